"""Shared test helpers: oracle calls on a Workload, an independent brute-force
formulation used to pin the oracle, and tolerance checks."""
from __future__ import annotations

import math

import numpy as np

import oracle
from block_sparse_paged_gbsa_b200.workloads import PAGE, Workload, bf16_bits


def elem_dtype(t) -> str:
    """The oracle's name of a torch tensor's 16-bit element type."""
    import torch

    return {torch.bfloat16: "bf16", torch.float16: "fp16"}[t.dtype]


def oracle_rows(w: Workload, q, kf, vf, rows, n_threads=None, lib=None):
    assert q.dtype == kf.dtype == vf.dtype
    return oracle.attention_rows(
        q_bits=bf16_bits(q), k_bits=bf16_bits(kf), v_bits=bf16_bits(vf),
        kv_page_stride=w.kv_page_stride, num_pages=w.num_pages, sparse_idx=w.sparse_idx,
        sparse_count=w.sparse_count, cu_seqlens_q=w.cu_seqlens_q, seqused_q=w.seqused_q,
        seqused_kv=w.kv_used, block_table=w.block_table, block_x=w.block_x, scale=w.scale,
        win_left=w.win_left, win_right=w.win_right, rows=rows, dtype=elem_dtype(q),
        n_threads=n_threads, lib=lib)


def oracle_all(w: Workload, q, kf, vf, n_threads=None, lib=None):
    T, N1 = w.T, w.N1
    tt, hh = np.meshgrid(np.arange(T), np.arange(N1), indexing="ij")
    rows = np.stack([tt.reshape(-1), hh.reshape(-1)], axis=1)
    out, lse = oracle_rows(w, q, kf, vf, rows, n_threads, lib=lib)
    return out.reshape(T, N1, w.D), lse.reshape(T, N1)


def oracle_rows_fp8(w: Workload, q8, kf8, vf8, scales, rows, n_threads=None):
    """Oracle rows for E4M3 inputs with per-tensor dequantization scales
    (q_scale, k_scale, v_scale): every E4M3 value is exact in fp16, so the
    values go to the oracle's fp16 decode unchanged; the scores carry
    scale * q_scale * k_scale and the output v_scale.  Returns (out, lse,
    out_abs) with out_abs = sum_p w_p |v_scale * v_p| (the error scale of a
    rounding of the weights)."""
    import torch

    qs, ks, vs = scales
    rows = np.asarray(rows, np.int64).reshape(-1, 2)
    out_abs = np.zeros((rows.shape[0], w.D), np.float64)
    out, lse = oracle.attention_rows(
        q_bits=bf16_bits(q8.to(torch.float16)), k_bits=bf16_bits(kf8.to(torch.float16)),
        v_bits=bf16_bits(vf8.to(torch.float16)), kv_page_stride=w.kv_page_stride,
        num_pages=w.num_pages, sparse_idx=w.sparse_idx, sparse_count=w.sparse_count,
        cu_seqlens_q=w.cu_seqlens_q, seqused_q=w.seqused_q, seqused_kv=w.kv_used,
        block_table=w.block_table, block_x=w.block_x, scale=w.scale * qs * ks,
        win_left=w.win_left, win_right=w.win_right, rows=rows, dtype="fp16", out_abs=out_abs,
        n_threads=n_threads)
    return out * vs, lse, out_abs * abs(vs)


def oracle_all_tnd(w: Workload, q, k_tnd, v_tnd, cu_kv, n_threads=None):
    """Oracle over every row with K/V in the TND layout (see workloads.tnd_kv)."""
    T, N1 = w.T, w.N1
    tt, hh = np.meshgrid(np.arange(T), np.arange(N1), indexing="ij")
    rows = np.stack([tt.reshape(-1), hh.reshape(-1)], axis=1)
    out, lse = oracle.attention_rows(
        q_bits=bf16_bits(q), k_bits=bf16_bits(k_tnd), v_bits=bf16_bits(v_tnd),
        kv_page_stride=0, num_pages=0, sparse_idx=w.sparse_idx, sparse_count=w.sparse_count,
        cu_seqlens_q=w.cu_seqlens_q, seqused_q=w.seqused_q, seqused_kv=w.kv_used,
        block_table=None, block_x=w.block_x, scale=w.scale, win_left=w.win_left,
        win_right=w.win_right, rows=rows, dtype=elem_dtype(q), cu_seqlens_kv=cu_kv,
        n_threads=n_threads)
    return out.reshape(T, N1, w.D), lse.reshape(T, N1)


def to_f64(bits: np.ndarray, dtype: str = "bf16") -> np.ndarray:
    """Exact float64 values of 16-bit patterns, decoded with numpy (a decoder
    independent of the oracle's C code): bf16 is the upper half of a
    binary32, fp16 is numpy's IEEE binary16."""
    bits = np.asarray(bits, np.uint16)
    if dtype == "fp16":
        return bits.view(np.float16).astype(np.float64)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def logical_kv(w: Workload, pool_bits: np.ndarray, b: int, dtype: str = "bf16") -> np.ndarray:
    """[ku, N2, D] fp64 keys (or values) of sequence b in logical order."""
    ku = int(w.kv_used[b])
    rows = []
    for lb in range(-(-ku // PAGE)):
        page = int(w.block_table[b, lb])
        start = page * w.kv_page_stride
        blk = pool_bits[start:start + PAGE * w.N2 * w.D].reshape(PAGE, w.N2, w.D)
        rows.append(blk)
    if not rows:
        return np.zeros((0, w.N2, w.D))
    return to_f64(np.concatenate(rows, 0)[:ku], dtype)


def brute_force(w: Workload, q, kf, vf, gap=False):
    """A second formulation of the operator: for every (token, head) the
    multiplicity of every logical key position is found by walking the block
    list entry by entry, the masks are applied as a dense boolean vector, and
    a dense fp64 softmax with those multiplicities as weights gives out/lse.
    With gap=True also returns sum_p w_p (max s - s_p) |v_p| per element."""
    dt = elem_dtype(q)
    qb_bits, kb, vb = bf16_bits(q), bf16_bits(kf), bf16_bits(vf)
    qd = to_f64(qb_bits, dt)
    out = np.zeros((w.T, w.N1, w.D))
    lse = np.full((w.T, w.N1), -np.inf)
    gap_abs = np.zeros((w.T, w.N1, w.D))
    G = w.N1 // w.N2
    qbase = 0
    for b in range(w.B):
        qs = int(w.cu_seqlens_q[b + 1] - w.cu_seqlens_q[b])
        qu = int(w.q_used[b]) if w.has_seqused_q else qs
        ku = int(w.kv_used[b])
        K = logical_kv(w, kb, b, dt)
        V = logical_kv(w, vb, b, dt)
        keys = np.arange(ku)
        for t in range(qu):
            tg = int(w.cu_seqlens_q[b]) + t
            qb = qbase + t // w.block_x
            pos = t + ku - qu
            allowed = keys <= pos
            if w.win_left >= 0:
                allowed &= keys >= pos - w.win_left
            if w.win_right >= 0:
                allowed &= keys <= pos + w.win_right
            for h in range(w.N1):
                kvh = h // G
                mult = np.zeros(ku)
                n = min(max(int(w.sparse_count[kvh, qb]), 0), w.top_k)
                for j in range(n):
                    lb = int(w.sparse_idx[kvh, qb, j])
                    if 0 <= lb < -(-ku // PAGE):
                        mult[lb * PAGE:min(lb * PAGE + PAGE, ku)] += 1
                wgt = mult * allowed
                if wgt.sum() == 0:
                    continue
                s = w.scale * (K[:, kvh, :] @ qd[tg, h])
                m = s[wgt > 0].max()
                e = np.where(wgt > 0, wgt * np.exp(np.where(wgt > 0, s - m, 0.0)), 0.0)
                out[tg, h] = e @ V[:, kvh, :] / e.sum()
                lse[tg, h] = m + math.log(e.sum())
                if gap:
                    g = np.where(wgt > 0, m - s, 0.0)
                    gap_abs[tg, h] = (e * g) @ np.abs(V[:, kvh, :]) / e.sum()
        qbase += -(-qs // w.block_x)
    return (out, lse, gap_abs) if gap else (out, lse)


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    """Half the bf16 spacing at |x| (the representation error of an exact
    value rounded to bf16)."""
    a = np.abs(np.asarray(x, np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 0.5 * 2.0 ** (e - 7)


OUT_TOL = 1e-2     # max abs error on the 16-bit output
LSE_TOL = 1e-3     # max abs error on the fp32 lse
RAW_BELOW = 2.0    # |exact| below which the raw error itself must stay within OUT_TOL


def out_errors(gpu_out, ref_out):
    """(raw max |gpu - exact| over entries with |exact| < 2, the same over all
    entries with the bf16 representation error of the exact value taken
    off)."""
    g = np.asarray(gpu_out, np.float64)
    r = np.asarray(ref_out, np.float64)
    diff = np.abs(g - r)
    small = np.abs(r) < RAW_BELOW
    raw = float(diff[small].max()) if small.any() else 0.0
    beyond = float((diff - bf16_half_ulp(r)).max()) if diff.size else 0.0
    return raw, beyond


def assert_out_close(gpu_out, ref_out, tol=OUT_TOL, what="out"):
    """The output tolerance: the raw error |gpu - exact| is at most tol
    wherever |exact| < 2, where a 16-bit output holds the exact value to
    within 2^-8; above that, bf16 cannot store the exact value closer than
    half its spacing (1.6e-2 at |x| >= 4), so the allowance is tol on top of
    that representation error."""
    g = np.asarray(gpu_out, np.float64)
    r = np.asarray(ref_out, np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite values"
    raw, beyond = out_errors(g, r)
    assert raw <= tol, f"{what}: raw max abs error {raw:.4g} > {tol} where |exact| < {RAW_BELOW}"
    assert beyond <= tol, f"{what}: max abs error {beyond:.4g} beyond bf16 rounding > {tol}"


def assert_lse_close(gpu_lse, ref_lse, tol=LSE_TOL):
    g = np.asarray(gpu_lse, np.float64)
    r = np.asarray(ref_lse, np.float64)
    inf_r = np.isneginf(r)
    assert np.array_equal(np.isneginf(g), inf_r), "lse: -inf pattern differs"
    if (~inf_r).any():
        worst = float(np.abs(g[~inf_r] - r[~inf_r]).max())
        assert worst <= tol, f"lse: max abs error {worst:.4g} > {tol}"


def keys_bound(w, rows):
    """An upper bound of the visible keys of each row: its clamped count x 128."""
    qbase = np.concatenate([[0], np.cumsum(-(-np.diff(w.cu_seqlens_q) // w.block_x))])
    b = np.searchsorted(w.cu_seqlens_q, rows[:, 0], side="right") - 1
    qb = qbase[b] + (rows[:, 0] - w.cu_seqlens_q[b]) // w.block_x
    cnt = np.clip(w.sparse_count[rows[:, 1] // w.G, qb], 0, w.top_k)
    return cnt.astype(np.float64) * PAGE


def r24_lse_bound(n_keys, ref_lse):
    """Per-row bound of |lse - exact| under R24 (softmaxPrecision 1).  lse =
    ln2 * (m + log2 l) with l the fp32 sum of the f16 weights P_p = 2^x_p; a
    weight's relative error is at most 2^-9.9 (ex2.approx.f16) plus
    ln2 * 2^-11 * |x_p| (the f16 rounding of x_p), |x_p| <= 8 (the reference
    lag) + log2(e) (M - S_p).  The error of l relative to l is the weighted
    mean of those, and the softmax-weighted mean of M - S_p is at most ln n
    (the weights' entropy ln Z + E[M - S] is at most ln n, with Z >= 1), so
    |ln(l' / l)| <= (1 + 2^-8) (2^-9.9 + ln2 2^-11 (8 + log2 n)); weights
    below the f16 range lose at most n 2^-24 of l >= 1; fp32 arithmetic
    adds 1e-5 |lse|."""
    n = np.maximum(np.asarray(n_keys, np.float64), 1.0)
    rel = (1.0 + 2.0 ** -8) * (2.0 ** -9.9 + math.log(2.0) * 2.0 ** -11 * (8.0 + np.log2(n)))
    r = np.asarray(ref_lse, np.float64)
    return rel + n * 2.0 ** -24 + 1e-5 * np.abs(np.where(np.isfinite(r), r, 0.0))


def assert_lse_close_r24(gpu_lse, ref_lse, n_keys):
    """lse under r24_lse_bound, with the same -inf pattern."""
    g = np.asarray(gpu_lse, np.float64)
    r = np.asarray(ref_lse, np.float64)
    inf_r = np.isneginf(r)
    assert np.array_equal(np.isneginf(g), inf_r), "lse: -inf pattern differs"
    fin = ~inf_r
    if fin.any():
        excess = np.abs(g[fin] - r[fin]) - r24_lse_bound(np.asarray(n_keys)[fin], r[fin])
        assert (excess <= 0).all(), f"lse: max excess over the R24 bound {excess.max():.3g}"


def r24_bound(dtype, ref, out_abs, gap_abs, n_keys, vmax):
    """The per-element bound of reading R24 (softmaxPrecision 1; derivation in
    tests/test_gpu_softmax_precision.py): the f16 exponent and exponential
    against the oracle's out_abs and gap_abs, the weights lost below the f16
    range, the 16-bit output, fp32 accumulation; bf16 adds the rounding of P
    to bf16, E4M3 the R22 bound of the weights' E4M3 cast."""
    d0 = 2.0 ** -9.9 + 8.0 * math.log(2.0) * 2.0 ** -11
    b = 2.0 * (1.0 + 2.0 ** -8) * (d0 * out_abs + 2.0 ** -11 * gap_abs)
    # the 16-bit output: u |exact|, u = 2^-8 for a bf16 out (8 significant
    # bits; E4M3 inputs give a bf16 out too), 2^-11 for fp16 (kept at 2^-9)
    u_out = 2.0 ** -9 if dtype == "fp16" else 2.0 ** -8
    b = b + 2.0 * n_keys[:, None] * 2.0 ** -24 * vmax + u_out * np.abs(ref) + 1e-5 * out_abs
    if dtype == "bf16":
        b = b + 2.0 ** -8 * out_abs  # P rounded to bf16 for the product
    if dtype == "e4m3":
        # the weights' E4M3 cast (R22): 2^-4 relative, 2^-10 below 2^-6
        b = b + 2.0 ** -4 * out_abs + 2.0 ** -18 * n_keys[:, None] * vmax
    return b
