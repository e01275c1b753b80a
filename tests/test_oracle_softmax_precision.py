"""The R24 tolerance of softmaxPrecision 1 (tests/helpers.py r24_bound; derived in
tests/test_gpu_softmax_precision.py)
is attainable: a numpy emulation of the mode's arithmetic -- keys in list
order, blocks of 128, the running reference max with the lazy threshold of 8,
the exponent rounded to f16 and its exponential rounded to f16, fp32 row sums
of those weights, P rounded to the element type for the product -- stays
within the bound against the fp64 oracle, with a mean error well below it,
and its lse within the R24 lse bound.  And the bounds have teeth: the same
emulation with the two weights of each f16 pair swapped (a plausible packing
mistake) breaks the output bound on the same rows, and its lse left in log2
units breaks the lse bound."""
import math

import numpy as np
import pytest
import torch

from block_sparse_paged_gbsa_b200.workloads import PAGE, bf16_bits, workload
from tests.helpers import (assert_lse_close_r24, keys_bound, logical_kv, r24_bound,
                           r24_lse_bound, to_f64)

LOG2E = 1.0 / math.log(2.0)


def _bf16(x):
    return torch.tensor(np.asarray(x, np.float32)).to(torch.bfloat16).float().numpy().astype(
        np.float64)


def _f16(x):
    return np.asarray(x, np.float32).astype(np.float16).astype(np.float64)


def _emulate(w, q, kf, vf, rows, dtype, round_exponent=_f16, swap_pairs=False, with_lse=False):
    dt = "bf16" if q.dtype == torch.bfloat16 else "fp16"
    qd = to_f64(bf16_bits(q), dt)
    kb, vb = bf16_bits(kf), bf16_bits(vf)
    qbase = np.concatenate([[0], np.cumsum(-(-np.diff(w.cu_seqlens_q) // w.block_x))])
    scale_log2 = np.float32(w.scale * LOG2E)
    out = np.zeros((rows.shape[0], w.D))
    lse = np.full(rows.shape[0], -np.inf)
    cache = {}
    for i, (tg, h) in enumerate(rows):
        b = int(np.searchsorted(w.cu_seqlens_q, tg, side="right") - 1)
        t = int(tg - w.cu_seqlens_q[b])
        qs = int(w.cu_seqlens_q[b + 1] - w.cu_seqlens_q[b])
        qu = int(w.q_used[b]) if w.has_seqused_q else qs
        ku = int(w.kv_used[b])
        if t >= qu:
            continue
        if b not in cache:
            cache[b] = (logical_kv(w, kb, b, dt), logical_kv(w, vb, b, dt))
        K, V = cache[b]
        kvh = h // w.G
        qb = int(qbase[b] + t // w.block_x)
        pos = t + ku - qu
        n = min(max(int(w.sparse_count[kvh, qb]), 0), w.top_k)
        m = -np.inf
        lsum = np.float32(0.0)
        acc = np.zeros(w.D)
        for j in range(n):
            lb = int(w.sparse_idx[kvh, qb, j])
            if not 0 <= lb < -(-ku // PAGE):
                continue
            p = np.arange(lb * PAGE, min(lb * PAGE + PAGE, ku))
            vis = p <= pos
            if w.win_left >= 0:
                vis &= p >= pos - w.win_left
            if not vis.any():
                continue
            s = (K[p, kvh, :] @ qd[tg, h]).astype(np.float32)       # fp32 accumulator
            s = np.where(vis, s, -np.inf).astype(np.float32)
            m_blk = np.float32(s.max() * scale_log2)
            m_new = max(m, m_blk)
            if m == -np.inf or m_new > m + 8.0:
                if m != -np.inf:
                    f = np.float32(2.0 ** (m - m_new))
                    lsum = np.float32(lsum * f)
                    acc = acc * f
                m = m_new
            x = (s.astype(np.float64) * scale_log2 - m).astype(np.float32)
            xr = round_exponent(x)
            P = np.exp2(xr).astype(np.float16).astype(np.float64)    # f16 weights
            P[~vis] = 0.0
            if swap_pairs:
                P = P.reshape(-1, 2)[:, ::-1].reshape(-1) if P.size % 2 == 0 else P
            lsum = np.float32(lsum + np.float32(P.sum()))
            Pu = _bf16(P) if dtype == "bf16" else P
            acc = acc + Pu @ V[p, kvh, :]
        if lsum > 0:
            out[i] = acc / float(lsum)
            lse[i] = (m + math.log2(float(lsum))) * math.log(2.0)
    return (out, lse) if with_lse else out


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("name", ["tiny", "dense_s16"])
def test_r24_bound_attainable_by_emulation(name, dtype):
    import oracle

    w = workload(name.split("_")[0], scale_down=16 if name.endswith("s16") else 1)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float16
    from block_sparse_paged_gbsa_b200.workloads import make_values
    q, kf, vf = make_values(w, "cpu", dtype=tdt)
    rng = np.random.default_rng(3)
    rows = np.stack([rng.integers(0, w.T, 600), rng.integers(0, w.N1, 600)], 1).astype(np.int64)
    n = rows.shape[0]
    oa, ga = np.zeros((n, w.D)), np.zeros((n, w.D))
    ro, rl = oracle.attention_rows(
        q_bits=bf16_bits(q), k_bits=bf16_bits(kf), v_bits=bf16_bits(vf),
        kv_page_stride=w.kv_page_stride, num_pages=w.num_pages, sparse_idx=w.sparse_idx,
        sparse_count=w.sparse_count, cu_seqlens_q=w.cu_seqlens_q, seqused_q=w.seqused_q,
        seqused_kv=w.kv_used, block_table=w.block_table, block_x=w.block_x, scale=w.scale,
        win_left=w.win_left, win_right=w.win_right, rows=rows, dtype=dtype, out_abs=oa,
        gap_abs=ga)
    em, em_lse = _emulate(w, q, kf, vf, rows, dtype, with_lse=True)
    vmax = float(vf.float().nan_to_num(0.0).abs().max())
    bound = r24_bound(dtype, ro, oa, ga, keys_bound(w, rows), vmax)
    err = np.abs(em - ro)
    assert (err <= bound).all(), float(np.max(err - bound))
    fin = np.isfinite(rl)
    scale = 2.0 * ((2.0 ** -9.9 + 8 * math.log(2) * 2.0 ** -11) * oa + 2.0 ** -11 * ga)
    assert err[fin].mean() <= 0.25 * scale[fin].mean()
    # swapped pair halves break the bound on these rows
    bad = _emulate(w, q, kf, vf, rows, dtype, swap_pairs=True)
    assert (np.abs(bad - ro) > bound).any()
    # the lse bound of R24 holds for the same arithmetic, and an lse left in
    # log2 units (the running max is kept in log2 units) breaks it
    n_keys = keys_bound(w, rows)
    assert_lse_close_r24(em_lse, rl, n_keys)
    fin = np.isfinite(rl)
    bad_lse = em_lse[fin] / math.log(2.0)
    assert (np.abs(bad_lse - rl[fin]) > r24_lse_bound(n_keys[fin], rl[fin])).any()
