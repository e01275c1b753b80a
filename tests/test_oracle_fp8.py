"""Pins of the oracle's E4M3 path (the NEXT row "FP8 E4M3 with static
dequantization scales", GBSA article "Constraints: data types" and the
quantised-input arguments of the PyTorch API).  E4M3 values reach the oracle
through fp16, which holds every one of them exactly; the dequantization
scales fold into the score scale and the output.  Pinned here: the E4M3
decode against the format's definition on all 256 patterns, the fp16
conversion, the scale folding, and the out_abs error scale."""
import glob
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from block_sparse_paged_gbsa_b200.workloads import PAGE, make_values, workload
from tests.helpers import oracle_rows, oracle_rows_fp8
from tests.test_oracle_pins import GOLDEN, _fixture_workload

ALL8 = torch.arange(256, dtype=torch.int32).to(torch.uint8)


def _e4m3_by_definition(byte: int) -> float:
    # 1 sign bit, 4 exponent bits (bias 7), 3 fraction bits; exponent 0 holds
    # the subnormals f/8 * 2^-6; S.1111.111 is NaN and there is no infinity
    s, e, f = byte >> 7, (byte >> 3) & 0xF, byte & 7
    if e == 15 and f == 7:
        return math.nan
    mag = (f / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + f / 8.0) * 2.0 ** (e - 7)
    return -mag if s else mag


def test_e4m3_decode_matches_the_format_on_every_pattern():
    got = ALL8.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ref = np.array([_e4m3_by_definition(b) for b in range(256)])
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all()
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9


def test_e4m3_values_are_exact_in_fp16():
    x = ALL8.view(torch.float8_e4m3fn)
    via16 = x.to(torch.float16).to(torch.float64).numpy()
    direct = x.to(torch.float64).numpy()
    assert ((via16 == direct) | (np.isnan(via16) & np.isnan(direct))).all()


def _fp8_inputs(w):
    q, kf, vf = make_values(w, "cpu", nan_fill=False)
    return tuple(t.float().clamp(-448, 448).to(torch.float8_e4m3fn) for t in (q, kf, vf))


def test_scales_fold_into_scores_and_output():
    # the same E4M3 codes with scales (qs, ks, vs) equal the dequantised values
    # qs*q, ks*k, vs*v run through the plain oracle (powers of two keep the
    # products exact in fp16)
    w = workload("tiny", scale_down=4)
    q8, k8, v8 = _fp8_inputs(w)
    qs, ks, vs = 0.5, 2.0, 0.25
    rows = np.stack([np.arange(w.T).repeat(w.N1), np.tile(np.arange(w.N1), w.T)], 1)
    out, lse, _ = oracle_rows_fp8(w, q8, k8, v8, (qs, ks, vs), rows)
    deq = lambda t, s: (t.to(torch.float16) * s)
    ro, rl = oracle_rows(w, deq(q8, qs), deq(k8, ks), deq(v8, vs), rows)
    assert np.array_equal(out, ro) and np.array_equal(lse, rl)


def test_out_abs_is_the_weighted_absolute_value():
    # V -> |V| leaves the weights unchanged, so out_abs must equal the output
    # of the same rows with |V|
    w = workload("tiny", scale_down=4)
    q8, k8, v8 = _fp8_inputs(w)
    rows = np.stack([np.arange(w.T).repeat(w.N1), np.tile(np.arange(w.N1), w.T)], 1)
    _, _, oa = oracle_rows_fp8(w, q8, k8, v8, (1.0, 1.0, 1.0), rows)
    ra, _, _ = oracle_rows_fp8(w, q8, k8, v8.abs(), (1.0, 1.0, 1.0), rows)
    assert np.allclose(oa, ra, rtol=1e-14, atol=0)
    assert (oa >= 0).all()


def _emulate_e4m3_p(w, q8, k8, v8, scales, rows, threshold=0.5):
    """The E4M3 mode's arithmetic as read from the pages (static cast of the
    weights, running reference max), in float64 except for the cast itself:
    keys in list order, per block a lazy reference max (kept unless the
    block max exceeds it by more than `threshold`, log2 units), weights
    P = e4m3(2^(x - m + 8)), row sum of the uncast weights."""
    from tests.helpers import logical_kv
    qs, ks, vs = scales
    qd = q8.to(torch.float64).numpy()
    G = w.N1 // w.N2
    out = np.zeros((len(rows), w.D))
    log2e = 1.0 / math.log(2.0)
    qbase, seq_of_tok = [], []
    base = 0
    for b in range(w.B):
        qn = int(w.cu_seqlens_q[b + 1] - w.cu_seqlens_q[b])
        qbase.append(base)
        seq_of_tok += [b] * qn
        base += -(-qn // w.block_x)
    kb = k8.to(torch.float16).view(torch.int16).numpy().view(np.uint16)
    vb = v8.to(torch.float16).view(torch.int16).numpy().view(np.uint16)
    cache = {}
    for r, (tg, h) in enumerate(rows):
        b = seq_of_tok[tg]
        if b not in cache:
            cache[b] = (logical_kv(w, kb, b, "fp16"), logical_kv(w, vb, b, "fp16"))
        K, V = cache[b]
        t = tg - int(w.cu_seqlens_q[b])
        qu = int(w.q_used[b]) if w.has_seqused_q else int(w.cu_seqlens_q[b + 1] - w.cu_seqlens_q[b])
        if t >= qu:
            continue
        ku = int(w.kv_used[b])
        pos = t + ku - qu
        kvh = h // G
        qb = qbase[b] + t // w.block_x
        n = min(max(int(w.sparse_count[kvh, qb]), 0), w.top_k)
        m, l, o = -np.inf, 0.0, np.zeros(w.D)
        for j in range(n):
            lb = int(w.sparse_idx[kvh, qb, j])
            if not 0 <= lb < -(-ku // PAGE):
                continue
            keys = np.arange(lb * PAGE, min(lb * PAGE + PAGE, ku))
            keys = keys[keys <= pos]
            if w.win_left >= 0:
                keys = keys[keys >= pos - w.win_left]
            if keys.size == 0:
                continue
            x = (w.scale * qs * ks * log2e) * (K[keys, kvh, :] @ qd[tg, h])
            m_new = max(m, x.max())
            if m == -np.inf or m_new > m + threshold:
                f = 0.0 if m == -np.inf else 2.0 ** (m - m_new)
                o *= f
                l *= f
                m = m_new
            p = 2.0 ** (x - m + 8.0)
            p8 = torch.from_numpy(p.astype(np.float32)).to(torch.float8_e4m3fn).to(torch.float64)
            l += p.sum()
            o += p8.numpy() @ V[keys, kvh, :]
        if l > 0:
            out[r] = o / l * vs
    return out


def _r22_check(w, ro, ra, got, fin, vmax):
    n_vis = w.top_k * 128
    bound = (2.0 ** -4 + 1e-5) * ra + 2.0 ** -8 * np.abs(ro) + 2.0 ** -18 * n_vis * vmax
    err = np.abs(got - ro)
    return bool((err <= bound).all()), float(err[fin].mean()), float((2.0 ** -4 * ra[fin]).mean())


@pytest.mark.parametrize("name,scale_down", [("tiny", 4), ("decode", 32), ("dense", 8)])
def test_r22_bound_holds_for_the_e4m3_reading(name, scale_down):
    # a correct implementation of the reading meets the R22 bound, with
    # errors that are real (not zero) and whose mean stays under a quarter of
    # the mean 2^-4 out_abs (observed: 2-7 %); with the 16-bit path's lazy
    # threshold (8) a 2^8 P can pass 448, the largest E4M3 value, and on rows
    # of many blocks the result is lost
    from block_sparse_paged_gbsa_b200.workloads import workload as wl
    w = wl(name, scale_down=scale_down)
    q8, k8, v8 = _fp8_inputs(w)
    scales = (0.37, 1.9, 0.61)
    rng = np.random.default_rng(7)
    rows = np.stack([rng.integers(0, w.T, 150), rng.integers(0, w.N1, 150)], 1)
    ro, rl, ra = oracle_rows_fp8(w, q8, k8, v8, scales, rows)
    fin = np.isfinite(rl)
    vmax = float(v8.to(torch.float64).abs().max()) * scales[2]
    got = _emulate_e4m3_p(w, q8, k8, v8, scales, rows)
    ok, mean_err, mean_bound = _r22_check(w, ro, ra, got, fin, vmax)
    assert ok
    assert 0.0 < mean_err <= 0.25 * mean_bound
    if name != "tiny":
        bad = _emulate_e4m3_p(w, q8, k8, v8, scales, rows, threshold=8.0)
        assert not _r22_check(w, ro, ra, bad, fin, vmax)[0]


@pytest.mark.parametrize("path", sorted(glob.glob(os.path.join(GOLDEN, "e4m3_*.json"))))
def test_e4m3_golden_fixture(path):
    # hand-derived closed forms of E4M3 codes with dequantization scales
    fx = json.load(open(path))
    w, q, kf, vf = _fixture_workload(fx)
    to8 = lambda t: t.float().to(torch.float8_e4m3fn)
    assert torch.equal(to8(q).float(), q.float())          # the codes are exact in E4M3
    rows = np.array([[e["t"], e["h"]] for e in fx["expected"]], np.int64)
    out, lse, _ = oracle_rows_fp8(w, to8(q), to8(kf), to8(vf), tuple(fx["scales"]), rows)
    for i, e in enumerate(fx["expected"]):
        assert lse[i] == pytest.approx(e["lse"], abs=1e-12)
        for d, val in e["out"].items():
            assert out[i, int(d)] == pytest.approx(val, abs=1e-12)
