"""E4M3 Q/K/V with per-tensor dequantization scales against the oracle (the
article's quantised mode 5, "static-cast P": FP8 inputs, the softmax weights
cast to FP8 for the P.V product, a 16-bit output).

Reading of the mode (the pages give the argument names only): q, k, v are
E4M3 codes times the scalars q/k/v_dequant_scale; scores are formed from the
dequantised values in fp32; the weights p = 2^(s - m) (m a running reference
max) are cast to E4M3 after a fixed factor 2^8 (the static cast), the row sum
uses the uncast weights; out is bf16.

Tolerance, per element, from that arithmetic: the E4M3 cast of a weight P
(2^8 p, with the reference max at most 0.5 below the row max, so the largest
P is 2^8.5 < 448 and nothing saturates) errs by at most 2^-4 P for P >= 2^-6
and by 2^-10 below, so |out - ref| <= 2^-4 out_abs + 2^-10 n |v|max / l8
with out_abs = sum_p w_p |v_p| from the oracle, n the row's visible keys and
l8 >= 2^8 the kernel's row sum; plus the bf16 rounding of out (2^-8 |ref|: 8 significant bits)
and fp32 accumulation (1e-5 out_abs).  lse does not see the cast: it keeps
the 16-bit bound.  The rounding errors have no common sign, so the mean error
must also stay well under the bound (a systematic mistake would not)."""
import numpy as np
import pytest
import torch

import block_sparse_paged_gbsa_b200 as gbsa
from block_sparse_paged_gbsa_b200.workloads import (PAGE, generate, make_values, pool_view,
                                                    tnd_kv, workload)
from tests.gpu_helpers import device_tensors, run_metadata
from tests.helpers import assert_lse_close, oracle_rows_fp8

pytestmark = pytest.mark.gpu

SCALES = (0.37, 1.9, 0.61)  # q, k, v dequantization scales (not powers of two)

CASES = {
    "tiny": lambda: workload("tiny"),
    "dense_s16": lambda: workload("dense", scale_down=16),
    "decode_s16": lambda: workload("decode", scale_down=16),
    "ragged_s16": lambda: workload("ragged", scale_down=16),
    "g8_bx16_window": lambda: generate(name="g8w", seed=80, q_storage=[1500, 900],
                                       q_used=[1480, 900], kv_used=[1500, 1000], N1=8, N2=1,
                                       block_x=16, top_k=12, selection="random_causal",
                                       win_left=700, win_right=0),
}


def _values(w):
    return make_values(w, "cuda", dtype=torch.float8_e4m3fn)


def _forward(w, q, k, v, forced=0, scales=SCALES, cu_kv=None):
    t = device_tensors(w)
    meta = run_metadata(w, t, forced=forced)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    kw = dict(block_table=t["bt"]) if cu_kv is None else dict(
        cu_seqlens_kv=torch.as_tensor(cu_kv, device="cuda"))
    out, lse = gbsa.forward(q, k, v, t["idx"], t["cnt"], [w.block_x, 128], metadata=meta,
                            cu_seqlens_q=t["cu"], seqused_q=t["squ"], seqused_kv=t["sku"],
                            softmax_scale=w.scale, win_left=w.win_left, win_right=w.win_right,
                            return_softmax_lse=True, max_blocks_per_split=forced,
                            dev_status=status, q_dequant_scale=scales[0],
                            k_dequant_scale=scales[1], v_dequant_scale=scales[2], **kw)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert out.dtype == torch.bfloat16
    return out, lse


def _all_rows(w):
    tt, hh = np.meshgrid(np.arange(w.T), np.arange(w.N1), indexing="ij")
    return np.stack([tt.reshape(-1), hh.reshape(-1)], axis=1)


def _check(w, q, kf, vf, out, lse, rows=None, scales=SCALES):
    rows = _all_rows(w) if rows is None else rows
    ro, rl, ra = oracle_rows_fp8(w, q.cpu(), kf.cpu(), vf.cpu(), scales, rows)
    o = out.float().cpu().numpy().astype(np.float64)[rows[:, 0], rows[:, 1]]
    l = lse.float().cpu().numpy()[..., 0].astype(np.float64)[rows[:, 0], rows[:, 1]]
    assert_lse_close(l, rl)
    fin = np.isfinite(rl)
    assert (o[~fin] == 0).all()                     # rows without a visible key
    vmax = float(vf.float().nan_to_num(0.0).abs().max()) * abs(scales[2])
    n_vis = w.top_k * PAGE
    bound = (2.0 ** -4 + 1e-5) * ra + 2.0 ** -8 * np.abs(ro) + 2.0 ** -18 * n_vis * vmax
    err = np.abs(o - ro)
    assert (err <= bound).all(), f"max excess {np.max(err - bound):.3g}"
    # no systematic error: the mean error is a small part of the mean bound
    assert err[fin].mean() <= 0.25 * ((2.0 ** -4) * ra[fin]).mean()


@pytest.mark.parametrize("name", sorted(CASES))
def test_fp8_matches_oracle(name):
    w = CASES[name]()
    q, kf, vf = _values(w)
    out, lse = _forward(w, q, pool_view(w, kf), pool_view(w, vf))
    _check(w, q, kf, vf, out, lse)


@pytest.mark.parametrize("name", ["decode_s16", "g8_bx16_window"])
def test_fp8_forced_splits(name):
    w = CASES[name]()
    q, kf, vf = _values(w)
    out, lse = _forward(w, q, pool_view(w, kf), pool_view(w, vf), forced=3)
    _check(w, q, kf, vf, out, lse)


def test_fp8_tnd_equals_paged():
    w = workload("ragged", scale_down=16)
    q, kf, vf = _values(w)
    kt, vt, cu_kv = tnd_kv(w, kf, vf)
    po, pl = _forward(w, q, pool_view(w, kf), pool_view(w, vf))
    to, tl = _forward(w, q, kt, vt, cu_kv=cu_kv)
    assert torch.equal(po, to) and torch.equal(pl, tl)


def test_fp8_scales_are_linear():
    # v_scale multiplies out exactly up to the bf16 rounding; q_scale and
    # k_scale enter only through their product
    w = workload("tiny")
    q, kf, vf = _values(w)
    kp, vp = pool_view(w, kf), pool_view(w, vf)
    o1, l1 = _forward(w, q, kp, vp, scales=(0.5, 3.0, 1.0))
    o2, l2 = _forward(w, q, kp, vp, scales=(3.0, 0.5, 4.0))
    assert torch.equal(l1, l2)
    assert torch.equal(o1.float() * 4.0, o2.float())


def test_fp8_dense_full_size_sampled_rows():
    w = workload("dense")
    q, kf, vf = _values(w)
    out, lse = _forward(w, q, pool_view(w, kf), pool_view(w, vf))
    rng = np.random.default_rng(5)
    rows = np.stack([rng.integers(0, w.T, 1500), rng.integers(0, w.N1, 1500)], 1)
    _check(w, q, kf, vf, out, lse, rows)


def test_fp8_decode_full_size_sampled_rows():
    w = workload("decode")
    q, kf, vf = _values(w)
    out, lse = _forward(w, q, pool_view(w, kf), pool_view(w, vf))
    rng = np.random.default_rng(6)
    rows = np.stack([rng.integers(0, w.T, 1500), rng.integers(0, w.N1, 1500)], 1)
    _check(w, q, kf, vf, out, lse, rows)


EDGE = {
    # narrow tiles (<= 8 live rows) with several tokens per tile
    "g2_bx4_narrow": lambda: generate(name="f1", seed=91, q_storage=[37, 130],
                                      kv_used=[700, 1200], N1=4, N2=2, block_x=4, top_k=6,
                                      selection="random_causal"),
    # G = 1, one-token blocks, lists with masked and duplicate-free random blocks
    "g1_bx1_any": lambda: generate(name="f2", seed=92, q_storage=[5, 3, 1], kv_used=[900, 300, 1500],
                                   N1=2, N2=2, block_x=1, top_k=8, selection="random_any"),
    # G = 128: one token per tile
    "g128": lambda: generate(name="f3", seed=93, q_storage=[10, 4], N1=128, N2=1, block_x=3,
                             top_k=3, selection="random_causal"),
}


@pytest.mark.parametrize("forced", [0, 3])
@pytest.mark.parametrize("name", sorted(EDGE))
def test_fp8_edge_shapes(name, forced):
    w = EDGE[name]()
    q, kf, vf = _values(w)
    out, lse = _forward(w, q, pool_view(w, kf), pool_view(w, vf), forced=forced)
    _check(w, q, kf, vf, out, lse)


def test_fp8_all_lists_empty():
    w = workload("tiny")
    w.sparse_count[:] = 0
    q, kf, vf = _values(w)
    out, lse = _forward(w, q, pool_view(w, kf), pool_view(w, vf))
    assert (out.float() == 0).all().item()
    assert torch.isneginf(lse).all().item()
