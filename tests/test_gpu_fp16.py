"""fp16 Q/K/V/out against the oracle (a NEXT-row widening: the article's fp16
data type with the fp32 online softmax of softmaxPrecision 0).  The kernels
switch the MMA operand type, P and the output to fp16; scheduling, masks and
the split-KV merge are the bf16 ones."""
import numpy as np
import pytest
import torch

from block_sparse_paged_gbsa_b200.workloads import generate, make_values, workload
from tests.gpu_helpers import run_gpu
from tests.helpers import assert_lse_close, assert_out_close, oracle_all, oracle_rows

pytestmark = pytest.mark.gpu

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
    return make_values(w, "cuda", dtype=torch.float16)


def _check(w, q, kf, vf, out, lse, rows=None):
    assert out.dtype == torch.float16
    o = out.float().cpu().numpy().astype(np.float64)
    l = lse.float().cpu().numpy()[..., 0].astype(np.float64)
    if rows is None:
        ro, rl = oracle_all(w, q.cpu(), kf.cpu(), vf.cpu())
        assert_out_close(o, ro)
        assert_lse_close(l, rl)
    else:
        ro, rl = oracle_rows(w, q.cpu(), kf.cpu(), vf.cpu(), rows)
        assert_out_close(o[rows[:, 0], rows[:, 1]], ro)
        assert_lse_close(l[rows[:, 0], rows[:, 1]], rl)


@pytest.mark.parametrize("name", sorted(CASES))
def test_fp16_matches_oracle(name):
    w = CASES[name]()
    q, kf, vf, meta, out, lse = run_gpu(w, values=_values(w))
    _check(w, q, kf, vf, out, lse)


@pytest.mark.parametrize("name", ["decode_s16", "g8_bx16_window"])
def test_fp16_forced_splits(name):
    w = CASES[name]()
    q, kf, vf, meta, out, lse = run_gpu(w, values=_values(w), forced=3)
    _check(w, q, kf, vf, out, lse)


def test_fp16_dense_full_size_sampled_rows():
    w = workload("dense")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    q, kf, vf, meta, out, lse = run_gpu(w, values=_values(w), dev_status=status)
    assert int(status.item()) == 0
    rng = np.random.default_rng(3)
    rows = np.stack([rng.integers(0, w.T, 2000), rng.integers(0, w.N1, 2000)], 1)
    _check(w, q, kf, vf, out, lse, rows)


def test_fp16_and_bf16_agree_on_values_both_hold():
    # the same 1/4-grid values in both types: the two kernels see identical
    # operands, so their outputs agree to fp16 / bf16 output rounding
    w = workload("tiny")
    q, kf, vf = make_values(w, "cuda")
    snap = lambda t: torch.round(t.float().clamp(-2, 2) * 4) / 4
    vb = tuple(snap(t).to(torch.bfloat16) for t in (q, kf, vf))
    vh = tuple(snap(t).to(torch.float16) for t in (q, kf, vf))
    *_, ob, lb = run_gpu(w, values=vb)
    *_, oh, lh = run_gpu(w, values=vh)
    fin = torch.isfinite(lb)
    assert torch.equal(fin, torch.isfinite(lh))
    assert (lb[fin] - lh[fin]).abs().max().item() < 2e-3
    assert (ob.float() - oh.float()).abs().max().item() < 2e-2
