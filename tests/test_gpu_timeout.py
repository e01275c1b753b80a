"""Failure detection on the GPU without a fault: every pipeline wait of the
forward kernel is bounded (gbsa_problem.wait_limit_ns, 1 s by default).  The
cases have long units (up to 128 prefill blocks, or 256 decode blocks, on 8
CTAs), so the epilogue waits a unit's whole run for its output,
far longer than the hardware may hold the first barrier probe on its own;
with a bound of 1 us that wait runs out.  The kernel must set the TIMEOUT
status bit, drain the copies and MMAs it issued, release its tensor memory,
put the work list's unit counters back to zero and return, and the next
call on the same stream and work list, with the default bound, must be
correct."""
import numpy as np
import pytest
import torch

import block_sparse_paged_gbsa_b200 as gbsa
from block_sparse_paged_gbsa_b200.workloads import generate, make_values, pool_view, workload
from tests.gpu_helpers import device_tensors, run_forward, run_metadata
from tests.helpers import assert_lse_close, assert_out_close, oracle_rows

pytestmark = pytest.mark.gpu

TIMEOUT_BIT = 0x20


def _sample(w, n=3000, seed=0):
    rng = np.random.default_rng(seed)
    return np.stack([rng.integers(0, w.T, n), rng.integers(0, w.N1, n)], 1).astype(np.int64)


CASES = {
    # two-tile units of up to 128 blocks: 16384 tokens, every causal block,
    # on 8 CTAs (the split length grows with the work per CTA: no splits)
    "causal_16k_8ctas": (lambda: generate(name="to", seed=95, q_storage=[16384], N1=8, N2=2,
                                          block_x=128, top_k=128, selection="all_causal"), 8),
    # the one-tile instantiation (units in halves, narrow tiles): decode
    # lists of up to 256 blocks on 8 CTAs (no splits)
    "decode_s2_8ctas": (lambda: workload("decode", scale_down=2), 8),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_wait_limit_runs_out_then_next_call_is_correct(name):
    make, ctas = CASES[name]
    w = make()
    q, kf, vf = make_values(w, "cuda")
    t = device_tensors(w)
    meta = run_metadata(w, t, num_ctas=ctas)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    gbsa.forward(q, pool_view(w, kf), pool_view(w, vf), t["idx"], t["cnt"], [w.block_x, 128],
                 metadata=meta, cu_seqlens_q=t["cu"], seqused_q=t["squ"], seqused_kv=t["sku"],
                 block_table=t["bt"], softmax_scale=w.scale, return_softmax_lse=True,
                 num_ctas=ctas, dev_status=status, wait_limit_ns=1000)
    torch.cuda.synchronize()               # the call returned
    assert int(status.item()) & TIMEOUT_BIT
    # its work counters (header words 26, 27) are back at zero for the next call
    assert int(meta[26].item()) == 0 and int(meta[27].item()) == 0
    for _ in range(2):
        status2 = torch.zeros(1, dtype=torch.int32, device="cuda")
        out, lse = run_forward(w, q, kf, vf, t, meta, num_ctas=ctas, dev_status=status2)
        torch.cuda.synchronize()
        assert int(status2.item()) == 0
    rows = _sample(w)
    ro, rl = oracle_rows(w, q.cpu(), kf.cpu(), vf.cpu(), rows)
    assert_out_close(out.float().cpu().numpy().astype(np.float64)[rows[:, 0], rows[:, 1]], ro)
    assert_lse_close(lse.cpu().numpy()[..., 0][rows[:, 0], rows[:, 1]], rl)


def test_negative_wait_limit_rejected_before_launch():
    w = workload("tiny")
    q, kf, vf = make_values(w, "cuda")
    t = device_tensors(w)
    meta = run_metadata(w, t)
    with pytest.raises(gbsa.GbsaError):
        gbsa.forward(q, pool_view(w, kf), pool_view(w, vf), t["idx"], t["cnt"], [w.block_x, 128],
                     metadata=meta, cu_seqlens_q=t["cu"], seqused_kv=t["sku"],
                     block_table=t["bt"], wait_limit_ns=-1)
