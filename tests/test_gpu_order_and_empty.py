"""GPU parity on the two input structures the named workloads never show:

* selection lists in other orders than ascending.  The article fixes no order
  for sparseBlockIdx ("Function / sparse attention mechanism" selects blocks
  by index; the result is a sum over the selected keys), so shuffled lists
  and descending lists (the diagonal, partly masked block first: the online
  softmax then starts from a masked block) must give the oracle's result;
* sequences with a storage length of 0 (a repeated cu_seqlens_q value: no Q
  block) and sequences with seqused_kv = 0 (no key: out 0, lse -inf), placed
  between ordinary ones ("Constraints / dual-length semantics").

Every case checks the metadata word for word against the oracle's rebuild,
the device status, and out / lse against the fp64 oracle, with whole units
and with forced split-KV pieces, in bf16 and in E4M3."""
import numpy as np
import pytest
import torch

from block_sparse_paged_gbsa_b200.workloads import generate, workload
from oracle import scheduler
from tests import test_gpu_fp8 as fp8
from tests.gpu_helpers import device_tensors, problem_dict, run_gpu, run_metadata, sm_count
from tests.helpers import assert_lse_close, assert_out_close, oracle_rows

pytestmark = pytest.mark.gpu

ORDERED = {
    "tiny": lambda o: workload("tiny", list_order=o),
    "ragged_s16": lambda o: workload("ragged", scale_down=16, list_order=o),
    "decode_s16": lambda o: workload("decode", scale_down=16, list_order=o),
    "g8_bx16_window": lambda o: generate(name="g8w", seed=80, q_storage=[1500, 900],
                                         q_used=[1480, 900], kv_used=[1500, 1000], N1=8, N2=1,
                                         block_x=16, top_k=12, selection="random_causal",
                                         win_left=700, win_right=0, list_order=o),
}

EMPTY = {
    # storage lengths 0 between non-empty sequences; a sequence with queries
    # and no key; a sequence with keys and no query
    "empty_between": lambda: generate(name="e1", seed=90, q_storage=[300, 0, 129, 0, 0, 64],
                                      kv_used=[300, 40, 0, 0, 77, 64], N1=8, N2=2,
                                      block_x=64, top_k=4, selection="random_causal"),
    # decode-shaped (one tile per Q block: units in halves, narrow tiles)
    "decode_zero_keys": lambda: generate(name="e2", seed=91,
                                         q_storage=[1, 1, 0, 1, 1, 0, 1, 1, 1, 1],
                                         q_used=[1, 1, 0, 1, 1, 0, 1, 1, 1, 1],
                                         kv_used=[5000, 0, 40, 300, 0, 0, 129, 1, 0, 7000],
                                         N1=16, N2=2, block_x=1, top_k=16, selection="decode",
                                         count_range=(1, 16), has_seqused_q=False),
    # G = 1, one token per Q block, a leading and a trailing empty sequence
    "g1_bx1": lambda: generate(name="e3", seed=92, q_storage=[0, 40, 0, 33, 0],
                               kv_used=[10, 0, 5, 33, 0], N1=2, N2=2, block_x=1, top_k=3,
                               selection="random_causal"),
    # used rows below storage, window, G = 5 (three tiles per Q block)
    "g5_window": lambda: generate(name="e4", seed=93, q_storage=[0, 700, 0, 333, 5],
                                  q_used=[0, 650, 0, 300, 5], kv_used=[0, 700, 9, 410, 0],
                                  N1=10, N2=2, block_x=64, top_k=6, selection="random_causal",
                                  win_left=200, win_right=0, page_stride_factor=1.25),
}


def _rows(w, limit=60000, seed=0):
    """Every (token, head) row of a small case, else a sample that keeps the
    first and last token of every non-empty sequence."""
    if w.T * w.N1 <= limit:
        tt, hh = np.meshgrid(np.arange(w.T), np.arange(w.N1), indexing="ij")
        return np.stack([tt.reshape(-1), hh.reshape(-1)], 1).astype(np.int64)
    rng = np.random.default_rng(seed)
    ends = np.concatenate([w.cu_seqlens_q[:-1], w.cu_seqlens_q[1:] - 1])
    tok = np.concatenate([rng.integers(0, w.T, 4000), ends[(ends >= 0) & (ends < w.T)]])
    return np.stack([tok, rng.integers(0, w.N1, tok.size)], 1).astype(np.int64)


def _metadata_matches_rebuild(w, forced):
    t = device_tensors(w)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    meta = run_metadata(w, t, 0, forced, status).cpu().numpy()
    ref = scheduler.build(problem_dict(w, sm_count(), forced), w.sparse_idx, w.sparse_count,
                          w.cu_seqlens_q, w.q_used, w.kv_used)
    mask = scheduler.defined_mask(ref)
    assert meta.size == ref.size
    assert np.array_equal(meta[mask], ref[mask])
    assert int(status.item()) == 0


def _check_bf16(w, forced):
    _metadata_matches_rebuild(w, forced)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    q, kf, vf, _, out, lse = run_gpu(w, forced=forced, dev_status=status)
    assert int(status.item()) == 0
    rows = _rows(w)
    ro, rl = oracle_rows(w, q.cpu(), kf.cpu(), vf.cpu(), rows)
    o = out.float().cpu().numpy().astype(np.float64)[rows[:, 0], rows[:, 1]]
    l = lse.cpu().numpy()[..., 0].astype(np.float64)[rows[:, 0], rows[:, 1]]
    assert_out_close(o, ro)
    assert_lse_close(l, rl)
    return out, lse


@pytest.mark.parametrize("forced", [0, 2])
@pytest.mark.parametrize("order", ["shuffled", "descending"])
@pytest.mark.parametrize("name", sorted(ORDERED))
def test_list_order_bf16(name, order, forced):
    _check_bf16(ORDERED[name](order), forced)


@pytest.mark.parametrize("forced", [0, 2])
@pytest.mark.parametrize("order", ["shuffled", "descending"])
@pytest.mark.parametrize("name", sorted(ORDERED))
def test_list_order_e4m3(name, order, forced):
    w = ORDERED[name](order)
    q, kf, vf = fp8._values(w)
    out, lse = fp8._forward(w, q, fp8.pool_view(w, kf), fp8.pool_view(w, vf), forced=forced)
    fp8._check(w, q, kf, vf, out, lse, _rows(w, limit=20000))


@pytest.mark.parametrize("forced", [0, 1])
@pytest.mark.parametrize("name", sorted(EMPTY))
def test_empty_sequences_and_zero_keys(name, forced):
    w = EMPTY[name]()
    assert (np.diff(w.cu_seqlens_q) == 0).any() or (w.kv_used == 0).any()
    out, lse = _check_bf16(w, forced)
    # every row of a sequence without a key: exactly 0 and -inf
    o, l = out.float().cpu(), lse.cpu()[..., 0]
    for b in np.nonzero(w.kv_used == 0)[0]:
        t0, t1 = int(w.cu_seqlens_q[b]), int(w.cu_seqlens_q[b + 1])
        assert torch.all(o[t0:t1] == 0)
        assert torch.all(torch.isneginf(l[t0:t1]))


@pytest.mark.parametrize("name", ["empty_between", "decode_zero_keys"])
def test_empty_sequences_e4m3(name):
    w = EMPTY[name]()
    q, kf, vf = fp8._values(w)
    for forced in (0, 1):
        out, lse = fp8._forward(w, q, fp8.pool_view(w, kf), fp8.pool_view(w, vf), forced=forced)
        fp8._check(w, q, kf, vf, out, lse, _rows(w, limit=20000))
