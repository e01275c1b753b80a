"""Non-paged TND K/V (k, v [T_kv, N2, D] with cu_seqlens_kv; the article's
"Constraints: layouts") on the GPU.  The same logical keys as TND must give
out and lse bit-identical to the paged pool, and match the oracle's TND
addressing.  NaN rows pad the sequences, so a stray read would show."""
import numpy as np
import pytest
import torch

import block_sparse_paged_gbsa_b200 as gbsa
from block_sparse_paged_gbsa_b200.workloads import generate, make_values, tnd_kv, workload
from tests.gpu_helpers import device_tensors, run_gpu, run_metadata
from tests.helpers import assert_lse_close, assert_out_close, oracle_all_tnd

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": lambda: workload("tiny"),
    "ragged_s16": lambda: workload("ragged", scale_down=16),
    "decode_s16": lambda: workload("decode", scale_down=16),
    "g8_bx16_window": lambda: generate(name="g8w", seed=80, q_storage=[1500, 900],
                                       q_used=[1480, 900], kv_used=[1500, 1000], N1=8, N2=1,
                                       block_x=16, top_k=12, selection="random_causal",
                                       win_left=700, win_right=0),
}


def _tnd_forward(w, q, kt, vt, cu_kv, forced=0):
    t = device_tensors(w)
    meta = run_metadata(w, t, forced=forced)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = gbsa.forward(q, kt, vt, t["idx"], t["cnt"], [w.block_x, 128], metadata=meta,
                            cu_seqlens_q=t["cu"], seqused_q=t["squ"], seqused_kv=t["sku"],
                            cu_seqlens_kv=torch.as_tensor(cu_kv, device="cuda"),
                            softmax_scale=w.scale, win_left=w.win_left, win_right=w.win_right,
                            return_softmax_lse=True, max_blocks_per_split=forced,
                            dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return out, lse


@pytest.mark.parametrize("name", sorted(CASES))
def test_tnd_equals_paged_and_oracle(name):
    w = CASES[name]()
    q, kf, vf = make_values(w, "cuda")
    kt, vt, cu_kv = tnd_kv(w, kf, vf)
    *_, po, pl = run_gpu(w, values=(q, kf, vf))
    to, tl = _tnd_forward(w, q, kt, vt, cu_kv)
    assert torch.equal(po, to) and torch.equal(pl, tl)
    ro, rl = oracle_all_tnd(w, q.cpu(), kt.cpu(), vt.cpu(), cu_kv)
    assert_out_close(to.float().cpu().numpy().astype(np.float64), ro)
    assert_lse_close(tl.float().cpu().numpy()[..., 0].astype(np.float64), rl)


@pytest.mark.parametrize("name", ["decode_s16", "g8_bx16_window"])
def test_tnd_forced_splits(name):
    w = CASES[name]()
    q, kf, vf = make_values(w, "cuda")
    kt, vt, cu_kv = tnd_kv(w, kf, vf)
    *_, po, pl = run_gpu(w, values=(q, kf, vf), forced=3)
    to, tl = _tnd_forward(w, q, kt, vt, cu_kv, forced=3)
    assert torch.equal(po, to) and torch.equal(pl, tl)
