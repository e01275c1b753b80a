"""Helpers for the GPU tests: run the CUDA path (through the C ABI) on a
Workload, and build the matching oracle work list."""
from __future__ import annotations

import numpy as np
import torch

import block_sparse_paged_gbsa_b200 as gbsa
from block_sparse_paged_gbsa_b200.workloads import Workload, make_values, pool_view


def device_tensors(w: Workload, dev="cuda"):
    to = lambda a, dt: torch.as_tensor(np.ascontiguousarray(a), dtype=dt, device=dev)
    return dict(idx=to(w.sparse_idx, torch.int32), cnt=to(w.sparse_count, torch.int32),
                cu=to(w.cu_seqlens_q, torch.int64),
                squ=to(w.q_used, torch.int32) if w.has_seqused_q else None,
                sku=to(w.kv_used, torch.int32), bt=to(w.block_table, torch.int32))


def run_metadata(w: Workload, t, num_ctas=0, forced=0, dev_status=None):
    return gbsa.metadata(t["idx"], t["cnt"], w.N1, w.N2, w.D, [w.block_x, 128],
                         cu_seqlens_q=t["cu"], seqused_q=t["squ"], seqused_kv=t["sku"],
                         num_tokens=w.T, win_left=w.win_left, win_right=w.win_right,
                         num_ctas=num_ctas, max_blocks_per_split=forced, dev_status=dev_status)


def run_forward(w: Workload, q, kf, vf, t, meta, num_ctas=0, forced=0, dev_status=None,
                return_lse=True):
    return gbsa.forward(q, pool_view(w, kf), pool_view(w, vf), t["idx"], t["cnt"],
                        [w.block_x, 128], metadata=meta, cu_seqlens_q=t["cu"],
                        seqused_q=t["squ"], seqused_kv=t["sku"], block_table=t["bt"],
                        softmax_scale=w.scale, win_left=w.win_left, win_right=w.win_right,
                        return_softmax_lse=return_lse, num_ctas=num_ctas,
                        max_blocks_per_split=forced, dev_status=dev_status)


def run_gpu(w: Workload, values=None, num_ctas=0, forced=0, dev_status=None):
    """(q, kf, vf, meta, out, lse) with values drawn on the GPU unless given."""
    q, kf, vf = values if values is not None else make_values(w, "cuda")
    t = device_tensors(w)
    meta = run_metadata(w, t, num_ctas, forced, dev_status)
    out, lse = run_forward(w, q, kf, vf, t, meta, num_ctas, forced, dev_status)
    torch.cuda.synchronize()
    return q, kf, vf, meta, out, lse


def sm_count() -> int:
    return torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count


def problem_dict(w: Workload, num_ctas: int, forced: int = 0) -> dict:
    p = w.problem_kwargs()
    p.update(num_ctas=num_ctas, max_blocks_per_split=forced, mask_mode=1)
    return p
