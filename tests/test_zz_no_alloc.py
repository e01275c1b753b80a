"""gbsa_forward_static_scratch(): the forward pass for callers that cannot
allocate device memory (hosts with a fixed device-memory budget, code running
inside an allocator or framework hook).  Its split-KV scratch is a static
device array inside the library; these tests call it through the C ABI and
check it against gbsa_forward() with a caller-provided workspace -- bit for
bit, since both run the same kernels on the same work list -- on calls in a
row with another problem between them (every call overwrites the shared
scratch), and check that an oversized problem is refused before launch."""
import ctypes

import numpy as np
import pytest
import torch

import block_sparse_paged_gbsa_b200 as gbsa
from block_sparse_paged_gbsa_b200.gbsa import _Problem, _Tensors, make_problem
from block_sparse_paged_gbsa_b200.workloads import make_values, pool_view, workload

pytestmark = pytest.mark.gpu

STATIC_SCRATCH_BYTES = 32 << 20


def _entry():
    lib = gbsa.gbsa.lib()
    f = lib.gbsa_forward_static_scratch
    f.argtypes = [ctypes.POINTER(_Problem), ctypes.POINTER(_Tensors), ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_void_p]
    f.restype = ctypes.c_int
    return f


def _setup(name, scale_down, seed=None):
    w = workload(name, seed=seed, scale_down=scale_down)
    q, kf, vf = make_values(w, "cuda")
    to = lambda a, dt: torch.as_tensor(np.ascontiguousarray(a), dtype=dt, device="cuda")
    t = dict(idx=to(w.sparse_idx, torch.int32), cnt=to(w.sparse_count, torch.int32),
             cu=to(w.cu_seqlens_q, torch.int64), sku=to(w.kv_used, torch.int32),
             bt=to(w.block_table, torch.int32))
    meta = gbsa.metadata(t["idx"], t["cnt"], w.N1, w.N2, w.D, [w.block_x, 128],
                         cu_seqlens_q=t["cu"], seqused_kv=t["sku"], num_tokens=w.T)
    return w, q, pool_view(w, kf), pool_view(w, vf), t, meta


def _static_call(f, w, q, k, v, t, meta, status):
    prob = make_problem(q, k, t["idx"], [w.block_x, 128], t["bt"], t["cu"],
                        softmax_scale=w.scale, return_softmax_lse=True)
    out = torch.full_like(q, float("nan"))
    lse = torch.full((w.T, w.N1, 1), float("nan"), dtype=torch.float32, device="cuda")
    ten = _Tensors(q=q.data_ptr(), k=k.data_ptr(), v=v.data_ptr(), sparse_idx=t["idx"].data_ptr(),
                   sparse_count=t["cnt"].data_ptr(), cu_seqlens_q=t["cu"].data_ptr(),
                   seqused_q=None, seqused_kv=t["sku"].data_ptr(), block_table=t["bt"].data_ptr(),
                   out=out.data_ptr(), lse=lse.data_ptr())
    rc = f(ctypes.byref(prob.as_c()), ctypes.byref(ten), meta.data_ptr(), status.data_ptr(),
           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return rc, out, lse


def _reference(w, q, k, v, t, meta, status):
    return gbsa.forward(q, k, v, t["idx"], t["cnt"], [w.block_x, 128], metadata=meta,
                        cu_seqlens_q=t["cu"], seqused_kv=t["sku"], block_table=t["bt"],
                        softmax_scale=w.scale, return_softmax_lse=True, dev_status=status)


def _same(out, lse, ref_out, ref_lse):
    # the same kernels on the same work list and CTA count as gbsa_forward():
    # bit-identical out, lse equal on the finite rows and -inf on the others
    assert torch.equal(out, ref_out)
    fin = torch.isfinite(ref_lse)
    assert torch.equal(torch.isfinite(lse), fin)
    assert torch.equal(lse[fin], ref_lse[fin])


def test_static_scratch_matches_workspace_entry_point():
    f = _entry()
    a = _setup("decode", 4)
    b = _setup("decode", 8, seed=4321)     # another problem, run between the two calls
    assert int(a[5][13].item()) > 0 and int(b[5][13].item()) > 0, \
        "the cases must exercise the split-KV merge"
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ref_a = _reference(*a, status)
    ref_b = _reference(*b, status)
    for case, ref in ((a, ref_a), (b, ref_b), (a, ref_a)):
        # every call overwrites the shared scratch; the merge must read only
        # what the same call wrote
        rc, out, lse = _static_call(f, *case, status)
        torch.cuda.synchronize()
        assert rc == 0, gbsa.gbsa.lib().gbsa_status_string(rc)
        assert int(status.item()) == 0
        _same(out, lse, *ref)


def test_static_scratch_refuses_oversized_problem():
    f = _entry()
    w, q, k, v, t, meta = _setup("dense", 16)
    prob = make_problem(q, k, t["idx"], [w.block_x, 128], t["bt"], t["cu"],
                        softmax_scale=w.scale, return_softmax_lse=True)
    assert gbsa.workspace_size(prob) > STATIC_SCRATCH_BYTES
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc, out, _ = _static_call(f, w, q, k, v, t, meta, status)
    torch.cuda.synchronize()
    assert gbsa.gbsa.lib().gbsa_status_string(rc) == b"GBSA_ERR_WORKSPACE_TOO_SMALL"
    assert torch.isnan(out.float()).all()    # nothing was launched
