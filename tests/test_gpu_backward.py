"""Gradients of the attention output on the GPU (gbsa.backward) against the
fp64 oracle's (oracle.attention_backward, pinned in test_oracle_backward).

Tolerance, from the arithmetic of the CUDA path: the products take the
exact 16-bit inputs with fp32 accumulation, and P = exp(s - lse) uses the
forward's fp32 lse.  Rounding to the element type errs by at most u = 2^-8
relative for bf16 (8 significant bits) and 2^-11 for fp16.  The delta
D = dO . O uses the forward's computed out, which errs per element by at
most 2u sum_p w_p |v_p| (its own 16-bit weights, then its 16-bit output), so
D errs by at most 2u A with A = sum_d |dO_d| sum_p w_p |v_p[d]|; P and dS
enter the products rounded (u of each term).  Every dS then errs by at most
2u P A + u |dS| <= 3u of the oracle's absolute-term sum for it,
P (|dO| . |V| + A); fp32 sums and the lse error stay far below.  So
|dq - dq_ref| and |dk - dk_ref| stay within 3u = 1.5 * 2^-7 of the oracle's
absolute-term sums and |dv - dv_ref| (no delta term) within u = 2^-8; the
test allows 2^-6 and 2^-7.  Keys nobody sees get exactly 0, and so do dq
rows with no key or past seqused_q."""
import numpy as np
import pytest
import torch

import block_sparse_paged_gbsa_b200 as gbsa
import oracle
from block_sparse_paged_gbsa_b200.workloads import PAGE, generate, make_values, pool_view, tnd_kv, workload
from tests.gpu_helpers import device_tensors, run_metadata
from tests.helpers import bf16_bits, elem_dtype

pytestmark = pytest.mark.gpu


def _cases():
    return {
        "tiny": lambda: workload("tiny"),
        # G = 5, Q blocks of 3 tiles (one-tile units), window, partial pages,
        # seqused_q, strided pool, shuffled lists with garbage past the counts
        "g5_window": lambda: generate(name="bw5", seed=71, q_storage=[300, 180], q_used=[290, 180],
                                      kv_used=[420, 250], N1=10, N2=2, block_x=64, top_k=6,
                                      selection="random_causal", win_left=200, win_right=0,
                                      page_stride_factor=1.5, list_order="shuffled"),
        # decode-shaped: one-token Q blocks, G = 8
        "decode_like": lambda: generate(name="bwd", seed=72, q_storage=[1] * 6, q_used=[1] * 6,
                                        kv_used=[700, 129, 1, 300, 1000, 64], N1=16, N2=2,
                                        block_x=1, top_k=8, selection="random_causal"),
        # duplicate entries count twice
        "duplicates": lambda: _with_duplicates(workload("tiny", seed=5)),
    }


def _with_duplicates(w):
    idx = w.sparse_idx.copy()
    cnt = w.sparse_count.copy()
    for h in range(w.N2):
        for qb in range(idx.shape[1]):
            c = int(cnt[h, qb])
            if 0 < c < w.top_k:
                idx[h, qb, c] = idx[h, qb, 0]
                cnt[h, qb] = c + 1
    w.sparse_idx, w.sparse_count = idx, cnt
    return w


def _compact(w, flat):
    """The oracle's pool-shaped gradient (page stride of the pool) as the
    compact [num_pages, 128, N2, D] layout of gbsa.backward."""
    per = PAGE * w.N2 * w.D
    a = np.zeros((w.num_pages, per), np.float64)
    for pg in range(w.num_pages):
        a[pg] = flat[pg * w.kv_page_stride:pg * w.kv_page_stride + per]
    return a.reshape(w.num_pages, PAGE, w.N2, w.D)


def _run(w, dtype, tnd=False, seed=0, ctas=0, forced=0):
    q, kf, vf = make_values(w, "cuda", dtype=dtype)
    t = device_tensors(w)
    meta = run_metadata(w, t, ctas, forced)
    g = torch.Generator(device="cuda").manual_seed(1234 + seed)
    dout = torch.randn(q.shape, generator=g, device="cuda", dtype=torch.float32).to(dtype)
    kw = dict(metadata=meta, cu_seqlens_q=t["cu"], seqused_q=t["squ"], seqused_kv=t["sku"],
              softmax_scale=w.scale, win_left=w.win_left, win_right=w.win_right,
              num_ctas=ctas, max_blocks_per_split=forced)
    if tnd:
        kt, vt, cu_kv = tnd_kv(w, kf, vf, seed=seed)
        kvkw = dict(cu_seqlens_kv=torch.as_tensor(cu_kv, device="cuda"))
        k_in, v_in = kt, vt
    else:
        kvkw = dict(block_table=t["bt"])
        k_in, v_in = pool_view(w, kf), pool_view(w, vf)
    out, lse = gbsa.forward(q, k_in, v_in, t["idx"], t["cnt"], [w.block_x, 128],
                            return_softmax_lse=True, **kw, **kvkw)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    dq, dk, dv = gbsa.backward(dout, q, k_in, v_in, out, lse, t["idx"], t["cnt"],
                               [w.block_x, 128], dev_status=status, **kw, **kvkw)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    okw = dict(sparse_idx=w.sparse_idx, sparse_count=w.sparse_count,
               cu_seqlens_q=w.cu_seqlens_q, seqused_q=w.seqused_q, seqused_kv=w.kv_used,
               block_x=w.block_x, scale=w.scale, win_left=w.win_left, win_right=w.win_right,
               dtype=elem_dtype(q), with_abs=True)
    if tnd:
        ref = oracle.attention_backward(q_bits=bf16_bits(q), k_bits=bf16_bits(kt), v_bits=bf16_bits(vt),
                                        dout_bits=bf16_bits(dout), kv_page_stride=0, num_pages=0,
                                        block_table=None, cu_seqlens_kv=cu_kv, **okw)
        shape = tuple(kt.shape)
        ref = [r if i % 3 == 0 else r.reshape(shape) for i, r in enumerate(ref)]
    else:
        ref = oracle.attention_backward(q_bits=bf16_bits(q), k_bits=bf16_bits(kf), v_bits=bf16_bits(vf),
                                        dout_bits=bf16_bits(dout), kv_page_stride=w.kv_page_stride,
                                        num_pages=w.num_pages, block_table=w.block_table, **okw)
        ref = [r if i % 3 == 0 else _compact(w, r) for i, r in enumerate(ref)]
    return (dq, dk, dv), ref


def _check(got, ref):
    dq_ref, dk_ref, dv_ref, dq_abs, dk_abs, dv_abs = ref
    for name, g, r, a, rel in (("dq", got[0], dq_ref, dq_abs, 2.0 ** -6),
                               ("dk", got[1], dk_ref, dk_abs, 2.0 ** -6),
                               ("dv", got[2], dv_ref, dv_abs, 2.0 ** -7)):
        g = g.double().cpu().numpy()
        assert g.shape == r.shape, name
        assert np.isfinite(g).all(), name
        err = np.abs(g - r)
        bound = rel * a + 1e-7 * max(a.max(), 1e-30)
        assert (err <= bound).all(), (name, float(np.max(err - bound)))
        assert np.array_equal(g[a == 0], np.zeros(int((a == 0).sum()))), name  # untouched: 0


@pytest.mark.parametrize("name", sorted(_cases()))
def test_backward_matches_oracle(name):
    w = _cases()[name]()
    got, ref = _run(w, torch.bfloat16)
    assert all(np.abs(r).max() > 0 for r in ref[:3])  # every gradient has nonzero entries
    _check(got, ref)


def test_backward_fp16():
    got, ref = _run(_cases()["g5_window"](), torch.float16, seed=1)
    _check(got, ref)


def test_backward_tnd():
    got, ref = _run(_cases()["g5_window"](), torch.bfloat16, tnd=True, seed=2)
    _check(got, ref)


def test_backward_with_split_work_list():
    """A work list built with forced splits and 7 CTAs: the backward reads
    only its item table and live lists, and takes the same problem (the
    list's signature covers num_ctas and the split length)."""
    got, ref = _run(_cases()["g5_window"](), torch.bfloat16, seed=3, ctas=7, forced=2)
    _check(got, ref)


def test_backward_metadata_of_another_problem_is_refused():
    """A work list built for other CTA settings: the kernel sets the
    mismatch bit and leaves dq alone."""
    w = _cases()["tiny"]()
    q, kf, vf = make_values(w, "cuda")
    t = device_tensors(w)
    meta = run_metadata(w, t, 7, 0)
    kw = dict(cu_seqlens_q=t["cu"], seqused_q=t["squ"], seqused_kv=t["sku"],
              block_table=t["bt"], softmax_scale=w.scale)
    out, lse = gbsa.forward(q, pool_view(w, kf), pool_view(w, vf), t["idx"], t["cnt"],
                            [w.block_x, 128], metadata=meta, num_ctas=7, return_softmax_lse=True,
                            **kw)
    dq = torch.full(q.shape, 7.0, dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    gbsa.backward(q, q, pool_view(w, kf), pool_view(w, vf), out, lse, t["idx"], t["cnt"],
                  [w.block_x, 128], metadata=meta, num_ctas=5, dq=dq, dev_status=status, **kw)
    torch.cuda.synchronize()
    assert int(status.item()) & 0x10
    assert bool((dq == 7.0).all())


def test_backward_rejects_e4m3():
    w = workload("tiny")
    q, kf, vf = make_values(w, "cuda", dtype=torch.float8_e4m3fn)
    t = device_tensors(w)
    meta = run_metadata(w, t)
    with pytest.raises(ValueError):
        gbsa.backward(q, q, pool_view(w, kf), pool_view(w, vf), q, None, t["idx"], t["cnt"],
                      [w.block_x, 128], metadata=meta, cu_seqlens_q=t["cu"], seqused_kv=t["sku"],
                      block_table=t["bt"])
