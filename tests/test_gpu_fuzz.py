"""Seeded random problems across the parameter space: group sizes 1..16, Q
block sizes from 1 to 200 tokens (several tiles, one tile, narrow tiles),
empty and partly used sequences, KV lengths with partial last pages or no
keys at all, sliding windows, every selection kind and list order, garbage
past each count, forced split lengths, CTA counts from 1 to 148, bf16, fp16
and E4M3, strided page pools.  For each: the work list is word for word the
sequential rebuild's (device status included), and sampled rows of out and
lse match the fp64 oracle: bf16 and fp16 under the output rule (raw 1e-2
where |exact| < 2, plus half a 16-bit ulp above) and the 1e-3 lse rule, E4M3
under its bound (R22, as in test_gpu_fp8).  The same keys in the non-paged
TND layout (NaN rows between the sequences) give bit-identical out and lse,
and so does a call without the lse output (out).
softmaxPrecision 1 on the same inputs stays within its R24 bound (as in
test_gpu_softmax_precision).  Every tenth case also runs the backward
(16-bit types) against the oracle's gradients under the bound of
test_gpu_backward (R25)."""
import math

import numpy as np
import pytest
import torch

import block_sparse_paged_gbsa_b200 as gbsa
from block_sparse_paged_gbsa_b200.workloads import PAGE, generate, make_values, pool_view, tnd_kv
from oracle import scheduler
from tests.gpu_helpers import device_tensors, problem_dict, run_metadata, sm_count
from tests.helpers import (assert_lse_close, assert_lse_close_r24, assert_out_close, keys_bound,
                           oracle_rows, oracle_rows_fp8, r24_bound)
from tests.test_gpu_softmax_precision import _oracle as oracle_mode1

pytestmark = pytest.mark.gpu

N_CASES = 150
FP8_SCALES = (0.37, 1.9, 0.61)  # q, k, v dequantization scales


def fuzz_case(k: int):
    """(workload, dtype, num_ctas, forced split length) of case k."""
    rng = np.random.default_rng(7000 + k)
    N2 = int(rng.choice([1, 2, 4]))
    G = int(rng.choice([1, 2, 3, 4, 5, 7, 8, 16]))
    block_x = int(rng.choice([1, 5, 16, 32, 64, 128, 200]))
    B = int(rng.integers(1, 5))
    qs = rng.integers(0, 600, size=B)
    if qs.sum() == 0:
        qs[0] = 1
    qu = np.array([int(rng.integers(0, q + 1)) if rng.random() < 0.3 else int(q) for q in qs])
    ku = np.array([max(0, int(u) + int(rng.integers(-50, 400))) if rng.random() < 0.85
                   else int(rng.integers(0, 3)) for u in qu])
    selection = str(rng.choice(["random_causal", "random_any", "all_causal", "sink_diag_random"]))
    window = rng.random() < 0.4
    w = generate(name=f"fuzz{k}", seed=5000 + k, q_storage=qs, q_used=qu, kv_used=ku,
                 N1=N2 * G, N2=N2, block_x=block_x, top_k=int(rng.integers(1, 25)),
                 selection=selection, win_left=int(rng.integers(0, 500)) if window else -1,
                 win_right=0 if window else -1,
                 page_stride_factor=float(rng.choice([1.0, 1.0, 1.5])),
                 list_order=str(rng.choice(["ascending", "descending", "shuffled"])))
    r = rng.random()
    dtype = torch.float8_e4m3fn if r < 0.2 else (torch.float16 if r < 0.45 else torch.bfloat16)
    ctas = int(rng.choice([0, 1, 7, 148]))
    forced = int(rng.choice([0, 0, 1, 2, 3]))
    return w, dtype, ctas, forced


def _rows(w, n=1500, seed=0):
    rng = np.random.default_rng(seed)
    ends = np.concatenate([w.cu_seqlens_q[:-1], w.cu_seqlens_q[1:] - 1])
    tok = np.concatenate([rng.integers(0, w.T, n), ends[(ends >= 0) & (ends < w.T)]])
    return np.stack([tok, rng.integers(0, w.N1, tok.size)], 1).astype(np.int64)


@pytest.mark.parametrize("k", range(N_CASES))
def test_fuzz_case(k):
    w, dtype, ctas, forced = fuzz_case(k)
    t = device_tensors(w)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    meta = run_metadata(w, t, ctas, forced, status)
    ref = scheduler.build(problem_dict(w, ctas or sm_count(), forced), w.sparse_idx,
                          w.sparse_count, w.cu_seqlens_q, w.q_used if w.has_seqused_q else None,
                          w.kv_used)
    m = meta.cpu().numpy()
    mask = scheduler.defined_mask(ref)
    assert m.size == ref.size and np.array_equal(m[mask], ref[mask])
    assert int(status.item()) == int(ref[15])
    q, kf, vf = make_values(w, "cuda", dtype=dtype)
    rows = _rows(w, seed=k)
    fp8 = dtype == torch.float8_e4m3fn
    scales = dict(q_dequant_scale=FP8_SCALES[0], k_dequant_scale=FP8_SCALES[1],
                  v_dequant_scale=FP8_SCALES[2]) if fp8 else {}

    def forward(k_, v_, mode=0, with_lse=True, **layout):
        o_, l_ = gbsa.forward(q, k_, v_, t["idx"], t["cnt"], [w.block_x, 128], metadata=meta,
                              cu_seqlens_q=t["cu"], seqused_q=t["squ"], seqused_kv=t["sku"],
                              softmax_scale=w.scale, win_left=w.win_left, win_right=w.win_right,
                              return_softmax_lse=with_lse, num_ctas=ctas,
                              max_blocks_per_split=forced, softmax_precision=mode, **scales,
                              **layout)
        torch.cuda.synchronize()
        return o_, l_

    o1, l1 = forward(pool_view(w, kf), pool_view(w, vf), mode=1, block_table=t["bt"])
    _check_mode1(w, q, kf, vf, o1, l1, rows, dtype)

    out, lse = forward(pool_view(w, kf), pool_view(w, vf), block_table=t["bt"])
    # without the lse output, out is the same
    o_nl, _ = forward(pool_view(w, kf), pool_view(w, vf), with_lse=False, block_table=t["bt"])
    assert torch.equal(out, o_nl)
    kt, vt, cu_kv = tnd_kv(w, kf, vf, seed=k)
    if cu_kv[-1] > 0:  # a TND K/V array needs at least one row
        to, tl = forward(kt, vt, cu_seqlens_kv=torch.as_tensor(cu_kv, device="cuda"))
        assert torch.equal(out, to) and torch.equal(lse, tl)
    if fp8:
        _check_e4m3(w, q, kf, vf, out, lse, rows)
        return
    assert out.dtype == dtype
    ro, rl = oracle_rows(w, q.cpu(), kf.cpu(), vf.cpu(), rows)
    o = out.float().cpu().numpy().astype(np.float64)[rows[:, 0], rows[:, 1]]
    l = lse.float().cpu().numpy()[..., 0].astype(np.float64)[rows[:, 0], rows[:, 1]]
    assert_out_close(o, ro)
    assert_lse_close(l, rl)


def _check_e4m3(w, q, kf, vf, out, lse, rows):
    """The E4M3 bound of test_gpu_fp8 (the weights' E4M3 cast: 2^-4 of
    out_abs, 2^-10 of the smallest weights; bf16 out; fp32 sums); the mean
    error condition only where enough rows see a key."""
    assert out.dtype == torch.bfloat16
    ro, rl, ra = oracle_rows_fp8(w, q.cpu(), kf.cpu(), vf.cpu(), FP8_SCALES, rows)
    o = out.float().cpu().numpy().astype(np.float64)[rows[:, 0], rows[:, 1]]
    l = lse.float().cpu().numpy()[..., 0].astype(np.float64)[rows[:, 0], rows[:, 1]]
    assert_lse_close(l, rl)
    fin = np.isfinite(rl)
    assert (o[~fin] == 0).all()
    vmax = float(vf.float().nan_to_num(0.0).abs().max()) * abs(FP8_SCALES[2])
    bound = (2.0 ** -4 + 1e-5) * ra + 2.0 ** -8 * np.abs(ro) + 2.0 ** -18 * w.top_k * PAGE * vmax
    err = np.abs(o - ro)
    assert (err <= bound).all(), f"max excess {np.max(err - bound):.3g}"
    if fin.sum() >= 100:
        assert err[fin].mean() <= 0.25 * ((2.0 ** -4) * ra[fin]).mean()


def _check_mode1(w, q, kf, vf, out, lse, rows, dtype):
    """softmaxPrecision 1 under R24 (per element; the mean error condition
    only where enough rows see a key)."""
    name = {torch.bfloat16: "bf16", torch.float16: "fp16", torch.float8_e4m3fn: "e4m3"}[dtype]
    scales = FP8_SCALES if name == "e4m3" else (1.0, 1.0, 1.0)
    ro, rl, oa, ga = oracle_mode1(w, q, kf, vf, rows, scales)
    o = out.float().cpu().numpy().astype(np.float64)[rows[:, 0], rows[:, 1]]
    l = lse.float().cpu().numpy()[..., 0].astype(np.float64)[rows[:, 0], rows[:, 1]]
    assert_lse_close_r24(l, rl, keys_bound(w, rows))
    fin = np.isfinite(rl)
    assert (o[~fin] == 0).all()
    vmax = float(vf.float().nan_to_num(0.0).abs().max()) * abs(scales[2])
    bound = r24_bound(name, ro, oa, ga, keys_bound(w, rows), vmax)
    err = np.abs(o - ro)
    assert (err <= bound).all(), f"mode 1: max excess {np.max(err - bound):.3g}"
    if fin.sum() >= 100:
        mean_scale = (2.0 ** -4 * oa if name == "e4m3" else
                      2.0 * ((2.0 ** -9.9 + 8 * math.log(2) * 2.0 ** -11) * oa + 2.0 ** -11 * ga))
        assert err[fin].mean() <= 0.25 * mean_scale[fin].mean()


@pytest.mark.parametrize("k", range(0, N_CASES, 10))
def test_fuzz_backward(k):
    """The gradients of every tenth random problem (16-bit element types)
    against the oracle's, under the bound of test_gpu_backward (R25)."""
    from tests.test_gpu_backward import _check, _compact
    import oracle
    from tests.helpers import bf16_bits, elem_dtype

    w, dtype, ctas, forced = fuzz_case(k)
    if dtype == torch.float8_e4m3fn:
        dtype = torch.bfloat16
    t = device_tensors(w)
    meta = run_metadata(w, t, ctas, forced)
    q, kf, vf = make_values(w, "cuda", dtype=dtype)
    g = torch.Generator(device="cuda").manual_seed(9000 + k)
    dout = torch.randn(q.shape, generator=g, device="cuda", dtype=torch.float32).to(dtype)
    kw = dict(metadata=meta, cu_seqlens_q=t["cu"], seqused_q=t["squ"], seqused_kv=t["sku"],
              block_table=t["bt"], softmax_scale=w.scale, win_left=w.win_left,
              win_right=w.win_right, num_ctas=ctas, max_blocks_per_split=forced)
    kp, vp = pool_view(w, kf), pool_view(w, vf)
    out, lse = gbsa.forward(q, kp, vp, t["idx"], t["cnt"], [w.block_x, 128],
                            return_softmax_lse=True, **kw)
    dq, dk, dv = gbsa.backward(dout, q, kp, vp, out, lse, t["idx"], t["cnt"], [w.block_x, 128],
                               **kw)
    torch.cuda.synchronize()
    ref = oracle.attention_backward(
        q_bits=bf16_bits(q), k_bits=bf16_bits(kf), v_bits=bf16_bits(vf), dout_bits=bf16_bits(dout),
        kv_page_stride=w.kv_page_stride, num_pages=w.num_pages, sparse_idx=w.sparse_idx,
        sparse_count=w.sparse_count, cu_seqlens_q=w.cu_seqlens_q, seqused_q=w.seqused_q,
        seqused_kv=w.kv_used, block_table=w.block_table, block_x=w.block_x, scale=w.scale,
        win_left=w.win_left, win_right=w.win_right, dtype=elem_dtype(q), with_abs=True)
    ref = [r if i % 3 == 0 else _compact(w, r) for i, r in enumerate(ref)]
    if np.abs(ref[0]).max() == 0 and np.abs(ref[2]).max() == 0:
        pytest.skip("no row sees a key")
    _check((dq, dk, dv), ref)
