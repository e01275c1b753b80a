"""softmaxPrecision 1 (GBSA article, "Softmax precision": the softmax in half
precision with the rescale in fp32) against the fp64 oracle, for bf16, fp16
and E4M3 inputs.

What the kernel computes in this mode: the exponent x = s * scale * log2(e) -
m (m the running reference max, at most 8 -- E4M3: 0.5 -- below the row max
M, fp32) is rounded to f16, one ex2.approx.f16x2 gives two weights P in f16;
the row sum adds those f16 weights in fp32; P enters the P.V product as f16
(fp16), rounded to bf16 (bf16) or cast to E4M3 after the 2^8 factor (E4M3).

Tolerance (reading R24), per element, with S_p the natural-log scores:
* the f16 rounding of x errs by at most 2^-11 |x|, and |x_p| <= t_p + 8 with
  t_p = (M - S_p) log2(e), so P is off by a factor within
  2^-9.9 (the PTX bound of ex2.approx.f16) + ln2 * 2^-11 * (8 + t_p);
* out = sum P v / sum P, with the same P above and below, so a relative error
  d_p in each weight moves out by at most 2 (1 + 2^-8) sum_p w_p d_p |v_p|,
  i.e. 2 (1 + 2^-8) [(2^-9.9 + 8 ln2 2^-11) out_abs + 2^-11 gap_abs] with
  out_abs = sum w_p |v_p| and gap_abs = sum w_p (M - S_p) |v_p| from the
  oracle;
* weights below the f16 range (2^-24) are lost: at most n 2^-24 |v|max over
  the n visible keys;
* bf16: P rounded to bf16 in the product only, 2^-8 out_abs (bf16 keeps 8
  significant bits: u = 2^-8); E4M3: the R22
  bound of the weights' E4M3 cast on top;
* the 16-bit output: u |exact| (2^-8 for a bf16 out, E4M3 included; fp16,
  u = 2^-11, keeps 2^-9); fp32 accumulation: 1e-5 out_abs.
The rounding errors have no common sign, so the mean error must also stay a
small part of the mean bound (a systematic mistake would not)."""
import math

import numpy as np
import pytest
import torch

import block_sparse_paged_gbsa_b200 as gbsa
import oracle
from block_sparse_paged_gbsa_b200.workloads import (PAGE, bf16_bits, generate, make_values,
                                                    pool_view, workload)
from tests.gpu_helpers import device_tensors, run_metadata
from tests.helpers import assert_lse_close_r24, keys_bound, r24_bound, r24_lse_bound

pytestmark = pytest.mark.gpu

DTYPES = {"bf16": torch.bfloat16, "fp16": torch.float16, "e4m3": torch.float8_e4m3fn}
SCALES = (0.37, 1.9, 0.61)  # E4M3 dequantization scales

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


def _run(w, q, kf, vf, mode, forced=0, scales=(1.0, 1.0, 1.0)):
    t = device_tensors(w)
    meta = run_metadata(w, t, forced=forced)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = gbsa.forward(q, pool_view(w, kf), pool_view(w, vf), t["idx"], t["cnt"],
                            [w.block_x, 128], metadata=meta, cu_seqlens_q=t["cu"],
                            seqused_q=t["squ"], seqused_kv=t["sku"], block_table=t["bt"],
                            softmax_scale=w.scale, win_left=w.win_left, win_right=w.win_right,
                            return_softmax_lse=True, max_blocks_per_split=forced,
                            dev_status=status, softmax_precision=mode,
                            q_dequant_scale=scales[0], k_dequant_scale=scales[1],
                            v_dequant_scale=scales[2])
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return out, lse


def _rows(w, limit=40000, seed=0):
    if w.T * w.N1 <= limit:
        tt, hh = np.meshgrid(np.arange(w.T), np.arange(w.N1), indexing="ij")
        return np.stack([tt.reshape(-1), hh.reshape(-1)], 1).astype(np.int64)
    rng = np.random.default_rng(seed)
    ends = np.concatenate([w.cu_seqlens_q[:-1], w.cu_seqlens_q[1:] - 1])
    tok = np.concatenate([rng.integers(0, w.T, 3000), ends[(ends >= 0) & (ends < w.T)]])
    return np.stack([tok, rng.integers(0, w.N1, tok.size)], 1).astype(np.int64)


def _oracle(w, q, kf, vf, rows, scales):
    """out, lse, out_abs and gap_abs of the rows (E4M3 values go to the
    oracle as fp16, exactly, with the scales folded in)."""
    fp8 = q.dtype == torch.float8_e4m3fn
    if fp8:
        q, kf, vf = (t.to(torch.float16) for t in (q, kf, vf))
    dt = "bf16" if q.dtype == torch.bfloat16 else "fp16"
    qs, ks, vs = scales if fp8 else (1.0, 1.0, 1.0)
    n = rows.shape[0]
    oa, ga = np.zeros((n, w.D)), np.zeros((n, w.D))
    out, lse = oracle.attention_rows(
        q_bits=bf16_bits(q.cpu()), k_bits=bf16_bits(kf.cpu()), v_bits=bf16_bits(vf.cpu()),
        kv_page_stride=w.kv_page_stride, num_pages=w.num_pages, sparse_idx=w.sparse_idx,
        sparse_count=w.sparse_count, cu_seqlens_q=w.cu_seqlens_q, seqused_q=w.seqused_q,
        seqused_kv=w.kv_used, block_table=w.block_table, block_x=w.block_x,
        scale=w.scale * qs * ks, win_left=w.win_left, win_right=w.win_right, rows=rows,
        dtype=dt, out_abs=oa, gap_abs=ga)
    return out * vs, lse, oa * abs(vs), ga * abs(vs)


def _check_mode1(w, dtype, forced=0):
    tdt = DTYPES[dtype]
    scales = SCALES if dtype == "e4m3" else (1.0, 1.0, 1.0)
    q, kf, vf = make_values(w, "cuda", dtype=tdt)
    out, lse = _run(w, q, kf, vf, 1, forced, scales)
    rows = _rows(w)
    ro, rl, oa, ga = _oracle(w, q, kf, vf, rows, scales)
    o = out.float().cpu().numpy().astype(np.float64)[rows[:, 0], rows[:, 1]]
    l = lse.cpu().numpy()[..., 0].astype(np.float64)[rows[:, 0], rows[:, 1]]
    assert_lse_close_r24(l, rl, keys_bound(w, rows))
    fin = np.isfinite(rl)
    assert (o[~fin] == 0).all()
    vmax = float(vf.float().nan_to_num(0.0).abs().max()) * abs(scales[2])
    bound = r24_bound(dtype, ro, oa, ga, keys_bound(w, rows), vmax)
    err = np.abs(o - ro)
    assert (err <= bound).all(), f"max excess {np.max(err - bound):.3g}"
    mean_scale = (2.0 ** -4 * oa if dtype == "e4m3" else
                  2.0 * ((2.0 ** -9.9 + 8 * math.log(2) * 2.0 ** -11) * oa + 2.0 ** -11 * ga))
    assert err[fin].mean() <= 0.25 * mean_scale[fin].mean()
    return q, kf, vf, out, lse, err[fin]


@pytest.mark.parametrize("dtype", sorted(DTYPES))
@pytest.mark.parametrize("name", sorted(CASES))
def test_mode1_matches_oracle(name, dtype):
    _check_mode1(CASES[name](), dtype)


@pytest.mark.parametrize("dtype", sorted(DTYPES))
@pytest.mark.parametrize("name", ["decode_s16", "g8_bx16_window"])
def test_mode1_forced_splits(name, dtype):
    _check_mode1(CASES[name](), dtype, forced=3)


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_mode1_is_its_own_path(dtype):
    """Mode 1 is not the fp32 softmax (the outputs differ somewhere) and stays
    close to it; its typical error is a small part of the raw 1e-2 target."""
    w = CASES["dense_s16"]()
    q, kf, vf, o1, l1, err = _check_mode1(w, dtype)
    o0, l0 = _run(w, q, kf, vf, 0)
    assert not torch.equal(o0, o1)
    # two roundings of nearly equal values may differ by one 16-bit spacing
    diff = (o0.float() - o1.float()).abs()
    assert (diff <= 1e-2 + 2.0 ** -8 * o0.float().abs()).all()
    # lse: mode 0 within 1e-3 of the exact value, mode 1 within R24's bound
    # (at most top_k * 128 visible keys); typically far closer
    fin = torch.isfinite(l0)
    l0n = l0[fin].double().cpu().numpy()
    dl = np.abs(l0n - l1[fin].double().cpu().numpy())
    assert (dl <= 1e-3 + r24_lse_bound(np.full(dl.shape, w.top_k * PAGE), l0n)).all()
    assert float(np.median(dl)) < 1e-3
    assert float(np.median(err)) < 1e-3


def test_mode1_dense_full_size_sampled_rows():
    """The full dense workload in the benchmark's launch configuration."""
    _check_mode1(workload("dense"), "bf16")
