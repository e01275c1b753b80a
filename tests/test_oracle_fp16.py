"""Pins of the oracle's fp16 input path (a NEXT-row widening: fp16 Q/K/V with
the fp32 softmax of softmaxPrecision 0, GBSA article "Constraints: data
types").  The decode is checked against numpy over every bit pattern, the
attention against the brute-force formulation with numpy's decoder, and the
dtype switch against values both types hold exactly."""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_paged_gbsa_b200.workloads import generate, make_values, workload
from tests.helpers import brute_force, oracle_all, to_f64

ALL = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)


def _same_or_both_nan(a, b):
    a, b = np.asarray(a), np.asarray(b)
    return bool(np.all((a == b) | (np.isnan(a) & np.isnan(b))))


def test_fp16_decode_matches_numpy_on_every_pattern():
    got = oracle.widen(ALL, "fp16")
    assert _same_or_both_nan(got, ALL.view(np.float16).astype(np.float64))
    assert np.signbit(got[0x8000]) and got[0x8000] == 0.0    # -0
    assert got[0x0001] == 2.0 ** -24 and got[0x7bff] == 65504.0


def test_bf16_decode_matches_binary32_upper_half_on_every_pattern():
    got = oracle.widen(ALL, "bf16")
    with np.errstate(invalid="ignore"):  # signalling-NaN patterns
        ref = (ALL.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert _same_or_both_nan(got, ref)


@pytest.mark.parametrize("case", ["tiny_s2", "window"])
def test_fp16_oracle_matches_brute_force(case):
    w = {"tiny_s2": lambda: workload("tiny", scale_down=2),
         "window": lambda: generate(name="w16", seed=5, q_storage=[150, 70], q_used=[140, 70],
                                    kv_used=[300, 70], N1=4, N2=2, block_x=32, top_k=3,
                                    selection="random_causal", win_left=90, win_right=0)}[case]()
    q, kf, vf = make_values(w, "cpu", dtype=torch.float16)
    out, lse = oracle_all(w, q, kf, vf)
    bo, bl = brute_force(w, q, kf, vf)
    fin = np.isfinite(bl)
    assert np.array_equal(np.isneginf(lse), np.isneginf(bl))
    assert np.abs(out - bo).max() < 1e-12
    assert np.abs(lse[fin] - bl[fin]).max() < 1e-12


def test_dtype_switch_changes_only_the_decoding():
    # values on a 1/4 grid in [-2, 2] are exact in bf16 and fp16: the two
    # encodings must give bit-identical fp64 results
    w = workload("tiny", scale_down=4)
    q, kf, vf = make_values(w, "cpu", nan_fill=False)
    snap = lambda t: (torch.round(t.float().clamp(-2, 2) * 4) / 4)
    qb, kb, vb = (snap(t).to(torch.bfloat16) for t in (q, kf, vf))
    qh, kh, vh = (snap(t).to(torch.float16) for t in (q, kf, vf))
    ob, lb = oracle_all(w, qb, kb, vb)
    oh, lh = oracle_all(w, qh, kh, vh)
    assert np.array_equal(ob, oh) and np.array_equal(lb, lh)
    # and the flag is not ignored: fp16 bits read as bf16 give other values
    assert not np.array_equal(to_f64(qh.view(torch.int16).numpy().view(np.uint16), "bf16"),
                              to_f64(qh.view(torch.int16).numpy().view(np.uint16), "fp16"))
