"""Pins of the oracle's E4M3 path (the NEXT row "FP8 E4M3 with static
dequantization scales", GBSA article "Constraints: data types" and the
quantised-input arguments of the PyTorch API).  E4M3 values reach the oracle
through fp16, which holds every one of them exactly; the dequantization
scales fold into the score scale and the output.  Pinned here: the E4M3
decode against the format's definition on all 256 patterns, the fp16
conversion, the scale folding, and the out_abs error scale."""
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_paged_gbsa_b200.workloads import make_values, workload
from tests.helpers import oracle_rows, oracle_rows_fp8

ALL8 = torch.arange(256, dtype=torch.int32).to(torch.uint8)


def _e4m3_by_definition(byte: int) -> float:
    # 1 sign bit, 4 exponent bits (bias 7), 3 fraction bits; exponent 0 holds
    # the subnormals f/8 * 2^-6; S.1111.111 is NaN and there is no infinity
    s, e, f = byte >> 7, (byte >> 3) & 0xF, byte & 7
    if e == 15 and f == 7:
        return math.nan
    mag = (f / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + f / 8.0) * 2.0 ** (e - 7)
    return -mag if s else mag


def test_e4m3_decode_matches_the_format_on_every_pattern():
    got = ALL8.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ref = np.array([_e4m3_by_definition(b) for b in range(256)])
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all()
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9


def test_e4m3_values_are_exact_in_fp16():
    x = ALL8.view(torch.float8_e4m3fn)
    via16 = x.to(torch.float16).to(torch.float64).numpy()
    direct = x.to(torch.float64).numpy()
    assert ((via16 == direct) | (np.isnan(via16) & np.isnan(direct))).all()


def _fp8_inputs(w):
    q, kf, vf = make_values(w, "cpu", nan_fill=False)
    return tuple(t.float().clamp(-448, 448).to(torch.float8_e4m3fn) for t in (q, kf, vf))


def test_scales_fold_into_scores_and_output():
    # the same E4M3 codes with scales (qs, ks, vs) equal the dequantised values
    # qs*q, ks*k, vs*v run through the plain oracle (powers of two keep the
    # products exact in fp16)
    w = workload("tiny", scale_down=4)
    q8, k8, v8 = _fp8_inputs(w)
    qs, ks, vs = 0.5, 2.0, 0.25
    rows = np.stack([np.arange(w.T).repeat(w.N1), np.tile(np.arange(w.N1), w.T)], 1)
    out, lse, _ = oracle_rows_fp8(w, q8, k8, v8, (qs, ks, vs), rows)
    deq = lambda t, s: (t.to(torch.float16) * s)
    ro, rl = oracle_rows(w, deq(q8, qs), deq(k8, ks), deq(v8, vs), rows)
    assert np.array_equal(out, ro) and np.array_equal(lse, rl)


def test_out_abs_is_the_weighted_absolute_value():
    # V -> |V| leaves the weights unchanged, so out_abs must equal the output
    # of the same rows with |V|
    w = workload("tiny", scale_down=4)
    q8, k8, v8 = _fp8_inputs(w)
    rows = np.stack([np.arange(w.T).repeat(w.N1), np.tile(np.arange(w.N1), w.T)], 1)
    _, _, oa = oracle_rows_fp8(w, q8, k8, v8, (1.0, 1.0, 1.0), rows)
    ra, _, _ = oracle_rows_fp8(w, q8, k8, v8.abs(), (1.0, 1.0, 1.0), rows)
    assert np.allclose(oa, ra, rtol=1e-14, atol=0)
    assert (oa >= 0).all()
