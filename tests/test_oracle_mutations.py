"""The pins must have teeth: plant plausible mistakes in a copy of the oracle's
C source (on the CPU), rebuild it, and check that the pin checks reject every
mutant while accepting the unmodified source."""
import glob
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from block_sparse_paged_gbsa_b200.workloads import (bf16_bits, generate, make_values, tnd_kv,
                                                    workload)
from tests.helpers import brute_force, logical_kv, oracle_all, oracle_rows, to_f64
from tests.test_oracle_pins import GOLDEN, _fixture_workload

SRC = os.path.join(os.path.dirname(oracle.__file__), "gbsa_oracle.c")

MUTANTS = {
    "top_left_causal": ("const int64_t pos = t + (ku - qu);", "const int64_t pos = t;"),
    "head_modulo": ("const int32_t kvh = h / G;", "const int32_t kvh = h % c->N2;"),
    "dropped_scale": ("score[i] = c->scale * dot;", "score[i] = dot;"),
    "window_off_by_one": ("p < pos - c->win_left", "p <= pos - c->win_left"),
    "no_block_table": ("page = c->block_table[(int64_t)b * c->max_pages_per_seq + lb];",
                       "page = lb;"),
    "lse_without_max": ("*lse = m + log(l);", "*lse = log(l);"),
    "qblock_without_base": ("const int64_t qb = c->q_block_base[b] + t / c->block_x;",
                            "const int64_t qb = t / c->block_x;"),
    "softmax_sign": ("const double w = exp(score[i] - m) / l;", "const double w = exp(m - score[i]) / l;"),
    "v_head_row_swapped": (
        "c->v + key_page[i] * c->kv_page_stride + ((int64_t)key_row[i] * c->N2 + kvh) * D;",
        "c->v + key_page[i] * c->kv_page_stride + ((int64_t)kvh * 128 + key_row[i]) * D;"),
    "seqused_q_ignored": ("const int64_t qu = c->seqused_q ? (int64_t)c->seqused_q[b] : qs;",
                          "const int64_t qu = qs;"),
    "count_not_clamped": ("if (n > c->top_k) n = c->top_k;", "if (n > c->top_k + 1) n = c->top_k + 1;"),
    "causal_strict": ("if (p > pos) continue;", "if (p >= pos) continue;"),
    # the fp16 decoder, the TND addressing and the E4M3 error scale
    "fp16_subnormal_scale": ("mag = ldexp((double)f, -24);", "mag = ldexp((double)f, -25);"),
    "fp16_exponent_bias": ("mag = ldexp((double)(1024 + f), e - 25);",
                           "mag = ldexp((double)(1024 + f), e - 24);"),
    "tnd_without_sequence_base": ("key_page[nk] = c->cu_seqlens_kv[b] + p;", "key_page[nk] = p;"),
    # a token at the start of a sequence given to an empty sequence that
    # shares its start (walking back to the first sequence starting there)
    "empty_sequence_owner": (
        "  while (lo + 1 < c->B && c->cu_seqlens_q[lo + 1] <= tg) lo++;",
        "  while (lo > 0 && c->cu_seqlens_q[lo - 1] == c->cu_seqlens_q[lo]) lo--;"),
    # a Q-block base that counts every sequence as at least one block
    "empty_sequence_counts_a_block": ("acc += (qs + block_x - 1) / block_x;",
                                      "acc += qs > 0 ? (qs + block_x - 1) / block_x : 1;"),
    "gap_abs_signed": ("gap_abs[d] += w * (m - score[i]) * fabs(c->widen(vrow[d]));",
                       "gap_abs[d] += w * (score[i] - m) * fabs(c->widen(vrow[d]));"),
    "gap_abs_unweighted": ("gap_abs[d] += w * (m - score[i]) * fabs(c->widen(vrow[d]));",
                           "gap_abs[d] += (m - score[i]) * fabs(c->widen(vrow[d]));"),
    "out_abs_signed": ("out_abs[d] += w * fabs(c->widen(vrow[d]));",
                       "out_abs[d] += w * c->widen(vrow[d]);"),
}


def _golden_ok(lib):
    for path in sorted(glob.glob(os.path.join(GOLDEN, "*.json"))):
        if path.endswith("example_call_shapes.json") or os.path.basename(path).startswith("e4m3_"):
            continue
        fx = json.load(open(path))
        w, q, kf, vf = _fixture_workload(fx)
        rows = np.array([[e["t"], e["h"]] for e in fx["expected"]], np.int64)
        try:
            out, lse = oracle_rows(w, q, kf, vf, rows, lib=lib)
        except ValueError:
            return False
        for i, e in enumerate(fx["expected"]):
            if abs(lse[i] - e["lse"]) > 1e-12:
                return False
            if any(abs(out[i, int(d)] - val) > 1e-12 for d, val in e["out"].items()):
                return False
    return True


def _brute_ok(lib):
    cases = [
        dict(q_storage=[200, 77], q_used=[190, 77], kv_used=[230, 77], N1=4, N2=2, block_x=64,
             top_k=3, selection="random_causal", win_left=90, win_right=0),
        dict(q_storage=[1, 1], q_used=[1, 1], kv_used=[300, 129], N1=4, N2=2, block_x=1,
             top_k=4, selection="decode", count_range=(1, 4)),
    ]
    for i, c in enumerate(cases):
        w = generate(name=f"m{i}", seed=300 + i, **c)
        w.sparse_count[0, 0] = w.top_k + 3          # exercises the count clamp
        q, kf, vf = make_values(w, "cpu")
        try:
            out, lse = oracle_all(w, q, kf, vf, lib=lib)
        except ValueError:
            return False
        bo, bl = brute_force(w, q, kf, vf)
        if not np.allclose(out, bo, atol=1e-10, rtol=0, equal_nan=False):
            return False
        if not np.array_equal(np.isneginf(lse), np.isneginf(bl)):
            return False
        fin = np.isfinite(bl)
        if not np.allclose(lse[fin], bl[fin], atol=1e-10, rtol=0):
            return False
    return True


def _sdpa_ok(lib):
    w = generate(name="sd", seed=21, q_storage=[256], N1=4, N2=2, block_x=128, top_k=2,
                 selection="all_causal")
    q, kf, vf = make_values(w, "cpu")
    out, _ = oracle_all(w, q, kf, vf, lib=lib)
    qq = q.double().transpose(0, 1)
    K = torch.from_numpy(logical_kv(w, bf16_bits(kf), 0)).transpose(0, 1).repeat_interleave(2, 0)
    V = torch.from_numpy(logical_kv(w, bf16_bits(vf), 0)).transpose(0, 1).repeat_interleave(2, 0)
    ref = torch.nn.functional.scaled_dot_product_attention(qq, K, V, is_causal=True, scale=w.scale)
    return np.allclose(out, ref.transpose(0, 1).numpy(), atol=1e-10, rtol=0)


def _widen_ok(lib):
    # both decoders against numpy's on every 16-bit pattern
    bits = np.arange(65536, dtype=np.uint16)
    for dt in ("bf16", "fp16"):
        with np.errstate(invalid="ignore"):  # the NaN patterns
            got, ref = oracle.widen(bits, dt, lib=lib), to_f64(bits, dt)
        if not ((got == ref) | (np.isnan(got) & np.isnan(ref))).all():
            return False
    return True


def _rows(lib, w, q, k, v, rows, **kw):
    args = dict(kv_page_stride=w.kv_page_stride, num_pages=w.num_pages,
                block_table=w.block_table)
    args.update(kw)
    return oracle.attention_rows(
        q_bits=bf16_bits(q), k_bits=bf16_bits(k), v_bits=bf16_bits(v), sparse_idx=w.sparse_idx,
        sparse_count=w.sparse_count, cu_seqlens_q=w.cu_seqlens_q, seqused_q=w.seqused_q,
        seqused_kv=w.kv_used, block_x=w.block_x, scale=w.scale, win_left=w.win_left,
        win_right=w.win_right, rows=rows, lib=lib, **args)


def _all_rows(w):
    return np.stack([np.arange(w.T).repeat(w.N1), np.tile(np.arange(w.N1), w.T)], 1)


def _tnd_ok(lib):
    # the same logical keys in the TND layout give the paged pool's rows
    w = generate(name="tw", seed=9, q_storage=[300, 90], q_used=[290, 90], kv_used=[500, 130],
                 N1=4, N2=2, block_x=64, top_k=4, selection="random_causal", win_left=150,
                 win_right=0, page_stride_factor=1.25)
    q, kf, vf = make_values(w, "cpu")
    kt, vt, cu = tnd_kv(w, kf, vf)
    rows = _all_rows(w)
    po, pl = _rows(lib, w, q, kf, vf, rows)
    to, tl = _rows(lib, w, q, kt, vt, rows, kv_page_stride=0, num_pages=0, block_table=None,
                   cu_seqlens_kv=cu)
    return np.array_equal(po, to) and np.array_equal(pl, tl) and np.isfinite(to).all()


def _out_abs_ok(lib):
    # out_abs is the output on |V| (the weights do not see V)
    w = workload("tiny", scale_down=4)
    q, kf, vf = make_values(w, "cpu", nan_fill=False)
    rows = _all_rows(w)
    oa = np.zeros((rows.shape[0], w.D))
    _rows(lib, w, q, kf, vf, rows, out_abs=oa)
    ra, _ = _rows(lib, w, q, kf, vf.abs(), rows)
    return bool(np.allclose(oa, ra, rtol=1e-14, atol=0) and (oa >= 0).all())


def _gap_abs_ok(lib):
    # gap_abs against the brute force's sum_p w_p (max s - s_p) |v_p|
    w = generate(name="ga", seed=12, q_storage=[150, 60], N1=4, N2=2, block_x=32, top_k=3,
                 selection="random_causal", win_left=70, win_right=0)
    q, kf, vf = make_values(w, "cpu")
    rows = _all_rows(w)
    ga = np.zeros((rows.shape[0], w.D))
    _rows(lib, w, q, kf, vf, rows, gap_abs=ga)
    _, _, bg = brute_force(w, q, kf, vf, gap=True)
    return bool(np.allclose(ga, bg.reshape(-1, w.D), atol=1e-10, rtol=0) and (ga >= 0).all())


def _all_pins_pass(lib):
    return (_golden_ok(lib) and _brute_ok(lib) and _sdpa_ok(lib) and _widen_ok(lib) and
            _tnd_ok(lib) and _out_abs_ok(lib) and _gap_abs_ok(lib))


def test_unmodified_oracle_passes(tmp_path):
    lib = oracle.load_library(oracle.compile_to(SRC, str(tmp_path / "orig.so")))
    assert _all_pins_pass(lib)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(old, new))
    lib = oracle.load_library(oracle.compile_to(str(path), str(tmp_path / f"{name}.so")))
    assert not _all_pins_pass(lib), f"pins did not catch the planted mistake {name!r}"
