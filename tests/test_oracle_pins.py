"""Pins for the fp64 oracle: each test ties it to something other than itself
(closed forms, hand-derived fixtures, a library routine, brute-force
enumeration, invariants), so that a dropped term, a wrong sign or index, or a
transposed operand in the oracle fails at least one of them."""
import glob
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from block_sparse_paged_gbsa_b200.workloads import PAGE, bf16_bits, generate, make_values, workload
from tests.helpers import brute_force, oracle_all, oracle_rows, to_f64

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------
# golden fixtures: hand-derived closed forms
# --------------------------------------------------------------------------
def _fixture_workload(fx):
    p = fx["problem"]
    w = generate(name="fixture", seed=5, q_storage=p["q_storage"], q_used=p["q_used"],
                 kv_used=p["kv_used"], N1=p["N1"], N2=p["N2"], block_x=p["block_x"],
                 top_k=p["top_k"], selection="random_causal", win_left=p["win_left"],
                 win_right=p["win_right"], scale=p["scale"])
    lists = fx["lists"]            # [N2][qb] -> list
    for kvh, per_qb in enumerate(lists):
        for qb, lst in enumerate(per_qb):
            w.sparse_count[kvh, qb] = len(lst)
            w.sparse_idx[kvh, qb, :len(lst)] = lst
    q = torch.zeros((w.T, w.N1, w.D), dtype=torch.bfloat16)
    kf = torch.zeros((w.pool_elems,), dtype=torch.bfloat16)
    vf = torch.zeros((w.pool_elems,), dtype=torch.bfloat16)

    def place(pool, p_log, kvh, d, val, b=0):
        page = int(w.block_table[b, p_log // PAGE])
        pool[page * w.kv_page_stride + ((p_log % PAGE) * w.N2 + kvh) * w.D + d] = val

    for t, h, d, val in fx["q"]:
        q[t, h, d] = val
    # entries [position, kvh, d, value] of sequence 0, or [..., b] of sequence b
    for e in fx["k"]:
        place(kf, *e)
    if fx["v"] == "ramp":
        for p_log in range(int(w.kv_used[0])):
            for kvh in range(w.N2):
                place(vf, p_log, kvh, 0, float(p_log))
    else:
        for e in fx["v"]:
            place(vf, *e)
    return w, q, kf, vf


@pytest.mark.parametrize("path", sorted(p for p in glob.glob(os.path.join(GOLDEN, "*.json"))
                                        if not p.endswith("example_call_shapes.json")
                                        and not os.path.basename(p).startswith("e4m3_")))
def test_golden_fixture(path):
    fx = json.load(open(path))
    w, q, kf, vf = _fixture_workload(fx)
    rows = np.array([[e["t"], e["h"]] for e in fx["expected"]], np.int64)
    out, lse = oracle_rows(w, q, kf, vf, rows)
    for i, e in enumerate(fx["expected"]):
        assert lse[i] == pytest.approx(e["lse"], abs=1e-12), (path, e)
        for d, val in e["out"].items():
            assert out[i, int(d)] == pytest.approx(val, abs=1e-12), (path, e, d)
    # the brute-force formulation agrees on the same fixture
    bo, bl = brute_force(w, q, kf, vf)
    for i, e in enumerate(fx["expected"]):
        assert bl[e["t"], e["h"]] == pytest.approx(e["lse"], abs=1e-12)


def test_example_call_shapes():
    """The pages' Python example: out has q's shape, lse is (T, N1, 1); its
    randint(0, 2) indices repeat blocks and must be accepted."""
    fx = json.load(open(os.path.join(GOLDEN, "example_call_shapes.json")))
    p = fx["problem"]
    rng = np.random.default_rng(0)
    w = generate(name="example", seed=11, q_storage=[p["Q_S"]], q_used=[p["Q_S"]],
                 kv_used=[p["KV_S"]], N1=p["N1"], N2=p["N2"], block_x=p["block_x"],
                 top_k=p["top_k"], selection="random_any", extra_pages=0)
    nb = fx["expected"]["num_blocks"]
    assert w.total_q_blocks == fx["expected"]["total_q_blocks"]
    assert w.num_pages == nb
    w.block_table[0, :nb] = np.arange(nb)
    w.sparse_idx[:] = rng.integers(0, nb, size=w.sparse_idx.shape)
    w.sparse_count[:] = p["top_k"]
    q, kf, vf = make_values(w, "cpu")
    out, lse = oracle_all(w, q, kf, vf)
    assert list(out.shape) == fx["expected"]["out_shape"]
    assert list(lse[..., None].shape) == fx["expected"]["lse_shape"]
    bo, bl = brute_force(w, q, kf, vf)
    np.testing.assert_allclose(out, bo, atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse, bl, atol=1e-12, rtol=0)


# --------------------------------------------------------------------------
# brute-force enumeration on tiny random cases
# --------------------------------------------------------------------------
TINY_CASES = [
    dict(q_storage=[200, 77], N1=4, N2=2, block_x=64, top_k=3, selection="random_causal"),
    dict(q_storage=[300], N1=2, N2=1, block_x=16, top_k=4, selection="random_causal",
         win_left=70, win_right=0),
    dict(q_storage=[150, 260], q_used=[140, 200], kv_used=[170, 200], N1=4, N2=4,
         block_x=32, top_k=3, selection="random_causal", page_stride_factor=1.5),
    dict(q_storage=[1, 1, 1], q_used=[1, 1, 1], kv_used=[300, 5, 129], N1=4, N2=2,
         block_x=1, top_k=4, selection="decode", count_range=(1, 4)),
    dict(q_storage=[90, 130], N1=3, N2=1, block_x=7, top_k=5, selection="random_any"),
    dict(q_storage=[256], q_used=[250], kv_used=[299], N1=2, N2=2, block_x=128, top_k=3,
         selection="random_causal", win_left=5, win_right=3),
]


@pytest.mark.parametrize("case", range(len(TINY_CASES)))
def test_brute_force_matches(case):
    w = generate(name=f"tiny{case}", seed=100 + case, **TINY_CASES[case])
    q, kf, vf = make_values(w, "cpu")
    out, lse = oracle_all(w, q, kf, vf)
    bo, bl = brute_force(w, q, kf, vf)
    assert np.isfinite(out).all()
    np.testing.assert_allclose(out, bo, atol=1e-12, rtol=0)
    inf = np.isneginf(bl)
    assert np.array_equal(np.isneginf(lse), inf)
    np.testing.assert_allclose(lse[~inf], bl[~inf], atol=1e-12, rtol=0)


def test_brute_force_matches_on_random_problems():
    # the same comparison on random tiny problems: sequence mixes with
    # unused rows, GQA groups, Q block sizes, list kinds (with duplicates and
    # masked blocks), both window sides, fp16 values and strided pools
    from hypothesis import HealthCheck, given, settings
    from hypothesis import strategies as st

    @settings(max_examples=40, deadline=None, derandomize=True,
              suppress_health_check=[HealthCheck.too_slow])
    @given(st.data())
    def run(data):
        # empty storage sequences (a repeated cu_seqlens_q value) and
        # sequences with seqused_kv = 0 are drawn too; one sequence is non-empty
        B = data.draw(st.integers(1, 3))
        qs = data.draw(st.lists(st.integers(0, 40), min_size=B, max_size=B))
        if sum(qs) == 0:
            qs[data.draw(st.integers(0, B - 1))] = data.draw(st.integers(1, 40))
        qu = [data.draw(st.integers(0, s)) for s in qs]
        ku = [data.draw(st.sampled_from([0, u]) | st.integers(0, u + 300)) for u in qu]
        N2 = data.draw(st.sampled_from([1, 2]))
        G = data.draw(st.sampled_from([1, 2, 3]))
        w = generate(name="hb", seed=data.draw(st.integers(0, 10_000)), q_storage=qs, q_used=qu,
                     kv_used=ku, N1=N2 * G, N2=N2, block_x=data.draw(st.sampled_from([1, 5, 16])),
                     top_k=data.draw(st.integers(1, 4)),
                     selection=data.draw(st.sampled_from(["random_causal", "random_any"])),
                     win_left=data.draw(st.sampled_from([-1, 0, 60])),
                     win_right=data.draw(st.sampled_from([-1, 0, 7])), has_seqused_q=True,
                     page_stride_factor=data.draw(st.sampled_from([1.0, 1.5])))
        dt = data.draw(st.sampled_from([torch.bfloat16, torch.float16]))
        q, kf, vf = make_values(w, "cpu", dtype=dt)
        out, lse = oracle_all(w, q, kf, vf)
        bo, bl = brute_force(w, q, kf, vf)
        np.testing.assert_allclose(out, bo, atol=1e-12, rtol=0)
        inf = np.isneginf(bl)
        assert np.array_equal(np.isneginf(lse), inf)
        np.testing.assert_allclose(lse[~inf], bl[~inf], atol=1e-12, rtol=0)

    run()


def test_counts_outside_range_and_bad_entries():
    """count > top_k is clamped, count < 0 is empty, entries outside the
    sequence's blocks contribute nothing (brute force applies the same reading)."""
    w = generate(name="bad", seed=3, q_storage=[256, 100], N1=2, N2=1, block_x=32, top_k=4,
                 selection="random_causal")
    w.sparse_count[0, 0] = 9
    w.sparse_count[0, 1] = -2
    w.sparse_idx[0, 2, 0] = 57
    w.sparse_idx[0, 3, 0] = -1
    w.sparse_count[0, 3] = max(w.sparse_count[0, 3], 1)
    q, kf, vf = make_values(w, "cpu")
    out, lse = oracle_all(w, q, kf, vf)
    bo, bl = brute_force(w, q, kf, vf)
    np.testing.assert_allclose(out, bo, atol=1e-12, rtol=0)
    assert np.all(np.isneginf(lse[32:64]))          # count < 0 -> no key for that Q block


# --------------------------------------------------------------------------
# special cases that reduce to a library routine or a closed form
# --------------------------------------------------------------------------
def test_all_causal_blocks_equal_dense_causal_sdpa():
    """Every causal block selected => dense causal attention; checked against
    torch's scaled_dot_product_attention in fp64 with GQA-expanded K/V."""
    w = generate(name="dense_small", seed=21, q_storage=[384, 256], N1=8, N2=2, block_x=128,
                 top_k=3, selection="all_causal")
    q, kf, vf = make_values(w, "cpu")
    out, lse = oracle_all(w, q, kf, vf)
    kb, vb = bf16_bits(kf), bf16_bits(vf)
    for b in range(w.B):
        t0, t1 = int(w.cu_seqlens_q[b]), int(w.cu_seqlens_q[b + 1])
        qq = q[t0:t1].double().transpose(0, 1)                       # [N1, S, D]
        from tests.helpers import logical_kv
        K = torch.from_numpy(logical_kv(w, kb, b)).transpose(0, 1)   # [N2, S, D]
        V = torch.from_numpy(logical_kv(w, vb, b)).transpose(0, 1)
        K = K.repeat_interleave(w.G, dim=0)
        V = V.repeat_interleave(w.G, dim=0)
        ref = torch.nn.functional.scaled_dot_product_attention(qq, K, V, is_causal=True,
                                                               scale=w.scale)
        np.testing.assert_allclose(out[t0:t1], ref.transpose(0, 1).numpy(), atol=1e-11, rtol=0)
        s = (qq @ K.transpose(1, 2)) * w.scale
        s = s.masked_fill(torch.ones_like(s, dtype=torch.bool).triu(1), -math.inf)
        np.testing.assert_allclose(lse[t0:t1], torch.logsumexp(s, -1).T.numpy(), atol=1e-11)


def test_values_all_ones_give_ones():
    """Softmax weights sum to 1: V = 1 gives out = 1 on every row with a key,
    V = c gives out = c."""
    w = workload("ragged", scale_down=16)
    q, kf, vf = make_values(w, "cpu")
    for c in (1.0, -2.5):
        vf2 = torch.where(torch.isnan(vf), vf, torch.full_like(vf, c))
        out, lse = oracle_all(w, q, kf, vf2)
        has = np.isfinite(lse)
        assert has.sum() > 100
        np.testing.assert_allclose(out[has], c, atol=1e-13, rtol=0)
        assert np.all(out[~has] == 0)


def test_single_key_row_closed_form():
    """A row with exactly one visible key: out = v exactly, lse = the score."""
    w = generate(name="single", seed=8, q_storage=[130], N1=2, N2=1, block_x=1, top_k=1,
                 selection="all_causal")
    # the first token of the sequence sees only key 0
    q, kf, vf = make_values(w, "cpu")
    kb, vb = bf16_bits(kf), bf16_bits(vf)
    out, lse = oracle_rows(w, q, kf, vf, np.array([[0, 0], [0, 1]]))
    page = int(w.block_table[0, 0])
    v0 = to_f64(vb[page * w.kv_page_stride:page * w.kv_page_stride + w.D])
    np.testing.assert_array_equal(out[0], v0)
    np.testing.assert_array_equal(out[1], v0)
    # score from a constructed q/k pair with an exactly known dot product
    q2 = torch.zeros_like(q)
    q2[0, 0, 5] = 3.0
    kf2 = kf.clone()
    kf2[page * w.kv_page_stride: page * w.kv_page_stride + w.D] = 0
    kf2[page * w.kv_page_stride + 5] = -0.25
    _, lse2 = oracle_rows(w, q2, kf2, vf, np.array([[0, 0]]))
    assert lse2[0] == pytest.approx(w.scale * 3.0 * -0.25, abs=1e-15)


def test_zero_queries_give_mean_of_visible_values():
    """q = 0: uniform weights, out = mean of v over the visible keys and
    lse = ln(#keys); with every causal block selected the visible keys of
    token t are 0..t, so out is the running mean of v (np.cumsum)."""
    w = generate(name="zeroq", seed=13, q_storage=[300], N1=2, N2=1, block_x=64, top_k=3,
                 selection="all_causal")
    q, kf, vf = make_values(w, "cpu")
    out, lse = oracle_all(w, torch.zeros_like(q), kf, vf)
    from tests.helpers import logical_kv
    V = logical_kv(w, bf16_bits(vf), 0)[:, 0, :]
    mean = np.cumsum(V, 0) / np.arange(1, 301)[:, None]
    for h in range(2):
        np.testing.assert_allclose(out[:, h], mean, atol=1e-12)
        np.testing.assert_allclose(lse[:, h], np.log(np.arange(1, 301)), atol=1e-13)


# --------------------------------------------------------------------------
# invariants
# --------------------------------------------------------------------------
def test_page_permutation_is_bit_identical():
    w = workload("tiny", scale_down=2)
    q, kf, vf = make_values(w, "cpu")
    out, lse = oracle_all(w, q, kf, vf)
    rng = np.random.default_rng(4)
    perm = rng.permutation(w.num_pages)           # physical page p moves to perm[p]
    k2, v2 = torch.empty_like(kf), torch.empty_like(vf)
    view = lambda f: f.view(w.num_pages, w.kv_page_stride)
    view(k2)[torch.as_tensor(perm)] = view(kf)
    view(v2)[torch.as_tensor(perm)] = view(vf)
    bt = w.block_table.copy()
    w.block_table[:] = np.where(bt >= 0, perm[np.maximum(bt, 0)], -1)
    out2, lse2 = oracle_all(w, q, k2, v2)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)
    # and the oracle really reads the table: the old table on moved pages differs
    w.block_table[:] = bt
    out3, _ = oracle_all(w, q, k2, v2)
    assert not np.array_equal(out, out3)


def test_page_stride_is_bit_identical():
    a = generate(name="s1", seed=31, q_storage=[256, 200], N1=4, N2=2, block_x=64, top_k=3,
                 selection="random_causal", page_stride_factor=1.0)
    b = generate(name="s2", seed=31, q_storage=[256, 200], N1=4, N2=2, block_x=64, top_k=3,
                 selection="random_causal", page_stride_factor=1.25)
    assert b.kv_page_stride > a.kv_page_stride
    q, kf, vf = make_values(a, "cpu")
    kb = torch.full((b.pool_elems,), float("nan"), dtype=torch.bfloat16)
    vb = kb.clone()
    pe = PAGE * a.N2 * a.D
    kb.view(b.num_pages, -1)[:, :pe] = kf.view(a.num_pages, -1)[:, :pe]
    vb.view(b.num_pages, -1)[:, :pe] = vf.view(a.num_pages, -1)[:, :pe]
    o1, l1 = oracle_all(a, q, kf, vf)
    o2, l2 = oracle_all(b, q, kb, vb)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_packed_gqa_equals_replicated_heads():
    w = generate(name="gqa", seed=41, q_storage=[200, 130], N1=8, N2=2, block_x=32, top_k=4,
                 selection="random_causal")
    q, kf, vf = make_values(w, "cpu")
    out, lse = oracle_all(w, q, kf, vf)
    G = w.G
    r = generate(name="gqa_rep", seed=41, q_storage=[200, 130], N1=8, N2=8, block_x=32,
                 top_k=4, selection="random_causal")
    r.block_table[:] = w.block_table
    r.sparse_idx = np.repeat(w.sparse_idx, G, axis=0)
    r.sparse_count = np.repeat(w.sparse_count, G, axis=0)
    r.num_pages, r.kv_page_stride = w.num_pages, PAGE * 8 * w.D

    def rep(f):
        pages = f.view(w.num_pages, w.kv_page_stride)[:, :PAGE * w.N2 * w.D]
        pages = pages.view(w.num_pages, PAGE, w.N2, w.D).repeat_interleave(G, dim=2)
        return pages.reshape(-1).contiguous()
    o2, l2 = oracle_all(r, q, rep(kf), rep(vf))
    assert np.array_equal(out, o2) and np.array_equal(lse, l2)


def test_padding_entries_and_unused_rows_change_nothing():
    w = workload("ragged", scale_down=16)
    q, kf, vf = make_values(w, "cpu")
    out, lse = oracle_all(w, q, kf, vf)
    rng = np.random.default_rng(9)
    j = np.arange(w.top_k)[None, None, :]
    pad = j >= w.sparse_count[:, :, None]
    w.sparse_idx = np.where(pad, rng.integers(-50, 500, size=w.sparse_idx.shape),
                            w.sparse_idx).astype(np.int32)
    q2 = q.clone()
    for b in range(w.B):                           # garbage in rows past seqused_q
        t0 = int(w.cu_seqlens_q[b]) + int(w.q_used[b])
        q2[t0:int(w.cu_seqlens_q[b + 1])] = float("nan")
    out2, lse2 = oracle_all(w, q2, kf, vf)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)
    for b in range(w.B):
        t0 = int(w.cu_seqlens_q[b]) + int(w.q_used[b])
        t1 = int(w.cu_seqlens_q[b + 1])
        assert np.all(out[t0:t1] == 0) and np.all(np.isneginf(lse[t0:t1]))


def test_oracle_rejects_bad_page():
    w = workload("tiny", scale_down=4)
    q, kf, vf = make_values(w, "cpu")
    w.block_table[0, 0] = w.num_pages + 3
    w.sparse_idx[0, 0, 0] = 0
    w.sparse_count[0, 0] = max(int(w.sparse_count[0, 0]), 1)
    with pytest.raises(ValueError):
        oracle_all(w, q, kf, vf)


@pytest.mark.parametrize("name", ["tiny", "window"])
def test_tnd_layout_equals_paged_pool(name):
    # the non-paged TND layout (k, v [T_kv, N2, D] with cu_seqlens_kv) holds the
    # same logical keys: the oracle must give bit-identical rows; NaN padding
    # between sequences must never be read
    from block_sparse_paged_gbsa_b200.workloads import tnd_kv
    from tests.helpers import oracle_all_tnd
    w = (workload("tiny") if name == "tiny" else
         generate(name="tw", seed=9, q_storage=[300, 90], q_used=[290, 90], kv_used=[500, 130],
                  N1=4, N2=2, block_x=64, top_k=4, selection="random_causal", win_left=150,
                  win_right=0, page_stride_factor=1.25))
    q, kf, vf = make_values(w, "cpu")
    kt, vt, cu = tnd_kv(w, kf, vf)
    po, pl = oracle_all(w, q, kf, vf)
    to, tl = oracle_all_tnd(w, q, kt, vt, cu)
    assert np.array_equal(po, to) and np.array_equal(pl, tl)
    assert np.isfinite(to).all()


def test_thread_count_changes_nothing():
    # rows are independent: any split of them over threads gives the same bits
    w = workload("tiny")
    q, kf, vf = make_values(w, "cpu")
    rows = np.stack([np.arange(w.T).repeat(w.N1), np.tile(np.arange(w.N1), w.T)], 1)
    o1, l1 = oracle_rows(w, q, kf, vf, rows, n_threads=1)
    for n in (2, 7):
        on, ln = oracle_rows(w, q, kf, vf, rows, n_threads=n)
        assert np.array_equal(o1, on) and np.array_equal(l1, ln)


@pytest.mark.parametrize("name", ["tiny", "window"])
def test_list_order_changes_nothing(name):
    """The selection is a set of blocks (a multiset with repeats): the same
    lists in ascending, descending and shuffled order give the same out and
    lse (to fp64 summation order), in the oracle and in the brute force."""
    def make(order):
        if name == "tiny":
            return workload("tiny", list_order=order)
        return generate(name="win", seed=41, q_storage=[300, 170], q_used=[290, 170],
                        kv_used=[310, 200], N1=4, N2=2, block_x=16, top_k=6,
                        selection="random_causal", win_left=90, win_right=0,
                        list_order=order)
    base = make("ascending")
    q, kf, vf = make_values(base, "cpu")
    ref_o, ref_l = oracle_all(base, q, kf, vf)
    for order in ("descending", "shuffled"):
        w = make(order)
        n = w.sparse_count
        for kvh in range(w.N2):
            for qb in range(w.total_q_blocks):
                c = int(n[kvh, qb])
                assert sorted(w.sparse_idx[kvh, qb, :c]) == sorted(base.sparse_idx[kvh, qb, :c])
        assert not np.array_equal(w.sparse_idx, base.sparse_idx)
        out, lse = oracle_all(w, q, kf, vf)
        np.testing.assert_allclose(out, ref_o, atol=1e-12, rtol=0)
        inf = np.isneginf(ref_l)
        assert np.array_equal(np.isneginf(lse), inf)
        np.testing.assert_allclose(lse[~inf], ref_l[~inf], atol=1e-12, rtol=0)
        bo, bl = brute_force(w, q, kf, vf)
        np.testing.assert_allclose(bo, ref_o, atol=1e-12, rtol=0)


def test_gap_abs_matches_brute_force_and_closed_forms():
    """gap_abs = sum_p w_p (m - s_p) |v_p| (the error scale of weights whose
    exponent is rounded in proportion to its size): equal to the brute
    force's, zero when every visible key has the same score (q = 0), and
    w_1 * 1 * |v_1| for two keys whose scores differ by 1."""
    w = generate(name="gp", seed=14, q_storage=[200, 90], q_used=[190, 90], kv_used=[260, 90],
                 N1=6, N2=2, block_x=16, top_k=4, selection="random_causal", win_left=80,
                 win_right=0)
    q, kf, vf = make_values(w, "cpu")
    tt, hh = np.meshgrid(np.arange(w.T), np.arange(w.N1), indexing="ij")
    rows = np.stack([tt.reshape(-1), hh.reshape(-1)], 1)
    ga = np.zeros((rows.shape[0], w.D))
    oracle_rows_gap(w, q, kf, vf, rows, ga)
    _, _, bg = brute_force(w, q, kf, vf, gap=True)
    np.testing.assert_allclose(ga, bg.reshape(-1, w.D), atol=1e-12, rtol=0)
    assert (ga >= 0).all() and ga.max() > 0
    # q = 0: every score is 0
    ga0 = np.zeros_like(ga)
    oracle_rows_gap(w, torch.zeros_like(q), kf, vf, rows, ga0)
    assert np.abs(ga0).max() == 0.0
    # two keys, scores 0 and -1 (scale 1, q.k = 0 and -1), v = 3 and -5 in dim 0
    t = generate(name="two", seed=15, q_storage=[1], q_used=[1], kv_used=[2], N1=1, N2=1,
                 block_x=1, top_k=1, selection="random_causal", scale=1.0)
    t.sparse_count[0, 0] = 1
    t.sparse_idx[0, 0, 0] = 0
    qq = torch.zeros((1, 1, 128), dtype=torch.bfloat16)
    qq[0, 0, 0] = 1.0
    kk = torch.zeros((t.pool_elems,), dtype=torch.bfloat16)
    vv = torch.zeros((t.pool_elems,), dtype=torch.bfloat16)
    page = int(t.block_table[0, 0]) * t.kv_page_stride
    kk[page + 128 * 1 + 0] = -1.0           # key 1 (row 1): q.k = -1
    vv[page + 0] = 3.0
    vv[page + 128 * 1 + 0] = -5.0
    g2 = np.zeros((1, 128))
    oracle_rows_gap(t, qq, kk, vv, np.array([[0, 0]]), g2)
    w1 = math.exp(-1.0) / (1.0 + math.exp(-1.0))
    assert g2[0, 0] == pytest.approx(w1 * 1.0 * 5.0, abs=1e-14)
    assert np.abs(g2[0, 1:]).max() == 0.0


def oracle_rows_gap(w, q, kf, vf, rows, gap_abs):
    return oracle.attention_rows(
        q_bits=bf16_bits(q), k_bits=bf16_bits(kf), v_bits=bf16_bits(vf),
        kv_page_stride=w.kv_page_stride, num_pages=w.num_pages, sparse_idx=w.sparse_idx,
        sparse_count=w.sparse_count, cu_seqlens_q=w.cu_seqlens_q, seqused_q=w.seqused_q,
        seqused_kv=w.kv_used, block_table=w.block_table, block_x=w.block_x, scale=w.scale,
        win_left=w.win_left, win_right=w.win_right, rows=rows, gap_abs=gap_abs)
