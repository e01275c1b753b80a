"""Invariants of the CPU rebuild of the work list (oracle/scheduler.py), checked
against definitions written independently here: liveness from per-row key
sets, coverage of every live (Q block, KV head, list entry) exactly once,
longest-first order, split lengths and the slot/combine bookkeeping."""
import numpy as np
import pytest

from block_sparse_paged_gbsa_b200.workloads import PAGE, generate, workload
from oracle import scheduler

CASES = {
    "tiny": lambda: workload("tiny"),
    "dense_small": lambda: workload("dense", scale_down=8),
    "decode_small": lambda: workload("decode", scale_down=16),
    "ragged_small": lambda: workload("ragged", scale_down=8),
    "long_small": lambda: workload("long", scale_down=64),
    "odd_blocks": lambda: generate(name="odd", seed=5, q_storage=[300, 1, 129], N1=6, N2=2,
                                   block_x=7, top_k=5, selection="random_any"),
    "window_qu_ku": lambda: generate(name="w", seed=6, q_storage=[400, 250],
                                     q_used=[390, 100], kv_used=[500, 180], N1=5, N2=1,
                                     block_x=64, top_k=6, selection="random_causal",
                                     win_left=150, win_right=0),
}


def _problem(w, num_ctas=148, forced=0):
    p = w.problem_kwargs()
    p.update(num_ctas=num_ctas, max_blocks_per_split=forced, mask_mode=1)
    return p


def _build(w, **kw):
    p = _problem(w, **kw)
    return p, scheduler.build(p, w.sparse_idx, w.sparse_count, w.cu_seqlens_q,
                              w.q_used, w.kv_used)


def _expected_live(w, qb, kvh):
    """(lb, mask, partial) of the live entries, from the key set of every used row."""
    b = int(np.searchsorted(np.cumsum([-(-int(s) // w.block_x) for s in w.q_storage]), qb,
                            side="right"))
    qbase = sum(-(-int(s) // w.block_x) for s in w.q_storage[:b])
    qbl = qb - qbase
    qs = int(w.q_storage[b])
    qu = int(w.q_used[b]) if w.has_seqused_q else qs
    ku = int(w.kv_used[b])
    rows = [t for t in range(qbl * w.block_x, min(qbl * w.block_x + w.block_x, qs)) if t < qu]
    n = min(max(int(w.sparse_count[kvh, qb]), 0), w.top_k)
    out = []
    for j in range(n):
        lb = int(w.sparse_idx[kvh, qb, j])
        if not 0 <= lb < -(-ku // PAGE):
            continue
        visible, hidden = 0, 0
        for t in rows:
            pos = t + ku - qu
            for p in range(lb * PAGE, lb * PAGE + PAGE):
                ok = p < ku and p <= pos and (w.win_left < 0 or p >= pos - w.win_left)
                visible += ok
                hidden += not ok
        if visible:
            out.append((lb, int(hidden > 0), int(lb * PAGE + PAGE > ku)))
    return out


@pytest.mark.parametrize("name", sorted(CASES))
def test_work_list_invariants(name):
    w = CASES[name]()
    p, m = _build(w)
    _check_invariants(w, p, m, name)


def _expected_status(w):
    """Status bits the inputs call for: a count outside [0, top_k] (0x04), a
    listed entry j < clamped count outside the sequence's blocks (0x02)."""
    bits = 0
    qb = 0
    for b in range(w.B):
        nblk = -(-int(w.kv_used[b]) // PAGE)
        for _ in range(-(-int(w.q_storage[b]) // w.block_x)):
            for kvh in range(w.N2):
                c = int(w.sparse_count[kvh, qb])
                if c < 0 or c > w.top_k:
                    bits |= 0x04
                for j in range(min(max(c, 0), w.top_k)):
                    if not 0 <= int(w.sparse_idx[kvh, qb, j]) < nblk:
                        bits |= 0x02
            qb += 1
    return bits


def _check_invariants(w, p, m, name):
    g = scheduler.geometry(p)
    assert m[0] == scheduler.MAGIC and m[1] == 1
    assert int(m[2]) & 0xFFFFFFFF == scheduler.signature(p)
    assert m[15] == _expected_status(w), "status bits are those the inputs call for"
    n_items, top_k = g["n_items"], w.top_k
    item = m[g["off_item"]:g["off_item"] + 8 * n_items].reshape(n_items, 8)
    lists = m[g["off_list"]:g["off_list"] + top_k * n_items].reshape(n_items, top_k)
    # liveness and flags, item by item (small cases: every item; larger: a sample)
    rng = np.random.default_rng(0)
    check = range(n_items) if n_items <= 600 else rng.choice(n_items, 600, replace=False)
    for i in check:
        qb, kvh = divmod(int(i), w.N2)
        exp = _expected_live(w, qb, kvh)
        n_live = int(item[i, 1])
        got = [(int(e) & 0xFFFFFF, (int(e) >> 24) & 1, (int(e) >> 25) & 1)
               for e in lists[i, :n_live]]
        assert got == exp, (name, i)
        assert np.all(lists[i, n_live:] == 0)
    # coverage: every (item, tile pair) splits [0, n_live) into disjoint pieces
    n_units, n_slots, n_comb, L = int(m[11]), int(m[12]), int(m[13]), int(m[14])
    units = m[g["off_unit"]:g["off_unit"] + 4 * n_units].reshape(n_units, 4)
    seen = {}
    for it, tp, jj, slot in units:
        j0, j1 = int(jj) & 0xFFFF, int(jj) >> 16
        seen.setdefault((int(it), int(tp)), []).append((j0, j1, int(slot)))
    for i in range(n_items):
        pairs = -(-int(item[i, 2]) // 2)
        for tp in range(pairs):
            pieces = sorted(seen.pop((i, tp)))
            assert pieces[0][0] == 0 and pieces[-1][1] == int(item[i, 1])
            for a, b in zip(pieces, pieces[1:]):
                assert a[1] == b[0]
            assert all(j1 - j0 <= L for j0, j1, _ in pieces) or len(pieces) == 1
            if len(pieces) > 1:
                slots = [s for *_, s in pieces]
                assert slots == list(range(slots[0], slots[0] + len(pieces)))
            else:
                assert pieces[0][2] == -1
    assert not seen, "pieces for items/tile pairs that do not exist"
    # longest first, stable
    lengths = (units[:, 2] >> 16) - (units[:, 2] & 0xFFFF)
    assert np.all(np.diff(lengths) <= 0)
    # split length rule and capacities
    total = sum(-(-int(item[i, 2]) // 2) * int(item[i, 1]) for i in range(n_items))
    assert (int(m[16]) | (int(m[17]) << 32)) == total
    assert L == max(8, -(-total // (4 * int(p["num_ctas"]))))
    assert n_units <= g["unit_cap"] and n_slots <= g["slot_cap"] and n_comb <= g["comb_cap"]
    comb = m[g["off_comb"]:g["off_comb"] + 4 * n_comb].reshape(n_comb, 4)
    assert int(comb[:, 3].sum()) == n_slots if n_comb else n_slots == 0


@pytest.mark.parametrize("name,forced,ctas", [("tiny", 1, 148), ("tiny", 3, 7),
                                              ("decode_small", 0, 148), ("ragged_small", 2, 7)])
def test_splits(name, forced, ctas):
    w = CASES[name]()
    p, m = _build(w, num_ctas=ctas, forced=forced)
    g = scheduler.geometry(p)
    n_units, n_slots, n_comb, L = int(m[11]), int(m[12]), int(m[13]), int(m[14])
    assert m[15] == 0
    if forced:
        assert L == forced
    units = m[g["off_unit"]:g["off_unit"] + 4 * n_units].reshape(n_units, 4)
    lengths = (units[:, 2] >> 16) - (units[:, 2] & 0xFFFF)
    assert lengths.max() <= L
    assert n_slots > 0 and n_comb > 0
    comb = m[g["off_comb"]:g["off_comb"] + 4 * n_comb].reshape(n_comb, 4)
    assert np.all(comb[:, 3] >= 2)
    assert np.array_equal(np.sort(units[units[:, 3] >= 0, 3]), np.arange(n_slots))


def test_bad_inputs_set_status():
    w = workload("tiny")
    w.sparse_idx[0, 0, 0] = 999
    w.sparse_count[1, 2] = w.top_k + 5
    p, m = _build(w)
    assert m[15] & scheduler.DEV_BAD_BLOCK_IDX and m[15] & scheduler.DEV_BAD_COUNT
    assert m[11] > 0
    w2 = workload("tiny")
    w2.cu_seqlens_q = w2.cu_seqlens_q.copy()
    w2.cu_seqlens_q[1] += 1                       # storage lengths no longer match the blocks
    p, m = _build(w2)
    assert m[15] & scheduler.DEV_BAD_SEQLEN and m[11] == 0


def test_signature_distinguishes_problems():
    w = workload("tiny")
    a = scheduler.signature(_problem(w))
    b = scheduler.signature(_problem(w, num_ctas=147))
    c = scheduler.signature(_problem(w, forced=4))
    assert len({a, b, c}) == 3


def test_work_list_invariants_on_random_problems():
    # the same independent checks on random small problems: sequence mixes
    # with empty and one-token sequences, seqused below storage, GQA groups
    # 1..8, Q block sizes, list kinds, windows and CTA counts
    from hypothesis import HealthCheck, given, settings
    from hypothesis import strategies as st

    @settings(max_examples=50, deadline=None, derandomize=True,
              suppress_health_check=[HealthCheck.too_slow])
    @given(st.data())
    def run(data):
        B = data.draw(st.integers(1, 4))
        # empty storage sequences (repeated cu_seqlens_q values) and
        # sequences with seqused_kv = 0; one sequence is non-empty
        qs = data.draw(st.lists(st.integers(0, 160), min_size=B, max_size=B))
        if sum(qs) == 0:
            qs[data.draw(st.integers(0, B - 1))] = data.draw(st.integers(1, 160))
        qu = [data.draw(st.integers(0, s)) for s in qs]
        ku = [data.draw(st.sampled_from([0, u]) | st.integers(0, u + 400)) for u in qu]
        N2 = data.draw(st.sampled_from([1, 2]))
        G = data.draw(st.sampled_from([1, 2, 3, 5, 8]))
        bx = data.draw(st.sampled_from([1, 3, 16, 64, 128]))
        top_k = data.draw(st.integers(1, 6))
        sel = data.draw(st.sampled_from(["random_causal", "random_any", "all_causal"]))
        win = data.draw(st.sampled_from([-1, 0, 100]))
        ctas = data.draw(st.sampled_from([3, 37, 148]))
        seed = data.draw(st.integers(0, 10_000))
        w = generate(name="h", seed=seed, q_storage=qs, q_used=qu, kv_used=ku, N1=N2 * G, N2=N2,
                     block_x=bx, top_k=top_k, selection=sel, win_left=win,
                     win_right=0 if win >= 0 else -1, has_seqused_q=True)
        p, m = _build(w, num_ctas=ctas)
        _check_invariants(w, p, m, "random")

    run()
