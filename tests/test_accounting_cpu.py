"""The benchmark's work accounting against independent counts: the exact
FLOPs from brute-force key membership, the block-granular FLOPs from the
work list the oracle's scheduler rebuild produces, and per-row sums."""
import numpy as np
import pytest

from block_sparse_paged_gbsa_b200.accounting import row_flops, work
from block_sparse_paged_gbsa_b200.workloads import PAGE, generate, workload
from oracle import scheduler


def _visible_pairs(w):
    """(row, head, key) triples with their multiplicity, enumerated directly."""
    total = 0
    qbase = 0
    G = w.G
    for b in range(w.B):
        qs = int(w.q_storage[b])
        qu = int(w.q_used[b]) if w.has_seqused_q else qs
        ku = int(w.kv_used[b])
        for t in range(qu):
            qb = qbase + t // w.block_x
            pos = t + ku - qu
            for h in range(w.N1):
                kvh = h // G
                n = min(max(int(w.sparse_count[kvh, qb]), 0), w.top_k)
                for j in range(n):
                    lb = int(w.sparse_idx[kvh, qb, j])
                    if not 0 <= lb < -(-ku // PAGE):
                        continue
                    lo = lb * PAGE if w.win_left < 0 else max(lb * PAGE, pos - w.win_left)
                    hi = min(lb * PAGE + PAGE - 1, ku - 1, pos)
                    total += max(0, hi - lo + 1)
        qbase += -(-qs // w.block_x)
    return total


CASES = [
    lambda: workload("tiny", scale_down=2),
    lambda: generate(name="w", seed=3, q_storage=[300, 129], q_used=[280, 129],
                     kv_used=[310, 200], N1=4, N2=2, block_x=32, top_k=5,
                     selection="random_causal", win_left=100, win_right=0),
    lambda: workload("decode", scale_down=32),
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_exact_flops_match_enumeration(case):
    w = CASES[case]()
    assert work(w)["flops_exact"] == 4 * w.D * _visible_pairs(w)


@pytest.mark.parametrize("case", range(len(CASES)))
def test_block_flops_match_work_list(case):
    w = CASES[case]()
    p = dict(w.problem_kwargs(), num_ctas=148, max_blocks_per_split=0, mask_mode=1)
    m = scheduler.build(p, w.sparse_idx, w.sparse_count, w.cu_seqlens_q, w.q_used, w.kv_used)
    g = scheduler.geometry(p)
    items = m[g["off_item"]:g["off_item"] + 8 * g["n_items"]].reshape(-1, 8)
    lists = m[g["off_list"]:g["off_list"] + w.top_k * g["n_items"]].reshape(-1, w.top_k)
    flops = 0
    for i in range(g["n_items"]):
        n_used, ku = int(items[i, 5]), int(items[i, 7])
        for e in lists[i, :items[i, 1]]:
            lb = int(e) & 0xFFFFFF
            flops += 4 * n_used * w.G * min(PAGE, ku - lb * PAGE) * w.D
    acc = work(w)
    assert acc["flops_block"] == flops
    assert acc["live_blocks"] == int(items[:, 1].sum())
    tt, hh = np.meshgrid(np.arange(w.T), np.arange(w.N1), indexing="ij")
    rows = np.stack([tt.reshape(-1), hh.reshape(-1)], 1)
    assert row_flops(w, rows) == flops


def _bench_module():
    import importlib.util
    import os
    path = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "bench.py")
    spec = importlib.util.spec_from_file_location("gbsa_bench", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_kernel_hash_ignores_comments_only():
    b = _bench_module()
    src = 'int a = 1; // note\n/* block\n comment */ asm("x // y /* z */"); char c = \'/\';\n'
    assert b.code_tokens(src) == b.code_tokens(src.replace("note", "other").replace("block", "b"))
    assert b.code_tokens(src) != b.code_tokens(src.replace("a = 1", "a = 2"))
    assert b.code_tokens(src) != b.code_tokens(src.replace("x // y", "x // w"))  # inside a string
    assert "note" not in b.code_tokens(src) and "x // y /* z */" in b.code_tokens(src)


def test_committed_traffic_records_are_well_formed():
    # bench.py reads a record only while its kernel_sha equals kernel_hash()
    import glob
    import json
    import os
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    recs = glob.glob(os.path.join(root, "profiles", "forward_*_traffic.json"))
    assert recs
    for r in recs:
        d = json.load(open(r))
        assert len(d["kernel_sha"]) == 16 and int(d["dram_bytes_per_launch"]) > 0, r
        assert "--clock-control none" in d["command"], r
