"""GPU edge cases against the oracle: empty lists, sequences without used
queries or with a single key, duplicate list entries, and the extreme GQA
group sizes (G = 1 with one-token Q blocks, G = 128 with one token per tile).

Readings (GBSA article, "Constraints"; the oracle module lists them): rows
with no visible key give out = 0 and lse = -inf; a duplicated list entry
contributes its keys twice; sequences with seqused_q = 0 produce only empty
rows."""
import numpy as np
import pytest
import torch

from block_sparse_paged_gbsa_b200.workloads import generate, make_values, workload
from tests.gpu_helpers import run_gpu
from tests.helpers import assert_lse_close, assert_out_close, oracle_all

pytestmark = pytest.mark.gpu


def _compare_all(w, q, kf, vf, out, lse):
    ro, rl = oracle_all(w, q.cpu(), kf.cpu(), vf.cpu())
    o = out.float().cpu().numpy().astype(np.float64)
    l = lse.float().cpu().numpy()[..., 0].astype(np.float64)
    assert_out_close(o, ro)
    assert_lse_close(l, rl)
    return ro, rl


def test_all_lists_empty():
    w = workload("tiny")
    w.sparse_count[:] = 0
    q, kf, vf, meta, out, lse = run_gpu(w)
    ro, rl = _compare_all(w, q, kf, vf, out, lse)
    assert np.isneginf(rl).all()
    assert (out.float() == 0).all().item()          # exact zeros, not just within tolerance
    assert torch.isneginf(lse).all().item()


def test_unused_queries_and_single_key():
    # seq 0 has no used query; seq 1 has one KV token, so only its last query
    # (bottom-right aligned) sees a key: out = v_0, lse = s_0 exactly; seq 2
    # is ordinary
    w = generate(name="e1", seed=81, q_storage=[200, 130, 64], q_used=[0, 130, 64],
                 kv_used=[128, 1, 300], N1=4, N2=2, block_x=64, top_k=4,
                 selection="random_causal", has_seqused_q=True)
    q, kf, vf, meta, out, lse = run_gpu(w)
    ro, rl = _compare_all(w, q, kf, vf, out, lse)
    assert np.isneginf(rl[:200]).all()                # seq 0: nothing used
    assert np.isneginf(rl[200:329]).all()             # seq 1: rows before the last see no key
    assert np.isfinite(rl[329]).all()                 # its last row sees key 0 only
    assert (out[:200].float() == 0).all().item()


def test_duplicate_list_entries_count_twice():
    w = workload("tiny")
    hit = 0
    for kvh in range(w.N2):
        for qb in range(w.sparse_count.shape[1]):
            if w.sparse_count[kvh, qb] >= 2:
                w.sparse_idx[kvh, qb, 1] = w.sparse_idx[kvh, qb, 0]
                hit += 1
    assert hit > 0
    q, kf, vf, meta, out, lse = run_gpu(w)
    _compare_all(w, q, kf, vf, out, lse)


@pytest.mark.parametrize("forced", [0, 3])
def test_group_of_one_one_token_blocks(forced):
    # G = 1 and block_x = 1: every Q block is one 1-row tile, so units of >= 4
    # blocks run on both tile slots; random_any lists include masked blocks
    w = generate(name="g1", seed=82, q_storage=[5, 3, 1], kv_used=[900, 300, 1500], N1=2, N2=2,
                 block_x=1, top_k=8, selection="random_any")
    q, kf, vf, meta, out, lse = run_gpu(w, forced=forced)
    _compare_all(w, q, kf, vf, out, lse)


def test_group_of_128_one_token_per_tile():
    # G = 128: a tile is one token x 128 heads; block_x = 3 gives a two-tile
    # unit and a one-tile unit per Q block
    w = generate(name="g128", seed=83, q_storage=[10, 4], N1=128, N2=1, block_x=3, top_k=3,
                 selection="random_causal")
    q, kf, vf, meta, out, lse = run_gpu(w)
    _compare_all(w, q, kf, vf, out, lse)


def test_unpacked_gqa_gives_the_same_rows():
    # is_packed_gqa = 0 (the article's per-head scheduling) is computed with
    # the packed tiles; every row's arithmetic is independent of the packing
    import block_sparse_paged_gbsa_b200 as gbsa
    from block_sparse_paged_gbsa_b200.workloads import pool_view
    from tests.gpu_helpers import device_tensors, run_metadata
    w = workload("tiny")
    q, kf, vf = make_values(w, "cuda")
    t = device_tensors(w)
    outs = []
    for packed in (True, False):
        meta = gbsa.metadata(t["idx"], t["cnt"], w.N1, w.N2, w.D, [w.block_x, 128],
                             cu_seqlens_q=t["cu"], seqused_q=t["squ"], seqused_kv=t["sku"],
                             num_tokens=w.T, is_packed_gqa=packed)
        outs.append(gbsa.forward(q, pool_view(w, kf), pool_view(w, vf), t["idx"], t["cnt"],
                                 [w.block_x, 128], metadata=meta, cu_seqlens_q=t["cu"],
                                 seqused_q=t["squ"], seqused_kv=t["sku"], block_table=t["bt"],
                                 softmax_scale=w.scale, is_packed_gqa=packed,
                                 return_softmax_lse=True))
    torch.cuda.synchronize()
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])


NARROW = {
    # tiles of at most 8 live rows take the narrow softmax (4 lanes per row);
    # with several tokens per tile the rows differ in causal position
    "g2_bx4": lambda: generate(name="n1", seed=84, q_storage=[37, 9, 130], q_used=[37, 7, 130],
                               kv_used=[700, 300, 1200], N1=4, N2=2, block_x=4, top_k=6,
                               selection="random_causal"),
    "g4_bx2_window": lambda: generate(name="n2", seed=85, q_storage=[21, 64], kv_used=[900, 2000],
                                      N1=8, N2=2, block_x=2, top_k=9, selection="random_any",
                                      win_left=300, win_right=0),
    "g1_bx8": lambda: generate(name="n3", seed=86, q_storage=[40, 17], kv_used=[1000, 640],
                               N1=3, N2=3, block_x=8, top_k=5, selection="random_causal"),
    "g2_bx3_rows6": lambda: generate(name="n5", seed=88, q_storage=[20, 11], q_used=[18, 11],
                                     kv_used=[520, 300], N1=4, N2=2, block_x=3, top_k=4,
                                     selection="random_causal", has_seqused_q=True),
    "g8_decode": lambda: generate(name="n4", seed=87, q_storage=[1] * 6,
                                  kv_used=[130, 1000, 4000, 129, 2500, 700], N1=16, N2=2,
                                  block_x=1, top_k=40, selection="decode"),
}


@pytest.mark.parametrize("forced", [0, 3])
@pytest.mark.parametrize("name", sorted(NARROW))
def test_narrow_tiles(name, forced):
    w = NARROW[name]()
    assert min(128 // w.G, w.block_x) * w.G <= 8      # the narrow path runs
    q, kf, vf, meta, out, lse = run_gpu(w, forced=forced)
    _compare_all(w, q, kf, vf, out, lse)
