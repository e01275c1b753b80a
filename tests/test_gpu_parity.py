"""GPU parity: the CUDA path (metadata + forward + combine, called through the
C ABI) against the fp64 oracle on the same seeded inputs.

Tolerances (from the target: max abs error 1e-2 on the bf16 output, 1e-3 on
the LSE): the output check allows 1e-2 of arithmetic error on top of the bf16
representation of the exact value (half an ulp at |out|), because an exact
value with |out| >= 4 cannot be stored in bf16 closer than 1.6e-2."""
import numpy as np
import pytest
import torch

import block_sparse_paged_gbsa_b200 as gbsa
from block_sparse_paged_gbsa_b200.workloads import generate, make_values, pool_view, workload
from oracle import scheduler
from tests.gpu_helpers import device_tensors, problem_dict, run_gpu, run_metadata, sm_count
from tests.helpers import assert_lse_close, assert_out_close, oracle_all, oracle_rows

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny": lambda: workload("tiny"),
    "dense_s16": lambda: workload("dense", scale_down=16),
    "decode_s16": lambda: workload("decode", scale_down=16),
    "ragged_s16": lambda: workload("ragged", scale_down=16),
    "long_s64": lambda: workload("long", scale_down=64),
    "odd_shapes": lambda: generate(name="odd", seed=77, q_storage=[300, 1, 129, 64], N1=6, N2=2,
                                   block_x=7, top_k=5, selection="random_any"),
    "g5_window": lambda: generate(name="g5", seed=78, q_storage=[700, 333],
                                  q_used=[650, 300], kv_used=[700, 410], N1=10, N2=2,
                                  block_x=64, top_k=6, selection="random_causal",
                                  win_left=200, win_right=0, page_stride_factor=1.25),
    "g16_bx200": lambda: generate(name="g16", seed=79, q_storage=[450], N1=16, N2=1,
                                  block_x=200, top_k=4, selection="random_causal"),
    # one tile per Q block (16 tokens x G=8 heads): units of >= 4 blocks run with
    # the two tile slots on the even / odd blocks, here with causal, window and
    # partial-page masks
    "g8_bx16_window": lambda: generate(name="g8w", seed=80, q_storage=[1500, 900],
                                       q_used=[1480, 900], kv_used=[1500, 1000], N1=8, N2=1,
                                       block_x=16, top_k=12, selection="random_causal",
                                       win_left=700, win_right=0),
}


def _sample_rows(w, n, seed=0):
    rng = np.random.default_rng(seed)
    T, N1 = w.T, w.N1
    tok = rng.integers(0, T, size=n)
    # plus the first and last token of every sequence
    ends = np.concatenate([w.cu_seqlens_q[:-1], w.cu_seqlens_q[1:] - 1])
    ends = ends[(ends >= 0) & (ends < T)]
    tok = np.concatenate([tok, np.repeat(ends, 1)])
    head = rng.integers(0, N1, size=tok.size)
    return np.stack([tok, head], 1).astype(np.int64)


def _compare(w, q, kf, vf, out, lse, rows=None):
    o = out.float().cpu().numpy().astype(np.float64)
    l = lse.float().cpu().numpy()[..., 0].astype(np.float64)
    if rows is None:
        ro, rl = oracle_all(w, q.cpu(), kf.cpu(), vf.cpu())
        assert_out_close(o, ro)
        assert_lse_close(l, rl)
    else:
        ro, rl = oracle_rows(w, q.cpu(), kf.cpu(), vf.cpu(), rows)
        assert_out_close(o[rows[:, 0], rows[:, 1]], ro)
        assert_lse_close(l[rows[:, 0], rows[:, 1]], rl)


def _first_diffs(gpu, ref, mask, n=6):
    """Where the GPU work list differs from the rebuild: region and words."""
    names = ["header", "seq", "item", "list", "unit", "combine"]
    bounds = [0] + [int(ref[k]) for k in (18, 19, 20, 21, 22, 23)]
    bad = np.nonzero((gpu != ref) & mask)[0]
    lines = []
    for i in bad[:n]:
        region = max(r for r in range(6) if bounds[r] <= i)
        lines.append(f"{names[region]}+{i - bounds[region]}: gpu {gpu[i]} ref {ref[i]}")
    return f"{bad.size} words differ: " + "; ".join(lines)


@pytest.mark.parametrize("name", sorted(SMALL))
def test_metadata_bit_exact(name):
    w = SMALL[name]()
    for ctas, forced in ((0, 0), (7, 0), (148, 2)):
        t = device_tensors(w)
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        meta = run_metadata(w, t, ctas, forced, status).cpu().numpy()
        p = problem_dict(w, ctas or sm_count(), forced)
        ref = scheduler.build(p, w.sparse_idx, w.sparse_count, w.cu_seqlens_q, w.q_used,
                              w.kv_used)
        assert meta.size == ref.size
        mask = scheduler.defined_mask(ref)
        assert np.array_equal(meta[mask], ref[mask]), _first_diffs(meta, ref, mask)
        assert int(status.item()) == 0


LARGE_META = {
    **{n: (lambda n=n: workload(n)) for n in ("dense", "long", "decode", "ragged")},
    # 50500 items: past the items whose fields the plan kernel stages in
    # shared memory, so the rest are re-read from the item table
    "many_items": lambda: generate(name="many", seed=81, q_storage=[60000, 41000], N1=16, N2=4,
                                   block_x=8, top_k=3, selection="random_causal"),
    # sequence counts around the paths of the sequence phase: derived in
    # every item CTA (up to 1024), a sequence kernel with the bases staged
    # in shared memory (up to 2048), and read from its table (beyond)
    **{f"decode_b{B}": (lambda B=B: _decode_batch(B)) for B in (1024, 1500, 2500)},
}


def _decode_batch(B, seed=82):
    rng = np.random.default_rng(seed + B)
    kv = rng.integers(1, 3000, size=B).astype(np.int32)
    return generate(name=f"db{B}", seed=seed, q_storage=[1] * B, q_used=[1] * B, kv_used=kv,
                    N1=8, N2=2, block_x=1, top_k=16, selection="decode", count_range=(1, 16),
                    has_seqused_q=False)


@pytest.mark.parametrize("name", sorted(LARGE_META))
def test_metadata_bit_exact_full_size(name):
    """The work list of the full-size workloads (the launch configuration the
    benchmark uses, and forced split lengths that give long and short pieces
    of many lengths) is word for word the sequential rebuild's."""
    w = LARGE_META[name]()
    t = device_tensors(w)
    for ctas, forced in ((0, 0), (148, 3), (64, 2)):
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        meta = run_metadata(w, t, ctas, forced, status).cpu().numpy()
        ref = scheduler.build(problem_dict(w, ctas or sm_count(), forced), w.sparse_idx,
                              w.sparse_count, w.cu_seqlens_q, w.q_used, w.kv_used)
        assert meta.size == ref.size
        mask = scheduler.defined_mask(ref)
        assert np.array_equal(meta[mask], ref[mask]), _first_diffs(meta, ref, mask)
        assert int(status.item()) == int(ref[15])


@pytest.mark.parametrize("name", sorted(SMALL))
def test_forward_matches_oracle(name):
    w = SMALL[name]()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    q, kf, vf, meta, out, lse = run_gpu(w, dev_status=status)
    assert int(status.item()) == 0, gbsa.gbsa.decode_dev_status(int(status.item()))
    rows = None if w.T * w.N1 <= 70000 else _sample_rows(w, 6000)
    _compare(w, q, kf, vf, out, lse, rows)


@pytest.mark.parametrize("name", ["tiny", "decode_s16", "g5_window", "g8_bx16_window"])
def test_split_kv_and_cta_counts(name):
    """Split-KV pieces and the combine: any CTA count / forced split length
    stays within tolerance of the oracle, and every repeat is bit-identical."""
    w = SMALL[name]()
    vals = make_values(w, "cuda")
    ref = oracle_all(w, *(v.cpu() for v in vals))
    combines = 0
    for ctas, forced in ((1, 0), (7, 1), (148, 3), (0, 2)):
        _, _, _, meta, out, lse = run_gpu(w, vals, ctas, forced)
        n_comb = int(meta[13].item())
        ref_meta = scheduler.build(problem_dict(w, ctas or sm_count(), forced), w.sparse_idx,
                                   w.sparse_count, w.cu_seqlens_q, w.q_used, w.kv_used)
        assert n_comb == int(ref_meta[13])
        combines += n_comb
        o = out.float().cpu().numpy().astype(np.float64)
        assert_out_close(o, ref[0])
        assert_lse_close(lse.cpu().numpy()[..., 0], ref[1])
        _, _, _, _, out2, lse2 = run_gpu(w, vals, ctas, forced)
        assert torch.equal(out, out2) and torch.equal(lse, lse2)
    assert combines > 0, "no configuration exercised the split-KV combine"


def test_values_one_give_one():
    w = workload("ragged", scale_down=16)
    q, kf, vf = make_values(w, "cuda")
    vf = torch.where(torch.isnan(vf), vf, torch.ones_like(vf))
    _, _, _, _, out, lse = run_gpu(w, (q, kf, vf))
    has = torch.isfinite(lse[..., 0])
    assert has.sum() > 1000
    err = (out.float()[has] - 1).abs().max().item()
    assert err <= 1e-2, err
    assert torch.all(out[~has] == 0)


def test_page_permutation_bit_identical():
    w = workload("tiny")
    q, kf, vf = make_values(w, "cuda")
    _, _, _, _, out, lse = run_gpu(w, (q, kf, vf))
    perm = torch.as_tensor(np.random.default_rng(3).permutation(w.num_pages), device="cuda")
    k2, v2 = torch.empty_like(kf), torch.empty_like(vf)
    k2.view(w.num_pages, -1)[perm] = kf.view(w.num_pages, -1)
    v2.view(w.num_pages, -1)[perm] = vf.view(w.num_pages, -1)
    bt = w.block_table
    w.block_table = np.where(bt >= 0, perm.cpu().numpy()[np.maximum(bt, 0)], -1).astype(np.int32)
    _, _, _, _, out2, lse2 = run_gpu(w, (q, k2, v2))
    assert torch.equal(out, out2) and torch.equal(lse, lse2)


def test_page_stride_bit_identical():
    kw = dict(seed=31, q_storage=[512, 300], N1=8, N2=2, block_x=64, top_k=4,
              selection="random_causal")
    a = generate(name="s1", page_stride_factor=1.0, **kw)
    b = generate(name="s2", page_stride_factor=1.25, **kw)
    q, kf, vf = make_values(a, "cuda")
    pe = 128 * a.N2 * a.D
    kb = torch.full((b.pool_elems,), float("nan"), dtype=torch.bfloat16, device="cuda")
    vb = kb.clone()
    kb.view(b.num_pages, -1)[:, :pe] = kf.view(a.num_pages, -1)[:, :pe]
    vb.view(b.num_pages, -1)[:, :pe] = vf.view(a.num_pages, -1)[:, :pe]
    _, _, _, _, o1, l1 = run_gpu(a, (q, kf, vf))
    _, _, _, _, o2, l2 = run_gpu(b, (q, kb, vb))
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_device_status_bits():
    w = workload("tiny")
    w.sparse_idx[0, 1, 0] = 10_000          # outside the sequence: skipped + flagged
    w.sparse_count[1, 2] = w.top_k + 3      # clamped + flagged
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    q, kf, vf, meta, out, lse = run_gpu(w, dev_status=status)
    bits = int(status.item())
    assert bits & 0x02 and bits & 0x04 and not bits & ~0x06
    _compare(w, q, kf, vf, out, lse)
    # the work list, header status word included, is still the rebuild's
    m = meta.cpu().numpy()
    ref = scheduler.build(problem_dict(w, sm_count()), w.sparse_idx, w.sparse_count,
                          w.cu_seqlens_q, w.q_used, w.kv_used)
    mask = scheduler.defined_mask(ref)
    assert int(m[15]) == int(ref[15]) == bits
    assert np.array_equal(m[mask], ref[mask]), _first_diffs(m, ref, mask)


@pytest.mark.parametrize("case", ["tiny", "decode_b1100"])
def test_bad_seqlen_status_matches_rebuild(case):
    """A negative seqused_kv: the header carries the sequence bit (and the
    plan is empty) on both paths of the sequence phase (2 and 1100
    sequences)."""
    w = _decode_batch(1100) if case == "decode_b1100" else workload("tiny")
    w.kv_used[1] = -1
    t = device_tensors(w)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    m = run_metadata(w, t, 0, 0, status).cpu().numpy()
    ref = scheduler.build(problem_dict(w, sm_count()), w.sparse_idx, w.sparse_count,
                          w.cu_seqlens_q, w.q_used if w.has_seqused_q else None, w.kv_used)
    assert int(ref[15]) & 0x01
    assert int(m[15]) == int(ref[15]) == int(status.item())
    mask = scheduler.defined_mask(ref)
    assert np.array_equal(m[mask], ref[mask]), _first_diffs(m, ref, mask)


def test_metadata_mismatch_leaves_output_untouched():
    w = workload("tiny")
    q, kf, vf = make_values(w, "cuda")
    t = device_tensors(w)
    meta = run_metadata(w, t, num_ctas=7)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out0 = torch.full_like(q, 3.0)
    out, _ = gbsa.forward(q, pool_view(w, kf), pool_view(w, vf), t["idx"], t["cnt"],
                          [w.block_x, 128], metadata=meta, cu_seqlens_q=t["cu"],
                          seqused_kv=t["sku"], block_table=t["bt"], softmax_scale=w.scale,
                          num_ctas=9, out=out0, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & 0x10
    assert torch.all(out == 3.0)


def test_host_rejections_before_launch():
    w = workload("tiny")
    q, kf, vf = make_values(w, "cuda")
    t = device_tensors(w)
    meta = run_metadata(w, t)
    with pytest.raises(ValueError):          # non-contiguous query
        gbsa.forward(q.transpose(0, 1), pool_view(w, kf), pool_view(w, vf), t["idx"], t["cnt"],
                     [w.block_x, 128], metadata=meta, cu_seqlens_q=t["cu"], seqused_kv=t["sku"],
                     block_table=t["bt"])
    with pytest.raises(gbsa.GbsaError):      # block_y must be the page size
        gbsa.forward(q, pool_view(w, kf), pool_view(w, vf), t["idx"], t["cnt"], [w.block_x, 64],
                     metadata=meta, cu_seqlens_q=t["cu"], seqused_kv=t["sku"],
                     block_table=t["bt"])


FULL = ["tiny", "dense", "long", "decode", "ragged"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled_rows(name):
    """The five named workloads at full size, in the launch configuration the
    benchmark times (all SMs, automatic split length), on sampled rows."""
    w = workload(name)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    q, kf, vf, meta, out, lse = run_gpu(w, dev_status=status)
    assert int(status.item()) == 0
    assert torch.isfinite(out.float()).all()
    rows = _sample_rows(w, 3000, seed=1)
    _compare(w, q, kf, vf, out, lse, rows)


@pytest.mark.parametrize("B,forced", [(1500, 0), (1500, 3), (2500, 0)])
def test_forward_with_many_sequences(B, forced):
    """Above 1024 sequences the sequence table comes from its own kernel (and
    above 2048 the item kernel looks it up in global memory): the forward on
    that work list matches the oracle on every row."""
    w = _decode_batch(B)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    q, kf, vf, meta, out, lse = run_gpu(w, forced=forced, dev_status=status)
    assert int(status.item()) == 0
    _compare(w, q, kf, vf, out, lse)
