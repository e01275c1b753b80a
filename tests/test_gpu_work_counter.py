"""Dynamic unit fetching.  CTA c of the forward starts with unit c of the
work list and takes the next untaken unit from a counter in the list's
header (word 26; word 27 counts the CTAs that finished).  gbsa_metadata()
leaves both at zero, and the last CTA of every forward puts them back, so one
work list serves repeated calls and CUDA graph replays.  Which CTA runs a
unit changes from call to call; the results must not: repeated calls and
graph replays are bit-identical, and the work list is unchanged by them."""
import pytest
import torch

import block_sparse_paged_gbsa_b200 as gbsa
from block_sparse_paged_gbsa_b200.workloads import make_values, pool_view, workload
from tests.gpu_helpers import device_tensors, run_forward, run_metadata, sm_count

pytestmark = pytest.mark.gpu

H_NUNITS, H_UNIT_NEXT, H_CTAS_DONE = 11, 26, 27

# (workload, scale-down, num_ctas (0: one per SM), forced split length)
CASES = [
    ("ragged", 8, 7, 0),    # two- and one-tile units, many per CTA
    ("ragged", 8, 0, 3),    # forced splits: partials and the combine
    ("dense", 4, 0, 0),
    ("decode", 4, 7, 0),    # units in halves, narrow tiles
    ("decode", 4, 0, 0),
    ("tiny", 1, 0, 0),      # fewer units than CTAs: no CTA fetches past its first
]


def _counters(meta):
    return int(meta[H_UNIT_NEXT].item()), int(meta[H_CTAS_DONE].item())


@pytest.mark.parametrize("name,sd,ctas,forced", CASES)
def test_counters_return_to_zero_and_calls_repeat_bit_identical(name, sd, ctas, forced):
    w = workload(name, scale_down=sd)
    q, kf, vf = make_values(w, "cuda")
    t = device_tensors(w)
    meta = run_metadata(w, t, ctas, forced)
    torch.cuda.synchronize()
    assert _counters(meta) == (0, 0)
    built = meta.clone()
    if name != "tiny":
        assert int(meta[H_NUNITS].item()) > 2 * (ctas or sm_count())  # the counter is used
    first = None
    for _ in range(3):
        out, lse = run_forward(w, q, kf, vf, t, meta, ctas, forced)
        torch.cuda.synchronize()
        assert _counters(meta) == (0, 0)
        if first is None:
            first = (out.clone(), lse.clone())
        else:
            assert torch.equal(out, first[0]) and torch.equal(lse, first[1])
    assert torch.equal(meta, built)


def test_graph_replays_bit_identical():
    w = workload("ragged", scale_down=8)
    q, kf, vf = make_values(w, "cuda")
    t = device_tensors(w)
    ctas = 7
    meta = run_metadata(w, t, ctas)
    ref_out, ref_lse = run_forward(w, q, kf, vf, t, meta, ctas)
    torch.cuda.synchronize()
    out, lse = torch.empty_like(ref_out), torch.empty_like(ref_lse)
    kp, vp = pool_view(w, kf), pool_view(w, vf)

    def call():
        gbsa.forward(q, kp, vp, t["idx"], t["cnt"], [w.block_x, 128], metadata=meta,
                     cu_seqlens_q=t["cu"], seqused_q=t["squ"], seqused_kv=t["sku"],
                     block_table=t["bt"], softmax_scale=w.scale, win_left=w.win_left,
                     win_right=w.win_right, return_softmax_lse=True, num_ctas=ctas, out=out,
                     lse=lse)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        call()  # warm-up on the capture stream
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    for _ in range(3):
        out.zero_()
        lse.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert _counters(meta) == (0, 0)
        assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)
    del graph


def test_separate_work_lists_run_concurrently():
    """Calls on two streams with their own work lists may overlap: each list
    has its own counters.  Each result equals the same call run alone."""
    cases = [(workload("ragged", scale_down=8), 7), (workload("dense", scale_down=4), 0)]
    prepared = []
    for w, ctas in cases:
        q, kf, vf = make_values(w, "cuda")
        t = device_tensors(w)
        meta = run_metadata(w, t, ctas)
        alone = run_forward(w, q, kf, vf, t, meta, ctas)
        torch.cuda.synchronize()
        prepared.append((w, ctas, q, kf, vf, t, meta, (alone[0].clone(), alone[1].clone())))
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    results = [[], []]
    for s in streams:
        s.wait_stream(torch.cuda.current_stream())
    for _ in range(3):
        for k, (w, ctas, q, kf, vf, t, meta, _) in enumerate(prepared):
            with torch.cuda.stream(streams[k]):
                results[k].append(run_forward(w, q, kf, vf, t, meta, ctas))
    torch.cuda.synchronize()
    for k, (w, ctas, q, kf, vf, t, meta, (ref_out, ref_lse)) in enumerate(prepared):
        assert _counters(meta) == (0, 0)
        for out, lse in results[k]:
            assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)
