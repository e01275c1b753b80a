#!/usr/bin/env python
"""Benchmark: block-sparse paged GQA attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload all]
    python bench.py --impl reference ...    # the fp64 CPU oracle arm

One step = the whole hot path over one batch of synthetic input: the
metadata (work list) launches, the forward kernel and the split-KV combine,
through the C ABI.  Inputs are resident in HBM before timing; L2 is flushed
(a 256 MiB write) between timed steps; every step is timed with CUDA events
on the launching stream; with N GPUs each rank runs its own seeded batch
(independent problems, no collective on the data path, weak scaling) and the
time is the max over ranks.  Prints one JSON line on rank 0.

By default (--workload all) one run times all five workloads: the line's
headline value, roofline, end-to-end figure and CPU baseline are those of the
largest one, the 131072-token long-context prefill, and ``per_config``
carries the same step, forward and roofline figures, with the clocks sampled
during each, for the other four.  --workload NAME times one workload alone.

Metric: effective TFLOPS counted over selected, unmasked (live) blocks, with
KV-page GB/s and the roofline fraction beside it.  The fp64 oracle is timed
on the host cores over a bounded sample of rows as the CPU baseline.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "effective TFLOPS + KV GB/s (selected blocks), % of roofline, 1×B200"
UNIT = "TFLOPS"
DESCRIPTIONS = {
    "dense": "dense-equivalent causal prefill: B=4 x 4096 tokens, N1=32, N2=8, D=128, "
             "block_shape=[128,128], 128-token pages, top_k=32, every causal block selected",
    "tiny": "tiny block-sparse prefill: B=2 x 512 tokens, N1=8, N2=2, block_shape=[64,128], "
            "top_k=4 random causal blocks incl. the diagonal",
    "long": "long-context block-sparse prefill: B=1 x 131072 tokens, N1=32, N2=4, "
            "block_shape=[128,128], top_k=64 (sink + diagonal + 62 random causal)",
    "decode": "decode with packed GQA: 64 x 1 query token, KV ~ U[8192,65536], N1=64, N2=8, "
              "block_shape=[1,128], top_k=256, count ~ U{64..256} incl. last page, split-KV",
    "ragged": "ragged varlen: 16 sequences lognormal(4096, 1.0) in [512,32768], seqused = "
              "storage - U[0,127], N1=40, N2=8, block_shape=[64,128], top_k=128, window "
              "(4096, 0), page stride 1.25x",
}
FLUSH_BYTES = 256 << 20
KERNEL_SOURCES = ["block_sparse_paged_gbsa_b200/csrc/gbsa_fwd.cu",
                  "block_sparse_paged_gbsa_b200/csrc/sm100.cuh",
                  "block_sparse_paged_gbsa_b200/csrc/gbsa_internal.cuh"]


HEADLINE = "long"
ORDER = ["long", "tiny", "dense", "decode", "ragged"]


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["gbsa", "reference"], default="gbsa")
    ap.add_argument("--workload", default="all", choices=["all"] + sorted(DESCRIPTIONS),
                    help="all (default): the long-context workload as the headline and the "
                         "other four in per_config; or one workload")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--dtype", default="bf16", choices=["bf16", "fp16", "e4m3"],
                    help="element type of q, k and v (e4m3: the quantised mode with "
                         "per-tensor dequantization scales, bf16 out)")
    ap.add_argument("--softmax-precision", type=int, default=0, choices=[0, 1],
                    help="the article's softmaxPrecision (0: fp32 online softmax; 1: "
                         "half-precision exponentials with fp32 rescale and row sums)")
    ap.add_argument("--backward", action="store_true",
                    help="time the gradient computation (gbsa.backward) of one workload "
                         "(dense unless --workload names another) instead of the forward")
    ap.add_argument("--scale-down", type=int, default=1,
                    help="shrink the workload's sequence lengths by this factor (same "
                         "structure); for profiler captures that must stay small")
    return ap.parse_args()


def headline_name(args) -> str:
    return HEADLINE if args.workload == "all" else args.workload


def describe(name, args) -> str:
    d = DESCRIPTIONS[name]
    if args.scale_down != 1:
        d += f" -- sequence lengths scaled down {args.scale_down}x (profiling case)"
    if args.dtype != "bf16":
        d += f" -- q, k, v in {args.dtype}"
    if args.softmax_precision:
        d += " -- softmaxPrecision 1"
    return d


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    except (OSError, KeyError, ValueError):
        return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0,
                    source="fallback")


def code_tokens(text: str) -> str:
    """C++ source without comments, whitespace runs collapsed: what the
    compiler sees, so that an edit of comments keeps the hash (string and
    character literals are kept verbatim)."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        elif c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def kernel_hash() -> str:
    """Identity of the forward kernel's source (comments excluded), matched
    against the ncu records under profiles/."""
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            h.update(code_tokens(f.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes per forward launch from the committed ncu summary, if it was
    taken on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", f"forward_{workload}_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    if d.get("kernel_sha") != kernel_hash():
        return None
    return d.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi sampling (50 ms) during the run; ``window`` summarises the
    samples of one timed region."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def _rows(self):
        self.file.flush()
        rows = []
        with open(self.file.name) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 10:
                    continue
                try:
                    ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                    frac = float("0." + parts[0].split(".")[1]) if "." in parts[0] else 0.0
                    rows.append((ts + frac, float(parts[2]), float(parts[3]), parts[6:10]))
                except ValueError:
                    continue
        return rows

    def window(self, t0: float, t1: float) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.12)  # the sample after the region
        rows = self._rows()
        inside = [r for r in rows if t0 - 0.06 <= r[0] <= t1 + 0.06]
        if not inside:
            after = [r for r in rows if r[0] >= t0 - 0.06]
            inside = after[:1]
        reasons = sorted({self.NAMES[i] for r in inside for i, v in enumerate(r[3])
                          if v == "Active"})
        sm = [r[1] for r in inside]
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": max((r[2] for r in inside), default=None), "reasons": reasons,
                "samples": len(inside)}

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            self.proc.wait()
            self.proc = None
        try:
            os.unlink(self.file.name)
        except OSError:
            pass


def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank draws its own batch of the same workload (weak scaling)."""
    return base_seed + 1000 * rank


def reduce_max(values, dist, device):
    """Max over ranks of a list of per-rank timings (host plumbing only)."""
    import torch
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def reduce_sum(values, dist, device):
    """Sum over ranks (the work each rank did)."""
    import torch
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return [float(x) for x in t.tolist()]


def job_value(total_flops: float, max_ms: float) -> float:
    """Whole-job TFLOPS: the work of all ranks over the slowest rank's time."""
    return total_flops / (max_ms * 1e-3) / 1e12


def dist_info():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def cpu_cores() -> int:
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()


def oracle_sample(w, q, kf, vf, target_s: float, seed: int = 0, scales=(1.0, 1.0, 1.0)):
    """Times the oracle on a bounded random sample of rows sized to about
    target_s seconds.  E4M3 values go to the oracle as fp16 (exact) with the
    dequantization scales folded in.  Returns (TFLOPS, seconds, rows,
    description)."""
    import torch
    import oracle
    from block_sparse_paged_gbsa_b200.accounting import row_flops
    from block_sparse_paged_gbsa_b200.workloads import bf16_bits

    if q.dtype == torch.float8_e4m3fn:
        q, kf, vf = (t.to(torch.float16) for t in (q, kf, vf))
        scale = w.scale * scales[0] * scales[1]
    else:
        scale = w.scale
    odt = "fp16" if q.dtype == torch.float16 else "bf16"
    qb, kb, vb = bf16_bits(q), bf16_bits(kf), bf16_bits(vf)
    rng = np.random.default_rng(seed)
    threads = cpu_cores()

    def run(n):
        rows = np.stack([rng.integers(0, w.T, n), rng.integers(0, w.N1, n)], 1).astype(np.int64)
        t0 = time.perf_counter()
        oracle.attention_rows(q_bits=qb, k_bits=kb, v_bits=vb, kv_page_stride=w.kv_page_stride,
                              num_pages=w.num_pages, sparse_idx=w.sparse_idx,
                              sparse_count=w.sparse_count, cu_seqlens_q=w.cu_seqlens_q,
                              seqused_q=w.seqused_q, seqused_kv=w.kv_used,
                              block_table=w.block_table, block_x=w.block_x, scale=scale,
                              win_left=w.win_left, win_right=w.win_right, rows=rows,
                              dtype=odt, n_threads=threads)
        return time.perf_counter() - t0, rows

    n = 4 * threads
    dt, rows = run(n)
    while dt < 0.5:
        n *= 4
        dt, rows = run(n)
    n = max(n, int(n * target_s / max(dt, 1e-6)))
    dt, rows = run(n)
    flops = row_flops(w, rows)
    return flops / dt / 1e12, dt, n, threads


def run_reference(args, world, rank):
    """The CPU oracle arm: each step is the oracle over a bounded random
    sample of rows of the headline workload, on the host cores."""
    if rank != 0:
        return
    from block_sparse_paged_gbsa_b200.workloads import make_values, workload

    import torch

    name = headline_name(args)
    w = workload(name, scale_down=args.scale_down)
    tdt = {"bf16": torch.bfloat16, "fp16": torch.float16, "e4m3": torch.float8_e4m3fn}[args.dtype]
    q, kf, vf = make_values(w, "cpu", dtype=tdt)  # the inputs of the GPU arm's --dtype
    per_step = max(0.5, min(5.0, 150.0 / max(1, args.steps + args.warmup)))
    vals = []
    for i in range(args.warmup + args.steps):
        tf, dt, n, threads = oracle_sample(w, q, kf, vf, per_step, seed=i)
        if i >= args.warmup:
            vals.append((tf, dt, n))
    tf = float(np.mean([v[0] for v in vals]))
    sample = (f"{int(np.mean([v[2] for v in vals]))} random (token, head) rows per step, "
              f"about {per_step:.1f} s of fp64 oracle work each")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(tf, 6), "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * float(np.mean([v[1] for v in vals])), 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": describe(name, args), "sample": sample},
        "cpu_baseline": {"value": round(tf, 6), "unit": UNIT, "cores": threads,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(tf, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def roofline(acc, fwd_ms, peaks, fp8, traffic):
    """The forward kernel's roofline object: the bound the workload's FLOPs
    and algorithmic bytes put it at, the achieved rate over the forward's
    device time, and its fraction of the measured peak."""
    t_peak = peaks["bf16_tflops"] * (2.0 if fp8 else 1.0)
    flops, nbytes = acc["flops_block"], acc["bytes"]
    tensor = flops / (t_peak * 1e12) >= nbytes / (peaks["hbm_gbs"] * 1e9)
    if tensor:
        achieved = flops / (fwd_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": round(achieved, 3), "peak": round(t_peak, 3),
                "unit": "TFLOP/s", "frac": round(achieved / t_peak, 4)}
    else:
        achieved = nbytes / (fwd_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 3), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4)}
    if tensor:
        # the same rate against the seconds-long, power-capped GEMM figure, the
        # fitting denominator when the timed region itself runs under the cap
        t_sus = peaks["bf16_tflops_sustained"] * (2.0 if fp8 else 1.0)
        roof["peak_sustained"] = round(t_sus, 3)
        roof["frac_sustained"] = round(achieved / t_sus, 4)
    roof["traffic"] = traffic
    roof["kernel"] = "gbsa forward (attention + split-KV combine launch)"
    roof["peak_source"] = peaks["source"] + " (burst)" + (
        "; E4M3 tensor peak = measured bf16 x 2 (nominal ratio)" if fp8 and tensor else "")
    return roof


def measure(name, args, dev, world, rank, sampler, dist, headline):
    """Times one workload: warm-up, then args.steps steps with CUDA events;
    for the headline also the end-to-end pipeline and the CPU baseline."""
    import torch

    import block_sparse_paged_gbsa_b200 as gbsa
    from block_sparse_paged_gbsa_b200.accounting import work
    from block_sparse_paged_gbsa_b200.workloads import make_values, pool_view, workload

    # each rank: its own seeded batch of the same workload (weak scaling)
    base = workload(name, scale_down=args.scale_down)
    w = workload(name, seed=rank_seed(base.seed, rank), scale_down=args.scale_down)
    tdt = {"bf16": torch.bfloat16, "fp16": torch.float16, "e4m3": torch.float8_e4m3fn}[args.dtype]
    fp8 = args.dtype == "e4m3"
    sp = args.softmax_precision
    scales = (1.0, 1.0, 1.0)  # E4M3 dequantization scales (the speed does not depend on them)
    acc = work(w, in_bytes=1 if fp8 else 2)
    q, kf, vf = make_values(w, dev, dtype=tdt)
    to = lambda a, dt: torch.as_tensor(np.ascontiguousarray(a), dtype=dt, device=dev)
    idx, cnt = to(w.sparse_idx, torch.int32), to(w.sparse_count, torch.int32)
    cu, sku, bt = to(w.cu_seqlens_q, torch.int64), to(w.kv_used, torch.int32), to(w.block_table, torch.int32)
    squ = to(w.q_used, torch.int32) if w.has_seqused_q else None
    k, v = pool_view(w, kf), pool_view(w, vf)
    block_shape = [w.block_x, 128]
    prob = gbsa.gbsa.make_problem(q, k, idx, block_shape, bt, cu, softmax_scale=w.scale,
                                  win_left=w.win_left, win_right=w.win_right,
                                  return_softmax_lse=w.return_lse, has_seqused_q=squ is not None,
                                  dequant_scales=scales, softmax_precision=sp)
    meta_buf = torch.empty(gbsa.metadata_size(prob) // 4, dtype=torch.int32, device=dev)
    ws = torch.empty(max(gbsa.workspace_size(prob), 16), dtype=torch.uint8, device=dev)
    out = torch.empty(q.shape, dtype=torch.bfloat16 if fp8 else tdt, device=dev)
    lse = torch.empty((w.T, w.N1, 1), dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step(qq=q, kk=k, vv=v, ii=idx, cc=cnt, uu=cu, su=squ, kv=sku, tb=bt, ev=None,
             oo=None, ll=None):
        if ev is not None:
            ev[0].record()
        meta = gbsa.metadata(ii, cc, w.N1, w.N2, w.D, block_shape, cu_seqlens_q=uu, seqused_q=su,
                             seqused_kv=kv, num_tokens=w.T, win_left=w.win_left,
                             win_right=w.win_right, dev_status=status, out=meta_buf)
        if ev is not None:
            ev[1].record()
        gbsa.forward(qq, kk, vv, ii, cc, block_shape, metadata=meta, cu_seqlens_q=uu,
                     seqused_q=su, seqused_kv=kv, block_table=tb, softmax_scale=w.scale,
                     win_left=w.win_left, win_right=w.win_right,
                     return_softmax_lse=w.return_lse, out=out if oo is None else oo,
                     lse=lse if ll is None else ll, workspace=ws, dev_status=status,
                     q_dequant_scale=scales[0], k_dequant_scale=scales[1],
                     v_dequant_scale=scales[2], softmax_precision=sp)
        if ev is not None:
            ev[2].record()

    for _ in range(max(3, args.warmup)):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    meta_host = meta_buf[:32].cpu().numpy()
    comb_cap = int(meta_host[10])
    # metadata (two kernels up to METADATA_FUSED_MAX_B sequences, else three),
    # the forward, and the combine when the work list can hold split pieces
    meta_launches = 2 if w.B <= gbsa.gbsa.METADATA_FUSED_MAX_B else 3
    launches_per_step = meta_launches + 1 + (1 if comb_cap > 0 else 0)

    events = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    for i in range(args.steps):
        flush.zero_()
        step(ev=events[i])
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t_wall1 = time.time()
    clocks = sampler.window(t_wall0, t_wall1)
    step_ms = float(np.mean([e[0].elapsed_time(e[2]) for e in events]))
    meta_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in events]))
    fwd_ms = float(np.mean([e[1].elapsed_time(e[2]) for e in events]))
    dev_bits = int(status.item())
    total_flops, total_kv = acc["flops_block"], acc["kv_bytes"]
    if world > 1:
        step_ms, meta_ms, fwd_ms = reduce_max([step_ms, meta_ms, fwd_ms], dist, dev)
        total_flops, total_kv = reduce_sum([total_flops, total_kv], dist, dev)

    # end to end through the public API: pinned host inputs -> device -> host
    # output, every step.  Steps are pipelined over two buffer sets and three
    # streams, as a serving loop would run them: step i's upload overlaps step
    # i-1's compute and step i-2's download.  The value is the steady-state
    # throughput, device time from the first upload to the last download over
    # the timed steps.
    e2e = None
    if headline and not args.no_e2e:
        host = {name_: t.cpu().pin_memory() for name_, t in
                dict(q=q, kf=kf, vf=vf, idx=idx, cnt=cnt, cu=cu, sku=sku, bt=bt).items()}
        if squ is not None:
            host["squ"] = squ.cpu().pin_memory()
        nbuf = 2
        dev_in = [{name_: torch.empty_like(t, device=dev) for name_, t in host.items()}
                  for _ in range(nbuf)]
        dev_out = [(torch.empty_like(out), torch.empty_like(lse)) for _ in range(nbuf)]
        host_out = [(torch.empty(out.shape, dtype=out.dtype).pin_memory(),
                     torch.empty(lse.shape, dtype=lse.dtype).pin_memory()) for _ in range(nbuf)]
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = out.numel() * out.element_size() + (lse.numel() * 4 if w.return_lse else 0)
        s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        ev_in = [torch.cuda.Event() for _ in range(nbuf)]
        ev_cmp = [torch.cuda.Event() for _ in range(nbuf)]
        ev_out = [torch.cuda.Event() for _ in range(nbuf)]

        def run_pipeline(n, t0=None, t1=None):
            for i in range(n):
                b = i % nbuf
                di, (do, dl), (ho, hl) = dev_in[b], dev_out[b], host_out[b]
                with torch.cuda.stream(s_in):
                    if i >= nbuf:
                        s_in.wait_event(ev_cmp[b])  # step i-2 no longer reads these inputs
                    if i == 0 and t0 is not None:
                        t0.record(s_in)
                    for name_, t in host.items():
                        di[name_].copy_(t, non_blocking=True)
                    ev_in[b].record(s_in)
                with torch.cuda.stream(s_cmp):
                    s_cmp.wait_event(ev_in[b])
                    if i >= nbuf:
                        s_cmp.wait_event(ev_out[b])  # step i-2's output has left
                    flush.zero_()
                    step(di["q"], pool_view(w, di["kf"]), pool_view(w, di["vf"]), di["idx"],
                         di["cnt"], di["cu"], di.get("squ"), di["sku"], di["bt"], oo=do, ll=dl)
                    ev_cmp[b].record(s_cmp)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_cmp[b])
                    ho.copy_(do, non_blocking=True)
                    if w.return_lse:
                        hl.copy_(dl, non_blocking=True)
                    ev_out[b].record(s_out)
                    if i == n - 1 and t1 is not None:
                        t1.record(s_out)
            torch.cuda.synchronize()

        run_pipeline(2 * nbuf)  # warm-up
        n_e2e = max(4, min(args.steps, 12))
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        run_pipeline(n_e2e, t0, t1)
        e2e_ms = t0.elapsed_time(t1) / n_e2e
        if world > 1:
            e2e_ms = reduce_max([e2e_ms], dist, dev)[0]
        e2e = {"value": round(job_value(total_flops, e2e_ms), 4),
               "unit": UNIT, "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": round(e2e_ms, 4),
               "pipelined": "two buffer sets; upload, compute and download of successive "
                            "steps overlap on three streams"}
        del host, dev_in, dev_out, host_out

    peaks = load_peaks()
    traffic = (profiled_traffic(name)
               if args.scale_down == 1 and args.dtype == "bf16" and sp == 0 else None)
    roof = roofline(acc, fwd_ms, peaks, fp8, traffic)
    t_peak = peaks["bf16_tflops"] * (2.0 if fp8 else 1.0)
    flops, nbytes = acc["flops_block"], acc["bytes"]
    t_roof = max(flops / (t_peak * 1e12), nbytes / (peaks["hbm_gbs"] * 1e9))

    cpu = None
    if headline and rank == 0 and world == 1 and not args.no_cpu_baseline:
        qc, kc, vc = q.cpu(), kf.cpu(), vf.cpu()
        tf, dt, n, threads = oracle_sample(w, qc, kc, vc, args.cpu_seconds, scales=scales)
        cpu = {"value": round(tf, 8), "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": f"{n} random (token, head) rows of the same workload, {dt:.1f} s"}

    res = {
        "workload": describe(name, args),
        "value": round(job_value(total_flops, step_ms), 4), "unit": UNIT,
        "ms_per_step": round(step_ms, 4), "metadata_ms": round(meta_ms, 4),
        "forward_ms": round(fwd_ms, 4),
        "kv_gbs": round(total_kv / (step_ms * 1e-3) / 1e9, 2),
        "roofline": roof,
        "roofline_step": {"time_ms": round(t_roof * 1e3, 5),
                          "frac": round(t_roof * 1e3 / step_ms, 4),
                          "flops": flops, "bytes": nbytes},
        "flops_exact": acc["flops_exact"],
        "clocks": clocks, "gpu_launches": launches_per_step * args.steps,
        "num_ctas": int(meta_host[7]), "dev_status": dev_bits,
    }
    del q, kf, vf, k, v, out, lse, ws, meta_buf, flush
    torch.cuda.empty_cache()
    return res, e2e, cpu


def measure_backward(name, args, dev, sampler):
    """Times gbsa.backward on one workload: the forward runs once first (out and
    lse are its inputs), then args.steps backward calls with CUDA events and
    the L2 flushed between them.  FLOPs: the five products per (tile, block)
    against the forward's two, block-granular."""
    import torch

    import block_sparse_paged_gbsa_b200 as gbsa
    from block_sparse_paged_gbsa_b200.accounting import work
    from block_sparse_paged_gbsa_b200.workloads import make_values, pool_view, workload

    w = workload(name, scale_down=args.scale_down)
    tdt = {"bf16": torch.bfloat16, "fp16": torch.float16}[args.dtype]
    acc = work(w, in_bytes=2)
    q, kf, vf = make_values(w, dev, dtype=tdt)
    to = lambda a, dt: torch.as_tensor(np.ascontiguousarray(a), dtype=dt, device=dev)
    idx, cnt = to(w.sparse_idx, torch.int32), to(w.sparse_count, torch.int32)
    cu, sku, bt = to(w.cu_seqlens_q, torch.int64), to(w.kv_used, torch.int32), to(w.block_table, torch.int32)
    squ = to(w.q_used, torch.int32) if w.has_seqused_q else None
    k, v = pool_view(w, kf), pool_view(w, vf)
    bs = [w.block_x, 128]
    meta = gbsa.metadata(idx, cnt, w.N1, w.N2, w.D, bs, cu_seqlens_q=cu, seqused_q=squ,
                         seqused_kv=sku, num_tokens=w.T, win_left=w.win_left,
                         win_right=w.win_right)
    kw = dict(metadata=meta, cu_seqlens_q=cu, seqused_q=squ, seqused_kv=sku, block_table=bt,
              softmax_scale=w.scale, win_left=w.win_left, win_right=w.win_right)
    out, lse = gbsa.forward(q, k, v, idx, cnt, bs, return_softmax_lse=True, **kw)
    g = torch.Generator(device=dev).manual_seed(99)
    dout = torch.randn(q.shape, generator=g, device=dev, dtype=torch.float32).to(tdt)
    dq = torch.empty(q.shape, dtype=torch.float32, device=dev)
    dk = torch.empty(k.shape, dtype=torch.float32, device=dev)
    dv = torch.empty(k.shape, dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step():
        gbsa.backward(dout, q, k, v, out, lse, idx, cnt, bs, dq=dq, dk=dk, dv=dv,
                      dev_status=status, **kw)

    for _ in range(max(3, args.warmup)):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    t_wall0 = time.time()
    for e in events:
        flush.zero_()
        e[0].record()
        step()
        e[1].record()
    torch.cuda.synchronize()
    clocks = sampler.window(t_wall0, time.time())
    ms = float(np.mean([e[0].elapsed_time(e[1]) for e in events]))
    flops = 2.5 * acc["flops_block"]
    peaks = load_peaks()
    achieved = flops / (ms * 1e-3) / 1e12
    return {
        "metric": "effective backward TFLOPS (dQ, dK, dV; block-granular FLOPs = 2.5 x the forward's)",
        "value": round(achieved, 4), "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": round(ms, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": args.dtype, "data": "synthetic",
        "config": {"workload": describe(name, args) + " -- backward",
                   "l2": "flushed between timed steps (256 MiB write)"},
        "roofline": {"bound": "tensor", "achieved": round(achieved, 3),
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": round(achieved / peaks["bf16_tflops"], 4), "traffic": None,
                     "kernel": "gbsa backward (delta + gradient kernels; mma.sync products)",
                     "peak_source": peaks["source"] + " (burst)"},
        "clocks": clocks, "gpu_launches": 2 * args.steps, "dev_status": int(status.item()),
        "e2e": None, "cpu_baseline": None,
    }


def main():
    args = parse_args()
    world, rank, local = dist_info()
    if args.impl == "reference":
        run_reference(args, world, rank)
        return

    import torch
    import torch.distributed as dist

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the CPU oracle arm is --impl reference)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    if args.backward:
        if world > 1:
            raise SystemExit("--backward runs on one GPU")
        sampler = ClockSampler(local)
        sampler.start()
        try:
            line = measure_backward("dense" if args.workload == "all" else args.workload, args,
                                    dev, sampler)
        finally:
            sampler.stop()
        print(json.dumps(line), flush=True)
        return

    names = ORDER if args.workload == "all" else [args.workload]
    head = headline_name(args)
    sampler = ClockSampler(local)
    sampler.start()
    results = {}
    try:
        for name in names:
            results[name] = measure(name, args, dev, world, rank, sampler, dist,
                                    headline=name == head)
    finally:
        sampler.stop()

    if rank == 0:
        res, e2e, cpu = results[head]
        line = {
            "metric": METRIC, "value": res["value"], "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": max(3, args.warmup),
            "ms_per_step": res["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": args.dtype, "data": "synthetic",
            "config": {"workload": res["workload"],
                       "parallelism": f"dp{world} (independent batches, no collective)",
                       "l2": "flushed between timed steps (256 MiB write)",
                       "num_ctas": res["num_ctas"]},
            "kv_gbs": res["kv_gbs"], "roofline_step": res["roofline_step"],
            "flops_exact": res["flops_exact"],
            "metadata_ms": res["metadata_ms"], "forward_ms": res["forward_ms"],
            "roofline": res["roofline"], "clocks": res["clocks"], "e2e": e2e,
            "cpu_baseline": cpu, "gpu_launches": res["gpu_launches"],
            "dev_status": res["dev_status"],
        }
        if len(names) > 1:
            line["per_config"] = {n: results[n][0] for n in names if n != head}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
