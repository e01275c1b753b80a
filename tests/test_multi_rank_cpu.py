"""The multi-GPU path of the benchmark, exercised on the CPU with two gloo
ranks: per-rank seeding gives independent batches, the timing reduction is
the max over ranks, and the whole-job value counts every rank's work."""
import os
import socket

import numpy as np
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from block_sparse_paged_gbsa_b200.accounting import work
from block_sparse_paged_gbsa_b200.workloads import workload


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        base = workload("tiny")
        w = workload("tiny", seed=bench.rank_seed(base.seed, rank))
        flops = work(w, exact=False)["flops_block"]
        local_ms = [1.0 + rank, 0.5 * (rank + 1)]          # rank 1 is the slow one
        mx = bench.reduce_max(local_ms, dist, "cpu")
        total = bench.reduce_sum([flops], dist, "cpu")[0]
        out[rank] = (w.seed, int(w.sparse_idx.sum()), flops, mx, total,
                     bench.job_value(total, mx[0]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:  # no fork of a threaded process
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    (s0, i0, f0, mx0, t0, v0), (s1, i1, f1, mx1, t1, v1) = res[0], res[1]
    assert s0 != s1 and i0 != i1                # independent batches
    assert mx0 == mx1 == [2.0, 1.0]             # max over ranks
    assert t0 == t1 == f0 + f1                  # every rank's own work counts
    assert v0 == v1 == (f0 + f1) / 2e-3 / 1e12
