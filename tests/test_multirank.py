"""Multi-rank host logic of the bench on CPU: two gloo ranks, no GPU.

The token mix has no exchange step, so N ranks each process their own grid
(weak scaling). What needs checking is the plumbing: each rank draws a
different grid, the job's step time is the slowest rank's, and the job
throughput counts every rank's tokens. The data-path computation here is the
CPU oracle standing in for the GPU kernels, run on a tiny grid per rank.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import workloads


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle

        cfg = workloads.CONFIGS["tiny"]
        inp = workloads.generate(cfg, seed=bench.rank_seed(rank))
        y = oracle.get().bissd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], 0, cfg.review)
        local_ms = 10.0 + 5.0 * rank              # a fake per-rank step time
        ms = bench.max_over_ranks(local_ms, dist)
        value = bench.job_throughput(cfg.tokens, world, ms)
        # every rank must see the same reduced time and value; the grids must differ
        checksum = torch.tensor([float(np.abs(y).sum())], dtype=torch.float64)
        gathered = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(gathered, checksum)
        out[rank] = (ms, value, [float(g.item()) for g in gathered])
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_weak_scaling():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    tokens = workloads.CONFIGS["tiny"].tokens
    for rank in range(world):
        ms, value, sums = out[rank]
        assert ms == pytest.approx(15.0)                               # max over ranks
        assert value == pytest.approx(tokens * world / 15e-3 / 1e6)    # all ranks' tokens
        assert sums[0] != pytest.approx(sums[1])                       # different grids per rank
    assert out[0][2] == out[1][2]


def test_single_rank_plumbing_is_identity():
    assert bench.max_over_ranks(3.5, None) == 3.5
    assert bench.rank_seed(0) == 0 and bench.rank_seed(3, base=10) == 13
    assert bench.job_throughput(1_000_000, 4, 1000.0) == pytest.approx(4.0)
