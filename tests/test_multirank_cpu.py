"""The N > 1 bench path on CPU: two gloo ranks exercise the same host logic
torchrun runs on GPUs (independent batches per rank, the max-over-ranks step
time, the whole-job rate, and the reference arm that only rank 0 runs)."""
from __future__ import annotations

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from long_context_sparse_lsa_b200 import workloads as wls


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # ranks time different amounts; every rank reports the maximum
        mine = 1.0 + rank * 0.5
        got = bench.max_over_ranks(mine, dist, torch.device("cpu"))
        wl = bench.rank_workload(wls.BATCH128K, rank)
        # the reference arm runs on rank 0 only: other ranks return at once
        ref_rc = None
        if rank != 0:
            args = type("A", (), {"warmup": 3, "steps": 1, "ref_seconds": 0.1, "gpus": world})()
            ref_rc = bench.run_reference(args, wls.TINY)
        out.put((rank, got, wl.seed, wl.lens, ref_rc))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_draw_independent_batches():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [1.5, 1.5]           # max over ranks, on every rank
    assert res[0][2] != res[1][2]                      # different seeds: independent batches
    assert res[0][3] == res[1][3]                      # same shape (weak scaling)
    assert res[1][4] == 0                              # reference arm: rank 1 exits without work


def test_job_rate_counts_every_rank():
    # 16 queries per rank on 4 ranks in 2 ms (the max over ranks) -> 32000 queries/s
    assert bench.job_rate(16, 4, 2.0) == pytest.approx(32000.0)
    assert bench.max_over_ranks(3.0, None, "cpu") == 3.0
