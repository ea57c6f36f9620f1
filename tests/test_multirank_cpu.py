"""The multi-rank host logic of bench.py (weak-scaled replicas: max-over-ranks step time and device status, whole-
job token count), run as two gloo ranks on the CPU."""

from __future__ import annotations

import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, out):
    import datetime

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench

        # rank r reports a step time of 10 + r ms and status 0, except rank 1 which reports status 4 (a timeout)
        ms, status = bench.max_over_ranks([10.0 + rank, 4 if rank == 1 else 0], world, "cpu")
        torch.distributed.barrier()
        tokens = bench.whole_job_tokens({"B": 1, "N": 524288}, world)
        out.put((rank, ms, status, tokens))
    finally:
        torch.distributed.destroy_process_group()


def test_max_over_ranks_and_whole_job_tokens():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(out.get(timeout=5) for _ in range(world))
    for rank, ms, status, tokens in res:
        assert ms == 11.0  # the slowest rank's time, on every rank
        assert status == 4  # a status raised on one rank reaches all of them (all raise together)
        assert tokens == 2 * 524288  # weak scaling: every rank's own batch counts


def test_single_rank_is_identity():
    import bench

    assert bench.max_over_ranks([3.5, 0], 1, "cpu") == [3.5, 0.0]
    assert bench.whole_job_tokens({"B": 2, "N": 4096}, 1) == 8192
