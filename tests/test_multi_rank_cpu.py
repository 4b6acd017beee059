"""Host logic of the N-GPU bench on CPU: two gloo ranks, replicas only.

Each rank times its own replica; the job's time is the slowest rank's and the
value counts every rank's units. No data-path collective exists (channels and
sequences shard with no exchange), so the only collectives are the timing
barrier and the max over ranks, exercised here with gloo on 127.0.0.1.
"""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        bench._barrier_sync(world)
        ms = 1.0 + rank  # rank 1 is the slowest
        ms_max = bench._max_over_ranks(ms, world)
        value = bench.whole_job_rate(1e9, world, ms_max)
        info = bench.dist_info()
        out.put((rank, ms_max, value, info))
        bench._barrier_sync(world)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms_max, value, info in res:
        assert ms_max == 2.0
        # 2 ranks x 1e9 units in 2 ms = 1000 G units/s
        assert value == pytest.approx(1000.0)
        assert info == (rank, rank, world)
