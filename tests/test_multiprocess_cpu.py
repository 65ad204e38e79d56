"""Host-side logic of the multi-GPU benchmark, on CPU with gloo (world size 2).

The layer does not exchange data between GPUs: each rank runs its own token
rows through a replica of the packed weight.  What the ranks share is the
timing: the step time is the max over ranks, and the reported throughput is
the work of all ranks over that time.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, times, out):
    import datetime

    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w, r, l = bench.dist_env()
        assert (w, r, l) == (world, rank, rank)
        t_max = bench.max_over_ranks(times[rank], world)
        out[rank] = (t_max, bench.aggregate(1e12, world, t_max))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_aggregate():
    world = 2
    times = [0.004, 0.005]          # rank 1 is slower
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_worker, args=(r, world, port, times, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    for r in range(world):
        t_max, value = res[r]
        assert t_max == pytest.approx(0.005)
        # 2 ranks x 1 TFLOP each over the slowest rank's 5 ms = 400 TFLOP/s
        assert value == pytest.approx(2 * 1e12 / 0.005 / 1e12)


def test_single_process_is_identity():
    import bench

    assert bench.max_over_ranks(1.25, 1) == 1.25
    assert bench.aggregate(2e12, 1, 0.5) == pytest.approx(4.0)
