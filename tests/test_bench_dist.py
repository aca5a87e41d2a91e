"""bench.py's multi-process plumbing on CPU: two gloo ranks (the one-process-
per-GPU layout of `torchrun bench.py --gpus N`, without GPUs) agree on the
slowest rank's time, pass the barrier, and turn it into the whole-job rate."""
import os
import socket

import pytest


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    ms_local = 10.0 + 5.0 * rank                      # rank 1 is the slower one
    bench.barrier(world)
    ms = bench.max_over_ranks(ms_local, world)
    rate = bench.whole_job_rate(3.0e12, 4, world, ms)
    bench.barrier(world)
    dist.destroy_process_group()
    out.put((rank, ms, rate))


def test_two_gloo_ranks_take_the_slowest_time():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [15.0, 15.0]
    # 2 ranks x 4 steps x 3e12 FLOP in 15 ms
    assert res[0][2] == pytest.approx(2 * 4 * 3.0e12 / 0.015)
    assert res[0][2] == res[1][2]


def test_single_process_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(7.5, 1) == 7.5
    assert bench.whole_job_rate(1.0, 10, 1, 1000.0) == pytest.approx(10.0)
