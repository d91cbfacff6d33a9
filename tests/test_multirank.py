"""The multi-rank bench plumbing on CPU: two gloo ranks (no GPU).

The path needs no collective, so N GPUs run N independent replicas; the only
cross-rank steps are the barrier around the timed region and the max-over-ranks
of the device time, from which the whole-job rate is computed.
"""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        my_ms = 10.0 + 5.0 * rank          # rank 1 is the slowest
        ms = bench.max_over_ranks(my_ms, world)
        rate = bench.job_throughput(1000.0, 4, ms, world)
        q.put((rank, ms, rate))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time_and_sum_the_work():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms, rate in res:
        assert ms == 15.0
        # 2 ranks x 1000 units x 4 steps in 15 ms.
        assert rate == pytest.approx(2 * 1000 * 4 / 0.015)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_throughput(10.0, 2, 1000.0, 1) == pytest.approx(20.0)
