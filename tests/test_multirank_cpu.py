"""Multi-rank host logic of bench.py on CPU: two gloo ranks on 127.0.0.1.

Data-parallel decode runs one replica of the workload per GPU (weak scaling): the
only cross-rank steps are a barrier and the max of the ranks' timed seconds. These
tests run that exact code (bench.max_over_ranks, bench.whole_job_rate) in two
processes with the gloo backend, so no GPU is involved.
"""
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_q):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        elapsed = 2.0 if rank == 1 else 1.5           # rank 1 is the slow one
        mx = bench.max_over_ranks(elapsed, world)
        rate, el = bench.whole_job_rate(10.0, 3, elapsed, world)
        out_q.put((rank, mx, rate, el))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
            pytest.fail("a rank did not finish")
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, mx, rate, el in got:
        assert mx == 2.0 and el == 2.0
        assert rate == pytest.approx(2 * 10.0 * 3 / 2.0)   # both replicas' units in the slowest time


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(1.25, 1) == 1.25
    rate, el = bench.whole_job_rate(4.0, 5, 2.0, 1)
    assert el == 2.0 and rate == pytest.approx(10.0)
