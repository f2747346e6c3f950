"""The benchmark's multi-rank plumbing on CPU: two gloo ranks take the
barrier, agree on the slowest rank's time, and report the whole job's
throughput from it (independent replicas, no collective in the data path)."""
import datetime
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, times, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        bench.barrier(world)
        ms_max = bench.max_over_ranks(times[rank], world)
        q.put((rank, ms_max, bench.job_throughput(world, 1000, ms_max)))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_report_the_slowest_rank():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    times = [12.5, 40.0]  # ms of timed steps on each rank
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, times, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for _, ms_max, value in got:
        assert ms_max == 40.0
        # 2 replicas x 1000 steps in the slowest rank's 40 ms
        assert value == pytest.approx(2 * 1000 / 0.040)


def test_single_rank_is_its_own_maximum():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25, 1) == 3.25
    assert bench.job_throughput(1, 500, 250.0) == pytest.approx(2000.0)
