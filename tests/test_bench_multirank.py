"""The multi-rank logic of bench.py on CPU: two gloo ranks report different timings, both
see the slowest rank's, and the whole-job rate counts every rank's bytes over that time."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [10.0 + rank, 20.0 - rank, 5.0 * (rank + 1)]
        got = bench.max_over_ranks(mine)
        rate = bench.job_rate(1e9, 4, world, got[0])
        q.put((rank, got, rate))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_max_over_ranks_and_job_rate_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(90)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=10) for _ in range(world))
    for _, got, rate in res:
        assert got == [11.0, 20.0, 10.0]                     # element-wise max over the ranks
        assert abs(rate - 1e9 * 4 * 2 / (11.0e-3) / 1e9) < 1e-9   # both ranks' bytes / slowest time


def test_single_process_is_identity():
    import bench
    assert bench.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
    assert bench.job_rate(2e9, 10, 1, 1000.0) == 20.0
