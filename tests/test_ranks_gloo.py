"""Multi-rank bookkeeping of bench.py on CPU ranks (gloo, world size 2): the
timing is the slowest rank's and the rate counts the units of all ranks."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    ms = 100.0 + 50.0 * rank                       # rank 1 is slower
    worst = bench.max_over_ranks_of(ms, world, torch.device("cpu"))
    rate = bench.whole_job_rate(1000, 10, world, worst)
    q.put((rank, worst, rate))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_rate_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, worst, rate in res:
        assert worst == 150.0
        assert rate == pytest.approx(2 * 1000 * 10 / 0.150)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks_of(3.5, 1, None) == 3.5
    assert bench.whole_job_rate(10, 2, 1, 1000.0) == 20.0
