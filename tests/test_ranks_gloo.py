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


# ------------------------------------------------ sequence-sharded step exchanges
def _fake_step(rank, world, log):
    """The exchange pattern of shard_step with stand-in tensors: a summed
    histogram, then a gather in rank order."""
    h = torch.full((3, 2048), rank + 1, dtype=torch.int32)
    h[0, rank] += 100
    yield ("sum", h)
    log.append(h.clone())
    src = torch.arange(5, dtype=torch.float32) + 10 * rank
    dst = torch.empty((world, 5))
    yield ("gather", src, dst)
    log.append(dst.clone())


def _shard_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from query_aware_sparse_decode_b200.shard import TorchCollectives
    log = []
    TorchCollectives().run(_fake_step(rank, world, log))
    q.put((rank, [t.tolist() for t in log]))
    dist.barrier()
    dist.destroy_process_group()


def _expected(world):
    from query_aware_sparse_decode_b200.shard import run_lockstep
    logs = [[] for _ in range(world)]
    run_lockstep(_fake_step(r, world, logs[r]) for r in range(world))
    return logs


def test_shard_exchanges_torch_distributed_world2_match_lockstep():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    want = _expected(2)
    for r in range(2):
        assert res[r] == [t.tolist() for t in want[r]]
    hsum, gathered = want[0]
    assert hsum[0, 0].item() == 103 and hsum[0, 1].item() == 103 and hsum[1, 5].item() == 3
    assert gathered[1].tolist() == [10.0, 11.0, 12.0, 13.0, 14.0]      # rank order


def test_lockstep_rejects_ranks_out_of_step():
    from query_aware_sparse_decode_b200.shard import run_lockstep

    def a():
        yield ("sum", torch.zeros(2, dtype=torch.int32))

    def b():
        yield ("gather", torch.zeros(2), torch.zeros((2, 2)))

    with pytest.raises(RuntimeError):
        run_lockstep([a(), b()])
    with pytest.raises(RuntimeError):
        run_lockstep([a(), iter(())])


# ------------------------------------------------ shard_step itself over torch.distributed
class _FakeLibrary:
    """Stands in for a rank's library context on the CPU: every call that
    shard_step makes records its inputs and writes rank-dependent values into
    the real ShardBuffers, so the exchanges move the shapes and contents the
    GPU path moves (no GPU in these tests)."""

    def __init__(self, cfg, rank):
        self.cfg, self.rank, self.seen = cfg, rank, []

    def append_kv(self, layer, k, v, stream=None):
        self.seen.append(("append", layer))

    def shard_set(self, layer, t0, glens):
        self.seen.append(("set", layer, t0, tuple(glens)))

    def score(self, layer, q_imp, scores, stream=None):
        scores.fill_(float(self.rank + 1))

    def shard_hist(self, layer, scores, p, state, hist, stream=None):
        hist.zero_()
        hist[:, 7 * p + self.rank] = 1 + p + 10 * self.rank

    def shard_pick(self, layer, p, hist, n_ranks, rank, state, stream=None):
        self.seen.append(("pick", p, n_ranks, rank, hist.clone()))

    def shard_mask(self, layer, scores, state, mask, stream=None):
        mask.fill_(self.rank)

    def sparse_attn_partial(self, layer, q, mask, mode, part, stream=None):
        part.copy_(torch.arange(part.numel(), dtype=torch.float32) + 1000 * self.rank)

    def merge_partials(self, parts, n, out, lse, stream=None):
        self.seen.append(("merge", n, parts.clone()))


def _shard_step_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from query_aware_sparse_decode_b200 import tb as TB
    from query_aware_sparse_decode_b200.shard import ShardBuffers, TorchCollectives, shard_step
    cfg = TB.make_config(2, 2, 8, 2, 64, 16, 1, 512, "bf16", 30, 4, 8, dense_layers=(0,))
    lib = _FakeLibrary(cfg, rank)
    bufs = ShardBuffers(cfg, world, torch.device("cpu"))
    for layer in (0, 1):   # a dense layer (partials only) and a sparse one (all exchanges)
        TorchCollectives().run(shard_step(lib, layer, rank, world, 256 * rank, [500, 480], None, None, None, bufs,
                                          "k" if rank == world - 1 else None, "v" if rank == world - 1 else None))
    q.put((rank, [(s[0],) + tuple(x.tolist() if torch.is_tensor(x) else x for x in s[1:]) for s in lib.seen]))
    dist.barrier()
    dist.destroy_process_group()


def test_shard_step_over_torch_distributed_world2_matches_lockstep():
    """shard_step's own exchange sequence (two summed histograms, a gathered
    histogram, gathered partials) with the real ShardBuffers shapes, run by
    TorchCollectives over two gloo processes, hands every library call the
    same tensors as the one-process lock-step runner, rank order kept."""
    from query_aware_sparse_decode_b200 import tb as TB
    from query_aware_sparse_decode_b200.shard import ShardBuffers, run_lockstep, shard_step
    ctx = mp.get_context("spawn")
    qu = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_step_worker, args=(r, 2, port, qu)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(qu.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    cfg = TB.make_config(2, 2, 8, 2, 64, 16, 1, 512, "bf16", 30, 4, 8, dense_layers=(0,))
    libs = [_FakeLibrary(cfg, r) for r in range(2)]
    bufs = [ShardBuffers(cfg, 2, torch.device("cpu")) for _ in range(2)]
    for layer in (0, 1):
        run_lockstep(shard_step(libs[r], layer, r, 2, 256 * r, [500, 480], None, None, None, bufs[r],
                                "k" if r == 1 else None, "v" if r == 1 else None) for r in range(2))
    for r in range(2):
        want = [(s[0],) + tuple(x.tolist() if torch.is_tensor(x) else x for x in s[1:]) for s in libs[r].seen]
        assert res[r] == want
    # the summed first digit holds both ranks' counts; the last digit is gathered in rank order
    picks = [s for s in libs[0].seen if s[0] == "pick"]
    assert picks[0][4][0, 0].item() == 1 and picks[0][4][0, 1].item() == 11
    assert picks[2][4].shape == (2, 2 * 8, 2048) and picks[2][4][1, 0, 15].item() == 13
    merges = [s for s in libs[1].seen if s[0] == "merge"]
    assert len(merges) == 2 and merges[1][2][1, 0].item() == 1000.0
