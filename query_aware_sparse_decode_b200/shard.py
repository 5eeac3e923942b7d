"""Sequence-sharded decode step: the order of the library calls on one rank
and the exchanges between ranks (include/tb.h, "Sequence-sharded decode").

Rank r holds, for every sequence, the contiguous global tokens
[t0_r, t0_r + len) of a layer's caches; ranks are in token order and the
last one receives the appended tokens.  `shard_step` is a generator: it
issues this rank's kernels on the stream and yields at every exchange,

    ("sum", t)             t summed over ranks, in place (radix histograms);
    ("gather", src, dst)   dst[r] = rank r's src (last-digit histograms, the
                           fp32 partial outputs);

and a runner carries the exchange out:

    TorchCollectives(group).run(step)   one rank per process, torch.distributed
                                        (NCCL over NVLink on GPUs);
    run_lockstep(steps)                 several ranks' steps in one process,
                                        each with its own context, exchanging
                                        by adding / copying their tensors; no
                                        kernel of one waits on another's.

Every step of the computation runs in the library's kernels; this module
only orders the calls and moves the exchanged tensors.
"""
from __future__ import annotations

import torch

from . import tb as TB

HIST_BINS = 2048


def sel_rows(cfg) -> int:
    """Selection rows per sequence: query heads, or KV groups with per-group selection."""
    return cfg.n_kv_heads if cfg.variant == TB.TB_BUTLER_GROUP else cfg.n_q_heads


class ShardBuffers:
    """Device buffers of one rank's sharded step (layouts in include/tb.h)."""

    def __init__(self, cfg, world: int, device=None):
        dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
        rows = sel_rows(cfg)
        nrow = cfg.batch * rows
        self.world = world
        self.scores = torch.empty((cfg.batch, rows, cfg.max_len), dtype=torch.float32, device=dev)
        self.hist = torch.empty((nrow, HIST_BINS), dtype=torch.int32, device=dev)
        self.hist_all = torch.empty((world, nrow, HIST_BINS), dtype=torch.int32, device=dev)
        self.state = torch.zeros((nrow, 4), dtype=torch.int32, device=dev)
        self.mask = torch.zeros((cfg.batch, rows, cfg.max_len // 32), dtype=torch.int32, device=dev)
        nq = cfg.batch * cfg.n_q_heads
        self.part = torch.empty(nq * cfg.head_dim + nq, dtype=torch.float32, device=dev)
        self.part_all = torch.empty((world, self.part.numel()), dtype=torch.float32, device=dev)


def shard_step(ctx: TB.Context, layer: int, rank: int, world: int, t0: int, global_lens, q, q_imp, out,
               bufs: ShardBuffers, k_new=None, v_new=None, stream=None):
    """One decode step of `layer` on this rank.  `global_lens`: every
    sequence's length after this step's append; `k_new`, `v_new`: the new
    token's K and V, given on the rank that holds the sequences' ends (it
    appends them and projects their K_imp).  `out` [B][Hq][D] receives the
    merged attention on every rank."""
    cfg = ctx.cfg
    if k_new is not None:
        ctx.append_kv(layer, k_new, v_new, stream)
    ctx.shard_set(layer, t0, global_lens)
    dense = ((cfg.dense_layer_mask >> layer) & 1) or cfg.keep_pct >= 100
    if dense:
        ctx.sparse_attn_partial(layer, q, None, TB.TB_MASK_DENSE, bufs.part, stream)
    else:
        ctx.score(layer, q_imp, bufs.scores, stream)
        for p in (0, 1):
            ctx.shard_hist(layer, bufs.scores, p, bufs.state, bufs.hist, stream)
            yield ("sum", bufs.hist)
            ctx.shard_pick(layer, p, bufs.hist, 1, 0, bufs.state, stream)
        ctx.shard_hist(layer, bufs.scores, 2, bufs.state, bufs.hist, stream)
        yield ("gather", bufs.hist, bufs.hist_all)
        ctx.shard_pick(layer, 2, bufs.hist_all, world, rank, bufs.state, stream)
        ctx.shard_mask(layer, bufs.scores, bufs.state, bufs.mask, stream)
        mode = TB.TB_MASK_GROUP if cfg.variant == TB.TB_BUTLER_GROUP else TB.TB_MASK_PER_HEAD
        ctx.sparse_attn_partial(layer, q, bufs.mask, mode, bufs.part, stream)
    yield ("gather", bufs.part, bufs.part_all)
    ctx.merge_partials(bufs.part_all, world, out, None, stream)


class TorchCollectives:
    """Exchanges through torch.distributed (one rank per process)."""

    def __init__(self, group=None):
        self.group = group

    def run(self, step) -> None:
        import torch.distributed as dist
        for op in step:
            if op[0] == "sum":
                dist.all_reduce(op[1], group=self.group)
            elif op[0] == "gather":
                src, dst = op[1], op[2]    # dst [world, *src.shape], as world stacked copies of src
                dist.all_gather_into_tensor(dst.view(-1, *src.shape[1:]), src, group=self.group)
            else:
                raise ValueError(f"unknown exchange {op[0]!r}")


def run_lockstep(steps) -> None:
    """Advance several ranks' steps (rank order) together in one process,
    carrying out each exchange between them."""
    steps = list(steps)
    while True:
        ops = [next(s, None) for s in steps]
        if all(o is None for o in ops):
            return
        exchange_in_process(ops)


def exchange_in_process(ops) -> None:
    """One exchange among ranks that share a process: ops[r] is rank r's
    request, all of the same kind."""
    if any(o is None for o in ops) or len({o[0] for o in ops}) != 1:
        raise RuntimeError("ranks out of step: " + ", ".join("done" if o is None else o[0] for o in ops))
    if ops[0][0] == "sum":
        total = ops[0][1].clone()
        for o in ops[1:]:
            total += o[1]
        for o in ops:
            o[1].copy_(total)
    elif ops[0][0] == "gather":
        for o in ops:
            for r, src in enumerate(ops):
                o[2][r].copy_(src[1])
    else:
        raise ValueError(f"unknown exchange {ops[0][0]!r}")
