"""Sequence-sharded decode on one GPU: R ranks, each with its own context
holding a contiguous token range of the same layer, run in lock step
(shard.run_lockstep; no kernel of one rank waits on another's).  The merged
step must select the oracle's set (decode_layer_sharded: the one-device
set) within the tie band, give the oracle's attention over the selected set
(the GPU's own set where the two differ inside the band), and, with
identical K_imp rows, select exactly what the one-context step selects.
The oracle never sees a GPU value other than a selected index set."""
import math

import numpy as np
import pytest
import torch

from oracle import tokenbutler as O
from query_aware_sparse_decode_b200 import synth as S
from query_aware_sparse_decode_b200 import tb as TB
from query_aware_sparse_decode_b200.shard import ShardBuffers, run_lockstep, sel_rows, shard_step

from harness import (assert_close_rows, bf16_score_slack, config_of, kimp_rows, make_layer, paged_copy, round_up,
                     sets_from_mask, tdtype, tie_band_ok, to_dev)

pytestmark = pytest.mark.gpu

WL = S.Workload("shard_bf16", n_layers=1, B=2, Hq=8, Hkv=2, D=128, d_imp=32, G=1, L=3000, dtype="bf16",
                keep_pct=30, sink=16, window=64, lens=(3000, 2500))


class _Slice:
    """The caches of one rank, shaped like a layer for paged_copy."""

    def __init__(self, k, v):
        self.k_cache, self.v_cache = k, v


def _rank_layer(ld, wl, t0, t1, lens0, variant, last, kimp_dtype="f32", paged=False):
    """A context holding global tokens [t0, t1) of the full layer `ld` (the
    last rank: [t0, len) and room for the appended token), dense or in
    shuffled pages."""
    n = [min(L, t1) - t0 for L in lens0]
    cap = round_up(max(n) + (1 if last else 0) + 1, 256)
    cfg = config_of(wl, max_len=cap, variant=variant, kimp_dtype=kimp_dtype)
    ctx = TB.Context(cfg)
    k = torch.zeros((wl.B, wl.Hkv, cap, wl.D), dtype=tdtype(wl), device="cuda")
    v = torch.zeros_like(k)
    for b in range(wl.B):
        k[b, :, :n[b]] = ld.k_cache[b, :, t0:t0 + n[b]]
        v[b, :, :n[b]] = ld.v_cache[b, :, t0:t0 + n[b]]
    kimp = TB.kimp_cache(cfg)
    if paged:
        # paged bf16 caches project K_imp with fp32 FMA, not the tensor cores:
        # take the one context's K_imp rows instead, so the scores stay equal
        kpool, vpool, table = paged_copy(_Slice(k, v), wl, cap, 64, 11 + t0)
        ctx.bind_layer_paged(0, kpool, vpool, table, kimp, ld.w_k)
        B, Hkv, nt, d, _ = ld.kimp.shape
        rows = ld.kimp.permute(0, 1, 2, 4, 3).reshape(B, Hkv, nt * 256, d)
        mine = torch.zeros((B, Hkv, cap, d), dtype=rows.dtype, device="cuda")
        for b in range(B):
            mine[b, :, :n[b]] = rows[b, :, t0:t0 + n[b]]
        kimp.copy_(mine.reshape(B, Hkv, cap // 256, 256, d).permute(0, 1, 2, 4, 3))
    else:
        ctx.bind_layer(0, k, v, kimp, ld.w_k)
    ctx.set_seq_lens(0, n)
    if not paged:
        ctx.project_kimp(0, 0, max(n))
    return ctx, kimp


def _run(wl, starts, variant=TB.TB_BUTLER, periodic=None, kimp_dtype="f32", paged_ranks=()):
    """One sharded decode step with ranks starting at `starts` (token
    indices, ascending, starts[0] = 0), compared with the oracle and with
    the one-context step."""
    group = variant == TB.TB_BUTLER_GROUP
    lens0 = [L - 1 for L in wl.seq_lens]
    full = TB.Context(config_of(wl, variant=variant, kimp_dtype=kimp_dtype))
    ld = make_layer(full, wl, 0, lens0)
    if periodic is not None:     # every candidate repeats the key of an earlier token: ties across ranks
        src = ld.k_cache.clone()
        for t in range(wl.sink + periodic, max(lens0)):
            ld.k_cache[:, :, t] = src[:, :, wl.sink + (t - wl.sink) % periodic]
        ld.K[:, :, :max(lens0)] = ld.k_cache[:, :, :max(lens0)].float().cpu().numpy()
    full.project_kimp(0, 0, max(lens0))
    R = len(starts)
    bounds = [(starts[r], starts[r + 1] if r + 1 < R else 1 << 30) for r in range(R)]
    ranks = [_rank_layer(ld, wl, t0, t1, lens0, variant, r == R - 1, kimp_dtype, r in paged_ranks)
             for r, (t0, t1) in enumerate(bounds)]
    k_raw, v_raw = S.kv_new(wl, 0)
    k_dev, v_dev = to_dev(k_raw, wl), to_dev(v_raw, wl)
    glens = [L + 1 for L in lens0]
    outs, bufs = [], []
    steps = []
    for r, (ctx, _) in enumerate(ranks):
        bufs.append(ShardBuffers(ctx.cfg, R))
        outs.append(torch.empty((wl.B, wl.Hq, wl.D), dtype=tdtype(wl), device="cuda"))
        last = r == R - 1
        steps.append(shard_step(ctx, 0, r, R, bounds[r][0], glens, ld.q_dev, ld.q_imp_dev, outs[r], bufs[r],
                                k_dev if last else None, v_dev if last else None))
    run_lockstep(steps)
    dense = wl.keep_pct >= 100
    # the one-context step
    out_full = torch.empty_like(outs[0])
    full.decode_step(0, k_dev, v_dev, ld.q_dev, ld.q_imp_dev, out_full)
    masks_full = None if dense else full.step_masks(sel_rows(full.cfg))
    torch.cuda.synchronize()
    for ctx, _ in ranks:
        assert ctx.check_status() == 0
    assert full.check_status() == 0
    for o in outs[1:]:
        assert torch.equal(o, outs[0])                 # every rank holds the merged output
    got = {}
    same_kimp = True
    if not dense:
        # global sets from the ranks' local masks
        for r, (ctx, kimp) in enumerate(ranks):
            n = ctx.seq_lens(0)
            for key, idx in sets_from_mask(bufs[r].mask, n).items():
                got.setdefault(key, []).append(idx + bounds[r][0])
            # K_imp rows of the rank (appended row included) against the one context's
            kr, kf = kimp_rows(kimp), kimp_rows(ld.kimp)
            t0 = bounds[r][0]
            for b in range(wl.B):
                same_kimp &= np.array_equal(kr[b, :, :n[b]], kf[b, :, t0:t0 + n[b]])
        got = {key: np.concatenate(v) for key, v in got.items()}
        if same_kimp:   # identical scores on both sides: identical sets
            for key, want in sets_from_mask(masks_full, glens).items():
                assert np.array_equal(got[key], want), f"row {key}: sharded != one-context"
    # oracle
    K = np.concatenate([ld.K, np.zeros((wl.B, wl.Hkv, 1, wl.D))], axis=2)
    V = np.concatenate([ld.V, np.zeros((wl.B, wl.Hkv, 1, wl.D))], axis=2)
    k64, v64 = S.widen(k_raw, wl.dtype), S.widen(v_raw, wl.dtype)
    for b, L in enumerate(glens):
        K[b, :, L - 1], V[b, :, L - 1] = k64[b], v64[b]
    obounds = [(t0, min(t1, max(glens))) for t0, t1 in bounds]
    storage = "bf16" if kimp_dtype == "bf16" else "f64"
    sel, ref, _, _ = O.decode_layer_sharded(ld.q, K, V, ld.W, ld.qimp, 0, wl.G, glens, wl.keep_pct, wl.sink,
                                            wl.window, obounds, group=group, kimp_storage=storage)
    _, _, _, sc = O.decode_layer(ld.q, K, V, ld.W, ld.qimp, 0, wl.G, glens, wl.keep_pct, wl.sink, wl.window,
                                 dense=False, group=group, kimp_storage=storage)
    o = outs[0].float().cpu().numpy()
    gs = wl.Hq // wl.Hkv
    mism = 0
    if dense:
        for (b, h), want in ref.items():
            assert_close_rows(o[b, h][None], want[None], wl.dtype, f"b{b} h{h}")
        return got, sel, same_kimp
    for b, L in enumerate(glens):
        for h in range(wl.Hq):
            r = h // gs if group else h
            slack = None
            if kimp_dtype == "bf16":
                g = h // gs
                qabs = np.abs(ld.qhat[b, g * gs:(g + 1) * gs]).sum(axis=0) if group else np.abs(ld.qhat[b, h])
                slack = bf16_score_slack(qabs, K[b, g, :L], ld.W)
            assert tie_band_ok(got[b, r], sel[b, h], sc[b, h], L, wl.keep_pct, wl.sink, wl.window, slack), \
                f"b{b} h{h}"
            want = ref[b, h]
            if not np.array_equal(got[b, r], sel[b, h]):
                mism += 1
                g = h // gs
                want, _ = O.attend(ld.q[b, h], K[b, g, :L], V[b, g, :L], got[b, r], 1.0 / math.sqrt(wl.D))
            assert_close_rows(o[b, h][None], want[None], wl.dtype, f"b{b} h{h}")
    assert mism <= max(1, wl.B * wl.Hq // 20)
    return got, sel, same_kimp


@pytest.mark.parametrize("starts", [(0,), (0, 1500), (0, 1000, 2100), (0, 700, 1400, 2400), (0, 1000, 2499)],
                         ids=["R1", "R2", "R3", "R4", "R3_last_rank_empty_before_the_append"])
@pytest.mark.parametrize("variant", [TB.TB_BUTLER, TB.TB_BUTLER_GROUP], ids=["per_head", "per_group"])
def test_sharded_step_matches_oracle_and_one_context(starts, variant):
    _run(WL, starts, variant)


@pytest.mark.parametrize("variant", [TB.TB_BUTLER, TB.TB_BUTLER_GROUP], ids=["per_head", "per_group"])
def test_sharded_ties_at_the_threshold_split_across_ranks(variant):
    """Candidates repeat 37 keys, so the k-th score is shared by tens of
    tokens on several ranks: lower ranks' copies are taken first, and the
    sets equal the oracle's exactly."""
    got, sel, same = _run(WL, (0, 900, 1800, 2400), variant, periodic=37)
    assert same
    gs = WL.Hq // WL.Hkv
    for (b, h), want in sel.items():
        r = h // gs if variant == TB.TB_BUTLER_GROUP else h
        assert np.array_equal(got[b, r], want), f"b{b} h{h}"


def test_sharded_full_budget_merges_attention_over_every_token():
    wl = WL.with_(keep_pct=100)
    _, sel, _ = _run(wl, (0, 1200))
    for key, idx in sel.items():
        assert idx.size == wl.seq_lens[key[0]]


@pytest.mark.parametrize("variant", [TB.TB_BUTLER, TB.TB_BUTLER_GROUP], ids=["per_head", "per_group"])
def test_sharded_step_with_bf16_kimp(variant):
    _run(WL, (0, 1000, 2100), variant, kimp_dtype="bf16")


def test_sharded_step_with_paged_ranks():
    """Ranks 0 and 2 keep their K/V in shuffled 64-token pages, rank 1 dense:
    the sets still equal the one-context step's bit for bit."""
    _, _, same = _run(WL, (0, 1000, 2100), paged_ranks=(0, 2))
    assert same
