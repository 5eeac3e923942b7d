"""GPU parity of the CUDA hot path (through the C ABI) against the fp64 oracle.

Criteria: K_imp within fp32 dot-product rounding; scores max-rel 1e-5;
selection bit-exact on identical fp32 scores; end-to-end selected sets equal
except for tokens within 1e-4 * max|score| of the k-th score; attention
max-abs 2e-3 (fp32) / 1e-2 relative (bf16)."""
import math

import numpy as np
import pytest
import torch

from oracle import tokenbutler as O
from query_aware_sparse_decode_b200 import synth as S
from query_aware_sparse_decode_b200 import tb as TB

from harness import (assert_close_rows, config_of, kimp_alloc, kimp_rows, make_layer, mask_from_sets, round_up,
                     sets_from_mask, tdtype, tie_band_ok, to_dev)

pytestmark = pytest.mark.gpu

SMALL_BF16 = S.Workload("small_bf16", n_layers=1, B=2, Hq=8, Hkv=2, D=128, d_imp=32, G=1, L=3000, dtype="bf16",
                        keep_pct=30, sink=16, window=64)
SMALL_D64 = S.Workload("small_bf16_d64", n_layers=1, B=1, Hq=8, Hkv=4, D=64, d_imp=16, G=1, L=1500, dtype="bf16",
                       keep_pct=50, sink=4, window=16)
RAGGED = S.Workload("ragged_bf16", n_layers=1, B=4, Hq=8, Hkv=2, D=128, d_imp=32, G=1, L=2300, dtype="bf16",
                    keep_pct=30, sink=16, window=64, lens=(2300, 1, 70, 1027))


def _kimp_tol(K, W):
    return 8e-6 * (np.abs(K) @ np.abs(W)) + 1e-30


# --------------------------------------------------------------------------- a1'
@pytest.mark.parametrize("wl", [S.TINY_F32, SMALL_BF16, SMALL_D64, RAGGED], ids=lambda w: w.name)
def test_project_kimp_matches_fp64(wl):
    ctx = TB.Context(config_of(wl))
    lens = wl.seq_lens
    ld = make_layer(ctx, wl, 0, lens)
    ctx.project_kimp(0, 0, max(lens))
    torch.cuda.synchronize()
    got = kimp_rows(ld.kimp)
    for b, L in enumerate(lens):
        ref = O.project_keys(ld.K[b, :, :L], ld.W)
        assert np.all(np.abs(got[b, :, :L] - ref) <= _kimp_tol(ld.K[b, :, :L], ld.W))
    assert ctx.check_status() == 0


# --------------------------------------------------------------------------- a1
@pytest.mark.parametrize("wl", [S.TINY_F32, SMALL_BF16], ids=lambda w: w.name)
def test_append_writes_rows_and_kimp(wl):
    ctx = TB.Context(config_of(wl))
    lens = wl.seq_lens
    ld = make_layer(ctx, wl, 0, lens)
    k_raw, v_raw = S.kv_new(wl, 0, step=3)
    ctx.append_kv(0, to_dev(k_raw, wl), to_dev(v_raw, wl))
    torch.cuda.synchronize()
    assert ctx.seq_lens(0) == [L + 1 for L in lens]
    k64, v64 = S.widen(k_raw, wl.dtype), S.widen(v_raw, wl.dtype)
    kc = ld.k_cache.float().cpu().numpy()
    vc = ld.v_cache.float().cpu().numpy()
    kimp = kimp_rows(ld.kimp)
    for b, L in enumerate(lens):
        assert np.array_equal(kc[b, :, L], k64[b]) and np.array_equal(vc[b, :, L], v64[b])
        ref = O.project_keys(k64[b], ld.W)
        assert np.all(np.abs(kimp[b, :, L] - ref) <= _kimp_tol(k64[b], ld.W))


@pytest.mark.parametrize("wl", [S.TINY_F32, SMALL_BF16, RAGGED], ids=lambda w: w.name)
def test_decode_step_append_matches_append_kernel(wl):
    """The rows the decode step appends must be the very bits the standalone
    append writes (both go through one device routine)."""
    lens = [max(L - 1, 0) for L in wl.seq_lens]
    outs = []
    for fused in (False, True):
        ctx = TB.Context(config_of(wl))
        ld = make_layer(ctx, wl, 0, lens)
        ctx.project_kimp(0, 0, max(lens))
        k_raw, v_raw = S.kv_new(wl, 0, step=1)
        k_dev, v_dev = to_dev(k_raw, wl), to_dev(v_raw, wl)
        if fused:
            out = torch.empty((wl.B, wl.Hq, wl.D), dtype=tdtype(wl), device="cuda")
            ctx.decode_step(0, k_dev, v_dev, ld.q_dev, ld.q_imp_dev, out)
        else:
            ctx.append_kv(0, k_dev, v_dev)
        torch.cuda.synchronize()
        assert ctx.check_status() == 0
        assert ctx.seq_lens(0) == [L + 1 for L in lens]
        outs.append((ld.k_cache.clone(), ld.v_cache.clone(), ld.kimp.clone()))
    for a, b in zip(*outs):
        assert torch.equal(a.view(torch.int32) if a.dtype == torch.float32 else a.view(torch.int16),
                           b.view(torch.int32) if b.dtype == torch.float32 else b.view(torch.int16))


# --------------------------------------------------------------------------- a2 + a3
@pytest.mark.parametrize("wl", [S.TINY_F32, SMALL_BF16, SMALL_D64, RAGGED,
                                S.TINY_F32.with_(name="tiny_G4_layer6", n_layers=8, G=4)], ids=lambda w: w.name)
def test_score_matches_oracle(wl):
    ctx = TB.Context(config_of(wl))
    lens = wl.seq_lens
    layer = wl.n_layers - 2 if wl.n_layers > 1 else 0
    ld = make_layer(ctx, wl, layer, lens)
    ctx.project_kimp(layer, 0, max(lens))
    scores = torch.full((wl.B, wl.Hq, ctx.cfg.max_len), float("nan"), device="cuda")
    ctx.score(layer, ld.q_imp_dev, scores)
    torch.cuda.synchronize()
    s = scores.cpu().numpy().astype(np.float64)
    gs = wl.Hq // wl.Hkv
    for b, L in enumerate(lens):
        for h in range(wl.Hq):
            ref = O.importance_scores(ld.qhat[b, h], O.project_keys(ld.K[b, h // gs, :L], ld.W))
            if L:
                assert np.max(np.abs(s[b, h, :L] - ref)) <= 1e-5 * np.max(np.abs(ref))
            assert np.all(np.isnan(s[b, h, L:]))      # entries past len are untouched


# --------------------------------------------------------------------------- a4 + a5
def _synthetic_scores(B, rows, Lmax, quant, seed_layer):
    x = S.fill_host(20, seed_layer, 0, B * rows, 0, Lmax, 1, "f32").reshape(B, rows, Lmax)
    if quant:
        x = (np.round(x * quant) / quant).astype(np.float32)   # many exact ties
        x[..., ::7] = np.float32(-0.0)                          # -0.0 vs +0.0 ties
        x[..., 3::11] = np.float32(0.0)
    return x


@pytest.mark.parametrize("case", [
    dict(lens=(512,), keep=50, sink=4, window=16, quant=0),
    dict(lens=(3000, 2999), keep=30, sink=16, window=64, quant=4),
    dict(lens=(4096, 100, 80, 1), keep=50, sink=16, window=64, quant=2),
    dict(lens=(9000,), keep=10, sink=0, window=0, quant=1),
    dict(lens=(777, 0), keep=100, sink=3, window=5, quant=8),
    dict(lens=(20000,), keep=0, sink=16, window=64, quant=0),
    dict(lens=(70000,), keep=30, sink=16, window=64, quant=16),
], ids=lambda c: f"L{c['lens']}-k{c['keep']}-q{c['quant']}")
def test_select_bit_exact_on_identical_scores(case):
    lens, rows = case["lens"], 4
    B = len(lens)
    wl = S.Workload("sel", n_layers=1, B=B, Hq=rows, Hkv=1, D=64, d_imp=16, G=1, L=max(lens), dtype="f32",
                    keep_pct=case["keep"], sink=case["sink"], window=case["window"], plant="none", lens=lens)
    cfg = config_of(wl)
    Lmax = cfg.max_len
    ctx = TB.Context(cfg)
    dummy = torch.zeros((B, 1, Lmax, 64), device="cuda")
    ctx.bind_layer(0, dummy, dummy.clone(), kimp_alloc(B, 1, 16, Lmax),
                   torch.zeros((64, 16), device="cuda"))
    ctx.set_seq_lens(0, lens)
    sc = _synthetic_scores(B, rows, Lmax, case["quant"], len(lens) * 100 + case["keep"])
    cap = max(lens) if max(lens) else 1
    idx = torch.full((B, rows, cap), -1, dtype=torch.int32, device="cuda")
    cnt = torch.full((B, rows), -1, dtype=torch.int32, device="cuda")
    mask = torch.zeros((B, rows, Lmax // 32), dtype=torch.int32, device="cuda")
    ctx.select(0, torch.from_numpy(sc).cuda(), rows, idx=idx, count=cnt, mask=mask)
    torch.cuda.synchronize()
    assert ctx.check_status() == 0
    idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    got_sets = sets_from_mask(mask, lens)
    for b, L in enumerate(lens):
        for r in range(rows):
            ref = O.select_tokens(sc[b, r].astype(np.float64), L, case["keep"], case["sink"], case["window"])
            assert cnt[b, r] == ref.size
            assert np.array_equal(idx[b, r, :ref.size], ref)
            assert np.array_equal(got_sets[b, r], ref)


@pytest.mark.parametrize("case", [
    dict(lens=(512,), keep=50, sink=4, window=16, quant=0, kind=None),
    dict(lens=(3000, 2999), keep=30, sink=16, window=64, quant=4, kind=None),
    dict(lens=(4096, 100, 80, 1), keep=50, sink=16, window=64, quant=2, kind=None),
    dict(lens=(9000,), keep=10, sink=0, window=0, quant=1, kind=None),
    dict(lens=(777, 0), keep=100, sink=3, window=5, quant=8, kind=None),
    dict(lens=(16384, 12000), keep=30, sink=16, window=64, quant=0, kind="three_values"),
    dict(lens=(16000,), keep=50, sink=16, window=64, quant=0, kind="two_digits"),
], ids=lambda c: f"L{c['lens']}-k{c['keep']}-q{c['quant']}-{c['kind']}")
def test_short_row_select_bit_exact_on_identical_scores(case):
    """Short rows without an index list (a cluster of few CTAs per row, some
    CTAs past a short row's end): exact sets and counts on identical fp32 scores,
    including quantised scores (-0.0 against +0.0) and rows where ties at
    the threshold decide most of the budget (an ordered quota)."""
    lens, rows = case["lens"], 4
    B = len(lens)
    wl = S.Workload("selr", n_layers=1, B=B, Hq=rows, Hkv=1, D=64, d_imp=16, G=1, L=max(lens), dtype="f32",
                    keep_pct=case["keep"], sink=case["sink"], window=case["window"], plant="none", lens=lens)
    cfg = config_of(wl)
    Lmax = cfg.max_len
    ctx = TB.Context(cfg)
    dummy = torch.zeros((B, 1, Lmax, 64), device="cuda")
    ctx.bind_layer(0, dummy, dummy.clone(), kimp_alloc(B, 1, 16, Lmax), torch.zeros((64, 16), device="cuda"))
    ctx.set_seq_lens(0, lens)
    if case["kind"] is None:
        sc = _synthetic_scores(B, rows, Lmax, case["quant"], len(lens) * 100 + case["keep"] + 7)
    else:
        sc = np.zeros((B, rows, Lmax), np.float32)
        for b, L in enumerate(lens):
            for r in range(rows):
                sc[b, r, :L] = _crowded_scores(case["kind"], L, 31 + 4 * b + r)
    cnt = torch.full((B, rows), -1, dtype=torch.int32, device="cuda")
    mask = torch.zeros((B, rows, Lmax // 32), dtype=torch.int32, device="cuda")
    ctx.select(0, torch.from_numpy(sc).cuda(), rows, count=cnt, mask=mask)
    torch.cuda.synchronize()
    assert ctx.check_status() == 0
    cnt = cnt.cpu().numpy()
    got_sets = sets_from_mask(mask, lens)
    for b, L in enumerate(lens):
        for r in range(rows):
            ref = O.select_tokens(sc[b, r].astype(np.float64), L, case["keep"], case["sink"], case["window"])
            assert cnt[b, r] == ref.size, f"b{b} r{r}"
            assert np.array_equal(got_sets[b, r], ref), f"b{b} r{r}"


def _crowded_scores(kind, L, seed):
    u = S.fill_host(21, seed, 0, 1, 0, L, 1, "f32").reshape(L).astype(np.float64)
    u = (u - u.min()) / (u.max() - u.min() + 1e-12)          # in [0, 1)
    if kind == "one_binade":      # [1, 2): the first digit has 4 occupied bins
        x = 1.0 + u
    elif kind == "two_digits":    # [1, 1 + 2**-12): the first two digits leave 2 bins
        x = 1.0 + np.floor(u * 2048) * 2.0 ** -23
    else:                         # three values: ties decide almost the whole budget
        x = np.floor(u * 3) - 1.0
    return x.astype(np.float32)


@pytest.mark.parametrize("kind", ["one_binade", "two_digits", "three_values"])
@pytest.mark.parametrize("keep", [10, 50])
def test_single_row_select_on_crowded_bins(kind, keep):
    """One shared row per sequence (the soft-voting shape) whose top digits
    leave far more keys in the threshold bin than a CTA's shared list
    holds: the re-read path must still give exactly the oracle's set
    (identical fp32 scores), with ties split across the cluster's CTAs."""
    lens = (200000, 150001)
    B = len(lens)
    wl = S.Workload("sel1", n_layers=1, B=B, Hq=1, Hkv=1, D=64, d_imp=16, G=1, L=max(lens), dtype="f32",
                    keep_pct=keep, sink=16, window=64, plant="none", lens=lens)
    cfg = config_of(wl)
    Lmax = cfg.max_len
    ctx = TB.Context(cfg)
    dummy = torch.zeros((B, 1, Lmax, 64), device="cuda")
    ctx.bind_layer(0, dummy, dummy.clone(), kimp_alloc(B, 1, 16, Lmax), torch.zeros((64, 16), device="cuda"))
    ctx.set_seq_lens(0, lens)
    sc = np.zeros((B, Lmax), np.float32)
    for b, L in enumerate(lens):
        sc[b, :L] = _crowded_scores(kind, L, 7 + b)
    idx = torch.full((B, 1, max(lens)), -1, dtype=torch.int32, device="cuda")
    cnt = torch.full((B, 1), -1, dtype=torch.int32, device="cuda")
    mask = torch.zeros((B, 1, Lmax // 32), dtype=torch.int32, device="cuda")
    ctx.select(0, torch.from_numpy(sc).cuda(), 1, idx=idx, count=cnt, mask=mask)
    torch.cuda.synchronize()
    assert ctx.check_status() == 0
    idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    got_sets = sets_from_mask(mask, lens)
    for b, L in enumerate(lens):
        ref = O.select_tokens(sc[b].astype(np.float64), L, keep, wl.sink, wl.window)
        assert cnt[b, 0] == ref.size
        assert np.array_equal(idx[b, 0, :ref.size], ref)
        assert np.array_equal(got_sets[b, 0], ref)


@pytest.mark.parametrize("kind,lens", [(None, (70000, 69001, 65537, 70000)),
                                       ("two_digits", (70000, 69001, 65537, 70000)),
                                       ("three_values", (70000, 69001, 65537, 70000)),
                                       (None, (70000, 1000, 1, 65537))],
                         ids=["random", "two_digits", "three_values", "ragged"])
def test_select_clusters_of_two_exchange_digit_two_in_shared_memory(kind, lens):
    """128 rows just over 65536 tokens: clusters of two CTAs (512 threads),
    the shape whose digit-2 histograms are summed through distributed shared
    memory.  Exact sets and counts on identical fp32 scores, including rows
    whose top two digits leave two bins (the exchanged histogram decides),
    rows where ties at the threshold take most of the budget, and short rows
    whose second CTA holds no token."""
    B, Hq, Hkv = len(lens), 32, 8
    keep = 30
    wl = S.Workload("sel_pair", n_layers=1, B=B, Hq=Hq, Hkv=Hkv, D=64, d_imp=16, G=1, L=max(lens), dtype="f32",
                    keep_pct=keep, sink=16, window=64, plant="none", lens=lens)
    cfg = config_of(wl)
    Lmax = cfg.max_len
    ctx = TB.Context(cfg)
    dummy = torch.zeros((B, Hkv, Lmax, 64), device="cuda")
    ctx.bind_layer(0, dummy, dummy.clone(), kimp_alloc(B, Hkv, 16, Lmax), torch.zeros((64, 16), device="cuda"))
    ctx.set_seq_lens(0, lens)
    if kind is None:
        sc = _synthetic_scores(B, Hq, Lmax, 0, 907)
    else:
        sc = np.zeros((B, Hq, Lmax), np.float32)
        for b, L in enumerate(lens):
            for r in range(Hq):
                sc[b, r, :L] = _crowded_scores(kind, L, 300 + 32 * b + r)
    cnt = torch.full((B, Hq), -1, dtype=torch.int32, device="cuda")
    mask = torch.zeros((B, Hq, Lmax // 32), dtype=torch.int32, device="cuda")
    ctx.select(0, torch.from_numpy(sc).cuda(), Hq, count=cnt, mask=mask)
    torch.cuda.synchronize()
    assert ctx.check_status() == 0
    cnt = cnt.cpu().numpy()
    got_sets = sets_from_mask(mask, lens)
    for b, L in enumerate(lens):
        for r in range(Hq):
            ref = O.select_tokens(sc[b, r].astype(np.float64), L, keep, wl.sink, wl.window)
            assert cnt[b, r] == ref.size, f"b{b} r{r}"
            assert np.array_equal(got_sets[b, r], ref), f"b{b} r{r}"


@pytest.mark.parametrize("kind", ["two_digits", "three_values"])
def test_decode_step_on_controlled_scores_in_clusters_of_two(kind):
    """The fused decode step (score kernel with its first-digit histogram,
    clusters of two CTAs exchanging digit 2 in shared memory, the scores
    dropped from L2 after the selection) on scores it computes exactly: the
    importance query is the first unit vector and K_imp holds crowded values
    in its first dimension (W_K = 0, so the appended token scores 0).  The
    step's masks must be the oracle's sets exactly."""
    lens0 = (69999, 69000, 65536, 69999)
    B, Hq, Hkv, D, dimp = len(lens0), 32, 8, 64, 16
    keep = 30
    wl = S.Workload("step_ctl", n_layers=1, B=B, Hq=Hq, Hkv=Hkv, D=D, d_imp=dimp, G=1, L=max(lens0) + 1, dtype="f32",
                    keep_pct=keep, sink=16, window=64, plant="none", lens=tuple(L + 1 for L in lens0))
    cfg = config_of(wl)
    Lmax = cfg.max_len
    ctx = TB.Context(cfg)
    k_cache = torch.zeros((B, Hkv, Lmax, D), device="cuda")
    v_cache = torch.zeros_like(k_cache)
    kimp = kimp_alloc(B, Hkv, dimp, Lmax)
    vals = np.zeros((B, Hkv, Lmax), np.float32)
    for b, L in enumerate(lens0):
        for g in range(Hkv):
            vals[b, g, :L] = _crowded_scores(kind, L, 500 + 8 * b + g)
    kimp[:, :, :, 0, :] = torch.from_numpy(vals.reshape(B, Hkv, Lmax // 256, 256)).cuda()
    ctx.bind_layer(0, k_cache, v_cache, kimp, torch.zeros((D, dimp), device="cuda"))
    ctx.set_seq_lens(0, list(lens0))
    q_imp = torch.zeros((B * Hq, 1, dimp), device="cuda")
    q_imp[:, 0, 0] = 1.0
    q = torch.from_numpy(S.fill_host(22, 3, 0, B * Hq, 0, D, 1, "f32").reshape(B, Hq, D)).cuda()
    zero_row = torch.zeros((B, Hkv, D), device="cuda")
    out = torch.empty((B, Hq, D), device="cuda")
    ctx.decode_step(0, zero_row, zero_row.clone(), q, q_imp, out)
    masks = ctx.step_masks(Hq)
    torch.cuda.synchronize()
    assert ctx.check_status() == 0
    lens = ctx.seq_lens(0)
    got_sets = sets_from_mask(masks, lens)
    for b, L in enumerate(lens):
        for h in range(Hq):
            row = np.zeros(L, np.float64)
            row[:L - 1] = vals[b, O.kv_head_of(h, Hq, Hkv), :L - 1]
            ref = O.select_tokens(row, L, keep, wl.sink, wl.window)
            assert np.array_equal(got_sets[b, h], ref), f"b{b} h{h}"


@pytest.mark.parametrize("kind", [None, "two_digits"])
def test_select_rows_beyond_one_cluster(kind):
    """Rows longer than a cluster of 16 CTAs of 65536 tokens (1048576) take
    the many-CTA scatter + resolve path: the same exact sets, counts and
    index lists on identical fp32 scores (one shared row per sequence, as in
    soft voting, and quantised per-head rows)."""
    lens = (1100000, 1048577)
    B = len(lens)
    rows = 1 if kind else 2
    keep = 30
    wl = S.Workload("sel_long", n_layers=1, B=B, Hq=rows, Hkv=1, D=64, d_imp=16, G=1, L=max(lens), dtype="f32",
                    keep_pct=keep, sink=16, window=64, plant="none", lens=lens)
    cfg = config_of(wl)
    Lmax = cfg.max_len
    ctx = TB.Context(cfg)
    dummy = torch.zeros((B, 1, Lmax, 64), device="cuda")
    ctx.bind_layer(0, dummy, dummy.clone(), kimp_alloc(B, 1, 16, Lmax), torch.zeros((64, 16), device="cuda"))
    ctx.set_seq_lens(0, lens)
    if kind is None:
        sc = _synthetic_scores(B, rows, Lmax, 4, 901)
    else:
        sc = np.zeros((B, rows, Lmax), np.float32)
        for b, L in enumerate(lens):
            sc[b, 0, :L] = _crowded_scores(kind, L, 77 + b)
    idx = torch.full((B, rows, max(lens)), -1, dtype=torch.int32, device="cuda")
    cnt = torch.full((B, rows), -1, dtype=torch.int32, device="cuda")
    mask = torch.zeros((B, rows, Lmax // 32), dtype=torch.int32, device="cuda")
    ctx.select(0, torch.from_numpy(sc).cuda(), rows, idx=idx, count=cnt, mask=mask)
    torch.cuda.synchronize()
    assert ctx.check_status() == 0
    idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    got_sets = sets_from_mask(mask, lens)
    for b, L in enumerate(lens):
        for r in range(rows):
            ref = O.select_tokens(sc[b, r].astype(np.float64), L, keep, wl.sink, wl.window)
            assert cnt[b, r] == ref.size
            assert np.array_equal(idx[b, r, :ref.size], ref)
            assert np.array_equal(got_sets[b, r], ref)


# --------------------------------------------------------------------------- a6
@pytest.mark.parametrize("wl", [S.TINY_F32, SMALL_BF16, SMALL_D64, RAGGED], ids=lambda w: w.name)
def test_sparse_attn_on_oracle_sets(wl):
    ctx = TB.Context(config_of(wl))
    lens = wl.seq_lens
    ld = make_layer(ctx, wl, 0, lens)
    gs = wl.Hq // wl.Hkv
    scale = 1.0 / math.sqrt(wl.D)
    sets = {}
    for b, L in enumerate(lens):
        for h in range(wl.Hq):
            s = O.importance_scores(ld.qhat[b, h], O.project_keys(ld.K[b, h // gs, :L], ld.W))
            sets[b, h] = O.select_tokens(s, L, wl.keep_pct, wl.sink, wl.window)
    mask = mask_from_sets(sets, wl.B, wl.Hq, ctx.cfg.max_len)
    out = torch.empty((wl.B, wl.Hq, wl.D), dtype=tdtype(wl), device="cuda")
    lse = torch.empty((wl.B, wl.Hq), device="cuda")
    ctx.sparse_attn(0, ld.q_dev, mask, TB.TB_MASK_PER_HEAD, out, lse)
    out_d = torch.empty_like(out)
    lse_d = torch.empty_like(lse)
    ctx.sparse_attn(0, ld.q_dev, None, TB.TB_MASK_DENSE, out_d, lse_d)
    torch.cuda.synchronize()
    o, l = out.float().cpu().numpy(), lse.cpu().numpy()
    od, ldn = out_d.float().cpu().numpy(), lse_d.cpu().numpy()
    for b, L in enumerate(lens):
        for h in range(wl.Hq):
            ref, ref_lse = O.attend(ld.q[b, h], ld.K[b, h // gs, :L], ld.V[b, h // gs, :L], sets[b, h], scale)
            assert_close_rows(o[b, h][None], ref[None], wl.dtype, f"sparse b{b} h{h}")
            assert abs(l[b, h] - ref_lse) <= 1e-3 * max(1.0, abs(ref_lse))
            refd, refd_lse = O.attend(ld.q[b, h], ld.K[b, h // gs, :L], ld.V[b, h // gs, :L], np.arange(L), scale)
            assert_close_rows(od[b, h][None], refd[None], wl.dtype, f"dense b{b} h{h}")
            assert abs(ldn[b, h] - refd_lse) <= 1e-3 * max(1.0, abs(refd_lse))


def test_sparse_attn_on_index_lists():
    """tb_sparse_attn_idx (the sets as the ascending index lists and counts
    that tb_select writes) equals tb_sparse_attn on the same sets' mask bit
    for bit and the oracle's attention; out-of-range indices are skipped and
    flagged."""
    wl = SMALL_BF16
    ctx = TB.Context(config_of(wl))
    ld = make_layer(ctx, wl, 0, wl.seq_lens)
    gs = wl.Hq // wl.Hkv
    sets = {}
    for b, L in enumerate(wl.seq_lens):
        for h in range(wl.Hq):
            s = O.importance_scores(ld.qhat[b, h], O.project_keys(ld.K[b, h // gs, :L], ld.W))
            sets[b, h] = O.select_tokens(s, L, wl.keep_pct, wl.sink, wl.window)
    cap = max(len(v) for v in sets.values()) + 3
    idx = np.full((wl.B, wl.Hq, cap), -1, np.int32)
    cnt = np.zeros((wl.B, wl.Hq), np.int32)
    for (b, h), v in sets.items():
        idx[b, h, :len(v)] = v
        cnt[b, h] = len(v)
    mask = mask_from_sets(sets, wl.B, wl.Hq, ctx.cfg.max_len)
    outs = []
    for use_idx in (True, False):
        out = torch.empty((wl.B, wl.Hq, wl.D), dtype=tdtype(wl), device="cuda")
        lse = torch.empty((wl.B, wl.Hq), device="cuda")
        if use_idx:
            ctx.sparse_attn_idx(0, ld.q_dev, torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda(), out, lse)
        else:
            ctx.sparse_attn(0, ld.q_dev, mask, TB.TB_MASK_PER_HEAD, out, lse)
        outs.append((out, lse))
    torch.cuda.synchronize()
    assert ctx.check_status() == 0
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
    o = outs[0][0].float().cpu().numpy()
    scale = 1.0 / math.sqrt(wl.D)
    for (b, h), v in sets.items():
        L = wl.seq_lens[b]
        want, _ = O.attend(ld.q[b, h], ld.K[b, h // gs, :L], ld.V[b, h // gs, :L], v, scale)
        assert_close_rows(o[b, h][None], want[None], wl.dtype, f"b{b} h{h}")
    # an index past the length: skipped and flagged
    idx[0, 0, 0] = wl.seq_lens[0] + 5
    out = torch.empty((wl.B, wl.Hq, wl.D), dtype=tdtype(wl), device="cuda")
    ctx.sparse_attn_idx(0, ld.q_dev, torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda(), out)
    torch.cuda.synchronize()
    assert ctx.check_status() == 0x1  # TB_DEV_ERR_INDEX


def test_sparse_attn_empty_set_and_single_token():
    wl = SMALL_BF16.with_(B=1)
    ctx = TB.Context(config_of(wl))
    ld = make_layer(ctx, wl, 0, (wl.L,))
    sets = {(0, h): (np.array([], np.int64) if h % 2 == 0 else np.array([1234])) for h in range(wl.Hq)}
    out = torch.empty((1, wl.Hq, wl.D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((1, wl.Hq), device="cuda")
    ctx.sparse_attn(0, ld.q_dev, mask_from_sets(sets, 1, wl.Hq, ctx.cfg.max_len), TB.TB_MASK_PER_HEAD, out, lse)
    torch.cuda.synchronize()
    o, l = out.float().cpu().numpy(), lse.cpu().numpy()
    for h in range(wl.Hq):
        if h % 2 == 0:
            assert np.all(o[0, h] == 0) and l[0, h] == -np.inf
        else:
            assert np.array_equal(o[0, h], ld.V[0, h // 4, 1234])   # bf16 value row, exact


# --------------------------------------------------------------------------- a1..a6 end to end
def _decode_e2e(wl, layer=0):
    cfg = config_of(wl)
    ctx = TB.Context(cfg)
    lens0 = [L - 1 for L in wl.seq_lens]
    ld = make_layer(ctx, wl, layer, lens0)
    ctx.project_kimp(layer, 0, max(lens0))
    k_raw, v_raw = S.kv_new(wl, layer)
    k_dev, v_dev = to_dev(k_raw, wl), to_dev(v_raw, wl)
    out = torch.empty((wl.B, wl.Hq, wl.D), dtype=tdtype(wl), device="cuda")
    ctx.decode_step(layer, k_dev, v_dev, ld.q_dev, ld.q_imp_dev, out)
    # the same step through the separate calls, keeping the selection
    lens = ctx.seq_lens(layer)
    scores = torch.empty((wl.B, wl.Hq, cfg.max_len), device="cuda")
    mask = torch.zeros((wl.B, wl.Hq, cfg.max_len // 32), dtype=torch.int32, device="cuda")
    out2 = torch.empty_like(out)
    dense = layer in wl.dense_layers or wl.keep_pct == 100
    if dense:
        ctx.sparse_attn(layer, ld.q_dev, None, TB.TB_MASK_DENSE, out2)
    else:
        ctx.score(layer, ld.q_imp_dev, scores)
        ctx.select(layer, scores, wl.Hq, mask=mask)
        ctx.sparse_attn(layer, ld.q_dev, mask, TB.TB_MASK_PER_HEAD, out2)
    torch.cuda.synchronize()
    assert ctx.check_status() == 0
    assert torch.equal(out, out2)
    # the step's own append: K and V rows exact, K_imp row within fp32 rounding
    k64, v64 = S.widen(k_raw, wl.dtype), S.widen(v_raw, wl.dtype)
    kc, vc = ld.k_cache.float().cpu().numpy(), ld.v_cache.float().cpu().numpy()
    kimp_now = kimp_rows(ld.kimp)
    for b, L in enumerate(lens):
        assert np.array_equal(kc[b, :, L - 1], k64[b]) and np.array_equal(vc[b, :, L - 1], v64[b])
        assert np.all(np.abs(kimp_now[b, :, L - 1] - O.project_keys(k64[b], ld.W)) <= _kimp_tol(k64[b], ld.W))
    # oracle on the full cache (prefill rows + the appended token)
    K = np.concatenate([ld.K, np.zeros((wl.B, wl.Hkv, 1, wl.D))], axis=2)
    V = np.concatenate([ld.V, np.zeros((wl.B, wl.Hkv, 1, wl.D))], axis=2)
    for b, L in enumerate(lens):
        K[b, :, L - 1], V[b, :, L - 1] = k64[b], v64[b]
    sel, ref, _, sc = O.decode_layer(ld.q, K, V, ld.W, ld.qimp, layer, wl.G, lens, wl.keep_pct, wl.sink,
                                     wl.window, dense=dense)
    o = out.float().cpu().numpy()
    got_sets = None if dense else sets_from_mask(mask, lens)
    scale = 1.0 / math.sqrt(wl.D)
    mism = 0
    for b in range(wl.B):
        for h in range(wl.Hq):
            want = ref[b, h]
            if not dense:
                assert tie_band_ok(got_sets[b, h], sel[b, h], sc[b, h], lens[b], wl.keep_pct, wl.sink, wl.window)
                if not np.array_equal(got_sets[b, h], sel[b, h]):
                    mism += 1
                    # the sets differ only inside the tie band: the output given
                    # a set is unique, so compare with the oracle on the GPU's set
                    g = O.kv_head_of(h, wl.Hq, wl.Hkv)
                    want, _ = O.attend(ld.q[b, h], K[b, g, :lens[b]], V[b, g, :lens[b]], got_sets[b, h], scale)
            assert_close_rows(o[b, h][None], want[None], wl.dtype, f"b{b} h{h}")
    assert mism <= max(1, wl.B * wl.Hq // 20)
    return ctx, sel, got_sets


def _decode_e2e_group(wl, layer=0):
    """The per-KV-group option: one set per (b, g) from the group's summed
    scores, attended by every head of the group."""
    cfg = config_of(wl, variant=TB.TB_BUTLER_GROUP)
    ctx = TB.Context(cfg)
    lens0 = [L - 1 for L in wl.seq_lens]
    ld = make_layer(ctx, wl, layer, lens0)
    ctx.project_kimp(layer, 0, max(lens0))
    k_raw, v_raw = S.kv_new(wl, layer)
    out = torch.empty((wl.B, wl.Hq, wl.D), dtype=tdtype(wl), device="cuda")
    ctx.decode_step(layer, to_dev(k_raw, wl), to_dev(v_raw, wl), ld.q_dev, ld.q_imp_dev, out)
    lens = ctx.seq_lens(layer)
    scores = torch.full((wl.B, wl.Hkv, cfg.max_len), float("nan"), device="cuda")
    mask = torch.zeros((wl.B, wl.Hkv, cfg.max_len // 32), dtype=torch.int32, device="cuda")
    out2 = torch.empty_like(out)
    ctx.score(layer, ld.q_imp_dev, scores)
    ctx.select(layer, scores, wl.Hkv, mask=mask)
    ctx.sparse_attn(layer, ld.q_dev, mask, TB.TB_MASK_GROUP, out2)
    torch.cuda.synchronize()
    assert ctx.check_status() == 0
    assert torch.equal(out, out2)
    K = np.concatenate([ld.K, np.zeros((wl.B, wl.Hkv, 1, wl.D))], axis=2)
    V = np.concatenate([ld.V, np.zeros((wl.B, wl.Hkv, 1, wl.D))], axis=2)
    k64, v64 = S.widen(k_raw, wl.dtype), S.widen(v_raw, wl.dtype)
    for b, L in enumerate(lens):
        K[b, :, L - 1], V[b, :, L - 1] = k64[b], v64[b]
    sel, ref, _, sc = O.decode_layer(ld.q, K, V, ld.W, ld.qimp, layer, wl.G, lens, wl.keep_pct, wl.sink,
                                     wl.window, dense=False, group=True)
    got_sets = sets_from_mask(mask, lens)
    s_gpu = scores.cpu().numpy().astype(np.float64)
    o = out.float().cpu().numpy()
    gs = wl.Hq // wl.Hkv
    scale = 1.0 / math.sqrt(wl.D)
    mism = 0
    for b, L in enumerate(lens):
        for g in range(wl.Hkv):
            lead = g * gs
            if L:
                assert np.max(np.abs(s_gpu[b, g, :L] - sc[b, lead])) <= 1e-5 * np.max(np.abs(sc[b, lead]))
            gset = got_sets[b, g]
            assert tie_band_ok(gset, sel[b, lead], sc[b, lead], L, wl.keep_pct, wl.sink, wl.window)
            if not np.array_equal(gset, sel[b, lead]):
                mism += 1
            for h in range(lead, lead + gs):
                want, _ = O.attend(ld.q[b, h], K[b, g, :L], V[b, g, :L], gset, scale)
                assert_close_rows(o[b, h][None], want[None], wl.dtype, f"group b{b} h{h}")
    assert mism <= max(1, wl.B * wl.Hkv // 10)


@pytest.mark.parametrize("wl", [S.TINY_F32, SMALL_BF16, SMALL_D64, RAGGED], ids=lambda w: w.name)
def test_group_selection_decode_step(wl):
    _decode_e2e_group(wl)


@pytest.mark.parametrize("wl", [S.TINY_F32, SMALL_BF16, SMALL_D64, RAGGED], ids=lambda w: w.name)
def test_decode_step_end_to_end(wl):
    _decode_e2e(wl)


def test_planted_tokens_selected_tiny_f32():
    wl = S.TINY_F32
    _, _, got = _decode_e2e(wl)
    planted = set(S.plant_list8(wl, 0).tolist())
    for h in range(wl.Hq):
        assert planted <= set(got[0, h].tolist())
        assert got[0, h].size == 256 + 4 + 16


def test_full_budget_equals_dense():
    _decode_e2e(SMALL_BF16.with_(keep_pct=100))
    _decode_e2e(SMALL_BF16.with_(dense_layers=(0,)))


@pytest.mark.parametrize("keep", [50, 100])
def test_llama8b_L32768_end_to_end(keep):
    _decode_e2e(S.LLAMA8B_L32K.with_(keep_pct=keep))


def test_attention_on_an_empty_sequence_and_repeated_calls():
    """A sequence with no cached token yields out = 0 and lse = -inf; the
    split tickets reset themselves, so back-to-back calls agree."""
    wl = SMALL_BF16.with_(lens=(1500, 0))
    ctx = TB.Context(config_of(wl))
    ld = make_layer(ctx, wl, 0, wl.seq_lens)
    outs = []
    for _ in range(3):
        out = torch.full((wl.B, wl.Hq, wl.D), 7.0, dtype=torch.bfloat16, device="cuda")
        lse = torch.zeros((wl.B, wl.Hq), device="cuda")
        ctx.sparse_attn(0, ld.q_dev, None, TB.TB_MASK_DENSE, out, lse)
        outs.append((out, lse))
    torch.cuda.synchronize()
    for out, lse in outs:
        assert torch.all(out[1] == 0) and torch.all(torch.isneginf(lse[1]))
        assert torch.equal(out, outs[0][0]) and torch.equal(lse, outs[0][1])
    ref, ref_lse = O.attend(ld.q[0, 0], ld.K[0, 0, :1500], ld.V[0, 0, :1500], np.arange(1500), 1 / math.sqrt(wl.D))
    assert_close_rows(outs[0][0][0, 0].float().cpu().numpy()[None], ref[None], "bf16")
