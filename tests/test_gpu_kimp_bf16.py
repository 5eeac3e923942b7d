"""The bf16 K_imp cache option against the oracle's bf16 storage (the exact
K W_K rounded once to the nearest bfloat16).

Every producer of K_imp (the tensor-core projection of dense caches, the
FMA projection of paged caches, the decode append) rounds an fp32 dot
product, which may sit on the other side of a rounding midpoint than the
exact value: those elements may hold the neighbouring bfloat16 value
(harness.bf16_kimp_bounds), and scores over them may move by that step
times |q_j| (harness.bf16_score_slack).  Everything else is compared as for
the fp32 cache: scores within fp32 accumulation, sets within the tie band,
outputs against the oracle's attention over the GPU's set."""
import math

import numpy as np
import pytest
import torch

from oracle import tokenbutler as O
from query_aware_sparse_decode_b200 import synth as S
from query_aware_sparse_decode_b200 import tb as TB

from harness import (assert_close_rows, bf16_kimp_ok, bf16_score_slack, config_of, kimp_rows, make_layer,
                     paged_copy, round_up, sets_from_mask, tdtype, tie_band_ok, to_dev)

pytestmark = pytest.mark.gpu

WL = S.Workload("kimp16_bf16", n_layers=1, B=2, Hq=8, Hkv=2, D=128, d_imp=32, G=1, L=3000, dtype="bf16",
                keep_pct=30, sink=16, window=64, lens=(3000, 1777))
WL_D64 = S.Workload("kimp16_d64", n_layers=1, B=1, Hq=8, Hkv=4, D=64, d_imp=16, G=1, L=1500, dtype="bf16",
                    keep_pct=50, sink=4, window=16)
WL_GS8 = S.Workload("kimp16_gs8", n_layers=1, B=2, Hq=16, Hkv=2, D=128, d_imp=32, G=1, L=2600, dtype="bf16",
                    keep_pct=10, sink=16, window=64, lens=(2600, 2049))
PAGE = 64


def _ctx(wl, variant=TB.TB_BUTLER, max_len=None):
    return TB.Context(config_of(wl, max_len=max_len, variant=variant, kimp_dtype="bf16"))


def test_bf16_kimp_needs_bf16_caches_and_a_bf16_tensor():
    with pytest.raises(TB.TBError):
        TB.Context(config_of(S.TINY_F32, kimp_dtype="bf16"))
    ctx = _ctx(WL)
    cfg = ctx.cfg
    k = torch.zeros((WL.B, WL.Hkv, cfg.max_len, WL.D), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((WL.D, WL.d_imp), dtype=torch.bfloat16, device="cuda")
    fp32_kimp = torch.zeros((WL.B, WL.Hkv, cfg.max_len // 256, WL.d_imp, 256), device="cuda")
    with pytest.raises(TypeError):
        ctx.bind_layer(0, k, k.clone(), fp32_kimp, w)
    assert TB.kimp_cache(cfg).dtype == torch.bfloat16


@pytest.mark.parametrize("layout", ["dense", "paged"])
@pytest.mark.parametrize("wl", [WL, WL_D64], ids=lambda w: w.name)
def test_bf16_kimp_projection_and_append(wl, layout):
    """Prefill rows projected (tensor cores on dense caches, FMA on paged
    ones), then one appended row per sequence."""
    ctx = _ctx(wl)
    lens0 = [L - 1 for L in wl.seq_lens]
    ld = make_layer(ctx, wl, 0, lens0)
    kimp = ld.kimp
    if layout == "paged":
        kpool, vpool, table = paged_copy(ld, wl, ctx.cfg.max_len, PAGE, 3)
        kimp = TB.kimp_cache(ctx.cfg)
        ctx.bind_layer_paged(0, kpool, vpool, table, kimp, ld.w_k)
        ctx.set_seq_lens(0, lens0)
    ctx.project_kimp(0, 0, max(lens0))
    k_raw, v_raw = S.kv_new(wl, 0)
    ctx.append_kv(0, to_dev(k_raw, wl), to_dev(v_raw, wl))
    torch.cuda.synchronize()
    assert ctx.check_status() == 0
    got = kimp_rows(kimp)
    k64 = S.widen(k_raw, wl.dtype)
    for b, L0 in enumerate(lens0):
        K = np.concatenate([ld.K[b, :, :L0], k64[b][:, None, :]], axis=1)   # [Hkv][L0 + 1][D]
        assert bf16_kimp_ok(got[b, :, :L0 + 1], K, ld.W), f"b{b}"
        # the bulk is the oracle's own rounding
        assert np.mean(got[b, :, :L0 + 1] == O.project_keys(K, ld.W, "bf16")) > 0.99


@pytest.mark.parametrize("wl", [WL, WL_D64, WL_GS8], ids=lambda w: w.name)
def test_bf16_kimp_scores(wl):
    """Scores over the stored bf16 K_imp: fp32 accumulation of exact products."""
    ctx = _ctx(wl)
    lens = wl.seq_lens
    ld = make_layer(ctx, wl, 0, lens)
    ctx.project_kimp(0, 0, max(lens))
    scores = torch.full((wl.B, wl.Hq, ctx.cfg.max_len), float("nan"), device="cuda")
    ctx.score(0, ld.q_imp_dev, scores)
    torch.cuda.synchronize()
    assert ctx.check_status() == 0
    sc = scores.cpu().numpy().astype(np.float64)
    gs = wl.Hq // wl.Hkv
    for b, L in enumerate(lens):
        for h in range(wl.Hq):
            K = ld.K[b, h // gs, :L]
            kb = O.project_keys(K, ld.W, "bf16")
            ref = O.importance_scores(ld.qhat[b, h], kb)
            tol = 4e-6 * (np.abs(kb) @ np.abs(ld.qhat[b, h])) + bf16_score_slack(np.abs(ld.qhat[b, h]), K, ld.W)
            assert np.all(np.abs(sc[b, h, :L] - ref) <= tol + 1e-30), f"b{b} h{h}"
            assert np.isnan(sc[b, h, L:]).all()     # entries past the length untouched


def _decode(wl, group):
    variant = TB.TB_BUTLER_GROUP if group else TB.TB_BUTLER
    ctx = _ctx(wl, variant)
    lens0 = [L - 1 for L in wl.seq_lens]
    ld = make_layer(ctx, wl, 0, lens0)
    ctx.project_kimp(0, 0, max(lens0))
    k_raw, v_raw = S.kv_new(wl, 0)
    out = torch.empty((wl.B, wl.Hq, wl.D), dtype=tdtype(wl), device="cuda")
    ctx.decode_step(0, to_dev(k_raw, wl), to_dev(v_raw, wl), ld.q_dev, ld.q_imp_dev, out)
    rows = wl.Hkv if group else wl.Hq
    masks = ctx.step_masks(rows)
    torch.cuda.synchronize()
    assert ctx.check_status() == 0
    lens = ctx.seq_lens(0)
    k64, v64 = S.widen(k_raw, wl.dtype), S.widen(v_raw, wl.dtype)
    K = np.concatenate([ld.K, np.zeros((wl.B, wl.Hkv, 1, wl.D))], axis=2)
    V = np.concatenate([ld.V, np.zeros((wl.B, wl.Hkv, 1, wl.D))], axis=2)
    for b, L in enumerate(lens):
        K[b, :, L - 1], V[b, :, L - 1] = k64[b], v64[b]
    sel, ref, _, sc = O.decode_layer(ld.q, K, V, ld.W, ld.qimp, 0, wl.G, lens, wl.keep_pct, wl.sink, wl.window,
                                     dense=False, group=group, kimp_storage="bf16")
    got = sets_from_mask(masks, lens)
    o = out.float().cpu().numpy()
    gs = wl.Hq // wl.Hkv
    mism = 0
    for b, L in enumerate(lens):
        for h in range(wl.Hq):
            g = h // gs
            r = g if group else h
            qabs = np.abs(ld.qhat[b, g * gs:(g + 1) * gs]).sum(axis=0) if group else np.abs(ld.qhat[b, h])
            slack = bf16_score_slack(qabs, K[b, g, :L], ld.W)
            assert tie_band_ok(got[b, r], sel[b, h], sc[b, h], L, wl.keep_pct, wl.sink, wl.window, slack), \
                f"b{b} h{h}"
            want = ref[b, h]
            if not np.array_equal(got[b, r], sel[b, h]):
                mism += 1
                want, _ = O.attend(ld.q[b, h], K[b, g, :L], V[b, g, :L], got[b, r], 1.0 / math.sqrt(wl.D))
            assert_close_rows(o[b, h][None], want[None], wl.dtype, f"b{b} h{h}")
    assert mism <= max(1, wl.B * wl.Hq // 20)


@pytest.mark.parametrize("group", [False, True], ids=["per_head", "per_group"])
@pytest.mark.parametrize("wl", [WL, WL_D64, WL_GS8], ids=lambda w: w.name)
def test_bf16_kimp_decode_step(wl, group):
    _decode(wl, group)


PF = S.Workload("kimp16_prefill", n_layers=8, B=2, Hq=8, Hkv=2, D=128, d_imp=32, G=4, L=3000, dtype="bf16",
                keep_pct=50, sink=16, window=64, dense_layers=(0,))


def test_bf16_kimp_prefill_rows():
    """Prefill rows over a bf16 K_imp: TF32 tiles need no split (bf16 is
    exact in TF32)."""
    wl, layer, row0, nrows = PF, 5, 2936, 64
    ctx = _ctx(wl, max_len=round_up(wl.L, 256))
    ld = make_layer(ctx, wl, layer, [wl.L] * wl.B)
    ctx.project_kimp(layer, 0, wl.L)
    prod = O.producer_of(layer, wl.G)
    qrows_raw = S.q_imp(wl, prod, rows=(row0, nrows))
    wpr = (row0 + nrows + 31) // 32
    masks = torch.zeros((wl.B, wl.Hq, nrows, wpr), dtype=torch.int32, device="cuda")
    ctx.select_prefill(layer, to_dev(qrows_raw, wl), row0, nrows, masks)
    torch.cuda.synchronize()
    assert ctx.check_status() == 0
    qrows = S.widen(qrows_raw, wl.dtype).reshape(wl.B, wl.Hq, wl.G, nrows, wl.d_imp)
    slot = O.consumer_slot(layer, wl.G)
    m = masks.cpu().numpy().view(np.uint32)
    gs = wl.Hq // wl.Hkv
    exact = checked = 0
    for b in range(wl.B):
        kb = O.project_keys(ld.K[b], ld.W, "bf16")
        ref = O.prefill_select(qrows[b, :, slot], kb, row0, wl.keep_pct, wl.sink, wl.window)
        for h in range(wl.Hq):
            for r in range(nrows):
                p = row0 + r
                bits = np.unpackbits(m[b, h, r].view(np.uint8), bitorder="little")
                assert not bits[p + 1:].any()
                got = np.nonzero(bits[:p + 1])[0]
                q = qrows[b, h, slot, r]
                s = O.importance_scores(q, kb[h // gs, :p + 1])
                slack = bf16_score_slack(np.abs(q), ld.K[b, h // gs, :p + 1], ld.W)
                assert tie_band_ok(got, ref[h, p], s, p + 1, wl.keep_pct, wl.sink, wl.window, slack)
                exact += np.array_equal(got, ref[h, p])
                checked += 1
    assert exact >= 0.95 * checked
