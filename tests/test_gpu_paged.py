"""Paged K/V caches: the same rows placed in shuffled pages of a pool.  The
paged decode step is checked against the oracle as the dense one is (K_imp
of the paged projection within fp32 rounding of the exact K W_K, sets within
the tie band, outputs against the oracle's attention over the GPU's set), and
against the dense layout: bit-identical results for every call that touches
K or V once both see the same K_imp."""
import math

import numpy as np
import pytest
import torch

from oracle import tokenbutler as O
from query_aware_sparse_decode_b200 import synth as S
from query_aware_sparse_decode_b200 import tb as TB

from harness import (KIMP_REL, assert_close_rows, config_of, kimp_alloc, kimp_rows, make_layer, paged_copy,
                     sets_from_mask, tdtype, tie_band_ok, to_dev)

pytestmark = pytest.mark.gpu

WL = S.Workload("paged_bf16", n_layers=1, B=2, Hq=8, Hkv=2, D=128, d_imp=32, G=1, L=3000, dtype="bf16",
                keep_pct=30, sink=16, window=64, lens=(3000, 1777))
PAGE = 64


def _check_against_oracle(wl, ld, variant, k_raw, v_raw, lens, kimp_dev, masks, out):
    """The paged step's K_imp, sets and outputs against the oracle on the
    same inputs (the full caches with the appended token)."""
    k64, v64 = S.widen(k_raw, wl.dtype), S.widen(v_raw, wl.dtype)
    K = np.concatenate([ld.K, np.zeros((wl.B, wl.Hkv, 1, wl.D))], axis=2)
    V = np.concatenate([ld.V, np.zeros((wl.B, wl.Hkv, 1, wl.D))], axis=2)
    for b, L in enumerate(lens):
        K[b, :, L - 1], V[b, :, L - 1] = k64[b], v64[b]
    o = out.float().cpu().numpy()
    scale = 1.0 / math.sqrt(wl.D)
    gs = wl.Hq // wl.Hkv
    got = sets_from_mask(masks, lens)
    if variant == TB.TB_SOFTVOTE:
        sel, _, _, votes = O.softvote_layer(ld.q, K, V, lens, wl.keep_pct, wl.sink, wl.window)
        for b, L in enumerate(lens):
            assert tie_band_ok(got[b, 0], sel[b], votes[b], L, wl.keep_pct, wl.sink, wl.window), f"b{b}"
            for h in range(wl.Hq):
                g = h // gs
                want, _ = O.attend(ld.q[b, h], K[b, g, :L], V[b, g, :L], got[b, 0], scale)
                assert_close_rows(o[b, h][None], want[None], wl.dtype, f"softvote b{b} h{h}")
        return
    # K_imp of the paged (fp32 FMA) projection and of the append, element by element
    kp = kimp_rows(kimp_dev)
    for b, L in enumerate(lens):
        for g in range(wl.Hkv):
            exact = O.project_keys(K[b, g, :L], ld.W)
            tol = KIMP_REL * (np.abs(K[b, g, :L]) @ np.abs(ld.W)) + 1e-30
            assert np.all(np.abs(kp[b, g, :L] - exact) <= tol), f"K_imp b{b} g{g}"
    group = variant == TB.TB_BUTLER_GROUP
    sel, ref, _, sc = O.decode_layer(ld.q, K, V, ld.W, ld.qimp, 0, wl.G, lens, wl.keep_pct, wl.sink, wl.window,
                                     dense=False, group=group)
    mism = 0
    for b, L in enumerate(lens):
        for h in range(wl.Hq):
            g = h // gs
            r = g if group else h
            assert tie_band_ok(got[b, r], sel[b, h], sc[b, h], L, wl.keep_pct, wl.sink, wl.window), f"b{b} h{h}"
            want = ref[b, h]
            if not np.array_equal(got[b, r], sel[b, h]):
                mism += 1
                want, _ = O.attend(ld.q[b, h], K[b, g, :L], V[b, g, :L], got[b, r], scale)
            assert_close_rows(o[b, h][None], want[None], wl.dtype, f"b{b} h{h}")
    assert mism <= max(1, wl.B * wl.Hq // 20)


@pytest.mark.parametrize("variant", [TB.TB_BUTLER, TB.TB_BUTLER_GROUP, TB.TB_SOFTVOTE],
                         ids=["butler", "group", "softvote"])
def test_paged_step_matches_oracle_and_dense(variant):
    wl = WL
    cfg = config_of(wl, max_len=3072, variant=variant)
    dense = TB.Context(cfg)
    lens0 = [L - 1 for L in wl.seq_lens]
    ld = make_layer(dense, wl, 0, lens0)
    paged = TB.Context(cfg)
    kpool, vpool, table = paged_copy(ld, wl, cfg.max_len, PAGE, 5)
    kimp_p = kimp_alloc(wl.B, wl.Hkv, wl.d_imp, cfg.max_len)
    paged.bind_layer_paged(0, kpool, vpool, table, kimp_p, ld.w_k)
    paged.set_seq_lens(0, lens0)
    k_raw, v_raw = S.kv_new(wl, 0)
    outs = []
    for ctx in (dense, paged):
        ctx.project_kimp(0, 0, max(lens0))
        out = torch.empty((wl.B, wl.Hq, wl.D), dtype=tdtype(wl), device="cuda")
        ctx.decode_step(0, to_dev(k_raw, wl), to_dev(v_raw, wl), ld.q_dev, ld.q_imp_dev, out)
        torch.cuda.synchronize()
        assert ctx.check_status() == 0
        outs.append(out.clone())
    assert paged.seq_lens(0) == [L for L in wl.seq_lens]
    # the appended rows landed in the pages the table names
    for b, L in enumerate(wl.seq_lens):
        page, off = table[b, (L - 1) // PAGE].item(), (L - 1) % PAGE
        assert torch.equal(kpool[page, :, off], ld.k_cache[b, :, L - 1])
        assert torch.equal(vpool[page, :, off], ld.v_cache[b, :, L - 1])
    if variant == TB.TB_SOFTVOTE:
        assert torch.equal(outs[0], outs[1])   # no K_imp on this path
    # the paged step against the oracle (the dense bf16 cache was projected on
    # the tensor cores, the paged one by fp32 FMA: each within fp32 rounding)
    rows = 1 if variant == TB.TB_SOFTVOTE else (wl.Hkv if variant == TB.TB_BUTLER_GROUP else wl.Hq)
    masks = paged.step_masks(rows)
    torch.cuda.synchronize()
    _check_against_oracle(wl, ld, variant, k_raw, v_raw, paged.seq_lens(0), kimp_p, masks, outs[1])


def test_paged_attention_and_selection_match_dense_on_identical_kimp():
    """With K_imp copied from the dense context, the paged step's selections
    and outputs are bit-identical to the dense step's."""
    wl = WL
    cfg = config_of(wl, max_len=3072)
    dense = TB.Context(cfg)
    lens0 = [L - 1 for L in wl.seq_lens]
    ld = make_layer(dense, wl, 0, lens0)
    dense.project_kimp(0, 0, max(lens0))
    paged = TB.Context(cfg)
    kpool, vpool, table = paged_copy(ld, wl, cfg.max_len, PAGE, 9)
    kimp_p = ld.kimp.clone()
    paged.bind_layer_paged(0, kpool, vpool, table, kimp_p, ld.w_k)
    paged.set_seq_lens(0, lens0)
    k_raw, v_raw = S.kv_new(wl, 0, step=2)
    res = []
    for ctx in (dense, paged):
        out = torch.empty((wl.B, wl.Hq, wl.D), dtype=tdtype(wl), device="cuda")
        ctx.decode_step(0, to_dev(k_raw, wl), to_dev(v_raw, wl), ld.q_dev, ld.q_imp_dev, out)
        masks = ctx.step_masks(wl.Hq)
        lse = torch.empty((wl.B, wl.Hq), device="cuda")
        out2 = torch.empty_like(out)
        ctx.sparse_attn(0, ld.q_dev, masks, TB.TB_MASK_PER_HEAD, out2, lse)
        torch.cuda.synchronize()
        assert ctx.check_status() == 0
        res.append((out, masks, out2, lse))
    # the appended K_imp row is computed by the same append kernel in both
    assert torch.equal(kimp_p, ld.kimp)
    (o_d, m_d, o2_d, l_d), (o_p, m_p, o2_p, l_p) = res
    lens = paged.seq_lens(0)
    sd, sp = sets_from_mask(m_d, lens), sets_from_mask(m_p, lens)  # words past the length are stale
    assert all(np.array_equal(sd[k], sp[k]) for k in sd)
    assert torch.equal(o_d, o_p) and torch.equal(o2_d, o2_p) and torch.equal(l_d, l_p)
