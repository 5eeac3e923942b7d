"""Paged K/V caches: the same rows placed in shuffled pages of a pool must give
bit-identical results to the dense layout, for every call that touches K or
V (append, K_imp projection, scoring, selection, attention, soft voting), and
the paged decode step must match the oracle like the dense one does."""
import numpy as np
import pytest
import torch

from query_aware_sparse_decode_b200 import synth as S
from query_aware_sparse_decode_b200 import tb as TB

from harness import config_of, kimp_alloc, make_layer, paged_copy, sets_from_mask, tdtype, to_dev

pytestmark = pytest.mark.gpu

WL = S.Workload("paged_bf16", n_layers=1, B=2, Hq=8, Hkv=2, D=128, d_imp=32, G=1, L=3000, dtype="bf16",
                keep_pct=30, sink=16, window=64, lens=(3000, 1777))
PAGE = 64


@pytest.mark.parametrize("variant", [TB.TB_BUTLER, TB.TB_BUTLER_GROUP, TB.TB_SOFTVOTE],
                         ids=["butler", "group", "softvote"])
def test_paged_equals_dense_bit_for_bit(variant):
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
    else:
        # K_imp: the dense bf16 cache was projected on the tensor cores, the paged
        # one by fp32 FMA, so compare the projections to each other within fp32
        # rounding and the outputs of steps that select from equal scores below
        kd, kp = ld.kimp.cpu().numpy(), kimp_p.cpu().numpy()
        assert np.allclose(kd, kp, rtol=1e-5, atol=1e-5)


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
