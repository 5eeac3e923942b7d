"""GPU parity of the soft-voting variant (TokenSelect per-head soft voting)
against the fp64 oracle: votes within 1e-4 * max|votes|, the shared
selected set equal except inside the tie band, attention outputs within the
bf16 tolerance against the oracle's attention over the GPU's set (the
oracle's own set where the two agree; the output given a set is unique)."""
import math

import numpy as np
import pytest
import torch

from oracle import tokenbutler as O
from query_aware_sparse_decode_b200 import synth as S
from query_aware_sparse_decode_b200 import tb as TB

from harness import assert_close_rows, config_of, make_layer, sets_from_mask, tie_band_ok, to_dev

pytestmark = pytest.mark.gpu

SV_SMALL = S.Workload("softvote_small", n_layers=1, B=2, Hq=8, Hkv=2, D=128, d_imp=32, G=1, L=5000, dtype="bf16",
                      keep_pct=30, sink=16, window=64, lens=(5000, 777))


def _softvote_case(wl):
    cfg = config_of(wl, variant=TB.TB_SOFTVOTE)
    ctx = TB.Context(cfg)
    lens = wl.seq_lens
    ld = make_layer(ctx, wl, 0, lens)
    votes = torch.full((wl.B, cfg.max_len), float("nan"), device="cuda")
    ctx.softvote_scores(0, ld.q_dev, votes)
    mask = torch.zeros((wl.B, 1, cfg.max_len // 32), dtype=torch.int32, device="cuda")
    ctx.select(0, votes, 1, mask=mask)
    out = torch.empty((wl.B, wl.Hq, wl.D), dtype=torch.bfloat16, device="cuda")
    ctx.sparse_attn(0, ld.q_dev, mask, TB.TB_MASK_SHARED, out)
    torch.cuda.synchronize()
    assert ctx.check_status() == 0
    v = votes.cpu().numpy().astype(np.float64)
    got = sets_from_mask(mask, lens)
    o = out.float().cpu().numpy()
    sel, ref, _, ref_votes = O.softvote_layer(ld.q, ld.K, ld.V, lens, wl.keep_pct, wl.sink, wl.window)
    scale = 1.0 / math.sqrt(wl.D)
    agree = 0
    for b, L in enumerate(lens):
        assert np.max(np.abs(v[b, :L] - ref_votes[b])) <= 1e-4 * np.max(np.abs(ref_votes[b]))
        assert abs(v[b, :L].sum() - wl.Hq) <= 1e-3 * wl.Hq
        assert tie_band_ok(got[b, 0], sel[b], ref_votes[b], L, wl.keep_pct, wl.sink, wl.window)
        same = np.array_equal(got[b, 0], sel[b])
        agree += same
        for h in range(wl.Hq):
            want = ref[b, h]
            if not same:
                g = O.kv_head_of(h, wl.Hq, wl.Hkv)
                want, _ = O.attend(ld.q[b, h], ld.K[b, g, :L], ld.V[b, g, :L], got[b, 0], scale)
            assert_close_rows(o[b, h][None], want[None], "bf16", f"b{b} h{h}")
    assert agree >= 1
    return ctx, ld


def test_softvote_small_ragged():
    _softvote_case(SV_SMALL)


def test_softvote_llama8b_L16384():
    _softvote_case(S.sweep(16384, 30))


def test_softvote_decode_step_matches_separate_calls():
    wl = SV_SMALL.with_(lens=None, B=1)
    cfg = config_of(wl, variant=TB.TB_SOFTVOTE)
    ctx = TB.Context(cfg)
    ld = make_layer(ctx, wl, 0, [wl.L - 1])
    ctx.project_kimp(0, 0, wl.L - 1)
    k_raw, v_raw = S.kv_new(wl, 0)
    out = torch.empty((1, wl.Hq, wl.D), dtype=torch.bfloat16, device="cuda")
    ctx.decode_step(0, to_dev(k_raw, wl), to_dev(v_raw, wl), ld.q_dev, None, out)
    votes = torch.empty((1, cfg.max_len), device="cuda")
    mask = torch.zeros((1, 1, cfg.max_len // 32), dtype=torch.int32, device="cuda")
    out2 = torch.empty_like(out)
    ctx.softvote_scores(0, ld.q_dev, votes)
    ctx.select(0, votes, 1, mask=mask)
    ctx.sparse_attn(0, ld.q_dev, mask, TB.TB_MASK_SHARED, out2)
    torch.cuda.synchronize()
    assert torch.equal(out, out2)
