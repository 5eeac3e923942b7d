"""GPU parity of the prefill importance path: K_imp = K . W_K on the tensor
cores (tcgen05, bf16 operands, fp32 accumulation) and the per-row causal
selection of a prefill query chunk, against the fp64 oracle."""
import numpy as np
import pytest
import torch

from oracle import tokenbutler as O
from query_aware_sparse_decode_b200 import synth as S
from query_aware_sparse_decode_b200 import tb as TB

from harness import (bf16_kimp_bounds, config_of, kimp_alloc, kimp_rows, make_layer, round_up, sets_from_mask,
                     tie_band_ok, to_dev)

pytestmark = pytest.mark.gpu


def _kimp_tol(K, W):
    return 8e-6 * (np.abs(K) @ np.abs(W)) + 1e-30


@pytest.mark.parametrize("start,count", [(0, 32768), (5, 1000), (32640, 100)])
def test_tcgen05_projection_prefill_scale(start, count):
    """One layer of the prefill workload: B=1, 8 KV heads, 32768 cached rows,
    D=128 -> d'=32; rows checked against fp64 on every KV head."""
    wl = S.PREFILL_L32K.with_(n_layers=1, dense_layers=())
    ctx = TB.Context(config_of(wl, max_len=32768 + 256))
    B, Hkv, D = wl.B, wl.Hkv, wl.D
    K_raw = S.kv_cache_host(wl, 0, S.K_CACHE, 0, 32768).reshape(B, Hkv, 32768, D)
    W_raw = S.w_k(wl, 0)
    k = torch.zeros((B, Hkv, ctx.cfg.max_len, D), dtype=torch.bfloat16, device="cuda")
    k[:, :, :32768] = to_dev(K_raw, wl)
    kimp = kimp_alloc(B, Hkv, wl.d_imp, ctx.cfg.max_len, float("nan"))
    ctx.bind_layer(0, k, torch.zeros_like(k), kimp, to_dev(W_raw, wl))
    ctx.set_seq_lens(0, [32768])
    ctx.project_kimp(0, start, count)
    torch.cuda.synchronize()
    assert ctx.check_status() == 0
    got = kimp_rows(kimp)
    K = S.widen(K_raw, wl.dtype)
    W = S.widen(W_raw, wl.dtype)
    for g in range(Hkv):
        ref = O.project_keys(K[0, g, start:start + count], W)
        assert np.all(np.abs(got[0, g, start:start + count] - ref) <= _kimp_tol(K[0, g, start:start + count], W))
        assert np.all(np.isnan(got[0, g, :start])) and np.all(np.isnan(got[0, g, start + count:]))


@pytest.mark.parametrize("kimp_dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [(128, 32), (64, 16)], ids=["D128_d32", "D64_d16"])
def test_tcgen05_projection_over_many_layers_in_one_launch(d, kimp_dtype):
    """tb_project_kimp_layers: one persistent launch over 6 layers (each its
    own cache, W_K and K_imp) equals tb_project_kimp layer by layer bit for
    bit, and the fp64 oracle within the fp32 bound; rows outside
    [start, start + count) stay untouched.  B=2, 2 KV heads, 3000 rows: a
    CTA's tiles cross layer boundaries with both W_K^T buffers in use."""
    D, dimp = d
    wl = S.Workload("prefill_layers", n_layers=6, B=2, Hq=4, Hkv=2, D=D, d_imp=dimp, G=2, L=3000, dtype="bf16",
                    keep_pct=50, sink=16, window=64, dense_layers=())
    cfg = config_of(wl, max_len=3072, kimp_dtype=kimp_dtype)
    multi, single = TB.Context(cfg), TB.Context(cfg)
    start, count = 37, 2900
    kd = torch.bfloat16 if kimp_dtype == "bf16" else torch.float32
    layers = []
    for layer in range(wl.n_layers):
        K_raw = S.kv_cache_host(wl, layer, S.K_CACHE, 0, wl.L).reshape(wl.B, wl.Hkv, wl.L, D)
        W_raw = S.w_k(wl, layer)
        k = torch.zeros((wl.B, wl.Hkv, cfg.max_len, D), dtype=torch.bfloat16, device="cuda")
        k[:, :, :wl.L] = to_dev(K_raw, wl)
        w = to_dev(W_raw, wl)
        km = kimp_alloc(wl.B, wl.Hkv, dimp, cfg.max_len, float("nan"), kd)
        ks = kimp_alloc(wl.B, wl.Hkv, dimp, cfg.max_len, float("nan"), kd)
        multi.bind_layer(layer, k, torch.zeros_like(k), km, w)
        single.bind_layer(layer, k, torch.zeros_like(k), ks, w)
        for ctx in (multi, single):
            ctx.set_seq_lens(layer, [wl.L] * wl.B)
        layers.append((K_raw, W_raw, km, ks))
    multi.project_kimp_layers(0, wl.n_layers, start, count)
    for layer in range(wl.n_layers):
        single.project_kimp(layer, start, count)
    torch.cuda.synchronize()
    assert multi.check_status() == 0 and single.check_status() == 0
    for layer, (K_raw, W_raw, km, ks) in enumerate(layers):
        assert torch.equal(km.view(torch.int16) if kd == torch.bfloat16 else km.view(torch.int32),
                           ks.view(torch.int16) if kd == torch.bfloat16 else ks.view(torch.int32)), f"layer {layer}"
        got = kimp_rows(km)
        K, W = S.widen(K_raw, wl.dtype), S.widen(W_raw, wl.dtype)
        for b in range(wl.B):
            for g in range(wl.Hkv):
                Kr = K[b, g, start:start + count]
                ref = O.project_keys(Kr, W)
                if kimp_dtype == "bf16":
                    lo, hi = bf16_kimp_bounds(Kr, W)
                    assert np.all((got[b, g, start:start + count] >= lo) & (got[b, g, start:start + count] <= hi))
                else:
                    assert np.all(np.abs(got[b, g, start:start + count] - ref) <= _kimp_tol(Kr, W)), f"l{layer}"
                assert np.all(np.isnan(got[b, g, :start])) and np.all(np.isnan(got[b, g, start + count:]))


PF_SMALL = S.Workload("prefill_small", n_layers=8, B=2, Hq=8, Hkv=2, D=128, d_imp=32, G=4, L=3000, dtype="bf16",
                      keep_pct=50, sink=16, window=64, dense_layers=(0,))


def _prefill_case(wl, layer, row0, nrows, heads=None, rows=None):
    cfg = config_of(wl, max_len=round_up(wl.L, 256))
    ctx = TB.Context(cfg)
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
    full = heads is None and rows is None
    heads = range(wl.Hq) if heads is None else heads
    rows = range(nrows) if rows is None else rows
    exact = checked = 0
    for b in range(wl.B):
        Kimp = O.project_keys(ld.K[b], ld.W)
        ref = O.prefill_select(qrows[b, :, slot], Kimp, row0, wl.keep_pct, wl.sink, wl.window) if full else None
        for h in heads:
            for r in rows:
                p = row0 + r
                bits = np.unpackbits(m[b, h, r].view(np.uint8), bitorder="little")
                assert not bits[p + 1:].any()          # causal: nothing after the row's position
                got = np.nonzero(bits[:p + 1])[0]
                s = O.importance_scores(qrows[b, h, slot, r], Kimp[h // gs, :p + 1])
                want = ref[h, p] if full else O.select_tokens(s, p + 1, wl.keep_pct, wl.sink, wl.window)
                assert tie_band_ok(got, want, s, p + 1, wl.keep_pct, wl.sink, wl.window)
                exact += np.array_equal(got, want)
                checked += 1
    assert exact >= 0.95 * checked


def test_prefill_rows_small():
    _prefill_case(PF_SMALL, layer=5, row0=2936, nrows=64)


def test_prefill_rows_short_prefix_and_edges():
    # rows 0..99: prefixes shorter than sink + window, then growing budgets
    _prefill_case(PF_SMALL.with_(L=400, B=1), layer=4, row0=0, nrows=100)


def test_prefill_rows_llama8b_L32768_sampled():
    """The prefill workload's chunk (last 1024 positions of 32768): 4 heads x
    64 sampled rows checked against the oracle."""
    wl = S.PREFILL_L32K.with_(n_layers=2)
    _prefill_case(wl, layer=1, row0=32768 - 1024, nrows=1024, heads=[0, 9, 18, 31], rows=range(0, 1024, 16))


def test_prefill_rows_with_massive_ties_take_the_one_row_path():
    """Keys drawn from three distinct rows: each row's scores take three
    values, so the threshold prefix holds thousands of equal keys and the
    blocked kernel hands every row to the one-row method.  Ties go to the
    lowest indices; the sets must equal the oracle's exactly."""
    wl = PF_SMALL.with_(B=1, L=2048, n_layers=1, G=1, dense_layers=())
    cfg = config_of(wl, max_len=round_up(wl.L, 256))
    ctx = TB.Context(cfg)
    B, Hkv, D, Lmax = wl.B, wl.Hkv, wl.D, cfg.max_len
    base = S.fill_host(S.K_CACHE, 0, 0, Hkv, 0, 3, D, "bf16")          # three rows per KV head
    K_raw = np.stack([base[g][np.arange(wl.L) % 3] for g in range(Hkv)])[None]   # [1][Hkv][L][D]
    W_raw = S.w_k(wl, 0)
    k = torch.zeros((B, Hkv, Lmax, D), dtype=torch.bfloat16, device="cuda")
    k[:, :, :wl.L] = to_dev(K_raw, wl)
    kimp = kimp_alloc(B, Hkv, wl.d_imp, Lmax)
    ctx.bind_layer(0, k, torch.zeros_like(k), kimp, to_dev(W_raw, wl))
    ctx.set_seq_lens(0, [wl.L])
    ctx.project_kimp(0, 0, wl.L)
    row0, nrows = wl.L - 40, 40
    qrows_raw = S.q_imp(wl, 0, rows=(row0, nrows))
    wpr = (row0 + nrows + 31) // 32
    masks = torch.full((B, wl.Hq, nrows, wpr), -1, dtype=torch.int32, device="cuda")
    ctx.select_prefill(0, to_dev(qrows_raw, wl), row0, nrows, masks)
    torch.cuda.synchronize()
    assert ctx.check_status() == 0
    qrows = S.widen(qrows_raw, wl.dtype).reshape(B, wl.Hq, 1, nrows, wl.d_imp)
    Kimp = O.project_keys(S.widen(K_raw, "bf16")[0], S.widen(W_raw, "bf16"))
    ref = O.prefill_select(qrows[0, :, 0], Kimp, row0, wl.keep_pct, wl.sink, wl.window)
    m = masks.cpu().numpy().view(np.uint32)
    for h in range(wl.Hq):
        for r in range(nrows):
            p = row0 + r
            bits = np.unpackbits(m[0, h, r].view(np.uint8), bitorder="little")
            assert not bits[p + 1:].any()
            assert np.array_equal(np.nonzero(bits[:p + 1])[0], ref[h, p])


def test_prefill_rows_longest_prefix_and_the_limit_beyond():
    """Rows up to the accepted prefix of 51200 tokens select exactly; one
    token more is refused before any launch (TB_ERR_UNSUPPORTED)."""
    wl = PF_SMALL.with_(B=1, L=51200, n_layers=6)
    _prefill_case(wl, layer=5, row0=51200 - 40, nrows=40, heads=[0, 3, 7], rows=[0, 7, 15, 16, 23, 24, 39])
    cfg = config_of(wl.with_(L=51201), max_len=round_up(51201, 256))
    ctx = TB.Context(cfg)
    make_layer(ctx, wl.with_(L=51201), 5, [51201])
    qrows = S.q_imp(wl, O.producer_of(5, wl.G), rows=(51201 - 16, 16))
    masks = torch.zeros((1, wl.Hq, 16, (51201 + 31) // 32), dtype=torch.int32, device="cuda")
    with pytest.raises(TB.TBError) as err:
        ctx.select_prefill(5, to_dev(qrows, wl), 51201 - 16, 16, masks)
    assert err.value.status == 7  # TB_ERR_UNSUPPORTED


def test_prefill_rows_blocked_partial_block_and_mixed_budgets():
    """nrows not a multiple of the 16-row block, rows whose prefixes are
    shorter than sink + window next to rows with a real top-k."""
    _prefill_case(PF_SMALL.with_(L=300, B=2), layer=6, row0=50, nrows=37)
