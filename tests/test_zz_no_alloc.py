"""tb_sparse_attn_static, the allocation-free attention entry point.

It serves callers that cannot allocate device memory (fixed-budget serving
loops, plug-ins in a host process that owns all device memory): it needs no
context and no workspace because its split partials live in a static device
array inside the library.  Its results must match the oracle's attention
over the same sets and tb_sparse_attn's, call after call, and requests too
large for the static array or for 32-bit cache rows must be refused.
This file is collected last so that a failure here leaves every other test
already run."""
import math

import numpy as np
import pytest
import torch

from oracle import tokenbutler as O
from query_aware_sparse_decode_b200 import synth as S
from query_aware_sparse_decode_b200 import tb as TB

from harness import assert_close_rows, config_of, make_layer, mask_from_sets

pytestmark = pytest.mark.gpu

WL = S.Workload("no_alloc_bf16", n_layers=1, B=2, Hq=8, Hkv=2, D=128, d_imp=32, G=1, L=3000, dtype="bf16",
                keep_pct=30, sink=16, window=64, lens=(3000, 1234))


def _sets(ld, wl):
    gs = wl.Hq // wl.Hkv
    sets = {}
    for b, L in enumerate(wl.seq_lens):
        for h in range(wl.Hq):
            s = O.importance_scores(ld.qhat[b, h], O.project_keys(ld.K[b, h // gs, :L], ld.W))
            sets[b, h] = O.select_tokens(s, L, wl.keep_pct, wl.sink, wl.window)
    return sets


@pytest.mark.parametrize("mode", [TB.TB_MASK_PER_HEAD, TB.TB_MASK_DENSE])
def test_static_attention_matches_context_attention_twice(mode):
    wl = WL
    ctx = TB.Context(config_of(wl))
    ld = make_layer(ctx, wl, 0, wl.seq_lens)
    mask = mask_from_sets(_sets(ld, wl), wl.B, wl.Hq, ctx.cfg.max_len) if mode == TB.TB_MASK_PER_HEAD else None
    ref = torch.empty((wl.B, wl.Hq, wl.D), dtype=torch.bfloat16, device="cuda")
    ref_lse = torch.empty((wl.B, wl.Hq), device="cuda")
    ctx.sparse_attn(0, ld.q_dev, mask, mode, ref, ref_lse)
    got = []
    for _ in range(2):  # the static scratch keeps the previous call's contents
        out = torch.full_like(ref, 3.0)
        lse = torch.full_like(ref_lse, 3.0)
        TB.sparse_attn_static(ld.k_cache, ld.v_cache, wl.seq_lens, wl.Hq, ld.q_dev, mask, mode, out, lse)
        got.append((out, lse))
    torch.cuda.synchronize()
    r, rl = ref.float().cpu().numpy(), ref_lse.cpu().numpy()
    # the oracle's attention over the same sets (every token for the dense mode)
    sets = _sets(ld, wl) if mode == TB.TB_MASK_PER_HEAD else None
    scale = 1.0 / math.sqrt(wl.D)
    gs = wl.Hq // wl.Hkv
    for out, lse in got:
        o, l = out.float().cpu().numpy(), lse.cpu().numpy()
        for b, L in enumerate(wl.seq_lens):
            assert_close_rows(o[b], r[b], "bf16", f"static vs context b{b}")
            assert np.all(np.abs(l[b] - rl[b]) <= 1e-3 * np.maximum(1.0, np.abs(rl[b])))
            for h in range(wl.Hq):
                idx = sets[b, h] if sets is not None else np.arange(L)
                want, want_lse = O.attend(ld.q[b, h], ld.K[b, h // gs, :L], ld.V[b, h // gs, :L], idx, scale)
                assert_close_rows(o[b, h][None], want[None], "bf16", f"static vs oracle b{b} h{h}")
                assert abs(l[b, h] - want_lse) <= 1e-3 * max(1.0, abs(want_lse))


def test_static_attention_refuses_requests_beyond_its_scratch():
    # B * Hq * (D + 2) fp32 partials of one split exceed the static array
    B, Hq, Hkv, D, max_len = 128, 128, 128, 128, 256
    assert B * Hq * (D + 2) * 4 > (8 << 20)
    small = torch.zeros(16, dtype=torch.bfloat16, device="cuda")  # never read: refused before any launch
    k = small.as_strided((B, Hkv, max_len, D), (0, 0, 0, 0))
    out = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    arr = (TB.ctypes.c_int32 * B)(*([10] * B))
    view = TB.CacheView(k.data_ptr(), k.data_ptr(), B, Hq, Hkv, D, max_len, TB.TB_BF16, arr)
    st = TB.lib().tb_sparse_attn_static(TB.ctypes.byref(view), TB.ctypes.c_void_p(small.data_ptr()), None,
                                        TB.TB_MASK_DENSE, TB.ctypes.c_void_p(out.data_ptr()), None, None)
    assert st == 3  # TB_ERR_CAPACITY


def test_static_attention_refuses_more_cache_rows_than_32_bits_hold():
    # B * Hkv * max_len >= 2^31: the gather lists hold 32-bit cache rows, so
    # the request is refused before any launch (a context refuses it too)
    B, Hq, Hkv, D, max_len = 128, 8, 8, 128, 1 << 21
    assert B * Hkv * max_len >= 1 << 31
    small = torch.zeros(16, dtype=torch.bfloat16, device="cuda")  # never read
    k = small.as_strided((B, Hkv, max_len, D), (0, 0, 0, 0))
    out = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    arr = (TB.ctypes.c_int32 * B)(*([10] * B))
    view = TB.CacheView(k.data_ptr(), k.data_ptr(), B, Hq, Hkv, D, max_len, TB.TB_BF16, arr)
    st = TB.lib().tb_sparse_attn_static(TB.ctypes.byref(view), TB.ctypes.c_void_p(small.data_ptr()), None,
                                        TB.TB_MASK_DENSE, TB.ctypes.c_void_p(out.data_ptr()), None, None)
    assert st == 2  # TB_ERR_SHAPE
