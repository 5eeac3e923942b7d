"""Shared set-up for the GPU parity tests: seeded inputs (from the generator
module), device buffers, a bound context, and comparison helpers.  Expected
values come only from the oracle."""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

from oracle import tokenbutler as O
from query_aware_sparse_decode_b200 import synth as S
from query_aware_sparse_decode_b200 import tb as TB


def tdtype(wl):
    return torch.bfloat16 if wl.dtype == "bf16" else torch.float32


def to_dev(arr: np.ndarray, wl) -> torch.Tensor:
    if wl.dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32)).cuda()


def round_up(x: int, m: int) -> int:
    return (x + m - 1) // m * m


@dataclass
class LayerData:
    layer: int
    W: np.ndarray          # [D][d'] float64
    qimp: np.ndarray       # producer tensor [(B*Hq)][G][1][d'] float64
    qhat: np.ndarray | None  # consumer queries [B][Hq][d'] float64 (None for dense layers)
    q: np.ndarray          # [B][Hq][D] float64
    K: np.ndarray          # [B][Hkv][Lfill][D] float64
    V: np.ndarray
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    kimp: torch.Tensor
    w_k: torch.Tensor
    q_imp_dev: torch.Tensor
    q_dev: torch.Tensor


def config_of(wl, max_len=None, keep_pct=None, variant=TB.TB_BUTLER, kimp_dtype="f32") -> TB.Config:
    return TB.make_config(wl.n_layers, wl.B, wl.Hq, wl.Hkv, wl.D, wl.d_imp, wl.G,
                          max_len if max_len is not None else round_up(wl.max_len + 1, 256), wl.dtype,
                          wl.keep_pct if keep_pct is None else keep_pct, wl.sink, wl.window,
                          dense_layers=wl.dense_layers, variant=variant, kimp_dtype=kimp_dtype)


def make_layer(ctx: TB.Context, wl, layer: int, lens, step: int = 0) -> LayerData:
    """Generates layer `layer` on the host, uploads it and binds it with the
    given per-sequence lengths (rows [0, len[b]) filled)."""
    B, Hq, Hkv, D, dimp, G = wl.B, wl.Hq, wl.Hkv, wl.D, wl.d_imp, wl.G
    Lmax = ctx.cfg.max_len
    Lfill = max(lens)
    W_raw = S.w_k(wl, layer)
    W = S.widen(W_raw, wl.dtype)
    prod = O.producer_of(layer, G)
    qimp_raw = S.q_imp(wl, prod, step)
    qimp = S.widen(qimp_raw, wl.dtype)
    dense = layer in wl.dense_layers
    qhat = None if dense else O.importance_queries(qimp, layer, G, B, Hq)
    delta = None if dense or wl.plant == "none" else S.plant_delta(W, qhat, Hkv)
    K_raw = S.kv_cache_host(wl, layer, S.K_CACHE, 0, Lfill, delta).reshape(B, Hkv, Lfill, D)
    V_raw = S.kv_cache_host(wl, layer, S.V_CACHE, 0, Lfill).reshape(B, Hkv, Lfill, D)
    q_raw = S.query(wl, layer, step)
    k_cache = torch.zeros((B, Hkv, Lmax, D), dtype=tdtype(wl), device="cuda")
    v_cache = torch.zeros_like(k_cache)
    k_cache[:, :, :Lfill] = to_dev(K_raw, wl)
    v_cache[:, :, :Lfill] = to_dev(V_raw, wl)
    kimp = TB.kimp_cache(ctx.cfg)
    w_k = to_dev(W_raw, wl)
    ctx.bind_layer(layer, k_cache, v_cache, kimp, w_k)
    ctx.set_seq_lens(layer, lens)
    return LayerData(layer, W, qimp, qhat, S.widen(q_raw, wl.dtype), S.widen(K_raw, wl.dtype),
                     S.widen(V_raw, wl.dtype), k_cache, v_cache, kimp, w_k, to_dev(qimp_raw, wl), to_dev(q_raw, wl))


def kimp_alloc(B, Hkv, dimp, Lmax, fill=0.0, dtype=torch.float32) -> torch.Tensor:
    """K_imp cache in the library's layout: 256-token tiles, dimension-major inside."""
    return torch.full((B, Hkv, Lmax // 256, dimp, 256), fill, dtype=dtype, device="cuda")


def kimp_rows(kimp: torch.Tensor) -> np.ndarray:
    """[B][Hkv][Lmax][d'] float64 view of a K_imp cache (fp32 or bf16)."""
    B, Hkv, nt, dimp, _ = kimp.shape
    return kimp.permute(0, 1, 2, 4, 3).reshape(B, Hkv, nt * 256, dimp).float().cpu().numpy().astype(np.float64)


KIMP_REL = 8e-6   # fp32 dot-product error bound of a K_imp element, relative to sum_d |K_d W_dj| (D <= 128)


def bf16_kimp_bounds(K: np.ndarray, W: np.ndarray):
    """The bfloat16 values a kernel may store for K_imp = K W: it rounds an
    fp32 dot product within KIMP_REL * sum|K_d W_dj| of the exact value, and
    rounding is monotone, so its value lies between the oracle's rounding of
    the two ends of that interval (equal ends: one possible value)."""
    x = np.asarray(K, np.float64) @ np.asarray(W, np.float64)
    tol = KIMP_REL * (np.abs(K) @ np.abs(W)) + 1e-30
    return O.round_to_bf16(x - tol), O.round_to_bf16(x + tol)


def bf16_kimp_ok(got: np.ndarray, K: np.ndarray, W: np.ndarray) -> bool:
    """A kernel's bf16 K_imp is the oracle's rounding of the exact K W,
    or, where the fp32 error interval straddles a rounding midpoint, the
    bfloat16 neighbour on the other side."""
    lo, hi = bf16_kimp_bounds(K, W)
    return bool(((got >= lo) & (got <= hi)).all())


def bf16_score_slack(qabs: np.ndarray, K: np.ndarray, W: np.ndarray) -> np.ndarray:
    """Per-token bound [L] on how far a score over a kernel's bf16 K_imp may
    sit from the same score over the oracle's: sum_j |q_j| (hi_j - lo_j).
    qabs: [d'] absolute importance query (a group's: the sum of |q| over
    its heads)."""
    lo, hi = bf16_kimp_bounds(K, W)
    return (hi - lo) @ np.asarray(qabs, np.float64)


def paged_copy(ld, wl, max_len, page, seed):
    """Pool [pages][Hkv][page][D] holding the dense caches' rows in shuffled
    pages (plus unused spare pages), and the page table [B][max_len/page]."""
    per_seq = max_len // page
    n_pages = wl.B * per_seq + 5
    perm = np.random.default_rng(seed).permutation(n_pages)[: wl.B * per_seq].reshape(wl.B, per_seq)
    kpool = torch.zeros((n_pages, wl.Hkv, page, wl.D), dtype=ld.k_cache.dtype, device="cuda")
    vpool = torch.zeros_like(kpool)
    for b in range(wl.B):
        for i in range(per_seq):
            kpool[perm[b, i]] = ld.k_cache[b, :, i * page:(i + 1) * page]
            vpool[perm[b, i]] = ld.v_cache[b, :, i * page:(i + 1) * page]
    table = torch.from_numpy(perm.astype(np.int32)).cuda()
    return kpool, vpool, table


def mask_from_sets(sets: dict, B: int, rows: int, Lmax: int) -> torch.Tensor:
    """uint32-as-int32 bitmask [B][rows][Lmax/32] from {(b, r): indices}."""
    m = np.zeros((B, rows, Lmax // 32), dtype=np.uint32)
    for (b, r), idx in sets.items():
        idx = np.asarray(idx, dtype=np.int64)
        np.bitwise_or.at(m[b, r], idx // 32, (np.uint32(1) << (idx % 32).astype(np.uint32)))
    return torch.from_numpy(m.view(np.int32)).cuda()


def sets_from_mask(mask: torch.Tensor, lens) -> dict:
    m = mask.cpu().numpy().view(np.uint32)
    out = {}
    B, rows, _ = m.shape
    for b in range(B):
        L = lens[b]
        for r in range(rows):
            bits = np.unpackbits(m[b, r].view(np.uint8), bitorder="little")[:L]
            out[b, r] = np.nonzero(bits)[0]
    return out


def assert_close_rows(got: np.ndarray, ref: np.ndarray, dtype: str, what: str = "") -> float:
    """fp32: max-abs <= 2e-3; bf16: max-abs <= 1e-2 * max|ref| per row.
    Returns the worst ratio error / allowed."""
    err = np.abs(got - ref)
    if dtype == "f32":
        allowed = 2e-3
        worst = float(err.max() / allowed)
    else:
        allowed = 1e-2 * np.maximum(np.abs(ref).max(axis=-1, keepdims=True), 1e-30)
        worst = float((err / allowed).max())
    assert worst <= 1.0, f"{what}: error {worst:.3f} x tolerance"
    return worst


def tie_band_ok(gpu_set, ref_set, scores64, L, keep_pct, sink, window, slack=None) -> bool:
    """Selected sets agree except on tokens whose oracle score lies within
    1e-4 * max|score| of the k-th candidate score (plus, with a bf16 K_imp,
    the token's own slack and the largest slack: `slack` [L])."""
    g, r = set(np.asarray(gpu_set).tolist()), set(np.asarray(ref_set).tolist())
    if g == r:
        return True
    if len(g) != len(r):
        return False
    cand = np.arange(sink, L - window) if L - window > sink else np.zeros(0, np.int64)
    k = min(O.token_budget(L, keep_pct), cand.size)
    if k == 0:
        return False
    sc = scores64[cand]
    kth = np.sort(sc)[::-1][k - 1]
    band = 1e-4 * np.abs(scores64[:L]).max()
    if slack is None:
        return all(abs(scores64[t] - kth) <= band for t in g ^ r)
    smax = float(np.max(slack[:L]))
    return all(abs(scores64[t] - kth) <= band + slack[t] + smax for t in g ^ r)


@dataclass
class DeviceLayer:
    """A layer whose caches were made on the device by the shared generator;
    the oracle regenerates any (b, KV head) slab on the host (same bits)."""
    wl: object
    layer: int
    L0: int
    W: np.ndarray            # [D][d'] float64
    qimp: np.ndarray         # producer tensor, float64
    qhat: np.ndarray | None  # [B][Hq][d'] float64
    delta: np.ndarray | None  # [B][Hkv][D] float32
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    kimp: torch.Tensor
    q_imp_dev: torch.Tensor
    q_dev: torch.Tensor
    q: np.ndarray            # [B][Hq][D] float64

    def slab(self, which: int, b: int, g: int) -> np.ndarray:
        """Rows [0, L0) of K (which=K_CACHE) or V of one (b, g), float64 [L0][D]."""
        wl = self.wl
        a = b * wl.Hkv + g
        delta = None
        mod = 0
        if which == S.K_CACHE and self.delta is not None:
            delta, mod = self.delta.reshape(wl.B * wl.Hkv, wl.D), 100
        raw = S.fill_host(which, self.layer, 0, 1, 0, self.L0, wl.D, wl.dtype, delta=delta, plant_mod=mod,
                          seed=wl.seed, a0=a)[0]
        return S.widen(raw, wl.dtype)


def make_layer_device(ctx: TB.Context, wl, layer: int, L0: int, step: int = 0) -> DeviceLayer:
    """Fills rows [0, L0) of every sequence on the device (1 % planted heavy
    hitters on consumer layers), binds the layer with len = L0 and projects
    K_imp with the library."""
    B, Hq, Hkv, D, dimp, G = wl.B, wl.Hq, wl.Hkv, wl.D, wl.d_imp, wl.G
    Lmax = ctx.cfg.max_len
    W_raw = S.w_k(wl, layer)
    W = S.widen(W_raw, wl.dtype)
    qimp_raw = S.q_imp(wl, O.producer_of(layer, G), step)
    qimp = S.widen(qimp_raw, wl.dtype)
    dense = layer in wl.dense_layers
    qhat = None if dense else O.importance_queries(qimp, layer, G, B, Hq)
    delta = None if dense or wl.plant == "none" else S.plant_delta(W, qhat, Hkv)
    k = torch.empty((B, Hkv, Lmax, D), dtype=tdtype(wl), device="cuda")
    v = torch.empty_like(k)
    dd = None if delta is None else torch.from_numpy(delta.reshape(B * Hkv, D)).cuda()
    S.fill_device(k, S.K_CACHE, layer, 0, B * Hkv, 0, L0, D, Lmax * D, D, wl.dtype, delta=dd,
                  plant_mod=100 if dd is not None else 0, seed=wl.seed)
    S.fill_device(v, S.V_CACHE, layer, 0, B * Hkv, 0, L0, D, Lmax * D, D, wl.dtype, seed=wl.seed)
    kimp = TB.kimp_cache(ctx.cfg)
    ctx.bind_layer(layer, k, v, kimp, to_dev(W_raw, wl))
    ctx.set_seq_lens(layer, [L0] * B)
    ctx.project_kimp(layer, 0, L0)
    q_raw = S.query(wl, layer, step)
    return DeviceLayer(wl, layer, L0, W, qimp, qhat, delta, k, v, kimp, to_dev(qimp_raw, wl), to_dev(q_raw, wl),
                       S.widen(q_raw, wl.dtype))
