"""The C++ fp64 oracle (oracle/tokenbutler.cpp) with the numpy oracle's
interface: the same function names, arguments and results as
oracle/tokenbutler.py, so every pin runs on both.

TEST INFRASTRUCTURE.  Only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  It builds the library on first use (oracle/build.py).  The
arithmetic is all in the C++ library; this module only converts arrays and
shapes, and composes the sharded step from the library's calls as the numpy
oracle does.  Threads: ``set_threads(n)`` (OpenMP over independent
(sequence, head) rows; the arithmetic inside a row does not depend on it).
"""
from __future__ import annotations

import ctypes
import math

import numpy as np

from oracle import build as _build

_LIB = None
_D = ctypes.POINTER(ctypes.c_double)
_L = ctypes.POINTER(ctypes.c_long)
_I = ctypes.POINTER(ctypes.c_int)


def lib():
    global _LIB
    if _LIB is None:
        h = ctypes.CDLL(_build.build())
        i, l, d, vp = ctypes.c_int, ctypes.c_long, ctypes.c_double, ctypes.c_void_p
        sig = {
            "tbo_set_threads": (None, [i]), "tbo_get_threads": (i, []),
            "tbo_producer_of": (i, [i, i]), "tbo_consumer_slot": (i, [i, i]), "tbo_kv_head_of": (i, [i, i, i]),
            "tbo_keep_pct_from_policy": (i, [ctypes.c_char_p]),
            "tbo_importance_queries": (None, [_D, i, i, i, i, i, i, i, _D]),
            "tbo_token_budget": (l, [l, i]),
            "tbo_round_to_bf16_array": (None, [_D, l, _D]),
            "tbo_project_keys": (None, [_D, l, i, _D, i, i, _D]),
            "tbo_importance_scores": (None, [_D, _D, l, i, _D]),
            "tbo_group_scores": (None, [_D, i, _D, l, i, _D]),
            "tbo_select_tokens": (l, [_D, l, i, i, i, _L]),
            "tbo_attend": (None, [_D, _D, _D, i, _L, l, d, _D, _D]),
            "tbo_softvote_scores": (None, [_D, i, _D, i, l, l, i, _D]),
            "tbo_reuse_decision": (i, [_D, _D, i, l, l, l, d, i, i, i]),
            "tbo_reused_set": (l, [_L, l, l, l, i, i, i, _L]),
            "tbo_merge_partials": (None, [_D, _D, i, i, _D, _D]),
            "tbo_decode_layer": (None, [_D, _D, _D, _D, _D, vp, l, i, i, i, i, i, l, i, i, _L, i, i, i, i, i, i,
                                        _I, i, l, _L, _L, _D, _D, vp]),
            "tbo_prefill_select": (None, [_D, i, i, i, _D, i, l, l, i, i, i, _L, _L]),
        }
        for name, (res, args) in sig.items():
            f = getattr(h, name)
            f.restype = res
            f.argtypes = args
        _LIB = h
    return _LIB


def _d(a: np.ndarray):
    return a.ctypes.data_as(_D)


def _l(a: np.ndarray):
    return a.ctypes.data_as(_L)


def _f64(x) -> np.ndarray:
    return np.ascontiguousarray(x, dtype=np.float64)


def set_threads(n: int) -> None:
    lib().tbo_set_threads(int(n))


def get_threads() -> int:
    return int(lib().tbo_get_threads())


# ------------------------------------------------------------------ layers
def producer_of(layer: int, G: int) -> int:
    return int(lib().tbo_producer_of(layer, G))


def consumer_slot(layer: int, G: int) -> int:
    return int(lib().tbo_consumer_slot(layer, G))


def kv_head_of(h: int, Hq: int, Hkv: int) -> int:
    return int(lib().tbo_kv_head_of(h, Hq, Hkv))


def keep_pct_from_policy(policy: str) -> int:
    v = int(lib().tbo_keep_pct_from_policy(policy.encode()))
    if v < 0:
        raise ValueError(f"unsupported policy {policy!r}")
    return v


def importance_queries(q_imp_producer, layer: int, G: int, B: int, Hq: int, position: int = 0) -> np.ndarray:
    q = _f64(q_imp_producer)
    out = np.empty((B, Hq, q.shape[-1]), np.float64)
    lib().tbo_importance_queries(_d(q), B, Hq, G, q.shape[2], q.shape[3], layer, position, _d(out))
    return out


def token_budget(L: int, keep_pct: int) -> int:
    return int(lib().tbo_token_budget(L, keep_pct))


# ------------------------------------------------------------------ a1: K_imp
def round_to_bf16(x) -> np.ndarray:
    a = _f64(x)
    out = np.empty_like(a)
    lib().tbo_round_to_bf16_array(_d(a), a.size, _d(out))
    return out


def project_keys(K, W_K, storage: str = "f64") -> np.ndarray:
    K = _f64(K)
    W = _f64(W_K)
    D, dimp = W.shape
    n = K.size // D
    out = np.empty(K.shape[:-1] + (dimp,), np.float64)
    lib().tbo_project_keys(_d(K), n, D, _d(W), dimp, 1 if storage == "bf16" else 0, _d(out))
    return out


# ------------------------------------------------------------------ a3: scores
def importance_scores(q_hat, K_imp) -> np.ndarray:
    q, k = _f64(q_hat), _f64(K_imp)
    out = np.empty(k.shape[0], np.float64)
    lib().tbo_importance_scores(_d(q), _d(k), k.shape[0], k.shape[1], _d(out))
    return out


def group_scores(q_hat_heads, K_imp) -> np.ndarray:
    q, k = _f64(q_hat_heads), _f64(K_imp)
    out = np.empty(k.shape[0], np.float64)
    lib().tbo_group_scores(_d(q), q.shape[0], _d(k), k.shape[0], k.shape[1], _d(out))
    return out


# ------------------------------------------------------------------ a4/a5: select
def select_tokens(scores, L: int, keep_pct: int, sink: int, window: int) -> np.ndarray:
    s = _f64(scores)
    out = np.empty(max(L, 1), np.int64)
    n = lib().tbo_select_tokens(_d(s), L, keep_pct, sink, window, _l(out))
    return out[:n].copy()


# ------------------------------------------------------------------ a6: attention
def attend(q, K, V, idx, scale: float):
    q, K, V = _f64(q), _f64(K), _f64(V)
    idx = np.ascontiguousarray(idx, dtype=np.int64)
    out = np.empty(q.shape[-1], np.float64)
    lse = np.empty(1, np.float64)
    lib().tbo_attend(_d(q), _d(K), _d(V), q.shape[-1], _l(idx), idx.size, scale, _d(out), _d(lse))
    return out, float(lse[0])


# ------------------------------------------------------------------ amortised selection
def reuse_decision(q_now, q_cached, L: int, len0: int, interval: int, tau: float, keep_pct: int, sink: int,
                   window: int) -> bool:
    a, c = _f64(q_now), _f64(q_cached)
    return bool(lib().tbo_reuse_decision(_d(a), _d(c), a.size, L, len0, interval, tau, keep_pct, sink, window))


def reused_set(cached, len0: int, L: int, sink: int, window: int, radius: int) -> np.ndarray:
    c = np.ascontiguousarray(cached, dtype=np.int64)
    out = np.empty(max(L, 1), np.int64)
    n = lib().tbo_reused_set(_l(c), c.size, len0, L, sink, window, radius, _l(out))
    return out[:n].copy()


# ------------------------------------------------------------------ one decode layer
def decode_layer(q, K, V, W_K, q_imp_producer, layer, G, L, keep_pct, sink, window, dense: bool,
                 K_imp=None, heads=None, batches=None, group: bool = False, kimp_storage: str = "f64"):
    """Same contract as the numpy oracle's decode_layer: dicts keyed by
    (b, h) of the selected indices, outputs [D], lse, and fp64 scores (None
    for dense layers)."""
    q = _f64(q)
    B, Hq, D = q.shape
    K, V = _f64(K), _f64(V)
    Hkv, ld = K.shape[1], K.shape[2]
    lens = np.array([L] * B if np.isscalar(L) else list(L), dtype=np.int64)
    heads = list(range(Hq) if heads is None else heads)
    batches = list(range(B) if batches is None else batches)
    rows = np.array([(b, h) for b in batches for h in heads], dtype=np.int32).reshape(-1)
    n_rows = rows.size // 2
    lmax = max(int(lens.max()) if lens.size else 0, 1)
    W = _f64(W_K)
    dimp = W.shape[1]
    qi = _f64(q_imp_producer) if not dense else np.zeros((B * Hq, G, 1, dimp))
    kimp = None if K_imp is None else _f64(K_imp)
    idx = np.empty((n_rows, lmax), np.int64)
    cnt = np.empty(n_rows, np.int64)
    out = np.empty((n_rows, D), np.float64)
    lse = np.empty(n_rows, np.float64)
    sc = None if dense else np.empty((n_rows, lmax), np.float64)
    lib().tbo_decode_layer(_d(q), _d(K), _d(V), _d(W), _d(qi), None if kimp is None else kimp.ctypes.data,
                           0 if kimp is None else kimp.shape[2], B, Hq, Hkv, D, dimp, ld, G, layer, _l(lens),
                           keep_pct, sink, window, int(bool(dense)), int(bool(group)),
                           1 if kimp_storage == "bf16" else 0, rows.ctypes.data_as(_I), n_rows, lmax, _l(idx),
                           _l(cnt), _d(out), _d(lse), None if sc is None else sc.ctypes.data)
    sel, o, l, scores = {}, {}, {}, {}
    for i in range(n_rows):
        b, h = int(rows[2 * i]), int(rows[2 * i + 1])
        sel[b, h] = idx[i, :cnt[i]].copy()
        o[b, h] = out[i].copy()
        l[b, h] = float(lse[i])
        scores[b, h] = None if dense else sc[i, :lens[b]].copy()
    return sel, o, l, scores


# ------------------------------------------------------------------ sequence sharding (R19)
def merge_partials(outs, lses):
    outs = _f64(outs)
    lses = _f64(lses)
    D = outs.shape[-1]
    out = np.empty(outs.shape[1:], np.float64)
    lse = np.empty(1, np.float64)
    lib().tbo_merge_partials(_d(outs), _d(lses), lses.size, D, _d(out), _d(lse))
    return out, float(lse[0])


def decode_layer_sharded(q, K, V, W_K, q_imp_producer, layer, G, L, keep_pct, sink, window, bounds,
                         group: bool = False, kimp_storage: str = "f64", heads=None, batches=None):
    """Reading R19, composed as in the numpy oracle: the unsharded set, each
    rank's attention over its part, the parts merged by log-sum-exp."""
    sel, _, _, _ = decode_layer(q, K, V, W_K, q_imp_producer, layer, G, L, keep_pct, sink, window, dense=False,
                                group=group, kimp_storage=kimp_storage, heads=heads, batches=batches)
    q = _f64(q)
    B, Hq, D = q.shape
    Hkv = K.shape[1]
    lens = [L] * B if np.isscalar(L) else list(L)
    scale = 1.0 / math.sqrt(D)
    out, lse, parts = {}, {}, {}
    for (b, h), idx in sel.items():
        g = kv_head_of(h, Hq, Hkv)
        pieces, outs, lses = [], [], []
        for t0, t1 in bounds:
            mine = idx[(idx >= t0) & (idx < t1)]
            o_r, l_r = attend(q[b, h], K[b, g, :lens[b]], V[b, g, :lens[b]], mine, scale)
            pieces.append(mine)
            outs.append(o_r)
            lses.append(l_r)
        out[b, h], lse[b, h] = merge_partials(outs, lses)
        parts[b, h] = pieces
    return sel, out, lse, parts


# ------------------------------------------------------------------ a7: prefill rows
def prefill_select(q_hat_rows, K_imp, row0: int, keep_pct: int, sink: int, window: int) -> dict:
    q = _f64(q_hat_rows)
    k = _f64(K_imp)
    Hq, nrows, dimp = q.shape
    Hkv = k.shape[0]
    lmax = row0 + nrows
    idx = np.empty((Hq * nrows, lmax), np.int64)
    cnt = np.empty(Hq * nrows, np.int64)
    lib().tbo_prefill_select(_d(q), Hq, nrows, dimp, _d(k), Hkv, k.shape[1], row0, keep_pct, sink, window, _l(idx),
                             _l(cnt))
    return {(h, row0 + r): idx[h * nrows + r, :cnt[h * nrows + r]].copy() for h in range(Hq) for r in range(nrows)}


# ------------------------------------------------------------------ a8: soft voting
def softvote_scores(q, K, L: int) -> np.ndarray:
    q, K = _f64(q), _f64(K)
    Hq, D = q.shape
    votes = np.empty(L, np.float64)
    lib().tbo_softvote_scores(_d(q), Hq, _d(K), K.shape[0], K.shape[1], L, D, _d(votes))
    return votes


def softvote_layer(q, K, V, L, keep_pct, sink, window, batches=None):
    """Soft-voting decode layer (TokenSelect README, per-head soft voting):
    one shared set per sequence, exact attention per head over it."""
    q = _f64(q)
    B, Hq, D = q.shape
    Hkv = K.shape[1]
    lens = [L] * B if np.isscalar(L) else list(L)
    batches = range(B) if batches is None else batches
    sel, out, lse, votes = {}, {}, {}, {}
    for b in batches:
        votes[b] = softvote_scores(q[b], K[b], lens[b])
        sel[b] = select_tokens(votes[b], lens[b], keep_pct, sink, window)
        for h in range(Hq):
            g = kv_head_of(h, Hq, Hkv)
            out[b, h], lse[b, h] = attend(q[b, h], K[b, g, :lens[b]], V[b, g, :lens[b]], sel[b],
                                          1.0 / math.sqrt(D))
    return sel, out, lse, votes
