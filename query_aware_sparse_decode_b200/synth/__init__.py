"""Seeded synthetic inputs shaped like Llama-3.1-8B decode (and the smaller
parity cases).  This module only builds inputs: it holds no step of the decode
method.  The same counter-based generator (``synth_core.h``) runs on the host
(``synth_host.c``) and on the device (``synth_dev.cu``) and gives identical
bits on both, so that large caches can be made on the GPU while the oracle
regenerates any slab of them on the CPU.

Value recipe (the model card's notation: D head dim, d' importance dim):

* K, V, the decode query q, the new token's k/v and the importance queries
  q_imp: Irwin-Hall(12) draws, mean 0, variance 1 (an N(0, 1) stand-in).
* W_K: the same draws times fp32(1/sqrt(D)), i.e. variance 1/D.
* Planted heavy hitters: a planted key row gets ``+ delta[b, g]`` where delta
  is chosen (in fp64, then rounded to fp32) so that the planted token's
  importance score rises by 4 standard deviations on average over the query
  heads of its KV group (see :func:`plant_delta`).
* bf16 tensors are rounded from fp32 to nearest even.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, field, replace

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_HOST_LIB = os.path.join(_HERE, "libtbsynth_host.so")
_DEV_LIB = os.path.join(_HERE, "libtbsynth_dev.so")

# tensor kinds (the stream id separates the draws of different tensors)
K_CACHE, V_CACHE, W_K, QUERY, Q_IMP, K_NEW, V_NEW, PLANT = 1, 2, 3, 4, 5, 6, 7, 8

BF16, F32 = 0, 1
_DTYPE_CODE = {"bf16": BF16, "f32": F32}


def stream_id(kind: int, layer: int = 0, step: int = 0) -> int:
    return (kind << 40) | (step << 16) | layer


_host = None
_dev = None


def _host_lib():
    global _host
    if _host is None:
        if not os.path.exists(_HOST_LIB):
            raise RuntimeError(f"{_HOST_LIB} is missing: run __graft_entry__.build() first")
        lib = ctypes.CDLL(_HOST_LIB)
        lib.tbs_fill_host.restype = ctypes.c_int
        lib.tbs_fill_host.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_int64,
                                      ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                      ctypes.c_int64,
                                      ctypes.c_uint64, ctypes.c_float, ctypes.c_void_p, ctypes.c_uint64,
                                      ctypes.c_uint32]
        lib.tbs_planted_host.restype = ctypes.c_int
        lib.tbs_planted_host.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                         ctypes.c_uint64, ctypes.c_uint32]
        lib.tbs_stream_key_host.restype = ctypes.c_uint64
        lib.tbs_stream_key_host.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        _host = lib
    return _host


def _dev_lib():
    global _dev
    if _dev is None:
        if not os.path.exists(_DEV_LIB):
            raise RuntimeError(f"{_DEV_LIB} is missing: run __graft_entry__.build() first")
        lib = ctypes.CDLL(_DEV_LIB)
        lib.tbs_fill_device.restype = ctypes.c_int
        lib.tbs_fill_device.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_longlong,
                                        ctypes.c_longlong,
                                        ctypes.c_longlong, ctypes.c_longlong, ctypes.c_longlong,
                                        ctypes.c_longlong, ctypes.c_ulonglong, ctypes.c_float, ctypes.c_void_p,
                                        ctypes.c_ulonglong, ctypes.c_uint, ctypes.c_void_p]
        _dev = lib
    return _dev


def key(seed: int, stream: int) -> int:
    return int(_host_lib().tbs_stream_key_host(seed, stream))


def fill_host(kind: int, layer: int, step: int, A: int, t0: int, t1: int, C: int, dtype: str,
              scale: float = 1.0, delta: np.ndarray | None = None, plant_mod: int = 0,
              seed: int = 0, a0: int = 0) -> np.ndarray:
    """Array [A][t1 - t0][C] of rows a0 .. a0+A-1: bf16 as uint16 bits, f32 as
    float32.  ``delta`` is indexed by the absolute row a: [a0 + A][C] at least."""
    code = _DTYPE_CODE[dtype]
    out = np.empty((A, t1 - t0, C), dtype=np.uint16 if code == BF16 else np.float32)
    dptr = None
    if delta is not None:
        delta = np.ascontiguousarray(delta, dtype=np.float32).reshape(-1, C)
        if delta.shape[0] < a0 + A:
            raise ValueError("delta has too few rows")
        dptr = delta.ctypes.data
    rc = _host_lib().tbs_fill_host(out.ctypes.data, code, a0, a0 + A, t0, t1, C, (t1 - t0) * C, C,
                                   key(seed, stream_id(kind, layer, step)), np.float32(scale),
                                   dptr, key(seed, stream_id(PLANT, layer)), plant_mod)
    if rc != 0:
        raise ValueError("tbs_fill_host: bad argument")
    return out


def fill_device(tensor, kind: int, layer: int, step: int, A: int, t0: int, t1: int, C: int,
                stride_a: int, stride_t: int, dtype: str, scale: float = 1.0, delta=None,
                plant_mod: int = 0, seed: int = 0, stream=None, dst_t0: int | None = None) -> None:
    """Fill rows t0 <= t < t1 of a device tensor whose element (a, t, c) sits
    at a*stride_a + (t - t0 + dst_t0)*stride_t + c (dst_t0 = t0 by default:
    row t of the tensor holds row t), with the same bits :func:`fill_host`
    gives.  ``delta`` is a device fp32 tensor [A][C] or None."""
    import torch
    if stream is None:
        stream = torch.cuda.current_stream().cuda_stream
    row = t0 if dst_t0 is None else dst_t0
    base = tensor.data_ptr() + row * stride_t * tensor.element_size()  # element (0, t0)
    rc = _dev_lib().tbs_fill_device(ctypes.c_void_p(base), _DTYPE_CODE[dtype], 0, A, t0, t1, C,
                                    stride_a, stride_t, key(seed, stream_id(kind, layer, step)),
                                    np.float32(scale), None if delta is None else ctypes.c_void_p(delta.data_ptr()),
                                    key(seed, stream_id(PLANT, layer)), plant_mod, ctypes.c_void_p(stream))
    if rc != 0:
        raise RuntimeError(f"tbs_fill_device failed with code {rc}")


def planted_flags(layer: int, A: int, t0: int, t1: int, plant_mod: int, seed: int = 0) -> np.ndarray:
    out = np.empty((A, t1 - t0), dtype=np.uint8)
    _host_lib().tbs_planted_host(out.ctypes.data, A, t0, t1, key(seed, stream_id(PLANT, layer)), plant_mod)
    return out.astype(bool)


# ---------------------------------------------------------------- bit helpers
def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))
    return (u >> np.uint64(16)).astype(np.uint16)


def widen(arr: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float64 values of a bf16-bits or fp32 array."""
    if dtype == "bf16":
        return bf16_bits_to_f32(arr).astype(np.float64)
    return np.asarray(arr, dtype=np.float32).astype(np.float64)


# ---------------------------------------------------------------- workloads
@dataclass(frozen=True)
class Workload:
    """Shapes and budget of one synthetic decode workload."""
    name: str
    n_layers: int
    B: int
    Hq: int
    Hkv: int
    D: int
    d_imp: int
    G: int
    L: int                      # cached tokens after the current token is appended
    dtype: str                  # "bf16" | "f32"
    keep_pct: int
    sink: int
    window: int
    dense_layers: tuple = ()    # layers attended densely
    plant: str = "pct1"         # "list8" | "pct1" | "none"
    seed: int = 0
    extra_len: int = 0          # spare cache capacity beyond L
    lens: tuple | None = None   # per-sequence lengths (ragged batch); default all L

    @property
    def max_len(self) -> int:
        return max(self.seq_lens) + self.extra_len

    @property
    def seq_lens(self) -> tuple:
        return tuple(self.lens) if self.lens is not None else (self.L,) * self.B

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


TINY_F32 = Workload("tiny_f32_L512", n_layers=1, B=1, Hq=4, Hkv=2, D=64, d_imp=16, G=1, L=512,
                    dtype="f32", keep_pct=50, sink=4, window=16, plant="list8")
LLAMA8B_L32K = Workload("llama8b_bf16_L32768", n_layers=1, B=1, Hq=32, Hkv=8, D=128, d_imp=32, G=1,
                        L=32768, dtype="bf16", keep_pct=50, sink=16, window=64)
DECODE32_B4_L128K = Workload("decode32_bf16_B4_L131072", n_layers=32, B=4, Hq=32, Hkv=8, D=128, d_imp=32,
                             G=4, L=131072, dtype="bf16", keep_pct=30, sink=16, window=64, dense_layers=(0,))
PREFILL_L32K = Workload("prefill_bf16_L32768", n_layers=32, B=1, Hq=32, Hkv=8, D=128, d_imp=32, G=4,
                        L=32768, dtype="bf16", keep_pct=50, sink=16, window=64, dense_layers=(0,))
SWEEP_LENGTHS = (4096, 16384, 65536, 131072, 262144)
SWEEP_KEEP = (10, 30, 50)


def sweep(L: int, keep_pct: int) -> Workload:
    return Workload(f"sweep_bf16_L{L}_keep{keep_pct}", n_layers=1, B=1, Hq=32, Hkv=8, D=128, d_imp=32, G=1,
                    L=L, dtype="bf16", keep_pct=keep_pct, sink=16, window=64)


# ---------------------------------------------------------------- tensors
def w_k(wl: Workload, layer: int) -> np.ndarray:
    """W_K of one layer, [D][d']: variance 1/D."""
    scale = np.float32(1.0 / np.sqrt(wl.D))
    return fill_host(W_K, layer, 0, 1, 0, wl.D, wl.d_imp, wl.dtype, scale, seed=wl.seed)[0]


def q_imp(wl: Workload, producer: int, step: int = 0, rows: tuple | None = None) -> np.ndarray:
    """Importance queries of one producer, [(B*Hq)][G][n][d'] for the positions
    ``rows = (row0, nrows)`` (default: one decode position, index 0)."""
    row0, n = rows if rows is not None else (0, 1)
    A = wl.B * wl.Hq * wl.G
    arr = fill_host(Q_IMP, producer, step, A, row0, row0 + n, wl.d_imp, wl.dtype, seed=wl.seed)
    return arr.reshape(wl.B * wl.Hq, wl.G, n, wl.d_imp)


def query(wl: Workload, layer: int, step: int = 0) -> np.ndarray:
    """Decode query q, [B][Hq][D]."""
    return fill_host(QUERY, layer, step, 1, 0, wl.B * wl.Hq, wl.D, wl.dtype, seed=wl.seed).reshape(
        wl.B, wl.Hq, wl.D)


def kv_new(wl: Workload, layer: int, step: int = 0) -> tuple[np.ndarray, np.ndarray]:
    """New token's key and value, each [B][Hkv][D]."""
    k = fill_host(K_NEW, layer, step, 1, 0, wl.B * wl.Hkv, wl.D, wl.dtype, seed=wl.seed)
    v = fill_host(V_NEW, layer, step, 1, 0, wl.B * wl.Hkv, wl.D, wl.dtype, seed=wl.seed)
    return k.reshape(wl.B, wl.Hkv, wl.D), v.reshape(wl.B, wl.Hkv, wl.D)


def plant_delta(w_k64: np.ndarray, qhat64: np.ndarray, Hkv: int) -> np.ndarray:
    """Offset added to every planted key row, [B][Hkv][D] float32.

    For query head h let w_h = W_K q_h (length D) and u_h = w_h / |w_h|.  With
    K ~ N(0, I), head h's importance scores over unplanted tokens have standard
    deviation sigma_h = |w_h|, and adding c*v to a key raises head h's score by
    c * sigma_h * (u_h . v).  We take v = normalise(sum_h u_h) over the heads
    of the KV group and c = 4 / mean_h(u_h . v), so the rise is 4 sigma on
    average over the group's heads.  ``qhat64`` is [B][Hq][d'], the importance
    queries the planted tokens should stand out for.
    """
    B, Hq, _ = qhat64.shape
    gs = Hq // Hkv
    out = np.zeros((B, Hkv, w_k64.shape[0]), dtype=np.float32)
    for b in range(B):
        for g in range(Hkv):
            u = []
            for h in range(g * gs, (g + 1) * gs):
                w = w_k64 @ qhat64[b, h]
                u.append(w / np.linalg.norm(w))
            u = np.array(u)
            v = u.sum(axis=0)
            v /= np.linalg.norm(v)
            c = 4.0 / float(np.mean(u @ v))
            out[b, g] = (c * v).astype(np.float32)
    return out


def plant_list8(wl: Workload, layer: int) -> np.ndarray:
    """Eight distinct planted positions in [sink, L - window), the same for
    every KV group: the candidates ordered by a seeded hash, first eight."""
    cand = np.arange(wl.sink, wl.L - wl.window, dtype=np.int64)
    flags_key = key(wl.seed, stream_id(PLANT, layer))
    # order candidates by their hash value (uint64 arithmetic wraps)
    z = np.uint64(flags_key) + cand.astype(np.uint64) * np.uint64(0x9E3779B97F4A7C15)
    z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
    z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
    z = z ^ (z >> np.uint64(31))
    return np.sort(cand[np.argsort(z, kind="stable")[:8]])


def kv_cache_host(wl: Workload, layer: int, which: int, t0: int, t1: int, delta: np.ndarray | None = None,
                  b_range: tuple | None = None) -> np.ndarray:
    """Host copy of cache rows [t0, t1) of K (which=K_CACHE) or V (V_CACHE),
    [nb*Hkv][t1-t0][D] for batches b_range=(b0, nb) (default all).  K rows of
    planted tokens get ``delta`` ([B][Hkv][D]) when given."""
    b0, nb = b_range if b_range is not None else (0, wl.B)
    A = nb * wl.Hkv
    a0 = b0 * wl.Hkv
    plant = which == K_CACHE and delta is not None and wl.plant != "none"
    if plant and wl.plant == "list8":
        raw = fill_host(which, layer, 0, A, t0, t1, wl.D, "f32", seed=wl.seed, a0=a0)
        pos = plant_list8(wl, layer)
        d = np.asarray(delta, dtype=np.float32).reshape(wl.B * wl.Hkv, wl.D)[a0:a0 + A]
        for p in pos:
            if t0 <= p < t1:
                raw[:, p - t0, :] = raw[:, p - t0, :] + d
        return raw if wl.dtype == "f32" else f32_to_bf16_bits(raw)
    if plant:
        dfull = np.asarray(delta, dtype=np.float32).reshape(wl.B * wl.Hkv, wl.D)
        return fill_host(which, layer, 0, A, t0, t1, wl.D, wl.dtype, delta=dfull, plant_mod=100,
                         seed=wl.seed, a0=a0)
    return fill_host(which, layer, 0, A, t0, t1, wl.D, wl.dtype, seed=wl.seed, a0=a0)
