"""Thin Python binding of ``libtb.so`` (the C ABI in ``include/tb.h``).

Argument marshalling only: every step of the decode path runs in the CUDA
kernels behind the C ABI.  PyTorch supplies device memory (the workspace and
the caller's tensors) and the current stream.  There is no fallback: a
missing or unloadable ``libtb.so`` raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libtb.so")

TB_OK = 0
TB_BF16, TB_F32 = 0, 1
TB_BUTLER, TB_SOFTVOTE, TB_BUTLER_GROUP = 0, 1, 2
TB_MASK_PER_HEAD, TB_MASK_SHARED, TB_MASK_DENSE, TB_MASK_GROUP = 0, 1, 2, 3
MAX_BATCH = 128
MAX_LAYERS = 64

STATUS_NAMES = {0: "TB_OK", 1: "TB_ERR_INVALID_ARG", 2: "TB_ERR_SHAPE", 3: "TB_ERR_CAPACITY",
                4: "TB_ERR_WORKSPACE", 5: "TB_ERR_CUDA", 6: "TB_ERR_DEVICE_STATUS", 7: "TB_ERR_UNSUPPORTED",
                8: "TB_ERR_STATE"}

# every symbol include/tb.h declares
EXPORTS = ("tb_workspace_size", "tb_init", "tb_bind_layer", "tb_set_seq_lens", "tb_get_seq_lens", "tb_set_budget",
           "tb_append_kv", "tb_project_kimp", "tb_project_kimp_layers", "tb_score", "tb_select", "tb_sparse_attn",
           "tb_sparse_attn_idx", "tb_decode_step", "tb_select_prefill", "tb_softvote_scores", "tb_sparse_attn_static", "tb_trace_events", "tb_launch_count",
           "tb_check_status", "tb_status_string", "tb_destroy", "tb_selftest_bounded_wait", "tb_selection_cache_size",
           "tb_bind_selection_cache", "tb_set_reuse", "tb_copy_step_masks", "tb_bind_layer_paged", "tb_shard_set",
           "tb_shard_hist", "tb_shard_pick", "tb_shard_mask", "tb_sparse_attn_partial", "tb_merge_partials")


class TBError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}")


class Config(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int), ("batch", ctypes.c_int), ("n_q_heads", ctypes.c_int),
                ("n_kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int), ("d_imp", ctypes.c_int),
                ("producer_freq", ctypes.c_int), ("max_len", ctypes.c_int), ("kv_dtype", ctypes.c_int),
                ("keep_pct", ctypes.c_int), ("sink", ctypes.c_int), ("window", ctypes.c_int),
                ("dense_layer_mask", ctypes.c_uint64), ("variant", ctypes.c_int), ("kimp_bf16", ctypes.c_int)]


class CacheView(ctypes.Structure):
    _fields_ = [("k_cache", ctypes.c_void_p), ("v_cache", ctypes.c_void_p), ("batch", ctypes.c_int),
                ("n_q_heads", ctypes.c_int), ("n_kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("max_len", ctypes.c_int), ("kv_dtype", ctypes.c_int), ("lens_host", ctypes.POINTER(ctypes.c_int32))]


_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is missing: build it with __graft_entry__.build()")
        L = ctypes.CDLL(_LIB_PATH)
        vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        P = ctypes.POINTER
        sig = {
            "tb_workspace_size": [P(Config), P(sz)],
            "tb_init": [P(Config), vp, sz, P(vp)],
            "tb_bind_layer": [vp, i32, vp, vp, vp, vp],
            "tb_set_seq_lens": [vp, i32, P(ctypes.c_int32)],
            "tb_get_seq_lens": [vp, i32, P(ctypes.c_int32)],
            "tb_set_budget": [vp, i32, i32, i32],
            "tb_append_kv": [vp, i32, vp, vp, vp],
            "tb_project_kimp": [vp, i32, i32, i32, vp],
            "tb_project_kimp_layers": [vp, i32, i32, i32, i32, vp],
            "tb_score": [vp, i32, vp, vp, vp],
            "tb_select": [vp, i32, vp, i32, vp, i32, vp, vp, vp],
            "tb_sparse_attn": [vp, i32, vp, vp, i32, vp, vp, vp],
            "tb_sparse_attn_idx": [vp, i32, vp, vp, i32, vp, vp, vp, vp],
            "tb_decode_step": [vp, i32, vp, vp, vp, vp, vp, vp],
            "tb_select_prefill": [vp, i32, vp, i32, i32, vp, i32, vp],
            "tb_softvote_scores": [vp, i32, vp, vp, vp],
            "tb_sparse_attn_static": [P(CacheView), vp, vp, i32, vp, vp, vp],
            "tb_trace_events": [vp, P(vp), i32],
            "tb_launch_count": [vp, P(ctypes.c_uint64)],
            "tb_check_status": [vp, P(ctypes.c_uint32)],
            "tb_status_string": [i32],
            "tb_destroy": [vp],
            "tb_selftest_bounded_wait": [vp, ctypes.c_longlong, i32, vp],
            "tb_selection_cache_size": [P(Config), P(sz)],
            "tb_bind_selection_cache": [vp, i32, vp, sz],
            "tb_set_reuse": [vp, ctypes.c_float, i32, i32],
            "tb_copy_step_masks": [vp, vp, sz, vp],
            "tb_bind_layer_paged": [vp, i32, vp, vp, i32, vp, i32, i32, vp, vp],
            "tb_shard_set": [vp, i32, i32, P(ctypes.c_int32)],
            "tb_shard_hist": [vp, i32, vp, i32, vp, vp, vp],
            "tb_shard_pick": [vp, i32, i32, vp, i32, i32, vp, vp],
            "tb_shard_mask": [vp, i32, vp, vp, vp, vp],
            "tb_sparse_attn_partial": [vp, i32, vp, vp, i32, vp, vp],
            "tb_merge_partials": [vp, vp, i32, vp, vp, vp],
        }
        for name, args in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = ctypes.c_int
        L.tb_status_string.restype = ctypes.c_char_p
        L.tb_destroy.restype = None
        _lib = L
    return _lib


def _check(status: int, what: str) -> None:
    if status != TB_OK:
        raise TBError(status, what)


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def make_config(n_layers, batch, n_q_heads, n_kv_heads, head_dim, d_imp, producer_freq, max_len, kv_dtype,
                keep_pct, sink, window, dense_layers=(0,), variant=TB_BUTLER, kimp_dtype="f32") -> Config:
    """kimp_dtype: "f32" (default) or "bf16" (a bf16 K_imp cache; bf16 K/V only)."""
    mask = 0
    for l in dense_layers:
        mask |= 1 << l
    if kimp_dtype not in ("f32", "bf16"):
        raise ValueError(f"kimp_dtype must be 'f32' or 'bf16', not {kimp_dtype!r}")
    return Config(n_layers, batch, n_q_heads, n_kv_heads, head_dim, d_imp, producer_freq, max_len,
                  TB_BF16 if kv_dtype in ("bf16", TB_BF16, torch.bfloat16) else TB_F32, keep_pct, sink, window,
                  mask, variant, 1 if kimp_dtype == "bf16" else 0)


def kimp_cache(cfg: Config, device="cuda", fill=0.0) -> torch.Tensor:
    """A K_imp cache for `cfg` in the library's layout [B][Hkv][max_len/256][d'][256]
    (256-token tiles, dimension-major inside), fp32 or bf16 as cfg says."""
    dt = torch.bfloat16 if cfg.kimp_bf16 else torch.float32
    return torch.full((cfg.batch, cfg.n_kv_heads, cfg.max_len // 256, cfg.d_imp, 256), fill, dtype=dt, device=device)


def workspace_size(cfg: Config) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().tb_workspace_size(ctypes.byref(cfg), ctypes.byref(n)), "tb_workspace_size")
    return n.value


def sparse_attn_static(k_cache, v_cache, lens, n_q_heads, q, mask, mask_mode, out, lse=None, stream=None) -> None:
    """tb_sparse_attn_static: the sparse attention without a context or a
    workspace (its scratch is a static device array inside the library), for
    callers that cannot allocate device memory.  k_cache, v_cache:
    [B][Hkv][max_len][D]; lens: per-sequence token counts."""
    B, Hkv, max_len, D = k_cache.shape
    arr = (ctypes.c_int32 * B)(*[int(x) for x in lens])
    view = CacheView(k_cache.data_ptr(), v_cache.data_ptr(), B, n_q_heads, Hkv, D, max_len,
                     TB_BF16 if k_cache.dtype == torch.bfloat16 else TB_F32, arr)
    _check(lib().tb_sparse_attn_static(ctypes.byref(view), _ptr(q), _ptr(mask), mask_mode, _ptr(out), _ptr(lse),
                                       _stream(stream)), "tb_sparse_attn_static")


class Context:
    """One tb_ctx plus the torch-allocated workspace it uses."""

    def __init__(self, cfg: Config, device=None):
        self.cfg = cfg
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        self.workspace = torch.empty(workspace_size(cfg), dtype=torch.uint8, device=self.device)
        h = ctypes.c_void_p()
        _check(lib().tb_init(ctypes.byref(cfg), _ptr(self.workspace), self.workspace.numel(), ctypes.byref(h)),
               "tb_init")
        self._h = h
        self._keep = {}  # tensors bound to layers stay alive with the context

    # -------------------------------------------------------------- setup
    def _kimp_type_ok(self, kimp_cache) -> None:
        want = torch.bfloat16 if self.cfg.kimp_bf16 else torch.float32
        if kimp_cache.dtype != want:
            raise TypeError(f"K_imp cache must be {want} for this config, got {kimp_cache.dtype}")

    def bind_layer(self, layer: int, k_cache, v_cache, kimp_cache, w_k) -> None:
        self._kimp_type_ok(kimp_cache)
        _check(lib().tb_bind_layer(self._h, layer, _ptr(k_cache), _ptr(v_cache), _ptr(kimp_cache), _ptr(w_k)),
               "tb_bind_layer")
        self._keep[layer] = (k_cache, v_cache, kimp_cache, w_k)

    def set_seq_lens(self, layer: int, lens) -> None:
        arr = (ctypes.c_int32 * self.cfg.batch)(*[int(x) for x in lens])
        _check(lib().tb_set_seq_lens(self._h, layer, arr), "tb_set_seq_lens")

    def seq_lens(self, layer: int) -> list:
        arr = (ctypes.c_int32 * self.cfg.batch)()
        _check(lib().tb_get_seq_lens(self._h, layer, arr), "tb_get_seq_lens")
        return list(arr)

    def set_budget(self, keep_pct: int, sink: int, window: int) -> None:
        _check(lib().tb_set_budget(self._h, keep_pct, sink, window), "tb_set_budget")
        self.cfg.keep_pct, self.cfg.sink, self.cfg.window = keep_pct, sink, window

    # -------------------------------------------------------------- hot path
    def append_kv(self, layer, k_new, v_new, stream=None) -> None:
        _check(lib().tb_append_kv(self._h, layer, _ptr(k_new), _ptr(v_new), _stream(stream)), "tb_append_kv")

    def project_kimp(self, layer, start, count, stream=None) -> None:
        _check(lib().tb_project_kimp(self._h, layer, start, count, _stream(stream)), "tb_project_kimp")

    def project_kimp_layers(self, first_layer, n_layers, start, count, stream=None) -> None:
        _check(lib().tb_project_kimp_layers(self._h, first_layer, n_layers, start, count, _stream(stream)),
               "tb_project_kimp_layers")

    def score(self, layer, q_imp, scores, stream=None) -> None:
        _check(lib().tb_score(self._h, layer, _ptr(q_imp), _ptr(scores), _stream(stream)), "tb_score")

    def select(self, layer, scores, rows_per_seq, idx=None, count=None, mask=None, stream=None) -> None:
        cap = 0 if idx is None else idx.shape[-1]
        _check(lib().tb_select(self._h, layer, _ptr(scores), rows_per_seq, _ptr(idx), cap, _ptr(count), _ptr(mask),
                               _stream(stream)), "tb_select")

    def sparse_attn(self, layer, q, mask, mask_mode, out, lse=None, stream=None) -> None:
        _check(lib().tb_sparse_attn(self._h, layer, _ptr(q), _ptr(mask), mask_mode, _ptr(out), _ptr(lse),
                                    _stream(stream)), "tb_sparse_attn")

    def sparse_attn_idx(self, layer, q, idx, count, out, lse=None, stream=None) -> None:
        """Attention over sets given as index lists: idx [B][Hq][cap], count [B][Hq] (int32)."""
        _check(lib().tb_sparse_attn_idx(self._h, layer, _ptr(q), _ptr(idx), idx.shape[-1], _ptr(count), _ptr(out),
                                        _ptr(lse), _stream(stream)), "tb_sparse_attn_idx")

    def decode_step(self, layer, k_new, v_new, q, q_imp, out, stream=None) -> None:
        _check(lib().tb_decode_step(self._h, layer, _ptr(k_new), _ptr(v_new), _ptr(q), _ptr(q_imp), _ptr(out),
                                    _stream(stream)), "tb_decode_step")

    def select_prefill(self, layer, q_imp_rows, row0, nrows, row_masks, stream=None) -> None:
        _check(lib().tb_select_prefill(self._h, layer, _ptr(q_imp_rows), row0, nrows, _ptr(row_masks),
                                       row_masks.shape[-1], _stream(stream)), "tb_select_prefill")

    def softvote_scores(self, layer, q, votes, stream=None) -> None:
        _check(lib().tb_softvote_scores(self._h, layer, _ptr(q), _ptr(votes), _stream(stream)), "tb_softvote_scores")

    def trace_events(self, events) -> None:
        """events: six torch.cuda.Event(enable_timing=True) (recorded by
        decode_step around its kernels), or None to stop tracing."""
        if events is None:
            _check(lib().tb_trace_events(self._h, None, 0), "tb_trace_events")
            return
        for e in events:
            if e.cuda_event == 0:  # torch creates the CUDA event lazily
                e.record()
        arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
        _check(lib().tb_trace_events(self._h, arr, len(events)), "tb_trace_events")
        self._trace = events

    def bind_layer_paged(self, layer, k_pool, v_pool, page_table, kimp_cache, w_k) -> None:
        """k_pool, v_pool: [pages][Hkv][page_size][D]; page_table: [B][max_pages] int32 (device)."""
        self._kimp_type_ok(kimp_cache)
        num_pages, _, page_size, _ = k_pool.shape
        max_pages = page_table.shape[1]
        _check(lib().tb_bind_layer_paged(self._h, layer, _ptr(k_pool), _ptr(v_pool), num_pages, _ptr(page_table),
                                         page_size, max_pages, _ptr(kimp_cache), _ptr(w_k)), "tb_bind_layer_paged")
        self._keep[layer] = (k_pool, v_pool, page_table, kimp_cache, w_k)

    def selection_cache(self, layer: int):
        """Allocate (zero-filled) and bind layer `layer`'s selection cache;
        returns the tensor, which must stay alive while bound."""
        n = ctypes.c_size_t(0)
        _check(lib().tb_selection_cache_size(ctypes.byref(self.cfg), ctypes.byref(n)), "tb_selection_cache_size")
        buf = torch.zeros(n.value + 256, dtype=torch.uint8, device=self.device)
        off = (-buf.data_ptr()) % 256
        view = buf[off:off + n.value]
        _check(lib().tb_bind_selection_cache(self._h, layer, ctypes.c_void_p(view.data_ptr()), n.value),
               "tb_bind_selection_cache")
        self._keep[("selection_cache", layer)] = buf
        return view

    def step_masks(self, rows: int, stream=None):
        """The last sparse decode step's selection masks, [B][rows][max_len/32] int32."""
        out = torch.zeros((self.cfg.batch, rows, self.cfg.max_len // 32), dtype=torch.int32, device=self.device)
        _check(lib().tb_copy_step_masks(self._h, ctypes.c_void_p(out.data_ptr()), out.numel() * 4, _stream(stream)),
               "tb_copy_step_masks")
        return out

    def set_reuse(self, tau: float, interval: int, radius: int = 0) -> None:
        _check(lib().tb_set_reuse(self._h, ctypes.c_float(tau), interval, radius), "tb_set_reuse")

    # ---- sequence-sharded decode (the step sequence is in shard.py)
    def shard_set(self, layer: int, t0: int, global_lens) -> None:
        arr = (ctypes.c_int32 * self.cfg.batch)(*[int(x) for x in global_lens])
        _check(lib().tb_shard_set(self._h, layer, int(t0), arr), "tb_shard_set")

    def shard_hist(self, layer, scores, pass_, state, hist, stream=None) -> None:
        _check(lib().tb_shard_hist(self._h, layer, _ptr(scores), pass_, _ptr(state), _ptr(hist), _stream(stream)),
               "tb_shard_hist")

    def shard_pick(self, layer, pass_, hist, n_ranks, rank, state, stream=None) -> None:
        _check(lib().tb_shard_pick(self._h, layer, pass_, _ptr(hist), n_ranks, rank, _ptr(state), _stream(stream)),
               "tb_shard_pick")

    def shard_mask(self, layer, scores, state, mask, stream=None) -> None:
        _check(lib().tb_shard_mask(self._h, layer, _ptr(scores), _ptr(state), _ptr(mask), _stream(stream)),
               "tb_shard_mask")

    def sparse_attn_partial(self, layer, q, mask, mask_mode, part, stream=None) -> None:
        _check(lib().tb_sparse_attn_partial(self._h, layer, _ptr(q), _ptr(mask), mask_mode, _ptr(part),
                                            _stream(stream)), "tb_sparse_attn_partial")

    def merge_partials(self, parts, n_parts, out, lse=None, stream=None) -> None:
        _check(lib().tb_merge_partials(self._h, _ptr(parts), n_parts, _ptr(out), _ptr(lse), _stream(stream)),
               "tb_merge_partials")

    def selftest_bounded_wait(self, cycles: int, arrive: bool, stream=None) -> None:
        """Launch the bounded-wait self-test (see include/tb.h); read the
        outcome with check_status() after a synchronisation."""
        _check(lib().tb_selftest_bounded_wait(self._h, int(cycles), 1 if arrive else 0, _stream(stream)),
               "tb_selftest_bounded_wait")

    def launch_count(self) -> int:
        n = ctypes.c_uint64(0)
        _check(lib().tb_launch_count(self._h, ctypes.byref(n)), "tb_launch_count")
        return n.value

    def check_status(self) -> int:
        flags = ctypes.c_uint32(0)
        st = lib().tb_check_status(self._h, ctypes.byref(flags))
        if st not in (TB_OK, 6):
            raise TBError(st, "tb_check_status")
        return flags.value

    def close(self) -> None:
        if getattr(self, "_h", None):
            lib().tb_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
