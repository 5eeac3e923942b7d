"""The C-ABI library loads on a machine without a GPU, exports every symbol
include/tb.h declares, and rejects bad arguments on the host before any CUDA
call."""
import ctypes
import os
import re

import pytest

from query_aware_sparse_decode_b200 import tb as TB

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "tb.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"TB_API\s+[\w\s\*]+?\b(tb_\w+)\s*\(", text)))


def test_header_declares_the_hot_path_calls():
    names = declared_symbols()
    for n in ("tb_init", "tb_append_kv", "tb_project_kimp", "tb_score", "tb_select", "tb_sparse_attn",
              "tb_decode_step"):
        assert n in names
    assert set(names) == set(TB.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = TB.lib()
    for n in declared_symbols():
        assert hasattr(lib, n), n


def _cfg(**kw):
    base = dict(n_layers=32, batch=4, n_q_heads=32, n_kv_heads=8, head_dim=128, d_imp=32, producer_freq=4,
                max_len=131328, kv_dtype="bf16", keep_pct=30, sink=16, window=64)
    base.update(kw)
    return TB.make_config(**base)


def _ws(cfg):
    n = ctypes.c_size_t(0)
    return TB.lib().tb_workspace_size(ctypes.byref(cfg), ctypes.byref(n)), n.value


def test_workspace_size_and_config_validation():
    st, n = _ws(_cfg())
    assert st == 0
    # scores [B][Hq][max_len] fp32 dominate: 4*32*131328*4 bytes
    assert n >= 4 * 32 * 131328 * 4
    bad = {
        "max_len": (1000, 2), "batch": (0, 2), "n_kv_heads": (5, 2), "head_dim": (96, 7), "d_imp": (48, 7),
        "producer_freq": (0, 2), "keep_pct": (101, 1), "sink": (-1, 1),
    }
    for field, (val, code) in bad.items():
        assert _ws(_cfg(**{field: val}))[0] == code, field
    assert _ws(_cfg(n_q_heads=48, n_kv_heads=4))[0] == 7       # group size 12 unsupported
    assert TB.lib().tb_workspace_size(None, None) == 1


def test_init_rejects_missing_or_small_workspace_without_cuda():
    cfg = _cfg()
    h = ctypes.c_void_p()
    assert TB.lib().tb_init(ctypes.byref(cfg), None, 0, ctypes.byref(h)) == 4
    assert TB.lib().tb_init(ctypes.byref(cfg), ctypes.c_void_p(256), 16, ctypes.byref(h)) == 4
    assert TB.lib().tb_init(ctypes.byref(cfg), ctypes.c_void_p(256), 1 << 40, None) == 1
    assert not h.value


def test_null_context_calls_fail_cleanly():
    L = TB.lib()
    assert L.tb_append_kv(None, 0, None, None, None) == 1
    assert L.tb_score(None, 0, None, None, None) == 1
    assert L.tb_select(None, 0, None, 32, None, 0, None, None, None) == 1
    assert L.tb_sparse_attn(None, 0, None, None, 0, None, None, None) == 1
    assert L.tb_decode_step(None, 0, None, None, None, None, None, None) == 1
    assert L.tb_set_budget(None, 30, 16, 64) == 1
    assert L.tb_check_status(None, None) == 1
    assert L.tb_trace_events(None, None, 0) == 1
    assert L.tb_shard_set(None, 0, 0, None) == 1
    assert L.tb_shard_hist(None, 0, None, 0, None, None, None) == 1
    assert L.tb_shard_pick(None, 0, 0, None, 1, 0, None, None) == 1
    assert L.tb_shard_mask(None, 0, None, None, None, None) == 1
    assert L.tb_sparse_attn_partial(None, 0, None, None, 0, None, None) == 1
    assert L.tb_merge_partials(None, None, 1, None, None, None) == 1
    assert L.tb_bind_layer_paged(None, 0, None, None, 1, None, 64, 1, None, None) == 1
    assert L.tb_set_reuse(None, 0.9, 3, 0) == 1
    L.tb_destroy(None)


def test_kimp_storage_option_validation():
    """bf16 K_imp needs bf16 caches; the flag is 0 or 1."""
    assert _ws(_cfg(kimp_dtype="bf16"))[0] == 0
    assert _ws(_cfg(kimp_dtype="bf16", kv_dtype="f32"))[0] == 7
    cfg = _cfg()
    cfg.kimp_bf16 = 2
    assert TB.lib().tb_workspace_size(ctypes.byref(cfg), ctypes.byref(ctypes.c_size_t(0))) == 1
    with pytest.raises(ValueError):
        _cfg(kimp_dtype="fp8")


def test_status_strings():
    L = TB.lib()
    for code in range(9):
        assert L.tb_status_string(code)
    assert L.tb_status_string(0) == b"ok"
