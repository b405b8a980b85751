"""The C-ABI library loads and exports what include/kvpop.h declares; host-side
validation (no device work, no GPU needed)."""
import ctypes
import os
import re

import pytest

import fixed_budget_kv_kvpop_b200 as kp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(kvpop_\w+)\s*\(", text))
    return names


def test_every_declared_symbol_is_exported():
    declared = _declared_symbols()
    assert declared, "no declarations found"
    for name in declared:
        assert hasattr(kp.lib, name), name
    assert declared == set(kp.EXPORTED_SYMBOLS)


def test_status_strings():
    for code in range(-7, 1):
        assert kp.lib.kvpop_status_string(code).decode() != "unknown status"
    assert kp.lib.kvpop_status_string(-99).decode() == "unknown status"


def _cfg(**kw):
    base = dict(batch=2, n_layers=3, n_q_heads=8, n_kv_heads=2, head_dim=128, sinks=4, window=16, topk=44,
                delay=0, dtype="bf16", scorer_hidden=64, external_scores=True, max_prefill_chunk=256)
    base.update(kw)
    return kp.make_config(**base)


def _bytes(cfg):
    n = ctypes.c_size_t(0)
    return kp.lib.kvpop_cache_bytes(ctypes.byref(cfg), ctypes.byref(n)), n.value


def test_cache_bytes_counts_the_cache():
    st, n = _bytes(_cfg())
    assert st == kp.KVPOP_OK
    units, slots, row = 2 * 2, 4 + 16 + 44, 2 * 128 * 2
    assert n >= 3 * units * slots * (row + 8)


@pytest.mark.parametrize("kw,code", [
    (dict(batch=0), kp.KVPOP_ERR_BAD_SHAPE),
    (dict(n_q_heads=6, n_kv_heads=4), kp.KVPOP_ERR_BAD_SHAPE),
    (dict(window=0), kp.KVPOP_ERR_BAD_SHAPE),
    (dict(topk=-1), kp.KVPOP_ERR_BAD_SHAPE),
    (dict(head_dim=96), kp.KVPOP_ERR_BAD_SHAPE),
    (dict(head_dim=128, dtype="f32"), kp.KVPOP_ERR_BAD_SHAPE),
    (dict(n_q_heads=16, n_kv_heads=2), kp.KVPOP_ERR_BAD_SHAPE),   # G = 8 at d = 128 not built
    (dict(external_scores=False), kp.KVPOP_ERR_INVALID_ARG),       # MLP mode without weights
    (dict(ref_context=8192, compression_ratio=0.75), kp.KVPOP_ERR_INVALID_ARG),  # B=64 != 2048
])
def test_invalid_configs_are_rejected(kw, code):
    st, _ = _bytes(_cfg(**kw))
    assert st == code


def test_compression_ratio_check_accepts_consistent_budget():
    # Qwen3-4B-shaped, 87.5% compression: B = 4 + 128 + 892 = 1024 = (1 - 0.875) * 8192
    st, _ = _bytes(_cfg(sinks=4, window=128, topk=892, ref_context=8192, compression_ratio=0.875))
    assert st == kp.KVPOP_OK


def test_null_arguments():
    assert kp.lib.kvpop_cache_bytes(None, None) == kp.KVPOP_ERR_INVALID_ARG
    h = ctypes.c_void_p()
    cfg = _cfg()
    assert kp.lib.kvpop_create(ctypes.byref(cfg), None, 0, ctypes.byref(h)) == kp.KVPOP_ERR_INVALID_ARG
    assert kp.lib.kvpop_prefill(None, 0, None, None, 0, None, None) == kp.KVPOP_ERR_INVALID_ARG
    assert kp.lib.kvpop_decode_step(None, 0, None, None, None, None, None, None) == kp.KVPOP_ERR_INVALID_ARG
    assert kp.lib.kvpop_destroy(None) == kp.KVPOP_ERR_INVALID_ARG
    assert kp.lib.kvpop_get_error(None, None) == kp.KVPOP_ERR_INVALID_ARG
    n = ctypes.c_size_t(0)
    assert kp.lib.kvpop_prefill_attention_workspace_bytes(None, 16, ctypes.byref(n)) == kp.KVPOP_ERR_INVALID_ARG
    assert kp.lib.kvpop_prefill_attention(None, 0, None, None, None, 16, None, None, None, None, 0,
                                          None) == kp.KVPOP_ERR_INVALID_ARG


def test_create_rejects_host_memory():
    cfg = _cfg()
    st, n = _bytes(cfg)
    buf = ctypes.create_string_buffer(n + 256)
    addr = (ctypes.addressof(buf) + 255) // 256 * 256
    h = ctypes.c_void_p()
    assert kp.lib.kvpop_create(ctypes.byref(cfg), ctypes.c_void_p(addr), n, ctypes.byref(h)) == kp.KVPOP_ERR_INVALID_ARG
    assert not h.value
