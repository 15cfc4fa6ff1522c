"""The C ABI library loads and exports every entry point include/kv4.h declares; host-side
validation returns status codes without touching a GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kv4.h")
LIB = os.path.join(ROOT, "int4_kv_cache_append_b200", "libkv4.so")


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB):
        from int4_kv_cache_append_b200 import build
        build.build()
    return ctypes.CDLL(LIB)


def declared_symbols():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(kv4_[a-z0-9_]+)\s*\(", txt)))


def test_header_declares_the_entry_points():
    syms = declared_symbols()
    for must in ("kv4_append", "kv4_decode_attn", "kv4_query_sizes", "kv4_cache_init", "kv4_bf16_decode_attn"):
        assert must in syms


def test_every_declared_symbol_is_exported(lib):
    missing = [s for s in declared_symbols() if not hasattr(lib, s)]
    assert not missing, f"declared in kv4.h but not exported: {missing}"


def test_binding_covers_every_symbol():
    from int4_kv_cache_append_b200 import kv4
    assert sorted(kv4.SYMBOLS) == declared_symbols()


def _cfg(**kw):
    from int4_kv_cache_append_b200 import kv4
    base = dict(num_layers=2, num_q_heads=32, num_kv_heads=8, head_dim=128, page_size=16, num_sinks=4,
                recent_window=128, hadamard_block=128, max_seqs=64, max_pages=100)
    base.update(kw)
    return kv4.kv4_config(**base)


def test_query_sizes_formula(lib):
    from int4_kv_cache_append_b200 import kv4
    pool, side = kv4.kv4_query_sizes(_cfg())
    assert pool == 2 * 100 * 8 * 16 * (128 + 8)
    assert side == 2 * 64 * 8 * ((4 + 128 + 15) // 16) * 16 * (2 * 128 + 4)
    # 4 + 32/128 bits per element: (D/2 + 4) bytes for K (or V) of one token-head
    assert pool / (2 * 100 * 8 * 16 * 2) * 8 / 128 == 4.25
    assert kv4.kv4_bf16_query_sizes(_cfg()) == 2 * 100 * 8 * 16 * 4 * 128


@pytest.mark.parametrize("kw,status", [
    (dict(head_dim=96), 2), (dict(head_dim=256), 2), (dict(num_q_heads=64), 2), (dict(num_q_heads=30), 1),
    (dict(page_size=8), 2), (dict(hadamard_block=48), 1), (dict(hadamard_block=256), 1), (dict(num_sinks=-1), 1),
    (dict(max_pages=0), 1), (dict(num_layers=0), 1),
])
def test_config_validation(lib, kw, status):
    from int4_kv_cache_append_b200 import kv4
    with pytest.raises(kv4.KV4Error) as e:
        kv4.kv4_query_sizes(_cfg(**kw))
    assert e.value.status == status


def test_init_and_host_validation_without_gpu(lib):
    from int4_kv_cache_append_b200 import kv4
    cfg = _cfg()
    # host handle only: fake, aligned device addresses are accepted (nothing is dereferenced)
    h = kv4.kv4_cache_init(cfg, 1 << 20, 1 << 21)
    try:
        # invalid arguments are rejected before any CUDA call
        assert lib.kv4_append(ctypes.c_void_p(h), 5, 1, None, 0, None, 0, None, None, None, None, 1, None) == 1
        assert lib.kv4_append(ctypes.c_void_p(h), 0, -1, None, 0, None, 0, None, None, None, None, 1, None) == 1
        assert lib.kv4_append(ctypes.c_void_p(h), 0, 0, None, 0, None, 0, None, None, None, None, 1, None) == 0
        assert lib.kv4_decode_attn(ctypes.c_void_p(h), 0, 65, None, 1, None, 1, None, 0, None, None, None,
                                   ctypes.c_size_t(0), None) == 1
        assert lib.kv4_decode_attn(ctypes.c_void_p(h), 0, 0, None, 1, None, 1, None, 0, None, None, None,
                                   ctypes.c_size_t(0), None) == 0
        # misaligned pool
        with pytest.raises(kv4.KV4Error):
            kv4.kv4_cache_init(cfg, (1 << 20) + 4, 1 << 21)
        # a BF16 handle is not an INT4 handle
        hb = kv4.kv4_bf16_cache_init(cfg, 1 << 20)
        assert lib.kv4_append(ctypes.c_void_p(hb), 0, 1, None, 0, None, 0, None, None, None, None, 1, None) == 1
        kv4.kv4_cache_destroy(hb)
    finally:
        kv4.kv4_cache_destroy(h)


def test_status_strings(lib):
    from int4_kv_cache_append_b200 import kv4
    assert kv4.status_string(0) == "ok"
    assert "workspace" in kv4.status_string(3)
    assert kv4.kv4_version() >= 100


def _mixed_cfg(**kw):
    base = dict(num_sinks=0, recent_window=0, hadamard_block=1, value_format=2, key_bits=3, value_bits=3)
    base.update(kw)
    return _cfg(**base)


def test_mixed_query_sizes_formula(lib):
    from int4_kv_cache_append_b200 import kv4
    pool, side = kv4.kv4_query_sizes(_mixed_cfg())
    # pages: key_bits*D/8 + value_bits*D/8 + 8 bytes per position and KV head; then one block
    # allocation record per (layer, KV head): D/2 fp32 scales + D/2 uint8 widths, 16-byte padded
    assert pool == 2 * 100 * 8 * 16 * (48 + 48 + 8) + 2 * 8 * 320
    assert side == 0
    pool, _ = kv4.kv4_query_sizes(_mixed_cfg(head_dim=64, key_bits=2, value_bits=8))
    assert pool == 2 * 100 * 8 * 16 * (16 + 64 + 8) + 2 * 8 * 160


@pytest.mark.parametrize("kw,status", [
    (dict(num_sinks=4), 1), (dict(recent_window=16), 1), (dict(hadamard_block=128), 1), (dict(key_bits=0), 1),
    (dict(key_bits=9), 1), (dict(value_bits=5), 2), (dict(value_bits=1), 2), (dict(value_format=3), 1),
])
def test_mixed_config_validation(lib, kw, status):
    from int4_kv_cache_append_b200 import kv4
    with pytest.raises(kv4.KV4Error) as e:
        kv4.kv4_query_sizes(_mixed_cfg(**kw))
    assert e.value.status == status


def test_mixed_host_validation_without_gpu(lib):
    import numpy as np
    from int4_kv_cache_append_b200 import kv4
    h = kv4.kv4_cache_init(_mixed_cfg(), 1 << 20, 0)
    try:
        v = ctypes.c_void_p
        # a layer without a block allocation: append and decode are refused before any launch
        assert lib.kv4_append(v(h), 0, 1, v(16), 0, v(16), 0, v(16), v(16), None, v(16), 1, None) == 6
        assert lib.kv4_decode_attn(v(h), 0, 1, v(16), 1, v(16), 1, v(16), 0, v(16), None, v(16),
                                   ctypes.c_size_t(1 << 30), None) == 6
        with pytest.raises(kv4.KV4Error) as e:
            kv4.kv4_get_key_allocation(h, 0, 8, 128, stream=0)
        assert e.value.status == kv4.KV4_ERR_NO_ALLOCATION
        assert "allocation" in kv4.status_string(6)
        # a caller allocation must spend exactly key_bits * D/2 bits per head, at most 8 per block,
        # with positive finite scales
        w = np.full((8, 64), 3, np.uint8)
        sg = np.ones((8, 64), np.float32)
        for bad_w, bad_s in ((w + 1, sg), (np.where(np.arange(64) == 0, 9, w).astype(np.uint8), sg),
                             (w, np.zeros_like(sg)), (w, np.full_like(sg, np.inf))):
            with pytest.raises(kv4.KV4Error) as e:
                kv4.kv4_set_key_allocation(h, 0, bad_w, bad_s, stream=0)
            assert e.value.status == 1
        # setters of the INT4 cache do not apply
        assert lib.kv4_set_value_rotation(v(h), 1) == 1
        # the row-copy test hook applies to this format only
        assert lib.kv4_debug_mixed_row_copies(v(h), 1) == 0 and lib.kv4_debug_mixed_row_copies(v(h), 0) == 0
        assert lib.kv4_debug_mixed_row_copies(None, 1) == 1
        # the INT4 entry points refuse an allocation call
        h4 = kv4.kv4_cache_init(_cfg(), 1 << 20, 1 << 21)
        assert lib.kv4_allocate_key_bits(v(h4), 0, 0, None, 1, None) == 1
        assert lib.kv4_debug_mixed_row_copies(v(h4), 1) == 1
        kv4.kv4_cache_destroy(h4)
    finally:
        kv4.kv4_cache_destroy(h)
