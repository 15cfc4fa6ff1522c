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
