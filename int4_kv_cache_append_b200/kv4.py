"""ctypes binding of libkv4.so (C ABI in include/kv4.h).

Each function has the name of the C entry point it wraps and only marshals arguments: torch
CUDA tensors become device pointers, streams become cudaStream_t handles, and a non-OK status
raises ``KV4Error``.  All computation happens in the CUDA kernels of libkv4.so; there is no
fallback path, and importing this module fails loudly when the library is missing.

``Cache`` and ``BF16Cache`` are conveniences that allocate the caller-owned buffers with torch
(PyTorch is used here for device memory and streams only).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkv4.so")

(KV4_OK, KV4_ERR_INVALID_ARG, KV4_ERR_UNSUPPORTED, KV4_ERR_WORKSPACE, KV4_ERR_CUDA, KV4_ERR_DEVICE,
 KV4_ERR_NO_ALLOCATION) = range(7)
KV4_F32, KV4_BF16, KV4_F16 = 0, 1, 2
KV4_DEVERR_PAGE_RANGE, KV4_DEVERR_WAIT_LIMIT, KV4_DEVERR_LENGTH, KV4_DEVERR_RANGE, KV4_DEVERR_RECORD = 0x1, 0x2, 0x4, 0x8, 0x10

# every entry point declared in include/kv4.h
SYMBOLS = (
    "kv4_query_sizes", "kv4_cache_init", "kv4_cache_destroy", "kv4_append", "kv4_decode_workspace_bytes",
    "kv4_decode_attn", "kv4_decode_attn_static", "kv4_set_decode_overlap", "kv4_debug_force_wait_timeout",
    "kv4_set_rotation_signs", "kv4_set_value_rotation", "kv4_bf16_query_sizes", "kv4_bf16_cache_init",
    "kv4_bf16_append", "kv4_bf16_decode_workspace_bytes", "kv4_bf16_decode_attn", "kv4_get_device_error",
    "kv4_launch_count", "kv4_status_string", "kv4_version", "kv4_allocate_key_bits", "kv4_set_key_allocation",
    "kv4_get_key_allocation", "kv4_debug_mixed_row_copies",
)


class KV4Error(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {status_string(status)} ({status})")
        self.status = status


KV4_VALUES_INT4, KV4_VALUES_BF16, KV4_KEYS_MIXED = 0, 1, 2


class kv4_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in (
        "num_layers", "num_q_heads", "num_kv_heads", "head_dim", "page_size", "num_sinks",
        "recent_window", "hadamard_block", "max_seqs", "max_pages", "value_format", "key_bits", "value_bits")]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing; build it with `python -m int4_kv_cache_append_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I, S, U = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_uint64
    cfgp = ctypes.POINTER(kv4_config)
    i32p = ctypes.c_void_p
    sig = {
        "kv4_query_sizes": (I, [cfgp, ctypes.POINTER(S), ctypes.POINTER(S)]),
        "kv4_cache_init": (I, [cfgp, P, P, ctypes.POINTER(P)]),
        "kv4_cache_destroy": (None, [P]),
        "kv4_append": (I, [P, I, I, P, I, P, I, i32p, i32p, i32p, i32p, I, P]),
        "kv4_decode_workspace_bytes": (I, [P, I, ctypes.POINTER(S)]),
        "kv4_decode_attn": (I, [P, I, I, P, I, i32p, I, i32p, I, P, P, P, S, P]),
        "kv4_decode_attn_static": (I, [P, I, I, P, I, i32p, I, i32p, I, P, P, P]),
        "kv4_set_decode_overlap": (I, [P, I]),
        "kv4_debug_force_wait_timeout": (I, [P, I]),
        "kv4_debug_mixed_row_copies": (I, [P, I]),
        "kv4_set_rotation_signs": (I, [P, P]),
        "kv4_set_value_rotation": (I, [P, I]),
        "kv4_bf16_query_sizes": (I, [cfgp, ctypes.POINTER(S)]),
        "kv4_bf16_cache_init": (I, [cfgp, P, ctypes.POINTER(P)]),
        "kv4_bf16_append": (I, [P, I, I, P, I, P, I, i32p, i32p, i32p, I, P]),
        "kv4_bf16_decode_workspace_bytes": (I, [P, I, ctypes.POINTER(S)]),
        "kv4_bf16_decode_attn": (I, [P, I, I, P, I, i32p, I, i32p, I, P, P, P, S, P]),
        "kv4_get_device_error": (I, [ctypes.POINTER(ctypes.c_uint32)]),
        "kv4_launch_count": (U, []),
        "kv4_status_string": (ctypes.c_char_p, [I]),
        "kv4_version": (I, []),
        "kv4_allocate_key_bits": (I, [P, I, I, P, I, P]),
        "kv4_set_key_allocation": (I, [P, I, P, P, P]),
        "kv4_get_key_allocation": (I, [P, I, P, P, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


lib = _load()


def status_string(status: int) -> str:
    return lib.kv4_status_string(status).decode()


def _check(fn: str, status: int) -> None:
    if status != KV4_OK:
        raise KV4Error(fn, status)


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("device tensor expected")
    if not t.is_contiguous():
        raise ValueError("contiguous tensor expected")
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def dtype_code(t: torch.Tensor) -> int:
    return {torch.float32: KV4_F32, torch.bfloat16: KV4_BF16, torch.float16: KV4_F16}[t.dtype]


# ------------------------------------------------------------------------ C entry points

def kv4_query_sizes(cfg: kv4_config) -> tuple[int, int]:
    pool, side = ctypes.c_size_t(), ctypes.c_size_t()
    _check("kv4_query_sizes", lib.kv4_query_sizes(ctypes.byref(cfg), ctypes.byref(pool), ctypes.byref(side)))
    return pool.value, side.value


def kv4_cache_init(cfg: kv4_config, page_pool, side_cache) -> int:
    h = ctypes.c_void_p()
    _check("kv4_cache_init", lib.kv4_cache_init(ctypes.byref(cfg), _ptr(page_pool), _ptr(side_cache), ctypes.byref(h)))
    return h.value


def kv4_cache_destroy(handle: int) -> None:
    lib.kv4_cache_destroy(handle)


def kv4_append(handle, layer, T, K, k_dtype, V, v_dtype, seq_slot, pos, lens_after, page_table, stride, stream=None):
    _check("kv4_append", lib.kv4_append(handle, layer, T, _ptr(K), k_dtype, _ptr(V), v_dtype, _ptr(seq_slot), _ptr(pos),
                                        _ptr(lens_after), _ptr(page_table), stride, _stream(stream)))


def kv4_decode_workspace_bytes(handle, B) -> int:
    n = ctypes.c_size_t()
    _check("kv4_decode_workspace_bytes", lib.kv4_decode_workspace_bytes(handle, B, ctypes.byref(n)))
    return n.value


def kv4_decode_attn(handle, layer, B, q, q_dtype, page_table, stride, lens, max_len_hint, out, lse, workspace,
                    ws_bytes, stream=None):
    _check("kv4_decode_attn", lib.kv4_decode_attn(handle, layer, B, _ptr(q), q_dtype, _ptr(page_table), stride,
                                                  _ptr(lens), max_len_hint, _ptr(out), _ptr(lse), _ptr(workspace),
                                                  ws_bytes, _stream(stream)))


def kv4_decode_attn_static(handle, layer, B, q, q_dtype, page_table, stride, lens, max_len_hint, out, lse,
                           stream=None):
    """kv4_decode_attn without a workspace argument, for callers that cannot allocate device
    memory: the split partials use the library's static per-GPU scratch array
    (KV4_STATIC_SCRATCH_BYTES = 16 MiB); larger batches are rejected with KV4_ERR_WORKSPACE.
    Calls that overlap on one GPU share that array and must not run concurrently."""
    _check("kv4_decode_attn_static", lib.kv4_decode_attn_static(handle, layer, B, _ptr(q), q_dtype, _ptr(page_table),
                                                                stride, _ptr(lens), max_len_hint, _ptr(out), _ptr(lse),
                                                                _stream(stream)))


KV4_STATIC_SCRATCH_BYTES = 16 << 20


def kv4_set_rotation_signs(handle, sign_bits):
    """Randomised-sign rotation: sign_bits is a sequence of uint32 words (bit d negates dim d before
    the Hadamard), or None to clear it.  Set before the first append."""
    if sign_bits is None:
        _check("kv4_set_rotation_signs", lib.kv4_set_rotation_signs(handle, None))
        return
    arr = (ctypes.c_uint32 * 4)(*[int(x) & 0xFFFFFFFF for x in list(sign_bits)[:4]])
    _check("kv4_set_rotation_signs", lib.kv4_set_rotation_signs(handle, ctypes.cast(arr, ctypes.c_void_p)))


def kv4_set_value_rotation(handle, enable: bool):
    """Store values rotated like the keys; outputs are rotated back.  Set before the first append."""
    _check("kv4_set_value_rotation", lib.kv4_set_value_rotation(handle, 1 if enable else 0))


def kv4_set_decode_overlap(handle, enable: bool):
    """With enable, the decode kernel builds its schedule from lens and page_table while the
    preceding kernel on the stream runs (they must not be written by that kernel)."""
    _check("kv4_set_decode_overlap", lib.kv4_set_decode_overlap(handle, 1 if enable else 0))


def kv4_debug_mixed_row_copies(handle, enable: bool):
    """Test hook (mixed bit-width keys): padded key rows by one bulk copy per row instead of the
    tensor copy, the path taken when the driver's tensor-map encoder is not available."""
    _check("kv4_debug_mixed_row_copies", lib.kv4_debug_mixed_row_copies(handle, 1 if enable else 0))


def kv4_debug_force_wait_timeout(handle, enable: bool):
    """Test hook: with enable, the decode's bounded waits are made to run out (1 ms limit), so the
    device-side failure path runs and KV4_DEVERR_WAIT_LIMIT is reported.  Off by default."""
    _check("kv4_debug_force_wait_timeout", lib.kv4_debug_force_wait_timeout(handle, 1 if enable else 0))


def kv4_allocate_key_bits(handle, layer, T, K, k_dtype, stream=None):
    """Mixed bit-width keys: score the T keys K [T][Hkv][D] per RoPE block and allocate the layer's
    key bits on the device."""
    _check("kv4_allocate_key_bits", lib.kv4_allocate_key_bits(handle, layer, T, _ptr(K), k_dtype, _stream(stream)))


def kv4_set_key_allocation(handle, layer, widths, sigma, stream=None):
    """Mixed bit-width keys: set a layer's allocation from host arrays widths uint8 [Hkv][D/2] and
    sigma float32 [Hkv][D/2] (NumPy)."""
    import numpy as np
    w = np.ascontiguousarray(widths, np.uint8)
    sg = np.ascontiguousarray(sigma, np.float32)
    _check("kv4_set_key_allocation", lib.kv4_set_key_allocation(handle, layer, w.ctypes.data_as(ctypes.c_void_p),
                                                                sg.ctypes.data_as(ctypes.c_void_p), _stream(stream)))


def kv4_get_key_allocation(handle, layer, Hkv, D, stream=None):
    """Mixed bit-width keys: (widths uint8 [Hkv][D/2], sigma float32 [Hkv][D/2]) of a layer."""
    import numpy as np
    w = np.zeros((Hkv, D // 2), np.uint8)
    sg = np.zeros((Hkv, D // 2), np.float32)
    _check("kv4_get_key_allocation", lib.kv4_get_key_allocation(handle, layer, w.ctypes.data_as(ctypes.c_void_p),
                                                                sg.ctypes.data_as(ctypes.c_void_p), _stream(stream)))
    return w, sg


def kv4_bf16_query_sizes(cfg: kv4_config) -> int:
    pool = ctypes.c_size_t()
    _check("kv4_bf16_query_sizes", lib.kv4_bf16_query_sizes(ctypes.byref(cfg), ctypes.byref(pool)))
    return pool.value


def kv4_bf16_cache_init(cfg: kv4_config, page_pool) -> int:
    h = ctypes.c_void_p()
    _check("kv4_bf16_cache_init", lib.kv4_bf16_cache_init(ctypes.byref(cfg), _ptr(page_pool), ctypes.byref(h)))
    return h.value


def kv4_bf16_append(handle, layer, T, K, k_dtype, V, v_dtype, seq_slot, pos, page_table, stride, stream=None):
    _check("kv4_bf16_append", lib.kv4_bf16_append(handle, layer, T, _ptr(K), k_dtype, _ptr(V), v_dtype, _ptr(seq_slot),
                                                  _ptr(pos), _ptr(page_table), stride, _stream(stream)))


def kv4_bf16_decode_workspace_bytes(handle, B) -> int:
    n = ctypes.c_size_t()
    _check("kv4_bf16_decode_workspace_bytes", lib.kv4_bf16_decode_workspace_bytes(handle, B, ctypes.byref(n)))
    return n.value


def kv4_bf16_decode_attn(handle, layer, B, q, q_dtype, page_table, stride, lens, max_len_hint, out, lse, workspace,
                         ws_bytes, stream=None):
    _check("kv4_bf16_decode_attn", lib.kv4_bf16_decode_attn(handle, layer, B, _ptr(q), q_dtype, _ptr(page_table), stride,
                                                            _ptr(lens), max_len_hint, _ptr(out), _ptr(lse),
                                                            _ptr(workspace), ws_bytes, _stream(stream)))


def kv4_get_device_error() -> int:
    v = ctypes.c_uint32()
    _check("kv4_get_device_error", lib.kv4_get_device_error(ctypes.byref(v)))
    return v.value


def kv4_launch_count() -> int:
    return int(lib.kv4_launch_count())


def kv4_version() -> int:
    return int(lib.kv4_version())


# ------------------------------------------------------------------------ conveniences

@dataclass
class Geometry:
    num_layers: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    page_size: int
    num_sinks: int
    recent_window: int
    hadamard_block: int
    max_seqs: int
    max_pages: int
    value_format: int = KV4_VALUES_INT4
    key_bits: int = 0      # KV4_KEYS_MIXED only
    value_bits: int = 0    # KV4_KEYS_MIXED only

    def c(self) -> kv4_config:
        return kv4_config(self.num_layers, self.num_q_heads, self.num_kv_heads, self.head_dim, self.page_size,
                          self.num_sinks, self.recent_window, self.hadamard_block, self.max_seqs, self.max_pages,
                          self.value_format, self.key_bits, self.value_bits)

    def page_bytes(self) -> int:
        """Bytes of one page (all KV heads) of one layer."""
        D, P, H = self.head_dim, self.page_size, self.num_kv_heads
        if self.value_format == KV4_KEYS_MIXED:
            return H * P * ((self.key_bits + self.value_bits) * D // 8 + 8)
        return H * P * (D // 2 + 4 + 2 * D if self.value_format == KV4_VALUES_BF16 else D + 8)


class Cache:
    """INT4 cache with torch-allocated page pool and side cache (uint8 tensors)."""

    def __init__(self, geo: Geometry, device="cuda", fill: int | None = None):
        self.geo = geo
        self.cfg = geo.c()
        pool_b, side_b = kv4_query_sizes(self.cfg)
        self.pool = torch.empty(max(pool_b, 16), dtype=torch.uint8, device=device)
        self.side = torch.empty(max(side_b, 16), dtype=torch.uint8, device=device)
        if fill is not None:
            self.pool.fill_(fill)
            self.side.fill_(fill)
        self.handle = kv4_cache_init(self.cfg, self.pool, self.side)
        self._ws = None

    def layer_views(self, layer: int):
        """(pages of the layer, side cache of the layer) as uint8 views."""
        pool_b, side_b = kv4_query_sizes(self.cfg)
        pl, sl = self.geo.page_bytes() * self.geo.max_pages, side_b // self.geo.num_layers
        return self.pool[layer * pl:(layer + 1) * pl], self.side[layer * sl:(layer + 1) * sl]

    def allocate_key_bits(self, layer, K, stream=None):
        """Mixed bit-width keys: allocate the layer's key bits from keys K [T][Hkv][D]."""
        kv4_allocate_key_bits(self.handle, layer, int(K.shape[0]), K, dtype_code(K), stream)

    def key_allocation(self, layer):
        return kv4_get_key_allocation(self.handle, layer, self.geo.num_kv_heads, self.geo.head_dim)

    def append(self, layer, K, V, seq_slot, pos, lens_after, page_table, stream=None):
        kv4_append(self.handle, layer, int(seq_slot.numel()), K, dtype_code(K), V, dtype_code(V), seq_slot, pos,
                   lens_after, page_table, int(page_table.shape[1]), stream)

    def workspace(self, B: int) -> torch.Tensor:
        n = kv4_decode_workspace_bytes(self.handle, B)
        if self._ws is None or self._ws.numel() < n:
            self._ws = torch.empty(n, dtype=torch.uint8, device=self.pool.device)
        return self._ws

    def decode(self, layer, q, page_table, lens, out=None, lse=None, max_len_hint=0, workspace=None, stream=None):
        B = int(lens.numel())
        if out is None:
            out = torch.empty((B, self.geo.num_q_heads, self.geo.head_dim), dtype=torch.float32, device=q.device)
        ws = workspace if workspace is not None else self.workspace(B)
        kv4_decode_attn(self.handle, layer, B, q, dtype_code(q), page_table, int(page_table.shape[1]), lens,
                        max_len_hint, out, lse, ws, ws.numel(), stream)
        return out

    def close(self):
        if self.handle:
            kv4_cache_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class BF16Cache:
    """BF16-KV baseline cache (same page table conventions, bf16 K and V in the pages)."""

    def __init__(self, geo: Geometry, device="cuda"):
        self.geo = geo
        self.cfg = geo.c()
        self.pool = torch.empty(max(kv4_bf16_query_sizes(self.cfg), 16), dtype=torch.uint8, device=device)
        self.handle = kv4_bf16_cache_init(self.cfg, self.pool)
        self._ws = None

    def append(self, layer, K, V, seq_slot, pos, page_table, stream=None):
        kv4_bf16_append(self.handle, layer, int(seq_slot.numel()), K, dtype_code(K), V, dtype_code(V), seq_slot, pos,
                        page_table, int(page_table.shape[1]), stream)

    def workspace(self, B: int) -> torch.Tensor:
        n = kv4_bf16_decode_workspace_bytes(self.handle, B)
        if self._ws is None or self._ws.numel() < n:
            self._ws = torch.empty(n, dtype=torch.uint8, device=self.pool.device)
        return self._ws

    def decode(self, layer, q, page_table, lens, out=None, lse=None, max_len_hint=0, workspace=None, stream=None):
        B = int(lens.numel())
        if out is None:
            out = torch.empty((B, self.geo.num_q_heads, self.geo.head_dim), dtype=torch.float32, device=q.device)
        ws = workspace if workspace is not None else self.workspace(B)
        kv4_bf16_decode_attn(self.handle, layer, B, q, dtype_code(q), page_table, int(page_table.shape[1]), lens,
                             max_len_hint, out, lse, ws, ws.numel(), stream)
        return out

    def close(self):
        if self.handle:
            kv4_cache_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
