"""ctypes binding for the plain-C CPU oracle (``kv4_oracle.c`` and ``gtq_oracle.c``).

TEST INFRASTRUCTURE ONLY.  The tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` are the only callers; the product package never imports this module.  It
shares no code with the CUDA library: the byte layout, the quantisers and the attention are
all restated in ``kv4_oracle.c``.

The oracle follows the method pages (KV4-RL, "Methodology in Plain English" paragraphs 2-3
and "Key Contributions" item 4; SAW-INT4 section 2; for the mixed bit-width key cache, "RoPE-Aware
Bit Allocation for KV-Cache Quantization", abstract).  Arrays are NumPy; every call here is
argument marshalling only.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCES = [os.path.join(_HERE, "kv4_oracle.c"), os.path.join(_HERE, "gtq_oracle.c")]
HEADERS = [os.path.join(_HERE, "kv4_oracle.h"), os.path.join(_HERE, "gtq_oracle.h")]
LIB_PATH = os.path.join(_HERE, "liboracle_kv4.so")

CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
          "-msse2", "-mfpmath=sse", "-fopenmp", "-Wall", "-Wextra"]

RN, RD, RU = 0, 1, 2
F32, BF16, F16 = 0, 1, 2
REGIONAL, SINGLE = 0, 1


def build(force: bool = False) -> str:
    """Compile the oracle into ``liboracle_kv4.so`` (skipped when up to date)."""
    if not force and os.path.exists(LIB_PATH):
        lib_t = os.path.getmtime(LIB_PATH)
        if all(lib_t >= os.path.getmtime(f) for f in SOURCES + HEADERS):
            return LIB_PATH
    tmp = LIB_PATH + f".tmp{os.getpid()}"
    subprocess.run(["gcc", *CFLAGS, "-o", tmp, *SOURCES, "-lm"], check=True)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


class _Cfg(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in (
        "num_q_heads", "num_kv_heads", "head_dim", "page_size", "num_sinks",
        "recent_window", "hadamard_block", "max_seqs")] + [("sign_bits", ctypes.c_uint32 * 4),
                                                           ("rotate_values", ctypes.c_int),
                                                           ("value_format", ctypes.c_int)]


@dataclass(frozen=True)
class Config:
    """Cache geometry (same meaning as the library's configuration record)."""
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    page_size: int
    num_sinks: int
    recent_window: int
    hadamard_block: int
    max_seqs: int
    sign_bits: tuple = (0, 0, 0, 0)  # randomised-sign rotation (bit d negates dim d); zero = plain
    rotate_values: int = 0  # values stored rotated like the keys
    value_format: int = 0  # 0: INT4 values; 1: bf16 values (keys as in 0)

    def c(self) -> _Cfg:
        return _Cfg(self.num_q_heads, self.num_kv_heads, self.head_dim, self.page_size,
                    self.num_sinks, self.recent_window, self.hadamard_block, self.max_seqs,
                    (ctypes.c_uint32 * 4)(*[int(x) & 0xFFFFFFFF for x in (list(self.sign_bits) + [0] * 4)[:4]]),
                    int(self.rotate_values), int(self.value_format))


class _GtqCfg(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in (
        "num_q_heads", "num_kv_heads", "head_dim", "page_size", "key_bits", "value_bits")]


@dataclass(frozen=True)
class GtqConfig:
    """Mixed bit-width key cache: key_bits average bits per key dimension (allocated per RoPE
    block), value_bits bits per value dimension."""
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    page_size: int
    key_bits: int
    value_bits: int

    def c(self) -> _GtqCfg:
        return _GtqCfg(self.num_q_heads, self.num_kv_heads, self.head_dim, self.page_size,
                       self.key_bits, self.value_bits)


_lib = None


def lib():
    global _lib
    if _lib is None:
        # KV4_ORACLE_LIB names an alternative build of this same source (the mutation test
        # compiles deliberately broken copies and checks that the pins reject them).
        path = os.environ.get("KV4_ORACLE_LIB") or build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I = ctypes.c_int
        S = ctypes.c_size_t
        cfgp = ctypes.POINTER(_Cfg)
        L.orc_f32_to_f16.argtypes = [ctypes.c_float, I]
        L.orc_f32_to_f16.restype = ctypes.c_uint16
        L.orc_f16_to_f32.argtypes = [ctypes.c_uint16]
        L.orc_f16_to_f32.restype = ctypes.c_float
        L.orc_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.orc_bf16_to_f32.restype = ctypes.c_float
        L.orc_fwht_f32.argtypes = [P, I, I]
        L.orc_fwht_f64.argtypes = [P, I, I]
        L.orc_rotate_key.argtypes = [ctypes.POINTER(_Cfg), P]
        L.orc_quant_int4.argtypes = [P, I, P, P, P]
        L.orc_quant_int4.restype = I
        L.orc_quant_int8.argtypes = [P, I, P, P]
        L.orc_quant_int8.restype = I
        for n in ("orc_page_bytes", "orc_side_slot_bytes"):
            getattr(L, n).argtypes = [cfgp]
            getattr(L, n).restype = S
        L.orc_side_tiles.argtypes = [cfgp]
        L.orc_side_tiles.restype = I
        L.orc_f32_to_bf16.argtypes = [ctypes.c_float]
        L.orc_f32_to_bf16.restype = ctypes.c_uint16
        for n in ("orc_k4_byte", "orc_v4_byte", "orc_p4_byte", "orc_k8_byte", "orc_v8_byte", "orc_s8_byte",
                  "orc_vb_byte", "orc_vb8_byte"):
            getattr(L, n).argtypes = [cfgp, I, I, I, I]
            getattr(L, n).restype = S
        L.orc_k4_high.argtypes = [cfgp, I, I]
        L.orc_k4_high.restype = I
        L.orc_append.argtypes = [cfgp, P, P, I, P, I, P, I, P, P, P, P, I]
        L.orc_append.restype = I
        L.orc_dequant_seq.argtypes = [cfgp, P, P, P, I, I, I, P, P, P]
        L.orc_dequant_seq.restype = I
        L.orc_decode.argtypes = [cfgp, P, P, I, P, I, P, I, P, P, P, I, I, I, I]
        L.orc_decode.restype = I
        gcp = ctypes.POINTER(_GtqCfg)
        L.orc_gtq_energy.argtypes = [I, I, I, P, I, P]
        L.orc_gtq_allocate.argtypes = [P, I, I, P]
        L.orc_gtq_allocate.restype = I
        L.orc_gtq_objective.argtypes = [P, I, P]
        L.orc_gtq_objective.restype = ctypes.c_double
        L.orc_gtq_scales.argtypes = [P, I, I, P]
        L.orc_gtq_quant_key.argtypes = [P, I, P, P, P, P]
        L.orc_gtq_quant_key.restype = I
        L.orc_gtq_dequant_key.argtypes = [ctypes.c_uint16, ctypes.c_float, I, I]
        L.orc_gtq_dequant_key.restype = ctypes.c_double
        L.orc_gtq_quant_value.argtypes = [P, I, I, P, P, P]
        L.orc_gtq_quant_value.restype = I
        L.orc_gtq_dequant_value.argtypes = [ctypes.c_uint16, ctypes.c_uint16, I, I]
        L.orc_gtq_dequant_value.restype = ctypes.c_double
        L.orc_gtq_pack.argtypes = [P, P, I, P]
        L.orc_gtq_unpack.argtypes = [P, P, I, P]
        for n in ("orc_gtq_key_row_bytes", "orc_gtq_value_row_bytes", "orc_gtq_tile_bytes", "orc_gtq_page_bytes"):
            getattr(L, n).argtypes = [gcp]
            getattr(L, n).restype = S
        for n in ("orc_gtq_key_row", "orc_gtq_value_row", "orc_gtq_param"):
            getattr(L, n).argtypes = [gcp, I, I, I]
            getattr(L, n).restype = S
        L.orc_gtq_append.argtypes = [gcp, P, P, P, I, P, I, P, I, P, P, P, I]
        L.orc_gtq_append.restype = I
        L.orc_gtq_dequant_seq.argtypes = [gcp, P, P, P, P, I, I, P, P]
        L.orc_gtq_dequant_seq.restype = I
        L.orc_gtq_decode.argtypes = [gcp, P, P, P, I, P, I, P, I, P, P, P, I]
        L.orc_gtq_decode.restype = I
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


# ---------------------------------------------------------------- scalar helpers

def f32_to_f16(x: float, mode: int = RN) -> int:
    return int(lib().orc_f32_to_f16(ctypes.c_float(float(x)), mode))


def f16_to_f32(bits: int) -> float:
    return float(lib().orc_f16_to_f32(ctypes.c_uint16(int(bits))))


def bf16_to_f32(bits: int) -> float:
    return float(lib().orc_bf16_to_f32(ctypes.c_uint16(int(bits))))


def f32_to_bf16(x: float) -> int:
    return int(lib().orc_f32_to_bf16(ctypes.c_float(float(x))))


def fwht_f32(x: np.ndarray, h: int) -> np.ndarray:
    y = np.ascontiguousarray(x, dtype=np.float32).copy()
    lib().orc_fwht_f32(_p(y), y.size, h)
    return y


def rotate_key(cfg: "Config", x: np.ndarray) -> np.ndarray:
    """The append's key rotation H diag(s) x (fp32)."""
    y = np.ascontiguousarray(x, dtype=np.float32).copy()
    assert y.size == cfg.head_dim
    c = cfg.c()
    lib().orc_rotate_key(ctypes.byref(c), _p(y))
    return y


def fwht_f64(x: np.ndarray, h: int) -> np.ndarray:
    y = np.ascontiguousarray(x, dtype=np.float64).copy()
    lib().orc_fwht_f64(_p(y), y.size, h)
    return y


def quant_int4(x: np.ndarray, with_flag: bool = False):
    """Returns (codes uint8[D], scale_bits, zero_bits), plus the out-of-range flag (a scale or
    zero that is not a finite fp16; the codes are then zero) when with_flag is set."""
    xf = np.ascontiguousarray(x, dtype=np.float32)
    codes = np.zeros(xf.size, np.uint8)
    sc = np.zeros(1, np.uint16)
    zr = np.zeros(1, np.uint16)
    flag = lib().orc_quant_int4(_p(xf), xf.size, _p(codes), _p(sc), _p(zr))
    return (codes, int(sc[0]), int(zr[0]), bool(flag)) if with_flag else (codes, int(sc[0]), int(zr[0]))


def quant_int8(x: np.ndarray, with_flag: bool = False):
    """Returns (codes int8[D], scale_bits), plus the out-of-range flag when with_flag is set."""
    xf = np.ascontiguousarray(x, dtype=np.float32)
    codes = np.zeros(xf.size, np.int8)
    sc = np.zeros(1, np.uint16)
    flag = lib().orc_quant_int8(_p(xf), xf.size, _p(codes), _p(sc))
    return (codes, int(sc[0]), bool(flag)) if with_flag else (codes, int(sc[0]))


# ---------------------------------------------------------------- cache-level calls

def page_bytes(cfg: Config) -> int:
    return int(lib().orc_page_bytes(ctypes.byref(cfg.c())))


def side_slot_bytes(cfg: Config) -> int:
    return int(lib().orc_side_slot_bytes(ctypes.byref(cfg.c())))


def side_tiles(cfg: Config) -> int:
    return int(lib().orc_side_tiles(ctypes.byref(cfg.c())))


def byte_offset(kind: str, cfg: Config, a: int, g: int, r: int, e: int) -> int:
    """kind in {k4, v4, p4, k8, v8, s8, vb, vb8}; (a, g, r, e) = (page or slot, kv head, position
    in page or side row, element or is_v).  vb / vb8: bf16 values (value_format 1)."""
    return int(getattr(lib(), f"orc_{kind}_byte")(ctypes.byref(cfg.c()), a, g, r, e))


def nibble_high(kind: str, cfg: Config, r: int, e: int) -> int:
    """1 if element e of the INT4 codes at position-in-page r is the high nibble of the byte
    byte_offset(kind, ...) names (kind k4 or v4), else 0."""
    if kind == "k4":
        return int(lib().orc_k4_high(ctypes.byref(cfg.c()), r, e))
    return e & 1


def _dtype_code(a: np.ndarray, declared: int | None) -> int:
    if declared is not None:
        return declared
    if a.dtype == np.float32:
        return F32
    raise TypeError("uint16 inputs need an explicit dtype code (BF16 or F16)")


def append(cfg: Config, pool: np.ndarray, side: np.ndarray, K: np.ndarray, V: np.ndarray,
           seq_slot: np.ndarray, pos: np.ndarray, lens_after: np.ndarray, page_table: np.ndarray,
           k_dtype: int | None = None, v_dtype: int | None = None) -> bool:
    """Append T tokens.  K, V: [T][Hkv][D] float32, or uint16 bit patterns with a dtype code.
    Returns True when some vector's fp16 scale or offset was not finite (stored with zero codes)."""
    K = np.ascontiguousarray(K)
    V = np.ascontiguousarray(V)
    seq_slot = np.ascontiguousarray(seq_slot, np.int32)
    pos = np.ascontiguousarray(pos, np.int32)
    lens_after = np.ascontiguousarray(lens_after, np.int32)
    page_table = np.ascontiguousarray(page_table, np.int32)
    T = int(seq_slot.size)
    rc = lib().orc_append(ctypes.byref(cfg.c()), _p(pool), _p(side), T, _p(K), _dtype_code(K, k_dtype),
                          _p(V), _dtype_code(V, v_dtype), _p(seq_slot), _p(pos), _p(lens_after),
                          _p(page_table), int(page_table.shape[1]))
    if rc < 0:
        raise RuntimeError(f"orc_append failed: {rc}")
    return rc == 1


def dequant_seq(cfg: Config, pool: np.ndarray, side: np.ndarray, page_row: np.ndarray, slot: int,
                L: int, g: int):
    """Dense fp64 (khat [L][D], vhat [L][D], region [L]) of one (sequence, kv head)."""
    D = cfg.head_dim
    khat = np.zeros((L, D), np.float64)
    vhat = np.zeros((L, D), np.float64)
    region = np.zeros(L, np.int32)
    page_row = np.ascontiguousarray(page_row, np.int32)
    rc = lib().orc_dequant_seq(ctypes.byref(cfg.c()), _p(pool), _p(side), _p(page_row), slot, L, g,
                               _p(khat), _p(vhat), _p(region))
    if rc != 0:
        raise RuntimeError(f"orc_dequant_seq failed: {rc}")
    return khat, vhat, region


def decode(cfg: Config, pool: np.ndarray, side: np.ndarray, q: np.ndarray, page_table: np.ndarray,
           lens: np.ndarray, mode: int = REGIONAL, chunk_tokens: int = 0, reverse: bool = False,
           q_dtype: int | None = None, nthreads: int = 1):
    """Decode attention for B = len(lens) sequences; returns (out [B][Hq][D], lse [B][Hq])."""
    q = np.ascontiguousarray(q)
    lens = np.ascontiguousarray(lens, np.int32)
    page_table = np.ascontiguousarray(page_table, np.int32)
    B = int(lens.size)
    out = np.zeros((B, cfg.num_q_heads, cfg.head_dim), np.float64)
    lse = np.zeros((B, cfg.num_q_heads), np.float64)
    rc = lib().orc_decode(ctypes.byref(cfg.c()), _p(pool), _p(side), B, _p(q), _dtype_code(q, q_dtype),
                          _p(page_table), int(page_table.shape[1]), _p(lens), _p(out), _p(lse), mode,
                          int(chunk_tokens), int(bool(reverse)), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"orc_decode failed: {rc}")
    return out, lse


# ---------------------------------------------------------------- mixed bit-width key cache

def gtq_energy(K: np.ndarray, k_dtype: int | None = None) -> np.ndarray:
    """Energy score [Hkv][D/2] of keys K [T][Hkv][D] (float32, or uint16 with a dtype code)."""
    K = np.ascontiguousarray(K)
    T, Hkv, D = K.shape
    E = np.zeros((Hkv, D // 2), np.float64)
    lib().orc_gtq_energy(T, Hkv, D, _p(K), _dtype_code(K, k_dtype), _p(E))
    return E


def gtq_allocate(energy: np.ndarray, key_bits: int) -> np.ndarray:
    """Greedy block widths (uint8) for one head's energies [D/2]."""
    e = np.ascontiguousarray(energy, np.float64)
    w = np.zeros(e.size, np.uint8)
    if lib().orc_gtq_allocate(_p(e), e.size, int(key_bits), _p(w)) != 0:
        raise ValueError("budget above 8 bits per dimension")
    return w


def gtq_objective(energy: np.ndarray, widths: np.ndarray) -> float:
    e = np.ascontiguousarray(energy, np.float64)
    w = np.ascontiguousarray(widths, np.uint8)
    return float(lib().orc_gtq_objective(_p(e), e.size, _p(w)))


def gtq_scales(energy: np.ndarray, T: int) -> np.ndarray:
    """Block scales (float32) of one head's energies [D/2] scored over T keys."""
    e = np.ascontiguousarray(energy, np.float64)
    sig = np.zeros(e.size, np.float32)
    lib().orc_gtq_scales(_p(e), e.size, int(T), _p(sig))
    return sig


def gtq_quant_key(x: np.ndarray, wc: np.ndarray, sc: np.ndarray):
    """(codes uint8[D], scale_bits, out_of_range) of one key with widths wc[D], scales sc[D]."""
    xf = np.ascontiguousarray(x, dtype=np.float32)
    w = np.ascontiguousarray(wc, np.uint8)
    s = np.ascontiguousarray(sc, np.float32)
    codes = np.zeros(xf.size, np.uint8)
    sb = np.zeros(1, np.uint16)
    flag = lib().orc_gtq_quant_key(_p(xf), xf.size, _p(w), _p(s), _p(codes), _p(sb))
    return codes, int(sb[0]), bool(flag)


def gtq_dequant_key(scale: int, sigma: float, w: int, code: int) -> float:
    return float(lib().orc_gtq_dequant_key(ctypes.c_uint16(scale), ctypes.c_float(sigma), int(w), int(code)))


def gtq_quant_value(x: np.ndarray, bits: int):
    """(codes uint8[D], zero_bits, range_bits, out_of_range) of one value."""
    xf = np.ascontiguousarray(x, dtype=np.float32)
    codes = np.zeros(xf.size, np.uint8)
    z = np.zeros(1, np.uint16)
    r = np.zeros(1, np.uint16)
    flag = lib().orc_gtq_quant_value(_p(xf), xf.size, int(bits), _p(codes), _p(z), _p(r))
    return codes, int(z[0]), int(r[0]), bool(flag)


def gtq_dequant_value(zero: int, rng: int, bits: int, code: int) -> float:
    return float(lib().orc_gtq_dequant_value(ctypes.c_uint16(zero), ctypes.c_uint16(rng), int(bits), int(code)))


def gtq_pack(codes: np.ndarray, wc: np.ndarray) -> np.ndarray:
    c = np.ascontiguousarray(codes, np.uint8)
    w = np.ascontiguousarray(wc, np.uint8)
    row = np.zeros((int(w.sum()) + 7) // 8, np.uint8)
    lib().orc_gtq_pack(_p(c), _p(w), c.size, _p(row))
    return row


def gtq_unpack(row: np.ndarray, wc: np.ndarray) -> np.ndarray:
    r = np.ascontiguousarray(row, np.uint8)
    w = np.ascontiguousarray(wc, np.uint8)
    codes = np.zeros(w.size, np.uint8)
    lib().orc_gtq_unpack(_p(r), _p(w), w.size, _p(codes))
    return codes


def gtq_sizes(cfg: GtqConfig) -> dict:
    c = cfg.c()
    L = lib()
    return {n: int(getattr(L, f"orc_gtq_{n}")(ctypes.byref(c)))
            for n in ("key_row_bytes", "value_row_bytes", "tile_bytes", "page_bytes")}


def gtq_offset(kind: str, cfg: GtqConfig, page: int, g: int, pp: int) -> int:
    """kind in {key_row, value_row, param}: byte offset in the page pool."""
    return int(getattr(lib(), f"orc_gtq_{kind}")(ctypes.byref(cfg.c()), page, g, pp))


def gtq_append(cfg: GtqConfig, widths: np.ndarray, sigma: np.ndarray, pool: np.ndarray, K: np.ndarray,
               V: np.ndarray, seq_slot: np.ndarray, pos: np.ndarray, page_table: np.ndarray,
               k_dtype: int | None = None, v_dtype: int | None = None) -> bool:
    """Append T tokens with block widths [Hkv][D/2] and block scales [Hkv][D/2].  Returns the
    out-of-range flag."""
    K = np.ascontiguousarray(K)
    V = np.ascontiguousarray(V)
    widths = np.ascontiguousarray(widths, np.uint8)
    seq_slot = np.ascontiguousarray(seq_slot, np.int32)
    pos = np.ascontiguousarray(pos, np.int32)
    page_table = np.ascontiguousarray(page_table, np.int32)
    sigma = np.ascontiguousarray(sigma, np.float32)
    rc = lib().orc_gtq_append(ctypes.byref(cfg.c()), _p(widths), _p(sigma), _p(pool), int(seq_slot.size), _p(K),
                              _dtype_code(K, k_dtype), _p(V), _dtype_code(V, v_dtype), _p(seq_slot), _p(pos),
                              _p(page_table), int(page_table.shape[1]))
    if rc < 0:
        raise RuntimeError(f"orc_gtq_append failed: {rc}")
    return rc == 1


def gtq_dequant_seq(cfg: GtqConfig, widths: np.ndarray, sigma: np.ndarray, pool: np.ndarray, page_row: np.ndarray,
                    L: int, g: int):
    D = cfg.head_dim
    khat = np.zeros((L, D), np.float64)
    vhat = np.zeros((L, D), np.float64)
    rc = lib().orc_gtq_dequant_seq(ctypes.byref(cfg.c()), _p(np.ascontiguousarray(widths, np.uint8)),
                                   _p(np.ascontiguousarray(sigma, np.float32)), _p(pool),
                                   _p(np.ascontiguousarray(page_row, np.int32)), L, g, _p(khat), _p(vhat))
    if rc != 0:
        raise RuntimeError(f"orc_gtq_dequant_seq failed: {rc}")
    return khat, vhat


def gtq_decode(cfg: GtqConfig, widths: np.ndarray, sigma: np.ndarray, pool: np.ndarray, q: np.ndarray,
               page_table: np.ndarray, lens: np.ndarray, q_dtype: int | None = None, nthreads: int = 1):
    """Decode attention; returns (out [B][Hq][D], lse [B][Hq])."""
    q = np.ascontiguousarray(q)
    lens = np.ascontiguousarray(lens, np.int32)
    page_table = np.ascontiguousarray(page_table, np.int32)
    B = int(lens.size)
    out = np.zeros((B, cfg.num_q_heads, cfg.head_dim), np.float64)
    lse = np.zeros((B, cfg.num_q_heads), np.float64)
    rc = lib().orc_gtq_decode(ctypes.byref(cfg.c()), _p(np.ascontiguousarray(widths, np.uint8)),
                              _p(np.ascontiguousarray(sigma, np.float32)), _p(pool), B, _p(q),
                              _dtype_code(q, q_dtype), _p(page_table), int(page_table.shape[1]), _p(lens),
                              _p(out), _p(lse), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"orc_gtq_decode failed: {rc}")
    return out, lse
