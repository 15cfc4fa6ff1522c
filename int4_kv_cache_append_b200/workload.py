"""Seeded synthetic workloads for the INT4 KV cache (inputs only: no cache arithmetic here).

This module is the one input generator that both the CUDA path's tests/benchmark and the
CPU oracle's tests use.  It holds none of the method's arithmetic (no rotation, no
quantisation, no attention); it only draws K, V, q, lengths, outlier channels and page
assignments.

Value generator (counter-based, so any element can be regenerated on its own):
  * SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number generators",
    OOPSLA 2014, in the form of Vigna's reference code): output k of the stream whose state
    starts at ``key`` is mix64(key + (k+1) * 0x9E3779B97F4A7C15), with
    mix64(z) = z ^= z>>30; z *= 0xBF58476D1CE4E5B9; z ^= z>>27; z *= 0x94D049BB133111EB; z ^ (z>>31).
  * Normal deviates: the sum of twelve independent uniform 16-bit integers taken from three
    consecutive outputs (outputs 3i, 3i+1, 3i+2 for element i), centred and scaled:
    z = (S - 393210) / 65536.  That is the classical "sum of twelve uniforms" N(0, 1)
    approximation (Irwin-Hall, variance 1); every step is integer arithmetic and the final
    float is exact, so the CPU (NumPy) and the GPU generator (``csrc/kv4gen.cu``) agree bit for
    bit.  The tails are cut at +-6, which synthetic inputs do not need.
  * Outlier channels are multiplied by 15 or 20 (exact in fp32 for these values); bf16 inputs
    are the fp32 values rounded to nearest-even.

Element index of a K or V value: ((b * 2**20 + pos) * Hkv + g) * D + d (stream per layer and
tensor); of a query value: (b * Hq + j) * D + d (stream per layer and decode step).
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass, field

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
M1 = np.uint64(0xBF58476D1CE4E5B9)
M2 = np.uint64(0x94D049BB133111EB)
POS_STRIDE = 1 << 20

KIND_K, KIND_V, KIND_Q = 1, 2, 3
F32, BF16 = "f32", "bf16"


def _mix64(z: np.ndarray) -> np.ndarray:
    z = z.copy()
    z ^= z >> np.uint64(30)
    z *= M1
    z ^= z >> np.uint64(27)
    z *= M2
    z ^= z >> np.uint64(31)
    return z


def splitmix64(key: int, k: np.ndarray) -> np.ndarray:
    """Output k (array, 0-based) of the SplitMix64 stream whose initial state is ``key``."""
    k = np.asarray(k, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix64(np.uint64(key) + (k + np.uint64(1)) * GAMMA)


def stream_key(seed: int, kind: int, layer: int, step: int = 0) -> int:
    """Key of the stream for (seed, tensor kind, layer, decode step)."""
    sel = (int(kind) << 56) | (int(step) << 24) | int(layer)
    return int(splitmix64(int(seed) & 0xFFFFFFFFFFFFFFFF, np.array([sel], np.uint64))[0])


def normal_f32(key: int, idx: np.ndarray, chunk: int = 1 << 16) -> np.ndarray:
    """Approximate N(0,1) deviates (float32, exact multiples of 2**-16) for element indices."""
    idx = np.asarray(idx, dtype=np.uint64).ravel()
    if idx.size > chunk:  # cache-sized pieces: same values, several times faster
        out = np.empty(idx.size, np.float32)
        for i in range(0, idx.size, chunk):
            out[i:i + chunk] = _normal_f32(key, idx[i:i + chunk])
        return out
    return _normal_f32(key, idx)


def _normal_f32(key: int, idx: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        base = idx * np.uint64(3)
    total = np.zeros(idx.shape, np.int64)
    for j in range(3):
        u = splitmix64(key, base + np.uint64(j))
        for sh in (0, 16, 32, 48):
            total += ((u >> np.uint64(sh)) & np.uint64(0xFFFF)).astype(np.int64)
    return ((total - 393210).astype(np.float32) * np.float32(1.0 / 65536.0)).astype(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even); returns the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def token_values(key: int, b: np.ndarray, pos: np.ndarray, Hkv: int, D: int,
                 factor: np.ndarray) -> np.ndarray:
    """K or V inputs [T][Hkv][D] float32 for tokens (b[t], pos[t]); factor [Hkv][D]."""
    b = np.asarray(b, np.int64).reshape(-1, 1, 1)
    pos = np.asarray(pos, np.int64).reshape(-1, 1, 1)
    g = np.arange(Hkv, dtype=np.int64).reshape(1, -1, 1)
    d = np.arange(D, dtype=np.int64).reshape(1, 1, -1)
    idx = ((b * POS_STRIDE + pos) * Hkv + g) * D + d
    z = normal_f32(key, idx).reshape(idx.shape)
    return (z * factor.astype(np.float32)[None]).astype(np.float32)


def query_values(key: int, B: int, Hq: int, D: int) -> np.ndarray:
    idx = np.arange(B * Hq * D, dtype=np.int64)
    return normal_f32(key, idx).reshape(B, Hq, D)


# ---------------------------------------------------------------------------- workloads

@dataclass
class Workload:
    """One synthetic configuration: geometry, lengths, value recipe and page assignment."""
    name: str
    seed: int
    layers: int
    B: int
    Hq: int
    Hkv: int
    D: int
    P: int
    s: int
    w: int
    h: int
    k_dtype: str
    v_dtype: str
    q_dtype: str
    n_outlier: int
    outlier_scale: float
    lens: np.ndarray = field(repr=False)
    max_lens: np.ndarray = field(repr=False)     # capacity per sequence (>= lens)
    outliers: np.ndarray = field(repr=False)     # [Hkv][n_outlier] channel ids
    page_table: np.ndarray = field(repr=False)   # [B][stride] int32
    num_pages: int = 0
    value_format: int = 0                        # 0: INT4 values, 1: bf16 values (K-INT4 / V-BF16)
    rope_outliers: bool = False                  # outliers as whole RoPE blocks, queries scaled alike
    key_bits: int = 0                            # value_format 2 (mixed bit-width keys): average key bits
    value_bits: int = 0                          # value_format 2: value bits per dimension

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def stride(self) -> int:
        return int(self.page_table.shape[1])

    def factor(self) -> np.ndarray:
        """Per-channel multiplier [Hkv][D] of the K and V inputs.  With rope_outliers an outlier
        channel o takes its rotary partner (o + D/2) mod D along, so the outlier is a whole
        two-dimensional RoPE block, as rotary position embedding makes it in real keys."""
        f = np.ones((self.Hkv, self.D), np.float32)
        for g in range(self.Hkv):
            f[g, self.outliers[g]] = np.float32(self.outlier_scale)
            if self.rope_outliers:
                f[g, (self.outliers[g] + self.D // 2) % self.D] = np.float32(self.outlier_scale)
        return f

    def kv_inputs(self, layer: int, b: np.ndarray, pos: np.ndarray):
        """(K, V) inputs for tokens (b, pos) of a layer, as fp32 arrays or bf16 bit arrays."""
        f = self.factor()
        K = token_values(stream_key(self.seed, KIND_K, layer), b, pos, self.Hkv, self.D, f)
        V = token_values(stream_key(self.seed, KIND_V, layer), b, pos, self.Hkv, self.D, f)
        if self.k_dtype == BF16:
            K = bf16_bits(K)
        if self.v_dtype == BF16:
            V = bf16_bits(V)
        return K, V

    def q_input(self, layer: int, step: int = 0, rows: np.ndarray | None = None):
        """Queries [B][Hq][D] (or only the given rows) as fp32 or bf16 bits."""
        q = query_values(stream_key(self.seed, KIND_Q, layer, step), self.B, self.Hq, self.D)
        if self.rope_outliers:  # queries carry the same block outliers as the keys of their head
            q = (q * np.repeat(self.factor(), self.G, axis=0)[None]).astype(np.float32)
        if rows is not None:
            q = q[np.asarray(rows)]
        return bf16_bits(q) if self.q_dtype == BF16 else q.astype(np.float32)

    def kv_bytes_int4(self, lens: np.ndarray | None = None) -> int:
        """Algorithmic KV bytes one decode reads: INT4 region codes + fp16 params, INT8 region
        codes + fp16 scales, K and V, all KV heads (bf16 values: 2D bytes of V per position in
        both regions instead of the V codes and parameters)."""
        L = np.asarray(self.lens if lens is None else lens, np.int64)
        if self.value_format == 2:  # mixed bit-width keys: packed K and V codes + 8 bytes, every position
            return int(self.Hkv * L.sum() * ((self.key_bits + self.value_bits) * self.D // 8 + 8))
        n4 = np.maximum(0, L - self.s - self.w)
        n8 = np.minimum(L, self.s + self.w)
        D = self.D
        b4, b8 = (D // 2 + 4 + 2 * D, 3 * D + 2) if self.value_format else (D + 8, 2 * D + 4)
        return int(self.Hkv * (n4 * b4 + n8 * b8).sum())

    def kv_bytes_bf16(self, lens: np.ndarray | None = None) -> int:
        L = np.asarray(self.lens if lens is None else lens, np.int64)
        return int(self.Hkv * L.sum() * 4 * self.D)


def _assign_pages(rng: np.random.Generator, max_lens: np.ndarray, P: int):
    need = (max_lens + P - 1) // P
    total = int(need.sum())
    perm = rng.permutation(total).astype(np.int32)
    stride = int(need.max())
    table = np.zeros((len(max_lens), stride), np.int32)
    off = 0
    for b, n in enumerate(need):
        table[b, :n] = perm[off:off + n]
        off += n
    return table, total


def make_workload(name: str, seed: int, layers: int, B: int, Hq: int, Hkv: int, D: int, P: int,
                  s: int, w: int, h: int, lens_fn, k_dtype: str, v_dtype: str, q_dtype: str,
                  n_outlier: int, outlier_scale: float, grow: int = 0) -> Workload:
    """Draw order: lengths, outlier channels, page permutation (all from default_rng(seed));
    K, V and q come from the counter-based streams keyed by the same seed."""
    rng = np.random.default_rng(seed)
    lens = np.asarray(lens_fn(rng), np.int64)
    outliers = np.stack([rng.choice(D, n_outlier, replace=False) for _ in range(Hkv)]).astype(np.int64)
    max_lens = lens + grow
    table, total = _assign_pages(rng, max_lens, P)
    return Workload(name, seed, layers, B, Hq, Hkv, D, P, s, w, h, k_dtype, v_dtype, q_dtype,
                    n_outlier, outlier_scale, lens.astype(np.int32), max_lens.astype(np.int32),
                    outliers, table, total)


def tiny_cfg() -> Workload:
    """1 layer, 2 ragged sequences (256, 200), 2 q heads on 1 KV head, D=64, P=16,
    s=4, w=32, h=64, fp32 K/V/q, 2 outlier channels x20."""
    return make_workload("tiny-2x256-D64", 0, 1, 2, 2, 1, 64, 16, 4, 32, 64,
                         lambda r: [256, 200], F32, F32, F32, 2, 20.0)


def qwen3_4b_decode(B: int = 64) -> Workload:
    """32q/8kv, D=128, bf16, lengths lognormal(median 2048, sigma 1) clipped to [1, 8192],
    P=16, s=4, w=128, h=128, 4 outlier channels x15."""
    def lens(r):
        return np.clip(np.rint(r.lognormal(mean=math.log(2048.0), sigma=1.0, size=B)), 1, 8192)
    return make_workload(f"qwen3-4b-decode-B{B}", 1, 1, B, 32, 8, 128, 16, 4, 128, 128, lens,
                         BF16, BF16, BF16, 4, 15.0)


def async_refill(B: int = 256) -> Workload:
    """B=256 slots, 32q/8kv, D=128, lengths ceil(Exp(mean 6144)) clipped to [1, 32768],
    s=4, w=128, h=64, fp32 K, bf16 V and q, 2 outlier channels x20."""
    def lens(r):
        return np.clip(np.ceil(r.exponential(6144.0, size=B)), 1, 32768)
    return make_workload(f"async-refill-B{B}", 2, 1, B, 32, 8, 128, 16, 4, 128, 64, lens,
                         F32, BF16, BF16, 2, 20.0)


def async_refill_snapshot(B: int = 256) -> Workload:
    """The async-refill shape drawn as a step of continuous refill rather than i.i.d. lengths:
    B slots, ceil(Exp(6144)) response lengths capped at 32768, context lengths of the slots at a
    random steady-state step (length-biased responses, uniform position; see concentration.py).
    Other parameters as async_refill."""
    from . import concentration as C

    def lens(r):
        return C.async_snapshot(C.exponential_lengths(6144.0, 32768), B, r, cap=32768)
    return make_workload(f"async-refill-snapshot-B{B}", 5, 1, B, 32, 8, 128, 16, 4, 128, 64, lens,
                         F32, BF16, BF16, 2, 20.0)


def long_context() -> Workload:
    """4 sequences of 32K/64K/128K/128K, 32q/8kv, D=128, P=64, s=4, w=256, h=128."""
    return make_workload("long-context-32k-128k", 3, 1, 4, 32, 8, 128, 64, 4, 256, 128,
                         lambda r: [32768, 65536, 131072, 131072], F32, F32, BF16, 2, 20.0)


def qwen3_8b_loop(B: int = 128, layers: int = 36, h: int = 128, steps: int = 64) -> Workload:
    """36 layers, 32q/8kv, D=128, B=128 lengths U{1024..16384}, s=16, w=128, P=16, bf16."""
    def lens(r):
        return r.integers(1024, 16384, size=B, endpoint=True)
    return make_workload(f"qwen3-8b-loop-h{h}", 4, layers, B, 32, 8, 128, 16, 16, 128, h, lens,
                         BF16, BF16, BF16, 4, 15.0, grow=steps)


WORKLOADS = {
    "tiny": tiny_cfg,
    "qwen3-4b-decode": qwen3_4b_decode,
    "async-refill": async_refill,
    "async-refill-snapshot": async_refill_snapshot,
    "long-context": long_context,
    "qwen3-8b-loop": qwen3_8b_loop,
}


# ---------------------------------------------------------------------------- device generator

_HERE = os.path.dirname(os.path.abspath(__file__))
GEN_LIB = os.path.join(_HERE, "libkv4gen.so")
_gen = None


def _genlib():
    global _gen
    if _gen is None:
        if not os.path.exists(GEN_LIB):
            raise RuntimeError(f"{GEN_LIB} is missing: run __graft_entry__.build()")
        L = ctypes.CDLL(GEN_LIB)
        P, I = ctypes.c_void_p, ctypes.c_int
        L.kv4gen_tokens.argtypes = [P, I, ctypes.c_uint64, P, P, I, I, I, P, P]
        L.kv4gen_tokens.restype = I
        L.kv4gen_normal.argtypes = [P, ctypes.c_int64, ctypes.c_uint64, ctypes.c_int64, I, P]
        L.kv4gen_normal.restype = I
        _gen = L
    return _gen


def device_token_values(key: int, b, pos, Hkv: int, D: int, factor, out_bf16: bool, stream=None):
    """GPU twin of ``token_values`` (same bits): b, pos int32 CUDA tensors [T], factor float32
    CUDA tensor [Hkv][D]; returns a CUDA tensor [T][Hkv][D] (float32, or bf16 bits as int16)."""
    import torch
    T = int(b.numel())
    out = torch.empty((T, Hkv, D), dtype=torch.int16 if out_bf16 else torch.float32, device=b.device)
    st = stream if stream is not None else torch.cuda.current_stream(b.device).cuda_stream
    rc = _genlib().kv4gen_tokens(out.data_ptr(), int(out_bf16), key & 0xFFFFFFFFFFFFFFFF, b.data_ptr(),
                                 pos.data_ptr(), T, Hkv, D, factor.data_ptr(), ctypes.c_void_p(st))
    if rc != 0:
        raise RuntimeError(f"kv4gen_tokens failed ({rc})")
    return out


def device_normal(key: int, n: int, start: int, out_bf16: bool, device):
    """GPU twin of ``normal_f32(key, start + arange(n))``."""
    import torch
    out = torch.empty(n, dtype=torch.int16 if out_bf16 else torch.float32, device=device)
    st = torch.cuda.current_stream(device).cuda_stream
    rc = _genlib().kv4gen_normal(out.data_ptr(), n, key & 0xFFFFFFFFFFFFFFFF, start, int(out_bf16),
                                 ctypes.c_void_p(st))
    if rc != 0:
        raise RuntimeError(f"kv4gen_normal failed ({rc})")
    return out
