"""Drive full-size synthetic workloads through the C ABI on one GPU.

Inputs are drawn on the device by the counter-based generator (libkv4gen.so, the GPU twin of
``workload.py``), so any sequence can be regenerated on the host for sampled checks.  Every
cache write goes through kv4_append / kv4_bf16_append.
"""
from __future__ import annotations

import numpy as np
import torch

from . import kv4
from . import workload as W


def geometry(wl: W.Workload, layers: int | None = None, value_format: int = kv4.KV4_VALUES_INT4) -> kv4.Geometry:
    mixed = value_format == kv4.KV4_KEYS_MIXED
    return kv4.Geometry(layers or wl.layers, wl.Hq, wl.Hkv, wl.D, wl.P, wl.s, wl.w, wl.h, wl.B, max(wl.num_pages, 1),
                        value_format, wl.key_bits if mixed else 0, wl.value_bits if mixed else 0)


def token_list(lens: np.ndarray, upto=None):
    """(b, pos) of every position [0, L_b) (or [0, upto_b))."""
    ends = np.asarray(lens if upto is None else upto, np.int64)
    b = np.repeat(np.arange(ends.size, dtype=np.int32), ends)
    starts = np.cumsum(ends) - ends
    p = (np.arange(int(ends.sum()), dtype=np.int64) - np.repeat(starts, ends)).astype(np.int32)
    return b, p


def device_kv(wl: W.Workload, layer: int, b: torch.Tensor, p: torch.Tensor, factor: torch.Tensor):
    kK = W.stream_key(wl.seed, W.KIND_K, layer)
    kV = W.stream_key(wl.seed, W.KIND_V, layer)
    K = W.device_token_values(kK, b, p, wl.Hkv, wl.D, factor, wl.k_dtype == W.BF16)
    V = W.device_token_values(kV, b, p, wl.Hkv, wl.D, factor, wl.v_dtype == W.BF16)
    K = K.view(torch.bfloat16) if wl.k_dtype == W.BF16 else K
    V = V.view(torch.bfloat16) if wl.v_dtype == W.BF16 else V
    return K, V


def prefill(cache, wl: W.Workload, layer: int, lens: np.ndarray, upto=None, chunk: int = 65536,
            bf16_pool: bool = False, allocate: bool = False):
    """Append positions [0, upto_b) of every sequence (lens_after = lens) in chunks.  allocate
    (mixed bit-width keys): the layer's key bits are first allocated from the keys of the first
    chunk (up to `chunk` prefill tokens, in sequence order)."""
    dev = cache.pool.device
    b_all, p_all = token_list(lens, upto)
    factor = torch.from_numpy(wl.factor()).to(dev)
    pt = torch.from_numpy(wl.page_table).to(dev)
    la = torch.from_numpy(np.asarray(lens, np.int32)).to(dev)
    for i in range(0, b_all.size, chunk):
        b = torch.from_numpy(b_all[i:i + chunk]).to(dev)
        p = torch.from_numpy(p_all[i:i + chunk]).to(dev)
        K, V = device_kv(wl, layer, b, p, factor)
        if allocate and i == 0:
            cache.allocate_key_bits(layer, K)
        if bf16_pool:
            cache.append(layer, K, V, b, p, pt)
        else:
            cache.append(layer, K, V, b, p, la, pt)
    torch.cuda.synchronize(dev)


def device_q(wl: W.Workload, layer: int, step: int, device) -> torch.Tensor:
    key = W.stream_key(wl.seed, W.KIND_Q, layer, step)
    q = W.device_normal(key, wl.B * wl.Hq * wl.D, 0, wl.q_dtype == W.BF16, device)
    q = q.view(wl.B, wl.Hq, wl.D)
    return q.view(torch.bfloat16) if wl.q_dtype == W.BF16 else q
