"""Helpers shared by the GPU parity tests: build the same cache on the GPU (through the C ABI)
and in the CPU oracle from the same seeded inputs, and compare."""
from __future__ import annotations

import numpy as np
import torch

from int4_kv_cache_append_b200 import workload as W
from oracle import oracle as O

# Output tolerance of the decode attention against the fp64 oracle on the same dequantised cache.
ATOL = 2e-3
REL_L2 = 1e-3
LSE_ATOL = 1e-4


def to_dev(a: np.ndarray) -> torch.Tensor:
    """fp32 array -> float32 CUDA tensor; uint16 array (bf16 bits) -> bfloat16 CUDA tensor."""
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def geometry(wl: W.Workload, max_seqs: int | None = None, layers: int | None = None, value_format: int = 0):
    from int4_kv_cache_append_b200 import kv4
    return kv4.Geometry(layers or wl.layers, wl.Hq, wl.Hkv, wl.D, wl.P, wl.s, wl.w, wl.h,
                        max_seqs or wl.B, max(wl.num_pages, 1), value_format)


def prefill_tokens(lens):
    b = np.concatenate([np.full(int(L), i, np.int32) for i, L in enumerate(lens)] or [np.zeros(0, np.int32)])
    p = np.concatenate([np.arange(int(L), dtype=np.int32) for L in lens] or [np.zeros(0, np.int32)])
    return b, p


def gpu_cache_from_host_inputs(wl: W.Workload, layer: int = 0, step_by_step: bool = False, fill: int = 0xA5,
                               lens=None, signs=None, rotate_values: bool = False, value_format: int = 0):
    """Append every token of the workload through kv4_append (inputs drawn on the host)."""
    from int4_kv_cache_append_b200 import kv4
    lens = np.asarray(wl.lens if lens is None else lens, np.int32)
    cache = kv4.Cache(geometry(wl, value_format=value_format), fill=fill)
    if signs is not None:
        kv4.kv4_set_rotation_signs(cache.handle, signs)
    if rotate_values:
        kv4.kv4_set_value_rotation(cache.handle, True)
    pt = torch.from_numpy(wl.page_table).cuda()
    if not step_by_step:
        b, p = prefill_tokens(lens)
        K, V = wl.kv_inputs(layer, b, p)
        cache.append(layer, to_dev(K), to_dev(V), torch.from_numpy(b).cuda(), torch.from_numpy(p).cuda(),
                     torch.from_numpy(lens).cuda(), pt)
    else:
        cur = np.zeros_like(lens)
        for t in range(int(lens.max())):
            rows = np.nonzero(lens > t)[0].astype(np.int32)
            cur[rows] = t + 1
            p = np.full(rows.size, t, np.int32)
            K, V = wl.kv_inputs(layer, rows, p)
            cache.append(layer, to_dev(K), to_dev(V), torch.from_numpy(rows).cuda(), torch.from_numpy(p).cuda(),
                         torch.from_numpy(cur.copy()).cuda(), pt)
    torch.cuda.synchronize()
    return cache


def oracle_cache(wl: W.Workload, layer: int = 0, step_by_step: bool = False, lens=None, signs=None,
                 rotate_values: bool = False, value_format: int = 0):
    cfg = O.Config(wl.Hq, wl.Hkv, wl.D, wl.P, wl.s, wl.w, wl.h, wl.B,
                   tuple(signs) if signs is not None else (0, 0, 0, 0), int(rotate_values), int(value_format))
    lens = np.asarray(wl.lens if lens is None else lens, np.int32)
    pool = np.full(O.page_bytes(cfg) * max(wl.num_pages, 1), 0xA5, np.uint8)
    side = np.full(O.side_slot_bytes(cfg) * wl.B, 0xA5, np.uint8)
    kd = O.BF16 if wl.k_dtype == W.BF16 else O.F32
    vd = O.BF16 if wl.v_dtype == W.BF16 else O.F32
    if not step_by_step:
        b, p = prefill_tokens(lens)
        K, V = wl.kv_inputs(layer, b, p)
        O.append(cfg, pool, side, K, V, b, p, lens, wl.page_table, kd, vd)
    else:
        cur = np.zeros_like(lens)
        for t in range(int(lens.max())):
            rows = np.nonzero(lens > t)[0].astype(np.int32)
            cur[rows] = t + 1
            p = np.full(rows.size, t, np.int32)
            K, V = wl.kv_inputs(layer, rows, p)
            O.append(cfg, pool, side, K, V, rows, p, cur, wl.page_table, kd, vd)
    return cfg, pool, side


def oracle_decode(wl: W.Workload, cfg, pool, side, q: np.ndarray, lens=None, **kw):
    qd = O.BF16 if q.dtype == np.uint16 else O.F32
    return O.decode(cfg, pool, side, q, wl.page_table, np.asarray(wl.lens if lens is None else lens, np.int32),
                    q_dtype=qd, **kw)


def assert_close(out_gpu: np.ndarray, out_ref: np.ndarray, lse_gpu=None, lse_ref=None, atol=ATOL, rel_l2=REL_L2,
                 lse_atol=LSE_ATOL, what=""):
    diff = np.abs(out_gpu.astype(np.float64) - out_ref)
    max_abs = float(diff.max()) if diff.size else 0.0
    denom = float(np.linalg.norm(out_ref)) or 1.0
    rl2 = float(np.linalg.norm(out_gpu.astype(np.float64) - out_ref)) / denom
    assert max_abs <= atol, f"{what}: max-abs {max_abs:.3e} > {atol}"
    assert rl2 <= rel_l2, f"{what}: rel-L2 {rl2:.3e} > {rel_l2}"
    if lse_gpu is not None:
        finite = np.isfinite(lse_ref)
        assert np.array_equal(finite, np.isfinite(lse_gpu)), f"{what}: lse finiteness differs"
        if finite.any():
            ld = float(np.abs(lse_gpu[finite].astype(np.float64) - lse_ref[finite]).max())
            assert ld <= lse_atol, f"{what}: lse max-abs {ld:.3e} > {lse_atol}"
    return max_abs, rl2


def gpu_decode(cache, wl: W.Workload, q_host: np.ndarray, layer: int = 0, lens=None, max_len_hint: int = 0):
    lens = np.asarray(wl.lens if lens is None else lens, np.int32)
    B = lens.size
    q = to_dev(q_host)
    lse = torch.empty((B, wl.Hq), dtype=torch.float32, device="cuda")
    out = cache.decode(layer, q, torch.from_numpy(wl.page_table).cuda(), torch.from_numpy(lens).cuda(), lse=lse,
                       max_len_hint=max_len_hint)
    torch.cuda.synchronize()
    return out.cpu().numpy(), lse.cpu().numpy()
