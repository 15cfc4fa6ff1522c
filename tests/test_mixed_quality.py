"""Quality of the mixed bit-width key cache against the INT4 cache, measured with the CPU oracle
against unquantised fp64 attention (a report, not a parity gate).

"RoPE-Aware Bit Allocation for KV-Cache Quantization" (searcharxiv abstract): high-energy RoPE
blocks are the sensitive ones and should receive more bits, and a budget allocated that way
preserves the query-key logits better than a uniform one at the same bits.  On keys whose
outliers are whole RoPE blocks (queries scaled alike), the oracle's decode error is measured for
the mixed cache with the energy-driven allocation and with uniform widths at 2, 3 and 4 bits per
key dimension (values at 4 bits), and, for scale, for the INT4 cache with and without the
Hadamard rotation (4 bits per key and value dimension plus parameters).  Run with -s to see the
figures.
"""
import dataclasses

import numpy as np
import pytest

from int4_kv_cache_append_b200 import workload as W
from oracle import oracle as O

LENS = (700, 520, 333, 900)


def _workload(scale: float, seed: int = 11, h: int = 1):
    wl = W.make_workload("mixq", seed, 1, len(LENS), 16, 4, 128, 16, 0, 0, h, lambda r: list(LENS),
                         W.F32, W.F32, W.F32, 4, scale)
    return dataclasses.replace(wl, rope_outliers=True)


def _inputs(wl):
    b = np.concatenate([np.full(L, i, np.int32) for i, L in enumerate(LENS)])
    p = np.concatenate([np.arange(L, dtype=np.int32) for L in LENS])
    K, V = wl.kv_inputs(0, b, p)
    return b, p, K, V, wl.q_input(0)


def _reference(wl, b, K, V, q):
    ref = np.zeros((wl.B, wl.Hq, wl.D))
    for i in range(wl.B):
        rows = np.nonzero(b == i)[0]
        for j in range(wl.Hq):
            g = j // wl.G
            lg = K[rows, g].astype(np.float64) @ q[i, j].astype(np.float64) / np.sqrt(wl.D)
            pr = np.exp(lg - lg.max())
            ref[i, j] = pr @ V[rows, g].astype(np.float64) / pr.sum()
    return ref


def _rel(out, ref):
    return float(np.linalg.norm(out - ref) / np.linalg.norm(ref))


def _mixed_error(wl, kb, vb, uniform: bool):
    b, p, K, V, q = _inputs(wl)
    cfg = O.GtqConfig(wl.Hq, wl.Hkv, wl.D, wl.P, kb, vb)
    E = O.gtq_energy(K)
    sigma = np.stack([O.gtq_scales(E[g], K.shape[0]) for g in range(wl.Hkv)])
    widths = (np.full((wl.Hkv, wl.D // 2), kb, np.uint8) if uniform
              else np.stack([O.gtq_allocate(E[g], kb) for g in range(wl.Hkv)]))
    pool = np.zeros(O.gtq_sizes(cfg)["page_bytes"] * wl.num_pages, np.uint8)
    O.gtq_append(cfg, widths, sigma, pool, K, V, b, p, wl.page_table)
    out, _ = O.gtq_decode(cfg, widths, sigma, pool, q, wl.page_table, np.array(LENS, np.int32))
    return _rel(out, _reference(wl, b, K, V, q))


def _int4_error(wl):
    b, p, K, V, q = _inputs(wl)
    cfg = O.Config(wl.Hq, wl.Hkv, wl.D, wl.P, 0, 0, wl.h, wl.B)
    pool = np.zeros(O.page_bytes(cfg) * wl.num_pages, np.uint8)
    side = np.zeros(max(O.side_slot_bytes(cfg), 1) * wl.B, np.uint8)
    O.append(cfg, pool, side, K, V, b, p, np.array(LENS, np.int32), wl.page_table)
    out, _ = O.decode(cfg, pool, side, q, wl.page_table, np.array(LENS, np.int32))
    return _rel(out, _reference(wl, b, K, V, q))


@pytest.mark.parametrize("scale", [4.0, 8.0])
def test_energy_allocation_beats_uniform_widths(scale):
    wl = _workload(scale)
    rows = []
    for kb in (2, 3, 4):
        e_alloc = _mixed_error(wl, kb, 4, uniform=False)
        e_unif = _mixed_error(wl, kb, 4, uniform=True)
        rows.append((kb, e_alloc, e_unif))
        assert e_alloc < e_unif, (scale, kb, e_alloc, e_unif)
    e_int4 = _int4_error(wl)
    e_int4_h = _int4_error(dataclasses.replace(wl, h=128))
    print(f"\nRoPE-block outliers x{scale:g}: output rel-L2 vs fp64 attention")
    for kb, ea, eu in rows:
        print(f"  mixed K{kb}V4  energy allocation {ea:.4f}  uniform widths {eu:.4f}")
    print(f"  INT4 cache (K4V4 + params)  h=1 {e_int4:.4f}  h=128 {e_int4_h:.4f}")
