"""Seeded random geometries, both cache formats, on the GPU against the CPU oracle.

Each case draws its geometry from a fixed seed: head dim 64 or 128, GQA group 1, 2 or 4, 1-4 KV
heads, page size 16-64, sinks and recent window (INT4 cache) or key / value bits (mixed cache),
Hadamard block, input dtypes, 1-6 sequences with ragged lengths including empty and one-token
ones.  The cache is filled with one prefill call, then a few single-token steps.  Every page
byte (and side-cache byte) must equal the oracle's, and the decode after each step must be
within the library's output tolerance of the oracle's fp64 attention.
"""
import dataclasses

import numpy as np
import pytest
import torch

from int4_kv_cache_append_b200 import workload as W
from oracle import oracle as O

import kv4_testlib as T

pytestmark = pytest.mark.gpu

N_CASES = 40


def _draw(seed: int, mixed: bool):
    r = np.random.default_rng(1000 + seed + (500 if mixed else 0))
    D = int(r.choice([64, 128]))
    G = int(r.choice([1, 2, 4]))
    Hkv = int(r.integers(1, 5))
    P = int(r.choice([16, 32, 48, 64]))
    B = int(r.integers(1, 7))
    lens = [int(x) for x in r.choice([0, 1, 2, 15, 16, 17, 33, 100, 250, 400], size=B)]
    if max(lens) == 0:
        lens[0] = 37
    dt = W.BF16 if r.random() < 0.5 else W.F32
    qdt = W.BF16 if r.random() < 0.7 else W.F32
    if mixed:
        s = w = 0
        h = 1
    else:
        s = int(r.choice([0, 1, 4, 16]))
        w = int(r.choice([0, 5, 32, 128]))
        h = int(r.choice([h for h in (1, 2, 8, 32, 64, 128) if h <= D]))
    grow = 3
    wl = W.make_workload(f"fuzz{'m' if mixed else ''}{seed}", 200 + seed, 1, B, G * Hkv, Hkv, D, P, s, w, h,
                         lambda _r: list(lens), dt, dt, qdt, 2, float(r.choice([1.0, 4.0, 15.0])), grow=grow)
    if mixed:
        wl = dataclasses.replace(wl, rope_outliers=True)
    kb = int(r.integers(1, 9))
    vb = int(r.choice([2, 3, 4, 8]))
    return wl, kb, vb, grow


def _kd(wl):
    return O.BF16 if wl.k_dtype == W.BF16 else O.F32


def _vd(wl):
    return O.BF16 if wl.v_dtype == W.BF16 else O.F32


def _steps(wl, grow):
    """(b, pos, lens_after) of the single-token steps after the prefill: every non-empty sequence
    grows by one token per step."""
    lens = np.asarray(wl.lens, np.int32).copy()
    out = []
    for _ in range(grow):
        rows = np.nonzero(lens > 0)[0].astype(np.int32)
        pos = lens[rows].astype(np.int32)
        lens[rows] += 1
        out.append((rows, pos, lens.copy()))
    return out


@pytest.mark.parametrize("seed", range(N_CASES))
def test_fuzz_int4_cache(seed):
    from int4_kv_cache_append_b200 import kv4
    wl, _, _, grow = _draw(seed, mixed=False)
    lens = np.asarray(wl.lens, np.int32)
    geo = kv4.Geometry(1, wl.Hq, wl.Hkv, wl.D, wl.P, wl.s, wl.w, wl.h, wl.B, max(wl.num_pages, 1))
    cache = kv4.Cache(geo, fill=0xA5)
    cfg = O.Config(wl.Hq, wl.Hkv, wl.D, wl.P, wl.s, wl.w, wl.h, wl.B)
    pool = np.full(O.page_bytes(cfg) * max(wl.num_pages, 1), 0xA5, np.uint8)
    side = np.full(max(O.side_slot_bytes(cfg), 1) * wl.B, 0xA5, np.uint8)
    pt = torch.from_numpy(wl.page_table).cuda()
    b, p = T.prefill_tokens(lens)
    calls = [(b, p, lens.copy())] + _steps(wl, grow)
    for i, (bb, pp, la) in enumerate(calls):
        if bb.size:
            K, V = wl.kv_inputs(0, bb, pp)
            cache.append(0, T.to_dev(K), T.to_dev(V), torch.from_numpy(bb).cuda(), torch.from_numpy(pp).cuda(),
                         torch.from_numpy(la).cuda(), pt)
            O.append(cfg, pool, side, K, V, bb, pp, la, wl.page_table, _kd(wl), _vd(wl))
        q = wl.q_input(0, step=i)
        out, lse = T.gpu_decode(cache, wl, q, lens=la)
        ro, rl = O.decode(cfg, pool, side, q, wl.page_table, la, q_dtype=O.BF16 if q.dtype == np.uint16 else O.F32)
        T.assert_close(out, ro, lse, rl, what=f"{wl.name} call {i}")
    gp, gs = cache.layer_views(0)
    assert np.array_equal(gp.cpu().numpy()[:pool.size], pool), f"{wl.name}: page bytes differ"
    if O.side_slot_bytes(cfg):
        assert np.array_equal(gs.cpu().numpy()[:side.size], side), f"{wl.name}: side bytes differ"
    assert kv4.kv4_get_device_error() == 0


@pytest.mark.parametrize("seed", range(N_CASES))
def test_fuzz_mixed_cache(seed):
    from int4_kv_cache_append_b200 import kv4
    wl, kb, vb, grow = _draw(seed, mixed=True)
    lens = np.asarray(wl.lens, np.int32)
    geo = kv4.Geometry(1, wl.Hq, wl.Hkv, wl.D, wl.P, 0, 0, 1, wl.B, max(wl.num_pages, 1), kv4.KV4_KEYS_MIXED, kb, vb)
    cache = kv4.Cache(geo, fill=0xA5)
    cfg = O.GtqConfig(wl.Hq, wl.Hkv, wl.D, wl.P, kb, vb)
    pool = np.full(O.gtq_sizes(cfg)["page_bytes"] * max(wl.num_pages, 1), 0xA5, np.uint8)
    pt = torch.from_numpy(wl.page_table).cuda()
    b, p = T.prefill_tokens(lens)
    K0, V0 = wl.kv_inputs(0, b, p)
    cache.allocate_key_bits(0, T.to_dev(K0))
    E = O.gtq_energy(K0, _kd(wl))
    widths = np.stack([O.gtq_allocate(E[g], kb) for g in range(wl.Hkv)])
    sigma = np.stack([O.gtq_scales(E[g], K0.shape[0]) for g in range(wl.Hkv)])
    w_gpu, s_gpu = cache.key_allocation(0)
    assert np.array_equal(w_gpu, widths) and np.array_equal(s_gpu.view(np.uint32), sigma.view(np.uint32))
    calls = [(b, p, lens.copy())] + _steps(wl, grow)
    for i, (bb, pp, la) in enumerate(calls):
        if bb.size:
            K, V = wl.kv_inputs(0, bb, pp)
            cache.append(0, T.to_dev(K), T.to_dev(V), torch.from_numpy(bb).cuda(), torch.from_numpy(pp).cuda(),
                         torch.from_numpy(la).cuda(), pt)
            O.gtq_append(cfg, widths, sigma, pool, K, V, bb, pp, wl.page_table, _kd(wl), _vd(wl))
        q = wl.q_input(0, step=i)
        out, lse = T.gpu_decode(cache, wl, q, lens=la)
        ro, rl = O.gtq_decode(cfg, widths, sigma, pool, q, wl.page_table, la,
                              q_dtype=O.BF16 if q.dtype == np.uint16 else O.F32)
        lse_tol = 1e-4 + 2.0 ** -20 * float(np.abs(rl[np.isfinite(rl)]).max(initial=0.0))
        T.assert_close(out, ro, lse, rl, lse_atol=lse_tol, what=f"{wl.name} K{kb}V{vb} call {i}")
    gp, _ = cache.layer_views(0)
    assert np.array_equal(gp.cpu().numpy()[:pool.size], pool), f"{wl.name}: page bytes differ"
    assert kv4.kv4_get_device_error() == 0
