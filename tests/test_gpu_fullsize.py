"""Full-size workloads, in the launch configuration the benchmark times, checked on sampled
(sequence, KV head) pairs that the oracle recomputes one by one.

The GPU cache is filled from inputs drawn on the device; for each sampled pair the host
regenerates that head's inputs (counter-based generator), the oracle appends and decodes that
one sequence, and the GPU's page bytes, side-cache bytes and outputs for the pair are compared:
bytes bit-exact, outputs within max-abs 2e-3 / rel-L2 1e-3, lse within 1e-4.
"""
import numpy as np
import pytest
import torch

from int4_kv_cache_append_b200 import workload as W
from oracle import oracle as O

import kv4_testlib as T

pytestmark = pytest.mark.gpu


def _oracle_one(wl: W.Workload, b: int, g: int, layer: int = 0):
    """Oracle cache and decode of sequence b, only KV head g populated (others zero inputs)."""
    L = int(wl.lens[b])
    npages = (L + wl.P - 1) // wl.P
    cfg = O.Config(wl.Hq, wl.Hkv, wl.D, wl.P, wl.s, wl.w, wl.h, 1)
    pool = np.full(O.page_bytes(cfg) * npages, 0xA5, np.uint8)
    side = np.full(O.side_slot_bytes(cfg), 0xA5, np.uint8)
    f = wl.factor()
    key_k = W.stream_key(wl.seed, W.KIND_K, layer)
    key_v = W.stream_key(wl.seed, W.KIND_V, layer)
    pos = np.arange(L, dtype=np.int64)
    idx = ((b * W.POS_STRIDE + pos[:, None]) * wl.Hkv + g) * wl.D + np.arange(wl.D)[None, :]
    Kg = W.normal_f32(key_k, idx).reshape(L, wl.D) * f[g][None]
    Vg = W.normal_f32(key_v, idx).reshape(L, wl.D) * f[g][None]
    K = np.zeros((L, wl.Hkv, wl.D), np.float32)
    V = np.zeros((L, wl.Hkv, wl.D), np.float32)
    K[:, g] = Kg
    V[:, g] = Vg
    kd = vd = O.F32
    if wl.k_dtype == W.BF16:
        K, kd = W.bf16_bits(K), O.BF16
    if wl.v_dtype == W.BF16:
        V, vd = W.bf16_bits(V), O.BF16
    pt = np.arange(npages, dtype=np.int32)[None, :]
    O.append(cfg, pool, side, K, V, np.zeros(L, np.int32), pos.astype(np.int32), np.array([L], np.int32), pt, kd, vd)
    q = wl.q_input(layer, 0, rows=[b])
    qd = O.BF16 if q.dtype == np.uint16 else O.F32
    out, lse = O.decode(cfg, pool, side, q, pt, np.array([L], np.int32), q_dtype=qd)
    return cfg, pool, side, out[0], lse[0]


@pytest.mark.parametrize("name", ["qwen3-4b-decode", "async-refill", "long-context", "qwen3-8b-loop"])
def test_fullsize_sampled_parity(name):
    from int4_kv_cache_append_b200 import harness as H, kv4
    wl = W.WORKLOADS[name]()
    cache = kv4.Cache(H.geometry(wl), fill=0xA5)
    H.prefill(cache, wl, 0, wl.lens)
    q = T.to_dev(wl.q_input(0))
    lse = torch.empty((wl.B, wl.Hq), device="cuda")
    out = cache.decode(0, q, torch.from_numpy(wl.page_table).cuda(), torch.from_numpy(wl.lens).cuda(), lse=lse,
                       max_len_hint=int(wl.lens.max()))
    torch.cuda.synchronize()
    assert kv4.kv4_get_device_error() == 0
    out = out.cpu().numpy()
    lse = lse.cpu().numpy()
    assert np.isfinite(out).all()
    order = np.argsort(wl.lens, kind="stable")
    picks = [(int(order[0]), 0), (int(order[len(order) // 2]), wl.Hkv // 2), (int(order[-1]), wl.Hkv - 1)]
    if name == "long-context":
        picks = [(0, 3)]
    pool_l, side_l = cache.layer_views(0)
    ocfg = None
    for b, g in picks:
        ocfg, opool, oside, oout, olse = _oracle_one(wl, b, g)
        L = int(wl.lens[b])
        # bytes of head g in every page of sequence b, and in its side-cache slot
        hb = wl.P * (wl.D + 8)
        for lp in range((L + wl.P - 1) // wl.P):
            page = int(wl.page_table[b, lp])
            gstart = page * O.page_bytes(ocfg) + g * hb
            ostart = lp * O.page_bytes(ocfg) + g * hb
            got = pool_l[gstart:gstart + hb].cpu().numpy()
            assert np.array_equal(got, opool[ostart:ostart + hb]), f"{name} b={b} g={g} page {lp} differs"
        sb = O.side_slot_bytes(ocfg) // wl.Hkv
        got = side_l[b * O.side_slot_bytes(ocfg) + g * sb:b * O.side_slot_bytes(ocfg) + (g + 1) * sb].cpu().numpy()
        assert np.array_equal(got, oside[g * sb:(g + 1) * sb]), f"{name} b={b} g={g} side cache differs"
        sl = slice(g * wl.G, (g + 1) * wl.G)
        T.assert_close(out[b, sl], oout[sl], lse[b, sl], olse[sl], what=f"{name} b={b} (L={L}) g={g}")


def test_device_generator_matches_host():
    from int4_kv_cache_append_b200 import harness as H
    wl = W.qwen3_4b_decode()
    b = np.array([0, 5, 63], np.int32)
    p = np.array([0, 77, 8191], np.int32)
    K, V = H.device_kv(wl, 0, torch.from_numpy(b).cuda(), torch.from_numpy(p).cuda(),
                       torch.from_numpy(wl.factor()).cuda())
    Kh, Vh = wl.kv_inputs(0, b, p)
    assert np.array_equal(K.view(torch.int16).cpu().numpy().view(np.uint16), Kh)
    assert np.array_equal(V.view(torch.int16).cpu().numpy().view(np.uint16), Vh)
    q = H.device_q(wl, 0, 0, "cuda")
    assert np.array_equal(q.view(torch.int16).cpu().numpy().view(np.uint16), wl.q_input(0))
