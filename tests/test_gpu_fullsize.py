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


def _oracle_replay(wl: W.Workload, b: int, g: int, layer: int, L0: int, steps: int):
    """Oracle cache of sequence b (only KV head g populated) built the way the step loop builds it:
    positions [0, L0) appended with lens_after = L0, then one position per step with lens_after =
    position + 1; returns the cache and the decode of the last step (query of that step)."""
    L = L0 + steps
    npages = (L + wl.P - 1) // wl.P
    cfg = O.Config(wl.Hq, wl.Hkv, wl.D, wl.P, wl.s, wl.w, wl.h, 1)
    pool = np.full(O.page_bytes(cfg) * npages, 0xA5, np.uint8)
    side = np.full(O.side_slot_bytes(cfg), 0xA5, np.uint8)
    f = wl.factor()
    pt = np.arange(npages, dtype=np.int32)[None, :]

    def inputs(pos):
        idx = ((b * W.POS_STRIDE + pos[:, None].astype(np.int64)) * wl.Hkv + g) * wl.D + np.arange(wl.D)[None, :]
        K = np.zeros((pos.size, wl.Hkv, wl.D), np.float32)
        V = np.zeros((pos.size, wl.Hkv, wl.D), np.float32)
        K[:, g] = W.normal_f32(W.stream_key(wl.seed, W.KIND_K, layer), idx).reshape(-1, wl.D) * f[g][None]
        V[:, g] = W.normal_f32(W.stream_key(wl.seed, W.KIND_V, layer), idx).reshape(-1, wl.D) * f[g][None]
        return (W.bf16_bits(K), O.BF16) if wl.k_dtype == W.BF16 else (K, O.F32), \
               (W.bf16_bits(V), O.BF16) if wl.v_dtype == W.BF16 else (V, O.F32)

    pos = np.arange(L0, dtype=np.int32)
    (K, kd), (V, vd) = inputs(pos)
    O.append(cfg, pool, side, K, V, np.zeros(L0, np.int32), pos, np.array([L0], np.int32), pt, kd, vd)
    for t in range(steps):
        p1 = np.array([L0 + t], np.int32)
        (K, kd), (V, vd) = inputs(p1)
        O.append(cfg, pool, side, K, V, np.zeros(1, np.int32), p1, p1 + 1, pt, kd, vd)
    q = wl.q_input(layer, steps - 1, rows=[b])
    qd = O.BF16 if q.dtype == np.uint16 else O.F32
    out, lse = O.decode(cfg, pool, side, q, pt, np.array([L], np.int32), q_dtype=qd)
    return cfg, pool, side, out[0], lse[0]


def test_loop_steps_sampled_parity():
    """The 36-layer loop at full size (128 sequences, 36 layers, about 44 GB of cache) in the
    benchmark's launch configuration (decode built while the append runs, max_len_hint set): after
    the prefill, 8 steps each append one token per sequence and decode, layer by layer.  Some
    sequences start just below s + w = 144, so that their first INT4 positions appear during the
    steps; in every longer one, one position per step leaves the recent ring for the INT4 region.
    Sampled (sequence, KV head, layer) triples are checked against the oracle replaying the same
    appends: page bytes and side-cache bytes bit-exact, last-step outputs within tolerance."""
    from int4_kv_cache_append_b200 import harness as H, kv4
    steps = 8
    wl = W.qwen3_8b_loop()
    lens0 = wl.lens.copy()
    lens0[:4] = [140, 143, 144, 9]  # below, at and past the s + w boundary; one inside the sinks
    wl.lens = lens0
    dev = torch.device("cuda")
    cache = kv4.Cache(H.geometry(wl), fill=0xA5)
    kv4.kv4_set_decode_overlap(cache.handle, True)
    for layer in range(wl.layers):
        H.prefill(cache, wl, layer, lens0)
    pt = torch.from_numpy(wl.page_table).to(dev)
    bt = torch.arange(wl.B, dtype=torch.int32, device=dev)
    factor = torch.from_numpy(wl.factor()).to(dev)
    maxlen = int(lens0.max()) + steps
    picks = [(0, 0, 0), (1, 3, 17), (2, 7, 35), (3, 1, 5), (int(np.argmax(lens0)), 5, 35),
             (int(np.argsort(lens0)[wl.B // 2]), 2, 20)]
    keep = {layer for _, _, layer in picks}
    outs, lses = {}, {}
    for t in range(steps):
        pos = torch.from_numpy((lens0 + t).astype(np.int32)).to(dev)
        la = pos + 1
        for layer in range(wl.layers):
            K, V = H.device_kv(wl, layer, bt, pos, factor)
            cache.append(layer, K, V, bt, pos, la, pt)
            q = H.device_q(wl, layer, t, dev)
            lse = torch.empty((wl.B, wl.Hq), device=dev)
            out = cache.decode(layer, q, pt, la, lse=lse, max_len_hint=maxlen)
            if t == steps - 1 and layer in keep:
                outs[layer], lses[layer] = out.clone(), lse.clone()
    torch.cuda.synchronize()
    assert kv4.kv4_get_device_error() == 0
    for b, g, layer in picks:
        L0 = int(lens0[b])
        ocfg, opool, oside, oout, olse = _oracle_replay(wl, b, g, layer, L0, steps)
        pool_l, side_l = cache.layer_views(layer)
        hb = wl.P * (wl.D + 8)
        for lp in range((L0 + steps + wl.P - 1) // wl.P):
            page = int(wl.page_table[b, lp])
            gstart = page * O.page_bytes(ocfg) + g * hb
            ostart = lp * O.page_bytes(ocfg) + g * hb
            got = pool_l[gstart:gstart + hb].cpu().numpy()
            want = opool[ostart:ostart + hb]
            assert np.array_equal(got, want), f"loop b={b} g={g} layer={layer} page {lp} differs"
        sb = O.side_slot_bytes(ocfg) // wl.Hkv
        s0 = b * O.side_slot_bytes(ocfg) + g * sb
        assert np.array_equal(side_l[s0:s0 + sb].cpu().numpy(), oside[g * sb:(g + 1) * sb]), \
            f"loop b={b} g={g} layer={layer} side cache differs"
        sl = slice(g * wl.G, (g + 1) * wl.G)
        T.assert_close(outs[layer][b, sl].cpu().numpy(), oout[sl], lses[layer][b, sl].cpu().numpy(), olse[sl],
                       what=f"loop b={b} (L={L0}+{steps}) g={g} layer={layer}")
