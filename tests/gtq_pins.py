"""Pins for the mixed bit-width key cache part of the CPU oracle (gtq_oracle.c).

Source: "RoPE-Aware Bit Allocation for KV-Cache Quantization" (searcharxiv abstract): a
label-free energy score per RoPE block of every (layer, KV head), integer bit widths handed out
greedily by marginal gain under the K budget, a packed cache.  The readings G1-G8 are listed in
oracle/gtq_oracle.h.  Each pin checks the oracle against something other than itself: the
hand-worked fixture tests/golden/gtq_allocation.txt, a brute-force search over every allocation,
error bounds of the quantiser, Python big-integer bit streams, and a decode written here from
the packed bytes.
"""
from __future__ import annotations

import itertools
import os

import numpy as np

from oracle import oracle as O
from int4_kv_cache_append_b200 import workload as W

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ----------------------------------------------------------------------------- allocation

def pin_gtq_allocation_golden():
    n = 0
    for line in open(os.path.join(GOLDEN, "gtq_allocation.txt")):
        if line.startswith("#") or not line.strip():
            continue
        kb, e, w = (x.split() for x in line.split("|"))
        got = O.gtq_allocate(np.array(e, np.float64), int(kb[0]))
        assert got.tolist() == [int(x) for x in w], (line.strip(), got.tolist())
        n += 1
    assert n >= 7


def _brute_min(E: np.ndarray, key_bits: int) -> float:
    """Least sum E_b 4^-w_b over every allocation with sum w = key_bits * nb, 0 <= w <= 8."""
    nb = E.size
    total = key_bits * nb
    best = np.inf
    for ws in itertools.product(range(9), repeat=nb):
        if sum(ws) != total:
            continue
        best = min(best, float(sum(E[b] * 0.25 ** ws[b] for b in range(nb))))
    return best


def pin_gtq_greedy_optimal(seed: int = 71):
    """Greedy by marginal gain is optimal for a separable convex model: its objective equals the
    brute-force minimum (ties may pick another optimum, so the objective is compared)."""
    rng = np.random.default_rng(seed)
    for trial in range(40):
        nb = int(rng.integers(2, 5))
        kb = int(rng.integers(1, 6))
        E = rng.exponential(1.0, nb) * 10.0 ** rng.integers(-3, 4, nb)
        if trial % 5 == 0:
            E[rng.integers(0, nb)] = 0.0
        w = O.gtq_allocate(E, kb)
        assert int(w.sum()) == kb * nb and int(w.max()) <= 8, (E, kb, w)
        mine = float(sum(E[b] * 0.25 ** int(w[b]) for b in range(nb)))
        brute = _brute_min(E, kb)
        assert abs(mine - brute) <= 1e-12 * max(brute, 1e-300), (E, kb, w, mine, brute)
        assert abs(O.gtq_objective(E, w) - mine) <= 1e-12 * max(mine, 1e-300)


def pin_gtq_allocation_invariances(seed: int = 73):
    """A common factor 4^k leaves the widths alone; permuting distinct energies permutes them;
    more energy never means fewer bits."""
    rng = np.random.default_rng(seed)
    for _ in range(30):
        nb = int(rng.integers(4, 65))
        kb = int(rng.integers(1, 8))
        E = rng.exponential(1.0, nb) * np.exp(rng.normal(0, 2, nb))
        w = O.gtq_allocate(E, kb)
        assert int(w.sum()) == kb * nb
        assert np.array_equal(O.gtq_allocate(E * 4.0 ** int(rng.integers(-5, 6)), kb), w)
        perm = rng.permutation(nb)
        assert np.array_equal(O.gtq_allocate(E[perm], kb), w[perm])
        order = np.argsort(E)
        assert np.all(np.diff(w[order].astype(int)) >= 0), (E[order], w[order])


# ----------------------------------------------------------------------------- energy score

def pin_gtq_energy(seed: int = 75):
    rng = np.random.default_rng(seed)
    # integer-valued keys: every partial sum is exact, so the score equals NumPy's sum exactly
    K = rng.integers(-40, 41, size=(37, 3, 16)).astype(np.float32)
    E = O.gtq_energy(K)
    want = (K[:, :, :8].astype(np.float64) ** 2 + K[:, :, 8:].astype(np.float64) ** 2).sum(axis=0)
    assert np.array_equal(E, want)
    # rotate-half pairing (G1): energy placed in coordinate b + D/2 belongs to block b
    D = 32
    for b in range(D // 2):
        K = np.zeros((5, 2, D), np.float32)
        K[:, 1, b + D // 2] = 3.0
        E = O.gtq_energy(K)
        assert E[1, b] == 45.0 and E.sum() == 45.0 and E[0].sum() == 0.0, (b, E)
    # bf16 inputs: the stored bit patterns are read as bf16
    Kf = rng.normal(0, 1, (9, 2, 16)).astype(np.float32)
    bits = (Kf.view(np.uint32) >> 16).astype(np.uint16)
    Kb = (bits.astype(np.uint32) << 16).view(np.float32)
    Eb = O.gtq_energy(bits, O.BF16)
    want = (Kb[:, :, :8].astype(np.float64) ** 2 + Kb[:, :, 8:].astype(np.float64) ** 2).sum(axis=0)
    assert np.allclose(Eb, want, rtol=1e-14, atol=0)


# ----------------------------------------------------------------------------- quantisers

def _f16(bits: int) -> float:
    return float(np.array([bits], np.uint16).view(np.float16)[0])


def pin_gtq_scales():
    # integer keys: the energy is exact, so the scale is sqrt(E / 2T) correctly rounded to fp32
    K = np.zeros((4, 1, 8), np.float32)
    K[:, 0, 0] = [1, -1, 3, 3]      # block 0: coordinates 0 and 4
    K[:, 0, 4] = [2, 0, 0, -1]
    K[:, 0, 1] = 5                  # block 1: only coordinate 1
    E = O.gtq_energy(K)[0]
    assert E.tolist() == [25.0, 100.0, 0.0, 0.0]
    sig = O.gtq_scales(E, 4)
    assert sig[0] == np.float32(np.sqrt(25.0 / 8)) and sig[1] == np.float32(np.sqrt(100.0 / 8))
    assert sig[2] == 1.0 and sig[3] == 1.0   # no energy: unit scale


def pin_gtq_key_quant_bounds(seed: int = 77):
    """Every coded coordinate lies within half a cell of its reconstruction (a cell is 2^(1-w)
    of the standardised range [-1, 1]); width-0 coordinates reconstruct as 0; the token scale
    covers every coded coordinate; codes stay in [0, 2^w - 1] and grow with x / sigma."""
    rng = np.random.default_rng(seed)
    for trial in range(300):
        D = int(rng.choice([16, 64, 128]))
        x = (rng.normal(0, 1, D) * 10.0 ** rng.integers(-3, 3)).astype(np.float32)
        wc = rng.integers(0, 9, D).astype(np.uint8)
        sc = np.exp(rng.normal(0, 1.5, D)).astype(np.float32)
        codes, sb, flag = O.gtq_quant_key(x, wc, sc)
        assert not flag
        s = _f16(sb)
        coded = wc > 0
        if coded.any():
            assert s >= float(np.max(np.abs(x[coded].astype(np.float64)) / sc[coded])) * (1 - 1e-6)
        for i in range(D):
            w = int(wc[i])
            if w == 0:
                assert codes[i] == 0 and O.gtq_dequant_key(sb, float(sc[i]), 0, 0) == 0.0
                continue
            assert 0 <= codes[i] <= (1 << w) - 1
            xh = O.gtq_dequant_key(sb, float(sc[i]), w, int(codes[i]))
            half = s * float(sc[i]) * 2.0 ** -w
            assert abs(float(x[i]) - xh) <= half * (1 + 1e-5), (trial, i, w, x[i], xh, half)
        for w in range(1, 9):
            idx = np.nonzero(wc == w)[0]
            if idx.size > 1:
                o = idx[np.argsort(x[idx].astype(np.float64) / sc[idx], kind="stable")]
                assert np.all(np.diff(codes[o].astype(int)) >= 0)


def pin_gtq_key_quant_cells():
    """Hand-placed values: x / (sigma s) at the cell centres of a 2-bit coordinate comes back
    exactly, and the cell edges fall to the upper cell (floor of (t + 1) 2^(w-1))."""
    sc = np.ones(5, np.float32)
    x = np.array([-0.75, -0.25, 0.25, 0.75, 1.0], np.float32)     # max |x| = 1 -> s = 1
    codes, sb, _ = O.gtq_quant_key(x, np.full(5, 2, np.uint8), sc)
    assert _f16(sb) == 1.0 and codes.tolist() == [0, 1, 2, 3, 3]
    assert [O.gtq_dequant_key(sb, 1.0, 2, c) for c in range(4)] == [-0.75, -0.25, 0.25, 0.75]
    x = np.array([-1.0, -0.5, 0.0, 0.5, 1.0], np.float32)
    codes, _, _ = O.gtq_quant_key(x, np.full(5, 2, np.uint8), sc)
    assert codes.tolist() == [0, 1, 2, 3, 3]
    codes, _, _ = O.gtq_quant_key(x, np.full(5, 1, np.uint8), sc)   # 1 bit: sign of t
    assert codes.tolist() == [0, 0, 1, 1, 1]
    # the block scale divides: the same x with sigma 2 uses a token scale of half
    codes2, sb2, _ = O.gtq_quant_key(x, np.full(5, 2, np.uint8), np.full(5, 2.0, np.float32))
    assert _f16(sb2) == 0.5 and codes2.tolist() == [0, 1, 2, 3, 3]


def pin_gtq_value_quant(seed: int = 78):
    rng = np.random.default_rng(seed)
    for trial in range(200):
        D = int(rng.choice([16, 64, 128]))
        bits = int(rng.integers(1, 9))
        x = (rng.normal(0, 1, D) * 10.0 ** rng.integers(-3, 3)).astype(np.float32)
        codes, zb, rb, flag = O.gtq_quant_value(x, bits)
        assert not flag
        z, r = _f16(zb), _f16(rb)
        top = (1 << bits) - 1
        assert z <= float(x.min()) and z + r >= float(x.max()) * (1 - 1e-7) - 1e-30
        assert int(codes.max()) <= top
        for i in range(D):
            xh = O.gtq_dequant_value(zb, rb, bits, int(codes[i]))
            assert abs(float(x[i]) - xh) <= 0.5 * r / top * (1 + 1e-5) + 1e-30, (trial, i, x[i], xh)
    # 8 bits on 256 evenly spaced fp16-exact values: codes are the ranks
    x = np.arange(256, dtype=np.float32) * np.float32(0.25) - np.float32(7.0)
    codes, zb, rb, _ = O.gtq_quant_value(x, 8)
    assert _f16(zb) == -7.0 and _f16(rb) == 63.75 and codes.tolist() == list(range(256))


def pin_gtq_quant_special():
    # constant value vector: zero range, all codes zero, reconstruction exact
    codes, zb, rb, flag = O.gtq_quant_value(np.full(8, 2.5, np.float32), 3)
    assert not flag and rb == 0 and _f16(zb) == 2.5 and not codes.any()
    assert O.gtq_dequant_value(zb, rb, 3, 0) == 2.5
    # zero key: token scale 0, codes zero, reconstruction 0
    codes, sb, flag = O.gtq_quant_key(np.zeros(8, np.float32), np.full(8, 3, np.uint8), np.ones(8, np.float32))
    assert not flag and sb == 0 and not codes.any() and O.gtq_dequant_key(sb, 1.0, 3, 0) == 0.0
    # beyond the fp16 range: reported, codes zero
    x = np.zeros(8, np.float32)
    x[3] = 1e6
    codes, sb, flag = O.gtq_quant_key(x, np.full(8, 4, np.uint8), np.ones(8, np.float32))
    assert flag and not codes.any()
    codes, zb, rb, flag = O.gtq_quant_value(x, 4)
    assert flag and not codes.any()
    # a width-0 coordinate does not enter the token scale
    x = np.array([100.0, 1.0, -0.5, 0.25], np.float32)
    _, sb, _ = O.gtq_quant_key(x, np.array([0, 2, 2, 2], np.uint8), np.ones(4, np.float32))
    assert _f16(sb) == 1.0


# ----------------------------------------------------------------------------- packing, layout

def _stream_pack(codes, wc) -> bytes:
    """The bit stream of G5 as one Python integer: code i shifted by the widths before it."""
    v, o = 0, 0
    for c, w in zip(codes, wc):
        v |= int(c) << o
        o += int(w)
    return v.to_bytes((o + 7) // 8, "little")


def pin_gtq_pack(seed: int = 79):
    rng = np.random.default_rng(seed)
    for _ in range(200):
        D = int(rng.choice([8, 16, 64, 128]))
        wc = rng.integers(0, 9, D).astype(np.uint8)
        codes = np.array([rng.integers(0, 1 << int(w)) if w else 0 for w in wc], np.uint8)
        row = O.gtq_pack(codes, wc)
        assert bytes(row.tobytes()) == _stream_pack(codes, wc)
        assert np.array_equal(O.gtq_unpack(row, wc), codes)


def _gtq_cfg(Hq=4, Hkv=2, D=32, P=16, kb=3, vb=3) -> O.GtqConfig:
    return O.GtqConfig(Hq, Hkv, D, P, kb, vb)


def pin_gtq_layout():
    """Key rows, value rows and parameter records of every (page, head, position) are disjoint
    and cover the page pool exactly."""
    for kb, vb, D, P in ((3, 3, 32, 16), (2, 4, 64, 16), (8, 1, 16, 32), (1, 8, 128, 16)):
        cfg = _gtq_cfg(D=D, P=P, kb=kb, vb=vb, Hkv=3, Hq=6)
        sz = O.gtq_sizes(cfg)
        assert sz["key_row_bytes"] == kb * D // 8 and sz["value_row_bytes"] == vb * D // 8
        npages = 3
        cover = np.zeros(sz["page_bytes"] * npages, np.int32)
        for page in range(npages):
            for g in range(3):
                for pp in range(P):
                    for kind, n in (("key_row", kb * D // 8), ("value_row", vb * D // 8), ("param", 8)):
                        o = O.gtq_offset(kind, cfg, page, g, pp)
                        cover[o:o + n] += 1
        assert np.all(cover == 1), (kb, vb, D, P)


# ----------------------------------------------------------------------------- append + decode

def gtq_workload(D=32, B=3, lens=(12, 7, 40), G=2, Hkv=2, P=16, seed=5, dt=W.F32, scale=4.0,
                 n_outlier=2) -> W.Workload:
    import dataclasses
    wl = W.make_workload("gtq-pin", seed, 1, B, G * Hkv, Hkv, D, P, 0, 0, 1, lambda r: list(lens),
                         dt, dt, dt, n_outlier, scale)
    return dataclasses.replace(wl, rope_outliers=True)


def gtq_oracle_cache(wl: W.Workload, kb: int, vb: int, widths=None, lens=None, sentinel: int = 0xA5):
    """(cfg, widths, sigma, pool) of a workload prefilled in one call; the widths default to the
    greedy allocation on the workload's own keys, the block scales always come from them."""
    cfg = O.GtqConfig(wl.Hq, wl.Hkv, wl.D, wl.P, kb, vb)
    lens = np.asarray(wl.lens if lens is None else lens, np.int32)
    b = np.concatenate([np.full(L, i, np.int32) for i, L in enumerate(lens)])
    p = np.concatenate([np.arange(L, dtype=np.int32) for L in lens])
    K, V = wl.kv_inputs(0, b, p)
    kd = O.BF16 if wl.k_dtype == W.BF16 else O.F32
    vd = O.BF16 if wl.v_dtype == W.BF16 else O.F32
    E = O.gtq_energy(K, kd)
    sigma = np.stack([O.gtq_scales(E[g], K.shape[0]) for g in range(wl.Hkv)])
    if widths is None:
        widths = np.stack([O.gtq_allocate(E[g], kb) for g in range(wl.Hkv)])
    pool = np.full(O.gtq_sizes(cfg)["page_bytes"] * max(wl.num_pages, 1), sentinel, np.uint8)
    O.gtq_append(cfg, widths, sigma, pool, K, V, b, p, wl.page_table, kd, vd)
    return cfg, widths, sigma, pool


def _brute_gtq_decode(wl, cfg, widths, sigma, pool, q, lens):
    """Decode from the packed bytes with Python integers and NumPy: parse each row as one
    little-endian integer, cut out the codes, rebuild keys and values, one softmax."""
    D, P, G = wl.D, wl.P, wl.Hq // wl.Hkv
    kr, vr = cfg.key_bits * D // 8, cfg.value_bits * D // 8
    tile = P * (kr + vr + 8)
    out = np.zeros((len(lens), wl.Hq, D))
    lse = np.zeros((len(lens), wl.Hq))
    for b, L in enumerate(lens):
        for g in range(wl.Hkv):
            wk = [int(widths[g][i % (D // 2)]) for i in range(D)]
            kh = np.zeros((L, D))
            vh = np.zeros((L, D))
            for t in range(L):
                page = int(wl.page_table[b, t // P])
                pp = t % P
                # slice of 16 positions: 16 key rows, 16 value rows, 16 records of 8 bytes
                base = (page * wl.Hkv + g) * tile + (pp // 16) * 16 * (kr + vr + 8)
                rr = pp % 16
                prm = pool[base + 16 * (kr + vr) + 8 * rr: base + 16 * (kr + vr) + 8 * rr + 8].view(np.float16).astype(float)
                kint = int.from_bytes(pool[base + rr * kr: base + (rr + 1) * kr].tobytes(), "little")
                vint = int.from_bytes(pool[base + 16 * kr + rr * vr: base + 16 * kr + (rr + 1) * vr].tobytes(), "little")
                o = 0
                for i in range(D):
                    w = wk[i]
                    c = (kint >> o) & ((1 << w) - 1)
                    o += w
                    sg = float(sigma[g][i % (D // 2)])
                    kh[t, i] = 0.0 if w == 0 else prm[0] * sg * ((2 * c + 1) / 2.0 ** w - 1)
                top = (1 << cfg.value_bits) - 1
                for i in range(D):
                    c = (vint >> (i * cfg.value_bits)) & top
                    vh[t, i] = prm[2] + c * prm[3] / top
            for j in range(G):
                qh = g * G + j
                s = kh @ q[b, qh].astype(np.float64) / np.sqrt(D)
                m = s.max()
                e = np.exp(s - m)
                out[b, qh] = e @ vh / e.sum()
                lse[b, qh] = m + np.log(e.sum())
    return out, lse


def pin_gtq_brute_force_decode():
    for kb, vb, lens, D, P in ((3, 3, (12, 7, 40), 32, 16), (2, 4, (1, 33, 16), 32, 16), (5, 2, (17, 3, 9), 16, 16),
                               (3, 3, (70, 5, 33), 32, 32), (4, 2, (100, 49, 17), 16, 48)):
        wl = gtq_workload(D=D, lens=lens, P=P)
        cfg, widths, sigma, pool = gtq_oracle_cache(wl, kb, vb)
        assert int(widths.sum()) == kb * D // 2 * wl.Hkv
        q = wl.q_input(0)
        out, lse = O.gtq_decode(cfg, widths, sigma, pool, q, wl.page_table, np.array(lens, np.int32))
        bo, bl = _brute_gtq_decode(wl, cfg, widths, sigma, pool, q, lens)
        assert np.allclose(out, bo, rtol=0, atol=1e-11), float(np.abs(out - bo).max())
        assert np.allclose(lse, bl, rtol=0, atol=1e-11)


def pin_gtq_unquantised_limit(seed: int = 81):
    """With 8 bits everywhere the decode is close to exact attention on the raw keys and values;
    the error shrinks as the key budget grows; and on keys and queries with RoPE-block outliers
    a budget spent by energy beats the same budget spread evenly (the abstract's claim)."""
    wl = gtq_workload(D=64, lens=(200, 150, 90), seed=seed, scale=4.0)
    lens = np.array(wl.lens, np.int32)
    b = np.concatenate([np.full(L, i, np.int32) for i, L in enumerate(lens)])
    p = np.concatenate([np.arange(L, dtype=np.int32) for L in lens])
    K, V = wl.kv_inputs(0, b, p)
    q = wl.q_input(0)
    G = wl.Hq // wl.Hkv
    ref = np.zeros((wl.B, wl.Hq, wl.D))
    for bi in range(wl.B):
        rows = np.nonzero(b == bi)[0]
        for qh in range(wl.Hq):
            g = qh // G
            sc = K[rows, g].astype(np.float64) @ q[bi, qh].astype(np.float64) / np.sqrt(wl.D)
            e = np.exp(sc - sc.max())
            ref[bi, qh] = e @ V[rows, g].astype(np.float64) / e.sum()

    def rel(out):
        return float(np.linalg.norm(out - ref) / np.linalg.norm(ref))
    errs = {}
    for kb in (2, 3, 5, 8):
        cfg, widths, sigma, pool = gtq_oracle_cache(wl, kb, 8)
        errs[kb] = rel(O.gtq_decode(cfg, widths, sigma, pool, q, wl.page_table, lens)[0])
    assert errs[8] < 0.03 and errs[8] < errs[5] < errs[3] < errs[2], errs
    for kb in (2, 3):
        uniform = np.full((wl.Hkv, wl.D // 2), kb, np.uint8)
        cfg, _, sigma, pool_u = gtq_oracle_cache(wl, kb, 8, widths=uniform)
        eu = rel(O.gtq_decode(cfg, uniform, sigma, pool_u, q, wl.page_table, lens)[0])
        assert errs[kb] < 0.8 * eu, (kb, errs[kb], eu)


GTQ_PINS = [
    pin_gtq_allocation_golden, pin_gtq_greedy_optimal, pin_gtq_allocation_invariances, pin_gtq_energy,
    pin_gtq_scales, pin_gtq_key_quant_bounds, pin_gtq_key_quant_cells, pin_gtq_value_quant,
    pin_gtq_quant_special, pin_gtq_pack, pin_gtq_layout, pin_gtq_brute_force_decode,
    pin_gtq_unquantised_limit,
]
