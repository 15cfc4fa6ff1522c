"""Pins for the CPU oracle: checks against what the method pages and mathematics fix.

Each ``pin_*`` function raises AssertionError when the oracle disagrees with an independent
fact: a library routine (NumPy's float16 rounding, scipy's Sylvester Hadamard), a closed
form, an invariant, a hand-worked fixture under ``tests/golden`` or a brute-force
restatement written here in Python/NumPy.  They are plain functions so that the mutation
test can run them against deliberately broken builds of the oracle.
"""
from __future__ import annotations

import os

import numpy as np
import scipy.linalg

from oracle import oracle as O
from int4_kv_cache_append_b200 import workload as W

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
MODES = {"RN": O.RN, "RD": O.RD, "RU": O.RU}


# ----------------------------------------------------------------------------- fp16

def _f16_up(h: np.float16) -> np.float16:
    return np.nextafter(h, np.float16(np.inf))


def _f16_down(h: np.float16) -> np.float16:
    return np.nextafter(h, np.float16(-np.inf))


def pin_fp16_golden():
    for line in open(os.path.join(GOLDEN, "fp16_rounding.txt")):
        if line.startswith("#") or not line.strip():
            continue
        xh, mode, want = line.split()[:3]
        x = np.array([int(xh, 16)], np.uint32).view(np.float32)[0]
        got = O.f32_to_f16(float(x), MODES[mode])
        assert got == int(want, 16), (xh, mode, hex(got), want)


def pin_fp16_vs_numpy(n: int = 20000, seed: int = 7):
    """RN equals NumPy's float32 -> float16 cast; RD/RU bracket x by adjacent fp16 values."""
    rng = np.random.default_rng(seed)
    bits = rng.integers(0, 2**32, size=n, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    x = x[np.isfinite(x)]
    # add values near the fp16 range and subnormals, where rounding is most fragile
    extra = np.concatenate([
        rng.uniform(-70000, 70000, 2000), rng.uniform(-1e-4, 1e-4, 2000),
        rng.uniform(-1e-7, 1e-7, 1000), rng.normal(0, 30, 2000)]).astype(np.float32)
    x = np.concatenate([x, extra])
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16)
    for xi, ri in zip(x, ref):
        got = O.f32_to_f16(float(xi), O.RN)
        assert got == int(ri.view(np.uint16)), (float(xi), hex(got), hex(int(ri.view(np.uint16))))
        rd = np.array([O.f32_to_f16(float(xi), O.RD)], np.uint16).view(np.float16)[0]
        ru = np.array([O.f32_to_f16(float(xi), O.RU)], np.uint16).view(np.float16)[0]
        xd = float(xi)
        assert float(rd) <= xd <= float(ru), (xd, float(rd), float(ru))
        if np.isfinite(rd) and float(rd) != xd:
            assert float(_f16_up(rd)) > xd or not np.isfinite(_f16_up(rd)), (xd, float(rd))
        if np.isfinite(ru) and float(ru) != xd:
            assert float(_f16_down(ru)) < xd or not np.isfinite(_f16_down(ru)), (xd, float(ru))
        if float(rd) == xd or float(ru) == xd:
            assert float(rd) == float(ru) == xd or (xd == 0.0)


def pin_fp16_decode_all():
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = allbits.view(np.float16).astype(np.float32)
    for b in range(0, 65536, 7):
        r = ref[b]
        got = O.f16_to_f32(b)
        if np.isnan(r):
            assert np.isnan(got)
        else:
            assert got == float(r), (hex(b), got, float(r))
    for b in (0x3F80, 0xC2F6, 0x0001, 0x7F7F):
        assert O.bf16_to_f32(b) == float(W.bf16_to_f32(np.array([b]))[0])


# ----------------------------------------------------------------------------- Hadamard

def pin_hadamard_matrix():
    """Butterfly applied to unit vectors gives blockdiag(H_h) (scipy Sylvester), H H^T = h I."""
    D = 128
    for h in (1, 2, 4, 8, 16, 32, 64, 128):
        cols = [O.fwht_f32(np.eye(D, dtype=np.float32)[i], h) for i in range(D)]
        M = np.stack(cols, axis=1).astype(np.int64)
        Hh = scipy.linalg.hadamard(h).astype(np.int64)
        ref = np.kron(np.eye(D // h, dtype=np.int64), Hh)
        assert np.array_equal(M, ref), h
        assert np.array_equal(M @ M.T, h * np.eye(D, dtype=np.int64)), h


def pin_hadamard_golden():
    txt = open(os.path.join(GOLDEN, "hadamard_sylvester.txt")).read().split("\n")
    mats, cur = {}, None
    for line in txt:
        if line.startswith("#") or not line.strip():
            continue
        if line.startswith("H"):
            cur = int(line[1:])
            mats[cur] = []
        else:
            mats[cur].append([int(v) for v in line.split()])
    for h, rows in mats.items():
        M = np.stack([O.fwht_f32(np.eye(h, dtype=np.float32)[i], h) for i in range(h)], axis=1)
        assert np.array_equal(M.astype(np.int64), np.array(rows)), h


def pin_hadamard_integer_exact(seed: int = 3):
    """On small-integer inputs every fp32 add is exact, so the butterfly equals the matrix
    product exactly; fp64 variant agrees too."""
    rng = np.random.default_rng(seed)
    for h in (2, 16, 64, 128):
        x = rng.integers(-1000, 1000, size=128).astype(np.float32)
        ref = np.kron(np.eye(128 // h), scipy.linalg.hadamard(h)) @ x.astype(np.float64)
        assert np.array_equal(O.fwht_f32(x, h).astype(np.float64), ref)
        assert np.array_equal(O.fwht_f64(x.astype(np.float64), h), ref)


# ----------------------------------------------------------------------------- quantisers

def _f16(bits: int) -> float:
    return float(np.array([bits], np.uint16).view(np.float16)[0])


def pin_quant_golden():
    lines = [ln for ln in open(os.path.join(GOLDEN, "quant_worked.txt"))
             if ln.strip() and not ln.startswith("#")]
    for a, b in zip(lines[0::2], lines[1::2]):
        kind, *vals = a.split()
        x = np.array([float(v) for v in vals], np.float32)
        want = b.split()[1:]
        if kind == "INT4":
            codes, sc, zr = O.quant_int4(x)
            assert sc == int(want[0], 16) and zr == int(want[1], 16), (a, hex(sc), hex(zr))
            assert codes.tolist() == [int(v) for v in want[2:]], (a, codes)
        else:
            codes, sc = O.quant_int8(x)
            assert sc == int(want[0], 16), (a, hex(sc))
            assert codes.tolist() == [int(v) for v in want[1:]], (a, codes)


def _vectors(seed: int, n: int, D: int):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        kind = i % 6
        if kind == 0:
            x = rng.normal(0, 1, D)
        elif kind == 1:
            x = rng.normal(0, 1, D)
            x[rng.choice(D, 2, replace=False)] *= 20
        elif kind == 2:
            x = rng.normal(0, 1e-4, D)
        elif kind == 3:
            x = rng.normal(5, 0.01, D)
        elif kind == 4:
            x = rng.uniform(-300, 300, D)
        else:
            x = np.full(D, rng.normal(0, 3))
        out.append(x.astype(np.float32))
    return out


def _requant_int4_numpy(x: np.ndarray):
    """Independent restatement of reading R3 with NumPy float32 arithmetic and NumPy float16
    neighbours for the directed roundings."""
    mn, mx = np.float32(x.min()) + np.float32(0), np.float32(x.max()) + np.float32(0)
    z = np.float16(mn)
    if float(z) > float(mn):
        z = _f16_down(z)
    zf = np.float32(z)
    r = np.float32(mx - zf)
    sq = np.float32(r / np.float32(15.0))
    with np.errstate(over="ignore"):
        s = np.float16(sq)
    if float(s) < float(sq):
        s = _f16_up(s)
    sf = np.float32(s)
    if sf == 0 or not (np.isfinite(sf) and np.isfinite(zf)):
        codes = np.zeros(x.size, np.uint8)
    else:
        t = ((x - zf).astype(np.float32) / sf).astype(np.float32)
        codes = np.clip(np.rint(t), 0, 15).astype(np.uint8)
    return codes, int(np.array([s]).view(np.uint16)[0]), int(np.array([z]).view(np.uint16)[0])


def pin_quant_int4_bounds(seed: int = 11, n: int = 600):
    for D in (32, 64, 128):
        for x in _vectors(seed + D, n // 3, D):
            codes, sc, zr = O.quant_int4(x)
            s, z = _f16(sc), _f16(zr)
            xd = x.astype(np.float64)
            assert codes.min() >= 0 and codes.max() <= 15
            assert z <= xd.min() and z + 15 * s >= xd.max()
            rec = z + s * codes.astype(np.float64)
            tol = s / 2 + 4 * np.spacing(np.maximum(np.abs(xd), abs(z))).astype(np.float64)
            assert np.all(np.abs(xd - rec) <= tol), np.max(np.abs(xd - rec) - tol)
            # the chosen level is the nearest of the 16 (ties excepted)
            levels = z + s * np.arange(16)
            dist = np.abs(xd[:, None] - levels[None, :])
            best = dist.min(axis=1)
            assert np.all(dist[np.arange(D), codes] <= best + 4 * np.spacing(np.abs(xd) + abs(z)))
            # zero is the largest fp16 <= min; scale the smallest fp16 >= fl32((max - zero)/15)
            assert float(_f16_up(np.float16(z))) > xd.min()
            rc, rs, rz = _requant_int4_numpy(x)
            assert (sc, zr) == (rs, rz) and np.array_equal(codes, rc)


def pin_quant_int4_constant():
    for v in (0.0, 1.0, -3.25, 1024.5, 2.0**-20):
        x = np.full(64, v, np.float32)
        codes, sc, zr = O.quant_int4(x)
        if float(np.float16(v)) == v:
            assert np.all(_f16(zr) + _f16(sc) * codes == v)


def pin_quant_range(seed: int = 17):
    """Vectors beyond the fp16 range: the largest fp16 <= min is -inf below -65504, the smallest
    fp16 >= (max - zero)/15 is +inf above 65504 (IEEE directed rounding of an overflow); such a
    vector gets all-zero codes and the out-of-range flag.  At the edge of the range the parameters
    are finite, the flag is clear and the reconstruction bound holds."""
    rng = np.random.default_rng(seed)
    big = np.float32(np.finfo(np.float16).max)  # 65504
    for D in (64, 128):
        x = rng.normal(0, 1, D).astype(np.float32)
        x[5] = -1.0e6  # zero overflows to -inf
        codes, sc, zr, bad = O.quant_int4(x, with_flag=True)
        assert bad and zr == 0xFC00 and sc == 0x7C00 and not codes.any(), (hex(sc), hex(zr))
        x = np.abs(rng.normal(0, 1, D)).astype(np.float32)
        x[7] = 1.0e6  # (max - zero)/15 = 66667 > 65504: scale overflows to +inf
        codes, sc, zr, bad = O.quant_int4(x, with_flag=True)
        z = _f16(zr)
        assert bad and sc == 0x7C00 and np.isfinite(z) and z <= x.min() < float(_f16_up(np.float16(z)))
        assert not codes.any()
        # INT8: max|x| / 127 stays finite up to 127 * 65504
        c8, s8, bad8 = O.quant_int8(x, with_flag=True)
        assert not bad8 and _f16(s8) >= 1.0e6 / 127
        x8 = x.copy()
        x8[7] = 1.0e7
        c8, s8, bad8 = O.quant_int8(x8, with_flag=True)
        assert bad8 and s8 == 0x7C00 and not c8.any()
        # the edge: min = -65504 exactly, range inside fp16 -> finite parameters, no flag
        x = rng.normal(0, 1, D).astype(np.float32)
        x[3] = -big
        codes, sc, zr, bad = O.quant_int4(x, with_flag=True)
        assert not bad and zr == 0xFBFF and np.isfinite(_f16(sc))
        rec = _f16(zr) + _f16(sc) * codes.astype(np.float64)
        assert np.all(np.abs(x.astype(np.float64) - rec) <= _f16(sc) / 2 + 4 * np.spacing(big))


def pin_append_range_flag(seed: int = 19):
    """The append reports a token whose parameters overflowed, and only then."""
    wl = small_workload(lens=(9,), B=1, s=2, w=3, h=8, seed=seed)
    cfg = oracle_cfg(wl)
    pool = np.zeros(O.page_bytes(cfg) * wl.num_pages, np.uint8)
    side = np.zeros(O.side_slot_bytes(cfg) * wl.B, np.uint8)
    b = np.zeros(9, np.int32)
    p = np.arange(9, dtype=np.int32)
    K, V = wl.kv_inputs(0, b, p)
    assert not O.append(cfg, pool, side, K, V, b, p, wl.lens, wl.page_table)
    V = V.copy()
    V[4, 1, 3] = 2.0e6
    assert O.append(cfg, pool, side, K, V, b, p, wl.lens, wl.page_table)


def pin_quant_int8_bounds(seed: int = 13, n: int = 300):
    for x in _vectors(seed, n, 128):
        codes, sc = O.quant_int8(x)
        s = _f16(sc)
        xd = x.astype(np.float64)
        assert np.abs(codes.astype(np.int64)).max() <= 127
        a = np.float32(np.abs(x).max())
        assert s >= float(np.float32(a / np.float32(127.0)))
        assert float(_f16_down(np.float16(s))) < float(np.float32(a / np.float32(127.0))) or s == 0
        if s > 0:
            err = np.abs(xd - s * codes)
            assert np.all(err <= s / 2 + 4 * np.spacing(np.abs(xd))), err.max()
            assert np.array_equal(codes, np.clip(np.rint((x / np.float32(s)).astype(np.float32)), -127, 127))


# ----------------------------------------------------------------------------- storage/layout

def pin_storage_bits():
    for line in open(os.path.join(GOLDEN, "storage_bits.txt")):
        if line.startswith("#") or not line.strip():
            continue
        D, bits = int(line.split()[0]), float(line.split()[1])
        cfg = O.Config(32, 8, D, 16, 4, 128, D, 4)
        # bytes per token per KV head for K (or V): page bytes / (P * Hkv * 2)
        per_vec = O.page_bytes(cfg) / (16 * 8 * 2)
        assert per_vec * 8 / D == bits


def pin_layout_bijection():
    """Every nibble and parameter byte of a page, and every byte of a side tile, is owned by
    exactly one (head, position, element) — no overlap, no gap."""
    for D, P, Hkv, s, w in ((64, 16, 2, 4, 32), (128, 64, 1, 4, 128), (32, 32, 1, 3, 10)):
        cfg = O.Config(Hkv, Hkv, D, P, s, w, 1, 2)
        pb = O.page_bytes(cfg)
        nib = np.zeros(2 * pb, np.int32)
        for g in range(Hkv):
            for pp in range(P):
                for e in range(D):
                    nib[2 * O.byte_offset("k4", cfg, 1, g, pp, e) - 2 * pb + O.nibble_high("k4", cfg, pp, e)] += 1
                    nib[2 * O.byte_offset("v4", cfg, 1, g, pp, e) - 2 * pb + O.nibble_high("v4", cfg, pp, e)] += 1
                for isv in (0, 1):
                    off = O.byte_offset("p4", cfg, 1, g, pp, isv) - pb
                    nib[2 * off:2 * off + 8] += 1
        assert np.all(nib == 1), (D, P, np.unique(nib, return_counts=True))
        sb = O.side_slot_bytes(cfg)
        nt = O.side_tiles(cfg)
        own = np.zeros(sb, np.int32)
        for g in range(Hkv):
            for row in range(nt * 16):
                for e in range(D):
                    own[O.byte_offset("k8", cfg, 1, g, row, e) - sb] += 1
                    own[O.byte_offset("v8", cfg, 1, g, row, e) - sb] += 1
                for isv in (0, 1):
                    off = O.byte_offset("s8", cfg, 1, g, row, isv) - sb
                    own[off:off + 2] += 1
        assert np.all(own == 1), (D, np.unique(own, return_counts=True))


def _bf16_rne(x: np.ndarray) -> np.ndarray:
    """fp32 -> bfloat16 bit patterns, nearest with ties to even, on the integer bits."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def pin_bf16_rounding(seed: int = 23):
    """orc_f32_to_bf16 is round-to-nearest-even on the 16 dropped bits: random finite patterns,
    exact halfway cases of both parities, and values already in bf16."""
    rng = np.random.default_rng(seed)
    bits = rng.integers(0, 2**32, size=20000, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    x = x[np.isfinite(x)]
    half = (np.arange(-300, 300, dtype=np.int64) << 16 | 0x8000).astype(np.uint32).view(np.float32)
    exact = (rng.integers(0, 2**16, size=500).astype(np.uint32) << 16).view(np.float32)
    for arr in (x, half[np.isfinite(half)], exact[np.isfinite(exact)]):
        want = _bf16_rne(arr)
        got = np.array([O.f32_to_bf16(float(v)) for v in arr], np.uint16)
        assert np.array_equal(got, want), np.nonzero(got != want)[0][:5]


def pin_layout_bijection_bf16_values():
    """bf16 values (value_format 1): every byte of a page tile (K nibbles, K parameters, V bf16)
    and of a side tile (K int8, K scale, V bf16) is owned by exactly one item."""
    for D, P, Hkv, s, w in ((64, 16, 2, 4, 32), (128, 32, 1, 3, 10), (32, 16, 1, 2, 5)):
        cfg = O.Config(Hkv, Hkv, D, P, s, w, 1, 2, value_format=1)
        pb = O.page_bytes(cfg)
        assert pb == Hkv * P * (D // 2 + 4 + 2 * D)
        nib = np.zeros(2 * pb, np.int32)
        for g in range(Hkv):
            for pp in range(P):
                for e in range(D):
                    nib[2 * O.byte_offset("k4", cfg, 1, g, pp, e) - 2 * pb + O.nibble_high("k4", cfg, pp, e)] += 1
                    off = O.byte_offset("vb", cfg, 1, g, pp, e) - pb
                    nib[2 * off:2 * off + 4] += 1
                off = O.byte_offset("p4", cfg, 1, g, pp, 0) - pb
                nib[2 * off:2 * off + 8] += 1
        assert np.all(nib == 1), (D, P, np.unique(nib, return_counts=True))
        sb = O.side_slot_bytes(cfg)
        assert sb == Hkv * O.side_tiles(cfg) * 16 * (3 * D + 2)
        own = np.zeros(sb, np.int32)
        for g in range(Hkv):
            for row in range(O.side_tiles(cfg) * 16):
                for e in range(D):
                    own[O.byte_offset("k8", cfg, 1, g, row, e) - sb] += 1
                    off = O.byte_offset("vb8", cfg, 1, g, row, e) - sb
                    own[off:off + 2] += 1
                off = O.byte_offset("s8", cfg, 1, g, row, 0) - sb
                own[off:off + 2] += 1
        assert np.all(own == 1), (D, np.unique(own, return_counts=True))


def pin_bf16_values_exact(seed: int = 29):
    """With bf16 values the dequantised values are the inputs rounded to bf16 (nearest even), in
    every region, and the keys dequantise exactly as in the INT4-value format."""
    for dt in (W.F32, W.BF16):
        wl = small_workload(D=64, lens=(40, 9, 70), s=3, w=8, h=16, seed=seed, dt=dt)
        cfg, pool, side = build_cache(wl, value_format=1)
        cfg0, pool0, side0 = build_cache(wl)
        for b, L in enumerate(wl.lens):
            _, V = wl.kv_inputs(0, np.full(L, b, np.int32), np.arange(L, dtype=np.int32))
            vb = V if V.dtype == np.uint16 else _bf16_rne(V)
            want = (vb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
            for g in range(wl.Hkv):
                kd, vd, _ = O.dequant_seq(cfg, pool, side, wl.page_table[b], b, L, g)
                kd0, _, _ = O.dequant_seq(cfg0, pool0, side0, wl.page_table[b], b, L, g)
                assert np.array_equal(vd, want[:, g]), (dt, b, g)
                assert np.array_equal(kd, kd0), (dt, b, g)


# ----------------------------------------------------------------------------- cache helpers

def build_cache(wl: W.Workload, layer: int = 0, lens=None, step_by_step: bool = False, sentinel: int = 0xA5,
                signs=(0, 0, 0, 0), rotate_values: int = 0, value_format: int = 0):
    """Oracle cache for a workload: prefill every token in position order (one call for all
    tokens with lens_after = L, or one call per position with lens_after = pos + 1)."""
    cfg = oracle_cfg(wl, signs, rotate_values, value_format)
    lens = np.asarray(wl.lens if lens is None else lens, np.int32)
    pool = np.full(O.page_bytes(cfg) * wl.num_pages, sentinel, np.uint8)
    side = np.full(O.side_slot_bytes(cfg) * wl.B, sentinel, np.uint8)
    kd = O.BF16 if wl.k_dtype == W.BF16 else O.F32
    vd = O.BF16 if wl.v_dtype == W.BF16 else O.F32
    if not step_by_step:
        b = np.concatenate([np.full(L, i, np.int32) for i, L in enumerate(lens)])
        p = np.concatenate([np.arange(L, dtype=np.int32) for L in lens])
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


def oracle_cfg(wl: W.Workload, signs=(0, 0, 0, 0), rotate_values: int = 0, value_format: int = 0) -> O.Config:
    return O.Config(wl.Hq, wl.Hkv, wl.D, wl.P, wl.s, wl.w, wl.h, wl.B, tuple(signs), rotate_values, value_format)


def small_workload(D=32, B=3, lens=(12, 7, 40), s=2, w=5, h=8, G=2, Hkv=2, P=16, seed=5,
                   dt=W.F32, scale=20.0) -> W.Workload:
    return W.make_workload("pin", seed, 1, B, G * Hkv, Hkv, D, P, s, w, h, lambda r: list(lens),
                           dt, dt, dt, 2, scale)


# ----------------------------------------------------------------------------- routing

def pin_routing(step_by_step: bool):
    for (s, w, lens) in ((2, 5, (12, 7, 40)), (0, 4, (9, 1, 3)), (3, 0, (5, 2, 1)), (4, 16, (3, 20, 33))):
        wl = small_workload(s=s, w=w, lens=lens)
        cfg, pool, side = build_cache(wl, step_by_step=step_by_step)
        sb = O.side_slot_bytes(cfg)
        for b, L in enumerate(wl.lens):
            rows_expected = {}
            for j in range(min(s, L)):
                rows_expected[j] = j
            for j in range(max(s, L - w), L):
                rows_expected[s + j % w] = j
            K, V = wl.kv_inputs(0, np.full(L, b, np.int32), np.arange(L, dtype=np.int32))
            for g in range(wl.Hkv):
                for row in range(O.side_tiles(cfg) * 16):
                    k_off = [O.byte_offset("k8", cfg, b, g, row, e) for e in range(wl.D)]
                    if row in rows_expected:
                        j = rows_expected[row]
                        kr = O.fwht_f32(K[j, g], wl.h)
                        codes, sc = O.quant_int8(kr)
                        assert np.array_equal(side[k_off].view(np.int8), codes), (s, w, b, row, j)
                        vcodes, vsc = O.quant_int8(V[j, g])
                        v_off = [O.byte_offset("v8", cfg, b, g, row, e) for e in range(wl.D)]
                        assert np.array_equal(side[v_off].view(np.int8), vcodes)
                    else:
                        assert np.all(side[k_off] == 0xA5), (s, w, b, row)
        assert side.size == sb * wl.B


# ----------------------------------------------------------------------------- decode

def _vbf(buf, base: int, D: int, r: int, e: int) -> float:
    """bf16 value element e of row r of a 16-row V block starting at base: rows 2p, 2p+1 form a
    pair, element group gq = e // (D/8); the pair's group chunk (D/2 bytes) sits at chunk index
    (p // 4) * 32 + gq * 4 + p % 4 and holds per element the pair's two bf16 (row 2p first); its
    16-byte units are permuted by xor with (p%4 & 2 | gq & 1) for 4 units, gq & 1 for 2."""
    p, dg = r // 2, D // 8
    gq, m = divmod(e, dg)
    units = D // 32
    swz = ((p % 4) & 2 | (gq & 1)) if units >= 4 else ((gq & 1) if units >= 2 else 0)
    chunk = base + (((p // 4) * 8 + gq) * 4 + p % 4) * (D // 2)
    byte = chunk + 16 * ((4 * m) // 16 ^ swz) + (4 * m) % 16 + 2 * (r % 2)
    bits = int(buf[byte]) | (int(buf[byte + 1]) << 8)
    return float(np.array([bits << 16], np.uint32).view(np.float32)[0])


def _brute_layout_decode(wl: W.Workload, pool, side, b: int, g: int, L: int, value_format: int = 0):
    """Independent restatement of the byte layout (written from the layout description, not
    from the C code) returning dense fp64 (khat rotated basis, vhat)."""
    D, P, s, w, Hkv = wl.D, wl.P, wl.s, wl.w, wl.Hkv
    vbf = value_format == 1
    tile4 = 16 * (D // 2 + 4 + 2 * D) if vbf else 16 * (D + 8)
    ntiles8 = (s + w + 15) // 16
    tile8 = 16 * (3 * D + 2) if vbf else 16 * (2 * D + 4)
    kh = np.zeros((L, D))
    vh = np.zeros((L, D))
    f16 = lambda buf, off: float(np.frombuffer(bytes(buf[off:off + 2]), np.float16)[0])
    for j in range(L):
        if j < min(s, L) or j >= max(s, L - w):
            row = j if j < s else s + j % w
            base = (b * Hkv + g) * ntiles8 * tile8 + (row // 16) * tile8
            r = row % 16
            ks = f16(side, base + 16 * D + 2 * r)
            vs = 0.0 if vbf else f16(side, base + 32 * D + 32 + 2 * r)
            for e in range(D):
                kb = base + r * D + 16 * ((e // 16) ^ (r & 1)) + e % 16
                kh[j, e] = ks * np.int8(side[kb])
                if vbf:
                    vh[j, e] = _vbf(side, base + 16 * D + 32, D, r, e)
                    continue
                p_, half, pl = (r >> 1), (r >> 1) >> 2, (r >> 1) & 3
                dg, ch8 = D // 8, D // 4
                gq, dd = e // dg, e % dg
                bb = (dd // 2) * 4 + (dd % 2) * 2 + (r & 1)
                if ch8 >= 32:
                    bb ^= 16 * (gq & 1)
                vb = base + 16 * D + 32 + ((half * 8 + gq) * 4 + pl) * ch8 + bb
                vh[j, e] = vs * np.int8(side[vb])
        else:
            page = wl.page_table[b, j // P]
            pp = j % P
            base = page * Hkv * P * (tile4 // 16) + g * P * (tile4 // 16) + (pp // 16) * tile4
            r = pp % 16
            kpar = base + (8 * D if vbf else 16 * D) + 4 * r
            ks, kz = f16(pool, kpar), f16(pool, kpar + 2)
            if not vbf:
                vs, vz = f16(pool, base + 16 * D + 64 + 4 * r), f16(pool, base + 16 * D + 64 + 4 * r + 2)
            for e in range(D):
                # K: pair-row r % 8 of D bytes, row r in the low (r < 8) or high nibble; element e
                # in 8-byte group e // 8 (even elements first); 16-byte halves of each 32 bytes
                # swapped in odd pair-rows when D >= 128
                pr = r % 8
                bi = 8 * (e // 8) + (e % 2) * 4 + (e % 8) // 2
                unit = (bi // 16) ^ ((pr % 2) if D >= 128 else 0)
                byte = pool[base + pr * D + 16 * unit + bi % 16]
                kh[j, e] = kz + ks * ((byte >> 4) if r >= 8 else (byte & 15))
                if vbf:
                    vh[j, e] = _vbf(pool, base + 8 * D + 64, D, r, e)
                    continue
                Q, k = e // 4, e % 4
                wpc = D // 32
                p_ = r >> 1
                off = (((p_ >> 2) * 8 + Q // wpc) * 4 + (p_ & 3)) * (4 * wpc) + 4 * (Q % wpc) + 2 * (r & 1) + (k >> 1)
                byte = pool[base + 8 * D + off]
                vh[j, e] = vz + vs * ((byte >> 4) if k & 1 else (byte & 15))
    return kh, vh


def pin_brute_force(seed: int = 21):
    """Tiny cases: the oracle's decode against a direct fp64 triple loop with an explicit
    Hadamard matrix, on a cache read back through an independent layout decoder (INT4 values,
    and bf16 values for the last two cases)."""
    for (lens, s, w, h, G, D, vf) in (((12, 7, 3), 2, 5, 8, 2, 32, 0), ((11, 1, 9), 0, 4, 32, 1, 32, 0),
                                      ((10, 12, 5), 3, 0, 4, 2, 32, 0), ((21, 3), 1, 2, 16, 1, 128, 0),
                                      ((19, 6, 2), 2, 4, 8, 2, 64, 1), ((21, 3), 1, 2, 16, 1, 128, 1)):
        wl = small_workload(D=D, lens=lens, s=s, w=w, h=h, G=G, seed=seed)
        cfg, pool, side = build_cache(wl, value_format=vf)
        q = wl.q_input(0)
        out, lse = O.decode(cfg, pool, side, q, wl.page_table, wl.lens)
        Hm = np.kron(np.eye(wl.D // h), scipy.linalg.hadamard(h)).astype(np.float64)
        for b, L in enumerate(wl.lens):
            for g in range(wl.Hkv):
                kh, vh = _brute_layout_decode(wl, pool, side, b, g, L, value_format=vf)
                kd, vd, _ = O.dequant_seq(cfg, pool, side, wl.page_table[b], b, L, g)
                assert np.array_equal(kh, kd) and np.array_equal(vh, vd)
                for i in range(G):
                    j = g * G + i
                    qr = Hm @ q[b, j].astype(np.float64) / h
                    logits = np.array([sum(qr[e] * kh[t, e] for e in range(wl.D)) for t in range(L)]) / np.sqrt(wl.D)
                    p = np.exp(logits - logits.max())
                    ref = (p[:, None] * vh).sum(0) / p.sum()
                    ref_lse = logits.max() + np.log(p.sum())
                    assert np.allclose(out[b, j], ref, rtol=1e-12, atol=1e-12), np.abs(out[b, j] - ref).max()
                    assert abs(lse[b, j] - ref_lse) <= 1e-12 * max(1, abs(ref_lse))


def pin_append_vs_numpy_requant(seed: int = 31):
    """Codes, scale and zero bits written by the oracle's append equal an independent NumPy
    re-quantisation (reading R3) of the rotated key / raw value, at the layout positions."""
    wl = small_workload(lens=(20, 33), B=2, s=2, w=5, h=16, seed=seed)
    cfg, pool, side = build_cache(wl)
    Hm = np.kron(np.eye(wl.D // wl.h), scipy.linalg.hadamard(wl.h))
    for b, L in enumerate(wl.lens):
        K, V = wl.kv_inputs(0, np.full(L, b, np.int32), np.arange(L, dtype=np.int32))
        for j in range(L):
            page, pp = wl.page_table[b, j // wl.P], j % wl.P
            for g in range(wl.Hkv):
                kr = O.fwht_f32(K[j, g], wl.h)
                assert np.allclose(kr, Hm @ K[j, g].astype(np.float64), rtol=1e-6, atol=1e-4)
                for isv, x in ((0, kr), (1, V[j, g])):
                    codes, sc, zr = _requant_int4_numpy(x)
                    kind = "v4" if isv else "k4"
                    got = np.array([(pool[O.byte_offset(kind, cfg, page, g, pp, e)]
                                     >> (4 * O.nibble_high(kind, cfg, pp, e))) & 15 for e in range(wl.D)])
                    assert np.array_equal(got, codes), (b, j, g, isv)
                    off = O.byte_offset("p4", cfg, page, g, pp, isv)
                    assert int(pool[off]) | (int(pool[off + 1]) << 8) == sc
                    assert int(pool[off + 2]) | (int(pool[off + 3]) << 8) == zr


def pin_regional_equals_single(seed: int = 41):
    for (lens, s, w, chunk) in (((300, 129, 40, 1), 4, 32, 37), ((257, 64), 0, 0, 50), ((90, 6), 16, 64, 7)):
        wl = small_workload(D=64, lens=lens, B=len(lens), s=s, w=w, h=64, seed=seed)
        cfg, pool, side = build_cache(wl)
        q = wl.q_input(0)
        o1, l1 = O.decode(cfg, pool, side, q, wl.page_table, wl.lens, mode=O.SINGLE)
        for ct, rev in ((0, False), (chunk, False), (chunk, True), (16, True)):
            o2, l2 = O.decode(cfg, pool, side, q, wl.page_table, wl.lens, mode=O.REGIONAL,
                              chunk_tokens=ct, reverse=rev)
            scale = np.abs(o1).max()
            assert np.abs(o1 - o2).max() <= 1e-12 * max(1.0, scale), (ct, rev, np.abs(o1 - o2).max())
            assert np.abs(l1 - l2).max() <= 1e-12 * max(1.0, np.abs(l1).max())


def sign_vector(words, D: int) -> np.ndarray:
    return np.array([-1.0 if (int(words[d >> 5]) >> (d & 31)) & 1 else 1.0 for d in range(D)])


def pin_signed_rotation_exact(seed: int = 53):
    """The append's key rotation with randomised signs is H diag(s) x: on integer vectors the fp32
    butterfly equals the explicit matrix product exactly."""
    rng = np.random.default_rng(seed)
    for D in (32, 64):
        for h in (1, 8, D):
            words = tuple(int(x) for x in rng.integers(0, 2**32, size=4, dtype=np.uint64))
            cfg = O.Config(2, 1, D, 16, 2, 4, h, 1, words)
            Hm = np.kron(np.eye(D // h), scipy.linalg.hadamard(h)).astype(np.float64)
            S = sign_vector(words, D)
            for _ in range(5):
                x = rng.integers(-7, 8, size=D).astype(np.float32)
                assert np.array_equal(O.rotate_key(cfg, x).astype(np.float64), Hm @ (S * x))


def pin_rotation_invariance(seed: int = 51):
    """tau * q_rot . khat_rot equals tau * q . (diag(s) H^T khat_rot / h): the stored rotated keys
    seen by the unrotated query through the inverse transform (H^T H = h I, s_d^2 = 1), with and
    without randomised signs."""
    rng = np.random.default_rng(seed)
    for h, words in ((1, (0, 0, 0, 0)), (8, (0, 0, 0, 0)), (32, (0, 0, 0, 0)),
                     (8, tuple(int(x) for x in rng.integers(0, 2**32, size=4, dtype=np.uint64))),
                     (32, tuple(int(x) for x in rng.integers(0, 2**32, size=4, dtype=np.uint64)))):
        wl = small_workload(D=32, lens=(30,), B=1, s=2, w=4, h=h, seed=seed)
        cfg, pool, side = build_cache(wl, signs=words)
        q = wl.q_input(0)
        out, _ = O.decode(cfg, pool, side, q, wl.page_table, wl.lens, mode=O.SINGLE)
        Hm = np.kron(np.eye(wl.D // h), scipy.linalg.hadamard(h)).astype(np.float64)
        kd, vd, _ = O.dequant_seq(cfg, pool, side, wl.page_table[0], 0, 30, 0)
        k_unrot = (kd @ Hm / h) * sign_vector(words, wl.D)[None, :]  # rows: diag(s) H^T khat / h
        for i in range(wl.G):
            logits = k_unrot @ q[0, i].astype(np.float64) / np.sqrt(wl.D)
            p = np.exp(logits - logits.max())
            ref = (p[:, None] * vd).sum(0) / p.sum()
            assert np.abs(out[0, i] - ref).max() <= 1e-12 * max(1, np.abs(ref).max())


def pin_value_rotation_invariance(seed: int = 57):
    """With values stored rotated (H diag(s) v) the decode output, rotated back, equals attention
    over the de-rotated dequantised values diag(s) H^T vhat_rot / h (and de-rotated keys)."""
    rng = np.random.default_rng(seed)
    for h in (1, 8, 32):
        words = tuple(int(x) for x in rng.integers(0, 2**32, size=4, dtype=np.uint64))
        wl = small_workload(D=32, lens=(30,), B=1, s=2, w=4, h=h, seed=seed)
        cfg, pool, side = build_cache(wl, signs=words, rotate_values=1)
        q = wl.q_input(0)
        out, _ = O.decode(cfg, pool, side, q, wl.page_table, wl.lens, mode=O.SINGLE)
        Hm = np.kron(np.eye(wl.D // h), scipy.linalg.hadamard(h)).astype(np.float64)
        S = sign_vector(words, wl.D)[None, :]
        kd, vd, _ = O.dequant_seq(cfg, pool, side, wl.page_table[0], 0, 30, 0)
        k_unrot = (kd @ Hm / h) * S
        v_unrot = (vd @ Hm / h) * S
        for i in range(wl.G):
            logits = k_unrot @ q[0, i].astype(np.float64) / np.sqrt(wl.D)
            p = np.exp(logits - logits.max())
            ref = (p[:, None] * v_unrot).sum(0) / p.sum()
            assert np.abs(out[0, i] - ref).max() <= 1e-12 * max(1, np.abs(ref).max())
        # the stored values are rotated: dequantised rows differ from the unrotated cache's
        _, vd0, _ = O.dequant_seq(*build_cache(wl, signs=words), wl.page_table[0], 0, 30, 0)
        assert not np.allclose(vd, vd0)


def pin_special_cases(seed: int = 61):
    # L = 1: a single position -> out equals its dequantised value exactly
    wl = small_workload(lens=(1, 1), B=2, s=2, w=5, seed=seed)
    cfg, pool, side = build_cache(wl)
    out, lse = O.decode(cfg, pool, side, wl.q_input(0), wl.page_table, wl.lens)
    for b in range(2):
        for g in range(wl.Hkv):
            _, vd, reg = O.dequant_seq(cfg, pool, side, wl.page_table[b], b, 1, g)
            for i in range(wl.G):
                assert np.array_equal(out[b, g * wl.G + i], vd[0])
    # q = 0: uniform weights -> mean of vhat over [0, L)
    wl = small_workload(lens=(37, 9), B=2, s=2, w=5, seed=seed + 1)
    cfg, pool, side = build_cache(wl)
    q0 = np.zeros((2, wl.Hq, wl.D), np.float32)
    out, lse = O.decode(cfg, pool, side, q0, wl.page_table, wl.lens)
    for b, L in enumerate(wl.lens):
        for g in range(wl.Hkv):
            _, vd, _ = O.dequant_seq(cfg, pool, side, wl.page_table[b], b, L, g)
            for i in range(wl.G):
                assert np.allclose(out[b, g * wl.G + i], vd.mean(0), rtol=1e-13, atol=1e-13)
                assert abs(lse[b, g * wl.G + i] - np.log(L)) < 1e-13
    # s = w = 0: pure INT4; L <= s + w: pure INT8 (regions reported by dequant_seq)
    for (s, w, L, want) in ((0, 0, 30, {1}), (4, 40, 30, {0, 2}), (4, 40, 3, {0})):
        wl = small_workload(lens=(L,), B=1, s=s, w=w, seed=seed + 2)
        cfg, pool, side = build_cache(wl)
        _, _, reg = O.dequant_seq(cfg, pool, side, wl.page_table[0], 0, L, 0)
        assert set(reg.tolist()) == want, (s, w, L, set(reg.tolist()))
    # region sizes: |S| = min(s, L), |R| = min(max(L - s, 0), w), |M| = max(0, L - s - w)
    for (s, w, L) in ((4, 32, 256), (4, 32, 20), (4, 32, 3), (0, 8, 5), (6, 0, 10)):
        wl = small_workload(lens=(L,), B=1, s=s, w=w, seed=seed + 3)
        cfg, pool, side = build_cache(wl)
        _, _, reg = O.dequant_seq(cfg, pool, side, wl.page_table[0], 0, L, 0)
        assert (reg == 0).sum() == min(s, L)
        assert (reg == 2).sum() == min(max(L - s, 0), w)
        assert (reg == 1).sum() == max(0, L - s - w)


ALL_PINS = [
    pin_fp16_golden, pin_fp16_vs_numpy, pin_fp16_decode_all, pin_hadamard_matrix,
    pin_hadamard_golden, pin_hadamard_integer_exact, pin_quant_golden, pin_quant_int4_bounds,
    pin_quant_int4_constant, pin_quant_int8_bounds, pin_storage_bits, pin_layout_bijection,
    lambda: pin_routing(False), lambda: pin_routing(True), pin_brute_force,
    pin_append_vs_numpy_requant, pin_regional_equals_single, pin_rotation_invariance,
    pin_special_cases, pin_signed_rotation_exact, pin_value_rotation_invariance, pin_quant_range,
    pin_append_range_flag, pin_bf16_rounding, pin_layout_bijection_bf16_values, pin_bf16_values_exact,
]

# the mixed bit-width key cache's pins run with the rest (the mutation test runs ALL_PINS)
import gtq_pins as _G  # noqa: E402

ALL_PINS = ALL_PINS + list(_G.GTQ_PINS)
