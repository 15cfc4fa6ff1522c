"""A Python model of the flattened split-K schedule of the decode kernels, checked on the CPU.

The decode kernel gives warp w the tiles whose first slot lies in [w*Q, (w+1)*Q) of the
sequence of all slots (per sequence b, per KV head g: the INT8 segment of ceil((s+w)/16) tiles
of 2 slots, then the INT4 segment of the 16-position tiles covering [s, max(s, L-w))), writes one
partial per (warp, segment) at index warp + segment_id, and the merge of (b, g) reads, for each
segment, the partials of warps floor(first_slot/Q) .. floor(last_tile_start/Q).  The merge kernel
numbers the partials of (b, g) j = 0.. (INT8-segment writers first, then INT4) and finds partial j
at index w8a + j + sid8 (INT8) or w4a + (j - n8p) + sid8 + 1 (INT4).  This model restates that
arithmetic and checks its invariants for many length mixes and grid sizes: every tile processed
exactly once, partial indices unique and inside the workspace, the merge reads exactly the
partials that were written (and finds each at the index its writer used), a (b, g) with a single
partial is recognised as such by its writer, and every bulk-copy source lies inside its buffer.
"""
import numpy as np
import pytest



def side_tiles_used(L, s, w, nt8):
    """The kernel's rule: tiles up to one past the last side row in use while the recent ring has
    not wrapped (rows end at L + (s mod w), or at L when L <= s), else all nt8."""
    smw = s % w if w > 0 else 0
    top = L if L <= s else L + smw
    return 0 if L <= 0 else ((top + 15) // 16 if top <= s + w else nt8)


def side_rows_used(L, s, w):
    """Side rows holding a position at length L: sinks j < min(s, L) at row j, recent
    j in [max(s, L - w), L) at row s + j mod w."""
    rows = set(range(min(s, L)))
    if w > 0:
        rows |= {s + j % w for j in range(max(s, L - w), L)}
    return rows


TIGHT_SIDE_TILES = 16  # side caches with more tiles visit only the tiles in use


def seg_info(L, s, w, nt8):
    n8 = side_tiles_used(L, s, w, nt8) if nt8 > TIGHT_SIDE_TILES else (nt8 if L > 0 else 0)
    m_end = max(s, L - w)
    t4a = s >> 4
    n4 = ((m_end - 1) >> 4) - t4a + 1 if m_end > s else 0
    return n8, n4, t4a, m_end


def model(lens, Hkv, s, w, P, stride, W):
    nt8 = (s + w + 15) // 16
    cap = stride * P
    lens = [min(max(L, 0), cap) for L in lens]
    # every tile: (start_slot, b, g, seg, i, nslots)
    tiles = []
    pos = 0
    for b, L in enumerate(lens):
        n8, n4, t4a, m_end = seg_info(L, s, w, nt8)
        for g in range(Hkv):
            for i in range(n8):
                tiles.append((pos, b, g, 0, i, 2))
                pos += 2
            for i in range(n4):
                tiles.append((pos, b, g, 1, i, 1))
                pos += 1
    total = pos
    Q = max(2, -(-total // W)) if total else 2
    owner = {}
    written = set()
    for (start, b, g, seg, i, n) in tiles:
        w_ = start // Q
        assert w_ < W
        owner[(b, g, seg, i)] = w_
        sid = 2 * (b * Hkv + g) + seg
        written.add((w_ + sid, b, g, seg, w_))
    # partial indices unique and within W + 2*B*Hkv
    idx = [x[0] for x in written]
    assert len(idx) == len(set(idx))
    assert all(0 <= v < W + 2 * len(lens) * Hkv for v in idx)
    # merge ranges
    pos = 0
    for b, L in enumerate(lens):
        n8, n4, t4a, m_end = seg_info(L, s, w, nt8)
        for g in range(Hkv):
            for seg, cnt, tc in ((0, n8, 2), (1, n4, 1)):
                cs = pos
                ce = cs + cnt * tc
                pos = ce
                if ce <= cs:
                    continue
                sid = 2 * (b * Hkv + g) + seg
                readers = set(range(cs // Q, (ce - tc) // Q + 1))
                writers = {x[4] for x in written if x[1] == b and x[2] == g and x[3] == seg}
                assert readers == writers, (b, g, seg, readers, writers)
        # ordinals and merge groups of each (b, g), as the kernel computes them
        for g in range(Hkv):
            cs8 = sum(Hkv * (2 * seg_info(lens[x], s, w, nt8)[0] + seg_info(lens[x], s, w, nt8)[1]) for x in range(b))
            cs8 += g * (2 * n8 + n4)
            cs4 = cs8 + 2 * n8
            w8a, w4a = cs8 // Q, cs4 // Q
            n8p = (cs4 - 2) // Q - w8a + 1 if n8 else 0
            n4p = (cs4 + n4 - 1) // Q - w4a + 1 if n4 else 0
            sid8 = 2 * (b * Hkv + g)
            parts = sorted(x[0] for x in written if x[1] == b and x[2] == g and x[3] == 0) + \
                sorted(x[0] for x in written if x[1] == b and x[2] == g and x[3] == 1)
            assert len(parts) == n8p + n4p
            for j, idx in enumerate(parts):
                kernel_idx = (w8a + j + sid8) if j < n8p else (w4a + (j - n8p) + sid8 + 1)
                assert kernel_idx == idx
                seg, wr = (0, idx - sid8) if j < n8p else (1, idx - sid8 - 1)
                jme = (wr - w8a) if seg == 0 else n8p + (wr - w4a)
                assert jme == j
            assert (len(parts) == 1) == (n8p + n4p == 1)
        # the visited side tiles hold every side row in use
        assert all(r < 16 * n8 for r in side_rows_used(L, s, w))
        # INT4 tiles address pages inside the page-table row
        for i in range(n4):
            ti = t4a + i
            assert (ti * 16) // P < stride
            assert ti * 16 < max(L, 1) + 15
    return total


@pytest.mark.parametrize("seed", range(40))
def test_schedule_invariants(seed):
    rng = np.random.default_rng(seed)
    B = int(rng.integers(1, 40))
    Hkv = int(rng.choice([1, 2, 8]))
    s = int(rng.choice([0, 1, 4, 16, 19]))
    w = int(rng.choice([0, 8, 32, 128]))
    P = int(rng.choice([16, 32, 64]))
    lens = rng.integers(0, 3000, size=B).tolist()
    if seed % 5 == 0:
        lens = [1, 0, s, s + 1, s + w, s + w + 1][:B] + lens[6:]
    if seed % 5 == 1:  # short sequences and the all-INT8 configuration (w above every length)
        lens = rng.integers(0, 2 * (s + w) + 3, size=B).tolist()
    if seed % 7 == 3:  # all-INT8: a side cache of more than 16 tiles, visited only where filled
        s, w = 0, int(max(lens)) + int(rng.integers(0, 40))
    if seed % 7 == 5:  # sinks and a long recent window (ring wraps for the longest sequences)
        s, w = int(rng.integers(1, 20)), int(rng.choice([300, 700]))
        lens = rng.integers(0, s + 2 * w, size=B).tolist()
    stride = max(1, (max(lens) + P - 1) // P)
    for W in (1, 3, 8, 37, 296, 2368):
        model(lens, Hkv, s, w, P, stride, W)


def test_lengths_beyond_page_table_are_clamped():
    # a length past stride*P is clamped to it (the merge kernel also raises a device error bit)
    model([10_000, 5], 2, 4, 32, 16, 4, 64)


def test_fast_division_multiplier():
    """The decode kernel divides by the per-launch unit count Q >= 2 as umulhi(n, m) with
    m = floor((2^32 - 1) / Q) + 1, corrected by one multiply-compare.  m equals ceil(2^32 / Q)
    for every Q >= 2, and the corrected quotient is exact for n < 2^31."""
    import numpy as np
    rng = np.random.default_rng(5)
    # Q < 2^31: the unit total is below 2^31 (the host refuses larger launches)
    ds = [2, 3, 4, 7, 8, 1000, 1024, 65535, 65536, 2**30 + 3, 2**31 - 1]
    ds += [int(x) for x in rng.integers(2, 2**31, size=200)]
    for d in ds:
        m = (2**32 - 1) // d + 1
        assert m == -(-2**32 // d)
        assert m < 2**32
        ns = [0, 1, d - 1, d, d + 1, 2**31 - 1] + [int(x) for x in rng.integers(0, 2**31, size=50)]
        for n in ns:
            if n >= 2**31:
                continue
            q = (n * m) >> 32                 # umulhi
            if (q * d) & 0xFFFFFFFF > n:      # 32-bit product, as in the kernel (q d < 2^32 here)
                q -= 1
            assert q == n // d, (n, d)


def test_side_tiles_used_cover_every_side_row():
    """Exhaustive over small budgets: the side tiles a decode visits hold every side row in use,
    and a sequence whose ring has not wrapped visits no tile past its last used row."""
    for s in range(0, 40, 3):
        for w in (0, 1, 5, 16, 17, 40):
            nt8 = (s + w + 15) // 16
            for L in range(0, 2 * (s + w) + 20):
                n8 = side_tiles_used(L, s, w, nt8)
                rows = side_rows_used(L, s, w)
                assert 0 <= n8 <= nt8
                assert all(r < 16 * n8 for r in rows), (s, w, L)
                if rows and n8 < nt8:
                    assert n8 == (max(rows) + 16) // 16, (s, w, L)
