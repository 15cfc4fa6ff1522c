"""GPU (C ABI) against the CPU oracle on the same seeded inputs.

Append: the page pool and side cache bytes written by kv4_append equal the oracle's byte for
byte (codes, fp16 scale/zero bits, INT8 routing, untouched bytes keep the 0xA5 fill).
Decode: kv4_decode_attn output within max-abs 2e-3 and relative-L2 1e-3 of the fp64 oracle on
the same dequantised cache, lse within 1e-4.
"""
import numpy as np
import pytest
import torch

from int4_kv_cache_append_b200 import workload as W
from oracle import oracle as O

import kv4_testlib as T

pytestmark = pytest.mark.gpu

# (name, D, Hq, Hkv, P, s, w, h, lens, k_dtype, v_dtype, q_dtype)
CASES = [
    ("tiny-cfg", None, None, None, None, None, None, None, None, None, None, None),
    ("d128-g4-bf16", 128, 8, 2, 16, 4, 16, 128, (300, 37, 1, 4, 5, 20, 21, 129), W.BF16, W.BF16, W.BF16),
    ("d128-g4-p64-h32", 128, 8, 2, 64, 4, 48, 32, (333, 64, 65, 200), W.F32, W.BF16, W.BF16),
    ("d64-g1-h1", 64, 2, 2, 16, 2, 8, 1, (50, 17, 3), W.F32, W.F32, W.F32),
    ("d128-g2-no-side", 128, 4, 2, 32, 0, 0, 64, (96, 33, 7), W.BF16, W.BF16, W.BF16),
    ("d128-g4-sinks-only", 128, 4, 1, 16, 8, 0, 16, (40, 8, 3), W.F32, W.F32, W.BF16),
    ("d64-g4-recent-only", 64, 8, 2, 16, 0, 24, 64, (90, 24, 25, 2), W.BF16, W.F32, W.F32),
    ("d128-g4-wide-s", 128, 4, 1, 16, 19, 13, 128, (100, 19, 20, 31, 32, 33), W.BF16, W.BF16, W.BF16),
    # KV8: no sinks and a recent window longer than every sequence, so every position is read
    # from the INT8 side cache
    ("d128-g4-kv8", 128, 8, 2, 16, 0, 208, 128, (200, 77, 1, 16, 17), W.BF16, W.BF16, W.BF16),
    # side caches of more than 16 tiles: the decode visits only the side tiles in use (all-INT8
    # with a window longer than every sequence; sinks with a long ring that wraps for some)
    ("d64-g2-kv8-long-window", 64, 4, 2, 16, 0, 400, 64, (350, 77, 1, 16, 17, 260), W.BF16, W.BF16, W.BF16),
    ("d128-g4-long-ring", 128, 8, 2, 16, 5, 300, 128, (20, 306, 400, 3, 305, 290), W.BF16, W.BF16, W.BF16),
    # more than 256 sequences: the decode prologue reads the lengths from memory instead of
    # keeping them in registers
    ("d64-g2-b300", 64, 4, 2, 16, 4, 16, 64,
     tuple(int(x) for x in np.random.default_rng(300).integers(0, 90, size=300)), W.BF16, W.BF16, W.BF16),
]


def make(case):
    name, D, Hq, Hkv, P, s, w, h, lens, kd, vd, qd = case
    if name == "tiny-cfg":
        return W.tiny_cfg()
    return W.make_workload(name, 17, 1, len(lens), Hq, Hkv, D, P, s, w, h, lambda r: list(lens), kd, vd, qd, 2, 20.0)


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
@pytest.mark.parametrize("step_by_step", [False, True], ids=["prefill", "stepwise"])
def test_append_bit_exact(case, step_by_step):
    wl = make(case)
    if step_by_step and wl.lens.max() > 160:
        wl.lens = np.minimum(wl.lens, 160).astype(np.int32)
    gc = T.gpu_cache_from_host_inputs(wl, step_by_step=step_by_step)
    cfg, pool, side = T.oracle_cache(wl, step_by_step=step_by_step)
    gp, gs = gc.layer_views(0)
    gp = gp.cpu().numpy()
    gs = gs.cpu().numpy()
    assert gp.size == pool.size and gs.size == side.size
    bad = np.nonzero(gp != pool)[0]
    assert bad.size == 0, f"page pool differs at {bad.size} bytes, first {bad[:8]}"
    bad = np.nonzero(gs != side)[0]
    assert bad.size == 0, f"side cache differs at {bad.size} bytes, first {bad[:8]}"
    from int4_kv_cache_append_b200 import kv4
    assert kv4.kv4_get_device_error() == 0


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_decode_matches_oracle(case):
    wl = make(case)
    gc = T.gpu_cache_from_host_inputs(wl)
    cfg, pool, side = T.oracle_cache(wl)
    q = wl.q_input(0)
    ref, ref_lse = T.oracle_decode(wl, cfg, pool, side, q)
    out, lse = T.gpu_decode(gc, wl, q)
    T.assert_close(out, ref, lse, ref_lse, what=case[0])
    # the regional merge equals one softmax over the whole dequantised cache
    single, _ = T.oracle_decode(wl, cfg, pool, side, q, mode=O.SINGLE)
    T.assert_close(out, single, what=case[0] + " vs single softmax")
    from int4_kv_cache_append_b200 import kv4
    assert kv4.kv4_get_device_error() == 0


def test_decode_on_oracle_built_cache():
    """The decode kernel alone: bytes written by the oracle, uploaded, decoded on the GPU."""
    wl = make(CASES[1])
    cfg, pool, side = T.oracle_cache(wl)
    from int4_kv_cache_append_b200 import kv4
    gc = kv4.Cache(T.geometry(wl))
    gp, gs = gc.layer_views(0)
    gp.copy_(torch.from_numpy(pool))
    gs.copy_(torch.from_numpy(side))
    q = wl.q_input(0)
    ref, ref_lse = T.oracle_decode(wl, cfg, pool, side, q)
    out, lse = T.gpu_decode(gc, wl, q)
    T.assert_close(out, ref, lse, ref_lse, what="oracle-built cache")


def test_decode_split_count_invariance():
    """Different grid sizes (hence different split points) give the same result within tolerance."""
    wl = W.make_workload("split", 23, 1, 3, 8, 2, 128, 16, 4, 32, 128, lambda r: [900, 517, 64],
                         W.BF16, W.BF16, W.BF16, 4, 15.0)
    gc = T.gpu_cache_from_host_inputs(wl)
    cfg, pool, side = T.oracle_cache(wl)
    q = wl.q_input(0)
    ref, ref_lse = T.oracle_decode(wl, cfg, pool, side, q)
    outs = []
    for hint in (0, 1, 16, 64, 900):
        out, lse = T.gpu_decode(gc, wl, q, max_len_hint=hint)
        T.assert_close(out, ref, lse, ref_lse, what=f"hint {hint}")
        outs.append(out)
    for o in outs[1:]:
        T.assert_close(o, outs[0].astype(np.float64), what="split vs split")


def test_page_permutation_invariance():
    """Moving pages to other physical slots (table updated) gives bit-identical outputs."""
    wl = make(CASES[1])
    q = wl.q_input(0)
    gc = T.gpu_cache_from_host_inputs(wl)
    out1, lse1 = T.gpu_decode(gc, wl, q)
    rng = np.random.default_rng(99)
    perm = rng.permutation(wl.num_pages).astype(np.int32)
    wl2 = W.Workload(**{**wl.__dict__, "page_table": np.where(wl.page_table >= 0, perm[wl.page_table], 0).astype(np.int32)})
    gc2 = T.gpu_cache_from_host_inputs(wl2)
    out2, lse2 = T.gpu_decode(gc2, wl2, q)
    assert np.array_equal(out1, out2) and np.array_equal(lse1, lse2)


def test_zero_length_and_single_token():
    wl = W.make_workload("edge", 29, 1, 4, 8, 2, 128, 16, 4, 16, 128, lambda r: [1, 0, 2, 23],
                         W.BF16, W.BF16, W.BF16, 2, 20.0)
    gc = T.gpu_cache_from_host_inputs(wl)
    cfg, pool, side = T.oracle_cache(wl)
    q = wl.q_input(0)
    ref, ref_lse = T.oracle_decode(wl, cfg, pool, side, q)
    out, lse = T.gpu_decode(gc, wl, q)
    assert np.all(out[1] == 0) and np.all(np.isneginf(lse[1]))
    T.assert_close(out, ref, lse, ref_lse, what="edge lengths")
    # L = 1: the output is the single (INT8) value exactly up to fp32 rounding
    _, vd, _ = O.dequant_seq(cfg, pool, side, wl.page_table[0], 0, 1, 0)
    assert np.abs(out[0, 0] - vd[0]).max() <= 1e-5 * max(1.0, np.abs(vd[0]).max())


def test_out_of_range_page_sets_error_bit_without_fault():
    """A page id outside the pool is caught by the kernels' guards: the access is skipped and
    the device error word reports it (the process and the context stay healthy)."""
    from int4_kv_cache_append_b200 import kv4
    wl = make(CASES[1])
    gc = T.gpu_cache_from_host_inputs(wl)
    assert kv4.kv4_get_device_error() == 0
    bad = wl.page_table.copy()
    bad[0, 5] = wl.num_pages + 1000
    q = T.to_dev(wl.q_input(0))
    lens = torch.from_numpy(wl.lens).cuda()
    gc.decode(0, q, torch.from_numpy(bad).cuda(), lens)
    torch.cuda.synchronize()
    assert kv4.kv4_get_device_error() & kv4.KV4_DEVERR_PAGE_RANGE
    out, _ = T.gpu_decode(gc, wl, wl.q_input(0))
    assert np.isfinite(out).all()


def _bf16_reference(wl, lens, q_host):
    """fp64 attention over bf16-rounded K/V (no rotation, no quantisation)."""
    out = np.zeros((len(lens), wl.Hq, wl.D))
    lse = np.zeros((len(lens), wl.Hq))
    q = W.bf16_to_f32(q_host).astype(np.float64) if q_host.dtype == np.uint16 else q_host.astype(np.float64)
    for b, L in enumerate(lens):
        if L == 0:
            lse[b] = -np.inf
            continue
        K, V = wl.kv_inputs(0, np.full(L, b, np.int32), np.arange(L, dtype=np.int32))
        K = W.bf16_to_f32(K if K.dtype == np.uint16 else W.bf16_bits(K)).astype(np.float64)
        V = W.bf16_to_f32(V if V.dtype == np.uint16 else W.bf16_bits(V)).astype(np.float64)
        for j in range(wl.Hq):
            g = j // wl.G
            lg = K[:, g] @ q[b, j] / np.sqrt(wl.D)
            p = np.exp(lg - lg.max())
            out[b, j] = (p[:, None] * V[:, g]).sum(0) / p.sum()
            lse[b, j] = lg.max() + np.log(p.sum())
    return out, lse


@pytest.mark.parametrize("case", [CASES[1], CASES[2], CASES[3]], ids=[CASES[i][0] for i in (1, 2, 3)])
def test_bf16_baseline_matches_reference(case):
    from int4_kv_cache_append_b200 import kv4
    wl = make(case)
    bc = kv4.BF16Cache(T.geometry(wl))
    b, p = T.prefill_tokens(wl.lens)
    K, V = wl.kv_inputs(0, b, p)
    pt = torch.from_numpy(wl.page_table).cuda()
    bc.append(0, T.to_dev(K), T.to_dev(V), torch.from_numpy(b).cuda(), torch.from_numpy(p).cuda(), pt)
    q = wl.q_input(0)
    lse = torch.empty((wl.B, wl.Hq), device="cuda")
    out = bc.decode(0, T.to_dev(q), pt, torch.from_numpy(wl.lens).cuda(), lse=lse)
    ref, ref_lse = _bf16_reference(wl, wl.lens, q)
    # fp32 queries enter as bf16 hi/lo halves (about 16 bits): a looser logit tolerance applies
    loose = q.dtype != np.uint16
    T.assert_close(out.cpu().numpy(), ref, lse.cpu().numpy(), ref_lse, atol=2e-2 if loose else 2e-3,
                   rel_l2=5e-3 if loose else 1e-3, lse_atol=1e-3 if loose else 1e-4, what="bf16 " + case[0])


@pytest.mark.parametrize("overlap", [False, True], ids=["stream-order", "overlap"])
def test_append_then_decode_on_one_stream(overlap):
    """The decode kernel launched right after an append on the same stream (the append lets its
    dependent launch early; with overlap the decode builds its schedule before waiting on the
    append): the result is the oracle's, and identical with and without overlap."""
    from int4_kv_cache_append_b200 import kv4
    wl = make(CASES[1])
    gc = T.gpu_cache_from_host_inputs(wl, lens=wl.lens - 1)  # every sequence short of its last token
    cfg, pool, side = T.oracle_cache(wl)
    q = wl.q_input(0)
    ref, ref_lse = T.oracle_decode(wl, cfg, pool, side, q)
    rows = np.nonzero(wl.lens > 0)[0].astype(np.int32)
    pos = (wl.lens[rows] - 1).astype(np.int32)
    K, V = wl.kv_inputs(0, rows, pos)
    pt = torch.from_numpy(wl.page_table).cuda()
    lens = torch.from_numpy(wl.lens).cuda()
    kv4.kv4_set_decode_overlap(gc.handle, overlap)
    outs = []
    for _ in range(2):
        gc.append(0, T.to_dev(K), T.to_dev(V), torch.from_numpy(rows).cuda(), torch.from_numpy(pos).cuda(), lens, pt)
        lse = torch.empty((wl.B, wl.Hq), device="cuda")
        out = gc.decode(0, T.to_dev(q), pt, lens, lse=lse)
        torch.cuda.synchronize()
        outs.append((out.cpu().numpy(), lse.cpu().numpy()))
    kv4.kv4_set_decode_overlap(gc.handle, False)
    T.assert_close(outs[0][0], ref, outs[0][1], ref_lse, what=f"append->decode overlap={overlap}")
    assert np.array_equal(outs[0][0], outs[1][0]) and np.array_equal(outs[0][1], outs[1][1])
    assert kv4.kv4_get_device_error() == 0


@pytest.mark.parametrize("case_id", [1, 3], ids=["d128-h128", "d64-h1"])
def test_randomised_sign_rotation(case_id):
    """kv4_set_rotation_signs: keys stored in the H diag(s) basis are bit-exact against the oracle's
    same reading, and the decode (query rotated with the same signs) matches it."""
    from int4_kv_cache_append_b200 import kv4
    wl = make(CASES[case_id])
    words = [int(x) for x in np.random.default_rng(77 + case_id).integers(0, 2**32, size=4, dtype=np.uint64)]
    words = words[:(wl.D + 31) // 32] + [0] * (4 - (wl.D + 31) // 32)
    gc = T.gpu_cache_from_host_inputs(wl, signs=words)
    cfg, pool, side = T.oracle_cache(wl, signs=words)
    gp, gs = gc.layer_views(0)
    assert np.array_equal(gp.cpu().numpy(), pool) and np.array_equal(gs.cpu().numpy(), side)
    q = wl.q_input(0)
    ref, ref_lse = T.oracle_decode(wl, cfg, pool, side, q)
    out, lse = T.gpu_decode(gc, wl, q)
    T.assert_close(out, ref, lse, ref_lse, what=f"signed rotation {CASES[case_id][0]}")
    # without the signs the stored keys differ (the option is not a no-op)
    plain = T.oracle_cache(wl)[1]
    assert not np.array_equal(plain, pool)
    assert kv4.kv4_get_device_error() == 0


@pytest.mark.parametrize("case_id", [1, 3, 8], ids=["d128-h128", "d64-h1", "d128-kv8"])
def test_value_rotation(case_id):
    """kv4_set_value_rotation (with random signs): values stored in the keys' rotated basis are
    bit-exact against the oracle's same reading, and the decode output, rotated back by the merge,
    matches the oracle's."""
    from int4_kv_cache_append_b200 import kv4
    wl = make(CASES[case_id])
    words = [int(x) for x in np.random.default_rng(91 + case_id).integers(0, 2**32, size=4, dtype=np.uint64)]
    words = words[:(wl.D + 31) // 32] + [0] * (4 - (wl.D + 31) // 32)
    gc = T.gpu_cache_from_host_inputs(wl, signs=words, rotate_values=True)
    cfg, pool, side = T.oracle_cache(wl, signs=words, rotate_values=True)
    gp, gs = gc.layer_views(0)
    assert np.array_equal(gp.cpu().numpy(), pool) and np.array_equal(gs.cpu().numpy(), side)
    q = wl.q_input(0)
    ref, ref_lse = T.oracle_decode(wl, cfg, pool, side, q)
    out, lse = T.gpu_decode(gc, wl, q)
    T.assert_close(out, ref, lse, ref_lse, what=f"value rotation {CASES[case_id][0]}")
    assert kv4.kv4_get_device_error() == 0



@pytest.mark.parametrize("case_id", [1, 3], ids=["d128-g4", "d64-g1"])
def test_decode_f16_query(case_id):
    """fp16 queries (KV4_F16): the kernel widens them exactly, like the oracle's fp16 input path."""
    from int4_kv_cache_append_b200 import kv4
    wl = make(CASES[case_id])
    gc = T.gpu_cache_from_host_inputs(wl)
    cfg, pool, side = T.oracle_cache(wl)
    q32 = W.query_values(W.stream_key(wl.seed, W.KIND_Q, 0), wl.B, wl.Hq, wl.D)
    qbits = np.ascontiguousarray(q32.astype(np.float16).view(np.uint16))
    ref, ref_lse = O.decode(cfg, pool, side, qbits, wl.page_table, wl.lens, q_dtype=O.F16)
    qd = torch.from_numpy(qbits.view(np.int16)).cuda().view(torch.float16)
    lse = torch.empty((wl.B, wl.Hq), device="cuda")
    out = gc.decode(0, qd, torch.from_numpy(wl.page_table).cuda(), torch.from_numpy(wl.lens).cuda(), lse=lse)
    torch.cuda.synchronize()
    T.assert_close(out.cpu().numpy(), ref, lse.cpu().numpy(), ref_lse, what=f"fp16 q {CASES[case_id][0]}")
    # the fp16 query is not the bf16 one: the two oracle results differ
    qb = np.ascontiguousarray(W.bf16_bits(q32))
    other, _ = O.decode(cfg, pool, side, qb, wl.page_table, wl.lens, q_dtype=O.BF16)
    assert not np.allclose(other, ref, rtol=0, atol=1e-7)
    assert kv4.kv4_get_device_error() == 0


def test_range_overflow_sets_error_bit():
    """A key element of 1e6 (spread by the rotation, the vector's minimum is below -65504: its fp16
    offset is -inf) and a value element of 2e6 ((max - zero)/15 above 65504: scale +inf): the append
    stores both vectors with all-zero codes and their non-finite parameters, byte for byte as the
    oracle does, and reports KV4_DEVERR_RANGE; the other vectors are unaffected."""
    from int4_kv_cache_append_b200 import kv4
    wl = W.make_workload("range", 37, 1, 2, 8, 2, 128, 16, 4, 16, 64, lambda r: [40, 25],
                         W.F32, W.F32, W.F32, 2, 20.0)
    b, p = T.prefill_tokens(wl.lens)
    K, V = wl.kv_inputs(0, b, p)
    K = K.copy()
    V = V.copy()
    K[3, 1, 17] = 1.0e6   # position 3 of sequence 0: a sink (also in the side cache)
    V[45, 0, 5] = 2.0e6   # position 5 of sequence 1: INT4 only
    gc = kv4.Cache(T.geometry(wl), fill=0xA5)
    pt = torch.from_numpy(wl.page_table).cuda()
    assert kv4.kv4_get_device_error() == 0
    gc.append(0, T.to_dev(K), T.to_dev(V), torch.from_numpy(b).cuda(), torch.from_numpy(p).cuda(),
              torch.from_numpy(wl.lens).cuda(), pt)
    torch.cuda.synchronize()
    assert kv4.kv4_get_device_error() & kv4.KV4_DEVERR_RANGE
    cfg = O.Config(wl.Hq, wl.Hkv, wl.D, wl.P, wl.s, wl.w, wl.h, wl.B)
    pool = np.full(O.page_bytes(cfg) * wl.num_pages, 0xA5, np.uint8)
    side = np.full(O.side_slot_bytes(cfg) * wl.B, 0xA5, np.uint8)
    assert O.append(cfg, pool, side, K, V, b, p, wl.lens, wl.page_table)
    gp, gs = gc.layer_views(0)
    assert np.array_equal(gp.cpu().numpy(), pool) and np.array_equal(gs.cpu().numpy(), side)
    # the flagged key's stored offset is -inf, the flagged value's scale +inf
    off = O.byte_offset("p4", cfg, int(wl.page_table[0, 0]), 1, 3, 0)
    assert int(pool[off + 2]) | (int(pool[off + 3]) << 8) == 0xFC00
    off = O.byte_offset("p4", cfg, int(wl.page_table[1, 0]), 0, 5, 1)
    assert int(pool[off]) | (int(pool[off + 1]) << 8) == 0x7C00
    # without the planted elements nothing is reported
    K0, V0 = wl.kv_inputs(0, b, p)
    gc.append(0, T.to_dev(K0), T.to_dev(V0), torch.from_numpy(b).cuda(), torch.from_numpy(p).cuda(),
              torch.from_numpy(wl.lens).cuda(), pt)
    torch.cuda.synchronize()
    assert kv4.kv4_get_device_error() == 0


@pytest.mark.parametrize("case_id", [1, 11], ids=["b8", "b300"])
def test_wait_limit_failure_path_reports_and_recovers(case_id):
    """The device-side failure path of the bounded waits, made to run with the test hook (no
    invalid copy involved): every decode warp's first wait is on a barrier that nothing arrives
    on, runs out after its 1 ms limit, sets KV4_DEVERR_WAIT_LIMIT, waits for its copies in flight
    and returns.  The merge kernel then meets the workspace's stale records (0xA5 fill), which
    point outside the workspace, skips them and reports KV4_DEVERR_RECORD.  The context stays
    usable: with the hook off the next decode matches the oracle and reports nothing."""
    from int4_kv_cache_append_b200 import kv4
    wl = make(CASES[case_id])
    gc = T.gpu_cache_from_host_inputs(wl)
    assert kv4.kv4_get_device_error() == 0
    q_host = wl.q_input(0)
    pt = torch.from_numpy(wl.page_table).cuda()
    lens = torch.from_numpy(wl.lens).cuda()
    ws = torch.full((kv4.kv4_decode_workspace_bytes(gc.handle, wl.B),), 0xA5, dtype=torch.uint8, device="cuda")
    kv4.kv4_debug_force_wait_timeout(gc.handle, True)
    try:
        gc.decode(0, T.to_dev(q_host), pt, lens, workspace=ws)
        torch.cuda.synchronize()
    finally:
        kv4.kv4_debug_force_wait_timeout(gc.handle, False)
    err = kv4.kv4_get_device_error()
    assert err & kv4.KV4_DEVERR_WAIT_LIMIT, hex(err)
    assert err & kv4.KV4_DEVERR_RECORD, hex(err)
    cfg, pool, side = T.oracle_cache(wl)
    ref, ref_lse = T.oracle_decode(wl, cfg, pool, side, q_host)
    out, lse = T.gpu_decode(gc, wl, q_host)
    T.assert_close(out, ref, lse, ref_lse, what="decode after the wait-limit path")
    assert kv4.kv4_get_device_error() == 0


# K-INT4 / V-BF16: keys as in KV4, values stored as bf16 in the pages and the side cache
VBF_CASES = [CASES[1], CASES[3], CASES[7], CASES[8], CASES[10], CASES[11]]


@pytest.mark.parametrize("case", VBF_CASES, ids=[c[0] for c in VBF_CASES])
@pytest.mark.parametrize("step_by_step", [False, True], ids=["prefill", "stepwise"])
def test_bf16_values_append_bit_exact(case, step_by_step):
    from int4_kv_cache_append_b200 import kv4
    wl = make(case)
    if step_by_step and wl.lens.max() > 160:
        wl.lens = np.minimum(wl.lens, 160).astype(np.int32)
    gc = T.gpu_cache_from_host_inputs(wl, step_by_step=step_by_step, value_format=1)
    cfg, pool, side = T.oracle_cache(wl, step_by_step=step_by_step, value_format=1)
    gp, gs = gc.layer_views(0)
    gp, gs = gp.cpu().numpy(), gs.cpu().numpy()
    assert gp.size == pool.size and gs.size == side.size
    bad = np.nonzero(gp != pool)[0]
    assert bad.size == 0, f"page pool differs at {bad.size} bytes, first {bad[:8]}"
    bad = np.nonzero(gs != side)[0]
    assert bad.size == 0, f"side cache differs at {bad.size} bytes, first {bad[:8]}"
    assert kv4.kv4_get_device_error() == 0


@pytest.mark.parametrize("case", VBF_CASES, ids=[c[0] for c in VBF_CASES])
def test_bf16_values_decode_matches_oracle(case):
    from int4_kv_cache_append_b200 import kv4
    wl = make(case)
    gc = T.gpu_cache_from_host_inputs(wl, value_format=1)
    cfg, pool, side = T.oracle_cache(wl, value_format=1)
    q = wl.q_input(0)
    ref, ref_lse = T.oracle_decode(wl, cfg, pool, side, q)
    out, lse = T.gpu_decode(gc, wl, q)
    T.assert_close(out, ref, lse, ref_lse, what="bf16 values " + case[0])
    single, _ = T.oracle_decode(wl, cfg, pool, side, q, mode=O.SINGLE)
    T.assert_close(out, single, what="bf16 values " + case[0] + " vs single softmax")
    # split points do not change the result beyond the tolerance
    out2, lse2 = T.gpu_decode(gc, wl, q, max_len_hint=1)
    T.assert_close(out2, ref, lse2, ref_lse, what="bf16 values, one CTA")
    assert kv4.kv4_get_device_error() == 0


def test_bf16_values_reject_value_rotation():
    from int4_kv_cache_append_b200 import kv4
    wl = make(CASES[1])
    gc = kv4.Cache(T.geometry(wl, value_format=1))
    with pytest.raises(kv4.KV4Error):
        kv4.kv4_set_value_rotation(gc.handle, True)
