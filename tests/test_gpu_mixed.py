"""Mixed bit-width key cache on the GPU against the CPU oracle (RoPE-Aware Bit Allocation for
KV-Cache Quantization, abstract: per-block energy score, greedy integer widths, packed cache).

The block allocation is an integer decision taken in fp64 in key order on both sides, so it must
match bit for bit, and so must every page byte the append writes; the decode is compared with the
oracle's fp64 attention within the library's output tolerance.  Expected values come from the
oracle only (its own allocation from the same seeded keys)."""
import dataclasses

import numpy as np
import pytest
import torch

from int4_kv_cache_append_b200 import workload as W
from oracle import oracle as O

import kv4_testlib as T

pytestmark = pytest.mark.gpu


def mixed_workload(name, seed, B, G, Hkv, D, P, lens, dt=W.BF16, qdt=None, scale=4.0, n_outlier=2):
    wl = W.make_workload(name, seed, 1, B, G * Hkv, Hkv, D, P, 0, 0, 1, lambda r: list(lens), dt, dt, qdt or dt,
                         n_outlier, scale)
    return dataclasses.replace(wl, rope_outliers=True)


# (workload, key_bits, value_bits)
CASES = [
    (mixed_workload("m-k3v3", 101, 4, 4, 8, 128, 16, [300, 17, 1, 64]), 3, 3),
    (mixed_workload("m-k2v2", 102, 3, 4, 2, 128, 16, [513, 40, 16]), 2, 2),
    (mixed_workload("m-k4v4-d64", 103, 3, 2, 4, 64, 32, [95, 200, 33]), 4, 4),
    (mixed_workload("m-k1v8-g1", 104, 2, 1, 4, 128, 16, [77, 128]), 1, 8),
    (mixed_workload("m-k8v3", 105, 2, 2, 2, 64, 16, [150, 9], dt=W.F32), 8, 3),
    (mixed_workload("m-k5v4-empty", 106, 3, 4, 2, 128, 48, [0, 250, 31]), 5, 4),
    (mixed_workload("m-k3v2-flat", 107, 3, 4, 2, 128, 16, [160, 99, 260], scale=1.0), 3, 2),
    # smallest rows (8-byte keys, 16-byte values) and an odd width on every block
    (mixed_workload("m-k1v2-d64", 108, 2, 4, 2, 64, 16, [33, 500]), 1, 2),
    (mixed_workload("m-k7v8-p32", 109, 2, 2, 4, 128, 32, [70, 301], dt=W.F32), 7, 8),
    # key rows of 16 and 32 words at D = 128: padded in shared memory, brought in by the tensor copy
    (mixed_workload("m-k4v4-d128", 110, 3, 4, 4, 128, 16, [260, 33, 129]), 4, 4),
    (mixed_workload("m-k8v8-p48", 111, 2, 2, 2, 128, 48, [200, 97], dt=W.F32), 8, 8),
]
IDS = [c[0].name for c in CASES]


def geometry(wl, kb, vb):
    from int4_kv_cache_append_b200 import kv4
    return kv4.Geometry(1, wl.Hq, wl.Hkv, wl.D, wl.P, 0, 0, 1, wl.B, max(wl.num_pages, 1), kv4.KV4_KEYS_MIXED, kb, vb)


def prefill(wl):
    lens = np.asarray(wl.lens, np.int32)
    b, p = T.prefill_tokens(lens)
    K, V = wl.kv_inputs(0, b, p)
    return b, p, K, V


def kd_code(wl):
    return O.BF16 if wl.k_dtype == W.BF16 else O.F32


def oracle_allocation(wl, kb, K):
    E = O.gtq_energy(K, kd_code(wl))
    widths = np.stack([O.gtq_allocate(E[g], kb) for g in range(wl.Hkv)])
    sigma = np.stack([O.gtq_scales(E[g], K.shape[0]) for g in range(wl.Hkv)])
    return widths, sigma


def oracle_pool(wl, kb, vb, widths, sigma, step_by_step=False):
    cfg = O.GtqConfig(wl.Hq, wl.Hkv, wl.D, wl.P, kb, vb)
    pool = np.full(O.gtq_sizes(cfg)["page_bytes"] * max(wl.num_pages, 1), 0xA5, np.uint8)
    vd = O.BF16 if wl.v_dtype == W.BF16 else O.F32
    lens = np.asarray(wl.lens, np.int32)
    if not step_by_step:
        b, p, K, V = prefill(wl)
        O.gtq_append(cfg, widths, sigma, pool, K, V, b, p, wl.page_table, kd_code(wl), vd)
    else:
        for t in range(int(lens.max()) if lens.size else 0):
            rows = np.nonzero(lens > t)[0].astype(np.int32)
            p = np.full(rows.size, t, np.int32)
            K, V = wl.kv_inputs(0, rows, p)
            O.gtq_append(cfg, widths, sigma, pool, K, V, rows, p, wl.page_table, kd_code(wl), vd)
    return cfg, pool


def gpu_cache(wl, kb, vb, step_by_step=False, allocation=None):
    """GPU cache: allocation from the prefill keys on the device (or set from host arrays), then
    the same appends as the oracle."""
    from int4_kv_cache_append_b200 import kv4
    cache = kv4.Cache(geometry(wl, kb, vb), fill=0xA5)
    b, p, K, V = prefill(wl)
    if allocation is None:
        cache.allocate_key_bits(0, T.to_dev(K))
    else:
        kv4.kv4_set_key_allocation(cache.handle, 0, allocation[0], allocation[1])
    pt = torch.from_numpy(wl.page_table).cuda()
    lens = np.asarray(wl.lens, np.int32)
    lt = torch.from_numpy(lens).cuda()
    if not step_by_step:
        cache.append(0, T.to_dev(K), T.to_dev(V), torch.from_numpy(b).cuda(), torch.from_numpy(p).cuda(), lt, pt)
    else:
        for t in range(int(lens.max()) if lens.size else 0):
            rows = np.nonzero(lens > t)[0].astype(np.int32)
            pp = np.full(rows.size, t, np.int32)
            Kt, Vt = wl.kv_inputs(0, rows, pp)
            cache.append(0, T.to_dev(Kt), T.to_dev(Vt), torch.from_numpy(rows).cuda(), torch.from_numpy(pp).cuda(), lt, pt)
    torch.cuda.synchronize()
    return cache


@pytest.mark.parametrize("wl,kb,vb", CASES, ids=IDS)
def test_allocation_matches_oracle(wl, kb, vb):
    _, _, K, _ = prefill(wl)
    cache = gpu_cache(wl, kb, vb)
    w_gpu, s_gpu = cache.key_allocation(0)
    w_orc, s_orc = oracle_allocation(wl, kb, K)
    assert np.array_equal(w_gpu, w_orc), (w_gpu, w_orc)
    assert np.array_equal(s_gpu.view(np.uint32), s_orc.view(np.uint32))
    assert (w_gpu.astype(int).sum(axis=1) == kb * wl.D // 2).all()


@pytest.mark.parametrize("step_by_step", [False, True], ids=["prefill", "stepwise"])
@pytest.mark.parametrize("wl,kb,vb", CASES, ids=IDS)
def test_append_bit_exact(wl, kb, vb, step_by_step):
    _, _, K, _ = prefill(wl)
    widths, sigma = oracle_allocation(wl, kb, K)
    cache = gpu_cache(wl, kb, vb, step_by_step=step_by_step)
    _, pool = oracle_pool(wl, kb, vb, widths, sigma, step_by_step=step_by_step)
    pages, _ = cache.layer_views(0)
    got = pages.cpu().numpy()[:pool.size]
    diff = np.nonzero(got != pool)[0]
    assert diff.size == 0, f"{diff.size} page bytes differ, first at {diff[:8]}"
    from int4_kv_cache_append_b200 import kv4
    assert kv4.kv4_get_device_error() == 0


@pytest.mark.parametrize("wl,kb,vb", CASES, ids=IDS)
def test_decode_matches_oracle(wl, kb, vb):
    _, _, K, _ = prefill(wl)
    widths, sigma = oracle_allocation(wl, kb, K)
    cfg, pool = oracle_pool(wl, kb, vb, widths, sigma)
    cache = gpu_cache(wl, kb, vb)
    q = wl.q_input(0)
    out, lse = T.gpu_decode(cache, wl, q)
    qd = O.BF16 if q.dtype == np.uint16 else O.F32
    ro, rl = O.gtq_decode(cfg, widths, sigma, pool, q, wl.page_table, np.asarray(wl.lens, np.int32), q_dtype=qd)
    T.assert_close(out, ro, lse, rl, what=wl.name)


@pytest.mark.parametrize("qdt", ["f32", "f16"])
def test_decode_query_dtypes(qdt):
    wl, kb, vb = CASES[0]
    _, _, K, _ = prefill(wl)
    widths, sigma = oracle_allocation(wl, kb, K)
    cfg, pool = oracle_pool(wl, kb, vb, widths, sigma)
    cache = gpu_cache(wl, kb, vb)
    q32 = wl.q_input(0).view(np.uint16).astype(np.uint32) << 16
    q32 = q32.view(np.float32) if wl.q_dtype == W.BF16 else wl.q_input(0)
    if qdt == "f16":
        qh = q32.astype(np.float16)
        q_dev = torch.from_numpy(qh).cuda()
        qo, qd = qh.view(np.uint16), O.F16
    else:
        q_dev = torch.from_numpy(q32).cuda()
        qo, qd = q32, O.F32
    lens = np.asarray(wl.lens, np.int32)
    lse = torch.empty((wl.B, wl.Hq), dtype=torch.float32, device="cuda")
    out = cache.decode(0, q_dev, torch.from_numpy(wl.page_table).cuda(), torch.from_numpy(lens).cuda(), lse=lse)
    torch.cuda.synchronize()
    ro, rl = O.gtq_decode(cfg, widths, sigma, pool, qo, wl.page_table, lens, q_dtype=qd)
    T.assert_close(out.cpu().numpy(), ro, lse.cpu().numpy(), rl, what=f"q {qdt}")


@pytest.mark.parametrize("wl,kb,vb", CASES[:4], ids=IDS[:4])
def test_decode_on_oracle_built_pool(wl, kb, vb):
    """The decode alone: the oracle's pool bytes and allocation copied into the GPU cache."""
    from int4_kv_cache_append_b200 import kv4
    _, _, K, _ = prefill(wl)
    widths, sigma = oracle_allocation(wl, kb, K)
    cfg, pool = oracle_pool(wl, kb, vb, widths, sigma)
    cache = kv4.Cache(geometry(wl, kb, vb), fill=0)
    kv4.kv4_set_key_allocation(cache.handle, 0, widths, sigma)
    pages, _ = cache.layer_views(0)
    pages[:pool.size].copy_(torch.from_numpy(pool).cuda())
    torch.cuda.synchronize()
    q = wl.q_input(0)
    out, lse = T.gpu_decode(cache, wl, q)
    ro, rl = O.gtq_decode(cfg, widths, sigma, pool, q, wl.page_table, np.asarray(wl.lens, np.int32),
                          q_dtype=O.BF16 if q.dtype == np.uint16 else O.F32)
    T.assert_close(out, ro, lse, rl, what=wl.name)


def test_set_allocation_round_trip_and_append():
    """A caller's allocation (here a uniform one) is used as given: get returns it, and the
    append and decode follow it."""
    from int4_kv_cache_append_b200 import kv4
    wl, kb, vb = CASES[1]
    _, _, K, _ = prefill(wl)
    widths = np.full((wl.Hkv, wl.D // 2), kb, np.uint8)
    _, sigma = oracle_allocation(wl, kb, K)
    cache = gpu_cache(wl, kb, vb, allocation=(widths, sigma))
    w2, s2 = cache.key_allocation(0)
    assert np.array_equal(w2, widths) and np.array_equal(s2, sigma)
    cfg, pool = oracle_pool(wl, kb, vb, widths, sigma)
    pages, _ = cache.layer_views(0)
    assert np.array_equal(pages.cpu().numpy()[:pool.size], pool)
    q = wl.q_input(0)
    out, lse = T.gpu_decode(cache, wl, q)
    ro, rl = O.gtq_decode(cfg, widths, sigma, pool, q, wl.page_table, np.asarray(wl.lens, np.int32), q_dtype=O.BF16)
    T.assert_close(out, ro, lse, rl, what="uniform allocation")


def test_decode_split_count_invariance():
    """The split-K grid changes with max_len_hint; the result must not (within rounding)."""
    wl, kb, vb = CASES[0]
    cache = gpu_cache(wl, kb, vb)
    q = wl.q_input(0)
    o1, l1 = T.gpu_decode(cache, wl, q, max_len_hint=0)
    o2, l2 = T.gpu_decode(cache, wl, q, max_len_hint=int(np.max(wl.lens)))
    assert np.abs(o1 - o2).max() <= 1e-5 and np.abs(l1 - l2).max() <= 1e-5


@pytest.mark.parametrize("name", ["m-k4v4-d128", "m-k8v8-p48", "m-k8v3"])
def test_row_copies_match_tensor_copy(name):
    """Padded key rows arrive by one tensor copy, or by one bulk copy per row when the tensor map
    cannot be had (forced here through the test hook); the decode must be bit-identical."""
    from int4_kv_cache_append_b200 import kv4
    wl, kb, vb = next(c for c in CASES if c[0].name == name)
    cache = gpu_cache(wl, kb, vb)
    q = wl.q_input(0)
    o1, l1 = T.gpu_decode(cache, wl, q)
    kv4.kv4_debug_mixed_row_copies(cache.handle, True)
    try:
        o2, l2 = T.gpu_decode(cache, wl, q)
    finally:
        kv4.kv4_debug_mixed_row_copies(cache.handle, False)
    assert kv4.kv4_get_device_error() == 0
    assert np.array_equal(o1.view(np.uint32), o2.view(np.uint32)) and np.array_equal(l1.view(np.uint32),
                                                                                     l2.view(np.uint32))


def test_wait_limit_failure_path_reports_and_recovers():
    """The device-side failure path of the decode's bounded waits, made to run with the test hook
    (no invalid copy involved): every warp's first wait is on a barrier that nothing arrives on,
    runs out after its 1 ms limit, sets KV4_DEVERR_WAIT_LIMIT, waits for its copies in flight and
    returns.  The context stays usable: with the hook off the next decode matches the oracle."""
    from int4_kv_cache_append_b200 import kv4
    wl, kb, vb = CASES[0]
    cache = gpu_cache(wl, kb, vb)
    assert kv4.kv4_get_device_error() == 0
    q = wl.q_input(0)
    kv4.kv4_debug_force_wait_timeout(cache.handle, True)
    try:
        T.gpu_decode(cache, wl, q)
    finally:
        kv4.kv4_debug_force_wait_timeout(cache.handle, False)
    err = kv4.kv4_get_device_error()
    assert err & kv4.KV4_DEVERR_WAIT_LIMIT, hex(err)
    _, _, K, _ = prefill(wl)
    widths, sigma = oracle_allocation(wl, kb, K)
    cfg, pool = oracle_pool(wl, kb, vb, widths, sigma)
    out, lse = T.gpu_decode(cache, wl, q)
    qd = O.BF16 if q.dtype == np.uint16 else O.F32
    ro, rl = O.gtq_decode(cfg, widths, sigma, pool, q, wl.page_table, np.asarray(wl.lens, np.int32), q_dtype=qd)
    T.assert_close(out, ro, lse, rl, what="decode after the wait-limit path")
    assert kv4.kv4_get_device_error() == 0


def test_range_overflow_sets_error_bit():
    """A key beyond the fp16 range is stored with zero codes and reported, as in the oracle."""
    from int4_kv_cache_append_b200 import kv4
    wl, kb, vb = CASES[4]  # fp32 inputs
    b, p, K, V = prefill(wl)
    widths, sigma = oracle_allocation(wl, kb, K)
    K = K.copy()
    K[5, 1, 3] = 1e6
    cache = kv4.Cache(geometry(wl, kb, vb), fill=0xA5)
    kv4.kv4_set_key_allocation(cache.handle, 0, widths, sigma)
    pt = torch.from_numpy(wl.page_table).cuda()
    lens = np.asarray(wl.lens, np.int32)
    cache.append(0, T.to_dev(K), T.to_dev(V), torch.from_numpy(b).cuda(), torch.from_numpy(p).cuda(),
                 torch.from_numpy(lens).cuda(), pt)
    torch.cuda.synchronize()
    assert kv4.kv4_get_device_error() & kv4.KV4_DEVERR_RANGE
    cfg = O.GtqConfig(wl.Hq, wl.Hkv, wl.D, wl.P, kb, vb)
    pool = np.full(O.gtq_sizes(cfg)["page_bytes"] * wl.num_pages, 0xA5, np.uint8)
    assert O.gtq_append(cfg, widths, sigma, pool, K, V, b, p, wl.page_table, O.F32, O.F32)
    pages, _ = cache.layer_views(0)
    assert np.array_equal(pages.cpu().numpy()[:pool.size], pool)


def _oracle_one_mixed(wl, kb, vb, widths, sigma, b, g):
    """Oracle cache (identity page table) and decode of sequence b of a full-size workload, only
    KV head g populated, with the given allocation."""
    L = int(wl.lens[b])
    npages = (L + wl.P - 1) // wl.P
    cfg = O.GtqConfig(wl.Hq, wl.Hkv, wl.D, wl.P, kb, vb)
    pool = np.full(O.gtq_sizes(cfg)["page_bytes"] * npages, 0xA5, np.uint8)
    f = wl.factor()
    pos = np.arange(L, dtype=np.int64)
    idx = ((b * W.POS_STRIDE + pos[:, None]) * wl.Hkv + g) * wl.D + np.arange(wl.D)[None, :]
    K = np.zeros((L, wl.Hkv, wl.D), np.float32)
    V = np.zeros((L, wl.Hkv, wl.D), np.float32)
    K[:, g] = W.normal_f32(W.stream_key(wl.seed, W.KIND_K, 0), idx).reshape(L, wl.D) * f[g][None]
    V[:, g] = W.normal_f32(W.stream_key(wl.seed, W.KIND_V, 0), idx).reshape(L, wl.D) * f[g][None]
    kd = vd = O.F32
    if wl.k_dtype == W.BF16:
        K, kd = W.bf16_bits(K), O.BF16
    if wl.v_dtype == W.BF16:
        V, vd = W.bf16_bits(V), O.BF16
    pt = np.arange(npages, dtype=np.int32)[None, :]
    O.gtq_append(cfg, widths, sigma, pool, K, V, np.zeros(L, np.int32), pos.astype(np.int32), pt, kd, vd)
    q = wl.q_input(0, 0, rows=[b])
    out, lse = O.gtq_decode(cfg, widths, sigma, pool, q, pt, np.array([L], np.int32),
                            q_dtype=O.BF16 if q.dtype == np.uint16 else O.F32)
    return cfg, pool, out[0], lse[0]


@pytest.mark.parametrize("name,kb,vb", [("async-refill", 3, 3), ("async-refill", 4, 4), ("long-context", 3, 3)])
def test_fullsize_mixed_sampled_parity(name, kb, vb):
    """The bench's mixed workloads at full size, in its launch configuration: the allocation from
    4096 host-drawn keys equals the oracle's; sampled (sequence, KV head) pairs are recomputed by
    the oracle one by one (page bytes bit-exact, outputs within the tolerance)."""
    from int4_kv_cache_append_b200 import harness as H, kv4
    wl = dataclasses.replace(W.WORKLOADS[name](), s=0, w=0, h=1, value_format=2, key_bits=kb, value_bits=vb,
                             rope_outliers=True)
    cache = kv4.Cache(H.geometry(wl, value_format=kv4.KV4_KEYS_MIXED), fill=0xA5)
    b_all, p_all = H.token_list(wl.lens)
    n = min(4096, b_all.size)
    Ka, _ = wl.kv_inputs(0, b_all[:n], p_all[:n])
    cache.allocate_key_bits(0, T.to_dev(Ka))
    kdc = O.BF16 if wl.k_dtype == W.BF16 else O.F32
    E = O.gtq_energy(Ka, kdc)
    widths = np.stack([O.gtq_allocate(E[g], kb) for g in range(wl.Hkv)])
    sigma = np.stack([O.gtq_scales(E[g], n) for g in range(wl.Hkv)])
    w_gpu, s_gpu = cache.key_allocation(0)
    assert np.array_equal(w_gpu, widths) and np.array_equal(s_gpu.view(np.uint32), sigma.view(np.uint32))
    H.prefill(cache, wl, 0, wl.lens)
    q = T.to_dev(wl.q_input(0))
    lse = torch.empty((wl.B, wl.Hq), device="cuda")
    out = cache.decode(0, q, torch.from_numpy(wl.page_table).cuda(), torch.from_numpy(wl.lens).cuda(), lse=lse,
                       max_len_hint=int(wl.lens.max()))
    torch.cuda.synchronize()
    assert kv4.kv4_get_device_error() == 0
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    assert np.isfinite(out).all()
    order = np.argsort(wl.lens, kind="stable")
    picks = [(int(order[0]), 0), (int(order[len(order) // 2]), wl.Hkv // 2), (int(order[-1]), wl.Hkv - 1)]
    if name == "long-context":
        picks = [(0, 3), (3, 6)]
    pages, _ = cache.layer_views(0)
    tile = wl.P * ((kb + vb) * wl.D // 8 + 8)
    for b, g in picks:
        ocfg, opool, oout, olse = _oracle_one_mixed(wl, kb, vb, widths, sigma, b, g)
        pb = O.gtq_sizes(ocfg)["page_bytes"]
        L = int(wl.lens[b])
        for lp in range((L + wl.P - 1) // wl.P):
            page = int(wl.page_table[b, lp])
            got = pages[page * pb + g * tile: page * pb + (g + 1) * tile].cpu().numpy()
            want = opool[lp * pb + g * tile: lp * pb + (g + 1) * tile]
            assert np.array_equal(got, want), f"{name}: seq {b} head {g} page {lp} differs"
        G = wl.Hq // wl.Hkv
        # The logits here reach several hundred (x20 RoPE-block outliers in both q and k), and the
        # decode forms them from query weights kept to ~22 bits (fp16 hi/lo halves), so the lse
        # bound grows with its magnitude: 1e-4 + 2^-20 |lse|.
        lse_tol = 1e-4 + 2.0 ** -20 * float(np.abs(olse[g * G:(g + 1) * G]).max())
        T.assert_close(out[b, g * G:(g + 1) * G], oout[g * G:(g + 1) * G], lse[b, g * G:(g + 1) * G],
                       olse[g * G:(g + 1) * G], lse_atol=lse_tol, what=f"{name} seq {b} head {g}")
