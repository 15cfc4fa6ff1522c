"""The seeded input generator (CPU side): published SplitMix64, exact normals, bf16 rounding."""
import numpy as np
import torch

from int4_kv_cache_append_b200 import workload as W

MASK = (1 << 64) - 1


def _splitmix_python(state: int, n: int):
    """SplitMix64 as in Vigna's reference implementation: the state advances by the golden
    gamma, and each output is the mixed state."""
    out = []
    for _ in range(n):
        state = (state + 0x9E3779B97F4A7C15) & MASK
        z = state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK
        out.append(z ^ (z >> 31))
    return out


def test_splitmix64_matches_sequential_definition():
    for key in (0, 1, 1234567, MASK):
        ref = _splitmix_python(key, 40)
        got = [int(v) for v in W.splitmix64(key, np.arange(40))]
        assert got == ref


def test_splitmix64_zero_seed_known_output():
    # first output of SplitMix64 from state 0 (widely tabulated): 0xE220A8397B1DCDAF
    assert int(W.splitmix64(0, np.array([0]))[0]) == 0xE220A8397B1DCDAF


def test_normals_exact_and_standardised():
    z = W.normal_f32(W.stream_key(9, W.KIND_K, 0), np.arange(400_000))
    assert z.dtype == np.float32
    assert np.all(z * 65536 == np.rint(z * 65536))           # exact multiples of 2^-16
    assert np.abs(z).max() <= 6.0
    assert abs(float(z.mean())) < 0.01 and abs(float(z.var()) - 1.0) < 0.01
    # counter-based: any element regenerates alone
    idx = np.array([5, 123456, 399_999])
    assert np.array_equal(W.normal_f32(W.stream_key(9, W.KIND_K, 0), idx), z[idx])


def test_bf16_rounding_matches_torch():
    x = W.normal_f32(W.stream_key(3, W.KIND_V, 1), np.arange(50_000)) * np.float32(37.0)
    x = np.concatenate([x, np.array([1.00390625, 1.01171875, -2.0**-130, 3.0e38], np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(W.bf16_bits(x), ref)
    assert np.array_equal(W.bf16_to_f32(ref), torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).float().numpy())


def test_workload_shapes_and_bytes():
    tiny = W.tiny_cfg()
    assert tiny.lens.tolist() == [256, 200]
    # INT4 region: 220 + 164 tokens x 72 B; INT8 region: 36 + 36 tokens x 132 B (1 KV head)
    assert tiny.kv_bytes_int4() == (220 + 164) * 72 + (36 + 36) * 132 == 37_152
    lc = W.long_context()
    assert lc.kv_bytes_int4() == 393_199_104 and lc.kv_bytes_bf16() == 1_476_395_008
    q = W.qwen3_4b_decode()
    assert q.lens.min() >= 1 and q.lens.max() <= 8192 and q.B == 64
    # every page of the pool is owned by exactly one (sequence, logical page)
    used = np.concatenate([q.page_table[b, :(q.max_lens[b] + 15) // 16] for b in range(q.B)])
    assert np.array_equal(np.sort(used), np.arange(q.num_pages))


def test_outliers_distinct_per_head():
    w = W.qwen3_4b_decode()
    for g in range(w.Hkv):
        assert len(set(w.outliers[g].tolist())) == w.n_outlier
    f = w.factor()
    assert (f == 15.0).sum() == w.Hkv * w.n_outlier
