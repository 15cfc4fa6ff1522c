"""kv4_decode_attn_static: the decode for callers that cannot allocate device memory.

Some callers of this library cannot hand it a workspace: code that runs inside another runtime's
memory pool that forbids foreign allocations, a serving process that reserved all device memory
up front for its page pools, or a caller with no allocator of its own.  For them the split-K
partials live in a fixed 16 MiB device array inside the library.  This test first runs that
entry point on a larger batch of another cache (so the shared array holds records and partials of
a different shape), then calls it through the C ABI twice in a row on the checked batch: both
results must equal kv4_decode_attn with a caller workspace bit for bit (same kernels, same grid,
same split points), so a record or partial left stale in the array would show.  It also checks
that a batch too large for the array is refused before anything is launched.  It sits in its own
file, collected last.
"""
import numpy as np
import pytest
import torch

from int4_kv_cache_append_b200 import workload as W

import kv4_testlib as T

pytestmark = pytest.mark.gpu


def _workspace_and_static(kv4, wl, gc):
    q = T.to_dev(wl.q_input(0))
    pt = torch.from_numpy(wl.page_table).cuda()
    lens = torch.from_numpy(wl.lens).cuda()
    ref_lse = torch.empty((wl.B, wl.Hq), device="cuda")
    ref = gc.decode(0, q, pt, lens, lse=ref_lse)
    out = torch.full((wl.B, wl.Hq, wl.D), float("nan"), device="cuda")
    lse = torch.full((wl.B, wl.Hq), float("nan"), device="cuda")
    kv4.kv4_decode_attn_static(gc.handle, 0, wl.B, q, kv4.KV4_BF16, pt, wl.stride, lens, 0, out, lse)
    torch.cuda.synchronize()
    return (ref.cpu().numpy(), ref_lse.cpu().numpy()), (out.cpu().numpy(), lse.cpu().numpy()), (q, pt, lens)


def test_static_scratch_decode_matches_workspace_decode():
    from int4_kv_cache_append_b200 import kv4
    # a larger batch with other lengths first: the shared array then holds its records and
    # partials (more (sequence, KV head) records, other split points) when the checked calls run
    big = W.make_workload("no-alloc-big", 41, 1, 40, 32, 8, 128, 16, 4, 128, 128,
                          lambda r: list(r.integers(1, 6000, size=40)), W.BF16, W.BF16, W.BF16, 4, 15.0)
    gb = T.gpu_cache_from_host_inputs(big)
    assert kv4.kv4_decode_workspace_bytes(gb.handle, big.B) <= kv4.KV4_STATIC_SCRATCH_BYTES
    (ref, ref_lse), (out, lse), _ = _workspace_and_static(kv4, big, gb)
    assert np.array_equal(out, ref) and np.array_equal(lse, ref_lse)
    wl = W.make_workload("no-alloc", 31, 1, 12, 32, 8, 128, 16, 4, 128, 128,
                         lambda r: [3000, 1, 130, 133, 2048, 517, 64, 900, 4096, 7, 1500, 260],
                         W.BF16, W.BF16, W.BF16, 4, 15.0)
    gc = T.gpu_cache_from_host_inputs(wl)
    assert kv4.kv4_decode_workspace_bytes(gc.handle, wl.B) <= kv4.KV4_STATIC_SCRATCH_BYTES
    (ref, ref_lse), (out, lse), (q, pt, lens) = _workspace_and_static(kv4, wl, gc)
    results = [(out, lse)]
    out2 = torch.full((wl.B, wl.Hq, wl.D), float("nan"), device="cuda")
    lse2 = torch.full((wl.B, wl.Hq), float("nan"), device="cuda")
    kv4.kv4_decode_attn_static(gc.handle, 0, wl.B, q, kv4.KV4_BF16, pt, wl.stride, lens, 0, out2, lse2)
    torch.cuda.synchronize()
    results.append((out2.cpu().numpy(), lse2.cpu().numpy()))
    for o, l in results:  # two calls in a row share (and overwrite) the static array
        assert np.array_equal(o, ref), f"static scratch vs workspace: max diff {np.nanmax(np.abs(o - ref)):.3e}"
        assert np.array_equal(l, ref_lse)
    assert kv4.kv4_get_device_error() == 0


def test_static_scratch_rejects_batches_beyond_its_size():
    from int4_kv_cache_append_b200 import kv4
    B = 512
    geo = kv4.Geometry(1, 32, 8, 128, 16, 4, 128, 128, B, 16)
    cache = kv4.Cache(geo)
    assert kv4.kv4_decode_workspace_bytes(cache.handle, B) > kv4.KV4_STATIC_SCRATCH_BYTES
    q = torch.zeros((B, 32, 128), dtype=torch.bfloat16, device="cuda")
    pt = torch.zeros((B, 1), dtype=torch.int32, device="cuda")
    lens = torch.zeros(B, dtype=torch.int32, device="cuda")
    out = torch.zeros((B, 32, 128), device="cuda")
    with pytest.raises(kv4.KV4Error) as e:
        kv4.kv4_decode_attn_static(cache.handle, 0, B, q, kv4.KV4_BF16, pt, 1, lens, 0, out, None)
    assert e.value.status == kv4.KV4_ERR_WORKSPACE
