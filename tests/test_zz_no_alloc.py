"""kv4_decode_attn_static: the decode for callers that cannot allocate device memory.

Some callers of this library cannot hand it a workspace: code that runs inside another runtime's
memory pool that forbids foreign allocations, a serving process that reserved all device memory
up front for its page pools, or a caller with no allocator of its own.  For them the split-K
partials live in a fixed 16 MiB device array inside the library.  This test calls that entry
point through the C ABI twice in a row and checks both results against kv4_decode_attn (with a
caller workspace) within the decode tolerance, and checks that a batch too large for the array is
refused before anything is launched.  It sits in its own file, collected last.
"""
import numpy as np
import pytest
import torch

from int4_kv_cache_append_b200 import workload as W

import kv4_testlib as T

pytestmark = pytest.mark.gpu


def test_static_scratch_decode_matches_workspace_decode():
    from int4_kv_cache_append_b200 import kv4
    wl = W.make_workload("no-alloc", 31, 1, 12, 32, 8, 128, 16, 4, 128, 128,
                         lambda r: [3000, 1, 130, 133, 2048, 517, 64, 900, 4096, 7, 1500, 260],
                         W.BF16, W.BF16, W.BF16, 4, 15.0)
    gc = T.gpu_cache_from_host_inputs(wl)
    assert kv4.kv4_decode_workspace_bytes(gc.handle, wl.B) <= kv4.KV4_STATIC_SCRATCH_BYTES
    q = T.to_dev(wl.q_input(0))
    pt = torch.from_numpy(wl.page_table).cuda()
    lens = torch.from_numpy(wl.lens).cuda()
    ref_lse = torch.empty((wl.B, wl.Hq), device="cuda")
    ref = gc.decode(0, q, pt, lens, lse=ref_lse)
    for _ in range(2):  # two calls in a row share (and overwrite) the static array
        out = torch.full((wl.B, wl.Hq, wl.D), float("nan"), device="cuda")
        lse = torch.full((wl.B, wl.Hq), float("nan"), device="cuda")
        kv4.kv4_decode_attn_static(gc.handle, 0, wl.B, q, kv4.KV4_BF16, pt, wl.stride, lens, 0, out, lse)
        torch.cuda.synchronize()
        T.assert_close(out.cpu().numpy(), ref.cpu().numpy().astype(np.float64), lse.cpu().numpy(),
                       ref_lse.cpu().numpy().astype(np.float64), what="static scratch vs workspace")
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
