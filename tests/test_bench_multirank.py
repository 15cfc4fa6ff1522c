"""Host logic of `bench.py --gpus N` on 2 CPU ranks over gloo.

Each rank runs its own batch (weak scaling); the only process-group traffic is a barrier and
the max-over-ranks reduction of the timed region.  The reference (oracle) arm runs on rank 0
alone.  No GPU is used.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import argparse

    import bench
    import torch.distributed as dist
    try:
        w, r, _ = bench.dist_setup("gloo")
        assert (w, r) == (world, rank)
        bench.barrier(w)
        ms = 10.0 + 5.0 * rank  # the slower rank decides the job time
        mx = bench.max_over_ranks(ms, w)
        rate = bench.whole_job_rate(64 * 100, w, mx)
        args = argparse.Namespace(workload="tiny", steps=1, warmup=0)
        line = bench.run_reference(args, w, r)
        q.put((rank, mx, rate, None if line is None else (line["impl"], line["n_gpus"], line["cpu_baseline"]["kind"])))
        dist.destroy_process_group()
    except Exception as e:  # surface the failure to the parent
        q.put((rank, "error", repr(e), None))


def test_two_rank_max_timing_and_reference_on_rank0_only():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, rate, ref in res:
        assert mx != "error", rate
        assert mx == pytest.approx(15.0)
        assert rate == pytest.approx(2 * 64 * 100 / 0.015)
    assert res[0][3] == ("reference", 2, "oracle")
    assert res[1][3] is None


def test_step_shape_of_the_workloads():
    """One-layer workloads cycle 4 resident layers at fixed lengths; the 36-layer loop runs all of
    its layers per step and may grow by the page capacity it was built with."""
    sys.path.insert(0, ROOT)
    import bench
    from int4_kv_cache_append_b200 import workload as W
    assert bench.step_shape(W.qwen3_4b_decode()) == (1, 4, 0)
    for h in (32, 64, 128):
        wl = W.qwen3_8b_loop(h=h)
        assert wl.h == h
        assert bench.step_shape(wl) == (36, 36, 64)


def test_sink_recent_overrides():
    """--sinks/--recent replace a workload's s and w (recent -1: every position, KV8) and name the
    workload after them; the lengths and pages are unchanged."""
    import argparse
    sys.path.insert(0, ROOT)
    import bench
    base = bench.make_wl(argparse.Namespace(workload="qwen3-4b-decode", h=None, sinks=None, recent=None))
    kv8 = bench.make_wl(argparse.Namespace(workload="qwen3-4b-decode", h=None, sinks=0, recent=-1))
    assert (kv8.s, kv8.w) == (0, int(base.max_lens.max()))
    assert kv8.name == f"{base.name}-s0-w{kv8.w}"
    assert (kv8.lens == base.lens).all() and (kv8.page_table == base.page_table).all()
    # every position read from the side cache: 2D + 4 bytes per token and KV head
    assert kv8.kv_bytes_int4() == base.Hkv * int(base.lens.astype(int).sum()) * (2 * base.D + 4)
    sw = bench.make_wl(argparse.Namespace(workload="qwen3-4b-decode", h=None, sinks=144, recent=0))
    assert (sw.s, sw.w) == (144, 0)


def test_hadamard_override_of_one_layer_workloads():
    """--h on a one-layer workload (the naive-INT4 h = 1 line beside h = 128) renames it and keeps
    everything else."""
    import argparse

    import bench
    from int4_kv_cache_append_b200 import workload as W
    base = W.qwen3_4b_decode()
    wl = bench.make_wl(argparse.Namespace(workload="qwen3-4b-decode", h=1, sinks=None, recent=None))
    assert wl.h == 1 and wl.name == base.name + "-h1"
    assert (wl.lens == base.lens).all() and (wl.page_table == base.page_table).all()
    loop = bench.make_wl(argparse.Namespace(workload="qwen3-8b-loop", h=64, sinks=None, recent=None))
    assert loop.h == 64 and loop.layers == 36
    names = [n for n, _, _ in bench.PER_CONFIG]
    vb = bench.make_wl(argparse.Namespace(workload="async-refill", h=None, sinks=None, recent=None, values="bf16"))
    assert vb.value_format == 1 and vb.name.endswith("-vbf16")
    base3 = W.async_refill()
    assert vb.kv_bytes_int4() > base3.kv_bytes_int4()
    assert {"tiny", "qwen3-4b-decode", "async-refill", "long-context"} <= set(names)
