#!/usr/bin/env python
"""Benchmark: decode steps of INT4-KV attention (append + decode) beside the BF16-KV kernel on
the same GPU and the CPU oracle on the host cores.  Default workload: the Qwen3-8B-like 36-layer
decode loop (32 q / 8 KV heads, head_dim 128, bf16, B = 128 sequences with lengths U{1024..16384}
growing by one token per step, P = 16, s = 16, w = 128, h = 128; about 44 GB of cache), the
largest configuration that fits one GPU.

A layer call = kv4_append of one new token per sequence (rotation, INT4 pack, INT8 routing)
followed by kv4_decode_attn over the whole cache (INT4 region + INT8 sink/recent regions,
split-K, regional merge).  The 36-layer workload: a step is all 36 layer calls, and every
sequence grows by one token per step.  One-layer workloads (`--workload qwen3-4b-decode |
async-refill | long-context | tiny ...`): a step is one layer call, steps cycle over 4 resident
layers (inputs larger than the 126 MB L2).  Each step is one CUDA graph (the decode a
programmatic dependent of the append); a second loop times the kernels one by one for the
roofline.  At N = 1 the line also carries `per_config`: the one-layer workloads measured in the
same process (decode time, roofline fraction, BF16-KV decode time, clocks; h = 1 beside h = 128).
Prints one JSON line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kv4|reference] [--workload NAME]
Under torchrun (N > 1) every rank runs its own batch on its own GPU (weak scaling, no
collective on the data path); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
METRIC = "INT4-KV decode attn: seq-steps/s and HBM GB/s (% of roofline) vs BF16-KV"
UNIT = "seq-steps/s"
LAYERS = 4
# sequences of the bench workload in the CPU oracle sample (the reference arm and the
# cpu_baseline leg time the same sample)
SAMPLE_SEQS = 8
INPUTS = ("synthetic, seeded: K, V, q are Irwin-Hall N(0,1) stand-ins (sum of 12 uniforms minus 6, "
          "tails cut at +-6) with fixed outlier channels per KV head")
# one-layer workloads measured beside the default line: (name, overrides, note); overrides: h
# (Hadamard block), values ("bf16": the K-INT4 / V-BF16 variant)
PER_CONFIG = (("tiny", {}, "37 KB of KV per decode: bound by launch and fixed cost, not by HBM"),
              ("qwen3-4b-decode", {}, None), ("qwen3-4b-decode", {"h": 1}, "h = 1: no rotation (naive INT4)"),
              ("async-refill", {}, None), ("async-refill", {"values": "bf16"}, "K-INT4 / V-BF16: bf16 values"),
              ("long-context", {}, None), ("long-context", {"h": 1}, "h = 1: no rotation (naive INT4)"),
              ("async-refill", {"mixed": (3, 3)}, "mixed bit-width keys K3V3 (RoPE-block bit allocation)"),
              ("async-refill", {"mixed": (4, 4)}, "mixed bit-width keys K4V4: the bytes of the INT4 cache"),
              ("long-context", {"mixed": (3, 3)}, "mixed bit-width keys K3V3 (RoPE-block bit allocation)"))


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default 2000; 64 for the growing 36-layer workload)")
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["kv4", "reference"], default="kv4")
    ap.add_argument("--workload", default="qwen3-8b-loop")
    ap.add_argument("--h", type=int, default=None, help="Hadamard block of the 36-layer workload (32, 64, 128)")
    ap.add_argument("--layers", type=int, default=None,
                    help="layers of the 36-layer workload (fewer for a small profiler capture: every layer's "
                         "launch is the same, only the resident KV shrinks)")
    ap.add_argument("--sinks", type=int, default=None, help="override s, the INT8 sink positions")
    ap.add_argument("--recent", type=int, default=None,
                    help="override w, the INT8 recent window (-1: every position, i.e. all-INT8 KV8)")
    ap.add_argument("--values", choices=["int4", "bf16"], default="int4",
                    help="value storage: INT4 (KV4) or bf16 (the K-INT4 / V-BF16 variant)")
    ap.add_argument("--mixed", default=None, metavar="KB,VB",
                    help="mixed bit-width key cache with KB average key bits and VB value bits per dimension "
                         "(RoPE-block bit allocation; no side cache, no rotation)")
    ap.add_argument("--no-bf16", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--no-overlap", action="store_true",
                    help="decode waits for the append before building its schedule (kv4_set_decode_overlap 0)")
    ap.add_argument("--e2e-steps", type=int, default=None, help="default 200 (20 for the 36-layer workload)")
    ap.add_argument("--no-per-config", action="store_true", help="skip the one-layer workloads beside the line")
    ap.add_argument("--per-config-steps", type=int, default=300)
    ap.add_argument("--soak-s", type=float, default=1.5, help="untimed identical steps sampled for clocks")
    args = ap.parse_args()
    if args.steps is None:
        args.steps = 64 if args.workload == "qwen3-8b-loop" else 2000
    if args.e2e_steps is None:
        args.e2e_steps = 20 if args.workload == "qwen3-8b-loop" else 200
    return args


def make_wl(args):
    sys.path.insert(0, ROOT)
    import dataclasses
    from int4_kv_cache_append_b200 import workload as W
    fn = W.WORKLOADS[args.workload]
    h = getattr(args, "h", None)
    nl = getattr(args, "layers", None)
    if args.workload == "qwen3-8b-loop" and (h is not None or nl is not None):
        kw = {"h": h} if h is not None else {}
        if nl is not None:
            kw["layers"] = nl
        wl = fn(**kw)
        if nl is not None:
            wl = dataclasses.replace(wl, name=f"{wl.name}-{nl}layers")
    else:
        if nl is not None:
            raise SystemExit("--layers applies to the 36-layer workload only")
        wl = fn()
        if h is not None and h != wl.h:
            wl = dataclasses.replace(wl, h=h, name=f"{wl.name}-h{h}")
    if getattr(args, "values", "int4") == "bf16":
        wl = dataclasses.replace(wl, value_format=1, name=f"{wl.name}-vbf16")
    if getattr(args, "mixed", None):
        kb, vb = (int(x) for x in args.mixed.split(","))
        wl = mixed_variant(wl, kb, vb)
    # sink / recent budgets (KV4-RL "Main Findings": s/w sweep; KV8 = every position in INT8)
    s, w = getattr(args, "sinks", None), getattr(args, "recent", None)
    if s is not None or w is not None:
        s = wl.s if s is None else s
        w = wl.w if w is None else (int(wl.max_lens.max()) if w < 0 else w)
        wl = dataclasses.replace(wl, s=s, w=w, name=f"{wl.name}-s{s}-w{w}")
    return wl


def mixed_variant(wl, kb: int, vb: int):
    """The workload on the mixed bit-width key cache: keys at kb bits per dimension on average,
    split over RoPE blocks; values at vb bits; outliers on whole RoPE blocks (queries alike); no
    side cache and no rotation."""
    import dataclasses
    return dataclasses.replace(wl, s=0, w=0, h=1, value_format=2, key_bits=kb, value_bits=vb, rope_outliers=True,
                               name=f"{wl.name}-k{kb}v{vb}")


# ----------------------------------------------------------------------------- helpers

def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def decode_sources_digest() -> str:
    h = hashlib.sha256()
    for f in ("kv4_decode.cu", "kv4_device.cuh", "kv4_layout.cuh"):
        h.update(open(os.path.join(ROOT, "int4_kv_cache_append_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes per decode launch from the committed ncu summary, if it was taken on these sources.

    profiles/decode_int4_traffic.txt holds lines `workload sources-digest bytes-per-launch`."""
    p = os.path.join(ROOT, "profiles", "decode_int4_traffic.txt")
    if not os.path.exists(p):
        return None
    for line in open(p):
        f = line.split()
        if len(f) == 3 and not line.startswith("#") and f[0] == workload and f[1] == decode_sources_digest():
            return int(f[2])
    return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons at 100 ms while running (read-only queries)."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.proc = None
        self.path = os.path.join("/tmp", f"kv4_clocks_{os.getpid()}.csv")
        self.uuid = uuid

    def start(self):
        try:
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
            if self.uuid:
                cmd += ["-i", self.uuid]
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(cmd, stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if not self.proc:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(mx)), "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(backend: str = "nccl"):
    """One process per GPU under torchrun; the process group carries only the barrier and the
    max-over-ranks timing reduction (no collective on the data path).  `gloo` is for the
    CPU tests of this host logic."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=60))
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: int, world: int, max_ms: float) -> float:
    """Weak scaling: every rank processes the same units; the job rate is all ranks' units over the
    slowest rank's time."""
    return world * units_per_rank / (max_ms / 1e3)


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ----------------------------------------------------------------------------- CPU oracle leg

def oracle_sample_setup(wl, nseq: int):
    """Host cache of the first nseq sequences, filled up to L-1 (untimed), plus the step inputs.
    Returns step(nthreads) (one layer call: append of one token per sequence, then the decode),
    its two halves append() and decode(nthreads), and the sample's lengths."""
    sys.path.insert(0, ROOT)
    from oracle import oracle as O
    from int4_kv_cache_append_b200 import workload as W
    lens = wl.lens[:nseq].astype(np.int32)
    cfg = O.Config(wl.Hq, wl.Hkv, wl.D, wl.P, wl.s, wl.w, wl.h, nseq)
    pool = np.zeros(O.page_bytes(cfg) * wl.num_pages, np.uint8)
    side = np.zeros(O.side_slot_bytes(cfg) * nseq, np.uint8)
    kd = O.BF16 if wl.k_dtype == W.BF16 else O.F32
    vd = O.BF16 if wl.v_dtype == W.BF16 else O.F32
    for b in range(nseq):
        L = int(lens[b])
        if L > 1:
            bb = np.full(L - 1, b, np.int32)
            pp = np.arange(L - 1, dtype=np.int32)
            K, V = wl.kv_inputs(0, bb, pp)
            O.append(cfg, pool, side, K, V, bb, pp, lens, wl.page_table[:nseq], kd, vd)
    bs = np.arange(nseq, dtype=np.int32)
    ps = (lens - 1).astype(np.int32)
    K1, V1 = wl.kv_inputs(0, bs, ps)
    q = wl.q_input(0, 0, rows=np.arange(nseq))
    qd = O.BF16 if wl.q_dtype == W.BF16 else O.F32
    pt = np.ascontiguousarray(wl.page_table[:nseq])

    def append():
        O.append(cfg, pool, side, K1, V1, bs, ps, lens, pt, kd, vd)

    def decode(nthreads):
        O.decode(cfg, pool, side, q, pt, lens, q_dtype=qd, nthreads=nthreads)

    def step(nthreads):
        append()
        decode(nthreads)

    return step, append, decode, lens


def _time_reps(fn, min_seconds: float, max_reps: int = 5000):
    fn()  # warm
    reps, t0 = 0, time.perf_counter()
    while True:
        fn()
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_seconds or reps >= max_reps:
            return reps, el


def cpu_baseline(wl, nseq: int = SAMPLE_SEQS, min_seconds: float = 8.0, per_step: int = 1):
    """The oracle's append + decode of one layer per step on a sample of sequences, on all host
    cores (OpenMP over (sequence, KV head) in the decode) and on one thread; the append (one
    thread) and the decode are also timed alone.  A step of per_step layers costs per_step such
    layer-steps (the layers are identical in shape)."""
    step, append, decode, lens = oracle_sample_setup(wl, nseq)
    cores = os.cpu_count() or 1
    reps, el = _time_reps(lambda: step(cores), min_seconds)
    reps1, el1 = _time_reps(lambda: step(1), min_seconds)
    repa, ela = _time_reps(append, min(2.0, min_seconds))
    repd, eld = _time_reps(lambda: decode(cores), min(4.0, min_seconds))
    per = f"; rate divided by the step's {per_step} layers" if per_step > 1 else ""
    return {"value": nseq * reps / el / per_step, "unit": UNIT, "cores": cores, "kind": "oracle",
            "single_thread": {"value": nseq * reps1 / el1 / per_step, "unit": UNIT, "cores": 1},
            "append_ms_per_layer": round(1e3 * ela / repa, 3), "decode_ms_per_layer": round(1e3 * eld / repd, 3),
            "sample": f"first {nseq} of {wl.B} sequences (lengths {int(lens.min())}..{int(lens.max())}), "
                      f"one layer call (append 1 token per sequence + decode), fp64 C oracle, OpenMP over "
                      f"(sequence, KV head) in the decode; {reps} layer calls in {el:.1f} s on {cores} threads, "
                      f"{reps1} in {el1:.1f} s on one{per}"}


def run_reference(args, world, rank):
    if rank != 0:
        return None
    sys.path.insert(0, ROOT)
    wl = make_wl(args)
    per_step = step_shape(wl)[0]
    nseq = min(SAMPLE_SEQS, wl.B)
    step, _, _, lens = oracle_sample_setup(wl, nseq)
    cores = os.cpu_count() or 1
    for _ in range(args.warmup):
        step(cores)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step(cores)
    el = time.perf_counter() - t0
    value = nseq * args.steps / el / per_step
    sample = (f"each step: first {nseq} of {wl.B} sequences (lengths {int(lens.min())}..{int(lens.max())}), "
              f"one layer call (append 1 token per sequence + decode), fp64 C oracle, OpenMP over "
              f"(sequence, KV head) in the decode; the same sample as the kv4 line's cpu_baseline"
              + (f"; rate divided by the step's {per_step} layers" if per_step > 1 else ""))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / args.steps * per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "B_sampled": nseq, "parallelism": "host cores", "inputs": INPUTS},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    return line


# ----------------------------------------------------------------------------- GPU leg

def step_shape(wl):
    """(layers one step runs, resident layers, positions each sequence may still grow by).

    One-layer workloads cycle over LAYERS resident layers, one layer per step, and append at the
    same position every step.  A workload with more layers than that (the 36-layer append + decode
    loop) runs every layer in one step, and its lengths grow by one token per step."""
    grow = int((wl.max_lens - wl.lens).min())
    if wl.layers > 1:
        return wl.layers, wl.layers, grow
    return 1, LAYERS, grow


def run_kv4(args, world, rank, local, wl=None, light=False):
    """The bench line of one workload.  light: a workload measured beside the line (per_config):
    args.per_config_steps steps after 5 warm-up steps, no e2e leg and no CPU baseline."""
    import torch
    sys.path.insert(0, ROOT)
    from int4_kv_cache_append_b200 import harness as H, kv4

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    wl = make_wl(args) if wl is None else wl
    B = wl.B
    lens0 = wl.lens.astype(np.int32)
    per_step, resident, grow = step_shape(wl)
    steps, warmup = (args.per_config_steps, 5) if light else (args.steps, args.warmup)
    if grow and steps > grow:
        raise SystemExit(f"{wl.name}: at most {grow} timed steps (page capacity for growth)")
    maxlen = int(lens0.max()) + grow
    stream = torch.cuda.Stream(dev)

    def setup(bf16: bool, layers: int):
        geo = H.geometry(wl, layers=layers, value_format=0 if bf16 else wl.value_format)
        cache = kv4.BF16Cache(geo, device=dev) if bf16 else kv4.Cache(geo, device=dev)
        for layer in range(layers):
            H.prefill(cache, wl, layer, lens0, upto=lens0 - 1, bf16_pool=bf16,
                      allocate=not bf16 and wl.value_format == kv4.KV4_KEYS_MIXED)
        factor = torch.from_numpy(wl.factor()).to(dev)
        bt = torch.arange(B, dtype=torch.int32, device=dev)
        pos = torch.from_numpy(lens0 - 1).to(dev)
        ins = []
        for layer in range(layers):
            K1, V1 = H.device_kv(wl, layer, bt, pos, factor)
            ins.append((K1, V1, H.device_q(wl, layer, 0, dev)))
        return cache, ins, bt

    class Steps:
        """Kernels of one layer (append, decode) and of one whole step, on `stream`.  `st` holds
        the new token's position (row 0) and the length after it (row 1) of every sequence; a
        growing workload advances both by one at the end of each step."""

        def __init__(self, cache, ins, bt, bf16, layers):
            self.cache, self.ins, self.bt, self.bf16, self.layers = cache, ins, bt, bf16, layers
            self.page_table = torch.from_numpy(wl.page_table).to(dev)
            self.st0 = torch.from_numpy(np.stack([lens0 - 1, lens0])).to(dev)
            self.st = self.st0.clone()
            self.out = torch.empty((B, wl.Hq, wl.D), dtype=torch.float32, device=dev)
            self.ws = cache.workspace(B)

        def append(self, layer):
            K1, V1, _ = self.ins[layer]
            if self.bf16:
                self.cache.append(layer, K1, V1, self.bt, self.st[0], self.page_table, stream=stream)
            else:
                self.cache.append(layer, K1, V1, self.bt, self.st[0], self.st[1], self.page_table, stream=stream)

        def decode(self, layer):
            self.cache.decode(layer, self.ins[layer][2], self.page_table, self.st[1], out=self.out,
                              max_len_hint=maxlen, workspace=self.ws, stream=stream)

        def advance(self):
            if grow:
                self.st.add_(1)

        def reset(self):
            self.st.copy_(self.st0)

        def step(self, i):
            """Step i: every layer (multi-layer workloads) or resident layer i % layers."""
            for layer in (range(self.layers) if per_step > 1 else [i % self.layers]):
                self.append(layer)
                self.decode(layer)
            self.advance()

    def capture(fns):
        """One CUDA graph per callable (each warmed once outside capture, which sets kernel
        attributes).  Returns the graphs and the library kernel launches one replay of each makes."""
        graphs, counts = [], []
        with torch.cuda.stream(stream):
            for fn in fns:
                fn()
            stream.synchronize()
            for fn in fns:
                n0 = kv4.kv4_launch_count()
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    fn()
                counts.append(kv4.kv4_launch_count() - n0)
                graphs.append(g)
        return graphs, counts

    def timed(S, steps, warmup, sampler=None, soak_s=0.0):
        """Two timed loops of `steps` steps each, after `warmup` untimed ones.

        Kernel loop: layer launches in turn (layer i % layers), each append and each decode as its
        own graph with CUDA events between them -> the mean append and decode (decode + merge
        kernels) durations.  Step loop: `steps` steps, each one graph holding the step's kernels
        in stream order, the decode a programmatic dependent of the append before it -> the step
        time.  Lengths are reset before each loop."""
        L = S.layers
        if args.no_graph:
            run_a = S.append
            run_d = S.decode
            run_s = S.step
            n0 = kv4.kv4_launch_count()
            S.step(0)
            torch.cuda.synchronize(dev)
            launches_per_step = kv4.kv4_launch_count() - n0
        else:
            gA, _ = capture([lambda l=l: S.append(l) for l in range(L)])
            gD, _ = capture([lambda l=l: S.decode(l) for l in range(L)])
            n_graphs = 1 if per_step > 1 else L
            gS, cS = capture([lambda i=i: S.step(i) for i in range(n_graphs)])
            launches_per_step = cS[0]
            run_a = lambda l: gA[l].replay()
            run_d = lambda l: gD[l].replay()
            run_s = lambda i: gS[i % n_graphs].replay()
        adv = S.advance
        with torch.cuda.stream(stream):
            S.reset()
            for i in range(warmup):
                run_s(i)
                if grow and (i + 1) % grow == 0:
                    S.reset()
            stream.synchronize()
            if sampler:
                sampler.start()
                t_end = time.perf_counter() + soak_s
                i = 0
                S.reset()
                while time.perf_counter() < t_end:
                    run_s(i)
                    i += 1
                    if grow and i % grow == 0:
                        S.reset()
                    if i % 16 == 0:
                        stream.synchronize()
                stream.synchronize()
            # kernel loop
            S.reset()
            barrier(world)
            torch.cuda.synchronize(dev)
            ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
            for i in range(steps):
                layer = i % L
                ev[i][0].record(stream)
                run_a(layer)
                ev[i][1].record(stream)
                run_d(layer)
                ev[i][2].record(stream)
                if layer == L - 1 or per_step == 1:
                    adv()
            torch.cuda.synchronize(dev)
            dec_ms = float(np.mean([e[1].elapsed_time(e[2]) for e in ev]))
            app_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in ev]))
            kernel_loop_lens = [int(i // L) if per_step > 1 else i for i in range(steps)] if grow else [0]
            # step loop
            S.reset()
            torch.cuda.synchronize(dev)
            barrier(world)
            torch.cuda.synchronize(dev)
            start = torch.cuda.Event(enable_timing=True)
            end = torch.cuda.Event(enable_timing=True)
            start.record(stream)
            for i in range(steps):
                run_s(i)
            end.record(stream)
            end.synchronize()
            torch.cuda.synchronize(dev)
        barrier(world)
        clocks = sampler.stop() if sampler else None
        total_ms = start.elapsed_time(end)
        return total_ms, dec_ms, app_ms, launches_per_step * steps, clocks, kernel_loop_lens

    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass

    # ---- INT4 cache (the product)
    cache, ins, bt = setup(False, resident)
    # lens and page_table are written before the step, never by the append: the decode may build
    # its schedule while the append runs
    mixed = wl.value_format == kv4.KV4_KEYS_MIXED
    if not mixed:
        kv4.kv4_set_decode_overlap(cache.handle, 0 if args.no_overlap else 1)
    S = Steps(cache, ins, bt, False, resident)
    total_ms, dec_ms, app_ms, launches, clocks, klens = timed(S, steps, warmup, sampler=ClockSampler(uuid),
                                                               soak_s=0.3 if light else args.soak_s)
    err = kv4.kv4_get_device_error()
    if err:
        raise RuntimeError(f"device error bits {err:#x} during the benchmark")
    total_ms = max_over_ranks(total_ms, world)
    value = whole_job_rate(B * steps, world, total_ms)

    # algorithmic bytes of one decode launch, averaged over the lengths the kernel loop saw
    def alg_of(kv_fn):
        kv = float(np.mean([kv_fn(lens0 + d) for d in klens]))
        pt = float(np.mean([4 * ((lens0 + d + wl.P - 1) // wl.P).sum() for d in klens]))
        return kv, pt
    kv_bytes, pt_bytes = alg_of(wl.kv_bytes_int4)
    io_bytes = B * wl.Hq * wl.D * (2 + 4)  # bf16 q in, fp32 out
    alg_bytes = kv_bytes + pt_bytes + io_bytes
    peak, peak_kind = peaks()
    achieved = alg_bytes / (dec_ms / 1e3) / 1e9
    roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "traffic": profiled_traffic(wl.name),
            "kernel": ("decode_mixed_kernel + merge_kernel (kv4_decode_attn on the mixed bit-width key cache)" if mixed
                       else "decode_int4_kernel + merge_int4_kernel (kv4_decode_attn: split-K tiles, then LSE merge)"),
            "bytes_per_launch": int(alg_bytes), "kv_bytes_per_launch": int(kv_bytes), "decode_ms": round(dec_ms, 5),
            "peak_source": f"{peak_kind} MEASURED_PEAKS.json hbm_gbs" if peak_kind == "measured" else "fallback"}
    spec_frac = achieved / 8000.0

    # ---- e2e through the public API with host buffers (pinned), every step.  Each step copies the
    # inputs of every layer call it makes (q, K, V, slots, positions, lengths) from pinned host
    # memory, runs append + decode through the C ABI and copies the (last layer's) output back.
    # The step's static inputs sit in one pinned buffer (one H2D copy), positions and lengths in a
    # second small one (they change every step of a growing workload); the C entry points are
    # called directly with device addresses.  Pipelined: inputs on an H2D stream and the output
    # on a D2H stream, device buffers double-buffered and ordered by events, so the copies of one
    # step overlap the kernels of the previous one.  The serial form (one stream) is reported
    # beside it.
    e2e = None
    if args.e2e_steps > 0 and not light:
        nl = per_step  # layer calls per step
        nsets = nl if per_step > 1 else 1
        parts = []  # (host tensor, offset) of the static inputs
        off = 0
        for l in range(nsets):
            for t in (ins[l][0], ins[l][1], ins[l][2]):
                parts.append((t.cpu().contiguous(), off))
                off += (t.numel() * t.element_size() + 255) // 256 * 256
        hb = bt.cpu()
        parts.append((hb, off))
        off += (hb.numel() * 4 + 255) // 256 * 256
        hpack = torch.empty(off, dtype=torch.uint8).pin_memory()
        for t, o in parts:
            nb = t.numel() * t.element_size()
            hpack[o:o + nb].copy_(t.view(-1).view(torch.uint8))
        nst = max(grow, 1)
        hst = [torch.from_numpy(np.stack([lens0 - 1 + k, lens0 + k])).pin_memory() for k in range(nst)]
        dpack = [torch.empty_like(hpack, device=dev) for _ in range(2)]
        dst = [torch.empty_like(hst[0], device=dev) for _ in range(2)]
        douts = [torch.empty_like(S.out) for _ in range(2)]
        houts = [torch.empty_like(S.out, device="cpu").pin_memory() for _ in range(2)]
        h2d = sum(t.numel() * t.element_size() for t, _ in parts) + hst[0].numel() * 4
        d2h = houts[0].numel() * houts[0].element_size()
        kd, vd, qd = kv4.dtype_code(ins[0][0]), kv4.dtype_code(ins[0][1]), kv4.dtype_code(ins[0][2])
        ws = S.ws
        pt_ptr, stride = S.page_table.data_ptr(), int(S.page_table.shape[1])
        calls = []  # per buffer: the (append args, decode args) of every layer call
        for j in range(2):
            base = dpack[j].data_ptr()
            slot_p = base + parts[-1][1]
            pos_p, len_p = dst[j].data_ptr(), dst[j].data_ptr() + 4 * B
            cj = []
            for li in range(nsets):
                kp, vp, qp = (base + parts[3 * li + x][1] for x in range(3))
                cj.append((kp, vp, qp, slot_p, pos_p, len_p))
            calls.append(cj)
        handle = cache.handle
        up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        sh_main = stream.cuda_stream
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        for e in ev_done + ev_out:
            e.record(stream)
        lib = kv4.lib

        def step_on(j, i, pipelined):
            if pipelined:
                up.wait_event(ev_done[j])  # the step that last used buffer j has finished
            with torch.cuda.stream(up if pipelined else stream):
                dpack[j].copy_(hpack, non_blocking=True)
                dst[j].copy_(hst[i % nst], non_blocking=True)
            if pipelined:
                ev_in[j].record(up)
                stream.wait_event(ev_in[j])
                stream.wait_event(ev_out[j])  # its previous output has been copied out
            layers = range(nl) if per_step > 1 else [i % resident]
            for (kp, vp, qp, slot_p, pos_p, len_p), layer in zip(calls[j], layers):
                st_ = lib.kv4_append(handle, layer, B, kp, kd, vp, vd, slot_p, pos_p, len_p, pt_ptr, stride, sh_main)
                sd_ = lib.kv4_decode_attn(handle, layer, B, qp, qd, pt_ptr, stride, len_p, maxlen,
                                          douts[j].data_ptr(), None, ws.data_ptr(), ws.numel(), sh_main)
                if st_ or sd_:
                    raise RuntimeError(f"kv4 call failed: append {st_}, decode {sd_}")
            if pipelined:
                ev_done[j].record(stream)
                down.wait_event(ev_done[j])
            with torch.cuda.stream(down if pipelined else stream):
                houts[j].copy_(douts[j], non_blocking=True)
            if pipelined:
                ev_out[j].record(down)

        def run(pipelined):
            for i in range(3):
                step_on(i % 2, i, pipelined)
            torch.cuda.synchronize(dev)
            barrier(world)
            s0 = torch.cuda.Event(enable_timing=True)
            s1 = torch.cuda.Event(enable_timing=True)
            s0.record(stream)
            for i in range(args.e2e_steps):
                step_on(i % 2, i, pipelined)
            if pipelined:
                stream.wait_event(ev_out[(args.e2e_steps - 1) % 2])
            s1.record(stream)
            s1.synchronize()
            return max_over_ranks(s0.elapsed_time(s1), world)

        serial_ms = run(False)
        e2e_ms = run(True)
        e2e = {"value": whole_job_rate(B * args.e2e_steps, world, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
               "e2e_serial": whole_job_rate(B * args.e2e_steps, world, serial_ms),
               "path": "kv4_append + kv4_decode_attn (C ABI) for every layer call of the step; every step copies "
                       "the inputs of those calls from pinned host memory (one packed buffer, plus positions and "
                       "lengths) and the last output back; copies on H2D/D2H streams overlap the previous step's "
                       "kernels (double-buffered); e2e_serial: the same on one stream"}

    del cache, ins, S
    torch.cuda.empty_cache()

    # ---- BF16-KV baseline kernel on the same GPU.  A multi-layer step is timed on LAYERS of its
    # layers (BF16 KV of every layer would not fit) and scaled by per_step / LAYERS: the layers
    # are identical in shape, so the per-layer cost is the same.
    bf = None
    if not args.no_bf16:
        bl = min(resident, LAYERS)
        bcache, bins, bbt = setup(True, bl)
        BS = Steps(bcache, bins, bbt, True, bl)
        b_total, b_dec, b_app, _, _, bklens = timed(BS, steps, warmup)
        scale = per_step / bl if per_step > 1 else 1.0
        b_total = max_over_ranks(b_total, world) * scale
        bkv = float(np.mean([wl.kv_bytes_bf16(lens0 + d) for d in bklens]))
        b_alg = bkv + pt_bytes + io_bytes
        bf = {"value": whole_job_rate(B * steps, world, b_total), "unit": UNIT, "ms_per_step": b_total / steps,
              "decode_ms": round(b_dec, 5), "append_ms": round(b_app, 5), "kv_bytes_per_launch": int(bkv),
              "achieved_GBps": round(b_alg / (b_dec / 1e3) / 1e9, 1),
              "frac": round(b_alg / (b_dec / 1e3) / 1e9 / peak, 4),
              "int4_speedup_step": round(value / whole_job_rate(B * steps, world, b_total), 3),
              "int4_speedup_decode": round(b_dec / dec_ms, 3)}
        if per_step > 1:
            bf["layers_timed"] = f"{bl} of {per_step} layers per step, time scaled by {scale:g}"
        del bcache, bins, BS
        torch.cuda.empty_cache()

    cpu = None
    if world == 1 and rank == 0 and not args.no_cpu_baseline and not light:
        cpu = cpu_baseline(wl, nseq=min(SAMPLE_SEQS, wl.B), per_step=per_step)

    resident_gb = resident * kv_bytes / 1e9
    line = {"metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": steps,
            "warmup": warmup, "ms_per_step": round(total_ms / steps, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": wl.name, "inputs": INPUTS, "B_per_gpu": B, "Hq": wl.Hq, "Hkv": wl.Hkv, "D": wl.D, "P": wl.P,
                       "s": wl.s, "w": wl.w, "h": wl.h, "len_mean": round(float(lens0.mean()), 1),
                       "len_max": int(lens0.max()), "layers_per_step": per_step,
                       "growth_per_step": 1 if grow else 0,
                       "kv_dtype": (f"packed K{wl.key_bits} (RoPE-block widths) V{wl.value_bits} pages" if mixed
                                    else "int4 K + bf16 V pages, int8 K + bf16 V side cache" if wl.value_format
                                    else "int4 pages + int8 side cache"),
                       "compute": ("QK^T and PV f16 MMA on integer codes with hi/lo f16 weights, f32 accumulate, "
                                   "f32 softmax" if mixed else
                                   "QK^T int8 MMA (exact int32), PV f16 MMA with f32 accumulate, f32 softmax"),
                       "l2": f"inputs larger than L2: {resident} resident layers cycled, {resident_gb:.2f} GB of KV "
                             f"between reuses",
                       "parallelism": f"dp{world} (independent batches per GPU, no collective)",
                       "graph": ("one graph per step (append -> decode programmatic edge)" if not args.no_graph
                                 else False),
                       "decode_overlap": not args.no_overlap, "append_ms": round(app_ms, 5),
                       "timing": "step loop (value) and kernel loop (decode_ms, append_ms), each `steps` long"},
            "roofline": roof, "hbm_frac_of_spec_8TBps": round(spec_frac, 4), "gpu_launches": int(launches),
            "clocks": clocks, "e2e": e2e, "bf16_kv": bf, "cpu_baseline": cpu}
    return line if rank == 0 else None


def per_config_record(line: dict, note: str | None) -> dict:
    """The figures of a one-layer workload's line that go into the default line's per_config."""
    r, b, c = line["roofline"], line["bf16_kv"], line["config"]
    rec = {"decode_ms": r["decode_ms"], "bytes_per_launch": r["bytes_per_launch"], "achieved_GBps": r["achieved"],
           "frac": r["frac"], "peak": r["peak"], "frac_of_spec_8TBps": line["hbm_frac_of_spec_8TBps"],
           "append_ms": c["append_ms"], "ms_per_step": line["ms_per_step"], "value": line["value"],
           "B": c["B_per_gpu"], "len_mean": c["len_mean"], "len_max": c["len_max"], "s": c["s"], "w": c["w"],
           "h": c["h"], "P": c["P"], "steps": line["steps"], "clocks": line["clocks"]}
    if b:
        rec.update({"bf16_decode_ms": b["decode_ms"], "bf16_frac": b["frac"],
                    "int4_over_bf16_decode": b["int4_speedup_decode"]})
    if note:
        rec["note"] = note
    return rec


def main():
    args = parse()
    if args.impl == "reference":
        # the host-core oracle: rank 0 alone runs and prints; other ranks exit without work
        world = int(os.environ.get("WORLD_SIZE", "1"))
        line = run_reference(args, world, int(os.environ.get("RANK", "0")))
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    world, rank, local = dist_setup("nccl")
    try:
        line = run_kv4(args, world, rank, local)
        if line is not None and rank == 0 and world == 1 and not args.no_per_config:
            # the other configurations, one after the other in this process (N = 1 only)
            import dataclasses

            from int4_kv_cache_append_b200 import workload as W
            per = {}
            for name, over, note in PER_CONFIG:
                wl = W.WORKLOADS[name]()
                if "h" in over:
                    wl = dataclasses.replace(wl, h=over["h"], name=f"{wl.name}-h{over['h']}")
                if over.get("values") == "bf16":
                    wl = dataclasses.replace(wl, value_format=1, name=f"{wl.name}-vbf16")
                if "mixed" in over:
                    wl = mixed_variant(wl, *over["mixed"])
                per[wl.name] = per_config_record(run_kv4(args, world, rank, local, wl=wl, light=True), note)
            line["per_config"] = per
        if line is not None and rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
