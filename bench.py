#!/usr/bin/env python
"""Benchmark of the B200 BitLinear hot path (y = F.linear(ActQuant(x), WeightQuant(W))).

Headline (one JSON line on rank 0):
  metric  BitLinear GB/s (M=1 decode) and int8 TOPS (prefill) as % of B200 roofline
  value   decode GB/s of the BitNet-b1.58-2B-4T layer set at M=1 (qkv 2560->3840,
          o 2560->2560, gate+up 2560->13824, down 6912->2560): one step = the four
          BitLinear forwards (ActQuant fused into the packed-weight GEMV, rescale
          in the epilogue), replayed from a CUDA graph. Weights rotate over 32
          copies (556 MB > 126 MB L2), so every step streams them from HBM.
  prefill the same path at M=4096 (qkv, gate+up, down with Laplace weights):
          TOPS of the tcgen05 GEMM kernel, GB/s of ActQuant.
  pack    WeightQuant + 2-bit pack of the gate+up weight (offline op).

Algorithmic bytes/ops count only what the method must move or compute:
decode = packed weights (N*K/4) + D (4N) + x (4MK) + y (4MN); prefill = 2*M*N*K.

Usage: python bench.py [--gpus N --steps K --warmup W] [--impl reference]
Under torchrun each rank runs an independent replica (weak scaling, no collective
on the data path); timings are device events, max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from bit_ternary_b200 import workloads as WL  # noqa: E402

METRIC = "BitLinear GB/s (M=1 decode) and int8 TOPS (prefill) as % of B200 roofline"
HEADLINE = "decode_layer_set"
PREFILL = "prefill_sweep"
PREFILL_M = 4096
ROTATE = 32
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
INT8_PER_BF16 = 2.0  # nominal dense ratio (4.5 POPS int8 / 2.25 PFLOPS bf16)


# --------------------------------------------------------------------------- utils
def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--ncu-small", action="store_true",
                    help="small decode-only run for profiler captures (4 weight copies, no extras)")
    ap.add_argument("--ncu-prefill", action="store_true",
                    help="small prefill-only run for profiler captures (gate_up layer, M=4096)")
    ap.add_argument("--ncu-layer", default=None, metavar="WORKLOAD:LAYER:M",
                    help="one layer of a workload, M tokens, for profiler captures (e.g. embed_batch:0:32768)")
    ap.add_argument("--ncu-rms", action="store_true",
                    help="with --ncu-layer: the RMSNorm + BitLinear forward (norm weight of ones)")
    ap.add_argument("--ncu-i2s", action="store_true",
                    help="I2_S export/import only (stacked gate_up weights), for profiler captures")
    ap.add_argument("--only", default=None, metavar="PARTS",
                    help="run only these parts (comma-separated: prefill, configs, bf16, rmsnorm, pack, "
                         "decode_stream, i2s) "
                         "and print their results; no headline line")
    ap.add_argument("--i2s-layouts", default="consecutive,quarters",
                    help="byte groupings timed by the I2_S part (comma-separated)")
    a = ap.parse_args(argv)
    a.warmup = max(3, a.warmup)
    a.steps = max(1, a.steps)
    return a


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(v, device=None):
    """Max of a per-rank float over the process group (identity without one)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(v)
    t = torch.tensor([float(v)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_gbs(world, bytes_per_step, steps, ms_max):
    """Whole-job GB/s: every rank moved bytes_per_step per step; time is the slowest rank's."""
    return world * bytes_per_step * steps / (ms_max * 1e-3) / 1e9


def decode_bytes(layers, M):
    tot = 0
    for l in layers:
        tot += l.N * l.K // 4 + 4 * l.N + 4 * M * l.K + 4 * M * l.N
    return tot


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while work runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append({"sm": float(parts[1]), "max": float(parts[2]), "power": float(parts[3]),
                                 "hw": parts[5], "hwt": parts[6], "swt": parts[7], "pcap": parts[8]})
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        pmax = max(r["power"] for r in rows)
        load = [r for r in rows if r["power"] >= 0.5 * pmax] or rows
        reasons = set()
        for r in load:
            for k, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                            ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[k].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in load), "sm_max_mhz": max(r["max"] for r in rows),
                "reasons": sorted(reasons), "samples": len(load), "power_w_max": pmax}


# ------------------------------------------------------------------- reference arm
def oracle_decode_step(layers, packs, xs, row_frac=1.0):
    """One layer-set forward by the CPU oracle (optionally on a row sample)."""
    import oracle as O

    done_bytes = 0
    for l, (p_ref, D_ref), x in zip(layers, packs, xs):
        n = max(1, int(round(l.N * row_frac)))
        O.bitlinear_forward(x, p_ref[:n], D_ref[:n], l.K)
        done_bytes += n * l.K // 4 + 4 * n + 4 * x.shape[0] * l.K + 4 * x.shape[0] * n
    return done_bytes


def prepare_oracle_inputs(key, M):
    import oracle as O

    wl = WL.WORKLOADS[key]
    packs, xs = [], []
    for li, l in enumerate(wl.layers):
        W = WL.weight(l.N, l.K, wl.w_dist, wl.seed, layer=li)
        packs.append(O.pack_weights(W))
        xs.append(WL.activations(M, l.K, wl.x_dist, wl.seed, layer=li, meta=wl.meta))
    return wl, packs, xs


def _oracle_worker(args):
    """One host process of the all-core oracle timing: whole layer-set forwards for `seconds`."""
    seconds, layers, packs, xs = args
    t0 = time.perf_counter()
    nbytes, steps = 0, 0
    while True:
        nbytes += oracle_decode_step(layers, packs, xs)
        steps += 1
        if time.perf_counter() - t0 >= seconds:
            break
    return nbytes, steps, time.perf_counter() - t0


def _oracle_processes():
    """Host processes for the all-core timing: one per core available to this process, capped
    so that their working sets (~0.6 GB each: the oracle unpacks a layer's codes to int64) fit
    in half of the host memory."""
    ncores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
    try:
        mem = os.sysconf("SC_PAGE_SIZE") * os.sysconf("SC_PHYS_PAGES")
        ncores = max(1, min(ncores, int(mem * 0.5 // (0.6 * 2**30))))
    except (ValueError, OSError, AttributeError):
        pass
    return ncores


def cpu_baseline(seconds):
    """The oracle on the host cores: one process (the plain single-thread figure), then one
    process per core over the same workload (processes started by spawn, after the GPU work:
    a forked child of a CUDA process can hang), then a sampled-token prefill layer."""
    import multiprocessing as mp

    wl, packs, xs = prepare_oracle_inputs(HEADLINE, 1)
    nbytes, steps, dt = _oracle_worker((seconds, wl.layers, packs, xs))
    one = nbytes / dt / 1e9
    nproc = _oracle_processes()
    all_cores = None
    if nproc > 1:
        with mp.get_context("spawn").Pool(nproc) as pool:
            res = pool.map(_oracle_worker, [(seconds, wl.layers, packs, xs)] * nproc)
        tot_bytes = sum(r[0] for r in res)
        tot_steps = sum(r[1] for r in res)
        wall = max(r[2] for r in res)
        all_cores = {"value": tot_bytes / wall / 1e9, "unit": "GB/s", "cores": nproc,
                     "sample": f"{nproc} processes x ~{seconds:.0f} s: {tot_steps} full layer-set forwards"}
    # Prefill (C4 gate_up at M=4096) on a sample of tokens: the oracle's cost is linear in M.
    import oracle as O

    pw = WL.WORKLOADS[PREFILL]
    li = 1
    l = pw.layers[li]
    p_ref, D_ref = O.pack_weights(WL.weight(l.N, l.K, pw.w_dist, pw.seed, layer=li))
    ms = 8
    x = WL.activations(ms, l.K, pw.x_dist, pw.seed, layer=li, meta=pw.meta)
    t0 = time.perf_counter()
    O.bitlinear_forward(x, p_ref, D_ref, l.K)
    tp = time.perf_counter() - t0
    prefill = {"value": 2.0 * ms * l.N * l.K / tp / 1e12, "unit": "TOPS", "cores": 1,
               "sample": f"{PREFILL} gate_up {l.K}->{l.N}: {ms} of the {PREFILL_M} tokens, all rows, "
                         f"{tp:.2f} s (cost linear in tokens)"}
    out = {"value": one, "unit": "GB/s", "cores": 1, "kind": "oracle",
           "sample": f"{steps} full layer-set forwards (M=1, all 4 layers, all rows) in {dt:.1f} s; "
                     "numpy int64 matmul, single thread",
           "prefill_sample": prefill}
    if all_cores is not None:
        out["all_cores"] = all_cores
    return out


def run_reference(a):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    wl, packs, xs = prepare_oracle_inputs(HEADLINE, 1)
    t0 = time.perf_counter()
    oracle_decode_step(wl.layers, packs, xs)
    t_full = time.perf_counter() - t0
    budget = 150.0  # seconds for warmup + timed steps
    frac = min(1.0, budget / max(1e-9, t_full * (a.steps + a.warmup)))
    for _ in range(a.warmup):
        oracle_decode_step(wl.layers, packs, xs, frac)
    t0 = time.perf_counter()
    nbytes = 0
    for _ in range(a.steps):
        nbytes += oracle_decode_step(wl.layers, packs, xs, frac)
    dt = time.perf_counter() - t0
    v = nbytes / dt / 1e9
    sample = (f"each step: the M=1 layer set on the first {100 * frac:.1f}% of every layer's output rows "
              f"(full step measured at {t_full:.2f} s); numpy int64 matmul, single thread")
    line = {"metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": world, "steps": a.steps, "warmup": a.warmup,
            "ms_per_step": dt / a.steps * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "i8", "data": "synthetic", "impl": "reference",
            "config": {"workload": f"{HEADLINE}: {wl.description} (qkv 2560->3840, o 2560->2560, "
                                   "gate_up 2560->13824, down 6912->2560)", "M": 1},
            "cpu_baseline": {"value": v, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------------ our arm
def run_ours(a):
    import torch
    import torch.distributed as dist

    from bit_ternary_b200 import build, _lib
    from bit_ternary_b200 import bitlinear as B

    rank, world, local = dist_env()
    build.build_library()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (there is no CPU fallback)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if _lib.lib().bitlinear_device_check() != 0:
        raise SystemExit("device is not sm_100 (B200)")
    if a.ncu_prefill or a.ncu_layer:
        return run_prefill_small(a, B, torch, dev)
    if a.ncu_i2s:
        peaks, _ = load_peaks()
        stream = torch.cuda.Stream(device=dev)
        print(json.dumps({"i2s": bench_i2s(B, torch, dev, stream, float(peaks["hbm_gbs"]), reps=2,
                                           layouts=tuple(a.i2s_layouts.split(",")))}))
        return 0
    if world > 1:
        import datetime

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    def max_ranks(v):
        return max_over_ranks(v, dev)

    peaks, peak_src = load_peaks()
    hbm_peak = float(peaks["hbm_gbs"])
    i8_burst = float(peaks["bf16_tflops"]) * INT8_PER_BF16
    i8_sust = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])) * INT8_PER_BF16
    stream = torch.cuda.Stream(device=dev)

    def capture(fn, n):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(n):
                fn(i)
        return g

    def time_graph(g):
        barrier()
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):  # replay() launches on the current stream
            e0.record(stream)
            g.replay()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        return e0.elapsed_time(e1)

    if a.only:
        parts = {
            "prefill": lambda: bench_prefill(a, B, torch, dev, stream, capture, time_graph, max_ranks, hbm_peak,
                                             i8_burst, i8_sust, rank),
            "configs": lambda: bench_configs(B, torch, dev, stream, capture, time_graph, max_ranks, hbm_peak,
                                             i8_burst, rank),
            "bf16": lambda: bench_bf16(B, torch, dev, stream, capture, time_graph, max_ranks, hbm_peak, rank),
            "rmsnorm": lambda: bench_rmsnorm(B, torch, dev, stream, capture, time_graph, max_ranks, hbm_peak,
                                             i8_burst),
            "pack": lambda: bench_pack(B, torch, dev, stream, hbm_peak),
            "decode_stream": lambda: bench_decode_stream(B, torch, dev, stream, capture, time_graph, max_ranks,
                                                         hbm_peak),
            "i2s": lambda: bench_i2s(B, torch, dev, stream, hbm_peak, layouts=tuple(a.i2s_layouts.split(","))),
            "block_scale": lambda: bench_block_scale(B, torch, dev, stream, capture, time_graph, max_ranks,
                                                     hbm_peak, i8_burst, rank),
        }
        res = {name: parts[name]() for name in a.only.split(",")}
        if rank == 0:
            print(json.dumps({"only": res}))
        return 0

    # ---------------------------------------------------------------- decode setup
    wl = WL.WORKLOADS[HEADLINE]
    M = 1
    layers = list(wl.layers)
    rot = 4 if a.ncu_small else ROTATE
    packs = []  # [rot][layer] -> (packed, D)
    base = []
    with torch.cuda.stream(stream):
        for li, l in enumerate(layers):
            W = torch.from_numpy(WL.weight(l.N, l.K, wl.w_dist, wl.seed + 17 * rank, layer=li)).to(dev)
            base.append(B.pack_weights(W))
            del W
        for r in range(rot):
            packs.append([(p.clone(), D.clone()) for (p, D) in base])
        xs = [[torch.from_numpy(WL.activations(M, l.K, wl.x_dist, wl.seed + r, layer=li, meta=wl.meta)).to(dev)
               for li, l in enumerate(layers)] for r in range(rot)]
        ys = [[torch.empty((M, l.N), dtype=torch.float32, device=dev) for l in layers] for _ in range(rot)]
        wss = [torch.zeros(max(256, B.workspace_size(M, l.N, l.K)), dtype=torch.uint8, device=dev) for l in layers]
    torch.cuda.synchronize(dev)
    step_bytes = decode_bytes(layers, M)

    EARLY = _lib.BL_FLAG_STREAM_WEIGHTS_EARLY

    def decode_step(i):
        # Four dependent-style BitLinear calls, one launch each; weights are
        # static, so each launch may stream them while the previous one runs.
        r = i % rot
        for li, l in enumerate(layers):
            p, D = packs[r][li]
            B.forward_batch([(xs[r][li], p, D, ys[r][li])], flags=EARLY, ws=wss[li])

    def decode_step_plain(i):
        r = i % rot
        for li, l in enumerate(layers):
            p, D = packs[r][li]
            B.forward(xs[r][li], p, D, out=ys[r][li], ws=wss[li])

    def decode_step_grouped(i):
        r = i % rot
        B.forward_batch([(xs[r][li], packs[r][li][0], packs[r][li][1], ys[r][li]) for li in range(len(layers))],
                        flags=EARLY, ws=wss[3])

    # warm-up: eager W steps, then the graph once
    with torch.cuda.stream(stream):
        for i in range(a.warmup):
            decode_step(i)
        if a.ncu_small:
            # grouped launches right after the per-layer warm-up (profiler captures)
            for i in range(3):
                decode_step_grouped(i)
    torch.cuda.synchronize(dev)
    g_dec = capture(decode_step, a.steps)
    gpu_id = None
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        gpu_id = str(local)
    clocks = ClockSampler(gpu_id)
    clocks.start()
    # soak: keep the GPU under this load ~1 s before the timed replay (clock samples)
    t_soak = time.perf_counter()
    while time.perf_counter() - t_soak < 1.0:
        with torch.cuda.stream(stream):
            g_dec.replay()
        torch.cuda.synchronize(dev)
    ms = max_ranks(time_graph(g_dec))
    clk = clocks.stop()
    variants = {}
    if not a.ncu_small:
        for name, fn in (("per_layer_plain", decode_step_plain), ("grouped_one_launch", decode_step_grouped)):
            gv = capture(fn, a.steps)
            with torch.cuda.stream(stream):
                gv.replay()
            msv = max_ranks(time_graph(gv))
            variants[name] = {"GB/s": round(weak_scaling_gbs(world, step_bytes, a.steps, msv), 1),
                              "us_per_step": round(msv / a.steps * 1e3, 3),
                              "frac_hbm": round(step_bytes / (msv / a.steps * 1e-3) / 1e9 / hbm_peak, 4)}
            del gv
    ms_step = ms / a.steps
    value = weak_scaling_gbs(world, step_bytes, a.steps, ms)
    launches_per_step = len(layers)
    achieved = step_bytes / (ms_step * 1e-3) / 1e9

    # per-layer breakdown (each layer alone, same rotation, own graph)
    per_layer = []
    if not a.ncu_small:
        nl = max(50, min(a.steps, 400))
        for li, l in enumerate(layers):
            def one(i, li=li):
                r = i % rot
                p, D = packs[r][li]
                B.forward_batch([(xs[r][li], p, D, ys[r][li])], flags=EARLY, ws=wss[li])
            g = capture(one, nl)
            with torch.cuda.stream(stream):
                g.replay()
            t = max_ranks(time_graph(g)) / nl
            b = decode_bytes([l], M)
            per_layer.append({"layer": l.name, "K": l.K, "N": l.N, "us": round(t * 1e3, 3),
                              "GB/s": round(b / (t * 1e-3) / 1e9, 1),
                              "frac_hbm": round(b / (t * 1e-3) / 1e9 / hbm_peak, 4)})
            del g

    # e2e through the public C ABI with host buffers (pinned): the step's four
    # activations sit in one pinned buffer and its four outputs in another, so
    # the batched host call moves each with one copy (H2D, four launches, D2H).
    x_all = torch.empty(sum(M * l.K for l in layers), dtype=torch.float32).pin_memory()
    y_all = torch.empty(sum(M * l.N for l in layers), dtype=torch.float32).pin_memory()
    x_host, y_host, xo, yo = [], [], 0, 0
    for li, l in enumerate(layers):
        xv = x_all[xo:xo + M * l.K].view(M, l.K)
        xv.copy_(torch.from_numpy(WL.activations(M, l.K, wl.x_dist, wl.seed, layer=li, meta=wl.meta)))
        x_host.append(xv)
        y_host.append(y_all[yo:yo + M * l.N].view(M, l.N))
        xo += M * l.K
        yo += M * l.N
    ws_batch_host = torch.zeros(B.batch_host_workspace_size([(M, l.N, l.K) for l in layers]), dtype=torch.uint8,
                                device=dev)
    ws_host = [torch.zeros(_lib.lib().bitlinear_host_workspace_size(M, l.N, l.K), dtype=torch.uint8, device=dev)
               for l in layers]
    h2d = sum(4 * M * l.K for l in layers)
    d2h = sum(4 * M * l.N for l in layers)
    ONE = _lib.BL_FLAG_ONE_LAUNCH_PER_CALL

    # The C call's descriptors, built once per weight rotation as a C caller
    # with persistent pinned buffers would; each step is then one call into
    # the library plus one synchronise.
    Lib = _lib.lib()
    call_arrays = []
    for r in range(rot):
        arr = (_lib.LinearCall * len(layers))()
        for li, l in enumerate(layers):
            arr[li] = _lib.LinearCall(x_host[li].data_ptr(), M, l.N, l.K, packs[r][li][0].data_ptr(),
                                      packs[r][li][1].data_ptr(), y_host[li].data_ptr())
        call_arrays.append(arr)
    ws_bh_ptr, ws_bh_bytes, stream_ptr = ws_batch_host.data_ptr(), ws_batch_host.numel(), stream.cuda_stream

    def e2e_step(i):
        # One batched host call per step; the step ends when its results are
        # in pinned host memory (one synchronise).
        st = Lib.bitlinear_forward_batch_host(call_arrays[i % rot], len(layers), EARLY | ONE, ws_bh_ptr,
                                              ws_bh_bytes, stream_ptr)
        if st != 0:
            raise RuntimeError(f"bitlinear_forward_batch_host failed: {st}")
        stream.synchronize()

    def e2e_step_binding(i):
        # The same step through the Python binding (argument checks each call).
        r = i % rot
        B.forward_batch_host([(x_host[li], packs[r][li][0], packs[r][li][1], y_host[li])
                              for li in range(len(layers))], flags=EARLY | ONE, ws=ws_batch_host)
        stream.synchronize()

    def e2e_step_per_call(i):
        # The same step as four single host calls (H2D + forward + D2H each).
        r = i % rot
        for li, l in enumerate(layers):
            p, D = packs[r][li]
            B.forward_host(x_host[li], p, D, y_host[li], ws=ws_host[li], sync=False)
        stream.synchronize()

    def time_e2e(fn):
        with torch.cuda.stream(stream):
            for i in range(a.warmup):
                fn(i)
            n = min(a.steps, 200)
            barrier()
            torch.cuda.synchronize(dev)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for i in range(n):
                fn(i)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            barrier()
        return max_ranks(e0.elapsed_time(e1)) / n

    ms_e2e = time_e2e(e2e_step)
    e2e_val = weak_scaling_gbs(world, step_bytes, 1, ms_e2e)
    ms_e2e_pc = time_e2e(e2e_step_per_call)
    e2e_per_call = {"GB/s": round(weak_scaling_gbs(world, step_bytes, 1, ms_e2e_pc), 3),
                    "ms_per_step": round(ms_e2e_pc, 4),
                    "api": "Python binding forward_host(sync=False) x4, one synchronise"}
    ms_e2e_b = time_e2e(e2e_step_binding)
    e2e_binding = {"GB/s": round(weak_scaling_gbs(world, step_bytes, 1, ms_e2e_b), 3),
                   "ms_per_step": round(ms_e2e_b, 4),
                   "api": "Python binding forward_batch_host (checks each call), one synchronise"}

    # free decode buffers before prefill
    del g_dec
    packs = xs = ys = None
    torch.cuda.synchronize(dev)
    torch.cuda.empty_cache()

    # ------------------------------------------------------------------ prefill
    prefill = None
    if not a.no_prefill and not a.ncu_small:
        prefill = bench_prefill(a, B, torch, dev, stream, capture, time_graph, max_ranks, hbm_peak,
                                i8_burst, i8_sust, rank)

    # ------------------------------------------------------- the other configs
    configs = None
    if not a.no_prefill and not a.ncu_small:
        configs = bench_configs(B, torch, dev, stream, capture, time_graph, max_ranks, hbm_peak, i8_burst, rank)

    # --------------------------------------------------------------------- pack
    pack = i2s = dstream = None
    if not a.ncu_small:
        dstream = bench_decode_stream(B, torch, dev, stream, capture, time_graph, max_ranks, hbm_peak)
        pack = bench_pack(B, torch, dev, stream, hbm_peak)
        i2s = bench_i2s(B, torch, dev, stream, hbm_peak, layouts=tuple(a.i2s_layouts.split(",")))

    # ----------------------------------------------------- RMSNorm + ActQuant
    rms = None
    if not a.no_prefill and not a.ncu_small:
        rms = bench_rmsnorm(B, torch, dev, stream, capture, time_graph, max_ranks, hbm_peak, i8_burst)

    # ------------------------------------------------------------- bf16 inputs
    bf16 = None
    if not a.no_prefill and not a.ncu_small:
        bf16 = bench_bf16(B, torch, dev, stream, capture, time_graph, max_ranks, hbm_peak, rank)

    # ------------------------------------------------- per-256-block scale variant
    blk = None
    if not a.no_prefill and not a.ncu_small:
        blk = bench_block_scale(B, torch, dev, stream, capture, time_graph, max_ranks, hbm_peak, i8_burst, rank)

    # --------------------------------------------------------------- cpu baseline
    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline and not a.ncu_small:
        cpu = cpu_baseline(a.cpu_seconds)

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0
    traffic = load_traffic("bl_ternary_decode_kernel")
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": a.steps,
        "warmup": a.warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "i8", "data": "synthetic",
        "config": {"workload": f"{HEADLINE}: {wl.description} (qkv 2560->3840, o 2560->2560, "
                               "gate_up 2560->13824, down 6912->2560), fp32 x in, fp32 y out; "
                               "four BitLinear calls per step, each its own launch, weights streamed early "
                               "(programmatic dependent launch), activations read after the previous launch",
                   "M": M, "bytes_per_step": step_bytes,
                   "l2": f"inputs larger than L2: weights rotate over {rot} copies "
                         f"({rot * sum(l.N * l.K // 4 for l in layers) / 1e6:.0f} MB)",
                   "parallelism": f"replica per GPU x{world} (independent decode streams)",
                   "graph": "CUDA graph of the timed steps"},
        "roofline": {"bound": "hbm", "kernel": "bl_ternary_decode_kernel (fused ActQuant + packed-weight ring + int8 MMA + rescale)",
                     "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
                     "frac": round(achieved / hbm_peak, 4), "traffic": traffic,
                     "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured" else
                     "fallback 6.65 TB/s", "per_launch_bytes": step_bytes / launches_per_step,
                     "avg_launch_us": round(ms_step * 1e3 / launches_per_step, 3)},
        "layers": per_layer,
        "decode_variants": variants,
        "e2e": {"value": round(e2e_val, 3), "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(ms_e2e, 4),
                "api": "C ABI bitlinear_forward_batch_host through ctypes, call descriptors built once (4 layers; "
                       "one pinned x buffer and one pinned y buffer: 1 H2D, 4 launches, 1 D2H) + one stream "
                       "synchronise per step",
                "binding_variant": e2e_binding, "per_call_variant": e2e_per_call},
        "gpu_launches": launches_per_step * a.steps,
        "clocks": clk,
        "prefill": prefill,
        "configs": configs,
        "decode_streaming": dstream,
        "pack": pack,
        "i2s": i2s,
        "bf16_inputs": bf16,
        "rmsnorm_actquant": rms,
        "block_scale": blk,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)
    return 0


def load_traffic(kernel):
    """DRAM bytes per launch from a committed ncu summary, if it matches the current kernel sources."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        with open(p) as f:
            d = json.load(f)
        from bit_ternary_b200 import build

        v = d.get("kernels", {}).get(kernel)
        if not isinstance(v, dict) or v.get("sha") != build.kernel_sha(kernel):
            return None
        return v.get("bytes_per_launch")
    except Exception:
        return None


L2_FLUSH_BYTES = 256 << 20  # twice the 126 MB L2: a rotation through this much traffic evicts it


def rotation(bytes_per_call, cap=16):
    """Copies of a call's buffers to cycle through so that the data one call
    touches was last touched at least L2_FLUSH_BYTES of traffic earlier."""
    return int(min(cap, max(2, -(-L2_FLUSH_BYTES // max(1, bytes_per_call)))))


def bench_prefill(a, B, torch, dev, stream, capture, time_graph, max_ranks, hbm_peak, i8_burst, i8_sust, rank):
    wl = WL.WORKLOADS[PREFILL]
    M = PREFILL_M
    layers = list(wl.layers)
    with torch.cuda.stream(stream):
        pk = []
        for li, l in enumerate(layers):
            W = torch.from_numpy(WL.weight(l.N, l.K, wl.w_dist, wl.seed + 31 * rank, layer=li)).to(dev)
            pk.append(B.pack_weights(W))
            del W
        xs = [torch.from_numpy(WL.activations(M, l.K, wl.x_dist, wl.seed, layer=li)).to(dev)
              for li, l in enumerate(layers)]
        ys = [torch.empty((M, l.N), dtype=torch.float32, device=dev) for l in layers]
        wss = [torch.zeros(B.workspace_size(M, l.N, l.K), dtype=torch.uint8, device=dev) for l in layers]
    torch.cuda.synchronize(dev)
    n = max(16, min(a.steps, 32))

    def whole(i):
        for li, l in enumerate(layers):
            p, D = pk[li]
            B.forward(xs[li], p, D, out=ys[li], ws=wss[li])

    with torch.cuda.stream(stream):
        for i in range(3):
            whole(i)
    torch.cuda.synchronize(dev)
    g = capture(whole, n)
    with torch.cuda.stream(stream):
        g.replay()
    ms_step = max_ranks(time_graph(g)) / n
    ops = sum(2 * M * l.N * l.K for l in layers)
    res = {"workload": f"{PREFILL}: M={M}, qkv 2560->3840, gate_up 2560->13824, down 6912->2560, "
                       "Laplace(0,0.02) weights", "ms_per_step": round(ms_step, 4),
           "TOPS_step": round(ops / (ms_step * 1e-3) / 1e12, 1), "layers": []}
    del g
    gemm_ops, gemm_ms = 0, 0.0
    for li, l in enumerate(layers):
        p, D = pk[li]
        # GEMM inputs (prepared codes in a workspace, packed weights) and outputs
        # rotate over copies, and so do ActQuant's x and workspace, so that
        # every call reads its inputs from HBM.
        rg = rotation(M * l.K + l.N * l.K // 4 + 4 * M * l.N)
        with torch.cuda.stream(stream):
            gitems = []
            for _ in range(rg):
                wsc = torch.zeros_like(wss[li])
                B.prepare_act(xs[li], wsc)
                gitems.append((p.clone(), D.clone(), wsc, torch.empty_like(ys[li])))
            rq = rotation(5 * M * l.K)
            qitems = [(xs[li].clone(), torch.zeros_like(wss[li])) for _ in range(rq)]
        torch.cuda.synchronize(dev)

        def gemm(i, l=l, gitems=gitems):
            pp, DD, wsc, yy = gitems[i % len(gitems)]
            B.forward_prepared(M, l.K, pp, DD, wsc, out=yy)

        def quant(i, qitems=qitems):
            xx, wsc = qitems[i % len(qitems)]
            B.prepare_act(xx, wsc)

        gg = capture(gemm, n)
        with torch.cuda.stream(stream):
            gg.replay()
        tg = max_ranks(time_graph(gg)) / n
        gq = capture(quant, n)
        with torch.cuda.stream(stream):
            gq.replay()
        tq = max_ranks(time_graph(gq)) / n
        o = 2 * M * l.N * l.K
        y_bytes = 4 * M * l.N
        x_bytes = M * l.K + 8 * M  # int8 codes + s_x + row sums read
        w_bytes = l.N * l.K // 4 + 4 * l.N
        t_mem = (y_bytes + x_bytes + w_bytes) / (hbm_peak * 1e9)
        t_cmp = o / (i8_burst * 1e12)
        tops = o / (tg * 1e-3) / 1e12
        q_bytes = 4 * M * l.K + M * l.K + 8 * M
        res["layers"].append({
            "layer": l.name, "K": l.K, "N": l.N, "gemm_us": round(tg * 1e3, 2), "TOPS": round(tops, 1),
            "frac_int8_peak": round(tops / i8_burst, 4),
            "frac_true_roofline": round(max(t_mem, t_cmp) / (tg * 1e-3), 4),
            "actquant_us": round(tq * 1e3, 2), "actquant_GBps": round(q_bytes / (tq * 1e-3) / 1e9, 1),
            "actquant_frac_hbm": round(q_bytes / (tq * 1e-3) / 1e9 / hbm_peak, 4),
            "l2": f"GEMM rotates over {rg} copies, ActQuant over {rq}"})
        gemm_ops += o
        gemm_ms += tg
        del gg, gq, gitems, qitems
    tops = gemm_ops / (gemm_ms * 1e-3) / 1e12
    res["roofline"] = {"bound": "tensor", "kernel": "gemm_kernel (tcgen05 kind::i8, TMEM A + TMEM accumulators)",
                       "achieved": round(tops, 1), "peak": round(i8_burst, 1), "unit": "TOPS",
                       "frac": round(tops / i8_burst, 4), "traffic": load_traffic("gemm_kernel"),
                       "peak_source": "measured bf16 burst x 2 (nominal int8/bf16 ratio)",
                       "frac_of_sustained_peak": round(tops / i8_sust, 4)}
    return res


def bench_configs(B, torch, dev, stream, capture, time_graph, max_ranks, hbm_peak, i8_burst, rank):
    """Every other configuration, one BitLinear call at a time (public forward: fused decode kernel
    for M <= 16, ActQuant + tensor-core GEMM above), against its true roofline
    max(algorithmic bytes / HBM peak, ops / int8 peak). Inputs rotate over enough copies to exceed
    the 126 MB L2."""
    cases = [("decode_2560", 1), ("siglip_m256", 256), ("prefill_sweep", 512), ("prefill_sweep", 2048),
             ("embed_batch", 32768)]
    out = []
    for key, M in cases:
        wl = WL.WORKLOADS[key]
        for li, l in enumerate(wl.layers):
            nbytes = l.N * l.K // 4 + 4 * l.N + 4 * M * l.K + 4 * M * l.N
            rot = int(min(128, max(1, -(-(256 << 20) // nbytes))))
            with torch.cuda.stream(stream):
                W = torch.from_numpy(WL.weight(l.N, l.K, wl.w_dist, wl.seed + 7 * rank, layer=li)).to(dev)
                p, D = B.pack_weights(W)
                del W
                x0 = torch.from_numpy(WL.activations(M, l.K, wl.x_dist, wl.seed, layer=li, meta=wl.meta)).to(dev)
                items = [(p.clone(), D.clone(), x0.clone(), torch.empty((M, l.N), dtype=torch.float32, device=dev))
                         for _ in range(rot)]
                del p, D, x0
                ws = torch.zeros(max(256, B.workspace_size(M, l.N, l.K)), dtype=torch.uint8, device=dev)
            torch.cuda.synchronize(dev)
            n = max(rot, 20)

            def call(i, items=items, ws=ws):
                pp, DD, xx, yy = items[i % len(items)]
                B.forward(xx, pp, DD, out=yy, ws=ws)

            with torch.cuda.stream(stream):
                for i in range(3):
                    call(i)
            torch.cuda.synchronize(dev)
            g = capture(call, n)
            with torch.cuda.stream(stream):
                g.replay()
            t = max_ranks(time_graph(g)) / n * 1e-3  # seconds per call
            ops = 2 * M * l.N * l.K
            t_mem, t_cmp = nbytes / (hbm_peak * 1e9), ops / (i8_burst * 1e12)
            out.append({"config": key, "layer": l.name, "M": M, "K": l.K, "N": l.N, "us": round(t * 1e6, 2),
                        "GB/s": round(nbytes / t / 1e9, 1), "TOPS": round(ops / t / 1e12, 1),
                        "bound": "hbm" if t_mem > t_cmp else "tensor",
                        "frac_true_roofline": round(max(t_mem, t_cmp) / t, 4),
                        "path": "fused decode kernel" if M <= 16 else "ActQuant + tcgen05 GEMM",
                        "l2": f"rotates over {rot} copies"})
            del g, items, ws
            torch.cuda.empty_cache()
    return out


def bench_bf16(B, torch, dev, stream, capture, time_graph, max_ranks, hbm_peak, rank):
    """bf16 inputs (bf16 master weights, bf16 activations; fp32 outputs), each against the HBM
    roofline with bf16 bytes counted at 2 per element."""
    out = {}
    wl = WL.WORKLOADS[HEADLINE]
    layers = list(wl.layers)
    rot = 16
    with torch.cuda.stream(stream):
        base = []
        for li, l in enumerate(layers):
            W = torch.from_numpy(WL.weight(l.N, l.K, wl.w_dist, wl.seed + 17 * rank, layer=li)).to(dev)
            base.append(B.pack_weights(W.to(torch.bfloat16)))
            del W
        packs = [[(p.clone(), D.clone()) for (p, D) in base] for _ in range(rot)]
        xs = [[torch.from_numpy(WL.activations(1, l.K, wl.x_dist, wl.seed + r, layer=li, meta=wl.meta)).to(dev)
               .to(torch.bfloat16) for li, l in enumerate(layers)] for r in range(rot)]
        ys = [torch.empty((1, l.N), dtype=torch.float32, device=dev) for l in layers]
        wss = [torch.zeros(max(256, B.workspace_size(1, l.N, l.K)), dtype=torch.uint8, device=dev) for l in layers]
    torch.cuda.synchronize(dev)

    def step(i):
        r = i % rot
        for li in range(len(layers)):
            p, D = packs[r][li]
            B.forward(xs[r][li], p, D, out=ys[li], ws=wss[li])

    with torch.cuda.stream(stream):
        for i in range(3):
            step(i)
    torch.cuda.synchronize(dev)
    n = 64
    g = capture(step, n)
    with torch.cuda.stream(stream):
        g.replay()
    t = max_ranks(time_graph(g)) / n * 1e-3
    nbytes = sum(l.N * l.K // 4 + 4 * l.N + 2 * l.K + 4 * l.N for l in layers)
    out["decode_layer_set"] = {"us_per_step": round(t * 1e6, 2), "GB/s": round(nbytes / t / 1e9, 1),
                               "frac_hbm": round(nbytes / t / 1e9 / hbm_peak, 4),
                               "note": "four dependent bitlinear_forward_bf16 launches per step, M=1, "
                                       f"weights rotating over {rot} copies"}
    del g, packs, xs
    M = PREFILL_M
    aq = []
    for K in (2560, 6912):
        qb = 2 * M * K + M * K + 12 * M
        r = rotation(qb)
        with torch.cuda.stream(stream):
            xb0 = torch.from_numpy(WL.activations(M, K, "normal", 3, layer=K)).to(dev).to(torch.bfloat16)
            xbs = [xb0.clone() for _ in range(r)]
            del xb0
        torch.cuda.synchronize(dev)
        g = capture(lambda i, xbs=xbs: B.quant_act(xbs[i % len(xbs)]), 32)
        with torch.cuda.stream(stream):
            g.replay()
        t = max_ranks(time_graph(g)) / 32 * 1e-3
        aq.append({"M": M, "K": K, "us": round(t * 1e6, 2), "GB/s": round(qb / t / 1e9, 1),
                   "frac_hbm": round(qb / t / 1e9 / hbm_peak, 4), "l2": f"rotates over {r} copies"})
        del g, xbs
    out["actquant"] = aq
    l = layers[2]
    with torch.cuda.stream(stream):
        Wb0 = torch.from_numpy(WL.weight(l.N, l.K, "normal", 5)).to(dev).to(torch.bfloat16)
        Wbs = [Wb0.clone() for _ in range(4)]  # 4 x 71 MB: each call's W was last read 212 MB earlier
        del Wb0
        ws = torch.zeros(B._lib.lib().bitlinear_pack_workspace_size(1, 16), dtype=torch.uint8, device=dev)
        B.pack_weights(Wbs[0], ws=ws)
        torch.cuda.synchronize(dev)
        ts = []
        for it in range(8):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            B.pack_weights(Wbs[(it + 1) % len(Wbs)], ws=ws)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            ts.append(e0.elapsed_time(e1))
    t = statistics.median(ts) * 1e-3
    alg = 2 * l.N * l.K + l.N * l.K // 4 + 4 * l.N
    out["pack"] = {"layer": f"gate_up {l.K}->{l.N}", "ms": round(t * 1e3, 4),
                   "GB/s_algorithmic": round(alg / t / 1e9, 1), "frac_hbm": round(alg / t / 1e9 / hbm_peak, 4),
                   "l2": "rotates over 4 weight copies"}
    del Wbs
    torch.cuda.empty_cache()
    return out


def bench_block_scale(B, torch, dev, stream, capture, time_graph, max_ranks, hbm_peak, i8_burst, rank):
    """The per-256-block scale variant (D [N, ceil(K/256)]): the decode layer set at M=1, the
    forward kernel's streaming rate on 16 stacked gate_up weights, a prefill-sized call on the
    CUDA-core path, and the per-block pack. Bytes per call: NK/4 packed + 4*N*nb scales + 4MK x
    + 4MN y."""
    out = {}
    wl = WL.WORKLOADS[HEADLINE]
    layers = list(wl.layers)
    rot = 16

    def nbytes(l, M):
        nb = (l.K + 255) // 256
        return l.N * l.K // 4 + 4 * l.N * nb + 4 * M * l.K + 4 * M * l.N

    with torch.cuda.stream(stream):
        base = []
        for li, l in enumerate(layers):
            W = torch.from_numpy(WL.weight(l.N, l.K, wl.w_dist, wl.seed + 17 * rank, layer=li)).to(dev)
            base.append(B.pack_weights_blocks(W))
            del W
        packs = [[(p.clone(), D.clone()) for (p, D) in base] for _ in range(rot)]
        xs = [[torch.from_numpy(WL.activations(1, l.K, wl.x_dist, wl.seed + r, layer=li, meta=wl.meta)).to(dev)
               for li, l in enumerate(layers)] for r in range(rot)]
        ys = [torch.empty((1, l.N), dtype=torch.float32, device=dev) for l in layers]
        wss = [torch.zeros(max(256, B.blocks_workspace_size(1, l.N, l.K)), dtype=torch.uint8, device=dev)
               for l in layers]
    torch.cuda.synchronize(dev)

    def step(i):
        r = i % rot
        for li in range(len(layers)):
            p, D = packs[r][li]
            B.forward_blocks(xs[r][li], p, D, out=ys[li], ws=wss[li])

    with torch.cuda.stream(stream):
        for i in range(3):
            step(i)
    torch.cuda.synchronize(dev)
    n = 64
    g = capture(step, n)
    with torch.cuda.stream(stream):
        g.replay()
    t = max_ranks(time_graph(g)) / n * 1e-3
    tot = sum(nbytes(l, 1) for l in layers)
    out["decode_layer_set"] = {"us_per_step": round(t * 1e6, 2), "GB/s": round(tot / t / 1e9, 1),
                               "frac_hbm": round(tot / t / 1e9 / hbm_peak, 4), "bytes_per_step": tot,
                               "note": "four bitlinear_forward_blocks calls per step (at M=1 one launch each: the "
                                       f"quantiser runs in every CTA), M=1, weights rotating over {rot} copies"}
    del g, packs, xs, base
    torch.cuda.empty_cache()

    # Streaming rate: one call over 16 stacked gate_up weights (141.6 MB packed).
    l = layers[2]
    Nst = 16 * l.N
    with torch.cuda.stream(stream):
        W1 = torch.from_numpy(WL.weight(l.N, l.K, wl.w_dist, wl.seed, layer=2)).to(dev)
        p1, D1 = B.pack_weights_blocks(W1)
        del W1
        pst, Dst = p1.repeat(16, 1).contiguous(), D1.repeat(16, 1).contiguous()
        copies = 2
        pk = [(pst.clone(), Dst.clone()) for _ in range(copies)]
        del pst, Dst
        x1 = torch.from_numpy(WL.activations(1, l.K, wl.x_dist, wl.seed, layer=2, meta=wl.meta)).to(dev)
        y1 = torch.empty((1, Nst), dtype=torch.float32, device=dev)
        ws1 = torch.zeros(max(256, B.blocks_workspace_size(1, Nst, l.K)), dtype=torch.uint8, device=dev)
    torch.cuda.synchronize(dev)
    g = capture(lambda i: B.forward_blocks(x1, pk[i % copies][0], pk[i % copies][1], out=y1, ws=ws1), 16)
    with torch.cuda.stream(stream):
        g.replay()
    t = max_ranks(time_graph(g)) / 16 * 1e-3
    sb = Nst * l.K // 4 + 4 * Nst * ((l.K + 255) // 256) + 4 * l.K + 4 * Nst
    out["streaming_m1"] = {"rows": Nst, "K": l.K, "us": round(t * 1e6, 2), "GB/s": round(sb / t / 1e9, 1),
                           "frac_hbm": round(sb / t / 1e9 / hbm_peak, 4),
                           "note": f"16 stacked gate_up weights, {copies} copies alternating (each 150 MB)"}
    del g, pk
    torch.cuda.empty_cache()

    # Prefill sizes: gate_up at M=512 and 4096 (one tensor-core GEMM per 256-column block).
    pre = []
    for M in (512, 4096):
        with torch.cuda.stream(stream):
            W1 = torch.from_numpy(WL.weight(l.N, l.K, "laplace", 9)).to(dev)
            pp, DD = B.pack_weights_blocks(W1)
            del W1
            xp = torch.from_numpy(WL.activations(M, l.K, "normal", 9)).to(dev)
            yp = torch.empty((M, l.N), dtype=torch.float32, device=dev)
            wsp = torch.zeros(max(256, B.blocks_workspace_size(M, l.N, l.K)), dtype=torch.uint8, device=dev)
        torch.cuda.synchronize(dev)
        g = capture(lambda i: B.forward_blocks(xp, pp, DD, out=yp, ws=wsp), 8)
        with torch.cuda.stream(stream):
            g.replay()
        t = max_ranks(time_graph(g)) / 8 * 1e-3
        ops = 2.0 * M * l.N * l.K
        nbk = (l.K + 255) // 256
        alg = 4 * M * l.K + l.N * l.K // 4 + 4 * l.N * nbk + 4 * M * l.N
        true_t = max(alg / (hbm_peak * 1e9), ops / (i8_burst * 1e12))
        pre.append({"M": M, "us": round(t * 1e6, 2), "TOPS": round(ops / t / 1e12, 2),
                    "frac_int8_peak": round(ops / t / 1e12 / i8_burst, 4),
                    "frac_true_roofline": round(true_t / t, 4)})
        del g, pp, DD, xp, yp, wsp
        torch.cuda.empty_cache()
    out["prefill_gate_up"] = {"cases": pre,
                              "note": "ActQuant, per-block row sums of the codes, then one tcgen05 GEMM per "
                                      f"256-column block ({(l.K + 255) // 256} launches), each epilogue adding "
                                      "its block's term to y (TMA reduce-add); the same input each call"}

    # Per-block pack of gate_up (offline).
    with torch.cuda.stream(stream):
        W0 = torch.from_numpy(WL.weight(l.N, l.K, "normal", 5)).to(dev)
        Ws = [W0.clone() for _ in range(4)]
        del W0
        ws = torch.zeros(B._lib.lib().bitlinear_pack_workspace_size(1, 16), dtype=torch.uint8, device=dev)
        B.pack_weights_blocks(Ws[0], ws=ws)
        torch.cuda.synchronize(dev)
        ts = []
        for it in range(8):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            B.pack_weights_blocks(Ws[(it + 1) % len(Ws)], ws=ws)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            ts.append(e0.elapsed_time(e1))
    t = statistics.median(ts) * 1e-3
    alg = 4 * l.N * l.K + l.N * l.K // 4 + 4 * l.N * ((l.K + 255) // 256)
    out["pack"] = {"layer": f"gate_up {l.K}->{l.N}", "ms": round(t * 1e3, 4),
                   "GB/s_algorithmic": round(alg / t / 1e9, 1), "frac_hbm": round(alg / t / 1e9 / hbm_peak, 4),
                   "note": "synchronous call (includes the status read-back); W rotates over 4 copies"}
    del Ws
    torch.cuda.empty_cache()
    return out


def bench_rmsnorm(B, torch, dev, stream, capture, time_graph, max_ranks, hbm_peak, i8_burst):
    """Fused per-projection RMSNorm + ActQuant (the embedding models of C5 normalise the input of
    every projection) against HBM: 4MK + 4K read, MK + 8M written. Also the forward with the
    fused norm on the first C5 layer, against its true roofline."""
    out = {"actquant": []}
    for (M, K) in ((32768, 1024), (32768, 3072), (4096, 2560), (4096, 6912)):
        nb = 4 * M * K + 4 * K + M * K + 12 * M
        r = rotation(nb)
        with torch.cuda.stream(stream):
            x0 = torch.from_numpy(WL.activations(M, K, "outlier_tokens", 7, layer=K,
                                                 meta={"frac": 0.01, "scale": 20.0, "df": 3.0})).to(dev)
            xs_r = [x0.clone() for _ in range(r)]
            del x0
            g = torch.from_numpy(WL.weight(1, K, "normal", 8).reshape(-1) + np.float32(1.0)).to(dev)
        torch.cuda.synchronize(dev)
        nrep = 16
        g_ = capture(lambda i, xs_r=xs_r, g=g: B.rmsnorm_quant_act(xs_r[i % len(xs_r)], g), nrep)
        with torch.cuda.stream(stream):
            g_.replay()
        t = max_ranks(time_graph(g_)) / nrep * 1e-3
        out["actquant"].append({"M": M, "K": K, "us": round(t * 1e6, 2), "GB/s": round(nb / t / 1e9, 1),
                                "frac_hbm": round(nb / t / 1e9 / hbm_peak, 4), "l2": f"rotates over {r} copies"})
        del g_, xs_r, g
    wl = WL.WORKLOADS["embed_batch"]
    l = wl.layers[2]  # 3072 -> 1024, compute-bound
    M = 32768
    with torch.cuda.stream(stream):
        W = torch.from_numpy(WL.weight(l.N, l.K, wl.w_dist, wl.seed, layer=2)).to(dev)
        p, D = B.pack_weights(W)
        del W
        x = torch.from_numpy(WL.activations(M, l.K, wl.x_dist, wl.seed, layer=2, meta=wl.meta)).to(dev)
        g = torch.from_numpy(WL.weight(1, l.K, "normal", 9).reshape(-1) + np.float32(1.0)).to(dev)
        y = torch.empty((M, l.N), dtype=torch.float32, device=dev)
        ws = torch.zeros(B.workspace_size(M, l.N, l.K), dtype=torch.uint8, device=dev)
    torch.cuda.synchronize(dev)
    gg = capture(lambda i: B.forward_rmsnorm(x, g, p, D, out=y, ws=ws), 10)
    with torch.cuda.stream(stream):
        gg.replay()
    t = max_ranks(time_graph(gg)) / 10 * 1e-3
    ops = 2 * M * l.N * l.K
    nb = 4 * M * l.K + 4 * l.K + l.N * l.K // 4 + 4 * l.N + 4 * M * l.N
    out["forward"] = {"layer": f"embed_batch {l.name} {l.K}->{l.N}, M={M}", "us": round(t * 1e6, 2),
                      "TOPS": round(ops / t / 1e12, 1),
                      "frac_true_roofline": round(max(nb / (hbm_peak * 1e9), ops / (i8_burst * 1e12)) / t, 4)}
    del gg, x, y, ws
    torch.cuda.empty_cache()
    # The decode layer set (M=1) with a norm before every projection: four
    # bitlinear_forward_rmsnorm calls per step, each one decode launch that
    # normalises and quantises x in every CTA. Bytes per layer: the BitLinear's
    # plus 4K of norm weight.
    dl = WL.WORKLOADS[HEADLINE]
    layers = list(dl.layers)
    rot = 16
    with torch.cuda.stream(stream):
        base = []
        for li, lay in enumerate(layers):
            W = torch.from_numpy(WL.weight(lay.N, lay.K, dl.w_dist, dl.seed, layer=li)).to(dev)
            base.append(B.pack_weights(W))
            del W
        packs = [[(pp.clone(), DD.clone()) for (pp, DD) in base] for _ in range(rot)]
        gs = [torch.from_numpy(WL.weight(1, lay.K, "normal", 30 + li).reshape(-1) + np.float32(1.0)).to(dev)
              for li, lay in enumerate(layers)]
        xs = [[torch.from_numpy(WL.activations(1, lay.K, dl.x_dist, dl.seed + r, layer=li, meta=dl.meta)).to(dev)
               for li, lay in enumerate(layers)] for r in range(rot)]
        ys = [torch.empty((1, lay.N), dtype=torch.float32, device=dev) for lay in layers]
        wss = [torch.zeros(max(256, B.workspace_size(1, lay.N, lay.K)), dtype=torch.uint8, device=dev)
               for lay in layers]
    torch.cuda.synchronize(dev)

    def step(i):
        r = i % rot
        for li in range(len(layers)):
            pp, DD = packs[r][li]
            B.forward_rmsnorm(xs[r][li], gs[li], pp, DD, out=ys[li], ws=wss[li])

    with torch.cuda.stream(stream):
        for i in range(3):
            step(i)
    torch.cuda.synchronize(dev)
    n = 64
    gd = capture(step, n)
    with torch.cuda.stream(stream):
        gd.replay()
    t = max_ranks(time_graph(gd)) / n * 1e-3
    tot = sum(lay.N * lay.K // 4 + 4 * lay.N + 4 * lay.K + 4 * lay.N + 4 * lay.K for lay in layers)
    out["decode_layer_set"] = {"us_per_step": round(t * 1e6, 2), "GB/s": round(tot / t / 1e9, 1),
                               "frac_hbm": round(tot / t / 1e9 / hbm_peak, 4),
                               "note": "four bitlinear_forward_rmsnorm calls per step (M=1, one decode launch "
                                       f"each, norm + ActQuant in every CTA), weights rotating over {rot} copies"}
    del gd, packs, xs
    torch.cuda.empty_cache()
    return out


def bench_decode_stream(B, torch, dev, stream, capture, time_graph, max_ranks, hbm_peak, copies=16):
    """The decode kernel's streaming ceiling: one call over `copies` stacked
    gate_up weights (2560 -> 13824 x copies, 141 MB packed), so launch and
    dependency latency are small against the weight stream. Two weight copies
    alternate, so every call reads its weights from HBM."""
    l = WL.WORKLOADS[HEADLINE].layers[2]
    with torch.cuda.stream(stream):
        W = torch.from_numpy(WL.weight(l.N, l.K, "normal", 11)).to(dev)
        p1, D1 = B.pack_weights(W)
        del W
        items = [(p1.repeat(copies, 1).contiguous(), D1.repeat(copies, 1).contiguous()) for _ in range(2)]
        del p1, D1
    N, K = items[0][0].shape[0], l.K
    out = {"weights": f"{copies} x gate_up stacked: [{N}, {K}], {N * K // 4 / 1e6:.1f} MB packed", "cases": []}
    for M in (1, 8):
        with torch.cuda.stream(stream):
            x = torch.from_numpy(WL.activations(M, K, "normal", 12)).to(dev)
            y = torch.empty((M, N), dtype=torch.float32, device=dev)
            ws = torch.zeros(max(256, B.workspace_size(M, N, K)), dtype=torch.uint8, device=dev)
        torch.cuda.synchronize(dev)
        nrep = 20
        g = capture(lambda i, x=x, y=y, ws=ws: B.forward(x, items[i % 2][0], items[i % 2][1], out=y, ws=ws), nrep)
        with torch.cuda.stream(stream):
            g.replay()
        t = max_ranks(time_graph(g)) / nrep * 1e-3
        nb = N * K // 4 + 4 * N + 4 * M * K + 4 * M * N
        out["cases"].append({"M": M, "us": round(t * 1e6, 2), "GB/s": round(nb / t / 1e9, 1),
                             "frac_hbm": round(nb / t / 1e9 / hbm_peak, 4)})
        del g, x, y, ws
    del items
    torch.cuda.empty_cache()
    return out


def bench_pack(B, torch, dev, stream, hbm_peak):
    l = WL.WORKLOADS[HEADLINE].layers[2]  # gate_up, the largest weight
    with torch.cuda.stream(stream):
        W0 = torch.from_numpy(WL.weight(l.N, l.K, "normal", 5)).to(dev)
        Ws = [W0, W0.clone()]  # 2 x 142 MB: each call's W was last read 283 MB earlier
        ws = torch.zeros(B._lib.lib().bitlinear_pack_workspace_size(1, 16), dtype=torch.uint8, device=dev)
        B.pack_weights(Ws[0], ws=ws)
        torch.cuda.synchronize(dev)
        ts = []
        for it in range(6):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            B.pack_weights(Ws[(it + 1) % 2], ws=ws)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            ts.append(e0.elapsed_time(e1))
        t = statistics.median(ts)
        # Asynchronous packs back to back (the pack's own kernels), one status read after them.
        ws_a = B.pack_workspace(dev)
        outs = [(torch.empty((l.N, l.K // 16), dtype=torch.int32, device=dev),
                 torch.empty((l.N, 1), dtype=torch.float32, device=dev)) for _ in range(2)]
        L = B._lib.lib()

        def pack_async(i):
            W = Ws[i % 2]
            p, D = outs[i % 2]
            B._lib.call("bitlinear_pack_weights_async", W.data_ptr(), l.N, l.K, p.data_ptr(), D.data_ptr(),
                        ws_a.data_ptr(), ws_a.numel(), stream.cuda_stream)

        for i in range(3):
            pack_async(i)
        torch.cuda.synchronize(dev)
        reps = 10
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(reps):
            pack_async(i + 1)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        t_async = e0.elapsed_time(e1) / reps
        st = L.bitlinear_pack_status(ws_a.data_ptr(), ws_a.numel(), stream.cuda_stream)
    alg = 4 * l.N * l.K + l.N * l.K // 4 + 4 * l.N
    return {"layer": f"gate_up {l.K}->{l.N}", "ms": round(t_async, 4),
            "GB/s_algorithmic": round(alg / (t_async * 1e-3) / 1e9, 1),
            "frac_hbm": round(alg / (t_async * 1e-3) / 1e9 / hbm_peak, 4),
            "sync_call_ms": round(t, 4), "sync_call_GB/s": round(alg / (t * 1e-3) / 1e9, 1),
            "status_after": int(st),
            "note": "ms / GB/s: bitlinear_pack_weights_async calls back to back (fp64 pass with the mean decided "
                    "in its last CTA, then ternarise+pack from the end of W), one status read after them; "
                    "sync_call: the synchronous call (status read-back and host wake-up included); "
                    "W rotates over 2 copies (283 MB)"}


def bench_i2s(B, torch, dev, stream, hbm_peak, copies=16, reps=10, layouts=("consecutive", "quarters")):
    """I2_S export and import of a stack of `copies` gate_up weights (larger
    than L2, so every call streams from HBM), both byte groupings: `reps`
    asynchronous conversions back to back between two events (one status
    check after them), and the synchronous call for comparison."""
    l = WL.WORKLOADS[HEADLINE].layers[2]
    with torch.cuda.stream(stream):
        W = torch.from_numpy(WL.weight(l.N, l.K, "normal", 6)).to(dev)
        p1, D1 = B.pack_weights(W)
        del W
        packed = p1.repeat(copies, 1).contiguous()
        D = D1.repeat(copies, 1).contiguous()
        del p1, D1
        N, K = packed.shape[0], packed.shape[1] * 16
        buf = torch.empty(B.i2s_bytes(N, K), dtype=torch.uint8, device=dev)
        p_in = torch.empty_like(packed)
        D_in = torch.empty_like(D)
        ws = B.i2s_workspace(dev)
        torch.cuda.synchronize(dev)
        alg = N * K // 2 + 4 * N + 4  # packed words + I2_S blocks + D + scale
        out = {"tensor": f"{copies} x gate_up stacked: [{N}, {K}]", "bytes_each_way": N * K // 4,
               "algorithmic_bytes_per_call": alg}
        for layout in layouts:
            calls = {
                "export": lambda sync: B.i2s_export(packed, D, layout, out=buf, ws=ws, sync=sync),
                "import": lambda sync: B.i2s_import(buf, N, K, layout, out=(p_in, D_in), ws=ws, sync=sync),
            }
            res = {}
            for name, fn in calls.items():
                for _ in range(3):
                    fn(False)
                torch.cuda.synchronize(dev)
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                for _ in range(reps):
                    fn(False)
                e1.record(stream)
                torch.cuda.synchronize(dev)
                if B.i2s_status(ws) != 0:
                    raise RuntimeError("I2_S conversion reported a format error")
                t = e0.elapsed_time(e1) / reps
                ts = []
                for _ in range(3):
                    f0 = torch.cuda.Event(enable_timing=True)
                    f1 = torch.cuda.Event(enable_timing=True)
                    f0.record(stream)
                    fn(True)
                    f1.record(stream)
                    torch.cuda.synchronize(dev)
                    ts.append(f0.elapsed_time(f1))
                res[name] = {"us": round(t * 1e3, 2), "GB/s_algorithmic": round(alg / (t * 1e-3) / 1e9, 1),
                             "frac_hbm": round(alg / (t * 1e-3) / 1e9 / hbm_peak, 4),
                             "sync_call_us": round(statistics.median(ts) * 1e3, 2)}
            out[layout] = res
        assert torch.equal(p_in, packed)
    out["note"] = ("us / GB/s: asynchronous calls back to back (one kernel each), one status check after them; "
                   "sync_call_us: the synchronous call (status clear, kernel, status read, host wake-up)")
    return out


def run_prefill_small(a, B, torch, dev):
    """Bounded case for profiler captures: one layer of one workload (default: the prefill
    gate_up layer, 2560->13824, at M=4096)."""
    key, li, M = PREFILL, 1, PREFILL_M
    if a.ncu_layer:
        k, i, m = a.ncu_layer.split(":")
        key, li, M = k, int(i), int(m)
    wl = WL.WORKLOADS[key]
    l = wl.layers[li]
    W = torch.from_numpy(WL.weight(l.N, l.K, wl.w_dist, wl.seed, layer=li)).to(dev)
    p, D = B.pack_weights(W)
    del W
    x = torch.from_numpy(WL.activations(M, l.K, wl.x_dist, wl.seed, layer=li, meta=wl.meta)).to(dev)
    y = torch.empty((M, l.N), dtype=torch.float32, device=dev)
    ws = torch.zeros(B.workspace_size(M, l.N, l.K), dtype=torch.uint8, device=dev)
    g = torch.ones(l.K, dtype=torch.float32, device=dev)
    for _ in range(a.warmup + a.steps):
        if a.ncu_rms:
            B.forward_rmsnorm(x, g, p, D, out=y, ws=ws)
        else:
            B.forward(x, p, D, out=y, ws=ws)
    torch.cuda.synchronize(dev)
    assert B.workspace_error(ws) == 0
    print(json.dumps({"prefill_small": "ok", "rmsnorm": bool(a.ncu_rms), "M": M, "K": l.K, "N": l.N,
                      "calls": a.warmup + a.steps}))
    return 0


def main(argv=None):
    a = parse_args(argv)
    if a.impl == "reference":
        return run_reference(a)
    return run_ours(a)


if __name__ == "__main__":
    sys.exit(main())
