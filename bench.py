#!/usr/bin/env python
"""Benchmark of the W4.4A8 linear layer (MixLLM) on B200.

One step = one pass of the hot path over one batch: activation quantization
(fp16 X -> int8 A_q + fp32 s_a) followed by the fused W4.4A8 GEMM (both
channel sets in one launch, fp16 Y scattered by channel index).  The weights
are quantized and packed once before timing (an offline step).

Default workload: Llama-3.1-8B q_proj shape, M=512 tokens, N=K=4096, 410 of
4096 output channels 8-bit (p10), group 128 -- synthetic seeded inputs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  Under torchrun (N > 1) every rank runs its own
batch with replicated weights (data parallel, no collective on the data path);
the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from mixed_precision_quantized_act_b200 import dist as dp  # noqa: E402
from mixed_precision_quantized_act_b200 import workloads as wl  # noqa: E402

METRIC = "W4.4A8 GEMM effective TOPS at M=512,N=K=4096; % of B200 int8 TC peak"
UNIT = "TOPS"
NOMINAL_INT8_OVER_BF16 = 4.5 / 2.25  # dense tensor peaks, ops per bf16 flop
GEMM_SRC = os.path.join(ROOT, "mixed_precision_quantized_act_b200", "csrc", "gemm_w4w8a8.cuh")
# ncu DRAM traffic per launch of the dominant kernel, per workload: a single
# entry or {"entries": [...]}, used while its source hash matches the CUDA sources
TRAFFIC_FILES = [os.path.join(ROOT, "profiles", f) for f in ("gemm_w4w8a8_traffic.json", "gemv_w4w8a8_traffic.json")]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=wl.Q_PROJ_P10.name)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--i2f", choices=["bias", "plain"], default="bias",
                    help="tiled GEMM's int32->float step: the 0x4b400000 bias trick (the method) or, as the "
                         "ablation of the fast-I2F design point, a plain convert per element (same Y)")
    ap.add_argument("--step", choices=["split", "fused"], default="split",
                    help="M > 64: split = quantize_act, then the GEMM as its programmatic dependent "
                         "(mixllm_linear's form); fused = one launch of the tiled GEMM that quantizes X "
                         "itself (mixllm_linear_one_launch); each line also times the other form")
    ap.add_argument("--dry-run", action="store_true",
                    help="argument and rank plumbing only (gloo on CPU, no kernels): rank 0 prints the "
                         "configuration, every rank's batch seed and the max over ranks of a stand-in time")
    return ap.parse_args()


def layer_for(name):
    try:
        return wl.by_name(name)
    except KeyError:
        raise SystemExit(f"unknown workload {name}")


# Few-token (decode) steps read a few MB of weights: instead of a flush, the
# timed steps cycle over enough copies of the packed weights to exceed L2
# twice over, as the layers of a decoder do, and run as one CUDA graph (the
# host cannot issue eager launches as fast as the device runs them).
ROTATE_BYTES = 300 * 1024 * 1024


def config_of(layer, n_gpus, rotate=0):
    l2 = (f"inputs larger than L2: {rotate} copies of the packed weights, step i uses copy i mod {rotate}"
          if rotate else "flushed by a 256 MiB device write before every timed step")
    return {"workload": layer.name, "M": layer.M, "N": layer.N, "K": layer.K, "N8": layer.N8,
            "N4": layer.N4, "group": 128, "l2": l2,
            "parallelism": f"dp{n_gpus} (weights replicated, M tokens per GPU)"}


def source_hash(files=None):
    """sha256 (16 hex digits) of CUDA sources of the library, in the order
    given (default: every file of csrc/, sorted)."""
    d = os.path.dirname(GEMM_SRC)
    h = hashlib.sha256()
    for f in files if files is not None else sorted(os.listdir(d)):
        with open(os.path.join(d, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except OSError:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, index, period_s=0.002):
        self.index, self.period = index, period_s
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self.ok = False

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        except Exception:
            self.ok = False
        return self

    def _run(self):
        nv, h = self._nv, self._h
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                for name, bit in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __exit__(self, *exc):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": len(self.samples), "source": "nvml unavailable"}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples), "source": "nvml, 2 ms period"}


# ------------------------------------------------------------------ oracle leg

def _oracle_rows_worker(name, seed, r0, target_s, sub_cols, start, out_q):
    """One host core's share of the oracle baseline: quantize + two-step GEMM
    on token rows r0, r0+1, ... (cycling over the batch) until about
    `target_s` seconds; puts (rows, seconds) on out_q."""
    import oracle
    layer = wl.by_name(name)
    X, W, is8 = wl.make_x(layer, seed), wl.make_w(layer, seed), wl.make_bitmap(layer, seed)
    if sub_cols is not None:
        W, is8 = W[:sub_cols], is8[:sub_cols]
    Wq = oracle.Quantized(W, is8)  # offline weight quantization, not timed
    A, s = oracle.quantize_act(X[r0:r0 + 1])  # warm-up and calibration row
    t0 = time.perf_counter()
    oracle.gemm_w4w8a8(A, s, Wq)
    per_row = max(time.perf_counter() - t0, 1e-6)
    rows = int(max(1, target_s / per_row))
    start.wait()  # every process has quantized its weights and calibrated
    done, r, t0 = 0, r0, time.perf_counter()
    while done < rows:
        r = r % layer.M
        n = min(rows - done, layer.M - r)
        A, s = oracle.quantize_act(X[r:r + n])
        oracle.gemm_w4w8a8(A, s, Wq)
        done += n
        r += n
    out_q.put((done, time.perf_counter() - t0))


def oracle_rate(layer, seed, target_s, cores=None, sub_cols=None):
    """Time the CPU oracle (quantize + two-step GEMM, unmodified) on the
    box's host cores: one spawned process per core, each on its own token
    rows of the workload, started together; returns (TOPS-equivalent over all
    rows / the slowest process's time, seconds, rows, cores).  Spawned, not
    forked: the parent may already hold a CUDA context."""
    import multiprocessing as mp
    cores = cores or os.cpu_count() or 1
    ctx = mp.get_context("spawn")
    start, out_q = ctx.Barrier(cores), ctx.Queue()
    procs = [ctx.Process(target=_oracle_rows_worker,
                         args=(layer.name, seed, (i * layer.M) // cores, target_s, sub_cols, start, out_q))
             for i in range(cores)]
    for pr in procs:
        pr.start()
    res = [out_q.get() for _ in procs]
    for pr in procs:
        pr.join()
    rows = sum(r for r, _ in res)
    secs = max(t for _, t in res)
    n = min(layer.N, sub_cols) if sub_cols else layer.N
    return 2.0 * rows * n * layer.K / secs / 1e12, secs, rows, cores


# ------------------------------------------------------------------ reference arm

def run_reference(args, layer, rank, world):
    """The oracle as it stands, on the machine's host cores, rank 0 only."""
    if rank != 0:
        return
    import oracle
    X, W, is8 = wl.make_x(layer, args.seed), wl.make_w(layer, args.seed), wl.make_bitmap(layer, args.seed)
    # one step = one token row of the workload through quantize + two-step GEMM,
    # restricted to the layer's first 512 output channels (a bounded sample)
    sub_cols = np.arange(min(layer.N, 512))
    Wq_s = oracle.Quantized(W[sub_cols], is8[sub_cols])
    ops_per_step = 2.0 * 1 * len(sub_cols) * layer.K
    for i in range(args.warmup):
        A, s = oracle.quantize_act(X[i % layer.M: i % layer.M + 1])
        oracle.gemm_w4w8a8(A, s, Wq_s)
    t0 = time.perf_counter()
    for i in range(args.steps):
        A, s = oracle.quantize_act(X[i % layer.M: i % layer.M + 1])
        oracle.gemm_w4w8a8(A, s, Wq_s)
    dt = time.perf_counter() - t0
    value = ops_per_step * args.steps / dt / 1e12
    sample = f"per step: 1 token row x {len(sub_cols)} output channels x K={layer.K} (quantize + two-step GEMM)"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": "synthetic", "config": config_of(layer, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "host_cores": os.cpu_count(), "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ our arm

def run_ours(args, layer, rank, world, local_rank):
    import torch
    import mixed_precision_quantized_act_b200 as mx

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    mx.load()
    stream = torch.cuda.current_stream()

    X = wl.make_x(layer, dp.batch_seed(args.seed, rank))
    W, is8 = wl.make_w(layer, args.seed), wl.make_bitmap(layer, args.seed)
    Xd = torch.from_numpy(X).to(dev)
    p = mx.pack_weights(torch.from_numpy(W).to(dev), torch.from_numpy(is8).to(dev))
    A_q = torch.empty((layer.M, layer.K), dtype=torch.int8, device=dev)
    s_a = torch.empty((layer.M, layer.K // 128), dtype=torch.float32, device=dev)
    Y = torch.empty((layer.M, layer.N), dtype=torch.float16, device=dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)

    # few tokens (decode): the split-K path with its workspace; otherwise the tiled kernel
    small = layer.M <= mx.SMALL_M_MAX
    other = None  # the tiled line's timing of the other M > 64 form
    copies = [p]
    if small:
        ws = mx.small_m_workspace(layer.M, p, dev)
        ncopy = max(2, -(-ROTATE_BYTES // p.nbytes()))
        copies += [mx.PackedLinear(**{k: (v.clone() if isinstance(v, torch.Tensor) else v) for k, v in vars(p).items()})
                   for _ in range(ncopy - 1)]

        def gemm(i=0):
            mx.gemm_w4w8a8_small_m_into(A_q, s_a, copies[i % len(copies)], Y, ws, stream)
    elif args.i2f == "plain":
        def gemm(i=0):
            mx.gemm_w4w8a8_plain_i2f_into(A_q, s_a, p, Y, stream)
    else:
        def gemm(i=0):
            mx.gemm_w4w8a8_into(A_q, s_a, p, Y, stream)

    def split_step(i=0):
        mx.quantize_act_into(Xd, A_q, s_a, stream)
        gemm(i)

    # M > 64: the tiled GEMM that quantizes X itself (one launch) when asked
    # for; the line times the other form too (not with the plain-convert ablation)
    one_ok = not small and args.i2f != "plain" and layer.G % 4 == 0
    fused = one_ok and args.step == "fused"
    if one_ok:
        ws_lin = mx.linear_workspace(layer.M, p, dev)

        def one_step(i=0):
            mx.linear_into(Xd, p, Y, ws_lin, stream, one_launch=True)

        for _ in range(3):
            one_step()
    step = one_step if fused else split_step

    for i in range(max(args.warmup, 3)):
        if not small:
            flush.fill_(1)
        step(i)
    mx.sync_status(stream)

    K = args.steps
    if small:
        # Timed region: one graph of exactly K steps (the GEMM of each is a
        # programmatic dependent of its quantizer), then one of Kk GEMMs alone
        # for the per-kernel duration (its launch gaps included).
        def captured(fn, n):
            g = torch.cuda.CUDAGraph()
            side = torch.cuda.Stream(device=dev)
            side.wait_stream(torch.cuda.current_stream(dev))
            with torch.cuda.stream(side):
                fn(0)  # warm the library's cached descriptors on the capturing stream
            torch.cuda.current_stream(dev).wait_stream(side)
            with torch.cuda.graph(g, stream=side):
                for i in range(n):
                    fn(i)
            return g

        def graph_step(i):
            mx.quantize_act_into(Xd, A_q, s_a, None)
            mx.gemm_w4w8a8_small_m_into(A_q, s_a, copies[i % len(copies)], Y, ws, None)

        def graph_gemm(i):
            mx.gemm_w4w8a8_small_m_into(A_q, s_a, copies[i % len(copies)], Y, ws, None)

        g_steps = captured(graph_step, K)
        g_steps.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        with ClockSampler(local_rank) as clocks:
            e0.record(stream)
            g_steps.replay()
            e1.record(stream)
            torch.cuda.synchronize()
        barrier(world)
        mx.sync_status(stream)
        t_step = max_over_ranks(e0.elapsed_time(e1) / K, world)
        del g_steps

        Kk = min(K, 500)
        g_gemm = captured(graph_gemm, Kk)
        g_gemm.replay()
        g_q = captured(lambda i: mx.quantize_act_into(Xd, A_q, s_a, None), Kk)
        g_q.replay()
        torch.cuda.synchronize()
        e2, e3, e4 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        e2.record(stream)
        g_gemm.replay()
        e3.record(stream)
        g_q.replay()
        e4.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        mx.sync_status(stream)
        t_gemm = max_over_ranks(e2.elapsed_time(e3) / Kk, world)
        t_quant = max_over_ranks(e3.elapsed_time(e4) / Kk, world)
        del g_gemm, g_q
        gemm_timed = f"{Kk} launches in one CUDA graph on rotating weight copies (launch gaps included)"
    else:
        # Timed region: whole steps.  The GEMM is launched as a programmatic
        # dependent of the quantizer, so nothing is recorded between the two.
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
        barrier(world)
        torch.cuda.synchronize()
        with ClockSampler(local_rank) as clocks:
            for i in range(K):
                flush.fill_(i & 0xFF)
                ev[i][0].record(stream)
                step()
                ev[i][1].record(stream)
            torch.cuda.synchronize()
        barrier(world)
        mx.sync_status(stream)
        t_step = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in ev) / K, world)

        # Per-kernel durations for the roofline: the split form's two kernels
        # with an event between them (which also keeps the GEMM from starting
        # early, so this is its stand-alone duration), and the split step as
        # the timed region runs it.
        Kk = min(K, 500)
        ek = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(Kk)]
        torch.cuda.synchronize()
        for i in range(Kk):
            flush.fill_(i & 0xFF)
            ek[i][0].record(stream)
            mx.quantize_act_into(Xd, A_q, s_a, stream)
            ek[i][1].record(stream)
            gemm()
            ek[i][2].record(stream)
        torch.cuda.synchronize()
        barrier(world)
        mx.sync_status(stream)
        t_gemm = max_over_ranks(sum(e[1].elapsed_time(e[2]) for e in ek) / Kk, world)
        t_quant = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in ek) / Kk, world)
        gemm_timed = f"{Kk} launches with an event before and after each, L2 flushed before each"
        if one_ok and not fused:
            eo = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(Kk)]
            torch.cuda.synchronize()
            for i in range(Kk):
                flush.fill_(i & 0xFF)
                eo[i][0].record(stream)
                one_step()
                eo[i][1].record(stream)
            torch.cuda.synchronize()
            barrier(world)
            mx.sync_status(stream)
            t_one = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in eo) / Kk, world)
            other = {"one_launch_step": {
                "ms": t_one, "tops": layer.ops() / (t_one * 1e-3) / 1e12,
                "timed": f"{Kk} launches of the GEMM that quantizes X itself (mixllm_linear_one_launch), "
                         "L2 flushed before each"}}
        if fused:
            # the fused step is one kernel: the timed steps are its launches
            t_split_gemm = t_gemm
            es = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(Kk)]
            torch.cuda.synchronize()
            for i in range(Kk):
                flush.fill_(i & 0xFF)
                es[i][0].record(stream)
                split_step()
                es[i][1].record(stream)
            torch.cuda.synchronize()
            barrier(world)
            mx.sync_status(stream)
            t_split = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in es) / Kk, world)
            other = {"split_step": {"step_ms": t_split, "step_tops": layer.ops() / (t_split * 1e-3) / 1e12,
                     "gemm_ms": t_split_gemm, "quantize_act_ms": t_quant,
                     "timed": f"{Kk} split steps (quantize_act, then the GEMM as its programmatic dependent), "
                              "L2 flushed before each; the two kernels apart as in quantize_act_kernel"}}
            t_gemm = t_step
            gemm_timed = (f"the timed steps: {K} launches of the GEMM that quantizes X itself, an event "
                          "before and after each, L2 flushed before each")

    # end to end through the public API: pinned host X in, host Y out
    Xh = torch.from_numpy(X).pin_memory()
    Yh = torch.empty((layer.M, layer.N), dtype=torch.float16).pin_memory()
    Ke = min(K, 200)
    ee = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(Ke)]
    for _ in range(3):
        Xd.copy_(Xh, non_blocking=True)
        step()
        Yh.copy_(Y, non_blocking=True)
    barrier(world)
    torch.cuda.synchronize()
    for i in range(Ke):
        if not small:
            flush.fill_(i & 0xFF)
        ee[i][0].record(stream)
        Xd.copy_(Xh, non_blocking=True)
        step(i)
        Yh.copy_(Y, non_blocking=True)
        ee[i][1].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    t_e2e_serial = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in ee) / Ke, world)

    # The same end-to-end steps pipelined as a server runs them: step i's
    # input copy (its own stream), compute (the library's two launches) and
    # output copy (a third stream) overlap the neighbouring steps' through
    # two device and two pinned host slots, ordered by events.  Every step
    # still moves its own X in and its own Y out.  No flush can sit between
    # overlapped steps, so the steps cycle over copies of the packed weights
    # larger than L2 together (the tiled path) instead.
    nslot = 2
    Xhs = [Xh] + [torch.from_numpy(X).pin_memory() for _ in range(nslot - 1)]
    Yhs = [Yh] + [torch.empty_like(Yh).pin_memory() for _ in range(nslot - 1)]
    Xds = [Xd] + [torch.empty_like(Xd) for _ in range(nslot - 1)]
    Yds = [Y] + [torch.empty_like(Y) for _ in range(nslot - 1)]
    wsets = copies if small else [p] + [
        mx.PackedLinear(**{k: (v.clone() if isinstance(v, torch.Tensor) else v) for k, v in vars(p).items()})
        for _ in range(max(1, -(-ROTATE_BYTES // p.nbytes())) - 1)]
    h2d, d2h = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    x_ready = [torch.cuda.Event() for _ in range(nslot)]
    x_free = [torch.cuda.Event() for _ in range(nslot)]
    y_ready = [torch.cuda.Event() for _ in range(nslot)]
    y_free = [torch.cuda.Event() for _ in range(nslot)]

    def pipelined(n):
        for i in range(n):
            b = i % nslot
            with torch.cuda.stream(h2d):
                if i >= nslot:
                    h2d.wait_event(x_free[b])
                Xds[b].copy_(Xhs[b], non_blocking=True)
                x_ready[b].record(h2d)
            stream.wait_event(x_ready[b])
            if i >= nslot:
                stream.wait_event(y_free[b])
            if fused:
                mx.linear_into(Xds[b], wsets[i % len(wsets)], Yds[b], ws_lin, stream, one_launch=True)
            elif small:
                mx.quantize_act_into(Xds[b], A_q, s_a, stream)
                mx.gemm_w4w8a8_small_m_into(A_q, s_a, wsets[i % len(wsets)], Yds[b], ws, stream)
            else:
                mx.quantize_act_into(Xds[b], A_q, s_a, stream)
                (mx.gemm_w4w8a8_plain_i2f_into if args.i2f == "plain" else mx.gemm_w4w8a8_into)(
                    A_q, s_a, wsets[i % len(wsets)], Yds[b], stream)
            x_free[b].record(stream)
            y_ready[b].record(stream)
            with torch.cuda.stream(d2h):
                d2h.wait_event(y_ready[b])
                Yhs[b].copy_(Yds[b], non_blocking=True)
                y_free[b].record(d2h)

    pipelined(max(args.warmup, 3))
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    p0.record(h2d)
    pipelined(Ke)
    d2h.wait_stream(h2d)
    d2h.wait_stream(stream)
    p1.record(d2h)
    torch.cuda.synchronize()
    barrier(world)
    mx.sync_status(stream)
    t_e2e = max_over_ranks(p0.elapsed_time(p1) / Ke, world)

    ops = layer.ops()
    value = ops * world / (t_step * 1e-3) / 1e12
    gemm_tops = ops / (t_gemm * 1e-3) / 1e12
    peaks, peak_src = measured_peaks()
    int8_peak = peaks["bf16_tflops"] * NOMINAL_INT8_OVER_BF16
    traffic = None
    for path in TRAFFIC_FILES:
        try:
            with open(path) as f:
                tr = json.load(f)
        except (OSError, ValueError):
            continue
        for e in tr.get("entries", [tr]):
            try:
                current = source_hash(e.get("sources"))
            except OSError:
                continue
            if e.get("source_hash") == current and e.get("workload") == layer.name:
                traffic = e.get("dram_bytes_per_launch")

    if small:  # HBM-bound: the packed weights are nearly all the bytes
        gemm_gbs = layer.algorithmic_bytes() / (t_gemm * 1e-3) / 1e9
        roofline = {"bound": "hbm", "achieved": gemm_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": gemm_gbs / peaks["hbm_gbs"], "traffic": traffic,
                    "peak_source": f"{peak_src} HBM copy {peaks['hbm_gbs']} GB/s",
                    "algorithmic_bytes": layer.algorithmic_bytes()}
    else:
        roofline = {"bound": "tensor", "achieved": gemm_tops, "peak": int8_peak, "unit": "TOPS",
                    "frac": gemm_tops / int8_peak, "traffic": traffic,
                    "peak_source": f"{peak_src} bf16 burst {peaks['bf16_tflops']} TFLOP/s x 2 (nominal int8/bf16)",
                    "algorithmic_bytes": layer.algorithmic_bytes()}

    line = None
    if rank == 0:
        cpu = None
        if world == 1:
            rate, secs, rows, cores = oracle_rate(layer, args.seed, args.cpu_seconds)
            cpu = {"value": rate, "unit": UNIT, "cores": cores, "host_cores": os.cpu_count(), "kind": "oracle",
                   "sample": f"{rows} token rows (cycling over the {layer.M}-row batch) x all {layer.N} "
                             f"channels x K={layer.K}, quantize + two-step GEMM, one process per host core "
                             f"on its own rows, {secs:.1f} s (slowest process)"}
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": t_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int8", "data": "synthetic (seeded N(0,1) X with x20 outlier "
            "columns, N(0,0.02) W, random 8-bit channel set)",
            "config": dict(config_of(layer, world, len(copies) if small else 0),
                           **({"i2f": "plain int->float convert (ablation)"} if args.i2f == "plain" and not small else {})),
            "gemm_kernel": {"path": mx.small_m_kernel(layer.M, layer.K, p.N4, p.N8) if small else
                            ("tiled, quantizing X itself" if fused else "tiled"),
                            "ms": t_gemm, "tops": gemm_tops,
                            "frac_of_int8_peak": gemm_tops / int8_peak,
                            "frac_of_nominal_4500": gemm_tops / 4500.0,
                            "timed": gemm_timed},
            "quantize_act_kernel": {"ms": t_quant,
                                    "gbs": (layer.M * layer.K * 3 + layer.M * layer.G * 4) / (t_quant * 1e-3) / 1e9,
                                    **({"note": "stand-alone quantizer of the split form, not in the fused step"}
                                       if fused else {})},
            **(other or {}),
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": {"value": ops * world / (t_e2e * 1e-3) / 1e12, "unit": UNIT,
                    "h2d_bytes_per_step": layer.M * layer.K * 2, "d2h_bytes_per_step": layer.M * layer.N * 2,
                    "ms_per_step": t_e2e,
                    "timed": f"{Ke} steps pipelined: X in on one copy stream, "
                             f"{'the fused GEMM' if fused else 'quantize + GEMM'}, Y out on "
                             f"another, two slots; weights cycled over {len(wsets)} copies",
                    "serial": {"value": ops * world / (t_e2e_serial * 1e-3) / 1e12, "ms_per_step": t_e2e_serial,
                               "timed": "copy in, compute, copy out on one stream, L2 flushed before each step"}},
            "gpu_launches": K if fused else 2 * K,
            "step": ("one launch of the fused GEMM that quantizes X itself: every CTA quantizes an even "
                     "share of the (token, group) pairs into the workspace, then loads A_q and s_a once "
                     "all shares are counted in (mixllm_linear)") if fused else
                    ("quantize_act then the fused GEMM, launched as its programmatic dependent (its "
                     "prologue overlaps the quantizer's tail; it reads A_q and s_a only after the quantizer ends)"
                     + ("; M <= 8 runs the GEMV, 9 <= M <= 64 the few-token tensor-core kernel (both split-K)"
                        if small else "")),
            "clocks": clocks.summary(),
        }
    return line


def barrier(world):
    dp.barrier(world)


def max_over_ranks(x, world):
    return dp.max_over_ranks(x, world, device="cuda")


LAYER_WORKLOAD = "llama3.1-8b_layer"  # the four linears of one decoder layer, "@M<m>" picks M


def run_layer(args, rank, world, local_rank):
    """The decoder layer's four linears (qkv, o_proj, gate_up, down), each as
    quantize + GEMM (or, for one token, the GEMV quantizing its own input).
    M > 64: one CUDA graph per step, L2 flushed before each step outside the
    graph.  M <= 64: the K steps as one CUDA graph over weight sets larger
    than L2 together.  Reports TOPS over the four GEMMs."""
    import torch
    import mixed_precision_quantized_act_b200 as mx
    from mixed_precision_quantized_act_b200.layer import LinearChain

    M = int(args.workload.split("@M")[1]) if "@M" in args.workload else 512
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    mx.load()
    layers = [l.with_m(M) for l in wl.LLAMA8B_LAYER]
    packed = [mx.pack_weights(torch.from_numpy(wl.make_w(l, args.seed)).to(dev),
                              torch.from_numpy(wl.make_bitmap(l, args.seed)).to(dev)) for l in layers]
    stream = torch.cuda.current_stream()
    K = args.steps
    if M <= mx.SMALL_M_MAX:
        # decode: rotate over weight sets larger than L2 together, K steps as one CUDA graph
        wbytes = sum(p.nbytes() for p in packed)
        ncopy = max(2, -(-ROTATE_BYTES // wbytes))
        sets = [packed] + [[mx.PackedLinear(**{k: (v.clone() if isinstance(v, torch.Tensor) else v)
                                               for k, v in vars(p).items()}) for p in packed]
                           for _ in range(ncopy - 1)]
        chains = [LinearChain(ps, M, dev) for ps in sets]
        for c in chains:
            for l, x in zip(layers, c.inputs):
                x.copy_(torch.from_numpy(wl.make_x(l, dp.batch_seed(args.seed, rank))))
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            for i in range(max(args.warmup, 3)):
                chains[i % ncopy].run()
        stream.wait_stream(side)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            for i in range(K):
                chains[i % ncopy].run()
        g.replay()
        mx.sync_status(stream)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        with ClockSampler(local_rank) as clocks:
            e0.record(stream)
            g.replay()
            e1.record(stream)
            torch.cuda.synchronize()
        barrier(world)
        mx.sync_status(stream)
        t_step = max_over_ranks(e0.elapsed_time(e1) / K, world)
        del g
        chain = chains[0]
        l2 = f"inputs larger than L2: {ncopy} sets of the layer's packed weights, step i uses set i mod {ncopy}"
    else:
        chain = LinearChain(packed, M, dev)
        for l, x in zip(layers, chain.inputs):
            x.copy_(torch.from_numpy(wl.make_x(l, dp.batch_seed(args.seed, rank))))
        chain.capture()
        flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
        for _ in range(max(args.warmup, 3)):
            flush.fill_(1)
            chain.replay()
        mx.sync_status(stream)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
        barrier(world)
        torch.cuda.synchronize()
        with ClockSampler(local_rank) as clocks:
            for i in range(K):
                flush.fill_(i & 0xFF)
                ev[i][0].record(stream)
                chain.replay()
                ev[i][1].record(stream)
            torch.cuda.synchronize()
        barrier(world)
        mx.sync_status(stream)
        t_step = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in ev) / K, world)
        l2 = "flushed by a 256 MiB device write before every timed step"
    chain.release()
    ops = chain.ops()
    if rank != 0:
        return None
    return {
        "metric": "W4.4A8 decoder-layer linears (qkv, o_proj, gate_up, down) effective TOPS",
        "value": ops * world / (t_step * 1e-3) / 1e12, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": t_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8",
        "data": "synthetic (seeded N(0,1) X with x20 outlier columns, N(0,0.02) W, random 8-bit channel sets)",
        "config": {"workload": f"{LAYER_WORKLOAD}@M{M}", "M": M, "linears": [l.name.split("_M")[0] for l in layers],
                   "l2": l2,
                   "parallelism": f"dp{world} (weights replicated, M tokens per GPU)"},
        "step": f"{chain.launches()} kernels (each linear: quantize_act + the GEMM, or for one token the GEMV "
                "quantizing its own activations) replayed as one CUDA graph",
        "gpu_launches": chain.launches() * K,
        "clocks": clocks.summary(),
    }


SEARCH_WORKLOAD = "llama3.1-8b_search_q_gate_D16"  # global salience search over two layers' channels


def run_search(args, rank, world, local_rank):
    """The global mixed-precision search (salience of every output channel,
    then the global top 10 %) over a q_proj-shaped (4096 x 4096) and a
    gate_proj-shaped (14336 x 4096) layer with 16 synthetic gradient samples
    per channel: 4.8 GB of gradients, larger than L2, so no flush."""
    import numpy as np
    import torch
    import mixed_precision_quantized_act_b200 as mx
    from mixed_precision_quantized_act_b200 import _lib

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    mx.load()
    D, K = 16, 4096
    Ns = [4096, 14336]
    gen = torch.Generator(device=dev)
    gen.manual_seed(args.seed * 1000 + rank)
    Ws = [torch.randn(N, K, device=dev, generator=gen) * 0.02 for N in Ns]
    Gs = [torch.randn(D, N, K, device=dev, generator=gen) for N in Ns]
    n_all = sum(Ns)
    T = n_all // 10
    S = torch.empty(n_all, dtype=torch.float32, device=dev)
    is8 = torch.empty(n_all, dtype=torch.uint8, device=dev)
    ws = _lib.select_top_t_workspace(n_all, dev)
    stream = torch.cuda.current_stream()
    offs = [0, Ns[0]]

    def salience():
        for W, G, o, N in zip(Ws, Gs, offs, Ns):
            _lib.channel_salience_into(W, G, S[o:o + N], stream)

    def step():
        salience()
        _lib.select_top_t_into(S, T, is8, ws, stream)

    for _ in range(max(args.warmup, 3)):
        step()
    mx.sync_status(stream)
    Kst = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(Kst)]
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clocks:
        for i in range(Kst):
            ev[i][0].record(stream)
            salience()
            ev[i][1].record(stream)
            _lib.select_top_t_into(S, T, is8, ws, stream)
            ev[i][2].record(stream)
        torch.cuda.synchronize()
    barrier(world)
    mx.sync_status(stream)
    t_step = max_over_ranks(sum(e[0].elapsed_time(e[2]) for e in ev) / Kst, world)
    t_sal = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in ev) / Kst, world)
    t_sel = max_over_ranks(sum(e[1].elapsed_time(e[2]) for e in ev) / Kst, world)
    sal_bytes = sum(D * N * K * 4 + N * K * 4 + N * 4 for N in Ns)
    step_bytes = sal_bytes + n_all * (6 * 4 + 1)  # + the selection: six passes over the scores, the bit map

    # end to end: gradients from pinned host memory every step, the bit map back
    Gh = [G.cpu().pin_memory() for G in Gs]
    is8_h = torch.empty(n_all, dtype=torch.uint8).pin_memory()
    Ke = min(Kst, 3)
    ee = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(Ke)]
    torch.cuda.synchronize()
    for i in range(Ke):
        ee[i][0].record(stream)
        for G, h in zip(Gs, Gh):
            G.copy_(h, non_blocking=True)
        step()
        is8_h.copy_(is8, non_blocking=True)
        ee[i][1].record(stream)
    torch.cuda.synchronize()
    t_e2e = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in ee) / Ke, world)

    if rank != 0:
        return None
    # the oracle on a sample of channels of the first layer
    rows = 512
    Wn = Ws[0][:rows].cpu().numpy()
    Gn = Gs[0][:, :rows].cpu().numpy()
    t0 = time.perf_counter()
    import oracle
    oracle.channel_salience(Wn, Gn)
    secs = time.perf_counter() - t0
    cpu_gbs = (D * rows * K * 4 + rows * K * 4) / secs / 1e9
    peaks, peak_src = measured_peaks()
    gbs = step_bytes * world / (t_step * 1e-3) / 1e9
    sal_gbs = sal_bytes / (t_sal * 1e-3) / 1e9
    return {
        "metric": "global salience search (channel salience of two layers + global top 10 %), bytes moved per second",
        "value": gbs, "unit": "GB/s", "n_gpus": world, "steps": Kst, "warmup": args.warmup,
        "ms_per_step": t_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded N(0,0.02) W, N(0,1) per-sample gradients)",
        "config": {"workload": SEARCH_WORKLOAD, "layers": [[N, K] for N in Ns], "samples": D, "T": T,
                   "l2": "inputs larger than L2 (4.8 GB of gradients)", "parallelism": f"dp{world}"},
        "salience_kernels": {"ms": t_sal, "gbs": sal_gbs}, "select_kernels": {"ms": t_sel},
        "roofline": {"bound": "hbm", "achieved": sal_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": sal_gbs / peaks["hbm_gbs"], "traffic": None,
                     "peak_source": f"{peak_src} HBM copy {peaks['hbm_gbs']} GB/s", "algorithmic_bytes": sal_bytes},
        "cpu_baseline": {"value": cpu_gbs, "unit": "GB/s", "cores": 1, "host_cores": os.cpu_count(), "kind": "oracle",
                         "sample": f"{rows} channels of the 4096 x 4096 layer x {D} samples, fp64, {secs:.2f} s"},
        "e2e": {"value": step_bytes / (t_e2e * 1e-3) / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": sum(G.numel() * 4 for G in Gs), "d2h_bytes_per_step": n_all},
        "gpu_launches": 14 * Kst,
        "step": "2 x channel_salience_kernel, then the radix select (init, 4 x (histogram + pick), count, scan, mark)",
        "clocks": clocks.summary(),
    }


def run_dry(args, rank, world):
    """The launch plumbing of a multi-GPU run without a GPU: the process group
    (gloo), each rank's batch seed, the barrier and the max over ranks of a
    per-rank time, and the whole-job unit count, as the timed runs use them."""
    import torch.distributed as tdist
    dp.init("gloo", timeout_s=60)
    try:
        name = args.workload
        if name.startswith(LAYER_WORKLOAD) or name == SEARCH_WORKLOAD:
            config, m = {"workload": name, "parallelism": f"dp{world}"}, None
        else:
            layer = layer_for(name)
            config, m = config_of(layer, world), layer.M
        seed = dp.batch_seed(args.seed, rank)
        seeds = [None] * world
        if world > 1:
            tdist.all_gather_object(seeds, seed)
        else:
            seeds = [seed]
        dp.barrier(world)
        tmax = dp.max_over_ranks(1.0 + 0.25 * rank, world)  # stand-in per-rank time (ms)
        if rank == 0:
            print(json.dumps({"dry_run": True, "impl": args.impl, "n_gpus": args.gpus, "world": world,
                              "steps": args.steps, "warmup": args.warmup, "config": config, "seeds": seeds,
                              "ms_per_step_max_over_ranks": tmax,
                              "units": dp.total_units(m, world) if m is not None else None}), flush=True)
    finally:
        dp.shutdown(world)


def main():
    args = parse()
    if args.dry_run:
        run_dry(args, int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")))
        return
    if args.workload == SEARCH_WORKLOAD:
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the search workload has no reference arm; "
                              "its cpu_baseline is the oracle on a channel sample"}), flush=True)
            return
        line = run_search(args, int(os.environ.get("RANK", "0")), 1, int(os.environ.get("LOCAL_RANK", "0")))
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.workload.startswith(LAYER_WORKLOAD):
        if args.impl == "reference":
            if rank == 0:
                print(json.dumps({"impl": "reference", "unavailable": "the decoder-layer workload has no "
                                  "CPU reference arm; use a single-linear workload"}), flush=True)
            return
        if world > 1:
            import torch
            torch.cuda.set_device(local_rank)
            dp.init("nccl", timeout_s=120, device=torch.device("cuda", local_rank))
        try:
            line = run_layer(args, rank, world, local_rank)
            if line is not None:
                print(json.dumps(line), flush=True)
        finally:
            dp.shutdown(world)
        return
    layer = layer_for(args.workload)
    if args.impl == "reference":
        run_reference(args, layer, rank, world)
        return
    if world > 1:
        import torch
        torch.cuda.set_device(local_rank)
        dp.init("nccl", timeout_s=120, device=torch.device("cuda", local_rank))
    try:
        line = run_ours(args, layer, rank, world, local_rank)
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        dp.shutdown(world)


if __name__ == "__main__":
    main()
