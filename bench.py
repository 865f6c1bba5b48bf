#!/usr/bin/env python
"""Benchmark of the Attn-QAT training attention step (forward + backward) on B200.

One step = attnqat_fwd + attnqat_bwd over one batch of the pages' shape:
B=1, H=6, Lq=Lk=31200, D=128, bf16, all four quantizers on, sm_scale=1/sqrt(128)
(the 6-head, 31200-token shape the fastvideo-kernel commit times).  The step
runs every kernel of the path: the three operand quantizers, the forward, the
Delta kernel, the kernel writing the fp16 copy of dO, the dK/dV kernel and the
dQ kernel.

Metric: nominal TFLOP/s of fwd+bwd (forward 4*B*H*Lq*Lk*D, backward 2.5x that),
also reported as fwd / bwd / fwd+bwd milliseconds and as a fraction of the
measured B200 BF16 tensor peak.  Inputs are seeded synthetic tensors; L2 is
flushed (a 256 MiB write) between timed steps, each step is timed with CUDA
events on the launching stream, and multi-GPU runs report the max over ranks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                  [--workload NAME] [--flags F] [--sparsity S | --causal]

--workload times another of the seeded workloads (tiny, outlier_channels_4096,
wan_6h_31200, scaled_heads_16384, large_40h_75600) and --flags another set of
quantizers (bits q=1, k=2, v=4, p=8; default all four).

--sparsity S times the block-sparse (VSA fine attention) step instead (with
--tile 64 the tile-64 profile: 64-token query and key blocks):
attnqat_vsa_select (the top max(1, min(ceil((1-S)*nk), nk)) of the nk key
tiles per 128-query tile by coarse tile-mean scores; the pages' VSA checkpoint
uses S = 0.9) + attnqat_sparse_fwd + attnqat_sparse_bwd on the same shape,
with TFLOP/s counted on the selected tiles only.

--causal times the causal step (ATTNQAT_CAUSAL on attnqat_fwd / attnqat_bwd,
query i attending keys j <= i) on the same shape, with TFLOP/s counted on the
unmasked (query, key) pairs, L(L+1)/2 per head.

The end-to-end leg ("e2e") runs the same step through the public API with the
inputs in pinned host memory: every step copies Q, K, V, dO to the device and
O, LSE, m, dQ, dK, dV back, on two copy streams, double-buffered so that one
step's copies overlap the neighbouring steps' kernels.

--impl reference times the float64 CPU oracle on the host cores instead (the
pages ship no runnable implementation): each step is a bounded sample of the
same workload, one head with the first query rows against all keys.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from quantization_aware_attention_nvfp4_b200 import workloads as W  # noqa: E402

WORKLOAD = "wan_6h_31200"
METRIC = "Attn-QAT fwd+bwd ms & TFLOP/s at H6 L31200 D128; % of B200 BF16 peak"
SPARSE_METRIC = ("Block-sparse (VSA) Attn-QAT fwd+bwd ms & TFLOP/s on the selected tiles at %s, "
                 "sparsity %g")
CAUSAL_METRIC = "Causal Attn-QAT fwd+bwd ms & TFLOP/s on the unmasked pairs at %s"
OTHER_METRIC = "Attn-QAT fwd+bwd ms & TFLOP/s at {}; % of B200 BF16 peak"
FLAG_NAMES = ((1, "q"), (2, "k"), (4, "v"), (8, "p"))
# nominal dense tensor rates of B200 per input type, relative to bf16/fp16
# (2.25 PFLOP/s bf16, 9 PFLOP/s fp4): the dK/dV kernel's S unit runs on the
# block-scaled NVFP4 pipe when Q and K are quantized
NVFP4_RATE_RATIO = 4.0
# query rows (= keys) of the oracle's causal sample: its cost grows with the
# square of the prefix, like the dense sample's rows x all keys
CAUSAL_SAMPLE_ROWS = int(os.environ.get("ATTNQAT_CAUSAL_BASELINE_ROWS", "15360"))
DATASHEET_BF16_TFLOPS = 2250.0
FALLBACK_PEAKS = dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0)
# rows of the oracle's bounded samples (query rows of head 0 against all keys):
# the CPU-baseline leg of the GPU run (~10-30 s on the machine's host cores) and
# each step of --impl reference
BASELINE_SAMPLE_ROWS = int(os.environ.get("ATTNQAT_BASELINE_ROWS", "6144"))
ORACLE_SAMPLE_ROWS = int(os.environ.get("ATTNQAT_ORACLE_SAMPLE_ROWS", "1024"))


def shape_name(w):
    return "B%d H%d L%d%s D%d" % (w.B, w.H, w.Lq, "" if w.Lq == w.Lk else "x%d" % w.Lk, w.D)


def flag_names(flags):
    return ",".join(n for b, n in FLAG_NAMES if flags & b) or "none"


def sample_rows(w, rows):
    """Query rows of an oracle sample with about the work of `rows` rows
    against 31200 keys (the cost of a row grows with Lk)."""
    return max(1, min(w.Lq, int(rows * 31200 / w.Lk)))


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return dict(hbm_gbs=p["hbm_gbs"], bf16_tflops=p["bf16_tflops"],
                    bf16_tflops_sustained=p["bf16_tflops_sustained"], source="measured")
    return dict(FALLBACK_PEAKS, source="fallback")


def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), \
        int(os.environ.get("LOCAL_RANK", "0"))


def max_over_ranks(values, device=None):
    """Element-wise max of per-rank timings over all ranks of the default
    process group (identity when there is none).  Every rank must call it the
    same number of times with the same number of values."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


# ------------------------------------------------------------------ clocks --

class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 50 ms while the
    timed region runs.  Entering waits (up to 10 s) for a first sample and
    leaving waits (up to 2 s) for one more, so even a region shorter than the
    sampling period is bracketed by a sample on each side."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        import threading
        self.lines = []
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return self
        first = threading.Event()

        def reader():
            for line in self.proc.stdout:
                self.lines.append(line)
                first.set()
            first.set()
        self.thread = threading.Thread(target=reader, daemon=True)
        self.thread.start()
        first.wait(10.0)
        del self.lines[:-1]  # keep only the latest sample before the region
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            n0 = len(self.lines)
            t0 = time.perf_counter()
            while len(self.lines) <= n0 and time.perf_counter() - t0 < 2.0 and self.proc.poll() is None:
                time.sleep(0.01)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=10)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.proc.wait()
            self.thread.join(timeout=10)
            self.out = "".join(self.lines)
        return False

    def summary(self):
        if self.proc is None or not getattr(self, "out", ""):
            return dict(sm_mhz=None, sm_max_mhz=None, reasons=["nvidia-smi unavailable"])
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return dict(sm_mhz=None, sm_max_mhz=None, reasons=["no samples"])
        loaded = [x for x in sm if x > 0.5 * max(sm)] or sm
        return dict(sm_mhz=float(statistics.median(loaded)), sm_max_mhz=float(max(smax)),
                    reasons=sorted(reasons), samples=len(sm))


# ----------------------------------------------------------------- GPU arm --

def selected_pairs(w, mask, T=W.SPARSE_TILE):
    """Sum over (b, h) of the (query row, key) pairs the T-token tile mask
    selects."""
    rows = np.minimum(T, w.Lq - T * np.arange(mask.shape[2]))
    keys = np.minimum(T, w.Lk - T * np.arange(mask.shape[3]))
    return float(np.einsum("bhij,i,j->", mask.astype(np.float64), rows, keys))


def dtype_weighted_peak(peak, n_units, fp4_units, ratio=NVFP4_RATE_RATIO):
    """Peak rate of a kernel whose n_units matmul units run fp4_units on the
    NVFP4 pipe (ratio times the bf16 rate) and the rest at the bf16 peak: the
    units over the time floor sum_u (1 / rate_u)."""
    return peak * n_units / ((n_units - fp4_units) + fp4_units / ratio)


def metric_name(args, w):
    if args.sparsity is not None:
        return SPARSE_METRIC % (shape_name(w) + ("" if args.tile == 128 else ", %d-token tiles" % args.tile),
                                args.sparsity)
    if args.causal:
        return CAUSAL_METRIC % shape_name(w)
    if w.name == WORKLOAD and args.flags == 15:
        return METRIC
    return OTHER_METRIC.format(shape_name(w))


def workload_name(args, w):
    name = w.name if args.flags == 15 else "%s_flags%d" % (w.name, args.flags)
    if args.sparsity is not None:
        return ("vsa_" if args.tile == 128 else "vsa%d_" % args.tile) + name
    return ("causal_" if args.causal else "") + name


def gpu_arm(args):
    import torch
    import torch.distributed as dist
    import quantization_aware_attention_nvfp4_b200 as A

    rank, world, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=300))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    w = W.get(args.workload)
    flops = w.nominal_flops()
    peaks = load_peaks()
    sparse = args.sparsity is not None
    causal = bool(args.causal)
    pairs = float(w.B * w.H * w.Lq * w.Lk)
    if causal:
        pairs = float(w.B * w.H) * w.Lq * (w.Lq + 1) / 2.0
        fwd_f = 4.0 * pairs * w.D
        flops = dict(fwd=fwd_f, bwd=2.5 * fwd_f, total=3.5 * fwd_f)
    T = args.tile
    nq, nk = -(-w.Lq // T), -(-w.Lk // T)
    topk = W.topk_tiles(nk, args.sparsity) if sparse else nk

    # seeded inputs (host), moved to the device once; the timed region starts
    # with them resident in HBM
    inp = W.inputs(w)
    host = {n: torch.from_numpy(inp[n].view(np.int16)).view(torch.bfloat16) for n in inp}
    q, k, v, do = (host[n].to(dev) for n in ("q", "k", "v", "do"))
    c = w.sm_scale
    flags = args.flags | (A.CAUSAL if causal else 0)
    if sparse:
        tm = torch.empty((w.B, w.H, nq, nk), dtype=torch.uint8, device=dev)
        sel_ws = torch.empty(A.load().attnqat_vsa_select_tiles_workspace_size(w.B, w.H, w.Lq, w.Lk, w.D, T),
                             dtype=torch.uint8, device=dev)
        ws_bytes = A.attnqat_sparse_workspace_size(w.B, w.H, w.Lq, w.Lk, w.D, flags)

        def fwd(qq, kk, vv, out, stream=None):
            # the selection belongs to the forward: coarse scores, top-k tiles
            A.attnqat_vsa_select(qq, kk, topk, out=tm, ws=sel_ws, stream=stream, tile=T)
            return A.attnqat_sparse_fwd(qq, kk, vv, tm, sm_scale=c, flags=flags, ws=ws, out=out, stream=stream,
                                        tile=T)

        def bwd(qq, kk, vv, ll, mm, dd, out, stream=None):
            return A.attnqat_sparse_bwd(qq, kk, vv, ll, mm, dd, ws, tm, sm_scale=c, flags=flags, out=out, tile=T,
                                        stream=stream)
    else:
        ws_bytes = A.attnqat_workspace_size(w.B, w.H, w.Lq, w.Lk, w.D, flags)

        def fwd(qq, kk, vv, out, stream=None):
            return A.attnqat_fwd(qq, kk, vv, sm_scale=c, flags=flags, ws=ws, out=out, stream=stream)

        def bwd(qq, kk, vv, ll, mm, dd, out, stream=None):
            return A.attnqat_bwd(qq, kk, vv, ll, mm, dd, ws, sm_scale=c, flags=flags, out=out, stream=stream)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.Lq), dtype=torch.float32, device=dev)
    m = torch.empty_like(lse)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        fwd(q, k, v, (o, lse, m))
        bwd(q, k, v, lse, m, do, (dq, dk, dv))

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    A.attnqat_device_status()
    if sparse:
        # the selection depends only on the inputs: count its pairs once
        mask_np = tm.cpu().numpy()
        pairs = selected_pairs(w, mask_np, T)
        fwd_f = 4.0 * pairs * w.D
        flops = dict(fwd=fwd_f, bwd=2.5 * fwd_f, total=3.5 * fwd_f)

    # ---- timed region: K steps, L2 flushed between steps, per-step events
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    A.attnqat_profile_enable(True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index) as clocks:
        wall0 = time.perf_counter()
        for i in range(args.steps):
            flush.zero_()
            e0, e1, e2 = ev[i]
            e0.record(stream)
            fwd(q, k, v, (o, lse, m))
            e1.record(stream)
            bwd(q, k, v, lse, m, do, (dq, dk, dv))
            e2.record(stream)
        torch.cuda.synchronize(dev)
        wall = time.perf_counter() - wall0
    if world > 1:
        dist.barrier()
    kernels = A.attnqat_profile_read(1 << 16)
    A.attnqat_profile_enable(False)
    A.attnqat_device_status()
    fwd_ms = sum(e0.elapsed_time(e1) for e0, e1, _ in ev)
    bwd_ms = sum(e1.elapsed_time(e2) for _, e1, e2 in ev)
    tot_ms = fwd_ms + bwd_ms
    tot_ms, fwd_ms, bwd_ms = max_over_ranks([tot_ms, fwd_ms, bwd_ms], dev)

    # ---- per-kernel durations inside the timed region (dominant kernel)
    per = {}
    for name, ms in kernels:
        per.setdefault(name, []).append(ms)
    units = 2.0 * pairs * w.D  # one matmul unit (over the selected pairs when sparse)
    algo_flops = {"attn_fwd": 2 * units, "attn_bwd_dkdv": 4 * units, "attn_bwd_dq": 1 * units}
    exec_flops = {"attn_fwd": 3 * units, "attn_bwd_dkdv": 4 * units, "attn_bwd_dq": 3 * units}
    tensor_kernels = {n: v for n, v in per.items() if n in algo_flops}
    dom = max(tensor_kernels, key=lambda n: sum(tensor_kernels[n]))
    dom_ms = statistics.mean(per[dom])
    achieved = algo_flops[dom] / (dom_ms * 1e-3) / 1e12
    # the kernels run inside an ~11 ms step, not a seconds-long loop: the
    # burst peak is the denominator
    peak = peaks["bf16_tflops"]
    # dtype-weighted: with Q and K quantized, one of dK/dV's four units (S)
    # runs on the NVFP4 pipe, whose nominal rate is 4x bf16's; the time floor
    # is then 3 units at the bf16 peak plus 1 at 4x it
    fp4_units = {"attn_bwd_dkdv": 1, "attn_fwd": 0, "attn_bwd_dq": 0}[dom] if (args.flags & 3) == 3 else 0
    weighted_peak = dtype_weighted_peak(peak, algo_flops[dom] / units, fp4_units)
    traffic = None if (sparse or causal or w.name != WORKLOAD or args.flags != 15) else load_traffic(dom)
    kernel_table = {n: dict(launches=len(v), mean_ms=round(statistics.mean(v), 4),
                            share=round(sum(v) / sum(sum(x) for x in per.values()), 4))
                    for n, v in per.items()}
    for n in algo_flops:
        if n in kernel_table:
            kernel_table[n]["algorithmic_tflops"] = round(algo_flops[n] / (kernel_table[n]["mean_ms"] * 1e-3) / 1e12, 1)
            kernel_table[n]["executed_tflops"] = round(exec_flops[n] / (kernel_table[n]["mean_ms"] * 1e-3) / 1e12, 1)

    # ---- end to end through the public API with host buffers
    e2e = None if args.no_e2e else e2e_arm(args, torch, dev, host, w, flops, fwd, bwd, world)

    value = world * flops["total"] * args.steps / (tot_ms * 1e-3) / 1e12
    ms_step = tot_ms / args.steps
    config = {"workload": workload_name(args, w), "B": w.B, "H": w.H, "Lq": w.Lq, "Lk": w.Lk, "D": w.D,
              "quantizers": flag_names(args.flags), "sm_scale": "%.6g" % c, "values": w.description,
              "global_batch": w.B * world, "seq_len": w.Lq,
              "parallelism": "replicas x%d (heads independent, no collective)" % world,
              "l2": "flushed between steps (256 MiB write); each step timed with CUDA events"}
    if sparse:
        config.update(sparsity=args.sparsity, tile=T,
                      key_tiles_per_query_tile=int(mask_np.sum(-1).max()),
                      selected_fraction=round(pairs / (w.B * w.H * w.Lq * w.Lk), 5),
                      selection="attnqat_vsa_select in the timed forward (tile means, top-%d coarse scores)" % topk)
    if causal:
        config.update(mask="causal (query i attends keys j <= i)",
                      unmasked_fraction=round(pairs / (w.B * w.H * w.Lq * w.Lk), 5))
    out = {
        "metric": metric_name(args, w),
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) float32 from numpy PCG64, rounded to bf16; %s)" % w.recipe,
        "config": config,
        "fwd_ms": round(fwd_ms / args.steps, 4),
        "bwd_ms": round(bwd_ms / args.steps, 4),
        "fwd_tflops": round(flops["fwd"] / (fwd_ms / args.steps * 1e-3) / 1e12, 1),
        "bwd_tflops": round(flops["bwd"] / (bwd_ms / args.steps * 1e-3) / 1e12, 1),
        "frac_of_bf16_peak": round(value / world / peaks["bf16_tflops"], 4),
        "frac_of_bf16_peak_sustained": round(value / world / peaks["bf16_tflops_sustained"], 4),
        "frac_of_datasheet_2250": round(value / world / DATASHEET_BF16_TFLOPS, 4),
        "peaks": "%s (bf16 %.1f burst / %.1f sustained TFLOP/s)" % (peaks["source"], peaks["bf16_tflops"],
                                                                  peaks["bf16_tflops_sustained"]),
        "roofline": {"kernel": dom, "bound": "tensor", "achieved": round(achieved, 1),
                     "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "traffic": traffic,
                     "algorithmic_flops_per_launch": algo_flops[dom],
                     "mean_launch_ms": round(dom_ms, 4),
                     "peak_kind": ("measured bf16 burst (cuBLAS 8192^3, best of 10; the kernel runs inside an "
                                   "~%.0f ms step)" % ms_step) if peaks["source"] == "measured" else "fallback",
                     "nvfp4_units_per_launch": fp4_units,
                     "dtype_weighted_peak": round(weighted_peak, 1),
                     "frac_dtype_weighted": round(achieved / weighted_peak, 4)},
        "kernels": kernel_table,
        # every profiled scope is one kernel launch except the selection
        # (three: tile means, coarse scores, top-k)
        "gpu_launches": len(kernels) + 2 * sum(1 for n, _ in kernels if n == "vsa_select"),
        "clocks": clocks.summary(),
        "wall_s_timed_region": round(wall, 3),
        "e2e": e2e,
    }
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            out["cpu_baseline"] = cpu_baseline_sample(
                w, args.flags, rows=sample_rows(w, CAUSAL_SAMPLE_ROWS if causal else BASELINE_SAMPLE_ROWS),
                topk=topk if sparse else None, causal=causal, T=T)
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def e2e_arm(args, torch, dev, host, w, flops, fwd, bwd, world):
    """Same step through the public API with host buffers: every step copies
    Q, K, V, dO from pinned host memory to the device and O, LSE, m, dQ, dK,
    dV back, all inside the timed region.

    The copies run on their own streams and are double-buffered: step i's
    inputs go to device slot i % 2 on the upload stream while step i-1
    computes, and step i's results leave slot i % 2 on the download stream
    while step i+1 computes.  Events order each copy against the kernels that
    read or write its slot (an upload waits until the kernels of step i-2 are
    done with the slot, the kernels wait for their upload and for the download
    of step i-2 to have drained their output slot).  Within a step the forward
    waits only for Q, K, V (dO lands while it runs) and O, LSE, m leave while
    the backward runs.  The region ends when the last download has landed in
    host memory."""
    pin = {n: t.pin_memory() for n, t in host.items()}
    shapes = dict(o=host["q"].shape, dq=host["q"].shape, dk=host["k"].shape, dv=host["v"].shape)
    stat_shape = (w.B, w.H, w.Lq)
    h_out = [dict({n: torch.empty(sh, dtype=torch.bfloat16).pin_memory() for n, sh in shapes.items()},
                  lse=torch.empty(stat_shape, dtype=torch.float32).pin_memory(),
                  m=torch.empty(stat_shape, dtype=torch.float32).pin_memory()) for _ in range(2)]
    d_in = [{n: torch.empty(t.shape, dtype=t.dtype, device=dev) for n, t in pin.items()} for _ in range(2)]
    d_out = [dict({n: torch.empty(sh, dtype=torch.bfloat16, device=dev) for n, sh in shapes.items()},
                  lse=torch.empty(stat_shape, dtype=torch.float32, device=dev),
                  m=torch.empty(stat_shape, dtype=torch.float32, device=dev)) for _ in range(2)]
    comp = torch.cuda.current_stream(dev)
    up = torch.cuda.Stream(dev)
    down = torch.cuda.Stream(dev)
    h2d = sum(t.numel() * t.element_size() for t in pin.values())
    d2h = sum(t.numel() * t.element_size() for t in h_out[0].values())

    fwd_in, fwd_out = ("q", "k", "v"), ("o", "lse", "m")

    def run(n_steps):
        # per slot: the forward's inputs landed, dO landed, the forward done,
        # the backward done, and every result of the slot downloaded
        up_f, up_b, fwd_done, computed, drained = ([torch.cuda.Event() for _ in range(2)] for _ in range(5))
        for i in range(n_steps):
            b = i % 2
            with torch.cuda.stream(up):
                if i >= 2:
                    up.wait_event(computed[b])  # the kernels of step i-2 are done with slot b
                for n in fwd_in:
                    d_in[b][n].copy_(pin[n], non_blocking=True)
                up_f[b].record(up)
                d_in[b]["do"].copy_(pin["do"], non_blocking=True)  # lands while the forward runs
                up_b[b].record(up)
            comp.wait_event(up_f[b])
            if i >= 2:
                comp.wait_event(drained[b])  # step i-2's results have left slot b
            x, y = d_in[b], d_out[b]
            fwd(x["q"], x["k"], x["v"], (y["o"], y["lse"], y["m"]), stream=comp)
            fwd_done[b].record(comp)
            with torch.cuda.stream(down):
                down.wait_event(fwd_done[b])  # O, LSE, m leave while the backward runs
                for n in fwd_out:
                    h_out[b][n].copy_(y[n], non_blocking=True)
            comp.wait_event(up_b[b])
            bwd(x["q"], x["k"], x["v"], y["lse"], y["m"], x["do"], (y["dq"], y["dk"], y["dv"]), stream=comp)
            computed[b].record(comp)
            with torch.cuda.stream(down):
                down.wait_event(computed[b])
                for n in h_out[b]:
                    if n not in fwd_out:
                        h_out[b][n].copy_(y[n], non_blocking=True)
                drained[b].record(down)
        comp.wait_stream(down)

    run(2)
    torch.cuda.synchronize(dev)
    # the same number of steps as the device timing: the pipeline's one fill
    # (the first upload) and one drain (the last download) are spread over them
    n = max(2, args.steps)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # the region opens on the compute stream before the first upload is queued
    up.wait_stream(comp)
    e0.record(comp)
    up.wait_event(e0)
    run(n)
    e1.record(comp)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks([e0.elapsed_time(e1)], dev)[0]
    value = world * flops["total"] * n / (ms * 1e-3) / 1e12
    return {"value": round(value, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": n, "ms_per_step": round(ms / n, 4),
            "copies": "pinned host <-> device every step, on upload/download streams, double-buffered"}


def load_traffic(kernel):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, if the
    summary was taken on the current attention kernel sources (else null)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    try:
        d = json.load(open(path))
        from quantization_aware_attention_nvfp4_b200 import build as B
        rec = d.get(kernel)
        if not rec or rec.get("sources_sha") != B.attention_sources_digest():
            return None
        return rec.get("dram_bytes_per_launch")
    except Exception:
        return None


# -------------------------------------------------------------- CPU oracle --

def cpu_baseline_sample(w, flags, rows: int, topk=None, causal=False, T=W.SPARSE_TILE):
    """The float64 oracle on a bounded sample of the workload: head 0, the
    first `rows` query rows against all keys, forward and backward (dQ for
    those rows, their dK/dV contributions for every key).  Returns the
    nominal TFLOP/s of that sub-problem.  With `topk`, block-sparse: the
    oracle's own selection of head 0 (inside the timed sample), counted on
    the selected keys.  With `causal`: the first `rows` tokens of head 0,
    which attend only to each other, counted on the unmasked pairs."""
    import oracle
    q = W.head_bits(w, "q", 0, 0)[:rows]
    k = W.head_bits(w, "k", 0, 0)
    v = W.head_bits(w, "v", 0, 0)
    if causal:
        k, v = k[:rows], v[:rows]
    do = W.head_bits(w, "do", 0, 0)[:rows]
    t0 = time.perf_counter()
    sel = None
    if topk is not None:
        sel = oracle.vsa_select(W.head_bits(w, "q", 0, 0), k, topk, tile=T)[0][: -(-rows // T)]
    hd = oracle.Head(q, k, v, w.sm_scale, flags | (oracle.CAUSAL if causal else 0), do, sel=sel, tile=T)
    hd.stats()
    hd.backward()
    dt = time.perf_counter() - t0
    nk = k.shape[0]
    pairs = float(rows * nk)
    if causal:
        pairs = rows * (rows + 1) / 2.0
    if sel is not None:
        keys = np.minimum(T, nk - T * np.arange(sel.shape[1]))
        rws = np.minimum(T, rows - T * np.arange(sel.shape[0]))
        pairs = float(rws @ sel.astype(np.float64) @ keys)
    flops = 3.5 * 4.0 * pairs * w.D
    what = "block-sparse, selected keys only, " if sel is not None else ("causal, " if causal else "")
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": oracle.num_threads(),
            "kind": "oracle", "seconds": round(dt, 2),
            "sample": "%s head 0, query rows [0,%d) x %s keys, %sfwd+bwd (float64 C oracle)" % (
                w.name, rows, ("the first %d" % rows) if causal else ("all %d" % nk), what)}


def reference_arm(args):
    """The oracle as the reference arm, on the same leg as the GPU arm (dense,
    --sparsity or --causal, the same workload and flags): each step is one
    bounded sample (see cpu_baseline_sample), timed on the host cores."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import oracle
    w = W.get(args.workload)
    sparse = args.sparsity is not None
    causal = bool(args.causal)
    topk = W.topk_tiles(-(-w.Lk // args.tile), args.sparsity) if sparse else None
    # the causal sample's cost grows with the square of its prefix
    rows = sample_rows(w, int(ORACLE_SAMPLE_ROWS * 2.5) if causal else ORACLE_SAMPLE_ROWS)
    for _ in range(max(0, min(args.warmup, 1))):
        cpu_baseline_sample(w, args.flags, rows=min(64, rows), topk=topk, causal=causal, T=args.tile)
    recs = [cpu_baseline_sample(w, args.flags, rows=rows, topk=topk, causal=causal, T=args.tile)
            for _ in range(args.steps)]
    seconds = sum(r["seconds"] for r in recs)
    # every step is the same sample: value = its flops over the mean time
    value = sum(r["value"] * r["seconds"] for r in recs) / seconds
    config = {"workload": workload_name(args, w), "B": w.B, "H": w.H, "Lq": w.Lq, "Lk": w.Lk, "D": w.D,
              "quantizers": flag_names(args.flags), "sample_rows": rows}
    if sparse:
        config.update(sparsity=args.sparsity, tile=args.tile)
    out = {
        "impl": "reference",
        "metric": metric_name(args, w), "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * seconds / len(recs), 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) float32 from numpy PCG64, rounded to bf16; %s)" % w.recipe,
        "config": config,
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": recs[0]["sample"] + ", one per step"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default=WORKLOAD, choices=[x.name for x in W.WORKLOADS],
                    help="seeded workload to time (default: the pages' H6 L31200 shape)")
    ap.add_argument("--flags", type=int, default=15,
                    help="quantizers on (bits q=1, k=2, v=4, p=8; default 15, all four)")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing leg")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the end-to-end leg (for short profiling runs; the line then has no e2e)")
    ap.add_argument("--sparsity", type=float, default=None,
                    help="time the block-sparse (VSA) step with this key-tile sparsity instead")
    ap.add_argument("--causal", action="store_true", help="time the causal step instead")
    ap.add_argument("--tile", type=int, default=128, choices=[64, 128],
                    help="token tile of the block-sparse leg (64: the tile-64 profile)")
    args = ap.parse_args()
    if args.causal and args.sparsity is not None:
        ap.error("--causal and --sparsity are separate legs")
    if not 0 <= args.flags <= 15:
        ap.error("--flags takes the quantizer bits 0..15")
    if args.warmup < 3 and args.impl == "native":
        args.warmup = 3
    if args.impl == "reference":
        reference_arm(args)
    else:
        gpu_arm(args)


if __name__ == "__main__":
    main()
