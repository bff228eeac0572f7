#!/usr/bin/env python
"""Benchmark of the ConvRot W8A8 linear on B200.

One step = one pass of the per-token hot path over one batch of synthetic
input: the rotate-quantise kernel (with the fused RMSNorm when the workload has
one) and the tcgen05 W8A8 GEMM with its dequant epilogue.  Weight preparation
(SmoothQuant calibration, rotation, per-row quantisation) is offline and not
timed.  The default workload is the largest single-GPU W8A8 configuration:
the fused gate+up projection at 8192 tokens (K = 4096, N = 24576).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   # the CPU oracle, timed on the host

The K timed steps are captured as one CUDA graph.  That graph is replayed
until at least MIN_TIMED_MS have passed (every replay is exactly K steps,
bracketed by a barrier and a device synchronisation); the median replay gives
ms_per_step.  Under torchrun every rank runs an independent replica (the
linear has no data exchange) and the max over ranks of the median is
reported.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

L2_BYTES = 126 * 1024 * 1024


# ------------------------------------------------------------------ ranks
def max_over_ranks(values, world: int, device):
    """Each entry's largest value over all ranks: a multi-rank measurement
    takes the slowest rank's device time.  One rank: the values themselves.
    Works on any process group (nccl on GPUs, gloo on CPU)."""
    vals = [float(v) for v in values]
    if world <= 1:
        return vals
    t = torch.tensor(vals, dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_throughput(units_per_rank_step: int, steps: int, world: int, ms: float) -> float:
    """Whole-job throughput: the units all ranks processed over the (max over
    ranks) elapsed time.  Every rank runs an independent replica of the same
    per-rank work (weak scaling)."""
    return units_per_rank_step * steps * world / (ms / 1e3)
METRIC = "ConvRot W8A8 linear TOPS and tokens/s vs INT8 tensor & HBM roofline"
DEFAULT_WORKLOAD = "gate_up_m8192"
# the timed graph (K steps) is replayed until at least this much device time
# has passed; the median replay is reported
MIN_TIMED_MS = 400.0
MIN_REPLAYS = 5
MAX_REPLAYS = 400
# dense int8 tensor peak = measured dense bf16 peak x the nominal int8:bf16 ratio (4.5 / 2.25)
INT8_PER_BF16 = 2.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--eager", action="store_true",
                    help="time eager ABI calls instead of replaying captured launches")
    ap.add_argument("--copies", type=int, default=0,
                    help="input copies rotated through to defeat L2 (0 = enough for 3x L2)")
    ap.add_argument("--no-library-reference", action="store_true",
                    help="skip timing torch._int_mm at 8192^3 (same-box context figure)")
    return ap.parse_args()


# ------------------------------------------------------------------ helpers
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# the sources each reported kernel is built from: its kernel header, the PTX
# helpers and the ABI file that plans and launches it
KERNEL_SOURCES = {
    "gemm": ("gemm.cuh", "gemm2sm.cuh", "ptx.cuh", "convrot_abi.cu"),
    "rotate_quant_act": ("actquant.cuh", "rowquant.cuh", "ptx.cuh", "convrot_abi.cu"),
}


def kernel_source_sha(kernel: str) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "w8a8_int8_quantized_rmsnorm_b200", "csrc")
    for name in sorted(KERNEL_SOURCES[kernel]):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, or None when the
    kernel's sources changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        t = json.load(f)
    e = t.get(workload, {}).get(kernel)
    if not e or e.get("source_sha") != kernel_source_sha(kernel):
        return None
    return e.get("dram_bytes_per_launch")


def agreed_replays(first_ms: float, world: int, device) -> int:
    """How many times the K-step region is replayed: enough for MIN_TIMED_MS
    of device time at the slowest rank's first replay, within [MIN_REPLAYS,
    MAX_REPLAYS].  Every rank gets the same count, so every rank takes the
    same collective steps."""
    first = max_over_ranks([first_ms], world, device)[0]
    return int(min(MAX_REPLAYS, max(MIN_REPLAYS, math.ceil(MIN_TIMED_MS / max(first, 1e-3)))))


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 20 ms; only the
    samples taken inside the timed region (between mark_start and mark_stop)
    are reported."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []  # (arrival time, line)
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark_start(self):
        self.t0 = time.time()

    def mark_stop(self):
        self.t1 = time.time()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.05)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        return summarize_clocks(self.lines, self.t0, self.t1)


def summarize_clocks(lines, t0=None, t1=None):
    """Median SM clock, max clock, median power and the throttle reasons seen
    in the (arrival time, nvidia-smi csv line) samples inside [t0, t1]."""
    sm, mx, pw, reasons = [], [], [], set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for t, ln in lines:
        if (t0 is not None and t < t0) or (t1 is not None and t > t1):
            continue
        parts = [p.strip() for p in ln.split(",")]
        if len(parts) < 9:
            continue
        try:
            sm.append(float(parts[1]))
            mx.append(float(parts[2]))
        except ValueError:
            continue
        try:
            pw.append(float(parts[3]))
        except ValueError:
            pass
        for n, v in zip(names, parts[5:9]):
            if v.lower().startswith("active"):
                reasons.add(n)
    return {"sm_mhz": statistics.median(sm) if sm else None,
            "sm_min_mhz": min(sm) if sm else None,
            "sm_max_mhz": max(mx) if mx else None,
            "power_w": statistics.median(pw) if pw else None,
            "reasons": sorted(reasons), "samples": len(sm), "period_ms": 20}


# ------------------------------------------------------------------ our arm
class Linear:
    def __init__(self, lin, Wq, s_row, group_in, swiglu=False):
        self.lin = lin
        self.Wq = Wq
        self.s_row = s_row
        self.group_in = group_in
        self.swiglu = swiglu  # gate/up GEMM whose epilogue writes SiLU(gate) * up
        self.out_cols = lin.N // 2 if swiglu else lin.N


def input_groups(w):
    """Linears that read the same activation share one rotate-quantise call."""
    if w.mlp:
        return [{"key": "mlp", "K": w.linears[0].K, "linears": [w.linears[0]]},
                {"key": "down", "K": w.linears[1].K, "linears": [w.linears[1]]}]
    groups = []
    for lin in w.linears:
        key = {"q_proj": "attn", "k_proj": "attn", "v_proj": "attn", "o_proj": "o",
               "gate_proj": "mlp", "up_proj": "mlp", "down_proj": "down"}.get(lin.name, lin.name)
        for g in groups:
            if g["key"] == key:
                g["linears"].append(lin)
                break
        else:
            groups.append({"key": key, "K": lin.K, "linears": [lin]})
    return groups


def prepare_mlp(cr, w, dev):
    """The MLP block's inputs and offline preparation (untimed): SmoothQuant
    into the norm weight and into up_proj's row scales, interleaved gate/up."""
    groups = input_groups(w)
    gu = w.linears[0]
    x = workloads.activations(w.M, gu.K, dist=w.dist, outlier_count=w.n_outliers(gu.K),
                              outlier_scale=w.outlier_scale).to(dev)
    nw = workloads.norm_weight(gu.K).to(dev)
    Wg, Wu, Wd = (t.to(dev) for t in workloads.mlp_weights(w, device=dev))
    mlp = cr.ConvRotMLP(Wg, Wu, Wd, norm_w=nw, x_calib=x)
    del Wg, Wu, Wd
    # the second group's input is the intermediate H, written by the gate/up GEMM
    h = torch.empty(w.M, gu.N // 2, dtype=torch.bfloat16, device=dev)
    layers = [Linear(gu, mlp.Wq_gu, mlp.s_gu, 0, swiglu=True), Linear(w.linears[1], mlp.Wq_d, mlp.s_d, 1)]
    torch.cuda.synchronize(dev)
    return groups, [x, h], [mlp.norm_w, None], layers, mlp


def prepare(cr, w, dev):
    """Synthetic inputs and offline weight preparation (untimed)."""
    if w.mlp:
        return prepare_mlp(cr, w, dev)[:4]
    groups = input_groups(w)
    inputs, norms = [], []
    for gi, g in enumerate(groups):
        lin0 = g["linears"][0]
        x = workloads.activations(w.M, lin0.K, dist=w.dist, outlier_count=w.n_outliers(lin0.K),
                                  outlier_scale=w.outlier_scale)
        nw = workloads.norm_weight(lin0.K) if w.norm else None
        inputs.append(x.to(dev))
        norms.append(None if nw is None else nw.to(dev))
    raw_norms = list(norms)
    layers = []
    for layer in range(w.layers):
        for gi, g in enumerate(groups):
            for lin in g["linears"]:
                gen_dev = "cpu" if lin.N * lin.K <= (1 << 27) and w.layers == 1 else dev
                W = workloads.weight(lin.N, lin.K, layer=layer, device=gen_dev).to(dev)
                col = None
                if raw_norms[gi] is not None:
                    # one norm-carrying linear per input group in these workloads
                    col, norms[gi] = cr.convrot_smoothquant_calibrate(inputs[gi], raw_norms[gi], W)
                if w.weight_bits == 8:
                    Wq, s_row = cr.convrot_quantize_weight(W, 256, col)
                else:
                    Wq, s_row = cr.convrot_quantize_weight_w4(W, 256, col)
                del W
                layers.append(Linear(lin, Wq, s_row, gi))
    torch.cuda.synchronize(dev)
    return groups, inputs, norms, layers


def run_ours(args, rank, world, dev):
    import w8a8_int8_quantized_rmsnorm_b200 as cr
    cr.lib()
    w = workloads.WORKLOADS[args.workload]
    peaks = load_peaks()
    torch.cuda.set_device(dev)
    groups, inputs, norms, layers = prepare(cr, w, dev)

    # copies of the per-step operands so that no step finds its inputs in L2
    # (the MLP block's H is produced inside the step: one buffer for all copies)
    step_bytes = sum(x.numel() * 2 for x in inputs) + sum(l.Wq.numel() for l in layers)
    copies = 1 if step_bytes > 2 * L2_BYTES else min(8, math.ceil(3 * L2_BYTES / step_bytes))
    if args.copies > 0:
        copies = args.copies
    x_sets = [inputs] + [[x if (w.mlp and gi == 1) else x.clone() for gi, x in enumerate(inputs)]
                         for _ in range(copies - 1)]
    w_sets = [[(l.Wq, l.s_row) for l in layers]] + \
             [[(l.Wq.clone(), l.s_row.clone()) for l in layers] for _ in range(copies - 1)]
    ws = cr.Workspace(dev.index)
    wo = w.weight_only
    Xq = [torch.empty(w.M, g["K"], dtype=torch.bfloat16 if wo else torch.int8, device=dev) for g in groups]
    st = [torch.empty(w.M, dtype=torch.float32, device=dev) for g in groups]
    Ys = [inputs[1] if l.swiglu else torch.empty(w.M, l.out_cols, dtype=torch.bfloat16, device=dev)
          for l in layers]
    linear = cr.convrot_int8_linear if w.weight_bits == 8 else cr.convrot_w4a8_linear
    swiglu = cr.convrot_int8_linear_swiglu if w.weight_bits == 8 else cr.convrot_w4a8_linear_swiglu

    stream = torch.cuda.current_stream(dev)
    n_k1 = len(groups)
    n_k2 = len(layers)

    def launch_k1(c, gi):
        if wo:
            cr.convrot_rotate_act_bf16(x_sets[c][gi], 256, norms[gi], 1e-6, out=Xq[gi])
        else:
            cr.convrot_rotate_quant_act(x_sets[c][gi], 256, norms[gi], 1e-6, out=(Xq[gi], st[gi]))

    def launch_k2(c, li):
        l = layers[li]
        Wq, s_row = w_sets[c][li]
        if wo:
            cr.convrot_weight_only_linear(Xq[l.group_in], Wq, s_row, out=Ys[li], workspace=ws)
            return
        (swiglu if l.swiglu else linear)(Xq[l.group_in], st[l.group_in], Wq, s_row, out=Ys[li],
                                         workspace=ws)

    # launch order of one step: every rotate-quantise, then every GEMM; the
    # MLP block is a chain (x -> gate/up -> H -> down)
    order = ([("k1", 0), ("k2", 0), ("k1", 1), ("k2", 1)] if w.mlp else
             [("k1", gi) for gi in range(len(groups))] + [("k2", li) for li in range(len(layers))])

    def launch(c, kind, idx):
        (launch_k1 if kind == "k1" else launch_k2)(c, idx)

    # Graph mode (default): the W warm-up steps and the K timed steps are each
    # captured as ONE CUDA graph of the same ABI calls (step i reads input copy
    # i % copies), as a serving stack captures a whole forward pass; the timed
    # region is one replay between two events on the launching stream.  Each
    # kernel's average duration comes from its own region: its K * launches
    # alone, captured and replayed the same way.  (An event-record node
    # between two kernels inside a graph costs ~5 us on this GPU, so kernels
    # are not bracketed one by one.)  --eager issues the same calls directly.
    for c in range(copies):  # eager warm-up: encodes and caches every tensor map
        for kind, idx in order:
            launch(c, kind, idx)
    torch.cuda.synchronize(dev)

    def step(i):
        for kind, idx in order:
            launch(i % copies, kind, idx)

    def k1_only(i):
        for gi in range(n_k1):
            launch_k1(i % copies, gi)

    def k2_only(i):
        for li in range(n_k2):
            launch_k2(i % copies, li)

    def region(fn, n):
        """The launches of fn(0..n-1): one captured graph, or None in eager mode."""
        if args.eager:
            return None
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=torch.cuda.Stream(dev)):
            for i in range(n):
                fn(i)
        return g

    def run(fn, n, graph):
        if graph is not None:
            graph.replay()
        else:
            for i in range(n):
                fn(i)

    def timed(fn, n, graph):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        a.record(stream)
        run(fn, n, graph)
        b.record(stream)
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b)

    def replays(fn, n, graph, sync_ranks):
        """Replays the K-step region until MIN_TIMED_MS of device time have
        passed (at least MIN_REPLAYS times); every replay is timed on its own
        between two events on the launching stream.  The replay count is agreed
        over ranks from the first replay, so every rank takes the same
        collective steps.  Returns (median ms, every replay's ms)."""
        def one():
            if sync_ranks and world > 1:
                torch.distributed.barrier()
            return timed(fn, n, graph)
        times = [one()]
        for _ in range(agreed_replays(times[0], world, dev) - 1):
            times.append(one())
        return statistics.median(times), times

    warm_graph = region(step, args.warmup)
    timed_graph = region(step, args.steps)
    k1_graph = region(k1_only, args.steps)
    k2_graph = region(k2_only, args.steps)
    torch.cuda.synchronize(dev)
    run(step, args.warmup, warm_graph)
    torch.cuda.synchronize(dev)
    status = cr.convrot_device_status(dev.index)
    if status:
        raise RuntimeError(f"device error word {status:#x} after warm-up")

    clocks = ClockSampler(dev.index)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    time.sleep(0.3)
    clocks.mark_start()
    median_ms, step_times = replays(step, args.steps, timed_graph, True)
    clocks.mark_stop()
    clk = clocks.stop()
    if world > 1:
        torch.distributed.barrier()
    elapsed_ms = max_over_ranks([median_ms], world, dev)[0]
    status = cr.convrot_device_status(dev.index)
    if status:
        raise RuntimeError(f"device error word {status:#x} in the timed region")

    # per-kernel regions, timed the same way (median of replays)
    k1_region_ms, _ = replays(k1_only, args.steps, k1_graph, False)
    k2_region_ms, _ = replays(k2_only, args.steps, k2_graph, False)
    k1_region_ms, k2_region_ms = max_over_ranks([k1_region_ms, k2_region_ms], world, dev)
    status = cr.convrot_device_status(dev.index)
    if status:
        raise RuntimeError(f"device error word {status:#x} in a kernel timing region")

    k1_ms = [k1_region_ms / args.steps]  # per step
    k2_ms = [k2_region_ms / args.steps]
    k1_avg = statistics.mean(k1_ms) / n_k1  # per launch
    k2_avg = statistics.mean(k2_ms) / n_k2

    ops = w.ops() * args.steps * world
    secs = elapsed_ms / 1e3
    # algorithmic bytes: K1 reads bf16 and writes int8 codes + scales (bf16 on
    # the weight-only path); K2 reads its activation (int8, or bf16 on the
    # weight-only path), the weight, the scales and writes bf16
    act_b = 2 if wo else 1
    k1_bytes = sum(w.M * g["K"] * (2 + act_b) + (0 if wo else 4 * w.M) +
                   (4 * g["K"] if norms[gi] is not None else 0) for gi, g in enumerate(groups))
    k2_bytes = sum(act_b * w.M * l.lin.K + l.Wq.numel() + 2 * w.M * l.out_cols +
                   (0 if wo else 4 * w.M) + 4 * l.lin.N for l in layers)
    k2_ops = w.ops()
    # the weight-only GEMM multiplies in bf16: its tensor peak is the bf16 one
    int8_peak = peaks["bf16_tflops"] * (1.0 if wo else INT8_PER_BF16)
    k2_achieved_tops = k2_ops / (statistics.mean(k2_ms) / 1e3) / 1e12
    k2_achieved_gbs = k2_bytes / (statistics.mean(k2_ms) / 1e3) / 1e9
    k1_achieved_gbs = k1_bytes / (statistics.mean(k1_ms) / 1e3) / 1e9
    # the GEMM dominates every workload's step; it is tensor-bound above the
    # ridge (~250 tokens) and weight-stream (HBM) bound below it
    ridge_bound = "tensor" if w.M > 256 else "hbm"
    if ridge_bound == "tensor":
        roof = {"bound": "tensor", "kernel": ("weight-only GEMM launch (tcgen05 kind::f16, int8 weight codes)"
                                              if wo else "W8A8/W4A8 GEMM launch (tcgen05 kind::i8)"),
                "achieved": round(k2_achieved_tops, 1), "peak": round(int8_peak, 1),
                "unit": "TOP/s", "frac": round(k2_achieved_tops / int8_peak, 4),
                "peak_note": (f"{peaks['source']}: dense bf16 burst {peaks['bf16_tflops']} TFLOP/s" if wo else
                              f"{peaks['source']}: 2 x dense bf16 burst {peaks['bf16_tflops']} TFLOP/s")}
        if peaks.get("bf16_tflops_sustained"):
            # the kernel region is replayed for MIN_TIMED_MS or more: the
            # power-capped (sustained) dense peak is reported beside the burst one
            sus = peaks["bf16_tflops_sustained"] * (1.0 if wo else INT8_PER_BF16)
            roof["peak_sustained"] = round(sus, 1)
            roof["frac_sustained"] = round(k2_achieved_tops / sus, 4)
    else:
        roof = {"bound": "hbm", "kernel": ("weight-only GEMM launch (tcgen05 kind::f16, int8 weight codes)"
                                           if wo else "W8A8/W4A8 GEMM launch (tcgen05 kind::i8)"),
                "achieved": round(k2_achieved_gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(k2_achieved_gbs / peaks["hbm_gbs"], 4),
                "peak_note": f"{peaks['source']} copy bandwidth"}
    roof["traffic"] = profiled_traffic("gemm", args.workload)
    roof["algorithmic_per_launch"] = (k2_ops / n_k2) if ridge_bound == "tensor" else (k2_bytes / n_k2)

    result = {
        "metric": METRIC,
        "value": round(job_throughput(w.M, args.steps, world, elapsed_ms), 1),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(elapsed_ms / args.steps, 5),
        "timed_replays": len(step_times),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if wo else "i8",
        "data": "synthetic (seeded; no trained weights or datasets)",
        "tops": round(ops / secs / 1e12, 1),
        "config": {
            "workload": args.workload, "M": w.M,
            "linears": [[l.name, l.N, l.K] for l in w.linears], "layers": w.layers,
            "weight_bits": w.weight_bits, "group": 256, "rmsnorm": w.norm,
            **({"path": "weight-only: rotated bf16 activations x int8 weight codes (bf16 MMA)"} if wo else {}),
            **({"block": "down(SiLU(gate(x)) * up(x)); gate/up as one GEMM with the SwiGLU epilogue"}
               if w.mlp else {}),
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "launch": ("eager ABI calls" if timed_graph is None else
                       "the K timed steps' ABI calls captured as one CUDA graph"),
            "timing": (f"{len(step_times)} replays of the K-step region, each timed between two "
                       f"events; median reported (min {min(step_times):.4f} ms, max "
                       f"{max(step_times):.4f} ms per replay, {sum(step_times):.1f} ms in total)"),
            "kernel_timing": ("each kernel's K * launches_per_step launches timed alone as one "
                              "region (same inputs and copies), replayed the same way; median"),
            "l2": (f"{copies} rotating copies of the step's inputs "
                   f"({copies * step_bytes / 1e6:.0f} MB > L2)") if copies > 1
                  else f"step inputs {step_bytes / 1e6:.0f} MB > 2x L2",
        },
        "roofline": roof,
        "kernels": {
            "rotate_quant_act": {"launches_per_step": n_k1, "avg_us": round(k1_avg * 1e3, 3),
                                 "bound": "hbm", "achieved_GBps": round(k1_achieved_gbs, 1),
                                 "frac": round(k1_achieved_gbs / peaks["hbm_gbs"], 4),
                                 "traffic": profiled_traffic("rotate_quant_act", args.workload),
                                 "algorithmic_bytes_per_step": k1_bytes},
            "gemm": {"launches_per_step": n_k2, "avg_us": round(k2_avg * 1e3, 3),
                     "achieved_TOPs": round(k2_achieved_tops, 1),
                     "tensor_frac": round(k2_achieved_tops / int8_peak, 4),
                     "achieved_GBps": round(k2_achieved_gbs, 1),
                     "hbm_frac": round(k2_achieved_gbs / peaks["hbm_gbs"], 4),
                     "algorithmic_bytes_per_step": k2_bytes, "ops_per_step": k2_ops},
        },
        "kernels_sum_ms_per_step": round((k1_region_ms + k2_region_ms) / args.steps, 5),
        "gpu_launches": (n_k1 + n_k2) * args.steps * len(step_times),
        "clocks": clk,
    }
    if not args.no_e2e:
        result["e2e"] = e2e_ours(cr, args, w, groups, inputs, norms, layers, dev, world)
    return result


def e2e_ours(cr, args, w, groups, inputs, norms, layers, dev, world):
    """Same metric through the public API with pinned host buffers: every step
    copies its activations host->device and its outputs device->host.

    Steps are double-buffered over three streams, as a serving loop would run
    them: step i's upload (copy-in stream) overlaps step i-1's kernels
    (compute stream) and step i-2's download (copy-out stream).  Events order
    each step's copy-in -> compute -> copy-out and keep a buffer from being
    reused before the step that last used it is done.  The timed region runs
    from the first upload to the last download."""
    ws = cr.Workspace(dev.index)
    linear = cr.convrot_int8_linear if w.weight_bits == 8 else cr.convrot_w4a8_linear
    swiglu = cr.convrot_int8_linear_swiglu if w.weight_bits == 8 else cr.convrot_w4a8_linear_swiglu
    steps = max(5, min(args.steps, 50))
    # the step's inputs (one activation per input group; the MLP block's only
    # input is x) and outputs (one per linear; the MLP block's is down_proj's)
    ins = [inputs[0]] if w.mlp else list(inputs)
    out_shapes = [(w.M, layers[1].out_cols)] if w.mlp else [(w.M, l.lin.N) for l in layers]
    host_x = [x.cpu().pin_memory() for x in ins]
    host_y = [[torch.empty(sh, dtype=torch.bfloat16).pin_memory() for sh in out_shapes] for _ in range(2)]
    dev_x = [[torch.empty_like(x, device=dev) for x in ins] for _ in range(2)]
    dev_y = [[torch.empty(sh, dtype=torch.bfloat16, device=dev) for sh in out_shapes] for _ in range(2)]
    s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    ev = lambda: torch.cuda.Event()
    up, done, down = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    for e in up + done + down:
        e.record(torch.cuda.current_stream(dev))

    def compute(xs, ys):
        if w.mlp:
            gu, dn = layers
            Xq, s_tok = cr.convrot_rotate_quant_act(xs[0], 256, norms[0], 1e-6)
            H = swiglu(Xq, s_tok, gu.Wq, gu.s_row, workspace=ws)
            Hq, s_h = cr.convrot_rotate_quant_act(H, 256, None, 1e-6)
            linear(Hq, s_h, dn.Wq, dn.s_row, out=ys[0], workspace=ws)
        elif w.weight_only:
            xr = [cr.convrot_rotate_act_bf16(xs[g], 256, norms[g], 1e-6) for g in range(len(groups))]
            for li, l in enumerate(layers):
                cr.convrot_weight_only_linear(xr[l.group_in], l.Wq, l.s_row, out=ys[li], workspace=ws)
        else:
            qs = [cr.convrot_rotate_quant_act(xs[g], 256, norms[g], 1e-6) for g in range(len(groups))]
            for li, l in enumerate(layers):
                linear(qs[l.group_in][0], qs[l.group_in][1], l.Wq, l.s_row, out=ys[li], workspace=ws)

    def step(i):
        b = i % 2
        with torch.cuda.stream(s_in):
            s_in.wait_event(done[b])            # step i-2's kernels have read dev_x[b]
            for h, d in zip(host_x, dev_x[b]):
                d.copy_(h, non_blocking=True)
            up[b].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(up[b])
            s_cmp.wait_event(down[b])           # step i-2's download has read dev_y[b]
            compute(dev_x[b], dev_y[b])
            done[b].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(done[b])
            for d, h in zip(dev_y[b], host_y[b]):
                h.copy_(d, non_blocking=True)
            down[b].record(s_out)

    for i in range(4):
        step(i)
    torch.cuda.synchronize(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    t0.record(s_in)
    for i in range(steps):
        step(i)
    t1.record(s_out)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks([t0.elapsed_time(t1)], world, dev)[0]
    return {"value": round(job_throughput(w.M, steps, world, ms), 1), "unit": "tokens/s",
            "h2d_bytes_per_step": sum(h.numel() * 2 for h in host_x),
            "d2h_bytes_per_step": sum(h.numel() * 2 for h in host_y[0]), "steps": steps,
            "pipelining": "double-buffered: copy-in, compute and copy-out streams ordered by events"}


# ------------------------------------------------------------------ oracle arm
def oracle_step_runner(w, sample_tokens):
    """Prepares the oracle's weights (untimed) and returns a callable that runs
    the oracle's per-token path on `sample_tokens` tokens of the workload."""
    from oracle import convrot_ref as ref
    if w.mlp:
        return oracle_mlp_runner(ref, w, sample_tokens)
    groups = input_groups(w)
    xs, nws, preps = [], [], []
    for g in groups:
        lin0 = g["linears"][0]
        x, _, nw = workloads.workload_inputs(w, lin0, M=min(w.M, max(sample_tokens, 1)))
        xs.append(x.float().double().numpy()[:sample_tokens])
        nws.append(None if nw is None else nw.double().numpy())
    for gi, g in enumerate(groups):
        for lin in g["linears"]:
            W = workloads.weight(lin.N, lin.K).float().double().numpy()
            col = None
            if nws[gi] is not None:
                col, nws[gi] = ref.smoothquant_scales(xs[gi], nws[gi], 1e-6, W)
            if w.weight_bits == 8:
                Wq, s_row, _ = ref.quantize_weight(W, 256, col)
                preps.append((gi, Wq, s_row, None))
            else:
                o = ref.quantize_weight_w4(W, 256, col)
                preps.append((gi, None, o["s_row"], o["packed"]))

    if w.weight_only:
        def run_wo():
            acts = [ref.to_bf16(ref.rotate_act(xs[g], 256, nws[g], 1e-6)) for g in range(len(groups))]
            for gi, Wq, s_row, _ in preps:
                ref.weight_only_linear(acts[gi], Wq, s_row)
        return run_wo

    def run():
        acts = [ref.rotate_quant_act(xs[g], 256, nws[g], 1e-6) for g in range(len(groups))]
        for gi, Wq, s_row, packed in preps:
            Xq, s_tok, _ = acts[gi]
            if packed is None:
                ref.int8_linear(Xq, s_tok, Wq, s_row)
            else:
                ref.w4a8_linear(Xq, s_tok, packed, s_row)
    return run


def oracle_mlp_runner(ref, w, sample_tokens):
    """The MLP block through the oracle: calibration and weight preparation on
    the sample (untimed), then norm + rotate-quantise, gate/up with SiLU(gate)
    * up, rotate-quantise of H and down_proj per call."""
    gu = w.linears[0]
    x, _, nw = workloads.workload_inputs(w, gu, M=min(w.M, max(sample_tokens, 1)))
    x64 = x.float().double().numpy()[:sample_tokens]
    Wg, Wu, Wd = (t.float().double().numpy() for t in workloads.mlp_weights(w))
    sc, wf = ref.smoothquant_scales(x64, nw.double().numpy(), 1e-6, np.concatenate([Wg, Wu]))
    qg, sg, _ = ref.quantize_weight(Wg, 256, sc)
    qu, su, _ = ref.quantize_weight(Wu, 256, sc)
    del Wg, Wu
    qgu = ref.interleave_gate_up(qg, qu)
    Xq, st, _ = ref.rotate_quant_act(x64, 256, wf, 1e-6)
    h0, _, _ = ref.swiglu_linear(Xq, st, qgu, ref.interleave_gate_up(sg, su))
    sd = ref.smoothquant_scales_of(h0, Wd)
    sgu = ref.interleave_gate_up(sg, ref.fold_smooth_into_rows(su, sd))
    qd, sdr, _ = ref.quantize_weight(Wd, 256, sd)
    del Wd

    def run():
        Xq, st, _ = ref.rotate_quant_act(x64, 256, wf, 1e-6)
        hb, _, _ = ref.swiglu_linear(Xq, st, qgu, sgu)
        Hq, sh, _ = ref.rotate_quant_act(hb, 256)
        ref.int8_linear(Hq, sh, qd, sdr)
    return run


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def library_int8_reference(dev, peak_tops, n=8192, reps=20):
    """A library int8 GEMM on the same GPU for context: torch._int_mm on
    n x n x n int8 operands (int32 result), timed with CUDA events after
    warm-up.  Not the target, and not part of the hot path."""
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    a = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev, generator=g)
    b = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev, generator=g)
    for _ in range(3):
        torch._int_mm(a, b)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        torch._int_mm(a, b)
    e1.record()
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / reps
    tops = 2.0 * n ** 3 / (ms / 1e3) / 1e12
    del a, b
    return {"op": "torch._int_mm", "shape": [n, n, n], "ms": round(ms, 4),
            "tops": round(tops, 1), "frac_of_int8_peak": round(tops / peak_tops, 4)}


def _time_oracle(run, target_s):
    run()  # warm
    reps, t = 0, 0.0
    t0 = time.perf_counter()
    while True:
        run()
        reps += 1
        t = time.perf_counter() - t0
        if t >= target_s or reps >= 1000:
            return reps, t


def cpu_baseline(w, target_s=10.0, single_s=3.0):
    """The oracle as it stands on the host cores, on a bounded sample; then
    the same sample on one BLAS thread."""
    sample = min(w.M, 64 if w.layers == 1 else 16)
    run = oracle_step_runner(w, sample)
    reps, t = _time_oracle(run, target_s)
    per_tok = t / (reps * sample * w.layers)
    res = {"value": round(1.0 / per_tok, 2), "unit": "tokens/s", "cores": blas_threads(),
           "kind": "oracle",
           "sample": f"{sample} tokens of {w.name} x {reps} repetitions "
                     f"({t:.1f} s; float64 numpy, every linear of the step"
                     + (f", 1 of {w.layers} layers, scaled" if w.layers > 1 else "") + ")"}
    try:
        from threadpoolctl import threadpool_limits
    except ImportError:
        return res
    with threadpool_limits(limits=1, user_api="blas"):
        reps1, t1 = _time_oracle(run, single_s)
    res["single_thread"] = {"value": round(reps1 * sample * w.layers / t1, 2), "unit": "tokens/s",
                            "cores": 1, "sample": f"the same sample x {reps1} repetitions ({t1:.1f} s)"}
    return res


def run_reference(args, rank, world):
    w = workloads.WORKLOADS[args.workload]
    if rank != 0:
        return None
    sample = min(w.M, 64 if w.layers == 1 else 16)
    run = oracle_step_runner(w, sample)
    for _ in range(max(1, min(args.warmup, 3))):
        run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run()
    secs = time.perf_counter() - t0
    tok_s = sample * args.steps / secs / w.layers
    return {
        "impl": "reference", "metric": METRIC, "value": round(tok_s, 2), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(secs / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)",
        "config": {"workload": args.workload, "M": w.M, "sample_tokens_per_step": sample},
        "cpu_baseline": {"value": round(tok_s, 2), "unit": "tokens/s", "cores": blas_threads(),
                         "kind": "oracle",
                         "sample": f"{sample} tokens of {w.name} per step"},
        "e2e": {"value": round(tok_s, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# ------------------------------------------------------------------ main
def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
    try:
        res = run_ours(args, rank, world, dev)
        if rank == 0:
            if not args.no_library_reference:
                peaks = load_peaks()
                res["library_reference"] = library_int8_reference(
                    dev, INT8_PER_BF16 * peaks["bf16_tflops"])
            if not args.no_cpu_baseline:
                res["cpu_baseline"] = cpu_baseline(workloads.WORKLOADS[args.workload])
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
