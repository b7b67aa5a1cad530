#!/usr/bin/env python
"""Throughput of the B200 Muon / NorMuon optimizer step.

One step = momentum + Nesterov + Frobenius norm (muon_momentum_norm), quintic
Newton-Schulz of every slice (muon_ns_batched or muon_gram_ns_batched) and
NorMuon + weight update (normuon_update), over every matrix of the workload,
with all inputs resident in HBM.  Prints ONE JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload llama8b]
                    [--variant standard|gram] [--impl ours|reference]

Metric: Newton-Schulz TFLOP/s of the whole step (the algorithmic flops of
the variant run -- one-triangle symmetric products -- divided by the step
time), with its fraction of the measured bf16 dense tensor-core peak and the
matrices (Newton-Schulz slices) per second.  Multi-GPU runs are independent
replicas (the step has no exchange): value = all ranks' work / max time.
``--impl reference`` times the fp64 CPU oracle on a bounded sample of the
same workload instead (rank 0 only).
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Muon step NS TFLOP/s & % bf16 TC peak; matrices/s at 1 B200 vs CPU oracle"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

DESCRIPTIONS = {
    "llama8b": "Llama-8B-shaped Muon step, 32 layers: q,o 4096x4096, k,v 1024x4096, gate,up 14336x4096, "
               "down 4096x14336 (224 matrices); bf16 G and M, fp32 master W + bf16 copy; NorMuon; lr 0.02",
    "moe": "MoE megabatch: 64 experts x (w1 2048x7168, w2 7168x2048) bf16; per-expert grad scale "
           "log-uniform [1e-2,1]; NorMuon; lr 0.02",
    "per_head": "q_proj 4096x4096 as 32 heads [32,128,4096] + 512x1024 + 1024x512, bf16, plain Muon",
    "conv_megabatch": "16 stacked Conv2d [16,64,64,3,3] -> [16,64,576] bf16, NorMuon, lr 0.02, wd 0.01",
    "single_256": "one 256x256 fp32 gradient, Muon, lr 0.05",
}



def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama8b", choices=sorted(DESCRIPTIONS))
    ap.add_argument("--variant", choices=["standard", "gram", "auto"], default=None,
                    help="auto: Gram form for slices with n >= 1.25 m, standard otherwise")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--scale-down", type=int, default=1, help="divide every parameter count (smoke runs only)")
    ap.add_argument("--coefficients", choices=["quintic", "polar-express"], default="quintic",
                    help="quintic: (3.4445, -4.7750, 2.0315) at every step; polar-express: the greedy "
                         "minimax schedule for singular values in [--pe-lower, 1]")
    ap.add_argument("--pe-lower", type=float, default=1e-3)
    ap.add_argument("--pe-safety", type=float, default=1.01)
    ap.add_argument("--schedule", choices=["serial", "two-stream"], default="serial",
                    help="serial: one call per stage over every shape; two-stream: per-shape calls, each shape's "
                         "Newton-Schulz on the main stream while the momentum of the next shape and the update of "
                         "the previous one run on a second stream (TwoStreamStep)")
    ap.add_argument("--graph", choices=["on", "off"], default="on",
                    help="on: the timed steps replay a CUDA graph of one whole step (the per-stage split "
                         "comes from eager steps after it); off: eager calls")
    return ap.parse_args()


def _peak_number(v):
    """A peak as a plain number, or from a record that holds one (value / median / mean / max)."""
    if isinstance(v, (int, float)) and v > 0:
        return float(v)
    if isinstance(v, dict):
        for k in ("value", "median", "mean", "max"):
            if isinstance(v.get(k), (int, float)) and v[k] > 0:
                return float(v[k])
    return None


def load_peaks(path=None):
    """The measured peaks (hbm_gbs, bf16_tflops, bf16_tflops_sustained) where the measurements file
    holds them, the fallback figures elsewhere; returns (peaks, {key: "measured" | "fallback"})."""
    p = path or os.path.join(ROOT, "MEASURED_PEAKS.json")
    d = {}
    if os.path.exists(p):
        try:
            with open(p) as f:
                raw = json.load(f)
            if isinstance(raw, dict):
                for k in FALLBACK_PEAKS:
                    v = _peak_number(raw.get(k))
                    if v is not None:
                        d[k] = v
        except (OSError, ValueError):
            d = {}
    peaks = dict(FALLBACK_PEAKS)
    peaks.update(d)
    return peaks, {k: ("measured" if k in d else "fallback") for k in FALLBACK_PEAKS}


AUTO_GRAM_RATIO = 1.25


def slice_variant(rows, cols, variant):
    if variant != "auto":
        return variant
    m, n = min(rows, cols), max(rows, cols)
    return "gram" if n > m and n >= AUTO_GRAM_RATIO * m else "standard"


GRAM_RESTART = 3        # the library's default restart period of the Gram form


def ns_flops(rows, cols, variant, steps, restart=GRAM_RESTART):
    """Work of one slice's orthogonalization, as the metric counts it (m = short side, n = long side).

    Standard, one triangle of each symmetric product: per step m^2 n (X X^T)
    + m^3 (b*A + c*A^2) + 2 m^2 n (B X).  Gram: m^2 n for X X^T, 2 m^2 n for
    the final Q X, per step one-triangle m^3 products: A^2, P Q (except at a
    segment's first step), the two factors of P A P (except at a segment's
    last step); each restart adds Q X (2 m^2 n) and X X^T (m^2 n).
    Both arms of the benchmark count the same work for the same variant.
    """
    m, n = min(rows, cols), max(rows, cols)
    variant = slice_variant(rows, cols, variant)
    if variant == "standard":
        return float(steps * (3 * m * m * n + m ** 3))

    def restart_at(k):
        return restart > 0 and 0 < k < steps and k % restart == 0

    prods, restarts, seg = 0, 0, 0
    for k in range(steps):
        if restart_at(k):
            restarts += 1
            seg = k
        prods += 1 + (k != seg) + 2 * (not (k == steps - 1 or restart_at(k + 1)))
    return float(3 * m * m * n + restarts * 3 * m * m * n + prods * m ** 3)


TRAFFIC_SOURCES = ("newton_schulz_ns_b200/csrc/ns_gemm.cuh", "newton_schulz_ns_b200/csrc/ptx_sm100.cuh",
                   "newton_schulz_ns_b200/csrc/muon_api.cu")


def kernel_source_hash():
    import hashlib
    h = hashlib.sha256()
    for f in TRAFFIC_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(key, variant):
    """DRAM bytes of one Newton-Schulz call, scaled from the committed ncu summary, or None.

    The summary holds per-launch captures of a one-layer case (a few launches
    per ncu run) and their scaling to one call of the full workload; it
    records the hash of the kernel sources it was captured with, and a
    different hash (the kernel changed since) gives None.
    """
    import re
    path = os.path.join(ROOT, "profiles", f"ns_gemm_{key}_{variant}_traffic_scaled.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_hash = re.search(r"source_hash:\s*([0-9a-f]+)", text)
    m_bytes = re.search(r"dram_bytes_per_ns_call_scaled:\s*([0-9.eE+]+)", text)
    if not m_hash or not m_bytes or m_hash.group(1) != kernel_source_hash():
        return None
    return float(m_bytes.group(1))


def default_variant(wl):
    return "gram" if wl.key == "moe" else "standard"


# ----------------------------------------------------------------------------- CPU oracle (baseline)

def small_kernel(r, c):
    """The fused kernel a slice takes (the library's shape rule), or None for the GEMM path."""
    m, n = min(r, c), max(r, c)
    if m > 128:
        return None
    if n <= 2048:
        return "ns_small_kernel"                 # columns resident on <= 4 CTAs
    if n % 8 == 0 and n <= 16384:
        return "ns_stream_kernel"                # columns streamed from L2, 4-CTA clusters
    if n <= 4096:
        return "ns_small_kernel"                 # resident on 8 CTAs
    return None


def ns_kernels_label(groups):
    """Which kernels one Newton-Schulz call of these batches runs."""
    names = []
    for b in groups:
        k = small_kernel(b.rows, b.cols) or "ns_gemm_pair_kernel / ns_gemm_kernel"
        if k not in names:
            names.append(k)
    return " + ".join(names) + " (all launches of one Newton-Schulz call)"


def ns_dtype(groups, variant):
    """The arithmetic type of the path: bf16 on the GEMM path; the fused kernels' standard form
    iterates in fp16 (bf16 in and out)."""
    if variant in ("gram", "auto"):
        return "bf16 (Gram form: fp16 m x m side)"
    fused = {small_kernel(b.rows, b.cols) is not None for b in groups}
    if fused == {False}:
        return "bf16"
    return "fp16 (bf16 in/out)" if fused == {True} else "bf16 + fp16 (short sides <= 128)"


def coefficients_desc(args):
    if args.coefficients == "polar-express":
        return (f"polar-express (greedy minimax quintics, singular values in [{args.pe_lower:g}, 1], "
                f"safety {args.pe_safety:g})")
    return "quintic (3.4445, -4.7750, 2.0315) at every step"


def cpu_sample_units(wl, variant):
    """The workload's distinct Newton-Schulz work shapes, one parameter each, with their counts.

    A unit is one parameter of a group (all its head slices); groups whose
    parameters have the same short side, long side, slices per parameter and
    variant cost the oracle the same and share a unit (Llama-8B: q/o, k/v and
    gate/up/down).  Each unit's weight is how many such parameters the
    workload holds.
    """
    units = {}
    for g in wl.groups:
        r, c = g.slice_rows, g.cols
        key = (min(r, c), max(r, c), g.slices // g.count, slice_variant(r, c, variant))
        if key in units:
            units[key][1] += g.count
            units[key][2].append(g.name)
        else:
            units[key] = [g, g.count, [g.name]]
    return [tuple(u) for u in units.values()]


def oracle_unit(wl, g, variant, abc=None):
    """The fp64 oracle's full step on parameter 0 of group g; returns (flops, slices, seconds)."""
    import numpy as np
    import oracle
    import workloads

    G = workloads.gradient(wl, g, 0, 0).float().double().numpy().reshape(g.slices // g.count, g.slice_rows, g.cols)
    W = workloads.initial_weight(wl, g, 0).float().double().numpy().reshape(G.shape)
    M = np.zeros_like(G)
    v = np.zeros(G.shape[:2]) if wl.normuon else None
    sv = slice_variant(g.slice_rows, g.cols, variant)
    t0 = time.perf_counter()
    oracle.muon_step_slices(G, M, W, v, mu=wl.momentum, nesterov=wl.nesterov, ns_eps=wl.ns_eps,
                            ns_steps=wl.ns_steps, abc=abc if abc is not None else oracle.QUINTIC_ABC,
                            variant=sv, restart=GRAM_RESTART if sv == "gram" else 0, normuon=wl.normuon,
                            beta2=wl.beta2, nor_eps=wl.nor_eps, lr=wl.lr, weight_decay=wl.weight_decay,
                            lr_scale=oracle.update_scale(g.rows, g.cols))
    dt = time.perf_counter() - t0
    return G.shape[0] * ns_flops(g.slice_rows, g.cols, variant, wl.ns_steps), G.shape[0], dt


def oracle_rate(units, times):
    """Workload-weighted rate from per-unit oracle times: (flops/s, slices/s) = sum w f / sum w t."""
    flops = sum(w * f for (_, w, _), (f, _, _) in zip(units, times))
    slices = sum(w * sl for (_, w, _), (_, sl, _) in zip(units, times))
    sec = sum(w * t for (_, w, _), (_, _, t) in zip(units, times))
    return flops / sec, slices / sec


def oracle_sample_desc(wl, units):
    names = "; ".join(f"{'/'.join(n)} (x{w})" for (_, w, n) in units)
    return (f"oracle (numpy fp64, full step incl. momentum/NorMuon/update) on ONE parameter of each distinct "
            f"Newton-Schulz shape of {wl.key}: {names}; the rate weights each shape's oracle time by its count "
            f"(an extrapolation from {len(units)} parameter(s) to the whole workload)")


def host_threads():
    import threadpoolctl
    info = threadpoolctl.threadpool_info()
    return max([i.get("num_threads", 1) for i in info] or [1])


def oracle_sample(wl, variant, abc=None):
    """Runs the oracle once on every unit; returns (flops/s, slices/s, seconds, cores, desc)."""
    import threadpoolctl
    units = cpu_sample_units(wl, variant)
    with threadpoolctl.threadpool_limits(limits=os.cpu_count() or 1):
        cores = host_threads()
        times = [oracle_unit(wl, g, variant, abc) for (g, _, _) in units]
    rate, slice_rate = oracle_rate(units, times)
    return rate, slice_rate, sum(t for (_, _, t) in times), cores, oracle_sample_desc(wl, units)


def workload_config(args, wl, variant):
    """The `config` both arms print: what workload, variant and coefficients the metric is on."""
    slices = wl.slices
    return {"workload": DESCRIPTIONS[wl.key], "key": wl.key, "variant": variant,
            "coefficients": coefficients_desc(args), "slices": slices,
            "ns_flop_per_step": sum(g.slices * ns_flops(g.slice_rows, g.cols, variant, wl.ns_steps)
                                    for g in wl.groups),
            "l2": "inputs larger than L2 (126 MB), no flush" if wl.key in ("llama8b", "moe")
            else "inputs smaller than L2: device-resident, no flush (latency-bound configuration)",
            "scale_down": args.scale_down}


# ----------------------------------------------------------------------------- GPU state

def build_state(wl, variant, dev, schedule=None):
    import torch
    import newton_schulz_ns_b200 as mn
    import workloads

    groups = []
    for g in wl.groups:
        n, r, c = g.slices, g.slice_rows, g.cols
        G = torch.empty((g.count, g.rows, g.cols), dtype=wl.grad_dtype, device=dev)
        W = torch.empty((g.count, g.rows, g.cols), dtype=wl.weight_dtype, device=dev)
        for i in range(g.count):
            G[i].copy_(workloads.gradient(wl, g, i, 0, device=dev).reshape(g.rows, g.cols))
            W[i].copy_(workloads.initial_weight(wl, g, i, device=dev).reshape(g.rows, g.cols))
        b = mn.Batch(n, r, c,
                     grad=G.view(n, r, c), momentum=torch.zeros((n, r, c), dtype=wl.mom_dtype, device=dev),
                     ns_in=torch.empty((n, r, c), dtype=torch.bfloat16, device=dev),
                     ns_out=torch.empty((n, r, c), dtype=torch.bfloat16, device=dev),
                     weight=W.view(n, r, c),
                     weight_copy=torch.empty((n, r, c), dtype=torch.bfloat16, device=dev)
                     if wl.weight_copy_bf16 else None,
                     sumsq=torch.zeros(n, dtype=torch.float32, device=dev),
                     variance=torch.zeros(n * r, dtype=torch.float32, device=dev) if wl.normuon else None,
                     row_sumsq=torch.zeros(n * r, dtype=torch.float32, device=dev) if wl.normuon else None,
                     fan_out=g.rows, fan_in=g.cols)
        groups.append(b)
    hp = mn.Hparams(mu=wl.momentum, nesterov=wl.nesterov, ns_eps=wl.ns_eps, ns_steps=wl.ns_steps,
                    abc_schedule=schedule,
                    beta2=wl.beta2, nor_eps=wl.nor_eps, lr=wl.lr, weight_decay=wl.weight_decay)
    ws = mn.allocate_workspace(groups, -1, dev)
    return groups, hp, ws


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons during a region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.proc = None
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", str(gpu_id)],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, power = [], [], []
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
                power.append(float(f[3]))
            except ValueError:
                continue
            for name, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "samples": len(sm),
                "power_w_max": max(power) if power else None, "reasons": sorted(reasons)}


def momentum_bytes(groups):
    """Algorithmic bytes of muon_momentum_norm: read G, M; write M, U (bf16)."""
    tot = 0
    for b in groups:
        e = b.n * b.rows * b.cols
        tot += e * (b.grad.element_size() + 2 * b.momentum.element_size() + 2)
    return tot


def update_bytes(groups, normuon):
    """Algorithmic bytes of normuon_update: read O and W, write W and the bf16 copy.

    With NorMuon the row sums of squares come from the Newton-Schulz call's
    last epilogue (row_sumsq), so O is read once; the per-row statistics
    (a few bytes per row) are not counted.
    """
    tot = 0
    for b in groups:
        e = b.n * b.rows * b.cols
        o_reads = 1 if (not normuon or b.row_sumsq is not None) else 2
        tot += e * (2 * o_reads + 2 * b.weight.element_size() + (2 if b.weight_copy is not None else 0))
    return tot


# ----------------------------------------------------------------------------- replicas

def max_over_ranks(values, device):
    """Element-wise maximum of a list of floats over all ranks (identity on one rank)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def replica_throughput(work_per_rank, world, seconds_max, scale=1e12):
    """Whole-job rate of `world` independent replicas timed by the slowest one."""
    return world * work_per_rank / seconds_max / scale


# ----------------------------------------------------------------------------- our arm

def run_ours(args, wl, variant, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import newton_schulz_ns_b200 as mn

    dev = f"cuda:{local_rank}"
    torch.cuda.set_device(dev)
    schedule = None
    if args.coefficients == "polar-express":
        schedule = mn.polar_express_schedule(args.pe_lower, wl.ns_steps, args.pe_safety)[0]
    groups, hp, ws = build_state(wl, variant, dev, schedule)
    if variant == "auto":
        def ns_fn(g, h, w, s):
            mn.muon_ns_auto_batched(g, h, w, AUTO_GRAM_RATIO, s)
    else:
        ns_fn = mn.muon_ns_batched if variant == "standard" else mn.muon_gram_ns_batched
    stream = torch.cuda.current_stream()

    ns_flop = sum(b.n * ns_flops(b.rows, b.cols, variant, wl.ns_steps) for b in groups)
    slices = sum(b.n for b in groups)

    two_stream = mn.TwoStreamStep(groups, hp, variant, wl.normuon, AUTO_GRAM_RATIO, dev) \
        if args.schedule == "two-stream" else None

    def step(ev=None):
        st = torch.cuda.current_stream()            # the capture stream while a graph is recorded
        if ev is None and two_stream is not None:
            two_stream(st)
            return
        if ev is not None:
            ev[0].record(st)
        mn.muon_momentum_norm(groups, hp, ws, st)
        if ev is not None:
            ev[1].record(st)
        ns_fn(groups, hp, ws, st)
        if ev is not None:
            ev[2].record(st)
        mn.normuon_update(groups, hp, wl.normuon, ws, st)
        if ev is not None:
            ev[3].record(st)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert mn.workspace_error(ws) == 0, "device-side wait timed out"
    if two_stream is not None:
        assert two_stream.workspace_errors() == 0, "device-side wait timed out"

    # ---- device-resident timing
    gpu_id = os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")[local_rank] \
        if os.environ.get("CUDA_VISIBLE_DEVICES") else str(local_rank)
    ns_events = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(4)) for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    graph = None
    if args.graph == "on":
        # One whole step (every kernel of momentum, Newton-Schulz and the
        # update) captured once and replayed: the timed region then measures
        # the device, not the host's enqueue rate.
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            step()
        stream.wait_stream(side)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        l0 = mn.kernel_launches()
        with torch.cuda.graph(graph):
            step()
        per_step_launches = mn.kernel_launches() - l0
        torch.cuda.synchronize()
        for _ in range(2):
            graph.replay()
        torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    clocks = Clocks(gpu_id)
    launches0 = mn.kernel_launches()
    start.record(stream)
    for k in range(args.steps):
        if graph is not None:
            graph.replay()
        else:
            step(ns_events[k])
    end.record(stream)
    torch.cuda.synchronize()
    launches = (per_step_launches * args.steps) if graph is not None else mn.kernel_launches() - launches0
    clk = clocks.stop()
    barrier()
    ms_total = start.elapsed_time(end)
    if graph is not None:
        del graph
        # the per-stage split, from eager steps after the timed region
        for k in range(args.steps):
            step(ns_events[k])
        torch.cuda.synchronize()
    ns_ms = [e[1].elapsed_time(e[2]) for e in ns_events]
    mom_ms = [e[0].elapsed_time(e[1]) for e in ns_events]
    upd_ms = [e[2].elapsed_time(e[3]) for e in ns_events]
    assert mn.workspace_error(ws) == 0, "device-side wait timed out"

    # ---- end to end: gradients H2D from pinned host memory, step, result D2H
    e2e = None
    need = sum(b.grad.numel() * b.grad.element_size() for b in groups)
    try:
        import psutil
        avail = psutil.virtual_memory().available
    except Exception:  # noqa: BLE001
        avail = 0
    e2e_skip = None if avail > 4 * need * max(1, world) else f"host memory {avail/1e9:.0f} GB too small for pinned gradients"
    if not args.no_e2e and e2e_skip is None:
        host_g = [torch.empty(b.grad.shape, dtype=b.grad.dtype, pin_memory=True) for b in groups]
        for h, b in zip(host_g, groups):
            h.copy_(b.grad)
        host_out = [torch.empty(b.n, dtype=torch.float32, pin_memory=True) for b in groups]
        h2d = sum(t.numel() * t.element_size() for t in host_g)
        d2h = sum(t.numel() * t.element_size() for t in host_out)
        # The public calls take a stream, so a caller can overlap the PCIe
        # transfer of one shape's gradients with the optimizer work on the
        # previous shape: copies run on their own stream, and each shape's
        # momentum, Newton-Schulz and update wait only for that shape's copy.
        copy_stream = torch.cuda.Stream(device=dev)
        copied = [torch.cuda.Event() for _ in groups]
        consumed = [torch.cuda.Event() for _ in groups]
        for ev in consumed:
            ev.record(stream)

        def e2e_step():
            for i, (b, h) in enumerate(zip(groups, host_g)):
                copy_stream.wait_event(consumed[i])     # last step's momentum has read this buffer
                with torch.cuda.stream(copy_stream):
                    b.grad.copy_(h, non_blocking=True)
                copied[i].record(copy_stream)
            for i, (b, h) in enumerate(zip(groups, host_out)):
                stream.wait_event(copied[i])
                mn.muon_momentum_norm([b], hp, ws, stream)
                consumed[i].record(stream)
                ns_fn([b], hp, ws, stream)
                mn.normuon_update([b], hp, wl.normuon, ws, stream)
                h.copy_(b.sumsq, non_blocking=True)

        for k in range(2):
            e2e_step()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        copy_stream.wait_event(e0)
        for k in range(args.steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        e2e_ms = e0.elapsed_time(e1)
        e2e = {"ms": e2e_ms, "h2d": h2d, "d2h": d2h}

    # ---- max over ranks
    ms_total, ns_mean, mom_mean, upd_mean, e2e_ms = max_over_ranks(
        [ms_total, statistics.mean(ns_ms), statistics.mean(mom_ms), statistics.mean(upd_ms),
         e2e["ms"] if e2e else 0.0], dev)
    if rank != 0:
        return None

    peaks, src = load_peaks()
    sec = ms_total / 1e3
    value = replica_throughput(ns_flop * args.steps, world, sec)
    ms_step = ms_total / args.steps
    achieved = ns_flop / (ns_mean / 1e3) / 1e12          # per NS call, averaged over the timed steps
    peak_s = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    peak_b = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    out = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": ns_dtype(groups, variant), "data": "synthetic (seeded torch Philox on the device)",
        "config": dict(workload_config(args, wl, variant), parallelism=f"replicas x{world} (no exchange)"),
        "launch": ("CUDA graph of one whole step, replayed for each timed step" if args.graph == "on"
                   else "eager calls"),
        "schedule": ("two streams: per-shape calls, each shape's Newton-Schulz overlapping the next shape's "
                     "momentum and the previous shape's NorMuon + update (TwoStreamStep); the per-stage split "
                     "in ms_breakdown comes from serial eager steps" if two_stream is not None
                     else "serial: one call per stage over every shape"),
        "pct_bf16_peak": round(100 * value / world / peak_s, 2),
        "pct_bf16_peak_burst": round(100 * value / world / peak_b, 2),
        "matrices_per_s": round(world * slices * args.steps / sec, 2),
        "ms_breakdown": {"momentum_norm": round(mom_mean, 3), "ns": round(ns_mean, 3),
                         "normuon_update": round(upd_mean, 3)},
        "hbm_kernels": {"momentum_gbs": round(momentum_bytes(groups) / (mom_mean / 1e3) / 1e9, 1),
                        "update_gbs": round(update_bytes(groups, wl.normuon) / (upd_mean / 1e3) / 1e9, 1),
                        "peak_gbs": peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]),
                        "peak_source": src["hbm_gbs"]},
        "roofline": {"bound": "tensor", "kernel": ns_kernels_label(groups),
                     "achieved": round(achieved, 2), "peak": peak_s, "unit": "TFLOP/s",
                     "frac": round(achieved / peak_s, 4), "frac_of_burst": round(achieved / peak_b, 4),
                     "peak_source": f"{src['bf16_tflops_sustained']} bf16_tflops_sustained (kernel timed inside a long "
                                    f"step)",
                     "traffic": measured_traffic(wl.key, variant) if args.scale_down == 1 else None,
                     "traffic_unit": "bytes per Newton-Schulz call: ncu dram__bytes_read.sum + write.sum of "
                                     "one-layer launches, scaled by the slices and steps of one call "
                                     f"(profiles/ns_gemm_{wl.key}_{variant}_traffic_scaled.md)"},
        "gpu_launches": int(launches),
        "clocks": clk,
    }
    if e2e_skip:
        out["e2e"] = {"value": None, "unit": "TFLOP/s", "skipped": e2e_skip}
    if e2e:
        out["e2e"] = {"value": round(replica_throughput(ns_flop * args.steps, world, e2e_ms / 1e3), 3),
                      "unit": "TFLOP/s",
                      "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                      "ms_per_step": round(e2e_ms / args.steps, 3),
                      "path": "public C-ABI calls per shape on one stream; each shape's gradients copied H2D "
                              "from pinned host memory on a second stream (overlapping the previous shape's "
                              "optimizer work) and its per-slice norms read back D2H, all inside the timed region"}
    if world == 1 and not args.no_cpu_baseline:
        rate, slice_rate, dt, cores, desc = oracle_sample(wl, variant, abc=oracle_schedule(args, wl))
        out["cpu_baseline"] = {"value": round(rate / 1e12, 6), "unit": "TFLOP/s", "cores": cores,
                               "kind": "oracle", "sample": desc, "seconds": round(dt, 2),
                               "matrices_per_s": round(slice_rate, 4)}
    return out


# ----------------------------------------------------------------------------- reference arm

def oracle_schedule(args, wl):
    """The oracle's own coefficients for the run (its linear-programming schedule for Polar Express)."""
    if args.coefficients != "polar-express":
        return None
    import oracle
    return oracle.polar_express_lp(args.pe_lower, wl.ns_steps, args.pe_safety)[0]


def run_reference(args, wl, variant):
    """The oracle on the host cores: step j runs the oracle on unit j mod U of the workload's sample
    (one parameter of each distinct shape), so every step stays a few seconds; the rate weights the
    units' mean times by their counts, as the cpu_baseline of the other arm does."""
    import threadpoolctl
    peaks, _ = load_peaks()
    abc = oracle_schedule(args, wl)
    units = cpu_sample_units(wl, variant)
    per_unit = [[] for _ in units]
    step_s = []
    with threadpoolctl.threadpool_limits(limits=os.cpu_count() or 1):
        cores = host_threads()
        for k in range(args.warmup + args.steps):
            u = (k - args.warmup) % len(units) if k >= args.warmup else k % len(units)
            res = oracle_unit(wl, units[u][0], variant, abc)
            if k >= args.warmup:
                per_unit[u].append(res)
                step_s.append(res[2])
        for u in range(len(units)):          # fewer timed steps than units: time the rest once
            if not per_unit[u]:
                per_unit[u].append(oracle_unit(wl, units[u][0], variant, abc))
    means = [(r[0][0], r[0][1], statistics.mean(x[2] for x in r)) for r in per_unit]
    rate, slice_rate = oracle_rate(units, means)
    value = rate / 1e12
    desc = oracle_sample_desc(wl, units) + f"; step j times unit j mod {len(units)}"
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * statistics.mean(step_s), 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(workload_config(args, wl, variant), parallelism=f"replicas x{args.gpus} (no exchange)"),
        "pct_bf16_peak": round(100 * value / peaks.get("bf16_tflops_sustained", 1400.0), 6),
        "matrices_per_s": round(slice_rate, 4),
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    import workloads
    wl = workloads.WORKLOADS[args.workload]
    if args.scale_down > 1:
        wl = workloads.scaled(wl, args.scale_down)
    variant = args.variant or default_variant(wl)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, wl, variant)), flush=True)
        return 0

    if args.warmup < 3:
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device(f"cuda:{local_rank}"))
    try:
        out = run_ours(args, wl, variant, rank, world, local_rank)
        if out is not None:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
