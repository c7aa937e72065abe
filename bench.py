#!/usr/bin/env python
"""Benchmark: expert-FFN HBM GB/s at batch-1 decode (MXFP4 DeepSeek-V4-Flash
MoE layer: 256 experts, top-6, hidden 4096, intermediate 2048, 1 token).

    python bench.py [--gpus N --steps K --warmup W] [--impl ours|reference]

A step is one pass of the hot path over one decode token of one layer:
router (softmax top-6) + routed-expert FFN (gate/up, SwiGLU, down, weighted
combine).  Steps rotate over `--layers` distinct resident layers (16 x 3.42 GB
by default), so each step's six experts are cold in L2 (inputs larger than L2).
The timed region replays pre-captured CUDA graphs (one router graph, one FFN
graph per layer); CUDA events bracket every FFN call for the roofline.

`value` = algorithmic bytes (the six selected experts' packed bytes, read
once) x steps / device time, summed over ranks (one independent replica per
GPU, weak scaling).  `e2e` repeats the measurement through the C ABI with
pinned host buffers and the host<->device copies inside the timed region.
`--impl reference` times the CPU oracle on the same workload and metric.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import re
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "expert-FFN HBM GB/s (% of peak) at bs=1 decode; prefill tokens/s per MoE layer"
WORKLOAD = "decode_mx"
WORKLOAD_DESC = ("decode MoE layer: 256 experts, top-6, hidden 4096, intermediate 2048, "
                 "batch 1, MXFP4 gate/up/down (e8m0 exponents 2^-9..2^0), bf16 N(0,1) "
                 "activations, softmax top-6 router")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=100)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--layers", type=int, default=16)
    ap.add_argument("--e2e-steps", type=int, default=2000)
    ap.add_argument("--cpu-sample-s", type=float, default=15.0)
    ap.add_argument("--reference-budget-s", type=float, default=150.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--prefill-steps", type=int, default=20,
                    help="timed repetitions of the 2048-token prefill layer (0: skip)")
    ap.add_argument("--prefill-experts", type=int, default=0,
                    help="profiling only: fewer experts in the prefill layer (0: the workload's 256)")
    ap.add_argument("--prefill-tokens", type=int, default=0,
                    help="profiling only: fewer prefill tokens (0: the workload's 2048)")
    ap.add_argument("--prefill-act", choices=["none", "e4m3", "mxfp4"], default="none",
                    help="activation mode of the prefill layer (default: bf16 activations)")
    ap.add_argument("--extra", choices=["all", "none"], default="all",
                    help="the other configurations' objects: NVFP4 decode at 1/4/16 tokens, the 43-layer "
                         "stack, the 16,384-token prefill layer and the W4A8 prefill layer")
    ap.add_argument("--stack-steps", type=int, default=5, help="timed passes over the 43-layer stack")
    return ap.parse_args()


# ------------------------------------------------------------------ clocks --
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML (read-only)."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x2: "applications_clocks_setting", 0x1: "gpu_idle"}

    def __init__(self, dev_index: int, period_s: float = 0.01):
        self.samples, self.reasons, self.ok = [], set(), False
        self.period = period_s
        self._stop = threading.Event()
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self.nv = pynvml
            p = torch.cuda.get_device_properties(dev_index)
            try:
                bus = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(dev_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def _reasons(self):
        try:
            return self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            return self.nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)

    def _one(self):
        self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
        r = self._reasons()
        for bit, name in self.REASONS.items():
            if r & bit and name != "gpu_idle":
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            self._one()
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._one()
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def stop(self):
        if self.ok:
            self._stop.set()
            self.t.join()
            self._one()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def _code_only(text: str) -> str:
    """Source text without comments and blank lines: what the compiler sees
    (string literals in these files hold no comment markers)."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(l.rstrip() for l in text.splitlines() if l.strip())


# The decode kernels' code: the kernel file first, then the headers it includes.
DECODE_KERNEL_FILES = ("qk_dmx.cu", "qk_group.cuh", "qk_route_table.cuh", "qk_device.cuh", "qk_common.cuh",
                       "qk_internal.h", "qk_tmap.h")


def kernel_source_hash() -> str:
    """Hash of the decode kernels' code (the kernel file and the headers it
    includes, comments excluded): a recorded DRAM traffic figure stays valid
    while the code it was measured on is unchanged."""
    from block_quantized_expert_mxfp4_b200 import build as b
    h = hashlib.sha256()
    for n in DECODE_KERNEL_FILES:
        h.update(_code_only(open(os.path.join(b.CSRC, n)).read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic():
    """dram bytes per FFN call from the committed ncu summary, if it was taken
    on the current kernel sources (else None)."""
    try:
        with open(os.path.join(ROOT, "profiles", "decode_mx_traffic.json")) as f:
            d = json.load(f)
        if d.get("kernel_source_hash") == kernel_source_hash():
            return d["dram_bytes_per_forward"]
    except Exception:
        pass
    return None


# -------------------------------------------------------------- CPU oracle --
def max_over_ranks(seconds: float, world: int, dev) -> float:
    """The job's time: the largest of the ranks' device times (every rank
    calls this at the same point; world 1 returns its own)."""
    import torch
    t = torch.tensor([seconds], dtype=torch.float64, device=dev)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def oracle_sample(seconds: float, max_steps: int = 1 << 30):
    """Time the CPU oracle on (token, expert) pairs of the decode workload.
    Returns (bytes, seconds, steps, threads)."""
    import numpy as np
    import oracle
    from block_quantized_expert_mxfp4_b200 import synth

    oracle.build()
    wl = synth.WORKLOADS[WORKLOAD]
    lg = synth.router_logits(7, 64, wl.E, stream=99)
    x = synth.activations(7, 64, wl.H, stream=99)
    ids, _ = oracle.route_topk(lg, wl.k)
    per_pair = 3 * (wl.I * wl.H // 2 + wl.I * wl.H // 32)
    done, t_used, steps = 0, 0.0, 0
    cache = {}
    while t_used < seconds and steps < max_steps:
        t, s = divmod(steps, wl.k)
        t %= 4  # the experts of 4 tokens (24 pairs) are generated once, then reused
        e = int(ids[t, s])
        if e not in cache:
            ws = []
            for pi, (rows, cols) in enumerate(((wl.I, wl.H), (wl.I, wl.H), (wl.H, wl.I))):
                q, sc = synth.mx_expert_bytes(0, 0, pi, rows, cols, wl.code_lo, wl.code_hi, [e],
                                              wl.E)
                ws.append(oracle.Weight(oracle.MXFP4, q, sc))
            cache[e] = oracle.Layer(*ws)
        L = cache[e]
        t0 = time.perf_counter()
        oracle.route_topk(lg[t:t + 1], wl.k)
        oracle.expert_ffn(L, 0, x[t])
        t_used += time.perf_counter() - t0
        done += per_pair
        steps += 1
    return done, t_used, steps, oracle.get_threads()


# ------------------------------------------------------------------ ours --
def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import block_quantized_expert_mxfp4_b200 as qk
    from block_quantized_expert_mxfp4_b200 import build as qk_build, synth, workload

    qk_build.build()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = synth.WORKLOADS[WORKLOAD]
    T, k = wl.T, wl.k
    L = args.layers
    layers = [workload.make_layer(wl, seed=rank, layer=l) for l in range(L)]
    expert_bytes = layers[0].expert_bytes()
    bytes_per_step = k * T * expert_bytes if T == 1 else None  # T=1: k distinct experts

    # per-slot inputs and outputs (distinct token per slot)
    xs = [synth.activations(rank, T, wl.H, stream=l).to(dev) for l in range(L)]
    lgs = [synth.router_logits(rank, T, wl.E, stream=l).to(dev) for l in range(L)]
    ids = [torch.empty((T, k), dtype=torch.int32, device=dev) for _ in range(L)]
    ws_ = [torch.empty((T, k), dtype=torch.float32, device=dev) for _ in range(L)]
    ys = [torch.empty((T, wl.H), dtype=torch.float32, device=dev) for _ in range(L)]
    lays = [lay.c() for lay in layers]
    wsp = torch.empty(qk.moe_expert_workspace_size(lays[0], T, k), dtype=torch.uint8, device=dev)

    def route(l, stream=None):
        qk.moe_route_topk(lgs[l], k, ids[l], ws_[l], stream)

    def ffn(l, stream=None):
        qk.moe_expert_forward(lays[l], xs[l], ids[l], ws_[l], ys[l], wsp, stream=stream)

    # warm-up eagerly (sets kernel attributes), then capture graphs
    for l in range(L):
        route(l)
        ffn(l)
    torch.cuda.synchronize()
    if qk.qk_last_device_status() != qk.QK_OK:
        raise RuntimeError("device status after warm-up")
    s = torch.cuda.Stream(device=dev)
    # G_all: L steps back to back (the throughput region); g_step[l]: one step;
    # G_ev: L steps with external event nodes bracketing every FFN call.
    ev_a = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(L)]
    ev_b = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(L)]
    G_all, G_ev, g_step = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph(), []
    with torch.cuda.stream(s):
        with torch.cuda.graph(G_all, stream=s):
            for l in range(L):
                route(l)
                ffn(l)
        with torch.cuda.graph(G_ev, stream=s):
            for l in range(L):
                route(l)
                ev_a[l].record(s)
                ffn(l)
                ev_b[l].record(s)
        for l in range(L):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                route(l)
                ffn(l)
            g_step.append(g)
    torch.cuda.synchronize()

    K, W = args.steps, max(3, args.warmup)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local_rank)
    with torch.cuda.stream(s):
        for i in range(W):
            g_step[i % L].replay()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        clocks.start()
        torch.cuda._sleep(20_000_000)  # lets the host queue ahead of the GPU (untimed)
        ev0.record(s)
        for _ in range(K // L):
            G_all.replay()
        for i in range(K % L):
            g_step[i].replay()
        ev1.record(s)
        torch.cuda.synchronize()
        clocks.stop()
        # roofline region: per-call device time of the FFN (events inside the graph)
        ffn_ms = []
        for _ in range(max(1, min(K, 2048) // L)):
            G_ev.replay()
            torch.cuda.synchronize()
            ffn_ms += [a.elapsed_time(b) for a, b in zip(ev_a, ev_b)]
    if world > 1:
        dist.barrier()
    st = qk.qk_last_device_status()
    if st != qk.QK_OK:
        raise RuntimeError(f"device status {qk.status_string(st)}")
    elapsed = ev0.elapsed_time(ev1) / 1e3
    ffn_s = statistics.fmean(ffn_ms) / 1e3
    elapsed_max = max_over_ranks(elapsed, world, dev)
    total_bytes = bytes_per_step * K * world
    value = total_bytes / elapsed_max / 1e9

    # ---- e2e through the C ABI with pinned host buffers
    E2 = min(args.e2e_steps, K)
    xh = [synth.activations(rank, T, wl.H, stream=1000 + i % 64).pin_memory() for i in range(64)]
    lh = [synth.router_logits(rank, T, wl.E, stream=1000 + i % 64).pin_memory() for i in range(64)]
    yh = torch.empty((T, wl.H), dtype=torch.float32).pin_memory()
    xd, ld = xs[0].clone(), lgs[0].clone()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s):
        for i in range(3):
            xd.copy_(xh[i], non_blocking=True)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0.record(s)
        for i in range(E2):
            l = i % L
            xd.copy_(xh[i % 64], non_blocking=True)
            ld.copy_(lh[i % 64], non_blocking=True)
            qk.moe_route_topk(ld, k, ids[l], ws_[l], s)
            qk.moe_expert_forward(lays[l], xd, ids[l], ws_[l], ys[l], wsp, stream=s)
            yh.copy_(ys[l], non_blocking=True)
        e1.record(s)
        torch.cuda.synchronize()
    e2e_value = bytes_per_step * E2 * world / max_over_ranks(e0.elapsed_time(e1) / 1e3, world, dev) / 1e9

    peak, peak_kind = peaks()
    achieved = bytes_per_step / ffn_s / 1e9
    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": K, "warmup": W, "ms_per_step": round(elapsed_max / K * 1e3, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e2m1 x e8m0 weights, activations as e4m3 terms x ue8m0 (block-scaled MMA), f32 accumulate",
        "data": "synthetic (seeded; random-init MXFP4 weights of the DeepSeek-V4-Flash expert shape)",
        "config": {"workload": WORKLOAD_DESC, "layers_resident": L,
                   "resident_weight_GB": round(L * wl.E * expert_bytes / 1e9, 2),
                   "bytes_per_step": bytes_per_step,
                   "l2": "inputs larger than L2: steps rotate over the resident layers",
                   "parallelism": f"replicas x{world}"},
        "roofline": {"kernel": "moe_expert_forward (k_dmx gate/up -> k_dmx down -> k_dmx_y combine, "
                               "block-scaled tcgen05, PDL-chained)",
                     "bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "frac_of_nominal_8tbs": round(achieved / 8000.0, 4),
                     "ffn_us": round(ffn_s * 1e6, 3), "ffn_calls_timed": len(ffn_ms),
                     "traffic": recorded_traffic()},
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s",
                "h2d_bytes_per_step": T * wl.H * 2 + T * wl.E * 4,
                "d2h_bytes_per_step": T * wl.H * 4, "steps": E2},
        "gpu_launches": 4 * K,  # route, gate/up, down, y
        "clocks": clocks.summary(),
    }
    del layers, lays
    torch.cuda.empty_cache()
    if args.prefill_steps > 0:
        out["prefill"] = run_prefill(args, rank, world, dev)
        # count, two tile-list scans, x split, gate/up GEMM (+ SwiGLU and the h split), down GEMM, combine
        out["gpu_launches"] += out["prefill"]["gpu_launches"]
    if args.extra == "all":
        # the other configurations, each timed in its own region (not part of `value`)
        out["decode_nvfp4"] = run_decode_nv(args, rank, world, dev)
        out["stack43"] = run_stack(args, rank, world, dev)
        out["prefill_16k"] = run_prefill(args, rank, world, dev, tokens=16384, steps=3)
        out["prefill_w4a8"] = run_prefill(args, rank, world, dev, act="e4m3", steps=10)
        out["prefill_w4a4"] = run_prefill(args, rank, world, dev, act="mxfp4", steps=10)
        out["prefill_w4a4_16k"] = run_prefill(args, rank, world, dev, tokens=16384, act="mxfp4", steps=3)
        out["prefill_w4a4_nvfp4"] = run_prefill(args, rank, world, dev, act="mxfp4", steps=10, nv=True)
        out["prefill_w4a4_nvfp4_16k"] = run_prefill(args, rank, world, dev, tokens=16384, act="mxfp4", steps=3,
                                                    nv=True)
        out["shared_fp8_prefill"] = run_shared_fp8(args, rank, world, dev)
        try:  # reported, never fatal to the line
            out["convert"] = run_convert(args, rank, world, dev)
        except Exception as e:  # noqa: BLE001
            out["convert"] = {"error": f"{type(e).__name__}: {e}", "gpu_launches": 0}
        for key in ("decode_nvfp4", "stack43", "prefill_16k", "prefill_w4a8", "prefill_w4a4", "prefill_w4a4_16k",
                    "prefill_w4a4_nvfp4", "prefill_w4a4_nvfp4_16k", "shared_fp8_prefill", "convert"):
            out["gpu_launches"] += out[key]["gpu_launches"]
    return out


def _graph_time(fn, K, world, dev, reps_warm=3):
    """Seconds per replay of a CUDA graph of fn() (CUDA events on its stream,
    after warm-up replays; max over ranks)."""
    import torch
    import torch.distributed as dist
    s = torch.cuda.Stream(device=dev)
    fn(None)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            fn(s)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s):
        for _ in range(reps_warm):
            g.replay()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0.record(s)
        for _ in range(K):
            g.replay()
        e1.record(s)
        torch.cuda.synchronize()
    t = max_over_ranks(e0.elapsed_time(e1) / 1e3 / K, world, dev)
    del g
    return t


def run_convert(args, rank, world, dev):
    """The scale-only conversions on the decode layer's three projections
    (256 experts; gate and up 2048 x 4096, down 4096 x 2048): MXFP4 -> NVFP4
    (e8m0 per 32 in, e4m3 per 16 and scale_2 out) and back; GB/s on the
    bytes read and written, against the measured HBM rate."""
    import torch

    import block_quantized_expert_mxfp4_b200 as qk
    from block_quantized_expert_mxfp4_b200 import synth, workload

    wl = synth.WORKLOADS["decode_mx"]
    layer = workload.make_layer(wl, rank, 0)
    projs = (layer.gate, layer.up, layer.down)
    e4 = [torch.empty((p.scales.shape[0], p.scales.shape[1], 2 * p.scales.shape[2]), dtype=torch.uint8,
                      device=dev) for p in projs]
    s2 = [torch.empty(p.scales.shape[0], dtype=torch.float32, device=dev) for p in projs]
    back = [torch.empty_like(p.scales) for p in projs]
    bad = torch.zeros(1, dtype=torch.int64, device=dev)
    peak, peak_kind = peaks()
    res = {"workload": "scale-only conversions of the decode layer's three projections (256 experts, "
                       "hidden 4096, intermediate 2048; e8m0 codes uniform in 118..127)",
           "peak_gbs": peak, "peak_kind": peak_kind}
    K = 10
    for name, fn, nbytes in (
            ("mxfp4_to_nvfp4", lambda i: qk.quant_convert_mxfp4_to_nvfp4(projs[i].scales, e4[i], s2[i], bad),
             sum(p.scales.numel() * 3 + p.scales.shape[0] * 4 for p in projs)),
            ("nvfp4_to_mxfp4", lambda i: qk.quant_convert_nvfp4_to_mxfp4(e4[i], s2[i], back[i], bad),
             sum(p.scales.numel() * 3 + p.scales.shape[0] * 4 for p in projs))):
        for _ in range(2):
            for i in range(3):
                fn(i)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(K):
            for i in range(3):
                fn(i)
        e1.record()
        torch.cuda.synchronize()
        t = max_over_ranks(e0.elapsed_time(e1) / 1e3 / K, world, dev)
        res[name] = {"us_per_layer": round(t * 1e6, 2), "bytes_per_layer": int(nbytes),
                     "achieved_gbs": round(nbytes / t / 1e9, 1), "frac": round(nbytes / t / 1e9 / peak, 4)}
    if qk.qk_last_device_status() != qk.QK_OK:
        raise RuntimeError("device status after the conversions")
    res["round_trip_identity"] = bool(all(torch.equal(b, p.scales) for b, p in zip(back, projs)))
    res["gpu_launches"] = 2 * (2 + K) * 3
    return res


def run_shared_fp8(args, rank, world, dev):
    """The FP8 E4M3 block-128 shared expert (4096 x 2048 SwiGLU) at prefill
    sizes (2048 and 16,384 rows), added into y: the block-scaled grouped
    GEMMs; tensor rate on the useful FLOPs and HBM rate on its bytes."""
    import torch

    import block_quantized_expert_mxfp4_b200 as qk
    from block_quantized_expert_mxfp4_b200 import synth, workload

    H, I = 4096, 2048
    sh = workload.make_fp8_shared(rank, 0, H, I, device=dev)
    peak, peak_kind = peaks()
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            bf16, src = float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        bf16, src = 1590.0, "fallback"
    res = {"workload": "FP8 E4M3 shared expert, hidden 4096, intermediate 2048, UE8M0 per 128x128 tile, "
                       "bf16 N(0,1) activations, result added into y",
           "path": "one group of M tokens on the block-scaled grouped GEMMs: x as 2 exact e4m3 terms, "
                   "e4m3 weights as stored (kind::mxf8f6f4), SwiGLU + 3-term h split in the gate/up epilogue, "
                   "add into y",
           "tensor_peak_tflops": 2 * bf16,
           "tensor_peak_kind": f"{src} bf16 x 2 (nominal fp8/bf16 ratio): kind::mxf8f6f4",
           "by_rows": {}}
    launches = 0
    for M in (2048, 16384):
        x = synth.activations(rank + 7, M, H).to(dev)
        y = torch.zeros((M, H), dtype=torch.float32, device=dev)
        ws = torch.empty(qk.fp8_shared_expert_workspace_size(M, H, I), dtype=torch.uint8, device=dev)

        def step(st):
            qk.fp8_shared_expert_forward(x, sh.wg, sh.sg, sh.wu, sh.su, sh.wd, sh.sd, y, ws, stream=st)
        K = 10
        t = _graph_time(step, K, world, dev)
        if qk.qk_last_device_status() != qk.QK_OK:
            raise RuntimeError("device status after the shared expert")
        flops = 2 * 3 * H * I * M
        res["by_rows"][str(M)] = {"ms": round(t * 1e3, 4), "rows_per_s": round(M * world / t, 1),
                                  "achieved_tflops": round(flops / t / 1e12, 1),
                                  "tensor_frac": round(flops / t / 1e12 / (2 * bf16), 4),
                                  "weight_bytes": sh.nbytes(), "hbm_frac": round(sh.nbytes() / t / 1e9 / peak, 4)}
        launches += K * 8  # route fill, count, two scans, x split, gate/up (+ h split), down, combine
        del x, y, ws
    res["gpu_launches"] = launches
    return res


def run_decode_nv(args, rank, world, dev):
    """The decode MoE layer in NVFP4 (the MXFP4 layer converted scale-only:
    e4m3 block scales per 16 and an fp32 scale_2 per expert) at 1, 4 and 16
    tokens: the FFN call alone, rotating over 4 resident layers."""
    import torch

    import block_quantized_expert_mxfp4_b200 as qk
    from block_quantized_expert_mxfp4_b200 import synth, workload

    wl = synth.WORKLOADS["decode_nv"]
    L = 4
    layers = [workload.make_layer(wl, seed=rank, layer=l) for l in range(L)]
    lays = [ly.c() for ly in layers]
    peak, peak_kind = peaks()
    res = {"workload": "decode MoE layer in NVFP4 (256 experts, top-6, hidden 4096, intermediate 2048; "
                       "e2m1 + e4m3 per 16 + fp32 scale_2, from the seeded MXFP4 layer by the scale-only "
                       "conversion), softmax top-6 router, bf16 N(0,1) activations",
           "layers_resident": L, "peak_gbs": peak, "peak_kind": peak_kind, "by_tokens": {}}
    launches = 0
    for T in (1, 4, 16):
        xs, ids_, ws_, nbytes = [], [], [], 0
        for l in range(L):
            x = synth.activations(rank * 131 + l, T, wl.H).to(dev)
            lg = synth.router_logits(rank * 131 + l, T, wl.E).to(dev)
            ids = torch.empty((T, wl.k), dtype=torch.int32, device=dev)
            w = torch.empty((T, wl.k), dtype=torch.float32, device=dev)
            qk.moe_route_topk(lg, wl.k, ids, w)
            xs.append(x), ids_.append(ids), ws_.append(w)
            nbytes += int(torch.unique(ids).numel()) * layers[l].expert_bytes()
        y = torch.empty((T, wl.H), dtype=torch.float32, device=dev)
        wsp = torch.empty(qk.moe_expert_workspace_size(lays[0], T, wl.k), dtype=torch.uint8, device=dev)
        reps = 10

        def step(st):
            for _ in range(reps):
                for l in range(L):
                    qk.moe_expert_forward(lays[l], xs[l], ids_[l], ws_[l], y, wsp, stream=st)
        t = _graph_time(step, 20, world, dev) / (reps * L)
        if qk.qk_last_device_status() != qk.QK_OK:
            raise RuntimeError("device status after the NVFP4 decode layer")
        b = nbytes / L
        res["by_tokens"][str(T)] = {"us_per_call": round(t * 1e6, 3), "bytes_per_call": int(b),
                                    "achieved_gbs": round(b / t / 1e9, 1), "frac": round(b / t / 1e9 / peak, 4),
                                    "tokens_per_s": round(T * world / t, 1)}
        launches += 20 * reps * L * 3  # gate/up, down and y kernels (f16 decode path) per call
    res["gpu_launches"] = launches
    res["path"] = "f16 decode kernels (k_decode: e2m1 and e4m3 scales decoded in registers, m16n8k16 MMA)"
    del layers, lays
    torch.cuda.empty_cache()
    return res


def run_stack(args, rank, world, dev):
    """The pruned 43-layer expert stack at 8 tokens: per layer the router, the
    routed experts (180 per layer, top-6, each projection's format drawn per
    layer) and the FP8 block-128 shared expert added into the same output;
    all 43 layers resident, one step = one pass over the stack."""
    import torch

    import block_quantized_expert_mxfp4_b200 as qk
    from block_quantized_expert_mxfp4_b200 import synth, workload

    wl = synth.WORKLOADS["stack43"]
    fm = synth.format_choice(rank, wl.layers)
    layers = [workload.make_layer(wl, rank, l, tuple(int(f) for f in fm[l])) for l in range(wl.layers)]
    lays = [ly.c() for ly in layers]
    shared = [workload.make_fp8_shared(rank, l, wl.H, wl.I, device=dev) for l in range(wl.layers)]
    T, k = wl.T, wl.k
    xs, lgs, ids_, ws_, ys = [], [], [], [], []
    nbytes = 0
    for l in range(wl.layers):
        xs.append(synth.activations(rank, T, wl.H, stream=l).to(dev))
        lgs.append(synth.router_logits(rank, T, wl.E, stream=l).to(dev))
        ids_.append(torch.empty((T, k), dtype=torch.int32, device=dev))
        ws_.append(torch.empty((T, k), dtype=torch.float32, device=dev))
        ys.append(torch.empty((T, wl.H), dtype=torch.float32, device=dev))
        qk.moe_route_topk(lgs[l], k, ids_[l], ws_[l])
        nbytes += int(torch.unique(ids_[l]).numel()) * layers[l].expert_bytes() + shared[l].nbytes()
    wsp = torch.empty(max(qk.moe_expert_workspace_size(ly, T, k) for ly in lays), dtype=torch.uint8, device=dev)
    wss = torch.empty(qk.fp8_shared_expert_workspace_size(T, wl.H, wl.I), dtype=torch.uint8, device=dev)

    def step(st):
        for l in range(wl.layers):
            qk.moe_route_topk(lgs[l], k, ids_[l], ws_[l], stream=st)
            qk.moe_expert_forward(lays[l], xs[l], ids_[l], ws_[l], ys[l], wsp, stream=st)
            sh = shared[l]
            qk.fp8_shared_expert_forward(xs[l], sh.wg, sh.sg, sh.wu, sh.su, sh.wd, sh.sd, ys[l], wss, stream=st)
    K = args.stack_steps
    t = _graph_time(step, K, world, dev)
    if qk.qk_last_device_status() != qk.QK_OK:
        raise RuntimeError("device status after the stack")
    peak, peak_kind = peaks()
    mixed = [sum(int(f == 1) for f in fm[l]) for l in range(wl.layers)]
    res = {"workload": f"pruned 43-layer expert stack: 180 experts per layer, top-6, hidden 4096, intermediate "
                       f"2048, {T} tokens; per layer and projection a seeded MXFP4 or NVFP4 format "
                       f"({sum(m == 3 for m in mixed)} layers all-MXFP4); FP8 E4M3 block-128 UE8M0 shared "
                       "expert 4096x2048 SwiGLU per layer",
           "ms_per_step": round(t * 1e3, 4), "tokens_per_s": round(T * world / t, 1), "steps": K,
           "bytes_per_step": nbytes, "achieved_gbs": round(nbytes / t / 1e9, 1), "peak_gbs": peak,
           "peak_kind": peak_kind, "frac": round(nbytes / t / 1e9 / peak, 4),
           "hbm_floor_ms": round(nbytes / peak / 1e6, 4),
           "gpu_launches": K * wl.layers * 6}  # router, routed gate/up, down and y, shared gate/up and down
    del layers, lays, shared
    torch.cuda.empty_cache()
    return res


def run_prefill(args, rank, world, dev, tokens=0, act=None, steps=0, nv=False):
    """The 2048-token Zipf prefill layer through moe_expert_forward (grouped
    path): tokens/s, HBM fraction on the touched experts' bytes, tensor rate.
    `tokens`, `act` and `steps` override the command line's choices; `nv`
    converts the layer to NVFP4 (scale-only conversion of the seeded MXFP4
    layer)."""
    import torch
    import torch.distributed as dist

    import block_quantized_expert_mxfp4_b200 as qk
    from block_quantized_expert_mxfp4_b200 import synth, workload

    wl = synth.WORKLOADS["prefill"]
    if args.prefill_experts or args.prefill_tokens or tokens:
        import dataclasses
        wl = dataclasses.replace(wl, E=args.prefill_experts or wl.E, T=tokens or args.prefill_tokens or wl.T)
    T, k = wl.T, wl.k
    act_name = act or args.prefill_act
    aq = {"none": qk.QK_ACT_NONE, "e4m3": qk.QK_ACT_E4M3, "mxfp4": qk.QK_ACT_MXFP4}[act_name]
    fmts = (qk.QK_FMT_NVFP4,) * 3 if nv else None
    layer = workload.make_layer(wl, seed=rank, layer=0, fmts=fmts)
    lay = layer.c()
    x = synth.activations(rank, T, wl.H).to(dev)
    lg = synth.zipf_logits(rank, T, wl.E, k).to(dev)
    ids = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), dtype=torch.float32, device=dev)
    qk.moe_route_topk(lg, k, ids, w)
    y = torch.empty((T, wl.H), dtype=torch.float32, device=dev)
    wsp = torch.empty(qk.moe_expert_workspace_size(lay, T, k, aq), dtype=torch.uint8, device=dev)
    touched = int(torch.unique(ids).numel())
    wbytes = touched * layer.expert_bytes()
    flops = 2 * 3 * wl.H * wl.I * T * k
    s = torch.cuda.Stream(device=dev)
    for _ in range(3):
        qk.moe_expert_forward(lay, x, ids, w, y, wsp, act_quant=aq)
    torch.cuda.synchronize()
    if qk.qk_last_device_status() != qk.QK_OK:
        raise RuntimeError("device status after prefill warm-up")
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            qk.moe_expert_forward(lay, x, ids, w, y, wsp, act_quant=aq, stream=s)
    torch.cuda.synchronize()
    K = steps or args.prefill_steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s):
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0.record(s)
        for _ in range(K):
            g.replay()
        e1.record(s)
        torch.cuda.synchronize()
    t = max_over_ranks(e0.elapsed_time(e1) / 1e3 / K, world, dev)
    if qk.qk_last_device_status() != qk.QK_OK:
        raise RuntimeError("device status after prefill")
    peak, peak_kind = peaks()
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            bf16, src = float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        bf16, src = 1590.0, "fallback"
    # The grouped GEMMs run kind::mxf8f6f4 (twice the bf16 rate, nominal ratio);
    # FP4 (kind::mxf4, four times) is the format's own ceiling.  `flops` is the
    # layer's useful work; the activation terms multiply the MMAs issued (2 for
    # gate/up, 3 for down) but not the work.
    if aq == qk.QK_ACT_MXFP4:  # both operands e2m1: kind::mxf4 (mxf4nvf4), four times the bf16 rate
        kind = "kind::mxf4nvf4" if nv else "kind::mxf4"
        tpeak, tkind = 4 * bf16, f"{src} bf16 x 4 (nominal fp4/bf16 ratio): the MMA kind used, {kind}"
    else:
        tpeak, tkind = 2 * bf16, f"{src} bf16 x 2 (nominal fp8/bf16 ratio): the MMA kind used, kind::mxf8f6f4"
    return {
        "workload": f"prefill MoE layer: {T} tokens, {wl.E} experts, top-6 Zipf(s=1) routing, hidden 4096, "
                    + ("intermediate 2048, NVFP4 gate/up/down (scale-only conversion of the seeded MXFP4 layer), "
                       if nv else "intermediate 2048, MXFP4 gate/up/down, ")
                    + "bf16 N(0,1) activations"
                    + ("" if aq == qk.QK_ACT_NONE else f", quantized in the layer to {act_name}"
                       " (one e8m0 scale per 32)"),
        "tokens_per_s": round(T * world / t, 1), "ms_per_layer": round(t * 1e3, 4), "steps": K,
        "experts_touched": touched,
        "hbm": {"bytes_per_layer": wbytes, "achieved_gbs": round(wbytes / t / 1e9, 1), "peak_gbs": peak,
                "peak_kind": peak_kind, "frac": round(wbytes / t / 1e9 / peak, 4)},
        "tensor": {"flop_per_layer": flops, "achieved_tflops": round(flops / t / 1e12, 1),
                   "peak_tflops": tpeak, "peak_kind": tkind, "frac": round(flops / t / 1e12 / tpeak, 4),
                   "frac_of_fp4_peak": round(flops / t / 1e12 / (4 * bf16), 4)},
        "path": ("counting sort by expert; x as 2 exact e4m3 terms; block-scaled tcgen05 grouped GEMMs "
                 "(e2m1 weights + e8m0 scales as stored): gate/up with SwiGLU + 3-term h split in its epilogue, "
                 "down; combine")
        if aq == qk.QK_ACT_NONE else
        (f"counting sort by expert; x and h quantized to {act_name} (one term per token, 128-token tiles); "
         + ("both operands packed e2m1, block-scaled tcgen05 kind::mxf4nvf4 grouped GEMMs (e2m1 + e4m3 per 16 "
            "as stored; activation scales as ue4m3 re-anchored per row; scale_2 in the epilogue)" if nv else
            "both operands packed e2m1, block-scaled tcgen05 kind::mxf4 grouped GEMMs (weights as stored)"
            if aq == qk.QK_ACT_MXFP4 else "block-scaled tcgen05 kind::mxf8f6f4 grouped GEMMs")
         + "; combine"),
        "gpu_launches": (8 if nv else 7) * K,  # the NVFP4 fp4 mode keeps the h split kernel
    }


def main():
    args = parse()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        if rank != 0:
            return 0
        from block_quantized_expert_mxfp4_b200 import synth
        wl = synth.WORKLOADS[WORKLOAD]
        nbytes, secs, steps, thr = oracle_sample(args.reference_budget_s, args.steps + args.warmup)
        v = nbytes / secs / 1e9
        line = {"impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": "GB/s",
                "n_gpus": 1, "steps": steps, "warmup": 0,
                "ms_per_step": round(secs / max(steps, 1) * 1e3, 3), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64 (exact dequantized weights)",
                "data": "synthetic (seeded)",
                "config": {"workload": WORKLOAD_DESC, "parallelism": "host cores"},
                "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": thr,
                                 "kind": "oracle",
                                 "sample": f"{steps} (token, expert) pairs of the decode layer "
                                           f"(13.37 MB of MXFP4 weights each), bounded by "
                                           f"{args.reference_budget_s:.0f} s"},
                "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return 0

    import torch
    import torch.distributed as dist

    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    out = run_ours(args, rank, world, local_rank)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        nbytes, secs, steps, thr = oracle_sample(args.cpu_sample_s)
        out["cpu_baseline"] = {
            "value": round(nbytes / secs / 1e9, 4), "unit": "GB/s", "cores": thr, "kind": "oracle",
            "sample": f"{steps} (token, expert) pairs of the decode layer, {secs:.1f} s of CPU time"}
    if rank == 0:
        print(json.dumps(out))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
