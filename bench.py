#!/usr/bin/env python
"""Throughput of the ds4 routed-MoE expert FFN layer on B200.

One step = one pass of the whole layer (router, top-k softmax, expert-gathered
dequant GEMVs with SwiGLU, down projection, gate-weighted combine with the
bf16 shared expert) over one batch of synthetic tokens.  Default workload:
the decode step -- 1 token through one layer of hidden 4096, expert
intermediate 2048, 256 routed experts top-8, one bf16 shared expert.

Timing: W warm-up steps, then exactly K steps replayed from CUDA graphs,
bracketed by a barrier and a device synchronize, timed with CUDA events on
the launching stream, maximum over ranks.  Weights rotate over several layer
instances (more bytes than L2) and every step reads a different token vector.

Prints one JSON line (rank 0).  `--impl reference` times the CPU oracle on
the same workload instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s (decode & prefill); expert-weight HBM GB/s vs B200 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# Secondary denominators: NVIDIA's nominal per-GPU figures for HGX B200 (dense, no sparsity).
NOMINAL = {"hbm_gbs": 7700.0, "bf16_tflops": 2250.0,
           "source": "NVIDIA nominal HGX B200 per-GPU figures: HBM3e 7.7 TB/s, dense bf16 2.25 PFLOP/s"}

WORKLOADS = {
    "decode": dict(n=1, H=4096, I=2048, E=256, k=8,
                   desc="decode step: 1 token, one MoE layer (hidden 4096, expert intermediate 2048, "
                        "256 routed experts top-8 in IQ2_XXS/Q2_K-style 2-bit blocks, 1 bf16 shared expert)"),
    "decode_q4": dict(n=1, H=4096, I=2048, E=256, k=8, expert_bits=4,
                      desc="decode step, 4-bit experts: 1 token, one MoE layer (hidden 4096, expert intermediate "
                           "2048, 256 routed experts top-8 in Q4_K-style blocks, 1 bf16 shared expert)"),
    "decode8": dict(n=8, H=4096, I=2048, E=256, k=8,
                    desc="MTP-verify style decode: 8 tokens, one MoE layer of the decode shape"),
    "decode2": dict(n=2, H=4096, I=2048, E=256, k=8,
                    desc="MTP-verify style decode: 2 tokens, one MoE layer of the decode shape"),
    "mtp8": dict(n=2, H=4096, I=2048, E=256, k=8, layers=8, router_std=1.0 / 64, chain_scales=True,
                 desc="MTP-verify style decode: 2 tokens through 8 chained MoE layers of the decode shape "
                      "(x_{l+1} = x_l + MoE_l(x_l)), router logits N(0,1)"),
    "prefill512": dict(n=512, H=4096, I=2048, E=256, k=8, zipf=1.1, bf16=True,
                       desc="short-prompt prefill: 512 bf16 tokens, one MoE layer of the decode shape, "
                            "Zipf(1.1) expert popularity"),
    "prefill512_q4": dict(n=512, H=4096, I=2048, E=256, k=8, zipf=1.1, bf16=True, expert_bits=4,
                          desc="short-prompt prefill, 4-bit experts: 512 bf16 tokens, one MoE layer of the decode "
                               "shape with Q4_K-style routed experts, Zipf(1.1) expert popularity"),
    "prefill11709": dict(n=11709, H=4096, I=2048, E=256, k=8, zipf=1.1, bf16=True,
                         desc="long-prompt prefill: 11,709 bf16 tokens, one MoE layer (hidden 4096, expert "
                              "intermediate 2048, 256 experts top-8 + shared), Zipf(1.1) expert popularity"),
}


def algorithmic_flops(w: dict) -> dict:
    """Tensor-core FLOPs of each prefill GEMM launch (2 per multiply-add)."""
    H, I, k, n = w["H"], w["I"], w["k"], w["n"]
    return {"k_moe_gemm<gate_up>": 2 * n * k * H * 2 * I, "k_moe_gemm<down>": 2 * n * k * I * H,
            "k_moe_gemm<shared_gate_up>": 2 * n * H * 2 * I, "k_moe_gemm<shared_down>": 2 * n * I * H}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------- bytes per launch
def algorithmic_bytes(w: dict, U: int) -> dict:
    """Bytes each decode kernel must move, from the canonical formats (U distinct experts)."""
    H, I, E, k, n = w["H"], w["I"], w["E"], w["k"], w["n"]
    iq2 = I * H // 256 * 66          # one gate or up matrix
    q2 = H * I // 256 * 84           # one down matrix
    if w.get("expert_bits") == 4:    # all three matrices in 144-byte Q4_K-style blocks
        iq2 = q2 = I * H // 256 * 144
    sh_gu, sh_d = 2 * I * H * 2, H * I * 2
    return {
        "k_router_decode": E * H * 4 + n * H * 4 + n * E * 4,
        # gate/up and down in one kernel: every selected expert and the shared expert once, x in, h out and
        # back in (two bf16 pieces per value), y out
        "k_moe_decode": U * (2 * iq2 + q2) + sh_gu + sh_d + n * H * 4 + 2 * (n * k + n) * I * 4 + (n * k + n) * H * 4,
        "k_combine_decode": (n * k + n) * H * 4 + n * H * 4,
        "routed": U * (2 * iq2 + q2),
        # prefill GEMMs (U = experts touched): weights once, permuted activations in, results out
        "k_moe_gemm<gate_up>": U * 2 * iq2 + n * k * H * 2 + n * k * I * 2,
        "k_moe_gemm<down>": U * q2 + n * k * I * 2 + n * k * H * 4,
        "layer": E * H * 4 + U * (2 * iq2 + q2) + sh_gu + sh_d,
    }


def traffic_from_profile(kernel: str, workload: str):
    """dram bytes per launch recorded under profiles/, if the kernel's sources are unchanged since.

    The summary names its sources ("source_files: a.cu b.cuh", under the
    package's csrc/) and the sha256 of their bytes concatenated in that order.
    """
    name = kernel.replace("<", "_").replace(">", "")
    p = os.path.join(ROOT, "profiles", "%s_%s.md" % (name, workload))
    if not os.path.exists(p):
        return None
    txt = open(p).read()
    m1 = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", txt)
    m2 = re.search(r"source_sha256:\s*([0-9a-f]+)", txt)
    m3 = re.search(r"source_files:\s*([A-Za-z0-9_. ]+)", txt)
    if not (m1 and m2 and m3):
        return None
    h = hashlib.sha256()
    for f in m3.group(1).split():
        src = os.path.join(ROOT, "bit_quantized_moe_softmax_b200", "csrc", f)
        if not os.path.exists(src):
            return None
        h.update(open(src, "rb").read())
    if h.hexdigest() != m2.group(1):
        return None
    return float(m1.group(1))


# --------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock, power and clock-event reasons of one GPU, read through NVML
    (read-only queries) by a thread every `period_s` while the sampler runs,
    so that even a timed region of a millisecond gets samples; nvidia-smi is
    the fallback when NVML cannot be loaded."""

    REASONS = (("sw_power_cap", 0x4), ("hw_slowdown", 0x8), ("sw_thermal_slowdown", 0x20),
               ("hw_thermal_slowdown", 0x40), ("hw_power_brake_slowdown", 0x80))

    def __init__(self, device: int, period_s: float = 0.002):
        self.device = device
        self.period_s = period_s
        self.samples = []          # (t, sm_mhz, max_mhz, power_w, reasons bitmask)
        self.marks = {}
        self._stop = None
        self._thread = None
        self.source = None

    def _handle(self):
        import pynvml

        pynvml.nvmlInit()
        try:
            uuid = str(torch.cuda.get_device_properties(self.device).uuid)
            return pynvml, pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.device)

    def start(self):
        import threading

        try:
            nv, h = self._handle()
            mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            self.source = "nvml"
        except Exception:
            self.source = None
            return
        self._stop = threading.Event()

        def loop():
            while not self._stop.is_set():
                try:
                    sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                    pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                    self.samples.append((time.perf_counter(), sm, mx, pw, rs))
                except Exception:
                    pass
                self._stop.wait(self.period_s)

        self._thread = threading.Thread(target=loop, daemon=True)
        self._thread.start()

    def mark(self, name):
        self.marks[name] = time.perf_counter()

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=5)
            self._thread = None

    def summary(self, t0=None, t1=None) -> dict:
        """Clocks over [t0, t1] (perf_counter times; default: everything sampled)."""
        if self.source is None:
            return ClockSmi(self.device).once()
        sel = [q for q in self.samples if (t0 is None or q[0] >= t0) and (t1 is None or q[0] <= t1)]
        if not sel:   # a region shorter than the sampling period: the samples around it
            if not self.samples:
                return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
            mid = 0.5 * ((t0 or 0.0) + (t1 or 0.0))
            sel = sorted(self.samples, key=lambda q: abs(q[0] - mid))[:3]
        reasons = sorted({nm for q in sel for nm, bit in self.REASONS if q[4] & bit})
        return {"sm_mhz": statistics.median(q[1] for q in sel), "sm_max_mhz": max(q[2] for q in sel),
                "reasons": reasons, "samples": len(sel), "power_w_median": round(statistics.median(q[3] for q in sel), 1),
                "source": "NVML, every %.0f ms during the timed region" % (self.period_s * 1e3)}


class ClockSmi:
    """One nvidia-smi query (fallback when NVML is unavailable)."""

    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index

    def once(self) -> dict:
        try:
            out = subprocess.run(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                                  "--format=csv,noheader,nounits"], capture_output=True, text=True, timeout=10).stdout
            f = [x.strip() for x in out.strip().split(",")]
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            return {"sm_mhz": float(f[0]), "sm_max_mhz": float(f[1]),
                    "reasons": [nm for nm, v in zip(names, f[2:6]) if v.lower().startswith("active")],
                    "source": "one nvidia-smi query after the timed region"}
        except Exception:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}


def host_cpu() -> dict:
    model = None
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except Exception:
        pass
    return {"cores": os.cpu_count(), "model": model}


# --------------------------------------------------------------- our arm
def run_ours(args, wl, rank, local, world):
    import bit_quantized_moe_softmax_b200 as m
    from bit_quantized_moe_softmax_b200 import dist as D
    from bit_quantized_moe_softmax_b200 import synth

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    n, H, I, E, k = wl["n"], wl["H"], wl["I"], wl["E"], wl["k"]
    prefill = n > 8
    C = wl.get("layers", 1)     # chained layers per step (x_{l+1} = x_l + MoE_l(x_l))
    chain = C > 1
    R = C if chain else (1 if prefill else args.instances)
    shape = synth.Shape(H=H, I=I, E=E, k=k)
    bias = synth.zipf_bias(E, wl["zipf"], seed=5).to(dev) if wl.get("zipf") else None
    act = m.DS4MOE_ACT_BF16 if wl.get("bf16") else m.DS4MOE_ACT_F32
    layers = []
    for r in range(R):
        L = synth.packed_layer(shape, seed=1000 * rank + r, router_std=wl.get("router_std", 0.02), bias=bias,
                               device=dev, d_range=synth.CHAIN_D_RANGE if wl.get("chain_scales") else None,
                               shared_std=synth.CHAIN_SHARED_STD if wl.get("chain_scales") else 0.02,
                               expert_bits=wl.get("expert_bits", 2))
        lay = m.MoELayer(H, I, E, k, max_tokens=max(n, 8), act_dtype=act, has_bias=bias is not None, device=dev,
                         expert_bits=wl.get("expert_bits", 0))
        lay.load(L)
        if args.steer:
            v = synth.normal((H,), 1.0, synth.gen(500 + r, dev), dev)
            lay.set_steering((v / v.double().norm().float()).contiguous(), args.steer)
        layers.append(lay)
        del L
    P = 2 if prefill else 64
    xs = synth.tokens(P * n, H, seed=77 + rank, device=dev,
                      dtype=torch.bfloat16 if act == m.DS4MOE_ACT_BF16 else torch.float32).view(P, n, H).contiguous()
    outs = torch.empty(P, n, H, dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(device=dev)
    nl = m.ds4moe_plan_launches(layers[0].h, n)
    names = [m.ds4moe_plan_kernel(layers[0].h, n, i) for i in range(nl)]

    cbufs = [torch.empty(n, H, dtype=torch.float32, device=dev) for _ in range(C)] if chain else []
    cwork = torch.empty(2, n, H, dtype=torch.float32, device=dev) if chain else None
    handles = [lay.h for lay in layers]

    def step(i, events=None):
        if chain and events is None:   # the whole chain in one call (layers as programmatic dependents)
            m.ds4moe_forward_chain(handles, xs[i % P], cbufs[-1], cwork, stream)
            return
        if chain:   # every layer of the chain, the residual added by each layer's combine kernel
            cur = xs[i % P]
            for l in range(C):
                if events is None:
                    m.ds4moe_forward_residual(layers[l].h, cur, cbufs[l], stream)
                else:
                    m.ds4moe_forward_residual_profiled(layers[l].h, cur, cbufs[l],
                                                       events[2 * nl * l:2 * nl * (l + 1)], stream)
                cur = cbufs[l]
            return
        lay = layers[i % R]
        if events is None:
            m.ds4moe_forward(lay.h, xs[i % P], outs[i % P], stream)
        else:
            m.ds4moe_forward_profiled(lay.h, xs[i % P], outs[i % P], events, stream)

    def distinct_experts():
        """Mean number of distinct experts per layer forward over the steps the graphs replay."""
        tot, cnt = 0, 0
        with torch.cuda.stream(stream):
            for i in range(min(4 if prefill else 64, P * R)):
                if chain:
                    cur = xs[i % P]
                    for l in range(C):
                        ids, _ = layers[l].route(cur)
                        tot += int(torch.unique(ids).numel())
                        cnt += 1
                        m.ds4moe_forward_residual(layers[l].h, cur, cbufs[l], stream)
                        cur = cbufs[l]
                else:
                    ids, _ = layers[i % R].route(xs[i % P])
                    tot += int(torch.unique(ids).numel())
                    cnt += 1
        stream.synchronize()
        return tot / cnt

    with torch.cuda.stream(stream):
        for i in range(max(2, R)):
            step(i)             # first calls set kernel attributes outside capture
    stream.synchronize()
    for lay in layers:          # a device-side check or bounded wait that failed ends the run here
        code = m.ds4moe_get_device_error(lay.h, stream)
        if code:
            raise SystemExit("device error code %d after the first forward calls" % code)

    sampler = ClockSampler(local)
    sampler.start()
    try:
        return _timed_run(args, wl, rank, local, world, dev, layers, xs, outs, stream, nl, names, step, distinct_experts,
                          chain, C, R, P, n, H, I, E, k, prefill, sampler, cbufs)
    finally:
        sampler.stop()


def _timed_run(args, wl, rank, local, world, dev, layers, xs, outs, stream, nl, names, step, distinct_experts, chain, C,
               R, P, n, H, I, E, k, prefill, sampler, cbufs):
    import bit_quantized_moe_softmax_b200 as m
    from bit_quantized_moe_softmax_b200 import dist as D

    S = max(1, min(args.steps, 2 if prefill else 64))

    def new_events(count):
        # torch creates the CUDA event on first record: record each once before capture
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * nl * C)] for _ in range(count)]
        for ev in evs:
            for e in ev:
                e.record(stream)
        stream.synchronize()
        return evs

    def capture(count, first, profiled):
        g = torch.cuda.CUDAGraph()
        evs = new_events(count) if profiled else []
        with torch.cuda.graph(g, stream=stream):
            for j in range(count):
                step(first + j, evs[j] if profiled else None)
        return g, evs

    def graphs_for(K, profiled):
        full, rem = divmod(K, S)
        out = []
        if full:
            out.append((capture(S, 0, profiled), full))
        if rem:
            out.append((capture(rem, 0, profiled), 1))
        return out

    # warm-up: W steps (graph replays of the same kind)
    warm = graphs_for(args.warmup, False)
    for (g, _), reps in warm:
        for _ in range(reps):
            g.replay()
    torch.cuda.synchronize(dev)
    timed = graphs_for(args.steps, False)
    for (g, _), _ in timed:
        g.replay()                # one untimed replay of each graph (first-launch upload)
    torch.cuda.synchronize(dev)
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    D.barrier()
    torch.cuda.synchronize(dev)
    t_start = time.perf_counter()
    with torch.cuda.stream(stream):
        start.record(stream)
        for (g, _), reps in timed:
            for _ in range(reps):
                g.replay()
        stop.record(stream)
    torch.cuda.synchronize(dev)
    t_stop = time.perf_counter()
    D.barrier()
    ms = start.elapsed_time(stop)
    # profiled pass over the same K steps: per-launch events around every kernel
    prof = graphs_for(args.steps, True)
    for (g, _), _ in prof:
        g.replay()
    torch.cuda.synchronize(dev)
    pstart, pstop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    durs = {nm: [] for nm in names}
    with torch.cuda.stream(stream):
        pstart.record(stream)
        for (g, evs), reps in prof:
            for _ in range(reps):
                g.replay()
        pstop.record(stream)
    torch.cuda.synchronize(dev)
    for (g, evs), reps in prof:
        for ev in evs:
            for l in range(C):
                for i, nm in enumerate(names):
                    durs[nm].append(ev[2 * nl * l + 2 * i].elapsed_time(ev[2 * nl * l + 2 * i + 1]))
    ms_prof = pstart.elapsed_time(pstop)
    clocks = sampler.summary(t_start, t_stop)

    ms_max = D.max_over_ranks(ms, dev)
    tokens = n * args.steps * world
    value = tokens / (ms_max / 1e3)
    ms_per_step = ms_max / args.steps

    # e2e: host buffers through the public API, copies inside the timed region
    K2 = max(1, min(args.steps, 2000))
    K2 = min(K2, 20) if prefill else K2
    xh = xs[: min(P, K2)].cpu().pin_memory()
    oh = torch.empty(xh.shape, dtype=torch.float32).pin_memory()

    def e2e_step(i):
        if chain:   # pinned host x -> device, the chain, device -> pinned host, synchronize
            xd = xs[0]
            with torch.cuda.stream(stream):
                xd.copy_(xh[i % xh.shape[0]], non_blocking=True)
                step(0)
                oh[i % xh.shape[0]].copy_(cbufs[-1], non_blocking=True)
            stream.synchronize()
        else:   # pipelined: this step's copies overlap its neighbours' kernels
            m.ds4moe_forward_host_async(layers[i % R].h, xh[i % xh.shape[0]], oh[i % xh.shape[0]], stream)

    def e2e_drain():
        if not chain:
            for lay in layers:
                m.ds4moe_host_sync(lay.h)
        stream.synchronize()

    for i in range(min(10, K2)):
        e2e_step(i)
    e2e_drain()
    D.barrier()
    t0 = time.perf_counter()
    for i in range(K2):
        e2e_step(i)
    e2e_drain()
    t1 = time.perf_counter()
    e2e_s = D.max_over_ranks(t1 - t0, dev)
    e2e = {"value": n * K2 * world / e2e_s, "unit": "tokens/s", "h2d_bytes_per_step": n * H * xh.element_size(),
           "d2h_bytes_per_step": n * H * 4, "steps": K2,
           "api": ("torch copies around one ds4moe_forward_chain call, synchronized per step" if chain
                   else "ds4moe_forward_host_async per step (two staging slots per layer), ds4moe_host_sync at the end")}

    # roofline of the dominant kernel
    wname = next(key for key, v in WORKLOADS.items() if v is wl)
    peaks, peak_kind = load_peaks()
    mean = {nm: (statistics.mean(v) if v else 0.0) for nm, v in durs.items()}
    dom = max(mean, key=lambda nm: mean[nm])
    U = distinct_experts()
    ab = algorithmic_bytes(wl, U if U is not None else n * k)
    if prefill:
        fl = algorithmic_flops(wl)
        achieved = fl[dom] / (mean[dom] * 1e-3) / 1e12
        # primary: the measured cuBLAS burst figure; the seconds-long sustained
        # figure (under the power cap) is reported beside it when the loop is long
        peak = peaks["bf16_tflops"]
        sustained_s = ms_per_step * args.steps / 1e3
        roofline = {"bound": "tensor", "kernel": dom, "achieved": round(achieved, 1), "peak": peak,
                    "unit": "TFLOP/s", "frac": round(achieved / peak, 4), "traffic": traffic_from_profile(dom, wname),
                    "algorithmic_flops_per_launch": fl[dom], "mean_launch_us": round(mean[dom] * 1e3, 2),
                    # the same launch against HBM: weights of the touched experts, activations in and out
                    "hbm_view": ({"achieved": round(ab[dom] / (mean[dom] * 1e-3) / 1e9, 1), "peak": peaks["hbm_gbs"],
                                  "unit": "GB/s", "frac": round(ab[dom] / (mean[dom] * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                                  "algorithmic_bytes_per_launch": int(round(ab[dom]))} if dom in ab else None),
                    "sustained_view": {"peak": peaks.get("bf16_tflops_sustained"),
                                       "frac": (round(achieved / peaks["bf16_tflops_sustained"], 4)
                                                if peaks.get("bf16_tflops_sustained") else None),
                                       "timed_loop_s": round(sustained_s, 3)},
                    "nominal": {"peak": NOMINAL["bf16_tflops"], "frac": round(achieved / NOMINAL["bf16_tflops"], 4),
                                "source": NOMINAL["source"]},
                    "peak_source": peak_kind + " (MEASURED_PEAKS.json bf16_tflops, cuBLAS burst)"}
    else:
        achieved = ab[dom] / (mean[dom] * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
        roofline = {"bound": "hbm", "kernel": dom, "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                    "frac": round(achieved / peak, 4), "traffic": traffic_from_profile(dom, wname),
                    "algorithmic_bytes_per_launch": int(round(ab[dom])), "mean_launch_us": round(mean[dom] * 1e3, 2),
                    "nominal": {"peak": NOMINAL["hbm_gbs"], "frac": round(achieved / NOMINAL["hbm_gbs"], 4),
                                "source": NOMINAL["source"]},
                    "peak_source": peak_kind + " (MEASURED_PEAKS.json hbm_gbs, burst copy)"}
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if prefill else "f32", "data": "synthetic",
        "config": {"workload": wl["desc"], "n_tokens_per_step": n, "hidden": H, "expert_inter": I,
                   "experts": E, "top_k": k, "layer_instances": R, "chained_layers": C, "token_vectors": P,
                   "mean_distinct_experts_per_layer": round(U, 2) if U else None,
                   "l2": ("%d chained layers (%.1f GB of weights) and %d token vectors per step: inputs larger "
                          "than L2" % (C, C * layers[0].weights.numel() / 1e9, P)) if chain else
                         ("weights rotate over %d layer instances (%.1f GB) and %d token vectors: inputs larger "
                          "than L2" % (R, R * layers[0].weights.numel() / 1e9, P)) if not prefill else
                         "one layer (%.1f GB of weights) and %d token batches per step: inputs larger than L2"
                         % (layers[0].weights.numel() / 1e9, n),
                   "parallelism": "dp%d replicas (no collective on the data path)" % world,
                   "steering_F": args.steer},
        "expert_weight_gbs": round(C * ab["routed"] / (ms_per_step * 1e-3) / 1e9, 1) if U else None,
        "layer_hbm_gbs": round(C * ab["layer"] / (ms_per_step * 1e-3) / 1e9, 1) if U else None,
        "layer_frac_of_hbm_peak": round(C * ab["layer"] / (ms_per_step * 1e-3) / 1e9 / peaks["hbm_gbs"], 4) if U else None,
        "kernel_us": {nm: round(mean[nm] * 1e3, 2) for nm in names},
        "ms_per_step_profiled": round(ms_prof / args.steps, 5),
        "roofline": roofline, "e2e": e2e, "gpu_launches": nl * C * args.steps, "clocks": clocks,
    }
    return line


# --------------------------------------------------------------- oracle (CPU) arm
def _pool_map(fn, items, budget_s):
    """Run fn over items on all host cores (threads: the oracle's C calls release the GIL and
    keep no global state), starting no new item after budget_s; returns (results, seconds)."""
    from concurrent.futures import ThreadPoolExecutor

    cores = os.cpu_count() or 1
    t0 = time.perf_counter()
    done = []

    def run(it):
        if time.perf_counter() - t0 > budget_s:
            return None
        return fn(it)

    with ThreadPoolExecutor(max_workers=cores) as ex:
        for r in ex.map(run, items):
            if r is not None:
                done.append(r)
    return done, time.perf_counter() - t0


def oracle_sample(wl, n_tokens, seed=0, budget_s=20.0, device="cuda", warmup=0):
    """Oracle tokens/s on a bounded sample of the workload (router + top-k + experts + shared), one token per
    task, on all host cores, after `warmup` untimed tokens.  Returns (tokens/s, tokens done, seconds, cores)."""
    import oracle
    from bit_quantized_moe_softmax_b200 import synth

    H, I, E, k = wl["H"], wl["I"], wl["E"], wl["k"]
    bias = synth.zipf_bias(E, wl["zipf"], seed=5) if wl.get("zipf") else None
    if wl.get("layers", 1) > 1:
        return oracle_chain_sample(wl, n_tokens, seed, budget_s, device, warmup)
    L = synth.packed_layer(synth.Shape(H=H, I=I, E=E, k=k), seed=seed, bias=bias, device=device,
                           expert_bits=wl.get("expert_bits", 2))
    x = synth.tokens(n_tokens, H, seed=seed + 5, dtype=torch.bfloat16 if wl.get("bf16") else torch.float32).float()
    mode = 1 if wl.get("bf16") else 0
    lg = oracle.router_logits(x.numpy(), L["W_r"].cpu().numpy(), None if bias is None else bias.numpy())
    rid, _ = oracle.topk_softmax(lg, k)
    lay = oracle.layer_from_torch(L, experts=rid.ravel())
    del L
    xs = x.numpy()
    if warmup:
        _pool_map(lambda t: oracle.moe_forward(lay, xs[t:t + 1], mode=mode), range(min(warmup, n_tokens)), budget_s)
    done, dt = _pool_map(lambda t: oracle.moe_forward(lay, xs[t:t + 1], mode=mode), range(n_tokens), budget_s)
    return len(done) / dt, len(done), dt, os.cpu_count() or 1


def oracle_chain_sample(wl, n_tokens, seed, budget_s, device, warmup=0):
    """Oracle tokens/s through the chain of layers (fp64 layers, binary32 between layers), one token per task
    on all host cores; each task routes its token layer by layer and runs the layer on the experts it picks."""
    import oracle
    from bit_quantized_moe_softmax_b200 import synth

    H, I, E, k, C = wl["H"], wl["I"], wl["E"], wl["k"], wl["layers"]
    Ls = [synth.packed_layer(synth.Shape(H=H, I=I, E=E, k=k), seed=seed + l, router_std=wl.get("router_std", 0.02),
                             device=device, d_range=synth.CHAIN_D_RANGE, shared_std=synth.CHAIN_SHARED_STD)
          for l in range(C)]
    lays = [oracle.layer_from_torch(L) for L in Ls]   # every expert on the host: any may be chosen
    del Ls
    x = synth.tokens(n_tokens, H, seed=seed + 5).numpy()

    def one(t):
        cur = x[t:t + 1].astype(np.float32)
        for lay in lays:
            y, _, _ = oracle.moe_forward(lay, cur, mode=0)
            cur = (cur.astype(np.float64) + y).astype(np.float32)
        return cur

    if warmup:
        _pool_map(one, range(min(warmup, n_tokens)), budget_s)
    done, dt = _pool_map(one, range(n_tokens), budget_s)
    return len(done) / dt, len(done), dt, os.cpu_count() or 1


def cpu_baseline_record(wl, n_tokens, budget_s, device):
    rate, done, dt, cores = oracle_sample(wl, n_tokens=n_tokens, budget_s=budget_s, device=device)
    cpu = host_cpu()
    return {"value": round(rate, 4), "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "cpu_model": cpu["model"],
            "sample": "%d tokens of the same workload through the CPU oracle in %.1f s on %d host threads "
                      "(one token per task; %s reading)" % (done, dt, cores,
                                                             "bf16 (mode 1)" if wl.get("bf16") else "fp64 (mode 0)")}


def run_reference(args, wl, rank, world):
    if rank != 0:
        return None
    budget = 120.0
    cores = os.cpu_count() or 1
    # the seeded layer is drawn on the GPU when there is one (the same bytes as our arm's); without one,
    # torch's CPU generator draws a layer of the same shape and distribution
    device = "cuda" if torch.cuda.is_available() else "cpu"
    warm = max(3, min(args.warmup, cores))   # untimed tokens first (one per host thread at most)
    rate, done, dt, cores = oracle_sample(wl, n_tokens=max(cores, args.steps), budget_s=budget, device=device,
                                          warmup=warm)
    cpu = host_cpu()
    sample = ("%d tokens (one per task; %d requested steps, n=%d per step in our arm) through the CPU oracle "
              "(canonical binary32 router, fp64 dequantized experts and shared expert) on %d host threads after %d "
              "untimed tokens, no new task after a %.0f s budget" % (done, args.steps, wl["n"], cores, warm, budget))
    return {"impl": "reference", "metric": METRIC, "value": round(rate, 4), "unit": "tokens/s", "n_gpus": world,
            "steps": done, "steps_requested": args.steps, "warmup": warm, "ms_per_step": round(dt / done * 1e3, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl["desc"], "n_tokens_per_step": wl["n"], "hidden": wl["H"],
                       "expert_inter": wl["I"], "experts": wl["E"], "top_k": wl["k"],
                       "chained_layers": wl.get("layers", 1), "parallelism": "oracle on the host cores of rank 0",
                       "steering_F": args.steer},
            "cpu_baseline": {"value": round(rate, 4), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "cpu_model": cpu["model"], "sample": sample},
            "e2e": {"value": round(rate, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


SUB_WORKLOADS = ("decode_q4", "mtp8", "prefill512", "prefill11709")


def sub_record(line: dict) -> dict:
    """The fields of a workload's line kept when it rides along the headline line."""
    keep = ("value", "unit", "ms_per_step", "dtype", "config", "roofline", "kernel_us", "e2e", "gpu_launches",
            "clocks", "cpu_baseline", "expert_weight_gbs", "layer_hbm_gbs", "layer_frac_of_hbm_peak")
    return {k: line[k] for k in keep if k in line}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=400)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decode", choices=sorted(WORKLOADS))
    ap.add_argument("--instances", type=int, default=4)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true",
                    help="with the default decode workload: skip the sub-records (4-bit decode, chain, prefill)")
    ap.add_argument("--steer", type=float, default=0.0,
                    help="directional steering strength F of every layer (unit direction, seeded); 0: off")
    args = ap.parse_args()
    wl = WORKLOADS[args.workload]
    from bit_quantized_moe_softmax_b200 import dist as D

    if args.impl == "reference":
        rank, local, world = D.env_rank()
        if rank == 0:
            print(json.dumps(run_reference(args, wl, rank, world)), flush=True)
        return
    rank, local, world = D.init("nccl")
    from bit_quantized_moe_softmax_b200 import build

    if rank == 0:
        build.build()
    D.barrier()
    dev = torch.device("cuda", local)
    baseline = rank == 0 and world == 1 and not args.no_cpu_baseline
    cores = os.cpu_count() or 1
    line = run_ours(args, wl, rank, local, world)
    if baseline:
        line["cpu_baseline"] = cpu_baseline_record(wl, n_tokens=4 * cores, budget_s=15.0, device=dev)
    # the metric covers decode and prefill: the default run adds the 4-bit decode step, the chained
    # verify step and both prefill workloads as sub-records
    if args.workload == "decode" and not args.no_prefill:
        subs = {}
        for name in SUB_WORKLOADS:
            import gc

            gc.collect()
            torch.cuda.empty_cache()
            sub = run_ours(args, WORKLOADS[name], rank, local, world)
            if baseline:
                sub["cpu_baseline"] = cpu_baseline_record(WORKLOADS[name], n_tokens=2 * cores, budget_s=10.0, device=dev)
            subs[name] = sub_record(sub)
        line["workloads"] = subs
    if rank == 0:
        print(json.dumps(line), flush=True)
    D.finish()


if __name__ == "__main__":
    main()
