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
    sh_gu, sh_d = 2 * I * H * 2, H * I * 2
    return {
        "k_router_decode": E * H * 4 + n * H * 4 + n * E * 4,
        "k_gateup_decode": U * 2 * iq2 + sh_gu + n * H * 4 + (n * k + n) * I * 4,
        "k_down_decode": U * q2 + sh_d + (n * k + n) * I * 4 + (n * k + n) * H * 4,
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
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="clocks", suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
                power.append(float(f[3]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        # samples under load: power above the midpoint of the observed range
        lo, hi = min(power), max(power)
        loaded = [s for s, p in zip(sm, power) if p >= lo + 0.5 * (hi - lo)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm), "samples_under_load": len(loaded)}


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
                               device=dev, d_range=synth.CHAIN_D_RANGE if wl.get("chain_scales") else (1e-3, 4e-3),
                               shared_std=synth.CHAIN_SHARED_STD if wl.get("chain_scales") else 0.02)
        lay = m.MoELayer(H, I, E, k, max_tokens=max(n, 8), act_dtype=act, has_bias=bias is not None, device=dev)
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

    def step(i, events=None):
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

    # graphs of S consecutive steps (cycling instances and token vectors)
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

    sampler = ClockSampler(local)
    sampler.start()
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
    with torch.cuda.stream(stream):
        start.record(stream)
        for (g, _), reps in timed:
            for _ in range(reps):
                g.replay()
        stop.record(stream)
    torch.cuda.synchronize(dev)
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
    clocks = sampler.stop()

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
           "api": ("torch copies around the chained ds4moe_forward_residual calls, synchronized per step" if chain
                   else "ds4moe_forward_host_async per step (two staging slots per layer), ds4moe_host_sync at the end")}

    # roofline of the dominant kernel
    peaks, peak_kind = load_peaks()
    mean = {nm: (statistics.mean(v) if v else 0.0) for nm, v in durs.items()}
    dom = max(mean, key=lambda nm: mean[nm])
    U = distinct_experts()
    ab = algorithmic_bytes(wl, U if U is not None else n * k)
    if prefill:
        fl = algorithmic_flops(wl)
        achieved = fl[dom] / (mean[dom] * 1e-3) / 1e12
        # a kernel timed inside a seconds-long loop runs under the power cap:
        # compare it with the sustained GEMM figure, a short run with the burst one
        sustained = ms_per_step * args.steps >= 1000.0
        peak = peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"]
        roofline = {"bound": "tensor", "kernel": dom, "achieved": round(achieved, 1), "peak": peak,
                    "unit": "TFLOP/s", "frac": round(achieved / peak, 4), "traffic": traffic_from_profile(dom, args.workload),
                    "algorithmic_flops_per_launch": fl[dom], "mean_launch_us": round(mean[dom] * 1e3, 2),
                    # the same launch against HBM: weights of the touched experts, activations in and out
                    "hbm_view": ({"achieved": round(ab[dom] / (mean[dom] * 1e-3) / 1e9, 1), "peak": peaks["hbm_gbs"],
                                  "unit": "GB/s", "frac": round(ab[dom] / (mean[dom] * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                                  "algorithmic_bytes_per_launch": int(round(ab[dom]))} if dom in ab else None),
                    "nominal": {"peak": NOMINAL["bf16_tflops"], "frac": round(achieved / NOMINAL["bf16_tflops"], 4),
                                "source": NOMINAL["source"]},
                    "peak_source": peak_kind + (" (MEASURED_PEAKS.json bf16_tflops_sustained, cuBLAS back to back "
                                                "for seconds: the timed loop lasts %.1f s)" % (ms_per_step * args.steps / 1e3)
                                                if sustained else " (MEASURED_PEAKS.json bf16_tflops, cuBLAS burst)")}
    else:
        achieved = ab[dom] / (mean[dom] * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
        roofline = {"bound": "hbm", "kernel": dom, "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                    "frac": round(achieved / peak, 4), "traffic": traffic_from_profile(dom, args.workload),
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
        "layer_frac_of_hbm_peak": round(C * ab["layer"] / (ms_per_step * 1e-3) / 1e9 / peak, 4) if U else None,
        "kernel_us": {nm: round(mean[nm] * 1e3, 2) for nm in names},
        "ms_per_step_profiled": round(ms_prof / args.steps, 5),
        "roofline": roofline, "e2e": e2e, "gpu_launches": nl * C * args.steps, "clocks": clocks,
    }
    return line


# --------------------------------------------------------------- oracle (CPU) arm
def oracle_sample(wl, n_tokens, seed=0, budget_s=20.0, device="cuda"):
    """Oracle tokens/s on a bounded sample of the workload (router + top-k + experts + shared, fp64)."""
    import oracle
    from bit_quantized_moe_softmax_b200 import synth

    H, I, E, k = wl["H"], wl["I"], wl["E"], wl["k"]
    bias = synth.zipf_bias(E, wl["zipf"], seed=5) if wl.get("zipf") else None
    if wl.get("layers", 1) > 1:
        return oracle_chain_sample(wl, n_tokens, seed, budget_s, device)
    L = synth.packed_layer(synth.Shape(H=H, I=I, E=E, k=k), seed=seed, bias=bias, device=device)
    x = synth.tokens(n_tokens, H, seed=seed + 5, dtype=torch.bfloat16 if wl.get("bf16") else torch.float32).float()
    mode = 1 if wl.get("bf16") else 0
    lg = oracle.router_logits(x.numpy(), L["W_r"].cpu().numpy(), None if bias is None else bias.numpy())
    rid, _ = oracle.topk_softmax(lg, k)
    lay = oracle.layer_from_torch(L, experts=rid.ravel())
    del L
    t0 = time.perf_counter()
    done = 0
    for t in range(n_tokens):
        oracle.moe_forward(lay, x[t:t + 1].numpy(), mode=mode)
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return done / dt, done, dt


def oracle_chain_sample(wl, n_tokens, seed, budget_s, device):
    """Oracle tokens/s through the chain of layers (fp64 layers, binary32 between layers); only the time
    of the oracle's router and layer calls counts (not the host copies of the selected experts' blocks)."""
    import oracle
    from bit_quantized_moe_softmax_b200 import synth

    H, I, E, k, C = wl["H"], wl["I"], wl["E"], wl["k"], wl["layers"]
    Ls = [synth.packed_layer(synth.Shape(H=H, I=I, E=E, k=k), seed=seed + l, router_std=wl.get("router_std", 0.02),
                             device=device, d_range=synth.CHAIN_D_RANGE, shared_std=synth.CHAIN_SHARED_STD)
          for l in range(C)]
    x = synth.tokens(n_tokens, H, seed=seed + 5).numpy()
    spent, done = 0.0, 0
    for t in range(n_tokens):
        cur = x[t:t + 1].astype(np.float32)
        for L in Ls:
            t0 = time.perf_counter()
            rid, _ = oracle.topk_softmax(oracle.router_logits(cur, L["W_r"].cpu().numpy()), k)
            spent += time.perf_counter() - t0
            lay = oracle.layer_from_torch(L, experts=rid.ravel())
            t0 = time.perf_counter()
            y, _, _ = oracle.moe_forward(lay, cur, mode=0)
            spent += time.perf_counter() - t0
            cur = (cur.astype(np.float64) + y).astype(np.float32)
        done += 1
        if spent > budget_s:
            break
    return done / spent, done, spent


def run_reference(args, wl, rank, world):
    if rank != 0:
        return None
    budget = 120.0
    rate, done, dt = oracle_sample(wl, n_tokens=max(1, args.steps), budget_s=budget)
    sample = ("%d of %d requested steps (1 token each, n=%d per step in our arm) through the CPU oracle "
              "(canonical binary32 router, fp64 dequantized experts and shared expert), single thread, "
              "stopped at a %.0f s budget" % (done, args.steps, wl["n"], budget))
    return {"impl": "reference", "metric": METRIC, "value": round(rate, 4), "unit": "tokens/s", "n_gpus": world,
            "steps": done, "steps_requested": args.steps, "warmup": 0, "ms_per_step": round(dt / done * 1e3, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl["desc"], "n_tokens_per_step": 1},
            "cpu_baseline": {"value": round(rate, 4), "unit": "tokens/s", "cores": 1, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(rate, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=400)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decode", choices=sorted(WORKLOADS))
    ap.add_argument("--instances", type=int, default=4)
    ap.add_argument("--no-cpu-baseline", action="store_true")
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
    line = run_ours(args, wl, rank, local, world)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, done, dt = oracle_sample(wl, n_tokens=16, budget_s=20.0, device=torch.device("cuda", local))
        line["cpu_baseline"] = {"value": round(rate, 4), "unit": "tokens/s", "cores": 1, "kind": "oracle",
                                "sample": "%d tokens of the same workload through the CPU oracle in %.1f s "
                                          "(single thread, fp64)" % (done, dt)}
    if rank == 0:
        print(json.dumps(line), flush=True)
    D.finish()


if __name__ == "__main__":
    main()
