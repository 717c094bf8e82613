"""Benchmark of the routed-expert MoE layer on B200 (synthetic seeded layers).

python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl strata|reference]

A step is one pass of the hot path over one batch: routing (router GEMV or
GEMM, softmax top-k, per-expert lists) and the experts (dequantised 2-bit
gate/up, SwiGLU, down, weighted combine). Workloads (seeded, synthetic):
  decode        d=2048 f=768 E=512 k=10, 1 token per step, uniform routing (default)
  verify4/16    48-layer stack, 4 or 16 tokens per step, Zipf(1.1) prior
  verify6       48-layer stack, 1 + 5 drafted tokens per step, Zipf(1.1) prior
  coder_decode  as decode with 256 experts per layer (the Coder variant)
  prefill       one layer, 8,192-token chunk, Zipf(1.1) prior
  prefill_stack 48 layers, 32,768 tokens in 8,192-token chunks, Zipf(1.1)
Inputs are resident in HBM before timing; the single-layer decode workloads
rotate over 8 seeded copies of the layer (6 GB at 512 experts) and 64 token
vectors so that no step finds its experts in L2. Multi-GPU runs are independent replicas (the layer does
not shard); value = units over all ranks / max-over-ranks time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE layer tokens/s (decode & 8K prefill) + % of HBM / tensor roofline"

# DRAM bytes (read + write) of one launch of each workload's dominant kernel
# from one ncu capture (profiles/*.md gives the command). Set to None when the
# kernel changes after the capture.
MEASURED_TRAFFIC = {
    "decode": 19056128,             # k_decode_fused<1>, profiles/decode_fused_T1.md
    "prefill": 683305984,           # k_expert_gemm<0>, profiles/prefill_expert_gemm_8192.md
}
PREFILL_KERNELS = 8

# default timed steps per workload (each a multiple of the steps one graph replay covers)
DEFAULT_STEPS = {"decode": 64 * 1024, "verify4": 200, "verify6": 150, "verify16": 100, "prefill": 200,
                 "prefill_stack": 3, "coder_decode": 64 * 1024}


def graph_steps(w) -> int:
    """Steps one CUDA-graph replay covers: 64 single-layer decode calls, 8
    prefill chunks, or one whole stack pass (captured by the library)."""
    if w.layers > 1:
        return 1
    return 64 if w.T <= 16 else 8


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        j = json.load(open(p))
        return j["hbm_gbs"], j["bf16_tflops"], j.get("bf16_tflops_sustained", j["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


class Clocks:
    """nvidia-smi sampler running during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.out = tempfile.NamedTemporaryFile(mode="w+", suffix=".csv", delete=False)

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.out, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        self.proc.wait(timeout=10)
        self.out.flush()
        rows = [l.split(",") for l in open(self.out.name).read().strip().splitlines() if l.strip()]
        os.unlink(self.out.name)
        sm = [float(r[1]) for r in rows if len(r) >= 9 and r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if len(r) >= 9 and r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in rows:
            if len(r) < 9:
                continue
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(rows)}


# ---------------------------------------------------------------- setup


def setup_dist(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def dist_max(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


class LayerData:
    """Device-resident inputs of one layer of a workload."""

    def __init__(self, S, w, layer_idx, layer_obj):
        import synth.device as sd
        self.W, self.bias = sd.layer_inputs(w, layer_idx)

        def pack(e, gc, gs, uc, us, dc, ds, dst):
            S.strata_moe_pack_expert_device(layer_obj.desc, gc, gs, uc, us, dc, ds, dst)

        self.blob = sd.layer_blob(w, layer_idx, pack)


# ---------------------------------------------------------------- workloads


def algorithmic_units(w, route_counts):
    """Selected-expert bytes of the decode/gate-up stage and expert FLOPs."""
    d, f = w.d, w.f
    gu_bytes_per_expert = 2 * d * f // 32 * 10
    return gu_bytes_per_expert, 2 * 2 * d * f  # bytes per active expert, flops per (token, expert) in gate/up


def run_strata(args, world, rank, local):
    import torch
    import bit_quantized_moe_warp_b200 as S
    import synth
    import synth.device as sd

    w = synth.WORKLOADS[args.workload]
    hbm, tf_burst, tf_sust, peak_src = load_peaks()
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    stacked = w.layers > 1
    T = w.T
    chunk = min(T, w.chunk)
    rotate = not stacked and T <= 16  # single-layer decode sizes: rotate layer copies and token vectors
    copies = args.copies if rotate else (w.layers if stacked else 1)
    ntok = 64 if rotate else 1
    layer_gb = (w.E * 3 * w.d * w.f // 32 * 10 + w.E * w.d * 4) / 1e9

    # inputs (each rank holds its own replica)
    bias_list = [None] * copies
    probe = S.MoELayer(w.d, w.f, w.E, w.k, chunk)
    layers = []
    for c in range(copies):
        layers.append(LayerData(S, w, c, probe))
        bias_list[c] = layers[-1].bias
    probe.close()
    if stacked:
        handle = S.MoELayer(w.d, w.f, w.E, w.k, chunk)
    else:
        handle = None
    xs = sd.x_bf16(w.seed, T * ntok, w.d, stream=rank).view(ntok, T, w.d) if not stacked else None
    x_stack0 = None
    if stacked:
        x_stack0 = sd.x_bf16(w.seed, T, w.d, stream=rank).float()
    torch.cuda.synchronize()

    # one layer handle per copy for the single-layer workloads (bias lives in the desc)
    handles = [S.MoELayer(w.d, w.f, w.E, w.k, T, router_bias=layers[c].bias) for c in range(copies)] if not stacked else []
    y = torch.zeros((T, w.d), dtype=torch.float32, device=dev)
    x_res = torch.empty((T, w.d), dtype=torch.float32, device=dev) if stacked else None

    def step(i):
        if stacked:
            handle.stack_forward([l.W for l in layers], [l.bias for l in layers] if w.zipf else None,
                                 [l.blob for l in layers], x_res, T, 1e-6)
        else:
            c = i % copies
            handles[c].forward(xs[i % ntok], layers[c].W, layers[c].blob, y, T)

    # graph of G steps (a whole stack pass is captured by the library itself)
    G = graph_steps(w)
    if stacked:
        x_res.copy_(x_stack0)
    for i in range(2):
        step(i)
    torch.cuda.synchronize()
    graph = None
    if not stacked:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for i in range(G):
                step(i)
        replay = graph.replay
    else:
        replay = lambda: step(0)
    if args.steps % G:
        raise SystemExit(f"--steps must be a multiple of {G} for this workload")
    reps = args.steps // G
    for _ in range(max(args.warmup, 3)):
        replay()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()

    clocks = Clocks(local)
    clocks.start()
    time.sleep(0.3)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        replay()
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1)
    barrier(world)
    ms = dist_max(ms, world)
    ms_step = ms / args.steps
    tokens = T * args.steps * world
    value = tokens / (ms / 1e3)
    print(f"# timed region: {ms_step * 1e3:.2f} us/step, {value:.1f} tokens/s", file=sys.stderr, flush=True)

    # stage timing of the dominant kernel (separate pass, events around it)
    dom = stage_timing(S, w, handles, handle, layers, xs, y, x_res, T, copies, ntok, stacked)
    roof = roofline(w, dom, hbm, tf_burst, peak_src)
    if stacked and T <= 16:
        roof = stack_roofline(S, w, layers, x_stack0, T, ms_step, hbm, peak_src)

    # end to end: pinned host input -> device, forward, result -> host, through the API
    e2e = end_to_end(S, w, handles, handle, layers, T, copies, stacked, world, args)

    # kernels of this library per step: decode = one fused layer kernel;
    # prefill = router GEMM, top-k, list scan, list scatter, gather, two
    # expert GEMMs; stacks add the RMSNorm kernel per layer and chunk on the
    # prefill path (the decode stack fuses it)
    launches_per_step = 1 if T <= 16 else PREFILL_KERNELS
    if stacked:
        per_layer = 1 if T <= 16 else PREFILL_KERNELS + 1
        launches_per_step = w.layers * per_layer * ((T + chunk - 1) // chunk)

    out = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "q2+fp32" if T <= 16 else "q2+fp16->fp32",
        "data": "synthetic (seeded; random-init 2-bit experts)",
        "config": {"workload": w.name, "d_model": w.d, "d_ff": w.f, "n_experts": w.E, "top_k": w.k,
                   "tokens_per_step": T, "layers": w.layers, "routing": "zipf1.1" if w.zipf else "uniform",
                   "l2": (f"inputs larger than L2: {copies} seeded layer copies ({copies * layer_gb:.1f} GB) and 64 token vectors rotated"
                          if rotate else f"inputs larger than L2 ({layer_gb:.2f} GB per layer)"),
                   "parallelism": "replicas" if world > 1 else "single"},
        "roofline": roof,
        "clocks": clk,
        "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps if launches_per_step else None,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(out), flush=True)


def stage_timing(S, w, handles, handle, layers, xs, y, x_res, T, copies, ntok, stacked):
    """Average duration of the dominant expert kernel, from CUDA events the
    library records around it, over one replay of G steps."""
    import torch
    if stacked:
        return None
    G = graph_steps(w)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(G)]
    for e in evs:
        for ev in e:
            ev.record()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(G):
            c = i % copies
            S.strata_moe_set_stage_events(handles[c].handle, evs[i])
            handles[c].forward(xs[i % ntok], layers[c].W, layers[c].blob, y, T)
    for h in handles:
        S.strata_moe_set_stage_events(h.handle, [])
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    dom = [evs[i][2].elapsed_time(evs[i][3]) for i in range(G)]
    tot = [evs[i][0].elapsed_time(evs[i][4]) for i in range(G)]
    # units: selected experts of each step (routing of the last replay)
    n_active = []
    for i in range(G):
        c = i % copies
        handles[c].forward(xs[i % ntok], layers[c].W, layers[c].blob, y, T)
        idx = handles[c].routing(T)[0].cpu().numpy()
        n_active.append(len(set(idx.ravel().tolist())))
    torch.cuda.synchronize()
    return {"dom_ms": float(np.mean(dom)), "step_ms": float(np.mean(tot)), "n_active": float(np.mean(n_active)),
            "T": T}


def decode_bytes(w, n_active):
    """Algorithmic bytes of one decode-layer launch: the selected experts'
    packed weights (all three matrices), the router weights and bias, x and y."""
    return n_active * (3 * w.d * w.f // 32 * 10) + w.E * w.d * 4 + w.E * 4 + w.T * w.d * (2 + 4)


def roofline(w, dom, hbm, tf_burst, peak_src):
    if dom is None:
        return None
    if dom["T"] <= 16:
        bytes_ = decode_bytes(w, dom["n_active"])
        ach = bytes_ / (dom["dom_ms"] * 1e-3) / 1e9
        return {"bound": "hbm", "kernel": "k_decode_fused (whole layer, one launch)", "achieved": ach, "peak": hbm,
                "unit": "GB/s", "frac": ach / hbm, "traffic": MEASURED_TRAFFIC.get(w.name),
                "algorithmic_bytes_per_launch": bytes_, "selected_experts_per_launch": dom["n_active"],
                "avg_launch_ms": dom["dom_ms"], "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)",
                "layer_call_ms": dom["step_ms"]}
    flops = dom["T"] * w.k * 2 * 2 * w.d * w.f
    ach = flops / (dom["dom_ms"] * 1e-3) / 1e12
    return {"bound": "tensor", "kernel": "k_expert_gemm<0> (gate/up + SwiGLU)", "achieved": ach, "peak": tf_burst,
            "unit": "TFLOP/s", "frac": ach / tf_burst, "traffic": MEASURED_TRAFFIC.get(w.name),
            "algorithmic_flops_per_launch": flops,
            "avg_launch_ms": dom["dom_ms"], "peak_source": f"{peak_src} (MEASURED_PEAKS.json bf16_tflops; fp16 same rate)",
            "layer_call_ms": dom["step_ms"],
            "layer_expert_TFLOPs": dom["T"] * w.k * 6 * w.d * w.f / (dom["step_ms"] * 1e-3) / 1e12}


def stack_roofline(S, w, layers, x0, T, ms_step, hbm, peak_src):
    """Decode stack: every layer is one fused launch. The selected experts of
    each layer come from running the same recurrence layer by layer through
    the library (RMSNorm kernel + fused layer with accumulation) and reading
    back each layer's routing; achieved = mean algorithmic bytes per layer /
    (step time / layers)."""
    import torch
    dev = torch.cuda.current_device()
    x = x0.clone()
    xn = torch.empty((T, w.d), dtype=torch.bfloat16, device=dev)
    n_active = []
    for l in range(w.layers):
        h = S.MoELayer(w.d, w.f, w.E, w.k, T, flags=S.STRATA_ACCUMULATE,
                       router_bias=layers[l].bias if w.zipf else None)
        S.strata_rmsnorm_bf16(x, xn, T, w.d, 1e-6)
        h.forward(xn, layers[l].W, layers[l].blob, x, T)
        idx = h.routing(T)[0].cpu().numpy()
        n_active.append(len(set(idx.ravel().tolist())))
        h.close()
    torch.cuda.synchronize()
    per_layer_ms = ms_step / w.layers
    bytes_ = float(np.mean([decode_bytes(w, n) for n in n_active]))
    ach = bytes_ / (per_layer_ms * 1e-3) / 1e9
    return {"bound": "hbm", "kernel": "k_decode_fused (one launch per layer)", "achieved": ach, "peak": hbm,
            "unit": "GB/s", "frac": ach / hbm, "traffic": None, "algorithmic_bytes_per_launch": bytes_,
            "selected_experts_per_launch": float(np.mean(n_active)), "avg_launch_ms": per_layer_ms,
            "avg_launch_ms_source": "step time / layers (the graph replays one launch per layer)",
            "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)"}


def end_to_end(S, w, handles, handle, layers, T, copies, stacked, world, args):
    import torch
    dev = torch.cuda.current_device()
    if stacked:
        xh = torch.empty((T, w.d), dtype=torch.float32).pin_memory()
        xh.copy_(torch.randn(T, w.d))
        outh = torch.empty((T, w.d), dtype=torch.float32).pin_memory()
        xd = torch.empty((T, w.d), dtype=torch.float32, device=dev)
    else:
        xh = torch.empty((64, T, w.d), dtype=torch.bfloat16).pin_memory()
        xh.copy_(torch.randn(64, T, w.d).to(torch.bfloat16))
        outh = torch.empty((T, w.d), dtype=torch.float32).pin_memory()
        xd = torch.empty((T, w.d), dtype=torch.bfloat16, device=dev)
    yd = torch.zeros((T, w.d), dtype=torch.float32, device=dev)
    n = max(8, min(args.steps, 2048 if T <= 16 else 8)) if not stacked else 2

    def one(i):
        if stacked:
            xd.copy_(xh, non_blocking=True)
            handle.stack_forward([l.W for l in layers], [l.bias for l in layers] if w.zipf else None,
                                 [l.blob for l in layers], xd, T, 1e-6)
            outh.copy_(xd, non_blocking=True)
        else:
            c = i % copies
            xd.copy_(xh[i % 64], non_blocking=True)
            handles[c].forward(xd, layers[c].W, layers[c].blob, yd, T)
            outh.copy_(yd, non_blocking=True)

    for i in range(3):
        one(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(n):
        one(i)
    e1.record()
    torch.cuda.synchronize()
    ms = dist_max(e0.elapsed_time(e1), world)
    h2d = T * w.d * (4 if stacked else 2)
    return {"value": T * n * world / (ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": T * w.d * 4, "steps": n,
            "note": "pinned host x -> device, forward through the C ABI (Python binding), y -> pinned host"}


# ---------------------------------------------------------------- CPU oracle


def cpu_baseline(w, seconds):
    """The CPU oracle as it stands, single thread, on a bounded sample."""
    import oracle
    import synth
    W = synth.gen_router_w(w.seed, 0, w.E, w.d)
    bias = synth.router_bias(w, 0)
    src_cache = {}

    def src(e):
        if e not in src_cache:
            src_cache[e] = synth.gen_expert(w.seed, 0, e, w.d, w.f)
        return src_cache[e]

    if w.T <= 16:
        # whole decode steps (route every token + all its experts)
        spent, toks, calls = 0.0, 0, 0
        while spent < seconds and calls < 64:
            x = synth.gen_x_bf16(w.seed, w.T, w.d, stream=100 + calls)
            r = oracle.route_layer(x, W, bias, w.k)
            for t in range(w.T):
                for e in r["idx"][t]:
                    src(int(e))
            t0 = time.perf_counter()
            r = oracle.route_layer(x, W, bias, w.k)
            oracle.layer_outputs(x, r, np.arange(w.T), src)
            spent += time.perf_counter() - t0
            toks += w.T
            calls += 1
        per_tok = spent / toks * (w.layers if w.layers > 1 else 1)
        return {"value": 1.0 / per_tok, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                "sample": f"{calls} calls of {w.T} token(s): routing + all selected experts in fp64"
                          + (f", one layer timed, scaled x{w.layers} layers" if w.layers > 1 else "")}
    # prefill: route a slice of the chunk, experts of a token sample, extrapolated
    n_route = 256
    x = synth.gen_x_bf16(w.seed, n_route, w.d)
    t0 = time.perf_counter()
    r = oracle.route_layer(x, W, bias, w.k)
    t_route = (time.perf_counter() - t0) / n_route
    toks = []
    spent = 0.0
    for t in range(n_route):
        for e in r["idx"][t]:
            src(int(e))
        t0 = time.perf_counter()
        oracle.layer_outputs(x, r, np.array([t]), src)
        spent += time.perf_counter() - t0
        toks.append(t)
        if spent > seconds:
            break
    per_tok = t_route + spent / len(toks)
    per_tok *= (w.layers if w.layers > 1 else 1)
    return {"value": 1.0 / per_tok, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"routing of {n_route} tokens + experts of {len(toks)} tokens (fp64), extrapolated per token"
                      + (f" x{w.layers} layers" if w.layers > 1 else "")}


def run_reference(args, world, rank):
    if rank != 0:
        return
    import synth
    w = synth.WORKLOADS[args.workload]
    per_step = []
    budget = args.cpu_seconds / max(1, args.steps + args.warmup)
    for i in range(args.warmup + args.steps):
        b = cpu_baseline(w, budget)
        if i >= args.warmup:
            per_step.append(b["value"])
    value = float(np.mean(per_step))
    ms_step = 1e3 * w.T / value
    out = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)", "impl": "reference",
           "config": {"workload": w.name, "d_model": w.d, "d_ff": w.f, "n_experts": w.E, "top_k": w.k,
                      "tokens_per_step": w.T, "layers": w.layers},
           "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                            "sample": b["sample"]},
           "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="decode", choices=list(DEFAULT_STEPS))
    ap.add_argument("--impl", default="strata", choices=["strata", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--copies", type=int, default=8,
                    help="single-layer decode sizes: seeded layer copies rotated (8 = 6 GB at 512 experts)")
    args = ap.parse_args()
    if args.steps is None:
        args.steps = DEFAULT_STEPS[args.workload]
        if args.impl == "reference":
            args.steps = 3
    world, rank, local = setup_dist(args)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_strata(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
