"""Benchmark of the routed-expert MoE layer on B200 (synthetic seeded layers).

python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl strata|reference]

A step is one pass of the hot path over one batch: routing (router GEMV or
GEMM, softmax top-k, per-expert lists) and the experts (dequantised 2-bit
gate/up, SwiGLU, down, weighted combine). Workloads (seeded, synthetic):
  decode        d=2048 f=768 E=512 k=10, 1 token per step, uniform routing
  prefill       one layer, 8,192-token chunk, Zipf(1.1) prior
  verify4/16    48-layer stack, 4 or 16 tokens per step, Zipf(1.1) prior
  verify6       48-layer stack, 1 + 5 drafted tokens per step, Zipf(1.1) prior
  coder_decode  as decode with 256 experts per layer (the Coder variant)
  prefill_stack 48 layers, 32,768 tokens in 8,192-token chunks, Zipf(1.1)
With no --workload the run measures both halves of the metric: the JSON line's
top level is the one-token decode layer and its "prefill" block the
8,192-token prefill layer, each timed over exactly --steps steps.

Inputs are resident in HBM before timing; the single-layer decode workloads
rotate over 8 seeded copies of the layer (6 GB at 512 experts) and 64 token
vectors so that no step finds its experts in L2. Multi-GPU runs are
independent replicas (the layer does not shard); value = units over all ranks
/ max-over-ranks time.
"""
from __future__ import annotations

import argparse
import hashlib
import re
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
CSRC = os.path.join(ROOT, "bit_quantized_moe_warp_b200", "csrc")

# DRAM bytes (read + write) of one launch of each workload's dominant kernel
# from one ncu capture (the profile under profiles/ gives the command), with
# the SHA-256 (first 16 hex digits) of the kernel's sources at capture time.
# When the sources differ the figure no longer describes the kernel and the
# line reports traffic null.
MEASURED_TRAFFIC = {
    "decode": {"bytes": 19053312, "sources": ("decode_fused.cu", "common.cuh", "topk.cuh"), "sha": "e59540585b4c4eee"},
    "decode_q4": {"bytes": 30853632, "sources": ("decode_fused.cu", "common.cuh", "topk.cuh"), "sha": "e59540585b4c4eee"},
    "prefill": {"bytes": 683609344, "sources": ("prefill_gemm.cu", "common.cuh"), "sha": "4c18aa910c077009"},
    "prefill_q4": {"bytes": 872128256, "sources": ("prefill_gemm.cu", "common.cuh"), "sha": "4c18aa910c077009"},
    # dram__bytes.sum.per_second x gpu__time_duration.sum of one launch each
    "kv4_128k_encode": {"bytes": 316971249, "sources": ("kv_codec.cu",), "sha": "a1739b8effd04803"},
    "kv4_128k_decode": {"bytes": 286000091, "sources": ("kv_codec.cu",), "sha": "a1739b8effd04803"},
}

# library kernels per single-layer call: decode = the one-launch layer kernel;
# prefill = W split, router GEMM, top-k, list scan, list scatter, gather, two
# expert GEMMs, combine
PREFILL_KERNELS = 9
DECODE_KERNELS = 1

# default timed steps per workload when --steps is not given
DEFAULT_STEPS = {"decode": 64 * 1024, "verify4": 200, "verify6": 150, "verify16": 100, "prefill": 200,
                 "prefill_stack": 3, "coder_decode": 64 * 1024,
                 "decode_q4": 64 * 1024, "verify4_q4": 200, "prefill_q4": 200}


def graph_steps(w) -> int:
    """Largest number of steps one CUDA-graph replay covers: 64 single-layer
    decode calls, 8 prefill chunks, or one whole stack pass (captured by the
    library itself)."""
    if w.layers > 1:
        return 1
    return 64 if w.T <= 16 else 8


def step_plan(steps: int, G: int):
    """(graph size, replays, remainder): exactly `steps` steps are timed as
    `replays` replays of a graph of `size` steps plus one replay of a graph of
    `remainder` steps (0: none)."""
    if steps < 1:
        raise ValueError("--steps must be >= 1")
    size = min(G, steps)
    reps = steps // size
    return size, reps, steps - reps * size


def sources_sha(names) -> str:
    """SHA-256 (16 hex digits) of the kernel sources' code: comments and
    blank lines are left out, so a comment edit keeps the recorded figure."""
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(CSRC, n), encoding="utf-8") as fh:
            text = re.sub(r"/\*.*?\*/", "", fh.read(), flags=re.S)
        for line in text.splitlines():
            code = line.split("//", 1)[0].rstrip()
            if code:
                h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


def measured_traffic(name: str):
    """(bytes, note): the ncu figure of the workload's dominant kernel, or
    None when there is none or the kernel's sources changed since."""
    m = MEASURED_TRAFFIC.get(name)
    if m is None:
        return None, "no capture of this shape"
    if sources_sha(m["sources"]) != m["sha"]:
        return None, "kernel changed since the last ncu capture"
    return m["bytes"], "ncu dram__bytes_read.sum + dram__bytes_write.sum, one launch"


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


# ---------------------------------------------------------------- algorithmic units


def expert_bytes(w) -> int:
    """Packed bytes of one expert: 3 matrices of d*f weights, 10 bytes per 32
    (2-bit codes + fp16 scale) or 18 (4-bit codes + fp16 scale)."""
    return 3 * w.d * w.f // 32 * (10 if w.bits == 2 else 18)


def decode_bytes(w, n_active):
    """Algorithmic bytes of one decode-layer launch: the selected experts'
    packed weights (all three matrices), the router weights and bias, x and y."""
    return n_active * expert_bytes(w) + w.E * w.d * 4 + w.E * 4 + w.T * w.d * (2 + 4)


def expert_flops(w, tokens) -> int:
    """Expert FLOPs of `tokens` tokens: k experts x (gate, up, down) x 2 d f."""
    return tokens * w.k * 6 * w.d * w.f


# ---------------------------------------------------------------- one workload


class Runner:
    """Inputs, handles and the step function of one workload on this rank."""

    def __init__(self, S, w, rank, copies_arg):
        import torch
        import synth.device as sd
        self.S, self.w = S, w
        self.dev = torch.device("cuda", torch.cuda.current_device())
        self.stacked = w.layers > 1
        self.T = w.T
        self.chunk = min(w.T, w.chunk)
        self.rotate = not self.stacked and w.T <= 16
        self.copies = copies_arg if self.rotate else (w.layers if self.stacked else 1)
        self.ntok = 64 if self.rotate else 1
        self.layer_gb = (w.E * expert_bytes(w) + w.E * w.d * 4) / 1e9
        probe = S.MoELayer(w.d, w.f, w.E, w.k, self.chunk, bits=w.bits)
        self.layers = [LayerData(S, w, c, probe) for c in range(self.copies)]
        probe.close()
        T = w.T
        if self.stacked:
            self.handle = S.MoELayer(w.d, w.f, w.E, w.k, self.chunk, bits=w.bits)
            self.handles = []
            self.x0 = sd.x_bf16(w.seed, T, w.d, stream=rank).float()
            self.x_res = torch.empty((T, w.d), dtype=torch.float32, device=self.dev)
            self.xs = None
        else:
            self.handle = None
            self.handles = [S.MoELayer(w.d, w.f, w.E, w.k, T, router_bias=self.layers[c].bias, bits=w.bits)
                            for c in range(self.copies)]
            self.xs = sd.x_bf16(w.seed, T * self.ntok, w.d, stream=rank).view(self.ntok, T, w.d)
            self.x_res = None
        self.y = torch.zeros((T, w.d), dtype=torch.float32, device=self.dev)
        torch.cuda.synchronize()

    def step(self, i):
        w = self.w
        if self.stacked:
            self.handle.stack_forward([l.W for l in self.layers], [l.bias for l in self.layers] if w.zipf else None,
                                      [l.blob for l in self.layers], self.x_res, self.T, 1e-6)
        else:
            c = i % self.copies
            self.handles[c].forward(self.xs[i % self.ntok], self.layers[c].W, self.layers[c].blob, self.y, self.T)

    def graph(self, n):
        """A replay function covering steps 0..n-1 (a CUDA graph for the single
        layer; the library captures and replays a whole stack pass itself)."""
        import torch
        if self.stacked:
            assert n == 1
            return lambda: self.step(0)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(n):
                self.step(i)
        self._keep = getattr(self, "_keep", []) + [g]
        return g.replay

    def close(self):
        for h in self.handles:
            h.close()
        if self.handle is not None:
            self.handle.close()
        self.layers = []


def time_steps(run, steps, warmup, world):
    """Exactly `steps` steps timed with CUDA events on the launching stream,
    after `warmup` untimed ones; returns the max over ranks in ms."""
    import torch
    stream = torch.cuda.current_stream()
    size, reps, rem = step_plan(steps, graph_steps(run.w))
    if run.stacked:
        run.x_res.copy_(run.x0)
    for i in range(2):
        run.step(i)
    torch.cuda.synchronize()
    main = run.graph(size)
    tail = run.graph(rem) if rem else None
    for _ in range(-(-max(warmup, 3) // size)):  # at least max(warmup, 3) untimed steps
        main()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        main()
    if tail is not None:
        tail()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    barrier(world)
    return dist_max(ms, world), {"graph_steps": size, "replays": reps, "remainder_steps": rem}


def stage_timing(run):
    """Average duration of the dominant expert kernel (prefill: the gate/up
    GEMM), from CUDA events the library records around it on the same stream,
    over one replay of a graph of 8 steps."""
    import torch
    S = run.S
    G = graph_steps(run.w)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(G)]
    for e in evs:
        for ev in e:
            ev.record()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(G):
            c = i % run.copies
            S.strata_moe_set_stage_events(run.handles[c].handle, evs[i])
            run.step(i)
    for h in run.handles:
        S.strata_moe_set_stage_events(h.handle, [])
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    dom = [evs[i][2].elapsed_time(evs[i][3]) for i in range(G)]
    tot = [evs[i][0].elapsed_time(evs[i][4]) for i in range(G)]
    return float(np.mean(dom)), float(np.mean(tot))


def active_experts(run, n):
    """Mean number of distinct selected experts over steps 0..n-1 (routing
    read back from the library after each call)."""
    import torch
    out = []
    for i in range(n):
        c = i % run.copies
        run.step(i)
        idx = run.handles[c].routing(run.T)[0].cpu().numpy()
        out.append(len(set(idx.ravel().tolist())))
    torch.cuda.synchronize()
    return float(np.mean(out))


def stack_active_experts(run):
    """Distinct selected experts of each layer of a decode stack, from the same
    recurrence run layer by layer through the library (RMSNorm kernel + layer
    call with accumulation) and each layer's routing read back."""
    import torch
    S, w, T = run.S, run.w, run.T
    x = run.x0.clone()
    xn = torch.empty((T, w.d), dtype=torch.bfloat16, device=run.dev)
    n_active = []
    for l in range(w.layers):
        h = S.MoELayer(w.d, w.f, w.E, w.k, T, flags=S.STRATA_ACCUMULATE, bits=w.bits,
                       router_bias=run.layers[l].bias if w.zipf else None)
        S.strata_rmsnorm_bf16(x, xn, T, w.d, 1e-6)
        h.forward(xn, run.layers[l].W, run.layers[l].blob, x, T)
        idx = h.routing(T)[0].cpu().numpy()
        n_active.append(len(set(idx.ravel().tolist())))
        h.close()
    torch.cuda.synchronize()
    return n_active


def decode_roofline(w, n_active, ms_per_launch, hbm, peak_src, launch_src):
    """HBM roofline of the one-launch decode layer on the selected experts'
    packed bytes (router bytes reported beside it)."""
    sel = n_active * expert_bytes(w)
    router = w.E * w.d * 4 + w.E * 4
    alg = decode_bytes(w, n_active)
    ach = sel / (ms_per_launch * 1e-3) / 1e9
    traffic, tnote = measured_traffic(w.name)
    return {"bound": "hbm", "kernel": "k_decode_fused (whole layer, one launch)", "achieved": ach, "peak": hbm,
            "unit": "GB/s", "frac": ach / hbm, "traffic": traffic, "traffic_note": tnote,
            "bytes_basis": "selected experts' packed weights (gate, up, down)",
            "selected_expert_bytes_per_launch": sel, "selected_experts_per_launch": n_active,
            "router_bytes_per_launch": router,
            "all_algorithmic_bytes_per_launch": alg,
            "achieved_all_bytes_gbs": alg / (ms_per_launch * 1e-3) / 1e9,
            "avg_launch_ms": ms_per_launch, "avg_launch_ms_source": launch_src,
            "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)"}


def prefill_roofline(w, dom_ms, layer_ms, peak, peak_src, peak_kind):
    """Tensor roofline of the gate/up GEMM (the dominant kernel) and of the
    whole layer on its expert FLOPs."""
    flops = w.T * w.k * 2 * 2 * w.d * w.f
    ach = flops / (dom_ms * 1e-3) / 1e12
    layer = expert_flops(w, w.T) / (layer_ms * 1e-3) / 1e12
    traffic, tnote = measured_traffic(w.name)
    return {"bound": "tensor", "kernel": f"k_expert_gemm<0, {w.bits}> (gate/up + SwiGLU)", "achieved": ach, "peak": peak,
            "unit": "TFLOP/s", "frac": ach / peak, "traffic": traffic, "traffic_note": tnote,
            "algorithmic_flops_per_launch": flops, "avg_launch_ms": dom_ms,
            "avg_launch_ms_source": "CUDA events recorded by the library around the kernel, inside the graph",
            "layer_expert_flops": expert_flops(w, w.T), "layer_ms": layer_ms,
            "layer_achieved": layer, "layer_frac": layer / peak,
            "peak_source": f"{peak_src} (MEASURED_PEAKS.json bf16_tflops {peak_kind}; fp16 kind::f16 runs at the same rate)"}


def measure(S, w, args, world, rank, local):
    """One workload: the timed region, roofline, end-to-end and CPU baseline;
    returns the JSON block (rank 0's view)."""
    import torch
    hbm, tf_burst, tf_sust, peak_src = load_peaks()
    steps = args.steps if args.steps is not None else DEFAULT_STEPS[w.name]
    run = Runner(S, w, rank, args.copies)
    clocks = Clocks(local)
    clocks.start()
    time.sleep(0.3)
    ms, plan = time_steps(run, steps, args.warmup, world)
    clk = clocks.stop()
    ms_step = ms / steps
    value = w.T * steps * world / (ms / 1e3)
    print(f"# {w.name}: {ms_step * 1e3:.2f} us/step, {value:.1f} tokens/s", file=sys.stderr, flush=True)

    T = w.T
    if not run.stacked and T <= 16:
        n_act = active_experts(run, min(steps, 64))
        roof = decode_roofline(w, n_act, ms_step, hbm, peak_src,
                               "graph-timed step (one kernel per step)")
    elif run.stacked and T <= 16:
        n_act = stack_active_experts(run)
        roof = decode_roofline(w, float(np.mean(n_act)), ms_step / w.layers, hbm, peak_src,
                               "step time / layers (the graph replays one launch per layer)")
    elif not run.stacked:
        dom_ms, _ = stage_timing(run)
        roof = prefill_roofline(w, dom_ms, ms_step, tf_burst, peak_src, "burst")
    else:
        layer_ms = ms_step / w.layers / (T // run.chunk)
        flops = expert_flops(w, run.chunk)
        ach = flops / (layer_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "kernel": "whole prefill layer (per 8,192-token chunk)", "achieved": ach,
                "peak": tf_sust, "unit": "TFLOP/s", "frac": ach / tf_sust, "traffic": None,
                "traffic_note": "no capture of this shape", "avg_launch_ms": layer_ms,
                "avg_launch_ms_source": "step time / (layers x chunks)",
                "peak_source": f"{peak_src} (MEASURED_PEAKS.json bf16_tflops_sustained)"}

    e2e = end_to_end(run, steps, world)
    if T <= 16:
        per_layer = DECODE_KERNELS
    else:
        per_layer = PREFILL_KERNELS + (1 if run.stacked else 0)
    launches = per_layer * w.layers * ((T + run.chunk - 1) // run.chunk) * steps
    block = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": f"q{w.bits}+fp32" if T <= 16 else f"q{w.bits}+fp16->fp32",
        "data": f"synthetic (seeded; random-init {w.bits}-bit experts)",
        "config": {"workload": w.name, "d_model": w.d, "d_ff": w.f, "n_experts": w.E, "top_k": w.k,
                   "tokens_per_step": T, "layers": w.layers, "routing": "zipf1.1" if w.zipf else "uniform",
                   "l2": (f"inputs larger than L2: {run.copies} seeded layer copies "
                          f"({run.copies * run.layer_gb:.1f} GB) and 64 token vectors rotated"
                          if run.rotate else f"inputs larger than L2 ({run.layer_gb:.2f} GB per layer)"),
                   "parallelism": "replicas" if world > 1 else "single", "timing": plan},
        "roofline": roof,
        "clocks": clk,
        "e2e": e2e,
        "gpu_launches": launches,
    }
    run.close()
    del run
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        block["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
    return block


def end_to_end(run, steps, world):
    """The same metric through the public API with host buffers: every step
    copies that step's x from pinned host memory, runs the layer (or stack)
    through the C ABI and reads y back into pinned host memory. Single layers
    of more than 16 tokens run as a two-buffer pipeline, as a serving loop
    does: the input and output copies (own streams, ordered by events) overlap
    the neighbouring steps' layer calls. At 16 tokens or fewer the copies are
    a few KB and the extra stream and event calls cost more host time than
    they hide, so the steps run on one stream."""
    import torch
    S, w, T = run.S, run.w, run.T
    dev = run.dev
    n = max(8, min(steps, 2048 if T <= 16 else 8)) if not run.stacked else 2
    h2d = T * w.d * (4 if run.stacked else 2)
    d2h = T * w.d * 4
    if not run.stacked and T <= 16:
        xh = torch.empty((64, T, w.d), dtype=torch.bfloat16).pin_memory()
        xh.copy_(torch.randn(64, T, w.d).to(torch.bfloat16))
        outh = torch.empty((T, w.d), dtype=torch.float32).pin_memory()
        xd = torch.empty((T, w.d), dtype=torch.bfloat16, device=dev)
        yd = torch.zeros((T, w.d), dtype=torch.float32, device=dev)
        st = torch.cuda.current_stream().cuda_stream
        args = [(run.handles[c].handle, run.layers[c].W.data_ptr(), run.layers[c].blob.data_ptr())
                for c in range(run.copies)]
        xp, yp = xd.data_ptr(), yd.data_ptr()
        xhs = [xh[i] for i in range(64)]

        def one(i):
            h, Wp, bp = args[i % run.copies]
            xd.copy_(xhs[i % 64], non_blocking=True)
            S.strata_moe_forward(h, xp, Wp, bp, yp, T, st)
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
        return {"value": T * n * world / (ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": n,
                "note": "every step: pinned host x -> device, forward through the C ABI (Python binding), "
                        "y -> pinned host, on one stream"}
    if run.stacked:
        xh = torch.empty((T, w.d), dtype=torch.float32).pin_memory()
        xh.copy_(torch.randn(T, w.d))
        outh = torch.empty((T, w.d), dtype=torch.float32).pin_memory()
        xd = torch.empty((T, w.d), dtype=torch.float32, device=dev)

        def one(i):
            xd.copy_(xh, non_blocking=True)
            run.handle.stack_forward([l.W for l in run.layers], [l.bias for l in run.layers] if w.zipf else None,
                                     [l.blob for l in run.layers], xd, T, 1e-6)
            outh.copy_(xd, non_blocking=True)

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
        return {"value": T * n * world / (ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": n,
                "note": "pinned host x -> device, stack through the C ABI (Python binding), x -> pinned host"}

    nx = 2
    xh = torch.empty((nx, T, w.d), dtype=torch.bfloat16).pin_memory()
    xh.copy_(torch.randn(nx, T, w.d).to(torch.bfloat16))
    outh = [torch.empty((T, w.d), dtype=torch.float32).pin_memory() for _ in range(2)]
    xd = [torch.empty((T, w.d), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    yd = [torch.zeros((T, w.d), dtype=torch.float32, device=dev) for _ in range(2)]
    s_c = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]   # x buffer b filled
    ev_k = [torch.cuda.Event() for _ in range(2)]    # layer call on buffer b done
    ev_out = [torch.cuda.Event() for _ in range(2)]  # y buffer b copied out
    st = s_c.cuda_stream
    # the layer call with plain device addresses and the stream handle
    args = [(run.handles[c].handle, run.layers[c].W.data_ptr(), run.layers[c].blob.data_ptr())
            for c in range(run.copies)]
    xp, yp = [t.data_ptr() for t in xd], [t.data_ptr() for t in yd]
    xhs = [xh[i] for i in range(nx)]

    def one(i):
        b = i & 1
        if i >= 2:
            s_in.wait_event(ev_k[b])       # the call two steps back has read xd[b]
        with torch.cuda.stream(s_in):
            xd[b].copy_(xhs[i % nx], non_blocking=True)
        ev_in[b].record(s_in)
        s_c.wait_event(ev_in[b])
        if i >= 2:
            s_c.wait_event(ev_out[b])      # yd[b] of two steps back is on the host
        h, Wp, bp = args[i % run.copies]
        S.strata_moe_forward(h, xp[b], Wp, bp, yp[b], T, st)
        ev_k[b].record(s_c)
        s_out.wait_event(ev_k[b])
        with torch.cuda.stream(s_out):
            outh[b].copy_(yd[b], non_blocking=True)
        ev_out[b].record(s_out)

    for i in range(4):
        one(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_c)
    s_in.wait_event(e0)
    s_out.wait_event(e0)
    for i in range(n):
        one(i)
    s_c.wait_stream(s_out)
    e1.record(s_c)
    torch.cuda.synchronize()
    ms = dist_max(e0.elapsed_time(e1), world)
    return {"value": T * n * world / (ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": n,
            "note": "every step: pinned host x -> device, forward through the C ABI (Python binding), "
                    "y -> pinned host; two buffers, copies on their own streams overlapping the neighbouring "
                    "steps' layer calls"}


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
            src_cache[e] = synth.gen_expert(w.seed, 0, e, w.d, w.f, w.bits)
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


# ---------------------------------------------------------------- KV codec


KV_STEPS = 50
KV_KERNELS = ("k_kv4_encode<128>", "k_kv4_decode<128>")


def kv_bytes(w) -> int:
    """Algorithmic bytes of one encode (or one decode) launch over all rows:
    bf16 rows (2 bytes per value) + codes (0.5) + fp16 scales (1/16)."""
    return w.rows * w.D * 2 + w.rows * w.D // 2 + w.rows * (w.D // 32) * 2


def kv_cpu_baseline(w, seconds):
    """The oracle's encode + decode on the host, on consecutive rows of the
    same workload until the time budget is spent."""
    import oracle
    import synth
    oracle.load()
    el = 0.0  # oracle time only; drawing the rows is not timed
    rows = 0
    chunk = 2048
    while el < seconds or rows == 0:
        x = synth.gen_kv_rows(w.seed, chunk, w.D, row0=rows)
        t1 = time.perf_counter()
        c, sc = oracle.kv4_encode(x)
        oracle.kv4_decode(c, sc)
        el += time.perf_counter() - t1
        rows += chunk
    return {"value": rows / (w.kv_heads * 2) / el, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{rows} rows ({rows // (w.kv_heads * 2)} tokens) of {w.name}, encode + fp64 decode"}


def measure_kv(S, w, args, world, rank, local):
    """The codec over one layer's 128K-token K and V cache: a step encodes every
    row and decodes every row; encode writes one of two code buffers while
    decode reads the other (written a step earlier, since evicted from L2)."""
    import torch
    import synth.device as sdev
    hbm, _, _, peak_src = load_peaks()
    steps = args.steps if args.steps is not None else KV_STEPS
    n, D = w.rows, w.D
    dev = torch.device("cuda", local)
    x = sdev.kv_rows(w.seed, n, D)
    codes = [torch.empty((n, D // 2), dtype=torch.uint8, device=dev) for _ in range(2)]
    scales = [torch.empty((n, D // 32), dtype=torch.int16, device=dev) for _ in range(2)]
    out = torch.empty((n, D), dtype=torch.bfloat16, device=dev)
    S.strata_kv4_encode(x, n, D, codes[1], scales[1])
    st = torch.cuda.current_stream()

    def step(i):
        a, b = i % 2, (i + 1) % 2
        S.strata_kv4_encode(x, n, D, codes[a], scales[a])
        S.strata_kv4_decode(codes[b], scales[b], n, D, out)

    for i in range(max(3, args.warmup)):
        step(i)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    clocks = Clocks(local)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(st)
    for i in range(steps):
        e0, e1, e2 = ev[i]
        e0.record(st)
        S.strata_kv4_encode(x, n, D, codes[i % 2], scales[i % 2])
        e1.record(st)
        S.strata_kv4_decode(codes[(i + 1) % 2], scales[(i + 1) % 2], n, D, out)
        e2.record(st)
    t_end.record(st)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    ms = dist_max(t_start.elapsed_time(t_end), world)
    enc_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in ev]))
    dec_ms = float(np.mean([e[1].elapsed_time(e[2]) for e in ev]))
    ms_step = ms / steps
    value = w.tokens * steps * world / (ms / 1e3)
    print(f"# {w.name}: {ms_step * 1e3:.2f} us/step (encode {enc_ms * 1e3:.2f} us, decode {dec_ms * 1e3:.2f} us), "
          f"{value:.4g} tokens/s", file=sys.stderr, flush=True)
    nb = kv_bytes(w)
    kern = {"encode": {"avg_launch_ms": enc_ms, "achieved_gbs": nb / (enc_ms * 1e-3) / 1e9,
                       "frac": nb / (enc_ms * 1e-3) / 1e9 / hbm},
            "decode": {"avg_launch_ms": dec_ms, "achieved_gbs": nb / (dec_ms * 1e-3) / 1e9,
                       "frac": nb / (dec_ms * 1e-3) / 1e9 / hbm}}
    dom = "encode" if enc_ms >= dec_ms else "decode"
    dms = kern[dom]["avg_launch_ms"]
    ach = nb / (dms * 1e-3) / 1e9
    traffic, tnote = measured_traffic(f"{w.name}_{dom}")
    for k in kern:
        kern[k]["traffic"], _ = measured_traffic(f"{w.name}_{k}")
    roof = {"bound": "hbm", "kernel": KV_KERNELS[0 if dom == "encode" else 1], "achieved": ach, "peak": hbm,
            "unit": "GB/s", "frac": ach / hbm, "traffic": traffic, "traffic_note": tnote,
            "algorithmic_bytes_per_launch": nb,
            "bytes_basis": "bf16 rows + 4-bit codes + fp16 scales, each moved once",
            "avg_launch_ms": dms, "avg_launch_ms_source": "CUDA events around each launch on its stream",
            "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)", "kernels": kern}
    e2e = kv_end_to_end(S, w, x, codes[0], scales[0], out, min(steps, 8), world)
    block = {
        "metric": "4-bit rotated KV codec: cached tokens/s (one layer's K and V encoded + decoded)",
        "value": value, "unit": "tokens/s", "n_gpus": world, "steps": steps, "warmup": max(3, args.warmup),
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32 (bf16 rows in and out, 4-bit codes + fp16 scales)",
        "data": "synthetic (seeded N(0,1) rows, 4 outlier channels x16)",
        "config": {"workload": w.name, "tokens": w.tokens, "kv_heads": w.kv_heads, "head_dim": D, "rows": n,
                   "l2": (f"inputs larger than L2 ({nb / 1e9:.2f} GB per launch); decode reads the codes the "
                          "previous step wrote"),
                   "parallelism": "replicas" if world > 1 else "single"},
        "roofline": roof, "clocks": clk, "e2e": e2e, "gpu_launches": 2 * steps,
    }
    del x, codes, scales, out
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        block["cpu_baseline"] = kv_cpu_baseline(w, args.cpu_seconds)
    return block


def kv_end_to_end(S, w, x, codes, scales, out, steps, world):
    """Through the C ABI from pinned host rows to pinned host rows: per step
    the rows go up, are encoded and decoded, and the decoded rows come back."""
    import torch
    n, D = w.rows, w.D
    hx = torch.empty((n, D), dtype=torch.bfloat16, pin_memory=True)
    hx.copy_(x, non_blocking=False)
    ho = torch.empty((n, D), dtype=torch.bfloat16, pin_memory=True)
    st = torch.cuda.current_stream()
    barrier(world)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(st)
    for _ in range(steps):
        x.copy_(hx, non_blocking=True)
        S.strata_kv4_encode(x, n, D, codes, scales)
        S.strata_kv4_decode(codes, scales, n, D, out)
        ho.copy_(out, non_blocking=True)
    b.record(st)
    torch.cuda.synchronize()
    ms = dist_max(a.elapsed_time(b), world)
    nbytes = n * D * 2
    return {"value": w.tokens * steps * world / (ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": nbytes,
            "d2h_bytes_per_step": nbytes, "steps": steps}


def kv_reference_block(w, args, world):
    steps = args.steps if args.steps is not None else 3
    budget = args.cpu_seconds / max(1, steps + args.warmup)
    vals = []
    b = None
    for i in range(args.warmup + steps):
        b = kv_cpu_baseline(w, budget)
        if i >= args.warmup:
            vals.append(b["value"])
    value = float(np.mean(vals))
    return {"metric": "4-bit rotated KV codec: cached tokens/s (one layer's K and V encoded + decoded)",
            "value": value, "unit": "tokens/s", "n_gpus": world, "steps": steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * w.tokens / value, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32 encode, f64 decode", "data": "synthetic (seeded)",
            "impl": "reference", "config": {"workload": w.name, "tokens": w.tokens, "kv_heads": w.kv_heads,
                                            "head_dim": w.D, "rows": w.rows},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                             "sample": f"each step: {b['sample']}"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def workloads_of(args):
    """(top-level workload, nested blocks): the default run is the one-token
    decode layer with the 8,192-token prefill layer nested."""
    import synth
    if args.workload is None:
        return synth.WORKLOADS["decode"], [("prefill", synth.WORKLOADS["prefill"])]
    return synth.WORKLOADS[args.workload], []


def reference_block(w, args, world):
    steps = args.steps if args.steps is not None else 3
    per_step = []
    budget = args.cpu_seconds / max(1, steps + args.warmup)
    b = None
    for i in range(args.warmup + steps):
        b = cpu_baseline(w, budget)
        if i >= args.warmup:
            per_step.append(b["value"])
    value = float(np.mean(per_step))
    ms_step = 1e3 * w.T / value
    return {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)", "impl": "reference",
            "config": {"workload": w.name, "d_model": w.d, "d_ff": w.f, "n_experts": w.E, "top_k": w.k,
                       "tokens_per_step": w.T, "layers": w.layers},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                             "sample": f"each step: {b['sample']}"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_reference(args, world, rank):
    """The oracle timed on the host cores on this arm's workloads (rank 0 only)."""
    if rank != 0:
        return
    import synth
    if args.workload in synth.KV_WORKLOADS:
        print(json.dumps(kv_reference_block(synth.KV_WORKLOADS[args.workload], args, world)), flush=True)
        return
    top, nested = workloads_of(args)
    out = reference_block(top, args, world)
    for key, w in nested:
        # the nested block is one bounded sample (its own cpu_seconds budget)
        nargs = argparse.Namespace(**vars(args))
        nargs.steps, nargs.warmup = 1, 0
        out[key] = reference_block(w, nargs, world)
    print(json.dumps(out), flush=True)


def run_strata(args, world, rank, local):
    import bit_quantized_moe_warp_b200 as S
    import synth
    if args.workload in synth.KV_WORKLOADS:
        out = measure_kv(S, synth.KV_WORKLOADS[args.workload], args, world, rank, local)
        if rank == 0:
            print(json.dumps(out), flush=True)
        return
    top, nested = workloads_of(args)
    out = measure(S, top, args, world, rank, local)
    for key, w in nested:
        out[key] = measure(S, w, args, world, rank, local)
    if rank == 0:
        print(json.dumps(out), flush=True)


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=None, choices=list(DEFAULT_STEPS) + ["kv4_128k"],
                    help="one workload only (default: decode, with the prefill layer nested); kv4_128k: "
                         "the 4-bit rotated KV-cache codec")
    ap.add_argument("--impl", default="strata", choices=["strata", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--copies", type=int, default=8,
                    help="single-layer decode sizes: seeded layer copies rotated (8 = 6 GB at 512 experts)")
    args = ap.parse_args(argv)
    if args.steps is not None and args.steps < 1:
        ap.error("--steps must be >= 1")
    if args.warmup < 0:
        ap.error("--warmup must be >= 0")
    return args


def main():
    args = parse_args()
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
