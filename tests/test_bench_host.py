"""bench.py on CPU: the command line the benchmark is run with, the step plan
that times exactly --steps steps for every workload, and the algorithmic
units the roofline divides by."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synth  # noqa: E402


def test_default_steps_name_generated_workloads():
    for name, steps in bench.DEFAULT_STEPS.items():
        assert name in synth.WORKLOADS, name
        assert steps > 0


def test_graph_steps_by_shape():
    W = synth.WORKLOADS
    assert bench.graph_steps(W["decode"]) == 64          # single layer, 1 token
    assert bench.graph_steps(W["coder_decode"]) == 64
    assert bench.graph_steps(W["prefill"]) == 8          # single layer, 8,192 tokens
    for name in ("verify4", "verify6", "verify16", "prefill_stack"):
        assert bench.graph_steps(W[name]) == 1           # the library captures the whole stack


@pytest.mark.parametrize("steps", [1, 3, 7, 8, 9, 20, 63, 64, 65, 100, 200, 64 * 1024, 64 * 1024 + 5])
def test_step_plan_times_exactly_the_requested_steps(steps):
    for name, w in synth.WORKLOADS.items():
        G = bench.graph_steps(w)
        size, reps, rem = bench.step_plan(steps, G)
        assert 1 <= size <= G and reps >= 1 and 0 <= rem < size, (name, steps)
        assert size * reps + rem == steps, (name, steps)


def test_driver_command_line_parses_and_plans_every_workload():
    args = bench.parse_args(["--gpus", "1", "--steps", "20", "--warmup", "5"])
    assert (args.gpus, args.steps, args.warmup, args.workload, args.impl) == (1, 20, 5, None, "strata")
    top, nested = bench.workloads_of(args)
    assert top.name == "decode" and [k for k, _ in nested] == ["prefill"]
    assert nested[0][1].T == 8192
    for w in [top] + [v for _, v in nested] + list(synth.WORKLOADS.values()):
        size, reps, rem = bench.step_plan(args.steps, bench.graph_steps(w))
        assert size * reps + rem == 20
    ref = bench.parse_args(["--impl", "reference", "--gpus", "1", "--steps", "20", "--warmup", "5"])
    assert ref.impl == "reference" and ref.steps == 20


def test_bad_step_counts_are_rejected():
    with pytest.raises(SystemExit):
        bench.parse_args(["--steps", "0"])
    with pytest.raises(ValueError):
        bench.step_plan(0, 64)


def test_decode_bytes_counts_selected_experts_router_and_activations():
    w = synth.WORKLOADS["decode"]
    per_expert = 3 * w.d * w.f // 32 * 10                # 2 bits + fp16 scale per 32 weights
    assert per_expert == bench.expert_bytes(w) == 1474560
    assert bench.decode_bytes(w, 10) == 10 * per_expert + w.E * w.d * 4 + w.E * 4 + w.T * w.d * 6
    assert bench.decode_bytes(w, 10) == 18954240


def test_decode_roofline_is_on_selected_expert_bytes_over_the_step():
    w = synth.WORKLOADS["decode"]
    r = bench.decode_roofline(w, 10.0, 0.01, 6500.0, "fallback", "graph-timed step")
    assert r["selected_expert_bytes_per_launch"] == 14745600
    assert abs(r["achieved"] - 14745600 / 1e-5 / 1e9) < 1e-6
    assert abs(r["frac"] - r["achieved"] / 6500.0) < 1e-12
    assert r["router_bytes_per_launch"] == w.E * w.d * 4 + w.E * 4


def test_prefill_flops():
    w = synth.WORKLOADS["prefill"]
    assert bench.expert_flops(w, w.T) == 8192 * 10 * 6 * 2048 * 768   # 773.1 GFLOP
    r = bench.prefill_roofline(w, 0.5, 1.0, 1600.0, "fallback", "burst")
    assert abs(r["layer_achieved"] - 773.094113280) < 1e-6
    assert abs(r["achieved"] - 515.39607552 / 0.5) < 1e-6


def test_traffic_is_dropped_when_kernel_sources_change():
    m = bench.MEASURED_TRAFFIC["decode"]
    saved = m["sha"]
    try:
        m["sha"] = bench.sources_sha(m["sources"])
        assert bench.measured_traffic("decode")[0] == m["bytes"]
        m["sha"] = "0" * 16
        assert bench.measured_traffic("decode")[0] is None
    finally:
        m["sha"] = saved


def test_traffic_guard_ignores_comments_only(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("// header\n__global__ void k(int *p) {\n    p[0] = 1;  // store\n}\n")
    monkeypatch.setattr(bench, "CSRC", str(tmp_path))
    h0 = bench.sources_sha(("k.cu",))
    src.write_text("/* a longer\n   header */\n__global__ void k(int *p) {\n\n    p[0] = 1;  // the store\n}\n")
    assert bench.sources_sha(("k.cu",)) == h0
    src.write_text("// header\n__global__ void k(int *p) {\n    p[0] = 2;  // store\n}\n")
    assert bench.sources_sha(("k.cu",)) != h0



def test_kv_workload_bytes_and_command_line():
    """The KV codec's line: the workload is accepted, its algorithmic bytes are
    2 + 0.5 + 1/16 bytes per value, and the recorded traffic matches the
    kernel's current code."""
    w = synth.KV_WORKLOADS["kv4_128k"]
    assert w.rows == 131072 * 4 * 2 and w.D == 128
    assert bench.kv_bytes(w) == w.rows * w.D * 2 + w.rows * w.D // 2 + w.rows * (w.D // 32) * 2 == 343932928
    args = bench.parse_args(["--workload", "kv4_128k", "--steps", "20", "--warmup", "5"])
    assert args.workload == "kv4_128k"
    for kern in ("encode", "decode"):
        b, note = bench.measured_traffic(f"kv4_128k_{kern}")
        assert b is not None, note
        assert 0.5 * bench.kv_bytes(w) < b <= bench.kv_bytes(w) * 1.05


def test_kv_reference_arm_prints_one_line(capsys):
    args = bench.parse_args(["--impl", "reference", "--workload", "kv4_128k", "--steps", "1", "--warmup", "0",
                             "--cpu-seconds", "0.05"])
    bench.run_reference(args, 1, 0)
    import json
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["config"]["workload"] == "kv4_128k"
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
