"""bench.py's workload table on CPU: every benchmarked workload exists in the
seeded generators, and every default step count is a whole number of CUDA-graph
replays (bench.py rejects any other count at run time)."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synth  # noqa: E402


def test_default_steps_cover_whole_graph_replays():
    for name, steps in bench.DEFAULT_STEPS.items():
        assert name in synth.WORKLOADS, name
        w = synth.WORKLOADS[name]
        assert steps > 0 and steps % bench.graph_steps(w) == 0, (name, steps, bench.graph_steps(w))


def test_graph_steps_by_shape():
    W = synth.WORKLOADS
    assert bench.graph_steps(W["decode"]) == 64          # single layer, 1 token
    assert bench.graph_steps(W["coder_decode"]) == 64
    assert bench.graph_steps(W["prefill"]) == 8          # single layer, 8,192 tokens
    for name in ("verify4", "verify6", "verify16", "prefill_stack"):
        assert bench.graph_steps(W[name]) == 1           # the library captures the whole stack


def test_decode_bytes_counts_selected_experts_router_and_activations():
    w = synth.WORKLOADS["decode"]
    per_expert = 3 * w.d * w.f // 32 * 10                # 2 bits + fp16 scale per 32 weights
    assert per_expert == 1474560
    assert bench.decode_bytes(w, 10) == 10 * per_expert + w.E * w.d * 4 + w.E * 4 + w.T * w.d * 6
    assert bench.decode_bytes(w, 10) == 18954240
