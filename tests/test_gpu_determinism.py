"""Routing is deterministic: the selected experts, their weights, the
per-expert offsets, token lists and pair slots are bit-identical over 100
calls of the same layer on the same input, on the one-launch decode path
(1 and 16 tokens) and on the prefill path (300 tokens). The outputs y may
differ in the last bits (fp32 atomics in the decode kernel), the routing may
not."""
import numpy as np
import pytest

import synth
from gpu_harness import S, device_blob, torch_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T", [1, 16, 300])
def test_routing_identical_over_100_calls(T):
    import torch
    import synth.device as sd
    lib = S()
    w = synth.WORKLOADS["verify4"]
    W, bias = sd.layer_inputs(w, 0)
    layer = lib.MoELayer(w.d, w.f, w.E, w.k, T, router_bias=bias)
    blob = device_blob(w, 0, layer.desc)
    x = sd.x_bf16(w.seed, T, w.d, stream=9)
    y = torch.zeros((T, w.d), dtype=torch.float32, device=torch_dev())
    first = None
    for it in range(100):
        layer.forward(x, W, blob, y, T)
        got = [a.cpu().numpy() for a in layer.routing(T)]
        if first is None:
            first = got
            continue
        for name, a, b in zip(("topk_idx", "topk_w", "offsets", "token_list", "pair_slot"), got, first):
            assert np.array_equal(a, b), f"call {it}: {name} differs"
    layer.check_status()
    layer.close()
