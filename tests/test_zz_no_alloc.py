"""The allocation-free routing call against the layer-handle routing call.

strata_moe_route_noalloc keeps its scratch in a fixed device array instead of
a layer workspace. Through the C ABI, on the full-size decode layer shape
with the Zipf(1.1) router prior, two calls in a row (different tokens) must
give the routing that strata_moe_route + strata_moe_get_routing give:
indices, per-expert offsets, token lists and slots bit-exact, weights within
1e-6. Collected last so that it also runs after every other GPU test; it
must pass alone in a fresh process as well."""
import numpy as np
import pytest

import synth
from gpu_harness import S, torch_dev

pytestmark = pytest.mark.gpu


def _handle_routing(lib, w, x, W, bias, T):
    layer = lib.MoELayer(w.d, w.f, w.E, w.k, 16, router_bias=bias)
    layer.route(x, W, T)
    out = [a.cpu().numpy() for a in layer.routing(T)]
    layer.check_status()
    layer.close()
    return out


def _noalloc_routing(lib, w, x, W, bias, T):
    import torch
    dev = torch_dev()
    desc = lib.make_desc(w.d, w.f, w.E, w.k, 16, 0, bias)
    P = T * w.k
    idx = torch.full((T, w.k), -7, dtype=torch.int32, device=dev)
    wt = torch.full((T, w.k), -7.0, dtype=torch.float32, device=dev)
    off = torch.full((w.E + 1,), -7, dtype=torch.int32, device=dev)
    tl = torch.full((P,), -7, dtype=torch.int32, device=dev)
    sl = torch.full((P,), -7, dtype=torch.int32, device=dev)
    lib.strata_moe_route_noalloc(desc, x, W, T, idx, wt, off, tl, sl)
    torch.cuda.synchronize()
    return [a.cpu().numpy() for a in (idx, wt, off, tl, sl)]


@pytest.mark.parametrize("T", [1, 4, 16])
def test_noalloc_routing_matches_layer_routing(T):
    import synth.device as sd
    lib = S()
    w = synth.WORKLOADS["verify16"]
    W, bias = sd.layer_inputs(w, 0)
    for call in range(2):  # two calls in a row, different tokens
        x = sd.x_bf16(w.seed, T, w.d, stream=50 + call)
        ref = _handle_routing(lib, w, x, W, bias, T)
        got = _noalloc_routing(lib, w, x, W, bias, T)
        names = ("topk_idx", "topk_w", "expert_offsets", "token_list", "pair_slot")
        for name, a, b in zip(names, got, ref):
            if name == "topk_w":
                assert np.allclose(a, b, rtol=1e-6, atol=0), f"call {call}: {name}"
            else:
                assert np.array_equal(a, b), f"call {call}: {name}"
        assert np.allclose(got[1].sum(axis=1), 1.0, atol=1e-5)


def _compare(got, ref, T, k, what):
    names = ("topk_idx", "topk_w", "expert_offsets", "token_list", "pair_slot")
    for name, a, b in zip(names, got, ref):
        if name == "topk_w":
            assert np.allclose(a, b, rtol=1e-6, atol=0), f"{what}: {name}"
        else:
            assert np.array_equal(a, b), f"{what}: {name}"
    assert got[2][-1] == T * k, f"{what}: offsets[E] is not T*k"
    assert np.allclose(got[1].sum(axis=1), 1.0, atol=1e-5)


def test_noalloc_routing_at_the_scratch_limits():
    """The largest shape the fixed scratch is sized for: 16 tokens, 1,024
    experts, top-32 (the last tile slots and the end of the array; E > 512
    takes the general warp top-k)."""
    import torch
    import synth.device as sd
    lib = S()
    w = synth.Workload("limits", 256, 128, 1024, 32, 16, 1, False, 11)
    W = torch.from_numpy(synth.gen_router_w(w.seed, 0, w.E, w.d)).to(torch_dev())
    for call in range(2):
        x = sd.x_bf16(w.seed, w.T, w.d, stream=70 + call)
        ref = _handle_routing(lib, w, x, W, None, w.T)
        got = _noalloc_routing(lib, w, x, W, None, w.T)
        _compare(got, ref, w.T, w.k, f"call {call}")


def test_noalloc_routing_ignores_max_tokens_and_flags():
    import torch
    import synth.device as sd
    lib = S()
    w = synth.WORKLOADS["tiny"]
    W = torch.from_numpy(synth.gen_router_w(w.seed, 0, w.E, w.d)).to(torch_dev())
    x = sd.x_bf16(w.seed, w.T, w.d, stream=3)
    ref = _handle_routing(lib, w, x, W, None, w.T)
    desc = lib.make_desc(w.d, w.f, w.E, w.k, 0, 0x80)   # max_tokens 0 and an unknown flag: not used here
    P = w.T * w.k
    dev = torch_dev()
    out = [torch.full((w.T, w.k), -7, dtype=torch.int32, device=dev),
           torch.full((w.T, w.k), -7.0, dtype=torch.float32, device=dev),
           torch.full((w.E + 1,), -7, dtype=torch.int32, device=dev),
           torch.full((P,), -7, dtype=torch.int32, device=dev),
           torch.full((P,), -7, dtype=torch.int32, device=dev)]
    lib.strata_moe_route_noalloc(desc, x, W, w.T, *out)
    torch.cuda.synchronize()
    _compare([a.cpu().numpy() for a in out], ref, w.T, w.k, "max_tokens 0")


def test_noalloc_routing_rejects_too_many_tokens():
    import torch
    lib = S()
    dev = torch_dev()
    d, f, E, k, T = 256, 128, 16, 4, 17
    desc = lib.make_desc(d, f, E, k, 64)
    x = torch.zeros((T, d), dtype=torch.bfloat16, device=dev)
    W = torch.zeros((E, d), dtype=torch.float32, device=dev)
    bufs = [torch.zeros(T * k, dtype=torch.int32, device=dev) for _ in range(2)]
    off = torch.zeros(E + 1, dtype=torch.int32, device=dev)
    wt = torch.zeros(T * k, dtype=torch.float32, device=dev)
    with pytest.raises(lib.StrataError) as ei:
        lib.strata_moe_route_noalloc(desc, x, W, T, bufs[0], wt, off, bufs[1], bufs[1])
    assert ei.value.status == lib.STRATA_ERR_TOO_MANY_TOKENS
