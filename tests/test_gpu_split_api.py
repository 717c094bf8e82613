"""strata_moe_route followed by strata_moe_experts: bit for bit the result of
one strata_moe_forward on the tensor-core path, within tolerance of the
oracle, and refused when the handle's last routing call built no tile lists."""
import numpy as np
import pytest

from gpu_harness import HostLayer, S, torch_dev
from test_gpu_layer import check_full

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,flags", [(8, 2), (40, 0), (300, 0)])
def test_route_then_experts_equals_forward(T, flags):
    import torch
    lib = S()
    dev = torch_dev()
    h = HostLayer(256, 128, 16, 4, T, seed=11 + T, zipf=True)
    layer = lib.MoELayer(h.d, h.f, h.E, h.k, T, flags=flags, router_bias=torch.from_numpy(h.bias).to(dev))
    xd, Wd, _, blob = h.to_device(layer.desc)
    y1 = torch.zeros((T, h.d), dtype=torch.float32, device=dev)
    layer.forward(xd, Wd, blob, y1, T)
    y2 = torch.full((T, h.d), 7.0, dtype=torch.float32, device=dev)  # overwritten: no accumulate flag
    layer.route(xd, Wd, T)
    layer.experts(xd, blob, y2, T)
    layer.check_status()
    assert torch.equal(y1, y2), "route + experts differs from forward"
    idx, w, off, tl, sl = (a.cpu().numpy() for a in layer.routing(T))
    logits = torch.empty((T, h.E), dtype=torch.float32, device=dev)
    layer.router_logits(xd, Wd, logits, T)
    g = dict(y=y2.cpu().numpy(), idx=idx, w=w, off=off, tl=tl, sl=sl, logits=logits.cpu().numpy())
    layer.close()
    check_full(h, g, exact_routing=False)


def test_experts_needs_tile_lists():
    import torch
    lib = S()
    dev = torch_dev()
    h = HostLayer(256, 128, 16, 4, 4, seed=5)
    layer = lib.MoELayer(h.d, h.f, h.E, h.k, 8)
    xd, Wd, _, blob = h.to_device(layer.desc)
    y = torch.zeros((4, h.d), dtype=torch.float32, device=dev)
    with pytest.raises(lib.StrataError) as ei:  # nothing routed yet
        layer.experts(xd, blob, y, 4)
    assert ei.value.status == lib.STRATA_ERR_INVALID_ARG
    layer.forward(xd, Wd, blob, y, 4)  # one-launch decode layer: no tile lists
    with pytest.raises(lib.StrataError) as ei:
        layer.experts(xd, blob, y, 4)
    assert ei.value.status == lib.STRATA_ERR_INVALID_ARG
    layer.route(xd, Wd, 4)
    with pytest.raises(lib.StrataError) as ei:  # another token count
        layer.experts(xd, blob, y, 3)
    assert ei.value.status == lib.STRATA_ERR_INVALID_ARG
    layer.experts(xd, blob, y, 4)
    layer.check_status()
    layer.close()
