"""The device input generator and the library's device packer reproduce the
host generator and the host packer bit for bit (so full-size layers built on
the GPU are the ones the oracle regenerates on the host)."""
import numpy as np
import pytest

import oracle
import synth
from gpu_harness import S, torch_dev

pytestmark = pytest.mark.gpu


def test_device_generator_matches_host():
    import synth.device as sd
    x = sd.x_bf16(3, 5, 256, tok0=7).cpu().view(dtype=__import__("torch").int16).numpy().view(np.uint16)
    assert np.array_equal(x, synth.gen_x_bf16(3, 5, 256, tok0=7))
    W = sd.router_w(2, 4, 64, 128).cpu().numpy()
    assert np.array_equal(W, synth.gen_router_w(2, 4, 64, 128))
    for bits in (2, 4):
        for mat, rows, K in ((synth.GATE, 768, 2048), (synth.DOWN, 256, 128)):
            c, s = sd.expert_codes_scales(1, 3, [0, 17, 511], mat, rows, K, bits)
            c, s = c.cpu().numpy(), s.cpu().numpy().view(np.uint16)
            for i, e in enumerate([0, 17, 511]):
                assert np.array_equal(c[i], synth.gen_codes(1, 3, e, mat, rows, K, bits))
                assert np.array_equal(s[i], synth.gen_scales(1, 3, e, mat, rows, K, bits).view(np.uint16))


@pytest.mark.parametrize("bits", [2, 4])
def test_device_packer_matches_host_packer(bits):
    import torch
    lib = S()
    d, f = 512, 256
    desc = lib.make_desc(d, f, 4, 2, 8, bits=bits)
    ex = synth.gen_expert(9, 0, 1, d, f, bits)
    eb = lib.strata_moe_expert_bytes(desc)
    host = np.zeros(eb, np.uint8)
    lib.strata_moe_pack_expert(desc, ex["gate_codes"], ex["gate_scales"], ex["up_codes"], ex["up_scales"],
                               ex["down_codes"], ex["down_scales"], host)
    dev = torch_dev()
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a.view(np.int16) if a.dtype == np.float16 else a)).to(dev)
    out = torch.zeros(eb, dtype=torch.uint8, device=dev)
    lib.strata_moe_pack_expert_device(desc, t(ex["gate_codes"]), t(ex["gate_scales"]), t(ex["up_codes"]),
                                      t(ex["up_scales"]), t(ex["down_codes"]), t(ex["down_scales"]), out)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy(), host)
    got = oracle.unpack_expert(host, d, f, bits)
    assert np.array_equal(got["down_codes"], ex["down_codes"])


def test_selftest_wait_times_out_and_context_survives():
    """A bounded device wait that nothing releases gives up and reports a
    timeout; the context keeps working afterwards."""
    import torch
    lib = S()
    rc = lib.strata_selftest_wait_timeout(50_000_000)  # 50 ms
    assert rc == lib.STRATA_ERR_TIMEOUT
    a = torch.ones(1024, device=torch_dev())
    assert float(a.sum()) == 1024.0
