"""The 4-bit Hadamard-rotated KV-cache codec on the GPU against the CPU oracle.

Codes and scales must match bit for bit: the encoder's fp32 steps (butterfly
stages of stride 1, 2, ..., D/2, the product by fp32(1/sqrt(D)), the block
rule) are fixed, so the integers they decide are too. Decoded rows are a
float result: each must lie within the bound of fp32 butterflies plus one
bf16 rounding of the oracle's exact fp64 inverse. Nothing may be written
outside the rows asked for."""
import math

import numpy as np
import pytest

import oracle
import synth
from gpu_harness import S, torch_dev

pytestmark = pytest.mark.gpu

GUARD = 0x5A


def _dev(a, dtype=None):
    import torch
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).to(torch_dev())


def _u16(t):
    return t.cpu().numpy().view(np.uint16)


def _nibbles(codes):
    c = np.empty((codes.shape[0], codes.shape[1] * 2), dtype=np.int64)
    c[:, 0::2] = codes & 15
    c[:, 1::2] = codes >> 4
    return c


def decode_bound(codes, scales, exact):
    """|GPU - exact| per value: the fp32 transform rounds each of its log2(D)
    stages (plus the product by the normalisation and that constant's own
    rounding) at 2^-24 of a partial sum no larger than the row's L1 norm
    divided by sqrt(D); the bf16 rounding adds 2^-9 of the value. Doubled."""
    D = codes.shape[1] * 2
    s = np.repeat(scales.view(np.float16).astype(np.float64), 32, axis=1)
    l1 = np.sum(np.abs((_nibbles(codes) - 8) * s), axis=1, keepdims=True) / math.sqrt(D)
    return 2.0 ** -8 * np.abs(exact) + (math.log2(D) + 2) * 2.0 ** -23 * l1


def gpu_encode(x_bits, D, pad_rows=0):
    """Encode on the GPU into guard-filled buffers; returns codes, scales (host)
    and whether the guard bytes after the last row survived."""
    import torch
    lib = S()
    n = x_bits.shape[0]
    xd = _dev(x_bits)
    cd = torch.full((n * D // 2 + 64,), GUARD, dtype=torch.uint8, device=torch_dev())
    sd = torch.full((n * D // 32 + 32,), 0x5A5A, dtype=torch.int16, device=torch_dev())
    lib.strata_kv4_encode(xd, n, D, cd, sd)
    torch.cuda.synchronize()
    c = cd.cpu().numpy()
    s = _u16(sd)
    intact = bool(np.all(c[n * D // 2:] == GUARD) and np.all(s[n * D // 32:] == 0x5A5A))
    return c[:n * D // 2].reshape(n, D // 2), s[:n * D // 32].reshape(n, D // 32), intact


def gpu_decode(codes, scales, D):
    import torch
    lib = S()
    n = codes.shape[0]
    out = torch.full((n * D + 64,), 0x5A5A, dtype=torch.int16, device=torch_dev())
    lib.strata_kv4_decode(_dev(codes), _dev(scales), n, D, out)
    torch.cuda.synchronize()
    o = _u16(out)
    return o[:n * D].reshape(n, D), bool(np.all(o[n * D:] == 0x5A5A))


def check_rows(x_bits, D):
    codes_o, scales_o = oracle.kv4_encode(x_bits)
    codes_g, scales_g, intact = gpu_encode(x_bits, D)
    assert intact, "encoder wrote past the last row"
    bad = np.nonzero(np.any(codes_g != codes_o, axis=1) | np.any(scales_g != scales_o, axis=1))[0]
    assert bad.size == 0, f"codes/scales differ from the oracle in rows {bad[:8]}"
    exact, _ = oracle.kv4_decode(codes_o, scales_o)
    out, intact = gpu_decode(codes_o, scales_o, D)
    assert intact, "decoder wrote past the last row"
    got = synth.bf16_bits_to_f32(out).astype(np.float64)
    err = np.abs(got - exact) - decode_bound(codes_o, scales_o, exact)
    assert np.all(err <= 0), f"decode off the oracle by {np.max(err):.3g} beyond its bound"


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("rows", [1, 5, 37, 1031])
def test_kv4_parity(D, rows):
    check_rows(synth.gen_kv_rows(40 + D + rows, rows, D), D)


@pytest.mark.parametrize("D", [64, 128, 256])
def test_kv4_special_rows(D):
    """Zero rows, rows too small for any half scale, saturating rows, one-hot
    rows, Hadamard columns and exact ties, in one batch."""
    import scipy.linalg
    H = scipy.linalg.hadamard(D).astype(np.float32)
    rows = [np.zeros(D, np.float32), np.full(D, 1e-8, np.float32), np.full(D, 61952.0, np.float32),
            np.full(D, -61952.0, np.float32), H[:, 3], -H[:, D - 1], np.eye(D, dtype=np.float32)[0],
            np.eye(D, dtype=np.float32)[D // 2 + 1] * 3.0]
    rng = np.random.default_rng(D)
    for _ in range(8):  # a few Hadamard columns with small integer weights: rotated values on a coarse grid
        rows.append(H[:, rng.integers(0, D, 3)] @ rng.integers(-7, 8, 3).astype(np.float32))
    x = synth.f32_to_bf16_bits(np.stack(rows).astype(np.float32))
    check_rows(x, D)


def test_kv4_append_at_row_offset():
    """Appending to a cache: pointers advanced by the first new row; earlier
    rows stay as they were."""
    import torch
    lib = S()
    D, n0, n1 = 128, 7, 45
    x = synth.gen_kv_rows(3, n0 + n1, D)
    codes_o, scales_o = oracle.kv4_encode(x)
    cd = torch.zeros((n0 + n1, D // 2), dtype=torch.uint8, device=torch_dev())
    sd = torch.zeros((n0 + n1, D // 32), dtype=torch.int16, device=torch_dev())
    xd = _dev(x)
    lib.strata_kv4_encode(xd[:n0], n0, D, cd[:n0], sd[:n0])
    lib.strata_kv4_encode(xd[n0:], n1, D, cd[n0:], sd[n0:])
    torch.cuda.synchronize()
    assert np.array_equal(cd.cpu().numpy(), codes_o)
    assert np.array_equal(_u16(sd), scales_o)


def test_kv4_zero_rows_is_noop():
    import torch
    lib = S()
    cd = torch.full((64,), GUARD, dtype=torch.uint8, device=torch_dev())
    sd = torch.full((4,), 0x5A5A, dtype=torch.int16, device=torch_dev())
    x = torch.zeros((1, 128), dtype=torch.int16, device=torch_dev())
    lib.strata_kv4_encode(x, 0, 128, cd, sd)
    out = torch.full((128,), 0x5A5A, dtype=torch.int16, device=torch_dev())
    lib.strata_kv4_decode(cd, sd, 0, 128, out)
    torch.cuda.synchronize()
    assert bool((cd == GUARD).all()) and bool((sd == 0x5A5A).all()) and bool((out == 0x5A5A).all())


def test_kv4_full_size_sampled():
    """The 128K-token workload in the benchmark's launch configuration:
    generated on the device, encoded and decoded whole; 1536 sampled rows
    (the first, the last and random ones) checked against the oracle."""
    import torch
    import synth.device as sdev
    lib = S()
    w = synth.KV_WORKLOADS["kv4_128k"]
    n, D = w.rows, w.D
    x = sdev.kv_rows(w.seed, n, D)
    cd = torch.empty((n, D // 2), dtype=torch.uint8, device=torch_dev())
    sd = torch.empty((n, D // 32), dtype=torch.int16, device=torch_dev())
    out = torch.empty((n, D), dtype=torch.bfloat16, device=torch_dev())
    lib.strata_kv4_encode(x, n, D, cd, sd)
    lib.strata_kv4_decode(cd, sd, n, D, out)
    torch.cuda.synchronize()
    rng = np.random.default_rng(128)
    pick = np.unique(np.concatenate([[0, 1, n - 2, n - 1], rng.integers(0, n, 1532)]))
    host = np.concatenate([synth.gen_kv_rows(w.seed, 1, D, row0=int(r)) for r in pick])
    idx = torch.from_numpy(pick).to(torch_dev())
    assert np.array_equal(x[idx].view(torch.int16).cpu().numpy().view(np.uint16), host), "device generator differs"
    codes_o, scales_o = oracle.kv4_encode(host)
    assert np.array_equal(cd[idx].cpu().numpy(), codes_o), "codes differ from the oracle"
    assert np.array_equal(_u16(sd[idx]), scales_o), "scales differ from the oracle"
    exact, _ = oracle.kv4_decode(codes_o, scales_o)
    got = out[idx].float().cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - exact) <= decode_bound(codes_o, scales_o, exact)), "decode outside its bound"
