"""Pins of the CPU oracle: checks against values that the pages, the format
definition and the mathematics fix, independently of the oracle's own code.

Each ``check_*`` raises AssertionError on a mismatch. They are run on the
oracle as built (``test_oracle_pins.py``) and on deliberately broken copies of
it (``test_oracle_mutants.py``), which must each fail at least one check.
"""
from __future__ import annotations

import itertools
import math
import os
from fractions import Fraction

import mpmath
import numpy as np

import oracle as O
import synth

GOLD = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
mpmath.mp.dps = 40


# ---------------------------------------------------------------- helpers


def silu_mp(v: float) -> float:
    v = mpmath.mpf(v)
    return float(v / (1 + mpmath.exp(-v)))


def bf16_rne_exact(v: float) -> int:
    """IEEE round-to-nearest-even of a double to bfloat16, in exact rational
    arithmetic (independent of the oracle's C code)."""
    if v == 0.0:
        return 0x8000 if math.copysign(1.0, v) < 0 else 0
    m, e = math.frexp(v)
    e = max(e, -125)
    q = Fraction(2) ** (e - 8)
    n = round(Fraction(v) / q)  # Python rounds half to even
    r = float(n * q)
    return int(np.array([r], dtype=np.float32).view(np.uint32)[0] >> 16)


def load_tile_example(name="q2_tile_example.txt", size=1280):
    blob = np.zeros(size, dtype=np.uint8)
    expects = []
    with open(os.path.join(GOLD, name)) as fh:
        for line in fh:
            t = line.split("#", 1)[0].split()
            if not t:
                continue
            if t[0] == "fill":
                a, b = int(t[1]), int(t[2])
                pat = [int(h, 16) for h in t[3:]]
                for i in range(a, b):
                    blob[i] = pat[(i - a) % len(pat)]
            elif t[0] == "bytes":
                off = int(t[1])
                for j, h in enumerate(t[2:]):
                    blob[off + j] = int(h, 16)
            elif t[0] == "expect":
                expects.append((int(t[1]), int(t[2]), int(t[3]), float(t[4])))
    return blob, expects


def const_expert(d, f, gate_code, up_code, down_code, scale=2.0, bits=2):
    """Expert whose three matrices hold one code everywhere, one scale."""
    s = np.float16(scale)
    return dict(bits=bits,
        gate_codes=np.full((f, d), gate_code, np.uint8), gate_scales=np.full((f, d // 32), s, np.float16),
        up_codes=np.full((f, d), up_code, np.uint8), up_scales=np.full((f, d // 32), s, np.float16),
        down_codes=np.full((d, f), down_code, np.uint8), down_scales=np.full((d, f // 32), s, np.float16))


def identity_like_expert(d, f, down_mult):
    """Gate = up = selector of coordinates 32j (j < f/32); down maps h_{32j}
    back to coordinate 32j times down_mult. Blocks not used have scale 0;
    inside a used block only position 0 carries a code that matters (code 2,
    scale 2 -> weight 1), because the inputs vanish elsewhere in the block."""
    z = lambda r, k: (np.full((r, k), 2, np.uint8), np.zeros((r, k // 32), np.float16))
    gc, gs = z(f, d)
    uc, us = z(f, d)
    dc, ds = z(d, f)
    for j in range(f // 32):
        gs[32 * j, j] = 2.0
        us[32 * j, j] = 2.0
        ds[32 * j, j] = 2.0 * down_mult
    return dict(gate_codes=gc, gate_scales=gs, up_codes=uc, up_scales=us, down_codes=dc, down_scales=ds)


def tiny_layer(seed=0, T=8, d=256, f=128, E=16, k=4, bits=2):
    x = synth.gen_x_bf16(seed, T, d)
    W = synth.gen_router_w(seed, 0, E, d)
    experts = [synth.gen_expert(seed, 0, e, d, f, bits) for e in range(E)]
    return x, W, experts


def rel(a, b):
    return np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300)


# ---------------------------------------------------------------- scalars


def check_fp16_decode():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    f = bits.view(np.float16)
    fin = np.isfinite(f)
    got = O.fp16_to_double(bits[fin])
    assert np.array_equal(got, f[fin].astype(np.float64)), "fp16 decode differs from IEEE binary16"


def check_bf16_convert():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    f = (bits.astype(np.uint32) << 16).view(np.float32)
    fin = np.isfinite(f)
    got = O.bf16_to_double(bits[fin])
    assert np.array_equal(got, f[fin].astype(np.float64)), "bf16 decode differs"
    # hand-worked rounding: 1 + 2^-8 is the midpoint of 1 and 1 + 2^-7 -> even
    # (1.0); 1 + 3*2^-8 is the midpoint of 1+2^-7 and 1+2^-6 -> even (0x3F82);
    # just above a midpoint rounds up
    hand = [(1.0, 0x3F80), (1 + 2 ** -8, 0x3F80), (1 + 3 * 2 ** -8, 0x3F82),
            (1 + 2 ** -8 + 2 ** -30, 0x3F81), (-2.0, 0xC000), (0.0, 0x0000),
            (-0.0, 0x8000), (3.0, 0x4040), (1e-40, None)]
    for v, want in hand:
        want = bf16_rne_exact(v) if want is None else want
        got = int(O.double_to_bf16([v])[0])
        assert got == want, f"bf16({v}) = {got:#x}, expected {want:#x}"
    rng = np.random.default_rng(7)
    vals = np.concatenate([rng.standard_normal(2000) * 10.0 ** rng.integers(-8, 8, 2000),
                           (1 + (2 * rng.integers(0, 128, 200) + 1) * 2.0 ** -8)])
    got = O.double_to_bf16(vals)
    for v, g in zip(vals, got):
        assert int(g) == bf16_rne_exact(float(v)), f"bf16 rounding of {v!r}"


# ---------------------------------------------------------------- format


def check_tile_example():
    blob, expects = load_tile_example()
    codes, scales = O.unpack_q2_tiled(blob, 64, 64)
    W = O.dequant(codes, scales)
    for r, c, code, val in expects:
        assert codes[r, c] == code, f"code at ({r},{c}) = {codes[r, c]}, expected {code}"
        assert W[r, c] == val, f"weight at ({r},{c}) = {W[r, c]}, expected {val}"
    # rows 2..62 are all code 0 with scale 1 -> -1.5 everywhere
    assert np.all(W[2:63] == -1.5)


def check_dequant_rules():
    # code c -> (c - 1.5) * s, one scale per 32 consecutive columns
    codes = np.tile(np.arange(4, dtype=np.uint8), (2, 16))  # [2, 64]
    scales = np.array([[0.25, 2.0], [1.0, 0.5]], dtype=np.float16)
    W = O.dequant(codes, scales)
    base = np.array([-1.5, -0.5, 0.5, 1.5])
    assert np.array_equal(W[0, :32], np.tile(base * 0.25, 8))
    assert np.array_equal(W[0, 32:], np.tile(base * 2.0, 8))
    assert np.array_equal(W[1, :32], np.tile(base * 1.0, 8))
    assert np.array_equal(W[1, 32:], np.tile(base * 0.5, 8))


def check_q4_tile_example():
    blob, expects = load_tile_example("q4_tile_example.txt", 2304)
    codes, scales = O.unpack_q4_tiled(blob, 64, 64)
    W = O.dequant(codes, scales, bits=4)
    for r, c, code, val in expects:
        assert codes[r, c] == code, f"4-bit code at ({r},{c}) = {codes[r, c]}, expected {code}"
        assert W[r, c] == val, f"4-bit weight at ({r},{c}) = {W[r, c]}, expected {val}"
    # row 0's codes are column % 16 everywhere; rows 2..62 all code 0 (-7.5)
    assert np.array_equal(codes[0], np.arange(64) % 16)
    assert np.all(W[2:63] == -7.5)


def check_q4_dequant_rules():
    # code c -> (c - 7.5) * s, one scale per 32 consecutive columns; codes c
    # and 15 - c are exact negatives
    codes = np.tile(np.arange(16, dtype=np.uint8), (2, 4))  # [2, 64]
    scales = np.array([[0.25, 2.0], [1.0, 0.5]], dtype=np.float16)
    W = O.dequant(codes, scales, bits=4)
    base = np.arange(16) - 7.5
    assert np.array_equal(W[0, :32], np.tile(base * 0.25, 2))
    assert np.array_equal(W[0, 32:], np.tile(base * 2.0, 2))
    assert np.array_equal(W[1, :32], np.tile(base * 1.0, 2))
    assert np.array_equal(W[1, 32:], np.tile(base * 0.5, 2))
    assert np.array_equal(W[:, :16], -W[:, 15::-1])


def check_q4_swiglu_closed_form():
    # gate code 9 (+1.5 s), up code 6 (-1.5 s), down code 8 (+0.5 s), scale 2:
    # W_gate = +3, W_up = -3, W_down = +1; x = 1/32 everywhere -> g = 3, u = -3
    d = f = 32
    X = np.full((1, d), 1.0 / 32)
    o = O.expert_ffn(X, const_expert(d, f, 9, 6, 8, bits=4))
    ref = 1.0 * f * (silu_mp(3.0) * -3.0)
    assert np.all(np.abs(o - ref) <= 1e-13 * abs(ref)), f"{o[0, 0]} vs {ref}"
    # code 0 gate (-15), code 15 up (+15), code 1 down (-13), scale 2, d = 64
    d, f = 64, 32
    X = np.full((1, d), 1.0 / 64)
    o = O.expert_ffn(X, const_expert(d, f, 0, 15, 1, bits=4))
    ref = -13.0 * f * (silu_mp(-15.0) * 15.0)
    assert np.all(np.abs(o - ref) <= 1e-13 * abs(ref)), f"{o[0, 0]} vs {ref}"


def check_q4_dense_equals_sparse():
    x, W, experts = tiny_layer(bits=4)
    E, k = W.shape[0], 4
    y, idx, w = O.moe_layer(x, W, None, experts, k)
    X = synth.bf16_bits_to_f32(x).astype(np.float64)
    gate = np.zeros((x.shape[0], E))
    for t in range(x.shape[0]):
        gate[t, idx[t]] = w[t]
    dense = sum(gate[:, e:e + 1] * O.expert_ffn(X, experts[e]) for e in range(E))
    assert rel(y, dense) <= 1e-12
    # the same layer read as 2-bit codes would be a different layer
    y2, _, _ = O.moe_layer(x, W, None, [dict(e, bits=2) for e in experts], k)
    assert rel(y2, y) > 1e-3


# ---------------------------------------------------------------- router


def check_router_onehot_and_bias():
    rng = np.random.default_rng(1)
    T, d, E = 5, 64, 12
    x = synth.f32_to_bf16_bits(rng.standard_normal((T, d)).astype(np.float32))
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    perm = rng.permutation(d)[:E]
    W = np.zeros((E, d), np.float32)
    W[np.arange(E), perm] = 1.0
    l = O.router_logits(x, W)
    assert np.array_equal(l, xf[:, perm]), "one-hot router rows must copy x"
    bias = rng.standard_normal(E).astype(np.float32)
    l0 = O.router_logits(x, np.zeros((E, d), np.float32), bias)
    assert np.array_equal(l0, np.broadcast_to(bias.astype(np.float64), (T, E))), "bias must be added"
    # against exactly rounded sums of the (exact) products
    W = (rng.standard_normal((E, d)) * 0.02).astype(np.float32)
    l = O.router_logits(x, W, bias)
    for t in range(T):
        for e in range(E):
            terms = [float(W[e, i]) * float(xf[t, i]) for i in range(d)] + [float(bias[e])]
            ref = math.fsum(terms)
            tol = 1e-14 * sum(abs(v) for v in terms)
            assert abs(l[t, e] - ref) <= tol, f"logit ({t},{e})"


# ---------------------------------------------------------------- top-k


def _valid_set(lf, S):
    ins = set(S)
    for a in ins:
        for b in range(len(lf)):
            if b in ins:
                continue
            if not (lf[a] > lf[b] or (lf[a] == lf[b] and a < b)):
                return False
    return True


def check_topk_bruteforce():
    rng = np.random.default_rng(2)
    for E in range(1, 9):
        for k in range(1, E + 1):
            for trial in range(6):
                # few distinct values -> many exact ties
                l = rng.integers(-3, 3, (1, E)).astype(np.float64) * 0.5
                if trial % 2:
                    l = l + rng.standard_normal((1, E)) * 1e-3
                idx, _ = O.topk_softmax(l, k)
                lf = l[0].astype(np.float32)
                valid = [S for S in itertools.combinations(range(E), k) if _valid_set(lf, S)]
                assert len(valid) == 1
                assert sorted(idx[0].tolist()) == list(valid[0]), f"E={E} k={k}: wrong set"
                order = sorted(valid[0], key=lambda e: (-float(lf[e]), e))
                assert idx[0].tolist() == order, f"E={E} k={k}: wrong slot order"
    # all equal -> lowest indices
    idx, _ = O.topk_softmax(np.zeros((1, 9)), 4)
    assert idx[0].tolist() == [0, 1, 2, 3]


def check_softmax_weights():
    rng = np.random.default_rng(3)
    l = rng.standard_normal((6, 16)) * 2.0
    for k in (1, 2, 4, 10):
        idx, w = O.topk_softmax(l, k)
        for t in range(l.shape[0]):
            sel = [int(e) for e in idx[t]]
            den = mpmath.fsum(mpmath.exp(mpmath.mpf(float(l[t, e]))) for e in sel)
            for j, e in enumerate(sel):
                ref = float(mpmath.exp(mpmath.mpf(float(l[t, e]))) / den)
                assert abs(w[t, j] - ref) <= 1e-14, f"weight k={k}"
            assert abs(w[t].sum() - 1.0) <= 1e-14
        if k == 1:
            assert np.all(w == 1.0)


def check_expert_lists():
    rng = np.random.default_rng(4)
    T, E, k = 37, 11, 3
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    off, tl, sl = O.expert_lists(idx, E)
    pairs = sorted((int(idx[t, j]), t, j) for t in range(T) for j in range(k))
    assert tl.tolist() == [p[1] for p in pairs]
    assert sl.tolist() == [p[2] for p in pairs]
    counts = np.bincount(idx.ravel(), minlength=E)
    assert off.tolist() == [0] + np.cumsum(counts).tolist()


# ---------------------------------------------------------------- experts


def check_swiglu_closed_form():
    # all weights equal: gate code 2, up code 1, down code 0, scale 2 ->
    # W_gate = +1, W_up = -1, W_down = -3.  x = 1/32 everywhere (exact in bf16)
    d = f = 32
    X = np.full((1, d), 1.0 / 32)
    o = O.expert_ffn(X, const_expert(d, f, 2, 1, 0))
    ref = -3.0 * f * (silu_mp(1.0) * -1.0)  # 96 silu(1)
    assert np.all(np.abs(o - ref) <= 1e-13 * abs(ref)), f"{o[0, 0]} vs {ref}"
    # code 3 gate (+3), code 0 up (-3), code 3 down (+3) on a non-square expert
    d, f = 64, 32
    X = np.full((1, d), 1.0 / 64)
    o = O.expert_ffn(X, const_expert(d, f, 3, 0, 3))
    ref = 3.0 * f * (silu_mp(3.0) * -3.0)
    assert np.all(np.abs(o - ref) <= 1e-13 * abs(ref)), f"{o[0, 0]} vs {ref}"


def check_zero_scale_expert():
    d, f = 64, 32
    ex = const_expert(d, f, 3, 3, 3, scale=0.0)
    X = np.random.default_rng(5).standard_normal((3, d))
    assert np.all(O.expert_ffn(X, ex) == 0.0)


def check_identity_like_layer():
    d, f, E, k, T = 256, 128, 4, 2, 6
    mult = [1.0, 2.0, 0.5, 4.0]
    experts = [identity_like_expert(d, f, m) for m in mult]
    rng = np.random.default_rng(6)
    xf = np.zeros((T, d), np.float32)
    xf[:, ::32] = rng.standard_normal((T, d // 32)) * 2
    x = synth.f32_to_bf16_bits(xf)
    xv = synth.bf16_bits_to_f32(x).astype(np.float64)
    W = (rng.standard_normal((E, d)) * 0.3).astype(np.float32)
    y, idx, w = O.moe_layer(x, W, None, experts, k)
    for t in range(T):
        a = sum(w[t, j] * mult[idx[t, j]] for j in range(k))
        for i in range(d):
            ref = a * silu_mp(xv[t, i]) * xv[t, i] if (i % 32 == 0 and i < f) else 0.0
            assert abs(y[t, i] - ref) <= 1e-13 * max(1.0, abs(ref)), f"y[{t},{i}]"


def check_dense_equals_sparse():
    x, W, experts = tiny_layer()
    E, k = W.shape[0], 4
    y, idx, w = O.moe_layer(x, W, None, experts, k)
    X = synth.bf16_bits_to_f32(x).astype(np.float64)
    gate = np.zeros((x.shape[0], E))
    for t in range(x.shape[0]):
        gate[t, idx[t]] = w[t]
    dense = sum(gate[:, e:e + 1] * O.expert_ffn(X, experts[e]) for e in range(E))
    assert rel(y, dense) <= 1e-12


def check_router_independence_when_k_equals_E():
    x, W, experts = tiny_layer(E=6)
    same = [experts[0]] * 6
    X = synth.bf16_bits_to_f32(x).astype(np.float64)
    ref = O.expert_ffn(X, experts[0])
    y1, _, _ = O.moe_layer(x, W, None, same, 6)
    y2, _, _ = O.moe_layer(x, W[::-1].copy() * 3, None, same, 6)
    assert rel(y1, ref) <= 1e-12 and rel(y2, ref) <= 1e-12


def check_permutations():
    x, W, experts = tiny_layer()
    E, k = W.shape[0], 4
    y, idx, w = O.moe_layer(x, W, None, experts, k)
    p = np.random.default_rng(8).permutation(E)  # new expert i is old p[i]
    y2, idx2, _ = O.moe_layer(x, W[p].copy(), None, [experts[i] for i in p], k)
    assert rel(y2, y) <= 1e-12
    assert np.array_equal(p[idx2], idx)
    q = np.random.default_rng(9).permutation(x.shape[0])
    y3, _, _ = O.moe_layer(x[q].copy(), W, None, experts, k)
    assert rel(y3, y[q]) <= 1e-14


def check_down_scale_doubling():
    x, W, experts = tiny_layer()
    k = 4
    y, idx, w = O.moe_layer(x, W, None, experts, k)
    e0 = int(idx[0, 0])
    ex2 = dict(experts[e0])
    ex2["down_scales"] = (experts[e0]["down_scales"].astype(np.float32) * 2).astype(np.float16)
    experts2 = list(experts)
    experts2[e0] = ex2
    y2, idx2, w2 = O.moe_layer(x, W, None, experts2, k)
    X = synth.bf16_bits_to_f32(x).astype(np.float64)
    o = O.expert_ffn(X, experts[e0])
    for t in range(x.shape[0]):
        js = np.nonzero(idx[t] == e0)[0]
        extra = w[t, js[0]] * o[t] if js.size else 0.0
        assert np.max(np.abs(y2[t] - (y[t] + extra))) <= 1e-12 * np.max(np.abs(y[t]))


# ---------------------------------------------------------------- stack glue


def check_rmsnorm():
    # x = (3, 4): mean square 12.5 -> x / sqrt(12.5)
    got = O.rmsnorm_bf16(np.array([3.0, 4.0]), 0.0)[0]
    ref = [bf16_rne_exact(float(mpmath.mpf(v) / mpmath.sqrt(mpmath.mpf("12.5")))) for v in (3, 4)]
    assert got.tolist() == ref
    # a constant vector normalises to +-1 (eps small), exactly 1 after bf16
    got = O.rmsnorm_bf16(np.full(16, -7.25), 1e-6)[0]
    assert np.all(got == 0xBF80)
    # eps enters under the root: x = (1, 1), eps = 3 -> 1/2
    got = O.rmsnorm_bf16(np.array([1.0, 1.0]), 3.0)[0]
    assert np.all(got == 0x3F00)
    rng = np.random.default_rng(10)
    v = rng.standard_normal(64) * 3
    got = O.rmsnorm_bf16(v, 1e-6)[0]
    ms = mpmath.fsum(mpmath.mpf(float(a)) ** 2 for a in v) / 64
    inv = 1 / mpmath.sqrt(ms + mpmath.mpf(1e-6))
    ref = [bf16_rne_exact(float(mpmath.mpf(float(a)) * inv)) for a in v]
    mism = sum(int(a) != b for a, b in zip(got, ref))
    assert mism == 0, f"{mism} bf16 mismatches"


def check_residual_add():
    rng = np.random.default_rng(11)
    x = rng.standard_normal(100).astype(np.float32)
    y = rng.standard_normal(100)
    got = O.residual_add_f32(x, y)
    assert np.array_equal(got, (x.astype(np.float64) + y).astype(np.float32))


# ------------------------------------------- 4-bit rotated KV-cache codec


def hadamard(D: int) -> np.ndarray:
    """Sylvester Hadamard matrix from scipy (a library routine, not the oracle)."""
    import scipy.linalg
    return scipy.linalg.hadamard(D).astype(np.float64)


def fp16_rne_exact(v: float) -> int:
    """IEEE binary16 round-to-nearest-even of a double, in exact rationals."""
    if v == 0.0:
        return 0x8000 if math.copysign(1.0, v) < 0 else 0
    m, e = math.frexp(abs(v))
    qe = max(e - 11, -24)
    n = round(Fraction(abs(v)) / Fraction(2) ** qe)
    return int(np.array([float(n * Fraction(2) ** qe) * (1 if v > 0 else -1)], dtype=np.float64)
               .astype(np.float16).view(np.uint16)[0])


def bf16_bits(v) -> np.ndarray:
    return (np.asarray(v, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def kv_rows(seed: int, rows: int, D: int) -> np.ndarray:
    """bf16 cache rows from the seeded generator: N(0,1) with outlier channels."""
    return synth.gen_kv_rows(seed, rows, D)


def load_kv_example():
    cases = []
    with open(os.path.join(GOLD, "kv4_example.txt")) as fh:
        for line in fh:
            t = line.split("#", 1)[0].split()
            if t:
                cases.append((t[0], dict(kv.split("=", 1) for kv in t[1:])))
    return cases


def check_fp16_encode():
    rng = np.random.default_rng(11)
    vals = np.concatenate([
        rng.standard_normal(3000) * 10.0 ** rng.integers(-9, 5, 3000),
        1 + (2 * rng.integers(0, 1024, 300) + 1) * 2.0 ** -11,  # ties in [1, 2)
        (2 * rng.integers(0, 512, 300) + 1) * 2.0 ** -25,  # ties in the subnormal range
        [65504.0, 65519.0, 65520.0, 2.0 ** -14, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26, 0.0, -0.0]])
    vals = vals.astype(np.float32)
    got = O.float_to_fp16(vals)
    with np.errstate(over="ignore"):
        lib = vals.astype(np.float16).view(np.uint16)  # numpy's IEEE conversion
    assert np.array_equal(got, lib), "fp16 rounding differs from IEEE round-to-nearest-even"
    for v in (1 + 2.0 ** -11, 1 + 3 * 2.0 ** -11, 2.0 ** -25, 3 * 2.0 ** -25, 0.017857142857142856):
        assert int(O.float_to_fp16([v])[0]) == fp16_rne_exact(float(np.float32(v))), v


def check_kv4_fwht_is_hadamard():
    rng = np.random.default_rng(12)
    for D in (32, 64, 128, 256):
        H = hadamard(D)
        for i in (0, 1, D // 2 + 3, D - 1):
            for j in (0, 2, D // 3, D - 1):
                assert O.hadamard_sign(i, j) == H[i, j], (D, i, j)
        v = rng.integers(-100, 101, D).astype(np.float32)  # exact in fp32 throughout
        assert np.array_equal(O.fwht_f32(v).astype(np.float64), H @ v.astype(np.float64)), D
        v = (rng.standard_normal(D) * 10.0 ** rng.integers(-3, 3, D)).astype(np.float32)
        ex = H @ v.astype(np.float64)
        bound = 2 * math.log2(D) * 2.0 ** -24 * np.sum(np.abs(v.astype(np.float64)))
        assert np.max(np.abs(O.fwht_f32(v) - ex)) <= bound, D


def check_kv4_quant_example():
    for kind, a in load_kv_example():
        if kind != "quant":
            continue
        vals = [float(v) for v in a["y"].split(",")]
        y = np.zeros(32, dtype=np.float32)
        y[:len(vals)] = vals
        code, sb = O.kv4_quantize_block(y)
        want = [int(c) for c in a["codes"].split(",")]
        assert sb == int(a["scale"], 16), f"scale {sb:#x}"
        assert list(code[:len(want)]) == want and np.all(code[len(want):] == int(a["rest"])), code


def check_kv4_encode_examples():
    for kind, a in load_kv_example():
        if kind != "enc":
            continue
        D = int(a["D"])
        H = hadamard(D)
        what, arg = a["x"].split(":")
        xv = np.zeros(D) if what == "onehot" else H[:, int(arg)].copy()
        if what == "onehot":
            xv[int(arg)] = 1.0
        codes, scales = O.kv4_encode(bf16_bits(xv)[None, :])
        want = np.full(D // 2, int(a["byte"], 16), dtype=np.uint8)
        if "byte_at" in a:
            i, b = a["byte_at"].split(":")
            want[int(i)] = int(b, 16)
        assert np.array_equal(codes[0], want), codes
        assert [int(v) for v in scales[0]] == [int(v, 16) for v in a["scales"].split(",")], scales
        out, bits = O.kv4_decode(codes, scales)
        if "at" in a:
            i, v = a["at"].split(":")
            exp = np.zeros(D)
            exp[int(i)] = float(v)
            assert np.allclose(out[0], exp, rtol=1e-14, atol=1e-15), out[0][:4]
            bi, bv = a["bf16_at"].split(":")
            assert int(bits[0, int(bi)]) == int(bv, 16) and int(np.count_nonzero(bits[0])) == 1
        else:
            col = H[:, int(a["sign"].split(":")[1])]
            assert np.allclose(out[0], col * float(a["abs"]), rtol=1e-14, atol=0)
            bf = int(a["bf16_abs"], 16)
            assert np.array_equal(bits[0], np.where(col > 0, bf, bf | 0x8000).astype(np.uint16))


def _exact_rotation(x_bits):
    x = (x_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    D = x.shape[1]
    return x, x @ hadamard(D).T / math.sqrt(D)


def _nibbles(codes):
    D = codes.shape[1] * 2
    c = np.empty((codes.shape[0], D), dtype=np.int64)
    c[:, 0::2] = codes & 15
    c[:, 1::2] = codes >> 4
    return c


def check_kv4_codes_match_exact_rounding():
    for D, seed in ((64, 21), (128, 22), (256, 23)):
        xb = kv_rows(seed, 96, D)
        codes, scales = O.kv4_encode(xb)
        _, y = _exact_rotation(xb)
        s = scales.view(np.float16).astype(np.float64)
        yb = y.reshape(y.shape[0], D // 32, 32)
        t = np.abs(yb).max(axis=2) / 7.0
        want_s = np.array([[fp16_rne_exact(float(v)) for v in row] for row in t], dtype=np.uint16)
        # the fp32 rotation may move t across an fp16 midpoint only when t sits
        # within its error bound of one
        frac = t / 2.0 ** (np.floor(np.log2(t)) - 10)
        near_mid = np.abs(frac - np.floor(frac) - 0.5) < 1e-4
        assert np.all((scales == want_s) | near_mid), "block scales differ from fp16(absmax / 7)"
        q = np.clip(np.rint(yb / s[:, :, None]), -7, 7).reshape(y.shape)
        ratio = (yb / s[:, :, None]).reshape(y.shape)
        tie = np.abs(np.abs(ratio - np.floor(ratio)) - 0.5) < 1e-4
        ok = (_nibbles(codes) - 8 == q) | tie
        assert np.all(ok) and np.mean(tie) < 0.01, "codes differ from round(y / s)"


def check_kv4_roundtrip_bound():
    for D, seed in ((64, 31), (128, 32), (256, 33)):
        xb = kv_rows(seed, 64, D)
        codes, scales = O.kv4_encode(xb)
        x, y = _exact_rotation(xb)
        out, bits = O.kv4_decode(codes, scales)
        s = np.repeat(scales.view(np.float16).astype(np.float64), 32, axis=1)
        yq = (_nibbles(codes) - 8) * s
        # per element in the rotated domain: within half a step (plus the fp32
        # rotation's own error)
        assert np.all(np.abs(y - yq) <= s / 2 + 1e-5 * np.abs(y).max(axis=1, keepdims=True)), D
        # the decode is the orthonormal inverse: equal 2-norm of the error
        e_rot = np.linalg.norm(y - yq, axis=1)
        e_x = np.linalg.norm(x - out, axis=1)
        assert np.allclose(e_x, e_rot, rtol=1e-9, atol=1e-12), D
        dec = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        assert np.all(np.abs(dec - out) <= np.abs(out) * 2.0 ** -8 + 1e-38), D


def check_kv4_single_code_decode():
    for D in (64, 128, 256):
        H = hadamard(D)
        for i in (0, 7, D // 2 + 5, D - 1):
            c = np.full(D, 8, dtype=np.uint8)
            c[i] = 9 if i % 3 else 6  # q = +1 or -2
            codes = (c[0::2] | (c[1::2] << 4)).astype(np.uint8)[None, :]
            scales = np.full((1, D // 32), 0x3800, dtype=np.uint16)  # 0.5
            out, _ = O.kv4_decode(codes, scales)
            want = H[:, i] * (int(c[i]) - 8) * 0.5 / math.sqrt(D)
            assert np.allclose(out[0], want, rtol=1e-15, atol=0), (D, i)


def check_kv4_zero_and_saturation():
    for D in (64, 256):
        codes, scales = O.kv4_encode(np.zeros((1, D), dtype=np.uint16))
        assert np.all(codes == 0x88) and np.all(scales == 0)
        out, bits = O.kv4_decode(codes, scales)
        assert np.all(out == 0) and np.all(bits == 0)
    # a row too small for any half scale: x = 1e-8 e_0 gives y = 1.25e-9
    # everywhere, absmax / 7 underflows fp16 to zero -> every code 8
    x = np.zeros((1, 64))
    x[0, 0] = 1e-8
    codes, scales = O.kv4_encode(bf16_bits(x))
    assert np.all(scales == 0) and np.all(codes == 0x88), codes
    # constant row of 61952 (a bf16 value): y = 61952 * sqrt(64) e_0 = 495616,
    # absmax / 7 above the largest half -> s saturates at 65504 (0x7bff);
    # 495616 / 65504 = 7.57 rounds to 8 and is clamped to 7 (code 15)
    codes, scales = O.kv4_encode(bf16_bits(np.full((1, 64), 61952.0)))
    assert int(scales[0, 0]) == 0x7BFF and int(scales[0, 1]) == 0, scales
    want = np.full(32, 0x88, dtype=np.uint8)
    want[0] = 0x8F
    assert np.array_equal(codes[0], want), codes


ALL_CHECKS = [v for k, v in sorted(globals().items()) if k.startswith("check_")]
