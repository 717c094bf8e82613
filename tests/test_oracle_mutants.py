"""Plausible mistakes planted in a copy of the CPU oracle must each fail at
least one pin. This shows the pins constrain every step of the oracle (a
dropped term, a wrong sign or index, a transposed operand, a wrong tie rule).
The mutants are compiled from a temporary copy; the oracle itself is never
modified. Runs without a GPU."""
import os

import pytest

import oracle
import pins_lib

MUTANTS = [
    ("code_offset", "W[(size_t)r * K + k] = (c - offset) * s;", "W[(size_t)r * K + k] = (c - offset + 0.5) * s;"),
    ("q4_offset", "double offset = ((double)(1 << bits) - 1.0) / 2.0;",
     "double offset = bits == 4 ? 7.0 : ((double)(1 << bits) - 1.0) / 2.0;"),
    ("q4_unpack_word", "const uint8_t *wp = tile + 32 * i + 4 * (2 * t + j / 2);",
     "const uint8_t *wp = tile + 32 * i + 4 * (2 * t + j % 2);"),
    ("q4_unpack_bit", "int bit = 16 * e + 8 * (j % 2) + 4 * sh;", "int bit = 16 * e + 4 * (j % 2) + 8 * sh;"),
    ("q4_unpack_scales", "const uint8_t *sp = tile + 2048 + 4 * i + 2 * b;", "const uint8_t *sp = tile + 2048 + 4 * i + 2 * (1 - b);"),
    ("q4_code_mask", "codes[(size_t)r * K + 64 * s + c] = (uint8_t)((w >> bit) & 15u);",
     "codes[(size_t)r * K + 64 * s + c] = (uint8_t)((w >> bit) & 7u);"),
    ("expert_bits_ignored", "oracle_dequant(f, d, bits, uc, us, Wu);", "oracle_dequant(f, d, 2, uc, us, Wu);"),
    ("scale_block", "scales[(size_t)r * nb + k / 32]", "scales[(size_t)r * nb + k / 64]"),
    ("silu_sign", "g / (1.0 + exp(-g))", "g / (1.0 + exp(g))"),
    ("gate_up_swapped", "h[r] = oracle_silu(g) * u;", "h[r] = oracle_silu(u) * g;"),
    ("down_transposed", "o += Wd[(size_t)i * f + r] * h[r];", "o += Wd[(size_t)r * d + i] * h[r];"),
    ("no_renormalise", "w[(size_t)t * k + j] = p[r[j].idx] / ps;", "w[(size_t)t * k + j] = p[r[j].idx];"),
    ("tie_to_higher", "return (x->idx > y->idx) - (x->idx < y->idx);", "return (x->idx < y->idx) - (x->idx > y->idx);"),
    ("ascending_order", "if (x->key > y->key)\n        return -1;", "if (x->key > y->key)\n        return 1;"),
    ("bias_dropped", "acc += (double)bias[e];", "acc += 0.0;"),
    ("softmax_no_shift", "p[e] = exp(l[e] - mx);", "p[e] = exp(l[e] - mx) + 1e-3;"),
    ("lists_slot_major", "for (int t = 0; t < T; ++t)\n            for (int j = 0; j < k; ++j)\n                if (idx[(size_t)t * k + j] == e) {",
     "for (int j = 0; j < k; ++j)\n            for (int t = 0; t < T; ++t)\n                if (idx[(size_t)t * k + j] == e) {"),
    ("unpack_bit", "int bit = 16 * h + 8 * sh + 6 - 2 * j;", "int bit = 16 * h + 8 * sh + 2 * j;"),
    ("unpack_word", "const uint8_t *wp = tile + 16 * i + 4 * t;", "const uint8_t *wp = tile + 16 * i + 4 * j;"),
    ("unpack_scale_order", "const uint8_t *sp = tile + 1024 + 4 * i + 2 * b;", "const uint8_t *sp = tile + 1024 + 4 * i + 2 * (1 - b);"),
    ("rms_no_mean", "double inv = 1.0 / sqrt(ss / d + eps);", "double inv = 1.0 / sqrt(ss + eps);"),
    ("rms_eps_outside", "double inv = 1.0 / sqrt(ss / d + eps);", "double inv = 1.0 / sqrt(ss / d) + eps;"),
    ("bf16_truncate", "double r = nearbyint(v / q) * q;", "double r = trunc(v / q) * q;"),
    ("fp16_subnormal", "v = ldexp((double)mant, -24);", "v = ldexp((double)mant, -25);"),
    ("residual_in_double", "x[i] = (float)((double)x[i] + y[i]);", "x[i] = (float)((double)x[i] + (float)y[i] * 1.0000001);"),
    ("kv_fwht_sign", "v[i + h] = a - b;", "v[i + h] = b - a;"),
    ("kv_fwht_last_stage", "for (int h = 1; h < D; h *= 2)", "for (int h = 1; h < D / 2; h *= 2)"),
    ("kv_norm_dropped", "y[i] = y[i] * r;", "y[i] = y[i];"),
    ("kv_scale_over_8", "float t = amax / 7.0f;", "float t = amax / 8.0f;"),
    ("kv_round_half_away", "double r = rint((double)y[i] * (double)inv);", "double r = round((double)y[i] * (double)inv);"),
    ("kv_product_rounded_first", "double r = rint((double)y[i] * (double)inv);", "double r = rintf(y[i] * inv);"),
    ("kv_clamp_8", "int q = r > 7.0 ? 7 :", "int q = r > 7.0 ? 8 :"),
    ("kv_zero_scale_inverse", "float inv = s > 0.0f ? 1.0f / s : 0.0f;", "float inv = 1.0f / s;"),
    ("kv_no_saturation", "if (t > 65504.0f)\n        t = 65504.0f;", "if (t > 65504.0f)\n        t = t;"),
    ("kv_code_offset", "code[i] = (uint8_t)(q + 8);", "code[i] = (uint8_t)(q + 7);"),
    ("kv_nibble_order", "(uint8_t)(q[2 * j] | (q[2 * j + 1] << 4));", "(uint8_t)(q[2 * j + 1] | (q[2 * j] << 4));"),
    ("kv_dec_sign", "acc += oracle_hadamard_sign(j, i) * y[i];", "acc += oracle_hadamard_sign(j, i ^ 1) * y[i];"),
    ("kv_dec_nibble", ">> (4 * (i % 2))) & 15;", ">> (4 * (1 - i % 2))) & 15;"),
    ("kv_dec_scale_block", "oracle_fp16_to_double(scales[(size_t)row * (D / 32) + i / 32]);",
     "oracle_fp16_to_double(scales[(size_t)row * (D / 32) + i / 64]);"),
    ("kv_dec_offset", "y[i] = (c - 8) *", "y[i] = (c - 7.5) *"),
    ("kv_dec_norm", "out[(size_t)row * D + j] = acc * inv;", "out[(size_t)row * D + j] = acc / D;"),
    ("hadamard_parity", "p ^= (int)(m & 1u);", "p ^= (int)((m >> 1) & 1u);"),
    ("fp16_subnormal_quantum", "qe = -24; /* subnormal range", "qe = -25; /* subnormal range"),
    ("fp16_no_carry", "n /= 2.0;\n        qe += 1;", "n -= 1.0;"),
    ("combine_weight_dropped", "y[(size_t)t * d + i] += w[(size_t)t * k + j] * o[i];", "y[(size_t)t * d + i] += o[i];"),
]


@pytest.mark.parametrize("name,find,repl", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_fails_a_pin(tmp_path, name, find, repl):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "strata_oracle.c")).read()
    assert src.count(find) == 1, f"mutation site for {name} not found exactly once"
    mut = tmp_path / f"oracle_{name}.c"
    mut.write_text(src.replace(find, repl))
    so = oracle.build(str(mut), str(tmp_path / f"liboracle_{name}.so"))
    saved = oracle._lib
    oracle._lib = oracle.load(so)
    failed = []
    try:
        for check in pins_lib.ALL_CHECKS:
            try:
                check()
            except AssertionError:
                failed.append(check.__name__)
    finally:
        oracle._lib = saved
    assert failed, f"mutant {name} passed every pin"
