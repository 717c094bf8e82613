"""CPU oracle of the routed-expert MoE layer (test infrastructure only).

Thin ctypes wrapper around ``strata_oracle.c`` (plain C, IEEE double, single
thread). Only the tests, the smoke check and the benchmark's CPU-baseline leg
may import this package; the library never does.

Parity status of each function and the pins that fix it are listed in the
header of ``strata_oracle.c`` and in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "strata_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
CFLAGS = ["-O2", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math", "-std=c99"]


def build(src: str = _SRC, out: str = _LIB, extra: tuple = ()) -> str:
    """Compile the oracle into a shared object (gcc, no FMA contraction)."""
    cmd = ["gcc", *CFLAGS, *extra, "-o", out, src, "-lm"]
    subprocess.run(cmd, check=True)
    return out


_lib = None


def load(path: str | None = None):
    """Load (building if needed) the oracle shared object."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    if _lib is None:
        if not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
            build()
        _lib = _bind(ctypes.CDLL(_LIB))
    return _lib


P = ctypes.c_void_p
I = ctypes.c_int


def _bind(lib):
    lib.oracle_bf16_to_double.restype = ctypes.c_double
    lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
    lib.oracle_fp16_to_double.restype = ctypes.c_double
    lib.oracle_fp16_to_double.argtypes = [ctypes.c_uint16]
    lib.oracle_double_to_bf16.restype = ctypes.c_uint16
    lib.oracle_double_to_bf16.argtypes = [ctypes.c_double]
    lib.oracle_dequant.argtypes = [I, I, I, P, P, P]
    lib.oracle_unpack_q2_tiled.argtypes = [I, I, P, ctypes.c_long, ctypes.c_long, P, P]
    lib.oracle_unpack_q4_tiled.argtypes = [I, I, P, ctypes.c_long, ctypes.c_long, P, P]
    lib.oracle_router_logits.argtypes = [I, I, I, P, P, P, P]
    lib.oracle_topk_softmax.argtypes = [I, I, I, P, P, P]
    lib.oracle_expert_lists.argtypes = [I, I, I, P, P, P, P]
    lib.oracle_expert_ffn.argtypes = [I, I, I, I, P, P, P, P, P, P, P, P]
    lib.oracle_moe_layer.argtypes = [I, I, I, I, I, I, P, P, P, P, P, P, P, P, P, P, P, P]
    lib.oracle_rmsnorm_bf16.argtypes = [I, P, ctypes.c_double, P]
    lib.oracle_residual_add_f32.argtypes = [I, P, P]
    lib.oracle_float_to_fp16.restype = ctypes.c_uint16
    lib.oracle_float_to_fp16.argtypes = [ctypes.c_float]
    lib.oracle_hadamard_sign.restype = I
    lib.oracle_hadamard_sign.argtypes = [I, I]
    L = ctypes.c_long
    lib.oracle_fwht_f32.argtypes = [I, P]
    lib.oracle_kv4_quantize_block.argtypes = [P, P, P]
    lib.oracle_kv4_encode.argtypes = [L, I, P, P, P]
    lib.oracle_kv4_decode.argtypes = [L, I, P, P, P]
    lib.oracle_round_bf16_array.argtypes = [L, P, P]
    for fn in ("oracle_fwht_f32", "oracle_kv4_quantize_block", "oracle_kv4_encode", "oracle_kv4_decode",
               "oracle_round_bf16_array"):
        getattr(lib, fn).restype = None
    for fn in ("oracle_dequant", "oracle_unpack_q2_tiled", "oracle_unpack_q4_tiled", "oracle_router_logits",
               "oracle_topk_softmax", "oracle_expert_lists", "oracle_expert_ffn",
               "oracle_moe_layer", "oracle_rmsnorm_bf16", "oracle_residual_add_f32"):
        getattr(lib, fn).restype = None
    return lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


# ----------------------------------------------------------------------------
# numpy-level API


def bf16_to_double(bits):
    lib = load()
    return np.array([lib.oracle_bf16_to_double(int(b)) for b in np.ravel(bits)]).reshape(np.shape(bits))


def fp16_to_double(bits):
    lib = load()
    return np.array([lib.oracle_fp16_to_double(int(b)) for b in np.ravel(bits)]).reshape(np.shape(bits))


def double_to_bf16(v):
    lib = load()
    return np.array([lib.oracle_double_to_bf16(float(x)) for x in np.ravel(v)], dtype=np.uint16).reshape(np.shape(v))


def dequant(codes, scales_fp16, bits: int = 2):
    """(c - (2^bits - 1)/2) * scale of the 32-column block, in double."""
    codes = _c(codes, np.uint8)
    sc = _c(np.asarray(scales_fp16).view(np.uint16) if np.asarray(scales_fp16).dtype == np.float16 else scales_fp16, np.uint16)
    rows, K = codes.shape
    W = np.empty((rows, K), dtype=np.float64)
    load().oracle_dequant(rows, K, bits, _p(codes), _p(sc), _p(W))
    return W


def unpack_q2_tiled(blob, rows: int, K: int, panel_stride: int = None, slice_stride: int = 1280):
    """Codes and scales of one matrix whose 64x64 tile (p, s) starts at
    ``blob + p * panel_stride + s * slice_stride`` (a lone matrix by default)."""
    blob = _c(blob, np.uint8)
    if panel_stride is None:
        panel_stride = (K // 64) * slice_stride
    last = (rows // 64 - 1) * panel_stride + (K // 64 - 1) * slice_stride
    assert blob.size >= last + 1280, "blob too small for rows x K"
    codes = np.empty((rows, K), dtype=np.uint8)
    scales = np.empty((rows, K // 32), dtype=np.uint16)
    load().oracle_unpack_q2_tiled(rows, K, _p(blob), panel_stride, slice_stride, _p(codes), _p(scales))
    return codes, scales.view(np.float16)


def unpack_q4_tiled(blob, rows: int, K: int, panel_stride: int = None, slice_stride: int = 2304):
    """Codes and scales of one 4-bit matrix (2304-byte tiles) whose tile
    (p, s) starts at ``blob + p * panel_stride + s * slice_stride``."""
    blob = _c(blob, np.uint8)
    if panel_stride is None:
        panel_stride = (K // 64) * slice_stride
    last = (rows // 64 - 1) * panel_stride + (K // 64 - 1) * slice_stride
    assert blob.size >= last + 2304, "blob too small for rows x K"
    codes = np.empty((rows, K), dtype=np.uint8)
    scales = np.empty((rows, K // 32), dtype=np.uint16)
    load().oracle_unpack_q4_tiled(rows, K, _p(blob), panel_stride, slice_stride, _p(codes), _p(scales))
    return codes, scales.view(np.float16)


def unpack_expert(blob, d: int, f: int, bits: int = 2) -> dict:
    """Codes/scales of one expert from its blob section (header's layout):
    gate/up tiles interleaved in (f-panel, d-slice) order, 2560-byte pairs;
    then the down matrix [d x f] with its tiles in (f-slice, d-panel) order."""
    blob = _c(blob, np.uint8)
    tb = 1280 if bits == 2 else 2304  # tile bytes
    un = unpack_q2_tiled if bits == 2 else unpack_q4_tiled
    gu = (f // 64) * (d // 64) * 2 * tb
    gc, gs = un(blob, f, d, (d // 64) * 2 * tb, 2 * tb)
    uc, us = un(blob[tb:], f, d, (d // 64) * 2 * tb, 2 * tb)
    dc, ds = un(blob[gu:], d, f, tb, (d // 64) * tb)
    return dict(gate_codes=gc, gate_scales=gs, up_codes=uc, up_scales=us, down_codes=dc, down_scales=ds, bits=bits)


def router_logits(x_bf16, W, bias=None):
    x = _c(x_bf16, np.uint16)
    W = _c(W, np.float32)
    T, d = x.shape
    E = W.shape[0]
    b = None if bias is None else _c(bias, np.float32)
    out = np.empty((T, E), dtype=np.float64)
    load().oracle_router_logits(T, d, E, _p(x), _p(W), _p(b), _p(out))
    return out


def topk_softmax(logits, k: int):
    l = _c(logits, np.float64)
    T, E = l.shape
    idx = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    load().oracle_topk_softmax(T, E, k, _p(l), _p(idx), _p(w))
    return idx, w


def expert_lists(idx, E: int):
    idx = _c(idx, np.int32)
    T, k = idx.shape
    off = np.empty(E + 1, dtype=np.int32)
    tl = np.empty(T * k, dtype=np.int32)
    sl = np.empty(T * k, dtype=np.int32)
    load().oracle_expert_lists(T, E, k, _p(idx), _p(off), _p(tl), _p(sl))
    return off, tl, sl


def _sc(a):
    a = np.asarray(a)
    return _c(a.view(np.uint16) if a.dtype == np.float16 else a, np.uint16)


def expert_ffn(X, ex: dict):
    """SwiGLU expert on rows of X (double [n, d]); ex holds codes/scales (and
    "bits", 2 when absent)."""
    X = _c(X, np.float64)
    n, d = X.shape
    f = ex["gate_codes"].shape[0]
    out = np.empty((n, d), dtype=np.float64)
    keep = [_c(ex["gate_codes"], np.uint8), _sc(ex["gate_scales"]),
            _c(ex["up_codes"], np.uint8), _sc(ex["up_scales"]),
            _c(ex["down_codes"], np.uint8), _sc(ex["down_scales"])]
    load().oracle_expert_ffn(d, f, n, int(ex.get("bits", 2)), _p(X), *[_p(a) for a in keep], _p(out))
    return out


def moe_layer(x_bf16, W, bias, experts: list, k: int):
    """Whole layer (small shapes): returns y (double [T, d]), idx, w."""
    x = _c(x_bf16, np.uint16)
    W = _c(W, np.float32)
    T, d = x.shape
    E = W.shape[0]
    f = experts[0]["gate_codes"].shape[0]
    b = None if bias is None else _c(bias, np.float32)
    keep = []

    def arr(name, conv):
        ptrs = (ctypes.c_void_p * E)()
        for e in range(E):
            a = conv(experts[e][name])
            keep.append(a)
            ptrs[e] = a.ctypes.data
        keep.append(ptrs)
        return ptrs

    u8 = lambda a: _c(a, np.uint8)
    pa = [arr("gate_codes", u8), arr("gate_scales", _sc), arr("up_codes", u8),
          arr("up_scales", _sc), arr("down_codes", u8), arr("down_scales", _sc)]
    y = np.empty((T, d), dtype=np.float64)
    idx = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    bits = int(experts[0].get("bits", 2))
    assert all(int(e.get("bits", 2)) == bits for e in experts), "one code width per layer"
    load().oracle_moe_layer(T, d, f, E, k, bits, _p(x), _p(W), _p(b),
                            *[ctypes.cast(p, ctypes.c_void_p) for p in pa], _p(y), _p(idx), _p(w))
    return y, idx, w


def rmsnorm_bf16(x, eps: float):
    """bf16 bits of RMSNorm(x) for each row of x (double)."""
    x = np.atleast_2d(_c(x, np.float64))
    out = np.empty(x.shape, dtype=np.uint16)
    lib = load()
    for t in range(x.shape[0]):
        lib.oracle_rmsnorm_bf16(x.shape[1], _p(x[t]), float(eps), _p(out[t]))
    return out


def residual_add_f32(x_f32, y):
    x = _c(x_f32, np.float32).copy()
    y = _c(y, np.float64)
    load().oracle_residual_add_f32(x.size, _p(x), _p(y))
    return x


# ----------------------------------------------------------------------------
# 4-bit Hadamard-rotated KV-cache codec


def float_to_fp16(v):
    """fp32 values -> fp16 bit patterns (round to nearest even)."""
    lib = load()
    return np.array([lib.oracle_float_to_fp16(float(x)) for x in np.ravel(np.asarray(v, dtype=np.float32))],
                    dtype=np.uint16).reshape(np.shape(v))


def hadamard_sign(i: int, j: int) -> int:
    return load().oracle_hadamard_sign(int(i), int(j))


def fwht_f32(v):
    """Unnormalised Walsh-Hadamard transform of one fp32 vector (fp32 steps)."""
    v = np.array(v, dtype=np.float32)
    load().oracle_fwht_f32(v.size, _p(v))
    return v


def kv4_quantize_block(y):
    """One 32-value block -> (codes uint8[32] in 1..15, fp16 scale bits)."""
    y = _c(y, np.float32)
    assert y.size == 32
    code = np.empty(32, dtype=np.uint8)
    sb = np.zeros(1, dtype=np.uint16)
    load().oracle_kv4_quantize_block(_p(y), _p(code), _p(sb))
    return code, int(sb[0])


def kv4_encode(x_bf16):
    """bf16 rows [rows, D] -> (codes uint8 [rows, D/2], scales fp16 bits uint16 [rows, D/32])."""
    x = _c(x_bf16, np.uint16)
    rows, D = x.shape
    codes = np.empty((rows, D // 2), dtype=np.uint8)
    scales = np.empty((rows, D // 32), dtype=np.uint16)
    load().oracle_kv4_encode(rows, D, _p(x), _p(codes), _p(scales))
    return codes, scales


def kv4_decode(codes, scales):
    """(codes, scales) -> (exact values as double [rows, D], their bf16 bits)."""
    codes = _c(codes, np.uint8)
    sc = _c(np.asarray(scales).view(np.uint16), np.uint16)
    rows, D = codes.shape[0], codes.shape[1] * 2
    out = np.empty((rows, D), dtype=np.float64)
    bits = np.empty((rows, D), dtype=np.uint16)
    lib = load()
    lib.oracle_kv4_decode(rows, D, _p(codes), _p(sc), _p(out))
    lib.oracle_round_bf16_array(out.size, _p(out), _p(bits))
    return out, bits


# ----------------------------------------------------------------------------
# workload-level helpers (experts generated on demand from the seeded source)


def route_layer(x_bf16, W, bias, k: int):
    """Routing of every token: logits (double), idx, w, per-expert lists."""
    logits = router_logits(x_bf16, W, bias)
    idx, w = topk_softmax(logits, k)
    off, tl, sl = expert_lists(idx, W.shape[0])
    return dict(logits=logits, idx=idx, w=w, offsets=off, token_list=tl, pair_slot=sl)


def layer_outputs(x_bf16, route: dict, tokens, expert_source):
    """y rows for the given tokens: sum_j w[t][j] * expert_{idx[t][j]}(x_t).

    ``expert_source(e)`` returns the codes/scales dict of expert e. Experts are
    visited once each, for all requested tokens that selected them."""
    tokens = np.asarray(tokens, dtype=np.int64)
    d = x_bf16.shape[1]
    idx, w = route["idx"], route["w"]
    y = np.zeros((tokens.size, d), dtype=np.float64)
    X = np.stack([_bf16_row(x_bf16[t]) for t in tokens]) if tokens.size else np.zeros((0, d))
    need = {}
    for r, t in enumerate(tokens):
        for j in range(idx.shape[1]):
            need.setdefault(int(idx[t, j]), []).append((r, j))
    for e in sorted(need):
        rows = need[e]
        out = expert_ffn(X[[r for r, _ in rows]], expert_source(e))
        for (r, j), o in zip(rows, out):
            y[r] += w[tokens[r], j] * o
    return y


def _bf16_row(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
