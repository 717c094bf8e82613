"""Device-side generation of the same seeded inputs (see ``synth``), for
workloads too large to draw on the host. Bit-identical to the numpy
generator; ``tests/test_gpu_synth.py`` checks that on samples."""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

from . import (DOWN, GATE, TAG_CODES, TAG_KV, TAG_ROUTER_W, TAG_SCALES, TAG_X, UP, Workload, kv_outlier_channels,
               router_bias, stream_key)

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth_dev.cu")
_LIB = os.path.join(_HERE, "libsynth.so")
_lib = None


def build(force: bool = False) -> str:
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.run(["/usr/local/cuda/bin/nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3",
                        "-Xcompiler", "-fPIC", "-shared", "-o", _LIB, _SRC], check=True)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB):
            raise RuntimeError(f"{_LIB} is missing: build it with synth.device.build()")
        lib = ctypes.CDLL(_LIB)
        V, I64 = ctypes.c_void_p, ctypes.c_int64
        lib.synth_codes.argtypes = [V, ctypes.c_int, I64, V, V]
        lib.synth_codes4.argtypes = [V, ctypes.c_int, I64, V, V]
        lib.synth_scales.argtypes = [V, ctypes.c_int, I64, ctypes.c_float, V, V]
        lib.synth_x_bf16.argtypes = [ctypes.c_uint64, I64, I64, V, V]
        lib.synth_router_w.argtypes = [ctypes.c_uint64, I64, V, V]
        for f in (lib.synth_codes, lib.synth_scales, lib.synth_x_bf16, lib.synth_router_w):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def _stream():
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _chk(rc):
    if rc != 0:
        raise RuntimeError(f"synth device kernel failed ({rc})")


def x_bf16(seed: int, T: int, d: int, stream: int = 0, tok0: int = 0):
    """torch.bfloat16 [T, d] on the current device (same as synth.gen_x_bf16)."""
    import torch
    out = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    _chk(_load().synth_x_bf16(stream_key(seed, TAG_X, stream), tok0 * d, T * d, out.data_ptr(), _stream()))
    return out


def kv_rows(seed: int, rows: int, D: int, row0: int = 0):
    """torch.bfloat16 [rows, D] on the current device (same as synth.gen_kv_rows)."""
    import torch
    out = torch.empty((rows, D), dtype=torch.bfloat16, device="cuda")
    _chk(_load().synth_x_bf16(stream_key(seed, TAG_KV), row0 * D, rows * D, out.data_ptr(), _stream()))
    ch = torch.from_numpy(kv_outlier_channels(seed, D)).cuda()
    out[:, ch] *= 16  # exact in bf16
    return out


def router_w(seed: int, layer: int, E: int, d: int):
    import torch
    out = torch.empty((E, d), dtype=torch.float32, device="cuda")
    _chk(_load().synth_router_w(stream_key(seed, TAG_ROUTER_W, layer), E * d, out.data_ptr(), _stream()))
    return out


def _keys(seed, tag, layer, experts, mat):
    import torch
    k = np.array([stream_key(seed, tag, layer, e, mat) for e in experts], dtype=np.uint64)
    return torch.from_numpy(k.view(np.int64)).to("cuda")


def expert_codes_scales(seed: int, layer: int, experts, mat: int, rows: int, K: int, bits: int = 2):
    """codes uint8 [n, rows, K] and scales (fp16 bits as int16) [n, rows, K/32]."""
    import torch
    experts = list(experts)
    n = len(experts)
    codes = torch.empty((n, rows, K), dtype=torch.uint8, device="cuda")
    scales = torch.empty((n, rows, K // 32), dtype=torch.int16, device="cuda")
    kc = _keys(seed, TAG_CODES, layer, experts, mat)
    ks = _keys(seed, TAG_SCALES, layer, experts, mat)
    gen = _load().synth_codes if bits == 2 else _load().synth_codes4
    _chk(gen(kc.data_ptr(), n, rows * K, codes.data_ptr(), _stream()))
    _chk(_load().synth_scales(ks.data_ptr(), n, rows * (K // 32), ctypes.c_float(1.0 if bits == 2 else 5.0),
                              scales.data_ptr(), _stream()))
    return codes, scales


def layer_blob(w: Workload, layer: int, pack_expert, out=None, batch: int = 32):
    """Packed expert blob of one layer on the device.

    ``pack_expert(e, gc, gs, uc, us, dc, ds, dst)`` is the caller's packer (the
    library's device packer); this module only supplies the codes/scales."""
    import torch
    d, f, E = w.d, w.f, w.E
    ebytes = 3 * (d // 64) * (f // 64) * (1280 if w.bits == 2 else 2304)
    if out is None:
        out = torch.empty(E * ebytes, dtype=torch.uint8, device="cuda")
    for e0 in range(0, E, batch):
        ex = list(range(e0, min(E, e0 + batch)))
        gc, gs = expert_codes_scales(w.seed, layer, ex, GATE, f, d, w.bits)
        uc, us = expert_codes_scales(w.seed, layer, ex, UP, f, d, w.bits)
        dc, ds = expert_codes_scales(w.seed, layer, ex, DOWN, d, f, w.bits)
        for i, e in enumerate(ex):
            pack_expert(e, gc[i], gs[i], uc[i], us[i], dc[i], ds[i], out[e * ebytes:(e + 1) * ebytes])
    return out


def layer_inputs(w: Workload, layer: int):
    """Router weights and bias of one layer on the device."""
    import torch
    W = router_w(w.seed, layer, w.E, w.d)
    b = router_bias(w, layer)
    bias = None if b is None else torch.from_numpy(b).to("cuda")
    return W, bias
