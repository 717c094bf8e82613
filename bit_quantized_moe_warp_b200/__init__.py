"""Python binding of the B200 routed-expert MoE layer (libstrata_moe.so).

Argument marshalling only: every function below forwards to the C ABI of
``include/strata_moe.h`` with the same name; tensors may be passed as torch
tensors (their ``data_ptr()``) or as integer device addresses. Every step of
the layer runs in the library's sm_100a kernels. Importing this package fails
loudly when the shared library has not been built.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# STRATA_MOE_LIB selects another build of the same library (e.g. the checked build,
# libstrata_moe_checked.so)
LIB_PATH = os.environ.get("STRATA_MOE_LIB") or os.path.join(_HERE, "libstrata_moe.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m bit_quantized_moe_warp_b200.build` "
                      "(or __graft_entry__.build())")

_lib = ctypes.CDLL(LIB_PATH)

# status codes (include/strata_moe.h)
STRATA_OK = 0
STRATA_ERR_INVALID_ARG = -1
STRATA_ERR_UNSUPPORTED = -2
STRATA_ERR_CUDA = -3
STRATA_ERR_OOM = -4
STRATA_ERR_TOO_MANY_TOKENS = -5
STRATA_ERR_BAD_BLOB = -6
STRATA_ERR_TIMEOUT = -7
STRATA_ERR_BOUNDS = -8

STRATA_FMT_Q2_0_TILED = 1
STRATA_FMT_Q4_0_TILED = 2
STRATA_ACCUMULATE = 1
STRATA_FORCE_PREFILL = 2
STRATA_DECODE_MAX_TOKENS = 16
STRATA_Q2_TILE_BYTES = 1280
STRATA_Q4_TILE_BYTES = 2304
STRATA_KV4_BLOCK = 32  # include/strata_kv.h
FORMAT_OF_BITS = {2: STRATA_FMT_Q2_0_TILED, 4: STRATA_FMT_Q4_0_TILED}


class strata_moe_desc(ctypes.Structure):
    _fields_ = [("d_model", ctypes.c_int32), ("d_ff", ctypes.c_int32), ("n_experts", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("max_tokens", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("weight_format", ctypes.c_int32), ("flags", ctypes.c_uint32), ("router_bias", ctypes.c_void_p)]


class StrataError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{_lib.strata_status_string(status).decode()} ({status}): {msg}")
        self.status = status


V, I32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
DP = ctypes.POINTER(strata_moe_desc)
_SIGS = {
    "strata_q2_matrix_bytes": (SZ, [I32, I32]),
    "strata_q4_matrix_bytes": (SZ, [I32, I32]),
    "strata_moe_expert_bytes": (SZ, [DP]),
    "strata_moe_expert_blob_bytes": (SZ, [DP]),
    "strata_moe_workspace_bytes": (SZ, [DP]),
    "strata_moe_layer_create": (I32, [DP, V, SZ, ctypes.POINTER(V)]),
    "strata_moe_layer_destroy": (I32, [V]),
    "strata_moe_forward": (I32, [V, V, V, V, V, I32, V]),
    "strata_moe_router_logits": (I32, [V, V, V, V, I32, V]),
    "strata_moe_route": (I32, [V, V, V, I32, V]),
    "strata_moe_experts": (I32, [V, V, V, V, I32, V]),
    "strata_moe_get_routing": (I32, [V, V, V, V, V, V, V]),
    "strata_moe_route_noalloc": (I32, [DP, V, V, I32, V, V, V, V, V, V]),
    "strata_moe_stack_forward": (I32, [V, I32, V, V, V, V, I32, ctypes.c_float, V]),
    "strata_rmsnorm_bf16": (I32, [V, V, I32, I32, ctypes.c_float, V]),
    "strata_moe_set_stage_events": (I32, [V, V, I32]),
    "strata_moe_check_status": (I32, [V]),
    "strata_q2_pack": (I32, [V, V, I32, I32, V]),
    "strata_q4_pack": (I32, [V, V, I32, I32, V]),
    "strata_moe_pack_expert": (I32, [DP, V, V, V, V, V, V, V]),
    "strata_moe_pack_expert_device": (I32, [DP, V, V, V, V, V, V, V, V]),
    "strata_selftest_wait_timeout": (I32, [ctypes.c_uint64, V]),
    "strata_selftest_bounds_check": (I32, [V]),
    "strata_is_checked_build": (I32, []),
    "strata_kv4_code_bytes": (SZ, [ctypes.c_int64, I32]),
    "strata_kv4_scale_bytes": (SZ, [ctypes.c_int64, I32]),
    "strata_kv4_encode": (I32, [V, ctypes.c_int64, I32, V, V, V]),
    "strata_kv4_decode": (I32, [V, V, ctypes.c_int64, I32, V, V]),
    "strata_status_string": (ctypes.c_char_p, [I32]),
    "strata_last_error": (ctypes.c_char_p, []),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args

EXPORTED = tuple(_SIGS)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int):
    if status != STRATA_OK:
        raise StrataError(status, _lib.strata_last_error().decode(errors="replace"))


def make_desc(d_model, d_ff, n_experts, top_k, max_tokens, flags=0, router_bias=None, bits=2) -> strata_moe_desc:
    """Layer descriptor; bits = 2 or 4 picks the weight format."""
    return strata_moe_desc(d_model, d_ff, n_experts, top_k, max_tokens, 32, FORMAT_OF_BITS.get(bits, 0), flags,
                           _ptr(router_bias))


# ---------------------------------------------------------------- C ABI


def strata_q2_matrix_bytes(rows, K):
    return _lib.strata_q2_matrix_bytes(rows, K)


def strata_q4_matrix_bytes(rows, K):
    return _lib.strata_q4_matrix_bytes(rows, K)


def strata_moe_expert_bytes(desc):
    return _lib.strata_moe_expert_bytes(ctypes.byref(desc))


def strata_moe_expert_blob_bytes(desc):
    return _lib.strata_moe_expert_blob_bytes(ctypes.byref(desc))


def strata_moe_workspace_bytes(desc):
    return _lib.strata_moe_workspace_bytes(ctypes.byref(desc))


def strata_moe_layer_create(desc, workspace=None, workspace_bytes=0):
    h = ctypes.c_void_p()
    _check(_lib.strata_moe_layer_create(ctypes.byref(desc), _ptr(workspace), workspace_bytes, ctypes.byref(h)))
    return h.value


def strata_moe_layer_destroy(layer):
    _check(_lib.strata_moe_layer_destroy(layer))


def strata_moe_forward(layer, x, router_w, expert_blob, y, n_tokens, stream=None):
    _check(_lib.strata_moe_forward(layer, _ptr(x), _ptr(router_w), _ptr(expert_blob), _ptr(y), n_tokens,
                                   _stream(stream)))


def strata_moe_router_logits(layer, x, router_w, logits, n_tokens, stream=None):
    _check(_lib.strata_moe_router_logits(layer, _ptr(x), _ptr(router_w), _ptr(logits), n_tokens, _stream(stream)))


def strata_moe_route(layer, x, router_w, n_tokens, stream=None):
    _check(_lib.strata_moe_route(layer, _ptr(x), _ptr(router_w), n_tokens, _stream(stream)))


def strata_moe_experts(layer, x, expert_blob, y, n_tokens, stream=None):
    _check(_lib.strata_moe_experts(layer, _ptr(x), _ptr(expert_blob), _ptr(y), n_tokens, _stream(stream)))


def strata_moe_get_routing(layer, topk_idx=None, topk_w=None, expert_offsets=None, token_list=None,
                           pair_slot=None, stream=None):
    _check(_lib.strata_moe_get_routing(layer, _ptr(topk_idx), _ptr(topk_w), _ptr(expert_offsets),
                                       _ptr(token_list), _ptr(pair_slot), _stream(stream)))


def strata_moe_route_noalloc(desc, x, router_w, n_tokens, topk_idx, topk_w, expert_offsets, token_list,
                             pair_slot, stream=None):
    _check(_lib.strata_moe_route_noalloc(ctypes.byref(desc), _ptr(x), _ptr(router_w), n_tokens, _ptr(topk_idx),
                                         _ptr(topk_w), _ptr(expert_offsets), _ptr(token_list), _ptr(pair_slot),
                                         _stream(stream)))


def strata_moe_stack_forward(layer, router_w, router_bias, expert_blobs, x_resid, n_tokens, rms_eps,
                             stream=None):
    n = len(router_w)
    W = (ctypes.c_void_p * n)(*[_ptr(w) for w in router_w])
    B = None if router_bias is None else (ctypes.c_void_p * n)(*[_ptr(b) for b in router_bias])
    X = (ctypes.c_void_p * n)(*[_ptr(b) for b in expert_blobs])
    _check(_lib.strata_moe_stack_forward(layer, n, ctypes.cast(W, V), None if B is None else ctypes.cast(B, V),
                                         ctypes.cast(X, V), _ptr(x_resid), n_tokens, float(rms_eps),
                                         _stream(stream)))


def strata_kv4_code_bytes(n_rows, head_dim):
    return _lib.strata_kv4_code_bytes(n_rows, head_dim)


def strata_kv4_scale_bytes(n_rows, head_dim):
    return _lib.strata_kv4_scale_bytes(n_rows, head_dim)


def strata_kv4_encode(x, n_rows, head_dim, codes, scales, stream=None):
    """bf16 rows [n_rows, head_dim] -> 4-bit codes [n_rows, head_dim/2] and fp16 scales [n_rows, head_dim/32]."""
    _check(_lib.strata_kv4_encode(_ptr(x), n_rows, head_dim, _ptr(codes), _ptr(scales), _stream(stream)))


def strata_kv4_decode(codes, scales, n_rows, head_dim, out, stream=None):
    """4-bit codes and fp16 scales of n_rows rows -> bf16 rows [n_rows, head_dim]."""
    _check(_lib.strata_kv4_decode(_ptr(codes), _ptr(scales), n_rows, head_dim, _ptr(out), _stream(stream)))


def strata_rmsnorm_bf16(x, out, n_tokens, d, eps, stream=None):
    _check(_lib.strata_rmsnorm_bf16(_ptr(x), _ptr(out), n_tokens, d, float(eps), _stream(stream)))


def strata_moe_set_stage_events(layer, events):
    """events: five torch.cuda.Event (timing enabled) or raw handles; [] clears."""
    import torch
    handles = []
    for e in events:
        if isinstance(e, torch.cuda.Event):
            if e.cuda_event == 0:
                e.record()
            handles.append(e.cuda_event)
        else:
            handles.append(int(e))
    arr = (ctypes.c_void_p * max(1, len(handles)))(*handles)
    _check(_lib.strata_moe_set_stage_events(layer, ctypes.cast(arr, V), len(handles)))


def strata_moe_check_status(layer):
    _check(_lib.strata_moe_check_status(layer))


def strata_q2_pack(codes, scales_fp16, rows, K, dst):
    """Host packer: numpy arrays (uint8 codes, uint16/float16 scales, uint8 dst)."""
    import numpy as np
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    s = np.ascontiguousarray(np.asarray(scales_fp16).view(np.uint16))
    _check(_lib.strata_q2_pack(c.ctypes.data, s.ctypes.data, rows, K, dst.ctypes.data))


def strata_q4_pack(codes, scales_fp16, rows, K, dst):
    """Host packer of the 4-bit format (codes 0..15), arguments as strata_q2_pack."""
    import numpy as np
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    s = np.ascontiguousarray(np.asarray(scales_fp16).view(np.uint16))
    _check(_lib.strata_q4_pack(c.ctypes.data, s.ctypes.data, rows, K, dst.ctypes.data))


def strata_moe_pack_expert(desc, gc, gs, uc, us, dc, ds, dst):
    """Host packer of one expert (numpy arrays)."""
    import numpy as np
    a = [np.ascontiguousarray(v, dtype=np.uint8) for v in (gc, uc, dc)]
    s = [np.ascontiguousarray(np.asarray(v).view(np.uint16)) for v in (gs, us, ds)]
    _check(_lib.strata_moe_pack_expert(ctypes.byref(desc), a[0].ctypes.data, s[0].ctypes.data, a[1].ctypes.data,
                                       s[1].ctypes.data, a[2].ctypes.data, s[2].ctypes.data, dst.ctypes.data))


def strata_moe_pack_expert_device(desc, gc, gs, uc, us, dc, ds, dst, stream=None):
    _check(_lib.strata_moe_pack_expert_device(ctypes.byref(desc), _ptr(gc), _ptr(gs), _ptr(uc), _ptr(us),
                                              _ptr(dc), _ptr(ds), _ptr(dst), _stream(stream)))


def strata_selftest_wait_timeout(timeout_ns, stream=None):
    return _lib.strata_selftest_wait_timeout(int(timeout_ns), _stream(stream))


def strata_selftest_bounds_check(stream=None):
    return _lib.strata_selftest_bounds_check(_stream(stream))


def strata_is_checked_build():
    return _lib.strata_is_checked_build()


def strata_status_string(status):
    return _lib.strata_status_string(status).decode()


def strata_last_error():
    return _lib.strata_last_error().decode(errors="replace")


# ---------------------------------------------------------------- handle


class MoELayer:
    """Owns a layer handle (and keeps the desc's bias tensor alive)."""

    def __init__(self, d_model, d_ff, n_experts, top_k, max_tokens, flags=0, router_bias=None, workspace=None,
                 bits=2):
        self._bias = router_bias
        self.desc = make_desc(d_model, d_ff, n_experts, top_k, max_tokens, flags, router_bias, bits)
        nbytes = strata_moe_workspace_bytes(self.desc) if workspace is not None else 0
        self.handle = strata_moe_layer_create(self.desc, workspace, nbytes)

    def close(self):
        if self.handle:
            strata_moe_layer_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def forward(self, x, router_w, blob, y, n_tokens, stream=None):
        strata_moe_forward(self.handle, x, router_w, blob, y, n_tokens, stream)

    def router_logits(self, x, router_w, logits, n_tokens, stream=None):
        strata_moe_router_logits(self.handle, x, router_w, logits, n_tokens, stream)

    def route(self, x, router_w, n_tokens, stream=None):
        strata_moe_route(self.handle, x, router_w, n_tokens, stream)

    def experts(self, x, blob, y, n_tokens, stream=None):
        strata_moe_experts(self.handle, x, blob, y, n_tokens, stream)

    def routing(self, n_tokens, stream=None):
        """Routing of the last call as torch tensors."""
        import torch
        k, E = self.desc.top_k, self.desc.n_experts
        dev = torch.device("cuda")
        idx = torch.empty((n_tokens, k), dtype=torch.int32, device=dev)
        w = torch.empty((n_tokens, k), dtype=torch.float32, device=dev)
        off = torch.empty(E + 1, dtype=torch.int32, device=dev)
        tl = torch.empty(n_tokens * k, dtype=torch.int32, device=dev)
        sl = torch.empty(n_tokens * k, dtype=torch.int32, device=dev)
        strata_moe_get_routing(self.handle, idx, w, off, tl, sl, stream)
        return idx, w, off, tl, sl

    def stack_forward(self, router_w, router_bias, blobs, x_resid, n_tokens, eps, stream=None):
        strata_moe_stack_forward(self.handle, router_w, router_bias, blobs, x_resid, n_tokens, eps, stream)

    def check_status(self):
        strata_moe_check_status(self.handle)

    def pack_expert_device(self, gc, gs, uc, us, dc, ds, dst, stream=None):
        strata_moe_pack_expert_device(self.desc, gc, gs, uc, us, dc, ds, dst, stream)
