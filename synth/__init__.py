"""Seeded synthetic inputs for the routed-expert layer (host side, numpy).

This module is shared by the CPU oracle's tests and by the GPU harness. It
holds no arithmetic of the layer itself: it only draws the inputs (token
activations, router weights, 2-bit codes, block scales, the expert-popularity
prior) from a counter-based generator, so that any element can be regenerated
on its own, on the host or on the device, with the same bits.

Generator (defined here; the device twin in ``synth_dev.cu`` restates it):

* ``mix64`` is the SplitMix64 output function (Steele, Lea & Flood, "Fast
  splittable pseudorandom number generators", OOPSLA 2014).
* A stream is a 64-bit key derived from a seed and a tuple of integer ids.
  Word ``i`` of a stream is ``mix64(key + (i + 1) * GAMMA)`` (mod 2**64), i.e.
  the SplitMix64 sequence started at ``key``.
* Uniform codes: word ``i`` supplies codes ``32 i .. 32 i + 31`` as its 2-bit
  fields, least significant first; 4-bit codes: word ``i`` supplies codes
  ``16 i .. 16 i + 15`` as its 4-bit fields.
* Normals: Irwin-Hall with 12 terms. Normal ``i`` takes words ``4 i .. 4 i + 3``,
  each split into three 20-bit uniforms (bits 0-19, 20-39, 40-59); with ``S``
  the integer sum of the 12 fields, ``z = (S - 6 * 2**20) * 2**-20``. ``z`` is
  an exact float32 (|S - 6*2**20| < 2**24), mean 0, variance 1, support
  (-6, 6). Every later step (bf16 / fp16 rounding, scaling by 0.02) is a single
  IEEE round-to-nearest-even operation, so host and device agree bit for bit.

Workloads (the layer's synthetic configurations):

* tiny:    d=256,  f=128, E=16,  k=4,  T=8,    1 layer, uniform routing, seed 0
* decode:  d=2048, f=768, E=512, k=10, T=1,    1 layer, uniform routing, seed 1
* verify:  d=2048, f=768, E=512, k=10, T=4/16, 48 layers, Zipf(1.1) prior, seed 2
* prefill: d=2048, f=768, E=512, k=10, T=8192, 1 layer, Zipf(1.1) prior, seed 3
* prefill_stack: 32768 tokens in 8192-token chunks, 48 layers, Zipf, seed 4

Value distributions: x ~ N(0,1) rounded to bf16; router W ~ N(0, 0.02) in
fp32; codes uniform in {0,1,2,3}; block scales fp16(|N(0, 0.02)| + 1e-3).
The Zipf prior is an additive router bias b_e = ln p(rank(e)) with
p(r) = r^-1.1 / sum_{r'=1..E} r'^-1.1 and a seeded permutation rank().
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

MASK64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15
MUL1 = 0xBF58476D1CE4E5B9
MUL2 = 0x94D049BB133111EB

# stream tags
TAG_X = 1
TAG_ROUTER_W = 2
TAG_CODES = 3
TAG_SCALES = 4
TAG_PERM = 5
TAG_KV = 6
TAG_KV_OUTLIERS = 7

# matrix ids inside one expert
GATE, UP, DOWN = 0, 1, 2


def mix64_int(z: int) -> int:
    z &= MASK64
    z = ((z ^ (z >> 30)) * MUL1) & MASK64
    z = ((z ^ (z >> 27)) * MUL2) & MASK64
    return z ^ (z >> 31)


def stream_key(seed: int, *ids: int) -> int:
    """64-bit key of the stream named by ``seed`` and ``ids``."""
    k = mix64_int(seed * GAMMA + 0x5851F42D4C957F2D)
    for i in ids:
        k = mix64_int(k ^ (((i + 1) * GAMMA) & MASK64))
    return k


def _mix64_np(z: np.ndarray) -> np.ndarray:
    z = z.astype(np.uint64, copy=True)
    with np.errstate(over="ignore"):
        z ^= z >> np.uint64(30)
        z *= np.uint64(MUL1)
        z ^= z >> np.uint64(27)
        z *= np.uint64(MUL2)
        z ^= z >> np.uint64(31)
    return z


def words(key: int, start: int, count: int) -> np.ndarray:
    """Words ``start .. start+count-1`` of stream ``key`` (uint64)."""
    i = np.arange(start, start + count, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(key) + (i + np.uint64(1)) * np.uint64(GAMMA)
    return _mix64_np(z)


def codes(key: int, n: int, start: int = 0) -> np.ndarray:
    """Codes ``start .. start+n-1`` (uint8 in {0..3}); ``start`` % 32 == 0."""
    assert start % 32 == 0
    nw = (n + 31) // 32
    w = words(key, start // 32, nw)
    sh = (np.arange(32, dtype=np.uint64) * np.uint64(2))[None, :]
    c = ((w[:, None] >> sh) & np.uint64(3)).astype(np.uint8).reshape(-1)
    return c[:n]


def codes4(key: int, n: int, start: int = 0) -> np.ndarray:
    """4-bit codes ``start .. start+n-1`` (uint8 in {0..15}); word ``i``
    supplies codes ``16 i .. 16 i + 15`` as its 4-bit fields, least
    significant first; ``start`` % 16 == 0."""
    assert start % 16 == 0
    nw = (n + 15) // 16
    w = words(key, start // 16, nw)
    sh = (np.arange(16, dtype=np.uint64) * np.uint64(4))[None, :]
    c = ((w[:, None] >> sh) & np.uint64(15)).astype(np.uint8).reshape(-1)
    return c[:n]


def normals(key: int, n: int, start: int = 0) -> np.ndarray:
    """Irwin-Hall(12) normals ``start .. start+n-1`` as exact float32."""
    w = words(key, 4 * start, 4 * n).reshape(n, 4)
    m = np.uint64(0xFFFFF)
    s = np.zeros(n, dtype=np.int64)
    for j in range(4):
        wj = w[:, j]
        s += (wj & m).astype(np.int64)
        s += ((wj >> np.uint64(20)) & m).astype(np.int64)
        s += ((wj >> np.uint64(40)) & m).astype(np.int64)
    z = (s - 6 * (1 << 20)).astype(np.float32) * np.float32(2.0 ** -20)
    return z


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even); returns uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ----------------------------------------------------------------------------
# per-tensor generators


def gen_x_bf16(seed: int, T: int, d: int, stream: int = 0, tok0: int = 0) -> np.ndarray:
    """Token activations x ~ N(0,1) in bf16, uint16 bits [T, d]; rows tok0.."""
    z = normals(stream_key(seed, TAG_X, stream), T * d, start=tok0 * d)
    return f32_to_bf16_bits(z).reshape(T, d)


def gen_router_w(seed: int, layer: int, E: int, d: int) -> np.ndarray:
    """Router weights W ~ N(0, 0.02) in fp32 [E, d]."""
    z = normals(stream_key(seed, TAG_ROUTER_W, layer), E * d)
    return (np.float32(0.02) * z).astype(np.float32).reshape(E, d)


def gen_codes(seed: int, layer: int, expert: int, mat: int, rows: int, K: int, bits: int = 2) -> np.ndarray:
    """Codes uint8 [rows, K] of one matrix of one expert: 2-bit codes in
    {0..3} or 4-bit codes in {0..15}."""
    key = stream_key(seed, TAG_CODES, layer, expert, mat)
    return (codes(key, rows * K) if bits == 2 else codes4(key, rows * K)).reshape(rows, K)


def gen_scales(seed: int, layer: int, expert: int, mat: int, rows: int, K: int, bits: int = 2) -> np.ndarray:
    """Block scales, float16 [rows, K/32]: fp16(|N(0,0.02)| + 1e-3) for 2-bit
    codes; for 4-bit codes the same value divided by 5, so that (c - 7.5) s
    spans the range (c - 1.5) s does with 2-bit codes."""
    nb = rows * (K // 32)
    z = normals(stream_key(seed, TAG_SCALES, layer, expert, mat), nb)
    t = np.abs(np.float32(0.02) * z) + np.float32(1e-3)
    if bits == 4:
        t = t / np.float32(5.0)
    return t.astype(np.float32).astype(np.float16).reshape(rows, K // 32)


def gen_expert(seed: int, layer: int, expert: int, d: int, f: int, bits: int = 2) -> dict:
    """Codes and scales of one expert: gate/up [f, d], down [d, f]."""
    out = {"bits": bits}
    for name, mat, rows, K in (("gate", GATE, f, d), ("up", UP, f, d), ("down", DOWN, d, f)):
        out[name + "_codes"] = gen_codes(seed, layer, expert, mat, rows, K, bits)
        out[name + "_scales"] = gen_scales(seed, layer, expert, mat, rows, K, bits)
    return out


def zipf_permutation(seed: int, layer: int, E: int) -> np.ndarray:
    """Seeded permutation rank[e] in 0..E-1 (Fisher-Yates on stream words)."""
    w = words(stream_key(seed, TAG_PERM, layer), 0, E)
    perm = np.arange(E, dtype=np.int64)
    for i in range(E - 1, 0, -1):
        j = int(w[i] % np.uint64(i + 1))
        perm[i], perm[j] = perm[j], perm[i]
    return perm


def gen_zipf_bias(seed: int, layer: int, E: int, s: float = 1.1) -> np.ndarray:
    """Additive router bias b_e = ln p(rank(e)), p(r) ∝ r^-s, fp32 [E]."""
    H = math.fsum(r ** -s for r in range(1, E + 1))
    rank = zipf_permutation(seed, layer, E)  # rank[e] in 0..E-1
    b = np.array([-s * math.log(int(rank[e]) + 1) - math.log(H) for e in range(E)], dtype=np.float64)
    return b.astype(np.float32)


# ----------------------------------------------------------------------------
# workloads


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    d: int
    f: int
    E: int
    k: int
    T: int
    layers: int
    zipf: bool
    seed: int
    chunk: int = 8192
    bits: int = 2  # code width: 2 (Q2) or 4 (Q4)

    def desc(self) -> str:
        return (f"d={self.d} f={self.f} E={self.E} k={self.k} T={self.T} layers={self.layers} "
                f"routing={'zipf1.1' if self.zipf else 'uniform'} seed={self.seed} bits={self.bits}")


WORKLOADS = {
    "tiny": Workload("tiny", 256, 128, 16, 4, 8, 1, False, 0),
    "decode": Workload("decode", 2048, 768, 512, 10, 1, 1, False, 1),
    "verify4": Workload("verify4", 2048, 768, 512, 10, 4, 48, True, 2),
    "verify16": Workload("verify16", 2048, 768, 512, 10, 16, 48, True, 2),
    # 1 + 5 tokens: a step that verifies the 5 tokens the suffix drafter drafts at once
    # ("Strata：把 125B 大模型塞进 12GB 显卡…", 再快一截：先猜再验的投机解码)
    "verify6": Workload("verify6", 2048, 768, 512, 10, 6, 48, True, 2),
    "prefill": Workload("prefill", 2048, 768, 512, 10, 8192, 1, True, 3),
    "prefill_stack": Workload("prefill_stack", 2048, 768, 512, 10, 32768, 48, True, 4),
    # the Coder variant of the model keeps 256 of the 512 experts per layer
    # ("Strata — 8~12GB 显存跑 125B 大模型的本地推理引擎", §5 models table)
    "coder_decode": Workload("coder_decode", 2048, 768, 256, 10, 1, 1, False, 5),
    # the 4-bit block format (a wider level of the pages' quality ladder,
    # "Strata：把 125B 大模型塞进 12GB 显卡…", 能跑多快 table)
    "decode_q4": Workload("decode_q4", 2048, 768, 512, 10, 1, 1, False, 6, bits=4),
    "verify4_q4": Workload("verify4_q4", 2048, 768, 512, 10, 4, 1, True, 6, bits=4),
    "prefill_q4": Workload("prefill_q4", 2048, 768, 512, 10, 8192, 1, True, 6, bits=4),
}


# ----------------------------------------------------------------------------
# KV-cache rows for the 4-bit rotated codec


@dataclasses.dataclass(frozen=True)
class KvWorkload:
    """One attention layer's K and V cache: tokens x kv_heads x 2 rows of D."""
    name: str
    tokens: int
    kv_heads: int
    D: int
    seed: int

    @property
    def rows(self) -> int:
        return self.tokens * self.kv_heads * 2

    def desc(self) -> str:
        return (f"tokens={self.tokens} kv_heads={self.kv_heads} head_dim={self.D} rows={self.rows} "
                f"outlier_channels=4x16 seed={self.seed}")


# a 128K-token context ("Strata：把 125B 大模型塞进 12GB 显卡…", 长上下文: the 4-bit
# cache is quoted at 128K); head_dim 128 and 4 KV heads are assumed shapes
KV_WORKLOADS = {
    "kv4_128k": KvWorkload("kv4_128k", 131072, 4, 128, 7),
}

KV_OUTLIERS = 4  # channels per head_dim scaled by 16 (an exact power of two)


def kv_outlier_channels(seed: int, D: int) -> np.ndarray:
    """The fixed channels (same in every row) that carry outliers."""
    w = words(stream_key(seed, TAG_KV_OUTLIERS), 0, 64)
    out = []
    for v in w:
        c = int(v % np.uint64(D))
        if c not in out:
            out.append(c)
        if len(out) == KV_OUTLIERS:
            break
    return np.array(sorted(out), dtype=np.int64)


def gen_kv_rows(seed: int, rows: int, D: int, row0: int = 0) -> np.ndarray:
    """Cached key/value rows, uint16 bf16 bits [rows, D]: bf16(z), z ~ N(0,1),
    times 16 in the outlier channels (exact in bf16), rows row0.."""
    z = f32_to_bf16_bits(normals(stream_key(seed, TAG_KV), rows * D, start=row0 * D)).reshape(rows, D)
    ch = kv_outlier_channels(seed, D)
    z[:, ch] = f32_to_bf16_bits(bf16_bits_to_f32(z[:, ch]) * np.float32(16.0))
    return z


def router_bias(w: Workload, layer: int):
    return gen_zipf_bias(w.seed, layer, w.E) if w.zipf else None
