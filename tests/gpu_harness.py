"""Shared helpers of the GPU parity tests: seeded inputs (host or device
generator), packing through the library, calls through the C ABI, and the
comparisons against the CPU oracle (gap rule for indices, per-row relative
error for outputs)."""
from __future__ import annotations

import numpy as np

import oracle
import synth

TOL = 2e-3          # max over a token row of |y - y_ref| / max |y_ref|
GAP = 1e-4          # index comparisons need l_(k) - l_(k+1) > GAP (or an exact tie)


def torch_dev():
    import torch
    return torch.device("cuda:0")


def S():
    import bit_quantized_moe_warp_b200 as S
    return S


# ---------------------------------------------------------------- inputs


class HostLayer:
    """All inputs of one layer generated on the host (small shapes)."""

    def __init__(self, d, f, E, k, T, seed=0, layer=0, zipf=False, experts=None, W=None, x=None, bias=None,
                 bits=2):
        self.d, self.f, self.E, self.k, self.T, self.bits = d, f, E, k, T, bits
        self.x = synth.gen_x_bf16(seed, T, d) if x is None else x
        self.W = synth.gen_router_w(seed, layer, E, d) if W is None else W
        self.bias = (synth.gen_zipf_bias(seed, layer, E) if zipf else None) if bias is None else bias
        self.experts = ([synth.gen_expert(seed, layer, e, d, f, bits) for e in range(E)]
                        if experts is None else experts)

    def blob(self, desc):
        eb = S().strata_moe_expert_bytes(desc)
        out = np.zeros(self.E * eb, np.uint8)
        for e, ex in enumerate(self.experts):
            S().strata_moe_pack_expert(desc, ex["gate_codes"], ex["gate_scales"], ex["up_codes"], ex["up_scales"],
                                       ex["down_codes"], ex["down_scales"], out[e * eb:(e + 1) * eb])
        return out

    def to_device(self, desc):
        import torch
        dev = torch_dev()
        xd = torch.from_numpy(np.ascontiguousarray(self.x).view(np.int16)).to(dev)
        Wd = torch.from_numpy(np.ascontiguousarray(self.W)).to(dev)
        bd = None if self.bias is None else torch.from_numpy(self.bias).to(dev)
        blob = torch.from_numpy(self.blob(desc)).to(dev)
        return xd, Wd, bd, blob

    def oracle(self):
        return oracle.moe_layer(self.x, self.W, self.bias, self.experts, self.k)


def device_blob(w: synth.Workload, layer: int, desc):
    """Packed blob of a full-size layer: device generator + library packer."""
    import synth.device as sd

    def pack(e, gc, gs, uc, us, dc, ds, dst):
        S().strata_moe_pack_expert_device(desc, gc, gs, uc, us, dc, ds, dst)

    return sd.layer_blob(w, layer, pack)


def expert_source(w: synth.Workload, layer: int):
    cache = {}

    def get(e):
        if e not in cache:
            cache[e] = synth.gen_expert(w.seed, layer, e, w.d, w.f, w.bits)
        return cache[e]

    return get


# ---------------------------------------------------------------- checks


def routing_check(logits_ref, k, idx_gpu, w_gpu=None, w_ref=None):
    """Gap rule. Returns (exempt token mask, list of mismatching tokens)."""
    T, E = logits_ref.shape
    lf = logits_ref.astype(np.float32)
    exempt = np.zeros(T, bool)
    bad = []
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-float(lf[t, e]), e))
        gap = np.inf if k == E else float(lf[t, order[k - 1]]) - float(lf[t, order[k]])
        if 0.0 < gap <= GAP:
            exempt[t] = True
            continue
        if sorted(order[:k]) != sorted(int(i) for i in idx_gpu[t]):
            bad.append(t)
            continue
        # slot order must match wherever adjacent gaps inside the top k+1 are large
        for j in range(k):
            g_next = np.inf if j + 1 >= E else float(lf[t, order[j]]) - float(lf[t, order[j + 1]])
            g_prev = np.inf if j == 0 else float(lf[t, order[j - 1]]) - float(lf[t, order[j]])
            if (g_next > GAP or g_next == 0.0) and (g_prev > GAP or g_prev == 0.0):
                if int(idx_gpu[t, j]) != order[j]:
                    bad.append(t)
                    break
    return exempt, bad


def lists_check(idx_ref, idx_gpu, exempt, E, off_gpu, tl_gpu, sl_gpu):
    """Per-expert lists must match the oracle's except for experts touched by
    an exempt token whose selection differs."""
    off_r, tl_r, sl_r = oracle.expert_lists(idx_ref, E)
    # slots: the slot of a pair is where its expert sits in the token's own
    # (GPU) rank order; that order was checked against the oracle's wherever
    # the adjacent logits are more than GAP apart (routing_check)
    for e in range(E):
        for p in range(off_gpu[e], off_gpu[e + 1]):
            assert int(idx_gpu[tl_gpu[p], sl_gpu[p]]) == e, f"pair {p}: slot does not point at expert {e}"
    skip = set()
    for t in np.nonzero(exempt)[0]:
        skip |= set(int(e) for e in idx_ref[t]) ^ set(int(e) for e in idx_gpu[t])
    if not skip:
        assert np.array_equal(off_gpu, off_r), "expert offsets differ"
        assert np.array_equal(tl_gpu, tl_r), "token lists differ"
        return
    for e in range(E):
        if e in skip:
            continue
        a = tl_gpu[off_gpu[e]:off_gpu[e + 1]]
        b = tl_r[off_r[e]:off_r[e + 1]]
        assert np.array_equal(a, b), f"token list of expert {e} differs"


def row_errors(y_gpu, y_ref):
    y_gpu = np.asarray(y_gpu, np.float64)
    den = np.max(np.abs(y_ref), axis=1)
    den[den == 0] = 1.0
    return np.max(np.abs(y_gpu - y_ref), axis=1) / den


WTOL = 1e-5         # renormalised routing weights (fp32 exp / sum against fp64)


def weights_check(idx_ref, w_ref, idx_gpu, w_gpu, exempt):
    """topk_w against the oracle's renormalised softmax weights, matched by
    expert (the slot order may differ inside near-ties), for every token whose
    selected set equals the oracle's; the weights sum to 1."""
    n = 0
    for t in range(idx_ref.shape[0]):
        ref = {int(e): float(v) for e, v in zip(idx_ref[t], w_ref[t])}
        got = {int(e): float(v) for e, v in zip(idx_gpu[t], w_gpu[t])}
        if set(ref) != set(got):
            assert exempt[t], f"token {t}: selected experts differ"
            continue
        for e, v in ref.items():
            assert abs(got[e] - v) <= WTOL, f"token {t} expert {e}: weight {got[e]} vs {v}"
        assert abs(sum(got.values()) - 1.0) <= 1e-5, f"token {t}: weights sum to {sum(got.values())}"
        n += 1
    assert n > 0
