"""Build the sm_100a shared library ``libstrata_moe.so`` in-tree with nvcc."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
OUT = os.path.join(HERE, "libstrata_moe.so")
# the same sources with every data-derived index bounds-checked into the status word
OUT_CHECKED = os.path.join(HERE, "libstrata_moe_checked.so")
SOURCES = ["strata_moe.cu", "route.cu", "decode_fused.cu", "prefill_gemm.cu", "misc.cu", "route_noalloc.cu", "router_gemm.cu", "kv_codec.cu"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-lineinfo",
         "-Xcompiler", "-fPIC", "-shared", "--expt-relaxed-constexpr"]


def needs_build(out: str = OUT) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    inc = os.path.join(HERE, "..", "include")
    deps += [os.path.join(inc, f) for f in os.listdir(inc) if f.endswith(".h")]
    return any(os.path.getmtime(p) > t for p in deps)


def build(verbose: bool = False, force: bool = False, checked: bool = False) -> str:
    out = OUT_CHECKED if checked else OUT
    if not force and not needs_build(out):
        return out
    cmd = [NVCC, *FLAGS, *(["-DSTRATA_CHECKED"] if checked else []), *(["-Xptxas", "-v"] if verbose else []),
           "-o", out, *[os.path.join(CSRC, s) for s in SOURCES], "-lcudart"]
    subprocess.run(cmd, check=True)
    return out


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv, force=True))
    print(build(verbose="-v" in sys.argv, force=True, checked=True))
