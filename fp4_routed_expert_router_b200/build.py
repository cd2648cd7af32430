"""Build the in-tree CUDA libraries for sm_100a with nvcc.

    python -m fp4_routed_expert_router_b200.build [--force]

Produces lib/libmoe_fp4.so (the compute path, C ABI of include/moe_fp4.h) and
lib/libmoe_synth.so (device-side synthetic-input generator).  nvcc
cross-compiles without a GPU.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIBDIR = os.path.join(PKG, "lib")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-shared", "-Xptxas", "-v"]

TARGETS = {
    "libmoe_fp4.so": ("moe_fp4_api.cu", []),
    "libmoe_synth.so": ("synth_fill.cu", []),
}


def _deps() -> list[str]:
    return glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(ROOT, "include", "*.h"))


def build(force: bool = False, verbose: bool = False) -> dict:
    os.makedirs(LIBDIR, exist_ok=True)
    newest = max(os.path.getmtime(p) for p in _deps())
    out = {}
    for lib, (src, extra) in TARGETS.items():
        dst = os.path.join(LIBDIR, lib)
        out[lib] = dst
        if not force and os.path.exists(dst) and os.path.getmtime(dst) >= newest:
            continue
        cmd = [NVCC, *ARCH, *FLAGS, os.path.join(CSRC, src), "-o", dst, *extra]
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            sys.stderr.write(res.stdout + res.stderr)
            raise RuntimeError(f"nvcc failed for {lib}")
        if verbose:
            sys.stderr.write(res.stderr)
    return out


if __name__ == "__main__":
    for k, v in build(force="--force" in sys.argv, verbose="-v" in sys.argv).items():
        print(k, v)
