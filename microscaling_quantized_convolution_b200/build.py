"""Build libmqv.so (the C-ABI library) in-tree with nvcc for sm_100a."""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libmqv.so")
SOURCES = ["mqv_api.cu"]
HEADERS = ["mqv_ptx.cuh", "mqv_quantize.cuh", "mqv_conv_common.cuh", "mqv_conv_kernels.cuh", "mqv_conv_halo.cuh", "mqv_conv_nvf4.cuh", "mqv_conv_wgk.cuh", "mqv_conv_narrow.cuh", "mqv_naive.cuh", "mqv_replay.cuh", "mqv_depthwise.cuh", "mqv_depthwise_core.h"]


def nvcc_cmd(out=LIB, extra=()):
    nvcc = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
    return [nvcc, "-std=c++17", "-O3", "-lineinfo",
            "-gencode", "arch=compute_100a,code=sm_100a",
            "-Xcompiler", "-fPIC,-O3", "-shared",
            "-I", os.path.join(ROOT, "include"),
            *extra,
            *[os.path.join(CSRC, s) for s in SOURCES],
            "-o", out]


def _stale(out):
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(ROOT, "include", "mqv.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    if force or _stale(LIB):
        cmd = nvcc_cmd()
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
            print(" ".join(cmd), file=sys.stderr)
        subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
