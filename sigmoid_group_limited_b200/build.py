"""Build libsgl_moe.so (the CUDA kernels + C-ABI) in-tree for sm_100a.

Usage: python -m sigmoid_group_limited_b200.build [--verbose]
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libsgl_moe.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(glob.glob(os.path.join(PKG, "csrc", "*.cu")))


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = sources() + glob.glob(os.path.join(PKG, "csrc", "*.cuh")) + \
        glob.glob(os.path.join(PKG, "csrc", "*.h")) + glob.glob(os.path.join(ROOT, "include", "*.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def build(verbose: bool = False, force: bool = False) -> str:
    if not force and not needs_build():
        return LIB
    cmd = [nvcc(), "-O3", "-std=c++17", *ARCH, "-lineinfo", "-Xcompiler", "-fPIC", "-shared",
           "-Xcompiler", "-fvisibility=hidden", "-I", os.path.join(ROOT, "include"),
           "-o", LIB + ".tmp", *sources()]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd))
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed")
    if verbose:
        sys.stderr.write(r.stderr)
    os.replace(LIB + ".tmp", LIB)
    return LIB


PEAK_SRC = os.path.join(PKG, "peak", "mma_peak.cu")
PEAK_LIB = os.path.join(PKG, "peak", "libsgl_peak.so")


def build_peak(force: bool = False) -> str:
    """libsgl_peak.so: the tensor-core throughput probe (peak/mma_peak.cu)."""
    if not force and os.path.exists(PEAK_LIB) and os.path.getmtime(PEAK_LIB) > os.path.getmtime(PEAK_SRC):
        return PEAK_LIB
    cmd = [nvcc(), "-O3", "-std=c++17", *ARCH, "-lineinfo", "-Xcompiler", "-fPIC", "-shared",
           "-Xcompiler", "-fvisibility=hidden", "-o", PEAK_LIB + ".tmp", PEAK_SRC]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed (peak probe)")
    os.replace(PEAK_LIB + ".tmp", PEAK_LIB)
    return PEAK_LIB


if __name__ == "__main__":
    build(verbose="--verbose" in sys.argv, force=True)
    build_peak(force=True)
    print(LIB)
    print(PEAK_LIB)
