"""Dense tensor-core instruction throughput on this GPU (libsgl_peak.so).

measure(kind, n, chains) launches one CTA per SM that issues back-to-back
tcgen05.mma instructions of one shape (M = 128, N = n) from shared memory,
and times the launch with CUDA events. kinds: "bf16" (kind::f16, K = 16),
"e2m1xe4m3" (kind::mxf8f6f4 block-scaled, K = 32), "e2m1xe2m1" (kind::mxf4
block-scaled, K = 64). The result is an instruction ceiling, not a GEMM
measurement: its ratio to the bf16 kind scales a measured bf16 GEMM peak to
the other kinds (`peaks()`).
"""
from __future__ import annotations

import ctypes
import os
import statistics

import torch

_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_DIR, "libsgl_peak.so")
KINDS = {"bf16": (0, 16), "e2m1xe4m3": (1, 32), "e2m1xe2m1": (2, 64)}
_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m sigmoid_group_limited_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        L.sgl_mma_peak.argtypes = [ctypes.c_int] * 6 + [ctypes.c_void_p, ctypes.c_void_p]
        L.sgl_mma_peak.restype = ctypes.c_int
        _lib = L
    return _lib


PATTERNS = {"same": 0, "two_tiles": 1, "ksplit": 2}


def measure(kind: str, n: int = 256, chains: int = 1, iters: int = 40000, repeats: int = 5,
            device=None, pattern: str = "same", commit: bool = False) -> dict:
    """Median over `repeats` launches of one probe configuration. pattern:
    "same" (every chain reads the same operands), "two_tiles" (two 128-row A
    tiles against one B tile: gate and up of a token tile), "ksplit" (the K
    step rotates per MMA); commit: a commit after every 8 MMAs."""
    code, K = KINDS[kind]
    dev = torch.device(device or "cuda")
    ctas = torch.cuda.get_device_properties(dev).multi_processor_count
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    times = []
    for r in range(repeats + 1):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        mode = PATTERNS[pattern] | (16 if commit else 0)
        rc = lib().sgl_mma_peak(code, n, chains, iters, ctas, mode, ctypes.c_void_p(status.data_ptr()),
                                ctypes.c_void_p(stream.cuda_stream))
        e1.record(stream)
        if rc != 0:
            raise RuntimeError(f"sgl_mma_peak({kind}, n={n}, chains={chains}) failed: cuda error {rc}")
        torch.cuda.synchronize(dev)
        if r > 0:                                   # the first launch is a warm-up
            times.append(e0.elapsed_time(e1) * 1e-3)
    if int(status.item()) != 0:
        raise RuntimeError("sgl_mma_peak: an MMA wait timed out")
    t = statistics.median(times)
    mmas = ctas * iters * chains
    flops = 2.0 * 128 * n * K * mmas
    return {"kind": kind, "M": 128, "N": n, "K": K, "chains": chains, "ctas": ctas, "pattern": pattern,
            "commit": commit,
            "tflops": flops / t / 1e12, "ns_per_mma": t / (iters * chains) * 1e9, "seconds": t}


# shapes every kind can run: the block-scaled kinds keep TMEM columns 384-399
# for their scale atoms, so at most 384 accumulator columns
COMMON_SHAPES = ((256, 1), (128, 2), (128, 3), (192, 2))


def peaks(device=None) -> dict:
    """Best instruction throughput per kind over the same shapes for every kind
    (COMMON_SHAPES), so that the ratios between kinds compare like with like."""
    out = {}
    for kind in KINDS:
        best = max((measure(kind, n, c, device=device) for n, c in COMMON_SHAPES), key=lambda r: r["tflops"])
        out[kind] = best
    return out
