"""Python binding of libsgl_moe.so, the B200 (sm_100a) sparse-MoE layer library.

Argument marshalling only: every stage runs in the library's CUDA kernels.
The names mirror the C-ABI in include/moe.h (moe_route, moe_permute,
moe_grouped_swiglu, moe_combine, moe_layer_forward). Tensors are torch CUDA
tensors (torch provides device memory and streams); bf16 tensors may be
torch.bfloat16 or int16/uint16 views of the same bytes.

There is no fallback: if the shared library is missing or the device is not
an sm_100 GPU, calls raise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsgl_moe.so")

MOE_W_BF16 = 0
MOE_W_MXFP4 = 1
MOE_W_MXFP4_A8 = 2
MOE_W_MXFP4_A8P = 3  # MOE_W_MXFP4_A8 with scales prepared by moe_prepare_weights
MOE_N_STAGE_EVENTS = 6
STATUS = {0: "MOE_OK", -1: "MOE_ERR_CFG", -2: "MOE_ERR_NULL", -3: "MOE_ERR_ALIGN",
          -4: "MOE_ERR_WORKSPACE", -5: "MOE_ERR_CUDA", -6: "MOE_ERR_DEVICE",
          -7: "MOE_ERR_UNSUPPORTED"}
DEVERR = {0: "none", 1: "expert id out of range", 2: "pipeline wait timed out",
          3: "work item out of range"}

C_FUNCTIONS = ("moe_workspace_size", "moe_route", "moe_permute", "moe_permute_static", "moe_route_stats",
               "moe_grouped_swiglu", "moe_prepare_weights",
               "moe_combine", "moe_layer_forward", "moe_read_error", "moe_status_string",
               "moe_version")


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


class moe_cfg(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int32), ("E", ctypes.c_int32), ("n_group", ctypes.c_int32),
                ("topk_group", ctypes.c_int32), ("K", ctypes.c_int32), ("I", ctypes.c_int32),
                ("I_shared", ctypes.c_int32), ("scale", ctypes.c_float),
                ("renorm", ctypes.c_int32), ("limit_routed", ctypes.c_float),
                ("limit_shared", ctypes.c_float), ("wfmt", ctypes.c_int32)]


class moe_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("Wg", "Wu", "Wd", "Wg_scale", "Wu_scale", "Wd_scale", "Wg_s", "Wu_s", "Wd_s")]


_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """Load libsgl_moe.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m sigmoid_group_limited_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    cp = ctypes.POINTER(moe_cfg)
    wp = ctypes.POINTER(moe_weights)
    L.moe_workspace_size.argtypes = [cp, i32]
    L.moe_workspace_size.restype = sz
    L.moe_route.argtypes = [cp, i32, vp, vp, vp, vp, vp, vp, sz, vp]
    L.moe_permute.argtypes = [cp, i32, vp, vp, vp, vp, vp, vp, sz, vp]
    L.moe_permute_static.argtypes = [cp, i32, vp, vp, vp, vp, vp, vp]
    L.moe_grouped_swiglu.argtypes = [cp, i32, vp, vp, vp, vp, wp, vp, vp, sz, vp]
    L.moe_combine.argtypes = [cp, i32, vp, i32, vp, vp]
    L.moe_layer_forward.argtypes = [cp, i32, vp, vp, vp, wp, vp, vp, vp, vp, vp, sz, vp, vp]
    L.moe_route_stats.argtypes = [cp, vp, vp, vp]
    L.moe_prepare_weights.argtypes = [cp, wp, vp, vp, vp, vp]
    L.moe_read_error.argtypes = [cp, i32, vp, sz, vp, ctypes.POINTER(i32)]
    L.moe_status_string.argtypes = [i32]
    L.moe_status_string.restype = ctypes.c_char_p
    L.moe_version.restype = ctypes.c_char_p
    for f in ("moe_route", "moe_permute", "moe_permute_static", "moe_route_stats", "moe_grouped_swiglu",
              "moe_combine", "moe_prepare_weights",
              "moe_layer_forward", "moe_read_error"):
        getattr(L, f).restype = i32
    _lib = L
    return L


def make_cfg(c) -> moe_cfg:
    """C struct from any object with the moe_cfg field names."""
    return moe_cfg(int(c.H), int(c.E), int(c.n_group), int(c.topk_group), int(c.K), int(c.I),
                   int(c.I_shared), float(c.scale), int(bool(c.renorm)), float(c.limit_routed),
                   float(c.limit_shared), int(c.wfmt))


def _p(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(st: int, where: str):
    if st != 0:
        raise MoEError(st, where)


def make_weights(Wg, Wu, Wd, Wg_s=None, Wu_s=None, Wd_s=None, Wg_scale=None, Wu_scale=None,
                 Wd_scale=None) -> moe_weights:
    return moe_weights(_p(Wg), _p(Wu), _p(Wd), _p(Wg_scale), _p(Wu_scale), _p(Wd_scale),
                       _p(Wg_s), _p(Wu_s), _p(Wd_s))


def workspace_size(cfg, T: int) -> int:
    c = make_cfg(cfg)
    n = lib().moe_workspace_size(ctypes.byref(c), int(T))
    if n == 0:
        raise MoEError(-1, "moe_workspace_size")
    return int(n)


def alloc_workspace(cfg, T: int, device=None) -> torch.Tensor:
    return torch.empty(workspace_size(cfg, T), dtype=torch.uint8, device=device or "cuda")


def moe_route(cfg, x, Wr, bias, idx, w, ws, stream=None):
    c = make_cfg(cfg)
    _check(lib().moe_route(ctypes.byref(c), x.shape[0], _p(x), _p(Wr), _p(bias), _p(idx), _p(w),
                           _p(ws), ws.numel(), _stream(stream)), "moe_route")


def moe_permute(cfg, T, idx, counts, offsets, perm, inv_perm, ws, stream=None):
    c = make_cfg(cfg)
    _check(lib().moe_permute(ctypes.byref(c), int(T), _p(idx), _p(counts), _p(offsets), _p(perm),
                             _p(inv_perm), _p(ws), ws.numel(), _stream(stream)), "moe_permute")


def moe_permute_static(cfg, T, idx, counts, offsets, perm, inv_perm, stream=None):
    """moe_permute without a workspace (scratch in a fixed array inside the
    library; T*K <= 65536). For callers that cannot allocate device memory."""
    c = make_cfg(cfg)
    _check(lib().moe_permute_static(ctypes.byref(c), int(T), _p(idx), _p(counts), _p(offsets),
                                    _p(perm), _p(inv_perm), _stream(stream)), "moe_permute_static")


MOE_N_ROUTE_STATS = 7
ROUTE_STATS_NAMES = ("entropy_bits", "entropy_normalized", "load_max", "load_mean", "max_over_mean",
                     "idle_experts", "slots")


def moe_route_stats(cfg, counts, stats, stream=None):
    """Routing statistics from expert counts into `stats` (float64 [7], device);
    see ROUTE_STATS_NAMES for the entries."""
    c = make_cfg(cfg)
    _check(lib().moe_route_stats(ctypes.byref(c), _p(counts), _p(stats), _stream(stream)),
           "moe_route_stats")


def moe_prepare_weights(cfg, weights: moe_weights, Wg_sf, Wu_sf, Wd_sf, stream=None):
    """Scale atoms of every expert for MOE_W_MXFP4_A8P (uint8 tensors shaped
    like the scale arrays they replace)."""
    _check(lib().moe_prepare_weights(ctypes.byref(make_cfg(cfg)), ctypes.byref(weights), _p(Wg_sf),
                                     _p(Wu_sf), _p(Wd_sf), _stream(stream)), "moe_prepare_weights")


def moe_grouped_swiglu(cfg, T, x, perm, offsets, w, weights: moe_weights, y_slot, ws, stream=None):
    c = make_cfg(cfg)
    _check(lib().moe_grouped_swiglu(ctypes.byref(c), int(T), _p(x), _p(perm), _p(offsets), _p(w),
                                    ctypes.byref(weights), _p(y_slot), _p(ws), ws.numel(),
                                    _stream(stream)), "moe_grouped_swiglu")


def moe_combine(cfg, T, y_slot, with_shared: bool, y, stream=None):
    c = make_cfg(cfg)
    _check(lib().moe_combine(ctypes.byref(c), int(T), _p(y_slot), int(bool(with_shared)), _p(y),
                             _stream(stream)), "moe_combine")


def moe_layer_forward(cfg, x, Wr, bias, weights: moe_weights, y, ws, idx_out=None, w_out=None,
                      counts_out=None, stream=None,
                      stage_events: Optional[Sequence[torch.cuda.Event]] = None):
    c = make_cfg(cfg)
    ev = None
    if stage_events is not None:
        if len(stage_events) != MOE_N_STAGE_EVENTS:
            raise ValueError(f"need {MOE_N_STAGE_EVENTS} events")
        for e in stage_events:          # torch creates CUDA events lazily, on first record
            if e.cuda_event == 0:
                e.record()
        ev = (ctypes.c_void_p * MOE_N_STAGE_EVENTS)(*[e.cuda_event for e in stage_events])
    _check(lib().moe_layer_forward(ctypes.byref(c), x.shape[0], _p(x), _p(Wr), _p(bias),
                                   ctypes.byref(weights), _p(y), _p(idx_out), _p(w_out),
                                   _p(counts_out), _p(ws), ws.numel(), _stream(stream), ev),
           "moe_layer_forward")


def moe_read_error(cfg, T, ws, stream=None) -> int:
    c = make_cfg(cfg)
    code = ctypes.c_int32(0)
    _check(lib().moe_read_error(ctypes.byref(c), int(T), _p(ws), ws.numel(), _stream(stream),
                                ctypes.byref(code)), "moe_read_error")
    return int(code.value)


def version() -> str:
    return lib().moe_version().decode()
