"""Shared helpers for the GPU parity tests: run the CUDA path through the
C-ABI binding and the oracle on host copies of the same seeded inputs."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import sigmoid_group_limited_b200 as sgl

NEAR_TIE = 1e-6        # routing margin below which a token is listed, not compared
W_TOL = 1e-6           # combine weights, absolute
Y_TOL_BF16 = 2e-2      # layer output, max |err| <= tol * RMS(y_oracle)


def bits(t: torch.Tensor) -> np.ndarray:
    """Host uint16 copy of a bf16 tensor's bytes."""
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def host_inputs(d):
    return dict(x=bits(d["x"]), Wr=d["Wr"].cpu().numpy(), bias=d["bias"].cpu().numpy(),
                Wg_s=bits(d["Wg_s"]), Wu_s=bits(d["Wu_s"]), Wd_s=bits(d["Wd_s"]))


class DeviceExperts:
    """Oracle weight accessor that copies one expert's bf16 weights from the
    device tensors on demand (the bytes the kernels read)."""

    def __init__(self, d):
        self.d = d

    def __call__(self, e: int):
        f = oracle.bf16_bits_to_f64
        return f(bits(self.d["Wg"][e])), f(bits(self.d["Wu"][e])), f(bits(self.d["Wd"][e]))


class DeviceExpertsMXFP4:
    """Oracle accessor for MXFP4 routed weights: host copies of one expert's
    packed codes and scales, dequantised by the oracle."""

    def __init__(self, d):
        self.d = d

    def __call__(self, e: int):
        d = self.d
        q = lambda k: d[k][e].cpu().numpy()  # noqa: E731
        return (oracle.mxfp4_dequantize(q("Wg_q"), q("Wg_sc")),
                oracle.mxfp4_dequantize(q("Wu_q"), q("Wu_sc")),
                oracle.mxfp4_dequantize(q("Wd_q"), q("Wd_sc")))


def experts_of(d):
    return DeviceExpertsMXFP4(d) if "Wg_q" in d else DeviceExperts(d)


def weights(d):
    if "Wg_q" in d:
        return sgl.make_weights(d["Wg_q"], d["Wu_q"], d["Wd_q"], d.get("Wg_s"), d.get("Wu_s"),
                                d.get("Wd_s"), d["Wg_sc"], d["Wu_sc"], d["Wd_sc"])
    return sgl.make_weights(d["Wg"], d["Wu"], d["Wd"], d.get("Wg_s"), d.get("Wu_s"), d.get("Wd_s"))


def run_layer(cfg, d, stream=None):
    T = d["x"].shape[0]
    dev = d["x"].device
    ws = sgl.alloc_workspace(cfg, T, dev)
    y = torch.empty(T, cfg.H, dtype=torch.bfloat16, device=dev)
    idx = torch.empty(T, cfg.K, dtype=torch.int32, device=dev)
    w = torch.empty(T, cfg.K, dtype=torch.float32, device=dev)
    counts = torch.empty(cfg.E, dtype=torch.int32, device=dev)
    sgl.moe_layer_forward(cfg, d["x"], d["Wr"], d["bias"], weights(d), y, ws, idx, w, counts,
                          stream=stream)
    torch.cuda.synchronize()
    assert sgl.moe_read_error(cfg, T, ws) == 0
    return dict(y=y, idx=idx, w=w, counts=counts, ws=ws)


def run_staged(cfg, d, idx: torch.Tensor, w: torch.Tensor):
    """Permute -> grouped SwiGLU (+ shared) -> combine, with given routing."""
    T = d["x"].shape[0]
    dev = d["x"].device
    ws = sgl.alloc_workspace(cfg, T, dev)
    counts = torch.empty(cfg.E, dtype=torch.int32, device=dev)
    offsets = torch.empty(cfg.E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(T * cfg.K, dtype=torch.int32, device=dev)
    inv = torch.empty(T * cfg.K, dtype=torch.int32, device=dev)
    y_slot = torch.zeros(T * cfg.K + T, cfg.H, dtype=torch.float32, device=dev)
    y = torch.empty(T, cfg.H, dtype=torch.bfloat16, device=dev)
    sgl.moe_permute(cfg, T, idx, counts, offsets, perm, inv, ws)
    sgl.moe_grouped_swiglu(cfg, T, d["x"], perm, offsets, w, weights(d), y_slot, ws)
    sgl.moe_combine(cfg, T, y_slot, cfg.I_shared > 0, y)
    torch.cuda.synchronize()
    assert sgl.moe_read_error(cfg, T, ws) == 0
    return dict(y=y, y_slot=y_slot, counts=counts, offsets=offsets, perm=perm, inv=inv)


def near_tie_tokens(ref) -> np.ndarray:
    return np.nonzero((ref["gmargin"] < NEAR_TIE) | (ref["emargin"] < NEAR_TIE))[0]


def check_routing(ref, idx_gpu: np.ndarray, w_gpu: np.ndarray):
    """idx bit-exact and |w - w_ref| <= 1e-6 on every token whose oracle
    margins are >= 1e-6; returns the listed near-tie tokens."""
    near = near_tie_tokens(ref)
    mask = np.ones(ref["idx"].shape[0], dtype=bool)
    mask[near] = False
    bad = np.nonzero((idx_gpu != ref["idx"]).any(axis=1) & mask)[0]
    assert bad.size == 0, f"idx mismatch on tokens {bad[:10]} (of {bad.size})"
    werr = np.abs(w_gpu[mask].astype(np.float64) - ref["w"][mask].astype(np.float64))
    assert werr.size == 0 or werr.max() <= W_TOL, f"max |w err| {werr.max():.3g}"
    return near


def check_y(y_gpu_bits: np.ndarray, y_ref_f32: np.ndarray, y_ref_bits: np.ndarray = None,
            tol: float = Y_TOL_BF16):
    """Layer output bar: max |y_gpu - y_oracle| <= tol * RMS(y_oracle), measured
    against the oracle's fp32 result before its final bf16 rounding.

    Why not against the oracle's bf16 result: one bf16 ulp is 2^-5 * RMS for
    |y| in [4, 8) * RMS, above the tolerance, and two correct results that
    straddle a rounding boundary differ by one ulp. The GPU's own rounding
    costs at most half an ulp (<= 2^-6 * RMS below 8 * RMS), which leaves
    room for the other legitimate differences (fp32 accumulation order, and
    h values whose bf16 rounding flips because of it)."""
    g = oracle.bf16_bits_to_f64(y_gpu_bits)
    r = np.asarray(y_ref_f32, dtype=np.float64)
    rms = np.sqrt(np.mean(r * r))
    assert np.all(np.isfinite(g)), "non-finite output"
    err = np.abs(g - r).max()
    assert err <= tol * rms, f"max |y err| {err:.4g} > {tol} * rms {rms:.4g}"
    return err / rms
