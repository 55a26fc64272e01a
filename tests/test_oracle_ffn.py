"""Pins for the oracle's expert stages: bf16 rounding, SwiGLU with limit, the
shared expert, the weighted combine and the whole-layer closed form."""
import math
import struct

import numpy as np
import pytest
import torch

import oracle
import workloads


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


# ---------------------------------------------------------------- bf16

def test_bf16_rounding_matches_torch_and_ties_to_even():
    rng = np.random.default_rng(0)
    a = np.concatenate([rng.normal(size=5000) * 10.0 ** rng.integers(-30, 30, 5000),
                        [0.0, -0.0, 1.0, 65504.0, 3.0e38, 1e-40]]).astype(np.float32)
    ref = _bits(torch.from_numpy(a).to(torch.bfloat16))
    assert np.array_equal(oracle.f32_to_bf16_bits(a), ref)
    # exact halfway cases: 1 + 2^-8 -> 1.0 (even), 1 + 3*2^-8 -> 1 + 2^-6 (even)
    ties = np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8], np.float32)
    assert list(oracle.f32_to_bf16_bits(ties)) == [0x3F80, 0x3F82]
    assert oracle.bf16_bits_to_f64(np.array([0x3F80, 0xC000, 0x0000], np.uint16)).tolist() == [1.0, -2.0, 0.0]


# ---------------------------------------------------------------- one expert, brute force

def _py_bf16(v: float) -> float:
    """bf16 rounding (nearest even) written with struct, independent of the oracle."""
    (u,) = struct.unpack("<I", struct.pack("<f", v))
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    (r,) = struct.unpack("<f", struct.pack("<I", u << 16))
    return r


def _f32(v: float) -> float:
    return struct.unpack("<f", struct.pack("<f", v))[0]


def _py_swiglu(xrow, Wg, Wu, Wd, L):
    """Pure-Python SwiGLU: exact dot products (fsum), then the same rounding points."""
    I, H = Wg.shape
    h = []
    for i in range(I):
        g = _f32(math.fsum(xrow[k] * Wg[i, k] for k in range(H)))
        u = _f32(math.fsum(xrow[k] * Wu[i, k] for k in range(H)))
        if L > 0:
            g = min(max(g, -L), L)
            u = min(max(u, -L), L)
        a = _f32(g / (1.0 + math.exp(-g)) * u)
        h.append(_py_bf16(a))
    return [_f32(math.fsum(h[i] * Wd[n, i] for i in range(I))) for n in range(Wd.shape[0])], h


@pytest.mark.parametrize("L", [0.0, 0.05])
def test_swiglu_against_pure_python(L):
    g = torch.Generator().manual_seed(7)
    H, I = 48, 24
    x = torch.randn(5, H, generator=g).to(torch.bfloat16)
    Wg = (torch.randn(I, H, generator=g) / H ** 0.5).to(torch.bfloat16)
    Wu = (torch.randn(I, H, generator=g) / H ** 0.5).to(torch.bfloat16)
    Wd = (torch.randn(H, I, generator=g) / I ** 0.5).to(torch.bfloat16)
    f = oracle.bf16_bits_to_f64
    x64, g64, u64, d64 = f(_bits(x)), f(_bits(Wg)), f(_bits(Wu)), f(_bits(Wd))
    o, h = oracle.swiglu_expert(x64, g64, u64, d64, L)
    for r in range(5):
        o_ref, h_ref = _py_swiglu(x64[r].tolist(), g64, u64, d64, L)
        assert np.array_equal(oracle.bf16_bits_to_f64(h[r]), np.array(h_ref))
        assert np.array_equal(o[r], np.array(o_ref, np.float32))


def test_swiglu_against_torch_float64_dense():
    """Textbook dense SwiGLU in torch float64 (no clamp) agrees to rounding."""
    g = torch.Generator().manual_seed(8)
    H, I = 256, 64
    x = torch.randn(32, H, generator=g, dtype=torch.float64)
    Wg = torch.randn(I, H, generator=g, dtype=torch.float64) / 16
    Wu = torch.randn(I, H, generator=g, dtype=torch.float64) / 16
    Wd = torch.randn(H, I, generator=g, dtype=torch.float64) / 8
    ref = (torch.nn.functional.silu(x @ Wg.T) * (x @ Wu.T)) @ Wd.T
    o, _ = oracle.swiglu_expert(x.numpy(), Wg.numpy(), Wu.numpy(), Wd.numpy(), 0.0)
    err = np.abs(o - ref.numpy()).max() / np.sqrt((ref.numpy() ** 2).mean())
    assert err < 2e-2        # h is rounded to bf16 on the way, nothing else differs


def test_limit_infinite_equals_no_limit_and_tiny_limit_saturates():
    g = torch.Generator().manual_seed(9)
    H, I = 64, 32
    x = torch.randn(8, H, generator=g, dtype=torch.float64) * 3
    Wg = torch.randn(I, H, generator=g, dtype=torch.float64)
    Wu = torch.randn(I, H, generator=g, dtype=torch.float64)
    Wd = torch.randn(H, I, generator=g, dtype=torch.float64)
    a = [t.numpy() for t in (x, Wg, Wu, Wd)]
    o0, h0 = oracle.swiglu_expert(*a, limit=0.0)
    o1, h1 = oracle.swiglu_expert(*a, limit=1e30)
    assert np.array_equal(o0, o1) and np.array_equal(h0, h1)
    # every |g|, |u| is far above L = 1e-3, so h = silu(+-L) * (+-L)
    L = 1e-3
    _, hL = oracle.swiglu_expert(*a, limit=L)
    gs = np.sign(a[0] @ a[1].T)
    us = np.sign(a[0] @ a[2].T)
    Lf = float(np.float32(L))
    silu_p, silu_m = Lf / (1 + math.exp(-Lf)), -Lf / (1 + math.exp(Lf))
    expect = np.where(gs > 0, silu_p, silu_m) * us * Lf
    assert np.allclose(oracle.bf16_bits_to_f64(hL), expect, rtol=2 ** -8, atol=0)


# ---------------------------------------------------------------- whole layer

def _tiny(cfg=None, T=64, **kw):
    cfg = (cfg or workloads.CONFIGS["tiny"]).with_(**kw)
    d = workloads.generate(cfg, "cpu", T=T)
    b = {k: (_bits(v) if v.dtype == torch.bfloat16 else v.numpy()) for k, v in d.items()}
    return cfg, b


def test_identical_experts_closed_form():
    """All routed experts equal: y = bf16(2.5 * FFN(x) + FFN_shared(x)) for every
    token, whatever the routing (the weights of the chosen 8 sum to 2.5)."""
    cfg, b = _tiny()
    Wg = np.repeat(b["Wg"][:1], cfg.E, axis=0)
    Wu = np.repeat(b["Wu"][:1], cfg.E, axis=0)
    Wd = np.repeat(b["Wd"][:1], cfg.E, axis=0)
    out = oracle.layer_forward(cfg, b["x"], b["Wr"], b["bias"],
                               oracle.dense_expert_weights(Wg, Wu, Wd), b["Wg_s"], b["Wu_s"], b["Wd_s"])
    f = oracle.bf16_bits_to_f64
    x64 = f(b["x"])
    o, _ = oracle.swiglu_expert(x64, f(Wg[0]), f(Wu[0]), f(Wd[0]))
    osh, _ = oracle.swiglu_expert(x64, f(b["Wg_s"]), f(b["Wu_s"]), f(b["Wd_s"]))
    expect = 2.5 * o.astype(np.float64) + osh.astype(np.float64)
    y = f(out["y"])
    # bf16 output: one rounding of the result plus fp32 summation error
    assert np.all(np.abs(y - expect) <= 2 ** -8 * np.abs(expect) + 1e-6)


def test_shared_expert_is_unscaled_and_always_on():
    """Routed experts with Wd = 0 contribute nothing: y = bf16(shared(x))."""
    cfg, b = _tiny()
    Wd0 = np.zeros_like(b["Wd"])
    out = oracle.layer_forward(cfg, b["x"], b["Wr"], b["bias"],
                               oracle.dense_expert_weights(b["Wg"], b["Wu"], Wd0),
                               b["Wg_s"], b["Wu_s"], b["Wd_s"])
    f = oracle.bf16_bits_to_f64
    osh, _ = oracle.swiglu_expert(f(b["x"]), f(b["Wg_s"]), f(b["Wu_s"]), f(b["Wd_s"]))
    assert np.array_equal(out["y"], oracle.f32_to_bf16_bits(osh))


def test_single_expert_slot_brute_force():
    """Token output from explicit per-slot loops (pure Python sums) equals the oracle's."""
    cfg, b = _tiny(T=4)
    out = oracle.layer_forward(cfg, b["x"], b["Wr"], b["bias"],
                               oracle.dense_expert_weights(b["Wg"], b["Wu"], b["Wd"]),
                               b["Wg_s"], b["Wu_s"], b["Wd_s"])
    f = oracle.bf16_bits_to_f64
    t = 2
    xr = f(b["x"][t]).tolist()
    acc = 0.0
    for k in range(cfg.K):
        e = int(out["idx"][t, k])
        o, _ = _py_swiglu(xr, f(b["Wg"][e]), f(b["Wu"][e]), f(b["Wd"][e]), 0.0)
        wk = float(out["w"][t, k])
        acc_vec = [_f32(wk * v) for v in o]
        acc = acc_vec if k == 0 else [_f32(a + c) for a, c in zip(acc, acc_vec)]
    osh, _ = _py_swiglu(xr, f(b["Wg_s"]), f(b["Wu_s"]), f(b["Wd_s"]), 0.0)
    y = [_py_bf16(_f32(a + c)) for a, c in zip(acc, osh)]
    assert np.array_equal(f(out["y"][t]), np.array(y))


def test_sampled_tokens_equal_full_run():
    cfg, b = _tiny()
    ew = oracle.dense_expert_weights(b["Wg"], b["Wu"], b["Wd"])
    full = oracle.layer_forward(cfg, b["x"], b["Wr"], b["bias"], ew, b["Wg_s"], b["Wu_s"], b["Wd_s"])
    some = oracle.layer_forward(cfg, b["x"], b["Wr"], b["bias"], ew, b["Wg_s"], b["Wu_s"], b["Wd_s"],
                                tokens=[63, 0, 17])
    assert np.array_equal(some["y"], full["y"][[63, 0, 17]])
