"""Seeded synthetic inputs for one sparse-MoE FFN layer.

This module only draws numbers: it holds shapes, seeds and distributions, and
none of the layer's arithmetic. The same tensors feed the CUDA path (through
the C-ABI) and the CPU oracle (as host copies of the very same bytes).

Shapes and constants follow the Ling-3.0-flash-VL MoE description
(lqnn.cn "Ling-3.0-flash-VL MoE routing" page, sections 2-4: hidden_size 2560,
moe_intermediate_size 768, 512 routed experts in n_group=8 groups keeping
topk_group=4, num_experts_per_tok=8, routed_scaling_factor 2.5,
norm_topk_prob, one always-on shared expert, SwiGLU limits) and the
lpnh.cn spec table (MXFP4 routed-expert weights).

Distributions: "N(0, v)" means variance v. Weights are N(0, 1/fan_in), the
router matrix N(0, 1/H) so that logits are about N(0, 1), x ~ N(0, 1),
the selection bias N(0, 0.1). Every tensor has its own stream: sub-seed
seed*16 + k (k = 0..8 for x, Wr, bias, Wg, Wu, Wd, Wg_s, Wu_s, Wd_s).
Values are drawn in fp32 by torch's seeded generator on the requested device
and cast to bf16 with round-to-nearest-even where the layer stores bf16.
"""
from __future__ import annotations

import dataclasses
import math
import os
from typing import Dict, Optional

import torch

MOE_W_BF16 = 0
MOE_W_MXFP4 = 1
MOE_W_MXFP4_A8 = 2   # MXFP4 routed weights, routed-expert activations in MXFP8
MOE_W_MXFP4_A8P = 3  # the same, scales prepared once into the tensor cores' atom layout


@dataclasses.dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int                  # tokens
    H: int                  # hidden_size
    E: int                  # routed experts
    n_group: int            # expert groups
    topk_group: int         # groups kept per token
    K: int                  # experts per token (num_experts_per_tok)
    I: int                  # moe_intermediate_size (routed)
    I_shared: int           # shared expert intermediate size
    scale: float = 2.5      # routed_scaling_factor
    renorm: bool = True     # norm_topk_prob
    limit_routed: float = 0.0   # SwiGLU limit on routed experts, <= 0 means off
    limit_shared: float = 0.0   # SwiGLU limit on the shared expert, <= 0 means off
    wfmt: int = MOE_W_BF16
    seed: int = 0
    bias_kind: str = "normal"   # "normal" (N(0, bias_var)), "zero", "zipf"
    bias_var: float = 0.1
    zipf_s: float = 1.1         # target popularity law p(r) ~ r^-zipf_s inside each group
    zipf_beta: float = 0.1      # fixed-formula bias scale (groups without a calibrated table)

    def with_(self, **kw) -> "MoEConfig":
        return dataclasses.replace(self, **kw)

    @property
    def experts_per_group(self) -> int:
        return self.E // self.n_group


_FULL = dict(H=2560, E=512, n_group=8, topk_group=4, K=8, I=768, I_shared=768)

CONFIGS: Dict[str, MoEConfig] = {
    # small case: every stage on a few tiles plus ragged tails
    "tiny": MoEConfig("tiny", T=64, H=256, E=32, n_group=4, topk_group=2, K=4,
                      I=64, I_shared=64, seed=0),
    # full-size layer, decode batch
    "decode": MoEConfig("decode", T=32, seed=1, **_FULL),
    # full-size layer, prefill batch
    "prefill": MoEConfig("prefill", T=4096, seed=2, **_FULL),
    # companion of the prefill batch with zero bias: near-uniform loads
    "prefill_bias0": MoEConfig("prefill_bias0", T=4096, seed=2, bias_kind="zero",
                               **_FULL),
    # skewed routing, Zipf-like popularity inside every group, SwiGLU limits 4 / 7
    "zipf": MoEConfig("zipf", T=16384, seed=3, bias_kind="zipf", limit_routed=4.0,
                      limit_shared=7.0, **_FULL),
    # routed expert weights in MXFP4 (e2m1 + e8m0 scale per 32 along K)
    "mxfp4": MoEConfig("mxfp4", T=8192, seed=4, wfmt=MOE_W_MXFP4, **_FULL),
    # the same inputs on block-scaled tensor cores: MXFP8 activations x MXFP4 weights
    "mxfp4_a8": MoEConfig("mxfp4_a8", T=8192, seed=4, wfmt=MOE_W_MXFP4_A8, **_FULL),
    # the same, with the weight scales prepared once into the tensor cores' atom layout
    "mxfp4_a8p": MoEConfig("mxfp4_a8p", T=8192, seed=4, wfmt=MOE_W_MXFP4_A8P, **_FULL),
    # small case of the block-scaled variant (its tiles need I % 128 == 0)
    "tiny_a8": MoEConfig("tiny_a8", T=64, H=256, E=32, n_group=4, topk_group=2, K=4,
                         I=128, I_shared=64, seed=0, wfmt=MOE_W_MXFP4_A8),
}


def _gen(device, sub_seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(sub_seed))
    return g


def _normal(shape, var: float, g: torch.Generator, device, chunk_rows: int = 0) -> torch.Tensor:
    """fp32 N(0, var) of the given shape, drawn in row chunks to bound temporaries."""
    std = math.sqrt(var)
    out = torch.empty(shape, dtype=torch.float32, device=device)
    if chunk_rows <= 0 or shape[0] <= chunk_rows:
        out.normal_(0.0, std, generator=g)
        return out
    for r0 in range(0, shape[0], chunk_rows):
        out[r0:r0 + chunk_rows].normal_(0.0, std, generator=g)
    return out


def _bf16(shape, var, g, device, chunk_rows=0) -> torch.Tensor:
    """bf16 N(0, var); drawn in fp32, rounded to nearest even per chunk."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    std = math.sqrt(var)
    rows = shape[0]
    if out.numel() == 0:
        return out
    step = chunk_rows if chunk_rows > 0 else rows
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        tmp = torch.empty((r1 - r0,) + tuple(shape[1:]), dtype=torch.float32, device=device)
        tmp.normal_(0.0, std, generator=g)
        out[r0:r1].copy_(tmp)  # fp32 -> bf16 is round-to-nearest-even
        del tmp
    return out


ZIPF_TABLE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "tests",
                          "golden", "zipf_bias_g64.txt")


def zipf_ranks(cfg: MoEConfig):
    """Within-group popularity rank r = 1..E/G of every expert (int64 [E]):
    a seeded permutation per group (rank 1 = the most favoured expert)."""
    import numpy as np
    per = cfg.experts_per_group
    gcpu = _gen("cpu", cfg.seed * 16 + 2)
    ranks = np.empty(cfg.E, dtype=np.int64)
    for grp in range(cfg.n_group):
        ranks[grp * per:(grp + 1) * per] = torch.randperm(per, generator=gcpu).numpy() + 1
    return ranks


def zipf_table(per: int):
    """Calibrated bias per rank (fp32 [per]) from tests/golden/zipf_bias_g64.txt
    (written by make_zipf_bias.py there), or None when the table is for
    another group size."""
    import numpy as np
    rows = []
    with open(ZIPF_TABLE) as f:
        for line in f:
            line = line.split("#", 1)[0].split()
            if line:
                rows.append(int(line[1], 16))
    if len(rows) != per:
        return None
    return np.array(rows, dtype=np.uint32).view(np.float32)


def selection_bias(cfg: MoEConfig, device="cpu") -> torch.Tensor:
    """Per-expert additive selection bias [E] fp32.

    normal: N(0, bias_var). zero: all 0. zipf: every expert gets the bias of
    its within-group popularity rank (zipf_ranks). With 64 experts per group
    the values per rank are the stored calibration of
    tests/golden/zipf_bias_g64.txt, which makes expert popularity inside each
    group follow p(r) ~ r^-1.1; other group sizes (the small test layers) use
    the fixed formula bias = -zipf_beta * zipf_s * ln(r), which is skewed but
    not calibrated.
    """
    g = _gen(device, cfg.seed * 16 + 2)
    if cfg.bias_kind == "zero":
        return torch.zeros(cfg.E, dtype=torch.float32, device=device)
    if cfg.bias_kind == "normal":
        return _normal((cfg.E,), cfg.bias_var, g, device)
    if cfg.bias_kind == "zipf":
        ranks = zipf_ranks(cfg)
        table = zipf_table(cfg.experts_per_group)
        if table is not None:
            return torch.from_numpy(table[ranks - 1].copy()).to(device)
        b = -cfg.zipf_beta * cfg.zipf_s * torch.log(torch.from_numpy(ranks).double())
        return b.to(torch.float32).to(device)
    raise ValueError(f"unknown bias_kind {cfg.bias_kind}")


def router_inputs(cfg: MoEConfig, device="cpu", T: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """x, Wr and bias of `cfg` alone (the same draws as generate(), without the
    expert weights)."""
    T = cfg.T if T is None else T
    s = cfg.seed * 16
    return {"x": _bf16((T, cfg.H), 1.0, _gen(device, s + 0), device, chunk_rows=8192),
            "Wr": _normal((cfg.E, cfg.H), 1.0 / cfg.H, _gen(device, s + 1), device),
            "bias": selection_bias(cfg, device)}


def generate(cfg: MoEConfig, device="cpu", T: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """All layer inputs for `cfg` on `device`.

    Returns x [T,H] bf16, Wr [E,H] f32, bias [E] f32, Wg/Wu [E,I,H] bf16,
    Wd [E,H,I] bf16, Wg_s/Wu_s [I_s,H] bf16, Wd_s [H,I_s] bf16. For the MXFP4
    format it also returns the packed routed weights (see `mxfp4_pack`):
    Wg_q/Wu_q/Wd_q (uint8 codes) and Wg_sc/Wu_sc/Wd_sc (uint8 e8m0 scales);
    the bf16 Wg/Wu/Wd are then dropped (the layer sees only packed bytes).
    """
    T = cfg.T if T is None else T
    s = cfg.seed * 16
    H, E, I, Is = cfg.H, cfg.E, cfg.I, cfg.I_shared
    out: Dict[str, torch.Tensor] = {}
    out["x"] = _bf16((T, H), 1.0, _gen(device, s + 0), device, chunk_rows=8192)
    out["Wr"] = _normal((E, H), 1.0 / H, _gen(device, s + 1), device)
    out["bias"] = selection_bias(cfg, device)
    chunk = 32  # experts per draw: bounds the fp32 temporary to ~250 MB at full size
    if cfg.wfmt == MOE_W_BF16:
        out["Wg"] = _bf16((E, I, H), 1.0 / H, _gen(device, s + 3), device, chunk)
        out["Wu"] = _bf16((E, I, H), 1.0 / H, _gen(device, s + 4), device, chunk)
        out["Wd"] = _bf16((E, H, I), 1.0 / I, _gen(device, s + 5), device, chunk)
    elif cfg.wfmt in (MOE_W_MXFP4, MOE_W_MXFP4_A8, MOE_W_MXFP4_A8P):
        for name, shape, var, k in (("Wg", (E, I, H), 1.0 / H, 3), ("Wu", (E, I, H), 1.0 / H, 4),
                                    ("Wd", (E, H, I), 1.0 / I, 5)):
            g = _gen(device, s + k)
            codes = torch.empty(shape[0], shape[1], shape[2] // 2, dtype=torch.uint8, device=device)
            scales = torch.empty(shape[0], shape[1], shape[2] // 32, dtype=torch.uint8, device=device)
            for e0 in range(0, E, chunk):
                e1 = min(E, e0 + chunk)
                w = torch.empty((e1 - e0,) + shape[1:], dtype=torch.float32, device=device)
                w.normal_(0.0, math.sqrt(var), generator=g)
                codes[e0:e1], scales[e0:e1] = mxfp4_pack(w)
                del w
            out[name + "_q"], out[name + "_sc"] = codes, scales
    else:
        raise ValueError("unknown weight format")
    out["Wg_s"] = _bf16((Is, H), 1.0 / H, _gen(device, s + 6), device)
    out["Wu_s"] = _bf16((Is, H), 1.0 / H, _gen(device, s + 7), device)
    out["Wd_s"] = _bf16((H, Is), 1.0 / max(Is, 1), _gen(device, s + 8), device)
    return out


def tokens(cfg: MoEConfig, T: int, step: int, device="cpu") -> torch.Tensor:
    """A fresh bf16 N(0,1) token batch [T,H] for step `step` (used for per-step inputs)."""
    return _bf16((T, cfg.H), 1.0, _gen(device, cfg.seed * 16 + 9 + 1000 * (step + 1)), device,
                 chunk_rows=8192)


# ---------------------------------------------------------------------------
# MXFP4 encoding of the routed weights (input format, OCP Microscaling v1.0):
# blocks of 32 consecutive values along K share one e8m0 scale 2^(X) with
# X = floor(log2(amax)) - 2 (2 = emax of e2m1); every value is v / 2^X rounded
# to the nearest e2m1 number (ties to even mantissa), saturating at +-6.
# Byte layout: codes [..., K/2], element 2j in the low nibble, 2j+1 in the
# high nibble; code = sign<<3 | magnitude index into {0,.5,1,1.5,2,3,4,6}.
# Scales [..., K/32], byte = X + 127 (0xFF, NaN, is never produced).
# ---------------------------------------------------------------------------
_E2M1_MAG = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)


def mxfp4_pack(w: torch.Tensor):
    """Encode fp32 `w` [..., K] (K % 32 == 0) as MXFP4 codes + e8m0 scales."""
    assert w.dtype == torch.float32 and w.shape[-1] % 32 == 0
    K = w.shape[-1]
    blk = w.reshape(*w.shape[:-1], K // 32, 32)
    amax = blk.abs().amax(dim=-1)
    # floor(log2(amax)) exactly, from the fp32 exponent field (amax > 0); amax == 0 -> X = -127
    bits = amax.view(torch.int32)
    expo = ((bits >> 23) & 0xFF).to(torch.int32) - 127
    sub = (bits >> 23) & 0xFF == 0
    if bool(sub.any()):  # subnormal amax: take log2 through float64
        l2 = torch.floor(torch.log2(amax.double().clamp_min(1e-300))).to(torch.int32)
        expo = torch.where(sub, l2, expo)
    X = expo - 2
    X = torch.where(amax == 0, torch.full_like(X, -127), X)
    X = X.clamp(-127, 127)
    scale_byte = (X + 127).to(torch.uint8)
    q = blk / torch.pow(2.0, X.to(torch.float32)).unsqueeze(-1)
    a = q.abs()
    # nearest e2m1 magnitude, ties to the even code (codes 0..7; even = mantissa bit 0)
    mags = torch.tensor(_E2M1_MAG, dtype=torch.float32, device=w.device)
    mid = (mags[1:] + mags[:-1]) / 2                       # 7 decision points
    code = torch.zeros_like(a, dtype=torch.int32)
    for i in range(7):
        above = a > mid[i]
        tie = a == mid[i]
        # at a tie go up only if the upper code (i+1) is even
        up = above | (tie & ((i + 1) % 2 == 0))
        code = code + up.to(torch.int32)
    code = code.clamp(0, 7)
    sign = (q < 0) & (code > 0)
    code = code | (sign.to(torch.int32) << 3)
    code = code.reshape(*w.shape[:-1], K)
    lo = code[..., 0::2]
    hi = code[..., 1::2]
    packed = (lo | (hi << 4)).to(torch.uint8)
    return packed, scale_byte.reshape(*w.shape[:-1], K // 32)


def expert_params(cfg: MoEConfig) -> int:
    """Parameters of one routed expert: gate, up and down matrices."""
    return 3 * cfg.H * cfg.I
