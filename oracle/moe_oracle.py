"""CPU oracle for one sparse-MoE FFN layer (sigmoid router, group-limited top-k,
SwiGLU experts, shared expert).

TEST INFRASTRUCTURE ONLY. This file is imported by the tests, by
`__graft_entry__.smoke()` and by the CPU-baseline leg of `bench.py`; the
product path (the CUDA library and its Python binding) never imports it.
It shares no code with the CUDA path.

It is written to be checked by eye against the method's description, not to
be fast: numpy float64 throughout, with a matrix product (a library
primitive) for every dot product and the rounding points listed below.

Sources (page title, section):
  [P3] "Ling-3.0-flash-VL MoE sparse routing" (lqnn.cn/news/282163)
       sec. 3 step 1  sigmoid scores, independent per expert, fp32 router
       sec. 3 step 2  n_group = 8 groups, keep topk_group = 4 by the highest
                      in-group score, then top-8 of the 256 candidates
       sec. 3 step 3  learnable per-expert bias for aux-loss-free balancing
       sec. 4         router_dtype fp32, routed_scaling_factor 2.5,
                      norm_topk_prob (weights of the chosen 8 sum to 1),
                      SwiGLU limit (+-4 routed, +-5/+-7 shared)
       sec. 2         1 shared expert per layer seen by every token; expert =
                      gate/up/down, hidden 2560, intermediate 768
  [P4] "Ling-3.0-flash-VL 42-layer hybrid backbone" (lpnh.cn/news/2815793),
       spec table: routed-expert weights in MXFP4 (4 bit).
  [P1] "Ling-3.0-flash-VL：层级化稀疏路由大模型硬核解析" (sheratonhq.com/news/113555),
       sec. 4.1: monitor the routing entropy of the expert selection
       frequencies and the experts that are never selected.

Readings where the pages are silent (each also listed in the design notes):
  R1 group score = max over the group of the BIASED score b = s + bias.
  R2 candidates are ranked by the biased score b.
  R3 the combine weights use the UNBIASED sigmoid score s (bias is for
     selection only).
  R4 renormalise first, then multiply by the scaling factor (sum w = 2.5).
  R5 ties (groups and experts) go to the lower index.
  R6 SwiGLU limit L clamps both gate and up to [-L, L] before silu(gate)*up;
     L <= 0 means no limit.
  R7 rounding: logits, scores and biased scores are fp32; gate/up/down dot
     products are accumulated exactly enough (float64) and rounded to fp32;
     h = silu(g)*u is rounded to fp32 then to bf16 (nearest even) before the
     down projection; y_slot = w * o in fp32; the token output is the fp32 sum
     over k in slot order plus the shared expert output, rounded to bf16.
  R8 slot order inside a token = selection rank; permutation order inside an
     expert = ascending flat index j = t*K + k (stable counting sort).
  R9 MXFP4 weights are used through their exact dequantised values
     (e2m1 magnitude * sign * 2^(scale - 127)).
  R15 block-scaled variant (weight format MXFP4_A8): the spec table of [P4]
     lists the quantisation scheme as FP8 + MXFP4. It is read as MXFP8
     activations (OCP Microscaling v1.0: e4m3 elements, one e8m0 scale per
     32 consecutive elements along the contraction) for the routed experts:
     x is quantised before gate/up, h (fp32) before down, instead of R7's
     bf16 h. Scale = 2^(floor(log2(amax)) - 8) (8 = e4m3's largest exponent),
     its byte clamped to [0, 254] (amax = 0 gives byte 0); elements are
     v / scale rounded to nearest e4m3, ties to even, saturating at +-448.
     The shared expert keeps the bf16 path of R7.

Parity pins: see tests/test_oracle_*.py (brute-force group enumeration, rank
counting, reductions to plain top-k and argmax, the all-ties case, closed
forms, invariants, MXFP4 code table). End-to-end agreement with the trained
Ling-3.0 model is not pinned: no trained weights and no worked numeric example
are printed on the pages ("parity unpinned" for that comparison only).
"""
from __future__ import annotations

import math
from typing import Callable, Optional, Sequence, Tuple

import numpy as np

# --------------------------------------------------------------------------
# number formats
# --------------------------------------------------------------------------


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64: a bf16 is the top half of an fp32."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest, ties to even (finite inputs)."""
    u = np.ascontiguousarray(np.asarray(a, dtype=np.float32)).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    return ((u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)).astype(np.uint16)


E2M1_MAGNITUDE = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)


def mxfp4_dequantize(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """MXFP4 (OCP Microscaling v1.0) -> float64.

    codes  [..., K/2] uint8: element 2j in the low nibble, 2j+1 in the high one;
           nibble = sign bit (8) | index into the e2m1 magnitudes.
    scales [..., K/32] uint8: e8m0 exponent, value 2^(byte - 127) (0xFF = NaN).
    [P4] spec table: the routed experts' weights are stored in MXFP4.
    """
    codes = np.asarray(codes, dtype=np.uint8)
    scales = np.asarray(scales, dtype=np.uint8)
    lo = codes & 0x0F
    hi = codes >> 4
    nib = np.stack([lo, hi], axis=-1).reshape(*codes.shape[:-1], codes.shape[-1] * 2)
    mag = np.asarray(E2M1_MAGNITUDE, dtype=np.float64)[nib & 7]
    val = np.where(nib & 8, -mag, mag)
    s = scales.astype(np.float64)
    scale = np.where(scales == 0xFF, np.nan, np.exp2(s - 127.0))
    scale = np.repeat(scale, 32, axis=-1)
    return val * scale


E4M3_MAX = 448.0
MOE_W_MXFP4_A8 = 2   # weight-format code of the block-scaled variant (R15)


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """OCP e4m3 (the "fn" variant: no infinities) -> float64.

    Bit 7 sign, bits 6..3 exponent (bias 7), bits 2..0 mantissa; exponent 0
    is subnormal (m/8 * 2^-6); exponent 15 with mantissa 7 is NaN."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


# the 127 finite non-negative e4m3 values, in code order (increasing)
_E4M3_POS = e4m3_decode(np.arange(0x7F, dtype=np.uint8))


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    """Nearest e4m3 code to each finite float64 value, ties to the even code
    (mantissa bit 0 clear), magnitudes above 448 saturate to 448 (R15); the
    sign bit is the input's, also when the magnitude rounds to zero."""
    v = np.asarray(v, dtype=np.float64)
    a = np.minimum(np.abs(v), E4M3_MAX)
    hi = np.clip(np.searchsorted(_E4M3_POS, a, side="left"), 0, 0x7E)  # first value >= a
    lo = np.maximum(hi - 1, 0)
    dlo = a - _E4M3_POS[lo]
    dhi = _E4M3_POS[hi] - a
    take_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0))
    code = np.where(take_hi, hi, lo).astype(np.uint8)
    return np.where(np.signbit(v), code | 0x80, code).astype(np.uint8)   # the sign is kept


def mxfp8_quantize(v: np.ndarray):
    """MXFP8 (e4m3 elements, e8m0 scale per 32 along the last axis), R15.

    v [..., K] float (K a multiple of 32) -> (codes uint8 [..., K],
    scales uint8 [..., K/32])."""
    v = np.asarray(v, dtype=np.float64)
    blk = v.reshape(*v.shape[:-1], v.shape[-1] // 32, 32)
    amax = np.abs(blk).max(axis=-1)
    _, ex = np.frexp(amax)                      # amax = f * 2^ex, f in [0.5, 1)
    floor_log2 = ex.astype(np.int64) - 1
    byte = np.where(amax > 0, np.clip(floor_log2 - 8 + 127, 0, 254), 0).astype(np.uint8)
    scale = np.exp2(byte.astype(np.float64) - 127.0)
    codes = e4m3_encode(blk / scale[..., None]).reshape(v.shape)
    return codes, byte


def mxfp8_dequantize(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Exact float64 values of MXFP8 codes and their e8m0 scales."""
    s = np.exp2(np.asarray(scales, dtype=np.float64) - 127.0)
    return e4m3_decode(codes) * np.repeat(s, 32, axis=-1)


# --------------------------------------------------------------------------
# routing  ([P3] sec. 3 and sec. 4)
# --------------------------------------------------------------------------


def router_logits(x_bits: np.ndarray, Wr: np.ndarray) -> np.ndarray:
    """z[t,e] = sum_h x[t,h] * Wr[e,h], accumulated in float64, rounded to fp32.

    [P3] sec. 3 step 1 (512 raw scores per token from the router matrix) and
    sec. 4 (router_dtype fp32: the router computes in fp32 even with bf16
    weights)."""
    x = bf16_bits_to_f64(x_bits)
    W = np.asarray(Wr, dtype=np.float32).astype(np.float64)
    return (x @ W.T).astype(np.float32)


def sigmoid_scores(z: np.ndarray) -> np.ndarray:
    """s = 1 / (1 + exp(-z)) per element, fp32.  [P3] sec. 3 step 1."""
    z64 = np.asarray(z, dtype=np.float32).astype(np.float64)
    return (1.0 / (1.0 + np.exp(-z64))).astype(np.float32)


def biased_scores(s: np.ndarray, bias: np.ndarray) -> np.ndarray:
    """b = s + bias[e] in fp32 (selection only).  [P3] sec. 3 step 3; R3."""
    return (np.asarray(s, np.float32).astype(np.float64)
            + np.asarray(bias, np.float32).astype(np.float64)[None, :]).astype(np.float32)


def group_limited_topk(b: np.ndarray, n_group: int, topk_group: int, K: int):
    """Group-limited top-k on biased scores b [T,E].  [P3] sec. 3 step 2.

    1. group score = max of b over the group's E/n_group experts (R1);
    2. keep the topk_group groups with the highest group score (ties: lower g);
    3. among the experts of the kept groups take the K with the highest b
       (ties: lower e), in rank order (R2, R5, R8).

    Returns idx [T,K] int32 and the two margins used to flag near ties:
    group margin = 4th minus 5th group score, expert margin = Kth minus
    (K+1)th candidate score (inf when there is no 5th group / (K+1)th
    candidate).
    """
    b = np.asarray(b, dtype=np.float32)
    T, E = b.shape
    per = E // n_group
    gscore = b.reshape(T, n_group, per).max(axis=2)
    # descending score, equal scores keep ascending index order (stable sort)
    gorder = np.argsort(-gscore, axis=1, kind="stable")
    kept = gorder[:, :topk_group]
    keep_mask = np.zeros((T, n_group), dtype=bool)
    np.put_along_axis(keep_mask, kept, True, axis=1)
    is_cand = np.repeat(keep_mask, per, axis=1)
    cand = np.where(is_cand, b.astype(np.float64), -np.inf)
    eorder = np.argsort(-cand, axis=1, kind="stable")
    idx = eorder[:, :K].astype(np.int32)

    gs = np.take_along_axis(gscore.astype(np.float64), gorder, axis=1)
    if topk_group < n_group:
        gmargin = gs[:, topk_group - 1] - gs[:, topk_group]
    else:
        gmargin = np.full(T, np.inf)
    cs = np.take_along_axis(cand, eorder, axis=1)
    if K < topk_group * per:
        emargin = cs[:, K - 1] - cs[:, K]
    else:
        emargin = np.full(T, np.inf)
    return idx, gmargin, emargin


def combine_weights(s: np.ndarray, idx: np.ndarray, scale: float, renorm: bool) -> np.ndarray:
    """w[t,k] = scale * s[t,idx_k] / sum_j s[t,idx_j] (renorm on), fp32.

    [P3] sec. 4: norm_topk_prob renormalises the chosen scores to sum to 1,
    routed_scaling_factor 2.5 multiplies the routed contribution (R3, R4)."""
    sel = np.take_along_axis(np.asarray(s, np.float32).astype(np.float64), idx, axis=1)
    if renorm:
        den = sel.sum(axis=1, keepdims=True)
        if np.any(den == 0.0):
            raise FloatingPointError("sum of selected sigmoid scores is zero")
        w = scale * (sel / den)
    else:
        w = scale * sel
    return w.astype(np.float32)


def route(x_bits, Wr, bias, n_group, topk_group, K, scale=2.5, renorm=True):
    """Stages 1-4 of the layer for every token: returns a dict with
    z, s, b (fp32 [T,E]), idx [T,K] int32, w [T,K] fp32, gmargin, emargin."""
    z = router_logits(x_bits, Wr)
    s = sigmoid_scores(z)
    b = biased_scores(s, bias)
    idx, gm, em = group_limited_topk(b, n_group, topk_group, K)
    w = combine_weights(s, idx, scale, renorm)
    return dict(z=z, s=s, b=b, idx=idx, w=w, gmargin=gm, emargin=em)


# --------------------------------------------------------------------------
# permutation (each token selects K experts; rows are grouped by expert)
# --------------------------------------------------------------------------


def permute(idx: np.ndarray, E: int):
    """Stable counting sort of the flat slots j = t*K + k by expert (R8).

    counts[e] = #{j : idx_flat[j] = e}; offsets = exclusive prefix sum (E+1);
    perm[r] = the slot at sorted position r; inv_perm[j] = position of slot j.
    """
    flat = np.asarray(idx, dtype=np.int64).reshape(-1)
    counts = np.bincount(flat, minlength=E).astype(np.int32)
    offsets = np.zeros(E + 1, dtype=np.int32)
    offsets[1:] = np.cumsum(counts)
    perm = np.argsort(flat, kind="stable").astype(np.int32)
    inv_perm = np.empty_like(perm)
    inv_perm[perm] = np.arange(perm.size, dtype=np.int32)
    return counts, offsets, perm, inv_perm


def route_stats(counts: np.ndarray, E: int) -> np.ndarray:
    """Load statistics of one routing pass from its expert counts ([P1] sec. 4.1).

    p_e = counts[e] / sum(counts); returns float64 [7]:
      0 H = -sum_{p_e > 0} p_e log2 p_e (bits), 1 H / log2 E, 2 max count,
      3 mean count (sum / E), 4 max / mean, 5 experts with count 0, 6 sum.
    With no slots at all every entry but the idle count (= E) is 0.
    """
    c = np.asarray(counts, dtype=np.int64)[:E]
    tot = float(c.sum())
    H = 0.0
    if tot > 0:
        p = c[c > 0] / tot
        H = float(-(p * np.log2(p)).sum())
    mx = float(c.max()) if E > 0 else 0.0
    mean = tot / E
    return np.array([H, H / math.log2(E) if E > 1 else 0.0, mx, mean,
                     mx / mean if mean > 0 else 0.0, float((c == 0).sum()), tot])


# --------------------------------------------------------------------------
# experts ([P3] sec. 2 and sec. 4)
# --------------------------------------------------------------------------


def swiglu_expert(x64: np.ndarray, Wg64: np.ndarray, Wu64: np.ndarray, Wd64: np.ndarray,
                  limit: float = 0.0, h_mxfp8: bool = False) -> Tuple[np.ndarray, np.ndarray]:
    """One SwiGLU expert on rows x64 [n,H] (float64 values of its inputs).

    g = x Wg^T, u = x Wu^T (fp32 results); with a limit L > 0 both are clamped
    to [-L, L] (R6); h = fp32(silu(g) * u), silu(g) = g / (1 + e^-g), rounded
    to bf16 (R7) or, with h_mxfp8, quantised to MXFP8 along I (R15);
    o = h Wd^T (fp32).  Returns (o fp32 [n,H_out], h): h as bf16 bits [n,I],
    or with h_mxfp8 the pair (codes [n,I], scales [n,I/32])."""
    g = (x64 @ Wg64.T).astype(np.float32)
    u = (x64 @ Wu64.T).astype(np.float32)
    if limit is not None and limit > 0.0 and math.isfinite(limit):
        L = np.float32(limit)
        g = np.clip(g, -L, L)
        u = np.clip(u, -L, L)
    g64 = g.astype(np.float64)
    a = ((g64 / (1.0 + np.exp(-g64))) * u.astype(np.float64)).astype(np.float32)
    if h_mxfp8:
        hq, hs = mxfp8_quantize(a)
        o = (mxfp8_dequantize(hq, hs) @ Wd64.T).astype(np.float32)
        return o, (hq, hs)
    h_bits = f32_to_bf16_bits(a)
    o = (bf16_bits_to_f64(h_bits) @ Wd64.T).astype(np.float32)
    return o, h_bits


ExpertFn = Callable[[int], Tuple[np.ndarray, np.ndarray, np.ndarray]]


def dense_expert_weights(Wg, Wu, Wd) -> ExpertFn:
    """Weight accessor over full bf16-bit arrays Wg/Wu [E,I,H], Wd [E,H,I]."""
    def get(e: int):
        return bf16_bits_to_f64(Wg[e]), bf16_bits_to_f64(Wu[e]), bf16_bits_to_f64(Wd[e])
    return get


def mxfp4_expert_weights(Wg_q, Wg_sc, Wu_q, Wu_sc, Wd_q, Wd_sc) -> ExpertFn:
    """Weight accessor over MXFP4-packed routed weights (R9)."""
    def get(e: int):
        return (mxfp4_dequantize(Wg_q[e], Wg_sc[e]), mxfp4_dequantize(Wu_q[e], Wu_sc[e]),
                mxfp4_dequantize(Wd_q[e], Wd_sc[e]))
    return get


def layer_forward(cfg, x_bits: np.ndarray, Wr: np.ndarray, bias: np.ndarray,
                  expert: ExpertFn, Wg_s, Wu_s, Wd_s,
                  tokens: Optional[Sequence[int]] = None):
    """Whole layer: route, permute, experts, weighted combine, shared expert.

    `cfg` needs H, E, n_group, topk_group, K, scale, renorm, limit_routed,
    limit_shared. With `tokens` given, routing still covers all rows of x but
    the expert stages run only for those tokens (sampled outputs of a large
    batch). Returns a dict with the routing results, permutation, h of the
    shared expert, y_slot [n,K,H] fp32, the fp32 output before its final
    rounding y_f32 [n,H] and y bf16 bits [n,H] for the evaluated tokens (in
    the order of `tokens`)."""
    r = route(x_bits, Wr, bias, cfg.n_group, cfg.topk_group, cfg.K, cfg.scale, cfg.renorm)
    counts, offsets, perm, inv_perm = permute(r["idx"], cfg.E)
    T = x_bits.shape[0]
    tok = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    x64 = bf16_bits_to_f64(x_bits[tok])
    n, K, H = tok.size, cfg.K, cfg.H
    act_mx = getattr(cfg, "wfmt", 0) == MOE_W_MXFP4_A8
    # R15: the routed experts see x through its MXFP8 values
    xr64 = mxfp8_dequantize(*mxfp8_quantize(x64)) if act_mx else x64
    y_slot = np.zeros((n, K, H), dtype=np.float32)
    idx = r["idx"][tok]
    w = r["w"][tok]
    for e in np.unique(idx):
        rows, ks = np.nonzero(idx == e)
        Wg, Wu, Wd = expert(int(e))
        o, _ = swiglu_expert(xr64[rows], Wg, Wu, Wd, cfg.limit_routed, h_mxfp8=act_mx)
        y_slot[rows, ks, :] = (w[rows, ks][:, None].astype(np.float32) * o).astype(np.float32)
    o_sh, h_sh = swiglu_expert(x64, bf16_bits_to_f64(Wg_s), bf16_bits_to_f64(Wu_s),
                               bf16_bits_to_f64(Wd_s), cfg.limit_shared)
    acc = np.zeros((n, H), dtype=np.float32)
    for k in range(K):                     # fp32 sum in slot order
        acc = (acc + y_slot[:, k, :]).astype(np.float32)
    acc = (acc + o_sh).astype(np.float32)
    y = f32_to_bf16_bits(acc)
    out = dict(r)
    out.update(counts=counts, offsets=offsets, perm=perm, inv_perm=inv_perm,
               tokens=tok, y_slot=y_slot, y_shared=o_sh, h_shared=h_sh, y_f32=acc, y=y)
    return out
