// router.cu - stages 1-5 of the layer: fp32 router logits, sigmoid scores,
// selection bias, group-limited top-k and renormalised, scaled weights.
//
// Page "Ling-3.0-flash-VL MoE sparse routing" (lqnn.cn/news/282163):
//   sec. 3 step 1: one raw score per expert, passed through an elementwise
//                  sigmoid (independent scores, not a softmax);
//   sec. 3 step 2: 8 groups of 64 experts, keep the 4 groups with the highest
//                  in-group score, then the 8 best of the 256 candidates;
//   sec. 3 step 3: a per-expert bias added to the scores for balancing;
//   sec. 4:        the router computes in fp32; the chosen scores are
//                  renormalised to sum to 1 and scaled by 2.5.
// Readings: the group score and the candidate ranking use the biased score;
// the weights use the unbiased one; ties go to the lower index.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <algorithm>
#include <type_traits>

#include "internal.h"
#include "ptx.cuh"

namespace sgl {
namespace {

// ---------------------------------------------------------------------------
// Logits for a set of rows, one warp per expert: the expert's fp32 router row
// is held in registers (a strided slice per lane) and up to 32 token rows are
// staged in shared memory as bf16; ILP tokens are accumulated at once.
//  EXACT = false: fp32 FMA accumulation (the pages' fp32 router), for small
//                 batches;
//  EXACT = true:  every product bf16 * fp32 is exact in float64 and the sum
//                 of H of them is accumulated in float64, so the one final
//                 rounding to fp32 gives the logit of an exact dot product.
//                 Used for the tokens whose fp32 decision was too close.
// With `list`, the rows are list[0 .. *list_n) instead of 0 .. T-1.
// ---------------------------------------------------------------------------
constexpr int kSmallT = 32;
constexpr int kRowRegs = 24;  // float4 per lane: H <= 24 * 128 = 3072
constexpr int kMaxExperts = 1024;
constexpr int kRowWarps = 4;  // experts per CTA
constexpr int kTokSplit = 2;  // warps per expert (they split the token rows)

// bf16 bits -> float64 by field arithmetic (no conversion instruction):
// sign, exponent rebiased from 127 to 1023, 7 mantissa bits on top.
__device__ __forceinline__ double bf16_bits_to_double(uint32_t b) {
  const uint32_t ex = (b >> 7) & 0xFFu;
  if (ex == 0u || ex == 0xFFu) return static_cast<double>(__uint_as_float(b << 16));
  const unsigned long long bits = (static_cast<unsigned long long>(b & 0x8000u) << 48) |
                                  (static_cast<unsigned long long>(ex + 896u) << 52) |
                                  (static_cast<unsigned long long>(b & 0x7Fu) << 45);
  return __longlong_as_double(static_cast<long long>(bits));
}

template <bool EXACT, int ILP>
__global__ void __launch_bounds__(kRowWarps * kTokSplit * 32) router_logits_rows(
    int T, int H, int E, const uint16_t* __restrict__ x, const float* __restrict__ Wr,
    float* __restrict__ z, const int32_t* __restrict__ list, const int32_t* __restrict__ list_n,
    int32_t* __restrict__ err) {
  using Acc = typename std::conditional<EXACT, double, float>::type;
  extern __shared__ __align__(128) uint16_t xs[];  // [kSmallT][H]
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int e = blockIdx.x * kRowWarps + (warp % kRowWarps);
  const int split = warp / kRowWarps;  // this warp takes token groups split, split+kTokSplit, ...
  const bool have = e < E;
  const int n = list ? min(*list_n, T) : T;
  if (n <= 0) return;
  if (tid == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  uint32_t phase = 0;
  float4 wv[kRowRegs];
  {
    // unconditional loads from clamped addresses (all in flight together),
    // then zero the slots past the row's end
    const float* row = Wr + static_cast<size_t>(have ? e : 0) * H;
#pragma unroll
    for (int j = 0; j < kRowRegs; ++j)
      wv[j] = *reinterpret_cast<const float4*>(row + min(4 * lane + 128 * j, H - 4));
#pragma unroll
    for (int j = 0; j < kRowRegs; ++j)
      if (4 * lane + 128 * j >= H) wv[j] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  const uint32_t row_bytes = static_cast<uint32_t>(H) * 2;
  for (int c0 = 0; c0 < n; c0 += kSmallT) {
    const int nc = min(kSmallT, n - c0);
    __syncthreads();  // everyone is done with the previous chunk
    if (tid == 0) {
      // one bulk copy per token row, all in flight at once
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(&bar, row_bytes * nc);
      for (int r = 0; r < nc; ++r) {
        const int t = list ? list[c0 + r] : c0 + r;
        bulk_load(xs + r * H, x + static_cast<size_t>(t) * H, row_bytes, &bar);
      }
    }
    mbar_wait(&bar, phase, &abort_flag, err, MOE_DEVERR_TIMEOUT);
    phase ^= 1;
    if (!have) continue;
    for (int r0 = split * ILP; r0 < nc; r0 += ILP * kTokSplit) {
      Acc acc[ILP];
#pragma unroll
      for (int q = 0; q < ILP; ++q) acc[q] = Acc(0);
#pragma unroll
      for (int j = 0; j < kRowRegs; ++j) {
        const int k = 4 * lane + 128 * j;
        if (k < H) {
          Acc w0, w1, w2, w3;
          if (EXACT) {
            w0 = static_cast<Acc>(wv[j].x); w1 = static_cast<Acc>(wv[j].y);
            w2 = static_cast<Acc>(wv[j].z); w3 = static_cast<Acc>(wv[j].w);
          } else {
            w0 = wv[j].x; w1 = wv[j].y; w2 = wv[j].z; w3 = wv[j].w;
          }
#pragma unroll
          for (int q = 0; q < ILP; ++q) {
            const int r = min(r0 + q, nc - 1);
            const uint2 p = *reinterpret_cast<const uint2*>(xs + r * H + k);
            if (EXACT) {
              acc[q] = fma(w0, static_cast<Acc>(bf16_bits_to_double(p.x & 0xFFFFu)), acc[q]);
              acc[q] = fma(w1, static_cast<Acc>(bf16_bits_to_double(p.x >> 16)), acc[q]);
              acc[q] = fma(w2, static_cast<Acc>(bf16_bits_to_double(p.y & 0xFFFFu)), acc[q]);
              acc[q] = fma(w3, static_cast<Acc>(bf16_bits_to_double(p.y >> 16)), acc[q]);
            } else {
              acc[q] = fmaf(w0, __uint_as_float(p.x << 16), acc[q]);
              acc[q] = fmaf(w1, __uint_as_float(p.x & 0xFFFF0000u), acc[q]);
              acc[q] = fmaf(w2, __uint_as_float(p.y << 16), acc[q]);
              acc[q] = fmaf(w3, __uint_as_float(p.y & 0xFFFF0000u), acc[q]);
            }
          }
        }
      }
#pragma unroll
      for (int q = 0; q < ILP; ++q) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc[q] += __shfl_xor_sync(0xffffffffu, acc[q], o);
      }
      if (lane < ILP) {
        Acc v = acc[0];
#pragma unroll
        for (int q = 1; q < ILP; ++q)
          if (lane == q) v = acc[q];
        if (r0 + lane < nc) {
          const int t = list ? list[c0 + r0 + lane] : c0 + r0 + lane;
          z[static_cast<size_t>(t) * E + e] = static_cast<float>(v);
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Logits for larger batches: a 128 (tokens) x 128 (experts) fp32 SIMT tile
// per CTA, 8x8 outputs per thread, K streamed in chunks of 16 through
// double-buffered shared memory.
// ---------------------------------------------------------------------------
constexpr int kRT = 128, kRE = 128, kRK = 16;

__global__ void __launch_bounds__(256) router_logits_tiled(int T, int H, int E,
                                                          const uint16_t* __restrict__ x,
                                                          const float* __restrict__ Wr,
                                                          float* __restrict__ z) {
  __shared__ __align__(16) float xs[2][kRK][kRT + 4];
  __shared__ __align__(16) float ws[2][kRK][kRE + 4];
  const int tid = threadIdx.x;
  const int t0 = blockIdx.x * kRT, e0 = blockIdx.y * kRE;
  // loader mapping: row = tid / 2 (token or expert), 8 consecutive k per thread
  const int lrow = tid >> 1, lk = (tid & 1) * 8;
  const bool xok = (t0 + lrow) < T, wok = (e0 + lrow) < E;
  const uint16_t* xsrc = x + static_cast<size_t>(t0 + lrow) * H + lk;
  const float* wsrc = Wr + static_cast<size_t>(e0 + lrow) * H + lk;

  uint4 xr;
  float4 wr0, wr1;
  auto gload = [&](int kc) {
    xr = xok ? *reinterpret_cast<const uint4*>(xsrc + kc) : make_uint4(0, 0, 0, 0);
    wr0 = wok ? *reinterpret_cast<const float4*>(wsrc + kc) : make_float4(0.f, 0.f, 0.f, 0.f);
    wr1 = wok ? *reinterpret_cast<const float4*>(wsrc + kc + 4) : make_float4(0.f, 0.f, 0.f, 0.f);
  };
  auto sstore = [&](int buf) {
    const uint32_t xv[4] = {xr.x, xr.y, xr.z, xr.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      xs[buf][lk + 2 * i][lrow] = __uint_as_float(xv[i] << 16);
      xs[buf][lk + 2 * i + 1][lrow] = __uint_as_float(xv[i] & 0xFFFF0000u);
    }
    ws[buf][lk + 0][lrow] = wr0.x;
    ws[buf][lk + 1][lrow] = wr0.y;
    ws[buf][lk + 2][lrow] = wr0.z;
    ws[buf][lk + 3][lrow] = wr0.w;
    ws[buf][lk + 4][lrow] = wr1.x;
    ws[buf][lk + 5][lrow] = wr1.y;
    ws[buf][lk + 6][lrow] = wr1.z;
    ws[buf][lk + 7][lrow] = wr1.w;
  };

  const int ty = tid >> 4, tx = tid & 15;
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  const int nk = H / kRK;
  gload(0);
  sstore(0);
  __syncthreads();
  for (int kc = 0; kc < nk; ++kc) {
    const int buf = kc & 1;
    if (kc + 1 < nk) gload((kc + 1) * kRK);
#pragma unroll
    for (int k = 0; k < kRK; ++k) {
      const float4 a0 = *reinterpret_cast<const float4*>(&xs[buf][k][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4*>(&xs[buf][k][64 + ty * 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&ws[buf][k][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4*>(&ws[buf][k][64 + tx * 4]);
      const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    if (kc + 1 < nk) sstore(buf ^ 1);
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int t = t0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + i - 4);
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = e0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + j - 4);
      if (e < E) z[static_cast<size_t>(t) * E + e] = acc[i][j];
    }
  }
}

// ---------------------------------------------------------------------------
// Scores and group-limited top-k: one warp per token. Lane l holds experts
// e = l + 32*j. The combine weights are computed in float64 from the fp32
// scores and rounded once.
//
// Two modes:
//  certified (tau > 0): scores from an fp32 sigmoid of the fp32 logits; the
//    kernel also measures its own decision margins (the topk_group-th minus
//    the next group score, and every gap between neighbours in the ranking
//    of the K+1 best candidates, since slot order is rank order) and appends
//    the token to `unc` when one is below tau (scaled by the token's logit
//    RMS); those tokens get exact logits and a second, exact pass.
//  exact (tau == 0): scores from a float64 sigmoid rounded to fp32 (the
//    reference definition), over the tokens in `list`.
// GJ > 0: every group spans GJ whole register slots (E/n_group a multiple of
// 32), so group maxima are reduced in registers, all groups at once.
// ---------------------------------------------------------------------------
template <int NV, int GJ>
__global__ void __launch_bounds__(256) router_topk(int T, int E, int n_group, int topk_group,
                                                   int K, float scale, int renorm,
                                                   const float* __restrict__ z,
                                                   const float* __restrict__ bias,
                                                   int32_t* __restrict__ idx,
                                                   float* __restrict__ wout, float tau,
                                                   int32_t* __restrict__ unc,
                                                   int32_t* __restrict__ unc_n,
                                                   const int32_t* __restrict__ list,
                                                   const int32_t* __restrict__ list_n) {
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  const int n = list ? min(*list_n, T) : T;
  const int per = E / n_group;
  for (int q = blockIdx.x * wpb + (threadIdx.x >> 5); q < n; q += gridDim.x * wpb) {
    const int t = list ? list[q] : q;
    const float* zr = z + static_cast<size_t>(t) * E;
    float s[NV], b[NV], zv[NV], bv0[NV];
    // all loads first, from clamped (always valid) addresses, so they are in
    // flight together; lanes past E are masked afterwards
#pragma unroll
    for (int j = 0; j < NV; ++j) zv[j] = zr[min(lane + 32 * j, E - 1)];
#pragma unroll
    for (int j = 0; j < NV; ++j) bv0[j] = bias ? bias[min(lane + 32 * j, E - 1)] : 0.f;
    float zz = 0.f;
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const bool in = lane + 32 * j < E;
      if (in) zz = fmaf(zv[j], zv[j], zz);
      s[j] = tau > 0.f ? 1.0f / (1.0f + expf(-zv[j]))
                       : static_cast<float>(1.0 / (1.0 + exp(-static_cast<double>(zv[j]))));
      b[j] = in ? s[j] + bv0[j] : -INFINITY;
      if (!in) s[j] = 0.f;
    }
    // ---- groups: keep topk_group by their max b (ties -> lower group)
    uint32_t kept_groups = 0;  // bit g set when group g is kept
    float gmargin = INFINITY;
    if (GJ > 0) {
      constexpr int G = GJ > 0 ? NV / GJ : 1;
      float gs[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float m = b[g * GJ];
#pragma unroll
        for (int i = 1; i < GJ; ++i) m = fmaxf(m, b[g * GJ + i]);
        gs[g] = m;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int g = 0; g < G; ++g) gs[g] = fmaxf(gs[g], __shfl_xor_sync(0xffffffffu, gs[g], o));
      float last = 0.f;
      for (int r = 0; r <= topk_group && r < G; ++r) {
        float bv = -INFINITY;
        int bi = -1;
#pragma unroll
        for (int g = 0; g < G; ++g)
          if (!((kept_groups >> g) & 1u) && (bi < 0 || gs[g] > bv)) {
            bv = gs[g];
            bi = g;
          }
        if (r < topk_group) {
          kept_groups |= 1u << bi;
          last = bv;
        } else {
          gmargin = last - bv;
        }
      }
    } else {
      // generic: group g's score is held by lane g
      float my_gscore = -INFINITY;
      for (int gg = 0; gg < n_group; ++gg) {
        float m = -INFINITY;
#pragma unroll
        for (int j = 0; j < NV; ++j)
          if (lane + 32 * j < E && (lane + 32 * j) / per == gg && b[j] > m) m = b[j];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == gg) my_gscore = m;
      }
      bool avail = lane < n_group;
      float last = 0.f;
      const int rounds = topk_group < n_group ? topk_group + 1 : topk_group;
      for (int r = 0; r < rounds; ++r) {
        float bv = avail ? my_gscore : -INFINITY;
        int bi = avail ? lane : 0x7fffffff;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
          const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
          if (ov > bv || (ov == bv && oi < bi)) {
            bv = ov;
            bi = oi;
          }
        }
        if (r < topk_group) {
          if (lane == bi) avail = false;
          kept_groups |= 1u << bi;
          last = bv;
        } else {
          gmargin = last - bv;
        }
      }
    }
    uint32_t cand = 0;
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const int e = lane + 32 * j;
      const int g = GJ > 0 ? j / (GJ > 0 ? GJ : 1) : e / per;
      if (e < E && ((kept_groups >> g) & 1u)) cand |= 1u << j;
    }
    // ---- K rounds of warp argmax over candidates (ties -> lower expert id),
    // plus one more for the last gap of the ranking
    int my_e = -1;
    float my_s = 0.f, last_b = 0.f, emargin = INFINITY;
    for (int k = 0; k <= K; ++k) {
      float bv = -INFINITY;
      int be = 0x7fffffff;
#pragma unroll
      for (int j = 0; j < NV; ++j) {
        if (((cand >> j) & 1u) && (be == 0x7fffffff || b[j] > bv)) {
          bv = b[j];
          be = lane + 32 * j;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oe = __shfl_xor_sync(0xffffffffu, be, o);
        if (ov > bv || (ov == bv && oe < be)) {
          bv = ov;
          be = oe;
        }
      }
      if (k > 0 && be != 0x7fffffff) emargin = fminf(emargin, last_b - bv);
      if (k == K) break;
      // owner lane removes the winner and publishes its unbiased score
      const int owner = be & 31, jw = be >> 5;
      float sw = 0.f;
#pragma unroll
      for (int j = 0; j < NV; ++j)
        if (j == jw && lane == owner) {
          sw = s[j];
          cand &= ~(1u << j);
        }
      sw = __shfl_sync(0xffffffffu, sw, owner);
      if (lane == k) {
        my_e = be;
        my_s = sw;
      }
      last_b = bv;
    }
    double den;
    {
      double v = (lane < K) ? static_cast<double>(my_s) : 0.0;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      den = v;  // exact: a sum of K <= 32 fp32 values of similar magnitude
    }
    if (lane < K) {
      const double sk = static_cast<double>(my_s);
      const double wv = renorm ? static_cast<double>(scale) * (sk / den)
                               : static_cast<double>(scale) * sk;
      idx[static_cast<size_t>(t) * K + lane] = my_e;
      wout[static_cast<size_t>(t) * K + lane] = static_cast<float>(wv);
    }
    if (tau > 0.f) {
      // the fp32 logit error grows with the logits' magnitude: scale the margin
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) zz += __shfl_xor_sync(0xffffffffu, zz, o);
      const float tau_t = tau * fmaxf(1.f, sqrtf(zz / E));
      if (lane == 0 && (gmargin < tau_t || emargin < tau_t)) unc[atomicAdd(unc_n, 1)] = t;
    }
  }
}

// ---------------------------------------------------------------------------
// Exact re-derivation of a close fp32 decision, one CTA per listed token.
// With every fp32 biased score within eps = tau_t / 2 of its exact value:
//  1. only groups whose fp32 score is within 2 eps of the (topk_group+1)-th
//     can be kept, and a group's exact maximum comes from its experts within
//     2 eps of its fp32 maximum: those experts get exact scores, and the kept
//     groups are chosen from the exact maxima;
//  2. among the kept groups' experts only those within 2 eps of the (K+1)-th
//     fp32 candidate can be in the exact top K+1: they get exact scores and
//     the K best are taken from them.
// An exact score is the float64 dot product of the bf16 token row with the
// fp32 router row (every product exact in float64), rounded once to fp32,
// then the float64 sigmoid rounded to fp32, plus the bias in fp32: the same
// arithmetic as the reference definition.
// ---------------------------------------------------------------------------
constexpr int kRefineThreads = 128;

template <int NV>
__device__ __forceinline__ void load_scores(const float* zr, const float* bias, int E, int lane,
                                            float* b, float* zz_out) {
  float zv[NV], bv0[NV];
#pragma unroll
  for (int j = 0; j < NV; ++j) zv[j] = zr[min(lane + 32 * j, E - 1)];
#pragma unroll
  for (int j = 0; j < NV; ++j) bv0[j] = bias ? bias[min(lane + 32 * j, E - 1)] : 0.f;
  float zz = 0.f;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const bool in = lane + 32 * j < E;
    if (in) zz = fmaf(zv[j], zv[j], zz);
    b[j] = in ? 1.0f / (1.0f + expf(-zv[j])) + bv0[j] : -INFINITY;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) zz += __shfl_xor_sync(0xffffffffu, zz, o);
  *zz_out = zz;
}

template <int NV>
__global__ void __launch_bounds__(kRefineThreads) router_refine(
    int T, int H, int E, int n_group, int topk_group, int K, float scale, int renorm,
    float tau, const uint16_t* __restrict__ x, const float* __restrict__ Wr,
    const float* __restrict__ z, const float* __restrict__ bias, int32_t* __restrict__ idx,
    float* __restrict__ wout, const int32_t* __restrict__ list,
    const int32_t* __restrict__ list_n) {
  __shared__ __align__(16) uint16_t xs[kRowRegs * 128];
  __shared__ int need[kMaxExperts];
  __shared__ float bex[kMaxExperts], sex[kMaxExperts];
  __shared__ uint32_t done[kMaxExperts / 32];
  __shared__ float gsc[32];
  __shared__ int kept_mask_s, n_need;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n = min(*list_n, T);
  const int per = E / n_group;
  for (int q = blockIdx.x; q < n; q += gridDim.x) {
    const int t = list[q];
    __syncthreads();  // smem of the previous token is no longer in use
    for (int i = tid; i < H / 8; i += blockDim.x)
      reinterpret_cast<uint4*>(xs)[i] = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * H)[i];
    for (int i = tid; i < (E + 31) / 32; i += blockDim.x) done[i] = 0u;
    if (tid == 0) n_need = 0;
    __syncthreads();

    // ---- warp 0: fp32 scores, group scores, the experts that decide group maxima
    float b[NV];
    float tau_t = 0.f, gth = -INFINITY;
    if (warp == 0) {
      float zz;
      load_scores<NV>(z + static_cast<size_t>(t) * E, bias, E, lane, b, &zz);
      tau_t = tau * fmaxf(1.f, sqrtf(zz / E));
      for (int g = 0; g < n_group; ++g) {
        float m = -INFINITY;
#pragma unroll
        for (int j = 0; j < NV; ++j)
          if ((lane + 32 * j) / per == g && b[j] > m) m = b[j];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) gsc[g] = m;
      }
      __syncwarp();
      // (topk_group+1)-th largest fp32 group score
      if (topk_group < n_group) {
        uint32_t taken = 0;
        for (int r = 0; r <= topk_group; ++r) {
          int bi = -1;
          for (int g = 0; g < n_group; ++g)
            if (!((taken >> g) & 1u) && (bi < 0 || gsc[g] > gsc[bi])) bi = g;
          taken |= 1u << bi;
          gth = gsc[bi];
        }
      }
#pragma unroll
      for (int j = 0; j < NV; ++j) {
        const int e = lane + 32 * j;
        bool nd = false;
        if (e < E) {
          const float gs = gsc[e / per];
          nd = gs >= gth - tau_t && b[j] >= gs - tau_t;
        }
        const unsigned bal = __ballot_sync(0xffffffffu, nd);
        const int base = n_need;
        __syncwarp();
        if (nd) need[base + __popc(bal & ((1u << lane) - 1u))] = e;
        __syncwarp();
        if (lane == 0) n_need = base + __popc(bal);
        __syncwarp();
      }
    }
    __syncthreads();

    // ---- exact scores for the listed experts: one warp per expert
    for (int round = 0; round < 2; ++round) {
      const int nn = n_need;
      for (int i = warp; i < nn; i += blockDim.x / 32) {
        const int e = need[i];
        const float* row = Wr + static_cast<size_t>(e) * H;
        float4 wv[kRowRegs];
#pragma unroll
        for (int j = 0; j < kRowRegs; ++j)
          wv[j] = *reinterpret_cast<const float4*>(row + min(4 * lane + 128 * j, H - 4));
        double acc = 0.0;
#pragma unroll
        for (int j = 0; j < kRowRegs; ++j) {
          const int k = 4 * lane + 128 * j;
          if (k < H) {
            const uint2 p = *reinterpret_cast<const uint2*>(xs + k);
            acc = fma(static_cast<double>(wv[j].x), bf16_bits_to_double(p.x & 0xFFFFu), acc);
            acc = fma(static_cast<double>(wv[j].y), bf16_bits_to_double(p.x >> 16), acc);
            acc = fma(static_cast<double>(wv[j].z), bf16_bits_to_double(p.y & 0xFFFFu), acc);
            acc = fma(static_cast<double>(wv[j].w), bf16_bits_to_double(p.y >> 16), acc);
          }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) {
          const float zf = static_cast<float>(acc);
          const float sf = static_cast<float>(1.0 / (1.0 + exp(-static_cast<double>(zf))));
          sex[e] = sf;
          bex[e] = sf + (bias ? bias[e] : 0.f);
          atomicOr(&done[e >> 5], 1u << (e & 31));
        }
      }
      __syncthreads();
      if (round == 1) break;
      // ---- warp 0: kept groups from exact maxima, then the candidates near the cut
      if (warp == 0) {
        // exact maximum of every group that can be kept
        float gex = -INFINITY;  // lane g holds group g's exact maximum
        for (int g = 0; g < n_group; ++g) {
          float m = -INFINITY;
          if (gsc[g] >= gth - tau_t) {
            for (int i = lane; i < nn; i += 32) {
              const int e = need[i];
              if (e / per == g) m = fmaxf(m, bex[e]);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
          }
          if (lane == g) gex = m;
        }
        uint32_t kept = 0;
        for (int r = 0; r < topk_group; ++r) {
          float bv = lane < n_group && !((kept >> lane) & 1u) ? gex : -INFINITY;
          int bi = lane < n_group && !((kept >> lane) & 1u) ? lane : 0x7fffffff;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (ov > bv || (ov == bv && oi < bi)) {
              bv = ov;
              bi = oi;
            }
          }
          kept |= 1u << bi;
        }
        // (K+1)-th largest fp32 score among the kept groups' experts
        uint32_t cand = 0;
#pragma unroll
        for (int j = 0; j < NV; ++j) {
          const int e = lane + 32 * j;
          if (e < E && ((kept >> (e / per)) & 1u)) cand |= 1u << j;
        }
        float bth = -INFINITY;
        {
          uint32_t c2 = cand;
          for (int k = 0; k <= K; ++k) {
            float bv = -INFINITY;
            int be = 0x7fffffff;
#pragma unroll
            for (int j = 0; j < NV; ++j)
              if (((c2 >> j) & 1u) && (be == 0x7fffffff || b[j] > bv)) {
                bv = b[j];
                be = lane + 32 * j;
              }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
              const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
              const int oe = __shfl_xor_sync(0xffffffffu, be, o);
              if (ov > bv || (ov == bv && oe < be)) {
                bv = ov;
                be = oe;
              }
            }
            if (be == 0x7fffffff) break;
            bth = bv;
            if ((be & 31) == lane) c2 &= ~(1u << (be >> 5));
          }
        }
        if (lane == 0) {
          kept_mask_s = static_cast<int>(kept);
          n_need = 0;
        }
        __syncwarp();
        // the final pool C (kept-group experts within 2 eps of the cut) goes to
        // need[]; the ones without an exact score yet are computed next round
#pragma unroll
        for (int j = 0; j < NV; ++j) {
          const int e = lane + 32 * j;
          const bool inC = ((cand >> j) & 1u) && b[j] >= bth - tau_t;
          const unsigned bal = __ballot_sync(0xffffffffu, inC);
          const int base = n_need;
          __syncwarp();
          if (inC) need[base + __popc(bal & ((1u << lane) - 1u))] = e;
          __syncwarp();
          if (lane == 0) n_need = base + __popc(bal);
          __syncwarp();
        }
      }
      __syncthreads();
      // skip experts that already have an exact score (compact the list in place)
      if (warp == 0) {
        const int nc = n_need;
        int m = 0;
        for (int i0 = 0; i0 < nc; i0 += 32) {
          const int i = i0 + lane;
          const int e = i < nc ? need[i] : 0;
          const bool todo = i < nc && !((done[e >> 5] >> (e & 31)) & 1u);
          const unsigned bal = __ballot_sync(0xffffffffu, todo);
          __syncwarp();
          // stash the full pool behind the to-do list: pool in bex-free slots is
          // rebuilt below from `done` and the kept groups, so only the to-do part
          // needs to stay in need[]
          if (todo) need[m + __popc(bal & ((1u << lane) - 1u))] = e;
          m += __popc(bal);
          __syncwarp();
        }
        if (lane == 0) n_need = m;
      }
      __syncthreads();
    }

    // ---- warp 0: final top K over the pool, from exact scores
    if (warp == 0) {
      const uint32_t kept = static_cast<uint32_t>(kept_mask_s);
      // recompute the pool membership (same rule as above) from registers
      uint32_t cand = 0;
#pragma unroll
      for (int j = 0; j < NV; ++j) {
        const int e = lane + 32 * j;
        if (e < E && ((kept >> (e / per)) & 1u)) cand |= 1u << j;
      }
      float bth = -INFINITY;
      {
        uint32_t c2 = cand;
        for (int k = 0; k <= K; ++k) {
          float bv = -INFINITY;
          int be = 0x7fffffff;
#pragma unroll
          for (int j = 0; j < NV; ++j)
            if (((c2 >> j) & 1u) && (be == 0x7fffffff || b[j] > bv)) {
              bv = b[j];
              be = lane + 32 * j;
            }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oe = __shfl_xor_sync(0xffffffffu, be, o);
            if (ov > bv || (ov == bv && oe < be)) {
              bv = ov;
              be = oe;
            }
          }
          if (be == 0x7fffffff) break;
          bth = bv;
          if ((be & 31) == lane) c2 &= ~(1u << (be >> 5));
        }
      }
      uint32_t pool = 0;
#pragma unroll
      for (int j = 0; j < NV; ++j)
        if (((cand >> j) & 1u) && b[j] >= bth - tau_t) pool |= 1u << j;
      int my_e = -1;
      float my_s = 0.f;
      for (int k = 0; k < K; ++k) {
        float bv = -INFINITY;
        int be = 0x7fffffff;
#pragma unroll
        for (int j = 0; j < NV; ++j) {
          if ((pool >> j) & 1u) {
            const float v = bex[lane + 32 * j];
            if (be == 0x7fffffff || v > bv) {
              bv = v;
              be = lane + 32 * j;
            }
          }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
          const int oe = __shfl_xor_sync(0xffffffffu, be, o);
          if (ov > bv || (ov == bv && oe < be)) {
            bv = ov;
            be = oe;
          }
        }
        if ((be & 31) == lane) pool &= ~(1u << (be >> 5));
        if (lane == k) {
          my_e = be;
          my_s = sex[be];
        }
      }
      double v = (lane < K) ? static_cast<double>(my_s) : 0.0;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane < K) {
        const double sk = static_cast<double>(my_s);
        const double wv = renorm ? static_cast<double>(scale) * (sk / v)
                                 : static_cast<double>(scale) * sk;
        idx[static_cast<size_t>(t) * K + lane] = my_e;
        wout[static_cast<size_t>(t) * K + lane] = static_cast<float>(wv);
      }
    }
  }
}

template <int NV, int GJ>
cudaError_t launch_topk(const moe_cfg& c, int T, const float* z, const float* bias, int32_t* idx,
                        float* w, float tau, int32_t* unc, int32_t* unc_n, const int32_t* list,
                        cudaStream_t s) {
  // small batches: one token per CTA, so every token's warp has an SM to itself
  const int warps = T <= 4 * num_sms() ? 1 : 8;
  int grid = cdiv(T, warps);
  if (list) grid = std::min(grid, num_sms() * 4);
  router_topk<NV, GJ><<<grid, warps * 32, 0, s>>>(T, c.E, c.n_group, c.topk_group, c.K, c.scale,
                                                  c.renorm, z, bias, idx, w, tau, unc, unc_n,
                                                  list, list ? unc_n : nullptr);
  return cudaGetLastError();
}

cudaError_t topk_dispatch(const moe_cfg& c, int T, const float* z, const float* bias,
                          int32_t* idx, float* w, float tau, int32_t* unc, int32_t* unc_n,
                          const int32_t* list, cudaStream_t s) {
  const int nv = cdiv(c.E, 32);
  const int per = c.E / c.n_group;
#define SGL_TOPK(NV_)                                                                    \
  if (nv <= NV_) {                                                                       \
    if (c.E == NV_ * 32 && per % 32 == 0 && per / 32 == 2 && NV_ >= 2)                   \
      return launch_topk<NV_, (NV_ >= 2 ? 2 : 1)>(c, T, z, bias, idx, w, tau, unc, unc_n, \
                                                  list, s);                              \
    if (c.E == NV_ * 32 && per % 32 == 0 && per / 32 == 1)                               \
      return launch_topk<NV_, 1>(c, T, z, bias, idx, w, tau, unc, unc_n, list, s);       \
    return launch_topk<NV_, 0>(c, T, z, bias, idx, w, tau, unc, unc_n, list, s);         \
  }
  SGL_TOPK(1)
  SGL_TOPK(2)
  SGL_TOPK(4)
  SGL_TOPK(8)
  SGL_TOPK(16)
  SGL_TOPK(32)
#undef SGL_TOPK
  return cudaErrorInvalidValue;
}

// The fp32 router matrix as three bf16 terms, w = hi + mid + lo: hi is w
// rounded to bf16, mid the rounded remainder, lo the rounded rest; for normal
// values the three 8-bit significands cover all 24 bits of w, so a bf16 token
// times each term is exact in fp32 and the tensor cores can form the fp32
// router product.
__global__ void __launch_bounds__(256) split_router(long long n, const float* __restrict__ w,
                                                    uint16_t* __restrict__ hi,
                                                    uint16_t* __restrict__ mid,
                                                    uint16_t* __restrict__ lo) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float v = w[i];
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    const float r1 = v - __bfloat162float(h);
    const __nv_bfloat16 m = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(m);
    hi[i] = __bfloat16_as_ushort(h);
    mid[i] = __bfloat16_as_ushort(m);
    lo[i] = __bfloat16_as_ushort(__float2bfloat16_rn(r2));
  }
}

template <int NV>
cudaError_t launch_refine_nv(const moe_cfg& c, int T, const uint16_t* x, const float* Wr,
                             const float* z, const float* bias, int32_t* idx, float* w, float tau,
                             const int32_t* list, const int32_t* list_n, cudaStream_t s) {
  const int grid = std::max(1, std::min(T, num_sms() * 4));
  router_refine<NV><<<grid, kRefineThreads, 0, s>>>(T, c.H, c.E, c.n_group, c.topk_group, c.K,
                                                    c.scale, c.renorm, tau, x, Wr, z, bias, idx,
                                                    w, list, list_n);
  return cudaGetLastError();
}

cudaError_t launch_refine(const moe_cfg& c, int T, const uint16_t* x, const float* Wr,
                          const float* z, const float* bias, int32_t* idx, float* w, float tau,
                          const int32_t* list, const int32_t* list_n, cudaStream_t s) {
  const int nv = cdiv(c.E, 32);
  if (nv <= 1) return launch_refine_nv<1>(c, T, x, Wr, z, bias, idx, w, tau, list, list_n, s);
  if (nv <= 2) return launch_refine_nv<2>(c, T, x, Wr, z, bias, idx, w, tau, list, list_n, s);
  if (nv <= 4) return launch_refine_nv<4>(c, T, x, Wr, z, bias, idx, w, tau, list, list_n, s);
  if (nv <= 8) return launch_refine_nv<8>(c, T, x, Wr, z, bias, idx, w, tau, list, list_n, s);
  if (nv <= 16) return launch_refine_nv<16>(c, T, x, Wr, z, bias, idx, w, tau, list, list_n, s);
  return launch_refine_nv<32>(c, T, x, Wr, z, bias, idx, w, tau, list, list_n, s);
}

template <bool EXACT, int ILP>
cudaError_t launch_rows(const moe_cfg& c, int T, const uint16_t* x, const float* Wr, float* z,
                        const int32_t* list, const int32_t* list_n, int32_t* err, cudaStream_t s) {
  const size_t smem = static_cast<size_t>(kSmallT) * c.H * sizeof(uint16_t);
  auto kern = router_logits_rows<EXACT, ILP>;
  cudaError_t e = ensure_dyn_smem(reinterpret_cast<const void*>(kern),
                                  kSmallT * kRowRegs * 128 * static_cast<int>(sizeof(uint16_t)));
  if (e != cudaSuccess) return e;
  kern<<<cdiv(c.E, kRowWarps), kRowWarps * kTokSplit * 32, smem, s>>>(T, c.H, c.E, x, Wr, z, list,
                                                                      list_n,
                                                          err);
  return cudaGetLastError();
}

}  // namespace

// Margin (on biased scores, per unit of logit RMS) below which an fp32
// decision is re-derived from exact logits. A 2560-term fp32 dot product of
// N(0,1) activations and N(0, 1/2560) router weights has a rounding error of
// about 1.2e-6 (one standard deviation), i.e. 3e-7 on a sigmoid score; the
// largest of millions of such errors stays below ~2e-6, a tenth of this.
constexpr float kCertifyMargin = 1.0f / 32768.0f;

cudaError_t launch_router(const moe_cfg& c, int T, const uint16_t* x, const float* Wr,
                          const float* bias, float* z, int32_t* idx, float* w, int32_t* unc,
                          int32_t* unc_n, int32_t* err, uint16_t* wr_split, cudaStream_t s) {
  cudaError_t e;
  if (c.H > kRowRegs * 128) return cudaErrorInvalidValue;
  if (T <= kSmallT) {
    e = launch_rows<false, 4>(c, T, x, Wr, z, nullptr, nullptr, err, s);
  } else if (wr_split != nullptr) {
    // tensor cores: split the router matrix, then one bf16 x 3 GEMM into z
    const long long n = static_cast<long long>(c.E) * c.H;
    uint16_t* hi = wr_split;
    uint16_t* mid = hi + n;
    uint16_t* lo = mid + n;
    split_router<<<num_sms() * 4, 256, 0, s>>>(n, Wr, hi, mid, lo);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    e = launch_router_gemm(c, T, x, hi, mid, lo, z, err, s);
  } else {
    dim3 grid(cdiv(T, kRT), cdiv(c.E, kRE));
    router_logits_tiled<<<grid, 256, 0, s>>>(T, c.H, c.E, x, Wr, z);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) return e;
  if ((e = topk_dispatch(c, T, z, bias, idx, w, kCertifyMargin, unc, unc_n, nullptr, s)) !=
      cudaSuccess)
    return e;
  (void)err;
  return launch_refine(c, T, x, Wr, z, bias, idx, w, kCertifyMargin, unc, unc_n, s);
}

}  // namespace sgl
