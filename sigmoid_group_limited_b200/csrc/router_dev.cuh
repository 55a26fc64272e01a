// router_dev.cuh - device code of the router (stages 1-5) shared by its own
// kernels (router.cu) and the fused decode front (front.cu): constants, the
// order-preserving score keys, and the per-token certified selection and
// exact re-derivation.
//
// Page "Ling-3.0-flash-VL MoE sparse routing" (lqnn.cn/news/282163): sec. 3
// steps 1-3 (sigmoid scores, 8 groups keep 4, top-8, selection bias), sec. 4
// (fp32 router, renormalised weights scaled by 2.5).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "internal.h"
#include "ptx.cuh"

namespace sgl {

// Margin (on biased scores, per unit of logit RMS) below which an fp32
// decision is re-derived from exact logits. A 2560-term fp32 dot product of
// N(0,1) activations and N(0, 1/2560) router weights has a rounding error of
// about 1.2e-6 (one standard deviation), i.e. 3e-7 on a sigmoid score; the
// largest of millions of such errors stays below ~2e-6, a tenth of this.
constexpr float kCertifyMargin = 1.0f / 32768.0f;

namespace {

constexpr int kSmallT = 32;
constexpr int kRowRegs = 24;  // float4 per lane in router_refine: H <= 24 * 128 = 3072
constexpr int kMaxExperts = 1024;
constexpr int kClusterK = 8;                               // CTAs splitting H
constexpr int kSplitE = 32;                                // experts per cluster
constexpr int kMaxChunk = kRowRegs * 128 / kClusterK;      // H <= 3072: 384 columns per CTA
constexpr int kXRow = kMaxChunk + 8;                       // bf16, padded: 8 lanes hit 8 bank groups
constexpr int kLogitsSmem = kSplitE * kMaxChunk * 4 + kSmallT * kXRow * 2 + kSmallT * (kSplitE + 1) * 4;

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

// Order-preserving map of a (non-NaN) float onto nonzero uint32 keys, and back.
__device__ __forceinline__ uint32_t order_key(float v) {
  const uint32_t u = __float_as_uint(v + 0.0f);  // -0 -> +0: equal values, equal keys
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// ---------------------------------------------------------------------------
// The same certified selection with one CTA per token and one warp per
// expert group, for groups of 32 or 64 experts (NG = 1 or 2 per lane), at
// most 16 groups and topk_group * (K+1) <= 64. Warp g scores its group
// (fp32 sigmoid + bias), finds the group maximum and its own top K+1 by
// rounds of warp max over order-preserving keys (ties -> lower expert id);
// warp 0 keeps topk_group groups (ties -> lower group) and ranks the kept
// groups' candidates (the overall top K+1 among the kept groups is among
// them). Margins, weights and the flagged-token list are as in router_topk.
// ---------------------------------------------------------------------------
constexpr int kSelMaxGroups = 16;
constexpr int kSelMaxCand = 33;  // K + 1 <= 33

// One token's selection (all threads of the block call it; warps >= n_group
// only join the barriers). zr: the token's E fp32 logits. Returns whether
// the token was flagged for exact re-derivation (also appended to unc).
template <int NG>
__device__ __forceinline__ bool select_token(int t, const float* __restrict__ zr, int E, int n_group,
                                             int topk_group, int K, float scale, int renorm,
                                             const float* __restrict__ bias, int32_t* __restrict__ idx,
                                             float* __restrict__ wout, float tau,
                                             int32_t* __restrict__ unc, int32_t* __restrict__ unc_n) {
  __shared__ uint32_t gkey[kSelMaxGroups];
  __shared__ float gzz[kSelMaxGroups];
  __shared__ uint32_t ckey[kSelMaxGroups][kSelMaxCand];
  __shared__ int cid[kSelMaxGroups][kSelMaxCand];
  __shared__ float cs[kSelMaxGroups][kSelMaxCand];
  __shared__ int flagged_s;
  const int lane = threadIdx.x & 31, g = threadIdx.x >> 5;
  const int per = 32 * NG, KP1 = K + 1;
  if (g < n_group) {
    float sv[NG];
    uint32_t key[NG];
    float zz = 0.f;
#pragma unroll
    for (int v = 0; v < NG; ++v) {
      const int e = g * per + lane + 32 * v;
      const float zv = zr[e];
      zz = fmaf(zv, zv, zz);
      sv[v] = 1.0f / (1.0f + expf(-zv));
      key[v] = order_key(sv[v] + (bias ? bias[e] : 0.f));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) zz += __shfl_xor_sync(0xffffffffu, zz, o);
    uint32_t mine = key[0];
    int mj = 0;
#pragma unroll
    for (int v = 1; v < NG; ++v)
      if (key[v] > mine) {
        mine = key[v];
        mj = v;
      }
    const uint32_t gmax = __reduce_max_sync(0xffffffffu, mine);
    if (lane == 0) {
      gkey[g] = gmax;
      gzz[g] = zz;
    }
    // this group's top K+1, best first
    uint32_t live = (1u << NG) - 1u;
    for (int r = 0; r < KP1; ++r) {
      const uint32_t mk = __reduce_max_sync(0xffffffffu, live ? mine : 0u);
      const uint32_t wid = __reduce_min_sync(
          0xffffffffu, (live && mine == mk) ? static_cast<uint32_t>(32 * mj + lane) : 0xffffffffu);
      if (wid == 0xffffffffu) {  // fewer candidates than K+1: mark the rest empty
        for (int rr = r + lane; rr < KP1; rr += 32) ckey[g][rr] = 0u;
        break;
      }
      if (lane == static_cast<int>(wid & 31)) {
        ckey[g][r] = mk;
        cid[g][r] = g * per + static_cast<int>(wid);
        cs[g][r] = sv[mj];
        live &= ~(1u << mj);
        mine = 0u;
#pragma unroll
        for (int v = 0; v < NG; ++v)
          if (((live >> v) & 1u) && key[v] > mine) {
            mine = key[v];
            mj = v;
          }
      }
    }
  }
  __syncthreads();
  if (g == 0) {
    // groups: lane gg holds group gg's maximum
    uint32_t gk = lane < n_group ? gkey[lane] : 0u;
    bool avail = lane < n_group;
    uint32_t kept = 0;
    float last = 0.f, gmargin = INFINITY;
    const int rounds = topk_group < n_group ? topk_group + 1 : topk_group;
    for (int r = 0; r < rounds; ++r) {
      const uint32_t mk = __reduce_max_sync(0xffffffffu, avail ? gk : 0u);
      const int gi = static_cast<int>(__reduce_min_sync(
          0xffffffffu, (avail && gk == mk) ? static_cast<uint32_t>(lane) : 0xffffffffu));
      if (r < topk_group) {
        kept |= 1u << gi;
        if (lane == gi) avail = false;
        last = key_value(mk);
      } else {
        gmargin = last - key_value(mk);
      }
    }
    // candidates of the kept groups, two slots per lane
    uint32_t k2[2];
    int i2[2];
    float s2[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int slot = lane + 32 * h;  // candidate number in kept-group order
      k2[h] = 0u;
      i2[h] = 0;
      s2[h] = 0.f;
      const int gsel = slot / KP1, r = slot - gsel * KP1;
      if (gsel < topk_group) {
        // the gsel-th kept group, in increasing group order
        uint32_t m = kept;
        for (int q = 0; q < gsel; ++q) m &= m - 1u;
        const int gg = __ffs(m) - 1;
        k2[h] = ckey[gg][r];
        i2[h] = cid[gg][r];
        s2[h] = cs[gg][r];
      }
    }
    int my_e = -1;
    float my_s = 0.f, last_b = 0.f, emargin = INFINITY;
    for (int k = 0; k <= K; ++k) {
      const uint32_t mine = k2[0] > k2[1] || (k2[0] == k2[1] && i2[0] < i2[1]) ? k2[0] : k2[1];
      const int mh = (k2[0] > k2[1] || (k2[0] == k2[1] && i2[0] < i2[1])) ? 0 : 1;
      const uint32_t mk = __reduce_max_sync(0xffffffffu, mine);
      if (mk == 0u) break;
      const uint32_t we = __reduce_min_sync(
          0xffffffffu, mine == mk ? static_cast<uint32_t>(mh ? i2[1] : i2[0]) : 0xffffffffu);
      const float bv = key_value(mk);
      if (k > 0) emargin = fminf(emargin, last_b - bv);
      if (k == K) break;
      float sw = 0.f;
      const bool own = mine == mk && static_cast<uint32_t>(mh ? i2[1] : i2[0]) == we;
      if (own) {
        sw = mh ? s2[1] : s2[0];
        if (mh) k2[1] = 0u;
        else k2[0] = 0u;
      }
      const unsigned ob = __ballot_sync(0xffffffffu, own);
      sw = __shfl_sync(0xffffffffu, sw, __ffs(ob) - 1);
      if (lane == k) {
        my_e = static_cast<int>(we);
        my_s = sw;
      }
      last_b = bv;
    }
    double den = (lane < K) ? static_cast<double>(my_s) : 0.0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    if (lane < K) {
      const double sk = static_cast<double>(my_s);
      const double wv = renorm ? static_cast<double>(scale) * (sk / den)
                               : static_cast<double>(scale) * sk;
      idx[static_cast<size_t>(t) * K + lane] = my_e;
      wout[static_cast<size_t>(t) * K + lane] = static_cast<float>(wv);
    }
    if (lane == 0) {
      float zz = 0.f;
      for (int q = 0; q < n_group; ++q) zz += gzz[q];
      const float tau_t = tau * fmaxf(1.f, sqrtf(zz / E));
      const bool flag = gmargin < tau_t || emargin < tau_t;
      if (flag) unc[atomicAdd(unc_n, 1)] = t;
      flagged_s = flag ? 1 : 0;
    }
  }
  __syncthreads();
  const bool flagged = flagged_s != 0;
  __syncthreads();  // shared candidates and the flag are reused by the next token
  return flagged;
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
constexpr int kRefineThreads = 256;  // 8 warps: exact scores of 8 experts at a time

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

// Value of the kth candidate (1-based) in the ranking by biased score, ties
// to the lower expert id; the last one found if there are fewer. Each lane
// keeps its own best; a round is a warp max of the keys, then the lowest id
// among the lanes holding it, and only the winning lane rescans.
template <int NV>
__device__ __forceinline__ float kth_candidate_value(uint32_t cand, const float* b, int kth,
                                                     int lane) {
  uint32_t lkey = 0u;
  int lj = 0;
  auto rescan = [&]() {
    lkey = 0u;
    float bv = -INFINITY;
#pragma unroll
    for (int j = 0; j < NV; ++j)
      if (((cand >> j) & 1u) && (lkey == 0u || b[j] > bv)) {
        bv = b[j];
        lj = j;
        lkey = order_key(bv);
      }
  };
  rescan();
  float v = -INFINITY;
  for (int k = 0; k < kth; ++k) {
    const uint32_t mk = __reduce_max_sync(0xffffffffu, lkey);
    if (mk == 0u) break;
    const uint32_t be = __reduce_min_sync(
        0xffffffffu, (lkey == mk) ? static_cast<uint32_t>(lj * 32 + lane) : 0xffffffffu);
    v = key_value(mk);
    if (lane == static_cast<int>(be & 31)) {
      cand &= ~(1u << (be >> 5));
      rescan();
    }
  }
  return v;
}

// Exact re-derivation of token t's decision (all threads of the block call
// it; blockDim.x a multiple of 32, at least 64).
template <int NV>
__device__ __forceinline__ void refine_token(int t, int H, int E, int n_group, int topk_group,
                                             int K, float scale, int renorm, float tau,
                                             const uint16_t* __restrict__ x,
                                             const float* __restrict__ Wr,
                                             const float* __restrict__ z,
                                             const float* __restrict__ bias,
                                             int32_t* __restrict__ idx, float* __restrict__ wout) {
  __shared__ __align__(16) uint16_t xs[kRowRegs * 128];
  __shared__ int need[kMaxExperts];
  __shared__ float bex[kMaxExperts], sex[kMaxExperts];
  __shared__ uint32_t done[kMaxExperts / 32];
  __shared__ float gsc[32];
  __shared__ int kept_mask_s, n_need;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int per = E / n_group;
  __syncthreads();  // smem of the previous token is no longer in use
  for (int i = tid; i < H / 8; i += blockDim.x)
    reinterpret_cast<uint4*>(xs)[i] = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * H)[i];
  for (int i = tid; i < (E + 31) / 32; i += blockDim.x) done[i] = 0u;
  if (tid == 0) n_need = 0;
  __syncthreads();

  // ---- warp 0: fp32 scores, group scores, the experts that decide group maxima
  float b[NV];
  int gj[NV];  // group of register slot j (-1 past E)
  float tau_t = 0.f, gth = -INFINITY;
  if (warp == 0) {
    float zz;
    load_scores<NV>(z + static_cast<size_t>(t) * E, bias, E, lane, b, &zz);
    tau_t = tau * fmaxf(1.f, sqrtf(zz / E));
#pragma unroll
    for (int j = 0; j < NV; ++j) gj[j] = lane + 32 * j < E ? (lane + 32 * j) / per : -1;
    for (int g = 0; g < n_group; ++g) {
      float m = -INFINITY;
#pragma unroll
      for (int j = 0; j < NV; ++j)
        if (gj[j] == g && b[j] > m) m = b[j];
      m = key_value(__reduce_max_sync(0xffffffffu, order_key(m)));
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
        const float gs = gsc[gj[j]];
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
      // every product is exact in float64; four independent float64 sums keep
      // the FMA units busy, then a fixed tree adds them
      double a4[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
      for (int j = 0; j < kRowRegs; ++j) {
        const int k = 4 * lane + 128 * j;
        if (k < H) {
          const uint2 p = *reinterpret_cast<const uint2*>(xs + k);
          a4[0] = fma(static_cast<double>(wv[j].x), bf16_bits_to_double(p.x & 0xFFFFu), a4[0]);
          a4[1] = fma(static_cast<double>(wv[j].y), bf16_bits_to_double(p.x >> 16), a4[1]);
          a4[2] = fma(static_cast<double>(wv[j].z), bf16_bits_to_double(p.y & 0xFFFFu), a4[2]);
          a4[3] = fma(static_cast<double>(wv[j].w), bf16_bits_to_double(p.y >> 16), a4[3]);
        }
      }
      double acc = (a4[0] + a4[1]) + (a4[2] + a4[3]);
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
          m = key_value(__reduce_max_sync(0xffffffffu, order_key(m)));
        }
        if (lane == g) gex = m;
      }
      uint32_t kept = 0;
      for (int r = 0; r < topk_group; ++r) {
        // best remaining group, ties to the lower group
        const bool avail = lane < n_group && !((kept >> lane) & 1u);
        const uint32_t mk = __reduce_max_sync(0xffffffffu, avail ? order_key(gex) : 0u);
        const uint32_t bi = __reduce_min_sync(
            0xffffffffu, (avail && order_key(gex) == mk) ? static_cast<uint32_t>(lane) : 0xffffffffu);
        kept |= 1u << bi;
      }
      // (K+1)-th largest fp32 score among the kept groups' experts
      uint32_t cand = 0;
#pragma unroll
      for (int j = 0; j < NV; ++j)
        if (gj[j] >= 0 && ((kept >> gj[j]) & 1u)) cand |= 1u << j;
      const float bth = kth_candidate_value<NV>(cand, b, K + 1, lane);
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
    for (int j = 0; j < NV; ++j)
      if (gj[j] >= 0 && ((kept >> gj[j]) & 1u)) cand |= 1u << j;
    const float bth = kth_candidate_value<NV>(cand, b, K + 1, lane);
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
      // best remaining pool member by exact score, ties to the lower expert id
      const uint32_t lk = be != 0x7fffffff ? order_key(bv) : 0u;
      const uint32_t mk = __reduce_max_sync(0xffffffffu, lk);
      be = static_cast<int>(__reduce_min_sync(
          0xffffffffu, (lk != 0u && lk == mk) ? static_cast<uint32_t>(be) : 0xffffffffu));
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
  __syncthreads();  // shared memory is reused by the next token
}

}  // namespace
}  // namespace sgl
