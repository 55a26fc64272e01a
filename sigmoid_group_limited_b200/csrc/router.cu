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
// Logits for small batches (T <= 32), split over K inside thread-block
// clusters: cluster b (8 CTAs) owns experts [32 b, 32 b + 32); CTA r of it
// forms the fp32 partial dot products of all tokens with those experts over
// hidden columns [r C, r C + C), C = H / 8 rounded up to 64. Lane t of every
// warp is token t, the block's router rows sit in shared memory and are read
// as broadcasts, and warp w accumulates experts 4w .. 4w+3: no cross-lane
// reduction. The eight partials are then added in rank order through
// distributed shared memory, each CTA finishing 4 of the 32 tokens, so z is
// the same whichever CTA finishes first.
// ---------------------------------------------------------------------------
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

__global__ void __cluster_dims__(kClusterK, 1, 1) __launch_bounds__(256)
    router_logits_cluster(int T, int H, int E, const uint16_t* __restrict__ x,
                          const float* __restrict__ Wr, float* __restrict__ z) {
  pdl_trigger();
  extern __shared__ __align__(16) uint8_t lsm[];
  float* ws = reinterpret_cast<float*>(lsm);                                  // [32][kMaxChunk]
  uint16_t* xs = reinterpret_cast<uint16_t*>(ws + kSplitE * kMaxChunk);       // [32][kXRow]
  float* out = reinterpret_cast<float*>(xs + kSmallT * kXRow);                // [32][33]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t r = cluster_ctarank();
  const int e0 = blockIdx.y * kSplitE;
  const int chunk = ((H / 64 + kClusterK - 1) / kClusterK) * 64;
  const int k0 = static_cast<int>(r) * chunk;
  const int kn = max(0, min(chunk, H - k0));  // a multiple of 64, possibly 0
  pdl_wait();  // x may come from an earlier kernel on the stream
  // the block's router rows and the batch's token columns, all copies in flight
  const uint64_t pol = policy_evict_first();
  for (int i = tid; i < kSplitE * (kMaxChunk / 4); i += blockDim.x) {
    const int row = i / (kMaxChunk / 4), c = 4 * (i % (kMaxChunk / 4));
    float* dst = ws + row * kMaxChunk + c;
    if (c < kn && e0 + row < E)
      cp_async16(dst, Wr + static_cast<size_t>(e0 + row) * H + k0 + c, pol);
    else
      *reinterpret_cast<float4*>(dst) = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  const uint64_t pol_x = policy_evict_last();
  for (int i = tid; i < kSmallT * (kMaxChunk / 8); i += blockDim.x) {
    const int row = i / (kMaxChunk / 8), c = 8 * (i % (kMaxChunk / 8));
    uint16_t* dst = xs + row * kXRow + c;
    if (row < T && c < kn)
      cp_async16(dst, x + static_cast<size_t>(row) * H + k0 + c, pol_x);
    else
      *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
  }
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();
  constexpr int EW = kSplitE / 8;  // experts per warp
  float acc[EW];
#pragma unroll
  for (int q = 0; q < EW; ++q) acc[q] = 0.f;
#pragma unroll 4
  for (int i = 0; i < kn / 8; ++i) {
    const uint4 xv8 = *reinterpret_cast<const uint4*>(xs + lane * kXRow + 8 * i);
    const uint32_t pk[4] = {xv8.x, xv8.y, xv8.z, xv8.w};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float xv0 = __uint_as_float(pk[2 * h] << 16);
      const float xv1 = __uint_as_float(pk[2 * h] & 0xFFFF0000u);
      const float xv2 = __uint_as_float(pk[2 * h + 1] << 16);
      const float xv3 = __uint_as_float(pk[2 * h + 1] & 0xFFFF0000u);
#pragma unroll
      for (int q = 0; q < EW; ++q) {
        const float4 wv = *reinterpret_cast<const float4*>(ws + (warp * EW + q) * kMaxChunk + 8 * i + 4 * h);
        acc[q] = fmaf(xv0, wv.x, acc[q]);
        acc[q] = fmaf(xv1, wv.y, acc[q]);
        acc[q] = fmaf(xv2, wv.z, acc[q]);
        acc[q] = fmaf(xv3, wv.w, acc[q]);
      }
    }
  }
#pragma unroll
  for (int q = 0; q < EW; ++q) out[lane * (kSplitE + 1) + warp * EW + q] = acc[q];
  cluster_sync();  // every CTA's partials are in its shared memory
  // CTA r adds tokens 4r .. 4r+3 over the eight partials, in rank order
  if (tid < (kSmallT / kClusterK) * kSplitE) {
    const int t = static_cast<int>(r) * (kSmallT / kClusterK) + tid / kSplitE, c = tid % kSplitE;
    const uint32_t loc = smem_u32(out + t * (kSplitE + 1) + c);
    float sum = 0.f;
#pragma unroll
    for (int q = 0; q < kClusterK; ++q) sum += ld_shared_cluster_f32(mapa_shared(loc, q));
    if (t < T && e0 + c < E) z[static_cast<size_t>(t) * E + e0 + c] = sum;
  }
  cluster_sync();  // no CTA exits while another may still read its partials
}

// Order-preserving map of a (non-NaN) float onto nonzero uint32 keys, and back.
__device__ __forceinline__ uint32_t order_key(float v) {
  const uint32_t u = __float_as_uint(v + 0.0f);  // -0 -> +0: equal values, equal keys
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

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
  pdl_trigger();
  pdl_wait();  // inputs come from earlier kernels on the stream
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
    for (int j = 0; j < NV; ++j) bv0[j] = bias ? bias[min(lane + 32 * j, E - 1)] : 0.f;
#pragma unroll
    for (int j = 0; j < NV; ++j) zv[j] = zr[min(lane + 32 * j, E - 1)];
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
      for (int g = 0; g < G; ++g)
        gs[g] = key_value(__reduce_max_sync(0xffffffffu, order_key(gs[g])));
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
    // plus one more for the last gap of the ranking. Each lane keeps its own
    // best candidate (lowest j among equals, i.e. lowest expert id); a round
    // is a warp max of the order-preserving keys, then the lowest expert id
    // among the lanes that hold that key, and only the winning lane rescans.
    int my_e = -1;
    float my_s = 0.f, last_b = 0.f, emargin = INFINITY;
    uint32_t lkey = 0u;  // 0: no candidate left in this lane
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
    for (int k = 0; k <= K; ++k) {
      const uint32_t mkey = __reduce_max_sync(0xffffffffu, lkey);
      const uint32_t be_u = __reduce_min_sync(
          0xffffffffu, (lkey == mkey && lkey != 0u) ? static_cast<uint32_t>(lj * 32 + lane) : 0xffffffffu);
      if (be_u == 0xffffffffu) break;  // no candidate left
      const int be = static_cast<int>(be_u);
      const float bv = key_value(mkey);
      if (k > 0) emargin = fminf(emargin, last_b - bv);
      if (k == K) break;
      // owner lane removes the winner and publishes its unbiased score
      const int owner = be & 31, jw = be >> 5;
      float sw = 0.f;
      if (lane == owner) {
#pragma unroll
        for (int j = 0; j < NV; ++j)
          if (j == jw) sw = s[j];
        cand &= ~(1u << jw);
        rescan();
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

template <int NG>
__global__ void __launch_bounds__(kSelMaxGroups * 32) router_select(
    int T, int E, int n_group, int topk_group, int K, float scale, int renorm,
    const float* __restrict__ z, const float* __restrict__ bias, int32_t* __restrict__ idx,
    float* __restrict__ wout, float tau, int32_t* __restrict__ unc, int32_t* __restrict__ unc_n) {
  pdl_trigger();
  pdl_wait();  // inputs come from earlier kernels on the stream
  __shared__ uint32_t gkey[kSelMaxGroups];
  __shared__ float gzz[kSelMaxGroups];
  __shared__ uint32_t ckey[kSelMaxGroups][kSelMaxCand];
  __shared__ int cid[kSelMaxGroups][kSelMaxCand];
  __shared__ float cs[kSelMaxGroups][kSelMaxCand];
  const int lane = threadIdx.x & 31, g = threadIdx.x >> 5;
  const int per = 32 * NG, KP1 = K + 1;
  for (int t = blockIdx.x; t < T; t += gridDim.x) {
    const float* zr = z + static_cast<size_t>(t) * E;
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
        if (gmargin < tau_t || emargin < tau_t) unc[atomicAdd(unc_n, 1)] = t;
      }
    }
    __syncthreads();  // shared candidates are reused by the next token
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

template <int NV>
__global__ void __launch_bounds__(kRefineThreads) router_refine(
    int T, int H, int E, int n_group, int topk_group, int K, float scale, int renorm,
    float tau, const uint16_t* __restrict__ x, const float* __restrict__ Wr,
    const float* __restrict__ z, const float* __restrict__ bias, int32_t* __restrict__ idx,
    float* __restrict__ wout, const int32_t* __restrict__ list,
    const int32_t* __restrict__ list_n) {
  pdl_trigger();
  pdl_wait();  // inputs come from earlier kernels on the stream
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
  }
}

template <int NV, int GJ>
cudaError_t launch_topk(const moe_cfg& c, int T, const float* z, const float* bias, int32_t* idx,
                        float* w, float tau, int32_t* unc, int32_t* unc_n, cudaStream_t s) {
  // small batches: one token per CTA, so every token's warp has an SM to itself
  const int warps = T <= 4 * num_sms() ? 1 : 8;
  const int grid = cdiv(T, warps);
  return launch_pdl(router_topk<NV, GJ>, dim3(grid), dim3(warps * 32), 0, s, T, c.E, c.n_group,
                    c.topk_group, c.K, c.scale, c.renorm, z, bias, idx, w, tau, unc, unc_n,
                    static_cast<const int32_t*>(nullptr), static_cast<const int32_t*>(nullptr));
}

cudaError_t topk_dispatch(const moe_cfg& c, int T, const float* z, const float* bias,
                          int32_t* idx, float* w, float tau, int32_t* unc, int32_t* unc_n,
                          cudaStream_t s) {
  const int nv = cdiv(c.E, 32);
  const int per = c.E / c.n_group;
  // small batches: a CTA per token (its groups in parallel); larger ones keep
  // the warp per token, which has more tokens in flight per SM
  if (T <= 4 * num_sms() && (per == 32 || per == 64) && c.n_group <= kSelMaxGroups &&
      c.K + 1 <= kSelMaxCand && c.topk_group * (c.K + 1) <= 64) {
    const int grid = T;
    auto kern = per == 32 ? router_select<1> : router_select<2>;
    return launch_pdl(kern, dim3(grid), dim3(c.n_group * 32), 0, s, T, c.E, c.n_group,
                      c.topk_group, c.K, c.scale, c.renorm, z, bias, idx, w, tau, unc, unc_n);
  }
#define SGL_TOPK(NV_)                                                                   \
  if (nv <= NV_) {                                                                      \
    if (c.E == NV_ * 32 && per % 32 == 0 && per / 32 == 2 && NV_ >= 2)                  \
      return launch_topk<NV_, (NV_ >= 2 ? 2 : 1)>(c, T, z, bias, idx, w, tau, unc, unc_n, s); \
    if (c.E == NV_ * 32 && per % 32 == 0 && per / 32 == 1)                              \
      return launch_topk<NV_, 1>(c, T, z, bias, idx, w, tau, unc, unc_n, s);            \
    return launch_topk<NV_, 0>(c, T, z, bias, idx, w, tau, unc, unc_n, s);              \
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
  pdl_trigger();
  pdl_wait();  // inputs come from earlier kernels on the stream
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
  return launch_pdl(router_refine<NV>, dim3(grid), dim3(kRefineThreads), 0, s, T, c.H, c.E,
                    c.n_group, c.topk_group, c.K, c.scale, c.renorm, tau, x, Wr, z, bias, idx, w,
                    list, list_n);
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
    // fp32 split-K logits in clusters of kClusterK CTAs
    e = ensure_dyn_smem(reinterpret_cast<const void*>(router_logits_cluster), kLogitsSmem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(router_logits_cluster, dim3(kClusterK, cdiv(c.E, kSplitE)), dim3(256),
                   static_cast<size_t>(kLogitsSmem), s, T, c.H, c.E, x, Wr, z);
  } else {
    // tensor cores: split the router matrix, then one bf16 x 3 GEMM into z
    if (wr_split == nullptr) return cudaErrorInvalidValue;
    const long long n = static_cast<long long>(c.E) * c.H;
    uint16_t* hi = wr_split;
    uint16_t* mid = hi + n;
    uint16_t* lo = mid + n;
    if ((e = launch_pdl(split_router, dim3(num_sms() * 4), dim3(256), 0, s, n, Wr, hi, mid, lo)) !=
        cudaSuccess)
      return e;
    e = launch_router_gemm(c, T, x, hi, mid, lo, z, err, s);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = topk_dispatch(c, T, z, bias, idx, w, kCertifyMargin, unc, unc_n, s)) != cudaSuccess)
    return e;
  return launch_refine(c, T, x, Wr, z, bias, idx, w, kCertifyMargin, unc, unc_n, s);
}

}  // namespace sgl
