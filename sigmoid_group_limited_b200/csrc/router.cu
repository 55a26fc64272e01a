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
#include "router_dev.cuh"

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

template <int NG>
__global__ void __launch_bounds__(kSelMaxGroups * 32) router_select(
    int T, int E, int n_group, int topk_group, int K, float scale, int renorm,
    const float* __restrict__ z, const float* __restrict__ bias, int32_t* __restrict__ idx,
    float* __restrict__ wout, float tau, int32_t* __restrict__ unc, int32_t* __restrict__ unc_n) {
  pdl_trigger();
  pdl_wait();  // inputs come from earlier kernels on the stream
  for (int t = blockIdx.x; t < T; t += gridDim.x)
    select_token<NG>(t, z + static_cast<size_t>(t) * E, E, n_group, topk_group, K, scale, renorm,
                     bias, idx, wout, tau, unc, unc_n);
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
  const int n = min(*list_n, T);
  for (int q = blockIdx.x; q < n; q += gridDim.x)
    refine_token<NV>(list[q], H, E, n_group, topk_group, K, scale, renorm, tau, x, Wr, z, bias, idx,
                     wout);
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
