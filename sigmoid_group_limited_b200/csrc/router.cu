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
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "internal.h"

namespace sgl {
namespace {

__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// ---------------------------------------------------------------------------
// Logits for small batches (T <= 32): one warp per expert. The tokens sit in
// shared memory as bf16; each lane holds a strided slice of the expert's
// fp32 router row in registers and accumulates lane partial sums in fp32,
// finished by a butterfly sum across the warp.
// ---------------------------------------------------------------------------
constexpr int kSmallT = 32;
constexpr int kRowRegs = 24;  // float4 per lane: H <= 24 * 128 = 3072

__global__ void __launch_bounds__(256) router_logits_small(int T, int H, int E,
                                                           const uint16_t* __restrict__ x,
                                                           const float* __restrict__ Wr,
                                                           float* __restrict__ z) {
  extern __shared__ __align__(16) uint16_t xs[];  // [T][H]
  const int tid = threadIdx.x;
  {
    const int n16 = T * H / 8;  // 16-byte chunks
    const uint4* src = reinterpret_cast<const uint4*>(x);
    uint4* dst = reinterpret_cast<uint4*>(xs);
    for (int i = tid; i < n16; i += blockDim.x) dst[i] = src[i];
  }
  __syncthreads();
  const int warp = tid >> 5, lane = tid & 31;
  const int e = blockIdx.x * 8 + warp;
  if (e >= E) return;
  const float* row = Wr + static_cast<size_t>(e) * H;
  float4 wv[kRowRegs];
#pragma unroll
  for (int j = 0; j < kRowRegs; ++j) {
    const int k = 4 * lane + 128 * j;
    wv[j] = (k < H) ? *reinterpret_cast<const float4*>(row + k) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  for (int t = 0; t < T; ++t) {
    const uint16_t* xr = xs + t * H;
    float acc = 0.f;
#pragma unroll
    for (int j = 0; j < kRowRegs; ++j) {
      const int k = 4 * lane + 128 * j;
      if (k < H) {
        const uint2 p = *reinterpret_cast<const uint2*>(xr + k);
        acc = fmaf(wv[j].x, __uint_as_float(p.x << 16), acc);
        acc = fmaf(wv[j].y, __uint_as_float(p.x & 0xFFFF0000u), acc);
        acc = fmaf(wv[j].z, __uint_as_float(p.y << 16), acc);
        acc = fmaf(wv[j].w, __uint_as_float(p.y & 0xFFFF0000u), acc);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) z[static_cast<size_t>(t) * E + e] = acc;
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
// e = l + 32*j. Scores use a float64 sigmoid rounded to fp32; the weights are
// computed in float64 from the fp32 scores and rounded once.
// ---------------------------------------------------------------------------
template <int NV>
__global__ void __launch_bounds__(256) router_topk(int T, int E, int n_group, int topk_group,
                                                   int K, float scale, int renorm,
                                                   const float* __restrict__ z,
                                                   const float* __restrict__ bias,
                                                   int32_t* __restrict__ idx,
                                                   float* __restrict__ wout) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  const int per = E / n_group;
  const float* zr = z + static_cast<size_t>(t) * E;
  float s[NV], b[NV];
  int g[NV];
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int e = lane + 32 * j;
    if (e < E) {
      const float zz = zr[e];
      s[j] = static_cast<float>(1.0 / (1.0 + exp(-static_cast<double>(zz))));
      b[j] = s[j] + (bias ? bias[e] : 0.f);
      g[j] = e / per;
    } else {
      s[j] = 0.f;
      b[j] = -INFINITY;
      g[j] = -1;
    }
  }
  // group score (max of b) held by lane g
  float my_gscore = -INFINITY;
  for (int gg = 0; gg < n_group; ++gg) {
    float m = -INFINITY;
#pragma unroll
    for (int j = 0; j < NV; ++j)
      if (g[j] == gg && b[j] > m) m = b[j];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float other = __shfl_xor_sync(0xffffffffu, m, o);
      m = other > m ? other : m;
    }
    if (lane == gg) my_gscore = m;
  }
  // keep topk_group groups: repeated argmax over lanes < n_group, ties -> lower lane
  bool my_kept = false;
  {
    float v = lane < n_group ? my_gscore : -INFINITY;
    bool avail = lane < n_group;
    for (int r = 0; r < topk_group; ++r) {
      float bv = avail ? v : -INFINITY;
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
      if (lane == bi) {
        my_kept = true;
        avail = false;
      }
    }
  }
  uint32_t cand = 0;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int src = g[j] < 0 ? 0 : g[j];
    const bool k = __shfl_sync(0xffffffffu, my_kept ? 1 : 0, src) != 0;
    if (k && g[j] >= 0) cand |= 1u << j;
  }
  // K rounds of warp argmax over candidates (ties -> lower expert id)
  int my_e = -1;
  float my_s = 0.f;
  for (int k = 0; k < K; ++k) {
    float bv = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      if ((cand >> j) & 1u) {
        if (b[j] > bv || be == 0x7fffffff) {
          bv = b[j];
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
  }
  double den = 0.0;
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
}

template <int NV>
cudaError_t launch_topk(const moe_cfg& c, int T, const float* z, const float* bias, int32_t* idx,
                        float* w, cudaStream_t s) {
  const int warps = 8;
  router_topk<NV><<<cdiv(T, warps), warps * 32, 0, s>>>(T, c.E, c.n_group, c.topk_group, c.K,
                                                        c.scale, c.renorm, z, bias, idx, w);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_router(const moe_cfg& c, int T, const uint16_t* x, const float* Wr,
                          const float* bias, float* z, int32_t* idx, float* w, cudaStream_t s) {
  if (T <= kSmallT && c.H <= kRowRegs * 128) {
    const size_t smem = static_cast<size_t>(T) * c.H * sizeof(uint16_t);
    static bool attr_set = false;
    if (!attr_set) {
      cudaFuncSetAttribute(router_logits_small, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kSmallT * kRowRegs * 128 * 2);
      attr_set = true;
    }
    router_logits_small<<<cdiv(c.E, 8), 256, smem, s>>>(T, c.H, c.E, x, Wr, z);
  } else {
    dim3 grid(cdiv(T, kRT), cdiv(c.E, kRE));
    router_logits_tiled<<<grid, 256, 0, s>>>(T, c.H, c.E, x, Wr, z);
  }
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const int nv = cdiv(c.E, 32);
  if (nv <= 1) return launch_topk<1>(c, T, z, bias, idx, w, s);
  if (nv <= 2) return launch_topk<2>(c, T, z, bias, idx, w, s);
  if (nv <= 4) return launch_topk<4>(c, T, z, bias, idx, w, s);
  if (nv <= 8) return launch_topk<8>(c, T, z, bias, idx, w, s);
  if (nv <= 16) return launch_topk<16>(c, T, z, bias, idx, w, s);
  return launch_topk<32>(c, T, z, bias, idx, w, s);
}

}  // namespace sgl
