// mxfp4.cu - routed expert weights stored as MXFP4 (page "Ling-3.0-flash-VL
// 42-layer hybrid backbone", lpnh.cn/news/2815793, spec table: the routed
// experts' weights are 4-bit), format per the OCP Microscaling spec: e2m1
// codes, two per byte (element 2j in the low nibble), one e8m0 scale per 32
// consecutive elements along K.
//
// The layer uses the exact values code * 2^(scale - 127): every such value
// has at most two significant bits, so it is exact in bf16. Each expert that
// the batch touches is dequantised once per forward into a compact bf16
// copy (slot order), which the bf16 grouped GEMMs then read through an
// expert -> slot map.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"
#include "ptx.cuh"

namespace sgl {
namespace {

// Touched experts in increasing id order: slot_of[e] (-1 when untouched),
// touched[slot] = e, ntouched[0] = count. One CTA of 1024 threads.
__global__ void __launch_bounds__(1024) mxfp4_slots(int E, const int32_t* __restrict__ offsets,
                                                    int32_t* __restrict__ slot_of,
                                                    int32_t* __restrict__ touched,
                                                    int32_t* __restrict__ ntouched) {
  pdl_trigger();
  pdl_wait();  // inputs come from earlier kernels on the stream
  __shared__ int wsum[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int base = 0;
  for (int e0 = 0; e0 < E; e0 += blockDim.x) {
    const int e = e0 + tid;
    const bool t = e < E && offsets[e + 1] > offsets[e];
    const unsigned bal = __ballot_sync(0xffffffffu, t);
    if (lane == 0) wsum[warp] = __popc(bal);
    __syncthreads();
    int before = 0, total = 0;
    for (int w = 0; w < 32; ++w) {
      before += w < warp ? wsum[w] : 0;
      total += wsum[w];
    }
    const int slot = base + before + __popc(bal & ((1u << lane) - 1u));
    if (e < E) slot_of[e] = t ? slot : -1;
    if (t) touched[slot] = e;
    base += total;
    __syncthreads();
  }
  if (tid == 0) *ntouched = base;
}

// 8 codes (one 32-bit word) -> 8 bf16 (16 bytes) at scale 2^(s - 127).
__device__ __forceinline__ uint4 dequant8(uint32_t codes, uint32_t s) {
  // 2^(s-127) as an fp32 (s == 0 is the subnormal 2^-127)
  const float scale = s == 0 ? __uint_as_float(0x00400000u) : __uint_as_float(s << 23);
  uint32_t out[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t h[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const uint32_t c = (codes >> (8 * i + 4 * k)) & 0xFu;
      const uint32_t m = c & 7u;
      // e2m1 magnitude as fp32 bits: 0, 0.5, then (1 + m0/2) * 2^(e-1)
      const uint32_t mb = m == 0u ? 0u
                          : m == 1u ? (126u << 23)
                                    : (((m >> 1) + 126u) << 23) | ((m & 1u) << 22);
      float v = __uint_as_float(mb) * scale;
      if (c & 8u) v = -v;
      h[k] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
    }
    out[i] = h[0] | (h[1] << 16);
  }
  return make_uint4(out[0], out[1], out[2], out[3]);
}

// Dequantise the three matrices of every touched expert into slot order.
// Unit u = 8 consecutive elements of one matrix row.
__global__ void __launch_bounds__(256) mxfp4_dequant(
    int I, int H, const int32_t* __restrict__ touched, const int32_t* __restrict__ ntouched,
    const uint8_t* __restrict__ gq, const uint8_t* __restrict__ gs,
    const uint8_t* __restrict__ uq, const uint8_t* __restrict__ us,
    const uint8_t* __restrict__ dq, const uint8_t* __restrict__ ds, uint16_t* __restrict__ gout,
    uint16_t* __restrict__ uout, uint16_t* __restrict__ dout) {
  pdl_trigger();
  pdl_wait();  // inputs come from earlier kernels on the stream
  const long long per_mat = static_cast<long long>(I) * H / 8;  // units per matrix
  const long long total = static_cast<long long>(*ntouched) * 3 * per_mat;
  for (long long u = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; u < total;
       u += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long slot = u / (3 * per_mat);
    const long long r = u - slot * 3 * per_mat;
    const int mat = static_cast<int>(r / per_mat);
    const long long v = r - mat * per_mat;
    const long long e = touched[slot];
    const long long el = e * I * H + v * 8;  // element index in the expert-major source
    const uint8_t* q = mat == 0 ? gq : mat == 1 ? uq : dq;
    const uint8_t* sc = mat == 0 ? gs : mat == 1 ? us : ds;
    uint16_t* o = mat == 0 ? gout : mat == 1 ? uout : dout;
    const uint32_t codes = *reinterpret_cast<const uint32_t*>(q + el / 2);
    const uint32_t s = sc[el / 32];
    *reinterpret_cast<uint4*>(o + slot * I * H + v * 8) = dequant8(codes, s);
  }
}

}  // namespace

cudaError_t launch_mxfp4_slots(const moe_cfg& c, const int32_t* offsets, int32_t* slot_of,
                               int32_t* touched, int32_t* ntouched, cudaStream_t s) {
  return launch_pdl(mxfp4_slots, dim3(1), dim3(1024), 0, s, c.E, offsets, slot_of, touched,
                    ntouched);
}

cudaError_t launch_mxfp4_expand(const moe_cfg& c, const int32_t* offsets, const moe_weights* W,
                                int32_t* slot_of, int32_t* touched, int32_t* ntouched,
                                uint16_t* gout, uint16_t* uout, uint16_t* dout, cudaStream_t s) {
  cudaError_t e = launch_mxfp4_slots(c, offsets, slot_of, touched, ntouched, s);
  if (e != cudaSuccess) return e;
  return launch_pdl(mxfp4_dequant, dim3(num_sms() * 8), dim3(256), 0, s, c.I, c.H,
                    static_cast<const int32_t*>(touched), static_cast<const int32_t*>(ntouched),
                    static_cast<const uint8_t*>(W->Wg), W->Wg_scale,
                    static_cast<const uint8_t*>(W->Wu), W->Wu_scale,
                    static_cast<const uint8_t*>(W->Wd), W->Wd_scale, gout, uout, dout);
}

}  // namespace sgl
