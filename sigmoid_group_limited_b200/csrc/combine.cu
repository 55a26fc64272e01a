// combine.cu - stage 9: weighted combine back to token order.
//
// Every token's output is the sum of its K routed-expert contributions
// (fp32, already multiplied by their combine weights) plus the shared
// expert's output (page "Ling-3.0-flash-VL MoE sparse routing", sec. 2 and sec. 4).
// The sum runs in fp32 in slot order k = 0..K-1, then adds the shared row,
// and is rounded once to bf16 (nearest even). 16-byte loads and stores; each
// thread owns 8 consecutive features of one token.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"
#include "ptx.cuh"

namespace sgl {
namespace {

__device__ __forceinline__ void add8(float* acc, const float4 a, const float4 b) {
  acc[0] += a.x;
  acc[1] += a.y;
  acc[2] += a.z;
  acc[3] += a.w;
  acc[4] += b.x;
  acc[5] += b.y;
  acc[6] += b.z;
  acc[7] += b.w;
}

__global__ void __launch_bounds__(256) combine_kernel(int T, int H, int K, int with_shared,
                                                      const float* __restrict__ y_slot,
                                                      uint16_t* __restrict__ y) {
  pdl_trigger();
  pdl_wait();  // inputs come from earlier kernels on the stream
  const int chunks = H / 8;
  const long long total = static_cast<long long>(T) * chunks;
  const float4* src = reinterpret_cast<const float4*>(y_slot);
  uint4* dst = reinterpret_cast<uint4*>(y);
  const long long TKrows = static_cast<long long>(T) * K;
  const long long row4 = H / 4;  // float4 per row
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long t = i / chunks;
    const int c = static_cast<int>(i - t * chunks);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
    for (int k = 0; k < K; ++k) {
      const float4* r = src + (t * K + k) * row4 + 2 * c;
      add8(acc, r[0], r[1]);
    }
    if (with_shared) {
      const float4* r = src + (TKrows + t) * row4 + 2 * c;
      add8(acc, r[0], r[1]);
    }
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(acc[2 * q]));
      const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(acc[2 * q + 1]));
      o[q] = lo | (hi << 16);
    }
    dst[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

}  // namespace

cudaError_t launch_combine(const moe_cfg& c, int T, const float* y_slot, int with_shared,
                           uint16_t* y, cudaStream_t s) {
  const long long total = static_cast<long long>(T) * (c.H / 8);
  const int threads = 256;
  long long blocks = (total + threads - 1) / threads;
  const long long cap = static_cast<long long>(num_sms()) * 8;
  if (blocks > cap) blocks = cap;
  return launch_pdl(combine_kernel, dim3(static_cast<int>(blocks)), dim3(threads), 0, s, T, c.H, c.K,
                    with_shared, y_slot, y);
}

}  // namespace sgl
