// mxfp8.cu - inputs of the block-scaled expert FFN (weight format
// MOE_W_MXFP4_A8): the routed experts' activations in MXFP8 and the weight
// scales in the layout the tensor cores take them in.
//
// Page "Ling-3.0-flash-VL 42-layer hybrid backbone" (lpnh.cn/news/2815793),
// spec table: the quantisation scheme is FP8 + MXFP4 (routed experts' weights
// in 4 bits). Format per the OCP Microscaling spec v1.0: e4m3 elements and
// one e8m0 scale per 32 consecutive elements along the contraction; the scale
// is 2^(floor(log2(amax)) - 8), 8 being the largest e4m3 exponent, and each
// element v / scale is rounded to the nearest e4m3 value (ties to even),
// saturating at 448.
//
// Scale atoms: tcgen05.mma kind::mxf8f6f4.block_scale reads its scales from
// tensor memory, where tcgen05.cp.32x128b.warpx4 puts them from a 512-byte
// shared-memory atom that covers 128 rows x one 128-wide k-block (four scales
// per row): the scale of row r and 32-element chunk k sits at byte
// (r % 32) * 16 + (r / 32) * 4 + k.
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"
#include "ptx.cuh"

namespace sgl {
namespace {

__device__ __forceinline__ int atom_offset(int r, int k) { return (r & 31) * 16 + (r >> 5) * 4 + k; }

// Weight scales of the touched experts as atoms, [slot][128-row tile][k-block]
// for each of Wg, Wu ([I, H]) and Wd ([H, I]). Unit = one row of one atom
// (four scale bytes, read as one 32-bit word); consecutive threads take
// consecutive rows of one atom.
__global__ void __launch_bounds__(256) mx_sf_repack(int H, int I, int max_touched,
                                                     const int32_t* __restrict__ touched,
                                                     const int32_t* __restrict__ ntouched,
                                                     const uint8_t* __restrict__ gs,
                                                     const uint8_t* __restrict__ us,
                                                     const uint8_t* __restrict__ ds,
                                                     uint8_t* __restrict__ sf_g,
                                                     uint8_t* __restrict__ sf_u,
                                                     uint8_t* __restrict__ sf_d) {
  pdl_trigger();
  pdl_wait();  // the touched list comes from the previous kernel
  const int nt = min(*ntouched, max_touched);
  const int kbh = H / 128, kbi = I / 128;
  const long long per_mat = static_cast<long long>(kbh) * kbi * 128;  // units per matrix (both shapes)
  const long long total = static_cast<long long>(nt) * 3 * per_mat;
  for (long long u = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; u < total;
       u += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long slot = u / (3 * per_mat);
    long long v = u - slot * 3 * per_mat;
    const int mat = static_cast<int>(v / per_mat);
    v -= mat * per_mat;
    const long long e = touched[slot];
    const int r = static_cast<int>(v & 127);
    const long long atom = v >> 7;  // (row tile, k-block) of this matrix
    const int nkb = mat < 2 ? kbh : kbi;  // k-blocks along the contraction
    const int kc = mat < 2 ? H / 32 : I / 32;  // scale bytes per row
    const long long rows = mat < 2 ? I : H;
    const int t = static_cast<int>(atom / nkb), b = static_cast<int>(atom % nkb);
    const uint8_t* src = (mat == 0 ? gs : mat == 1 ? us : ds) + (e * rows + t * 128 + r) * kc + b * 4;
    uint8_t* dst = (mat == 0 ? sf_g : mat == 1 ? sf_u : sf_d) + (slot * per_mat / 128 + atom) * 512;
    *reinterpret_cast<uint32_t*>(dst + atom_offset(r, 0)) = *reinterpret_cast<const uint32_t*>(src);
  }
}

// x [T, H] bf16 -> x_q [T, H] e4m3 codes, x_sf [T, H/32] e8m0. One thread per
// 32-element block.
__global__ void __launch_bounds__(256) mx_quant_x(long long nblocks, int H,
                                                   const uint16_t* __restrict__ x,
                                                   uint8_t* __restrict__ xq,
                                                   uint8_t* __restrict__ xsf) {
  pdl_trigger();
  pdl_wait();  // x may come from an earlier kernel on the stream
  for (long long b = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; b < nblocks;
       b += static_cast<long long>(gridDim.x) * blockDim.x) {
    const uint4* src = reinterpret_cast<const uint4*>(x + b * 32);
    uint4 raw[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) raw[i] = src[i];
    const uint32_t* w = reinterpret_cast<const uint32_t*>(raw);
    float v[32];
    uint32_t amax_bits = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
      amax_bits = max(amax_bits, __float_as_uint(v[2 * i]) & 0x7FFFFFFFu);
      amax_bits = max(amax_bits, __float_as_uint(v[2 * i + 1]) & 0x7FFFFFFFu);
    }
    // floor(log2(amax)) - 8 + 127 from amax's exponent field, clamped to [0, 254]
    const int byte = min(max(static_cast<int>(amax_bits >> 23) - 8, 0), 254);
    const int ie = 254 - byte;  // 1/scale = 2^(127 - byte)
    const float inv = ie > 0 ? __uint_as_float(static_cast<uint32_t>(ie) << 23)
                             : __uint_as_float(0x00400000u);
    uint32_t out[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const __nv_fp8x2_storage_t lo =
          __nv_cvt_float2_to_fp8x2(make_float2(v[4 * i] * inv, v[4 * i + 1] * inv), __NV_SATFINITE, __NV_E4M3);
      const __nv_fp8x2_storage_t hi =
          __nv_cvt_float2_to_fp8x2(make_float2(v[4 * i + 2] * inv, v[4 * i + 3] * inv), __NV_SATFINITE, __NV_E4M3);
      out[i] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
    }
    uint4* dst = reinterpret_cast<uint4*>(xq + b * 32);
    dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
    dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
    xsf[b] = static_cast<uint8_t>(byte);
  }
}

}  // namespace

cudaError_t launch_mx_prep(const moe_cfg& c, int T, const int32_t* offsets, const moe_weights* W,
                           const uint16_t* x, int32_t* slot_of, int32_t* touched,
                           int32_t* ntouched, uint8_t* sf_g, uint8_t* sf_u, uint8_t* sf_d,
                           uint8_t* x_q, uint8_t* x_sf, cudaStream_t s) {
  cudaError_t e = launch_mxfp4_slots(c, offsets, slot_of, touched, ntouched, s);
  if (e != cudaSuccess) return e;
  const long long TK = static_cast<long long>(T) * c.K;
  const int max_touched = static_cast<int>(TK < c.E ? TK : c.E);
  e = launch_pdl(mx_sf_repack, dim3(num_sms() * 4), dim3(256), 0, s, c.H, c.I, max_touched,
                 static_cast<const int32_t*>(touched), static_cast<const int32_t*>(ntouched),
                 W->Wg_scale, W->Wu_scale, W->Wd_scale, sf_g, sf_u, sf_d);
  if (e != cudaSuccess) return e;
  const long long nblocks = static_cast<long long>(T) * (c.H / 32);
  long long grid = (nblocks + 255) / 256;
  if (grid > num_sms() * 8) grid = num_sms() * 8;
  return launch_pdl(mx_quant_x, dim3(static_cast<int>(grid)), dim3(256), 0, s, nblocks, c.H, x,
                    x_q, x_sf);
}

}  // namespace sgl
