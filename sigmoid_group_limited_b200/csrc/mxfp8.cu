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

// Weight scales of the touched experts as atoms, [slot][128-row tile][k-block]
// for each of Wg, Wu ([I, H]) and Wd ([H, I]). One warp per (slot, matrix,
// 128-row tile), eight k-blocks at a time: the warp reads the tile's 128 rows
// x 32 scale bytes with 4-byte loads in which eight lanes cover one row
// (whole sectors), transposes them through shared memory, and writes each
// atom as one 512-byte store: lane l's 16 bytes at l * 16 are the four scale
// bytes of rows l, l+32, l+64 and l+96.
constexpr int kRepackWarps = 8;
constexpr int kRepackKb = 8;  // k-blocks per pass
__global__ void __launch_bounds__(32 * kRepackWarps) mx_sf_repack(int H, int I, int max_touched,
                                                     const int32_t* __restrict__ touched,
                                                     const int32_t* __restrict__ ntouched,
                                                     const uint8_t* __restrict__ gs,
                                                     const uint8_t* __restrict__ us,
                                                     const uint8_t* __restrict__ ds,
                                                     uint8_t* __restrict__ sf_g,
                                                     uint8_t* __restrict__ sf_u,
                                                     uint8_t* __restrict__ sf_d) {
  __shared__ uint32_t tr[kRepackWarps][128][kRepackKb + 1];  // +1: conflict-free columns
  pdl_trigger();
  pdl_wait();  // the touched list comes from the previous kernel
  // touched == nullptr: every expert, slot = expert id (max_touched = E)
  const int nt = touched ? min(*ntouched, max_touched) : max_touched;
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  uint32_t (*sw)[kRepackKb + 1] = tr[wib];
  const int tiles_gu = I / 128, tiles_d = H / 128;  // 128-row tiles of Wg / Wu, of Wd
  const int per_slot = 2 * tiles_gu + tiles_d;
  const long long total = static_cast<long long>(nt) * per_slot;
  const long long nwarps = static_cast<long long>(gridDim.x) * kRepackWarps;
  for (long long w = static_cast<long long>(blockIdx.x) * kRepackWarps + wib; w < total; w += nwarps) {
    const long long slot = w / per_slot;
    const int v = static_cast<int>(w - slot * per_slot);
    const int mat = v < tiles_gu ? 0 : (v < 2 * tiles_gu ? 1 : 2);
    const int t = mat < 2 ? v - mat * tiles_gu : v - 2 * tiles_gu;  // row tile
    const long long e = touched ? touched[slot] : slot;
    const int kw = mat < 2 ? H / 128 : I / 128;  // scale words per row = k-blocks
    const long long rows = mat < 2 ? I : H;
    const int tiles = mat < 2 ? tiles_gu : tiles_d;
    const uint32_t* src = reinterpret_cast<const uint32_t*>(mat == 0 ? gs : mat == 1 ? us : ds) +
                          (e * rows + t * 128) * kw;
    uint8_t* dst = (mat == 0 ? sf_g : mat == 1 ? sf_u : sf_d) + ((slot * tiles + t) * kw) * 512 + lane * 16;
    for (int b0 = 0; b0 < kw; b0 += kRepackKb) {
      const int nb = min(kRepackKb, kw - b0);
      __syncwarp();  // the previous pass's reads of sw are done
      // lane l: word l % 8 of rows l / 8, l / 8 + 4, ...
      const int c = lane & 7;
      if (c < nb) {
#pragma unroll 4
        for (int r = lane >> 3; r < 128; r += 4) sw[r][c] = src[static_cast<size_t>(r) * kw + b0 + c];
      }
      __syncwarp();
      for (int b = 0; b < nb; ++b)
        *reinterpret_cast<uint4*>(dst + (b0 + b) * 512) =
            make_uint4(sw[lane][b], sw[lane + 32][b], sw[lane + 64][b], sw[lane + 96][b]);
    }
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
  e = launch_pdl(mx_sf_repack, dim3(num_sms() * 4), dim3(32 * kRepackWarps), 0, s, c.H, c.I, max_touched,
                 static_cast<const int32_t*>(touched), static_cast<const int32_t*>(ntouched),
                 W->Wg_scale, W->Wu_scale, W->Wd_scale, sf_g, sf_u, sf_d);
  if (e != cudaSuccess) return e;
  return launch_mx_quant(c, T, x, x_q, x_sf, s);
}

cudaError_t launch_mx_quant(const moe_cfg& c, int T, const uint16_t* x, uint8_t* x_q, uint8_t* x_sf,
                            cudaStream_t s) {
  const long long nblocks = static_cast<long long>(T) * (c.H / 32);
  long long grid = (nblocks + 255) / 256;
  if (grid > num_sms() * 8) grid = num_sms() * 8;
  return launch_pdl(mx_quant_x, dim3(static_cast<int>(grid)), dim3(256), 0, s, nblocks, c.H, x,
                    x_q, x_sf);
}

cudaError_t launch_mx_sf_atoms(const moe_cfg& c, const moe_weights* W, uint8_t* sf_g, uint8_t* sf_u,
                               uint8_t* sf_d, cudaStream_t s) {
  return launch_pdl(mx_sf_repack, dim3(num_sms() * 4), dim3(32 * kRepackWarps), 0, s, c.H, c.I, c.E,
                    static_cast<const int32_t*>(nullptr), static_cast<const int32_t*>(nullptr),
                    W->Wg_scale, W->Wu_scale, W->Wd_scale, sf_g, sf_u, sf_d);
}

}  // namespace sgl
