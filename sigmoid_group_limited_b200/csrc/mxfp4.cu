// mxfp4.cu - routed expert weights stored as MXFP4 (page "Ling-3.0-flash-VL
// 42-layer hybrid backbone", lpnh.cn/news/2815793, spec table: the routed
// experts' weights are 4-bit), format per the OCP Microscaling spec: e2m1
// codes, two per byte (element 2j in the low nibble), one e8m0 scale per 32
// consecutive elements along K.
//
// The bf16 FFN kernel expands the codes to their exact values
// code * 2^(scale - 127) in shared memory (ffn.cu). What remains here is the
// list of the experts a batch touches, which the block-scaled path uses to
// repack their scales once per forward.
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

}  // namespace

cudaError_t launch_mxfp4_slots(const moe_cfg& c, const int32_t* offsets, int32_t* slot_of,
                               int32_t* touched, int32_t* ntouched, cudaStream_t s) {
  return launch_pdl(mxfp4_slots, dim3(1), dim3(1024), 0, s, c.E, offsets, slot_of, touched,
                    ntouched);
}

}  // namespace sgl
