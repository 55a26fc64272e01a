// permute_dev.cuh - device code of stage 6 shared by the permutation kernels
// (permute.cu) and the fused decode front (front.cu): the block scan, the FFN
// work-list builder and the one-CTA permutation.
//
// Each token selects K experts (page "Ling-3.0-flash-VL MoE sparse routing",
// sec. 3 step 2); the permutation is a stable counting sort of the flat slot
// index j = t*K + k by expert id.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"
#include "ptx.cuh"

namespace sgl {
namespace {

constexpr int kMaxE = 1024;

__device__ __forceinline__ int ld_acquire_gpu(const int32_t* a) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(a) : "memory");
  return v;
}

// Grid barrier n (1, 2, ...) of a cooperative launch on a monotonic counter
// that is zero at launch; false if it timed out (the error word is set;
// every CTA then leaves).
__device__ bool grid_barrier(int32_t* bar, int n, int32_t* err) {
  __shared__ int ok_s;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();  // this CTA's writes before its arrival
    atomicAdd(bar, 1);
    const int need = n * static_cast<int>(gridDim.x);
    const long long t0 = clock64();
    int ok = 1;
    while (ld_acquire_gpu(bar) < need) {  // waits last a few microseconds: spin
      if (clock64() - t0 > kWaitLimitCycles) {
        atomicExch(err, MOE_DEVERR_TIMEOUT);
        ok = 0;
        break;
      }
    }
    ok_s = ok;
  }
  __syncthreads();
  return ok_s != 0;
}

// Block-wide exclusive scan of up to 2 values per thread (1024 threads).
// Returns the exclusive prefix of this thread's first value; *total gets the sum.
__device__ int block_exscan2(int v0, int v1, int* scratch /*32*/, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int v = v0 + v1;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    int s = lane < nw ? scratch[lane] : 0;
    int si = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, si, o);
      if (lane >= o) si += y;
    }
    if (lane < nw) scratch[lane] = si - s;
    if (lane == 31) scratch[32] = si;
  }
  __syncthreads();
  const int ex = scratch[warp] + incl - v;
  *total = scratch[32];
  __syncthreads();
  return ex;
}

struct SchedArgs {
  int T, K, E, H, I, Is, has_shared, bn;
  int gu_ft, dn_ft;   // output features per gate/up item and per down item
  int32_t* gu_start;  // [E+2] first gate/up work item of slot e (e == E: shared expert)
  int32_t* dn_start;  // [E+2] first down work item of slot e
  int32_t* ready;     // nullable: [gate/up items] zeroed for the fused FFN's row-tile counters
  int ready_len;      // > 0: zero ready[0, ready_len) whole (the FFN picks its own tile)
  int32_t* nitems;    // [2] totals
};

// Work lists of the two grouped GEMMs, as prefix sums of per-slot item counts.
// Slot e (e == E: the shared expert, whose rows are the T tokens) has
// ceil(rows/bn) row tiles times its output tiles; the GEMM kernels decode an
// item index back to (slot, row tile, output tile) with a binary search over
// these starts. Needs blockDim.x == 1024 and counts in shared memory.
__device__ void build_schedule(const SchedArgs& a, const int* cnt, int* scratch) {
  const int nslots = a.E + (a.has_shared ? 1 : 0);
  const int nt_gu_r = cdiv_dev(a.I, a.gu_ft), nt_gu_s = cdiv_dev(a.Is, a.gu_ft);
  const int nt_dn = cdiv_dev(a.H, a.dn_ft);
  int ngu[2] = {0, 0}, ndn[2] = {0, 0};
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const int e = 2 * threadIdx.x + q;
    if (e < nslots) {
      const bool sh = e == a.E;
      const int rows = sh ? a.T : cnt[e];
      const int nm = (rows + a.bn - 1) / a.bn;
      ngu[q] = nm * (sh ? nt_gu_s : nt_gu_r);
      ndn[q] = nm * nt_dn;
    }
  }
  int tot_gu, tot_dn;
  const int base_gu = block_exscan2(ngu[0], ngu[1], scratch, &tot_gu);
  const int base_dn = block_exscan2(ndn[0], ndn[1], scratch, &tot_dn);
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const int e = 2 * threadIdx.x + q;
    if (e <= a.E + 1) {
      const bool real = e < nslots;
      a.gu_start[e] = real ? base_gu + (q ? ngu[0] : 0) : tot_gu;
      a.dn_start[e] = real ? base_dn + (q ? ndn[0] : 0) : tot_dn;
    }
  }
  if (a.ready && a.ready_len > 0) {
    // the FFN derives its work lists for a tile it picks itself: every
    // counter it may use
    for (int i = threadIdx.x; i < a.ready_len; i += blockDim.x) a.ready[i] = 0;
  } else if (a.ready) {
    // one counter per (slot, row tile): the slot's first nm gate/up item indices
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int e = 2 * threadIdx.x + q;
      if (e < nslots) {
        const int ntg = e == a.E ? nt_gu_s : nt_gu_r;
        const int nm = ntg > 0 ? (q ? ngu[1] : ngu[0]) / ntg : 0;
        const int b0 = base_gu + (q ? ngu[0] : 0);
        for (int m = 0; m < nm; ++m) a.ready[b0 + m] = 0;
      }
    }
  }
  if (threadIdx.x == 0) {
    a.nitems[0] = tot_gu;
    a.nitems[1] = tot_dn;
    a.nitems[2] = 0;  // the fused FFN's item counter
  }
}

// The whole permutation in one CTA (all T*K entries in one tile: decode
// batches): per-warp histograms of contiguous chunks, per-expert totals and
// their exclusive scan, per-warp bases, stable positions, and optionally the
// GEMM work lists, with no round trip through global memory in between.
// whist: [warps][E] ints of shared memory; 2 * blockDim.x >= E + 2.
__device__ __forceinline__ void perm_block(int TK, int E, const int32_t* __restrict__ idx,
                                           int32_t* __restrict__ counts,
                                           int32_t* __restrict__ offsets,
                                           int32_t* __restrict__ perm,
                                           int32_t* __restrict__ inv_perm,
                                           int32_t* __restrict__ err, const SchedArgs& sa,
                                           int build, int* whist) {
  __shared__ int cnt[kMaxE + 1];
  __shared__ int off[kMaxE + 1];
  __shared__ int scratch[33];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  for (int i = tid; i < nw * E; i += blockDim.x) whist[i] = 0;
  __syncthreads();
  const int chunk = ((cdiv_dev(TK, nw) + 31) / 32) * 32;
  const int c0 = warp * chunk, c1 = min(c0 + chunk, TK);
  const unsigned lt = (1u << lane) - 1u;
  int* wh = whist + warp * E;
  for (int r = c0; r < c1; r += 32) {
    const int i = r + lane;
    int e = -1;
    if (i < c1) {
      e = idx[i];
      if (e < 0 || e >= E) {
        atomicExch(err, MOE_DEVERR_EXPERT_ID);
        e = -1;
      }
    }
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && (peers & lt) == 0) wh[e] += __popc(peers);
  }
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) {
    int tot = 0;
    for (int w = 0; w < nw; ++w) tot += whist[w * E + e];
    cnt[e] = tot;
  }
  __syncthreads();
  int total;
  const int e0 = 2 * tid;
  const int v0 = e0 < E ? cnt[e0] : 0, v1 = e0 + 1 < E ? cnt[e0 + 1] : 0;
  const int ex = block_exscan2(v0, v1, scratch, &total);
  if (e0 < E) off[e0] = ex;
  if (e0 + 1 < E) off[e0 + 1] = ex + v0;
  if (tid == 0) off[E] = total;
  __syncthreads();
  for (int e = tid; e <= E; e += blockDim.x) {
    offsets[e] = off[e];
    if (e < E) counts[e] = cnt[e];
  }
  for (int e = tid; e < E; e += blockDim.x) {
    int run = off[e];
    for (int w = 0; w < nw; ++w) {
      const int v = whist[w * E + e];
      whist[w * E + e] = run;
      run += v;
    }
  }
  __syncthreads();
  for (int r = c0; r < c1; r += 32) {
    const int i = r + lane;
    int e = -1;
    if (i < c1) {
      e = idx[i];
      if (e < 0 || e >= E) e = -1;
    }
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    int pos = -1;
    if (e >= 0) pos = wh[e] + __popc(peers & lt);
    __syncwarp();
    if (e >= 0 && (peers & lt) == 0) wh[e] += __popc(peers);
    __syncwarp();
    if (i < c1) {
      if (e >= 0 && (pos < 0 || pos >= TK)) {
        atomicExch(err, MOE_DEVERR_SCHEDULE);
        e = -1;
        pos = -1;
      }
      if (e >= 0) perm[pos] = i;
      if (inv_perm) inv_perm[i] = pos;
    }
  }
  if (build) build_schedule(sa, cnt, scratch);
}

SchedArgs make_sched(const moe_cfg& c, int T, const WsLayout& L, int32_t* gu_start,
                     int32_t* dn_start, int32_t* ready, int32_t* nitems) {
  SchedArgs a;
  a.T = T;
  a.K = c.K;
  a.E = c.E;
  a.H = c.H;
  a.I = c.I;
  a.Is = c.I_shared;
  a.has_shared = c.I_shared > 0;
  a.bn = L.bn;
  a.gu_ft = L.gu_ft;
  a.dn_ft = L.dn_ft;
  a.gu_start = gu_start;
  a.dn_start = dn_start;
  a.ready = ready;
  a.ready_len = ffn_adaptive(L) ? L.max_items_gu : 0;
  a.nitems = nitems;
  return a;
}


}  // namespace
}  // namespace sgl
