// ffn_common.cuh - parameters and device helpers shared by the expert-FFN
// kernels (ffn.cu: one CTA per item; ffn_pair.cu: a CTA pair per item;
// ffn_mx.cu: block-scaled MXFP8 x MXFP4).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"
#include "ptx.cuh"

namespace sgl {
namespace {

struct FfnParams {
  int T, K, E, H, I, Is;
  int has_shared;
  float lim_r, lim_s;        // <= 0: no limit
  const uint16_t* x;         // [T, H]
  const int32_t* perm;       // [T*K] sorted position -> flat slot j
  const float* w;            // [T*K] routing weights
  uint16_t* h_r;             // [T*K, I] permuted rows
  uint16_t* h_s;             // [T, Is]
  float* y_slot;             // [(T*K + T), H] fp32
  const int32_t* offsets;    // [E+1]
  const int32_t* wslot;      // nullable: weight row block of expert e
  const int32_t* gu_start;   // [E+2]
  const int32_t* dn_start;   // [E+2]
  const int32_t* nitems;     // [2] item totals; [2] is the claim counter
  int32_t* counter;
  int32_t* ready;            // [max_gu] finished gate/up tiles per (slot, row tile)
  int max_gu, max_dn;
  int32_t* err;
  const int32_t* sched_counts;  // nullable: derive the work lists from the expert counts
  int bn, gu_ft, dn_ft;         // token tile and output features per item (for that)
  // MXFP4 routed weights (the expanding kernel): codes [E*rows, K/2] and e8m0
  // scales [E*rows, K/32] of Wg, Wu (K = H) and Wd (K = I), expert-major
  const uint8_t *q_g, *q_u, *q_d, *s_g, *s_u, *s_d;
  // test hooks of the scheduler's wait (0 in normal use): its limit in cycles,
  // and a count added to the tiles it waits for (one that is never reached
  // makes the wait run out)
  long long wait_limit;
  int ready_extra;
};

// In-place exclusive scan of a[0..n) in shared memory by the whole CTA
// (each thread sums a contiguous run, then one block scan of the run sums);
// wsum: 33 ints of shared memory. Ends with a CTA barrier.
__device__ __forceinline__ void smem_exscan(int* a, int n, int* wsum) {
  const int per = (n + static_cast<int>(blockDim.x) - 1) / static_cast<int>(blockDim.x);
  const int b = static_cast<int>(threadIdx.x) * per, e = min(n, b + per);
  int s = 0;
  for (int i = b; i < e; ++i) s += a[i];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int nw = static_cast<int>(blockDim.x) >> 5;
    const int v = lane < nw ? wsum[lane] : 0;
    int vi = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, vi, o);
      if (lane >= o) vi += y;
    }
    if (lane < nw) wsum[lane] = vi - v;
  }
  __syncthreads();
  int run = wsum[warp] + incl - s;
  for (int i = b; i < e; ++i) {
    const int v = a[i];
    a[i] = run;
    run += v;
  }
  __syncthreads();
}

// Rows of expert e: from the counts, else from the row offsets.
__device__ __forceinline__ int expert_rows(const FfnParams& p, int e) {
  return max(0, p.sched_counts ? p.sched_counts[e] : p.offsets[e + 1] - p.offsets[e]);
}

// The FFN work lists from the expert loads, in shared memory: the row
// offsets s_off[0..E] (exclusive scan of the loads) and the per-slot item
// starts s_gu / s_dn [E+2] (slot E the shared expert, entry E+1 the total)
// for token tiles of bn rows, as the schedule builder of the permutation
// writes them for its tile. Returns the item totals.
__device__ __forceinline__ void derive_schedule(const FfnParams& p, int bn, int* s_gu, int* s_dn,
                                                int* s_off, int* wsum, int* n_gu, int* n_dn) {
  const int nslots = p.E + (p.has_shared ? 1 : 0);
  const int nt_gu_r = cdiv_dev(p.I, p.gu_ft), nt_gu_s = cdiv_dev(p.Is, p.gu_ft);
  const int nt_dn = cdiv_dev(p.H, p.dn_ft);
  for (int e = threadIdx.x; e < p.E + 2; e += blockDim.x) {
    int gu = 0, dn = 0, c = 0;
    if (e < p.E) c = expert_rows(p, e);
    if (e < nslots) {
      const bool sh = e == p.E;
      const int rows = sh ? p.T : c;
      const int nm = (rows + bn - 1) / bn;
      gu = nm * (sh ? nt_gu_s : nt_gu_r);
      dn = nm * nt_dn;
    }
    s_gu[e] = gu;
    s_dn[e] = dn;
    if (e < p.E + 1) s_off[e] = c;
  }
  __syncthreads();
  smem_exscan(s_gu, p.E + 2, wsum);
  smem_exscan(s_dn, p.E + 2, wsum);
  smem_exscan(s_off, p.E + 1, wsum);
  *n_gu = s_gu[p.E + 1];
  *n_dn = s_dn[p.E + 1];
}

// Token tile of the adaptive kernel: an MMA costs about the same for any N,
// so 256-row tiles pay when they cut the number of row tiles, which they do
// only for experts with more than 128 rows; otherwise the 128-row geometry
// (more pipeline stages, double-buffered accumulators) is faster. 256 when
// the 256-row tiles number at most 4/5 of the 128-row ones. Every CTA reads
// the same loads, so all take the same decision. tot: 2 ints of shared
// memory. Ends with a CTA barrier.
__device__ __forceinline__ int adaptive_bn(const FfnParams& p, int* tot) {
  if (threadIdx.x < 2) tot[threadIdx.x] = 0;
  __syncthreads();
  int t128 = 0, t256 = 0;
  for (int e = threadIdx.x; e <= p.E; e += blockDim.x) {
    const int rows = e < p.E ? expert_rows(p, e) : (p.has_shared ? p.T : 0);
    t128 += (rows + 127) / 128;
    t256 += (rows + 255) / 256;
  }
  atomicAdd(&tot[0], t128);
  atomicAdd(&tot[1], t256);
  __syncthreads();
  return 5 * tot[1] <= 4 * tot[0] ? 256 : 128;
}

__device__ __forceinline__ float clampL(float v, float L) {
  return L > 0.f ? fminf(fmaxf(v, -L), L) : v;
}

// Named barrier 1 over the epilogue warps (NT threads).
template <int NT>
__device__ __forceinline__ void epi_bar() {
  asm volatile("bar.sync 1, %0;" ::"n"(NT) : "memory");
}

// silu(g) * u after the clamp, with the hardware exponential and the
// hardware's approximate reciprocal (h is rounded to bf16 right after, whose
// half-ulp is far above either error).
__device__ __forceinline__ float swiglu(float g, float u, float L) {
  const float gg = clampL(g, L), uu = clampL(u, L);
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(1.0f + __expf(-gg)));
  return gg * r * uu;
}


__device__ __forceinline__ uint16_t f2bf(float v) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Epilogue stores through a per-warp shared-memory tile (kEpiTileWords
// 32-bit words): a lane of an epilogue warp holds one output feature (its
// TMEM lane) for consecutive token columns, while the outputs are token rows
// of features. Going through the tile turns 32 single-value stores per row
// group into 16-byte stores of row pieces.
constexpr int kEpiTileWords = 256;

// h (bf16) of 16 token columns: hv[c] is this lane's feature fbase + lane of
// token row `row0 + c`; rows c >= nvalid are not stored. hout + row * ncols
// + fbase must be 16-byte aligned for every row (ncols and fbase multiples
// of 8).
__device__ __forceinline__ void store_h16(const float* hv, uint32_t* tile, uint16_t* hout,
                                          int ncols, int row0, int nvalid, int fbase, int lane) {
  const bool odd = (lane & 1) != 0;
  // token pair (2k, 2k+1): the even lane of a lane pair packs features
  // (l, l+1) of token 2k, the odd lane those of token 2k+1
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float mine = odd ? hv[2 * k + 1] : hv[2 * k];
    const float other = __shfl_xor_sync(0xffffffffu, odd ? hv[2 * k] : hv[2 * k + 1], 1);
    tile[(2 * k + (odd ? 1 : 0)) * 16 + (lane >> 1)] =
        odd ? pack_bf16x2(other, mine) : pack_bf16x2(mine, other);
  }
  __syncwarp();
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int r = half * 8 + (lane >> 2);  // token row; the lane's 8 features at 8 * (lane & 3)
    const uint4 v = *reinterpret_cast<const uint4*>(tile + r * 16 + 4 * (lane & 3));
    if (r < nvalid)
      *reinterpret_cast<uint4*>(hout + static_cast<size_t>(row0 + r) * ncols + fbase +
                                8 * (lane & 3)) = v;
  }
  __syncwarp();
}

// fp32 rows of 8 token columns: v[i] (already weighted) is this lane's
// feature fbase + lane of y_slot row j[i] (j < 0: not stored). y + j * H +
// fbase must be 16-byte aligned (H and fbase multiples of 4).
__device__ __forceinline__ void store_y8(const float* v, const int* j, uint32_t* tile, float* y,
                                         int H, int fbase, int lane) {
  float* t = reinterpret_cast<float*>(tile);
#pragma unroll
  for (int i = 0; i < 8; ++i) t[i * 32 + lane] = v[i];
  __syncwarp();
#pragma unroll
  for (int pass = 0; pass < 2; ++pass) {
    const int i = pass * 4 + (lane >> 3);  // row; the lane's 4 features at 4 * (lane & 7)
    const float4 q = *reinterpret_cast<const float4*>(t + i * 32 + 4 * (lane & 7));
    const int jj = j[i];
    if (jj >= 0)
      *reinterpret_cast<float4*>(y + static_cast<size_t>(jj) * H + fbase + 4 * (lane & 7)) = q;
  }
  __syncwarp();
}

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ int ld_acquire(const int32_t* a) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(a) : "memory");
  return v;
}

// Bounded wait of a scheduler until *addr >= need (acquire): the count of
// gate/up tiles that other CTAs have published for a down item's row tile.
// Gives up after `limit` cycles (kWaitLimitCycles when 0), or at once if the
// CTA's abort flag is up. A timeout sets the error word but not the abort
// flag: the scheduler then queues the end of its work, and every role of the
// CTA finishes the items already queued and leaves, with no copy or MMA left
// in flight.
__device__ __forceinline__ bool wait_count(const int32_t* addr, int need, volatile int* abort_flag,
                                           int* err, long long limit = 0) {
  const long long t0 = clock64();
  const long long lim = limit > 0 ? limit : kWaitLimitCycles;
  while (ld_acquire(addr) < need) {
    if (*abort_flag) return false;
    if (clock64() - t0 > lim) {
      atomicExch(err, MOE_DEVERR_TIMEOUT);
      return false;
    }
    __nanosleep(100);
  }
  return true;
}

// Bounded wait until the producer's progress word reaches `need`.
__device__ __forceinline__ bool wait_progress(const volatile long long* prog, long long need,
                                              volatile int* abort_flag, int* err) {
  const long long t0 = clock64();
  while (*prog < need) {
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitLimitCycles) {
      *abort_flag = 1;
      atomicExch(err, MOE_DEVERR_TIMEOUT);
      return false;
    }
    __nanosleep(32);
  }
  return true;
}

// Same validity rule in every role, so all roles skip the same items.
// gu_tile / dn_tile: output features per gate/up and per down item.
__device__ __forceinline__ bool item_ok(const FfnParams& p, const WorkItem& it, bool gu, int bn,
                                        int gu_tile = kTileN, int dn_tile = kDownTile) {
  const bool sh = it.e == p.E;
  if (it.e < 0 || it.e > p.E || (sh && !p.has_shared)) return false;
  if (it.nrows <= 0 || it.nrows > bn || it.row0 < 0) return false;
  if (it.row0 + it.nrows > (sh ? p.T : p.T * p.K)) return false;
  if (it.ntile < 0) return false;
  return gu ? it.ntile * gu_tile < (sh ? p.Is : p.I) : it.ntile * dn_tile < p.H;
}

// Work item `i` of one kind from its per-slot item prefix sums (in shared
// memory): the slot is the last one whose first item is <= i; within a slot
// the row tile varies fastest, so CTAs that run at the same time share a
// weight tile in L2.
__device__ __forceinline__ WorkItem decode_item(int i, const int* s_start, const int* s_off,
                                                int nslots, int E, int T, int bn) {
  int lo = 0, hi = nslots;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s_start[mid] <= i) lo = mid;
    else hi = mid;
  }
  const int e = lo;
  const bool sh = e == E;
  const int rows = sh ? T : s_off[e + 1] - s_off[e];
  const int r0 = sh ? 0 : s_off[e];
  const int nm = max(1, (rows + bn - 1) / bn);
  const int local = i - s_start[e];
  const int n = local / nm, m = local - n * nm;
  return WorkItem{e, r0 + m * bn, min(bn, rows - m * bn), n};
}

}  // namespace
}  // namespace sgl
