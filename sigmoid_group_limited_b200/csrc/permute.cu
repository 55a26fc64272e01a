// permute.cu - stage 6: group the T*K (token, slot) pairs by expert.
//
// Each token selects K experts (page "Ling-3.0-flash-VL MoE sparse routing",
// sec. 3 step 2); the expert FFNs then run on the rows routed to them. The
// order is a stable counting sort of the flat slot index j = t*K + k by
// expert id, so it is deterministic and equal to the oracle's.
//
// Three kernels over tiles of kPermTile flat entries:
//   perm_hist    per-tile expert histogram (shared-memory atomics; counts do
//                not depend on their order),
//   perm_scan    one CTA: per-expert totals, exclusive offsets, per-(expert,
//                tile) bases, and the GEMM work lists,
//   perm_scatter per tile: stable ranks from warp match/ballot in flat order,
//                then perm / inv_perm.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace sgl {
namespace {

constexpr int kMaxE = 1024;
constexpr int kScanSmemInts = 48 * 1024;  // tile counts perm_scan stages in shared memory (192 KB)
constexpr int kScatterWarps = 8;

__global__ void __launch_bounds__(256) perm_hist(int TK, int E, int n_ptiles,
                                                 const int32_t* __restrict__ idx,
                                                 int32_t* __restrict__ tile_cnt,  // [E][n_ptiles]
                                                 int32_t* __restrict__ err) {
  pdl_trigger();
  pdl_wait();  // inputs come from earlier kernels on the stream
  __shared__ int hist[kMaxE];
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int base = blockIdx.x * kPermTile;
  const int n = min(kPermTile, TK - base);
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int e = idx[base + i];
    if (e < 0 || e >= E) {
      atomicExch(err, MOE_DEVERR_EXPERT_ID);
      continue;
    }
    atomicAdd(&hist[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    tile_cnt[static_cast<size_t>(e) * n_ptiles + blockIdx.x] = hist[e];
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
  if (a.ready) {
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

__global__ void __launch_bounds__(1024) perm_scan(int E, int n_ptiles,
                                                  const int32_t* __restrict__ tile_cnt,
                                                  int32_t* __restrict__ tile_base,
                                                  int32_t* __restrict__ counts,
                                                  int32_t* __restrict__ offsets, SchedArgs sa,
                                                  int build, int stage_smem) {
  pdl_trigger();
  pdl_wait();  // inputs come from earlier kernels on the stream
  __shared__ int cnt[kMaxE + 1];
  __shared__ int off[kMaxE + 1];
  __shared__ int scratch[33];
  extern __shared__ int tc_s[];  // the tile counts, when they fit (else read from global)
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int ncnt = E * n_ptiles;
  const int32_t* tc = tile_cnt;
  if (stage_smem && ncnt <= kScanSmemInts) {  // the launch provided E * n_ptiles ints
    // one coalesced sweep, all loads in flight, instead of a dependent load per expert
    for (int i = threadIdx.x; i < ncnt; i += blockDim.x) tc_s[i] = tile_cnt[i];
    __syncthreads();
    tc = tc_s;
  }
  // per-expert totals: one warp per expert, lanes over tiles
  for (int e = warp; e < E; e += nw) {
    int s = 0;
    for (int t = lane; t < n_ptiles; t += 32) s += tc[static_cast<size_t>(e) * n_ptiles + t];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) cnt[e] = s;
  }
  __syncthreads();
  int total;
  const int e0 = 2 * threadIdx.x;
  const int c0 = e0 < E ? cnt[e0] : 0, c1 = e0 + 1 < E ? cnt[e0 + 1] : 0;
  const int ex = block_exscan2(c0, c1, scratch, &total);
  if (e0 < E) off[e0] = ex;
  if (e0 + 1 < E) off[e0 + 1] = ex + c0;
  if (threadIdx.x == 0) off[E] = total;
  __syncthreads();
  for (int e = threadIdx.x; e <= E; e += blockDim.x) {
    offsets[e] = off[e];
    if (e < E) counts[e] = cnt[e];
  }
  // per-(expert, tile) exclusive bases: one warp per expert, warp scan over tiles
  for (int e = warp; e < E; e += nw) {
    int carry = off[e];
    for (int t0 = 0; t0 < n_ptiles; t0 += 32) {
      const int t = t0 + lane;
      const int v = t < n_ptiles ? tc[static_cast<size_t>(e) * n_ptiles + t] : 0;
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (t < n_ptiles) tile_base[static_cast<size_t>(e) * n_ptiles + t] = carry + incl - v;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
  if (build) build_schedule(sa, cnt, scratch);
}

__global__ void __launch_bounds__(1024) schedule_only(const int32_t* __restrict__ offsets,
                                                      SchedArgs sa) {
  pdl_trigger();
  pdl_wait();  // inputs come from earlier kernels on the stream
  __shared__ int cnt[kMaxE + 1];
  __shared__ int scratch[33];
  for (int e = threadIdx.x; e < sa.E; e += blockDim.x) cnt[e] = offsets[e + 1] - offsets[e];
  __syncthreads();
  build_schedule(sa, cnt, scratch);
}

__global__ void __launch_bounds__(kScatterWarps * 32) perm_scatter(
    int TK, int E, int n_ptiles, const int32_t* __restrict__ idx,
    const int32_t* __restrict__ tile_base, int32_t* __restrict__ perm,
    int32_t* __restrict__ inv_perm, int32_t* __restrict__ err) {
  pdl_trigger();
  pdl_wait();  // inputs come from earlier kernels on the stream
  __shared__ int whist[kScatterWarps][kMaxE];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < kScatterWarps * E; i += blockDim.x) whist[i / E][i % E] = 0;
  __syncthreads();
  const int tbase = blockIdx.x * kPermTile;
  const int n = min(kPermTile, TK - tbase);
  constexpr int chunk = kPermTile / kScatterWarps;
  const int c0 = warp * chunk, c1 = min(c0 + chunk, n);
  const unsigned lt = (1u << lane) - 1u;
  // pass 1: this warp's per-expert counts (its chunk is contiguous in flat order)
  for (int r = c0; r < c1; r += 32) {
    const int i = r + lane;
    int e = -1;
    if (i < c1) {
      e = idx[tbase + i];
      if (e < 0 || e >= E) e = -1;
    }
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && (peers & lt) == 0) whist[warp][e] += __popc(peers);
  }
  __syncthreads();
  // exclusive scan over warps, seeded with the tile's base for each expert
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = tile_base[static_cast<size_t>(e) * n_ptiles + blockIdx.x];
#pragma unroll
    for (int w = 0; w < kScatterWarps; ++w) {
      const int v = whist[w][e];
      whist[w][e] = run;
      run += v;
    }
  }
  __syncthreads();
  // pass 2: stable positions
  for (int r = c0; r < c1; r += 32) {
    const int i = r + lane;
    int e = -1;
    if (i < c1) {
      e = idx[tbase + i];
      if (e < 0 || e >= E) e = -1;
    }
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    int pos = -1;
    if (e >= 0) pos = whist[warp][e] + __popc(peers & lt);
    __syncwarp();
    if (e >= 0 && (peers & lt) == 0) whist[warp][e] += __popc(peers);
    __syncwarp();
    if (i < c1) {
      const int j = tbase + i;
      if (e >= 0 && (pos < 0 || pos >= TK)) {  // cannot happen for consistent counts
        atomicExch(err, MOE_DEVERR_SCHEDULE);
        pos = -1;
        e = -1;
      }
      if (e >= 0) perm[pos] = j;
      if (inv_perm) inv_perm[j] = pos;
    }
  }
}

// The whole permutation in one CTA when all T*K entries fit one tile (decode
// batches): per-warp histograms of contiguous chunks, per-expert totals and
// their exclusive scan, per-warp bases, stable positions, and optionally the
// GEMM work lists, with no round trip through global memory in between.
__global__ void __launch_bounds__(1024) perm_single(int TK, int E, const int32_t* __restrict__ idx,
                                                    int32_t* __restrict__ counts,
                                                    int32_t* __restrict__ offsets,
                                                    int32_t* __restrict__ perm,
                                                    int32_t* __restrict__ inv_perm,
                                                    int32_t* __restrict__ err, SchedArgs sa,
                                                    int build) {
  pdl_trigger();
  pdl_wait();  // inputs come from earlier kernels on the stream
  extern __shared__ int whist[];  // [32 warps][E]
  __shared__ int cnt[kMaxE + 1];
  __shared__ int off[kMaxE + 1];
  __shared__ int scratch[33];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < 32 * E; i += blockDim.x) whist[i] = 0;
  __syncthreads();
  const int chunk = ((cdiv_dev(TK, 32) + 31) / 32) * 32;
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
    for (int w = 0; w < 32; ++w) tot += whist[w * E + e];
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
    for (int w = 0; w < 32; ++w) {
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
  const bool mx = c.wfmt == MOE_W_MXFP4_A8;
  a.gu_ft = mx ? kMxGuTile : kTileN;
  a.dn_ft = mx ? kMxDnTile : kDownTile;
  a.gu_start = gu_start;
  a.dn_start = dn_start;
  a.ready = ready;
  a.nitems = nitems;
  return a;
}

}  // namespace

cudaError_t launch_permute(const moe_cfg& c, int T, const int32_t* idx, int32_t* tile_cnt,
                           int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv_perm,
                           int32_t* err, const WsLayout& L, int32_t* gu_start,
                           int32_t* dn_start, int32_t* ready, int32_t* nitems, cudaStream_t s) {
  const int TK = T * c.K;
  const int np = L.n_ptiles;
  SchedArgs sa = make_sched(c, T, L, gu_start, dn_start, ready, nitems);
  if (np == 1) {
    const int smem = 32 * c.E * static_cast<int>(sizeof(int));
    cudaError_t e = ensure_dyn_smem(reinterpret_cast<const void*>(perm_single),
                                    32 * kMaxE * static_cast<int>(sizeof(int)));
    if (e != cudaSuccess) return e;
    return launch_pdl(perm_single, dim3(1), dim3(1024), smem, s, TK, c.E, idx, counts, offsets, perm,
                      inv_perm, err, sa, gu_start != nullptr ? 1 : 0);
  }
  int32_t* tile_base = tile_cnt + static_cast<size_t>(c.E) * np;
  cudaError_t e = launch_pdl(perm_hist, dim3(np), dim3(256), 0, s, TK, c.E, np, idx, tile_cnt, err);
  if (e != cudaSuccess) return e;
  const int scan_smem = c.E * np <= kScanSmemInts ? c.E * np * static_cast<int>(sizeof(int)) : 0;
  if (scan_smem > 0) {
    e = ensure_dyn_smem(reinterpret_cast<const void*>(perm_scan),
                        kScanSmemInts * static_cast<int>(sizeof(int)));
    if (e != cudaSuccess) return e;
  }
  e = launch_pdl(perm_scan, dim3(1), dim3(1024), scan_smem, s, c.E, np,
                 static_cast<const int32_t*>(tile_cnt), tile_base, counts, offsets, sa,
                 gu_start != nullptr ? 1 : 0, scan_smem > 0 ? 1 : 0);
  if (e != cudaSuccess) return e;
  return launch_pdl(perm_scatter, dim3(np), dim3(kScatterWarps * 32), 0, s, TK, c.E, np, idx,
                    static_cast<const int32_t*>(tile_base), perm, inv_perm, err);
}

// ---------------------------------------------------------------------------
// Scratch for moe_permute_static, for callers that cannot allocate device
// memory: the per-(expert, tile) counts and bases of the three kernels above
// plus an error word, in one file-scope device array of fixed size. Every
// device that loads the library holds it until the process exits.
// Layout (int32): [0] error word, [1..63] unused, [64, 64 + E*n_tiles)
// counts, then E*n_tiles bases.
// ---------------------------------------------------------------------------
constexpr int kStaticScratchHead = 64;
constexpr int kStaticScratchInts =
    kStaticScratchHead + 2 * kStaticMaxExperts * (kStaticMaxSlots / kPermTile);
static __device__ __align__(256) int32_t g_permute_scratch[kStaticScratchInts];

// Device address of g_permute_scratch on the current device, looked up once
// per device (with that device current) and cached; nullptr on failure.
static int32_t* static_scratch_address() {
  static std::mutex mu;
  static int32_t* addr[kMaxDevices] = {};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<int32_t*>(p);
  }
  return addr[dev];
}

cudaError_t launch_permute_static(const moe_cfg& c, int T, const int32_t* idx, int32_t* counts,
                                  int32_t* offsets, int32_t* perm, int32_t* inv_perm,
                                  cudaStream_t s) {
  const int TK = T * c.K;
  const int np = cdiv(TK, kPermTile);
  int32_t* base = static_scratch_address();
  if (base == nullptr) return cudaErrorInvalidSymbol;
  int32_t* err = base;
  int32_t* tile_cnt = base + kStaticScratchHead;
  int32_t* tile_base = tile_cnt + static_cast<size_t>(c.E) * np;
  // the error word must start at zero; the tile arrays are fully written
  cudaError_t e = cudaMemsetAsync(err, 0, sizeof(int32_t), s);
  if (e != cudaSuccess) return e;
  perm_hist<<<np, 256, 0, s>>>(TK, c.E, np, idx, tile_cnt, err);
  SchedArgs sa{};
  sa.nitems = base + 1;
  sa.ready = nullptr;
  perm_scan<<<1, 1024, 0, s>>>(c.E, np, tile_cnt, tile_base, counts, offsets, sa, 0, 0);
  perm_scatter<<<np, kScatterWarps * 32, 0, s>>>(TK, c.E, np, idx, tile_base, perm, inv_perm,
                                                 err);
  return cudaGetLastError();
}

cudaError_t launch_schedule(const moe_cfg& c, int T, const int32_t* offsets, const WsLayout& L,
                            int32_t* gu_start, int32_t* dn_start, int32_t* ready,
                            int32_t* nitems, cudaStream_t s) {
  SchedArgs sa = make_sched(c, T, L, gu_start, dn_start, ready, nitems);
  return launch_pdl(schedule_only, dim3(1), dim3(1024), 0, s, offsets, sa);
}

}  // namespace sgl
