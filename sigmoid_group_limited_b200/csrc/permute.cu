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
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <string.h>

#include <mutex>

#include "internal.h"
#include "permute_dev.cuh"
#include "ptx.cuh"

namespace sgl {
namespace {

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

// The permutation in one CTA of 1024 threads (decode batches).
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
  perm_block(TK, E, idx, counts, offsets, perm, inv_perm, err, sa, build, whist);
}

// The permutation of batches that span several tiles, in one cooperative
// launch of one CTA (1024 threads) per tile of kPermTile flat entries:
//   phase 1  per-warp expert histograms of the tile's 32 contiguous chunks
//            (shared memory), the tile's totals to tile_cnt [E][n_tiles];
//   barrier  (bounded, on a counter that is zero at launch);
//   phase 2  every CTA reads all tiles' counts, forms the per-expert totals,
//            their exclusive scan (the offsets) and the counts of the tiles
//            before its own, turns its warps' histograms into bases and
//            places its entries in flat order: the same stable counting sort
//            as the three-kernel form. CTA 0 writes counts, offsets and the
//            FFN work lists.
__global__ void __launch_bounds__(1024, 1) perm_fused(int TK, int E, int n_ptiles,
                                                      const int32_t* __restrict__ idx,
                                                      int32_t* __restrict__ tile_cnt,
                                                      int32_t* __restrict__ counts,
                                                      int32_t* __restrict__ offsets,
                                                      int32_t* __restrict__ perm,
                                                      int32_t* __restrict__ inv_perm,
                                                      int32_t* __restrict__ bar, int32_t* __restrict__ err,
                                                      SchedArgs sa, int build) {
  pdl_trigger();
  pdl_wait();  // inputs come from earlier kernels on the stream
  extern __shared__ int whist[];  // [32 warps][E]
  __shared__ int cnt[kMaxE + 1];
  __shared__ int off[kMaxE + 1];
  __shared__ int scratch[33];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int kWarps = 32, kChunk = kPermTile / kWarps;
  const int tbase = blockIdx.x * kPermTile;
  const int n = min(kPermTile, TK - tbase);
  const int c0 = warp * kChunk, c1 = min(c0 + kChunk, n);
  const unsigned lt = (1u << lane) - 1u;
  int* wh = whist + warp * E;
  for (int i = tid; i < kWarps * E; i += blockDim.x) whist[i] = 0;
  __syncthreads();
  // phase 1: this warp's per-expert counts of its chunk
  for (int r = c0; r < c1; r += 32) {
    const int i = r + lane;
    int e = -1;
    if (i < c1) {
      e = idx[tbase + i];
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
    for (int w = 0; w < kWarps; ++w) tot += whist[w * E + e];
    tile_cnt[static_cast<size_t>(e) * n_ptiles + blockIdx.x] = tot;
  }
  if (!grid_barrier(bar, 1, err)) return;
  // phase 2: totals, offsets and this tile's base per expert
  int before[2] = {0, 0};
  int tot2[2] = {0, 0};
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const int e = 2 * tid + q;
    if (e < E) {
      const int32_t* row = tile_cnt + static_cast<size_t>(e) * n_ptiles;
      int a = 0, b = 0;
      for (int t = 0; t < n_ptiles; ++t) {
        const int v = __ldcg(row + t);  // written by other CTAs before the barrier
        a += v;
        b += t < static_cast<int>(blockIdx.x) ? v : 0;
      }
      tot2[q] = a;
      before[q] = b;
      cnt[e] = a;
    }
  }
  int total;
  const int ex = block_exscan2(tot2[0], tot2[1], scratch, &total);
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const int e = 2 * tid + q;
    if (e < E) off[e] = ex + (q ? tot2[0] : 0);
  }
  if (tid == 0) off[E] = total;
  __syncthreads();
  if (blockIdx.x == 0) {
    for (int e = tid; e <= E; e += blockDim.x) {
      offsets[e] = off[e];
      if (e < E) counts[e] = cnt[e];
    }
  }
  // per-warp bases, seeded with the expert's offset plus the earlier tiles' counts
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const int e = 2 * tid + q;
    if (e < E) {
      int run = off[e] + before[q];
      for (int w = 0; w < kWarps; ++w) {
        const int v = whist[w * E + e];
        whist[w * E + e] = run;
        run += v;
      }
    }
  }
  __syncthreads();
  // stable positions
  for (int r = c0; r < c1; r += 32) {
    const int i = r + lane;
    int e = -1;
    if (i < c1) {
      e = idx[tbase + i];
      if (e < 0 || e >= E) e = -1;
    }
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    int pos = -1;
    if (e >= 0) pos = wh[e] + __popc(peers & lt);
    __syncwarp();
    if (e >= 0 && (peers & lt) == 0) wh[e] += __popc(peers);
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
  if (build && blockIdx.x == 0) build_schedule(sa, cnt, scratch);
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
  if (np <= num_sms() && getenv("SGL_MOE_PERM") == nullptr) {
    // one cooperative launch, one CTA per tile (all resident: the barrier ends);
    // err[2] of the control block is its barrier counter, zero at this point
    const int smem = 32 * c.E * static_cast<int>(sizeof(int));
    cudaError_t e = ensure_dyn_smem(reinterpret_cast<const void*>(perm_fused),
                                    32 * kMaxE * static_cast<int>(sizeof(int)));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t lc;
    memset(&lc, 0, sizeof(lc));
    lc.gridDim = dim3(np);
    lc.blockDim = dim3(1024);
    lc.dynamicSmemBytes = smem;
    lc.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    lc.attrs = attr;
    lc.numAttrs = 1;
    return cudaLaunchKernelEx(&lc, perm_fused, TK, c.E, np, idx, tile_cnt, counts, offsets, perm,
                              inv_perm, err + 2, err, sa, gu_start != nullptr ? 1 : 0);
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
// moe_permute_static accepts any E that the configuration check accepts
static_assert(kStaticMaxExperts >= kMaxExpertsCfg, "static scratch smaller than the largest E");

// Device address of g_permute_scratch in the calling thread's current CUDA
// context, looked up once per context (with that context current) and cached
// under the context handle, so a device reset or another context on the same
// device gets its own lookup; nullptr on failure.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

static CUcontext current_context() {
  static const CtxGetCurrentFn fn = [] {  // the driver's function, found once (thread-safe)
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<CtxGetCurrentFn>(nullptr);
    return reinterpret_cast<CtxGetCurrentFn>(f);
  }();
  CUcontext ctx = nullptr;
  if (fn == nullptr || fn(&ctx) != CUDA_SUCCESS) return nullptr;
  return ctx;
}

static int32_t* static_scratch_address() {
  static std::mutex mu;
  static CUcontext ctx_of[kMaxDevices] = {};
  static int32_t* addr[kMaxDevices] = {};
  static int used = 0;
  void* p = nullptr;
  CUcontext ctx = current_context();
  if (ctx == nullptr) {
    // no context bound to this thread yet: the runtime binds the current
    // device's primary context on this first call
    if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess) return nullptr;
    ctx = current_context();
    if (ctx == nullptr) return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < used; ++i)
    if (ctx_of[i] == ctx) return addr[i];
  if (p == nullptr && cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess) return nullptr;
  const int slot = used < kMaxDevices ? used++ : kMaxDevices - 1;  // keep the newest when full
  ctx_of[slot] = ctx;
  addr[slot] = static_cast<int32_t*>(p);
  return addr[slot];
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
