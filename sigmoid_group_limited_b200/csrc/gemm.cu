// gemm.cu - stages 7 and 8: the grouped SwiGLU expert FFN and the shared
// expert, as two persistent tcgen05 GEMM kernels.
//
// Page "Ling-3.0-flash-VL MoE sparse routing" (lqnn.cn/news/282163): sec. 2
// (an expert is a gate / up / down SwiGLU FFN, hidden 2560, intermediate 768;
// one shared expert sees every token) and sec. 4 (SwiGLU limit +-4 on routed
// experts, +-5/+-7 on the shared expert). The limit clamps gate and up to
// [-L, L] before silu(gate) * up.
//
// Both kernels compute D = W_tile * X_tile^T with the weights as the MMA's
// 128-row A operand and a tile of BN tokens as its N (the tokens of one
// expert are few, so the weights fill the 128-row side):
//   gate/up: D_g, D_u [128 features x BN tokens] over K = H, epilogue
//            h = bf16(silu(clamp(D_g)) * clamp(D_u)), stored in permuted row
//            order; the token rows are gathered from x with TMA gather4.
//   down:    D [128 features x BN rows] over K = I, epilogue
//            y_slot[j] = w_j * D (fp32) written to the slot's flat index j.
// Work items (expert, row tile, output tile) come from a device-built list;
// each CTA walks the list with a grid stride. Warp roles per CTA:
//   warp 0  TMA producer (one lane), warp 1  MMA issuer (one lane) and TMEM
//   owner, warps 2..5  epilogue (TMEM lanes 32*(warp%4) ...).
// Pipelines: STAGES shared-memory stages (full/empty mbarriers) and two TMEM
// accumulators (tmem_full/tmem_empty) so the epilogue of one item overlaps
// the main loop of the next. Every wait is bounded (ptx.cuh).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>

#include "internal.h"
#include "ptx.cuh"

namespace sgl {
namespace {

// Warps: 0 weight TMA, 1 MMA, 2..5 epilogue; gate/up adds 6..9 token gatherers.
constexpr int kGatherWarps = 4;
__host__ __device__ constexpr int threads_for(int mode) { return mode == 0 ? 320 : 192; }
constexpr int kSmemBudget = 200 * 1024;

struct GemmParams {
  int T, K, E, H, I, Is;
  const uint16_t* x;  // [T, H] tokens (gate/up operand)
  int has_shared;
  float lim_r, lim_s;  // <= 0: no limit
  const int32_t* perm;
  const float* w;
  uint16_t* h_r;  // [T*K, I] permuted rows
  uint16_t* h_s;  // [T, Is]
  float* z;       // router mode: logits [T, E]
  float* y_slot;   // [(T*K + T), H] fp32
  const int32_t* offsets;  // [E+1] routed row offsets
  const int32_t* wslot;    // nullable: weight row block of expert e
  const int32_t* start;    // [E+2] first work item of each slot (slot E: shared expert)
  const int32_t* nitems;   // device count of valid items
  int max_items;
  int32_t* err;
};

__host__ __device__ constexpr int pow2_at_least(int v) {
  int p = 32;
  while (p < v) p <<= 1;
  return p;
}

template <int MODE, int BN>
struct Cfg {
  // weight tiles per stage: gate + up (0), down (1), router hi + mid + lo (2)
  static constexpr int NA = MODE == 0 ? 2 : (MODE == 2 ? 3 : 1);
  static constexpr int A_BYTES = kTileN * 128;       // 128 rows x 64 bf16
  static constexpr int B_BYTES = BN * 128;           // BN rows x 64 bf16
  static constexpr int STAGE_BYTES = NA * A_BYTES + B_BYTES;
  static constexpr int STAGES_RAW = kSmemBudget / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
  // fp32 columns per accumulator buffer: gate and up side by side (0), one (1, 2)
  static constexpr int ACC_COLS = (MODE == 0 ? 2 : 1) * BN;
  // router mode: two hi-term chunk buffers + the mid and lo accumulators
  static constexpr int TMEM_COLS = pow2_at_least(MODE == 2 ? 4 * BN : 2 * ACC_COLS);
  static_assert(TMEM_COLS <= 512, "two accumulator buffers must fit the 512 TMEM columns");
  static constexpr int SMEM = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/ +
                             BN * 4 /*token rows*/ + BN * 8 /*row metadata*/;
};

// Named barrier 1 over the four epilogue warps (128 threads).
__device__ __forceinline__ void epilogue_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ float clampL(float v, float L) {
  return L > 0.f ? fminf(fmaxf(v, -L), L) : v;
}

__device__ __forceinline__ uint16_t f2bf(float v) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

// Same validity rule in every role, so all roles skip the same items.
__device__ __forceinline__ bool item_ok(const GemmParams& p, const WorkItem& it, int mode,
                                        int bn) {
  if (mode == 2)
    return it.e == 0 && it.nrows > 0 && it.nrows <= bn && it.row0 >= 0 &&
           it.row0 + it.nrows <= p.T && it.ntile >= 0 && it.ntile * kTileN < p.E;
  const bool sh = it.e == p.E;
  if (it.e < 0 || it.e > p.E || (sh && !p.has_shared)) return false;
  if (it.nrows <= 0 || it.nrows > bn || it.row0 < 0) return false;
  const int rows = sh ? p.T : p.T * p.K;
  if (it.row0 + it.nrows > rows) return false;
  const int nt = mode == 0 ? (sh ? p.Is : p.I) : p.H;
  if (it.ntile < 0 || it.ntile * kTileN >= nt) return false;
  return true;
}

// Work item `i` from the per-slot item prefix sums (staged in shared memory):
// the slot is the last one whose first item is <= i; within a slot the row
// tile varies fastest, so neighbouring CTAs share a weight tile in L2.
__device__ __forceinline__ WorkItem decode_item(int i, const int* s_start, const int* s_off,
                                                int nslots, int E, int T, int bn, int mode,
                                                int nt_r, int nt_s) {
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
  (void)mode;
  (void)nt_r;
  (void)nt_s;
  return WorkItem{e, r0 + m * bn, min(bn, rows - m * bn), n};
}

template <int MODE, int BN>
__global__ void __launch_bounds__(threads_for(MODE), 1)
    moe_gemm(const __grid_constant__ GemmParams p, const __grid_constant__ CUtensorMap tA0,
             const __grid_constant__ CUtensorMap tA1, const __grid_constant__ CUtensorMap tS0,
             const __grid_constant__ CUtensorMap tS1, const __grid_constant__ CUtensorMap tB0,
             const __grid_constant__ CUtensorMap tB1) {
  using C = Cfg<MODE, BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* tfull = empty + C::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* hfull = tempty + 2;   // router mode: hi-term chunk buffers
  uint64_t* hempty = hfull + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(hempty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* tok = reinterpret_cast<int*>(smem + C::STAGES * C::STAGE_BYTES + 256);
  int* meta_j = tok + BN;                                       // down: slot of each row
  float* meta_w = reinterpret_cast<float*>(meta_j + BN);        // down: its routing weight
  int* s_start = reinterpret_cast<int*>(meta_w + BN);           // [E+2] item starts
  int* s_off = s_start + (p.E + 2);                             // [E+1] row offsets

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      // gate/up: the weight TMA arrival plus one arrival per token-gatherer thread
      mbar_init(&full[s], MODE == 0 ? 1 + kGatherWarps * 32 : 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);
      mbar_init(&hfull[a], 1);
      mbar_init(&hempty[a], 4);
    }
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tA0);
    prefetch_tmap(&tB0);
    if (p.has_shared) prefetch_tmap(&tS0);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (MODE != 2) {
    for (int i = threadIdx.x; i < p.E + 2; i += blockDim.x) s_start[i] = p.start[i];
    for (int i = threadIdx.x; i < p.E + 1; i += blockDim.x) s_off[i] = p.offsets[i];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int nslots = p.E + (p.has_shared ? 1 : 0);
  auto item_at = [&](int i) {
    if (MODE == 2) {  // router: output tile n of 128 experts x token tile m
      const int nm = (p.T + BN - 1) / BN;
      const int n = i / nm, m = i - n * nm;
      return WorkItem{0, m * BN, min(BN, p.T - m * BN), n};
    }
    return decode_item(i, s_start, s_off, nslots, p.E, p.T, BN, MODE, 0, 0);
  };
  const int n_items = p.nitems ? min(*p.nitems, p.max_items) : p.max_items;
  const int KB_r = (MODE == 1 ? p.I : p.H) / 64;
  const int KB_s = (MODE == 1 ? p.Is : p.H) / 64;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    const uint64_t pol_w = policy_evict_first();
    const uint64_t pol_x = policy_evict_last();
    int stage = 0;
    uint32_t phase = 0;
    bool live = true;
    for (int item = blockIdx.x; item < n_items && live; item += gridDim.x) {
      const WorkItem it = item_at(item);
      if (!item_ok(p, it, MODE, BN)) {
        if (lane == 0) atomicExch(p.err, MOE_DEVERR_SCHEDULE);
        continue;
      }
      const bool sh = it.e == p.E;
      if (lane == 0) {
        const int nkb = sh ? KB_s : KB_r;
        const int wblk = (MODE != 2 && p.wslot) ? p.wslot[it.e] : it.e;
        const int arow = (sh || MODE == 2) ? it.ntile * kTileN
                                           : wblk * (MODE == 0 ? p.I : p.H) + it.ntile * kTileN;
        const CUtensorMap* mA0 = sh ? &tS0 : &tA0;
        const CUtensorMap* mA1 = sh ? &tS1 : &tA1;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) {
            live = false;
            break;
          }
          uint8_t* sA = smem + stage * C::STAGE_BYTES;
          uint8_t* sB = sA + C::NA * C::A_BYTES;
          if (MODE == 0) {
            // weights only; the token rows come from the gatherer warps
            mbar_arrive_expect_tx(&full[stage], C::NA * C::A_BYTES);
            tma_load_2d(sA, mA0, &full[stage], kb * 64, arow, pol_w);
            tma_load_2d(sA + C::A_BYTES, mA1, &full[stage], kb * 64, arow, pol_w);
          } else if (MODE == 2) {
            // router: the three bf16 terms of the fp32 router rows, and the tokens
            mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
            tma_load_2d(sA, &tA0, &full[stage], kb * 64, arow, pol_x);
            tma_load_2d(sA + C::A_BYTES, &tA1, &full[stage], kb * 64, arow, pol_x);
            tma_load_2d(sA + 2 * C::A_BYTES, &tS0, &full[stage], kb * 64, arow, pol_x);
            tma_load_2d(sB, &tB0, &full[stage], kb * 64, it.row0, pol_w);
          } else {
            mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
            tma_load_2d(sA, mA0, &full[stage], kb * 64, arow, pol_w);
            tma_load_2d(sB, sh ? &tB1 : &tB0, &full[stage], kb * 64, it.row0, pol_x);
          }
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      live = __shfl_sync(0xffffffffu, live ? 1 : 0, 0) != 0;
      __syncwarp();
    }
    // drain: every stage must be released by its MMA commit before teardown
    if (lane == 0 && live) {
      for (int i = 0; i < C::STAGES; ++i) {
        if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) break;
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && MODE == 2) {
      // Router: the hi term goes into a fresh chunk accumulator per 64-wide
      // k-block (double-buffered; the epilogue adds the chunks in fp32
      // registers), mid and lo accumulate over the whole K in their own
      // buffers. Short accumulations keep the tensor cores' fp32 rounding small.
      constexpr uint32_t idesc = idesc_bf16(kTileN, BN);
      int stage = 0, ck = 0;
      uint32_t phase = 0, tph = 0;
      bool live = true;
      const uint32_t d_mid = tmem_base + 2 * BN, d_lo = tmem_base + 3 * BN;
      for (int item = blockIdx.x; item < n_items && live; item += gridDim.x) {
        const WorkItem it = item_at(item);
        if (!item_ok(p, it, MODE, BN)) continue;
        if (!mbar_wait(&tempty[0], tph ^ 1, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) break;
        tc_fence_after();
        for (int kb = 0; kb < KB_r; ++kb, ++ck) {
          const int hb = ck & 1;
          const uint32_t hph = (ck >> 1) & 1;
          if (!mbar_wait(&hempty[hb], hph ^ 1, abort_flag, p.err, MOE_DEVERR_TIMEOUT) ||
              !mbar_wait(&full[stage], phase, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) {
            live = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + stage * C::STAGE_BYTES);
          const uint32_t b0 = a0 + C::NA * C::A_BYTES;
          const uint32_t d_hi = tmem_base + hb * BN;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bd = sdesc_k128(b0 + kk * 32);
            const uint32_t acc_all = (kb | kk) != 0 ? 1u : 0u;
            umma_bf16(d_hi, sdesc_k128(a0 + kk * 32), bd, idesc, kk != 0 ? 1u : 0u);
            umma_bf16(d_mid, sdesc_k128(a0 + C::A_BYTES + kk * 32), bd, idesc, acc_all);
            umma_bf16(d_lo, sdesc_k128(a0 + 2 * C::A_BYTES + kk * 32), bd, idesc, acc_all);
          }
          umma_commit(&empty[stage]);
          umma_commit(&hfull[hb]);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!live) break;
        umma_commit(&tfull[0]);
        tph ^= 1;
      }
    } else if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(kTileN, BN);
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool live = true;
      for (int item = blockIdx.x; item < n_items && live; item += gridDim.x) {
        const WorkItem it = item_at(item);
        if (!item_ok(p, it, MODE, BN)) continue;
        const int nkb = it.e == p.E ? KB_s : KB_r;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + acc * C::ACC_COLS;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) {
            live = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + stage * C::STAGE_BYTES);
          const uint32_t b0 = a0 + C::NA * C::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bd = sdesc_k128(b0 + kk * 32);
            const uint32_t accum = (kb | kk) != 0 ? 1u : 0u;
            umma_bf16(d0, sdesc_k128(a0 + kk * 32), bd, idesc, accum);
            if (MODE == 0) umma_bf16(d0 + BN, sdesc_k128(a0 + C::A_BYTES + kk * 32), bd, idesc, accum);
            if (MODE == 2) {  // x * (hi + mid + lo): every product exact, one fp32 accumulator
              umma_bf16(d0, sdesc_k128(a0 + C::A_BYTES + kk * 32), bd, idesc, 1u);
              umma_bf16(d0, sdesc_k128(a0 + 2 * C::A_BYTES + kk * 32), bd, idesc, 1u);
            }
          }
          umma_commit(&empty[stage]);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!live) break;
        umma_commit(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
    }
    __syncwarp();
  } else if (MODE == 0 && warp >= 6) {
    // ------------------------------------------------------------ token gatherers
    // Thread g copies 16-byte chunk (g % 8) of rows g/8, g/8 + 16, ... of the
    // stage's BN x 64 token tile, straight into the 128-byte-swizzled layout
    // (chunk c of row r lands at chunk c ^ (r % 8)). A stage's copies are
    // retired two stages later: wait for the group, make it visible to the
    // tensor cores (proxy fence), then arrive on the stage's full barrier.
    constexpr int kRowsPerThread = BN / 16;
    constexpr int kLag = 2;
    const int g = tid - 6 * 32;
    const int chunk = g & 7, rbase = g >> 3;
    const uint64_t pol_x = policy_evict_last();
    int stage = 0;
    uint32_t phase = 0;
    int pend0 = -1, pend1 = -1;  // stages issued two and one steps ago, not yet retired
    bool live = true;
    for (int item = blockIdx.x; item < n_items && live; item += gridDim.x) {
      const WorkItem it = item_at(item);
      if (!item_ok(p, it, MODE, BN)) continue;
      const bool sh = it.e == p.E;
      const int nkb = sh ? KB_s : KB_r;
      const uint16_t* src[kRowsPerThread];
#pragma unroll
      for (int i = 0; i < kRowsPerThread; ++i) {
        const int row = it.row0 + min(rbase + 16 * i, it.nrows - 1);
        int t = sh ? row : p.perm[row] / p.K;
        t = min(max(t, 0), p.T - 1);
        src[i] = p.x + static_cast<size_t>(t) * p.H + chunk * 8;
      }
      for (int kb = 0; kb < nkb; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) {
          live = false;
          break;
        }
        uint8_t* sB = smem + stage * C::STAGE_BYTES + C::NA * C::A_BYTES;
#pragma unroll
        for (int i = 0; i < kRowsPerThread; ++i) {
          const int r = rbase + 16 * i;
          cp_async16(sB + r * 128 + ((chunk ^ (r & 7)) << 4), src[i] + kb * 64, pol_x);
        }
        cp_async_commit();
        if (pend0 >= 0) {
          cp_async_wait<kLag>();  // all but the two newest groups have landed
          fence_proxy_async_smem();
          mbar_arrive(&full[pend0]);
        }
        pend0 = pend1;
        pend1 = stage;
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    cp_async_wait<0>();  // nothing may still be landing in shared memory at exit
    fence_proxy_async_smem();
    if (live) {
      if (pend0 >= 0) mbar_arrive(&full[pend0]);
      if (pend1 >= 0) mbar_arrive(&full[pend1]);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                  // TMEM lane quarter of this warp
    const int orow = q * 32 + lane;          // output feature within the tile
    int acc = 0;
    uint32_t acc_phase = 0;
    if (MODE == 2) {
      // router: z = sum over k-blocks of the hi chunks (fp32, in order) + mid + lo
      int ck = 0;
      uint32_t tph = 0;
      const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
      for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        const WorkItem it = item_at(item);
        if (!item_ok(p, it, MODE, BN)) continue;
        float sum[BN];
#pragma unroll
        for (int c = 0; c < BN; ++c) sum[c] = 0.f;
        bool live = true;
        for (int kb = 0; kb < KB_r; ++kb, ++ck) {
          const int hb = ck & 1;
          if (!mbar_wait(&hfull[hb], (ck >> 1) & 1, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) {
            live = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int c0 = 0; c0 < BN; c0 += 32) {
            float v0[16], v1[16];
            tmem_ld16(lane_base + hb * BN + c0, v0);
            tmem_ld16(lane_base + hb * BN + c0 + 16, v1);
            tmem_ld_wait();
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              sum[c0 + c] += v0[c];
              sum[c0 + 16 + c] += v1[c];
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&hempty[hb]);
        }
        if (!live || !mbar_wait(&tfull[0], tph, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) break;
        tc_fence_after();
#pragma unroll
        for (int c0 = 0; c0 < BN; c0 += 16) {
          float vm[16], vl[16];
          tmem_ld16(lane_base + 2 * BN + c0, vm);
          tmem_ld16(lane_base + 3 * BN + c0, vl);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 16; ++c) sum[c0 + c] += vm[c] + vl[c];
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[0]);
        tph ^= 1;
        const int e = it.ntile * kTileN + orow;
        if (e < p.E) {
#pragma unroll
          for (int c = 0; c < BN; ++c)
            if (c < it.nrows) p.z[static_cast<size_t>(it.row0 + c) * p.E + e] = sum[c];
        }
      }
    }
    for (int item = blockIdx.x; item < (MODE == 2 ? 0 : n_items); item += gridDim.x) {
      const WorkItem it = item_at(item);
      if (!item_ok(p, it, MODE, BN)) continue;
      const bool sh = it.e == p.E;
      if (MODE == 1) {
        // destination slot and routing weight of every row of the item, loaded
        // while the item's MMAs run (the store loop then touches no metadata in
        // global memory)
        epilogue_bar();  // all four warps are done with the previous item's rows
        if (orow < BN) {
          int j = -1;
          float wt = 0.f;
          if (orow < it.nrows) {
            const int row = it.row0 + orow;
            if (sh) {
              j = p.T * p.K + row;
              wt = 1.0f;
            } else {
              j = p.perm[row];
              if (j < 0 || j >= p.T * p.K) {  // a bad permutation: report, never store
                atomicExch(p.err, MOE_DEVERR_SCHEDULE);
                j = -1;
              } else {
                wt = p.w[j];
              }
            }
          }
          meta_j[orow] = j;
          meta_w[orow] = wt;
        }
        epilogue_bar();
      }
      if (!mbar_wait(&tfull[acc], acc_phase, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * C::ACC_COLS;
      const int nfeat = it.ntile * kTileN + orow;
      if (MODE == 0) {
        const int ncols = sh ? p.Is : p.I;
        const bool ok = nfeat < ncols;
        const float L = sh ? p.lim_s : p.lim_r;
        uint16_t* hout = sh ? p.h_s : p.h_r;
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 16) {
          float gv[16], uv[16];
          tmem_ld16(taddr + c0, gv);
          tmem_ld16(taddr + BN + c0, uv);
          tmem_ld_wait();
          if (ok) {
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const int r = c0 + c;
              if (r < it.nrows) {
                const float g = clampL(gv[c], L), u = clampL(uv[c], L);
                const float hval = (g / (1.0f + expf(-g))) * u;
                hout[static_cast<size_t>(it.row0 + r) * ncols + nfeat] = f2bf(hval);
              }
            }
          }
        }
      } else {
        const bool ok = nfeat < p.H;
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 16) {
          float ov[16];
          tmem_ld16(taddr + c0, ov);
          tmem_ld_wait();
          if (ok) {
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const int j = meta_j[c0 + c];
              if (j >= 0) p.y_slot[static_cast<size_t>(j) * p.H + nfeat] = meta_w[c0 + c] * ov[c];
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ===========================================================================
// Fused expert FFN: gate/up and down in one persistent, cooperative launch.
// Item space: [0, Ngu) gate/up items, then [Ngu, Ngu + Ndn) down items, both
// decoded from their per-slot prefix sums. Items are claimed dynamically: a
// CTA's producer takes the next index from a global counter and hands it to
// the CTA's other roles through a small shared-memory queue. Indices are
// claimed in increasing order, so every gate/up item is claimed before any
// down item.
// A down item (slot e, row tile m) reads h rows written by the gate/up
// epilogues of other CTAs: those epilogues count finished output tiles per
// (e, m) in ready[] (stores, proxy fence, CTA barrier, threadfence, atomic);
// the producer waits with an acquire load until all of the slot's output tiles
// are in. Gate/up items never wait, and the cooperative launch keeps every CTA
// resident, so every waited-for item is owned by a running CTA that does it
// first. Waits are bounded like every other wait here.
// ===========================================================================
constexpr int kFusedThreads = 320;

struct FusedParams {
  GemmParams g;
  const int32_t* gu_start;  // [E+2]
  const int32_t* dn_start;  // [E+2]
  int32_t* ready;           // [max_gu] finished gate/up output tiles per (slot, row tile)
  int32_t* counter;         // next unclaimed item (zeroed by the schedule builder)
  int max_gu, max_dn;
};
constexpr int kQueue = 4;  // items a CTA's producer may run ahead of its slowest role

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}
__device__ __forceinline__ int ld_acquire(const int32_t* a) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(a) : "memory");
  return v;
}

// Bounded wait until *addr >= need (acquire). Same abort protocol as mbar_wait.
__device__ __forceinline__ bool wait_count(const int32_t* addr, int need, volatile int* abort_flag,
                                           int* err) {
  const long long t0 = clock64();
  while (ld_acquire(addr) < need) {
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitLimitCycles) {
      *abort_flag = 1;
      atomicExch(err, MOE_DEVERR_TIMEOUT);
      return false;
    }
    __nanosleep(100);
  }
  return true;
}

template <int BN>
__global__ void __launch_bounds__(kFusedThreads, 1)
    moe_ffn_fused(const __grid_constant__ FusedParams fp, const __grid_constant__ CUtensorMap tWg,
                  const __grid_constant__ CUtensorMap tWu, const __grid_constant__ CUtensorMap tWgS,
                  const __grid_constant__ CUtensorMap tWuS, const __grid_constant__ CUtensorMap tWd,
                  const __grid_constant__ CUtensorMap tWdS, const __grid_constant__ CUtensorMap tH,
                  const __grid_constant__ CUtensorMap tHs) {
  using C = Cfg<0, BN>;  // stage = gate + up tiles + token tile (down uses one A tile)
  const GemmParams& p = fp.g;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* tfull = empty + C::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* qfull = tempty + 2;   // item queue: producer -> the other roles
  uint64_t* qempty = qfull + kQueue;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(qempty + kQueue);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* qitem = reinterpret_cast<volatile int*>(tmem_slot + 2);  // [kQueue]
  int* meta_j = reinterpret_cast<int*>(smem + C::STAGES * C::STAGE_BYTES + 256);
  float* meta_w = reinterpret_cast<float*>(meta_j + BN);
  int* s_gu = reinterpret_cast<int*>(meta_w + BN);  // [E+2]
  int* s_dn = s_gu + (p.E + 2);                      // [E+2]
  int* s_off = s_dn + (p.E + 2);                     // [E+1]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1 + kGatherWarps);  // weight TMA + one arrival per gatherer warp
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);
    }
    for (int q = 0; q < kQueue; ++q) {
      mbar_init(&qfull[q], 1);
      mbar_init(&qempty[q], 1 + 4 + kGatherWarps);  // MMA lane, epilogue and gatherer warps
    }
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tWg);
    prefetch_tmap(&tWd);
    prefetch_tmap(&tH);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  for (int i = tid; i < p.E + 2; i += blockDim.x) {
    s_gu[i] = fp.gu_start[i];
    s_dn[i] = fp.dn_start[i];
  }
  for (int i = tid; i < p.E + 1; i += blockDim.x) s_off[i] = p.offsets[i];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int nslots = p.E + (p.has_shared ? 1 : 0);
  const int n_gu = min(p.nitems[0], fp.max_gu);
  const int n_dn = min(p.nitems[1], fp.max_dn);
  const int n_all = n_gu + n_dn;
  // item i -> (is gate/up, work item)
  auto item_at = [&](int i, bool& gu) {
    gu = i < n_gu;
    return gu ? decode_item(i, s_gu, s_off, nslots, p.E, p.T, BN, 0, 0, 0)
              : decode_item(i - n_gu, s_dn, s_off, nslots, p.E, p.T, BN, 1, 0, 0);
  };
  // ready[] index of (slot, row tile) of an item
  auto ready_idx = [&](const WorkItem& it) {
    const int r0 = it.e == p.E ? 0 : s_off[it.e];
    return s_gu[it.e] + (it.row0 - r0) / BN;
  };
  // next item index from the queue (every role reads every entry once);
  // -1 ends the walk. One arrival per warp (lane 0) frees the entry.
  // whole_warp: every lane of the calling warp takes part (else lane 0 alone)
  auto next_item = [&](int n, int& item, bool whole_warp) -> bool {
    const int q = n % kQueue;
    if (!mbar_wait(&qfull[q], (n / kQueue) & 1, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) return false;
    item = qitem[q];
    if (whole_warp) __syncwarp();
    if (lane == 0) mbar_arrive(&qempty[q]);
    return item >= 0;
  };
  const int KB_gu = p.H / 64;
  const int KB_dn_r = p.I / 64, KB_dn_s = p.Is / 64;
  auto nkb_of = [&](bool gu, bool sh) { return gu ? KB_gu : (sh ? KB_dn_s : KB_dn_r); };

  if (warp == 0) {
    // ------------------------------------------------------------ weight / h TMA
    const uint64_t pol_w = policy_evict_first();
    const uint64_t pol_h = policy_evict_last();
    int stage = 0;
    uint32_t phase = 0;
    bool live = true;
    for (int n = 0; live; ++n) {
      // claim the next item (dynamic: whoever is free takes it) and queue it
      int item = -1;
      if (lane == 0) {
        const int q = n % kQueue;
        if (!mbar_wait(&qempty[q], ((n / kQueue) & 1) ^ 1, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) {
          live = false;
        } else {
          item = atomicAdd(fp.counter, 1);
          if (item >= n_all) item = -1;
          qitem[q] = item;
          mbar_arrive(&qfull[q]);
        }
      }
      item = __shfl_sync(0xffffffffu, item, 0);
      live = __shfl_sync(0xffffffffu, live ? 1 : 0, 0) != 0;
      if (!live || item < 0) break;
      bool gu;
      const WorkItem it = item_at(item, gu);
      if (!item_ok(p, it, gu ? 0 : 1, BN)) {
        if (lane == 0) atomicExch(p.err, MOE_DEVERR_SCHEDULE);
        continue;
      }
      const bool sh = it.e == p.E;
      if (lane == 0) {
        if (!gu) {
          // every gate/up output tile of this (slot, row tile) must be in h
          const int need = cdiv_dev(sh ? p.Is : p.I, kTileN);
          if (!wait_count(fp.ready + ready_idx(it), need, abort_flag, p.err)) live = false;
          fence_proxy_async_global();
        }
        const int wblk = p.wslot ? p.wslot[it.e] : it.e;
        const int nkb = nkb_of(gu, sh);
        for (int kb = 0; kb < nkb && live; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) {
            live = false;
            break;
          }
          uint8_t* sA = smem + stage * C::STAGE_BYTES;
          uint8_t* sB = sA + C::NA * C::A_BYTES;
          if (gu) {
            const int arow = sh ? it.ntile * kTileN : wblk * p.I + it.ntile * kTileN;
            mbar_arrive_expect_tx(&full[stage], 2 * C::A_BYTES);
            tma_load_2d(sA, sh ? &tWgS : &tWg, &full[stage], kb * 64, arow, pol_w);
            tma_load_2d(sA + C::A_BYTES, sh ? &tWuS : &tWu, &full[stage], kb * 64, arow, pol_w);
          } else {
            const int arow = sh ? it.ntile * kTileN : wblk * p.H + it.ntile * kTileN;
            mbar_arrive_expect_tx(&full[stage], C::A_BYTES + C::B_BYTES);
            tma_load_2d(sA, sh ? &tWdS : &tWd, &full[stage], kb * 64, arow, pol_w);
            tma_load_2d(sB, sh ? &tHs : &tH, &full[stage], kb * 64, it.row0, pol_h);
          }
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      live = __shfl_sync(0xffffffffu, live ? 1 : 0, 0) != 0;
      __syncwarp();
    }
    if (lane == 0 && live) {
      for (int i = 0; i < C::STAGES; ++i) {
        if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) break;
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(kTileN, BN);
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool live = true;
      for (int n = 0; live; ++n) {
        int item;
        if (!next_item(n, item, false)) break;
        bool gu;
        const WorkItem it = item_at(item, gu);
        if (!item_ok(p, it, gu ? 0 : 1, BN)) continue;
        const int nkb = nkb_of(gu, it.e == p.E);
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + acc * C::ACC_COLS;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) {
            live = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + stage * C::STAGE_BYTES);
          const uint32_t b0 = a0 + C::NA * C::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bd = sdesc_k128(b0 + kk * 32);
            const uint32_t accum = (kb | kk) != 0 ? 1u : 0u;
            umma_bf16(d0, sdesc_k128(a0 + kk * 32), bd, idesc, accum);
            if (gu) umma_bf16(d0 + BN, sdesc_k128(a0 + C::A_BYTES + kk * 32), bd, idesc, accum);
          }
          umma_commit(&empty[stage]);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!live) break;
        umma_commit(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
    }
    __syncwarp();
  } else if (warp >= 6) {
    // ------------------------------------------------------------ token gatherers
    // gate/up items: copy the routed token rows into the swizzled stage layout
    // (as in the separate gate/up kernel); down items: nothing to copy, but the
    // stage sequence and the full-barrier arrivals stay the same (an empty
    // copy group completes at once).
    constexpr int kRowsPerThread = BN / 16;
    constexpr int kLag = 2;
    const int g = tid - 6 * 32;
    const int chunk = g & 7, rbase = g >> 3;
    const uint64_t pol_x = policy_evict_last();
    int stage = 0;
    uint32_t phase = 0;
    int pend0 = -1, pend1 = -1;
    bool live = true;
    for (int n = 0; live; ++n) {
      int item;
      if (!next_item(n, item, true)) break;
      bool gu;
      const WorkItem it = item_at(item, gu);
      if (!item_ok(p, it, gu ? 0 : 1, BN)) continue;
      const bool sh = it.e == p.E;
      const int nkb = nkb_of(gu, sh);
      const uint16_t* src[kRowsPerThread];
#pragma unroll
      for (int i = 0; i < kRowsPerThread; ++i) {
        const int row = it.row0 + min(rbase + 16 * i, it.nrows - 1);
        int t = 0;
        if (gu) t = sh ? row : p.perm[row] / p.K;
        t = min(max(t, 0), p.T - 1);
        src[i] = p.x + static_cast<size_t>(t) * p.H + chunk * 8;
      }
      for (int kb = 0; kb < nkb; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) {
          live = false;
          break;
        }
        if (gu) {
          uint8_t* sB = smem + stage * C::STAGE_BYTES + C::NA * C::A_BYTES;
#pragma unroll
          for (int i = 0; i < kRowsPerThread; ++i) {
            const int r = rbase + 16 * i;
            cp_async16(sB + r * 128 + ((chunk ^ (r & 7)) << 4), src[i] + kb * 64, pol_x);
          }
        }
        cp_async_commit();
        if (pend0 >= 0) {
          cp_async_wait<kLag>();      // this lane's copies for stage pend0 have landed
          fence_proxy_async_smem();   // ... and are visible to the tensor cores
          __syncwarp();
          if (lane == 0) mbar_arrive(&full[pend0]);
        }
        pend0 = pend1;
        pend1 = stage;
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    cp_async_wait<0>();
    fence_proxy_async_smem();
    __syncwarp();
    if (live && lane == 0) {
      if (pend0 >= 0) mbar_arrive(&full[pend0]);
      if (pend1 >= 0) mbar_arrive(&full[pend1]);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int orow = q * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int n = 0;; ++n) {
      int item;
      if (!next_item(n, item, true)) break;
      bool gu;
      const WorkItem it = item_at(item, gu);
      if (!item_ok(p, it, gu ? 0 : 1, BN)) continue;
      const bool sh = it.e == p.E;
      if (!gu) {
        epilogue_bar();
        if (orow < BN) {
          int j = -1;
          float wt = 0.f;
          if (orow < it.nrows) {
            const int row = it.row0 + orow;
            if (sh) {
              j = p.T * p.K + row;
              wt = 1.0f;
            } else {
              j = p.perm[row];
              if (j < 0 || j >= p.T * p.K) {
                atomicExch(p.err, MOE_DEVERR_SCHEDULE);
                j = -1;
              } else {
                wt = p.w[j];
              }
            }
          }
          meta_j[orow] = j;
          meta_w[orow] = wt;
        }
        epilogue_bar();
      }
      if (!mbar_wait(&tfull[acc], acc_phase, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * C::ACC_COLS;
      const int nfeat = it.ntile * kTileN + orow;
      if (gu) {
        const int ncols = sh ? p.Is : p.I;
        const bool ok = nfeat < ncols;
        const float L = sh ? p.lim_s : p.lim_r;
        uint16_t* hout = sh ? p.h_s : p.h_r;
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 16) {
          float gv[16], uv[16];
          tmem_ld16(taddr + c0, gv);
          tmem_ld16(taddr + BN + c0, uv);
          tmem_ld_wait();
          if (ok) {
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const int r = c0 + c;
              if (r < it.nrows) {
                const float gg = clampL(gv[c], L), uu = clampL(uv[c], L);
                hout[static_cast<size_t>(it.row0 + r) * ncols + nfeat] =
                    f2bf((gg / (1.0f + expf(-gg))) * uu);
              }
            }
          }
        }
      } else {
        const bool ok = nfeat < p.H;
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 16) {
          float ov[16];
          tmem_ld16(taddr + c0, ov);
          tmem_ld_wait();
          if (ok) {
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const int j = meta_j[c0 + c];
              if (j >= 0) p.y_slot[static_cast<size_t>(j) * p.H + nfeat] = meta_w[c0 + c] * ov[c];
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
      if (gu) {
        // publish this output tile of h: stores -> async proxy -> CTA -> GPU
        fence_proxy_async_global();
        epilogue_bar();
        if (warp == 2 && lane == 0) {
          __threadfence();
          atomicAdd(fp.ready + ready_idx(it), 1);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  }
  return fn;
}

// bf16 row-major [rows, cols] matrix, box = box_rows x 64 columns, 128B swizzle.
bool map_bf16(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr || ptr == nullptr || rows == 0) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

GemmParams make_params(const GemmArgs& a, int mode) {
  const moe_cfg& c = *a.cfg;
  GemmParams p;
  p.T = a.T;
  p.K = c.K;
  p.E = c.E;
  p.H = c.H;
  p.I = c.I;
  p.Is = c.I_shared;
  p.has_shared = (c.I_shared > 0 && a.W->Wg_s != nullptr) ? 1 : 0;
  p.lim_r = (c.limit_routed > 0.f && isfinite(c.limit_routed)) ? c.limit_routed : 0.f;
  p.lim_s = (c.limit_shared > 0.f && isfinite(c.limit_shared)) ? c.limit_shared : 0.f;
  p.perm = a.perm;
  p.x = a.x;
  p.w = a.w;
  p.h_r = a.h_r;
  p.h_s = a.h_s;
  p.y_slot = a.y_slot;
  p.offsets = a.offsets;
  p.wslot = a.wslot;
  p.start = mode == 0 ? a.gu_start : a.dn_start;
  p.nitems = a.nitems + mode;
  p.max_items = mode == 0 ? a.max_items_gu : a.max_items_dn;
  p.err = a.err;
  return p;
}

template <int MODE, int BN>
cudaError_t launch_mode(const GemmArgs& a, cudaStream_t s) {
  using C = Cfg<MODE, BN>;
  const moe_cfg& c = *a.cfg;
  GemmParams p = make_params(a, MODE);
  CUtensorMap tA0, tA1, tS0, tS1, tB0, tB1;
  const int T = a.T, TK = a.T * c.K;
  bool ok = true;
  if (MODE == 0) {
    ok &= map_bf16(&tA0, a.Wg, static_cast<uint64_t>(a.wrows) * c.I, c.H, kTileN);
    ok &= map_bf16(&tA1, a.Wu, static_cast<uint64_t>(a.wrows) * c.I, c.H, kTileN);
    ok &= map_bf16(&tB0, a.x, T, c.H, 1);
    tB1 = tB0;
    if (p.has_shared) {
      ok &= map_bf16(&tS0, a.W->Wg_s, c.I_shared, c.H, kTileN);
      ok &= map_bf16(&tS1, a.W->Wu_s, c.I_shared, c.H, kTileN);
    } else {
      tS0 = tA0;
      tS1 = tA1;
    }
  } else {
    ok &= map_bf16(&tA0, a.Wd, static_cast<uint64_t>(a.wrows) * c.H, c.I, kTileN);
    tA1 = tA0;
    ok &= map_bf16(&tB0, a.h_r, TK, c.I, BN);
    if (p.has_shared) {
      ok &= map_bf16(&tS0, a.W->Wd_s, c.H, c.I_shared, kTileN);
      ok &= map_bf16(&tB1, a.h_s, T, c.I_shared, BN);
    } else {
      tS0 = tA0;
      tB1 = tB0;
    }
    tS1 = tS0;
  }
  if (!ok) return cudaErrorInvalidValue;
  auto kern = moe_gemm<MODE, BN>;
  const int smem = C::SMEM + (2 * c.E + 3) * static_cast<int>(sizeof(int));
  cudaError_t e = ensure_dyn_smem(reinterpret_cast<const void*>(kern),
                                  C::SMEM + (2 * 1024 + 3) * static_cast<int>(sizeof(int)));
  if (e != cudaSuccess) return e;
  const int max_items = p.max_items;
  const int grid = max(1, min(num_sms(), max_items));
  kern<<<grid, threads_for(MODE), smem, s>>>(p, tA0, tA1, tS0, tS1, tB0, tB1);
  return cudaGetLastError();
}

}  // namespace

// Router logits on the tensor cores: z[T,E] = x [T,H] . (hi + mid + lo)^T with
// the fp32 router matrix split into three bf16 terms (exact for normal values).
cudaError_t launch_router_gemm(const moe_cfg& c, int T, const uint16_t* x, const uint16_t* w_hi,
                               const uint16_t* w_mid, const uint16_t* w_lo, float* z,
                               int32_t* err, cudaStream_t s) {
  constexpr int BN = 128;
  using C = Cfg<2, BN>;
  GemmParams p;
  memset(&p, 0, sizeof(p));
  p.T = T;
  p.K = c.K;
  p.E = c.E;
  p.H = c.H;
  p.I = c.I;
  p.Is = c.I_shared;
  p.x = x;
  p.z = z;
  p.err = err;
  p.nitems = nullptr;
  p.max_items = cdiv(c.E, kTileN) * cdiv(T, BN);
  CUtensorMap tA0, tA1, tS0, tB0;
  bool ok = map_bf16(&tA0, w_hi, c.E, c.H, kTileN) && map_bf16(&tA1, w_mid, c.E, c.H, kTileN) &&
            map_bf16(&tS0, w_lo, c.E, c.H, kTileN) && map_bf16(&tB0, x, T, c.H, BN);
  if (!ok) return cudaErrorInvalidValue;
  auto kern = moe_gemm<2, BN>;
  const int smem = C::SMEM + (2 * 1024 + 3) * static_cast<int>(sizeof(int));
  cudaError_t e = ensure_dyn_smem(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  const int grid = std::max(1, std::min(num_sms(), p.max_items));
  kern<<<grid, threads_for(2), smem, s>>>(p, tA0, tA1, tS0, tS0, tB0, tB0);
  return cudaGetLastError();
}

namespace {

template <int BN>
cudaError_t launch_fused_bn(const GemmArgs& a, cudaStream_t s) {
  using C = Cfg<0, BN>;
  const moe_cfg& c = *a.cfg;
  FusedParams fp;
  memset(&fp, 0, sizeof(fp));
  fp.g = make_params(a, 0);
  fp.gu_start = a.gu_start;
  fp.dn_start = a.dn_start;
  fp.ready = a.ready;
  fp.counter = const_cast<int32_t*>(a.nitems) + 2;
  fp.max_gu = a.max_items_gu;
  fp.max_dn = a.max_items_dn;
  const int T = a.T, TK = a.T * c.K;
  CUtensorMap tWg, tWu, tWgS, tWuS, tWd, tWdS, tH, tHs;
  bool ok = map_bf16(&tWg, a.Wg, static_cast<uint64_t>(a.wrows) * c.I, c.H, kTileN) &&
            map_bf16(&tWu, a.Wu, static_cast<uint64_t>(a.wrows) * c.I, c.H, kTileN) &&
            map_bf16(&tWd, a.Wd, static_cast<uint64_t>(a.wrows) * c.H, c.I, kTileN) &&
            map_bf16(&tH, a.h_r, TK, c.I, BN);
  if (fp.g.has_shared) {
    ok = ok && map_bf16(&tWgS, a.W->Wg_s, c.I_shared, c.H, kTileN) &&
         map_bf16(&tWuS, a.W->Wu_s, c.I_shared, c.H, kTileN) &&
         map_bf16(&tWdS, a.W->Wd_s, c.H, c.I_shared, kTileN) &&
         map_bf16(&tHs, a.h_s, T, c.I_shared, BN);
  } else {
    tWgS = tWg;
    tWuS = tWu;
    tWdS = tWd;
    tHs = tH;
  }
  if (!ok) return cudaErrorInvalidValue;
  auto kern = moe_ffn_fused<BN>;
  const int smem_max = C::SMEM + (3 * 1024 + 5) * static_cast<int>(sizeof(int));
  const int smem = C::SMEM + (3 * c.E + 5) * static_cast<int>(sizeof(int));
  cudaError_t e = ensure_dyn_smem(reinterpret_cast<const void*>(kern), smem_max);
  if (e != cudaSuccess) return e;
  // one CTA per SM, all resident at once (down items wait on other CTAs)
  cudaLaunchConfig_t lc;
  memset(&lc, 0, sizeof(lc));
  lc.gridDim = dim3(num_sms());
  lc.blockDim = dim3(kFusedThreads);
  lc.dynamicSmemBytes = smem;
  lc.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  return cudaLaunchKernelEx(&lc, kern, fp, tWg, tWu, tWgS, tWuS, tWd, tWdS, tH, tHs);
}

template <int MODE>
cudaError_t launch_bn(const GemmArgs& a, cudaStream_t s) {
  switch (a.bn) {
    case 16: return launch_mode<MODE, 16>(a, s);
    case 32: return launch_mode<MODE, 32>(a, s);
    case 64: return launch_mode<MODE, 64>(a, s);
    case 128: return launch_mode<MODE, 128>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_gemm_gateup(const GemmArgs& a, cudaStream_t s) { return launch_bn<0>(a, s); }
cudaError_t launch_ffn_fused(const GemmArgs& a, cudaStream_t s) {
  switch (a.bn) {
    case 16: return launch_fused_bn<16>(a, s);
    case 32: return launch_fused_bn<32>(a, s);
    case 64: return launch_fused_bn<64>(a, s);
    case 128: return launch_fused_bn<128>(a, s);
    default: return cudaErrorInvalidValue;
  }
}
cudaError_t launch_gemm_down(const GemmArgs& a, cudaStream_t s) { return launch_bn<1>(a, s); }

}  // namespace sgl
