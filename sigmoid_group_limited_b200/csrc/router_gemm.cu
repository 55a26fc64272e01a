// router_gemm.cu - stage 1 for batches above 32 tokens: the router logits
// z = x . Wr^T on the tensor cores.
//
// Page "Ling-3.0-flash-VL MoE sparse routing" (lqnn.cn/news/282163), sec. 4:
// the router runs in fp32. The fp32 router matrix is split (split_router in
// router.cu) into three bf16 terms hi + mid + lo, which represent every
// normal fp32 value exactly, and bf16 x times each term is exact in the MMA's
// products. What is left is fp32 accumulation, and the tensor cores' fp32
// sums are not rounded to nearest at every step, so long sums drift. The hi
// term, which carries almost all of the value, therefore goes into a fresh
// accumulator for every 64-wide k-block; the epilogue adds those chunks in
// fp32 registers, in k order. mid and lo accumulate over the whole K in their
// own accumulators: their contribution is below 2^-8 of the total, so their
// drift is too. The router's top-k certifies every decision against the
// remaining error and re-derives close calls exactly (router.cu).
//
// One tile = 128 experts (MMA M, the three terms as three A operands) x 128
// tokens (MMA N). Warp roles: 0 TMA producer, 1 MMA issuer and TMEM owner,
// 2..5 epilogue. All waits are bounded (ptx.cuh).
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>

#include "internal.h"
#include "ptx.cuh"

namespace sgl {
namespace {

constexpr int kRBN = 128;                  // tokens per tile (MMA N)
constexpr int kRA = kTileN * 128;          // one A tile: 128 rows x 64 bf16
constexpr int kRB = kRBN * 128;            // token tile: 128 rows x 64 bf16
constexpr int kRStage = 3 * kRA + kRB;     // hi + mid + lo + tokens
constexpr int kRStages = 3;
// TMEM: two hi-chunk buffers, then the mid and lo accumulators (BN columns each)
constexpr int kRTmemCols = 4 * kRBN;
constexpr int kRSmem = kRStages * kRStage + 1024 + 256;
constexpr int kRThreads = 192;

struct RouterGemmParams {
  int T, E, H;
  float* z;  // [T, E]
  int32_t* err;
};

__global__ void __launch_bounds__(kRThreads, 1)
    router_logits_tc(const __grid_constant__ RouterGemmParams p,
                     const __grid_constant__ CUtensorMap tHi, const __grid_constant__ CUtensorMap tMid,
                     const __grid_constant__ CUtensorMap tLo, const __grid_constant__ CUtensorMap tX) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kRStages * kRStage);
  uint64_t* empty = full + kRStages;
  uint64_t* tfull = empty + kRStages;  // mid + lo done for the tile
  uint64_t* tempty = tfull + 1;
  uint64_t* hfull = tempty + 1;        // [2] hi chunk ready
  uint64_t* hempty = hfull + 2;        // [2] hi chunk consumed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(hempty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_trigger();
  if (tid == 0) {
    for (int s = 0; s < kRStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tfull, 1);
    mbar_init(tempty, 4);
    for (int a = 0; a < 2; ++a) {
      mbar_init(&hfull[a], 1);
      mbar_init(&hempty[a], 4);
    }
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tHi);
    prefetch_tmap(&tX);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kRTmemCols);
    tmem_relinquish();
  }
  pdl_wait();  // the split router matrix comes from the kernel before
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int nm = (p.T + kRBN - 1) / kRBN;
  const int n_items = nm * ((p.E + kTileN - 1) / kTileN);
  const int KB = p.H / 64;

  if (warp == 0) {
    if (lane == 0) {
      // the router matrix and the tokens are both re-read by other tiles: keep them in L2
      const uint64_t pol = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      bool live = true;
      for (int item = blockIdx.x; item < n_items && live; item += gridDim.x) {
        const int n = item / nm, m = item - n * nm;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) {
            live = false;
            break;
          }
          uint8_t* s = smem + stage * kRStage;
          mbar_arrive_expect_tx(&full[stage], kRStage);
          tma_load_2d(s, &tHi, &full[stage], kb * 64, n * kTileN, pol);
          tma_load_2d(s + kRA, &tMid, &full[stage], kb * 64, n * kTileN, pol);
          tma_load_2d(s + 2 * kRA, &tLo, &full[stage], kb * 64, n * kTileN, pol);
          tma_load_2d(s + 3 * kRA, &tX, &full[stage], kb * 64, m * kRBN, pol);
          if (++stage == kRStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // every stage must be released by its MMA commit before teardown
      for (int i = 0; i < kRStages && live; ++i) {
        if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) break;
        if (++stage == kRStages) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(kTileN, kRBN);
      const uint32_t d_mid = tmem_base + 2 * kRBN, d_lo = tmem_base + 3 * kRBN;
      int stage = 0, ck = 0;
      uint32_t phase = 0, tph = 0;
      bool live = true;
      for (int item = blockIdx.x; item < n_items && live; item += gridDim.x) {
        if (!mbar_wait(tempty, tph ^ 1, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) break;
        tc_fence_after();
        for (int kb = 0; kb < KB; ++kb, ++ck) {
          const int hb = ck & 1;
          if (!mbar_wait(&hempty[hb], ((ck >> 1) & 1) ^ 1, abort_flag, p.err, MOE_DEVERR_TIMEOUT) ||
              !mbar_wait(&full[stage], phase, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) {
            live = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + stage * kRStage);
          const uint32_t b0 = a0 + 3 * kRA;
          const uint32_t d_hi = tmem_base + hb * kRBN;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bd = sdesc_k128(b0 + kk * 32);
            const uint32_t acc_all = (kb | kk) != 0 ? 1u : 0u;
            umma_bf16(d_hi, sdesc_k128(a0 + kk * 32), bd, idesc, kk != 0 ? 1u : 0u);
            umma_bf16(d_mid, sdesc_k128(a0 + kRA + kk * 32), bd, idesc, acc_all);
            umma_bf16(d_lo, sdesc_k128(a0 + 2 * kRA + kk * 32), bd, idesc, acc_all);
          }
          umma_commit(&empty[stage]);
          umma_commit(&hfull[hb]);
          if (++stage == kRStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!live) break;
        umma_commit(tfull);
        tph ^= 1;
      }
    }
    __syncwarp();
  } else {
    // epilogue: z = (sum over k-blocks of the hi chunks, in order) + mid + lo
    const int q = warp & 3;
    const int orow = q * 32 + lane;  // expert within the tile
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    int ck = 0;
    uint32_t tph = 0;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
      const int n = item / nm, m = item - n * nm;
      const int row0 = m * kRBN, nrows = min(kRBN, p.T - row0);
      float sum[kRBN];
#pragma unroll
      for (int c = 0; c < kRBN; ++c) sum[c] = 0.f;
      bool live = true;
      for (int kb = 0; kb < KB; ++kb, ++ck) {
        const int hb = ck & 1;
        if (!mbar_wait(&hfull[hb], (ck >> 1) & 1, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) {
          live = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c0 = 0; c0 < kRBN; c0 += 32) {
          float v0[16], v1[16];
          tmem_ld16(lane_base + hb * kRBN + c0, v0);
          tmem_ld16(lane_base + hb * kRBN + c0 + 16, v1);
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
      if (!live || !mbar_wait(tfull, tph, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) break;
      tc_fence_after();
#pragma unroll
      for (int c0 = 0; c0 < kRBN; c0 += 16) {
        float vm[16], vl[16];
        tmem_ld16(lane_base + 2 * kRBN + c0, vm);
        tmem_ld16(lane_base + 3 * kRBN + c0, vl);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 16; ++c) sum[c0 + c] += vm[c] + vl[c];
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty);
      tph ^= 1;
      const int e = n * kTileN + orow;
      if (e < p.E) {
#pragma unroll
        for (int c = 0; c < kRBN; ++c)
          if (c < nrows) p.z[static_cast<size_t>(row0 + c) * p.E + e] = sum[c];
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kRTmemCols);
  }
}

}  // namespace

cudaError_t launch_router_gemm(const moe_cfg& c, int T, const uint16_t* x, const uint16_t* w_hi,
                               const uint16_t* w_mid, const uint16_t* w_lo, float* z,
                               int32_t* err, cudaStream_t s) {
  RouterGemmParams p;
  memset(&p, 0, sizeof(p));
  p.T = T;
  p.E = c.E;
  p.H = c.H;
  p.z = z;
  p.err = err;
  CUtensorMap tHi, tMid, tLo, tX;
  const bool ok = map_bf16(&tHi, w_hi, c.E, c.H, kTileN) && map_bf16(&tMid, w_mid, c.E, c.H, kTileN) &&
                  map_bf16(&tLo, w_lo, c.E, c.H, kTileN) && map_bf16(&tX, x, T, c.H, kRBN);
  if (!ok) return cudaErrorInvalidValue;
  cudaError_t e = ensure_dyn_smem(reinterpret_cast<const void*>(router_logits_tc), kRSmem);
  if (e != cudaSuccess) return e;
  const int n_items = cdiv(c.E, kTileN) * cdiv(T, kRBN);
  const int grid = std::max(1, std::min(num_sms(), n_items));
  return launch_pdl(router_logits_tc, dim3(grid), dim3(kRThreads), kRSmem, s, p, tHi, tMid, tLo, tX);
}

}  // namespace sgl
