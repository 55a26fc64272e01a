// ffn_mx.cu - stages 7 and 8 on block-scaled tensor cores (weight format
// MOE_W_MXFP4_A8): the routed experts as MXFP8 activations x MXFP4 weights,
// the shared expert in bf16, in one persistent kernel.
//
// Pages: "Ling-3.0-flash-VL MoE sparse routing" (lqnn.cn/news/282163) sec. 2
// and sec. 4 (SwiGLU experts, hidden 2560, intermediate 768, shared expert,
// SwiGLU limits); "Ling-3.0-flash-VL 42-layer hybrid backbone"
// (lpnh.cn/news/2815793) spec table (quantisation FP8 + MXFP4, routed experts
// in 4 bits). Formats per the OCP Microscaling spec v1.0 (see mxfp8.cu).
//
// Same items as the bf16 kernel (ffn.cu), with a token tile of 112 rows:
//   gate/up (slot e, row tile m, feature tile n of 128): A0 = Wg rows, A1 = Wu
//       rows, B = the routed rows of x (MXFP8 codes and scales, gathered);
//       two accumulators, so the gate and up MMAs of a k step are independent
//       (a chain of MMAs into one accumulator runs at its latency, ~1.4x
//       slower). Routed h = silu(g) * u is quantised to MXFP8 in the epilogue
//       (one warp = 32 consecutive features = one scale block); shared h ->
//       bf16.
//   down (slot e, row tile m, output tile n of 256): A0 / A1 = Wd rows
//       [256n, 256n+128) / [256n+128, 256n+256), B = h rows; y_slot[j] = w_j * D.
// Routed items run tcgen05.mma kind::mxf8f6f4.block_scale (e2m1 weights read
// in place by TMA, unpacked to one byte per element; e4m3 activations; K = 128
// per stage); their scale atoms go shared memory -> tensor memory with
// tcgen05.cp once per stage. Shared-expert items run kind::f16 (K = 64 per
// stage) on the same pipeline. TMEM: two buffers of gate | up accumulators
// (2 x 2 x 112 columns), then the three scale atoms.
//
// Claiming, readiness counters, warp roles and bounded waits are those of
// ffn.cu (480 threads: TMA producer, MMA issuer, 8 epilogue warps, 4 gatherer
// warps, scheduler).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "ffn_common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace sgl {
namespace {

constexpr int kXEpiWarps = 8;
constexpr int kXEpiThreads = 32 * kXEpiWarps;
constexpr int kXGatherWarp0 = 2 + kXEpiWarps;  // warps 10..13
constexpr int kXGatherWarps = 4;
constexpr int kXSchedWarp = kXGatherWarp0 + kXGatherWarps;  // warp 14
constexpr int kXThreads = 32 * (kXSchedWarp + 1);
constexpr int kXQueue = 4;
constexpr int kXLead = 4;
constexpr long long kXProgStride = 1024;
constexpr int kXA = 128 * 128;              // one A tile: 128 rows x 128 bytes
constexpr int kXB = kMxTileN * 128;         // B tile: up to 112 rows x 128 bytes
constexpr int kXSfOff = 2 * kXA + kXB;      // scale atoms: A0, A1, B (512 bytes each)
constexpr int kXStage = (kXSfOff + 3 * 512 + 1023) / 1024 * 1024;
constexpr int kXStages = 4;
constexpr int kXAccCols = 2 * kMxTileN;     // gate | up of one buffer
constexpr int kXSfCol = 2 * kXAccCols;      // scale atoms after the two buffers
constexpr int kXTmemCols = 512;
constexpr int kXCtrl = 512;
constexpr int kXHBox = 16;                  // h rows per TMA box
constexpr int kXSmem =
    kXStages * kXStage + 1024 + kXCtrl + kMxTileN * 8 + kXEpiWarps * kEpiTileWords * 4;
static_assert(kXSmem + (3 * kMaxExpertsCfg + 5) * 4 <= 227 * 1024, "shared memory");
static_assert(kXSfCol + 12 <= kXTmemCols, "TMEM");
static_assert(kMxTileN % 16 == 0 && kMxTileN <= 128, "token tile");

struct MxParams {
  FfnParams f;
  const uint8_t* x_q;    // [T, H] e4m3
  const uint8_t* x_sf;   // [T, H/32] e8m0
  uint8_t* h_q;          // [T*K, I] e4m3, permuted rows
  uint8_t* h_sf;         // [routed row tiles][I/128][512] atoms
  const uint8_t* sf_g;   // [slot][I/128][H/128][512]
  const uint8_t* sf_u;   // [slot][I/128][H/128][512]
  const uint8_t* sf_d;   // [slot][H/128][I/128][512]
  const int32_t* slot_of;  // nullptr: prepared atoms, indexed by expert id
};

struct MxMaps {
  CUtensorMap wg, wu, wd;     // MXFP4 codes, 128-row boxes
  CUtensorMap hq;             // h codes [T*K, I] bytes, 16-row boxes
  CUtensorMap wgs, wus, wds;  // shared expert bf16, 128-row boxes
  CUtensorMap hs;             // shared h [T, Is] bf16, 16-row boxes
};

__device__ __forceinline__ int atom_off(int r, int k) { return (r & 31) * 16 + (r >> 5) * 4 + k; }

// e4m3 code of v (already divided by the block scale), nearest even, saturating.
__device__ __forceinline__ uint8_t to_e4m3(float v) {
  return static_cast<uint8_t>(__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3));
}

__global__ void __launch_bounds__(kXThreads, 1)
    moe_ffn_mx(const __grid_constant__ MxParams q, const __grid_constant__ MxMaps m) {
  const FfnParams& p = q.f;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* ctrl = smem + kXStages * kXStage;
  uint64_t* full = reinterpret_cast<uint64_t*>(ctrl);
  uint64_t* empty = full + kXStages;
  uint64_t* tfull = empty + kXStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* qfull = tempty + 2;
  uint64_t* qempty = qfull + kXQueue;
  volatile long long* prog = reinterpret_cast<volatile long long*>(qempty + kXQueue);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(const_cast<long long*>(prog) + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* qitem = abort_flag + 1;  // [kXQueue]
  int* meta_j = reinterpret_cast<int*>(ctrl + kXCtrl);
  float* meta_w = reinterpret_cast<float*>(meta_j + kMxTileN);
  uint32_t* epi_tile = reinterpret_cast<uint32_t*>(meta_w + kMxTileN);    // [warps][kEpiTileWords]
  int* s_gu = reinterpret_cast<int*>(epi_tile + kXEpiWarps * kEpiTileWords);  // [E+2]
  int* s_dn = s_gu + (p.E + 2);                           // [E+2]
  int* s_off = s_dn + (p.E + 2);                          // [E+1]
  static_assert(8 * (2 * kXStages + 4 + 2 * kXQueue) + 8 + 4 * (2 + kXQueue) <= kXCtrl, "ctrl");

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_trigger();
  if (tid == 0) {
    for (int s = 0; s < kXStages; ++s) {
      mbar_init(&full[s], 1 + 32 * kXGatherWarps);  // producer's expect_tx + one per gatherer thread
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], kXEpiWarps);
    }
    for (int i = 0; i < kXQueue; ++i) {
      mbar_init(&qfull[i], 1);
      mbar_init(&qempty[i], 1 + 1 + kXEpiWarps + kXGatherWarps);
    }
    *prog = 0;
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&m.wg);
    prefetch_tmap(&m.wu);
    prefetch_tmap(&m.wd);
    prefetch_tmap(&m.hq);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kXTmemCols);
    tmem_relinquish();
  }
  pdl_wait();  // the schedule, the routing, x and its MXFP8 copy come from earlier kernels
  for (int i = tid; i < p.E + 2; i += blockDim.x) {
    s_gu[i] = p.gu_start[i];
    s_dn[i] = p.dn_start[i];
  }
  for (int i = tid; i < p.E + 1; i += blockDim.x) s_off[i] = p.offsets[i];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int nslots = p.E + (p.has_shared ? 1 : 0);
  const int n_gu = min(p.nitems[0], p.max_gu);
  const int n_dn = min(p.nitems[1], p.max_dn);
  const int n_all = n_gu + n_dn;
  const int kbh = p.H / 128, kbi = p.I / 128, ftg = cdiv_dev(p.I, kMxGuTile);
  auto item_at = [&](int i, bool& gu) {
    gu = i < n_gu;
    return gu ? decode_item(i, s_gu, s_off, nslots, p.E, p.T, kMxTileN)
              : decode_item(i - n_gu, s_dn, s_off, nslots, p.E, p.T, kMxTileN);
  };
  auto ok_item = [&](const WorkItem& it, bool gu) {
    return item_ok(p, it, gu, kMxTileN, kMxGuTile, kMxDnTile);
  };
  // k-blocks: 128 wide for the 8-bit routed operands, 64 for bf16
  auto nkb_of = [&](bool gu, bool sh) {
    return gu ? (sh ? p.H / 64 : kbh) : (sh ? p.Is / 64 : kbi);
  };
  // a down item's second 128-row half exists unless it starts past H
  auto two_halves = [&](const WorkItem& it, bool gu) {
    return gu || it.ntile * kMxDnTile + 128 < p.H;
  };
  auto mma_n = [&](const WorkItem& it) { return (min(it.nrows, kMxTileN) + 15) & ~15; };
  // dense index of a routed (slot, row tile): every routed slot has ftg gate/up tiles per row tile
  auto row_tile = [&](const WorkItem& it) { return s_gu[it.e] / ftg + (it.row0 - s_off[it.e]) / kMxTileN; };
  auto next_item = [&](int n, int& item, bool whole_warp) -> bool {
    const int qi = n % kXQueue;
    if (!mbar_wait(&qfull[qi], (n / kXQueue) & 1, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) return false;
    item = qitem[qi];
    if (whole_warp) __syncwarp();
    if (lane == 0) mbar_arrive(&qempty[qi]);
    return item >= 0;
  };

  if (warp == kXSchedWarp) {
    // ------------------------------------------------------------ scheduler
    if (lane == 0) {
      int prev_nkb = 0;
      for (int n = 0;; ++n) {
        const int qi = n % kXQueue;
        if (!mbar_wait(&qempty[qi], ((n / kXQueue) & 1) ^ 1, abort_flag, p.err, MOE_DEVERR_TIMEOUT))
          break;
        if (n > 0 && !wait_progress(prog, (n - 1) * kXProgStride + max(0, prev_nkb - kXLead),
                                    abort_flag, p.err))
          break;
        int item = atomicAdd(p.counter, 1);
        if (item >= n_all) item = -1;
        prev_nkb = 0;
        if (item >= 0) {
          bool gu;
          const WorkItem it = item_at(item, gu);
          if (ok_item(it, gu)) {
            const bool sh = it.e == p.E;
            prev_nkb = nkb_of(gu, sh);
            if (!gu) {
              // every gate/up feature tile of this (slot, row tile) must be in h
              const int r0 = sh ? 0 : s_off[it.e];
              const int ridx = s_gu[it.e] + (it.row0 - r0) / kMxTileN;
              if (!wait_count(p.ready + ridx, cdiv_dev(sh ? p.Is : p.I, kMxGuTile), abort_flag,
                              p.err))
                item = -1;
            }
          } else {
            atomicExch(p.err, MOE_DEVERR_SCHEDULE);
          }
        }
        qitem[qi] = item;
        mbar_arrive(&qfull[qi]);
        if (item < 0) break;
      }
    }
    __syncwarp();
  } else if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // Weight tiles and their scale atoms; for down items also the h rows and
    // their scale atom. MXFP4 boxes count their packed bytes.
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_h = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      bool live = true;
      for (int n = 0; live; ++n) {
        int item;
        if (!next_item(n, item, false)) break;
        *prog = n * kXProgStride;
        bool gu;
        const WorkItem it = item_at(item, gu);
        if (!ok_item(it, gu)) continue;
        const bool sh = it.e == p.E;
        if (!gu) fence_proxy_async_global();  // h was published by other CTAs
        const int nkb = nkb_of(gu, sh);
        const bool two = two_halves(it, gu);
        const int na = two ? 2 : 1;
        const int nhbox = gu ? 0 : mma_n(it) / kXHBox;
        const int slot = sh ? 0 : (q.slot_of ? q.slot_of[it.e] : it.e);  // prepared atoms: by expert
        uint32_t bytes;
        if (sh) bytes = na * kXA + nhbox * kXHBox * 128;
        else bytes = na * (128 * 64 + 512) + (gu ? 0 : nhbox * kXHBox * 128 + 512);
        // first weight row of A0 (A1 follows 128 rows later for down items)
        const int arow = gu ? it.ntile * kMxGuTile : it.ntile * kMxDnTile;
        const uint8_t* sfa0 = nullptr;
        const uint8_t* sfa1 = nullptr;
        const uint8_t* sfb = nullptr;
        if (!sh) {
          if (gu) {
            sfa0 = q.sf_g + (static_cast<size_t>(slot) * (p.I / 128) + arow / 128) * kbh * 512;
            sfa1 = q.sf_u + (static_cast<size_t>(slot) * (p.I / 128) + arow / 128) * kbh * 512;
          } else {
            sfa0 = q.sf_d + (static_cast<size_t>(slot) * (p.H / 128) + arow / 128) * kbi * 512;
            sfa1 = sfa0 + static_cast<size_t>(kbi) * 512;  // the next 128-row tile
            sfb = q.h_sf + static_cast<size_t>(row_tile(it)) * kbi * 512;
          }
        }
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) {
            live = false;
            break;
          }
          uint8_t* sA = smem + stage * kXStage;
          uint8_t* sB = sA + 2 * kXA;
          uint8_t* sSF = sA + kXSfOff;
          mbar_arrive_expect_tx(&full[stage], bytes);
          if (sh) {
            const CUtensorMap* a0 = gu ? &m.wgs : &m.wds;
            const CUtensorMap* a1 = gu ? &m.wus : &m.wds;
            tma_load_2d(sA, a0, &full[stage], kb * 64, arow, pol_w);
            if (two) tma_load_2d(sA + kXA, a1, &full[stage], kb * 64, gu ? arow : arow + 128, pol_w);
            for (int hb = 0; hb < nhbox; ++hb)
              tma_load_2d(sB + hb * kXHBox * 128, &m.hs, &full[stage], kb * 64, it.row0 + hb * kXHBox,
                          pol_h);
          } else {
            if (gu) {
              tma_load_2d(sA, &m.wg, &full[stage], kb * 128, it.e * p.I + arow, pol_w);
              tma_load_2d(sA + kXA, &m.wu, &full[stage], kb * 128, it.e * p.I + arow, pol_w);
            } else {
              tma_load_2d(sA, &m.wd, &full[stage], kb * 128, it.e * p.H + arow, pol_w);
              if (two) tma_load_2d(sA + kXA, &m.wd, &full[stage], kb * 128, it.e * p.H + arow + 128, pol_w);
              for (int hb = 0; hb < nhbox; ++hb)
                tma_load_2d(sB + hb * kXHBox * 128, &m.hq, &full[stage], kb * 128,
                            it.row0 + hb * kXHBox, pol_h);
              bulk_load(sSF + 1024, sfb + kb * 512, 512, &full[stage]);
            }
            bulk_load(sSF, sfa0 + kb * 512, 512, &full[stage]);
            if (two) bulk_load(sSF + 512, sfa1 + kb * 512, 512, &full[stage]);
          }
          *prog = n * kXProgStride + kb + 1;
          if (++stage == kXStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // every stage must be released by its MMA commit before teardown
      for (int i = 0; i < kXStages && live; ++i) {
        if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) break;
        if (++stage == kXStages) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool live = true;
      const uint32_t sf_t = tmem_base + kXSfCol;  // A0, A1, B scale atoms: 4 columns each
      for (int n = 0; live; ++n) {
        int item;
        if (!next_item(n, item, false)) break;
        bool gu;
        const WorkItem it = item_at(item, gu);
        if (!ok_item(it, gu)) continue;
        const bool sh = it.e == p.E;
        const int nkb = nkb_of(gu, sh);
        const bool two = two_halves(it, gu);
        const int N = mma_n(it);
        const uint32_t idesc_f16 = idesc_bf16(128, N);
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + acc * kXAccCols, d1 = d0 + kMxTileN;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) {
            live = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + stage * kXStage), a1 = a0 + kXA, b0 = a0 + 2 * kXA;
          if (sh) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t bd = sdesc_k128(b0 + kk * 32);
              const uint32_t accum = (kb | kk) != 0 ? 1u : 0u;
              umma_bf16(d0, sdesc_k128(a0 + kk * 32), bd, idesc_f16, accum);
              if (two) umma_bf16(d1, sdesc_k128(a1 + kk * 32), bd, idesc_f16, accum);
            }
          } else {
            // this stage's scales into tensor memory: ordered before the MMAs
            // below and after those of the previous stage that read the columns
            const uint32_t sf_s = a0 + kXSfOff;
            tmem_cp_atom(sf_t, sf_s);
            if (two) tmem_cp_atom(sf_t + 4, sf_s + 512);
            tmem_cp_atom(sf_t + 8, sf_s + 1024);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint32_t sel = static_cast<uint32_t>(kk) << 30;
              const uint64_t bd = sdesc_k128(b0 + kk * 32);
              const uint32_t idesc = idesc_mx_e2m1_e4m3(128, N, kk);
              const uint32_t accum = (kb | kk) != 0 ? 1u : 0u;
              umma_mx(d0, sdesc_k128(a0 + kk * 32), bd, idesc, accum, sf_t | sel, (sf_t + 8) | sel);
              if (two)
                umma_mx(d1, sdesc_k128(a1 + kk * 32), bd, idesc, accum, (sf_t + 4) | sel,
                        (sf_t + 8) | sel);
            }
          }
          umma_commit(&empty[stage]);
          if (++stage == kXStages) {
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
  } else if (warp >= kXGatherWarp0) {
    // ------------------------------------------------------------ token gatherers
    // Gate/up items: thread g copies 16-byte chunk (g % 8) of rows g/8,
    // g/8 + 16, ... of the stage's token tile (128 bytes per row: 128 e4m3
    // codes, or 64 bf16 for the shared expert) into the 128-byte-swizzled
    // layout, and for routed items the four scale bytes of row g into the B
    // scale atom. Each thread then hands the stage's full barrier an arrival
    // that fires when its copies have landed (as in ffn.cu); down items keep
    // the stage sequence and the arrivals.
    constexpr int kRowsPerThread = kMxTileN / 16;
    const int g = tid - kXGatherWarp0 * 32;
    const int chunk = g & 7, rbase = g >> 3;
    const uint64_t pol_x = policy_evict_last();
    int stage = 0;
    uint32_t phase = 0;
    bool live = true;
    for (int n = 0; live; ++n) {
      int item;
      if (!next_item(n, item, true)) break;
      bool gu;
      const WorkItem it = item_at(item, gu);
      if (!ok_item(it, gu)) continue;
      const bool sh = it.e == p.E;
      const int nkb = nkb_of(gu, sh);
      const int nb = mma_n(it);
      const uint8_t* src[kRowsPerThread];
      const uint8_t* sf_src = nullptr;
#pragma unroll
      for (int i = 0; i < kRowsPerThread; ++i) {
        const int row = it.row0 + min(rbase + 16 * i, it.nrows - 1);
        int t = 0;
        if (gu) t = sh ? row : p.perm[row] / p.K;
        t = min(max(t, 0), p.T - 1);
        src[i] = sh ? reinterpret_cast<const uint8_t*>(p.x + static_cast<size_t>(t) * p.H) + chunk * 16
                    : q.x_q + static_cast<size_t>(t) * p.H + chunk * 16;
      }
      if (gu && !sh && g < nb) {
        const int row = it.row0 + min(g, it.nrows - 1);
        const int t = min(max(p.perm[row] / p.K, 0), p.T - 1);
        sf_src = q.x_sf + static_cast<size_t>(t) * (p.H / 32);
      }
      for (int kb = 0; kb < nkb; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) {
          live = false;
          break;
        }
        if (gu) {
          uint8_t* sB = smem + stage * kXStage + 2 * kXA;
          // 128 bytes of a row per k-block: 64 bf16 or 128 e4m3
#pragma unroll
          for (int i = 0; i < kRowsPerThread; ++i) {
            const int r = rbase + 16 * i;
            if (r < nb) cp_async16(sB + r * 128 + ((chunk ^ (r & 7)) << 4), src[i] + kb * 128, pol_x);
          }
          if (sf_src) cp_async4(smem + stage * kXStage + kXSfOff + 1024 + atom_off(g, 0), sf_src + kb * 4);
        }
        cp_async_mbar_arrive_noinc(&full[stage]);
        if (++stage == kXStages) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    cp_async_wait_all();  // nothing may still be landing in shared memory at exit
  } else {
    // ------------------------------------------------------------ epilogue
    const int qd = warp & 3;            // TMEM lane quarter
    const int et = tid - 2 * 32;        // epilogue thread 0..255
    const int cpart = et >> 7;          // the two warps of a quarter: alternate column chunks
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int n = 0;; ++n) {
      int item;
      if (!next_item(n, item, true)) break;
      bool gu;
      const WorkItem it = item_at(item, gu);
      if (!ok_item(it, gu)) continue;
      const bool sh = it.e == p.E;
      if (!gu) {
        epi_bar<kXEpiThreads>();  // the previous item's rows are no longer read
        for (int rr = et; rr < kMxTileN; rr += kXEpiThreads) {
          int j = -1;
          float wt = 0.f;
          if (rr < it.nrows) {
            const int row = it.row0 + rr;
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
          meta_j[rr] = j;
          meta_w[rr] = wt;
        }
        epi_bar<kXEpiThreads>();
      }
      if (!mbar_wait(&tfull[acc], acc_phase, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(qd * 32) << 16) + acc * kXAccCols;
      const int ncol = mma_n(it);
      uint32_t* tile = epi_tile + (warp - 2) * kEpiTileWords;
      if (gu) {
        const int fbase = it.ntile * kMxGuTile + qd * 32;  // this warp's 32 features
        const int ncols = sh ? p.Is : p.I;
        const bool ok = fbase < ncols;  // I and Is are multiples of 64: whole warps
        const float L = sh ? p.lim_s : p.lim_r;
        // routed: this warp's 32 features are one MXFP8 block, chunk qd of the
        // h scale atom of (row tile, k-block ntile)
        uint8_t* hsf = sh ? nullptr : q.h_sf + (static_cast<size_t>(row_tile(it)) * kbi + it.ntile) * 512;
        uint8_t* tb = reinterpret_cast<uint8_t*>(tile);
#pragma unroll 1
        for (int c0 = 16 * cpart; c0 < ncol; c0 += 32) {
          float gv[16], uv[16];
          tmem_ld16(taddr + c0, gv);
          tmem_ld16(taddr + kMxTileN + c0, uv);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 16; ++c) gv[c] = ok ? swiglu(gv[c], uv[c], L) : 0.f;
          if (sh) {
            if (ok) store_h16(gv, tile, p.h_s, p.Is, it.row0 + c0, it.nrows - c0, fbase, lane);
            continue;
          }
          // e4m3 codes of the 16 token rows, byte (row c, feature lane) of the tile
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const float h = gv[c];
            const uint32_t amax = __reduce_max_sync(0xffffffffu, __float_as_uint(h) & 0x7FFFFFFFu);
            const int byte = min(max(static_cast<int>(amax >> 23) - 8, 0), 254);
            const int ie = 254 - byte;  // 1 / scale = 2^(127 - byte)
            const float inv = ie > 0 ? __uint_as_float(static_cast<uint32_t>(ie) << 23)
                                     : __uint_as_float(0x00400000u);
            tb[c * 32 + lane] = to_e4m3(h * inv);
            if (lane == 0 && c0 + c < it.nrows) hsf[atom_off(c0 + c, qd)] = static_cast<uint8_t>(byte);
          }
          __syncwarp();
          {  // lane: 16 codes of token row lane / 2
            const int r = lane >> 1;
            if (ok && c0 + r < it.nrows)
              *reinterpret_cast<uint4*>(q.h_q + static_cast<size_t>(it.row0 + c0 + r) * p.I + fbase +
                                        16 * (lane & 1)) =
                  *reinterpret_cast<const uint4*>(tb + r * 32 + 16 * (lane & 1));
          }
          __syncwarp();
        }
      } else {
        const bool two = two_halves(it, gu);
#pragma unroll 1
        for (int half = 0; half < (two ? 2 : 1); ++half) {
          const int fbase = it.ntile * kMxDnTile + half * 128 + qd * 32;  // this warp's features
          const bool ok = fbase < p.H;  // H is a multiple of 64: whole warps
#pragma unroll 1
          for (int c0 = 16 * cpart; c0 < ncol && ok; c0 += 32) {
            float ov[16];
            tmem_ld16(taddr + half * kMxTileN + c0, ov);
            tmem_ld_wait();
#pragma unroll
            for (int g8 = 0; g8 < 2; ++g8) {
              float v[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) v[i] = meta_w[c0 + 8 * g8 + i] * ov[8 * g8 + i];
              store_y8(v, meta_j + c0 + 8 * g8, tile, p.y_slot, p.H, fbase, lane);
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
        // publish this feature tile of h: stores -> async proxy -> CTA -> GPU
        fence_proxy_async_global();
        epi_bar<kXEpiThreads>();
        if (warp == 2 && lane == 0) {
          __threadfence();
          const int r0 = sh ? 0 : s_off[it.e];
          atomicAdd(p.ready + s_gu[it.e] + (it.row0 - r0) / kMxTileN, 1);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kXTmemCols);
  }
}

}  // namespace

cudaError_t launch_ffn_mx(const GemmArgs& a, cudaStream_t s) {
  const moe_cfg& c = *a.cfg;
  if (a.bn != kMxTileN || a.x_q == nullptr) return cudaErrorInvalidValue;
  MxParams q;
  memset(&q, 0, sizeof(q));
  FfnParams& p = q.f;
  p.T = a.T;
  p.K = c.K;
  p.E = c.E;
  p.H = c.H;
  p.I = c.I;
  p.Is = c.I_shared;
  p.has_shared = (c.I_shared > 0 && a.W->Wg_s != nullptr) ? 1 : 0;
  p.lim_r = (c.limit_routed > 0.f && isfinite(c.limit_routed)) ? c.limit_routed : 0.f;
  p.lim_s = (c.limit_shared > 0.f && isfinite(c.limit_shared)) ? c.limit_shared : 0.f;
  p.x = a.x;
  p.perm = a.perm;
  p.w = a.w;
  p.h_r = a.h_r;
  p.h_s = a.h_s;
  p.y_slot = a.y_slot;
  p.offsets = a.offsets;
  p.wslot = nullptr;
  p.gu_start = a.gu_start;
  p.dn_start = a.dn_start;
  p.nitems = a.nitems;
  p.counter = const_cast<int32_t*>(a.nitems) + 2;
  p.ready = a.ready;
  p.max_gu = a.max_items_gu;
  p.max_dn = a.max_items_dn;
  p.err = a.err;
  q.x_q = a.x_q;
  q.x_sf = a.x_sf;
  q.h_q = a.h_q;
  q.h_sf = a.h_sf;
  q.sf_g = a.sf_g;
  q.sf_u = a.sf_u;
  q.sf_d = a.sf_d;
  q.slot_of = a.slot_of;
  const int T = a.T, TK = a.T * c.K;
  const uint64_t E = static_cast<uint64_t>(c.E);
  MxMaps m;
  bool ok = map_fp4(&m.wg, a.Wg, E * c.I, c.H, 128) && map_fp4(&m.wu, a.Wu, E * c.I, c.H, 128) &&
            map_fp4(&m.wd, a.Wd, E * c.H, c.I, 128) && map_u8(&m.hq, a.h_q, TK, c.I, kXHBox);
  if (p.has_shared) {
    ok = ok && map_bf16(&m.wgs, a.W->Wg_s, c.I_shared, c.H, 128) &&
         map_bf16(&m.wus, a.W->Wu_s, c.I_shared, c.H, 128) &&
         map_bf16(&m.wds, a.W->Wd_s, c.H, c.I_shared, 128) &&
         map_bf16(&m.hs, a.h_s, T, c.I_shared, kXHBox);
  } else {
    m.wgs = m.wus = m.wds = m.hs = m.hq;  // never read
  }
  if (!ok) return cudaErrorInvalidValue;
  const int smem_max = kXSmem + (3 * kMaxExpertsCfg + 5) * static_cast<int>(sizeof(int));
  const int smem = kXSmem + (3 * c.E + 5) * static_cast<int>(sizeof(int));
  cudaError_t e = ensure_dyn_smem(reinterpret_cast<const void*>(moe_ffn_mx), smem_max);
  if (e != cudaSuccess) return e;
  return launch_pdl(moe_ffn_mx, dim3(num_sms()), dim3(kXThreads), smem, s, q, m);
}

}  // namespace sgl
