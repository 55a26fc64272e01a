// ffn_pair.cu - stages 7 and 8 for large batches: the grouped SwiGLU experts
// and the shared expert on CTA pairs (tcgen05 cta_group::2).
//
// Page "Ling-3.0-flash-VL MoE sparse routing" (lqnn.cn/news/282163): sec. 2
// (an expert is a gate / up / down SwiGLU FFN, hidden 2560, intermediate 768;
// one shared expert sees every token) and sec. 4 (SwiGLU limits).
//
// Same scheduling as ffn.cu, but each item runs on a pair of CTAs (a cluster
// of two) that issue M = 256 MMAs: each CTA holds 128 rows of A and half of
// the item's N token rows of B, and gets its 128 rows of D in its own TMEM.
// TMEM holds two 256-column accumulators (halves 0 and 1).
//   gate/up item (slot, 256-token tile, 256 features f0..f0+255): CTA r holds
//       gate rows f0 + 128r .. +127 and up rows f0 + 128r .. +127 as two A
//       operands; gate accumulates in half 0 and up in half 1, two
//       independent MMA chains issued alternately (an MMA waits for the
//       previous one into the same accumulator, so one chain alone issues
//       at about two thirds of the rate of two). B = the item's token rows,
//       copied from x by the gatherer warps of each CTA (16-byte cp.async
//       into the swizzled tile). Per CTA and 64-wide k-block: 32 KB of A and
//       up to 16 KB of B for 2 x 128 x 256 x 64 MACs of this SM.
//   down item (slot, 256-token tile, 256 hidden features): CTA r holds Wd rows
//       256 n + 128 r .. +127; B = h rows; one accumulator, the halves taken
//       in turn, so a down item's epilogue overlaps the next down item.
// A gate/up item holds both halves, so its epilogue does not overlap the
// next item's MMAs; eight epilogue warps keep that drain short.
// A and the h rows of down items arrive by TMA (no multicast): each CTA loads
// its own halves and the byte counts complete on the leader CTA's full
// barrier, where the gatherer warps of both CTAs also arrive; the leader's
// MMA thread releases a stage in both CTAs with one multicast commit.
//
// Warp roles per CTA (480 threads):
//   0      TMA producer (lane 0), both CTAs
//   1      TMEM allocation in both CTAs; MMA issuer (lane 0) in the leader
//   2..9   epilogue, both CTAs: two warps per TMEM lane quarter (warp % 4),
//          alternate column chunks
//   10..13 token gatherers, both CTAs
//   14     scheduler (lane 0), leader: claims items, waits for their inputs
//          and writes them into the item queues of both CTAs
// Barriers filled by TMA bytes or by tcgen05.commit only are waited on at
// CTA scope; the ones other threads of the pair arrive on (full stages, item
// queues, the leader's accumulator-empty barriers) at cluster scope.
// Every wait is bounded; the two CTAs meet at a cluster barrier after setup
// and before exit, so no CTA touches the other's shared memory after it left.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "ffn_common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace sgl {
namespace {

constexpr int kPEpiWarps = 8;              // warps 2..9, two per TMEM lane quarter
constexpr int kPEpiThreads = 32 * kPEpiWarps;
constexpr int kPGatherWarp0 = 2 + kPEpiWarps;   // warps 10..13
constexpr int kPGatherWarps = 4;
constexpr int kPSchedWarp = kPGatherWarp0 + kPGatherWarps;  // warp 14
constexpr int kPThreads = 32 * (kPSchedWarp + 1);
constexpr int kPQueue = 4;
constexpr int kPLead = 4;                  // claim the next item this many k-blocks early
constexpr long long kPProgStride = 1024;
constexpr int kPStages = 4;
constexpr int kPA = 128 * 128;             // one A operand: this CTA's 128 rows x 64 bf16
constexpr int kPB = kPairTileN / 2 * 128;  // B half: up to 128 rows x 64 bf16
constexpr int kPStage = 2 * kPA + kPB;     // gate A, up A (down: Wd rows only), B
constexpr int kPBox = 32;                  // token rows per B box
constexpr int kPAccCols = kPairTileN;      // fp32 columns of one accumulator (a TMEM half)
constexpr int kPTmemCols = 2 * kPAccCols;  // halves 0 and 1
constexpr int kPCtrl = 512;
constexpr int kPSmem =
    kPStages * kPStage + 1024 + kPCtrl + kPairTileN * 8 + kPEpiWarps * kEpiTileWords * 4;
static_assert(kPTmemCols <= 512, "TMEM");
static_assert(kPSmem + (3 * kMaxExpertsCfg + 5) * 4 <= 227 * 1024, "shared memory");
// consumers of a queue entry, counted on the leader's qempty: leader producer,
// MMA, epilogue and gatherer warps; peer producer, epilogue and gatherer warps
constexpr int kPQueueConsumers = 1 + 1 + kPEpiWarps + kPGatherWarps + 1 + kPEpiWarps + kPGatherWarps;

// MMA N of an item: its rows rounded up to 64 (each CTA then holds a whole
// number of 32-row boxes of B)
__device__ __forceinline__ int pair_n(const WorkItem& it) {
  return (min(it.nrows, kPairTileN) + 63) & ~63;
}

struct PairMaps {
  CUtensorMap wg, wu, wgs, wus;  // gate / up rows, 128-row boxes
  CUtensorMap wd, wds;           // down rows, 128-row boxes
  CUtensorMap h, hs;             // h rows, 32-row boxes
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPThreads, 1)
    moe_ffn_pair(const __grid_constant__ FfnParams p, const __grid_constant__ PairMaps m) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* ctrl = smem + kPStages * kPStage;
  uint64_t* full = reinterpret_cast<uint64_t*>(ctrl);  // [kPStages] (the leader's count)
  uint64_t* empty = full + kPStages;                    // [kPStages]
  uint64_t* tfull = empty + kPStages;                   // [2]
  uint64_t* tempty = tfull + 2;                         // [2] (the leader's count)
  uint64_t* qfull = tempty + 2;                         // [kPQueue]
  uint64_t* qempty = qfull + kPQueue;                   // [kPQueue] (the leader's count)
  volatile long long* prog = reinterpret_cast<volatile long long*>(qempty + kPQueue);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(const_cast<long long*>(prog) + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* qitem = abort_flag + 1;  // [kPQueue]
  int* meta_j = reinterpret_cast<int*>(ctrl + kPCtrl);              // [kPairTileN]
  float* meta_w = reinterpret_cast<float*>(meta_j + kPairTileN);    // [kPairTileN]
  uint32_t* epi_stage = reinterpret_cast<uint32_t*>(meta_w + kPairTileN);  // [warps][kEpiTileWords]
  int* s_gu = reinterpret_cast<int*>(epi_stage + kPEpiWarps * kEpiTileWords);  // [E+2]
  int* s_dn = s_gu + (p.E + 2);                                      // [E+2]
  int* s_off = s_dn + (p.E + 2);                                     // [E+1]
  static_assert(8 * (2 * kPStages + 4 + 2 * kPQueue) + 8 + 4 * (2 + kPQueue) <= kPCtrl, "ctrl");

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank() & 1u;
  const bool leader = rank == 0;
  pdl_trigger();
  if (tid == 0) {
    for (int s = 0; s < kPStages; ++s) {
      // the leader's expect_tx arrival (+ both CTAs' TMA bytes) and one
      // arrival per gatherer warp of both CTAs (the peer's are remote)
      mbar_init(&full[s], 1 + 2 * kPGatherWarps);
      mbar_init(&empty[s], 1);  // the leader's multicast commit
    }
    for (int a = 0; a < 2; ++a) {  // one pair per TMEM half
      mbar_init(&tfull[a], 1);   // multicast commit
      mbar_init(&tempty[a], 2 * kPEpiWarps);  // the epilogue warps of both CTAs
    }
    for (int q = 0; q < kPQueue; ++q) {
      mbar_init(&qfull[q], 1);
      mbar_init(&qempty[q], kPQueueConsumers);
    }
    *prog = 0;
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&m.wg);
    prefetch_tmap(&m.wd);
    prefetch_tmap(&m.h);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kPTmemCols);
    tmem_relinquish_pair();
  }
  pdl_wait();  // the schedule, the routing and x come from earlier kernels
  for (int i = tid; i < p.E + 2; i += blockDim.x) {
    s_gu[i] = p.gu_start[i];
    s_dn[i] = p.dn_start[i];
  }
  for (int i = tid; i < p.E + 1; i += blockDim.x) s_off[i] = p.offsets[i];
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any remote arrival
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int nslots = p.E + (p.has_shared ? 1 : 0);
  const int n_gu = min(p.nitems[0], p.max_gu);
  const int n_dn = min(p.nitems[1], p.max_dn);
  const int n_all = n_gu + n_dn;
  auto item_at = [&](int i, bool& gu) {
    gu = i < n_gu;
    return gu ? decode_item(i, s_gu, s_off, nslots, p.E, p.T, kPairTileN)
              : decode_item(i - n_gu, s_dn, s_off, nslots, p.E, p.T, kPairTileN);
  };
  auto valid = [&](const WorkItem& it, bool gu) {
    return item_ok(p, it, gu, kPairTileN, kPairGuTile, kDownTile);
  };
  const int KB_gu = p.H / 64, KB_dn_r = p.I / 64, KB_dn_s = p.Is / 64;
  auto nkb_of = [&](bool gu, bool sh) { return gu ? KB_gu : (sh ? KB_dn_s : KB_dn_r); };
  // the leader's copy of a barrier, as a cluster address
  auto at_leader = [&](uint64_t* bar) { return mapa_shared(smem_u32(bar), 0); };
  // queue entry n: wait, read, release (one arrival per warp, on the leader's qempty)
  auto next_item = [&](int n, int& item, bool whole_warp) -> bool {
    const int q = n % kPQueue;
    if (!mbar_wait_cluster(&qfull[q], (n / kPQueue) & 1, abort_flag, p.err, MOE_DEVERR_TIMEOUT))
      return false;
    item = qitem[q];
    if (whole_warp) __syncwarp();
    if (lane == 0) {
      if (leader) mbar_arrive(&qempty[q]);
      else mbar_arrive_cluster(at_leader(&qempty[q]));
    }
    return item >= 0;
  };

  if (warp == kPSchedWarp) {
    // ------------------------------------------------------------ scheduler (leader)
    if (leader && lane == 0) {
      int prev_nkb = 0;
      for (int n = 0;; ++n) {
        const int q = n % kPQueue;
        if (!mbar_wait_cluster(&qempty[q], ((n / kPQueue) & 1) ^ 1, abort_flag, p.err,
                               MOE_DEVERR_TIMEOUT))
          break;
        // claim item n when the producer is kPLead k-blocks from the end of item n-1
        if (n > 0 && !wait_progress(prog, (n - 1) * kPProgStride + max(0, prev_nkb - kPLead),
                                    abort_flag, p.err))
          break;
        int item = atomicAdd(p.counter, 1);
        if (item >= n_all) item = -1;
        prev_nkb = 0;
        if (item >= 0) {
          bool gu;
          const WorkItem it = item_at(item, gu);
          if (valid(it, gu)) {
            const bool sh = it.e == p.E;
            prev_nkb = nkb_of(gu, sh);
            if (!gu) {
              // both halves of every gate/up output tile of this (slot, row tile) are in h
              const int r0 = sh ? 0 : s_off[it.e];
              const int ridx = s_gu[it.e] + (it.row0 - r0) / kPairTileN;
              if (!wait_count(p.ready + ridx, 2 * cdiv_dev(sh ? p.Is : p.I, kPairGuTile),
                              abort_flag, p.err))
                item = -1;
            }
          } else {
            atomicExch(p.err, MOE_DEVERR_SCHEDULE);
          }
        }
        // the peer's copy first, then both arrivals (release at cluster scope)
        st_shared_cluster(mapa_shared(smem_u32(const_cast<int*>(&qitem[q])), 1), item);
        qitem[q] = item;
        mbar_arrive_cluster(mapa_shared(smem_u32(&qfull[q]), 1));
        mbar_arrive(&qfull[q]);
        if (item < 0) break;
      }
    }
    __syncwarp();
  } else if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    // This CTA's 128 rows of A, and for down items its half of the h rows;
    // the token rows of gate/up items come from the gatherer warps.
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_h = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      bool live = true;
      for (int n = 0; live; ++n) {
        int item;
        if (!next_item(n, item, false)) break;
        if (leader) *prog = n * kPProgStride;
        bool gu;
        const WorkItem it = item_at(item, gu);
        if (!valid(it, gu)) continue;
        const bool sh = it.e == p.E;
        // h rows of a down item were published by other CTAs (acquired by the
        // leader's scheduler, released to this CTA through the queue)
        if (!gu) fence_proxy_async_global();
        const int wblk = sh ? 0 : (p.wslot ? p.wslot[it.e] : it.e);
        const int nkb = nkb_of(gu, sh);
        const int nhalf = pair_n(it) / 2;  // this CTA's B rows (a multiple of 32)
        const int brow = it.row0 + static_cast<int>(rank) * nhalf;
        const int nbox = gu ? 0 : nhalf / kPBox;
        const uint32_t pair_bytes = 2u * ((gu ? 2 : 1) * kPA + nbox * kPBox * 128);
        int arow0;
        const CUtensorMap *ma0, *ma1 = nullptr;
        if (gu) {
          arow0 = (sh ? 0 : wblk * p.I) + it.ntile * kPairGuTile + static_cast<int>(rank) * 128;
          ma0 = sh ? &m.wgs : &m.wg;
          ma1 = sh ? &m.wus : &m.wu;
        } else {
          arow0 = (sh ? 0 : wblk * p.H) + it.ntile * kDownTile + static_cast<int>(rank) * kTileN;
          ma0 = sh ? &m.wds : &m.wd;
        }
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) {
            live = false;
            break;
          }
          uint8_t* sA = smem + stage * kPStage;
          uint8_t* sB = sA + 2 * kPA;
          const uint32_t lbar = at_leader(&full[stage]);
          if (leader) mbar_arrive_expect_tx(&full[stage], pair_bytes);
          if (gu) {
            tma_load_2d_pair(sA, ma0, lbar, kb * 64, arow0, pol_w);        // gate rows
            tma_load_2d_pair(sA + kPA, ma1, lbar, kb * 64, arow0, pol_w);  // up rows
          } else {
            tma_load_2d_pair(sA, ma0, lbar, kb * 64, arow0, pol_w);
          }
          for (int b = 0; b < nbox; ++b)
            tma_load_2d_pair(sB + b * kPBox * 128, sh ? &m.hs : &m.h, lbar, kb * 64,
                             brow + b * kPBox, pol_h);
          if (leader) *prog = n * kPProgStride + kb + 1;
          if (++stage == kPStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // every stage must be released by the MMA before teardown
      for (int i = 0; i < kPStages && live; ++i) {
        if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err, MOE_DEVERR_TIMEOUT))
          break;
        if (++stage == kPStages) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader)
    if (leader && lane == 0) {
      int stage = 0, dn_half = 0;
      uint32_t phase = 0;
      uint32_t used0 = 0u, used1 = 0u;  // items that took TMEM half 0 / 1 so far
      bool live = true;
      for (int n = 0; live; ++n) {
        int item;
        if (!next_item(n, item, false)) break;
        bool gu;
        const WorkItem it = item_at(item, gu);
        if (!valid(it, gu)) continue;
        const int nkb = nkb_of(gu, it.e == p.E);
        const uint32_t idesc = idesc_bf16(2 * kTileN, pair_n(it));
        // gate/up: both halves (gate in 0, up in 1); down: the next half in turn
        const int h0 = gu ? 0 : dn_half, h1 = gu ? 1 : dn_half;
        const uint32_t par0 = (h0 ? used1 : used0) & 1u, par1 = (h1 ? used1 : used0) & 1u;
        if (!mbar_wait_cluster(&tempty[h0], par0 ^ 1u, abort_flag, p.err, MOE_DEVERR_TIMEOUT))
          break;
        if (gu && !mbar_wait_cluster(&tempty[h1], par1 ^ 1u, abort_flag, p.err, MOE_DEVERR_TIMEOUT))
          break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + h0 * kPAccCols;
        const uint32_t d1 = tmem_base + h1 * kPAccCols;
        for (int kb = 0; kb < nkb; ++kb) {
          // acquire at cluster scope: the peer's gatherers arrive from the other CTA
          if (!mbar_wait_cluster(&full[stage], phase, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) {
            live = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + stage * kPStage);
          const uint32_t b0 = a0 + 2 * kPA;
          if (gu) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint32_t acc = (kb | kk) != 0 ? 1u : 0u;
              umma_bf16_pair(d0, sdesc_k128(a0 + kk * 32), sdesc_k128(b0 + kk * 32), idesc, acc);
              umma_bf16_pair(d1, sdesc_k128(a0 + kPA + kk * 32), sdesc_k128(b0 + kk * 32), idesc,
                             acc);
            }
          } else {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_bf16_pair(d0, sdesc_k128(a0 + kk * 32), sdesc_k128(b0 + kk * 32), idesc,
                             (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit_pair_mc(&empty[stage], 0x3);  // frees the stage in both CTAs
          if (++stage == kPStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!live) break;
        umma_commit_pair_mc(&tfull[h0], 0x3);
        if (gu) {
          umma_commit_pair_mc(&tfull[h1], 0x3);
          ++used0;
          ++used1;
        } else {
          if (h0) ++used1;
          else ++used0;
          dn_half ^= 1;
        }
      }
    }
    __syncwarp();
  } else if (warp >= kPGatherWarp0 && warp < kPSchedWarp) {
    // ------------------------------------------------------------ token gatherers (both CTAs)
    // Gate/up items: thread g copies 16-byte chunk (g % 8) of rows g/8,
    // g/8 + 16, ... of this CTA's half of the token tile into the
    // 128-byte-swizzled layout (chunk c of row r lands at c ^ (r % 8)). A
    // stage's copies retire two stages later: wait for the group, make it
    // visible to the tensor cores (proxy fence), then one arrival per warp on
    // the leader's full barrier. Down items copy nothing but keep the stage
    // sequence and the arrivals.
    constexpr int kRowsPerThread = kPairTileN / 2 / 16;
    constexpr int kLag = 2;
    const int g = tid - kPGatherWarp0 * 32;
    const int chunk = g & 7, rbase = g >> 3;
    const uint64_t pol_x = policy_evict_last();
    int stage = 0;
    uint32_t phase = 0;
    int pend[2] = {-1, -1};  // stages issued and not yet retired, oldest first
    bool live = true;
    // The peer's copies are in its own shared memory: a release restricted to
    // shared memory, then a relaxed arrive on the leader's barrier (a full
    // cluster-scope release would also wait for the copies still in flight).
    auto retire = [&](int st) {
      if (leader) {
        mbar_arrive(&full[st]);
      } else {
        fence_release_shared_cluster();
        mbar_arrive_cluster_relaxed(at_leader(&full[st]));
      }
    };
    for (int n = 0; live; ++n) {
      // The scheduler may hold the next item back until gate/up tiles this
      // pair is still finishing are published, and the MMA cannot finish them
      // before their stages retire: if the next item is not queued yet,
      // retire the pending stages before waiting for it.
      const int q = n % kPQueue;
      const bool queued = __shfl_sync(
          0xffffffffu, lane == 0 ? (mbar_try_wait_cluster(&qfull[q], (n / kPQueue) & 1) ? 1 : 0) : 0, 0) != 0;
      if (!queued && (pend[0] >= 0 || pend[1] >= 0)) {
        cp_async_wait<0>();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (pend[0] >= 0) retire(pend[0]);
          if (pend[1] >= 0) retire(pend[1]);
        }
        pend[0] = pend[1] = -1;
      }
      int item;
      if (!next_item(n, item, true)) break;
      bool gu;
      const WorkItem it = item_at(item, gu);
      if (!valid(it, gu)) continue;
      const bool sh = it.e == p.E;
      const int nkb = nkb_of(gu, sh);
      const int nhalf = pair_n(it) / 2;  // this CTA's B rows
      const int brow = it.row0 + static_cast<int>(rank) * nhalf;
      const uint16_t* src[kRowsPerThread];
#pragma unroll
      for (int i = 0; i < kRowsPerThread; ++i) {
        // rows past the item repeat its last row (their columns are never stored)
        const int row = min(brow + rbase + 16 * i, it.row0 + it.nrows - 1);
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
          uint8_t* sB = smem + stage * kPStage + 2 * kPA;
#pragma unroll
          for (int i = 0; i < kRowsPerThread; ++i) {
            const int r = rbase + 16 * i;
            if (r < nhalf) cp_async16(sB + r * 128 + ((chunk ^ (r & 7)) << 4), src[i] + kb * 64, pol_x);
          }
        }
        cp_async_commit();
        if (pend[0] >= 0) {
          cp_async_wait<kLag>();     // this lane's copies for the oldest pending stage landed
          fence_proxy_async_smem();  // ... and are visible to the tensor cores
          __syncwarp();
          if (lane == 0) retire(pend[0]);
        }
        pend[0] = pend[1];
        pend[1] = stage;
        if (++stage == kPStages) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    cp_async_wait<0>();  // nothing may still be landing in shared memory at exit
    fence_proxy_async_smem();
    __syncwarp();
    if (live && lane == 0) {
      if (pend[0] >= 0) retire(pend[0]);
      if (pend[1] >= 0) retire(pend[1]);
    }
  } else if (warp >= 2 && warp < 2 + kPEpiWarps) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;            // TMEM lane quarter
    const int orow = q * 32 + lane;    // row of this CTA's D
    const int et = tid - 64;           // epilogue thread 0..255
    const int cpart = et >> 7;         // column chunks of this warp: alternate ones
    int dn_half = 0;
    uint32_t used0 = 0u, used1 = 0u;  // the MMA issuer's sequence of TMEM halves
    for (int n = 0;; ++n) {
      int item;
      if (!next_item(n, item, true)) break;
      bool gu;
      const WorkItem it = item_at(item, gu);
      if (!valid(it, gu)) continue;
      const bool sh = it.e == p.E;
      const int ncol = pair_n(it);
      if (!gu) {
        // destination slot and routing weight of every row, staged while the MMAs run
        epi_bar<kPEpiThreads>();
        for (int rr = et; rr < kPairTileN; rr += kPEpiThreads) {
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
        epi_bar<kPEpiThreads>();
      }
      const int h0 = gu ? 0 : dn_half, h1 = gu ? 1 : dn_half;
      const uint32_t par0 = (h0 ? used1 : used0) & 1u, par1 = (h1 ? used1 : used0) & 1u;
      if (!mbar_wait(&tfull[h0], par0, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) break;
      if (gu && !mbar_wait(&tfull[h1], par1, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) break;
      tc_fence_after();
      const uint32_t tq = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
      const uint32_t taddr = tq + h0 * kPAccCols;
      if (gu) {
        // lane = feature: gate in half 0, up in half 1 of the same lane. Per
        // 16-token chunk the warp's 32 features x 16 tokens of h go through
        // its shared-memory tile, so that each lane then stores 16-byte
        // pieces of token rows (8 features) instead of single values.
        const int fbase = it.ntile * kPairGuTile + static_cast<int>(rank) * 128 + q * 32;
        const int ncols = sh ? p.Is : p.I;
        const bool ok = fbase < ncols;  // I and Is are multiples of 64: whole warps
        const float L = sh ? p.lim_s : p.lim_r;
        uint16_t* hout = sh ? p.h_s : p.h_r;
        uint32_t* tile = epi_stage + (warp - 2) * kEpiTileWords;
#pragma unroll 1
        for (int c0 = 16 * cpart; c0 < ncol && ok; c0 += 32) {
          float g[16], u[16];
          tmem_ld16(tq + c0, g);
          tmem_ld16(tq + kPAccCols + c0, u);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 16; ++c) g[c] = swiglu(g[c], u[c], L);
          store_h16(g, tile, hout, ncols, it.row0 + c0, it.nrows - c0, fbase, lane);
        }
      } else {
        const int fbase = it.ntile * kDownTile + static_cast<int>(rank) * kTileN + q * 32;
        const bool ok = fbase < p.H;  // H is a multiple of 64: whole warps
        uint32_t* tile = epi_stage + (warp - 2) * kEpiTileWords;
        // 32 columns per TMEM wait (ncol is a multiple of 64), alternate groups per warp
#pragma unroll 1
        for (int c0 = 32 * cpart; c0 < ncol && ok; c0 += 64) {
          float ov[32];
          tmem_ld16(taddr + c0, ov);
          tmem_ld16(taddr + c0 + 16, ov + 16);
          tmem_ld_wait();
#pragma unroll
          for (int g8 = 0; g8 < 4; ++g8) {
            float v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = meta_w[c0 + 8 * g8 + i] * ov[8 * g8 + i];
            store_y8(v, meta_j + c0 + 8 * g8, tile, p.y_slot, p.H, fbase, lane);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader) mbar_arrive(&tempty[h0]);
        else mbar_arrive_cluster(at_leader(&tempty[h0]));
        if (gu) {
          if (leader) mbar_arrive(&tempty[h1]);
          else mbar_arrive_cluster(at_leader(&tempty[h1]));
        }
      }
      if (gu) {
        ++used0;
        ++used1;
      } else {
        if (h0) ++used1;
        else ++used0;
        dn_half ^= 1;
      }
      if (gu) {
        // publish this CTA's half of the output tile of h
        fence_proxy_async_global();
        epi_bar<kPEpiThreads>();
        if (warp == 2 && lane == 0) {
          __threadfence();
          const int r0 = sh ? 0 : s_off[it.e];
          atomicAdd(p.ready + s_gu[it.e] + (it.row0 - r0) / kPairTileN, 1);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no CTA leaves while the other may still arrive on its barriers
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kPTmemCols);
  }
}

}  // namespace

cudaError_t launch_ffn_pair(const GemmArgs& a, cudaStream_t s) {
  const moe_cfg& c = *a.cfg;
  const int T = a.T, TK = a.T * c.K;
  FfnParams p;
  memset(&p, 0, sizeof(p));
  p.T = T;
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
  p.wslot = a.wslot;
  p.gu_start = a.gu_start;
  p.dn_start = a.dn_start;
  p.nitems = a.nitems;
  p.counter = const_cast<int32_t*>(a.nitems) + 2;
  p.ready = a.ready;
  p.max_gu = a.max_items_gu;
  p.max_dn = a.max_items_dn;
  p.err = a.err;
  PairMaps m;
  const uint64_t wr = static_cast<uint64_t>(a.wrows);
  bool ok = map_bf16(&m.wg, a.Wg, wr * c.I, c.H, 128) && map_bf16(&m.wu, a.Wu, wr * c.I, c.H, 128) &&
            map_bf16(&m.wd, a.Wd, wr * c.H, c.I, kTileN) &&
            map_bf16(&m.h, a.h_r, TK, c.I, kPBox);
  if (p.has_shared) {
    ok = ok && map_bf16(&m.wgs, a.W->Wg_s, c.I_shared, c.H, 128) &&
         map_bf16(&m.wus, a.W->Wu_s, c.I_shared, c.H, 128) &&
         map_bf16(&m.wds, a.W->Wd_s, c.H, c.I_shared, kTileN) &&
         map_bf16(&m.hs, a.h_s, T, c.I_shared, kPBox);
  } else {
    m.wgs = m.wg;
    m.wus = m.wu;
    m.wds = m.wd;
    m.hs = m.h;
  }
  if (!ok) return cudaErrorInvalidValue;
  const int smem_max = kPSmem + (3 * kMaxExpertsCfg + 5) * static_cast<int>(sizeof(int));
  const int smem = kPSmem + (3 * c.E + 5) * static_cast<int>(sizeof(int));
  cudaError_t e = ensure_dyn_smem(reinterpret_cast<const void*>(moe_ffn_pair), smem_max);
  if (e != cudaSuccess) return e;
  // clusters of two CTAs, one per SM; items are claimed by running CTAs only,
  // so every wait is on work a resident CTA has already taken
  const int grid = num_sms() & ~1;
  return launch_pdl(moe_ffn_pair, dim3(grid), dim3(kPThreads), smem, s, p, m);
}

}  // namespace sgl
