// ffn.cu - stages 7 and 8: the grouped SwiGLU experts and the shared expert,
// in one persistent tcgen05 kernel.
//
// Page "Ling-3.0-flash-VL MoE sparse routing" (lqnn.cn/news/282163): sec. 2
// (an expert is a gate / up / down SwiGLU FFN, hidden 2560, intermediate 768;
// one shared expert sees every token) and sec. 4 (SwiGLU limit +-4 on routed
// experts, +-5/+-7 on the shared expert). The limit clamps gate and up to
// [-L, L] before silu(gate) * up.
//
// Every product is D = W_tile * X_tile^T with the weights as the MMA's 128-row
// A operand and a tile of BN rows (tokens) as its N: an expert sees few tokens,
// so the weights fill the 128-row side. Two kinds of work item, both with two
// A tiles and one B tile per pipeline stage and two accumulators:
//   gate/up (slot e, row tile m, feature tile n of 128), K = H:
//       A0 = Wg rows, A1 = Wu rows, B = the routed token rows of x (gathered);
//       epilogue h = bf16(silu(clamp(D0)) * clamp(D1)) in permuted row order.
//   down (slot e, row tile m, output tile n of 256), K = I:
//       A0 / A1 = Wd rows [256n, 256n+128) / [256n+128, 256n+256), B = h rows;
//       epilogue y_slot[j] = w_j * D (fp32) at the row's flat slot index j.
// Slot E is the shared expert: its rows are the T tokens, its weight 1.
//
// The work lists (per-slot item starts and row offsets) come from the
// permutation kernels, or, after the fused decode front, are derived from the
// expert counts in every CTA's prologue (the same values).
//
// Items are claimed dynamically from one global counter: gate/up items
// [0, Ngu), then down items. A down item reads h rows that other CTAs' gate/up
// epilogues wrote; those epilogues count finished tiles per (slot, row tile)
// in ready[] (stores, async-proxy fence, CTA barrier, threadfence, atomic)
// and the claiming CTA waits for the count with an acquire load. Gate/up items
// never wait, every CTA is resident (cooperative launch), and a claimed
// gate/up item runs on its CTA's pipeline whatever that CTA's scheduler is
// waiting for, so every wait ends.
//
// Warp roles per CTA (480 threads):
//   0      TMA producer (lane 0): weight tiles, and h tiles of down items
//   1      MMA issuer (lane 0), owner of the TMEM accumulators
//   2..9   epilogue: two warps per TMEM lane quarter (warp % 4), alternate
//          column chunks
//   10..13 token gatherers: cp.async of the routed x rows into the swizzled
//          B tile of gate/up stages, completion tracked by the stage's barrier
//   14     scheduler (lane 0): claims the next item while the current one is
//          still streaming, waits for its inputs, and queues it for the others
// Pipelines: STAGES shared-memory stages (full / empty mbarriers), two TMEM
// accumulator buffers (tfull / tempty) so the epilogue of one item overlaps
// the MMAs of the next, and a 4-entry item queue (qfull / qempty). Every wait
// is bounded (ptx.cuh); a timeout raises the CTA's abort flag and the error
// word, and the kernel winds down.
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

constexpr int kEpiWarps = 8;      // warps 2..9: two per TMEM lane quarter
constexpr int kGatherWarp0 = 2 + kEpiWarps;
constexpr int kGatherWarps = 4;   // warps 10..13
constexpr int kSchedWarp = kGatherWarp0 + kGatherWarps;  // warp 14
constexpr int kFfnThreads = 32 * (kSchedWarp + 1);
constexpr int kQueue = 4;                 // item queue entries
constexpr int kLead = 4;                  // claim the next item this many k-blocks early
constexpr long long kProgStride = 1024;   // producer progress = n * stride + k-blocks issued
constexpr int kSmemBudget = 210 * 1024;   // pipeline stages

template <int BN>
struct Cfg {
  static constexpr int A_BYTES = kTileN * 128;  // 128 rows x 64 bf16
  static constexpr int B_BYTES = BN * 128;      // BN rows x 64 bf16
  static constexpr int STAGE_BYTES = 2 * A_BYTES + B_BYTES;
  static constexpr int STAGES_RAW = kSmemBudget / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
  static constexpr int ACC_COLS = 2 * BN;       // two fp32 accumulators side by side
  // accumulator buffers: two (the epilogue of one item overlaps the MMAs of
  // the next) while they fit the 512 TMEM columns, else one
  static constexpr int NACC = 2 * ACC_COLS <= 512 ? 2 : 1;
  static constexpr int TMEM_COLS = NACC * ACC_COLS < 32 ? 32 : NACC * ACC_COLS;
  static constexpr int H_BOX = BN < 64 ? BN : 64;  // rows per TMA box of h
  static_assert((TMEM_COLS & (TMEM_COLS - 1)) == 0 && TMEM_COLS <= 512, "TMEM allocation");
  static constexpr int CTRL_BYTES = 512;        // barriers, queue, flags
  // + the per-slot item starts and row offsets, (3E + 5) ints, added at launch
  static constexpr int SMEM = STAGES * STAGE_BYTES + 1024 /*align*/ + CTRL_BYTES + BN * 8;
  static_assert(8 * (2 * 8 + 2 * 2 + 2 * kQueue) + 8 + 4 * (2 + kQueue) <= CTRL_BYTES,
                "control block");
};

template <int BN>
__global__ void __launch_bounds__(kFfnThreads, 1)
    moe_ffn(const __grid_constant__ FfnParams p, const __grid_constant__ CUtensorMap tWg,
            const __grid_constant__ CUtensorMap tWu, const __grid_constant__ CUtensorMap tWgS,
            const __grid_constant__ CUtensorMap tWuS, const __grid_constant__ CUtensorMap tWd,
            const __grid_constant__ CUtensorMap tWdS, const __grid_constant__ CUtensorMap tH,
            const __grid_constant__ CUtensorMap tHs) {
  using C = Cfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* ctrl = smem + C::STAGES * C::STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(ctrl);
  uint64_t* empty = full + 8;
  uint64_t* tfull = empty + 8;
  uint64_t* tempty = tfull + 2;
  uint64_t* qfull = tempty + 2;
  uint64_t* qempty = qfull + kQueue;
  volatile long long* prog = reinterpret_cast<volatile long long*>(qempty + kQueue);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(const_cast<long long*>(prog) + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* qitem = abort_flag + 1;  // [kQueue]
  int* meta_j = reinterpret_cast<int*>(ctrl + C::CTRL_BYTES);
  float* meta_w = reinterpret_cast<float*>(meta_j + BN);
  int* s_gu = reinterpret_cast<int*>(meta_w + BN);  // [E+2]
  int* s_dn = s_gu + (p.E + 2);                      // [E+2]
  int* s_off = s_dn + (p.E + 2);                     // [E+1]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_trigger();
  if (tid == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1 + 32 * kGatherWarps);  // weight TMA + one arrival per gatherer thread
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], kEpiWarps);
    }
    for (int q = 0; q < kQueue; ++q) {
      mbar_init(&qfull[q], 1);
      mbar_init(&qempty[q], 1 + 1 + kEpiWarps + kGatherWarps);  // producer, MMA, epilogue, gatherers
    }
    *prog = 0;
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tWg);
    prefetch_tmap(&tWu);
    prefetch_tmap(&tWd);
    prefetch_tmap(&tH);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  pdl_wait();  // the schedule, the routing and x come from earlier kernels
  int n_gu_all, n_dn_all;
  if (p.sched_counts) {
    __shared__ int wsum[33];
    derive_schedule(p, s_gu, s_dn, s_off, wsum, &n_gu_all, &n_dn_all);
  } else {
    for (int i = tid; i < p.E + 2; i += blockDim.x) {
      s_gu[i] = p.gu_start[i];
      s_dn[i] = p.dn_start[i];
    }
    for (int i = tid; i < p.E + 1; i += blockDim.x) s_off[i] = p.offsets[i];
    n_gu_all = p.nitems[0];
    n_dn_all = p.nitems[1];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int nslots = p.E + (p.has_shared ? 1 : 0);
  const int n_gu = min(n_gu_all, p.max_gu);
  const int n_dn = min(n_dn_all, p.max_dn);
  const int n_all = n_gu + n_dn;
  auto item_at = [&](int i, bool& gu) {
    gu = i < n_gu;
    return gu ? decode_item(i, s_gu, s_off, nslots, p.E, p.T, BN)
              : decode_item(i - n_gu, s_dn, s_off, nslots, p.E, p.T, BN);
  };
  const int KB_gu = p.H / 64, KB_dn_r = p.I / 64, KB_dn_s = p.Is / 64;
  auto nkb_of = [&](bool gu, bool sh) { return gu ? KB_gu : (sh ? KB_dn_s : KB_dn_r); };
  // a down item's second 128-row half exists unless it starts past H
  auto two_halves = [&](const WorkItem& it, bool gu) {
    return gu || it.ntile * kDownTile + kTileN < p.H;
  };
  auto mma_n = [&](const WorkItem& it) { return (min(it.nrows, BN) + 15) & ~15; };
  // queue entry n: wait for it, read it, release it (one arrival per warp)
  auto next_item = [&](int n, int& item, bool whole_warp) -> bool {
    const int q = n % kQueue;
    if (!mbar_wait(&qfull[q], (n / kQueue) & 1, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) return false;
    item = qitem[q];
    if (whole_warp) __syncwarp();
    if (lane == 0) mbar_arrive(&qempty[q]);
    return item >= 0;
  };

  if (warp == kSchedWarp) {
    // ------------------------------------------------------------ scheduler
    if (lane == 0) {
      int prev_nkb = 0;
      for (int n = 0;; ++n) {
        const int q = n % kQueue;
        if (!mbar_wait(&qempty[q], ((n / kQueue) & 1) ^ 1, abort_flag, p.err, MOE_DEVERR_TIMEOUT))
          break;
        // claim item n only when the producer is kLead k-blocks from the end
        // of item n-1: early enough to hide the claim and the input wait,
        // late enough not to hoard work other CTAs could start sooner
        if (n > 0 && !wait_progress(prog, (n - 1) * kProgStride + max(0, prev_nkb - kLead),
                                    abort_flag, p.err))
          break;
        int item = atomicAdd(p.counter, 1);
        if (item >= n_all) item = -1;
        prev_nkb = 0;
        if (item >= 0) {
          bool gu;
          const WorkItem it = item_at(item, gu);
          if (item_ok(p, it, gu, BN)) {
            const bool sh = it.e == p.E;
            prev_nkb = nkb_of(gu, sh);
            if (!gu) {
              // every gate/up output tile of this (slot, row tile) must be in h
              const int r0 = sh ? 0 : s_off[it.e];
              const int ridx = s_gu[it.e] + (it.row0 - r0) / BN;
              if (!wait_count(p.ready + ridx, cdiv_dev(sh ? p.Is : p.I, kTileN), abort_flag, p.err))
                item = -1;
            }
          } else {
            atomicExch(p.err, MOE_DEVERR_SCHEDULE);
          }
        }
        qitem[q] = item;
        mbar_arrive(&qfull[q]);
        if (item < 0) break;
      }
    }
    __syncwarp();
  } else if (warp == 0) {
    // ------------------------------------------------------------ weight / h TMA
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_h = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      bool live = true;
      for (int n = 0; live; ++n) {
        int item;
        if (!next_item(n, item, false)) break;
        *prog = n * kProgStride;
        bool gu;
        const WorkItem it = item_at(item, gu);
        if (!item_ok(p, it, gu, BN)) continue;
        const bool sh = it.e == p.E;
        const bool two = two_halves(it, gu);
        // h rows of a down item were published by other CTAs (the scheduler
        // acquired them); order the async-proxy reads after that
        if (!gu) fence_proxy_async_global();
        const int wblk = sh ? 0 : (p.wslot ? p.wslot[it.e] : it.e);
        const int nkb = nkb_of(gu, sh);
        const CUtensorMap* mA0 = gu ? (sh ? &tWgS : &tWg) : (sh ? &tWdS : &tWd);
        const CUtensorMap* mA1 = gu ? (sh ? &tWuS : &tWu) : mA0;
        const int arow0 = gu ? (sh ? 0 : wblk * p.I) + it.ntile * kTileN
                             : (sh ? 0 : wblk * p.H) + it.ntile * kDownTile;
        const int arow1 = gu ? arow0 : arow0 + kTileN;
        const int nhbox = gu ? 0 : (mma_n(it) + C::H_BOX - 1) / C::H_BOX;
        const uint32_t bytes = (two ? 2 : 1) * C::A_BYTES + nhbox * C::H_BOX * 128;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) {
            live = false;
            break;
          }
          uint8_t* sA = smem + stage * C::STAGE_BYTES;
          mbar_arrive_expect_tx(&full[stage], bytes);
          tma_load_2d(sA, mA0, &full[stage], kb * 64, arow0, pol_w);
          if (two) tma_load_2d(sA + C::A_BYTES, mA1, &full[stage], kb * 64, arow1, pol_w);
          for (int hb = 0; hb < nhbox; ++hb)
            tma_load_2d(sA + 2 * C::A_BYTES + hb * C::H_BOX * 128, sh ? &tHs : &tH, &full[stage],
                        kb * 64, it.row0 + hb * C::H_BOX, pol_h);
          *prog = n * kProgStride + kb + 1;
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // every stage must be released by its MMA commit before teardown
      for (int i = 0; i < C::STAGES && live; ++i) {
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
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool live = true;
      for (int n = 0; live; ++n) {
        int item;
        if (!next_item(n, item, false)) break;
        bool gu;
        const WorkItem it = item_at(item, gu);
        if (!item_ok(p, it, gu, BN)) continue;
        const int nkb = nkb_of(gu, it.e == p.E);
        const bool two = two_halves(it, gu);
        // MMA N = the item's rows rounded up to 16 (the B rows past it are never read)
        const uint32_t idesc = idesc_bf16(kTileN, mma_n(it));
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
          const uint32_t b0 = a0 + 2 * C::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bd = sdesc_k128(b0 + kk * 32);
            const uint32_t accum = (kb | kk) != 0 ? 1u : 0u;
            umma_bf16(d0, sdesc_k128(a0 + kk * 32), bd, idesc, accum);
            if (two) umma_bf16(d0 + BN, sdesc_k128(a0 + C::A_BYTES + kk * 32), bd, idesc, accum);
          }
          umma_commit(&empty[stage]);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!live) break;
        umma_commit(&tfull[acc]);
        if (++acc == C::NACC) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
    }
    __syncwarp();
  } else if (warp >= kGatherWarp0) {
    // ------------------------------------------------------------ token gatherers
    // Gate/up items: thread g copies 16-byte chunk (g % 8) of rows g/8,
    // g/8 + 16, ... of the stage's BN x 64 token tile straight into the
    // 128-byte-swizzled layout (chunk c of row r lands at c ^ (r % 8)). Each
    // thread then hands the stage's full barrier an arrival that fires when
    // its copies have landed (cp.async.mbarrier.arrive.noinc), so gatherers
    // run as far ahead as the free stages allow. Down items copy nothing but
    // keep the stage sequence and the arrivals.
    constexpr int kRowsPerThread = BN / 16;
    const int g = tid - kGatherWarp0 * 32;
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
      if (!item_ok(p, it, gu, BN)) continue;
      const bool sh = it.e == p.E;
      const int nkb = nkb_of(gu, sh);
      const int nb = mma_n(it);  // B rows the MMA reads
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
          uint8_t* sB = smem + stage * C::STAGE_BYTES + 2 * C::A_BYTES;
#pragma unroll
          for (int i = 0; i < kRowsPerThread; ++i) {
            const int r = rbase + 16 * i;
            if (r < nb) cp_async16(sB + r * 128 + ((chunk ^ (r & 7)) << 4), src[i] + kb * 64, pol_x);
          }
        }
        cp_async_mbar_arrive_noinc(&full[stage]);
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    cp_async_wait_all();  // nothing may still be landing in shared memory at exit
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;            // TMEM lane quarter of this warp
    const int orow = q * 32 + lane;    // output feature within a 128-row half
    const int et = tid - 2 * 32;       // epilogue thread 0..255
    const int cpart = et >> 7;         // which of the two warps of the quarter: column chunks
    constexpr int kEpiThreads = 32 * kEpiWarps;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int n = 0;; ++n) {
      int item;
      if (!next_item(n, item, true)) break;
      bool gu;
      const WorkItem it = item_at(item, gu);
      if (!item_ok(p, it, gu, BN)) continue;
      const bool sh = it.e == p.E;
      if (!gu) {
        // destination slot and routing weight of every row, staged while the
        // item's MMAs run (the store loop then touches no metadata in global)
        epi_bar<kEpiThreads>();  // every epilogue warp is done with the previous item's rows
        for (int rr = et; rr < BN; rr += kEpiThreads) {
          int j = -1;
          float wt = 0.f;
          if (rr < it.nrows) {
            const int row = it.row0 + rr;
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
          meta_j[rr] = j;
          meta_w[rr] = wt;
        }
        epi_bar<kEpiThreads>();
      }
      if (!mbar_wait(&tfull[acc], acc_phase, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * C::ACC_COLS;
      if (gu) {
        const int nfeat = it.ntile * kTileN + orow;
        const int ncols = sh ? p.Is : p.I;
        const bool ok = nfeat < ncols;
        const float L = sh ? p.lim_s : p.lim_r;
        uint16_t* hout = sh ? p.h_s : p.h_r;
        const int ncol = mma_n(it);
        // the two warps of a lane quarter take alternate 16-column chunks
#pragma unroll 1
        for (int c0 = 16 * cpart; c0 < ncol; c0 += 32) {
          float gv[16], uv[16];
          tmem_ld16(taddr + c0, gv);
          tmem_ld16(taddr + BN + c0, uv);
          tmem_ld_wait();
          if (ok) {
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const int r = c0 + c;
              if (r < it.nrows)
                hout[static_cast<size_t>(it.row0 + r) * ncols + nfeat] = f2bf(swiglu(gv[c], uv[c], L));
            }
          }
        }
      } else {
        const int ncol = mma_n(it);
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
          const int nfeat = it.ntile * kDownTile + half * kTileN + orow;
          const bool ok = nfeat < p.H;
          // kCols columns per TMEM wait (the loads of one group are in flight
          // together); the two warps of a lane quarter take alternate groups
          constexpr int kCols = BN >= 32 ? 32 : 16;
#pragma unroll 1
          for (int c0 = kCols * cpart; c0 < ncol; c0 += 2 * kCols) {
            float ov[kCols];
#pragma unroll
            for (int u = 0; u < kCols; u += 16) tmem_ld16(taddr + half * BN + c0 + u, ov + u);
            tmem_ld_wait();
            if (ok) {
#pragma unroll
              for (int c = 0; c < kCols; ++c) {
                const int j = meta_j[c0 + c];
                if (j >= 0) p.y_slot[static_cast<size_t>(j) * p.H + nfeat] = meta_w[c0 + c] * ov[c];
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (++acc == C::NACC) {
        acc = 0;
        acc_phase ^= 1;
      }
      if (gu) {
        // publish this output tile of h: stores -> async proxy -> CTA -> GPU
        fence_proxy_async_global();
        epi_bar<kEpiThreads>();
        if (warp == 2 && lane == 0) {
          __threadfence();
          const int r0 = sh ? 0 : s_off[it.e];
          atomicAdd(p.ready + s_gu[it.e] + (it.row0 - r0) / BN, 1);
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

template <int BN>
cudaError_t launch_bn(const GemmArgs& a, cudaStream_t s) {
  using C = Cfg<BN>;
  const moe_cfg& c = *a.cfg;
  FfnParams p;
  memset(&p, 0, sizeof(p));
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
  p.wslot = a.wslot;
  p.gu_start = a.gu_start;
  p.dn_start = a.dn_start;
  p.nitems = a.nitems;
  p.counter = const_cast<int32_t*>(a.nitems) + 2;
  p.ready = a.ready;
  p.max_gu = a.max_items_gu;
  p.max_dn = a.max_items_dn;
  p.err = a.err;
  p.sched_counts = a.sched_counts;
  p.bn = BN;
  p.gu_ft = kTileN;
  p.dn_ft = kDownTile;
  const int T = a.T, TK = a.T * c.K;
  CUtensorMap tWg, tWu, tWgS, tWuS, tWd, tWdS, tH, tHs;
  bool ok = map_bf16(&tWg, a.Wg, static_cast<uint64_t>(a.wrows) * c.I, c.H, kTileN) &&
            map_bf16(&tWu, a.Wu, static_cast<uint64_t>(a.wrows) * c.I, c.H, kTileN) &&
            map_bf16(&tWd, a.Wd, static_cast<uint64_t>(a.wrows) * c.H, c.I, kTileN) &&
            map_bf16(&tH, a.h_r, TK, c.I, C::H_BOX);
  if (p.has_shared) {
    ok = ok && map_bf16(&tWgS, a.W->Wg_s, c.I_shared, c.H, kTileN) &&
         map_bf16(&tWuS, a.W->Wu_s, c.I_shared, c.H, kTileN) &&
         map_bf16(&tWdS, a.W->Wd_s, c.H, c.I_shared, kTileN) &&
         map_bf16(&tHs, a.h_s, T, c.I_shared, C::H_BOX);
  } else {
    tWgS = tWg;
    tWuS = tWu;
    tWdS = tWd;
    tHs = tH;
  }
  if (!ok) return cudaErrorInvalidValue;
  auto kern = moe_ffn<BN>;
  const int smem_max = C::SMEM + (3 * kMaxExpertsCfg + 5) * static_cast<int>(sizeof(int));
  const int smem = C::SMEM + (3 * c.E + 5) * static_cast<int>(sizeof(int));
  cudaError_t e = ensure_dyn_smem(reinterpret_cast<const void*>(kern), smem_max);
  if (e != cudaSuccess) return e;
  // One CTA per SM. Items are claimed only by running CTAs, so a down item
  // only ever waits on gate/up tiles a resident CTA has taken: no
  // co-residency guarantee is needed.
  return launch_pdl(kern, dim3(num_sms()), dim3(kFfnThreads), smem, s, p, tWg, tWu, tWgS, tWuS, tWd,
                    tWdS, tH, tHs);
}

}  // namespace

cudaError_t launch_ffn(const GemmArgs& a, cudaStream_t s) {
  if (a.ffn == kFfnPair) return a.bn == kPairTileN ? launch_ffn_pair(a, s) : cudaErrorInvalidValue;
  if (a.ffn != kFfnNarrow) return cudaErrorInvalidValue;
  switch (a.bn) {
    case 16: return launch_bn<16>(a, s);
    case 32: return launch_bn<32>(a, s);
    case 64: return launch_bn<64>(a, s);
    case 128: return launch_bn<128>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace sgl
