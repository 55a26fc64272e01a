// ffn.cu - stages 7 and 8: the grouped SwiGLU experts and the shared expert,
// in one persistent tcgen05 kernel.
//
// Page "Ling-3.0-flash-VL MoE sparse routing" (lqnn.cn/news/282163): sec. 2
// (an expert is a gate / up / down SwiGLU FFN, hidden 2560, intermediate 768;
// one shared expert sees every token) and sec. 4 (SwiGLU limit +-4 on routed
// experts, +-5/+-7 on the shared expert). The limit clamps gate and up to
// [-L, L] before silu(gate) * up.
//
// Two kinds of work item, each with two 128-row weight tiles (W0, W1) and one
// tile of up to BN token rows (X) per pipeline stage:
//   gate/up (slot e, row tile m, feature tile n of 128), K = H:
//       W0 = Wg rows, W1 = Wu rows, X = the routed token rows of x (gathered);
//       epilogue h = bf16(silu(clamp(gate)) * clamp(up)) in permuted row order.
//   down (slot e, row tile m, output tile n of 256), K = I:
//       W0 / W1 = Wd rows [256n, 256n+128) / [256n+128, 256n+256), X = h rows;
//       epilogue y_slot[j] = w_j * out (fp32) at the row's flat slot index j.
// Slot E is the shared expert: its rows are the T tokens, its weight 1.
// Two MMA orientations share that stage layout:
//   small batches (BN = 16..64): the weights are the 128-row A operand and the
//       few token rows the N; two MMAs per k-step, D0 = W0 X^T and D1 = W1 X^T
//       (an expert sees few tokens, so the weights fill the 128-row side);
//   large batches (BN = 128, "token rows as M", selected with
//       SGL_MOE_FFN=tokens_m): X is the 128-row A operand and W0 and W1,
//       adjacent in shared memory, form one 256-row B operand; one M = 128,
//       N = 256 MMA per k-step writes gate | up (or the two Wd halves) side by
//       side. The even and odd k-steps go to two partial accumulators (all 512
//       TMEM columns, one buffer) that the epilogue adds: an MMA waits for the
//       previous one into the same accumulator, so two chains issue faster
//       than one. Each epilogue thread owns one token row and stores whole
//       32-byte runs of h and y_slot.
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
// MXFP4 routed weights: warps 15..22 expand the packed codes of the stage's
// two weight tiles into bf16 (one weight row per thread); warp 23 loads the
// packed code tiles by TMA into a staging ring of their own
constexpr int kExpWarp0 = kSchedWarp + 1;
constexpr int kExpWarps = 8;
constexpr int kCodeWarp = kExpWarp0 + kExpWarps;
constexpr int kFfnThreadsF4 = 32 * (kCodeWarp + 1);
constexpr int kExpDepth = 2;       // k-blocks of scale bytes an expander holds in registers ahead
constexpr int kCodeTile = 128 * 32;  // one weight tile's codes of one k-block (128 rows x 32 bytes)
constexpr int kQueue = 4;                 // item queue entries
constexpr int kLead = 4;                  // claim the next item this many k-blocks early
constexpr long long kProgStride = 1024;   // producer progress = n * stride + k-blocks issued
constexpr int kSmemLimit = 227 * 1024;    // dynamic shared memory of one CTA
constexpr int kMaxStages = 8;             // full / empty barriers in the control block

template <int BN, bool TM = false, bool F4 = false>
struct Cfg {
  static constexpr int A_BYTES = kTileN * 128;  // 128 rows x 64 bf16
  static constexpr int B_BYTES = BN * 128;      // BN rows x 64 bf16
  static constexpr int STAGE_BYTES = 2 * A_BYTES + B_BYTES;
  // MXFP4: a ring of packed-code slots (two code tiles each) ahead of the
  // bf16 stages, which the expanders fill from shared memory and so need
  // less depth
  static constexpr int STG = F4 ? 6 : 0;
  static constexpr int STG_BYTES = 2 * kCodeTile;
  static constexpr int CTRL_BYTES = 512;        // barriers, queue, flags
  // everything but the stages: alignment slack, control block, row metadata,
  // the epilogue warps' store tiles, and the per-slot item starts and row
  // offsets of the largest E, (3E + 5) ints (added at launch for the real E)
  static constexpr int FIXED_BYTES =
      1024 + CTRL_BYTES + BN * 8 + kEpiWarps * kEpiTileWords * 4;
  static constexpr int STAGES_RAW =
      (kSmemLimit - STG * STG_BYTES - FIXED_BYTES - (3 * kMaxExpertsCfg + 5) * 4) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > kMaxStages ? kMaxStages : STAGES_RAW;
  // weights as M: two fp32 accumulators (gate | up, or the two Wd halves) of
  // BN columns side by side; token rows as M: two partial sums of 256
  // columns each (even and odd k-steps: two independent MMA chains)
  static constexpr int ACC_COLS = TM ? 4 * kTileN : 2 * BN;
  // accumulator buffers: two (the epilogue of one item overlaps the MMAs of
  // the next) while they fit the 512 TMEM columns, else one
  static constexpr int NACC = 2 * ACC_COLS <= 512 ? 2 : 1;
  static constexpr int TMEM_COLS = NACC * ACC_COLS < 32 ? 32 : NACC * ACC_COLS;
  static constexpr int H_BOX = BN < 64 ? BN : 64;  // rows per TMA box of h
  static_assert((TMEM_COLS & (TMEM_COLS - 1)) == 0 && TMEM_COLS <= 512, "TMEM allocation");
  // + the per-slot item starts and row offsets, (3E + 5) ints, added at launch
  static constexpr int SMEM = STAGES * STAGE_BYTES + STG * STG_BYTES + FIXED_BYTES;
  static_assert(8 * (2 * 8 + 2 * 2 + 2 * kQueue + 2 * 8) + 8 + 4 * (2 + kQueue) <= CTRL_BYTES,
                "control block");
  static_assert(STG <= 8 && STAGES >= 2, "rings");
  static_assert(SMEM + (3 * kMaxExpertsCfg + 5) * 4 <= kSmemLimit, "shared memory");
};

// ---------------------------------------------------------------------------
// MXFP4 -> bf16 in shared memory. A weight is code * 2^(s - 127) with an e2m1
// code (sign bit 3, magnitude index m = bits 0-2 into {0, .5, 1, 1.5, 2, 3, 4,
// 6}) and the e8m0 scale byte s of its 32-element block; every such value
// has at most two significant bits, so bf16 holds it exactly. For
// 2 <= s <= 252 the bf16 of magnitude m is normal, with exponent field
// s - 1 + {0, 0, 1, 1, 2, 2, 3, 3}[m] (for m >= 1) and mantissa 0x40 for
// m = 3, 5, 7: two byte tables (high and low bytes of the eight bf16 values)
// built once per scale feed byte permutes that expand four codes at a time.
// Other scales take an fp32 multiply per element (also exact).
// ---------------------------------------------------------------------------
struct F4Tables {
  uint32_t h0, h1, l0, l1;  // high / low bytes of the bf16 of magnitudes 0-3 and 4-7
};

__device__ __forceinline__ F4Tables f4_tables(uint32_t s) {
  const uint32_t brep = (s - 1u) * 0x01010101u;    // exponent field of 0.5 * 2^(s - 127)
  const uint32_t ev0 = brep + 0x01010000u;         // magnitudes 0..3: +0 (unused), +0, +1, +1
  const uint32_t ev1 = brep + 0x03030202u;         // magnitudes 4..7: +2, +2, +3, +3
  F4Tables t;
  t.h0 = (ev0 >> 1) & 0x7F7F7F00u;                 // magnitude 0 -> 0
  t.h1 = (ev1 >> 1) & 0x7F7F7F7Fu;
  t.l0 = ((ev0 << 7) & 0x80808000u) | 0x40000000u; // 1.5: mantissa 0x40
  t.l1 = ((ev1 << 7) & 0x80808080u) | 0x40004000u; // 3 and 6: mantissa 0x40
  return t;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// 8 codes (one 32-bit word, element 2j in the low nibble of byte j) -> 8 bf16
// (16 bytes, element order) with the tables of their scale.
__device__ __forceinline__ uint4 f4_expand8(uint32_t w, const F4Tables& t) {
  uint32_t out[4];
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const uint32_t ws = half ? (w >> 16) : w;
    const uint32_t sel = ws & 0x7777u;                   // four magnitude indices
    uint32_t hb = __byte_perm(t.h0, t.h1, sel);
    const uint32_t lb = __byte_perm(t.l0, t.l1, sel);
    // prmt's sign-replicate mode: bytes of negative codes (selector bit 3)
    // come out 0xFF, the others 0x80; bit 0 moved to bit 7 is the sign
    const uint32_t sg = prmt(0x80808080u, 0x80808080u, ws & 0xFFFFu);
    hb |= (sg << 7) & 0x80808080u;
    out[2 * half] = __byte_perm(lb, hb, 0x5140);        // elements 4 half + 0, + 1
    out[2 * half + 1] = __byte_perm(lb, hb, 0x7362);    // elements 4 half + 2, + 3
  }
  return make_uint4(out[0], out[1], out[2], out[3]);
}

// The same 8 codes at any scale byte, through fp32 (exact: s == 0 is the
// subnormal 2^-127, s == 255 gives NaN).
__device__ __forceinline__ uint4 f4_expand8_exact(uint32_t w, uint32_t s) {
  const float scale = s == 255u ? __uint_as_float(0x7FC00000u)
                      : s == 0u ? __uint_as_float(0x00400000u)
                                : __uint_as_float(s << 23);
  uint32_t out[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t h[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const uint32_t c = (w >> (8 * i + 4 * k)) & 0xFu, m = c & 7u;
      const uint32_t mb = m == 0u ? 0u
                          : m == 1u ? (126u << 23)
                                    : (((m >> 1) + 126u) << 23) | ((m & 1u) << 22);
      float v = __uint_as_float(mb) * scale;
      if (c & 8u) v = -v;
      h[k] = f2bf(v);
    }
    out[i] = h[0] | (h[1] << 16);
  }
  return make_uint4(out[0], out[1], out[2], out[3]);
}

// One weight row's k-block of 64 elements (32 bytes of codes, scales s0 for
// elements 0-31 and s1 for 32-63) into the 128-byte swizzled smem row `row`
// of a tile at `tile` (chunk c of row r at c ^ (r % 8)).
__device__ __forceinline__ void f4_store_row(uint8_t* tile, int row, const uint4& c0, const uint4& c1,
                                             uint32_t s0, uint32_t s1) {
  uint8_t* dst = tile + row * 128;
  const int sw = row & 7;
  const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
  if (s0 >= 2u && s0 <= 252u && s1 >= 2u && s1 <= 252u) {
    const F4Tables t0 = f4_tables(s0), t1 = f4_tables(s1);
#pragma unroll
    for (int c = 0; c < 8; ++c)
      *reinterpret_cast<uint4*>(dst + ((c ^ sw) << 4)) = f4_expand8(words[c], c < 4 ? t0 : t1);
  } else {
#pragma unroll
    for (int c = 0; c < 8; ++c)
      *reinterpret_cast<uint4*>(dst + ((c ^ sw) << 4)) = f4_expand8_exact(words[c], c < 4 ? s0 : s1);
  }
}

template <int BN, bool TM, bool F4>
__global__ void __launch_bounds__(F4 ? kFfnThreadsF4 : kFfnThreads, 1)
    moe_ffn(const __grid_constant__ FfnParams p, const __grid_constant__ CUtensorMap tWg,
            const __grid_constant__ CUtensorMap tWu, const __grid_constant__ CUtensorMap tWgS,
            const __grid_constant__ CUtensorMap tWuS, const __grid_constant__ CUtensorMap tWd,
            const __grid_constant__ CUtensorMap tWdS, const __grid_constant__ CUtensorMap tH,
            const __grid_constant__ CUtensorMap tHs) {
  using C = Cfg<BN, TM, F4>;
  static_assert(!TM || BN == kTileN, "token rows as M: tiles of 128 rows");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* stg = smem + C::STAGES * C::STAGE_BYTES;  // MXFP4 code slots
  uint8_t* ctrl = stg + C::STG * C::STG_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(ctrl);
  uint64_t* empty = full + 8;
  uint64_t* tfull = empty + 8;
  uint64_t* tempty = tfull + 2;
  uint64_t* qfull = tempty + 2;
  uint64_t* qempty = qfull + kQueue;
  uint64_t* sfull = qempty + kQueue;   // code slot loaded
  uint64_t* sempty = sfull + 8;        // code slot expanded
  volatile long long* prog = reinterpret_cast<volatile long long*>(sempty + 8);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(const_cast<long long*>(prog) + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* qitem = abort_flag + 1;  // [kQueue]
  int* meta_j = reinterpret_cast<int*>(ctrl + C::CTRL_BYTES);
  float* meta_w = reinterpret_cast<float*>(meta_j + BN);
  uint32_t* epi_tile = reinterpret_cast<uint32_t*>(meta_w + BN);       // [warps][kEpiTileWords]
  int* s_gu = reinterpret_cast<int*>(epi_tile + kEpiWarps * kEpiTileWords);  // [E+2]
  int* s_dn = s_gu + (p.E + 2);                      // [E+2]
  int* s_off = s_dn + (p.E + 2);                     // [E+1]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_trigger();
  if (tid == 0) {
    for (int s = 0; s < kMaxStages; ++s) {  // the adaptive kernel may use more than C::STAGES
      // weight / h TMA + one arrival per gatherer thread (+ one per expander warp)
      mbar_init(&full[s], 1 + 32 * kGatherWarps + (F4 ? kExpWarps : 0));
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], kEpiWarps);
    }
    for (int q = 0; q < kQueue; ++q) {
      mbar_init(&qfull[q], 1);
      // producer, MMA, epilogue, gatherers (and expanders, code loader)
      mbar_init(&qempty[q], 1 + 1 + kEpiWarps + kGatherWarps + (F4 ? kExpWarps + 1 : 0));
    }
    for (int s = 0; s < C::STG; ++s) {
      mbar_init(&sfull[s], 1);
      mbar_init(&sempty[s], kExpWarps);
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
  // Token tile and stage geometry. Fixed for every instantiation but the
  // adaptive one (256-row tiles, weights as M, bf16 weights), which picks
  // 128 or 256 from the expert loads and, at 128, splits the same stage ring
  // into 128-row stages and double-buffers the accumulators. (The MXFP4 form
  // keeps 256: with its code ring only two stages fit, and the runtime
  // geometry measured 6 % slower there than the fixed one.)
  constexpr bool kAdaptive = BN == 256 && !TM && !F4;
  int bn = BN;
  int n_gu_all, n_dn_all;
  if (kAdaptive || p.sched_counts) {
    __shared__ int wsum[33];
    if (kAdaptive) bn = adaptive_bn(p, wsum);
    derive_schedule(p, bn, s_gu, s_dn, s_off, wsum, &n_gu_all, &n_dn_all);
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
  const bool split = kAdaptive && bn < BN;
  const int stage_bytes = split ? 2 * C::A_BYTES + kTileN * 128 : C::STAGE_BYTES;
  const int nstages = split ? C::STAGES * C::STAGE_BYTES / stage_bytes : C::STAGES;
  const int acc_cols = split ? 2 * kTileN : C::ACC_COLS;
  const int nacc = split ? 2 : C::NACC;
  const int nslots = p.E + (p.has_shared ? 1 : 0);
  const int n_gu = min(n_gu_all, p.max_gu);
  const int n_dn = min(n_dn_all, p.max_dn);
  const int n_all = n_gu + n_dn;
  auto item_at = [&](int i, bool& gu) {
    gu = i < n_gu;
    return gu ? decode_item(i, s_gu, s_off, nslots, p.E, p.T, bn)
              : decode_item(i - n_gu, s_dn, s_off, nslots, p.E, p.T, bn);
  };
  const int KB_gu = p.H / 64, KB_dn_r = p.I / 64, KB_dn_s = p.Is / 64;
  auto nkb_of = [&](bool gu, bool sh) { return gu ? KB_gu : (sh ? KB_dn_s : KB_dn_r); };
  // a down item's second 128-row half exists unless it starts past H
  auto two_halves = [&](const WorkItem& it, bool gu) {
    return gu || it.ntile * kDownTile + kTileN < p.H;
  };
  auto mma_n = [&](const WorkItem& it) { return (min(it.nrows, bn) + 15) & ~15; };
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
          if (item_ok(p, it, gu, bn)) {
            const bool sh = it.e == p.E;
            prev_nkb = nkb_of(gu, sh);
            if (!gu) {
              // every gate/up output tile of this (slot, row tile) must be in h
              const int r0 = sh ? 0 : s_off[it.e];
              const int ridx = s_gu[it.e] + (it.row0 - r0) / bn;
              if (!wait_count(p.ready + ridx, cdiv_dev(sh ? p.Is : p.I, kTileN) + p.ready_extra,
                              abort_flag, p.err, p.wait_limit))
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
        if (!item_ok(p, it, gu, bn)) continue;
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
        // MXFP4 routed weights are expanded into the stage by the expander warps
        const bool wtma = !F4 || sh;
        const uint32_t bytes = (wtma ? (two ? 2 : 1) * C::A_BYTES : 0) + nhbox * C::H_BOX * 128;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) {
            live = false;
            break;
          }
          uint8_t* sA = smem + stage * stage_bytes;
          mbar_arrive_expect_tx(&full[stage], bytes);
          if (wtma) {
            tma_load_2d(sA, mA0, &full[stage], kb * 64, arow0, pol_w);
            if (two) tma_load_2d(sA + C::A_BYTES, mA1, &full[stage], kb * 64, arow1, pol_w);
          }
          for (int hb = 0; hb < nhbox; ++hb)
            tma_load_2d(sA + 2 * C::A_BYTES + hb * C::H_BOX * 128, sh ? &tHs : &tH, &full[stage],
                        kb * 64, it.row0 + hb * C::H_BOX, pol_h);
          *prog = n * kProgStride + kb + 1;
          if (++stage == nstages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // every stage must be released by its MMA commit before teardown
      for (int i = 0; i < nstages && live; ++i) {
        if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) break;
        if (++stage == nstages) {
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
        if (!item_ok(p, it, gu, bn)) continue;
        const int nkb = nkb_of(gu, it.e == p.E);
        const bool two = two_halves(it, gu);
        // weights as M: MMA N = the item's rows rounded up to 16 (the B rows past
        // it are never read); token rows as M: M = 128 whatever the rows (the
        // accumulator lanes past them are never read), N = both weight tiles
        const uint32_t idesc =
            TM ? idesc_bf16(kTileN, two ? 2 * kTileN : kTileN) : idesc_bf16(kTileN, mma_n(it));
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + acc * acc_cols;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) {
            live = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + stage * stage_bytes);
          const uint32_t b0 = a0 + 2 * C::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bd = sdesc_k128(b0 + kk * 32);
            const uint32_t accum = (kb | kk) != 0 ? 1u : 0u;
            if constexpr (TM) {
              // A = the 128 token rows, B = W0 then W1 (256 rows, contiguous);
              // even k-steps into the first partial sum, odd ones into the
              // second, so consecutive MMAs do not wait on each other
              umma_bf16(d0 + (kk & 1) * (2 * kTileN), bd, sdesc_k128(a0 + kk * 32), idesc,
                        (kb | (kk >> 1)) != 0 ? 1u : 0u);
            } else {
              umma_bf16(d0, sdesc_k128(a0 + kk * 32), bd, idesc, accum);
              if (two) umma_bf16(d0 + bn, sdesc_k128(a0 + C::A_BYTES + kk * 32), bd, idesc, accum);
            }
          }
          umma_commit(&empty[stage]);
          if (++stage == nstages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!live) break;
        umma_commit(&tfull[acc]);
        if (++acc == nacc) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
    }
    __syncwarp();
  } else if (F4 && warp == kCodeWarp) {
    // ------------------------------------------------------------ MXFP4 code loader
    // Routed items: per k-block one TMA box of 128 rows x 32 bytes per weight
    // tile into the next code slot, as far ahead of the expanders as the
    // ring allows (across items). Shared-expert items use no slot.
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();
      int slot = 0;
      uint32_t sphase = 0;
      bool live = true;
      for (int n = 0; live; ++n) {
        int item;
        if (!next_item(n, item, false)) break;
        bool gu;
        const WorkItem it = item_at(item, gu);
        if (!item_ok(p, it, gu, bn) || it.e == p.E) continue;
        const bool two = two_halves(it, gu);
        const int nkb = nkb_of(gu, false);
        const CUtensorMap* m0 = gu ? &tWg : &tWd;  // the code maps of this kernel
        const CUtensorMap* m1 = gu ? &tWu : &tWd;
        const int row0 = gu ? it.e * p.I + it.ntile * kTileN : it.e * p.H + it.ntile * kDownTile;
        const int row1 = gu ? row0 : row0 + kTileN;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&sempty[slot], sphase ^ 1, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) {
            live = false;
            break;
          }
          uint8_t* dst = stg + slot * C::STG_BYTES;
          mbar_arrive_expect_tx(&sfull[slot], (two ? 2 : 1) * kCodeTile);
          tma_load_2d(dst, m0, &sfull[slot], kb * 32, row0, pol_w);
          if (two) tma_load_2d(dst + kCodeTile, m1, &sfull[slot], kb * 32, row1, pol_w);
          if (++slot == C::STG) {
            slot = 0;
            sphase ^= 1;
          }
        }
      }
      // every slot must have been consumed before teardown
      for (int i = 0; i < C::STG && live; ++i) {
        if (!mbar_wait(&sempty[slot], sphase ^ 1, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) break;
        if (++slot == C::STG) {
          slot = 0;
          sphase ^= 1;
        }
      }
    }
    __syncwarp();
  } else if (F4 && warp >= kExpWarp0) {
    // ------------------------------------------------------------ MXFP4 expanders
    // Routed items: thread x (0..255) owns row x of the stage's 256 weight
    // rows (W0 = rows 0-127, W1 = 128-255). Per k-block it waits for the code
    // slot and for the stage, reads its row's 32 bytes of codes from the
    // slot, takes the 2 scale bytes it loaded kExpDepth k-blocks ahead, and
    // writes the 64 bf16 into the swizzled tile; each warp then fences its
    // writes for the tensor cores and arrives once on the stage's full
    // barrier and on the slot's empty barrier. Shared-expert items (bf16, by
    // TMA) only keep the stage sequence and the arrivals.
    const int x = tid - kExpWarp0 * 32;
    const int half = x >> 7, r = x & (kTileN - 1);
    int stage = 0, slot = 0;
    uint32_t phase = 0, sphase = 0;
    bool live = true;
    for (int n = 0; live; ++n) {
      int item;
      if (!next_item(n, item, true)) break;
      bool gu;
      const WorkItem it = item_at(item, gu);
      if (!item_ok(p, it, gu, bn)) continue;
      const bool sh = it.e == p.E;
      const bool two = two_halves(it, gu);
      const int nkb = nkb_of(gu, sh);
      // this thread's weight row: its scale bytes (rows past the last expert
      // arrive as zero codes from the TMA; their scale is irrelevant)
      const uint8_t* srow = nullptr;
      if (!sh && (half == 0 || two)) {
        const long long nrows_all = static_cast<long long>(p.E) * (gu ? p.I : p.H);
        const long long grow = gu ? static_cast<long long>(it.e) * p.I + it.ntile * kTileN + r
                                  : static_cast<long long>(it.e) * p.H + it.ntile * kDownTile + half * kTileN + r;
        if (grow < nrows_all) srow = (gu ? (half ? p.s_u : p.s_g) : p.s_d) + grow * ((gu ? p.H : p.I) / 32);
      }
      uint32_t sc[kExpDepth];
      auto fetch = [&](int kb, int d) {
        sc[d] = (srow != nullptr && kb < nkb) ? __ldg(reinterpret_cast<const uint16_t*>(srow + kb * 2)) : 0u;
      };
#pragma unroll
      for (int d = 0; d < kExpDepth; ++d) fetch(d, d);
      // k-blocks in groups of kExpDepth, so the register slots are static
      for (int kb0 = 0; kb0 < nkb && live; kb0 += kExpDepth) {
#pragma unroll
        for (int d = 0; d < kExpDepth; ++d) {
          const int kb = kb0 + d;
          if (kb >= nkb) break;
          if (!sh && !mbar_wait(&sfull[slot], sphase, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) {
            live = false;
            break;
          }
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) {
            live = false;
            break;
          }
          if (!sh && (half == 0 || two)) {
            const uint4* src = reinterpret_cast<const uint4*>(stg + slot * C::STG_BYTES + half * kCodeTile + r * 32);
            f4_store_row(smem + stage * stage_bytes + half * C::A_BYTES, r, src[0], src[1], sc[d] & 0xFFu,
                         sc[d] >> 8);
          }
          fetch(kb + kExpDepth, d);
          fence_proxy_async_smem();  // generic-proxy writes before the tensor cores read them
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&full[stage]);
            if (!sh) mbar_arrive(&sempty[slot]);
          }
          if (++stage == nstages) {
            stage = 0;
            phase ^= 1;
          }
          if (!sh && ++slot == C::STG) {
            slot = 0;
            sphase ^= 1;
          }
        }
      }
    }
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
      if (!item_ok(p, it, gu, bn)) continue;
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
          uint8_t* sB = smem + stage * stage_bytes + 2 * C::A_BYTES;
#pragma unroll
          for (int i = 0; i < kRowsPerThread; ++i) {
            const int r = rbase + 16 * i;
            if (r < nb) cp_async16(sB + r * 128 + ((chunk ^ (r & 7)) << 4), src[i] + kb * 64, pol_x);
          }
        }
        cp_async_mbar_arrive_noinc(&full[stage]);
        if (++stage == nstages) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    cp_async_wait_all();  // nothing may still be landing in shared memory at exit
  } else if constexpr (TM) {
    // ------------------------------------------------------------ epilogue, token rows as M
    // Accumulator lane = token row of the tile, column = output feature, as
    // two partial sums [0, 256) and [256, 512): gate/up items hold gate in
    // columns [0, 128) and up in [128, 256) of each; down items the tile's
    // 256 hidden features. The thread of lane r of quarter q
    // owns row 32q + r; of the quarter's two warps, one takes the first half
    // of the columns and one the second.
    const int q = warp & 3;
    const int et = tid - 2 * 32;       // epilogue thread 0..255
    const int cpart = et >> 7;         // column half of this warp
    const int r = q * 32 + lane;       // token row of the tile owned by this thread
    constexpr int kEpiThreads = 32 * kEpiWarps;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int n = 0;; ++n) {
      int item;
      if (!next_item(n, item, true)) break;
      bool gu;
      const WorkItem it = item_at(item, gu);
      if (!item_ok(p, it, gu, bn)) continue;
      const bool sh = it.e == p.E;
      const bool live = r < it.nrows;
      // down items: the row's flat slot and routing weight, read while the
      // item's MMAs run
      int j = -1;
      float wt = 0.f;
      if (!gu && live) {
        const int row = it.row0 + r;
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
      if (!mbar_wait(&tfull[acc], acc_phase, abort_flag, p.err, MOE_DEVERR_TIMEOUT)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * acc_cols;
      if (gu) {
        const int ncols = sh ? p.Is : p.I;
        const float L = sh ? p.lim_s : p.lim_r;
        const int f0 = it.ntile * kTileN;
        uint16_t* hrow = (sh ? p.h_s : p.h_r) + static_cast<size_t>(it.row0 + r) * ncols + f0;
        // 64 features per warp, 16 per TMEM wait; a 16-feature run of h is 32 bytes
#pragma unroll 1
        for (int c0 = 64 * cpart; c0 < 64 * cpart + 64; c0 += 16) {
          float gv[16], uv[16], t1[16];
          tmem_ld16(taddr + c0, gv);               // gate, even k-steps
          tmem_ld16(taddr + 2 * kTileN + c0, t1);  // gate, odd k-steps
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 16; ++c) gv[c] += t1[c];
          tmem_ld16(taddr + kTileN + c0, uv);      // up, even
          tmem_ld16(taddr + 3 * kTileN + c0, t1);  // up, odd
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 16; ++c) uv[c] += t1[c];
          if (live && f0 + c0 < ncols) {
            uint32_t pk[8];
#pragma unroll
            for (int c = 0; c < 8; ++c)
              pk[c] = static_cast<uint32_t>(f2bf(swiglu(gv[2 * c], uv[2 * c], L))) |
                      (static_cast<uint32_t>(f2bf(swiglu(gv[2 * c + 1], uv[2 * c + 1], L))) << 16);
            uint4* dst = reinterpret_cast<uint4*>(hrow + c0);
            dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          }
        }
      } else {
        // 128 hidden features per warp (a half of the tile), 16 per TMEM wait
        const int f0 = it.ntile * kDownTile + cpart * kTileN;
        const bool ok = j >= 0 && f0 < p.H;
        float* yrow = p.y_slot + static_cast<size_t>(ok ? j : 0) * p.H + f0;
#pragma unroll 1
        for (int c0 = 0; c0 < kTileN; c0 += 16) {
          float ov[16], o1[16];
          tmem_ld16(taddr + cpart * kTileN + c0, ov);               // even k-steps
          tmem_ld16(taddr + 2 * kTileN + cpart * kTileN + c0, o1);  // odd k-steps
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 16; ++c) ov[c] += o1[c];
          if (ok) {
            float4* dst = reinterpret_cast<float4*>(yrow + c0);
#pragma unroll
            for (int c = 0; c < 4; ++c)
              dst[c] = make_float4(wt * ov[4 * c], wt * ov[4 * c + 1], wt * ov[4 * c + 2],
                                   wt * ov[4 * c + 3]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (++acc == nacc) {
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
          atomicAdd(p.ready + s_gu[it.e] + (it.row0 - r0) / bn, 1);
        }
      }
    }
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
      if (!item_ok(p, it, gu, bn)) continue;
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
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * acc_cols;
      uint32_t* tile = epi_tile + (warp - 2) * kEpiTileWords;
      if (gu) {
        const int fbase = it.ntile * kTileN + q * 32;  // this warp's 32 features
        const int ncols = sh ? p.Is : p.I;
        const bool ok = fbase < ncols;  // I and Is are multiples of 64: whole warps
        const float L = sh ? p.lim_s : p.lim_r;
        uint16_t* hout = sh ? p.h_s : p.h_r;
        const int ncol = mma_n(it);
        // the two warps of a lane quarter take alternate 16-column chunks
#pragma unroll 1
        for (int c0 = 16 * cpart; c0 < ncol && ok; c0 += 32) {
          float gv[16], uv[16];
          tmem_ld16(taddr + c0, gv);
          tmem_ld16(taddr + bn + c0, uv);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 16; ++c) gv[c] = swiglu(gv[c], uv[c], L);
          store_h16(gv, tile, hout, ncols, it.row0 + c0, it.nrows - c0, fbase, lane);
        }
      } else {
        const int ncol = mma_n(it);
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
          const int fbase = it.ntile * kDownTile + half * kTileN + q * 32;  // this warp's features
          const bool ok = fbase < p.H;  // H is a multiple of 64: whole warps
          // kCols columns per TMEM wait (the loads of one group are in flight
          // together); the two warps of a lane quarter take alternate groups
          constexpr int kCols = BN >= 32 ? 32 : 16;
#pragma unroll 1
          for (int c0 = kCols * cpart; c0 < ncol && ok; c0 += 2 * kCols) {
            float ov[kCols];
#pragma unroll
            for (int u = 0; u < kCols; u += 16) tmem_ld16(taddr + half * bn + c0 + u, ov + u);
            tmem_ld_wait();
#pragma unroll
            for (int g8 = 0; g8 < kCols / 8; ++g8) {
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
      if (++acc == nacc) {
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
          atomicAdd(p.ready + s_gu[it.e] + (it.row0 - r0) / bn, 1);
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

template <int BN, bool TM, bool F4>
cudaError_t launch_bn(const GemmArgs& a, cudaStream_t s) {
  using C = Cfg<BN, TM, F4>;
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
  // test hooks (see FfnParams): SGL_MOE_TEST_WAIT_CYCLES, SGL_MOE_TEST_READY_EXTRA
  if (const char* v = getenv("SGL_MOE_TEST_WAIT_CYCLES")) p.wait_limit = strtoll(v, nullptr, 10);
  if (const char* v = getenv("SGL_MOE_TEST_READY_EXTRA")) p.ready_extra = static_cast<int>(strtol(v, nullptr, 10));
  const int T = a.T, TK = a.T * c.K;
  CUtensorMap tWg, tWu, tWgS, tWuS, tWd, tWdS, tH, tHs;
  bool ok = map_bf16(&tH, a.h_r, TK, c.I, C::H_BOX);
  if (F4) {
    // packed routed weights: the code tiles by TMA (maps in the routed weight
    // maps' places), the scales read by the expanders
    p.q_g = static_cast<const uint8_t*>(a.W->Wg);
    p.q_u = static_cast<const uint8_t*>(a.W->Wu);
    p.q_d = static_cast<const uint8_t*>(a.W->Wd);
    p.s_g = a.W->Wg_scale;
    p.s_u = a.W->Wu_scale;
    p.s_d = a.W->Wd_scale;
    ok = ok && map_codes(&tWg, a.W->Wg, static_cast<uint64_t>(c.E) * c.I, c.H / 2) &&
         map_codes(&tWu, a.W->Wu, static_cast<uint64_t>(c.E) * c.I, c.H / 2) &&
         map_codes(&tWd, a.W->Wd, static_cast<uint64_t>(c.E) * c.H, c.I / 2);
  } else {
    ok = ok && map_bf16(&tWg, a.Wg, static_cast<uint64_t>(a.wrows) * c.I, c.H, kTileN) &&
         map_bf16(&tWu, a.Wu, static_cast<uint64_t>(a.wrows) * c.I, c.H, kTileN) &&
         map_bf16(&tWd, a.Wd, static_cast<uint64_t>(a.wrows) * c.H, c.I, kTileN);
  }
  if (p.has_shared) {
    ok = ok && map_bf16(&tWgS, a.W->Wg_s, c.I_shared, c.H, kTileN) &&
         map_bf16(&tWuS, a.W->Wu_s, c.I_shared, c.H, kTileN) &&
         map_bf16(&tWdS, a.W->Wd_s, c.H, c.I_shared, kTileN) &&
         map_bf16(&tHs, a.h_s, T, c.I_shared, C::H_BOX);
  } else if (F4) {  // no bf16 weight at all: any valid map stands in (never read)
    tWgS = tWuS = tWdS = tHs = tH;
  } else {
    tWgS = tWg;
    tWuS = tWu;
    tWdS = tWd;
    tHs = tH;
  }
  if (!ok) return cudaErrorInvalidValue;
  auto kern = moe_ffn<BN, TM, F4>;
  const int smem_max = C::SMEM + (3 * kMaxExpertsCfg + 5) * static_cast<int>(sizeof(int));
  const int smem = C::SMEM + (3 * c.E + 5) * static_cast<int>(sizeof(int));
  cudaError_t e = ensure_dyn_smem(reinterpret_cast<const void*>(kern), smem_max);
  if (e != cudaSuccess) return e;
  // One CTA per SM. Items are claimed only by running CTAs, so a down item
  // only ever waits on gate/up tiles a resident CTA has taken: no
  // co-residency guarantee is needed.
  return launch_pdl(kern, dim3(num_sms()), dim3(F4 ? kFfnThreadsF4 : kFfnThreads), smem, s, p, tWg, tWu,
                    tWgS, tWuS, tWd,
                    tWdS, tH, tHs);
}

}  // namespace

cudaError_t launch_ffn(const GemmArgs& a, cudaStream_t s) {
  if (a.ffn == kFfnPair) return a.bn == kPairTileN ? launch_ffn_pair(a, s) : cudaErrorInvalidValue;
  if (a.ffn != kFfnNarrow) return cudaErrorInvalidValue;
  // the 128-row tiles run with the weights as M unless SGL_MOE_FFN=tokens_m
  const bool tm = ffn_env_is("tokens_m");
  if (a.cfg->wfmt == MOE_W_MXFP4) {  // MXFP4 routed weights expanded in shared memory
    switch (a.bn) {
      case 16: return launch_bn<16, false, true>(a, s);
      case 32: return launch_bn<32, false, true>(a, s);
      case 64: return launch_bn<64, false, true>(a, s);
      case 128: return tm ? launch_bn<128, true, true>(a, s) : launch_bn<128, false, true>(a, s);
      case 256: return launch_bn<256, false, true>(a, s);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (a.bn) {
    case 16: return launch_bn<16, false, false>(a, s);
    case 32: return launch_bn<32, false, false>(a, s);
    case 64: return launch_bn<64, false, false>(a, s);
    case 128: return tm ? launch_bn<128, true, false>(a, s) : launch_bn<128, false, false>(a, s);
    case 256: return launch_bn<256, false, false>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace sgl
