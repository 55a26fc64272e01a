// internal.h - host-side declarations shared by the library's translation
// units: workspace layout, GEMM work items and kernel launchers.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "../../include/moe.h"

namespace sgl {

// One expert-FFN work item: expert `e` (e == E: the shared expert), rows
// [row0, row0 + nrows) of that expert's row range, output tile `ntile`
// (kTileN intermediate features for gate/up, kDownTile hidden features for
// down). Rows are positions in the permuted row space for
// routed experts (offsets[e] + m*BN) and token ids for the shared expert.
// Items are not stored: the GEMM kernels decode an item index from the
// per-slot item prefix sums (gu_start / dn_start) and the row offsets.
struct WorkItem {
  int32_t e;
  int32_t row0;
  int32_t nrows;
  int32_t ntile;
};

constexpr int kPermTile = 2048;   // (token, slot) entries per permutation tile
constexpr int kFrontMaxT = 64;    // largest batch of the fused decode front
constexpr int kTileN = 128;       // output features per GEMM tile (MMA M)
constexpr int kDownTile = 256;    // hidden features per down item (two MMA tiles)
constexpr int kPairTileN = 256;   // token tile of the CTA-pair FFN (large batches)
constexpr int kPairGuTile = 256;  // intermediate features per gate/up item of the CTA-pair FFN
// Block-scaled FFN (MOE_W_MXFP4_A8): token tile (MMA N; two double-buffered
// gate/up accumulators of this width and the scale columns fill the 512 TMEM
// columns), intermediate features per gate/up item and hidden features per
// down item (as the bf16 kernel).
constexpr int kMxTileN = 112;
constexpr int kMxGuTile = 128;
constexpr int kMxDnTile = 256;
constexpr int kMaxExpertsCfg = 1024;  // largest E a configuration may have

// The block-scaled weight formats (per-call scale repack, or prepared atoms).
inline bool mx_a8(int wfmt) { return wfmt == MOE_W_MXFP4_A8 || wfmt == MOE_W_MXFP4_A8P; }

// Which expert-FFN kernel a batch runs on.
enum FfnKind {
  kFfnNarrow = 0,  // moe_ffn<BN>: BN <= 128 tokens, 128 gate + 128 up features per item
  kFfnPair = 1,    // moe_ffn_pair: a CTA pair per item (tcgen05 cta_group::2)
  kFfnMx = 2,      // moe_ffn_mx: block-scaled MXFP8 x MXFP4
};

// The expert-FFN kernel for large batches: one CTA per item with 256-token
// tiles (default); the environment variable SGL_MOE_FFN selects 128-token
// tiles ("narrow"), token rows as the MMA's M ("tokens_m", 128-token tiles) or
// a CTA pair per item ("pair"). Read at every call, so the workspace layout
// and the launch always agree.
inline bool ffn_env_is(const char* name) {
  const char* v = getenv("SGL_MOE_FFN");
  return v != nullptr && strcmp(v, name) == 0;
}

// Kernel and token-tile width (MMA N) for a batch: narrow tiles for decode,
// wide ones for prefill. T*K/E is the mean load over all experts. Above 48,
// 256-token tiles: an MMA costs about the same for any N, so the widest tile
// issues the fewest instructions, at the price of single-buffered
// accumulators (two 256-column chains fill TMEM).
inline FfnKind choose_ffn(int T, int K, int E, int* bn) {
  const double avg = static_cast<double>(T) * K / E;
  if (avg <= 12.0) return *bn = 16, kFfnNarrow;
  if (avg <= 24.0) return *bn = 32, kFfnNarrow;
  if (avg <= 48.0) return *bn = 64, kFfnNarrow;
  if (ffn_env_is("pair")) return *bn = kPairTileN, kFfnPair;
  if (ffn_env_is("narrow") || ffn_env_is("tokens_m")) return *bn = 128, kFfnNarrow;
  return *bn = 256, kFfnNarrow;
}

// Output features per gate/up item and per down item of each kernel.
inline void ffn_tiles(int kind, int* gu_ft, int* dn_ft) {
  switch (kind) {
    case kFfnMx: *gu_ft = kMxGuTile, *dn_ft = kMxDnTile; break;
    case kFfnPair: *gu_ft = kPairGuTile, *dn_ft = kDownTile; break;
    default: *gu_ft = kTileN, *dn_ft = kDownTile; break;
  }
}

inline int cdiv(long long a, long long b) { return static_cast<int>((a + b - 1) / b); }
__host__ __device__ inline int cdiv_dev(int a, int b) { return (a + b - 1) / b; }

// Per-call control block at the start of the workspace, zeroed by every
// entry point that routes: [0] device error word, [1] count of tokens whose
// routing is re-derived exactly, [2] grid barrier counter of the fused
// decode front.
constexpr int kCtrlBytes = 256;

struct WsLayout {
  size_t z, unc, tile_hist, idx, w, counts, offsets, perm, inv_perm, gu_start, dn_start, ready, nitems, h_r,
      h_s, y_slot, err, total;
  // block-scaled format with per-call scale repack: touched-expert slots
  size_t slot_of, touched, ntouched;
  // MOE_W_MXFP4_A8 only: MXFP8 x (codes [T,H], scales [T,H/32]); the scales
  // of h (codes reuse h_r) as 512-byte atoms per (row tile, 128-wide k-block);
  // the touched experts' weight scales as atoms per (128-row tile, k-block)
  // of Wg, Wu and Wd
  size_t x_q, x_sf, h_sf, sf_g, sf_u, sf_d;
  int max_row_tiles;
  size_t wr_split;  // router matrix as three bf16 terms (batches above 32 tokens)
  size_t zp;        // partial router logits [8][kFrontMaxT][E] of the fused decode front
  int max_touched;
  int n_ptiles, bn, max_items_gu, max_items_dn;
  int ffn, gu_ft, dn_ft;  // FfnKind and its output features per gate/up and down item
  int adaptive;           // the FFN picks its token tile on the device (see ffn_adaptive)
};

WsLayout ws_layout(const moe_cfg& c, int T);

// The 256-token-tile FFN with bf16 weights picks its token tile (128 or 256)
// from the expert loads on the device and derives its own work lists; its
// workspace is sized for the 128-row tiles (more items).
inline bool ffn_adaptive(const WsLayout& L) { return L.adaptive != 0; }

// Launchers (return cudaGetLastError()).
// Routing. unc [T] / unc_n: scratch list (and its count, zeroed by the
// caller) of tokens whose fp32 decision is re-derived from exact logits.
// wr_split: scratch [3][E][H] bf16 for the router matrix as three bf16 terms
// (tensor-core logits, T > 32); nullptr for smaller batches.
cudaError_t launch_router(const moe_cfg& c, int T, const uint16_t* x, const float* Wr,
                          const float* bias, float* z, int32_t* idx, float* w, int32_t* unc,
                          int32_t* unc_n, int32_t* err, uint16_t* wr_split, cudaStream_t s);

// The decode front in one cooperative launch (T <= kFrontMaxT, see front.cu):
// routing (logits via zp, certified selection, exact re-derivation of close
// calls), then the permutation and the FFN work lists. bar: a zeroed grid
// barrier counter. decode_front_ok: whether a configuration qualifies.
bool decode_front_ok(const moe_cfg& c, int T);
cudaError_t launch_decode_front(const moe_cfg& c, int T, const uint16_t* x, const float* Wr,
                                const float* bias, float* zp, float* z, int32_t* idx, float* w,
                                int32_t* unc, int32_t* unc_n, int32_t* bar, int32_t* err,
                                int32_t* counts, int32_t* offsets, int32_t* perm,
                                int32_t* inv_perm, const WsLayout& L, int32_t* gu_start,
                                int32_t* dn_start, int32_t* ready, int32_t* nitems,
                                const moe_weights* W, bool build_sched, cudaStream_t s);
// Bytes of routed gate / up weights the decode front asks L2 for (about what
// HBM delivers between the routing decision and the FFN's first loads): the
// environment variable SGL_MOE_PREFETCH in MiB, 0 turning every prefetch of
// the front off; 32 MiB when unset.
inline uint64_t front_prefetch_budget() {
  const char* v = getenv("SGL_MOE_PREFETCH");
  if (v == nullptr || *v == 0) return 32ull << 20;
  const long mb = strtol(v, nullptr, 10);
  return mb > 0 ? static_cast<uint64_t>(mb) << 20 : 0;
}

cudaError_t launch_permute(const moe_cfg& c, int T, const int32_t* idx, int32_t* tile_hist,
                           int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv_perm,
                           int32_t* err, const WsLayout& L, int32_t* gu_start, int32_t* dn_start,
                           int32_t* ready, int32_t* nitems, cudaStream_t s);

// Allocation-free permutation (moe_permute_static): scratch in a fixed
// device array; needs T*K <= kStaticMaxSlots and E <= kStaticMaxExperts.
constexpr int kStaticMaxSlots = 65536;
constexpr int kStaticMaxExperts = 1024;
constexpr int kMaxDevices = 64;
cudaError_t launch_permute_static(const moe_cfg& c, int T, const int32_t* idx, int32_t* counts,
                                  int32_t* offsets, int32_t* perm, int32_t* inv_perm,
                                  cudaStream_t s);

cudaError_t launch_schedule(const moe_cfg& c, int T, const int32_t* offsets, const WsLayout& L,
                            int32_t* gu_start, int32_t* dn_start, int32_t* ready,
                            int32_t* nitems, cudaStream_t s);

struct GemmArgs {
  const moe_cfg* cfg;
  int T;
  const uint16_t* x;
  const int32_t* perm;
  const float* w;
  const moe_weights* W;
  const void* Wg;            // routed weights the GEMMs read (bf16), expert- or slot-major
  const void* Wu;
  const void* Wd;
  const int32_t* wslot;      // nullable: row block of expert e is wslot[e] instead of e
  int wrows;                 // row blocks in Wg/Wu/Wd (E, or the slot capacity)
  uint16_t* h_r;
  uint16_t* h_s;
  float* y_slot;
  const int32_t* offsets;   // [E+1] routed row offsets
  const int32_t* gu_start;  // [E+2] item prefix sums, gate/up
  const int32_t* dn_start;  // [E+2] item prefix sums, down
  int32_t* ready;           // [max_items_gu] per (slot, row tile) finished gate/up tiles
  const int32_t* nitems;
  int32_t* err;
  int bn;
  int ffn;  // FfnKind
  // nullable (narrow kernel): the expert counts [E] from which the FFN derives
  // its work lists and row offsets itself, instead of reading gu_start /
  // dn_start / offsets / nitems[0..1]
  const int32_t* sched_counts;
  int max_items_gu;
  int max_items_dn;
  // MOE_W_MXFP4_A8: the MXFP4 codes are a.Wg/Wu/Wd (expert-major), read in place
  const uint8_t* x_q;        // [T, H] e4m3
  const uint8_t* x_sf;       // [T, H/32] e8m0
  uint8_t* h_q;              // [T*K, I] e4m3 (permuted rows)
  uint8_t* h_sf;             // [row tiles][I/128][512] e8m0 atoms
  const uint8_t* sf_g;       // [slot][I/128][H/128][512]
  const uint8_t* sf_u;       // [slot][I/128][H/128][512]
  const uint8_t* sf_d;       // [slot][H/128][I/128][512]
  const int32_t* slot_of;    // [E] touched slot of expert e; nullptr: sf_* indexed by expert
};

// The expert FFN: gate/up and down in one cooperative persistent launch
// (counters in a.ready and a.nitems[2], zeroed by the schedule builder).
cudaError_t launch_ffn(const GemmArgs& a, cudaStream_t s);
// The expert FFN on CTA pairs (token tile kPairTileN).
cudaError_t launch_ffn_pair(const GemmArgs& a, cudaStream_t s);
cudaError_t launch_router_gemm(const moe_cfg& c, int T, const uint16_t* x, const uint16_t* w_hi,
                               const uint16_t* w_mid, const uint16_t* w_lo, float* z,
                               int32_t* err, cudaStream_t s);

// The block-scaled expert FFN (MOE_W_MXFP4_A8): routed items on
// tcgen05.mma kind::mxf8f6f4 (e2m1 weights x e4m3 activations, e8m0 scales),
// shared-expert items on kind::f16, in one persistent launch.
cudaError_t launch_ffn_mx(const GemmArgs& a, cudaStream_t s);
// MOE_W_MXFP4_A8 inputs of that FFN: touched-expert slots, their weight
// scales repacked as atoms (sf_g / sf_u / sf_d) and x quantised to MXFP8.
cudaError_t launch_mx_prep(const moe_cfg& c, int T, const int32_t* offsets, const moe_weights* W,
                           const uint16_t* x, int32_t* slot_of, int32_t* touched,
                           int32_t* ntouched, uint8_t* sf_g, uint8_t* sf_u, uint8_t* sf_d,
                           uint8_t* x_q, uint8_t* x_sf, cudaStream_t s);
// MXFP8 x alone (MOE_W_MXFP4_A8P: the weight scales are prepared atoms).
cudaError_t launch_mx_quant(const moe_cfg& c, int T, const uint16_t* x, uint8_t* x_q, uint8_t* x_sf,
                            cudaStream_t s);
// Every expert's weight scales as atoms (moe_prepare_weights).
cudaError_t launch_mx_sf_atoms(const moe_cfg& c, const moe_weights* W, uint8_t* sf_g, uint8_t* sf_u,
                               uint8_t* sf_d, cudaStream_t s);
// Touched experts of a batch in increasing id order (slot_of[e], -1 if none).
cudaError_t launch_mxfp4_slots(const moe_cfg& c, const int32_t* offsets, int32_t* slot_of,
                               int32_t* touched, int32_t* ntouched, cudaStream_t s);


cudaError_t launch_combine(const moe_cfg& c, int T, const float* y_slot, int with_shared,
                           uint16_t* y, cudaStream_t s);

// Whether launches on this host thread use programmatic dependent launch.
// It pays for small batches, whose kernels are short and latency-bound; on
// large ones the early-resident grids cost more than the launch gaps they
// hide. Set per call by the entry points (PdlScope).
constexpr int kPdlMaxTokens = 256;
inline bool& pdl_enabled() {
  static thread_local bool on = false;
  return on;
}
struct PdlScope {
  bool prev;
  explicit PdlScope(int T) : prev(pdl_enabled()) { pdl_enabled() = T <= kPdlMaxTokens; }
  ~PdlScope() { pdl_enabled() = prev; }
};

// Launches `kern`, with programmatic stream serialization when enabled (see
// pdl_wait in ptx.cuh); returns cudaLaunchKernelEx's status.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
  cudaLaunchConfig_t lc;
  memset(&lc, 0, sizeof(lc));
  lc.gridDim = grid;
  lc.blockDim = block;
  lc.dynamicSmemBytes = smem;
  lc.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&lc, kern, static_cast<Args&&>(args)...);
}

// Routing statistics from expert counts (see moe_route_stats in moe.h).
cudaError_t launch_route_stats(const moe_cfg& c, const int32_t* counts, double* stats,
                               cudaStream_t s);

int num_sms();

// Tensor map of a bf16 row-major [rows, cols] matrix for TMA: box of
// box_rows x 64 columns, 128-byte swizzle. False if it cannot be encoded.
bool map_bf16(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows);
// Row-major [rows, cols] bytes (e4m3 codes): box of box_rows x 128 bytes,
// 128-byte swizzle.
bool map_u8(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows);
// Packed MXFP4 codes as bytes: [rows, row_bytes] uint8, box of 128 rows x 32
// bytes (64 elements: one k-block), no swizzle (rows 32 bytes apart in
// shared memory). Needs row_bytes % 32 == 0 and a 16-byte aligned base.
bool map_codes(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t row_bytes);
// MXFP4 codes [rows, cols/2] (cols 4-bit elements per row, two per byte):
// box of box_rows x 128 elements, unpacked to one byte per element in shared
// memory (16 elements per 16 bytes: 8 code bytes + 8 bytes of gap) with the
// 128-byte swizzle, the operand layout of tcgen05.mma kind::mxf8f6f4.
// Needs a 32-byte aligned base and cols % 128 == 0.
bool map_fp4(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows);

// Raises `func`'s dynamic shared-memory limit to at least `bytes`, once per
// device (later calls with a size already granted cost a table lookup).
cudaError_t ensure_dyn_smem(const void* func, int bytes);

}  // namespace sgl
