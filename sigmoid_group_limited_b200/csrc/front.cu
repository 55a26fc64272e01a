// front.cu - the decode front of the layer in one launch (batches of up to 64
// tokens): router logits, certified group-limited top-k with the exact
// re-derivation of close calls, permutation and FFN work lists. The separate
// kernels for these stages are latency-bound at this size; one cooperative
// launch with two grid barriers replaces four launches.
//
// Page "Ling-3.0-flash-VL MoE sparse routing" (lqnn.cn/news/282163): sec. 3
// steps 1-3 and sec. 4 (fp32 router, sigmoid scores, bias for selection, 8
// groups keep 4, top-8, weights renormalised and scaled by 2.5); the
// permutation groups each expert's rows (stable counting sort by expert).
//
// Phases (every CTA runs phase 1; barriers are bounded):
//   1. CTA b = 8 * eb + r forms the fp32 partial logits of experts
//      [32 eb, 32 eb + 32) over hidden chunk r (as the cluster kernel of
//      router.cu: router rows and token columns staged in shared memory, lane
//      = token) and writes them to zp[r][t][e].
//   2. CTA t < T adds its token's eight partials in chunk order (the same z as
//      the cluster kernel), then runs the certified selection and, if the
//      token was flagged, its exact re-derivation.
//   3. Permutation: the selecting CTAs count their experts with atomics in
//      phase 2 (order-free); after the second barrier CTA t places its own
//      K slots at offsets[e] + (the number of earlier flat slots with the
//      same expert), the stable counting-sort position, and CTA 0 writes the
//      offsets and, unless the FFN derives them from the counts itself, its
//      work lists (whose ready counters phase 1 zeroed).
// L2 prefetch for the expert FFN that follows: HBM is nearly idle while the
// front runs, so phase 1 asks L2 for the shared expert's weights (known
// before routing), and after the second barrier the CTAs without a token ask
// for the gate and up weights of the lowest-numbered touched experts (the
// FFN's first work items), up to a byte budget.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include "internal.h"
#include "permute_dev.cuh"
#include "ptx.cuh"
#include "router_dev.cuh"

namespace sgl {
namespace {

constexpr int kFrontThreads = 512;
constexpr int kFrontChunks = 8;   // hidden chunks per expert block
constexpr int kFrontExperts = 32;  // experts per block
constexpr int kFrontRed = 8 * 4 * kFrontMaxT;  // floats: the second K half's partials
constexpr int kFrontSmem = kFrontExperts * kMaxChunk * 4 + kFrontMaxT * kXRow * 2 + kFrontRed * 4;

struct FrontParams {
  int T, H, E, n_group, topk_group, K, renorm;
  float scale;
  const uint16_t* x;
  const float* Wr;
  const float* bias;
  float* zp;          // [8][kFrontMaxT][E] partial logits
  float* z;           // [T][E] logits
  int32_t* idx;
  float* w;
  int32_t* unc;
  int32_t* unc_n;
  int32_t* bar;       // grid barrier counter (zero at launch)
  int32_t* err;
  int32_t* counts;
  int32_t* offsets;
  int32_t* perm;
  int32_t* inv_perm;
  SchedArgs sa;
  int n_ready;        // ready counters to zero (the FFN's largest gate/up item count)
  int build_sched;    // 0: the FFN derives its work lists from the counts itself
  // L2 prefetch (null / 0: none): the shared expert's three matrices, and the
  // routed gate and up weights (expert e at e * pf_expert_bytes) of at most
  // pf_experts touched experts
  const uint8_t* pf_shared[3];
  uint32_t pf_shared_bytes;
  const uint8_t* pf_g;
  const uint8_t* pf_u;
  uint32_t pf_expert_bytes;
  int pf_experts;
};

constexpr uint32_t kPrefetchPiece = 16384;  // bytes per bulk L2 prefetch

// Prefetch pieces [first, n) step `stride` of [base, base + bytes) into L2.
__device__ __forceinline__ void prefetch_range(const uint8_t* base, uint32_t bytes, int first, int stride) {
  const int n = static_cast<int>((bytes + kPrefetchPiece - 1) / kPrefetchPiece);
  for (int c = first; c < n; c += stride) {
    const uint32_t at = static_cast<uint32_t>(c) * kPrefetchPiece;
    prefetch_l2_bulk(base + at, min(kPrefetchPiece, bytes - at));
  }
}


template <int NG, int NV>
__global__ void __launch_bounds__(kFrontThreads, 1) decode_front(const __grid_constant__ FrontParams p) {
  pdl_trigger();  // the FFN may start its prologue; it waits for this grid to finish
  extern __shared__ __align__(16) uint8_t fsm[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int T = p.T, H = p.H, E = p.E;
  // ---- phase 1: partial logits
  {
    float* ws = reinterpret_cast<float*>(fsm);                            // [32][kMaxChunk]
    uint16_t* xs = reinterpret_cast<uint16_t*>(ws + kFrontExperts * kMaxChunk);  // [kFrontMaxT][kXRow]
    const int eb = blockIdx.x / kFrontChunks, r = blockIdx.x % kFrontChunks;
    const int e0 = eb * kFrontExperts;
    const int chunk = ((H / 64 + kFrontChunks - 1) / kFrontChunks) * 64;
    const int k0 = r * chunk;
    const int kn = max(0, min(chunk, H - k0));  // a multiple of 64, possibly 0
    const uint64_t pol = policy_evict_first();
    for (int i = tid; i < kFrontExperts * (kMaxChunk / 4); i += blockDim.x) {
      const int row = i / (kMaxChunk / 4), c = 4 * (i % (kMaxChunk / 4));
      float* dst = ws + row * kMaxChunk + c;
      if (c < kn && e0 + row < E)
        cp_async16(dst, p.Wr + static_cast<size_t>(e0 + row) * H + k0 + c, pol);
      else
        *reinterpret_cast<float4*>(dst) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const uint64_t pol_x = policy_evict_last();
    for (int i = tid; i < kFrontMaxT * (kMaxChunk / 8); i += blockDim.x) {
      const int row = i / (kMaxChunk / 8), c = 8 * (i % (kMaxChunk / 8));
      uint16_t* dst = xs + row * kXRow + c;
      if (row < T && c < kn)
        cp_async16(dst, p.x + static_cast<size_t>(row) * H + k0 + c, pol_x);
      else
        *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
    }
    cp_async_commit();
    // the shared expert's weights: piece c of each matrix goes to CTA c % grid
    if (tid < 3 && p.pf_shared[tid])
      prefetch_range(p.pf_shared[tid], p.pf_shared_bytes, blockIdx.x, gridDim.x);
    cp_async_wait<0>();
    __syncthreads();
    // warp w: experts 4 (w % 8) .. +3 over K half w / 8; lane = token, in
    // passes of 32 tokens (token 32 tp + lane)
    constexpr int EW = 4;
    float* red = reinterpret_cast<float*>(xs + kFrontMaxT * kXRow);  // [8 warps][4][kFrontMaxT tokens]
    const int wq = warp & 7, kh = warp >> 3;
    const int nk8 = kn / 8, half = nk8 / 2;  // kn is a multiple of 64: nk8 even
    const int ntp = (T + 31) / 32;
    for (int tp = 0; tp < ntp; ++tp) {
      const int tok = 32 * tp + lane;
      float acc[EW];
#pragma unroll
      for (int q = 0; q < EW; ++q) acc[q] = 0.f;
#pragma unroll 4
      for (int i = kh * half; i < (kh + 1) * half; ++i) {
        const uint4 xv8 = *reinterpret_cast<const uint4*>(xs + tok * kXRow + 8 * i);
        const uint32_t pk[4] = {xv8.x, xv8.y, xv8.z, xv8.w};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float xv0 = __uint_as_float(pk[2 * h] << 16);
          const float xv1 = __uint_as_float(pk[2 * h] & 0xFFFF0000u);
          const float xv2 = __uint_as_float(pk[2 * h + 1] << 16);
          const float xv3 = __uint_as_float(pk[2 * h + 1] & 0xFFFF0000u);
#pragma unroll
          for (int q = 0; q < EW; ++q) {
            const float4 wv = *reinterpret_cast<const float4*>(ws + (wq * EW + q) * kMaxChunk + 8 * i + 4 * h);
            acc[q] = fmaf(xv0, wv.x, acc[q]);
            acc[q] = fmaf(xv1, wv.y, acc[q]);
            acc[q] = fmaf(xv2, wv.z, acc[q]);
            acc[q] = fmaf(xv3, wv.w, acc[q]);
          }
        }
      }
      if (kh == 1) {
#pragma unroll
        for (int q = 0; q < EW; ++q) red[(wq * EW + q) * kFrontMaxT + tok] = acc[q];
      }
      __syncthreads();
      if (kh == 0 && tok < T) {
#pragma unroll
        for (int q = 0; q < EW; ++q) {
          const int e = e0 + wq * EW + q;
          // the two K halves in a fixed order
          if (e < E)
            p.zp[(static_cast<size_t>(r) * kFrontMaxT + tok) * E + e] =
                acc[q] + red[(wq * EW + q) * kFrontMaxT + tok];
        }
      }
    }
  }
  // warm the bias in L2 for the selection (it may have been evicted)
  if (blockIdx.x == 0 && p.bias)
    for (int e = tid * 32; e < E; e += blockDim.x * 32)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(p.bias + e));
  // counts (the selecting CTAs add to them), the FFN's ready counters and its
  // item claim counter start at zero
  if (blockIdx.x == 0 && tid == 0) p.sa.nitems[2] = 0;
  for (int i = blockIdx.x * blockDim.x + tid; i < E + p.n_ready; i += gridDim.x * blockDim.x) {
    if (i < E) p.counts[i] = 0;
    else p.sa.ready[i - E] = 0;
  }
  if (!grid_barrier(p.bar, 1, p.err)) return;
  // ---- phase 2: one CTA per token
  if (static_cast<int>(blockIdx.x) < T) {
    const int t = blockIdx.x;
    // the token's logits (eight partials in chunk order) and the bias, in
    // shared memory for the selection; z also goes to global for a re-derivation
    float* zs = reinterpret_cast<float*>(fsm);   // [E]
    float* bs = zs + kMaxExperts;                // [E]
    float* zr = p.z + static_cast<size_t>(t) * E;
    for (int e = tid; e < E; e += blockDim.x) {
      float sum = 0.f;
#pragma unroll
      for (int q = 0; q < kFrontChunks; ++q) sum += p.zp[(static_cast<size_t>(q) * kFrontMaxT + t) * E + e];
      zs[e] = sum;
      zr[e] = sum;
      bs[e] = p.bias ? p.bias[e] : 0.f;
    }
    __syncthreads();
    const bool flagged = select_token<NG>(t, zs, E, p.n_group, p.topk_group, p.K, p.scale, p.renorm,
                                          bs, p.idx, p.w, kCertifyMargin, p.unc, p.unc_n);
    if (flagged)
      refine_token<NV>(t, H, E, p.n_group, p.topk_group, p.K, p.scale, p.renorm, kCertifyMargin, p.x,
                       p.Wr, p.z, p.bias, p.idx, p.w);
    __syncthreads();  // this token's final idx is written
    if (tid < p.K) {
      const int e = p.idx[static_cast<size_t>(t) * p.K + tid];
      if (e >= 0 && e < E) atomicAdd(p.counts + e, 1);
      else atomicExch(p.err, MOE_DEVERR_EXPERT_ID);
    }
  }
  if (!grid_barrier(p.bar, 2, p.err)) return;
  // ---- phase 3: permutation (CTA t: token t's slots) and work lists (CTA 0)
  if (static_cast<int>(blockIdx.x) < T) {
    int* cnt = reinterpret_cast<int*>(fsm);  // [E + 1]
    int* off = cnt + kMaxE + 1;              // [E + 1]
    int* sidx = off + kMaxE + 1;             // [T * K]
    __shared__ int scratch[33];
    const int TK = T * p.K, t = blockIdx.x;
    for (int e = tid; e < E; e += blockDim.x) cnt[e] = ld_acquire_gpu(p.counts + e);
    for (int j = tid; j < TK; j += blockDim.x) sidx[j] = p.idx[j];
    __syncthreads();
    int total;
    const int e0 = 2 * tid;
    const int v0 = e0 < E ? cnt[e0] : 0, v1 = e0 + 1 < E ? cnt[e0 + 1] : 0;
    const int ex = block_exscan2(v0, v1, scratch, &total);
    if (e0 < E) off[e0] = ex;
    if (e0 + 1 < E) off[e0 + 1] = ex + v0;
    if (tid == 0) off[E] = total;
    __syncthreads();
    // warp k places slot j = t*K + k: its rank among earlier slots of the same expert
    if (warp < p.K) {
      const int j = t * p.K + warp;
      const int e = sidx[j];
      int rank = 0;
      for (int j0 = 0; j0 < j; j0 += 32) {
        const int jj = j0 + lane;
        rank += __popc(__ballot_sync(0xffffffffu, jj < j && sidx[jj] == e));
      }
      if (lane == 0 && e >= 0 && e < E) {
        const int pos = off[e] + rank;
        if (pos < TK) {
          p.perm[pos] = j;
          if (p.inv_perm) p.inv_perm[j] = pos;
        } else {
          atomicExch(p.err, MOE_DEVERR_SCHEDULE);
        }
      }
    }
    if (t == 0) {
      for (int e = tid; e <= E; e += blockDim.x) p.offsets[e] = off[e];
      if (p.build_sched) {
        SchedArgs sa = p.sa;
        sa.ready = nullptr;  // zeroed in phase 1
        build_schedule(sa, cnt, scratch);
      }
    }
  } else if (p.pf_experts > 0) {
    // gate and up weights of the first touched experts, in the FFN's item
    // order (increasing expert id); CTA T + i of the idle ones takes piece c
    // when c % n_idle == i
    __shared__ int pf_list[kSelMaxCand];
    __shared__ int pf_n;
    if (warp == 0) {
      int n = 0;
      for (int e0 = 0; e0 < E && n < p.pf_experts; e0 += 32) {
        const int e = e0 + lane;
        unsigned m = __ballot_sync(0xffffffffu, e < E && ld_acquire_gpu(p.counts + e) > 0);
        while (m && n < p.pf_experts) {
          const int b = __ffs(m) - 1;
          m &= m - 1;
          if (lane == 0) pf_list[n] = e0 + b;
          ++n;
        }
      }
      if (lane == 0) pf_n = n;
    }
    __syncthreads();
    const int n_idle = static_cast<int>(gridDim.x) - T, i = static_cast<int>(blockIdx.x) - T;
    const int per = static_cast<int>((p.pf_expert_bytes + kPrefetchPiece - 1) / kPrefetchPiece);
    for (int c = i + n_idle * tid; c < 2 * pf_n * per; c += n_idle * static_cast<int>(blockDim.x)) {
      const int q = c / per, piece = c - q * per;
      const uint8_t* base = (q & 1 ? p.pf_u : p.pf_g) + static_cast<size_t>(pf_list[q >> 1]) * p.pf_expert_bytes;
      const uint32_t at = static_cast<uint32_t>(piece) * kPrefetchPiece;
      prefetch_l2_bulk(base + at, min(kPrefetchPiece, p.pf_expert_bytes - at));
    }
  }
}

}  // namespace

bool decode_front_ok(const moe_cfg& c, int T) {
  const int per = c.E / c.n_group;
  // phase 2 takes one CTA per token: T <= the grid (32 CTAs for E = 128)
  return T <= kFrontMaxT && T <= kFrontChunks * c.E / kFrontExperts &&
         (c.E == 128 || c.E == 256 || c.E == 512) && (per == 32 || per == 64) &&
         c.n_group <= kSelMaxGroups && c.K + 1 <= kSelMaxCand && c.topk_group * (c.K + 1) <= 64 &&
         c.H <= kRowRegs * 128 && T * c.K <= kPermTile && 2 * kFrontThreads >= c.E + 2;
}

cudaError_t launch_decode_front(const moe_cfg& c, int T, const uint16_t* x, const float* Wr,
                                const float* bias, float* zp, float* z, int32_t* idx, float* w,
                                int32_t* unc, int32_t* unc_n, int32_t* bar, int32_t* err,
                                int32_t* counts, int32_t* offsets, int32_t* perm,
                                int32_t* inv_perm, const WsLayout& L, int32_t* gu_start,
                                int32_t* dn_start, int32_t* ready, int32_t* nitems,
                                const moe_weights* W, bool build_sched, cudaStream_t s) {
  if (!decode_front_ok(c, T)) return cudaErrorInvalidValue;
  FrontParams p;
  memset(&p, 0, sizeof(p));
  p.T = T;
  p.H = c.H;
  p.E = c.E;
  p.n_group = c.n_group;
  p.topk_group = c.topk_group;
  p.K = c.K;
  p.renorm = c.renorm;
  p.scale = c.scale;
  p.x = x;
  p.Wr = Wr;
  p.bias = bias;
  p.zp = zp;
  p.z = z;
  p.idx = idx;
  p.w = w;
  p.unc = unc;
  p.unc_n = unc_n;
  p.bar = bar;
  p.err = err;
  p.counts = counts;
  p.offsets = offsets;
  p.perm = perm;
  p.inv_perm = inv_perm;
  p.sa = make_sched(c, T, L, gu_start, dn_start, ready, nitems);
  p.n_ready = L.max_items_gu;
  p.build_sched = build_sched ? 1 : 0;
  const uint64_t budget = front_prefetch_budget();
  if (W && budget > 0) {
    // bf16 matrices whose sizes (multiples of 64 x 64 elements) keep every
    // piece 16-byte aligned
    const uint64_t shared_bytes = static_cast<uint64_t>(c.I_shared) * c.H * 2;
    if (c.I_shared > 0 && W->Wg_s && W->Wu_s && W->Wd_s && shared_bytes < (1ull << 31)) {
      p.pf_shared[0] = static_cast<const uint8_t*>(W->Wg_s);
      p.pf_shared[1] = static_cast<const uint8_t*>(W->Wu_s);
      p.pf_shared[2] = static_cast<const uint8_t*>(W->Wd_s);
      p.pf_shared_bytes = static_cast<uint32_t>(shared_bytes);
    }
    const uint64_t expert_bytes = static_cast<uint64_t>(c.I) * c.H * 2;
    if (c.wfmt == MOE_W_BF16 && W->Wg && W->Wu && expert_bytes < (1ull << 31)) {
      p.pf_g = static_cast<const uint8_t*>(W->Wg);
      p.pf_u = static_cast<const uint8_t*>(W->Wu);
      p.pf_expert_bytes = static_cast<uint32_t>(expert_bytes);
      const uint64_t n = budget / (2 * expert_bytes);
      p.pf_experts = static_cast<int>(n < kSelMaxCand ? n : kSelMaxCand);
    }
  }
  const int per = c.E / c.n_group;
  void (*kern)(FrontParams) = nullptr;
  const int nv = c.E / 32;
  if (per == 32) kern = nv == 4 ? decode_front<1, 4> : nv == 8 ? decode_front<1, 8> : decode_front<1, 16>;
  else kern = nv == 4 ? decode_front<2, 4> : nv == 8 ? decode_front<2, 8> : decode_front<2, 16>;
  const int smem = kFrontSmem;  // phase 3 needs 2 (kMaxE + 1) + T * K ints, far less
  cudaError_t e = ensure_dyn_smem(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t lc;
  memset(&lc, 0, sizeof(lc));
  lc.gridDim = dim3(kFrontChunks * c.E / kFrontExperts);
  lc.blockDim = dim3(kFrontThreads);
  lc.dynamicSmemBytes = smem;
  lc.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // every CTA resident: the grid barriers end
  attr[0].val.cooperative = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  return cudaLaunchKernelEx(&lc, kern, p);
}

}  // namespace sgl
