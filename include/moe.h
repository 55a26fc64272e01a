/*
 * moe.h - C-ABI of the B200 (sm_100a) sparse-MoE FFN layer library
 *         (libsgl_moe.so).
 *
 * One layer, as described for the Ling-3.0-flash(-VL) models on the page
 * "Ling-3.0-flash-VL MoE sparse routing" (lqnn.cn/news/282163), sections 2-4:
 *   1. fp32 router logits z = x Wr^T (sec. 4, router_dtype fp32),
 *   2. sigmoid scores s = 1/(1+e^-z), independent per expert (sec. 3 step 1),
 *   3. selection bias b = s + bias[e] (sec. 3 step 3),
 *   4. group-limited top-k: n_group groups, keep the topk_group groups with the
 *      highest in-group maximum of b, then the K best experts by b among them
 *      (sec. 3 step 2); ties go to the lower index,
 *   5. combine weights w = scale * s_k / sum_j s_j of the unbiased scores
 *      (sec. 4, norm_topk_prob and routed_scaling_factor),
 *   6. permutation of the T*K (token, slot) pairs by expert,
 *   7. SwiGLU experts h = silu(clamp(g)) * clamp(u), o = h Wd^T with an
 *      optional limit L (sec. 4, SwiGLU limit), y_slot = w * o,
 *   8. one always-on shared expert (sec. 2), unscaled, with its own limit,
 *   9. y[t] = sum_k y_slot[t,k] + y_shared[t].
 * The routed weights may be MXFP4 (page "Ling-3.0-flash-VL 42-layer hybrid
 * backbone", lpnh.cn/news/2815793, spec table: routed experts in 4 bit).
 *
 * Conventions for every call:
 *  - Pointers marked "device" are CUDA device pointers owned by the caller;
 *    the library never allocates on these paths and keeps no global state.
 *    Every device pointer must be 16-byte aligned (MOE_ERR_ALIGN otherwise).
 *  - `stream` is a cudaStream_t (NULL = legacy default stream); every call is
 *    asynchronous on it. A status other than MOE_OK means nothing was
 *    launched (host-side validation) or a launch failed (MOE_ERR_CUDA).
 *  - Kernels that detect bad data (an expert id out of range, a wait that
 *    timed out) set an error word inside the workspace instead of trapping;
 *    read it with moe_read_error(). moe_route, moe_permute and
 *    moe_layer_forward clear the word when they start; moe_grouped_swiglu
 *    and moe_combine only add to it.
 *  - bf16 tensors are raw bfloat16 (uint16) arrays; all matrices are
 *    row-major with the reduction (K) dimension contiguous: Wr [E,H] fp32,
 *    Wg/Wu [E,I,H], Wd [E,H,I], Wg_s/Wu_s [I_s,H], Wd_s [H,I_s].
 *  - Supported shapes: H, I, I_shared multiples of 64; E a multiple of 32
 *    and of n_group, E <= 1024; n_group <= 32; K <= 32 and K <= the
 *    candidate count; 1 <= T <= 1<<20.
 */
#ifndef SGL_MOE_H
#define SGL_MOE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_W_BF16 0   /* routed weights are bf16 */
#define MOE_W_MXFP4 1  /* routed weights are MXFP4 codes + e8m0 scales */
/* Routed weights MXFP4 as above, and the routed experts' activations MXFP8:
 * page "Ling-3.0-flash-VL 42-layer hybrid backbone" (lpnh.cn/news/2815793),
 * spec table, gives the quantisation scheme as FP8 + MXFP4. x is quantised
 * before gate/up and h before down (OCP Microscaling v1.0: e4m3 elements, one
 * e8m0 scale per 32 consecutive elements along the contraction; scale
 * 2^(floor(log2(amax)) - 8), elements rounded to nearest even, saturating at
 * 448), and the routed GEMMs run on block-scaled tensor cores. The shared
 * expert stays bf16. Needs H % 128 == 0 and I % 128 == 0. */
#define MOE_W_MXFP4_A8 2
/* MOE_W_MXFP4_A8 with the three weight-scale arrays already in the block-
 * scaled tensor cores' atom layout, written once by moe_prepare_weights: the
 * forward then skips the per-call repack of the touched experts' scales. The
 * arithmetic is that of MOE_W_MXFP4_A8, bit for bit. */
#define MOE_W_MXFP4_A8P 3

/* Layer configuration; field names follow the model's config keys. */
typedef struct moe_cfg {
  int32_t H;            /* hidden_size (2560) */
  int32_t E;            /* routed experts (512) */
  int32_t n_group;      /* expert groups (8) */
  int32_t topk_group;   /* groups kept per token (4) */
  int32_t K;            /* num_experts_per_tok (8) */
  int32_t I;            /* moe_intermediate_size (768) */
  int32_t I_shared;     /* shared expert intermediate size (768); 0 = no shared expert */
  float scale;          /* routed_scaling_factor (2.5) */
  int32_t renorm;       /* norm_topk_prob (1) */
  float limit_routed;   /* SwiGLU limit of routed experts; <= 0 or inf: off */
  float limit_shared;   /* SwiGLU limit of the shared expert; <= 0 or inf: off */
  int32_t wfmt;         /* MOE_W_BF16, MOE_W_MXFP4, MOE_W_MXFP4_A8 or MOE_W_MXFP4_A8P */
} moe_cfg;

typedef enum moe_status {
  MOE_OK = 0,
  MOE_ERR_CFG = -1,         /* configuration or T outside the supported range */
  MOE_ERR_NULL = -2,        /* a required pointer is NULL */
  MOE_ERR_ALIGN = -3,       /* a device pointer is not 16-byte aligned */
  MOE_ERR_WORKSPACE = -4,   /* workspace NULL or smaller than moe_workspace_size() */
  MOE_ERR_CUDA = -5,        /* a CUDA runtime/driver call or launch failed */
  MOE_ERR_DEVICE = -6,      /* a kernel reported bad data (moe_read_error) */
  MOE_ERR_UNSUPPORTED = -7  /* device is not sm_100 or format not built */
} moe_status;

/* Expert weights. Routed bf16: Wg,Wu [E,I,H], Wd [E,H,I] bf16, scales NULL.
 * Routed MXFP4 (MOE_W_MXFP4 and MOE_W_MXFP4_A8): Wg,Wu [E,I,H/2], Wd [E,H,I/2]
 * uint8 codes (element 2j in the low nibble) and Wg_scale,Wu_scale [E,I,H/32],
 * Wd_scale [E,H,I/32] e8m0; with MOE_W_MXFP4_A8 the codes must be 32-byte
 * aligned. MOE_W_MXFP4_A8P: the same codes, and the scale arrays in the atom
 * layout of moe_prepare_weights (same byte counts).
 * Shared expert (bf16): Wg_s,Wu_s [I_s,H], Wd_s [H,I_s]; all three NULL when
 * cfg->I_shared == 0. All device pointers. */
typedef struct moe_weights {
  const void* Wg;
  const void* Wu;
  const void* Wd;
  const uint8_t* Wg_scale;
  const uint8_t* Wu_scale;
  const uint8_t* Wd_scale;
  const void* Wg_s;
  const void* Wu_s;
  const void* Wd_s;
} moe_weights;

/* Number of stage events moe_layer_forward records when given an array. */
#define MOE_N_STAGE_EVENTS 6

/* Bytes of device workspace the calls below need for T tokens (0 on a bad
 * cfg). One workspace serves every call for the same (cfg, T). */
MOE_API size_t moe_workspace_size(const moe_cfg* cfg, int32_t T);

/* Stages 1-5, routing (page 3 sec. 3 steps 1-3, sec. 4).
 * x [T,H] bf16, Wr [E,H] fp32, bias [E] fp32 (may be NULL = zero bias);
 * out: idx [T,K] int32 (experts in rank order), w [T,K] fp32. All device. */
MOE_API moe_status moe_route(const moe_cfg* cfg, int32_t T, const void* x, const float* Wr,
                     const float* bias, int32_t* idx, float* w, void* ws, size_t ws_bytes,
                     void* stream);

/* Stage 6, permutation (page "Ling-3.0-flash-VL MoE sparse routing", sec. 1:
 * the router picks a few experts for every token, and each expert then works
 * on the tokens routed to it; page at 2kiu.com/news/4837473 on the sparse
 * activation of Ling-3.0-flash-VL, sec. 4: the compute fans out from the
 * router into 8 expert branches per token). The rows routed to each expert
 * are grouped together: a stable counting sort of the flat slots
 * j = t*K + k by expert (order inside an expert = ascending j), deterministic.
 * in: idx [T,K] int32; out: counts [E], offsets [E+1] (exclusive prefix sum),
 * perm [T*K] (sorted position -> slot j), inv_perm [T*K] (slot -> position).
 * inv_perm may be NULL. All device. An id outside [0,E) sets the error word. */
MOE_API moe_status moe_permute(const moe_cfg* cfg, int32_t T, const int32_t* idx, int32_t* counts,
                       int32_t* offsets, int32_t* perm, int32_t* inv_perm, void* ws,
                       size_t ws_bytes, void* stream);

/* moe_permute without a workspace, for callers that cannot allocate device
 * memory: a plugin whose host framework owns all device memory and hands out
 * no workspace, or a real-time loop or embedded runtime that must not
 * allocate once it runs. The pages describe no such call; it exists only for
 * those callers. Same inputs, outputs and results as moe_permute (all device
 * pointers, owned by the caller).
 * Scratch: a fixed array inside the library, 256.25 KiB per device, held by
 * every GPU that loads the library until the process exits. Limits:
 * T*K <= 65536 and E <= 1024, else MOE_ERR_WORKSPACE and nothing runs.
 * The first call in a CUDA context looks the array's address up (once per
 * context, with that context current; a device reset or another context on
 * the device gets a fresh lookup): make that first call before any stream
 * capture. All calls share the array, so calls that overlap on the GPU (other
 * streams, other threads) race: serialise them. Expert ids outside [0,E) are
 * dropped as in moe_permute; there is no error word to read back. Allocates
 * nothing (no cudaMalloc, no cudaFree). */
MOE_API moe_status moe_permute_static(const moe_cfg* cfg, int32_t T, const int32_t* idx,
                                      int32_t* counts, int32_t* offsets, int32_t* perm,
                                      int32_t* inv_perm, void* stream);

/* Stage 7 (and 8 when shared weights are given): grouped SwiGLU experts on
 * tcgen05 tensor cores (page 3 sec. 2 and sec. 4).
 * in: x [T,H] bf16, perm and offsets from moe_permute, w [T,K] fp32;
 * out: y_slot [(T*K + T), H] fp32 where row j = t*K + k holds
 *      w[t,k] * Expert_{idx[t,k]}(x_t) and row T*K + t holds the shared
 *      expert's output for token t (left untouched without shared weights).
 * All device. */
MOE_API moe_status moe_grouped_swiglu(const moe_cfg* cfg, int32_t T, const void* x, const int32_t* perm,
                              const int32_t* offsets, const float* w, const moe_weights* W,
                              void* y_slot, void* ws, size_t ws_bytes, void* stream);

/* Stage 9, weighted combine back to token order (page at
 * 2kiu.com/news/4837473 on the sparse activation of Ling-3.0-flash-VL,
 * sec. 4: the 8 expert branches' outputs are aggregated before the next
 * layer; page "Ling-3.0-flash-VL MoE sparse routing", sec. 2: the shared
 * expert's output is added for every token):
 * y[t] = bf16( (sum over k = 0..K-1 of y_slot[t*K+k]) + y_slot[T*K+t] ),
 * summed in fp32 in slot order; the shared row is added only when
 * with_shared != 0. y_slot (fp32) as produced by moe_grouped_swiglu;
 * y [T,H] bf16, rounded once (nearest even). */
MOE_API moe_status moe_combine(const moe_cfg* cfg, int32_t T, const void* y_slot, int32_t with_shared,
                       void* y, void* stream);

/* The whole layer (stages 1-9) in one call.
 * x [T,H] bf16, Wr [E,H] fp32, bias [E] fp32 (NULL = zero), W weights;
 * out: y [T,H] bf16; optional (NULL allowed) idx_out [T,K], w_out [T,K],
 * counts_out [E]. ws/ws_bytes: workspace. stage_events: NULL, or an array of
 * MOE_N_STAGE_EVENTS cudaEvent_t recorded on `stream` after: start, route,
 * permute, gate/up GEMM, down GEMM, combine. All pointers device except
 * cfg, W, stage_events. */
MOE_API moe_status moe_layer_forward(const moe_cfg* cfg, int32_t T, const void* x, const float* Wr,
                             const float* bias, const moe_weights* W, void* y, int32_t* idx_out,
                             float* w_out, int32_t* counts_out, void* ws, size_t ws_bytes,
                             void* stream, void* const* stage_events);

/* One-time preparation of MXFP4 routed weights for MOE_W_MXFP4_A8P (page
 * "Ling-3.0-flash-VL 42-layer hybrid backbone", spec table: FP8 + MXFP4).
 * cfg->wfmt: MOE_W_MXFP4_A8 or MOE_W_MXFP4_A8P (only the shapes are read);
 * in: W->Wg_scale, Wu_scale [E,I,H/32], Wd_scale [E,H,I/32] e8m0 (device);
 * out (device, caller-owned, the same byte counts as the inputs, 16-byte
 * aligned): Wg_sf, Wu_sf [E][I/128][H/128][512] and Wd_sf [E][H/128][I/128]
 * [512]: the 512-byte atom (expert e, 128-row tile t, 128-wide k-block b)
 * holds the scale of row 128t + r and 32-element chunk 4b + k at byte
 * (r % 32) * 16 + (r / 32) * 4 + k, the layout tcgen05.cp.32x128b.warpx4
 * copies into tensor memory for the block-scaled MMA. Pass the three outputs
 * as the scale pointers of a moe_weights used with MOE_W_MXFP4_A8P.
 * Errors: MOE_ERR_CFG (not a block-scaled format, or H or I not a multiple
 * of 128), MOE_ERR_NULL, MOE_ERR_ALIGN, MOE_ERR_CUDA. Asynchronous on
 * `stream`. */
MOE_API moe_status moe_prepare_weights(const moe_cfg* cfg, const moe_weights* W, uint8_t* Wg_sf,
                                       uint8_t* Wu_sf, uint8_t* Wd_sf, void* stream);

/* Routing statistics from the expert counts that moe_permute and
 * moe_layer_forward produce: the load monitoring of page 1 ("Ling-3.0-flash-VL：
 * 层级化稀疏路由大模型硬核解析", sec. 4.1: routing entropy and experts that are
 * never selected), for the balancing that page 3 sec. 3 step 3 describes.
 * in: counts [E] int32 (device; negative entries count as 0);
 * out: stats [MOE_N_ROUTE_STATS] float64 (device):
 *   [0] entropy H = -sum_e p_e log2 p_e, p_e = counts_e / sum(counts), bits
 *       (0 when the sum is 0)
 *   [1] H / log2(E)  (1 = every expert equally loaded)
 *   [2] max load      [3] mean load = sum / E      [4] max / mean
 *   [5] idle experts (count 0)                      [6] sum of the counts
 * Deterministic (fixed summation order). Asynchronous on `stream`. */
#define MOE_N_ROUTE_STATS 7
MOE_API moe_status moe_route_stats(const moe_cfg* cfg, const int32_t* counts, double* stats,
                                   void* stream);

/* Reads (synchronously, on `stream`) and clears the workspace error word.
 * *code = 0 when no kernel reported a problem; otherwise one of the
 * MOE_DEVERR_* values below. Returns MOE_OK or MOE_ERR_CUDA. */
MOE_API moe_status moe_read_error(const moe_cfg* cfg, int32_t T, void* ws, size_t ws_bytes,
                          void* stream, int32_t* code);

#define MOE_DEVERR_EXPERT_ID 1   /* routing index outside [0, E) */
#define MOE_DEVERR_TIMEOUT 2     /* a pipeline wait in a GEMM kernel gave up */
#define MOE_DEVERR_SCHEDULE 3    /* a GEMM work item was out of range */

/* Human-readable name of a status. Never NULL. */
MOE_API const char* moe_status_string(moe_status s);

/* Library version string. */
MOE_API const char* moe_version(void);

#ifdef __cplusplus
}
#endif
#endif /* SGL_MOE_H */
