// capi.cu - the library's C-ABI (include/moe.h): argument validation,
// workspace layout and the stage sequence of one MoE layer forward.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <map>
#include <mutex>
#include <utility>

#include "internal.h"

namespace sgl {

int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (cache[dev] == 0) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    cache[dev] = v > 0 ? v : 1;
  }
  return cache[dev];
}

cudaError_t ensure_dyn_smem(const void* func, int bytes) {
  static std::mutex mu;
  static std::map<std::pair<int, const void*>, int> granted;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  int& have = granted[std::make_pair(dev, func)];
  if (have >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) have = bytes;
  return e;
}

static size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

WsLayout ws_layout(const moe_cfg& c, int T) {
  WsLayout L;
  memset(&L, 0, sizeof(L));
  const size_t TK = static_cast<size_t>(T) * c.K;
  L.n_ptiles = cdiv(static_cast<long long>(TK), kPermTile);
  const bool mx = mx_a8(c.wfmt);
  if (mx) {
    L.bn = kMxTileN;
    L.ffn = kFfnMx;
  } else {
    L.ffn = choose_ffn(T, c.K, c.E, &L.bn);
    // MXFP4 weights are expanded by the one-CTA kernel
    if (c.wfmt == MOE_W_MXFP4 && L.ffn == kFfnPair) L.ffn = kFfnNarrow, L.bn = 256;
  }
  ffn_tiles(L.ffn, &L.gu_ft, &L.dn_ft);
  L.adaptive = L.ffn == kFfnNarrow && L.bn == 256 && c.wfmt == MOE_W_BF16 ? 1 : 0;
  const int gu_ft = L.gu_ft, dn_ft = L.dn_ft;
  const int rt_gu = cdiv(c.I, gu_ft), st_gu = cdiv(c.I_shared, gu_ft), nt_dn = cdiv(c.H, dn_ft);
  const int bn_items = ffn_adaptive(L) ? kTileN : L.bn;  // the smallest tile the FFN may pick
  const long long mt_r = cdiv(static_cast<long long>(TK), bn_items) +
                         (static_cast<long long>(TK) < c.E ? static_cast<long long>(TK) : c.E);
  const long long mt_s = c.I_shared > 0 ? cdiv(T, bn_items) : 0;
  L.max_items_gu = static_cast<int>(mt_r * rt_gu + mt_s * st_gu);
  L.max_row_tiles = static_cast<int>(mt_r);
  L.max_items_dn = static_cast<int>((mt_r + mt_s) * nt_dn);
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align_up(o + bytes, 256);
    return at;
  };
  L.err = take(kCtrlBytes);
  L.nitems = take(16);
  L.z = take(static_cast<size_t>(T) * c.E * 4);
  L.unc = take(static_cast<size_t>(T) * 4);
  L.tile_hist = take(static_cast<size_t>(2) * c.E * L.n_ptiles * 4);
  L.idx = take(TK * 4);
  L.w = take(TK * 4);
  L.counts = take(static_cast<size_t>(c.E) * 4);
  L.offsets = take(static_cast<size_t>(c.E + 1) * 4);
  L.perm = take(TK * 4);
  L.inv_perm = take(TK * 4);
  L.gu_start = take(static_cast<size_t>(c.E + 2) * 4);
  L.dn_start = take(static_cast<size_t>(c.E + 2) * 4);
  L.ready = take(static_cast<size_t>(L.max_items_gu) * 4);
  L.h_r = take(TK * c.I * 2);
  L.h_s = take(static_cast<size_t>(T) * (c.I_shared > 0 ? c.I_shared : 0) * 2);
  L.y_slot = take((TK + T) * c.H * 4);
  L.wr_split = T > 32 ? take(static_cast<size_t>(3) * c.E * c.H * 2) : 0;
  L.zp = T <= kFrontMaxT ? take(static_cast<size_t>(8) * kFrontMaxT * c.E * 4) : 0;
  if (mx) {
    // h_r holds the e4m3 h codes; the rest is scales
    L.max_touched = static_cast<int>(TK < static_cast<size_t>(c.E) ? TK : c.E);
    const size_t kb_h = static_cast<size_t>(c.H / 128), kb_i = static_cast<size_t>(c.I / 128);
    if (c.wfmt == MOE_W_MXFP4_A8) {  // touched-expert slots of the per-call scale repack
      L.slot_of = take(static_cast<size_t>(c.E) * 4);
      L.touched = take(static_cast<size_t>(c.E) * 4);
      L.ntouched = take(16);
    }
    L.x_q = take(static_cast<size_t>(T) * c.H);
    L.x_sf = take(static_cast<size_t>(T) * (c.H / 32));
    L.h_sf = take(static_cast<size_t>(L.max_row_tiles) * kb_i * 512);
    if (c.wfmt == MOE_W_MXFP4_A8) {
      const size_t atoms = static_cast<size_t>(L.max_touched) * kb_h * kb_i * 512;
      L.sf_g = take(atoms);
      L.sf_u = take(atoms);
      L.sf_d = take(atoms);
    }
  }
  L.total = o;
  return L;
}

}  // namespace sgl

using namespace sgl;

namespace {

bool cfg_ok(const moe_cfg* c) {
  if (c == nullptr) return false;
  if (c->H <= 0 || c->H % 64 != 0 || c->H > 16384) return false;
  if (c->E <= 0 || c->E % 32 != 0 || c->E > kMaxExpertsCfg) return false;
  if (c->n_group <= 0 || c->n_group > 32 || c->E % c->n_group != 0) return false;
  if (c->topk_group <= 0 || c->topk_group > c->n_group) return false;
  if (c->K <= 0 || c->K > 32 || c->K > c->topk_group * (c->E / c->n_group)) return false;
  if (c->I <= 0 || c->I % 64 != 0 || c->I > 16384) return false;
  if (c->I_shared < 0 || c->I_shared % 64 != 0 || c->I_shared > 16384) return false;
  if (isnan(c->scale) || isinf(c->scale)) return false;
  if (isnan(c->limit_routed) || isnan(c->limit_shared)) return false;
  if (c->wfmt != MOE_W_BF16 && c->wfmt != MOE_W_MXFP4 && !mx_a8(c->wfmt)) return false;
  if (mx_a8(c->wfmt) && (c->H % 128 != 0 || c->I % 128 != 0)) return false;
  return true;
}

bool T_ok(int32_t T) { return T >= 1 && T <= (1 << 20); }

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// SGL_MOE_FRONT=separate keeps the separate routing and permutation kernels
// for decode batches (read at every call; for comparisons and tests).
bool fused_front_disabled() {
  const char* v = getenv("SGL_MOE_FRONT");
  return v != nullptr && strcmp(v, "separate") == 0;
}

// sm_100 check, cached per device.
moe_status device_ok() {
  static int cache[64] = {0};  // 0 unknown, 1 ok, 2 not ok
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= 64) return MOE_ERR_UNSUPPORTED;
  if (cache[dev] == 0) {
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    cache[dev] = (major == 10 && minor == 0) ? 1 : 2;
  }
  return cache[dev] == 1 ? MOE_OK : MOE_ERR_UNSUPPORTED;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

moe_status cu(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

moe_status check_weights(const moe_cfg* c, const moe_weights* W) {
  if (W == nullptr || W->Wg == nullptr || W->Wu == nullptr || W->Wd == nullptr) return MOE_ERR_NULL;
  if (!al16(W->Wg) || !al16(W->Wu) || !al16(W->Wd)) return MOE_ERR_ALIGN;
  if (c->wfmt == MOE_W_MXFP4 || mx_a8(c->wfmt)) {
    if (!W->Wg_scale || !W->Wu_scale || !W->Wd_scale) return MOE_ERR_NULL;
    if (!al16(W->Wg_scale) || !al16(W->Wu_scale) || !al16(W->Wd_scale)) return MOE_ERR_ALIGN;
  }
  if (mx_a8(c->wfmt)) {  // TMA of unpacked 4-bit codes wants 32-byte bases
    auto al32 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; };
    if (!al32(W->Wg) || !al32(W->Wu) || !al32(W->Wd)) return MOE_ERR_ALIGN;
  }
  if (c->I_shared > 0) {
    if (W->Wg_s == nullptr || W->Wu_s == nullptr || W->Wd_s == nullptr) return MOE_ERR_NULL;
    if (!al16(W->Wg_s) || !al16(W->Wu_s) || !al16(W->Wd_s)) return MOE_ERR_ALIGN;
  }
  return MOE_OK;
}

// Stages 7-8 after the schedule: the weight-format preparation (MXFP4_A8:
// scale atoms and MXFP8 x), then the expert FFN kernel of the format (MXFP4
// weights are expanded to bf16 inside the FFN kernel).
cudaError_t run_ffn(const moe_cfg* cfg, int T, const uint16_t* x, const int32_t* perm,
                    const int32_t* offsets, const float* w, const moe_weights* W, float* y_slot,
                    void* ws, const WsLayout& L, cudaStream_t s,
                    const int32_t* sched_counts = nullptr) {
  GemmArgs a;
  memset(&a, 0, sizeof(a));
  a.sched_counts = sched_counts;
  a.cfg = cfg;
  a.T = T;
  a.x = x;
  a.perm = perm;
  a.w = w;
  a.W = W;
  a.Wg = W->Wg;
  a.Wu = W->Wu;
  a.Wd = W->Wd;
  a.wslot = nullptr;
  a.wrows = cfg->E;
  a.h_r = at<uint16_t>(ws, L.h_r);
  a.h_s = at<uint16_t>(ws, L.h_s);
  a.y_slot = y_slot;
  a.offsets = offsets;
  a.gu_start = at<int32_t>(ws, L.gu_start);
  a.dn_start = at<int32_t>(ws, L.dn_start);
  a.ready = at<int32_t>(ws, L.ready);
  a.nitems = at<int32_t>(ws, L.nitems);
  a.err = at<int32_t>(ws, L.err);
  a.bn = L.bn;
  a.ffn = L.ffn;
  a.max_items_gu = L.max_items_gu;
  a.max_items_dn = L.max_items_dn;
  if (mx_a8(cfg->wfmt)) {
    if (cfg->wfmt == MOE_W_MXFP4_A8) {  // touched experts' scales repacked for this call
      cudaError_t e = launch_mx_prep(*cfg, T, offsets, W, x, at<int32_t>(ws, L.slot_of),
                                     at<int32_t>(ws, L.touched), at<int32_t>(ws, L.ntouched),
                                     at<uint8_t>(ws, L.sf_g), at<uint8_t>(ws, L.sf_u),
                                     at<uint8_t>(ws, L.sf_d), at<uint8_t>(ws, L.x_q),
                                     at<uint8_t>(ws, L.x_sf), s);
      if (e != cudaSuccess) return e;
      a.sf_g = at<uint8_t>(ws, L.sf_g);
      a.sf_u = at<uint8_t>(ws, L.sf_u);
      a.sf_d = at<uint8_t>(ws, L.sf_d);
      a.slot_of = at<int32_t>(ws, L.slot_of);
    } else {  // prepared atoms of every expert (moe_prepare_weights)
      cudaError_t e = launch_mx_quant(*cfg, T, x, at<uint8_t>(ws, L.x_q), at<uint8_t>(ws, L.x_sf), s);
      if (e != cudaSuccess) return e;
      a.sf_g = W->Wg_scale;
      a.sf_u = W->Wu_scale;
      a.sf_d = W->Wd_scale;
      a.slot_of = nullptr;
    }
    a.x_q = at<uint8_t>(ws, L.x_q);
    a.x_sf = at<uint8_t>(ws, L.x_sf);
    a.h_q = at<uint8_t>(ws, L.h_r);
    a.h_sf = at<uint8_t>(ws, L.h_sf);
    return launch_ffn_mx(a, s);
  }
  return launch_ffn(a, s);
}

}  // namespace

extern "C" {

size_t moe_workspace_size(const moe_cfg* cfg, int32_t T) {
  if (!cfg_ok(cfg) || !T_ok(T)) return 0;
  return ws_layout(*cfg, T).total;
}

moe_status moe_route(const moe_cfg* cfg, int32_t T, const void* x, const float* Wr,
                     const float* bias, int32_t* idx, float* w, void* ws, size_t ws_bytes,
                     void* stream) {
  PdlScope pdl_scope(T);  // programmatic dependent launch for small batches
  if (!cfg_ok(cfg) || !T_ok(T)) return MOE_ERR_CFG;
  if (!x || !Wr || !idx || !w) return MOE_ERR_NULL;
  if (!al16(x) || !al16(Wr) || !al16(idx) || !al16(w) || (bias && !al16(bias))) return MOE_ERR_ALIGN;
  const WsLayout L = ws_layout(*cfg, T);
  if (ws == nullptr || ws_bytes < L.total || !al16(ws)) return MOE_ERR_WORKSPACE;
  moe_status st = device_ok();
  if (st != MOE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(at<int32_t>(ws, L.err), 0, kCtrlBytes, s) != cudaSuccess) return MOE_ERR_CUDA;
  return cu(launch_router(*cfg, T, static_cast<const uint16_t*>(x), Wr, bias, at<float>(ws, L.z),
                          idx, w, at<int32_t>(ws, L.unc), at<int32_t>(ws, L.err) + 1,
                          at<int32_t>(ws, L.err), T > 32 ? at<uint16_t>(ws, L.wr_split) : nullptr,
                          s));
}

moe_status moe_permute(const moe_cfg* cfg, int32_t T, const int32_t* idx, int32_t* counts,
                       int32_t* offsets, int32_t* perm, int32_t* inv_perm, void* ws,
                       size_t ws_bytes, void* stream) {
  PdlScope pdl_scope(T);  // programmatic dependent launch for small batches
  if (!cfg_ok(cfg) || !T_ok(T)) return MOE_ERR_CFG;
  if (!idx || !counts || !offsets || !perm) return MOE_ERR_NULL;
  if (!al16(idx) || !al16(counts) || !al16(offsets) || !al16(perm) || (inv_perm && !al16(inv_perm)))
    return MOE_ERR_ALIGN;
  const WsLayout L = ws_layout(*cfg, T);
  if (ws == nullptr || ws_bytes < L.total || !al16(ws)) return MOE_ERR_WORKSPACE;
  moe_status st = device_ok();
  if (st != MOE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(at<int32_t>(ws, L.err), 0, 16, s) != cudaSuccess) return MOE_ERR_CUDA;
  return cu(launch_permute(*cfg, T, idx, at<int32_t>(ws, L.tile_hist), counts, offsets, perm,
                           inv_perm, at<int32_t>(ws, L.err), L, nullptr, nullptr, nullptr,
                           at<int32_t>(ws, L.nitems), s));
}

moe_status moe_permute_static(const moe_cfg* cfg, int32_t T, const int32_t* idx, int32_t* counts,
                              int32_t* offsets, int32_t* perm, int32_t* inv_perm, void* stream) {
  if (!cfg_ok(cfg) || !T_ok(T)) return MOE_ERR_CFG;
  if (!idx || !counts || !offsets || !perm) return MOE_ERR_NULL;
  if (!al16(idx) || !al16(counts) || !al16(offsets) || !al16(perm) || (inv_perm && !al16(inv_perm)))
    return MOE_ERR_ALIGN;
  if (static_cast<long long>(T) * cfg->K > kStaticMaxSlots || cfg->E > kStaticMaxExperts)
    return MOE_ERR_WORKSPACE;
  moe_status st = device_ok();
  if (st != MOE_OK) return st;
  return cu(launch_permute_static(*cfg, T, idx, counts, offsets, perm, inv_perm,
                                  static_cast<cudaStream_t>(stream)));
}

moe_status moe_grouped_swiglu(const moe_cfg* cfg, int32_t T, const void* x, const int32_t* perm,
                              const int32_t* offsets, const float* w, const moe_weights* W,
                              void* y_slot, void* ws, size_t ws_bytes, void* stream) {
  PdlScope pdl_scope(T);  // programmatic dependent launch for small batches
  if (!cfg_ok(cfg) || !T_ok(T)) return MOE_ERR_CFG;
  if (!x || !perm || !offsets || !w || !y_slot) return MOE_ERR_NULL;
  if (!al16(x) || !al16(perm) || !al16(offsets) || !al16(w) || !al16(y_slot)) return MOE_ERR_ALIGN;
  moe_status st = check_weights(cfg, W);
  if (st != MOE_OK) return st;
  const WsLayout L = ws_layout(*cfg, T);
  if (ws == nullptr || ws_bytes < L.total || !al16(ws)) return MOE_ERR_WORKSPACE;
  st = device_ok();
  if (st != MOE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t* gu = at<int32_t>(ws, L.gu_start);
  int32_t* dn = at<int32_t>(ws, L.dn_start);
  int32_t* nitems = at<int32_t>(ws, L.nitems);
  cudaError_t e = launch_schedule(*cfg, T, offsets, L, gu, dn, at<int32_t>(ws, L.ready), nitems, s);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  return cu(run_ffn(cfg, T, static_cast<const uint16_t*>(x), perm, offsets, w, W,
                    static_cast<float*>(y_slot), ws, L, s));
}

moe_status moe_combine(const moe_cfg* cfg, int32_t T, const void* y_slot, int32_t with_shared,
                       void* y, void* stream) {
  PdlScope pdl_scope(T);  // programmatic dependent launch for small batches
  if (!cfg_ok(cfg) || !T_ok(T)) return MOE_ERR_CFG;
  if (!y_slot || !y) return MOE_ERR_NULL;
  if (!al16(y_slot) || !al16(y)) return MOE_ERR_ALIGN;
  moe_status st = device_ok();
  if (st != MOE_OK) return st;
  return cu(launch_combine(*cfg, T, static_cast<const float*>(y_slot), with_shared ? 1 : 0,
                           static_cast<uint16_t*>(y), static_cast<cudaStream_t>(stream)));
}

moe_status moe_layer_forward(const moe_cfg* cfg, int32_t T, const void* x, const float* Wr,
                             const float* bias, const moe_weights* W, void* y, int32_t* idx_out,
                             float* w_out, int32_t* counts_out, void* ws, size_t ws_bytes,
                             void* stream, void* const* stage_events) {
  PdlScope pdl_scope(T);  // programmatic dependent launch for small batches
  if (!cfg_ok(cfg) || !T_ok(T)) return MOE_ERR_CFG;
  if (!x || !Wr || !y) return MOE_ERR_NULL;
  if (!al16(x) || !al16(Wr) || !al16(y) || (bias && !al16(bias)) || (idx_out && !al16(idx_out)) ||
      (w_out && !al16(w_out)) || (counts_out && !al16(counts_out)))
    return MOE_ERR_ALIGN;
  moe_status st = check_weights(cfg, W);
  if (st != MOE_OK) return st;
  const WsLayout L = ws_layout(*cfg, T);
  if (ws == nullptr || ws_bytes < L.total || !al16(ws)) return MOE_ERR_WORKSPACE;
  st = device_ok();
  if (st != MOE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  auto rec = [&](int i) {
    if (stage_events && stage_events[i])
      cudaEventRecord(static_cast<cudaEvent_t>(stage_events[i]), s);
  };
  int32_t* idx = idx_out ? idx_out : at<int32_t>(ws, L.idx);
  float* w = w_out ? w_out : at<float>(ws, L.w);
  int32_t* counts = counts_out ? counts_out : at<int32_t>(ws, L.counts);
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* perm = at<int32_t>(ws, L.perm);
  int32_t* err = at<int32_t>(ws, L.err);
  int32_t* gu = at<int32_t>(ws, L.gu_start);
  int32_t* dn = at<int32_t>(ws, L.dn_start);
  int32_t* nitems = at<int32_t>(ws, L.nitems);
  float* y_slot = at<float>(ws, L.y_slot);
  cudaError_t e;
  rec(0);
  if (cudaMemsetAsync(err, 0, kCtrlBytes, s) != cudaSuccess) return MOE_ERR_CUDA;
  // decode batches: routing and permutation in one launch; the narrow FFN
  // kernel then derives its work lists from the counts (off the front's tail)
  const bool front = decode_front_ok(*cfg, T) && !fused_front_disabled();
  const bool ffn_derives = front && L.ffn == kFfnNarrow;
  if (front) {
    if ((e = launch_decode_front(*cfg, T, static_cast<const uint16_t*>(x), Wr, bias,
                                 at<float>(ws, L.zp), at<float>(ws, L.z), idx, w,
                                 at<int32_t>(ws, L.unc), err + 1, err + 2, err, counts, offsets,
                                 perm, at<int32_t>(ws, L.inv_perm), L, gu, dn,
                                 at<int32_t>(ws, L.ready), nitems, W, !ffn_derives, s)) != cudaSuccess)
      return MOE_ERR_CUDA;
    rec(1);
  } else {
    if ((e = launch_router(*cfg, T, static_cast<const uint16_t*>(x), Wr, bias, at<float>(ws, L.z),
                           idx, w, at<int32_t>(ws, L.unc), err + 1, err,
                           T > 32 ? at<uint16_t>(ws, L.wr_split) : nullptr, s)) != cudaSuccess)
      return MOE_ERR_CUDA;
    rec(1);
    if ((e = launch_permute(*cfg, T, idx, at<int32_t>(ws, L.tile_hist), counts, offsets, perm,
                            at<int32_t>(ws, L.inv_perm), err, L, gu, dn, at<int32_t>(ws, L.ready),
                            nitems, s)) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  rec(2);
  if ((e = run_ffn(cfg, T, static_cast<const uint16_t*>(x), perm, offsets, w, W, y_slot, ws, L, s,
                   ffn_derives ? counts : nullptr)) != cudaSuccess)
    return MOE_ERR_CUDA;
  rec(3);
  rec(4);
  if ((e = launch_combine(*cfg, T, y_slot, cfg->I_shared > 0 ? 1 : 0, static_cast<uint16_t*>(y),
                          s)) != cudaSuccess)
    return MOE_ERR_CUDA;
  rec(5);
  return MOE_OK;
}

moe_status moe_prepare_weights(const moe_cfg* cfg, const moe_weights* W, uint8_t* Wg_sf,
                               uint8_t* Wu_sf, uint8_t* Wd_sf, void* stream) {
  if (!cfg_ok(cfg) || !mx_a8(cfg->wfmt)) return MOE_ERR_CFG;
  if (!W || !W->Wg_scale || !W->Wu_scale || !W->Wd_scale || !Wg_sf || !Wu_sf || !Wd_sf)
    return MOE_ERR_NULL;
  if (!al16(W->Wg_scale) || !al16(W->Wu_scale) || !al16(W->Wd_scale) || !al16(Wg_sf) ||
      !al16(Wu_sf) || !al16(Wd_sf))
    return MOE_ERR_ALIGN;
  moe_status st = device_ok();
  if (st != MOE_OK) return st;
  return cu(launch_mx_sf_atoms(*cfg, W, Wg_sf, Wu_sf, Wd_sf, static_cast<cudaStream_t>(stream)));
}

moe_status moe_route_stats(const moe_cfg* cfg, const int32_t* counts, double* stats,
                           void* stream) {
  if (!cfg_ok(cfg)) return MOE_ERR_CFG;
  if (!counts || !stats) return MOE_ERR_NULL;
  if (!al16(counts) || !al16(stats)) return MOE_ERR_ALIGN;
  moe_status st = device_ok();
  if (st != MOE_OK) return st;
  return cu(launch_route_stats(*cfg, counts, stats, static_cast<cudaStream_t>(stream)));
}

moe_status moe_read_error(const moe_cfg* cfg, int32_t T, void* ws, size_t ws_bytes, void* stream,
                          int32_t* code) {
  if (!cfg_ok(cfg) || !T_ok(T)) return MOE_ERR_CFG;
  if (!code) return MOE_ERR_NULL;
  const WsLayout L = ws_layout(*cfg, T);
  if (ws == nullptr || ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t v = 0;
  if (cudaMemcpyAsync(&v, at<int32_t>(ws, L.err), 4, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemsetAsync(at<int32_t>(ws, L.err), 0, 4, s) != cudaSuccess) return MOE_ERR_CUDA;
  *code = v;
  return MOE_OK;
}

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_CFG: return "MOE_ERR_CFG: configuration or token count outside the supported range";
    case MOE_ERR_NULL: return "MOE_ERR_NULL: a required pointer is NULL";
    case MOE_ERR_ALIGN: return "MOE_ERR_ALIGN: a device pointer is not 16-byte aligned";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE: workspace missing or too small";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA: a CUDA call or kernel launch failed";
    case MOE_ERR_DEVICE: return "MOE_ERR_DEVICE: a kernel reported bad data";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED: device or weight format not supported";
  }
  return "MOE_ERR_UNKNOWN";
}

const char* moe_version(void) { return "sgl-moe 0.1 (sm_100a)"; }

}  // extern "C"
