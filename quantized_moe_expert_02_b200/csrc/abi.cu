// C ABI entry points: argument checks, workspace carving, dispatch between
// the decode kernels (T <= 8) and the general path.
#include <mutex>

#include "moe_internal.cuh"
#include "trace.h"

namespace moe {

moe_status launch_route(const uint16_t* x, int T, int H, const uint16_t* wr,
                        int E, const float* bias, int k, int32_t* topk_idx,
                        float* topk_w, float* logits, int32_t* err,
                        cudaStream_t s);
moe_status launch_group(const int32_t* idx, int T, int k, int E,
                        int32_t* offsets, int32_t* pair_ids, int32_t* active,
                        int32_t* n_active, int32_t* scratch, int32_t* err,
                        cudaStream_t s);
moe_status launch_up_generic(const moe_layer_desc& d, const uint16_t* x,
                             int T, int k, const int32_t* offsets,
                             const int32_t* pair_ids, const int32_t* active,
                             const int32_t* n_active,
                             const int32_t* blob_index, float* h,
                             int32_t* err, cudaStream_t s);
moe_status launch_down_generic(const moe_layer_desc& d, int T, int k,
                               const int32_t* offsets,
                               const int32_t* pair_ids, const int32_t* active,
                               const int32_t* n_active,
                               const int32_t* blob_index, const float* h,
                               float* y, int32_t* err, cudaStream_t s);
moe_status launch_combine(const float* y, const float* w, int T, int k,
                          int H, const float* residual, float* out,
                          uint16_t* out_bf16, cudaStream_t s);
bool ffn_decode_supported(const moe_layer_desc& d, int T, int k);
moe_status launch_up_decode(const moe_layer_desc& d, const uint16_t* x,
                            int T, int k, const int32_t* offsets,
                            const int32_t* pair_ids, const int32_t* active,
                            const int32_t* n_active, const int32_t* blob_index,
                            const FfnWs& ws, cudaStream_t s, bool pdl);
moe_status launch_down_decode(const moe_layer_desc& d, int T, int k,
                              const int32_t* offsets, const int32_t* pair_ids,
                              const int32_t* active, const int32_t* n_active,
                              const int32_t* blob_index, const FfnWs& ws,
                              float* y, const float* topk_w,
                              const float* residual, float* out,
                              uint16_t* out_bf16, cudaStream_t s, bool pdl);

bool pf_supported(const moe_layer_desc& d, int T);
int64_t pf_max_tiles(int64_t P);
moe_status launch_pf_up(const moe_layer_desc& d, const uint16_t* x, int T,
                        int k, const int32_t* offsets,
                        const int32_t* pair_ids, const int32_t* blob_index,
                        const FfnWs& w, cudaStream_t s);
moe_status launch_pf_up_gemm(const moe_layer_desc& d, int T, int k,
                             const int32_t* pair_ids,
                             const int32_t* blob_index, const FfnWs& w,
                             cudaStream_t s);
moe_status launch_pf_down(const moe_layer_desc& d, int T, int k,
                          const int32_t* pair_ids, const int32_t* blob_index,
                          const FfnWs& w, float* y, cudaStream_t s);

bool decode_layer_supported(const moe_layer_desc& d, int T, int k);
size_t decode_layer_ws_bytes(int T, int k, int H, int F);
moe_status launch_decode_layer(const moe_layer_desc& d, const uint16_t* x,
                               const float* r_in, int T, int k,
                               const uint16_t* wr, const float* bias,
                               const int32_t* blob_index,
                               const float* residual, float* out,
                               uint16_t* out_bf16, int32_t* topk_idx,
                               float* topk_w, float* logits, void* ws,
                               int32_t* err, cudaStream_t s, int mode,
                               const StageArgs* stg = nullptr);
moe_status launch_rmsnorm_bf16(const float* r, int T, int H, uint16_t* x,
                               cudaStream_t s);

int num_sms() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cached[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) !=
            cudaSuccess || n <= 0)
      n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

moe_status ensure_smem(const void* kernel, size_t bytes) {
  struct Entry { const void* fn; int dev; int bytes; };
  static Entry table[256];
  static int n = 0;
  static std::mutex mu;
  if (bytes <= 48 * 1024) return MOE_OK;
  int dev = 0;
  MOE_CUDA_TRY(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < n; ++i)
    if (table[i].fn == kernel && table[i].dev == dev &&
        table[i].bytes >= (int)bytes)
      return MOE_OK;
  MOE_CUDA_TRY(cudaFuncSetAttribute(
      kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes));
  for (int i = 0; i < n; ++i)
    if (table[i].fn == kernel && table[i].dev == dev) {
      table[i].bytes = (int)bytes;
      return MOE_OK;
    }
  if (n < 256) table[n++] = {kernel, dev, (int)bytes};
  return MOE_OK;
}

struct Carver {
  size_t off = 0;
  size_t take(size_t bytes) {
    const size_t o = off;
    off += (bytes + 255) & ~(size_t)255;
    return o;
  }
};

struct Layout {
  size_t err, up_cnt, dn_cnt, up_part, bfrag, bscale, y_int, h;
  size_t x16, xscale, inv, tiles, n_tiles, total;
};

static Layout ffn_layout(int T, int k, int H, int F) {
  Carver c;
  Layout L;
  const int64_t P = (int64_t)T * k;
  const bool dec = T <= DEC_TMAX;
  const int64_t nrt = F / 32;
  L.err = c.take(64);
  L.up_cnt = c.take(dec ? P * nrt * 4 : 0);
  L.dn_cnt = c.take(dec ? (int64_t)(H / 16) * 4 : 0);
  L.up_part = c.take(dec ? P * nrt * NSPLIT_MAX * 2 * 256 * 4 : 0);
  L.bfrag = c.take(dec ? P * nrt * BF_NT * 64 * 4 : 0);
  L.bscale = c.take(dec ? P * nrt * 8 * 4 : 0);
  L.y_int = c.take(P * H * 4);
  L.h = c.take(P * F * 4);
  L.x16 = c.take(dec ? 0 : P * H * 2);
  L.xscale = c.take(dec ? 0 : P * 4);
  L.inv = c.take(dec ? 0 : P * 4);
  L.tiles = c.take(dec ? 0 : pf_max_tiles(P) * 16);
  L.n_tiles = c.take(64);
  L.total = c.off;
  return L;
}

FfnWs carve_ffn_ws(void* base, int T, int k, int H, int F) {
  const Layout L = ffn_layout(T, k, H, F);
  uint8_t* b = static_cast<uint8_t*>(base);
  FfnWs w;
  w.err = reinterpret_cast<int32_t*>(b + L.err);
  w.up_cnt = reinterpret_cast<int32_t*>(b + L.up_cnt);
  w.dn_cnt = reinterpret_cast<int32_t*>(b + L.dn_cnt);
  w.up_part = reinterpret_cast<float*>(b + L.up_part);
  w.bfrag = reinterpret_cast<uint32_t*>(b + L.bfrag);
  w.bscale = reinterpret_cast<float*>(b + L.bscale);
  w.y_int = reinterpret_cast<float*>(b + L.y_int);
  w.h = reinterpret_cast<float*>(b + L.h);
  w.x16 = reinterpret_cast<__half*>(b + L.x16);
  w.xscale = reinterpret_cast<float*>(b + L.xscale);
  w.inv = reinterpret_cast<int32_t*>(b + L.inv);
  w.tiles = reinterpret_cast<int4*>(b + L.tiles);
  w.n_tiles = reinterpret_cast<int32_t*>(b + L.n_tiles);
  w.logits = nullptr;
  w.grp = nullptr;
  w.bytes = L.total;
  return w;
}

// Layer workspace = FFN workspace, then routing and grouping buffers.
struct LayerWs {
  FfnWs ffn;
  void* fused;       // workspace of the one-kernel decode layer
  float* logits;
  int32_t* offsets;
  int32_t* pair_ids;
  int32_t* active;
  int32_t* n_active;
  int32_t* grp;
  uint16_t* xr;      // bf16 [T][H]: rmsnorm of the residual (T > 8)
  size_t bytes;
};

static LayerWs carve_layer_ws(void* base, int T, int k, int E, int H, int F) {
  LayerWs w;
  w.ffn = carve_ffn_ws(base, T, k, H, F);
  Carver c;
  c.off = w.ffn.bytes;
  const int64_t P = (int64_t)T * k;
  const size_t lo = c.take((size_t)T * E * 4);
  const size_t of = c.take((size_t)(E + 1) * 4);
  const size_t pi = c.take((size_t)P * 4);
  const size_t ac = c.take((size_t)E * 4);
  const size_t na = c.take(64);
  const size_t gr = c.take(group_ws_bytes(T, k, E));
  const size_t fu = c.take(T <= DEC_TMAX ? decode_layer_ws_bytes(T, k, H, F)
                                         : 0);
  const size_t xr = c.take(T <= DEC_TMAX ? 0 : (size_t)T * H * 2);
  uint8_t* b = static_cast<uint8_t*>(base);
  w.fused = base ? static_cast<void*>(b + fu) : nullptr;
  w.logits = base ? reinterpret_cast<float*>(b + lo) : nullptr;
  w.offsets = base ? reinterpret_cast<int32_t*>(b + of) : nullptr;
  w.pair_ids = base ? reinterpret_cast<int32_t*>(b + pi) : nullptr;
  w.active = base ? reinterpret_cast<int32_t*>(b + ac) : nullptr;
  w.n_active = base ? reinterpret_cast<int32_t*>(b + na) : nullptr;
  w.grp = base ? reinterpret_cast<int32_t*>(b + gr) : nullptr;
  w.xr = base ? reinterpret_cast<uint16_t*>(b + xr) : nullptr;
  w.bytes = c.off;
  return w;
}

static moe_status check_desc(const moe_layer_desc* d) {
  if (!d || !d->pool) return MOE_ERR_INVALID;
  if (!fmt_valid(d->fmt_up_gate) || !fmt_valid(d->fmt_down))
    return MOE_ERR_INVALID;
  if (d->E <= 0 || d->E > EMAX) return MOE_ERR_SHAPE;
  if (!packed_shape_ok(d->fmt_up_gate, d->F, d->H)) return MOE_ERR_SHAPE;
  if (!packed_shape_ok(d->fmt_down, d->H, d->F)) return MOE_ERR_SHAPE;
  if (d->F % 32 || d->H % 32) return MOE_ERR_SHAPE;
  const int64_t blob = 2 * tensor_bytes_of(d->fmt_up_gate, d->F, d->H) +
                       tensor_bytes_of(d->fmt_down, d->H, d->F);
  if (d->blob_stride < blob || d->blob_stride % 16) return MOE_ERR_SHAPE;
  if ((uintptr_t)d->pool % 16) return MOE_ERR_INVALID;
  return MOE_OK;
}

static moe_status check_ffn_args(const moe_layer_desc* desc, int T, int k,
                                 const int32_t* offsets,
                                 const int32_t* pair_ids,
                                 const int32_t* active,
                                 const int32_t* n_active, void* ws,
                                 size_t ws_bytes) {
  moe_status st = check_desc(desc);
  if (st != MOE_OK) return st;
  if (!offsets || !pair_ids || !active || !n_active) return MOE_ERR_INVALID;
  if (T <= 0 || k <= 0 || k > 32 || k > desc->E) return MOE_ERR_SHAPE;
  if (!ws) return MOE_ERR_WORKSPACE;
  if (ws_bytes < ffn_layout(T, k, desc->H, desc->F).total)
    return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

// Up/gate + SwiGLU (result stays in the workspace).
static moe_status run_up(const moe_layer_desc& d, const uint16_t* x, int T,
                         int k, const int32_t* offsets,
                         const int32_t* pair_ids, const int32_t* active,
                         const int32_t* n_active, const int32_t* blob_index,
                         const FfnWs& w, cudaStream_t s, bool pdl) {
  if (ffn_decode_supported(d, T, k))
    return launch_up_decode(d, x, T, k, offsets, pair_ids, active, n_active,
                            blob_index, w, s, pdl);
  if (pf_supported(d, T))
    return launch_pf_up(d, x, T, k, offsets, pair_ids, blob_index, w, s);
  return launch_up_generic(d, x, T, k, offsets, pair_ids, active, n_active,
                           blob_index, w.h, w.err, s);
}

// Down projection, optionally followed by the combine.
static moe_status run_down(const moe_layer_desc& d, int T, int k,
                           const int32_t* offsets, const int32_t* pair_ids,
                           const int32_t* active, const int32_t* n_active,
                           const int32_t* blob_index, const FfnWs& w,
                           float* y_pairs, const float* topk_w,
                           const float* residual, float* out,
                           uint16_t* out_bf16, cudaStream_t s, bool pdl) {
  float* y = y_pairs ? y_pairs : w.y_int;
  if (ffn_decode_supported(d, T, k))
    return launch_down_decode(d, T, k, offsets, pair_ids, active, n_active,
                              blob_index, w, y, topk_w, residual, out,
                              out_bf16, s, pdl);
  moe_status st =
      pf_supported(d, T)
          ? launch_pf_down(d, T, k, pair_ids, blob_index, w, y, s)
          : launch_down_generic(d, T, k, offsets, pair_ids, active, n_active,
                                blob_index, w.h, y, w.err, s);
  if (st != MOE_OK || !out) return st;
  return launch_combine(y, topk_w, T, k, d.H, residual, out, out_bf16, s);
}

}  // namespace moe

using namespace moe;

extern "C" const char* moe_status_string(int st) {
  switch (st) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID: return "invalid argument";
    case MOE_ERR_SHAPE: return "unsupported shape";
    case MOE_ERR_UNSUPPORTED: return "unsupported";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_DEVICE: return "device error word set";
    case MOE_ERR_CAPACITY: return "slot pool capacity exceeded";
    case MOE_ERR_TIMEOUT: return "device wait timed out";
    case MOE_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

extern "C" moe_status moe_route_topk(const uint16_t* x, int T, int H,
                                     const uint16_t* w_router, int E,
                                     const float* bias, int k,
                                     int32_t* topk_idx, float* topk_w,
                                     float* logits_out, void* stream) {
  MOE_TRACE();
  if (!x || !w_router || !topk_idx || !topk_w || !logits_out)
    return logits_out ? MOE_ERR_INVALID : MOE_ERR_WORKSPACE;
  if (T <= 0 || H <= 0 || H % 8 || E <= 0 || E > EMAX || k < 1 || k > 32 ||
      k > E)
    return MOE_ERR_SHAPE;
  if (((uintptr_t)x | (uintptr_t)w_router) % 16) return MOE_ERR_INVALID;
  return launch_route(x, T, H, w_router, E, bias, k, topk_idx, topk_w,
                      logits_out, nullptr, (cudaStream_t)stream);
}

extern "C" size_t moe_group_workspace_bytes(int T, int k, int E) {
  if (T <= 0 || k <= 0 || E <= 0) return 0;
  return 256 + group_ws_bytes(T, k, E);
}

extern "C" moe_status moe_group_tokens(const int32_t* topk_idx, int T, int k,
                                       int E, int32_t* expert_offsets,
                                       int32_t* pair_ids, int32_t* active,
                                       int32_t* n_active, void* ws,
                                       size_t ws_bytes, void* stream) {
  MOE_TRACE();
  if (!topk_idx || !expert_offsets || !pair_ids || !active || !n_active)
    return MOE_ERR_INVALID;
  if (T <= 0 || k <= 0 || E <= 0 || E > EMAX) return MOE_ERR_SHAPE;
  if (!ws || ws_bytes < moe_group_workspace_bytes(T, k, E))
    return MOE_ERR_WORKSPACE;
  int32_t* err = static_cast<int32_t*>(ws);
  int32_t* scratch = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + 256);
  return launch_group(topk_idx, T, k, E, expert_offsets, pair_ids, active,
                      n_active, scratch, err, (cudaStream_t)stream);
}

extern "C" size_t moe_ffn_workspace_bytes(int T, int k, int H, int F) {
  if (T <= 0 || k <= 0 || H <= 0 || F <= 0) return 0;
  return ffn_layout(T, k, H, F).total;
}

extern "C" size_t moe_layer_workspace_bytes(int T, int k, int E, int H,
                                            int F) {
  if (T <= 0 || k <= 0 || E <= 0 || H <= 0 || F <= 0) return 0;
  return carve_layer_ws(nullptr, T, k, E, H, F).bytes;
}

extern "C" moe_status moe_workspace_init(void* ws, size_t ws_bytes,
                                         void* stream) {
  MOE_TRACE();
  if (!ws) return MOE_ERR_WORKSPACE;
  MOE_CUDA_TRY(cudaMemsetAsync(ws, 0, ws_bytes, (cudaStream_t)stream));
  return MOE_OK;
}

extern "C" moe_status moe_expert_up_q(
    const moe_layer_desc* desc, const uint16_t* x, int T, int k,
    const int32_t* expert_offsets, const int32_t* pair_ids,
    const int32_t* active, const int32_t* n_active,
    const int32_t* blob_index, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRACE();
  if (!x || ((uintptr_t)x & 15)) return MOE_ERR_INVALID;
  moe_status st = check_ffn_args(desc, T, k, expert_offsets, pair_ids, active,
                                 n_active, ws, ws_bytes);
  if (st != MOE_OK) return st;
  const FfnWs w = carve_ffn_ws(ws, T, k, desc->H, desc->F);
  return run_up(*desc, x, T, k, expert_offsets, pair_ids, active, n_active,
                blob_index, w, (cudaStream_t)stream, false);
}

extern "C" moe_status moe_expert_up_gemm_q(
    const moe_layer_desc* desc, int T, int k, const int32_t* expert_offsets,
    const int32_t* pair_ids, const int32_t* active, const int32_t* n_active,
    const int32_t* blob_index, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRACE();
  moe_status st = check_ffn_args(desc, T, k, expert_offsets, pair_ids, active,
                                 n_active, ws, ws_bytes);
  if (st != MOE_OK) return st;
  if (ffn_decode_supported(*desc, T, k) || !pf_supported(*desc, T))
    return MOE_ERR_UNSUPPORTED;
  const FfnWs w = carve_ffn_ws(ws, T, k, desc->H, desc->F);
  return launch_pf_up_gemm(*desc, T, k, pair_ids, blob_index, w,
                           (cudaStream_t)stream);
}

extern "C" moe_status moe_expert_down_q(
    const moe_layer_desc* desc, int T, int k, const int32_t* expert_offsets,
    const int32_t* pair_ids, const int32_t* active, const int32_t* n_active,
    const int32_t* blob_index, float* y_pairs, const float* topk_w,
    const float* residual, float* out, uint16_t* out_bf16, void* ws,
    size_t ws_bytes, void* stream) {
  MOE_TRACE();
  if (!y_pairs && !out) return MOE_ERR_INVALID;
  if (out && !topk_w) return MOE_ERR_INVALID;
  moe_status st = check_ffn_args(desc, T, k, expert_offsets, pair_ids, active,
                                 n_active, ws, ws_bytes);
  if (st != MOE_OK) return st;
  const FfnWs w = carve_ffn_ws(ws, T, k, desc->H, desc->F);
  return run_down(*desc, T, k, expert_offsets, pair_ids, active, n_active,
                  blob_index, w, y_pairs, topk_w, residual, out, out_bf16,
                  (cudaStream_t)stream, false);
}

extern "C" moe_status moe_expert_ffn_q(
    const moe_layer_desc* desc, const uint16_t* x, int T, int k,
    const int32_t* expert_offsets, const int32_t* pair_ids,
    const int32_t* active, const int32_t* n_active,
    const int32_t* blob_index, float* y_pairs, void* ws, size_t ws_bytes,
    void* stream) {
  MOE_TRACE();
  if (!y_pairs || !x || ((uintptr_t)x & 15)) return MOE_ERR_INVALID;
  moe_status st = check_ffn_args(desc, T, k, expert_offsets, pair_ids, active,
                                 n_active, ws, ws_bytes);
  if (st != MOE_OK) return st;
  const FfnWs w = carve_ffn_ws(ws, T, k, desc->H, desc->F);
  cudaStream_t s = (cudaStream_t)stream;
  st = run_up(*desc, x, T, k, expert_offsets, pair_ids, active, n_active,
              blob_index, w, s, false);
  if (st != MOE_OK) return st;
  return run_down(*desc, T, k, expert_offsets, pair_ids, active, n_active,
                  blob_index, w, y_pairs, nullptr, nullptr, nullptr, nullptr,
                  s, true);
}

extern "C" moe_status moe_expert_ffn_combine_q(
    const moe_layer_desc* desc, const uint16_t* x, int T, int k,
    const int32_t* expert_offsets, const int32_t* pair_ids,
    const int32_t* active, const int32_t* n_active,
    const int32_t* blob_index, const float* topk_w, const float* residual,
    float* out, uint16_t* out_bf16, void* ws, size_t ws_bytes,
    void* stream) {
  MOE_TRACE();
  if (!out || !topk_w || !x || ((uintptr_t)x & 15)) return MOE_ERR_INVALID;
  moe_status st = check_ffn_args(desc, T, k, expert_offsets, pair_ids, active,
                                 n_active, ws, ws_bytes);
  if (st != MOE_OK) return st;
  const FfnWs w = carve_ffn_ws(ws, T, k, desc->H, desc->F);
  cudaStream_t s = (cudaStream_t)stream;
  st = run_up(*desc, x, T, k, expert_offsets, pair_ids, active, n_active,
              blob_index, w, s, false);
  if (st != MOE_OK) return st;
  return run_down(*desc, T, k, expert_offsets, pair_ids, active, n_active,
                  blob_index, w, nullptr, topk_w, residual, out, out_bf16, s,
                  true);
}

extern "C" moe_status moe_layer_forward(
    const moe_layer_desc* desc, const uint16_t* x, int T, int k,
    const uint16_t* w_router, const float* bias, const int32_t* blob_index,
    const float* residual, float* out, uint16_t* out_bf16, int32_t* topk_idx,
    float* topk_w, float* logits_out, void* ws, size_t ws_bytes,
    void* stream) {
  MOE_TRACE();
  moe_status st = check_desc(desc);
  if (st != MOE_OK) return st;
  if (!x || !w_router || !out || !topk_idx || !topk_w) return MOE_ERR_INVALID;
  if (T <= 0 || k < 1 || k > 32 || k > desc->E) return MOE_ERR_SHAPE;
  if (desc->H % 8 || ((uintptr_t)x | (uintptr_t)w_router) % 16)
    return MOE_ERR_INVALID;
  if (!ws) return MOE_ERR_WORKSPACE;
  const LayerWs w = carve_layer_ws(ws, T, k, desc->E, desc->H, desc->F);
  if (ws_bytes < w.bytes) return MOE_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  float* logits = logits_out ? logits_out : w.logits;
  if (decode_layer_supported(*desc, T, k))
    return launch_decode_layer(*desc, x, nullptr, T, k, w_router, bias,
                               blob_index, residual, out, out_bf16, topk_idx,
                               topk_w, logits, w.fused, w.ffn.err, s, DL_FULL);
  st = launch_route(x, T, desc->H, w_router, desc->E, bias, k, topk_idx,
                    topk_w, logits, w.ffn.err, s);
  if (st != MOE_OK) return st;
  st = launch_group(topk_idx, T, k, desc->E, w.offsets, w.pair_ids, w.active,
                    w.n_active, w.grp, w.ffn.err, s);
  if (st != MOE_OK) return st;
  st = run_up(*desc, x, T, k, w.offsets, w.pair_ids, w.active, w.n_active,
              blob_index, w.ffn, s, true);
  if (st != MOE_OK) return st;
  return run_down(*desc, T, k, w.offsets, w.pair_ids, w.active, w.n_active,
                  blob_index, w.ffn, nullptr, topk_w, residual, out, out_bf16,
                  s, true);
}

// ------------------------------------------------ pre-norm residual stack
// One layer of the residual stack: x = bf16(rmsnorm(r)), r_out = r + MoE(x),
// as one call or as its routing and FFN halves.

static moe_status check_residual_args(const moe_layer_desc* desc,
                                      const float* r, int T, int k,
                                      void* ws, size_t ws_bytes,
                                      LayerWs* w) {
  moe_status st = check_desc(desc);
  if (st != MOE_OK) return st;
  if (!r) return MOE_ERR_INVALID;
  if (T <= 0 || k < 1 || k > 32 || k > desc->E) return MOE_ERR_SHAPE;
  if (desc->H % 8 || ((uintptr_t)r % 16)) return MOE_ERR_INVALID;
  if (!ws) return MOE_ERR_WORKSPACE;
  *w = carve_layer_ws(ws, T, k, desc->E, desc->H, desc->F);
  if (ws_bytes < w->bytes) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

extern "C" moe_status moe_layer_forward_residual(
    const moe_layer_desc* desc, const float* r, int T, int k,
    const uint16_t* w_router, const float* bias, const int32_t* blob_index,
    float* r_out, uint16_t* out_bf16, int32_t* topk_idx, float* topk_w,
    float* logits_out, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRACE();
  LayerWs w;
  moe_status st = check_residual_args(desc, r, T, k, ws, ws_bytes, &w);
  if (st != MOE_OK) return st;
  if (!w_router || !r_out || !topk_idx || !topk_w) return MOE_ERR_INVALID;
  if ((uintptr_t)w_router % 16) return MOE_ERR_INVALID;
  cudaStream_t s = (cudaStream_t)stream;
  float* logits = logits_out ? logits_out : w.logits;
  if (decode_layer_supported(*desc, T, k))
    return launch_decode_layer(*desc, nullptr, r, T, k, w_router, bias,
                               blob_index, r, r_out, out_bf16, topk_idx,
                               topk_w, logits, w.fused, w.ffn.err, s, DL_FULL);
  st = launch_rmsnorm_bf16(r, T, desc->H, w.xr, s);
  if (st != MOE_OK) return st;
  st = launch_route(w.xr, T, desc->H, w_router, desc->E, bias, k, topk_idx,
                    topk_w, logits, w.ffn.err, s);
  if (st != MOE_OK) return st;
  st = launch_group(topk_idx, T, k, desc->E, w.offsets, w.pair_ids, w.active,
                    w.n_active, w.grp, w.ffn.err, s);
  if (st != MOE_OK) return st;
  st = run_up(*desc, w.xr, T, k, w.offsets, w.pair_ids, w.active, w.n_active,
              blob_index, w.ffn, s, true);
  if (st != MOE_OK) return st;
  return run_down(*desc, T, k, w.offsets, w.pair_ids, w.active, w.n_active,
                  blob_index, w.ffn, nullptr, topk_w, r, r_out, out_bf16, s,
                  true);
}

extern "C" moe_status moe_layer_route_residual(
    const moe_layer_desc* desc, const float* r, int T, int k,
    const uint16_t* w_router, const float* bias, int32_t* topk_idx,
    float* topk_w, float* logits_out, void* ws, size_t ws_bytes,
    void* stream) {
  MOE_TRACE();
  LayerWs w;
  moe_status st = check_residual_args(desc, r, T, k, ws, ws_bytes, &w);
  if (st != MOE_OK) return st;
  if (!w_router || !topk_idx || !topk_w) return MOE_ERR_INVALID;
  if ((uintptr_t)w_router % 16) return MOE_ERR_INVALID;
  cudaStream_t s = (cudaStream_t)stream;
  float* logits = logits_out ? logits_out : w.logits;
  if (decode_layer_supported(*desc, T, k))
    return launch_decode_layer(*desc, nullptr, r, T, k, w_router, bias,
                               nullptr, nullptr, nullptr, nullptr, topk_idx,
                               topk_w, logits, w.fused, w.ffn.err, s,
                               DL_ROUTE);
  st = launch_rmsnorm_bf16(r, T, desc->H, w.xr, s);
  if (st != MOE_OK) return st;
  return launch_route(w.xr, T, desc->H, w_router, desc->E, bias, k, topk_idx,
                      topk_w, logits, w.ffn.err, s);
}

extern "C" moe_status moe_layer_ffn_residual(
    const moe_layer_desc* desc, const float* r, int T, int k,
    const int32_t* topk_idx, const float* topk_w, const int32_t* blob_index,
    float* r_out, uint16_t* out_bf16, void* ws, size_t ws_bytes,
    void* stream) {
  MOE_TRACE();
  LayerWs w;
  moe_status st = check_residual_args(desc, r, T, k, ws, ws_bytes, &w);
  if (st != MOE_OK) return st;
  if (!r_out || !topk_idx || !topk_w) return MOE_ERR_INVALID;
  cudaStream_t s = (cudaStream_t)stream;
  if (decode_layer_supported(*desc, T, k))
    return launch_decode_layer(*desc, nullptr, r, T, k, nullptr, nullptr,
                               blob_index, r, r_out, out_bf16,
                               const_cast<int32_t*>(topk_idx),
                               const_cast<float*>(topk_w), w.logits, w.fused,
                               w.ffn.err, s, DL_FFN);
  st = launch_rmsnorm_bf16(r, T, desc->H, w.xr, s);
  if (st != MOE_OK) return st;
  st = launch_group(topk_idx, T, k, desc->E, w.offsets, w.pair_ids, w.active,
                    w.n_active, w.grp, w.ffn.err, s);
  if (st != MOE_OK) return st;
  st = run_up(*desc, w.xr, T, k, w.offsets, w.pair_ids, w.active, w.n_active,
              blob_index, w.ffn, s, true);
  if (st != MOE_OK) return st;
  return run_down(*desc, T, k, w.offsets, w.pair_ids, w.active, w.n_active,
                  blob_index, w.ffn, nullptr, topk_w, r, r_out, out_bf16, s,
                  true);
}

extern "C" moe_status moe_stage_misses(const int32_t* n_miss,
                                       const int32_t* miss_expert,
                                       const int32_t* miss_slot, int P,
                                       int layer, int L, int E,
                                       const uint64_t* table, uint8_t* pool,
                                       int slot_base, int n_slots,
                                       int64_t pool_slots,
                                       int64_t blob_stride,
                                       int64_t blob_bytes, int32_t* err,
                                       void* stream);

extern "C" moe_status moe_layer_ffn_residual_staged(
    const moe_layer_desc* desc, const float* r, int T, int k,
    const int32_t* topk_idx, const float* topk_w, const int32_t* blob_index,
    float* r_out, uint16_t* out_bf16, const int32_t* n_miss,
    const int32_t* miss_expert, const int32_t* miss_slot, int layer, int L,
    const uint64_t* table, int slot_base, int n_slots, int64_t pool_slots,
    void* ws, size_t ws_bytes, void* stream) {
  MOE_TRACE();
  LayerWs w;
  moe_status st = check_residual_args(desc, r, T, k, ws, ws_bytes, &w);
  if (st != MOE_OK) return st;
  if (!r_out || !topk_idx || !topk_w || !blob_index || !n_miss ||
      !miss_expert || !miss_slot || !table)
    return MOE_ERR_INVALID;
  if (layer < 0 || layer >= L || slot_base < 0 || n_slots < 1 ||
      pool_slots < 1 || slot_base + (int64_t)n_slots > pool_slots)
    return MOE_ERR_SHAPE;
  const int64_t blob = 2 * tensor_bytes_of(desc->fmt_up_gate, desc->F,
                                           desc->H) +
                       tensor_bytes_of(desc->fmt_down, desc->H, desc->F);
  if (blob % 16) return MOE_ERR_SHAPE;
  cudaStream_t s = (cudaStream_t)stream;
  if (decode_layer_supported(*desc, T, k)) {
    const StageArgs sa{n_miss, miss_expert, miss_slot, table, layer,
                       slot_base, n_slots, pool_slots, blob};
    return launch_decode_layer(*desc, nullptr, r, T, k, nullptr, nullptr,
                               blob_index, r, r_out, out_bf16,
                               const_cast<int32_t*>(topk_idx),
                               const_cast<float*>(topk_w), w.logits, w.fused,
                               w.ffn.err, s, DL_FFN, &sa);
  }
  // other shapes: the pull kernel, then the FFN half
  st = moe_stage_misses(n_miss, miss_expert, miss_slot, T * k, layer, L,
                        desc->E, table, const_cast<uint8_t*>(desc->pool),
                        slot_base, n_slots, pool_slots, desc->blob_stride,
                        blob, w.ffn.err, stream);
  if (st != MOE_OK) return st;
  return moe_layer_ffn_residual(desc, r, T, k, topk_idx, topk_w, blob_index,
                                r_out, out_bf16, ws, ws_bytes, stream);
}

extern "C" moe_status moe_get_device_status(void* ws, int32_t* host_err,
                                            void* stream) {
  MOE_TRACE();
  if (!ws) return MOE_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  int32_t v = 0;
  MOE_CUDA_TRY(cudaMemcpyAsync(&v, ws, 4, cudaMemcpyDeviceToHost, s));
  MOE_CUDA_TRY(cudaStreamSynchronize(s));
  if (v != 0) MOE_CUDA_TRY(cudaMemsetAsync(ws, 0, 4, s));
  if (host_err) *host_err = v;
  return v ? MOE_ERR_DEVICE : MOE_OK;
}
