// C ABI of libmoe_b200: argument checks, workspace layout and the launch
// sequence of the MoE layer forward pass.  Every compute step runs in the
// kernels of this library; this file only validates and enqueues.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "internal.h"
#include "moe.h"

namespace moe {

// Device error word (MOE_DEVERR_* bits), one per device that loads the library.
__device__ int g_moe_device_error;

namespace {

constexpr int kMaxDevices = 64;
Ctx g_ctx[kMaxDevices];
std::mutex g_ctx_mu;

// Driver entry points that identify the current context (resolved once).
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);
CtxGetCurrentFn g_ctx_get_current = nullptr;
CtxGetIdFn g_ctx_get_id = nullptr;
std::once_flag g_ctx_fn_once;

void resolve_ctx_fns() {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(p);
  p = nullptr;
  if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_ctx_get_id = reinterpret_cast<CtxGetIdFn>(p);
  (void)cudaGetLastError();
}

// Device facts of the current device, cached per device and context: the
// symbol lookup also makes the device's primary context current if it was not.
moe_status_t get_ctx(Ctx& out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_ctx_mu);
  Ctx& c = g_ctx[dev];
  unsigned long long id = 0;
  if (c.dev != dev || !current_context_id(&id) || id != c.ctx_id) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return MOE_ERR_CUDA;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_moe_device_error) != cudaSuccess) return MOE_ERR_CUDA;
    if (!current_context_id(&id)) return MOE_ERR_CUDA;
    c.num_sms = sms;
    c.err = static_cast<int*>(p);
    c.dev = dev;
    c.ctx_id = id;
  }
  out = c;
  return MOE_OK;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t esize(const moe_config_t& c) { return c.dtype == MOE_BF16 ? 2 : 4; }

moe_status_t check_config(const moe_config_t* cfg) {
  if (!cfg) return MOE_ERR_INVALID_ARG;
  const moe_config_t& c = *cfg;
  if (c.T < 0 || c.d <= 0 || c.f <= 0 || c.reserved != 0) return MOE_ERR_INVALID_ARG;
  if (!(c.capacity_factor > 0.0)) return MOE_ERR_INVALID_ARG;  // rejects NaN too
  if (c.dtype != MOE_F32 && c.dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (c.E != 8 || c.top_k != 2) return MOE_ERR_UNSUPPORTED;
  if (c.T > (int64_t)1 << 24 || c.d > (int64_t)1 << 20 || c.f > (int64_t)1 << 20) return MOE_ERR_UNSUPPORTED;
  const int64_t mult = c.dtype == MOE_BF16 ? 128 : 64;
  if (c.d % mult != 0 || c.f % mult != 0) return MOE_ERR_UNSUPPORTED;
  if (c.dtype == MOE_F32 && (slot_rows(c) + 63) / 64 + 8 > 65535) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

// ceil(cf * T * k / E) in double, in that order; never more than T, which no
// expert can exceed anyway (a token reaches an expert at most once).
int64_t capacity_of(const moe_config_t& c) {
  if (isinf(c.capacity_factor)) return c.T;
  const double v = ceil(c.capacity_factor * (double)(c.T * c.top_k) / (double)c.E);
  if (v >= (double)c.T) return c.T;
  return (int64_t)v;
}

size_t round_up(size_t v) { return (v + 255) & ~(size_t)255; }

// Scratch of moe_dispatch: per-block expert histograms.
size_t dispatch_ws(const moe_config_t& c) { return round_up((size_t)dispatch_blocks(c) * c.E * sizeof(int32_t)); }

// Workspace of moe_layer_forward, carved in this order.
struct Layout {
  size_t topk_idx, topk_w, route, perm, slot_of, row_scale, disp, x_perm, h, y, x_in, out, total;
};

Layout layout_of(const moe_config_t& c) {
  Layout L;
  const size_t rows = (size_t)slot_rows(c);
  size_t o = 0;
  auto take = [&](size_t bytes) {
    size_t at = o;
    o += round_up(bytes);
    return at;
  };
  L.topk_idx = take(rows * 4);
  L.topk_w = take(rows * 4);
  L.route = take((size_t)(3 * c.E + 2 + 8) * 4);  // counts_raw, counts_kept, offsets, stats
  L.perm = take(rows * 4);
  L.slot_of = take(rows * 4);
  L.row_scale = take(rows * 4);
  L.disp = take(dispatch_ws(c));
  L.x_perm = take(rows * c.d * esize(c));
  L.h = take(rows * c.f * esize(c));
  L.y = take(rows * c.d * 4);
  L.x_in = take((size_t)c.T * c.d * esize(c));
  L.out = take((size_t)c.T * c.d * esize(c));
  L.total = o;
  return L;
}

moe_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// Batches averaging at most 64 rows per expert stream the expert weights
// rather than reuse them; they run on the kernel that puts the weights on
// the MMA's M side and spends no tensor time on padded token rows.
bool weight_streaming(const moe_config_t& c) { return c.T * (int64_t)c.top_k <= 64 * (int64_t)c.E; }

// The one-call bf16 layer with row-major tensor-core tiles runs the down pass
// with the combine fused (the Y region holds the fp32 sums: T*d <= T*k*d).
bool fused_layer(const moe_config_t& c) {
  return c.dtype == MOE_BF16 && !weight_streaming(c) && c.d % 256 == 0 && c.top_k == 2;
}

moe_status_t run_gate_up(const moe_config_t& c, const void* x_perm, const int32_t* offsets, const void* wg,
                         const void* wu, void* h, cudaStream_t s, const Ctx& ctx) {
  if (c.dtype == MOE_BF16 && weight_streaming(c))
    return cuda_status(launch_decode_gate_up(c, x_perm, offsets, wg, wu, h, s, ctx));
  if (c.dtype == MOE_BF16) return cuda_status(launch_tc_gate_up(c, x_perm, offsets, wg, wu, h, s, ctx));
  return cuda_status(launch_ffn_simt_gate_up(c, static_cast<const float*>(x_perm), offsets,
                                             static_cast<const float*>(wg), static_cast<const float*>(wu),
                                             static_cast<float*>(h), s, ctx));
}

moe_status_t run_down(const moe_config_t& c, const void* h, const int32_t* offsets, const void* wd,
                      const float* row_scale, float* y, cudaStream_t s, const Ctx& ctx) {
  if (c.dtype == MOE_BF16 && weight_streaming(c))
    return cuda_status(launch_decode_down(c, h, offsets, wd, row_scale, y, s, ctx));
  if (c.dtype == MOE_BF16) return cuda_status(launch_tc_down(c, h, offsets, wd, row_scale, y, s, ctx));
  return cuda_status(launch_ffn_simt_down(c, static_cast<const float*>(h), offsets, static_cast<const float*>(wd),
                                          row_scale, y, s, ctx));
}

}  // namespace

bool current_context_id(unsigned long long* id) {
  std::call_once(g_ctx_fn_once, resolve_ctx_fns);
  CUcontext c = nullptr;
  return g_ctx_get_current && g_ctx_get_id && g_ctx_get_current(&c) == CUDA_SUCCESS && c != nullptr &&
         g_ctx_get_id(c, id) == CUDA_SUCCESS;
}

moe_status_t validate_config(const moe_config_t* cfg) { return check_config(cfg); }

moe_status_t current_ctx(Ctx& out) { return get_ctx(out); }

bool encode_tmap(CUtensorMap* map, const void* base, int rank, const uint64_t* dims, const uint64_t* strides_bytes,
                 const uint32_t* box, CUtensorMapSwizzle swz) {
  return encode_tmap_dtype(map, base, rank, dims, strides_bytes, box, swz, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
}

bool encode_tmap_dtype(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                       const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swz,
                       CUtensorMapDataType dtype) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gd[5], gs[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i + 1 < rank; ++i) gs[i] = strides_bytes[i];
  CUresult r = fn(map, dtype, (cuuint32_t)rank, const_cast<void*>(base), gd, gs, bx, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace moe

using namespace moe;

extern "C" {

int32_t moe_abi_version(void) { return 1; }

const char* moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_DEVICE_CHECK: return "MOE_ERR_DEVICE_CHECK";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
  }
  return "MOE_ERR_UNKNOWN";
}

int64_t moe_capacity(const moe_config_t* cfg) {
  if (check_config(cfg) != MOE_OK) return -1;
  return capacity_of(*cfg);
}

size_t moe_dispatch_workspace_size(const moe_config_t* cfg) {
  if (check_config(cfg) != MOE_OK) return 0;
  return dispatch_ws(*cfg);
}

size_t moe_expert_ffn_workspace_size(const moe_config_t* cfg) {
  if (check_config(cfg) != MOE_OK) return 0;
  return 0;
}

size_t moe_workspace_size(const moe_config_t* cfg) {
  if (check_config(cfg) != MOE_OK) return 0;
  return layout_of(*cfg).total;
}

moe_status_t moe_router_topk(const moe_config_t* cfg, const void* x, const void* w_router, const float* logit_bias,
                             float* logits, int32_t* topk_idx, float* topk_w, moe_stream_t stream) {
  Range range_("moe_router_topk");
  moe_status_t st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;
  if (!x || !w_router || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_router) || !aligned16(topk_idx) || !aligned16(topk_w) ||
      (logits && !aligned16(logits)) || (logit_bias && !aligned16(logit_bias)))
    return MOE_ERR_INVALID_ARG;
  Ctx ctx;
  if ((st = get_ctx(ctx)) != MOE_OK) return st;
  return cuda_status(launch_router(*cfg, x, w_router, logit_bias, logits, topk_idx, topk_w, stream, ctx));
}

moe_status_t moe_dispatch(const moe_config_t* cfg, const void* x, const int32_t* topk_idx, const float* topk_w,
                          int32_t* counts_raw, int32_t* counts_kept, int32_t* offsets, int32_t* perm, int32_t* slot_of,
                          float* row_scale, void* x_perm, void* ws, size_t ws_bytes, moe_stream_t stream) {
  Range range_("moe_dispatch");
  moe_status_t st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (!topk_idx || !topk_w || !counts_raw || !counts_kept || !offsets || !perm || !slot_of || !row_scale)
    return MOE_ERR_INVALID_ARG;
  if (x_perm && !x) return MOE_ERR_INVALID_ARG;
  if (!aligned16(topk_idx) || !aligned16(topk_w) || !aligned16(slot_of) || (x_perm && !aligned16(x_perm)) ||
      (x && !aligned16(x)))
    return MOE_ERR_INVALID_ARG;
  if (ws_bytes < dispatch_ws(*cfg) || (dispatch_ws(*cfg) > 0 && !ws)) return MOE_ERR_WORKSPACE;
  Ctx ctx;
  if ((st = get_ctx(ctx)) != MOE_OK) return st;
  const moe_config_t& c = *cfg;
  cudaError_t e = launch_dispatch(c, capacity_of(c), topk_idx, topk_w, counts_raw, counts_kept, offsets, perm,
                                  slot_of, row_scale, static_cast<int32_t*>(ws), nullptr, stream, ctx);
  if (e == cudaSuccess && x_perm && c.T > 0) e = launch_gather(c, x, perm, offsets, x_perm, stream, ctx);
  return cuda_status(e);
}

moe_status_t moe_gather_rows(const void* src, int64_t n_src, const int32_t* idx, int64_t n, int64_t row_bytes,
                             void* dst, moe_stream_t stream) {
  Range range_("moe_gather_rows");
  if (n < 0 || n_src < 0 || row_bytes <= 0 || row_bytes % 16 != 0 || n > ((int64_t)1 << 31) ||
      n_src > ((int64_t)1 << 31))
    return MOE_ERR_INVALID_ARG;
  if (n == 0) return MOE_OK;
  if (!src || !idx || !dst || !aligned16(src) || !aligned16(dst)) return MOE_ERR_INVALID_ARG;
  Ctx ctx;
  moe_status_t st = get_ctx(ctx);
  if (st != MOE_OK) return st;
  return cuda_status(launch_gather_index(src, idx, n, n_src, row_bytes, dst, stream, ctx));
}

moe_status_t moe_route_counts(const moe_config_t* cfg, const int32_t* topk_idx, int32_t* counts,
                              moe_stream_t stream) {
  moe_status_t st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (!counts || (cfg->T > 0 && (!topk_idx || !aligned16(topk_idx)))) return MOE_ERR_INVALID_ARG;
  Ctx ctx;
  if ((st = get_ctx(ctx)) != MOE_OK) return st;
  return cuda_status(launch_route_counts(*cfg, topk_idx, counts, stream, ctx));
}

moe_status_t moe_dispatch_shard(const moe_config_t* cfg, int64_t capacity, const int32_t* shard_counts,
                                int32_t n_shards, int32_t shard, const void* x, const int32_t* topk_idx,
                                const float* topk_w, int32_t* counts_raw, int32_t* counts_kept, int32_t* offsets,
                                int32_t* perm, int32_t* slot_of, float* row_scale, void* x_perm, void* ws,
                                size_t ws_bytes, moe_stream_t stream) {
  Range range_("moe_dispatch_shard");
  moe_status_t st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (capacity < 0 || n_shards < 1 || shard < 0 || shard >= n_shards || !shard_counts) return MOE_ERR_INVALID_ARG;
  if (!topk_idx || !topk_w || !counts_raw || !counts_kept || !offsets || !perm || !slot_of || !row_scale)
    return MOE_ERR_INVALID_ARG;
  if (x_perm && !x) return MOE_ERR_INVALID_ARG;
  if (!aligned16(topk_idx) || !aligned16(topk_w) || !aligned16(slot_of) || (x_perm && !aligned16(x_perm)) ||
      (x && !aligned16(x)))
    return MOE_ERR_INVALID_ARG;
  if (ws_bytes < dispatch_ws(*cfg) || (dispatch_ws(*cfg) > 0 && !ws)) return MOE_ERR_WORKSPACE;
  Ctx ctx;
  if ((st = get_ctx(ctx)) != MOE_OK) return st;
  const moe_config_t& c = *cfg;
  cudaError_t e = launch_dispatch(c, capacity, topk_idx, topk_w, counts_raw, counts_kept, offsets, perm, slot_of,
                                  row_scale, static_cast<int32_t*>(ws), nullptr, stream, ctx, shard_counts, shard);
  if (e == cudaSuccess && x_perm && c.T > 0) e = launch_gather(c, x, perm, offsets, x_perm, stream, ctx);
  return cuda_status(e);
}

moe_status_t moe_expert_gate_up(const moe_config_t* cfg, const void* x_perm, const int32_t* offsets,
                                const void* w_gate, const void* w_up, void* h, moe_stream_t stream) {
  Range range_("moe_expert_gate_up");
  moe_status_t st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;
  if (!x_perm || !offsets || !w_gate || !w_up || !h) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x_perm) || !aligned16(w_gate) || !aligned16(w_up) || !aligned16(h)) return MOE_ERR_INVALID_ARG;
  Ctx ctx;
  if ((st = get_ctx(ctx)) != MOE_OK) return st;
  return run_gate_up(*cfg, x_perm, offsets, w_gate, w_up, h, stream, ctx);
}

moe_status_t moe_expert_down(const moe_config_t* cfg, const void* h, const int32_t* offsets, const void* w_down,
                             const float* row_scale, float* y, void* ws, size_t ws_bytes, moe_stream_t stream) {
  Range range_("moe_expert_down");
  (void)ws;
  (void)ws_bytes;
  moe_status_t st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;
  if (!h || !offsets || !w_down || !y) return MOE_ERR_INVALID_ARG;
  if (!aligned16(h) || !aligned16(w_down) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  Ctx ctx;
  if ((st = get_ctx(ctx)) != MOE_OK) return st;
  return run_down(*cfg, h, offsets, w_down, row_scale, y, stream, ctx);
}

size_t moe_expert_down_combine_workspace_size(const moe_config_t* cfg) {
  if (check_config(cfg) != MOE_OK) return 0;
  return round_up((size_t)cfg->T * cfg->d * 4);
}

moe_status_t moe_expert_down_combine(const moe_config_t* cfg, const void* h, const int32_t* offsets,
                                     const void* w_down, const float* row_scale, const int32_t* perm, void* out,
                                     void* ws, size_t ws_bytes, moe_stream_t stream) {
  Range range_("moe_expert_down_combine");
  moe_status_t st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;
  if (!fused_layer(*cfg)) return MOE_ERR_UNSUPPORTED;
  if (!h || !offsets || !w_down || !perm || !out) return MOE_ERR_INVALID_ARG;
  if (!aligned16(h) || !aligned16(w_down) || !aligned16(out) || (row_scale && !aligned16(row_scale)))
    return MOE_ERR_INVALID_ARG;
  if (!ws || ws_bytes < moe_expert_down_combine_workspace_size(cfg)) return MOE_ERR_WORKSPACE;
  if (!aligned16(ws)) return MOE_ERR_INVALID_ARG;
  Ctx ctx;
  if ((st = get_ctx(ctx)) != MOE_OK) return st;
  float* out32 = static_cast<float*>(ws);
  cudaError_t e = launch_zero_rows(*cfg, out32, stream, ctx);
  if (e == cudaSuccess) e = launch_tc_down_scatter(*cfg, h, offsets, w_down, row_scale, perm, out32, stream, ctx);
  if (e == cudaSuccess) e = launch_round_out(*cfg, out32, out, stream, ctx);
  return cuda_status(e);
}

moe_status_t moe_expert_ffn(const moe_config_t* cfg, const void* x_perm, const int32_t* offsets, const void* w_gate,
                            const void* w_up, const void* w_down, const float* row_scale, void* h, float* y, void* ws,
                            size_t ws_bytes, moe_stream_t stream) {
  moe_status_t st = moe_expert_gate_up(cfg, x_perm, offsets, w_gate, w_up, h, stream);
  if (st != MOE_OK) return st;
  return moe_expert_down(cfg, h, offsets, w_down, row_scale, y, ws, ws_bytes, stream);
}

moe_status_t moe_combine(const moe_config_t* cfg, const float* y, const int32_t* slot_of, const float* topk_w,
                         int32_t weights_applied, void* out, moe_stream_t stream) {
  Range range_("moe_combine");
  moe_status_t st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;
  if (!y || !slot_of || !out || (!weights_applied && !topk_w)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(y) || !aligned16(slot_of) || !aligned16(out) || (topk_w && !aligned16(topk_w)))
    return MOE_ERR_INVALID_ARG;
  Ctx ctx;
  if ((st = get_ctx(ctx)) != MOE_OK) return st;
  return cuda_status(launch_combine(*cfg, y, slot_of, topk_w, weights_applied, out, stream, ctx));
}

static moe_status_t layer_forward_impl(const moe_config_t& c, const void* x, const void* w_router,
                                       const float* logit_bias, const void* w_gate, const void* w_up,
                                       const void* w_down, void* out, int32_t* stats, uint8_t* ws, cudaStream_t s,
                                       const Ctx& ctx) {
  const Layout L = layout_of(c);
  int32_t* topk_idx = reinterpret_cast<int32_t*>(ws + L.topk_idx);
  float* topk_w = reinterpret_cast<float*>(ws + L.topk_w);
  int32_t* route = reinterpret_cast<int32_t*>(ws + L.route);
  int32_t* counts_raw = route;
  int32_t* counts_kept = route + c.E;
  int32_t* offsets = route + 2 * c.E;
  int32_t* perm = reinterpret_cast<int32_t*>(ws + L.perm);
  int32_t* slot_of = reinterpret_cast<int32_t*>(ws + L.slot_of);
  float* row_scale = reinterpret_cast<float*>(ws + L.row_scale);
  int32_t* disp = reinterpret_cast<int32_t*>(ws + L.disp);
  void* x_perm = ws + L.x_perm;
  void* h = ws + L.h;
  float* y = reinterpret_cast<float*>(ws + L.y);

  cudaError_t e = launch_router(c, x, w_router, logit_bias, nullptr, topk_idx, topk_w, s, ctx);
  if (e == cudaSuccess)
    e = launch_dispatch(c, capacity_of(c), topk_idx, topk_w, counts_raw, counts_kept, offsets, perm, slot_of,
                        row_scale, disp, stats, s, ctx);
  if (e == cudaSuccess) e = launch_gather(c, x, perm, offsets, x_perm, s, ctx);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  if (fused_layer(c)) {
    // down accumulates straight into out32 by token (in the Y region, which this
    // path does not use); one rounding pass writes out
    float* out32 = y;
    e = launch_zero_rows(c, out32, s, ctx);
    if (e == cudaSuccess) e = launch_tc_gate_up(c, x_perm, offsets, w_gate, w_up, h, s, ctx);
    if (e == cudaSuccess) e = launch_tc_down_scatter(c, h, offsets, w_down, row_scale, perm, out32, s, ctx);
    if (e == cudaSuccess) e = launch_round_out(c, out32, out, s, ctx);
    return cuda_status(e);
  }
  moe_status_t st = run_gate_up(c, x_perm, offsets, w_gate, w_up, h, s, ctx);
  if (st == MOE_OK) st = run_down(c, h, offsets, w_down, row_scale, y, s, ctx);
  if (st == MOE_OK) st = cuda_status(launch_combine(c, y, slot_of, topk_w, 1, out, s, ctx));
  return st;
}

static moe_status_t check_layer_args(const moe_config_t* cfg, const void* w_router, const float* logit_bias,
                                     const void* w_gate, const void* w_up, const void* w_down, void* ws,
                                     size_t ws_bytes) {
  moe_status_t st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (!w_router || !w_gate || !w_up || !w_down) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w_router) || !aligned16(w_gate) || !aligned16(w_up) || !aligned16(w_down) ||
      (logit_bias && !aligned16(logit_bias)))
    return MOE_ERR_INVALID_ARG;
  if (cfg->T > 0 && (!ws || ws_bytes < layout_of(*cfg).total)) return MOE_ERR_WORKSPACE;
  if (ws && !aligned16(ws)) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

moe_status_t moe_layer_forward(const moe_config_t* cfg, const void* x, const void* w_router, const float* logit_bias,
                               const void* w_gate, const void* w_up, const void* w_down, void* out, int32_t* stats,
                               void* ws, size_t ws_bytes, moe_stream_t stream) {
  Range range_("moe_layer_forward");
  moe_status_t st = check_layer_args(cfg, w_router, logit_bias, w_gate, w_up, w_down, ws, ws_bytes);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;
  if (!x || !out || !aligned16(x) || !aligned16(out) || (stats && !aligned16(stats))) return MOE_ERR_INVALID_ARG;
  Ctx ctx;
  if ((st = get_ctx(ctx)) != MOE_OK) return st;
  return layer_forward_impl(*cfg, x, w_router, logit_bias, w_gate, w_up, w_down, out, stats,
                            static_cast<uint8_t*>(ws), stream, ctx);
}

moe_status_t moe_layer_forward_host(const moe_config_t* cfg, const void* x_host, const void* w_router,
                                    const float* logit_bias, const void* w_gate, const void* w_up, const void* w_down,
                                    void* out_host, void* ws, size_t ws_bytes, moe_stream_t stream) {
  Range range_("moe_layer_forward_host");
  moe_status_t st = check_layer_args(cfg, w_router, logit_bias, w_gate, w_up, w_down, ws, ws_bytes);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;
  if (!x_host || !out_host) return MOE_ERR_INVALID_ARG;
  Ctx ctx;
  if ((st = get_ctx(ctx)) != MOE_OK) return st;
  const moe_config_t& c = *cfg;
  const Layout L = layout_of(c);
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  const size_t bytes = (size_t)c.T * c.d * esize(c);
  if (cudaMemcpyAsync(w8 + L.x_in, x_host, bytes, cudaMemcpyHostToDevice, stream) != cudaSuccess)
    return MOE_ERR_CUDA;
  st = layer_forward_impl(c, w8 + L.x_in, w_router, logit_bias, w_gate, w_up, w_down, w8 + L.out, nullptr, w8,
                          stream, ctx);
  if (st != MOE_OK) return st;
  if (cudaMemcpyAsync(out_host, w8 + L.out, bytes, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return MOE_ERR_CUDA;
  return cuda_status(cudaStreamSynchronize(stream));
}

size_t moe_workspace_size_host_batches(const moe_config_t* cfg) {
  if (check_config(cfg) != MOE_OK) return 0;
  return layout_of(*cfg).total + 2 * round_up((size_t)cfg->T * cfg->d * esize(*cfg));
}

}  // extern "C"

namespace moe {
namespace {
// The copy streams and events of moe_layer_forward_host_batches, created on a
// device's first call and kept for the process (re-created when the device's
// context changes, e.g. after cudaDeviceReset: the old handles died with it).
// A call holds its device's lock from start to end (the call waits for its own
// copies), so calls from several host threads on one device take turns.
struct CopyPipe {
  std::mutex mu;
  bool ready = false;
  unsigned long long ctx_id = 0;
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t ev[7] = {};  // start, xin[2], comp[2], outfree[2]
};
CopyPipe g_pipes[kMaxDevices];

// With the pipe's lock held: makes sure its streams and events exist in the current context.
bool pipe_ready(CopyPipe& p, const Ctx& ctx) {
  if (p.ready && p.ctx_id == ctx.ctx_id) return true;
  p.ready = false;
  p.h2d = p.d2h = nullptr;
  for (cudaEvent_t& e : p.ev) e = nullptr;
  bool ok = cudaStreamCreateWithFlags(&p.h2d, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&p.d2h, cudaStreamNonBlocking) == cudaSuccess;
  for (int i = 0; ok && i < 7; ++i) ok = cudaEventCreateWithFlags(&p.ev[i], cudaEventDisableTiming) == cudaSuccess;
  if (!ok) {
    for (cudaEvent_t e : p.ev)
      if (e) cudaEventDestroy(e);
    if (p.h2d) cudaStreamDestroy(p.h2d);
    if (p.d2h) cudaStreamDestroy(p.d2h);
    p.h2d = p.d2h = nullptr;
    for (cudaEvent_t& e : p.ev) e = nullptr;
    (void)cudaGetLastError();
    return false;
  }
  p.ctx_id = ctx.ctx_id;
  p.ready = true;
  return true;
}
}  // namespace
}  // namespace moe

extern "C" {

// Two-slot copy/compute pipeline: batch i uses staging slot i % 2 (x and out).
//   h2d stream : wait comp[s] (batch i-2 done with slot s), copy x_host[i] -> x slot, record xin[s]
//   stream     : wait xin[s] and outfree[s] (batch i-2's result copied out), layer, record comp[s]
//   d2h stream : wait comp[s], copy out slot -> out_host[i], record outfree[s]
// Enqueued in that order for each i, so batch i+1's copy-in and batch i-1's
// copy-out run while batch i computes.  cudaStreamWaitEvent binds the event's
// latest record at enqueue time, which is always the batch two steps back.
moe_status_t moe_layer_forward_host_batches(const moe_config_t* cfg, int64_t n_batches, const void* const* x_host,
                                            const void* w_router, const float* logit_bias, const void* w_gate,
                                            const void* w_up, const void* w_down, void* const* out_host, void* ws,
                                            size_t ws_bytes, moe_stream_t stream) {
  Range range_("moe_layer_forward_host_batches");
  moe_status_t st = check_layer_args(cfg, w_router, logit_bias, w_gate, w_up, w_down, ws, ws_bytes);
  if (st != MOE_OK) return st;
  if (n_batches < 0) return MOE_ERR_INVALID_ARG;
  if (n_batches == 0 || cfg->T == 0) return MOE_OK;
  if (!x_host || !out_host) return MOE_ERR_INVALID_ARG;
  for (int64_t i = 0; i < n_batches; ++i)
    if (!x_host[i] || !out_host[i]) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < moe_workspace_size_host_batches(cfg)) return MOE_ERR_WORKSPACE;
  Ctx ctx;
  if ((st = get_ctx(ctx)) != MOE_OK) return st;
  const moe_config_t& c = *cfg;
  const Layout L = layout_of(c);
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  const size_t bytes = (size_t)c.T * c.d * esize(c);
  uint8_t* x_slot[2] = {w8 + L.x_in, w8 + L.total};
  uint8_t* out_slot[2] = {w8 + L.out, w8 + L.total + round_up(bytes)};

  CopyPipe& pipe = g_pipes[ctx.dev];
  std::lock_guard<std::mutex> pipe_lock(pipe.mu);
  if (!pipe_ready(pipe, ctx)) return MOE_ERR_CUDA;
  cudaStream_t h2d = pipe.h2d, d2h = pipe.d2h;
  cudaEvent_t* ev = pipe.ev;
  cudaEvent_t &start = ev[0], *xin = ev + 1, *comp = ev + 3, *outfree = ev + 5;
  // the whole pipeline starts after the work already in `stream`
  bool ok = cudaEventRecord(start, stream) == cudaSuccess && cudaStreamWaitEvent(h2d, start, 0) == cudaSuccess &&
       cudaStreamWaitEvent(d2h, start, 0) == cudaSuccess;
  for (int64_t i = 0; ok && i < n_batches; ++i) {
    const int sl = (int)(i & 1);
    if (i >= 2) ok = cudaStreamWaitEvent(h2d, comp[sl], 0) == cudaSuccess;
    ok = ok && cudaMemcpyAsync(x_slot[sl], x_host[i], bytes, cudaMemcpyHostToDevice, h2d) == cudaSuccess &&
         cudaEventRecord(xin[sl], h2d) == cudaSuccess && cudaStreamWaitEvent(stream, xin[sl], 0) == cudaSuccess;
    if (ok && i >= 2) ok = cudaStreamWaitEvent(stream, outfree[sl], 0) == cudaSuccess;
    if (!ok) break;
    st = layer_forward_impl(c, x_slot[sl], w_router, logit_bias, w_gate, w_up, w_down, out_slot[sl], nullptr, w8,
                            stream, ctx);
    if (st != MOE_OK) break;
    ok = cudaEventRecord(comp[sl], stream) == cudaSuccess && cudaStreamWaitEvent(d2h, comp[sl], 0) == cudaSuccess &&
         cudaMemcpyAsync(out_host[i], out_slot[sl], bytes, cudaMemcpyDeviceToHost, d2h) == cudaSuccess &&
         cudaEventRecord(outfree[sl], d2h) == cudaSuccess;
  }
  // later work in `stream` is ordered after the last copy-out; then wait for all of it
  if (ok && st == MOE_OK) ok = cudaEventRecord(start, d2h) == cudaSuccess && cudaStreamWaitEvent(stream, start, 0) == cudaSuccess;
  cudaError_t sync = cudaStreamSynchronize(d2h);
  if (sync == cudaSuccess) sync = cudaStreamSynchronize(h2d);
  if (sync == cudaSuccess) sync = cudaStreamSynchronize(stream);
  if (st != MOE_OK) return st;
  if (!ok) return MOE_ERR_CUDA;
  return cuda_status(sync);
}

moe_status_t moe_quantize_int8(const moe_config_t* cfg, const void* w, int64_t K, int64_t N, int8_t* q, float* scale,
                               moe_stream_t stream) {
  Range range_("moe_quantize_int8");
  moe_status_t st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (cfg->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (K <= 0 || N <= 0 || K > ((int64_t)1 << 20) || N > ((int64_t)1 << 20)) return MOE_ERR_INVALID_ARG;
  if (N % 64 != 0) return MOE_ERR_UNSUPPORTED;
  if (!w || !q || !scale || !aligned16(w) || !aligned16(q) || !aligned16(scale)) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_quantize_int8(cfg->E, w, K, N, q, scale, stream));
}

static moe_status_t check_w8(const moe_config_t* cfg, const void* qg, const float* sg, const void* qu,
                             const float* su, const void* qd, const float* sd) {
  moe_status_t st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (cfg->dtype != MOE_BF16 || cfg->d % 256 != 0) return MOE_ERR_UNSUPPORTED;
  if (!qg || !sg || !qu || !su || !qd || !sd) return MOE_ERR_INVALID_ARG;
  if (!aligned16(qg) || !aligned16(qu) || !aligned16(qd) || !aligned16(sg) || !aligned16(su) || !aligned16(sd))
    return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

}  // extern "C"

namespace moe {
namespace {

// Scratch of the int8-weight expert FFN, carved in this order:
// row codes of x_perm (hi, lo planes and per-row scales), H in fp32, row codes of H.
struct W8Layout {
  size_t x_hi, x_lo, x_scale, h, h_hi, h_lo, h_scale, y_parts, total;
};

W8Layout w8_layout_of(const moe_config_t& c) {
  W8Layout L;
  const size_t rows = (size_t)slot_rows(c);
  size_t o = 0;
  auto take = [&](size_t bytes) {
    size_t at = o;
    o += round_up(bytes);
    return at;
  };
  L.x_hi = take(rows * c.d);
  L.x_lo = take(rows * c.d);
  L.x_scale = take(rows * 4);
  L.h = take(rows * c.f * 4);
  L.h_hi = take(rows * c.f);
  L.h_lo = take(rows * c.f);
  L.h_scale = take(rows * 4);
  L.y_parts = take((rows > 64 * (size_t)c.E ? 1 : kMaxDownSplits) * rows * c.d * 4);
  L.total = o;
  return L;
}

// x_rows: x_perm, or (with perm) x itself read by slot; y == nullptr leaves the
// down pass's K-split partials unsummed (the layer's combine adds them in order).
cudaError_t run_ffn_w8(const moe_config_t& c, const void* x_rows, const int32_t* offsets, const int8_t* qg,
                       const float* sg, const int8_t* qu, const float* su, const int8_t* qd, const float* sd,
                       const float* row_scale, float* y, uint8_t* ws, cudaStream_t s, const Ctx& ctx,
                       const int32_t* perm = nullptr) {
  const W8Layout L = w8_layout_of(c);
  const int64_t rows = slot_rows(c);
  int8_t* x_hi = reinterpret_cast<int8_t*>(ws + L.x_hi);
  int8_t* x_lo = reinterpret_cast<int8_t*>(ws + L.x_lo);
  float* x_sc = reinterpret_cast<float*>(ws + L.x_scale);
  float* h = reinterpret_cast<float*>(ws + L.h);
  int8_t* h_hi = reinterpret_cast<int8_t*>(ws + L.h_hi);
  int8_t* h_lo = reinterpret_cast<int8_t*>(ws + L.h_lo);
  float* h_sc = reinterpret_cast<float*>(ws + L.h_scale);
  cudaError_t e = launch_quantize_rows(x_rows, false, offsets, rows, c.d, x_hi, x_lo, x_sc, ctx.num_sms, s, perm, c.T,
                                       ctx.err);
  if (e == cudaSuccess) e = launch_i8_gate_up(c, x_hi, x_lo, x_sc, offsets, qg, sg, qu, su, h, s, ctx);
  if (e == cudaSuccess) e = launch_quantize_rows(h, true, offsets, rows, c.f, h_hi, h_lo, h_sc, ctx.num_sms, s);
  float* y_parts = reinterpret_cast<float*>(ws + L.y_parts);
  if (e == cudaSuccess) e = launch_i8_down(c, h_hi, h_lo, h_sc, offsets, qd, sd, row_scale, y_parts, s, ctx);
  if (e == cudaSuccess && y) e = launch_sum_partials(c, y_parts, offsets, y, s, ctx);
  return e;
}

// The K-split partials of the 8-bit down pass, for a combine that sums them.
const float* w8_partials(const moe_config_t& c, const uint8_t* ws) {
  return reinterpret_cast<const float*>(ws + w8_layout_of(c).y_parts);
}

}  // namespace
}  // namespace moe

extern "C" {

size_t moe_expert_ffn_w8_workspace_size(const moe_config_t* cfg) {
  if (check_config(cfg) != MOE_OK) return 0;
  return w8_layout_of(*cfg).total;
}

size_t moe_workspace_size_w8(const moe_config_t* cfg) {
  if (check_config(cfg) != MOE_OK) return 0;
  return layout_of(*cfg).total + w8_layout_of(*cfg).total;
}

moe_status_t moe_expert_ffn_w8(const moe_config_t* cfg, const void* x_perm, const int32_t* offsets,
                               const int8_t* q_gate, const float* s_gate, const int8_t* q_up, const float* s_up,
                               const int8_t* q_down, const float* s_down, const float* row_scale, float* y, void* ws,
                               size_t ws_bytes, moe_stream_t stream) {
  Range range_("moe_expert_ffn_w8");
  moe_status_t st = check_w8(cfg, q_gate, s_gate, q_up, s_up, q_down, s_down);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;
  if (!x_perm || !offsets || !y || !aligned16(x_perm) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  if (!ws || !aligned16(ws) || ws_bytes < w8_layout_of(*cfg).total) return MOE_ERR_WORKSPACE;
  Ctx ctx;
  if ((st = get_ctx(ctx)) != MOE_OK) return st;
  return cuda_status(run_ffn_w8(*cfg, x_perm, offsets, q_gate, s_gate, q_up, s_up, q_down, s_down, row_scale, y,
                                static_cast<uint8_t*>(ws), stream, ctx));
}

moe_status_t moe_layer_forward_w8(const moe_config_t* cfg, const void* x, const void* w_router,
                                  const float* logit_bias, const int8_t* q_gate, const float* s_gate,
                                  const int8_t* q_up, const float* s_up, const int8_t* q_down, const float* s_down,
                                  void* out, int32_t* stats, void* ws, size_t ws_bytes, moe_stream_t stream) {
  Range range_("moe_layer_forward_w8");
  moe_status_t st = check_w8(cfg, q_gate, s_gate, q_up, s_up, q_down, s_down);
  if (st != MOE_OK) return st;
  if (!w_router || !aligned16(w_router) || (logit_bias && !aligned16(logit_bias))) return MOE_ERR_INVALID_ARG;
  if (cfg->T == 0) return MOE_OK;
  if (!ws || ws_bytes < moe_workspace_size_w8(cfg) || !aligned16(ws)) return MOE_ERR_WORKSPACE;
  if (!x || !out || !aligned16(x) || !aligned16(out) || (stats && !aligned16(stats))) return MOE_ERR_INVALID_ARG;
  Ctx ctx;
  if ((st = get_ctx(ctx)) != MOE_OK) return st;
  const moe_config_t& c = *cfg;
  const Layout L = layout_of(c);
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  int32_t* topk_idx = reinterpret_cast<int32_t*>(w8 + L.topk_idx);
  float* topk_w = reinterpret_cast<float*>(w8 + L.topk_w);
  int32_t* route = reinterpret_cast<int32_t*>(w8 + L.route);
  int32_t* offsets = route + 2 * c.E;
  int32_t* perm = reinterpret_cast<int32_t*>(w8 + L.perm);
  int32_t* slot_of = reinterpret_cast<int32_t*>(w8 + L.slot_of);
  float* row_scale = reinterpret_cast<float*>(w8 + L.row_scale);
  cudaError_t e = launch_router(c, x, w_router, logit_bias, nullptr, topk_idx, topk_w, stream, ctx);
  if (e == cudaSuccess)
    e = launch_dispatch(c, capacity_of(c), topk_idx, topk_w, route, route + c.E, offsets, perm, slot_of, row_scale,
                        reinterpret_cast<int32_t*>(w8 + L.disp), stats, stream, ctx);
  // x rows are coded straight from x by slot (no x_perm), and the combine adds the
  // down pass's K-split partials itself, in the order the partial sum would
  if (e == cudaSuccess)
    e = run_ffn_w8(c, x, offsets, q_gate, s_gate, q_up, s_up, q_down, s_down, row_scale, nullptr, w8 + L.total,
                   stream, ctx, perm);
  if (e == cudaSuccess)
    e = launch_combine(c, w8_partials(c, w8 + L.total), slot_of, topk_w, 1, out, stream, ctx,
                       down_splits(c, ctx.num_sms), slot_rows(c) * c.d);
  return cuda_status(e);
}

moe_status_t moe_expert_utilization(const int32_t* stats, int32_t E, int64_t* counts, float* utilization,
                                    moe_stream_t stream) {
  Range range_("moe_expert_utilization");
  if (!stats || !counts || !utilization || E < 1 || E > 64) return MOE_ERR_INVALID_ARG;
  Ctx ctx;
  moe_status_t st = get_ctx(ctx);
  if (st != MOE_OK) return st;
  return cuda_status(launch_utilization(stats, E, counts, utilization, stream));
}

moe_status_t moe_check_bounded_wait(int64_t limit_ns, moe_stream_t stream) {
  if (limit_ns < 1000 || limit_ns > 1000000000) return MOE_ERR_INVALID_ARG;
  Ctx ctx;
  moe_status_t st = get_ctx(ctx);
  if (st != MOE_OK) return st;
  return cuda_status(launch_wait_check(limit_ns, stream, ctx));
}

moe_status_t moe_set_gemm_tiles(int32_t mode, int32_t* previous) {
  if (mode != MOE_TILES_AUTO && mode != MOE_TILES_SINGLE && mode != MOE_TILES_PAIR) return MOE_ERR_INVALID_ARG;
  const int prev = set_tile_mode(mode);
  if (previous) *previous = prev;
  return MOE_OK;
}

moe_status_t moe_get_device_error(int32_t* code, int32_t clear) {
  if (!code) return MOE_ERR_INVALID_ARG;
  Ctx ctx;
  moe_status_t st = get_ctx(ctx);
  if (st != MOE_OK) return st;
  if (cudaDeviceSynchronize() != cudaSuccess) return MOE_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, ctx.err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (clear) {
    const int zero = 0;
    if (cudaMemcpy(ctx.err, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return MOE_ERR_CUDA;
  }
  *code = v;
  return v ? MOE_ERR_DEVICE_CHECK : MOE_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------- training
namespace moe {
namespace {

// Workspace of the training pair: the forward's layout, then what the backward
// reads (G, U) and its own scratch.
struct TrainLayout {
  Layout base;
  size_t g, u, dout_perm, dy_perm, dg, du, dw_part, dlogits, dweight, dx32, wr_part, total;
};

TrainLayout train_layout_of(const moe_config_t& c) {
  TrainLayout L;
  L.base = layout_of(c);
  const size_t rows = (size_t)slot_rows(c);
  size_t o = L.base.total;
  auto take = [&](size_t bytes) {
    size_t at = o;
    o += round_up(bytes);
    return at;
  };
  L.g = take(rows * c.f * 2);
  L.u = take(rows * c.f * 2);
  L.dout_perm = take(rows * c.d * 2);
  L.dy_perm = take(rows * c.d * 2);
  L.dg = take(rows * c.f * 2);
  L.du = take(rows * c.f * 2);
  L.dw_part = take(rows * (size_t)(c.f / 256) * bwd_dh_parts_per_tile() * 4);
  L.dlogits = take((size_t)c.T * c.E * 4);
  L.dweight = take((size_t)c.T * c.top_k * 4);
  L.dx32 = take((size_t)c.T * c.d * 4);
  L.wr_part = take((size_t)kRouterBwdChunks * c.E * c.d * 4);
  L.total = o;
  return L;
}

bool train_supported(const moe_config_t& c) {
  return c.dtype == MOE_BF16 && c.d % 256 == 0 && c.f % 256 == 0 && c.top_k == 2;
}

}  // namespace
}  // namespace moe

extern "C" {

size_t moe_workspace_size_train(const moe_config_t* cfg) {
  if (check_config(cfg) != MOE_OK || !train_supported(*cfg)) return 0;
  return train_layout_of(*cfg).total;
}

moe_status_t moe_layer_forward_train(const moe_config_t* cfg, const void* x, const void* w_router,
                                     const float* logit_bias, const void* w_gate, const void* w_up,
                                     const void* w_down, void* out, void* ws, size_t ws_bytes, moe_stream_t stream) {
  Range range_("moe_layer_forward_train");
  moe_status_t st = check_layer_args(cfg, w_router, logit_bias, w_gate, w_up, w_down, ws, ws_bytes);
  if (st != MOE_OK) return st;
  if (!train_supported(*cfg)) return MOE_ERR_UNSUPPORTED;
  if (cfg->T == 0) return MOE_OK;
  if (!x || !out || !aligned16(x) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < moe_workspace_size_train(cfg)) return MOE_ERR_WORKSPACE;
  Ctx ctx;
  if ((st = get_ctx(ctx)) != MOE_OK) return st;
  const moe_config_t& c = *cfg;
  const TrainLayout TL = train_layout_of(c);
  const Layout& L = TL.base;
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  int32_t* topk_idx = reinterpret_cast<int32_t*>(w8 + L.topk_idx);
  float* topk_w = reinterpret_cast<float*>(w8 + L.topk_w);
  int32_t* route = reinterpret_cast<int32_t*>(w8 + L.route);
  int32_t* offsets = route + 2 * c.E;
  int32_t* perm = reinterpret_cast<int32_t*>(w8 + L.perm);
  int32_t* slot_of = reinterpret_cast<int32_t*>(w8 + L.slot_of);
  float* row_scale = reinterpret_cast<float*>(w8 + L.row_scale);
  float* y = reinterpret_cast<float*>(w8 + L.y);
  cudaError_t e;
  {
    PhaseMark m(MOE_PHASE_FWD_ROUTER, stream);
    e = launch_router(c, x, w_router, logit_bias, nullptr, topk_idx, topk_w, stream, ctx);
  }
  if (e == cudaSuccess) {
    PhaseMark m(MOE_PHASE_FWD_DISPATCH, stream);
    e = launch_dispatch(c, capacity_of(c), topk_idx, topk_w, route, route + c.E, offsets, perm, slot_of, row_scale,
                        reinterpret_cast<int32_t*>(w8 + L.disp), nullptr, stream, ctx);
  }
  if (e == cudaSuccess) {
    PhaseMark m(MOE_PHASE_FWD_GATHER, stream);
    e = launch_gather(c, x, perm, offsets, w8 + L.x_perm, stream, ctx);
  }
  // the row-major tensor-core kernels at every batch size: gate/up keeps G and U
  if (e == cudaSuccess) {
    PhaseMark m(MOE_PHASE_FWD_GATE_UP, stream);
    e = launch_tc_gate_up(c, w8 + L.x_perm, offsets, w_gate, w_up, w8 + L.h, stream, ctx, w8 + TL.g, w8 + TL.u);
  }
  if (e == cudaSuccess) {
    PhaseMark m(MOE_PHASE_FWD_DOWN, stream);
    e = launch_tc_down(c, w8 + L.h, offsets, w_down, row_scale, y, stream, ctx);
  }
  if (e == cudaSuccess) {
    PhaseMark m(MOE_PHASE_FWD_COMBINE, stream);
    e = launch_combine(c, y, slot_of, topk_w, 1, out, stream, ctx);
  }
  return cuda_status(e);
}

moe_status_t moe_layer_backward(const moe_config_t* cfg, const void* x, const void* w_router, const void* w_gate,
                                const void* w_up, const void* w_down, const void* dout, void* dx, float* dw_router,
                                float* dbias, float* dw_gate, float* dw_up, float* dw_down, void* ws,
                                size_t ws_bytes, moe_stream_t stream) {
  Range range_("moe_layer_backward");
  moe_status_t st = check_layer_args(cfg, w_router, nullptr, w_gate, w_up, w_down, ws, ws_bytes);
  if (st != MOE_OK) return st;
  if (!train_supported(*cfg)) return MOE_ERR_UNSUPPORTED;
  if (!dw_router || !dw_gate || !dw_up || !dw_down) return MOE_ERR_INVALID_ARG;
  if (!aligned16(dw_router) || !aligned16(dw_gate) || !aligned16(dw_up) || !aligned16(dw_down) ||
      (dbias && !aligned16(dbias)))
    return MOE_ERR_INVALID_ARG;
  if (cfg->T > 0 && (!x || !dout || !dx || !aligned16(x) || !aligned16(dout) || !aligned16(dx)))
    return MOE_ERR_INVALID_ARG;
  if (cfg->T > 0 && ws_bytes < moe_workspace_size_train(cfg)) return MOE_ERR_WORKSPACE;
  Ctx ctx;
  if ((st = get_ctx(ctx)) != MOE_OK) return st;
  const moe_config_t& c = *cfg;
  if (c.T == 0) {
    // no tokens: every gradient is zero
    cudaError_t e = cudaMemsetAsync(dw_router, 0, (size_t)c.E * c.d * 4, stream);
    if (e == cudaSuccess && dbias) e = cudaMemsetAsync(dbias, 0, (size_t)c.E * 4, stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(dw_gate, 0, (size_t)c.E * c.d * c.f * 4, stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(dw_up, 0, (size_t)c.E * c.d * c.f * 4, stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(dw_down, 0, (size_t)c.E * c.d * c.f * 4, stream);
    return cuda_status(e);
  }
  const TrainLayout TL = train_layout_of(c);
  const Layout& L = TL.base;
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  const int32_t* topk_idx = reinterpret_cast<const int32_t*>(w8 + L.topk_idx);
  const float* topk_w = reinterpret_cast<const float*>(w8 + L.topk_w);
  const int32_t* offsets = reinterpret_cast<const int32_t*>(w8 + L.route) + 2 * c.E;
  const int32_t* perm = reinterpret_cast<const int32_t*>(w8 + L.perm);
  const int32_t* slot_of = reinterpret_cast<const int32_t*>(w8 + L.slot_of);
  const float* row_scale = reinterpret_cast<const float*>(w8 + L.row_scale);
  float* dw_part = reinterpret_cast<float*>(w8 + TL.dw_part);
  float* dx32 = reinterpret_cast<float*>(w8 + TL.dx32);
  const int n_parts = (int)(c.f / 256) * bwd_dh_parts_per_tile();
  cudaError_t e;
  {
    PhaseMark m(MOE_PHASE_BWD_GATHER, stream);
    e = launch_bwd_gather(c, dout, perm, offsets, row_scale, w8 + TL.dout_perm, w8 + TL.dy_perm, stream, ctx);
  }
  if (e == cudaSuccess) {
    PhaseMark m(MOE_PHASE_BWD_DH, stream);
    e = launch_bwd_dh(c, w8 + TL.dout_perm, offsets, w_down, w8 + TL.g, w8 + TL.u, w8 + L.h, row_scale, w8 + TL.dg,
                      w8 + TL.du, dw_part, stream, ctx);
  }
  if (e == cudaSuccess) {
    PhaseMark m(MOE_PHASE_BWD_ZERO, stream);
    e = launch_zero_rows(c, dx32, stream, ctx);
  }
  if (e == cudaSuccess) {
    PhaseMark m(MOE_PHASE_BWD_DX, stream);
    e = launch_bwd_dx(c, w8 + TL.dg, w8 + TL.du, offsets, w_gate, w_up, perm, dx32, stream, ctx);
  }
  if (e == cudaSuccess) {
    PhaseMark m(MOE_PHASE_BWD_ROUTER, stream);
    e = launch_router_bwd(c, dw_part, n_parts, slot_of, topk_idx, topk_w, w_router, dx32, x,
                          reinterpret_cast<float*>(w8 + TL.dlogits), reinterpret_cast<float*>(w8 + TL.dweight), dx,
                          dw_router, dbias, reinterpret_cast<float*>(w8 + TL.wr_part), stream, ctx);
  }
  // weight gradients: the larger operand's blocks outermost, so the smaller one stays in L2
  if (e == cudaSuccess) {
    PhaseMark m(MOE_PHASE_BWD_WG_DOWN, stream);
    e = launch_bwd_wgrad(c, w8 + L.h, c.f, w8 + TL.dy_perm, c.d, offsets, dw_down, c.f >= c.d, stream, ctx);
  }
  if (e == cudaSuccess) {
    PhaseMark m(MOE_PHASE_BWD_WG_GATE, stream);
    e = launch_bwd_wgrad(c, w8 + L.x_perm, c.d, w8 + TL.dg, c.f, offsets, dw_gate, c.d >= c.f, stream, ctx);
  }
  if (e == cudaSuccess) {
    PhaseMark m(MOE_PHASE_BWD_WG_UP, stream);
    e = launch_bwd_wgrad(c, w8 + L.x_perm, c.d, w8 + TL.du, c.f, offsets, dw_up, c.d >= c.f, stream, ctx);
  }
  return cuda_status(e);
}

}  // extern "C"
