// Host-side declarations shared by the translation units of libmoe_b200.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <nvtx3/nvToolsExt.h>

#include <utility>

#include "moe.h"

namespace moe {

// NVTX range around an entry point (visible in Nsight timelines; no cost
// without a tool attached).
struct Range {
  explicit Range(const char* name) { nvtxRangePushA(name); }
  ~Range() { nvtxRangePop(); }
  Range(const Range&) = delete;
  Range& operator=(const Range&) = delete;
};

// Phase timing (moe_profile_phases): while enabled, a PhaseMark records one
// CUDA event on `s` when constructed and another at end(); the pair is kept
// for moe_profile_read under MOE_PHASE_* index `phase`.  Disabled, it does
// nothing.
class PhaseMark {
 public:
  PhaseMark(int phase, cudaStream_t s);
  void end();
  ~PhaseMark() { end(); }
  PhaseMark(const PhaseMark&) = delete;
  PhaseMark& operator=(const PhaseMark&) = delete;

 private:
  int phase_;
  cudaStream_t s_;
  cudaEvent_t a_ = nullptr, b_ = nullptr;
};

// Per-device facts the launchers need (looked up again when the device's
// context changes, e.g. after cudaDeviceReset).
struct Ctx {
  int dev = -1;
  int num_sms = 0;
  int* err = nullptr;  // device address of the device error word
  unsigned long long ctx_id = 0;
};

// Unique id of the current CUDA context (cuCtxGetId); false when none is current.
bool current_context_id(unsigned long long* id);

// Launch with programmatic stream serialization: the kernel is launched while
// the previous kernel of the stream is finishing (its launch overlaps that
// kernel's exit); the kernel calls pdl_wait() before it touches global memory.  `extra` adds one more launch attribute (e.g. a cluster
// shape) when its id is not cudaLaunchAttributeIgnore.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              const cudaLaunchAttribute& extra, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  unsigned n = 1;
  if (extra.id != cudaLaunchAttributeIgnore) attr[n++] = extra;
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}
inline cudaLaunchAttribute no_extra_attr() {
  cudaLaunchAttribute a = {};
  a.id = cudaLaunchAttributeIgnore;
  return a;
}

// Rows of the grouped buffers (x_perm, h, y): every assignment may be kept.
inline int64_t slot_rows(const moe_config_t& c) { return c.T * (int64_t)c.top_k; }

// Tokens handled by one block of the dispatch kernels.
constexpr int kDispatchBlockTokens = 256;
inline int64_t dispatch_blocks(const moe_config_t& c) {
  return (c.T + kDispatchBlockTokens - 1) / kDispatchBlockTokens;
}

cudaError_t launch_router(const moe_config_t& c, const void* x, const void* wr, const float* bias,
                          float* logits, int32_t* idx, float* w, cudaStream_t s, const Ctx& ctx);

cudaError_t launch_dispatch(const moe_config_t& c, int64_t cap, const int32_t* idx, const float* w,
                            int32_t* counts_raw, int32_t* counts_kept, int32_t* offsets,
                            int32_t* perm, int32_t* slot_of, float* row_scale, int32_t* block_hist,
                            int32_t* stats, cudaStream_t s, const Ctx& ctx,
                            const int32_t* shard_counts = nullptr, int shard = 0);
// dst[i] = src[idx[i]], i < n: rows of row_bytes (a multiple of 16) from a source of n_src rows.
cudaError_t launch_gather_index(const void* src, const int32_t* idx, int64_t n, int64_t n_src, int64_t row_bytes,
                                void* dst, cudaStream_t s, const Ctx& ctx);
// counts[e] = number of assignments routed to expert e (one block, fixed order).
cudaError_t launch_route_counts(const moe_config_t& c, const int32_t* idx, int32_t* counts, cudaStream_t s,
                                const Ctx& ctx);

cudaError_t launch_gather(const moe_config_t& c, const void* x, const int32_t* perm,
                          const int32_t* offsets, void* x_perm, cudaStream_t s, const Ctx& ctx);

cudaError_t launch_combine(const moe_config_t& c, const float* y, const int32_t* slot_of,
                           const float* topk_w, int weights_applied, void* out, cudaStream_t s,
                           const Ctx& ctx,
                           int n_parts = 1, int64_t part_stride = 0);

// fp32 expert FFN on the CUDA cores (exact fp32 FMA; no TF32).
cudaError_t launch_ffn_simt_gate_up(const moe_config_t& c, const float* x_perm,
                                    const int32_t* offsets, const float* wg, const float* wu,
                                    float* h, cudaStream_t s, const Ctx& ctx);
cudaError_t launch_ffn_simt_down(const moe_config_t& c, const float* h, const int32_t* offsets,
                                 const float* wd, const float* row_scale, float* y,
                                 cudaStream_t s, const Ctx& ctx);

// bf16 expert FFN on the tcgen05 tensor cores.
// g_save / u_save (training): also write the pre-activations G, U [T*k, f] (bf16).
cudaError_t launch_tc_gate_up(const moe_config_t& c, const void* x_perm, const int32_t* offsets,
                              const void* wg, const void* wu, void* h, cudaStream_t s,
                              const Ctx& ctx, void* g_save = nullptr, void* u_save = nullptr);
cudaError_t launch_tc_down(const moe_config_t& c, const void* h, const int32_t* offsets,
                           const void* wd, const float* row_scale, float* y, cudaStream_t s,
                           const Ctx& ctx);

// Tile shape of the bf16 grouped GEMMs (MOE_TILES_*): one CTA per 128-row tile,
// or CTA pairs (2-SM MMAs) per 256-row tile.  set_tile_mode returns the previous mode.
int set_tile_mode(int mode);
bool use_pair_tiles(const moe_config_t& c);

// Down with the combine fused: adds row_scale * (H W_down) into a zeroed fp32
// out32 [T, d] by token (perm) instead of writing Y.  With n_peers > 0 the
// destinations are other ranks' sums: perm holds p * peer_tokens + t and the
// row goes to peer_out[p] + t * d (out32 unused).
cudaError_t launch_tc_down_scatter(const moe_config_t& c, const void* h, const int32_t* offsets, const void* wd,
                                   const float* row_scale, const int32_t* perm, float* out32, cudaStream_t s,
                                   const Ctx& ctx, int n_peers = 0, float* const* peer_out = nullptr,
                                   int64_t peer_tokens = 0);
// Backward of the expert FFNs (bf16, d and f multiples of 256): dG / dU and the
// routing-weight partials, dx (added into a zeroed fp32 dx32 by token), and
// the weight gradients dW[e] = A_e^T B_e over each expert's rows ([E, M, N] fp32).
// Routing-weight partials the dH kernel writes per row and N tile.
int bwd_dh_parts_per_tile();
cudaError_t launch_bwd_dh(const moe_config_t& c, const void* dout_perm, const int32_t* offsets, const void* wd,
                          const void* G, const void* U, const void* H, const float* row_scale, void* dG, void* dU,
                          float* dw_part, cudaStream_t s, const Ctx& ctx);
cudaError_t launch_bwd_dx(const moe_config_t& c, const void* dG, const void* dU, const int32_t* offsets,
                          const void* wg, const void* wu, const int32_t* perm, float* dx32, cudaStream_t s,
                          const Ctx& ctx);
cudaError_t launch_bwd_wgrad(const moe_config_t& c, const void* a_rows, int64_t M, const void* b_rows, int64_t N,
                             const int32_t* offsets, float* dW, bool m_outer, cudaStream_t s, const Ctx& ctx);
// dout_perm[r] = dout[perm[r]],  dy_perm[r] = bf16(row_scale[r] * dout[perm[r]])  (r < offsets[E])
cudaError_t launch_bwd_gather(const moe_config_t& c, const void* dout, const int32_t* perm, const int32_t* offsets,
                              const float* row_scale, void* dout_perm, void* dy_perm, cudaStream_t s, const Ctx& ctx);
// Router backward: routing-weight gradients from the partials, logit gradients
// through the softmax over the two selected logits, dx = round(dx32 + dlogits W_r),
// dW_r = dlogits^T x and dbias = column sums of dlogits (fixed summation orders).
cudaError_t launch_router_bwd(const moe_config_t& c, const float* dw_part, int n_parts, const int32_t* slot_of,
                              const int32_t* topk_idx, const float* topk_w, const void* w_router, const float* dx32,
                              const void* x, float* dlogits, float* dweight, void* dx, float* dw_router,
                              float* dbias, float* wr_part, cudaStream_t s, const Ctx& ctx);
constexpr int kRouterBwdChunks = 128;  // token chunks of the dW_r partial sums

// out32 <- 0 ([T, d] fp32), and out <- out32 rounded to cfg's dtype.
cudaError_t launch_zero_rows(const moe_config_t& c, float* out32, cudaStream_t s, const Ctx& ctx);
cudaError_t launch_round_out(const moe_config_t& c, const float* out32, void* out, cudaStream_t s, const Ctx& ctx);

// One block waits on an mbarrier nothing completes, bounded by limit_ns; sets
// MOE_DEVERR_TIMEOUT when the wait gives up (check of the bounded-wait path).
cudaError_t launch_wait_check(int64_t limit_ns, cudaStream_t s, const Ctx& ctx);

// counts[e] += stats[e] and utilization[e] = counts[e] * E / sum(counts) (one block).
cudaError_t launch_utilization(const int32_t* stats, int E, int64_t* counts, float* util, cudaStream_t s);

// Argument check shared by the entry points (MOE_OK when the config is usable).
moe_status_t validate_config(const moe_config_t* cfg);
// Device facts of the current device (cached per device).
moe_status_t current_ctx(Ctx& out);

// Encodes a tiled TMA descriptor (driver entry point resolved once); bf16 elements.
bool encode_tmap(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                 const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swz);
bool encode_tmap_dtype(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                       const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swz,
                       CUtensorMapDataType dtype);

// Per-output-channel int8 quantisation of E matrices [K, N] (bf16 in).
cudaError_t launch_quantize_int8(int E, const void* w, int64_t K, int64_t N, int8_t* q, float* scale,
                                 cudaStream_t s);

// Expert GEMMs with the weights on the MMA's M side (small token counts,
// bf16 weights).
cudaError_t launch_decode_gate_up(const moe_config_t& c, const void* x_perm, const int32_t* offsets,
                                  const void* wg, const void* wu, void* h, cudaStream_t s, const Ctx& ctx);
cudaError_t launch_decode_down(const moe_config_t& c, const void* h, const int32_t* offsets,
                               const void* wd, const float* row_scale, float* y, cudaStream_t s,
                               const Ctx& ctx);

// 15-bit row codes (hi/lo int8 planes + per-row scale) of the first offsets[E]
// rows of src ([rows, K], bf16 or fp32).
cudaError_t launch_quantize_rows(const void* src, bool src_f32, const int32_t* offsets, int64_t max_rows,
                                 int64_t K, int8_t* hi, int8_t* lo, float* scale, int num_sms, cudaStream_t s,
                                 const int32_t* perm = nullptr, int64_t n_src = 0, int* err = nullptr);

// Expert GEMMs on the int8 tensor cores: int8 weights x row-code planes.
cudaError_t launch_i8_gate_up(const moe_config_t& c, const int8_t* x_hi, const int8_t* x_lo,
                              const float* x_scale, const int32_t* offsets, const int8_t* qg,
                              const float* sg, const int8_t* qu, const float* su, float* h, cudaStream_t s,
                              const Ctx& ctx);
// K splits of the int8 down pass (1 .. kMaxDownSplits; each split writes an fp32
// partial [T*k, d], summed in split order).
constexpr int kMaxDownSplits = 8;
int down_splits(const moe_config_t& c, int num_sms);
// Writes down_splits(c) K-split partials [splits, T*k, d] fp32; launch_sum_partials adds them into y.
cudaError_t launch_i8_down(const moe_config_t& c, const int8_t* h_hi, const int8_t* h_lo, const float* h_scale,
                           const int32_t* offsets, const int8_t* qd, const float* sd, const float* row_scale,
                           float* y_parts, cudaStream_t s, const Ctx& ctx);
cudaError_t launch_sum_partials(const moe_config_t& c, const float* y_parts, const int32_t* offsets, float* y,
                                cudaStream_t s, const Ctx& ctx);

}  // namespace moe
