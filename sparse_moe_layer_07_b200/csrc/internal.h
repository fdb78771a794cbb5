// Host-side declarations shared by the translation units of libmoe_b200.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

// Per-device facts the launchers need.
struct Ctx {
  int dev = -1;
  int num_sms = 0;
  int* err = nullptr;  // device address of the device error word
};

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
                            int32_t* stats, cudaStream_t s, const Ctx& ctx);

cudaError_t launch_gather(const moe_config_t& c, const void* x, const int32_t* perm,
                          const int32_t* offsets, void* x_perm, cudaStream_t s, const Ctx& ctx);

cudaError_t launch_combine(const moe_config_t& c, const float* y, const int32_t* slot_of,
                           const float* topk_w, int weights_applied, void* out, cudaStream_t s,
                           const Ctx& ctx);

// fp32 expert FFN on the CUDA cores (exact fp32 FMA; no TF32).
cudaError_t launch_ffn_simt_gate_up(const moe_config_t& c, const float* x_perm,
                                    const int32_t* offsets, const float* wg, const float* wu,
                                    float* h, cudaStream_t s, const Ctx& ctx);
cudaError_t launch_ffn_simt_down(const moe_config_t& c, const float* h, const int32_t* offsets,
                                 const float* wd, const float* row_scale, float* y,
                                 cudaStream_t s, const Ctx& ctx);

// bf16 expert FFN on the tcgen05 tensor cores.
cudaError_t launch_tc_gate_up(const moe_config_t& c, const void* x_perm, const int32_t* offsets,
                              const void* wg, const void* wu, void* h, cudaStream_t s,
                              const Ctx& ctx);
cudaError_t launch_tc_down(const moe_config_t& c, const void* h, const int32_t* offsets,
                           const void* wd, const float* row_scale, float* y, cudaStream_t s,
                           const Ctx& ctx);

// Argument check shared by the entry points (MOE_OK when the config is usable).
moe_status_t validate_config(const moe_config_t* cfg);
// Device facts of the current device (cached per device).
moe_status_t current_ctx(Ctx& out);

// Encodes a tiled TMA descriptor (driver entry point resolved once).
bool encode_tmap(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                 const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swz);

}  // namespace moe
