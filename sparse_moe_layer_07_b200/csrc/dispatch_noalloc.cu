// moe_dispatch_noalloc: the capacity dispatch for callers that cannot allocate
// device memory.
//
// moe_dispatch needs a small scratch buffer (one expert histogram per block of
// 256 tokens) that the caller normally allocates and passes in.  Some callers
// have no way to do that: a plug-in hosted by an inference runtime that owns
// all device memory and hands its plug-ins no workspace, or a latency-critical
// loop that cannot afford cudaMalloc's implicit device-wide synchronisation.
// This entry point keeps that scratch in a fixed, file-scope device array
// instead, so it performs no allocation of any kind (no cudaMalloc, no
// cudaFree, no allocating library routine).
//
// Costs and limits:
//   - every GPU that loads the library holds kNoallocScratchInts int32
//     (MOE_NOALLOC_MAX_TOKENS / 256 * 8 = 128 KiB) until the process exits;
//   - T above MOE_NOALLOC_MAX_TOKENS is rejected with MOE_ERR_UNSUPPORTED;
//   - all calls share the one array, so calls that overlap on the GPU (for
//     example on two streams at once) race and give wrong results;
//   - the array keeps the last call's contents; nothing has to start at zero,
//     because each call writes every histogram entry it later reads;
//   - the first call on a device looks up the array's device address (with
//     that device current) and caches it, keyed by the current context's
//     unique id, so after a cudaDeviceReset (a new primary context) the next
//     call looks the address up again; make the first call on a device, and
//     the first after a reset, before any stream capture.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "internal.h"
#include "moe.h"

namespace moe {
namespace {

constexpr int64_t kNoallocBlocks = (MOE_NOALLOC_MAX_TOKENS + kDispatchBlockTokens - 1) / kDispatchBlockTokens;
constexpr int64_t kNoallocScratchInts = kNoallocBlocks * 8;

// The scratch itself.  In host code this name is only a stand-in for the
// symbol, not a device address: kernels receive the address looked up below.
static __device__ __align__(256) int32_t g_dispatch_scratch[kNoallocScratchInts];

constexpr int kMaxDev = 64;
int32_t* g_scratch_ptr[kMaxDev];
unsigned long long g_scratch_ctx_id[kMaxDev];
bool g_scratch_ready[kMaxDev];
std::mutex g_scratch_mu;

// Device address of the scratch on the current device, looked up with that
// device current the first time, and again whenever the current context is
// not the one the cached address belongs to.
moe_status_t scratch_on_current_device(int32_t** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  unsigned long long id = 0;
  const bool have_id = current_context_id(&id);
  if (!g_scratch_ready[dev] || !have_id || id != g_scratch_ctx_id[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dispatch_scratch) != cudaSuccess) return MOE_ERR_CUDA;
    // the lookup makes the device's primary context current if it was not yet
    if (!current_context_id(&id)) return MOE_ERR_CUDA;
    g_scratch_ptr[dev] = static_cast<int32_t*>(p);
    g_scratch_ctx_id[dev] = id;
    g_scratch_ready[dev] = true;
  }
  *out = g_scratch_ptr[dev];
  return MOE_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status_t moe_dispatch_noalloc(const moe_config_t* cfg, const void* x, const int32_t* topk_idx,
                                             const float* topk_w, int32_t* counts_raw, int32_t* counts_kept,
                                             int32_t* offsets, int32_t* perm, int32_t* slot_of, float* row_scale,
                                             void* x_perm, moe_stream_t stream) {
  Range range_("moe_dispatch_noalloc");
  moe_status_t st = validate_config(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T > MOE_NOALLOC_MAX_TOKENS) return MOE_ERR_UNSUPPORTED;
  const int64_t cap = moe_capacity(cfg);
  if (!topk_idx || !topk_w || !counts_raw || !counts_kept || !offsets || !perm || !slot_of || !row_scale)
    return MOE_ERR_INVALID_ARG;
  if (x_perm && !x) return MOE_ERR_INVALID_ARG;
  if (!aligned16(topk_idx) || !aligned16(topk_w) || !aligned16(slot_of) || (x_perm && !aligned16(x_perm)) ||
      (x && !aligned16(x)))
    return MOE_ERR_INVALID_ARG;
  int32_t* scratch = nullptr;
  if ((st = scratch_on_current_device(&scratch)) != MOE_OK) return st;
  Ctx ctx;
  if ((st = current_ctx(ctx)) != MOE_OK) return st;
  cudaError_t e = launch_dispatch(*cfg, cap, topk_idx, topk_w, counts_raw, counts_kept, offsets, perm, slot_of,
                                  row_scale, scratch, nullptr, stream, ctx);
  if (e == cudaSuccess && x_perm && cfg->T > 0) e = launch_gather(*cfg, x, perm, offsets, x_perm, stream, ctx);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
