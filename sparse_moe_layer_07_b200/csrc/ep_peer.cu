// Expert parallelism over peer memory ("Expert parallelism vs. tensor
// parallelism", moe_layer_ep_forward).  The pages' version exchanges token rows
// with two all-to-alls (dispatch to the expert's owner, outputs back to the
// source).  Here the exchanges are stores issued by the kernels that produce
// the data:
//   dispatch: one kernel per source rank reads each kept row x[perm[r]] and
//             stores it, with its source id and routing weight, at its final
//             place in the owner's expert-major grouped buffer (no x_perm, no
//             send buffer, no regrouping on the receiving side);
//   combine:  the owner's down projection (the tensor-core kernel with the
//             fused combine epilogue) adds routing_weight * (h W_down) into the
//             source rank's fp32 sums with vector atomics; the source then
//             rounds its own sums once.
// Neither kernel signals another rank: the phases are separated by barriers
// the caller puts after them on the stream.
// Within an owner's buffer, expert e's rows come from source 0, 1, ... in
// turn, each source's rows in its kept (token) order, so every rank computes
// every destination from the all-gathered table of kept counts alone.
//
// Peer addresses come from CUDA IPC (moe_peer_export / moe_peer_import): an
// address inside another process's cudaMalloc block, mapped here.
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kE = 8;      // experts (the layer's fixed expert count)
constexpr int kWarps = 8;  // rows in flight per block of the dispatch kernel

struct EpDispatchArgs {
  const uint4* x;           // [T, d] this rank's tokens, row_vec 16-byte words per row
  const int32_t* table;     // [world, E] kept rows of each rank by expert
  const int32_t* offsets;   // [E + 1] this rank's kept rows by expert
  const int32_t* perm;      // source token of each kept row
  const float* row_scale;   // routing weight of each kept row
  int32_t* grp_offsets;     // [E + 1] out: this rank's received rows by expert
  int64_t T;                // tokens of every rank
  int64_t rows_cap;         // rows of every grouped buffer: world * T * top_k
  float* sums;              // this rank's fp32 sums [T, d], cleared here
  int row_vec;
  int world, rank;
  uint4* x_grp[MOE_EP_MAX_WORLD];
  int32_t* src[MOE_EP_MAX_WORLD];
  float* scale[MOE_EP_MAX_WORLD];
  int* err;
};

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint4* peer_select(const EpDispatchArgs& a, int q) {
  uint4* d = a.x_grp[0];
#pragma unroll
  for (int i = 1; i < MOE_EP_MAX_WORLD; ++i)
    if (i == q) d = a.x_grp[i];
  return d;
}
__device__ __forceinline__ int32_t* src_select(const EpDispatchArgs& a, int q) {
  int32_t* d = a.src[0];
#pragma unroll
  for (int i = 1; i < MOE_EP_MAX_WORLD; ++i)
    if (i == q) d = a.src[i];
  return d;
}
__device__ __forceinline__ float* scale_select(const EpDispatchArgs& a, int q) {
  float* d = a.scale[0];
#pragma unroll
  for (int i = 1; i < MOE_EP_MAX_WORLD; ++i)
    if (i == q) d = a.scale[i];
  return d;
}

// Work items of one warp: a 2 KB segment of a kept row (32 lanes x 4 vectors
// of 16 bytes) to copy into its owner's buffer, or, after all of those, 2 KB
// of this rank's fp32 sums to clear.  Every block first derives, one thread per
// expert, dst[e] = first row in the owner's buffer of this rank's rows of
// expert e = (rows of the owner's earlier experts, from every source) + (rows
// of expert e from sources before this rank), and checks the table.
constexpr int kSegVec = 128;  // 16-byte vectors per work item

__global__ void __launch_bounds__(32 * kWarps) ep_dispatch_peers_kernel(const __grid_constant__ EpDispatchArgs a) {
  __shared__ int s_offs[kE + 1];
  __shared__ int s_dst[kE];
  __shared__ int s_tab[MOE_EP_MAX_WORLD * kE];
  pdl_wait();
  const int per = kE / a.world;
  // one round of loads: the offsets (threads 0-8) and the table (threads 32-95);
  // at 75 MB per call the kernel is latency-bound, and a second dependent round
  // cost 4 us of 18 (a grid of one resident wave, 4 us more: the extra blocks
  // hide latency better than they cost in prologues)
  if (threadIdx.x <= kE) s_offs[threadIdx.x] = __ldg(a.offsets + threadIdx.x);
  if (threadIdx.x >= 32 && threadIdx.x < 32 + a.world * kE) s_tab[threadIdx.x - 32] = __ldg(a.table + threadIdx.x - 32);
  __syncthreads();
  bool ok = true;
  if (threadIdx.x < kE) {
    const int e = threadIdx.x;
    const int q = e / per;
    if (s_offs[e + 1] - s_offs[e] != s_tab[a.rank * kE + e]) ok = false;
    int64_t pos = 0, total = 0;
    for (int e2 = q * per; e2 < (q + 1) * per; ++e2)
      for (int p = 0; p < a.world; ++p) {
        const int c = s_tab[p * kE + e2];
        if (c < 0) ok = false;
        if (e2 < e || (e2 == e && p < a.rank)) pos += c;
        total += c;
      }
    if (total > a.rows_cap) ok = false;
    s_dst[e] = (int)pos;
  }
  if (threadIdx.x == 0 && (s_offs[0] != 0 || s_offs[kE] > a.T * 2)) ok = false;
  ok = __syncthreads_and(ok);
  if (blockIdx.x == 0 && threadIdx.x <= kE) {
    // this rank as an owner: its experts in order, other experts empty
    int run = 0;
    for (int e2 = a.rank * per; e2 < (a.rank + 1) * per && e2 < (int)threadIdx.x; ++e2)
      for (int p = 0; p < a.world; ++p) run += s_tab[p * kE + e2];
    a.grp_offsets[threadIdx.x] = ok ? run : 0;
    if (!ok && threadIdx.x == 0) flag_error(a.err, MOE_DEVERR_OFFSETS);
  }
  if (!ok) return;
  const int lane = threadIdx.x & 31;
  const int n = s_offs[kE];
  const int nv = a.row_vec;
  const int segs = (nv + kSegVec - 1) / kSegVec;
  const int64_t copy_items = (int64_t)n * segs;
  const int64_t zero_vec = a.T * (int64_t)nv * 2;  // the sums hold T rows of 4 * d bytes
  const int64_t items = copy_items + (zero_vec + kSegVec - 1) / kSegVec;
  const int64_t warps = (int64_t)gridDim.x * kWarps;
  for (int64_t it = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5); it < items; it += warps) {
    if (it < copy_items) {
      const int r = (int)(it / segs);
      const int v0 = (int)(it - (int64_t)r * segs) * kSegVec;
      int e = 0;
#pragma unroll
      for (int k = 1; k < kE; ++k)
        if (r >= s_offs[k]) e = k;
      const int q = e / per;
      const int64_t dst = (int64_t)s_dst[e] + (r - s_offs[e]);
      const int t = __ldg(a.perm + r);
      if (t < 0 || (int64_t)t >= a.T) {
        if (lane == 0) flag_error(a.err, MOE_DEVERR_SLOT_INDEX);
        continue;
      }
      const uint4* srow = a.x + (int64_t)t * nv;
      uint4* drow = peer_select(a, q) + dst * nv;
      uint4 v[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int i = v0 + lane + 32 * j;
        if (i < nv) v[j] = ld_stream(srow + i);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int i = v0 + lane + 32 * j;
        if (i < nv) drow[i] = v[j];
      }
      if (v0 == 0 && lane == 0) {
        src_select(a, q)[dst] = (int32_t)(a.rank * a.T + t);
        scale_select(a, q)[dst] = __ldg(a.row_scale + r);
      }
    } else {
      const int64_t z0 = (it - copy_items) * kSegVec;
      uint4* z = reinterpret_cast<uint4*>(a.sums);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t i = z0 + lane + 32 * j;
        if (i < zero_vec) z[i] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
  }
  // No fence: the owners read these rows only after a barrier that the caller
  // orders after this kernel on the stream (a collective, an event or a host
  // barrier), and a kernel's completion makes all its stores, peer memory
  // included, visible.  A fence per block cost 6 us of 25 at 75 MB per rank
  // (one per thread: 11 us).
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The checks every entry point shares: a bf16 top-2 layer of E = kE experts in
// the fused down + combine scope and a consistent peer table.
moe_status_t check_ep(const moe_config_t* cfg, const moe_ep_peers_t* peers) {
  moe_status_t st = validate_config(cfg);
  if (st != MOE_OK) return st;
  if (!peers) return MOE_ERR_INVALID_ARG;
  const int w = peers->world;
  if (w < 1 || w > MOE_EP_MAX_WORLD || peers->rank < 0 || peers->rank >= w) return MOE_ERR_INVALID_ARG;
  if (cfg->dtype != MOE_BF16 || cfg->top_k != 2 || cfg->E != kE || kE % w != 0 || cfg->d % 256 != 0)
    return MOE_ERR_UNSUPPORTED;
  if ((int64_t)w * cfg->T > ((int64_t)1 << 30)) return MOE_ERR_INVALID_ARG;
  for (int q = 0; q < w; ++q)
    if (!peers->x_grp[q] || !peers->src[q] || !peers->scale[q] || !peers->sums[q] || !aligned16(peers->x_grp[q]) ||
        !aligned16(peers->sums[q]) || (reinterpret_cast<uintptr_t>(peers->src[q]) & 3u) != 0 ||
        (reinterpret_cast<uintptr_t>(peers->scale[q]) & 3u) != 0)
      return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

// Driver entry point of cuMemGetAddressRange (resolved once): the base of the
// allocation holding an address, which is what CUDA IPC exports.
using MemGetAddressRangeFn = CUresult (*)(CUdeviceptr*, size_t*, CUdeviceptr);
MemGetAddressRangeFn g_get_range = nullptr;
std::once_flag g_get_range_once;

void resolve_get_range() {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_get_range = reinterpret_cast<MemGetAddressRangeFn>(p);
  (void)cudaGetLastError();
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status_t moe_ep_dispatch_peers(const moe_config_t* cfg, const moe_ep_peers_t* peers,
                                              const int32_t* table, const void* x, const int32_t* offsets,
                                              const int32_t* perm, const float* row_scale, int32_t* grp_offsets,
                                              moe_stream_t stream) {
  Range range_("moe_ep_dispatch_peers");
  moe_status_t st = check_ep(cfg, peers);
  if (st != MOE_OK) return st;
  if (!table || !offsets || !grp_offsets || (cfg->T > 0 && (!x || !perm || !row_scale || !aligned16(x))))
    return MOE_ERR_INVALID_ARG;
  Ctx ctx;
  if ((st = current_ctx(ctx)) != MOE_OK) return st;
  const int r = peers->rank;
  EpDispatchArgs a = {};
  a.sums = peers->sums[r];
  a.x = static_cast<const uint4*>(x);
  a.table = table;
  a.offsets = offsets;
  a.perm = perm;
  a.row_scale = row_scale;
  a.grp_offsets = grp_offsets;
  a.T = cfg->T;
  a.rows_cap = (int64_t)peers->world * slot_rows(*cfg);
  a.row_vec = (int)(cfg->d * 2 / 16);
  a.world = peers->world;
  a.rank = r;
  for (int q = 0; q < peers->world; ++q) {
    a.x_grp[q] = static_cast<uint4*>(peers->x_grp[q]);
    a.src[q] = peers->src[q];
    a.scale[q] = peers->scale[q];
  }
  a.err = ctx.err;
  // one warp per 2 KB item: enough blocks for the most items (every row kept)
  // up to 8 blocks per SM
  const int64_t segs = (a.row_vec + kSegVec - 1) / kSegVec;
  const int64_t items = slot_rows(*cfg) * segs + (cfg->T * (int64_t)a.row_vec * 2 + kSegVec - 1) / kSegVec;
  int64_t blocks = (items + kWarps - 1) / kWarps;
  if (blocks > (int64_t)ctx.num_sms * 8) blocks = (int64_t)ctx.num_sms * 8;
  if (blocks < 1) blocks = 1;
  cudaError_t e = launch_pdl(ep_dispatch_peers_kernel, dim3((unsigned)blocks), dim3(32 * kWarps), 0, stream, no_extra_attr(), a);
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" moe_status_t moe_ep_expert_ffn_peers(const moe_config_t* cfg, const moe_ep_peers_t* peers,
                                                const int32_t* grp_offsets, const void* w_gate, const void* w_up,
                                                const void* w_down, void* h, moe_stream_t stream) {
  Range range_("moe_ep_expert_ffn_peers");
  moe_status_t st = check_ep(cfg, peers);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;
  if (!grp_offsets || !w_gate || !w_up || !w_down || !h || !aligned16(w_gate) || !aligned16(w_up) ||
      !aligned16(w_down) || !aligned16(h))
    return MOE_ERR_INVALID_ARG;
  Ctx ctx;
  if ((st = current_ctx(ctx)) != MOE_OK) return st;
  // the grouped buffers hold world * T * top_k rows: the tensor-core kernels
  // see a layer of world * T tokens whose offsets cover this rank's experts
  moe_config_t ce = *cfg;
  ce.T = cfg->T * peers->world;
  const int r = peers->rank;
  cudaError_t e = launch_tc_gate_up(ce, peers->x_grp[r], grp_offsets, w_gate, w_up, h, stream, ctx);
  if (e == cudaSuccess)
    e = launch_tc_down_scatter(ce, h, grp_offsets, w_down, peers->scale[r], peers->src[r], nullptr, stream, ctx,
                               peers->world, peers->sums, cfg->T);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" moe_status_t moe_ep_combine_peers(const moe_config_t* cfg, const moe_ep_peers_t* peers, void* out,
                                             moe_stream_t stream) {
  Range range_("moe_ep_combine_peers");
  moe_status_t st = check_ep(cfg, peers);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;
  if (!out || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  Ctx ctx;
  if ((st = current_ctx(ctx)) != MOE_OK) return st;
  return launch_round_out(*cfg, peers->sums[peers->rank], out, stream, ctx) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" moe_status_t moe_peer_export(const void* ptr, moe_peer_handle_t* handle) {
  if (!ptr || !handle) return MOE_ERR_INVALID_ARG;
  std::call_once(g_get_range_once, resolve_get_range);
  if (!g_get_range) return MOE_ERR_CUDA;
  CUdeviceptr base = 0;
  size_t size = 0;
  if (g_get_range(&base, &size, reinterpret_cast<CUdeviceptr>(ptr)) != CUDA_SUCCESS) return MOE_ERR_CUDA;
  cudaIpcMemHandle_t h;
  if (cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base)) != cudaSuccess) {
    (void)cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  static_assert(sizeof(h) == sizeof(handle->ipc), "IPC handle size");
  memcpy(handle->ipc, &h, sizeof(h));
  handle->offset = (uint64_t)(reinterpret_cast<CUdeviceptr>(ptr) - base);
  return MOE_OK;
}

extern "C" moe_status_t moe_peer_import(const moe_peer_handle_t* handle, void** ptr) {
  if (!handle || !ptr) return MOE_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  memcpy(&h, handle->ipc, sizeof(h));
  void* base = nullptr;
  if (cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) {
    (void)cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  *ptr = static_cast<uint8_t*>(base) + handle->offset;
  return MOE_OK;
}

extern "C" moe_status_t moe_peer_release(void* ptr, const moe_peer_handle_t* handle) {
  if (!ptr || !handle) return MOE_ERR_INVALID_ARG;
  void* base = static_cast<uint8_t*>(ptr) - handle->offset;
  if (cudaIpcCloseMemHandle(base) != cudaSuccess) {
    (void)cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}
