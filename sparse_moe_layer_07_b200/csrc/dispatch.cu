// Capacity-factor dispatch and the row gather.
//
// "How does Grok-1 use a mixture-of-experts design?", section "Routing: top-2
// without auxiliary loss": a dispatch mask from the top-2 indices, then
// `_apply_capacity` drops overflow beyond capacity_factor x the per-expert
// share; section "The high-level architecture": `_dispatch_and_combine` groups
// tokens by expert.  Capacity is ceil(cf * T * k / E) and overflow is dropped
// lowest-token-index-first, i.e. assignment (t, e) is kept iff fewer than
// `cap` tokens before t were routed to e.
//
// A batch split into token shards (one per rank) keeps the global rule: shard i
// is told how many assignments each expert received from shards 0..i-1 and
// keeps (t, e) iff that prior count plus t's rank inside the shard is below the
// global capacity.
//
// Three deterministic passes, no atomics on any output:
//   hist : block b counts its tokens' assignments per expert   -> block_hist[b][e]
//   scan : exclusive scan over blocks per expert, counts, caps, offsets
//   rank : each assignment's rank = block base + rank inside the block (warp
//          ballots in token order); kept ones get slot offsets[e] + rank.
// Ranks inside a block follow token order, then slot j within the token.
#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kE = 8;
constexpr int kBT = kDispatchBlockTokens;  // one token per thread
constexpr int kWarps = kBT / 32;

__device__ __forceinline__ void load_pair(const int32_t* idx, int64_t t, int64_t T, int& e0, int& e1, int* err) {
  e0 = -1;
  e1 = -1;
  if (t < T) {
    const int2 p = __ldg(reinterpret_cast<const int2*>(idx) + t);
    e0 = p.x;
    e1 = p.y;
    if (e0 < 0 || e0 >= kE) { flag_error(err, MOE_DEVERR_EXPERT_INDEX); e0 = -1; }
    if (e1 < 0 || e1 >= kE) { flag_error(err, MOE_DEVERR_EXPERT_INDEX); e1 = -1; }
  }
}

__global__ void __launch_bounds__(kBT) dispatch_hist_kernel(const int32_t* __restrict__ idx, int64_t T,
                                                           int32_t* __restrict__ block_hist, int* err) {
  __shared__ int s_cnt[kWarps][kE];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t t = (int64_t)blockIdx.x * kBT + threadIdx.x;
  pdl_wait();
  int e0, e1;
  load_pair(idx, t, T, e0, e1, err);
#pragma unroll
  for (int e = 0; e < kE; ++e) {
    const unsigned b0 = __ballot_sync(0xffffffffu, e0 == e);
    const unsigned b1 = __ballot_sync(0xffffffffu, e1 == e);
    if (lane == 0) s_cnt[warp][e] = __popc(b0) + __popc(b1);
  }
  __syncthreads();
  if (threadIdx.x < kE) {
    int s = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) s += s_cnt[w][threadIdx.x];
    block_hist[(int64_t)blockIdx.x * kE + threadIdx.x] = s;
  }
}

// Assignments routed to each expert by the tokens of earlier shards (the first
// `shard` rows of shard_counts [n_shards, E]), 0 without shards.
__device__ __forceinline__ int64_t prior_count(const int32_t* shard_counts, int shard, int e) {
  int64_t p = 0;
  if (shard_counts)
    for (int r = 0; r < shard; ++r) p += shard_counts[r * kE + e];
  return p;
}

// One block of 8 warps; warp e scans block_hist[:, e] in chunks of 32 blocks.
// With shards, expert e has cap - prior slots left for this shard's tokens.
__global__ void __launch_bounds__(256) dispatch_scan_kernel(int32_t* __restrict__ block_hist, int64_t nblk, int64_t cap,
                                                           const int32_t* __restrict__ shard_counts, int shard,
                                                           int32_t* __restrict__ counts_raw,
                                                           int32_t* __restrict__ counts_kept,
                                                           int32_t* __restrict__ offsets, int32_t* __restrict__ stats) {
  __shared__ int s_total[kE];
  const int lane = threadIdx.x & 31, e = threadIdx.x >> 5;
  pdl_wait();
  int running = 0;
  for (int64_t b0 = 0; b0 < nblk; b0 += 32) {
    const int64_t b = b0 + lane;
    const int v = b < nblk ? block_hist[b * kE + e] : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    if (b < nblk) block_hist[b * kE + e] = running + incl - v;  // exclusive base of block b
    running += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) s_total[e] = running;
  __syncthreads();
  if (threadIdx.x == 0) {
    int off = 0, dropped = 0;
    for (int k = 0; k < kE; ++k) {
      const int raw = s_total[k];
      int64_t left = cap - prior_count(shard_counts, shard, k);
      if (left < 0) left = 0;
      const int kept = (int64_t)raw < left ? raw : (int)left;
      counts_raw[k] = raw;
      counts_kept[k] = kept;
      offsets[k] = off;
      off += kept;
      dropped += raw - kept;
      if (stats) {
        stats[k] = raw;
        stats[kE + k] = kept;
        stats[2 * kE + k] = off - kept;
      }
    }
    offsets[kE] = off;
    if (stats) {
      stats[3 * kE] = off;
      stats[3 * kE + 1] = dropped;
    }
  }
}

__global__ void __launch_bounds__(kBT) dispatch_rank_kernel(const int32_t* __restrict__ idx, const float* __restrict__ w,
                                                           int64_t T, int64_t cap,
                                                           const int32_t* __restrict__ shard_counts, int shard,
                                                           const int32_t* __restrict__ block_base,
                                                           const int32_t* __restrict__ offsets,
                                                           int32_t* __restrict__ perm, int32_t* __restrict__ slot_of,
                                                           float* __restrict__ row_scale, int* err) {
  __shared__ int s_cnt[kWarps][kE];
  __shared__ int s_base[kE];
  __shared__ int s_off[kE];
  __shared__ int64_t s_prior[kE];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t t = (int64_t)blockIdx.x * kBT + threadIdx.x;
  pdl_wait();
  int e0, e1;
  load_pair(idx, t, T, e0, e1, err);
  if (threadIdx.x < kE) {
    s_base[threadIdx.x] = block_base[(int64_t)blockIdx.x * kE + threadIdx.x];
    s_off[threadIdx.x] = offsets[threadIdx.x];
    s_prior[threadIdx.x] = prior_count(shard_counts, shard, threadIdx.x);
  }
  const unsigned lt = (1u << lane) - 1u;
  int pre0 = 0, pre1 = 0;  // in-warp prefix for this lane's slot 0 / slot 1
#pragma unroll
  for (int e = 0; e < kE; ++e) {
    const unsigned b0 = __ballot_sync(0xffffffffu, e0 == e);
    const unsigned b1 = __ballot_sync(0xffffffffu, e1 == e);
    const int p = __popc(b0 & lt) + __popc(b1 & lt);
    if (e0 == e) pre0 = p;
    if (e1 == e) pre1 = p + (e0 == e ? 1 : 0);
    if (lane == 0) s_cnt[warp][e] = __popc(b0) + __popc(b1);
  }
  __syncthreads();
  if (t >= T) return;
  float2 wt = __ldg(reinterpret_cast<const float2*>(w) + t);
  int slots[2] = {-1, -1};
  const int es[2] = {e0, e1};
  const int pres[2] = {pre0, pre1};
  const float ws[2] = {wt.x, wt.y};
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int e = es[j];
    if (e < 0) continue;
    int r = s_base[e] + pres[j];
    for (int k = 0; k < warp; ++k) r += s_cnt[k][e];
    if (s_prior[e] + r < cap) {
      const int s = s_off[e] + r;
      slots[j] = s;
      perm[s] = (int32_t)t;
      row_scale[s] = ws[j];
    }
  }
  reinterpret_cast<int2*>(slot_of)[t] = make_int2(slots[0], slots[1]);
}

// x_perm[s, :] = x[perm[s], :] for s < offsets[E]; one warp per row, 16-byte vectors.
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ perm,
                                                         const int32_t* __restrict__ offsets, int64_t T,
                                                         int64_t row_vec, uint4* __restrict__ x_perm, int* err) {
  pdl_wait();
  int64_t n = offsets[kE];
  const int lane = threadIdx.x & 31;
  if (n < 0 || n > 2 * T) {
    if (blockIdx.x == 0 && threadIdx.x == 0) flag_error(err, MOE_DEVERR_OFFSETS);
    n = 0;
  }
  const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t s = gw; s < n; s += nw) {
    const int32_t t = __ldg(perm + s);
    if (t < 0 || t >= T) {
      if (lane == 0) flag_error(err, MOE_DEVERR_SLOT_INDEX);
      continue;
    }
    const uint4* src = x + (int64_t)t * row_vec;
    uint4* dst = x_perm + s * row_vec;
    int64_t v = lane;
    for (; v + 96 < row_vec; v += 128) {
      const uint4 a = __ldg(src + v), b = __ldg(src + v + 32), c = __ldg(src + v + 64), d = __ldg(src + v + 96);
      dst[v] = a;
      dst[v + 32] = b;
      dst[v + 64] = c;
      dst[v + 96] = d;
    }
    for (; v < row_vec; v += 32) dst[v] = __ldg(src + v);
  }
}

}  // namespace

cudaError_t launch_dispatch(const moe_config_t& c, int64_t cap, const int32_t* idx, const float* w,
                            int32_t* counts_raw, int32_t* counts_kept, int32_t* offsets,
                            int32_t* perm, int32_t* slot_of, float* row_scale, int32_t* block_hist,
                            int32_t* stats, cudaStream_t s, const Ctx& ctx, const int32_t* shard_counts,
                            int shard) {
  const int64_t nblk = dispatch_blocks(c);
  cudaError_t e = cudaSuccess;
  if (nblk > 0) {
    e = launch_pdl(dispatch_hist_kernel, dim3((unsigned)nblk), dim3(kBT), 0, s, no_extra_attr(), idx, c.T, block_hist,
                   ctx.err);
    if (e != cudaSuccess) return e;
  }
  e = launch_pdl(dispatch_scan_kernel, dim3(1), dim3(256), 0, s, no_extra_attr(), block_hist, nblk, cap,
                 shard_counts, shard, counts_raw, counts_kept, offsets, stats);
  if (e != cudaSuccess) return e;
  if (nblk > 0) {
    e = launch_pdl(dispatch_rank_kernel, dim3((unsigned)nblk), dim3(kBT), 0, s, no_extra_attr(), idx, w, c.T, cap,
                   shard_counts, shard, static_cast<const int32_t*>(block_hist), static_cast<const int32_t*>(offsets),
                   perm, slot_of, row_scale, ctx.err);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

namespace {

// counts[e] = assignments routed to e over the whole batch: one block, each
// thread counts a strided share of the tokens, then a fixed-order reduction.
__global__ void __launch_bounds__(256) route_counts_kernel(const int32_t* __restrict__ idx, int64_t T,
                                                          int32_t* __restrict__ counts, int* err) {
  __shared__ int s[kE][256];
  int c[kE];
#pragma unroll
  for (int e = 0; e < kE; ++e) c[e] = 0;
  for (int64_t t = threadIdx.x; t < T; t += blockDim.x) {
    int e0, e1;
    load_pair(idx, t, T, e0, e1, err);
#pragma unroll
    for (int e = 0; e < kE; ++e) c[e] += (e0 == e) + (e1 == e);
  }
#pragma unroll
  for (int e = 0; e < kE; ++e) s[e][threadIdx.x] = c[e];
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if ((int)threadIdx.x < w)
#pragma unroll
      for (int e = 0; e < kE; ++e) s[e][threadIdx.x] += s[e][threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x < kE) counts[threadIdx.x] = s[threadIdx.x][0];
}

}  // namespace

cudaError_t launch_route_counts(const moe_config_t& c, const int32_t* idx, int32_t* counts, cudaStream_t s,
                                const Ctx& ctx) {
  route_counts_kernel<<<1, 256, 0, s>>>(idx, c.T, counts, ctx.err);
  return cudaGetLastError();
}

namespace {

// dst[i] = src[idx[i]] for i < n (rows of row_vec 16-byte vectors); an index
// outside [0, n_src) leaves its row untouched and sets the error word.
__global__ void __launch_bounds__(256) gather_index_kernel(const uint4* __restrict__ src, const int32_t* __restrict__ idx,
                                                          int64_t n, int64_t n_src, int64_t row_vec,
                                                          uint4* __restrict__ dst, int* err) {
  const int lane = threadIdx.x & 31;
  const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t i = gw; i < n; i += nw) {
    const int32_t r = __ldg(idx + i);
    if (r < 0 || r >= n_src) {
      if (lane == 0) flag_error(err, MOE_DEVERR_SLOT_INDEX);
      continue;
    }
    for (int64_t v = lane; v < row_vec; v += 32) dst[i * row_vec + v] = __ldg(src + (int64_t)r * row_vec + v);
  }
}

}  // namespace

cudaError_t launch_gather_index(const void* src, const int32_t* idx, int64_t n, int64_t n_src, int64_t row_bytes,
                                void* dst, cudaStream_t s, const Ctx& ctx) {
  if (n == 0) return cudaSuccess;
  int64_t blocks = (n + 7) / 8;
  const int64_t cap_blocks = (int64_t)ctx.num_sms * 8;
  if (blocks > cap_blocks) blocks = cap_blocks;
  gather_index_kernel<<<(unsigned)blocks, 256, 0, s>>>(static_cast<const uint4*>(src), idx, n, n_src, row_bytes / 16,
                                                       static_cast<uint4*>(dst), ctx.err);
  return cudaGetLastError();
}

cudaError_t launch_gather(const moe_config_t& c, const void* x, const int32_t* perm,
                          const int32_t* offsets, void* x_perm, cudaStream_t s, const Ctx& ctx) {
  const int64_t esz = c.dtype == MOE_BF16 ? 2 : 4;
  const int64_t row_vec = c.d * esz / 16;
  const int64_t rows = slot_rows(c);
  if (rows == 0) return cudaSuccess;
  int64_t blocks = (rows + 7) / 8;  // 8 warps per block, one row per warp
  const int64_t cap_blocks = (int64_t)ctx.num_sms * 8;
  if (blocks > cap_blocks) blocks = cap_blocks;
  const cudaError_t e = launch_pdl(gather_rows_kernel, dim3((unsigned)blocks), dim3(256), 0, s, no_extra_attr(),
                                   static_cast<const uint4*>(x), perm, offsets, c.T, row_vec,
                                   static_cast<uint4*>(x_perm), ctx.err);
  return e != cudaSuccess ? e : cudaGetLastError();
}


namespace {
// counts[e] += stats[e]; utilization[e] = counts[e] * E / sum(counts), one
// thread, experts in order (the sum does not depend on timing).
__global__ void utilization_kernel(const int32_t* __restrict__ stats, int E, int64_t* __restrict__ counts,
                                   float* __restrict__ util) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  int64_t total = 0;
  for (int e = 0; e < E; ++e) {
    const int64_t c = counts[e] + (int64_t)stats[e];
    counts[e] = c;
    total += c;
  }
  for (int e = 0; e < E; ++e)
    util[e] = total > 0 ? (float)((double)counts[e] * (double)E / (double)total) : 0.0f;
}
}  // namespace

cudaError_t launch_utilization(const int32_t* stats, int E, int64_t* counts, float* util, cudaStream_t s) {
  utilization_kernel<<<1, 32, 0, s>>>(stats, E, counts, util);
  return cudaGetLastError();
}

}  // namespace moe
