// Router logits + top-2 + softmax over the two selected logits.
//
// "How does Grok-1 use a mixture-of-experts design?", section "Routing: top-2
// without auxiliary loss" (grok_router_forward): logits = hidden @ W_r.T with
// W_r stored [E, hidden]; topk(logits, 2); softmax of the two selected values.
//
// HBM-bound on x: a block of 8 warps takes 4 tokens (1 for decode-sized
// batches) and splits the hidden dimension over its 256 threads; each thread
// streams its 16-byte slices of the 4 token rows and reuses every W_r slice
// (E rows, L1/L2 resident) for the 4 tokens.  Partial sums are reduced in a
// fixed order (lanes, then warps), so results do not depend on timing.
#include <cuda_bf16.h>
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "tc_ptx.cuh"

namespace moe {
namespace {

constexpr int kE = 8;
constexpr int kWarps = 8;

// Top-2 of one token's (biased) logits and the softmax over the two selected.
__device__ __forceinline__ void finish_token(const float (&l)[kE], int64_t t, float* logits, int32_t* idx, float* w) {
  if (logits) {
    float4* lp = reinterpret_cast<float4*>(logits + t * kE);
    lp[0] = make_float4(l[0], l[1], l[2], l[3]);
    lp[1] = make_float4(l[4], l[5], l[6], l[7]);
  }
  // descending; strict '>' keeps the lower expert index on equal logits
  int i0 = 0;
  float v0 = l[0];
#pragma unroll
  for (int e = 1; e < kE; ++e)
    if (l[e] > v0) { v0 = l[e]; i0 = e; }
  int i1 = i0 == 0 ? 1 : 0;
  float v1 = l[i1];
#pragma unroll
  for (int e = 0; e < kE; ++e)
    if (e != i0 && l[e] > v1) { v1 = l[e]; i1 = e; }
  // softmax over the two selected logits: w0 = 1 / (1 + e^(l1 - l0))
  const float ex = expf(v1 - v0);
  const float inv = 1.0f / (1.0f + ex);
  idx[2 * t] = i0;
  idx[2 * t + 1] = i1;
  w[2 * t] = inv;
  w[2 * t + 1] = ex * inv;
}

// kTPB tokens per block; the 8 warps split the hidden dimension (each thread 8
// consecutive elements per 2048-wide step, for every token of the block, so
// each W_r load serves kTPB tokens) and their partial logits are summed in warp
// order.  kTPB = 1 for decode-sized batches (latency: a few steps instead of
// d/256), 4 for large ones (many blocks in flight, x streamed once).
template <typename Tin, int kTPB>
__global__ void __launch_bounds__(kWarps * 32) router_top2_split_kernel(const Tin* __restrict__ x,
                                                                       const Tin* __restrict__ wr,
                                                                       const float* __restrict__ bias,
                                                                       float* __restrict__ logits,
                                                                       int32_t* __restrict__ idx,
                                                                       float* __restrict__ w, int64_t T, int64_t d) {
  __shared__ float s_part[kWarps][kTPB][kE];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int64_t t0 = (int64_t)blockIdx.x * kTPB;
  float acc[kTPB][kE];
#pragma unroll
  for (int j = 0; j < kTPB; ++j)
#pragma unroll
    for (int e = 0; e < kE; ++e) acc[j][e] = 0.f;
  for (int64_t c = (int64_t)threadIdx.x * 8; c < d; c += kWarps * 32 * 8) {
    float xv[kTPB][8];
#pragma unroll
    for (int j = 0; j < kTPB; ++j) {
      const int64_t t = t0 + j < T ? t0 + j : T - 1;  // clamp: duplicate rows are discarded below
      load8(x + t * d + c, xv[j]);
    }
#pragma unroll
    for (int e = 0; e < kE; ++e) {
      float wv[8];
      load8(wr + (int64_t)e * d + c, wv);
#pragma unroll
      for (int j = 0; j < kTPB; ++j)
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[j][e] = fmaf(xv[j][i], wv[i], acc[j][e]);
    }
  }
#pragma unroll
  for (int j = 0; j < kTPB; ++j)
#pragma unroll
    for (int e = 0; e < kE; ++e) {
      float v = acc[j][e];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) s_part[warp][j][e] = v;
    }
  __syncthreads();
  if (threadIdx.x < kTPB && t0 + threadIdx.x < T) {
    const int j = threadIdx.x;
    float l[kE];
#pragma unroll
    for (int e = 0; e < kE; ++e) {
      float v = 0.f;
      for (int k = 0; k < kWarps; ++k) v += s_part[k][j][e];
      l[e] = v + (bias ? __ldg(bias + e) : 0.f);
    }
    finish_token(l, t0 + j, logits, idx, w);
  }
}

// ------------------------------------------------------------------ tensor cores
// The logits of a bf16 layer as tcgen05 MMAs per 64-token tile: A = 64 rows of
// x (K-major, 128-byte swizzle, streamed by TMA in 64-column K blocks), B = the
// 8 rows of W_r (K-major), D = 64 x 8 fp32 in TMEM.  The contraction is the
// page's hidden @ W_r.T itself; T*d*E multiply-adds on the CUDA cores take
// about as long as reading x from HBM once the clocks sit at the power cap, so
// on the tensor cores the kernel is left with only the stream of x.
//
// Every logit is the same fixed sum of four partial sums over the quarters of
// the hidden dimension, (q0 + q1) + (q2 + q3), each quarter accumulated in its
// own TMEM columns.  A tile's quarters are shared by a cluster of 1, 2 or 4
// CTAs (chosen from the batch size, so that enough CTAs stream x at once);
// the other CTAs send their quarter sums to the cluster's first CTA through
// distributed shared memory, and that CTA adds them in the fixed order and
// finishes the tile's tokens.  The result therefore does not depend on the
// batch size or on the split.  Per CTA, 128 threads: warp 0 lane 0 issues the
// TMA loads into a ring of kRtStages stages, warp 1 lane 0 the MMAs (warp 1
// owns 32 TMEM columns: quarter j at columns 8 j), and all four warps read the
// accumulators (M = 64: tile row 16 q + i sits in lane i < 16 of TMEM lane
// quarter q).  Every wait is bounded; a timeout flags the device error word.
constexpr int kRtM = 64;
constexpr int kRtBK = 64;
constexpr int kRtKB = 2;       // K blocks per stage: one TMA box of [2 blocks][64 rows][64]
constexpr int kRtStages = 5;   // with the receive buffer: two CTAs fit one SM's shared memory
constexpr int kRtParts = 4;             // K quarters
constexpr int kRtA1 = kRtM * kRtBK * 2;  // 8 KB of x per K block
constexpr int kRtB1 = kE * kRtBK * 2;    // 1 KB of W_r per K block (one 8-row swizzle atom)
constexpr int kRtA = kRtKB * kRtA1;
constexpr int kRtB = kRtKB * kRtB1;
constexpr int kRtRecv = kRtParts * kRtM * kE * 4;  // quarter sums received by the first CTA
constexpr int kRtSmem = 1024 + kRtStages * (kRtA + kRtB) + kRtRecv + 256;
constexpr uint32_t kRtIdesc = ptx::idesc_bf16_f32(kRtM, kE, false, false);
static_assert(2 * (kRtSmem + 1024) <= 228 * 1024, "two router CTAs per SM");

// First K block of quarter j of num_kb blocks.
__device__ __forceinline__ int rt_part_begin(int j, int num_kb) { return j * num_kb / kRtParts; }

__global__ void __launch_bounds__(128) router_tc_kernel(const __grid_constant__ CUtensorMap tmx,
                                                        const __grid_constant__ CUtensorMap tmw,
                                                        const float* __restrict__ bias, float* __restrict__ logits,
                                                        int32_t* __restrict__ idx, float* __restrict__ w, int64_t T,
                                                        int num_kb, int nsplit, int* err) {
  using namespace ptx;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* sA = smem;
  uint8_t* sB = smem + kRtStages * kRtA;
  float* recv = reinterpret_cast<float*>(sB + kRtStages * kRtB);  // [quarter][row][expert]
  uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(recv) + kRtRecv);
  uint64_t* empty = full + kRtStages;
  uint64_t* done = empty + kRtStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int m0 = (int)(blockIdx.x / (unsigned)nsplit) * kRtM;
  // this CTA's quarters [j0, j1) and K blocks [kb0, kb1)
  const int per = kRtParts / nsplit;
  const int j0 = (int)rank * per, j1 = j0 + per;
  const int kb0 = rt_part_begin(j0, num_kb), kb1 = rt_part_begin(j1, num_kb);
  const int n_kb = kb1 - kb0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRtStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 1) {
    prefetch_tmap(&tmx);
    prefetch_tmap(&tmw);
  }
  pdl_wait();
  if (warp == 1) {
    tmem_alloc(tmem_slot, 32);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- producer
    const uint64_t once = policy_evict_first();
    const uint64_t keep = policy_evict_last();
    // stage i holds K blocks kb0 + kRtKB i .. + kRtKB - 1 (a box may run past this
    // CTA's range or the tensor's end: those blocks are loaded, or zero-filled,
    // and not multiplied)
    const int n_st = (n_kb + kRtKB - 1) / kRtKB;
    int i = 0;
    for (; i < n_st; ++i) {
      const int s = i % kRtStages;
      const uint32_t ph = (uint32_t)(i / kRtStages) & 1u;
      if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) {
        flag_error(err, MOE_DEVERR_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      mbar_arrive_expect_tx(&full[s], kRtA + kRtB);
      tma_load_3d_hint(sA + s * kRtA, &tmx, &full[s], 0, m0, kb0 + kRtKB * i, once);
      tma_load_3d_hint(sB + s * kRtB, &tmw, &full[s], 0, 0, kb0 + kRtKB * i, keep);
    }
    // drain: every issued load must land before the CTA can exit
    const int first = i > kRtStages ? i - kRtStages : 0;
    for (int j = first; j < i; ++j)
      mbar_wait(&full[j % kRtStages], (uint32_t)(j / kRtStages) & 1u, nullptr, 100000000ull);
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------------- MMA issuer
    bool issued = false;
    int j = j0;
    const int n_st = (n_kb + kRtKB - 1) / kRtKB;
    for (int i = 0; i < n_st; ++i) {
      const int s = i % kRtStages;
      const uint32_t ph = (uint32_t)(i / kRtStages) & 1u;
      if (!mbar_wait(&full[s], ph, abort_flag)) {
        flag_error(err, MOE_DEVERR_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int u = 0; u < kRtKB; ++u) {
        const int kb = kb0 + kRtKB * i + u;
        if (kb >= kb1) break;
        while (kb >= rt_part_begin(j + 1, num_kb)) ++j;  // the quarter this K block belongs to
        const uint32_t a_addr = smem_u32(sA + s * kRtA + u * kRtA1);
        const uint32_t b_addr = smem_u32(sB + s * kRtB + u * kRtB1);
        const uint32_t d_tmem = tmem_base + (uint32_t)(kE * (j - j0));
        const bool first_of_part = kb == rt_part_begin(j, num_kb);
#pragma unroll
        for (int kk = 0; kk < kRtBK / 16; ++kk)
          umma_bf16(d_tmem, sw128_desc(a_addr + kk * 32, 16, 1024), sw128_desc(b_addr + kk * 32, 16, 1024),
                    kRtIdesc, (first_of_part && kk == 0) ? 0u : 1u);
      }
      issued = true;
      umma_commit(&empty[s]);
    }
    // the epilogue waits for every MMA issued; this lane also waits (without
    // the abort flag) so that TMEM is never released under a running MMA
    if (issued) {
      umma_commit(done);
      mbar_wait(done, 0, nullptr, 100000000ull);
    }
  }
  __syncwarp();

  // ------------------------------------------------------------------ epilogue
  // quarter sums of this CTA (a quarter with no K block sums to 0)
  const bool ok = n_kb == 0 || (mbar_wait(done, 0, abort_flag) && !*abort_flag);
  tc_fence_after();
  __syncwarp();
  float part[kRtParts][kE];
#pragma unroll
  for (int q = 0; q < kRtParts; ++q) {
    uint32_t v[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (q < per && n_kb > 0) {
      tmem_ld8(tmem_base + ((uint32_t)(warp * 32) << 16) + (uint32_t)(kE * q), v);
      tmem_wait_ld();
    }
    const int jq = j0 + q;
    const bool empty_part = rt_part_begin(jq, num_kb) == rt_part_begin(jq + 1, num_kb);
#pragma unroll
    for (int e = 0; e < kE; ++e) part[q][e] = empty_part ? 0.f : __uint_as_float(v[e]);
  }
  const int r = warp * 16 + lane;  // tile row held by this thread (lanes < 16)
  if (rank != 0 && lane < 16) {
    // send this CTA's quarter sums to the first CTA of the cluster
    const uint32_t dst = mapa_shared(smem_u32(recv), 0);
#pragma unroll
    for (int q = 0; q < kRtParts; ++q)
      if (q < per) {
#pragma unroll
        for (int e = 0; e < kE; ++e)
          st_cluster_u32(dst + 4u * (uint32_t)(((j0 + q) * kRtM + r) * kE + e), __float_as_uint(part[q][e]));
      }
  }
  if (!ok && lane == 0) flag_error(err, MOE_DEVERR_TIMEOUT);
  tc_fence_before();
  cluster_sync();  // quarter sums delivered; every CTA's TMEM reads are done
  if (rank == 0 && lane < 16) {
    const int64_t t = (int64_t)m0 + r;
    if (t < T) {
      float q4[kRtParts][kE];
#pragma unroll
      for (int q = 0; q < kRtParts; ++q)
#pragma unroll
        for (int e = 0; e < kE; ++e) q4[q][e] = q < per ? part[q][e] : recv[(q * kRtM + r) * kE + e];
      float l[kE];
#pragma unroll
      for (int e = 0; e < kE; ++e)
        l[e] = ((q4[0][e] + q4[1][e]) + (q4[2][e] + q4[3][e])) + (bias ? __ldg(bias + e) : 0.f);
      finish_token(l, t, logits, idx, w);
    }
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 32);
  }
}

cudaError_t launch_router_tc(const moe_config_t& c, const void* x, const void* wr, const float* bias, float* logits,
                             int32_t* idx, float* w, cudaStream_t s, const Ctx& ctx) {
  // 3-D views {64 columns, rows, K block}: a box of kRtKB blocks lands as kRtKB
  // consecutive [rows][64] tiles, each a run of 128-byte swizzle atoms
  CUtensorMap tx, tw;
  const uint64_t x_dims[3] = {(uint64_t)kRtBK, (uint64_t)c.T, (uint64_t)(c.d / kRtBK)};
  const uint64_t w_dims[3] = {(uint64_t)kRtBK, (uint64_t)kE, (uint64_t)(c.d / kRtBK)};
  const uint64_t str[2] = {(uint64_t)c.d * 2, (uint64_t)kRtBK * 2};
  const uint32_t x_box[3] = {kRtBK, kRtM, kRtKB};
  const uint32_t w_box[3] = {kRtBK, kE, kRtKB};
  if (!encode_tmap(&tx, x, 3, x_dims, str, x_box, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap(&tw, wr, 3, w_dims, str, w_box, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(router_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kRtSmem);
  if (e != cudaSuccess) return e;
  const int64_t tiles = (c.T + kRtM - 1) / kRtM;
  // CTAs per tile: enough that about 1.5 CTAs per SM stream x at once (two fit per SM)
  int nsplit = 1;
  while (nsplit < kRtParts && tiles * nsplit * 2 < (int64_t)ctx.num_sms * 3) nsplit *= 2;
  cudaLaunchAttribute cluster = {};
  cluster.id = cudaLaunchAttributeClusterDimension;
  cluster.val.clusterDim.x = (unsigned)nsplit;
  cluster.val.clusterDim.y = 1;
  cluster.val.clusterDim.z = 1;
  e = launch_pdl(router_tc_kernel, dim3((unsigned)(tiles * nsplit), 1, 1), dim3(128, 1, 1), kRtSmem, s, cluster, tx, tw, bias, logits, idx, w, c.T, (int)(c.d / kRtBK), nsplit,
                         ctx.err);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int kTPB>
cudaError_t launch_router_split(const moe_config_t& c, const void* x, const void* wr, const float* bias,
                                float* logits, int32_t* idx, float* w, cudaStream_t s) {
  const int64_t blocks = (c.T + kTPB - 1) / kTPB;
  if (c.dtype == MOE_BF16)
    router_top2_split_kernel<__nv_bfloat16, kTPB><<<(unsigned)blocks, kWarps * 32, 0, s>>>(
        static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(wr), bias, logits, idx, w, c.T, c.d);
  else
    router_top2_split_kernel<float, kTPB><<<(unsigned)blocks, kWarps * 32, 0, s>>>(
        static_cast<const float*>(x), static_cast<const float*>(wr), bias, logits, idx, w, c.T, c.d);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_router(const moe_config_t& c, const void* x, const void* wr, const float* bias,
                          float* logits, int32_t* idx, float* w, cudaStream_t s, const Ctx& ctx) {
  if (c.T == 0) return cudaSuccess;
  // bf16: the tensor-core kernel at every batch size, so a token's logits do not
  // depend on the batch it arrives in
  if (c.dtype == MOE_BF16 && c.E == kE && c.d % kRtBK == 0)
    return launch_router_tc(c, x, wr, bias, logits, idx, w, s, ctx);
  if (c.T <= (int64_t)ctx.num_sms * 2) return launch_router_split<1>(c, x, wr, bias, logits, idx, w, s);
  return launch_router_split<4>(c, x, wr, bias, logits, idx, w, s);
}

}  // namespace moe
