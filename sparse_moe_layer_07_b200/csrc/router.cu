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
  if (c.T <= (int64_t)ctx.num_sms * 2) return launch_router_split<1>(c, x, wr, bias, logits, idx, w, s);
  return launch_router_split<4>(c, x, wr, bias, logits, idx, w, s);
}

}  // namespace moe
