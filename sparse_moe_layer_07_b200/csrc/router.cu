// Router logits + top-2 + softmax over the two selected logits.
//
// "How does Grok-1 use a mixture-of-experts design?", section "Routing: top-2
// without auxiliary loss" (grok_router_forward): logits = hidden @ W_r.T with
// W_r stored [E, hidden]; topk(logits, 2); softmax of the two selected values.
//
// HBM-bound on x for large batches: each warp streams 4 token rows with 16-byte
// loads and reuses every W_r chunk (E rows, L1/L2 resident) for the 4 tokens;
// smaller batches use one token per warp, and decode-sized ones one token per
// block with the hidden dimension split over 8 warps.  Partial sums are reduced
// in a fixed order, so results do not depend on timing.
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

// kTokPerWarp tokens share each W_r chunk a warp loads: 4 for large batches
// (less L1 traffic), 2 or 1 for smaller ones (more warps in flight).
template <typename Tin, int kTokPerWarp>
__global__ void __launch_bounds__(kWarps * 32) router_top2_kernel(const Tin* __restrict__ x, const Tin* __restrict__ wr,
                                                                 const float* __restrict__ bias, float* __restrict__ logits,
                                                                 int32_t* __restrict__ idx, float* __restrict__ w,
                                                                 int64_t T, int64_t d) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int64_t t0 = ((int64_t)blockIdx.x * kWarps + warp) * kTokPerWarp;
  if (t0 >= T) return;

  float acc[kTokPerWarp][kE];
#pragma unroll
  for (int j = 0; j < kTokPerWarp; ++j)
#pragma unroll
    for (int e = 0; e < kE; ++e) acc[j][e] = 0.f;

  for (int64_t c = (int64_t)lane * 8; c < d; c += 256) {
    float wv[kE][8];
#pragma unroll
    for (int e = 0; e < kE; ++e) load8(wr + (int64_t)e * d + c, wv[e]);
#pragma unroll
    for (int j = 0; j < kTokPerWarp; ++j) {
      const int64_t t = t0 + j < T ? t0 + j : T - 1;  // clamp: duplicate rows are discarded below
      float xv[8];
      load8(x + t * d + c, xv);
#pragma unroll
      for (int e = 0; e < kE; ++e)
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[j][e] = fmaf(xv[i], wv[e][i], acc[j][e]);
    }
  }

#pragma unroll
  for (int j = 0; j < kTokPerWarp; ++j)
#pragma unroll
    for (int e = 0; e < kE; ++e) {
      float v = acc[j][e];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      acc[j][e] = v;
    }

  if (lane < kTokPerWarp) {
    // lane j finalises token t0 + j (register arrays indexed by a runtime lane
    // would spill, so select with a static loop)
    float l[kE];
#pragma unroll
    for (int j = 0; j < kTokPerWarp; ++j)
      if (lane == j)
#pragma unroll
        for (int e = 0; e < kE; ++e) l[e] = acc[j][e];
    const int64_t t = t0 + lane;
    if (t < T) {
      if (bias) {
#pragma unroll
        for (int e = 0; e < kE; ++e) l[e] += __ldg(bias + e);
      }
      finish_token(l, t, logits, idx, w);
    }
  }
}

// Small batches: one token per block, the 8 warps split the hidden dimension
// (each thread 8 consecutive elements per 2048-wide step) and their partial
// logits are summed in warp order, so latency is a few steps instead of d/256.
template <typename Tin>
__global__ void __launch_bounds__(kWarps * 32) router_top2_split_kernel(const Tin* __restrict__ x,
                                                                       const Tin* __restrict__ wr,
                                                                       const float* __restrict__ bias,
                                                                       float* __restrict__ logits,
                                                                       int32_t* __restrict__ idx,
                                                                       float* __restrict__ w, int64_t d) {
  __shared__ float s_part[kWarps][kE];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int64_t t = blockIdx.x;
  float acc[kE];
#pragma unroll
  for (int e = 0; e < kE; ++e) acc[e] = 0.f;
  for (int64_t c = (int64_t)threadIdx.x * 8; c < d; c += kWarps * 32 * 8) {
    float xv[8];
    load8(x + t * d + c, xv);
#pragma unroll
    for (int e = 0; e < kE; ++e) {
      float wv[8];
      load8(wr + (int64_t)e * d + c, wv);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[e] = fmaf(xv[i], wv[i], acc[e]);
    }
  }
#pragma unroll
  for (int e = 0; e < kE; ++e) {
    float v = acc[e];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) s_part[warp][e] = v;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float l[kE];
#pragma unroll
    for (int e = 0; e < kE; ++e) {
      float v = 0.f;
      for (int k = 0; k < kWarps; ++k) v += s_part[k][e];
      l[e] = v + (bias ? __ldg(bias + e) : 0.f);
    }
    finish_token(l, t, logits, idx, w);
  }
}

template <int kTPW>
cudaError_t launch_router_t(const moe_config_t& c, const void* x, const void* wr, const float* bias, float* logits,
                            int32_t* idx, float* w, cudaStream_t s) {
  const int64_t tok_per_block = kWarps * kTPW;
  const int64_t blocks = (c.T + tok_per_block - 1) / tok_per_block;
  if (blocks == 0) return cudaSuccess;
  if (c.dtype == MOE_BF16)
    router_top2_kernel<__nv_bfloat16, kTPW><<<(unsigned)blocks, kWarps * 32, 0, s>>>(
        static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(wr), bias, logits, idx, w, c.T, c.d);
  else
    router_top2_kernel<float, kTPW><<<(unsigned)blocks, kWarps * 32, 0, s>>>(
        static_cast<const float*>(x), static_cast<const float*>(wr), bias, logits, idx, w, c.T, c.d);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_router(const moe_config_t& c, const void* x, const void* wr, const float* bias,
                          float* logits, int32_t* idx, float* w, cudaStream_t s, const Ctx& ctx) {
  if (c.T == 0) return cudaSuccess;
  if (c.T <= (int64_t)ctx.num_sms * 2) {
    if (c.dtype == MOE_BF16)
      router_top2_split_kernel<__nv_bfloat16><<<(unsigned)c.T, kWarps * 32, 0, s>>>(
          static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(wr), bias, logits, idx, w, c.d);
    else
      router_top2_split_kernel<float><<<(unsigned)c.T, kWarps * 32, 0, s>>>(
          static_cast<const float*>(x), static_cast<const float*>(wr), bias, logits, idx, w, c.d);
    return cudaGetLastError();
  }
  // tokens per warp: as many as keep at least two blocks per SM (x is streamed
  // once, so warps in flight set the speed; more tokens per warp share W_r loads)
  if (c.T <= (int64_t)ctx.num_sms * kWarps) return launch_router_t<1>(c, x, wr, bias, logits, idx, w, s);
  if (c.T <= (int64_t)ctx.num_sms * kWarps * 4 * 2) return launch_router_t<2>(c, x, wr, bias, logits, idx, w, s);
  return launch_router_t<4>(c, x, wr, bias, logits, idx, w, s);
}

}  // namespace moe
