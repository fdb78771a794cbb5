// Weighted combine back to token order.
//
// "How does Grok-1 use a mixture-of-experts design?", section "The high-level
// architecture": `_dispatch_and_combine(...).view_as(x)` returns, for every
// token, the routing-weighted sum of its experts' outputs (the page "Let Grok
// spill the beans on Grok" names it a weighted sum); section "Expert
// parallelism vs. tensor parallelism" scales each expert output by its weight.
//
// out[t] = sum_{j: slot_of[t,j] >= 0} s_j * y[slot_of[t,j]] in fp32, j = 0
// first, then one rounding to the output type.  A fixed order and a zero start
// make the result independent of scheduling.  HBM-bound: one block per token
// row per iteration, 16-byte loads of y.
#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

// y of a slot = sum over p < n_parts of y[p * part_stride + slot * d + ...], parts
// added in order (K-split partials of the 8-bit down pass; 1 part otherwise).
__device__ __forceinline__ float4 slot_row(const float* y, int n_parts, int64_t part_stride, int64_t off) {
  float4 a = __ldg(reinterpret_cast<const float4*>(y + off));
  for (int p = 1; p < n_parts; ++p) {
    const float4 b = __ldg(reinterpret_cast<const float4*>(y + p * part_stride + off));
    a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
  }
  return a;
}

template <bool kBf16Out>
__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ y, int n_parts, int64_t part_stride,
                                                     const int32_t* __restrict__ slot_of,
                                                     const float* __restrict__ topk_w, int weights_applied, int64_t T,
                                                     int64_t d, int64_t max_slot, void* __restrict__ out, int* err) {
  const int64_t nvec = d / 4;  // float4 groups per row
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    const int2 sl = __ldg(reinterpret_cast<const int2*>(slot_of) + t);
    int s0 = sl.x, s1 = sl.y;
    if (s0 >= max_slot || s0 < -1 || s1 >= max_slot || s1 < -1) {
      if (threadIdx.x == 0) flag_error(err, MOE_DEVERR_SLOT_INDEX);
      if (s0 >= max_slot || s0 < -1) s0 = -1;
      if (s1 >= max_slot || s1 < -1) s1 = -1;
    }
    float c0 = 1.f, c1 = 1.f;
    if (!weights_applied) {
      const float2 wt = __ldg(reinterpret_cast<const float2*>(topk_w) + t);
      c0 = wt.x;
      c1 = wt.y;
    }
    const int64_t r0 = (int64_t)(s0 < 0 ? 0 : s0) * d, r1 = (int64_t)(s1 < 0 ? 0 : s1) * d;
    for (int64_t v = threadIdx.x; v < nvec; v += blockDim.x) {
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
      if (s0 >= 0) {
        const float4 p = slot_row(y, n_parts, part_stride, r0 + 4 * v);
        a.x += c0 * p.x; a.y += c0 * p.y; a.z += c0 * p.z; a.w += c0 * p.w;
      }
      if (s1 >= 0) {
        const float4 p = slot_row(y, n_parts, part_stride, r1 + 4 * v);
        a.x += c1 * p.x; a.y += c1 * p.y; a.z += c1 * p.z; a.w += c1 * p.w;
      }
      if (kBf16Out) {
        uint2 o;
        o.x = pack_bf16x2(a.x, a.y);
        o.y = pack_bf16x2(a.z, a.w);
        reinterpret_cast<uint2*>(out)[t * nvec + v] = o;
      } else {
        reinterpret_cast<float4*>(out)[t * nvec + v] = a;
      }
    }
  }
}

__global__ void __launch_bounds__(256) zero_kernel(float4* __restrict__ p, int64_t n4) {
  pdl_wait();
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x)
    p[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// The fused down pass leaves out32[t] = fp32 sum of the token's weighted expert
// outputs; one rounding to the output type finishes the combine.
template <bool kBf16Out>
__global__ void __launch_bounds__(256) round_out_kernel(const float4* __restrict__ src, void* __restrict__ out,
                                                        int64_t n4) {
  pdl_wait();
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x) {
    const float4 a = __ldg(src + i);
    if (kBf16Out) {
      uint2 o;
      o.x = pack_bf16x2(a.x, a.y);
      o.y = pack_bf16x2(a.z, a.w);
      reinterpret_cast<uint2*>(out)[i] = o;
    } else {
      reinterpret_cast<float4*>(out)[i] = a;
    }
  }
}

unsigned grid_for(int64_t n4, const Ctx& ctx) {
  const int64_t want = (n4 + 255) / 256;
  const int64_t cap = (int64_t)ctx.num_sms * 8;
  return (unsigned)(want < cap ? (want < 1 ? 1 : want) : cap);
}

}  // namespace

cudaError_t launch_zero_rows(const moe_config_t& c, float* out32, cudaStream_t s, const Ctx& ctx) {
  const int64_t n4 = c.T * c.d / 4;
  if (n4 == 0) return cudaSuccess;
  const cudaError_t e = launch_pdl(zero_kernel, dim3(grid_for(n4, ctx)), dim3(256), 0, s, no_extra_attr(),
                                   reinterpret_cast<float4*>(out32), n4);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_round_out(const moe_config_t& c, const float* out32, void* out, cudaStream_t s, const Ctx& ctx) {
  const int64_t n4 = c.T * c.d / 4;
  if (n4 == 0) return cudaSuccess;
  const cudaError_t e =
      launch_pdl(c.dtype == MOE_BF16 ? round_out_kernel<true> : round_out_kernel<false>, dim3(grid_for(n4, ctx)),
                 dim3(256), 0, s, no_extra_attr(), reinterpret_cast<const float4*>(out32), out, n4);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_combine(const moe_config_t& c, const float* y, const int32_t* slot_of,
                           const float* topk_w, int weights_applied, void* out, cudaStream_t s,
                           const Ctx& ctx, int n_parts, int64_t part_stride) {
  if (c.T == 0) return cudaSuccess;
  int64_t blocks = c.T;
  const int64_t cap_blocks = (int64_t)ctx.num_sms * 8;
  if (blocks > cap_blocks) blocks = cap_blocks;
  const int64_t max_slot = slot_rows(c);
  if (c.dtype == MOE_BF16)
    combine_kernel<true><<<(unsigned)blocks, 256, 0, s>>>(y, n_parts, part_stride, slot_of, topk_w, weights_applied,
                                                          c.T, c.d, max_slot, out, ctx.err);
  else
    combine_kernel<false><<<(unsigned)blocks, 256, 0, s>>>(y, n_parts, part_stride, slot_of, topk_w,
                                                           weights_applied, c.T, c.d, max_slot, out, ctx.err);
  return cudaGetLastError();
}

}  // namespace moe
