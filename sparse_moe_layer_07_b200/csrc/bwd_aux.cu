// Memory-bound pieces of the layer's backward (training), on the CUDA cores.
//
// The router of "How does Grok-1 use a mixture-of-experts design?" (section
// "Routing: top-2 without auxiliary loss") computes logits = x W_r^T (+ bias),
// keeps the two largest and takes a softmax over those two.  With the routing
// decisions held fixed, the gradient reaches the router through the softmax:
//   dweight[t, j] = <dout_t, y_{t,j}>  (0 for a dropped assignment)
//   dlogits[t, idx[t, j]] = w_j * (dweight_j - sum_i w_i dweight_i)
//   dx_t += dlogits_t W_r,  dW_r = dlogits^T x,  dbias = sum_t dlogits_t
// dweight arrives as per-tile partial dot products from the kDH GEMM epilogue
// and is summed here in tile order; every reduction has a fixed order, so the
// results do not depend on scheduling.
#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kE = 8;

__device__ __forceinline__ void unpack8(const uint4 q, float (&v)[8]) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}

// One warp per grouped row: dout_perm[r] = dout[perm[r]] (a copy) and
// dy_perm[r] = bf16(row_scale[r] * dout[perm[r]]), 8 values per 16-byte vector.
__global__ void __launch_bounds__(256) bwd_gather_kernel(const uint4* __restrict__ dout, const int32_t* __restrict__ perm,
                                                        const int32_t* __restrict__ offsets,
                                                        const float* __restrict__ row_scale, int64_t T,
                                                        int64_t row_vec, uint4* __restrict__ dout_perm,
                                                        uint4* __restrict__ dy_perm, int* err) {
  int64_t n = offsets[kE];
  if (n < 0 || n > 2 * T) {
    if (blockIdx.x == 0 && threadIdx.x == 0) flag_error(err, MOE_DEVERR_OFFSETS);
    n = 0;
  }
  const int lane = threadIdx.x & 31;
  const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t r = gw; r < n; r += nw) {
    const int32_t t = __ldg(perm + r);
    if (t < 0 || t >= T) {
      if (lane == 0) flag_error(err, MOE_DEVERR_SLOT_INDEX);
      continue;
    }
    const float w = __ldg(row_scale + r);
    for (int64_t v = lane; v < row_vec; v += 32) {
      const uint4 q = __ldg(dout + t * row_vec + v);
      dout_perm[r * row_vec + v] = q;
      float f[8];
      unpack8(q, f);
      dy_perm[r * row_vec + v] =
          make_uint4(pack_bf16x2(w * f[0], w * f[1]), pack_bf16x2(w * f[2], w * f[3]),
                     pack_bf16x2(w * f[4], w * f[5]), pack_bf16x2(w * f[6], w * f[7]));
    }
  }
}

// One warp per token: lanes 0 and 1 form the routing-weight gradient of slot
// 0 / 1 (partials summed in tile order), every lane then has the two logit
// gradients, lanes 0-7 write the token's dlogits row, and the warp streams
// dx[t] = round(dx32[t] + dl_0 W_r[i_0] + dl_1 W_r[i_1]) (slot 0 first), four
// columns per lane and 16-byte vector, four vectors in flight per lane.
__global__ void __launch_bounds__(256) router_bwd_token_kernel(
    const float* __restrict__ dw_part, int n_parts, const int32_t* __restrict__ slot_of,
    const int32_t* __restrict__ topk_idx, const float* __restrict__ topk_w, const __nv_bfloat16* __restrict__ wr,
    const float* __restrict__ dx32, int64_t T, int64_t d, int64_t max_slot, float* __restrict__ dlogits,
    float* __restrict__ dweight, __nv_bfloat16* __restrict__ dx, int* err) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int nq = (int)(d / 4);  // 4-column groups of a row (d is a multiple of 128)
  for (int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += warps) {
    int e = 0;
    float w = 0.f, dw = 0.f;
    if (lane < 2) {
      int sl = slot_of[2 * t + lane];
      e = topk_idx[2 * t + lane];
      w = topk_w[2 * t + lane];
      if (sl >= max_slot || sl < -1) {
        flag_error(err, MOE_DEVERR_SLOT_INDEX);
        sl = -1;
      }
      if (e < 0 || e >= kE) {
        flag_error(err, MOE_DEVERR_EXPERT_INDEX);
        e = 0;
        w = 0.f;
      }
      if (sl >= 0)
        for (int p = 0; p < n_parts; ++p) dw += dw_part[(int64_t)sl * n_parts + p];
      dweight[2 * t + lane] = dw;
    }
    const int e0 = __shfl_sync(0xffffffffu, e, 0), e1 = __shfl_sync(0xffffffffu, e, 1);
    const float w0 = __shfl_sync(0xffffffffu, w, 0), w1 = __shfl_sync(0xffffffffu, w, 1);
    const float dw0 = __shfl_sync(0xffffffffu, dw, 0), dw1 = __shfl_sync(0xffffffffu, dw, 1);
    const float mean = w0 * dw0 + w1 * dw1;
    const float dl0 = w0 * (dw0 - mean);
    const float dl1 = w1 * (dw1 - mean);
    if (lane < kE) {
      float v = 0.f;
      if (e0 == lane) v += dl0;
      if (e1 == lane) v += dl1;
      dlogits[t * kE + lane] = v;
    }
    const float4* a4 = reinterpret_cast<const float4*>(dx32 + t * d);
    const uint2* p2 = reinterpret_cast<const uint2*>(wr + (int64_t)e0 * d);
    const uint2* q2 = reinterpret_cast<const uint2*>(wr + (int64_t)e1 * d);
    uint2* o2 = reinterpret_cast<uint2*>(dx + t * d);
    for (int g0 = lane; g0 < nq; g0 += 128) {
      float4 a[4];
      uint2 pb[4], qb[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int g = g0 + 32 * k;
        if (g < nq) {
          a[k] = __ldcs(a4 + g);
          pb[k] = p2[g];
          qb[k] = q2[g];
        }
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int g = g0 + 32 * k;
        if (g < nq) {
          const float2 p01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pb[k].x));
          const float2 p23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pb[k].y));
          const float2 q01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qb[k].x));
          const float2 q23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qb[k].y));
          float v0 = a[k].x + dl0 * p01.x, v1 = a[k].y + dl0 * p01.y;
          float v2 = a[k].z + dl0 * p23.x, v3 = a[k].w + dl0 * p23.y;
          v0 = v0 + dl1 * q01.x;
          v1 = v1 + dl1 * q01.y;
          v2 = v2 + dl1 * q23.x;
          v3 = v3 + dl1 * q23.y;
          o2[g] = make_uint2(pack_bf16x2(v0, v1), pack_bf16x2(v2, v3));
        }
      }
    }
  }
}

// dW_r partial sums over token chunks: part[c][e][i] = sum_{t in chunk c} dlogits[t, e] x[t, i]
// (tokens in increasing order); a thread owns 8 adjacent columns (one 16-byte
// vector of x per token) for all 8 experts, and keeps two tokens' loads in flight.
__global__ void __launch_bounds__(256) router_bwd_weight_kernel(const float* __restrict__ dlogits,
                                                               const __nv_bfloat16* __restrict__ x, int64_t T,
                                                               int64_t d, int chunks, float* __restrict__ part) {
  const int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // 8-column group
  const int c = blockIdx.y;
  const int64_t per = (T + chunks - 1) / chunks;
  const int64_t t0 = c * per;
  const int64_t t1 = t0 + per < T ? t0 + per : T;
  const int64_t nv = d / 8;
  if (v >= nv) return;
  float acc[kE][8];
#pragma unroll
  for (int e = 0; e < kE; ++e)
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[e][k] = 0.f;
  const uint4* x4 = reinterpret_cast<const uint4*>(x);
  int64_t t = t0;
  for (; t + 1 < t1; t += 2) {
    const uint4 qa = __ldcs(x4 + t * nv + v);
    const uint4 qb = __ldcs(x4 + (t + 1) * nv + v);
    float xa[8], xb[8];
    unpack8(qa, xa);
    unpack8(qb, xb);
#pragma unroll
    for (int e = 0; e < kE; ++e) {
      const float la = __ldg(dlogits + t * kE + e);
      const float lb = __ldg(dlogits + (t + 1) * kE + e);
#pragma unroll
      for (int k = 0; k < 8; ++k) acc[e][k] = fmaf(lb, xb[k], fmaf(la, xa[k], acc[e][k]));
    }
  }
  if (t < t1) {
    float xa[8];
    unpack8(__ldcs(x4 + t * nv + v), xa);
#pragma unroll
    for (int e = 0; e < kE; ++e) {
      const float la = __ldg(dlogits + t * kE + e);
#pragma unroll
      for (int k = 0; k < 8; ++k) acc[e][k] = fmaf(la, xa[k], acc[e][k]);
    }
  }
#pragma unroll
  for (int e = 0; e < kE; ++e) {
    float4* o = reinterpret_cast<float4*>(part + ((int64_t)c * kE + e) * d + v * 8);
    o[0] = make_float4(acc[e][0], acc[e][1], acc[e][2], acc[e][3]);
    o[1] = make_float4(acc[e][4], acc[e][5], acc[e][6], acc[e][7]);
  }
}

// dW_r[e][i] = sum over chunks in order; block 0 also forms dbias[e] = sum_t dlogits[t, e]
// (each thread a strided subset of tokens, then a fixed tree).
__global__ void __launch_bounds__(256) router_bwd_reduce_kernel(const float* __restrict__ part, int chunks,
                                                               const float* __restrict__ dlogits, int64_t T,
                                                               int64_t d, float* __restrict__ dw_router,
                                                               float* __restrict__ dbias) {
  const int64_t n = (int64_t)kE * d;
  for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < n; k += (int64_t)gridDim.x * blockDim.x) {
    float acc = 0.f;
    for (int c = 0; c < chunks; ++c) acc += part[(int64_t)c * n + k];
    dw_router[k] = acc;
  }
  if (blockIdx.x != 0 || dbias == nullptr) return;
  __shared__ float s[kE][256];
  float acc[kE];
#pragma unroll
  for (int e = 0; e < kE; ++e) acc[e] = 0.f;
  for (int64_t t = threadIdx.x; t < T; t += blockDim.x)
#pragma unroll
    for (int e = 0; e < kE; ++e) acc[e] += dlogits[t * kE + e];
#pragma unroll
  for (int e = 0; e < kE; ++e) s[e][threadIdx.x] = acc[e];
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if ((int)threadIdx.x < w)
#pragma unroll
      for (int e = 0; e < kE; ++e) s[e][threadIdx.x] += s[e][threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x < kE) dbias[threadIdx.x] = s[threadIdx.x][0];
}

unsigned capped(int64_t want, const Ctx& ctx, int per_sm = 8) {
  const int64_t cap = (int64_t)ctx.num_sms * per_sm;
  return (unsigned)(want < 1 ? 1 : (want < cap ? want : cap));
}

}  // namespace

cudaError_t launch_bwd_gather(const moe_config_t& c, const void* dout, const int32_t* perm, const int32_t* offsets,
                              const float* row_scale, void* dout_perm, void* dy_perm, cudaStream_t s, const Ctx& ctx) {
  const int64_t rows = slot_rows(c);
  if (rows == 0) return cudaSuccess;
  bwd_gather_kernel<<<capped((rows + 7) / 8, ctx), 256, 0, s>>>(
      static_cast<const uint4*>(dout), perm, offsets, row_scale, c.T, c.d / 8, static_cast<uint4*>(dout_perm),
      static_cast<uint4*>(dy_perm), ctx.err);
  return cudaGetLastError();
}

cudaError_t launch_router_bwd(const moe_config_t& c, const float* dw_part, int n_parts, const int32_t* slot_of,
                              const int32_t* topk_idx, const float* topk_w, const void* w_router, const float* dx32,
                              const void* x, float* dlogits, float* dweight, void* dx, float* dw_router,
                              float* dbias, float* wr_part, cudaStream_t s, const Ctx& ctx) {
  if (c.T == 0) return cudaSuccess;
  router_bwd_token_kernel<<<capped((c.T + 7) / 8, ctx), 256, 0, s>>>(
      dw_part, n_parts, slot_of, topk_idx, topk_w, static_cast<const __nv_bfloat16*>(w_router), dx32, c.T, c.d,
      slot_rows(c), dlogits, dweight, static_cast<__nv_bfloat16*>(dx), ctx.err);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((c.d / 8 + 255) / 256), (unsigned)kRouterBwdChunks);
  router_bwd_weight_kernel<<<grid, 256, 0, s>>>(dlogits, static_cast<const __nv_bfloat16*>(x), c.T, c.d,
                                                kRouterBwdChunks, wr_part);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  router_bwd_reduce_kernel<<<capped((kE * c.d + 255) / 256, ctx), 256, 0, s>>>(wr_part, kRouterBwdChunks, dlogits,
                                                                             c.T, c.d, dw_router, dbias);
  return cudaGetLastError();
}

}  // namespace moe
