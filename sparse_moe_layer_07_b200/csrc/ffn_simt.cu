// fp32 expert FFN on the CUDA cores.
//
// Same operation as the tensor-core path ("How does Grok-1 use a
// mixture-of-experts design?", section "Expert implementation: SwiGLU at
// scale": y = W_down(silu(W_gate x) * W_up x)), for fp32 layers.  TF32 tensor
// cores carry a 10-bit mantissa, too coarse for an fp32 result, so this path
// uses plain fp32 FMA with a fixed accumulation order.
//
// Grouped tiling: blockIdx.y enumerates the 64-row blocks of every expert
// (read from the device offsets), blockIdx.x the 64-column output blocks.
// 256 threads, each owns a 4 x 4 sub-tile; K advances 16 at a time through
// shared memory.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kE = 8;
constexpr int TM = 64, TN = 64, TK = 16;

// Locate the 64-row block `mb` among the experts; false if past the end.
__device__ __forceinline__ bool find_block(const int32_t* offsets, int64_t max_rows, int mb, int& e_out, int& m0,
                                           int& rows, int* err) {
  int acc = 0;
  int prev = 0;
  for (int e = 0; e < kE; ++e) {
    const int lo = offsets[e], hi = offsets[e + 1];
    if (lo < prev || hi < lo || (int64_t)hi > max_rows) {
      if (threadIdx.x == 0 && blockIdx.x == 0) flag_error(err, MOE_DEVERR_OFFSETS);
      return false;
    }
    prev = lo;
    const int nb = (hi - lo + TM - 1) / TM;
    if (mb < acc + nb) {
      e_out = e;
      m0 = lo + (mb - acc) * TM;
      rows = hi - m0 < TM ? hi - m0 : TM;
      return true;
    }
    acc += nb;
  }
  return false;
}

template <bool kGateUp>
__global__ void __launch_bounds__(256) ffn_simt_kernel(const float* __restrict__ A, const int32_t* __restrict__ offsets,
                                                      const float* __restrict__ W0, const float* __restrict__ W1,
                                                      const float* __restrict__ row_scale, float* __restrict__ out,
                                                      int64_t K, int64_t N, int64_t max_rows, int* err) {
  __shared__ float sA[TK][TM + 4];
  __shared__ float sW0[TK][TN];
  __shared__ float sW1[kGateUp ? TK : 1][TN];
  int e, m0, rows;
  if (!find_block(offsets, max_rows, blockIdx.y, e, m0, rows, err)) return;
  const int n0 = blockIdx.x * TN;
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const float* W0e = W0 + (int64_t)e * K * N;
  const float* W1e = kGateUp ? W1 + (int64_t)e * K * N : nullptr;

  float acc0[4][4], acc1[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc0[i][j] = acc1[i][j] = 0.f;

  const int ar = tid >> 2, ak = (tid & 3) * 4;    // A tile loader: row, k
  const int wk = tid >> 4, wn = (tid & 15) * 4;  // W tile loader: k, n
  for (int64_t k0 = 0; k0 < K; k0 += TK) {
    float4 av = make_float4(0.f, 0.f, 0.f, 0.f);
    if (ar < rows) av = __ldg(reinterpret_cast<const float4*>(A + (int64_t)(m0 + ar) * K + k0 + ak));
    sA[ak + 0][ar] = av.x;
    sA[ak + 1][ar] = av.y;
    sA[ak + 2][ar] = av.z;
    sA[ak + 3][ar] = av.w;
    *reinterpret_cast<float4*>(&sW0[wk][wn]) =
        __ldg(reinterpret_cast<const float4*>(W0e + (k0 + wk) * N + n0 + wn));
    if (kGateUp)
      *reinterpret_cast<float4*>(&sW1[wk][wn]) =
          __ldg(reinterpret_cast<const float4*>(W1e + (k0 + wk) * N + n0 + wn));
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float a[4], b0[4], b1[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = sA[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b0[j] = sW0[kk][tx * 4 + j];
      if (kGateUp) {
#pragma unroll
        for (int j = 0; j < 4; ++j) b1[j] = sW1[kk][tx * 4 + j];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc0[i][j] = fmaf(a[i], b0[j], acc0[i][j]);
          if (kGateUp) acc1[i][j] = fmaf(a[i], b1[j], acc1[i][j]);
        }
    }
    __syncthreads();
  }

#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = ty * 4 + i;
    if (r >= rows) continue;
    float v[4];
    if (kGateUp) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float g = acc0[i][j];
        v[j] = g / (1.0f + expf(-g)) * acc1[i][j];
      }
    } else {
      const float sc = row_scale ? __ldg(row_scale + m0 + r) : 1.0f;
#pragma unroll
      for (int j = 0; j < 4; ++j) v[j] = sc * acc0[i][j];
    }
    *reinterpret_cast<float4*>(out + (int64_t)(m0 + r) * N + n0 + tx * 4) = make_float4(v[0], v[1], v[2], v[3]);
  }
}

inline unsigned max_row_blocks(const moe_config_t& c) {
  return (unsigned)((slot_rows(c) + TM - 1) / TM + kE);
}

}  // namespace

cudaError_t launch_ffn_simt_gate_up(const moe_config_t& c, const float* x_perm, const int32_t* offsets,
                                    const float* wg, const float* wu, float* h, cudaStream_t s, const Ctx& ctx) {
  if (slot_rows(c) == 0) return cudaSuccess;
  dim3 grid((unsigned)(c.f / TN), max_row_blocks(c));
  ffn_simt_kernel<true><<<grid, 256, 0, s>>>(x_perm, offsets, wg, wu, nullptr, h, c.d, c.f, slot_rows(c), ctx.err);
  return cudaGetLastError();
}

cudaError_t launch_ffn_simt_down(const moe_config_t& c, const float* h, const int32_t* offsets, const float* wd,
                                 const float* row_scale, float* y, cudaStream_t s, const Ctx& ctx) {
  if (slot_rows(c) == 0) return cudaSuccess;
  dim3 grid((unsigned)(c.d / TN), max_row_blocks(c));
  ffn_simt_kernel<false><<<grid, 256, 0, s>>>(h, offsets, wd, nullptr, row_scale, y, c.f, c.d, slot_rows(c), ctx.err);
  return cudaGetLastError();
}

}  // namespace moe
