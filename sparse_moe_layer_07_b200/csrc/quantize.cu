// Per-output-channel symmetric int8 quantisation of expert weights.
//
// The pages report that the released Grok-1 weights were quantised ("Benchmarking
// xAI's Grok-1", section "Grok-1: In Practice"; "8-Bit Quantization" in the
// feature list of "Let Grok spill the beans on Grok") but give no scheme.  The
// scheme here, with every decision in IEEE fp32:
//   amax[e, n]  = max_k |w[e, k, n]|
//   scale[e, n] = amax[e, n] / 127
//   q[e, k, n]  = clamp(rint(w[e, k, n] / scale[e, n]), -127, 127)   (0 where scale = 0)
// One block owns 64 output channels of one expert: 32 threads x 2 channels
// across (bf16x2 loads, coalesced along the channel axis) and 8 row groups;
// pass 1 reduces amax over K, pass 2 writes the codes.
#include <cuda_bf16.h>
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kRowGroups = 8;

__global__ void __launch_bounds__(32 * kRowGroups) quantize_int8_kernel(const __nv_bfloat16* __restrict__ w, int64_t K,
                                                                       int64_t N, int8_t* __restrict__ q,
                                                                       float* __restrict__ scale) {
  __shared__ float s_amax[kRowGroups][64];
  __shared__ float s_scale[64];
  const int e = blockIdx.y;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int64_t n = (int64_t)blockIdx.x * 64 + 2 * tx;
  const __nv_bfloat16* we = w + (int64_t)e * K * N;
  float a0 = 0.f, a1 = 0.f;
  for (int64_t k = ty; k < K; k += kRowGroups) {
    const float2 v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(we + k * N + n));
    a0 = fmaxf(a0, fabsf(v.x));
    a1 = fmaxf(a1, fabsf(v.y));
  }
  s_amax[ty][2 * tx] = a0;
  s_amax[ty][2 * tx + 1] = a1;
  __syncthreads();
  if (ty == 0) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      float m = 0.f;
#pragma unroll
      for (int g = 0; g < kRowGroups; ++g) m = fmaxf(m, s_amax[g][2 * tx + j]);
      const float sc = m / 127.0f;
      s_scale[2 * tx + j] = sc;
      scale[(int64_t)e * N + n + j] = sc;
    }
  }
  __syncthreads();
  const float s0 = s_scale[2 * tx], s1 = s_scale[2 * tx + 1];
  int8_t* qe = q + (int64_t)e * K * N;
  for (int64_t k = ty; k < K; k += kRowGroups) {
    const float2 v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(we + k * N + n));
    const float r0 = s0 > 0.f ? fminf(fmaxf(rintf(v.x / s0), -127.f), 127.f) : 0.f;
    const float r1 = s1 > 0.f ? fminf(fmaxf(rintf(v.y / s1), -127.f), 127.f) : 0.f;
    char2 c;
    c.x = (signed char)(int)r0;
    c.y = (signed char)(int)r1;
    *reinterpret_cast<char2*>(qe + k * N + n) = c;
  }
}

// 15-bit code of each activation row (the first offsets[E] rows of src):
//   scale = max_k |v_k| / 32512,  c_k = clamp(rint(v_k / scale), -32512, 32512)
//   hi_k = floor((c_k + 128) / 256),  lo_k = c_k - 256 * hi_k   (int8 each)
// One block per row (256 threads, 1024 for rows of 16K values or more): a max
// reduction, then the codes, 4 values per thread step.
constexpr float kRowCodeMax = 32512.0f;

__device__ __forceinline__ void load4(const __nv_bfloat16* p, float (&v)[4]) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
  v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
}
__device__ __forceinline__ void load4(const float* p, float (&v)[4]) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
}

// Row r of the source is src row perm[r] when perm is given (rows gathered on
// the fly, e.g. x by slot), else src row r.
template <typename Tin>
__global__ void __launch_bounds__(1024) quantize_rows_kernel(const Tin* __restrict__ src, const int32_t* __restrict__ perm,
                                                           int64_t n_src, const int32_t* __restrict__ offsets,
                                                           int64_t max_rows, int64_t K, int8_t* __restrict__ hi,
                                                           int8_t* __restrict__ lo, float* __restrict__ scale, int* err) {
  __shared__ float s_max[32];
  int64_t n = offsets[8];
  if (n < 0 || n > max_rows) n = 0;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int64_t r = blockIdx.x; r < n; r += gridDim.x) {
    int64_t sr = r;
    if (perm) {
      sr = perm[r];
      if (sr < 0 || sr >= n_src) {
        if (threadIdx.x == 0) flag_error(err, MOE_DEVERR_SLOT_INDEX);
        continue;  // uniform over the block: every thread skips this row
      }
    }
    const Tin* row = src + sr * K;
    float m = 0.f;
    for (int64_t k = 4 * (int64_t)threadIdx.x; k < K; k += 4 * (int64_t)blockDim.x) {
      float v[4];
      load4(row + k, v);
      m = fmaxf(m, fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3]))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) s_max[warp] = m;
    __syncthreads();
    float amax = 0.f;
    const int nw = blockDim.x >> 5;
    for (int w = 0; w < nw; ++w) amax = fmaxf(amax, s_max[w]);
    const float sc = amax / kRowCodeMax;
    if (threadIdx.x == 0) scale[r] = sc;
    for (int64_t k = 4 * (int64_t)threadIdx.x; k < K; k += 4 * (int64_t)blockDim.x) {
      float v[4];
      load4(row + k, v);
      char4 h, l;
      int c[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) c[j] = sc > 0.f ? (int)fminf(fmaxf(rintf(v[j] / sc), -kRowCodeMax), kRowCodeMax) : 0;
      h.x = (signed char)((c[0] + 128) >> 8); l.x = (signed char)(c[0] - 256 * ((c[0] + 128) >> 8));
      h.y = (signed char)((c[1] + 128) >> 8); l.y = (signed char)(c[1] - 256 * ((c[1] + 128) >> 8));
      h.z = (signed char)((c[2] + 128) >> 8); l.z = (signed char)(c[2] - 256 * ((c[2] + 128) >> 8));
      h.w = (signed char)((c[3] + 128) >> 8); l.w = (signed char)(c[3] - 256 * ((c[3] + 128) >> 8));
      *reinterpret_cast<char4*>(hi + r * K + k) = h;
      *reinterpret_cast<char4*>(lo + r * K + k) = l;
    }
    __syncthreads();  // s_max is reused by the next row
  }
}

}  // namespace

cudaError_t launch_quantize_rows(const void* src, bool src_f32, const int32_t* offsets, int64_t max_rows,
                                 int64_t K, int8_t* hi, int8_t* lo, float* scale, int num_sms, cudaStream_t s,
                                 const int32_t* perm, int64_t n_src, int* err) {
  if (max_rows == 0) return cudaSuccess;
  int64_t blocks = max_rows < (int64_t)num_sms * 4 ? max_rows : (int64_t)num_sms * 4;
  const int threads = K >= 16384 ? 1024 : 256;  // long rows (H) get more threads per row
  if (src_f32)
    quantize_rows_kernel<float><<<(unsigned)blocks, threads, 0, s>>>(static_cast<const float*>(src), perm, n_src,
                                                                     offsets, max_rows, K, hi, lo, scale, err);
  else
    quantize_rows_kernel<__nv_bfloat16><<<(unsigned)blocks, threads, 0, s>>>(
        static_cast<const __nv_bfloat16*>(src), perm, n_src, offsets, max_rows, K, hi, lo, scale, err);
  return cudaGetLastError();
}

cudaError_t launch_quantize_int8(int E, const void* w, int64_t K, int64_t N, int8_t* q, float* scale,
                                 cudaStream_t s) {
  if (E == 0 || K == 0 || N == 0) return cudaSuccess;
  dim3 grid((unsigned)(N / 64), (unsigned)E);
  quantize_int8_kernel<<<grid, 32 * kRowGroups, 0, s>>>(static_cast<const __nv_bfloat16*>(w), K, N, q, scale);
  return cudaGetLastError();
}

}  // namespace moe
