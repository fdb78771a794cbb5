// Device helpers shared by the kernels: bf16 packing, error reporting.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

template <typename T>
struct Elem;
template <>
struct Elem<float> {
  static __device__ __forceinline__ float to_f32(float v) { return v; }
};
template <>
struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
};

// Eight consecutive elements loaded as fp32 (16-byte bf16 or 32-byte fp32 load).
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&v)[8]) {
  uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
  float4 a = __ldg(reinterpret_cast<const float4*>(p));
  float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// Round two fp32 to bf16 (nearest even) and pack them, low half first.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&p);
}

// SiLU(g) * u of the bf16 tensor-core forward epilogues.  __expf and the
// approximate divide keep it at two special-function operations and a few
// FMAs, where the IEEE quotient g / (1 + e^-g) costs a call per element that
// serialised the gate/up epilogue (10 us per 128 x 128 tile against 3 us this
// way).  It stays within a few fp32 ulp of the IEEE form, far inside the bf16
// rounding of H; for g -> -inf the denominator passes 2^126, where __fdividef
// returns 0, the limit of the function.  (The backward's dH epilogue keeps the
// IEEE sigmoid: there the fast form made the kernel 7% slower at Grok size.)
__device__ __forceinline__ float silu_mul_fast(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }

// Programmatic dependent launch (kernels started with launch_pdl): the kernel
// is launched while the previous kernel of its stream finishes, and
// pdl_wait() blocks until that kernel has completed with its writes visible,
// so every kernel of the forward path calls it before its first access to
// global memory.  No kernel triggers its dependents early
// (griddepcontrol.launch_dependents): with the trigger at the start of each
// kernel, the next kernel's CTAs waited on the SMs through the whole GEMM and
// the Grok-size step took 12% longer; without it the launch overlaps only the
// previous kernel's exit, 3% off the mid-size step and neutral at Grok size.
// A no-op for a kernel launched without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void flag_error(int* err, int bits) {
  if (err) atomicOr(err, bits);
}

}  // namespace moe
