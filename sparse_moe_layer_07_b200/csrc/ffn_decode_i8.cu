// Expert GEMMs with 8-bit expert weights on the int8 tensor cores.
//
// The layer of "How does Grok-1 use a mixture-of-experts design?" (section
// "Expert implementation: SwiGLU at scale") with the expert weights stored as
// int8 codes and per-output-channel scales (quantize.cu), for the
// weight-streaming regime (few tokens per expert).  Every activation row r
// enters as a 15-bit code c = 256 * hi + lo with a per-row scale s_r (hi and
// lo are two int8 planes, quantize_rows in quantize.cu), so each MMA is an
// exact int8 x int8 -> int32 product:
//   acc_hi[n, t] = sum_k q[k, n] * hi[t, k],  acc_lo[n, t] = sum_k q[k, n] * lo[t, k]
//   value[n, t]  = s_w[n] * s_r[t] * (256 * acc_hi + acc_lo)
// No weight is converted on the SM: the int8 tiles go from HBM to shared
// memory by TMA and straight into tcgen05.mma kind::i8, so each stage holds
// only int8 weights and the ring keeps ~160 KB of weights in flight per SM.
// Like ffn_decode.cu the weights are the M = 128 operand (MN-major) and the
// tokens the N operand (up to 32 per tile, K-major planes).
//   gate/up : accumulators [gate_hi | gate_lo | up_hi | up_lo]; the epilogue
//             writes H = silu(g) * u in fp32 (re-coded by quantize_rows for down)
//   down    : Y = row_scale * value.
// Warp roles as in ffn_decode.cu (warp 0 TMA, warp 1 MMA + TMEM, warps 2-5
// epilogue); all waits bounded.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"
#include "tc_ptx.cuh"

namespace moe {
namespace {

using namespace ptx;

constexpr int kE = 8;
constexpr int CH = 128;              // weight channels per tile (MMA M)
constexpr int BK = 128;              // K per stage (128 int8 = one 128-byte swizzle row)
constexpr int TOK = 32;              // tokens per tile at most (MMA N)
constexpr int W_TILE = CH * BK;      // 16 KB: int8 [128 K][128 channels]
constexpr int PLANE = TOK * BK;      // 4 KB: int8 [32 tokens][128 K]
constexpr int XBOX = 16;             // token rows per TMA box
constexpr int kThreads = 192;
constexpr int kTmemCols = 256;

enum Mode { kGateUp = 0, kDown = 1 };

}  // namespace

// K splits of the int8 down pass.  With decode-sized batches (one token block
// per expert) the down pass has only E * d / 256 tiles, too few to fill the
// GPU evenly, so K is split into s ranges (each writing its own fp32 partial,
// summed later in split order); s is the count in 1..kMaxDownSplits whose tile
// count E * (d / 256) * s fills the last wave best.  Larger batches have enough
// tiles and use one split.
int down_splits(const moe_config_t& c, int num_sms) {
  const int64_t kb = c.f / 128;
  if (slot_rows(c) > 64 * (int64_t)c.E) return 1;
  const int64_t base = (int64_t)c.E * (c.d / 256);
  int best = 1;
  double best_eff = 0.0;
  for (int sp = 1; sp <= kMaxDownSplits && sp <= kb; ++sp) {
    const int64_t tiles = base * sp;
    const int64_t waves = (tiles + num_sms - 1) / num_sms;
    const double eff = (double)tiles / (double)(waves * num_sms);
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best = sp;
    }
  }
  return best;
}

namespace {

// Both passes stream two 16 KB weight tiles per stage: gate/up the gate and up
// tiles of one 128-channel block; down two adjacent 128-channel blocks of W_down
// (256 output channels per tile), so each stage moves 32 KB of weights and the
// 5-stage ring keeps 160 KB in flight per SM.
template <int MODE>
struct I8Cfg {
  static constexpr int kMats = 2;
  static constexpr int kChW = MODE == kGateUp ? CH : 2 * CH;   // output channels per tile
  static constexpr int STAGE = kMats * W_TILE + 2 * PLANE;     // 40 KB
  static constexpr int kStages = 5;
  static constexpr int kAccs = 2 * kMats;                       // hi and lo per matrix
  static constexpr int kAccStride = kAccs * TOK;                 // 128 / 64 columns
  static constexpr int SMEM_BYTES = 1024 + kStages * STAGE + 256;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
  static_assert(2 * kAccStride <= kTmemCols, "TMEM budget");
  static constexpr uint32_t IDESC_BASE = idesc_s8_s32(128, 8, true, false) & ~(0x3Fu << 17);
};

struct I8Args {
  const int32_t* offsets;
  int64_t rows_alloc;
  int n_cb;                 // output channels / channels per tile
  int n_out;                // output channels
  int num_kb;               // K / 128 (all splits together)
  int ksplit;               // K splits (down: each split's range writes its own partial output)
  int64_t split_stride;     // elements between the partial outputs
  void* out;                // H fp32 [rows, f] or Y fp32 [rows, d]
  int64_t ld_out;
  const float* wscale0;     // [E, n_out]: gate (or down)
  const float* wscale1;     // [E, n_out]: up
  const float* row_code_scale;  // [rows]: scale of each input row's code
  const float* row_scale;   // down: routing weight per row (NULL: 1)
  int* err;
};

struct Sched8 {
  int offs[kE + 1];
  int chunks[kE];
  int prefix[kE + 1];
};

struct Tile8 {
  int e, m0, rows, n0, ntok, ks;
};

// Tile order: expert, token block, K split, channel block.
__device__ __forceinline__ Tile8 tile8(const Sched8& s, int L, int n_cb, int ksplit, int chw) {
  int e = 0;
#pragma unroll
  for (int k = 1; k < kE; ++k)
    if (L >= s.prefix[k]) e = k;
  const int local = L - s.prefix[e];
  const int per_chunk = n_cb * ksplit;
  const int ch = local / per_chunk;
  const int r = local - ch * per_chunk;
  Tile8 t;
  t.e = e;
  t.ks = r / n_cb;
  t.n0 = (r - t.ks * n_cb) * chw;
  t.m0 = s.offs[e] + ch * TOK;
  const int left = s.offs[e + 1] - t.m0;
  t.rows = left < TOK ? left : TOK;
  t.ntok = (t.rows + 15) & ~15;
  return t;
}

__device__ __forceinline__ float code_value(uint32_t hi, uint32_t lo) {
  return fmaf(256.0f, (float)(int)hi, (float)(int)lo);
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    decode_i8_kernel(const __grid_constant__ CUtensorMap tmW0, const __grid_constant__ CUtensorMap tmW1,
                     const __grid_constant__ CUtensorMap tmHi, const __grid_constant__ CUtensorMap tmLo,
                     const I8Args args) {
  using C = I8Cfg<MODE>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* stages = smem;  // S x [kMats weight tiles | hi plane | lo plane]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * C::STAGE);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  __shared__ Sched8 sched;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 1) {
    prefetch_tmap(&tmW0);
    prefetch_tmap(&tmW1);
    prefetch_tmap(&tmHi);
    prefetch_tmap(&tmLo);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  if (warp == 2 && lane == 0) {
    bool ok = true;
    int prev = 0;
    for (int k = 0; k <= kE; ++k) {
      const int v = args.offsets[k];
      sched.offs[k] = v;
      if (v < prev || (int64_t)v > args.rows_alloc) ok = false;
      prev = v;
    }
    if (sched.offs[0] < 0) ok = false;
    int acc = 0;
    for (int k = 0; k < kE; ++k) {
      const int n = ok ? sched.offs[k + 1] - sched.offs[k] : 0;
      sched.chunks[k] = (n + TOK - 1) / TOK;
      sched.prefix[k] = acc;
      acc += sched.chunks[k] * args.n_cb * args.ksplit;
    }
    sched.prefix[kE] = acc;
    if (!ok) flag_error(args.err, MOE_DEVERR_OFFSETS);
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = sched.prefix[kE];

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ producer
      const uint64_t keep = policy_evict_last();
      uint32_t it = 0;
      bool ok = true;
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
        const Tile8 t = tile8(sched, L, args.n_cb, args.ksplit, C::kChW);
        const int kb_lo = t.ks * args.num_kb / args.ksplit, kb_hi = (t.ks + 1) * args.num_kb / args.ksplit;
        for (int kb = kb_lo; kb < kb_hi; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* st = stages + s * C::STAGE;
          mbar_arrive_expect_tx(&full[s], C::kMats * W_TILE + 2 * t.ntok * BK);
          const int k0 = kb * BK;
          tma_load_3d(st, &tmW0, &full[s], t.n0, k0, t.e);
          if (MODE == kGateUp)
            tma_load_3d(st + W_TILE, &tmW1, &full[s], t.n0, k0, t.e);
          else
            tma_load_3d(st + W_TILE, &tmW0, &full[s], t.n0 + CH, k0, t.e);
          uint8_t* ph_hi = st + C::kMats * W_TILE;
          uint8_t* ph_lo = ph_hi + PLANE;
          for (int b = 0; b < t.ntok / XBOX; ++b) {
            tma_load_2d_hint(ph_hi + b * XBOX * BK, &tmHi, &full[s], k0, t.m0 + b * XBOX, keep);
            tma_load_2d_hint(ph_lo + b * XBOX * BK, &tmLo, &full[s], k0, t.m0 + b * XBOX, keep);
          }
        }
      }
      if (!ok) {
        flag_error(args.err, MOE_DEVERR_TIMEOUT);
        *abort_flag = 1;
      }
      const uint32_t first = it > (uint32_t)S ? it - S : 0u;
      for (uint32_t j = first; j < it; ++j) mbar_wait(&full[j % S], (j / S) & 1u, nullptr, 100000000ull);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      uint32_t it = 0, tc = 0;
      bool ok = true, issued = false;
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x, ++tc) {
        const Tile8 t = tile8(sched, L, args.n_cb, args.ksplit, C::kChW);
        const uint32_t idesc = C::IDESC_BASE | ((uint32_t)(t.ntok >> 3) << 17);
        const uint32_t buf = tc & 1u;
        const uint32_t tph = (tc >> 1) & 1u;
        if (!mbar_wait(&tempty[buf], tph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d0 = tmem_base + buf * C::kAccStride;
        const int kb_lo = t.ks * args.num_kb / args.ksplit, kb_hi = (t.ks + 1) * args.num_kb / args.ksplit;
        for (int kb = kb_lo; kb < kb_hi; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1u;
          if (!mbar_wait(&full[s], ph, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = smem_u32(stages + s * C::STAGE);
          const uint32_t p_hi = st + C::kMats * W_TILE;
          const uint32_t p_lo = p_hi + PLANE;
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk) {
            const uint64_t b_hi = sw128_desc(p_hi + kk * 32, 16, 1024);
            const uint64_t b_lo = sw128_desc(p_lo + kk * 32, 16, 1024);
            const uint32_t acc = (kb != kb_lo || kk != 0) ? 1u : 0u;
#pragma unroll
            for (int m = 0; m < C::kMats; ++m) {
              const uint64_t ad = sw128_desc(st + m * W_TILE + kk * 4096, 8192, 1024);
              umma_s8(d0 + (2 * m) * TOK, ad, b_hi, idesc, acc);
              umma_s8(d0 + (2 * m + 1) * TOK, ad, b_lo, idesc, acc);
            }
          }
          issued = true;
          umma_commit(&empty[s]);
        }
        if (!ok) break;
        umma_commit(&tfull[buf]);
      }
      if (!ok) {
        flag_error(args.err, MOE_DEVERR_TIMEOUT);
        *abort_flag = 1;
      }
      if (issued) {
        umma_commit(drain);
        mbar_wait(drain, 0, nullptr, 100000000ull);
      }
    }
  } else {
    // -------------------------------------------------- epilogue
    const int q = warp & 3;
    const int c_local = q * 32 + lane;
    uint32_t tc = 0;
    for (int L = blockIdx.x; L < total; L += gridDim.x, ++tc) {
      const Tile8 t = tile8(sched, L, args.n_cb, args.ksplit, C::kChW);
      const uint32_t buf = tc & 1u;
      const uint32_t tph = (tc >> 1) & 1u;
      if (!mbar_wait(&tfull[buf], tph, abort_flag)) {
        if (lane == 0) flag_error(args.err, MOE_DEVERR_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const int n = t.n0 + c_local;
      const uint32_t tacc = tmem_base + buf * C::kAccStride + ((uint32_t)(q * 32) << 16);
      float* out = static_cast<float*>(args.out) + (int64_t)t.ks * args.split_stride;
      if (MODE == kGateUp) {
        const float sg = __ldg(args.wscale0 + (int64_t)t.e * args.n_out + n);
        const float su = __ldg(args.wscale1 + (int64_t)t.e * args.n_out + n);
        for (int j0 = 0; j0 < t.ntok; j0 += 16) {
          uint32_t gh[16], gl[16], uh[16], ul[16];
          tmem_ld16(tacc + 0 * TOK + j0, gh);
          tmem_ld16(tacc + 1 * TOK + j0, gl);
          tmem_ld16(tacc + 2 * TOK + j0, uh);
          tmem_ld16(tacc + 3 * TOK + j0, ul);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            if (j0 + j < t.rows) {
              const int64_t row = t.m0 + j0 + j;
              const float sr = __ldg(args.row_code_scale + row);
              const float g = sg * sr * code_value(gh[j], gl[j]);
              const float u = su * sr * code_value(uh[j], ul[j]);
              out[row * args.ld_out + n] = silu_mul_fast(g, u);
            }
          }
        }
      } else {
#pragma unroll 1
        for (int m = 0; m < 2; ++m) {
          const int nm = n + m * CH;
          const float sd = __ldg(args.wscale0 + (int64_t)t.e * args.n_out + nm);
          for (int j0 = 0; j0 < t.ntok; j0 += 16) {
            uint32_t vh[16], vl[16];
            tmem_ld16(tacc + (2 * m) * TOK + j0, vh);
            tmem_ld16(tacc + (2 * m + 1) * TOK + j0, vl);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              if (j0 + j < t.rows) {
                const int64_t row = t.m0 + j0 + j;
                const float rs = args.row_scale ? __ldg(args.row_scale + row) : 1.0f;
                out[row * args.ld_out + nm] = rs * (sd * __ldg(args.row_code_scale + row) * code_value(vh[j], vl[j]));
              }
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[buf]);
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

template <int MODE>
cudaError_t launch_i8(const CUtensorMap& w0, const CUtensorMap& w1, const CUtensorMap& hi, const CUtensorMap& lo,
                      const I8Args& a, cudaStream_t s, const Ctx& ctx) {
  using C = I8Cfg<MODE>;
  auto kern = decode_i8_kernel<MODE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  kern<<<ctx.num_sms, kThreads, C::SMEM_BYTES, s>>>(w0, w1, hi, lo, a);
  return cudaGetLastError();
}

bool code_weight_map(CUtensorMap* m, const void* q, int64_t K, int64_t N, int E) {
  const uint64_t dims[3] = {(uint64_t)N, (uint64_t)K, (uint64_t)E};
  const uint64_t str[2] = {(uint64_t)N, (uint64_t)K * N};
  const uint32_t box[3] = {128, BK, 1};
  return encode_tmap_dtype(m, q, 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_DATA_TYPE_UINT8);
}

bool plane_map(CUtensorMap* m, const void* p, int64_t rows, int64_t K) {
  const uint64_t dims[2] = {(uint64_t)K, (uint64_t)rows};
  const uint64_t str[1] = {(uint64_t)K};
  const uint32_t box[2] = {BK, XBOX};
  return encode_tmap_dtype(m, p, 2, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_DATA_TYPE_UINT8);
}

// y[r, :] = ((parts[0] + parts[1]) + parts[2]) + ... for the first offsets[E] rows.
__global__ void __launch_bounds__(256) sum_partials_kernel(const float4* __restrict__ parts, const int32_t* offsets,
                                                          int64_t max_rows, int64_t row_vec, int64_t split_vec,
                                                          int nsplit, float4* __restrict__ y) {
  int64_t n = offsets[kE];
  if (n < 0 || n > max_rows) n = 0;
  const int64_t total = n * row_vec;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    float4 a = parts[i];
    for (int p = 1; p < nsplit; ++p) {
      const float4 b = parts[p * split_vec + i];
      a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
    }
    y[i] = a;
  }
}

}  // namespace

cudaError_t launch_sum_partials(const moe_config_t& c, const float* y_parts, const int32_t* offsets, float* y,
                                cudaStream_t s, const Ctx& ctx) {
  const int64_t rows = slot_rows(c);
  if (rows == 0) return cudaSuccess;
  const int nsplit = down_splits(c, ctx.num_sms);
  sum_partials_kernel<<<ctx.num_sms * 4, 256, 0, s>>>(reinterpret_cast<const float4*>(y_parts), offsets, rows,
                                                      c.d / 4, rows * c.d / 4, nsplit, reinterpret_cast<float4*>(y));
  return cudaGetLastError();
}

cudaError_t launch_i8_gate_up(const moe_config_t& c, const int8_t* x_hi, const int8_t* x_lo, const float* x_scale,
                              const int32_t* offsets, const int8_t* qg, const float* sg, const int8_t* qu,
                              const float* su, float* h, cudaStream_t s, const Ctx& ctx) {
  const int64_t rows = slot_rows(c);
  if (rows == 0) return cudaSuccess;
  CUtensorMap tg, tu, th, tl;
  if (!code_weight_map(&tg, qg, c.d, c.f, c.E) || !code_weight_map(&tu, qu, c.d, c.f, c.E) ||
      !plane_map(&th, x_hi, rows, c.d) || !plane_map(&tl, x_lo, rows, c.d))
    return cudaErrorInvalidValue;
  I8Args a;
  a.offsets = offsets;
  a.rows_alloc = rows;
  a.n_cb = (int)(c.f / CH);
  a.n_out = (int)c.f;
  a.num_kb = (int)(c.d / BK);
  a.ksplit = 1;
  a.split_stride = 0;
  a.out = h;
  a.ld_out = c.f;
  a.wscale0 = sg;
  a.wscale1 = su;
  a.row_code_scale = x_scale;
  a.row_scale = nullptr;
  a.err = ctx.err;
  return launch_i8<kGateUp>(tg, tu, th, tl, a, s, ctx);
}

// The down pass has only d / 256 channel blocks per token block (24 at d = 6144),
// so its K range is split (four ways when f / 128 allows): each part writes
// its own fp32 partial [rows, d] and a fixed-order sum (sum_partials) forms
// y = ((p0 + p1) + p2) + p3.
cudaError_t launch_i8_down(const moe_config_t& c, const int8_t* h_hi, const int8_t* h_lo, const float* h_scale,
                           const int32_t* offsets, const int8_t* qd, const float* sd, const float* row_scale,
                           float* y_parts, cudaStream_t s, const Ctx& ctx) {
  const int64_t rows = slot_rows(c);
  if (rows == 0) return cudaSuccess;
  CUtensorMap tw, th, tl;
  if (!code_weight_map(&tw, qd, c.f, c.d, c.E) || !plane_map(&th, h_hi, rows, c.f) || !plane_map(&tl, h_lo, rows, c.f))
    return cudaErrorInvalidValue;
  I8Args a;
  a.offsets = offsets;
  a.rows_alloc = rows;
  a.n_cb = (int)(c.d / (2 * CH));
  a.n_out = (int)c.d;
  a.ksplit = down_splits(c, ctx.num_sms);
  a.num_kb = (int)(c.f / BK);
  a.split_stride = rows * c.d;
  a.out = y_parts;
  a.ld_out = c.d;
  a.wscale0 = sd;
  a.wscale1 = nullptr;
  a.row_code_scale = h_scale;
  a.row_scale = row_scale;
  a.err = ctx.err;
  return launch_i8<kDown>(tw, tw, th, tl, a, s, ctx);
}

}  // namespace moe
