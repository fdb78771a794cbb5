// Grouped expert GEMMs for small token counts (decode): weights on the M side.
//
// Same layer as ffn_tc.cu ("How does Grok-1 use a mixture-of-experts design?",
// section "Expert implementation: SwiGLU at scale"), for batches where each
// expert sees only a few rows, so the pass is bound by streaming the expert
// weights from HBM.  The operands are swapped: one tcgen05 MMA computes
//   D[channel, token] (+)= W^T[channel, k] * X^T[k, token]
// with M = 128 weight channels (A, MN-major straight from the [E, K, N] weight
// layout) and N = the expert's tokens rounded up to 16 (B, K-major rows of
// x_perm or H), so no tensor work is spent on padded token rows.
//   gate/up : two accumulators (gate columns at +0, up at +128 in TMEM); the
//             epilogue applies silu(gate) * up and writes H[token, channel].
//   down    : Y[token, channel] = row_scale[token] * acc.
// Weights are bf16 here; the 8-bit weight path (int8 tensor-core MMAs) lives
// in ffn_decode_i8.cu.
//
// Schedule: persistent, one CTA per SM, tile = (expert, block of up to 128
// tokens, block of 128 output channels).  Warp roles: warp 0 issues TMA, warp
// 1 issues MMAs and owns 512 TMEM columns (two double-buffered accumulator
// sets), warps 2-5 run the epilogue.  All waits are bounded.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"
#include "tc_ptx.cuh"

namespace moe {
namespace {

using namespace ptx;

constexpr int kE = 8;
constexpr int CH = 128;                   // weight channels per tile (MMA M)
constexpr int BK = 64;                    // K per stage
constexpr int TOK = 128;                  // tokens per tile at most (MMA N)
constexpr int W_CHUNK = 64 * BK * 2;      // 8 KB: 64 channels x 64 K
constexpr int W_TILE = 2 * W_CHUNK;       // 16 KB: 128 channels
constexpr int X_TILE = TOK * BK * 2;      // 16 KB: up to 128 token rows
constexpr int XBOX = 16;                  // token rows per TMA box
constexpr int kThreads = 192;
constexpr int kTmemCols = 512;
constexpr int kAccStride = 256;           // TMEM columns per accumulator set
constexpr int kUpOffset = 128;            // up accumulator column offset in a set

enum Mode { kGateUp = 0, kDown = 1 };

template <int MODE>
struct DCfg {
  static constexpr int kMats = MODE == kGateUp ? 2 : 1;
  static constexpr int STAGE = kMats * W_TILE + X_TILE;
  static constexpr int kStages = MODE == kGateUp ? 4 : 6;
  static constexpr int SMEM_BYTES = 1024 + kStages * STAGE + 256;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
  // M = 128, A (weights) MN-major, B (tokens) K-major; N is set per tile.
  static constexpr uint32_t IDESC_BASE = idesc_bf16_f32(128, 8, true, false) & ~(0x3Fu << 17);
};

struct DecArgs {
  const int32_t* offsets;  // [E + 1], device
  int64_t rows_alloc;      // rows of the token operand and of the output buffers
  int n_cb;                // output channels / 128
  int num_kb;              // K / 64
  void* out;               // H (bf16) or Y (fp32)
  int64_t ld_out;
  const float* row_scale;  // down only; NULL means 1
  int* err;
};

struct DSched {
  int offs[kE + 1];
  int chunks[kE];
  int prefix[kE + 1];
};

struct DTile {
  int e, m0, rows, n0, ntok;
};

__device__ __forceinline__ DTile decode_dtile(const DSched& s, int L, int n_cb) {
  int e = 0;
#pragma unroll
  for (int k = 1; k < kE; ++k)
    if (L >= s.prefix[k]) e = k;
  const int local = L - s.prefix[e];
  const int ch = local / n_cb;
  DTile t;
  t.e = e;
  t.n0 = (local - ch * n_cb) * CH;
  t.m0 = s.offs[e] + ch * TOK;
  const int left = s.offs[e + 1] - t.m0;
  t.rows = left < TOK ? left : TOK;
  t.ntok = (t.rows + 15) & ~15;
  return t;
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    decode_gemm_kernel(const __grid_constant__ CUtensorMap tmW0, const __grid_constant__ CUtensorMap tmW1,
                       const __grid_constant__ CUtensorMap tmX, const DecArgs args) {
  using C = DCfg<MODE>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* stages = smem;  // S x [kMats weight tiles | token rows]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * C::STAGE);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  __shared__ DSched sched;

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
    prefetch_tmap(&tmX);
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
      acc += sched.chunks[k] * args.n_cb;
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
        const DTile t = decode_dtile(sched, L, args.n_cb);
        for (int kb = 0; kb < args.num_kb; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* st = stages + s * C::STAGE;
          mbar_arrive_expect_tx(&full[s], C::kMats * W_TILE + t.ntok * 128);
#pragma unroll
          for (int m = 0; m < C::kMats; ++m) {
            const CUtensorMap* tw = m == 0 ? &tmW0 : &tmW1;
            tma_load_3d(st + m * W_TILE, tw, &full[s], t.n0, kb * BK, t.e);
            tma_load_3d(st + m * W_TILE + W_CHUNK, tw, &full[s], t.n0 + 64, kb * BK, t.e);
          }
          uint8_t* xs = st + C::kMats * W_TILE;
          for (int b = 0; b < t.ntok / XBOX; ++b)
            tma_load_2d_hint(xs + b * XBOX * 128, &tmX, &full[s], kb * BK, t.m0 + b * XBOX, keep);
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
        const DTile t = decode_dtile(sched, L, args.n_cb);
        const uint32_t idesc = C::IDESC_BASE | ((uint32_t)(t.ntok >> 3) << 17);
        const uint32_t buf = tc & 1u;
        const uint32_t tph = (tc >> 1) & 1u;
        if (!mbar_wait(&tempty[buf], tph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d0 = tmem_base + buf * kAccStride;
        for (int kb = 0; kb < args.num_kb; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1u;
          if (!mbar_wait(&full[s], ph, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = smem_u32(stages + s * C::STAGE);
          const uint32_t xs = st + C::kMats * W_TILE;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t bd = sw128_desc(xs + kk * 32, 16, 1024);
#pragma unroll
            for (int m = 0; m < C::kMats; ++m) {
              const uint64_t ad = sw128_desc(st + m * W_TILE + kk * 2048, W_CHUNK, 1024);
              umma_bf16(d0 + m * kUpOffset, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
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
      const DTile t = decode_dtile(sched, L, args.n_cb);
      const uint32_t buf = tc & 1u;
      const uint32_t tph = (tc >> 1) & 1u;
      if (!mbar_wait(&tfull[buf], tph, abort_flag)) {
        if (lane == 0) flag_error(args.err, MOE_DEVERR_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const int n = t.n0 + c_local;
      const uint32_t tacc = tmem_base + buf * kAccStride + ((uint32_t)(q * 32) << 16);
      if (MODE == kGateUp) {
        __nv_bfloat16* H = static_cast<__nv_bfloat16*>(args.out);
        for (int j0 = 0; j0 < t.ntok; j0 += 16) {
          uint32_t g[16], u[16];
          tmem_ld16(tacc + j0, g);
          tmem_ld16(tacc + kUpOffset + j0, u);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (j0 + j < t.rows)
              H[(int64_t)(t.m0 + j0 + j) * args.ld_out + n] =
                  __float2bfloat16_rn(silu_mul_fast(__uint_as_float(g[j]), __uint_as_float(u[j])));
        }
      } else {
        float* Y = static_cast<float*>(args.out);
        for (int j0 = 0; j0 < t.ntok; j0 += 16) {
          uint32_t v[16];
          tmem_ld16(tacc + j0, v);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            if (j0 + j < t.rows) {
              const int64_t row = t.m0 + j0 + j;
              const float rs = args.row_scale ? __ldg(args.row_scale + row) : 1.0f;
              Y[row * args.ld_out + n] = rs * __uint_as_float(v[j]);
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
cudaError_t launch_decode(const CUtensorMap& w0, const CUtensorMap& w1, const CUtensorMap& x, const DecArgs& a,
                          cudaStream_t s, const Ctx& ctx) {
  using C = DCfg<MODE>;
  auto kern = decode_gemm_kernel<MODE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  kern<<<ctx.num_sms, kThreads, C::SMEM_BYTES, s>>>(w0, w1, x, a);
  return cudaGetLastError();
}

bool weight_map(CUtensorMap* m, const void* w, int64_t K, int64_t N, int E) {
  const uint64_t dims[3] = {(uint64_t)N, (uint64_t)K, (uint64_t)E};
  const uint64_t str[2] = {(uint64_t)N * 2, (uint64_t)K * N * 2};
  const uint32_t box[3] = {64, 64, 1};
  return encode_tmap(m, w, 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

bool token_map(CUtensorMap* m, const void* x, int64_t rows, int64_t K) {
  const uint64_t dims[2] = {(uint64_t)K, (uint64_t)rows};
  const uint64_t str[1] = {(uint64_t)K * 2};
  const uint32_t box[2] = {64, XBOX};
  return encode_tmap(m, x, 2, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

cudaError_t launch_decode_gate_up(const moe_config_t& c, const void* x_perm, const int32_t* offsets, const void* wg,
                                  const void* wu, void* h, cudaStream_t s, const Ctx& ctx) {
  const int64_t rows = slot_rows(c);
  if (rows == 0) return cudaSuccess;
  CUtensorMap tg, tu, tx;
  if (!weight_map(&tg, wg, c.d, c.f, c.E) || !weight_map(&tu, wu, c.d, c.f, c.E) || !token_map(&tx, x_perm, rows, c.d))
    return cudaErrorInvalidValue;
  DecArgs a;
  a.offsets = offsets;
  a.rows_alloc = rows;
  a.n_cb = (int)(c.f / CH);
  a.num_kb = (int)(c.d / BK);
  a.out = h;
  a.ld_out = c.f;
  a.row_scale = nullptr;
  a.err = ctx.err;
  return launch_decode<kGateUp>(tg, tu, tx, a, s, ctx);
}

cudaError_t launch_decode_down(const moe_config_t& c, const void* h, const int32_t* offsets, const void* wd,
                               const float* row_scale, float* y, cudaStream_t s, const Ctx& ctx) {
  const int64_t rows = slot_rows(c);
  if (rows == 0) return cudaSuccess;
  CUtensorMap tw, tx;
  if (!weight_map(&tw, wd, c.f, c.d, c.E) || !token_map(&tx, h, rows, c.f)) return cudaErrorInvalidValue;
  DecArgs a;
  a.offsets = offsets;
  a.rows_alloc = rows;
  a.n_cb = (int)(c.d / CH);
  a.num_kb = (int)(c.f / BK);
  a.out = y;
  a.ld_out = c.d;
  a.row_scale = row_scale;
  a.err = ctx.err;
  return launch_decode<kDown>(tw, tw, tx, a, s, ctx);
}

}  // namespace moe
