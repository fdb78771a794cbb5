// Backward of the expert FFNs on the tcgen05 tensor cores (training).
//
// The pages give the forward pass only ("How does Grok-1 use a
// mixture-of-experts design?", sections "Expert implementation: SwiGLU at
// scale" and "Expert parallelism vs. tensor parallelism"); training
// differentiates that forward with the routing decisions held fixed.  For
// the kept rows r of expert e (token t = perm[r], weight w = row_scale[r]),
// with G = X W_gate, U = X W_up, H = silu(G) * U saved by the forward:
//   kDH : dHu[r, :] = dout[t, :] W_down[e]^T        (A = dout rows, B = W_down K-major)
//         epilogue: dH = w * dHu,  dG = dH * U * silu'(G),  dU = dH * silu(G),
//         and per-tile partials of <dHu, H> (= the routing weight's gradient
//         <dout, y>), summed later in a fixed order
//   kDX : dx[t, :] += dG[r, :] W_gate[e]^T + dU[r, :] W_up[e]^T
//         (K runs over both halves; B = W_gate / W_up read K-major straight from
//         their [E, d, f] layout; the epilogue adds into an fp32 sum by token:
//         two terms per token, so the order of the adds does not matter)
//   kWG : dW[e] = A_e^T B_e over the rows of expert e  (A, B MN-major:
//         dW_down = H^T (w * dout),  dW_gate = X^T dG,  dW_up = X^T dU); K is
//         the ragged row count: the expert's last K block issues only the
//         16-row MMA steps that hold its rows, and the rows of the last step
//         past the expert's end are zeroed in shared memory before the MMA
//         (by warp 6, which only kWG has).
// Pipeline as in ffn_tc.cu: persistent CTAs, warp 0 TMA, warp 1 MMA (lane 0
// alone) + TMEM (two 128 x 256 fp32 accumulators), warps 2-5 epilogue; every
// wait bounded.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"
#include "tc_ptx.cuh"

namespace moe {
namespace {

using namespace ptx;

constexpr int kE = 8;
constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;
// Epilogue warps: 4, one per TMEM lane quarter.  (The layout also allows 8, two
// per quarter each taking half of the tile's columns; for kDH that measured 14%
// slower than 4 relative to the forward GEMMs in the same capture.)
template <int MODE>
struct Warps {
  static constexpr int kEpi = 4;
  // weight gradients: one more warp zeroes the rows past an expert's end in its
  // last K block, so the MMA warp does not stall on it
  static constexpr int kZeroWarp = MODE == 2 ? 2 + kEpi : -1;
  static constexpr int kThreads = 64 + 32 * kEpi + (MODE == 2 ? 32 : 0);
};
constexpr int kTmemCols = 512;
constexpr int kAccStride = 256;
constexpr int CHUNK = 64 * BK * 2;      // 8 KB: 64 x 64 bf16
constexpr int A_BYTES = 2 * CHUNK;      // 16 KB: 128 x 64
constexpr int B_BYTES = 4 * CHUNK;      // 32 KB: 256 x 64
constexpr int STAGE = A_BYTES + B_BYTES;
constexpr int kStages = 4;
// weight gradients: each epilogue warp stages 32 rows x 32 fp32 (4 KB, 128-byte
// swizzled) for a TMA tile store, double buffered
constexpr int OUT_STAGE = 32 * 32 * 4;
constexpr int OUT_BYTES = 4 * 2 * OUT_STAGE;
constexpr int SMEM_BYTES = 1024 + kStages * STAGE + OUT_BYTES + 256;
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
// full, empty, zeroed (kStages each), tfull, tempty (2 each), drain, then the
// TMEM slot, the abort flag and the producer's stage count
static_assert((3 * kStages + 5) * 8 + 12 <= 256, "barrier area");

enum Mode { kDH = 0, kDX = 1, kWG = 2 };

struct BwdArgs {
  const int32_t* offsets;  // [E + 1]
  int64_t rows_alloc;      // rows of the grouped buffers
  int n_tiles;             // N / BN
  int m_tiles;             // kWG: M / BM
  int num_kb;              // kDH: d / BK;  kDX: 2 f / BK
  int half_kb;             // kDX: f / BK (first half dG x W_gate, second dU x W_up)
  int m_outer;             // kWG: tiles of one expert ordered M-block major
  const int32_t* perm;     // kDX: token of each row
  int64_t n_tok;
  const float* row_scale;  // kDH
  const __nv_bfloat16* G;  // kDH inputs [rows, f]
  const __nv_bfloat16* U;
  const __nv_bfloat16* H;
  __nv_bfloat16* dG;       // kDH outputs [rows, f]
  __nv_bfloat16* dU;
  float* dw_part;          // kDH: [rows, n_tiles * parts per tile]
  float* out;              // kDX: dx32 [T, d];  kWG: dW [E, M, N]
  int64_t ld;              // kDH: f;  kDX: d;  kWG: N
  int64_t M;               // kWG
  int* err;
};

struct Sched {
  int offs[kE + 1];
  int mt[kE];              // row blocks (kDH, kDX) of each expert
  int prefix[kE + 1];
};

struct Tile {
  int e, m0, rows, n0, nb;
  int row0, nrows, nkb;    // kWG: the expert's grouped rows and K blocks
};

template <int MODE>
__device__ __forceinline__ Tile decode_tile(const Sched& s, const BwdArgs& a, int L) {
  Tile t;
  int e = 0;
#pragma unroll
  for (int k = 1; k < kE; ++k)
    if (L >= s.prefix[k]) e = k;
  const int local = L - s.prefix[e];
  t.e = e;
  t.row0 = s.offs[e];
  t.nrows = s.offs[e + 1] - s.offs[e];
  if (MODE == kWG) {
    int mb, nb;
    if (a.m_outer) {
      mb = local / a.n_tiles;
      nb = local - mb * a.n_tiles;
    } else {
      nb = local / a.m_tiles;
      mb = local - nb * a.m_tiles;
    }
    t.m0 = mb * BM;
    t.rows = BM;
    t.n0 = nb * BN;
    t.nb = nb;
    t.nkb = (t.nrows + BK - 1) / BK;
  } else {
    const int nb = local / s.mt[e];
    const int mi = local - nb * s.mt[e];
    t.m0 = s.offs[e] + mi * BM;
    const int left = s.offs[e + 1] - t.m0;
    t.rows = left < BM ? left : BM;
    t.n0 = nb * BN;
    t.nb = nb;
    t.nkb = MODE == kDH ? a.num_kb : 2 * a.half_kb;
  }
  return t;
}

template <int MODE>
__device__ __forceinline__ void build_schedule(Sched& sched, const BwdArgs& args) {
  bool ok = true;
  int prev = 0;
  for (int k = 0; k <= kE; ++k) {
    const int v = args.offsets[k];
    sched.offs[k] = v;
    if (v < prev || (int64_t)v > args.rows_alloc) ok = false;
    prev = v;
  }
  if (sched.offs[0] < 0) ok = false;
  if (!ok)
    for (int k = 0; k <= kE; ++k) sched.offs[k] = 0;
  int acc = 0;
  for (int k = 0; k < kE; ++k) {
    const int n = sched.offs[k + 1] - sched.offs[k];
    sched.mt[k] = (n + BM - 1) / BM;
    sched.prefix[k] = acc;
    // weight gradients: every expert owns its M x N tiles (zero when it has no rows)
    acc += MODE == kWG ? (ok ? args.m_tiles * args.n_tiles : 0) : sched.mt[k] * args.n_tiles;
  }
  sched.prefix[kE] = acc;
  if (!ok) flag_error(args.err, MOE_DEVERR_OFFSETS);
}

__device__ __forceinline__ void unpack8_bf16(const uint4 q, float (&v)[8]) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}

template <int MODE>
__global__ void __launch_bounds__(Warps<MODE>::kThreads, 1)
    bwd_gemm_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                    const __grid_constant__ CUtensorMap tmB0, const __grid_constant__ CUtensorMap tmB1,
                    const __grid_constant__ CUtensorMap tmOut, const BwdArgs args) {
  constexpr int S = kStages;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* sA = smem;
  uint8_t* sB = smem + S * A_BYTES;
  uint8_t* sOut = smem + S * STAGE;  // 1024-byte aligned: S * STAGE is a multiple of 1024
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * STAGE + OUT_BYTES);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* zeroed = drain + 1;  // kWG: stage s of a ragged last K block is zeroed and ready
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(zeroed + S);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // kWG: K blocks whose loads the producer has issued (the zeroing warp waits on
  // a stage's full barrier only once its loads are issued, so the barrier is at
  // that K block's phase and not at an earlier phase of the same parity)
  volatile uint32_t* issued_kb = reinterpret_cast<volatile uint32_t*>(tmem_slot + 2);
  __shared__ Sched sched;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    *issued_kb = 0;
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&zeroed[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 32 * Warps<MODE>::kEpi);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 1) {
    prefetch_tmap(&tmA0);
    prefetch_tmap(&tmB0);
    if (MODE == kDX) {
      prefetch_tmap(&tmA1);
      prefetch_tmap(&tmB1);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  if (warp == 2 && lane == 0) build_schedule<MODE>(sched, args);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = sched.prefix[kE];

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      uint32_t it = 0;
      bool ok = true;
      const uint64_t keep = policy_evict_last();
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
        const Tile t = decode_tile<MODE>(sched, args, L);
        for (int kb = 0; kb < t.nkb; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], STAGE);
          uint8_t* a = sA + s * A_BYTES;
          uint8_t* b = sB + s * B_BYTES;
          if (MODE == kDH) {
            tma_load_2d_hint(a, &tmA0, &full[s], kb * BK, t.m0, keep);
#pragma unroll
            for (int c = 0; c < 4; ++c) tma_load_3d_hint(b + c * CHUNK, &tmB0, &full[s], kb * BK, t.n0 + 64 * c, t.e, keep);
          } else if (MODE == kDX) {
            const bool first = kb < args.half_kb;
            const int k0 = (first ? kb : kb - args.half_kb) * BK;
            tma_load_2d_hint(a, first ? &tmA0 : &tmA1, &full[s], k0, t.m0, keep);
#pragma unroll
            for (int c = 0; c < 4; ++c)
              tma_load_3d_hint(b + c * CHUNK, first ? &tmB0 : &tmB1, &full[s], k0, t.n0 + 64 * c, t.e, keep);
          } else {
            const int r0 = t.row0 + kb * BK;
            tma_load_3d_hint(a, &tmA0, &full[s], 0, r0, t.m0 / 64, keep);
            tma_load_3d_hint(b, &tmB0, &full[s], 0, r0, t.n0 / 64, keep);
            *issued_kb = it + 1;
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
    // -------------------------------------------------------------- MMA issuer
    // Lane 0 alone waits and issues, as in the forward GEMMs: a warp-wide loop
    // with a shuffle and a warp sync per K block held the dH and dx kernels
    // 25-35% below the MMA rate.
    if (lane == 0) {
      constexpr bool kMN = MODE == kWG;
      constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN, kMN, kMN);
      constexpr uint32_t IDESC_M64 = idesc_bf16_f32(64, BN, kMN, kMN);
      uint32_t it = 0, tc = 0, zphase = 0;  // zphase: parity bit per stage of `zeroed`
      bool ok = true, issued = false;
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x, ++tc) {
        const Tile t = decode_tile<MODE>(sched, args, L);
        // a row block of at most 64 rows (an expert's last) runs M = 64 MMAs
        const uint32_t idesc = (MODE != kWG && t.rows <= 64) ? IDESC_M64 : IDESC;
        const uint32_t buf = tc & 1u;
        const uint32_t tph = (tc >> 1) & 1u;
        if (!mbar_wait(&tempty[buf], tph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * kAccStride;
        for (int kb = 0; kb < t.nkb; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1u;
          // K steps of 16 rows issued for this block: the expert's last block
          // issues only the steps that hold its rows; when the last such step
          // also holds rows past the expert's end, the zeroing warp clears them
          // in both operands and releases the stage on zeroed[s] instead.
          int ksteps = BK / 16;
          bool ragged = false;
          if (MODE == kWG) {
            const int valid = t.nrows - kb * BK;
            if (valid < BK) {
              ksteps = (valid + 15) / 16;
              ragged = ksteps * 16 > valid;
            }
          }
          if (ragged) {
            if (!mbar_wait(&zeroed[s], (zphase >> s) & 1u, abort_flag)) {
              ok = false;
              break;
            }
            zphase ^= 1u << s;
          } else if (!mbar_wait(&full[s], ph, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + s * A_BYTES);
          const uint32_t b_addr = smem_u32(sB + s * B_BYTES);
          auto mma_step = [&](int kk) {
            uint64_t ad, bd;
            if (kMN) {
              ad = sw128_desc(a_addr + kk * 2048, CHUNK, 1024);
              bd = sw128_desc(b_addr + kk * 2048, CHUNK, 1024);
            } else {
              ad = sw128_desc(a_addr + kk * 32, 16, 1024);
              bd = sw128_desc(b_addr + kk * 32, 16, 1024);
            }
            umma_bf16(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
          };
          // full K blocks issue their four steps without a branch: a bound check
          // inside this loop cost the weight gradients 11% of the MMA rate
          if (ksteps == BK / 16) {
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) mma_step(kk);
          } else {
            for (int kk = 0; kk < ksteps; ++kk) mma_step(kk);
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
  } else if (warp == Warps<MODE>::kZeroWarp) {
    // ------------------------------------------------ ragged-row zeroing (kWG)
    // The tile's last K block may hold rows past the expert's end (the next
    // expert's rows, or rows past the kept ones): once the stage has landed,
    // zero those rows of the last 16-row step in all six 8 KB chunks (a row is
    // 128 bytes of a chunk, so the swizzle does not matter), make the writes
    // visible to the tensor core and release the stage to the MMA warp.  Every
    // lane waits for the stage itself, so its stores follow the TMA's.
    uint32_t it = 0;
    for (int L = blockIdx.x; L < total; L += gridDim.x) {
      const Tile t = decode_tile<MODE>(sched, args, L);
      const uint32_t it_last = it + (uint32_t)t.nkb - 1u;
      it += (uint32_t)t.nkb;
      if (t.nkb == 0) continue;
      const int valid = t.nrows - (t.nkb - 1) * BK;
      const int pad = (valid + 15) / 16 * 16 - valid;
      if (valid >= BK || pad == 0) continue;
      const int s = it_last % S;
      // bounded: the producer issues this K block's loads unless the kernel aborts
      const uint64_t t0 = globaltimer_ns();
      bool go = true;
      while ((int)(*issued_kb - it_last) <= 0) {
        if (*abort_flag || globaltimer_ns() - t0 > 2000000000ull) {
          go = false;
          break;
        }
        __nanosleep(32);
      }
      if (!go || !mbar_wait(&full[s], (it_last / S) & 1u, abort_flag)) {
        if (!*abort_flag) {
          if (lane == 0) flag_error(args.err, MOE_DEVERR_TIMEOUT);
          *abort_flag = 1;
        }
        break;
      }
      const int per_chunk = pad * 8;  // 16-byte pieces
      for (int i = lane; i < 6 * per_chunk; i += 32) {
        const int c = i / per_chunk;
        const int j = i - c * per_chunk;
        uint8_t* chunk = c < 2 ? sA + s * A_BYTES + c * CHUNK : sB + s * B_BYTES + (c - 2) * CHUNK;
        *reinterpret_cast<uint4*>(chunk + valid * 128 + j * 16) = make_uint4(0u, 0u, 0u, 0u);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&zeroed[s]);
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int q = warp & 3;
    // column chunks of 32 this warp covers: all 8, or one half with 8 epilogue warps
    constexpr int kSplit = Warps<MODE>::kEpi / 4;
    const int half = kSplit == 1 ? 0 : (warp - 2) / 4;
    const int c_begin = half * (BN / 32) / kSplit, c_end = c_begin + (BN / 32) / kSplit;
    uint32_t tc = 0;
    for (int L = blockIdx.x; L < total; L += gridDim.x, ++tc) {
      const Tile t = decode_tile<MODE>(sched, args, L);
      const uint32_t buf = tc & 1u;
      const uint32_t tph = (tc >> 1) & 1u;
      if (!mbar_wait(&tfull[buf], tph, abort_flag)) {
        if (lane == 0) flag_error(args.err, MOE_DEVERR_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t tacc = tmem_base + buf * kAccStride + ((uint32_t)(q * 32) << 16);
      // tile row of this thread; M = 64 accumulators hold row 16 q + i in lane i (< 16) of quarter q
      const int r = (MODE != kWG && t.rows <= 64) ? (lane < 16 ? q * 16 + lane : BM) : q * 32 + lane;
      if (MODE == kDH) {
        const bool valid = r < t.rows;
        const int64_t row = t.m0 + r;
        const float w = valid ? __ldg(args.row_scale + row) : 0.f;
        const int64_t base = row * args.ld + t.n0;
        float dot = 0.f;
        // G, U, H of a 32-column chunk: 4 x 16 bytes each; the next chunk's are
        // loaded while this one is computed, so the loads overlap the math.  They
        // and the dG, dU stores stream through L2 (evict-first): each is touched
        // once here, and keeping them from pushing out the operand tiles made
        // the kernel 5% faster at Grok size
        uint4 qg[4], qu[4], qh[4];
        auto load_chunk = [&](int c, uint4 (&a)[4], uint4 (&b)[4], uint4 (&hh)[4]) {
          const int64_t o = base + c * 32;
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            a[p] = __ldcs(reinterpret_cast<const uint4*>(args.G + o + p * 8));
            b[p] = __ldcs(reinterpret_cast<const uint4*>(args.U + o + p * 8));
            hh[p] = __ldcs(reinterpret_cast<const uint4*>(args.H + o + p * 8));
          }
        };
        if (valid) load_chunk(c_begin, qg, qu, qh);
#pragma unroll 1
        for (int c = c_begin; c < c_end; ++c) {
          uint32_t v[32];
          tmem_ld32(tacc + c * 32, v);
          const bool more = c + 1 < c_end;
          uint4 ng[4], nu[4], nh[4];
          if (valid && more) load_chunk(c + 1, ng, nu, nh);
          tmem_wait_ld();
          if (valid) {
#pragma unroll
            for (int p = 0; p < 4; ++p) {
              const int64_t o = base + c * 32 + p * 8;
              float g[8], u[8], h[8];
              unpack8_bf16(qg[p], g);
              unpack8_bf16(qu[p], u);
              unpack8_bf16(qh[p], h);
              uint32_t og[4], ou[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                float dg2[2], du2[2];
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                  const int j = 2 * i + k;
                  const float dhu = __uint_as_float(v[p * 8 + j]);
                  dot = fmaf(dhu, h[j], dot);
                  const float dh = w * dhu;
                  const float sg = 1.0f / (1.0f + __expf(-g[j]));
                  const float sl = g[j] * sg;
                  dg2[k] = dh * u[j] * (sg * (1.0f + g[j] * (1.0f - sg)));
                  du2[k] = dh * sl;
                }
                og[i] = pack_bf16x2(dg2[0], dg2[1]);
                ou[i] = pack_bf16x2(du2[0], du2[1]);
              }
              __stcs(reinterpret_cast<uint4*>(args.dG + o), make_uint4(og[0], og[1], og[2], og[3]));
              __stcs(reinterpret_cast<uint4*>(args.dU + o), make_uint4(ou[0], ou[1], ou[2], ou[3]));
            }
          }
          if (more) {
#pragma unroll
            for (int p = 0; p < 4; ++p) {
              qg[p] = ng[p];
              qu[p] = nu[p];
              qh[p] = nh[p];
            }
          }
        }
        if (valid) args.dw_part[row * (int64_t)args.n_tiles * kSplit + t.nb * kSplit + half] = dot;
      } else if (MODE == kDX) {
        int tok = -1;
        if (r < t.rows) {
          tok = __ldg(args.perm + t.m0 + r);
          if (tok < 0 || (int64_t)tok >= args.n_tok) {
            flag_error(args.err, MOE_DEVERR_SLOT_INDEX);
            tok = -1;
          }
        }
        float* dst = args.out + (int64_t)(tok < 0 ? 0 : tok) * args.ld + t.n0;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tacc + c * 32, v);
          tmem_wait_ld();
          if (tok >= 0) {
            float4* d4 = reinterpret_cast<float4*>(dst + c * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              atomicAdd(d4 + i, make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                            __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3])));
          }
        }
      } else {
        // 32 rows x 32 columns per TMA store: lane = row, its 8 16-byte pieces
        // placed with the 128-byte swizzle (piece j of row r at j ^ (r % 8))
        const bool zero = t.nkb == 0;
        uint8_t* stage0 = sOut + (q * 2) * OUT_STAGE;
        const int y = t.e * (int)args.M + t.m0 + q * 32;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tacc + c * 32, v);
          tmem_wait_ld();
          uint8_t* st = stage0 + (c & 1) * OUT_STAGE;
          if (lane == 0) bulk_wait_group_read<1>();  // the store that last read this buffer is done with it
          __syncwarp();
          float4* row = reinterpret_cast<float4*>(st + lane * 128);
#pragma unroll
          for (int j = 0; j < 8; ++j)
            row[j ^ (lane & 7)] = zero ? make_float4(0.f, 0.f, 0.f, 0.f)
                                       : make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                                     __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmOut, st, t.n0 + c * 32, y);
            bulk_commit_group();
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[buf]);
    }
  }

  // tile stores still in flight must finish before the CTA (and its shared memory) goes
  if (MODE == kWG && warp >= 2 && lane == 0) bulk_wait_group_all();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

template <int MODE>
cudaError_t launch_bwd(const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& b0, const CUtensorMap& b1,
                       const CUtensorMap& out, const BwdArgs& args, cudaStream_t s, const Ctx& ctx) {
  auto kern = bwd_gemm_kernel<MODE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  kern<<<ctx.num_sms, Warps<MODE>::kThreads, SMEM_BYTES, s>>>(a0, a1, b0, b1, out, args);
  return cudaGetLastError();
}

BwdArgs base_args(const moe_config_t& c, const int32_t* offsets, const Ctx& ctx) {
  BwdArgs a = {};
  a.offsets = offsets;
  a.rows_alloc = slot_rows(c);
  a.n_tok = c.T;
  a.err = ctx.err;
  return a;
}

bool map_rows(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, uint32_t box_rows) {
  const uint64_t dims[2] = {(uint64_t)cols, (uint64_t)rows};
  const uint64_t str[1] = {(uint64_t)cols * 2};
  const uint32_t box[2] = {64, box_rows};
  return encode_tmap(m, base, 2, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

// [E, R, C] weights, box of 64 columns x 64 rows of one expert
bool map_weights(CUtensorMap* m, const void* base, int E, int64_t R, int64_t C) {
  const uint64_t dims[3] = {(uint64_t)C, (uint64_t)R, (uint64_t)E};
  const uint64_t str[2] = {(uint64_t)C * 2, (uint64_t)R * C * 2};
  const uint32_t box[3] = {64, 64, 1};
  return encode_tmap(m, base, 3, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

int bwd_dh_parts_per_tile() { return Warps<kDH>::kEpi / 4; }

cudaError_t launch_bwd_dh(const moe_config_t& c, const void* dout_perm, const int32_t* offsets, const void* wd,
                          const void* G, const void* U, const void* H, const float* row_scale, void* dG, void* dU,
                          float* dw_part, cudaStream_t s, const Ctx& ctx) {
  const int64_t rows = slot_rows(c);
  if (rows == 0) return cudaSuccess;
  CUtensorMap ta, tb;
  // W_down [E, f, d] read K-major: rows = f (N), columns = d (K)
  if (!map_rows(&ta, dout_perm, rows, c.d, 128) || !map_weights(&tb, wd, c.E, c.f, c.d))
    return cudaErrorInvalidValue;
  BwdArgs a = base_args(c, offsets, ctx);
  a.n_tiles = (int)(c.f / BN);
  a.num_kb = (int)(c.d / BK);
  a.row_scale = row_scale;
  a.G = static_cast<const __nv_bfloat16*>(G);
  a.U = static_cast<const __nv_bfloat16*>(U);
  a.H = static_cast<const __nv_bfloat16*>(H);
  a.dG = static_cast<__nv_bfloat16*>(dG);
  a.dU = static_cast<__nv_bfloat16*>(dU);
  a.dw_part = dw_part;
  a.ld = c.f;
  return launch_bwd<kDH>(ta, ta, tb, tb, ta, a, s, ctx);
}

cudaError_t launch_bwd_dx(const moe_config_t& c, const void* dG, const void* dU, const int32_t* offsets,
                          const void* wg, const void* wu, const int32_t* perm, float* dx32, cudaStream_t s,
                          const Ctx& ctx) {
  const int64_t rows = slot_rows(c);
  if (rows == 0) return cudaSuccess;
  CUtensorMap ta0, ta1, tb0, tb1;
  // W_gate / W_up [E, d, f] read K-major: rows = d (N), columns = f (K)
  if (!map_rows(&ta0, dG, rows, c.f, 128) || !map_rows(&ta1, dU, rows, c.f, 128) ||
      !map_weights(&tb0, wg, c.E, c.d, c.f) || !map_weights(&tb1, wu, c.E, c.d, c.f))
    return cudaErrorInvalidValue;
  BwdArgs a = base_args(c, offsets, ctx);
  a.n_tiles = (int)(c.d / BN);
  a.half_kb = (int)(c.f / BK);
  a.num_kb = 2 * a.half_kb;
  a.perm = perm;
  a.out = dx32;
  a.ld = c.d;
  return launch_bwd<kDX>(ta0, ta1, tb0, tb1, ta0, a, s, ctx);
}

cudaError_t launch_bwd_wgrad(const moe_config_t& c, const void* a_rows, int64_t M, const void* b_rows, int64_t N,
                             const int32_t* offsets, float* dW, bool m_outer, cudaStream_t s, const Ctx& ctx) {
  const int64_t rows = slot_rows(c);
  if (rows == 0 || M % BM != 0 || N % BN != 0) return rows == 0 ? cudaSuccess : cudaErrorInvalidValue;
  CUtensorMap ta, tb, to;
  {
    // [rows, C] viewed as [C / 64 chunks][rows][64]: one box = nch chunks of 64 x 64
    const uint64_t a_dims[3] = {64, (uint64_t)rows, (uint64_t)(M / 64)};
    const uint64_t a_str[2] = {(uint64_t)M * 2, 128};
    const uint32_t a_box[3] = {64, 64, 2};
    const uint64_t b_dims[3] = {64, (uint64_t)rows, (uint64_t)(N / 64)};
    const uint64_t b_str[2] = {(uint64_t)N * 2, 128};
    const uint32_t b_box[3] = {64, 64, 4};
    if (!encode_tmap(&ta, a_rows, 3, a_dims, a_str, a_box, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tmap(&tb, b_rows, 3, b_dims, b_str, b_box, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  // dW [E * M, N] fp32, stored 32 x 32 at a time from the swizzled staging tiles
  const uint64_t o_dims[2] = {(uint64_t)N, (uint64_t)c.E * M};
  const uint64_t o_str[1] = {(uint64_t)N * 4};
  const uint32_t o_box[2] = {32, 32};
  if (!encode_tmap_dtype(&to, dW, 2, o_dims, o_str, o_box, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_DATA_TYPE_FLOAT32))
    return cudaErrorInvalidValue;
  BwdArgs a = base_args(c, offsets, ctx);
  a.m_tiles = (int)(M / BM);
  a.n_tiles = (int)(N / BN);
  a.m_outer = m_outer ? 1 : 0;
  a.out = dW;
  a.ld = N;
  a.M = M;
  return launch_bwd<kWG>(ta, ta, tb, tb, to, a, s, ctx);
}

}  // namespace moe
