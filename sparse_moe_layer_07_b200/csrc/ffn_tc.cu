// Grouped expert GEMMs on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// "How does Grok-1 use a mixture-of-experts design?", section "Expert
// implementation: SwiGLU at scale": every expert is y = W_down(silu(W_gate x) *
// W_up x) without bias, and FusedSwiGLUExpert computes gate and up with one
// matmul of width 2f.  Here:
//   gate/up : rows r of expert e:  H[r, n0:n0+128] = silu(X W_gate[e]) * (X W_up[e])
//             one 128 x 256 x 16 MMA per K step covers the gate AND up columns
//             of the tile (two 64-column chunks of each weight side by side in
//             shared memory), so the SwiGLU is applied in the epilogue straight
//             from the TMEM accumulator and H is written once, in bf16.
//   down    : Y[r, n0:n0+BN] = row_scale[r] * (H W_down[e])   (fp32 out)
//
// Layouts: X / H row-major [rows, K] (K-major A); weights row-major [E, K, N]
// (N contiguous, so B is MN-major, legal for 16-bit UMMA).  One TMA box per
// 128 B x 64 rows, 128-byte swizzle on both sides.
//
// Schedule: persistent, one CTA per SM.  The tile list is every
// (expert, 128-row block, N block); tiles of one expert are ordered N-block
// major so CTAs running at the same time share weight tiles and row blocks in
// L2 (row-block-major order measured 50% slower), and both operands are
// loaded with an evict-last L2 policy (1-2% faster than the default policy;
// evict-first on the weights was 13% slower).  Rows of an expert's last block that belong to the next expert are
// computed but not stored.  Warp roles (192 threads):
//   warp 0 lane 0 : TMA producer over a kStages ring (full/empty mbarriers)
//   warp 1 lane 0 : MMA issuer; warp 1 owns the 512 TMEM columns
//                   (two 256-column fp32 accumulators, double buffered)
//   warps 2..5    : epilogue; warp w reads TMEM lanes 32*(w%4) .. +31
// Every mbarrier wait is bounded; on a timeout the CTA flags the device error
// word, the other roles stop, in-flight copies and MMAs are drained and TMEM is
// released before the CTA exits.
#include <cuda.h>
#include <cuda_bf16.h>

#include <atomic>

#include "common.cuh"
#include "internal.h"
#include "tc_ptx.cuh"

namespace moe {
namespace {

using namespace ptx;

constexpr int kE = 8;
constexpr int BM = 128;
constexpr int BK = 64;
constexpr int kThreads = 192;
constexpr int kTmemCols = 512;
constexpr int kAccStride = 256;  // TMEM columns between the two accumulators
constexpr int A_BYTES = BM * BK * 2;      // 16 KB
constexpr int CHUNK_BYTES = 64 * BK * 2;  // 8 KB: 64 N-columns x 64 K-rows

enum Mode { kGateUp = 0, kDown = 1 };

template <int MODE, int MMA_N>
struct Cfg {
  static constexpr int kChunks = MMA_N / 64;
  static constexpr int B_BYTES = kChunks * CHUNK_BYTES;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int kStages = MMA_N == 256 ? 4 : 6;
  static constexpr int BN_OUT = MODE == kGateUp ? MMA_N / 2 : MMA_N;  // output columns per tile
  static constexpr int kBarBytes = 256;
  static constexpr int SMEM_BYTES = 1024 + kStages * STAGE_BYTES + kBarBytes;
  static constexpr uint32_t IDESC = idesc_bf16_f32(BM, MMA_N, false, true);
  // an expert's last row block with at most 64 rows runs M = 64 MMAs (half the
  // work; measured, an M = 64 MMA takes as many clocks as an M = 128 one)
  static constexpr uint32_t IDESC_M64 = idesc_bf16_f32(64, MMA_N, false, true);
};

struct TcArgs {
  const int32_t* offsets;  // [E + 1], device
  int64_t rows_alloc;      // rows of the A and output buffers
  int n_tiles;             // output N / BN_OUT
  int num_kb;              // K / BK
  void* out;
  int64_t ld_out;          // elements per output row
  const float* row_scale;  // down only; NULL means 1
  const int32_t* perm;     // fused variants: source token of each row
  int64_t n_tok;           // fused variants: rows of x / out (tokens)
  // fused down over peer memory: perm holds p * n_tok + t and row t of source
  // rank p's sums is peer_out[p] + t * ld_out (n_peers == 0: out is the one
  // destination)
  int n_peers = 0;
  float* peer_out[MOE_EP_MAX_WORLD] = {};
  void* save_g;            // gate/up for training: also write G and U (bf16) or NULL
  void* save_u;
  int* err;
};

struct Sched {
  int offs[kE + 1];
  int mt[kE];
  int prefix[kE + 1];
};

struct Tile {
  int e, m0, rows, n0;
};

__device__ __forceinline__ Tile decode_tile(const Sched& s, int L, int bn, int bm = BM) {
  int e = 0;
#pragma unroll
  for (int k = 1; k < kE; ++k)
    if (L >= s.prefix[k]) e = k;
  const int local = L - s.prefix[e];
  const int nt = local / s.mt[e];
  const int mi = local - nt * s.mt[e];
  Tile t;
  t.e = e;
  t.m0 = s.offs[e] + mi * bm;
  const int left = s.offs[e + 1] - t.m0;
  t.rows = left < bm ? left : bm;
  t.n0 = nt * bn;
  return t;
}

// Reads and checks the expert offsets, then lays out the tile list: expert e
// has ceil(rows_e / bm) row blocks times n_tiles column blocks.
__device__ __forceinline__ void build_schedule(Sched& sched, const TcArgs& args, int bm) {
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
    sched.mt[k] = (n + bm - 1) / bm;
    sched.prefix[k] = acc;
    acc += sched.mt[k] * args.n_tiles;
  }
  sched.prefix[kE] = acc;
  if (!ok) flag_error(args.err, MOE_DEVERR_OFFSETS);
}

// Source token of grouped row `row` for the fused variants (0 for rows past the
// kept ones, which are computed and never stored; a bad index is flagged).
__device__ __forceinline__ int source_token(const TcArgs& args, int row, int n_rows) {
  if (row >= n_rows) return 0;
  const int t = __ldg(args.perm + row);
  if (t < 0 || (int64_t)t >= args.n_tok * (args.n_peers > 0 ? args.n_peers : 1)) {
    flag_error(args.err, MOE_DEVERR_SLOT_INDEX);
    return -1;
  }
  return t;
}

// Epilogue of one tile for one thread: the thread's TMEM lane holds tile row r
// of this CTA (global grouped row row0 + r), output columns [n0, n0 + n_cols)
// from TMEM column `tacc` on (gate/up: the matching up columns u_off further
// on).  Rows with valid == false are read (the TMEM loads are warp-wide) but
// not stored.  n_rows = kept rows.
template <int MODE, bool kScatter>
__device__ __forceinline__ void epilogue_rows(const TcArgs& args, int n_rows, int row0, int r, bool valid, int n0,
                                              int n_cols, int u_off, uint32_t tacc) {
  if (MODE == kGateUp) {
    __nv_bfloat16* H = static_cast<__nv_bfloat16*>(args.out);
    __nv_bfloat16* dst_row = H + (int64_t)(row0 + r) * args.ld_out + n0;
    // 32-column chunks (n_cols <= 128); the TMEM loads of chunk c + 1 are in
    // flight while chunk c is computed and stored (the loop is unrolled so the
    // two register sets stay in registers)
    const int nch = n_cols / 32;
    uint32_t gb[2][32], ub[2][32];
    tmem_ld32(tacc, gb[0]);
    tmem_ld32(tacc + u_off, ub[0]);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      if (c >= nch) break;
      tmem_wait_ld();
      tmem_regs_ready(gb[c & 1]);
      tmem_regs_ready(ub[c & 1]);
      if (c + 1 < nch) {
        tmem_ld32(tacc + (c + 1) * 32, gb[(c + 1) & 1]);
        tmem_ld32(tacc + u_off + (c + 1) * 32, ub[(c + 1) & 1]);
      }
      const uint32_t(&g)[32] = gb[c & 1];
      const uint32_t(&u)[32] = ub[c & 1];
      uint32_t p[16];
#pragma unroll
      for (int i = 0; i < 16; ++i)
        p[i] = pack_bf16x2(silu_mul_fast(__uint_as_float(g[2 * i]), __uint_as_float(u[2 * i])),
                           silu_mul_fast(__uint_as_float(g[2 * i + 1]), __uint_as_float(u[2 * i + 1])));
      if (valid) {
        // streaming stores: H is read back by the next launch, not by this one, so
        // its lines should not push the operand tiles out of L2 (1-2% faster)
        uint4* d4 = reinterpret_cast<uint4*>(dst_row + c * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i) __stcs(d4 + i, make_uint4(p[4 * i], p[4 * i + 1], p[4 * i + 2], p[4 * i + 3]));
        if (args.save_g) {
          // training: keep the pre-activations for the backward pass
          const int64_t o = (int64_t)(row0 + r) * args.ld_out + n0 + c * 32;
          uint4* g4 = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(args.save_g) + o);
          uint4* u4 = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(args.save_u) + o);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            g4[i] = make_uint4(pack_bf16x2(__uint_as_float(g[8 * i]), __uint_as_float(g[8 * i + 1])),
                               pack_bf16x2(__uint_as_float(g[8 * i + 2]), __uint_as_float(g[8 * i + 3])),
                               pack_bf16x2(__uint_as_float(g[8 * i + 4]), __uint_as_float(g[8 * i + 5])),
                               pack_bf16x2(__uint_as_float(g[8 * i + 6]), __uint_as_float(g[8 * i + 7])));
            u4[i] = make_uint4(pack_bf16x2(__uint_as_float(u[8 * i]), __uint_as_float(u[8 * i + 1])),
                               pack_bf16x2(__uint_as_float(u[8 * i + 2]), __uint_as_float(u[8 * i + 3])),
                               pack_bf16x2(__uint_as_float(u[8 * i + 4]), __uint_as_float(u[8 * i + 5])),
                               pack_bf16x2(__uint_as_float(u[8 * i + 6]), __uint_as_float(u[8 * i + 7])));
          }
        }
      }
    }
  } else if (kScatter) {
    float* O = static_cast<float*>(args.out);
    int tok = valid ? source_token(args, row0 + r, n_rows) : -1;
    const bool store = tok >= 0;
    if (store && args.n_peers > 0) {
      const int p = tok / (int)args.n_tok;
      tok -= p * (int)args.n_tok;
#pragma unroll
      for (int i = 0; i < MOE_EP_MAX_WORLD; ++i)
        if (i == p) O = args.peer_out[i];
    }
    float* dst_row = O + (int64_t)(store ? tok : 0) * args.ld_out + n0;
    const float sc = (store && args.row_scale) ? __ldg(args.row_scale + row0 + r) : 1.0f;
#pragma unroll 1
    for (int c = 0; c < n_cols / 32; ++c) {
      uint32_t v[32];
      tmem_ld32(tacc + c * 32, v);
      tmem_wait_ld();
      if (store) {
        float4* d4 = reinterpret_cast<float4*>(dst_row + c * 32);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          atomicAdd(d4 + i, make_float4(sc * __uint_as_float(v[4 * i]), sc * __uint_as_float(v[4 * i + 1]),
                                        sc * __uint_as_float(v[4 * i + 2]), sc * __uint_as_float(v[4 * i + 3])));
      }
    }
  } else {
    float* Y = static_cast<float*>(args.out);
    float* dst_row = Y + (int64_t)(row0 + r) * args.ld_out + n0;
    const float sc = (valid && args.row_scale) ? __ldg(args.row_scale + row0 + r) : 1.0f;
#pragma unroll 1
    for (int c = 0; c < n_cols / 32; ++c) {
      uint32_t v[32];
      tmem_ld32(tacc + c * 32, v);
      tmem_wait_ld();
      if (valid) {
        float4* d4 = reinterpret_cast<float4*>(dst_row + c * 32);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          d4[i] = make_float4(sc * __uint_as_float(v[4 * i]), sc * __uint_as_float(v[4 * i + 1]),
                              sc * __uint_as_float(v[4 * i + 2]), sc * __uint_as_float(v[4 * i + 3]));
      }
    }
  }
}

// FUSED = true (down only): instead of writing Y by grouped row, the epilogue
// adds row_scale * (H W_down) into a zeroed fp32 out[token] with vector
// atomics.  With top-2 a token receives at most two terms and 0 + a + b rounds
// the same in either order, so the result is the combine's fp32 sum bit for
// bit, without the Y buffer.
template <int MODE, int MMA_N, bool FUSED>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                           const __grid_constant__ CUtensorMap tmB1, const TcArgs args) {
  using C = Cfg<MODE, MMA_N>;
  constexpr bool kScatter = FUSED && MODE == kDown;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* sA = smem;
  uint8_t* sB = smem + S * A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * C::STAGE_BYTES);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  __shared__ Sched sched;

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
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB0);
    prefetch_tmap(&tmB1);
  }
  // everything above is local to the CTA; what follows reads the previous kernels' outputs
  pdl_wait();
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  if (warp == 2 && lane == 0) build_schedule(sched, args, BM);
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
        const Tile t = decode_tile(sched, L, C::BN_OUT);
        for (int kb = 0; kb < args.num_kb; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], C::STAGE_BYTES);
          uint8_t* b = sB + s * C::B_BYTES;
          tma_load_2d_hint(sA + s * A_BYTES, &tmA, &full[s], kb * BK, t.m0, keep);
          if (MODE == kGateUp) {
#pragma unroll
            for (int c = 0; c < C::kChunks / 2; ++c) {
              tma_load_3d_hint(b + c * CHUNK_BYTES, &tmB0, &full[s], t.n0 + 64 * c, kb * BK, t.e, keep);
              tma_load_3d_hint(b + (C::kChunks / 2 + c) * CHUNK_BYTES, &tmB1, &full[s], t.n0 + 64 * c, kb * BK, t.e, keep);
            }
          } else {
#pragma unroll
            for (int c = 0; c < C::kChunks; ++c)
              tma_load_3d_hint(b + c * CHUNK_BYTES, &tmB0, &full[s], t.n0 + 64 * c, kb * BK, t.e, keep);
          }
        }
      }
      if (!ok) {
        flag_error(args.err, MOE_DEVERR_TIMEOUT);
        *abort_flag = 1;
      }
      // drain: every issued load must land before the CTA can exit
      const uint32_t first = it > (uint32_t)S ? it - S : 0u;
      for (uint32_t j = first; j < it; ++j) mbar_wait(&full[j % S], (j / S) & 1u, nullptr, 100000000ull);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      uint32_t it = 0, tc = 0;
      bool ok = true, issued = false;
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x, ++tc) {
        const uint32_t buf = tc & 1u;
        const uint32_t tph = (tc >> 1) & 1u;
        const uint32_t idesc = decode_tile(sched, L, C::BN_OUT).rows <= 64 ? C::IDESC_M64 : C::IDESC;
        if (!mbar_wait(&tempty[buf], tph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * kAccStride;
        for (int kb = 0; kb < args.num_kb; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1u;
          if (!mbar_wait(&full[s], ph, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + s * A_BYTES);
          const uint32_t b_addr = smem_u32(sB + s * C::B_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = sw128_desc(a_addr + kk * 32, 16, 1024);
            const uint64_t bd = sw128_desc(b_addr + kk * 2048, CHUNK_BYTES, 1024);
            umma_bf16(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
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
        // all MMAs must finish before TMEM and shared memory are released
        umma_commit(drain);
        mbar_wait(drain, 0, nullptr, 100000000ull);
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    uint32_t tc = 0;
    for (int L = blockIdx.x; L < total; L += gridDim.x, ++tc) {
      const Tile t = decode_tile(sched, L, C::BN_OUT);
      const uint32_t buf = tc & 1u;
      const uint32_t tph = (tc >> 1) & 1u;
      if (!mbar_wait(&tfull[buf], tph, abort_flag)) {
        if (lane == 0) flag_error(args.err, MOE_DEVERR_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      // M = 64 accumulators hold tile row 16 q + i in lane i (< 16) of lane quarter q
      const int r = t.rows <= 64 ? (lane < 16 ? q * 16 + lane : BM) : q * 32 + lane;
      const bool valid = r < t.rows;
      const uint32_t tacc = tmem_base + buf * kAccStride + ((uint32_t)(q * 32) << 16);
      epilogue_rows<MODE, kScatter>(args, sched.offs[kE], t.m0, r, valid, t.n0, C::BN_OUT, C::BN_OUT, tacc);
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

// ------------------------------------------------------------------ CTA pairs
// The same grouped GEMMs on CTA pairs (clusters of 2 on the two SMs of a TPC):
// one 256 x 256 x 16 MMA per K step spans both SMs.  Each CTA stages its own
// 128 A rows and half of the B columns (gate/up: the leader stages the 128
// W_gate columns of the tile, the other CTA the matching 128 W_up columns; down:
// each stages 128 of the 256 W_down columns), so a CTA moves 32 KB per K step
// instead of 48 KB and the ring holds 6 stages.  The leader (cluster rank 0)
// issues every MMA; both CTAs run their own epilogue on the 128 accumulator
// rows in their TMEM (tile row 128 r + i in lane i of CTA r).
//
// An expert's last row block with at most 128 rows runs M = 128 pair MMAs: CTA
// r supplies tile rows 64 r .. 64 r + 63, and its TMEM holds row 64 r + i in
// lane i for accumulator columns [0, 128) and in lane 64 + i for columns
// [128, 256), both at TMEM columns [0, 128).  For gate/up the two CTAs then
// stage W_gate and W_up chunks side by side (CTA r: the 64 gate and 64 up
// columns n0 + 64 r ..), so every lane sees a gate column and its up column 64
// TMEM columns apart.  Rows past an expert's end are computed, never stored.
//
// Barriers: full[s] lives in the leader and counts both CTAs' bytes (each CTA's
// TMA signals it); empty[s] and tfull[b] live in both CTAs and are signalled
// together by the leader's commits (the async proxy orders the data behind
// these three, so their waits are CTA-scope); tempty[b] lives in the leader and
// takes one release-at-cluster-scope arrival per epilogue warp of either CTA.
// A timeout in either CTA raises the abort flag of both.
constexpr int PBM = 256;           // rows per pair tile
constexpr int kPairStages = 6;
constexpr int PB_BYTES = 2 * CHUNK_BYTES;  // B columns a CTA stages per K step (128)
constexpr int PSTAGE_BYTES = A_BYTES + PB_BYTES;
constexpr int PAIR_SMEM_BYTES = 1024 + kPairStages * PSTAGE_BYTES + 256;
constexpr uint32_t IDESC_PAIR = idesc_bf16_f32(256, 256, false, true);
constexpr uint32_t IDESC_PAIR_M128 = idesc_bf16_f32(128, 256, false, true);

template <int MODE, bool FUSED>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_tc_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                                const __grid_constant__ CUtensorMap tmB1, const TcArgs args) {
  constexpr bool kScatter = FUSED && MODE == kDown;
  constexpr int S = kPairStages;
  constexpr int BN_OUT = MODE == kGateUp ? 128 : 256;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* sA = smem;
  uint8_t* sB = smem + S * A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * PSTAGE_BYTES);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  __shared__ Sched sched;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1;
  const int n_pairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 8);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 1) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB0);
    prefetch_tmap(&tmB1);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
    tc_fence_before();
  }
  if (warp == 2 && lane == 0) build_schedule(sched, args, PBM);
  __syncthreads();
  cluster_sync();  // both CTAs' barriers are initialised before either signals the other's
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = sched.prefix[kE];
  const uint32_t full_lead = mapa_shared(smem_u32(full), 0);
  const uint32_t tempty_lead = mapa_shared(smem_u32(tempty), 0);
  const uint32_t abort_peer = mapa_shared(smem_u32(const_cast<int*>(abort_flag)), rank ^ 1u);
  auto raise_abort = [&]() {
    *abort_flag = 1;
    st_cluster_u32(abort_peer, 1u);
  };

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producers (both CTAs)
      uint32_t it = 0;
      bool ok = true;
      const uint64_t keep = policy_evict_last();
      for (int L = pair; L < total && ok; L += n_pairs) {
        const Tile t = decode_tile(sched, L, BN_OUT, PBM);
        const bool half = t.rows <= 128;
        const int a_row = t.m0 + (int)rank * (half ? 64 : 128);
        // B columns of the two chunks this CTA stages (see the layouts above)
        const CUtensorMap* tb0 = (MODE == kGateUp && rank && !half) ? &tmB1 : &tmB0;
        const CUtensorMap* tb1 = (MODE == kGateUp && (rank || half)) ? &tmB1 : &tmB0;
        int c0, c1;
        if (MODE == kGateUp) {
          c0 = half ? t.n0 + 64 * (int)rank : t.n0;
          c1 = half ? c0 : t.n0 + 64;
        } else {
          c0 = t.n0 + 128 * (int)rank;
          c1 = c0 + 64;
        }
        for (int kb = 0; kb < args.num_kb; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * PSTAGE_BYTES);
          const uint32_t bar = full_lead + 8u * (uint32_t)s;
          uint8_t* b = sB + s * PB_BYTES;
          tma_load_2d_pair(sA + s * A_BYTES, &tmA, bar, kb * BK, a_row, keep);
          tma_load_3d_pair(b, tb0, bar, c0, kb * BK, t.e, keep);
          tma_load_3d_pair(b + CHUNK_BYTES, tb1, bar, c1, kb * BK, t.e, keep);
        }
      }
      if (!ok) {
        flag_error(args.err, MOE_DEVERR_TIMEOUT);
        raise_abort();
      }
      if (rank == 0) {
        // drain: the leader's full barriers count both CTAs' loads
        const uint32_t first = it > (uint32_t)S ? it - S : 0u;
        for (uint32_t j = first; j < it; ++j) mbar_wait(&full[j % S], (j / S) & 1u, nullptr, 100000000ull);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ------------------------------------------------------------ MMA issuer (leader)
      uint32_t it = 0, tc = 0;
      bool ok = true, issued = false;
      for (int L = pair; L < total && ok; L += n_pairs, ++tc) {
        const uint32_t buf = tc & 1u;
        const uint32_t tph = (tc >> 1) & 1u;
        if (!mbar_wait<true>(&tempty[buf], tph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * kAccStride;
        const uint32_t idesc = decode_tile(sched, L, BN_OUT, PBM).rows <= 128 ? IDESC_PAIR_M128 : IDESC_PAIR;
        for (int kb = 0; kb < args.num_kb; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1u;
          if (!mbar_wait(&full[s], ph, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + s * A_BYTES);
          const uint32_t b_addr = smem_u32(sB + s * PB_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = sw128_desc(a_addr + kk * 32, 16, 1024);
            const uint64_t bd = sw128_desc(b_addr + kk * 2048, CHUNK_BYTES, 1024);
            umma_bf16_pair(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          issued = true;
          umma_commit_pair_to(&empty[s], 0x3);
        }
        if (!ok) break;
        umma_commit_pair_to(&tfull[buf], 0x3);
      }
      if (!ok) {
        flag_error(args.err, MOE_DEVERR_TIMEOUT);
        raise_abort();
      }
      if (issued) {
        // all MMAs must finish before either CTA releases TMEM or shared memory
        umma_commit_pair(drain);
        mbar_wait(drain, 0, nullptr, 100000000ull);
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue (both CTAs)
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    uint32_t tc = 0;
    for (int L = pair; L < total; L += n_pairs, ++tc) {
      const Tile t = decode_tile(sched, L, BN_OUT, PBM);
      const uint32_t buf = tc & 1u;
      const uint32_t tph = (tc >> 1) & 1u;
      if (!mbar_wait(&tfull[buf], tph, abort_flag)) {
        if (lane == 0) {
          flag_error(args.err, MOE_DEVERR_TIMEOUT);
          raise_abort();
        }
        break;
      }
      tc_fence_after();
      const uint32_t tacc = tmem_base + buf * kAccStride + ((uint32_t)(q * 32) << 16);
      if (t.rows > 128) {
        const int r = q * 32 + lane;
        epilogue_rows<MODE, kScatter>(args, sched.offs[kE], t.m0 + (int)rank * 128, r, r < t.rows - (int)rank * 128,
                                      t.n0, BN_OUT, BN_OUT, tacc);
      } else {
        // M = 128 pair tile: lane quarters 0 / 1 hold rows 0-31 / 32-63 of this
        // CTA's 64 with the first half of the columns, quarters 2 / 3 the same
        // rows with the second half
        const int r = (q & 1) * 32 + lane;
        const int cols = BN_OUT / 2;
        epilogue_rows<MODE, kScatter>(args, sched.offs[kE], t.m0 + (int)rank * 64, r, r < t.rows - (int)rank * 64,
                                      t.n0 + (q >> 1) * cols, cols, cols, tacc);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_lead + 8u * buf);
    }
  }

  __syncthreads();
  cluster_sync();  // neither CTA leaves while the other may still signal it or use its TMEM
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

// Pairs that fit on the device at once (clusters of 2 at one CTA per SM);
// cached per kernel.
template <int MODE, bool FUSED>
int pair_grid(const Ctx& ctx) {
  static std::atomic<int> cached[64];
  const int slot = ctx.dev >= 0 && ctx.dev < 64 ? ctx.dev : 0;
  const int known = cached[slot].load(std::memory_order_relaxed);
  if (known > 0) return known;
  auto kern = grouped_gemm_tc_pair_kernel<MODE, FUSED>;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = PAIR_SMEM_BYTES;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) {
    (void)cudaGetLastError();
    n = ctx.num_sms / 2;
  }
  if (n > ctx.num_sms / 2) n = ctx.num_sms / 2;
  if (n < 1) n = 1;
  cached[slot].store(n, std::memory_order_relaxed);
  return n;
}

template <int MODE, bool FUSED>
cudaError_t launch_pair(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1, const TcArgs& args,
                        cudaStream_t s, const Ctx& ctx) {
  auto kern = grouped_gemm_tc_pair_kernel<MODE, FUSED>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, PAIR_SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int pairs = pair_grid<MODE, FUSED>(ctx);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = PAIR_SMEM_BYTES;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, a, b0, b1, args);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int MODE, int MMA_N, bool FUSED = false>
cudaError_t launch_grouped(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1, const TcArgs& args,
                           cudaStream_t s, const Ctx& ctx) {
  using C = Cfg<MODE, MMA_N>;
  auto kern = grouped_gemm_tc_kernel<MODE, MMA_N, FUSED>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  e = launch_pdl(kern, dim3(ctx.num_sms), dim3(kThreads), C::SMEM_BYTES, s, no_extra_attr(), a, b0, b1, args);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace

namespace {
std::atomic<int> g_tile_mode{MOE_TILES_AUTO};
}  // namespace

int set_tile_mode(int mode) { return g_tile_mode.exchange(mode); }

// Automatic choice: single-CTA tiles.  Timed back to back in one process on a
// power-capped B200, the pair kernels were 7% slower than the single-CTA ones
// at the Grok-1 prefill shape (T 8192, d 6144, f 32768: gate/up 11.83 vs 11.03
// ms, down + combine 6.06 vs 5.67 ms) and gate/up 9% slower at T 4096, f 8192
// (down 2% faster there): the pair's tensor pipe was busy 80% of the time
// against 88% for single CTAs, and the halved operand traffic buys nothing
// once the single-CTA kernel is bound by the tensor pipe at the capped clock.
bool use_pair_tiles(const moe_config_t& c) {
  (void)c;
  return g_tile_mode.load(std::memory_order_relaxed) == MOE_TILES_PAIR;
}

cudaError_t launch_tc_gate_up(const moe_config_t& c, const void* x_perm, const int32_t* offsets,
                              const void* wg, const void* wu, void* h, cudaStream_t s, const Ctx& ctx, void* g_save,
                              void* u_save) {
  const int64_t rows = slot_rows(c);
  if (rows == 0) return cudaSuccess;
  CUtensorMap ta, tg, tu;
  const uint64_t a_dims[2] = {(uint64_t)c.d, (uint64_t)rows};
  const uint64_t a_str[1] = {(uint64_t)c.d * 2};
  const uint32_t a_box[2] = {64, 128};
  const uint64_t w_dims[3] = {(uint64_t)c.f, (uint64_t)c.d, (uint64_t)c.E};
  const uint64_t w_str[2] = {(uint64_t)c.f * 2, (uint64_t)c.d * c.f * 2};
  const uint32_t w_box[3] = {64, 64, 1};
  if (!encode_tmap(&ta, x_perm, 2, a_dims, a_str, a_box, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap(&tg, wg, 3, w_dims, w_str, w_box, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap(&tu, wu, 3, w_dims, w_str, w_box, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  TcArgs args;
  args.offsets = offsets;
  args.rows_alloc = rows;
  args.n_tiles = (int)(c.f / Cfg<kGateUp, 256>::BN_OUT);
  args.num_kb = (int)(c.d / BK);
  args.out = h;
  args.ld_out = c.f;
  args.row_scale = nullptr;
  args.perm = nullptr;
  args.n_tok = c.T;
  args.save_g = g_save;
  args.save_u = u_save;
  args.err = ctx.err;
  if (use_pair_tiles(c)) return launch_pair<kGateUp, false>(ta, tg, tu, args, s, ctx);
  return launch_grouped<kGateUp, 256>(ta, tg, tu, args, s, ctx);
}

cudaError_t launch_tc_down(const moe_config_t& c, const void* h, const int32_t* offsets, const void* wd,
                           const float* row_scale, float* y, cudaStream_t s, const Ctx& ctx) {
  const int64_t rows = slot_rows(c);
  if (rows == 0) return cudaSuccess;
  CUtensorMap ta, tw;
  const uint64_t a_dims[2] = {(uint64_t)c.f, (uint64_t)rows};
  const uint64_t a_str[1] = {(uint64_t)c.f * 2};
  const uint32_t a_box[2] = {64, 128};
  const uint64_t w_dims[3] = {(uint64_t)c.d, (uint64_t)c.f, (uint64_t)c.E};
  const uint64_t w_str[2] = {(uint64_t)c.d * 2, (uint64_t)c.f * c.d * 2};
  const uint32_t w_box[3] = {64, 64, 1};
  if (!encode_tmap(&ta, h, 2, a_dims, a_str, a_box, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap(&tw, wd, 3, w_dims, w_str, w_box, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  TcArgs args;
  args.offsets = offsets;
  args.rows_alloc = rows;
  args.num_kb = (int)(c.f / BK);
  args.out = y;
  args.ld_out = c.d;
  args.row_scale = row_scale;
  args.perm = nullptr;
  args.n_tok = c.T;
  args.save_g = nullptr;
  args.save_u = nullptr;
  args.err = ctx.err;
  if (c.d % 256 == 0) {
    args.n_tiles = (int)(c.d / 256);
    if (use_pair_tiles(c)) return launch_pair<kDown, false>(ta, tw, tw, args, s, ctx);
    return launch_grouped<kDown, 256>(ta, tw, tw, args, s, ctx);
  }
  args.n_tiles = (int)(c.d / 128);
  return launch_grouped<kDown, 128>(ta, tw, tw, args, s, ctx);
}

cudaError_t launch_tc_down_scatter(const moe_config_t& c, const void* h, const int32_t* offsets, const void* wd,
                                   const float* row_scale, const int32_t* perm, float* out32, cudaStream_t s,
                                   const Ctx& ctx, int n_peers, float* const* peer_out, int64_t peer_tokens) {
  const int64_t rows = slot_rows(c);
  if (rows == 0) return cudaSuccess;
  if (c.d % 256 != 0) return cudaErrorInvalidValue;
  CUtensorMap ta, tw;
  const uint64_t a_dims[2] = {(uint64_t)c.f, (uint64_t)rows};
  const uint64_t a_str[1] = {(uint64_t)c.f * 2};
  const uint32_t a_box[2] = {64, 128};
  const uint64_t w_dims[3] = {(uint64_t)c.d, (uint64_t)c.f, (uint64_t)c.E};
  const uint64_t w_str[2] = {(uint64_t)c.d * 2, (uint64_t)c.f * c.d * 2};
  const uint32_t w_box[3] = {64, 64, 1};
  if (!encode_tmap(&ta, h, 2, a_dims, a_str, a_box, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap(&tw, wd, 3, w_dims, w_str, w_box, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  TcArgs args;
  args.offsets = offsets;
  args.rows_alloc = rows;
  args.num_kb = (int)(c.f / BK);
  args.out = out32;
  args.ld_out = c.d;
  args.row_scale = row_scale;
  args.perm = perm;
  args.n_tok = c.T;
  args.save_g = nullptr;
  args.save_u = nullptr;
  args.err = ctx.err;
  args.n_tiles = (int)(c.d / 256);
  if (n_peers > 0) {
    if (n_peers > MOE_EP_MAX_WORLD || !peer_out || peer_tokens <= 0) return cudaErrorInvalidValue;
    args.n_peers = n_peers;
    args.n_tok = peer_tokens;
    for (int p = 0; p < n_peers; ++p) args.peer_out[p] = peer_out[p];
  }
  if (use_pair_tiles(c)) return launch_pair<kDown, true>(ta, tw, tw, args, s, ctx);
  return launch_grouped<kDown, 256, true>(ta, tw, tw, args, s, ctx);
}

}  // namespace moe
