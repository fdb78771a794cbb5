/*
 * Seeded synthetic inputs for the MoE layer: counter-based normal variates.
 *
 * This file holds no arithmetic of the MoE layer itself.  It only turns
 * (seed, tensor id, element index) into a reproducible number, so that the
 * CUDA path and the CPU oracle see bit-identical inputs.
 *
 * Generator: Philox4x32-10, as defined by Salmon, Moraes, Dror and Shaw,
 * "Parallel random numbers: as easy as 1, 2, 3" (SC'11): 10 rounds of two
 * 32x32->64 multiplies per round with multipliers 0xD2511F53 / 0xCD9E8D57 and
 * Weyl key increments 0x9E3779B9 / 0xBB67AE85.
 *
 * Element i of a tensor uses counter block m = i / 2 and takes lane i % 2 of a
 * Box-Muller pair built from two 53-bit uniforms of that block:
 *   key     = (low32(seed), low32(tensor_id))
 *   counter = (low32(m), high32(m), high32(seed), high32(tensor_id))
 *   u1 = (bits53(r0, r1) + 0.5) / 2^53,  u2 = (bits53(r2, r3) + 0.5) / 2^53
 *   z0 = sqrt(-2 ln u1) cos(2 pi u2),    z1 = sqrt(-2 ln u1) sin(2 pi u2)
 * value = mean + std * z, computed in double, then rounded once (round to
 * nearest, ties to even) to the storage type (fp32 or bf16).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define PHILOX_M0 0xD2511F53u
#define PHILOX_M1 0xCD9E8D57u
#define PHILOX_W0 0x9E3779B9u
#define PHILOX_W1 0xBB67AE85u

static inline void philox_round(uint32_t c[4], const uint32_t k[2]) {
  uint64_t p0 = (uint64_t)PHILOX_M0 * (uint64_t)c[0];
  uint64_t p1 = (uint64_t)PHILOX_M1 * (uint64_t)c[2];
  uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
  uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
  uint32_t n0 = hi1 ^ c[1] ^ k[0];
  uint32_t n2 = hi0 ^ c[3] ^ k[1];
  c[0] = n0;
  c[1] = lo1;
  c[2] = n2;
  c[3] = lo0;
}

/* Philox4x32-10 block function: out = philox(ctr, key). */
void synth_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
  uint32_t c[4] = {ctr[0], ctr[1], ctr[2], ctr[3]};
  uint32_t k[2] = {key[0], key[1]};
  for (int r = 0; r < 10; ++r) {
    philox_round(c, k);
    if (r < 9) {
      k[0] += PHILOX_W0;
      k[1] += PHILOX_W1;
    }
  }
  memcpy(out, c, sizeof(c));
}

static inline double u53(uint32_t a, uint32_t b) {
  uint64_t v = ((uint64_t)(a >> 5) << 26) | (uint64_t)(b >> 6);
  return ((double)v + 0.5) * (1.0 / 9007199254740992.0);
}

static inline void normal_pair(uint64_t seed, uint64_t tid, uint64_t m, double z[2]) {
  uint32_t key[2] = {(uint32_t)seed, (uint32_t)tid};
  uint32_t ctr[4] = {(uint32_t)m, (uint32_t)(m >> 32), (uint32_t)(seed >> 32), (uint32_t)(tid >> 32)};
  uint32_t r[4];
  synth_philox4x32_10(ctr, key, r);
  double u1 = u53(r[0], r[1]);
  double u2 = u53(r[2], r[3]);
  double rad = sqrt(-2.0 * log(u1));
  double th = 6.283185307179586476925286766559 * u2;
  z[0] = rad * cos(th);
  z[1] = rad * sin(th);
}

/* Round a finite double to bf16 (round to nearest, ties to even) and return its bits. */
static inline uint16_t bf16_rne_from_double(double v) {
  uint64_t b;
  memcpy(&b, &v, 8);
  /* keep 1 + 7 mantissa bits: drop the low 45 of the 52 stored bits */
  uint64_t lsb = (b >> 45) & 1u;
  b += ((uint64_t)1 << 44) - 1 + lsb;
  b &= ~(((uint64_t)1 << 45) - 1);
  double r;
  memcpy(&r, &b, 8);
  float f = (float)r; /* exact: r has at most 8 significant bits */
  uint32_t fb;
  memcpy(&fb, &f, 4);
  return (uint16_t)(fb >> 16);
}

typedef void (*store_fn)(void* out, uint64_t j, double v);

static void store_f64(void* out, uint64_t j, double v) { ((double*)out)[j] = v; }
static void store_f32(void* out, uint64_t j, double v) { ((float*)out)[j] = (float)v; }
static void store_bf16(void* out, uint64_t j, double v) { ((uint16_t*)out)[j] = bf16_rne_from_double(v); }

static void fill(uint64_t seed, uint64_t tid, uint64_t start, uint64_t n, double mean, double std,
                 void* out, store_fn st) {
  const uint64_t chunk = 1u << 16;
  const int64_t nchunks = (int64_t)((n + chunk - 1) / chunk);
#pragma omp parallel for schedule(static)
  for (int64_t c = 0; c < nchunks; ++c) {
    uint64_t j0 = (uint64_t)c * chunk;
    uint64_t j1 = j0 + chunk < n ? j0 + chunk : n;
    uint64_t j = j0;
    while (j < j1) {
      uint64_t i = start + j;
      double z[2];
      normal_pair(seed, tid, i >> 1, z);
      st(out, j, mean + std * z[i & 1]);
      ++j;
      if ((i & 1) == 0 && j < j1) {
        st(out, j, mean + std * z[1]);
        ++j;
      }
    }
  }
}

/* Elements [start, start+n) of tensor `tid`, as doubles (before any rounding). */
void synth_normal_f64(uint64_t seed, uint64_t tid, uint64_t start, uint64_t n, double mean, double std,
                      double* out) {
  fill(seed, tid, start, n, mean, std, out, store_f64);
}

void synth_normal_f32(uint64_t seed, uint64_t tid, uint64_t start, uint64_t n, double mean, double std,
                      float* out) {
  fill(seed, tid, start, n, mean, std, out, store_f32);
}

void synth_normal_bf16(uint64_t seed, uint64_t tid, uint64_t start, uint64_t n, double mean, double std,
                       uint16_t* out) {
  fill(seed, tid, start, n, mean, std, out, store_bf16);
}

/* Rounding helper exposed for tests of the bf16 storage rule. */
void synth_round_bf16(const double* in, uint64_t n, uint16_t* out) {
  for (uint64_t j = 0; j < n; ++j) out[j] = bf16_rne_from_double(in[j]);
}
