/*
 * Seeded synthetic inputs for the RRAttention prefill operator.
 *
 * This module only draws numbers.  It holds none of the method's arithmetic
 * (no sampling, pooling, scoring, selection or attention); both the CUDA path
 * and the fp64 oracle take their inputs from here.
 *
 * Random numbers: a counter-based generator.  Element n of stream `tid` is
 *     bits = splitmix64(splitmix64(seed ^ tid * 0xD6E8FEB86659FD93) + n)
 * (splitmix64 as published by Steele, Lea and Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014), turned into one N(0,1) value
 * by Box-Muller: u1 = (bits[63:40] + 1) / 2^24, u2 = bits[39:16] / 2^24,
 * z = sqrt(-2 ln u1) cos(2 pi u2), evaluated in double.  Every element is a
 * pure function of (seed, tid, n), so the result does not depend on the
 * number of threads.
 *
 * Streams: Q=1, K=2, V=3, u=4, w=5, z=6.
 *
 * Structures (the workloads the RRAttention pages measure on, stood in for by
 * synthetic data of the same shape):
 *   RR_GEN_IID          Q, K, V ~ N(0,1).
 *   RR_GEN_PLANTED      u = N(0, I_d) normalised to unit length (one vector,
 *                       shared by all heads).  K[j] += 3u for j in {0,1,2,3}
 *                       and for every j with j mod 1021 == 0.  Q += u at
 *                       every position and head.  V ~ N(0,1).
 *   RR_GEN_PLANTED_BAND as RR_GEN_PLANTED, plus K[j] += 0.5 w[j mod 4096],
 *                       w in R^{4096 x d} ~ N(0,1) shared by all kv heads.
 *   RR_GEN_VIDEO        frames of 256 tokens; z in R^{256 x Hkv x d} ~ N(0,1).
 *                       K[f*256+t, kv] = z[t, kv] + 0.3 N(0,1);
 *                       Q[f*256+t, h]  = z[t, h / (H/Hkv)] + 0.3 N(0,1)
 *                       (independent noise); V ~ N(0,1).
 *
 * Each value is formed in double, rounded to fp32, then rounded to bf16 with
 * round-to-nearest-even.  Output layout: [L, heads, d] row-major bf16 bits.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

enum { RR_GEN_IID = 0, RR_GEN_PLANTED = 1, RR_GEN_PLANTED_BAND = 2, RR_GEN_VIDEO = 3 };
enum { RR_ROLE_Q = 0, RR_ROLE_K = 1, RR_ROLE_V = 2 };

static inline uint64_t splitmix64(uint64_t z) {
  z += 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

static inline double normal_at(uint64_t key, uint64_t n) {
  uint64_t bits = splitmix64(key + n);
  double u1 = (double)((bits >> 40) + 1) * (1.0 / 16777216.0);
  double u2 = (double)((bits >> 16) & 0xFFFFFFull) * (1.0 / 16777216.0);
  return sqrt(-2.0 * log(u1)) * cos(6.283185307179586476925 * u2);
}

static inline uint64_t stream_key(uint64_t seed, uint64_t tid) {
  return splitmix64(seed ^ (tid * 0xD6E8FEB86659FD93ull));
}

static inline uint16_t f32_to_bf16_rne(float f) {
  union { float f; uint32_t u; } v;
  v.f = f;
  uint32_t u = v.u;
  if ((u & 0x7F800000u) == 0x7F800000u) return (uint16_t)((u >> 16) | ((u & 0xFFFFu) ? 0x40u : 0u));
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

/* One N(0,1) draw, exposed so tests can check the stream definition. */
double rr_gen_normal(uint64_t seed, uint64_t tid, uint64_t n) {
  return normal_at(stream_key(seed, tid), n);
}

/*
 * Fill one input tensor.
 *   structure: RR_GEN_*; role: RR_ROLE_Q / K / V.
 *   L: positions; H, Hkv: query / kv heads; d: head dim.
 *   out: L * (role == Q ? H : Hkv) * d bf16 values.
 * Returns 0, or -1 on bad arguments.
 */
int rr_gen_fill(int structure, uint64_t seed, int role, int64_t L, int H, int Hkv, int d,
                uint16_t* out) {
  if (!out || L <= 0 || H <= 0 || Hkv <= 0 || d <= 0 || H % Hkv) return -1;
  if (structure < RR_GEN_IID || structure > RR_GEN_VIDEO) return -1;
  if (role < RR_ROLE_Q || role > RR_ROLE_V) return -1;
  const int heads = role == RR_ROLE_Q ? H : Hkv;
  const int g = H / Hkv;
  const uint64_t tid = (uint64_t)role + 1;
  const uint64_t key = stream_key(seed, tid);

  double* u = NULL;  /* planted direction */
  double* w = NULL;  /* local band slots */
  double* z = NULL;  /* per-frame token templates */
  if (structure == RR_GEN_PLANTED || structure == RR_GEN_PLANTED_BAND) {
    u = (double*)malloc(sizeof(double) * (size_t)d);
    if (!u) return -1;
    double nrm = 0.0;
    uint64_t ku = stream_key(seed, 4);
    for (int x = 0; x < d; ++x) { u[x] = normal_at(ku, (uint64_t)x); nrm += u[x] * u[x]; }
    nrm = sqrt(nrm);
    for (int x = 0; x < d; ++x) u[x] /= nrm;
  }
  if (structure == RR_GEN_PLANTED_BAND && role == RR_ROLE_K) {
    w = (double*)malloc(sizeof(double) * 4096 * (size_t)d);
    if (!w) { free(u); return -1; }
    uint64_t kw = stream_key(seed, 5);
    for (size_t n = 0; n < 4096 * (size_t)d; ++n) w[n] = normal_at(kw, n);
  }
  if (structure == RR_GEN_VIDEO && role != RR_ROLE_V) {
    z = (double*)malloc(sizeof(double) * 256 * (size_t)Hkv * (size_t)d);
    if (!z) { free(u); free(w); return -1; }
    uint64_t kz = stream_key(seed, 6);
    for (size_t n = 0; n < 256 * (size_t)Hkv * (size_t)d; ++n) z[n] = normal_at(kz, n);
  }

#pragma omp parallel for schedule(static)
  for (int64_t p = 0; p < L; ++p) {
    for (int hh = 0; hh < heads; ++hh) {
      const size_t base = ((size_t)p * heads + hh) * (size_t)d;
      for (int x = 0; x < d; ++x) {
        double n = normal_at(key, base + (size_t)x);
        double val;
        if (structure == RR_GEN_VIDEO && role != RR_ROLE_V) {
          int kv = role == RR_ROLE_Q ? hh / g : hh;
          val = z[((size_t)(p % 256) * Hkv + kv) * d + x] + 0.3 * n;
        } else {
          val = n;
          if (u && role == RR_ROLE_Q) val += u[x];
          if (u && role == RR_ROLE_K && (p < 4 || p % 1021 == 0)) val += 3.0 * u[x];
          if (w) val += 0.5 * w[(size_t)(p % 4096) * d + x];
        }
        out[base + x] = f32_to_bf16_rne((float)val);
      }
    }
  }
  free(u);
  free(w);
  free(z);
  return 0;
}
