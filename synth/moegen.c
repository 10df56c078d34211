/*
 * moegen.c - seeded synthetic inputs for the routed 2-bit MoE FFN layer.
 *
 * This file draws random numbers and lays them into the input planes. It holds
 * none of the layer's arithmetic: no dequantisation, no routing, no FFN. Both
 * the CPU oracle and the CUDA library are fed from the buffers it fills.
 *
 * Random source: splitmix64 (G. Steele, D. Lea, C. Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014). A stream with seed s yields
 * x_i = mix(s + (i+1) * 0x9E3779B97F4A7C15), i = 0, 1, 2, ... which is the
 * generator's own next() sequence written in counter form, so any element can
 * be produced independently (the loops below are split across threads).
 *
 * Recipes (one stream per tensor, seed = moegen_seed(cfg, layer, tensor, expert)):
 *   bytes             uniform: byte j = byte (j mod 8) of x_{j/8}, little-endian
 *   uniform double    u = (x >> 11) * 2^-53
 *   normal            Box-Muller on (x_{2i}, x_{2i+1}) in double
 *   bf16 / fp16       round-to-nearest-even from the double (via fp32 for bf16)
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define GOLDEN_GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t sm_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

static inline uint64_t sm_at(uint64_t seed, uint64_t i) {
  return sm_mix(seed + (i + 1) * GOLDEN_GAMMA);
}

uint64_t moegen_splitmix64_at(uint64_t seed, uint64_t i) { return sm_at(seed, i); }

/* Stream seed for one tensor of one layer of one configuration. */
uint64_t moegen_seed(uint64_t cfg_seed, uint32_t layer, uint32_t tensor, uint32_t expert) {
  uint64_t s = sm_mix(cfg_seed ^ 0x6D6F6567656E3031ULL);
  s = sm_mix(s + (uint64_t)layer * GOLDEN_GAMMA);
  s = sm_mix(s + ((uint64_t)tensor << 32 | (uint64_t)expert));
  return s;
}

static inline double u01(uint64_t x) { return (double)(x >> 11) * (1.0 / 9007199254740992.0); }

/* fp32 -> bf16, round to nearest even (inputs here are finite). */
static inline uint16_t f32_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  uint32_t r = u + 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(r >> 16);
}

/* double -> fp16, round to nearest even, normal and subnormal range, saturating
 * to inf above 65504 (never reached by the recipes). */
static uint16_t f64_to_f16(double v) {
  uint16_t sign = 0;
  if (v < 0) { sign = 0x8000; v = -v; }
  if (v == 0) return sign;
  if (v >= 65520.0) return sign | 0x7C00;
  int e;
  double m = frexp(v, &e); /* v = m * 2^e, m in [0.5, 1) */
  int exp16 = e - 1 + 15;  /* biased exponent for 1.f form */
  if (exp16 >= 1) {
    /* normal: 10 fraction bits */
    double scaled = ldexp(m, 11); /* in [1024, 2048) */
    double fl = floor(scaled);
    double rem = scaled - fl;
    uint32_t mant = (uint32_t)fl;
    if (rem > 0.5 || (rem == 0.5 && (mant & 1u))) mant++;
    if (mant == 2048) { mant = 1024; exp16++; }
    if (exp16 >= 31) return sign | 0x7C00;
    return sign | (uint16_t)(exp16 << 10) | (uint16_t)(mant - 1024);
  }
  /* subnormal: value = mant * 2^-24 */
  double scaled = ldexp(v, 24);
  double fl = floor(scaled);
  double rem = scaled - fl;
  uint32_t mant = (uint32_t)fl;
  if (rem > 0.5 || (rem == 0.5 && (mant & 1u))) mant++;
  return sign | (uint16_t)mant; /* mant == 1024 rolls into the smallest normal */
}

void moegen_bytes(uint64_t seed, uint8_t* out, int64_t n) {
  int64_t nw = n / 8;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < nw; ++i) {
    uint64_t x = sm_at(seed, (uint64_t)i);
    memcpy(out + 8 * i, &x, 8); /* little-endian host */
  }
  if (n % 8) {
    uint64_t x = sm_at(seed, (uint64_t)nw);
    for (int64_t j = 0; j < n % 8; ++j) out[8 * nw + j] = (uint8_t)(x >> (8 * j));
  }
}

static inline void box_muller(uint64_t seed, int64_t pair, double* z0, double* z1) {
  double u1 = u01(sm_at(seed, 2 * (uint64_t)pair));
  double u2 = u01(sm_at(seed, 2 * (uint64_t)pair + 1));
  double r = sqrt(-2.0 * log(1.0 - u1));
  double th = 6.283185307179586476925286766559 * u2;
  *z0 = r * cos(th);
  *z1 = r * sin(th);
}

void moegen_normal_f32(uint64_t seed, float* out, int64_t n, double stddev) {
  int64_t np = (n + 1) / 2;
#pragma omp parallel for schedule(static)
  for (int64_t p = 0; p < np; ++p) {
    double z0, z1;
    box_muller(seed, p, &z0, &z1);
    out[2 * p] = (float)(z0 * stddev);
    if (2 * p + 1 < n) out[2 * p + 1] = (float)(z1 * stddev);
  }
}

void moegen_normal_bf16(uint64_t seed, uint16_t* out, int64_t n, double stddev) {
  int64_t np = (n + 1) / 2;
#pragma omp parallel for schedule(static)
  for (int64_t p = 0; p < np; ++p) {
    double z0, z1;
    box_muller(seed, p, &z0, &z1);
    out[2 * p] = f32_to_bf16((float)(z0 * stddev));
    if (2 * p + 1 < n) out[2 * p + 1] = f32_to_bf16((float)(z1 * stddev));
  }
}

/* fp16 scales: out[i] = fp16((0.75 + 0.5 u_i) * base). */
void moegen_f16_scale(uint64_t seed, uint16_t* out, int64_t n, double base) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = f64_to_f16((0.75 + 0.5 * u01(sm_at(seed, (uint64_t)i))) * base);
}

/* Q2K-style scale pair plane: low half fp16 d = (0.75 + 0.5 u) * base,
 * high half fp16 dmin = fp16(1.5 * d). */
void moegen_q2k_dd(uint64_t seed, uint32_t* out, int64_t n, double base) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    uint16_t d = f64_to_f16((0.75 + 0.5 * u01(sm_at(seed, (uint64_t)i))) * base);
    /* decode d exactly to double: fp16 -> value */
    int ex = (d >> 10) & 31, mant = d & 1023;
    double dv = ex ? ldexp(1024 + mant, ex - 25) : ldexp(mant, -24);
    uint16_t dm = f64_to_f16(1.5 * dv);
    out[i] = (uint32_t)d | ((uint32_t)dm << 16);
  }
}

/* Uniform random permutation of 0..n-1 (Fisher-Yates, draw i uses x_i). */
void moegen_permutation(uint64_t seed, int32_t* out, int32_t n) {
  for (int32_t i = 0; i < n; ++i) out[i] = i;
  for (int32_t i = n - 1; i > 0; --i) {
    uint64_t x = sm_at(seed, (uint64_t)(n - 1 - i));
    int32_t j = (int32_t)((x >> 33) % (uint64_t)(i + 1));
    int32_t t = out[i];
    out[i] = out[j];
    out[j] = t;
  }
}

/* Zipf-style router bias: b[e] = -s * ln(rank_e), ranks 1..n from a seeded
 * random permutation. */
void moegen_zipf_bias(uint64_t seed, float* out, int32_t n, double s) {
  int32_t perm[4096];
  if (n > 4096) return;
  moegen_permutation(seed, perm, n);
  for (int32_t e = 0; e < n; ++e) out[e] = (float)(-s * log((double)(perm[e] + 1)));
}
