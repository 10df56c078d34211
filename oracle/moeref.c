/*
 * moeref.c - CPU oracle for the routed 2-bit MoE FFN layer.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path links, loads or calls
 * this file; only the tests, the package's smoke check and the CPU-baseline leg
 * of the benchmark do. It shares no code, header, table or constant generator
 * with the CUDA library.
 *
 * What the sources fix (ds4 engine pages):
 *   - "ds4 : analyse pratique pour un usage documenté" (hysenlabs.com),
 *     section « Support de modèles et choix de quantification »: only the routed
 *     MoE experts are quantized, up/gate in IQ2_XXS and down in Q2_K; shared
 *     experts, projections and routing stay unquantized.
 *   - "antirez/ds4 - Moteur local d'inférence DeepSeek V4 Flash pour Metal"
 *     (news.hada.io), section « Poids du modèle »: the same split.
 *   - "Un modèle de 284 milliards de paramètres tourne désormais sur un Mac de
 *     128 Go. Qui y perd ?" (tiblogics.com), section « Comment un modèle de 284
 *     milliards de paramètres tient sur une seule machine »: a router picks a
 *     few experts per token; the routed experts hold most of the weights.
 * The pages name the formats but do not define them bit by bit; the layouts
 * below are this project's own specification of "IQ2_XXS-style" and
 * "Q2_K-style" blocks (256 weights per super-block, along the reduction axis).
 *
 * Arithmetic: every weight is decoded exactly (it fits fp32 exactly), every
 * dot product is accumulated in double, outputs are rounded to fp32 once.
 *
 * Parity status of each function is stated at its definition.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define QK 256
#define IQ2_BYTES 64
#define Q2K_BYTES 80

enum { REF_OK = 0, REF_ERR_ARG = 1, REF_ERR_SHAPE = 2, REF_ERR_NOMEM = 3 };
enum { REF_F32 = 0, REF_BF16 = 1 };

typedef struct {
  int32_t hidden, inter, n_experts, top_k, shared_inter;
} moeref_desc;

typedef struct {
  const uint16_t* router_w;  /* bf16 [E][H] */
  const float* router_bias;  /* [E] or NULL */
  const uint8_t* gate_codes; /* [E][I*H/256][64] */
  const uint16_t* gate_d;    /* [E][I*H/256] fp16 */
  const uint8_t* up_codes;
  const uint16_t* up_d;
  const uint8_t* down_codes; /* [E][H*I/256][80] */
  const uint32_t* down_dd;   /* [E][H*I/256] fp16 d | fp16 dmin << 16 */
  const uint16_t* sh_gate;   /* bf16 [Is][H] */
  const uint16_t* sh_up;     /* bf16 [Is][H] */
  const uint16_t* sh_down;   /* bf16 [H][Is] */
  /* second expert format: REF_FMT_MXFP4 takes the routed matrices from the
     code planes above read as MXFP4 codes [rows][K/2] with these E8M0 planes
     [rows][K/32]; the d / dd planes are then unused */
  int32_t expert_format;
  const uint8_t* gate_scales;
  const uint8_t* up_scales;
  const uint8_t* down_scales;
} moeref_weights;

enum { REF_FMT_IQ2_Q2K = 0, REF_FMT_MXFP4 = 1, REF_FMT_Q4 = 2, REF_FMT_MXFP4_A8 = 3 };
/* With REF_FMT_Q4 the three scale pointers hold fp16 d per block, [rows][K/32] uint16.
   REF_FMT_MXFP4_A8: the MXFP4 weights of REF_FMT_MXFP4, and the two routed
   contractions take their activations (x, then h) quantised to MXFP8 first
   (moeref_quant_mxfp8 below); the shared expert is unaffected. */

/* ---------------------------------------------------------------- scalars */

/* IEEE binary16 -> double, exact (normal, subnormal, zero; inf/nan as such). */
double moeref_f16_to_f64(uint16_t h) {
  int s = h >> 15, e = (h >> 10) & 31, m = h & 1023;
  double v;
  if (e == 0) v = ldexp((double)m, -24);
  else if (e == 31) v = m ? NAN : INFINITY;
  else v = ldexp((double)(1024 + m), e - 25);
  return s ? -v : v;
}

/* bfloat16 -> double, exact: the top half of an IEEE binary32. */
double moeref_bf16_to_f64(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

static double act_in(const void* x, int dtype, int64_t i) {
  return dtype == REF_F32 ? (double)((const float*)x)[i] : moeref_bf16_to_f64(((const uint16_t*)x)[i]);
}

/* ----------------------------------------------------------------- grid D2
 * Codebook of the IQ2-style format: 256 rows of 8 magnitudes in {8, 25, 43}.
 * Specification (this project's): splitmix64 (Steele, Lea, Flood, OOPSLA 2014)
 * with seed 0x4951325F47524944; draw c = (next() >> 32) mod 6561; keep c if not
 * drawn before; stop at 256 rows, in acceptance order. Element e of a row is the
 * base-3 digit e of c (least significant first) mapped 0->8, 1->25, 2->43.
 * Pinned by: splitmix64's published first output, invariants, a regression hash. */
uint64_t moeref_splitmix64_next(uint64_t* state) {
  uint64_t z = (*state += 0x9E3779B97F4A7C15ULL);
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

void moeref_grid(uint8_t out[256 * 8]) {
  static const uint8_t level[3] = {8, 25, 43};
  uint64_t st = 0x4951325F47524944ULL;
  uint32_t rows[256];
  int n = 0;
  while (n < 256) {
    uint32_t c = (uint32_t)((moeref_splitmix64_next(&st) >> 32) % 6561u);
    int dup = 0;
    for (int i = 0; i < n; ++i) dup |= rows[i] == c;
    if (!dup) rows[n++] = c;
  }
  for (int r = 0; r < 256; ++r) {
    uint32_t c = rows[r];
    for (int e = 0; e < 8; ++e) {
      out[r * 8 + e] = level[c % 3];
      c /= 3;
    }
  }
}

/* ------------------------------------------------------- block formats D1/D3
 * IQ2-style block (256 weights, 64 code bytes + one fp16 d in its own plane).
 * Sub-block s (0..7) is bytes 8s..8s+7 and covers weights 32s..32s+31 as four
 * groups j of 8. Bytes 8s+j (j=0..3) hold the grid row index of group j. Bytes
 * 8s+4..8s+7 form a little-endian u32 v: bits 7j..7j+6 are the sign field
 * sigma_j of group j (bit e set => element e negative, e = 0..6), bits 28..31
 * the 4-bit scale ls. Element 7 is negative iff popcount(sigma_j) is odd, so a
 * group always has an even number of negatives. Value:
 *     w[32s + 8j + e] = d * (2 ls + 1) * grid[idx_j][e] * sign_e / 8.
 * Parity: pinned by hand-worked blocks, invariants and exhaustive checks. */
void moeref_dequant_iq2(const uint8_t* codes, const uint16_t* d, int64_t nblocks, float* out) {
  uint8_t grid[256 * 8];
  moeref_grid(grid);
  /* blocks are independent */
#pragma omp parallel for schedule(static)
  for (int64_t b = 0; b < nblocks; ++b) {
    const uint8_t* q = codes + b * IQ2_BYTES;
    double db = moeref_f16_to_f64(d[b]);
    for (int s = 0; s < 8; ++s) {
      uint32_t v = (uint32_t)q[8 * s + 4] | (uint32_t)q[8 * s + 5] << 8 | (uint32_t)q[8 * s + 6] << 16 |
                   (uint32_t)q[8 * s + 7] << 24;
      int ls = (int)(v >> 28);
      for (int j = 0; j < 4; ++j) {
        int idx = q[8 * s + j];
        uint32_t sigma = (v >> (7 * j)) & 127u;
        int neg_count = 0;
        for (int e = 0; e < 7; ++e) neg_count += (sigma >> e) & 1u;
        for (int e = 0; e < 8; ++e) {
          int neg = e < 7 ? (int)((sigma >> e) & 1u) : (neg_count & 1);
          double w = db * (double)(2 * ls + 1) * (double)grid[idx * 8 + e] / 8.0;
          out[b * QK + 32 * s + 8 * j + e] = (float)(neg ? -w : w);
        }
      }
    }
  }
}

/* Q2K-style block (256 weights, 80 code bytes + one u32 d|dmin in its plane).
 * Bytes 0..15: sub-block s (weights 16s..16s+15) scale byte, sc = low nibble,
 * m = high nibble. Bytes 16..79: byte 16+i holds weights 4i..4i+3, weight 4i+r
 * in bits 2r..2r+1 (q in 0..3). Plane word: fp16 d in bits 0..15, fp16 dmin in
 * bits 16..31. Value: w = d * sc * q - dmin * m. Both products are exact in
 * double and the difference is exact in double; the cast to fp32 is the only
 * rounding. Parity: pinned by hand-worked blocks and exhaustive checks. */
void moeref_dequant_q2k(const uint8_t* codes, const uint32_t* dd, int64_t nblocks, float* out) {
  /* blocks are independent */
#pragma omp parallel for schedule(static)
  for (int64_t b = 0; b < nblocks; ++b) {
    const uint8_t* q = codes + b * Q2K_BYTES;
    double dv = moeref_f16_to_f64((uint16_t)(dd[b] & 0xFFFFu));
    double dm = moeref_f16_to_f64((uint16_t)(dd[b] >> 16));
    for (int i = 0; i < QK; ++i) {
      int s = i / 16;
      int sc = q[s] & 15, m = q[s] >> 4;
      int qq = (q[16 + i / 4] >> (2 * (i % 4))) & 3;
      double w = dv * (double)sc * (double)qq - dm * (double)m;
      out[b * QK + i] = (float)w;
    }
  }
}

/* Dequantise expert e's [rows][K] matrix into dense floats. Blocks run over the
 * row-major flattened index of the matrix, so when K < 256 one block spans
 * 256/K consecutive rows. */
/* ------------------------------------------------------------------ MXFP4
 * OCP Microscaling Formats (MX) v1.0: an MXFP4 block is 32 FP4 E2M1 elements
 * and one E8M0 scale. E2M1: bit 3 sign, bits 2..1 exponent (bias 1), bit 0
 * mantissa; exponent 0 is subnormal (value = mantissa * 2^(1-1) * 0.5), else
 * (1 + mantissa / 2) * 2^(exponent - 1); no infinities or NaN. E8M0: the value
 * 2^(E - 127) (E = 255 is NaN and is not used here). The library's packing:
 * element 2i of a block in the low nibble of byte i, element 2i+1 in the high
 * nibble ("ds4 : analyse pratique pour un usage documenté", « Support de
 * modèles et choix de quantification », names the MXFP4 variant of the routed
 * experts; the bits are the MX specification's).
 * Parity: pinned by the specification's table of E2M1 values, E8M0 powers of
 * two, a hand-decoded block and a dense float64 FFN over independently decoded
 * weights. */
double moeref_e2m1(unsigned c) {
  const unsigned ex = (c >> 1) & 3u, man = c & 1u;
  const double mag = ex == 0 ? 0.5 * man : (1.0 + 0.5 * man) * ldexp(1.0, (int)ex - 1);
  return (c & 8u) ? -mag : mag;
}

void moeref_dequant_mxfp4(const uint8_t* codes, const uint8_t* scales, int64_t nblocks, float* out) {
  for (int64_t b = 0; b < nblocks; ++b) {
    const double sc = ldexp(1.0, (int)scales[b] - 127);
    for (int i = 0; i < 32; ++i) {
      const unsigned byte = codes[b * 16 + i / 2];
      const unsigned c = (i & 1) ? (byte >> 4) : (byte & 15u);
      out[b * 32 + i] = (float)(moeref_e2m1(c) * sc);
    }
  }
}

static void dequant_matrix_mxfp4(const uint8_t* codes, const uint8_t* scales, int e, int rows, int K, float* out) {
  const int64_t nb = (int64_t)rows * K / 32;
  moeref_dequant_mxfp4(codes + (int64_t)e * nb * 16, scales + (int64_t)e * nb, nb, out);
}

/* ------------------------------------------------------------------ MXFP8
 * Activations for a block-scaled FP4 x FP8 contraction: OCP Microscaling
 * Formats (MX) v1.0, the FP8 E4M3 element type with one E8M0 scale per block
 * of 32 (the MXFP8 format of that specification). E4M3: sign bit 7, exponent
 * bits 6..3 with bias 7, mantissa bits 2..0; exponent field 0 holds the
 * subnormals m * 2^-9; S.1111.111 is NaN and there is no infinity, so the
 * largest finite magnitude is 1.75 * 2^8 = 448.
 * Conversion of a block (the specification's rule): the shared exponent is
 * X = floor(log2(max |v_i|)) - emax, emax = 8 for E4M3 (the exponent of the
 * largest normal), clamped to the E8M0 range [-127, 127]; each element is
 * v_i / 2^X rounded to the nearest E4M3 value, ties to the even code, and
 * magnitudes beyond 448 saturate to 448 (the specification leaves overflow of
 * FP8 to the implementation; saturation is the reading taken here). A block of
 * zeros gets X = -127. The scale byte is X + 127.
 * Parity: pinned by the E4M3 value table of the specification, a library
 * float8_e4m3fn conversion on in-range values, hand-computed blocks and a
 * dense float64 MoE with an independent implementation of the block rule. */
double moeref_e4m3_decode(unsigned c) {
  const unsigned ex = (c >> 3) & 15u, man = c & 7u;
  if (ex == 15u && man == 7u) return NAN;
  const double mag = ex == 0 ? ldexp((double)man, -9) : ldexp(1.0 + man / 8.0, (int)ex - 7);
  return (c & 0x80u) ? -mag : mag;
}

/* nearest finite E4M3 code to v (ties to the even code), saturating at 448;
   a binary search over the increasing magnitudes of codes 0x00..0x7E */
unsigned moeref_e4m3_encode(double v) {
  const unsigned sign = (v < 0.0 || (v == 0.0 && signbit(v))) ? 0x80u : 0u;
  const double a = fabs(v);
  unsigned lo = 0, hi = 0x7Eu; /* invariant: value(lo) <= a (or lo = 0), answer in [lo, hi] */
  if (a >= moeref_e4m3_decode(0x7Eu)) return sign | 0x7Eu;
  while (hi - lo > 1u) {
    const unsigned mid = (lo + hi) / 2u;
    if (moeref_e4m3_decode(mid) <= a) lo = mid; else hi = mid;
  }
  /* a lies in [value(lo), value(hi)) */
  const double dl = a - moeref_e4m3_decode(lo), dh = moeref_e4m3_decode(hi) - a;
  unsigned c;
  if (dl < dh) c = lo;
  else if (dh < dl) c = hi;
  else c = (lo & 1u) ? hi : lo;
  return sign | c;
}

/* n blocks of 32 values -> E4M3 codes [n][32] and E8M0 scale bytes [n] */
void moeref_quant_mxfp8(const double* v, int64_t nblocks, uint8_t* elem, uint8_t* scale) {
  for (int64_t b = 0; b < nblocks; ++b) {
    double amax = 0.0;
    for (int i = 0; i < 32; ++i) amax = fmax(amax, fabs(v[b * 32 + i]));
    int X = -127;
    if (amax > 0.0) {
      int e2;
      frexp(amax, &e2); /* amax = f * 2^e2, f in [0.5, 1): floor(log2 amax) = e2 - 1 */
      X = (e2 - 1) - 8;
      if (X < -127) X = -127;
      if (X > 127) X = 127;
    }
    scale[b] = (uint8_t)(X + 127);
    for (int i = 0; i < 32; ++i) elem[b * 32 + i] = (uint8_t)moeref_e4m3_encode(ldexp(v[b * 32 + i], -X));
  }
}

/* the values an MXFP8 block represents: element * 2^(scale - 127), in place */
static void mxfp8_round_trip(double* v, int64_t nblocks) {
  uint8_t el[32], sc;
  for (int64_t b = 0; b < nblocks; ++b) {
    moeref_quant_mxfp8(v + b * 32, 1, el, &sc);
    for (int i = 0; i < 32; ++i) v[b * 32 + i] = ldexp(moeref_e4m3_decode(el[i]), (int)sc - 127);
  }
}

/* -------------------------------------------------------------------- Q4
 * The 4-bit routed-expert variant the pages mention ("Un modèle de 284
 * milliards ...", « Comment un 284B tient »: Q4 models; "antirez/ds4 ...":
 * checkpoints shared between the 2-bit and 4-bit routed-expert variants) has
 * no published layout. This project's Q4-style block: 32 weights along the
 * reduction axis, one fp16 scale d and 32 unsigned 4-bit codes q (element 2i
 * in the low nibble of code byte i, 2i+1 in the high nibble):
 * w = d * (q - 8), exact in fp32.
 * Parity: pinned by a hand-decoded block, the affine law in q and the scaling
 * law in d, and a dense float64 MoE over the decoded weights. */
void moeref_dequant_q4(const uint8_t* codes, const uint16_t* d, int64_t nblocks, float* out) {
  for (int64_t b = 0; b < nblocks; ++b) {
    const double s = moeref_f16_to_f64(d[b]);
    for (int i = 0; i < 32; ++i) {
      const unsigned byte = codes[b * 16 + i / 2];
      const int q = (int)((i & 1) ? (byte >> 4) : (byte & 15u));
      out[b * 32 + i] = (float)(s * (double)(q - 8));
    }
  }
}

static void dequant_matrix_q4(const uint8_t* codes, const uint16_t* d, int e, int rows, int K, float* out) {
  const int64_t nb = (int64_t)rows * K / 32;
  moeref_dequant_q4(codes + (int64_t)e * nb * 16, d + (int64_t)e * nb, nb, out);
}

static void dequant_matrix_iq2(const uint8_t* codes, const uint16_t* d, int e, int rows, int K, float* out) {
  int64_t nb = (int64_t)rows * K / QK;
  moeref_dequant_iq2(codes + (int64_t)e * nb * IQ2_BYTES, d + (int64_t)e * nb, nb, out);
}
static void dequant_matrix_q2k(const uint8_t* codes, const uint32_t* dd, int e, int rows, int K, float* out) {
  int64_t nb = (int64_t)rows * K / QK;
  moeref_dequant_q2k(codes + (int64_t)e * nb * Q2K_BYTES, dd + (int64_t)e * nb, nb, out);
}

/* ------------------------------------------------------------------ router
 * Router (unquantized, per the quantization section cited above): logits
 * l[t][e] = sum_h x[t][h] * Wr[e][h] (+ bias[e]), in double from the exact
 * inputs. Top-k: the k largest logits, slots in descending order, ties to the
 * lower expert index. Weights: softmax over all experts renormalised over the
 * chosen k, which equals exp(l_j - l_max) / sum over the chosen of exp(l_i -
 * l_max) because the full denominator cancels.
 * Parity: pinned by brute-force sort, k = E plain softmax, sum-to-one. */
int moeref_route(int H, int E, int k, const uint16_t* router_w, const float* router_bias, const void* x,
                 int x_dtype, int T, int32_t* topk_idx, float* topk_w, double* logits_out) {
  if (H <= 0 || E <= 0 || k <= 0 || k > E || T < 0 || !router_w || (T && (!x || !topk_idx || !topk_w)))
    return REF_ERR_ARG;
  int rc = REF_OK;
  /* tokens are independent; with OpenMP they are spread over threads (the
     arithmetic of each token is the same sequential loop either way) */
#pragma omp parallel for schedule(dynamic, 1)
  for (int t = 0; t < T; ++t) {
    double* l = (double*)malloc(sizeof(double) * (size_t)E);
    char* taken = (char*)malloc((size_t)E);
    double* lw = (double*)malloc(sizeof(double) * (size_t)k);
    if (!l || !taken || !lw) {
      free(l); free(taken); free(lw);
#pragma omp critical
      rc = REF_ERR_NOMEM;
      continue;
    }
    for (int e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int h = 0; h < H; ++h)
        acc += act_in(x, x_dtype, (int64_t)t * H + h) * moeref_bf16_to_f64(router_w[(int64_t)e * H + h]);
      if (router_bias) acc += (double)router_bias[e];
      l[e] = acc;
      taken[e] = 0;
      if (logits_out) logits_out[(int64_t)t * E + e] = acc;
    }
    for (int j = 0; j < k; ++j) {
      int best = -1;
      for (int e = 0; e < E; ++e)
        if (!taken[e] && (best < 0 || l[e] > l[best])) best = e;
      taken[best] = 1;
      topk_idx[(int64_t)t * k + j] = best;
      lw[j] = l[best];
    }
    double z = 0.0;
    for (int j = 0; j < k; ++j) z += exp(lw[j] - lw[0]);
    for (int j = 0; j < k; ++j) topk_w[(int64_t)t * k + j] = (float)(exp(lw[j] - lw[0]) / z);
    free(l);
    free(taken);
    free(lw);
  }
  return rc;
}

/* ------------------------------------------------------------- permutation
 * Assignment a = t*k + j. counts[e] = #{a : idx[a] == e}; offsets = exclusive
 * prefix sum (offsets[E] = T*k); perm[offsets[e] + r] = the r-th smallest a with
 * idx[a] == e (stable); inv[perm[p]] = p.
 * Parity: pinned by a library stable sort on (idx[a], a) and invariants. */
int moeref_permute(int T, int k, int E, const int32_t* topk_idx, int32_t* offsets, int32_t* perm, int32_t* inv) {
  if (T < 0 || k <= 0 || E <= 0 || !offsets || (T && (!topk_idx || !perm || !inv))) return REF_ERR_ARG;
  int64_t n = (int64_t)T * k;
  for (int e = 0; e <= E; ++e) offsets[e] = 0;
  for (int64_t a = 0; a < n; ++a) {
    int e = topk_idx[a];
    if (e < 0 || e >= E) return REF_ERR_ARG;
    offsets[e + 1]++;
  }
  for (int e = 0; e < E; ++e) offsets[e + 1] += offsets[e];
  int32_t* fill = (int32_t*)calloc((size_t)E, sizeof(int32_t));
  if (!fill) return REF_ERR_NOMEM;
  for (int64_t a = 0; a < n; ++a) {
    int e = topk_idx[a];
    int32_t p = offsets[e] + fill[e]++;
    perm[p] = (int32_t)a;
    inv[a] = p;
  }
  free(fill);
  return REF_OK;
}

/* -------------------------------------------------------------- expert FFN
 * For each assignment (t, j) with expert e = idx[t][j]:
 *   g = Wg_e x_t, u = Wu_e x_t         (Wg, Wu: [I][H], IQ2-style)
 *   h = silu(g) * u, silu(z) = z / (1 + exp(-z))   (no clamp)
 *   o = Wd_e h                          (Wd: [H][I], Q2K-style)
 * Shared expert (bf16, weight 1, no gate; I_s = 0 means none):
 *   s = Wsd (silu(Wsg x_t) * (Wsu x_t))
 * Combine: y[t] = sum_j w[t][j] o_{t,j} (j ascending) + s[t] (+ residual[t]).
 * All in double, y rounded to fp32 once.
 * Parity: pinned by a dense float64 MoE loop over library matmuls, the E=k=1
 * dense case, d=dmin=0, x=0 and relabelling/permutation invariance. */
static double silu(double z) { return z / (1.0 + exp(-z)); }

int moeref_expert_ffn(const moeref_desc* desc, const moeref_weights* W, const void* x, int x_dtype, int T,
                      const int32_t* topk_idx, const float* topk_w, const float* residual, float* y) {
  if (!desc || !W || T < 0) return REF_ERR_ARG;
  const int H = desc->hidden, I = desc->inter, E = desc->n_experts, k = desc->top_k, Is = desc->shared_inter;
  if (H <= 0 || I <= 0 || E <= 0 || k <= 0 || k > E || Is < 0) return REF_ERR_ARG;
  const int q4 = W->expert_format == REF_FMT_Q4;
  const int a8 = W->expert_format == REF_FMT_MXFP4_A8;
  const int mx = W->expert_format == REF_FMT_MXFP4 || q4 || a8; /* block-32 formats with scale planes */
  if (W->expert_format != REF_FMT_IQ2_Q2K && !mx) return REF_ERR_ARG;
  if (((int64_t)H * I) % QK || (mx && (H % 32 || I % 32))) return REF_ERR_SHAPE;
  if (T == 0) return REF_OK;
  if (!x || !topk_idx || !topk_w || !y || !W->gate_codes || !W->up_codes || !W->down_codes)
    return REF_ERR_ARG;
  if (mx ? (!W->gate_scales || !W->up_scales || !W->down_scales) : (!W->gate_d || !W->up_d || !W->down_dd))
    return REF_ERR_ARG;
  if (Is > 0 && (!W->sh_gate || !W->sh_up || !W->sh_down)) return REF_ERR_ARG;

  const int64_t nA = (int64_t)T * k;
  double* o = (double*)calloc((size_t)(nA * H), sizeof(double)); /* per assignment */
  float* wg = (float*)malloc(sizeof(float) * (size_t)I * H);
  float* wu = (float*)malloc(sizeof(float) * (size_t)I * H);
  float* wd = (float*)malloc(sizeof(float) * (size_t)H * I);
  if (!o || !wg || !wu || !wd) { free(o); free(wg); free(wu); free(wd); return REF_ERR_NOMEM; }

  int64_t* mine = (int64_t*)malloc(sizeof(int64_t) * (size_t)(nA > 0 ? nA : 1));
  if (!mine) { free(o); free(wg); free(wu); free(wd); return REF_ERR_NOMEM; }
  for (int e = 0; e < E; ++e) {
    int64_t na = 0;
    for (int64_t a = 0; a < nA; ++a)
      if (topk_idx[a] == e) mine[na++] = a;
    if (!na) continue;
    if (q4) {
      dequant_matrix_q4(W->gate_codes, (const uint16_t*)W->gate_scales, e, I, H, wg);
      dequant_matrix_q4(W->up_codes, (const uint16_t*)W->up_scales, e, I, H, wu);
      dequant_matrix_q4(W->down_codes, (const uint16_t*)W->down_scales, e, H, I, wd);
    } else if (mx) {
      dequant_matrix_mxfp4(W->gate_codes, W->gate_scales, e, I, H, wg);
      dequant_matrix_mxfp4(W->up_codes, W->up_scales, e, I, H, wu);
      dequant_matrix_mxfp4(W->down_codes, W->down_scales, e, H, I, wd);
    } else {
      dequant_matrix_iq2(W->gate_codes, W->gate_d, e, I, H, wg);
      dequant_matrix_iq2(W->up_codes, W->up_d, e, I, H, wu);
      dequant_matrix_q2k(W->down_codes, W->down_dd, e, H, I, wd);
    }
    /* the assignments of expert e (and, with OpenMP, their rows) are
       independent; each dot product is the same sequential loop */
    double* hh = (double*)malloc(sizeof(double) * (size_t)na * I);
    double* xa = (double*)malloc(sizeof(double) * (size_t)na * H); /* exact widening of x_t */
    if (!hh || !xa) { free(hh); free(xa); free(mine); free(o); free(wg); free(wu); free(wd); return REF_ERR_NOMEM; }
    for (int64_t i = 0; i < na; ++i)
      for (int c = 0; c < H; ++c) xa[i * H + c] = act_in(x, x_dtype, (mine[i] / k) * H + c);
    if (a8) mxfp8_round_trip(xa, na * H / 32); /* rows of H, blocks of 32 along H */
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t i = 0; i < na; ++i)
      for (int r = 0; r < I; ++r) {
        double g = 0.0, u = 0.0;
        for (int c = 0; c < H; ++c) {
          double xv = xa[i * H + c];
          g += (double)wg[(int64_t)r * H + c] * xv;
          u += (double)wu[(int64_t)r * H + c] * xv;
        }
        hh[i * I + r] = silu(g) * u;
      }
    if (a8) mxfp8_round_trip(hh, na * I / 32); /* rows of I, blocks of 32 along I */
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t i = 0; i < na; ++i)
      for (int r = 0; r < H; ++r) {
        double acc = 0.0;
        for (int c = 0; c < I; ++c) acc += (double)wd[(int64_t)r * I + c] * hh[i * I + c];
        o[mine[i] * H + r] = acc;
      }
    free(hh);
    free(xa);
  }
  free(mine);
  free(wg);
  free(wu);
  free(wd);

  int rc = REF_OK;
  /* tokens are independent (shared expert and combine) */
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t t = 0; t < T; ++t) {
    double* hs = (double*)malloc(sizeof(double) * (size_t)(Is > 0 ? Is : 1));
    double* s = (double*)malloc(sizeof(double) * (size_t)H);
    double* xt = (double*)malloc(sizeof(double) * (size_t)H); /* exact widening of x_t */
    if (!hs || !s || !xt) {
      free(hs); free(s); free(xt);
#pragma omp critical
      rc = REF_ERR_NOMEM;
      continue;
    }
    for (int r = 0; r < H; ++r) s[r] = 0.0;
    for (int c = 0; c < H; ++c) xt[c] = act_in(x, x_dtype, t * H + c);
    if (Is > 0) {
      for (int r = 0; r < Is; ++r) {
        double g = 0.0, u = 0.0;
        for (int c = 0; c < H; ++c) {
          double xv = xt[c];
          g += moeref_bf16_to_f64(W->sh_gate[(int64_t)r * H + c]) * xv;
          u += moeref_bf16_to_f64(W->sh_up[(int64_t)r * H + c]) * xv;
        }
        hs[r] = silu(g) * u;
      }
      for (int r = 0; r < H; ++r) {
        double acc = 0.0;
        for (int c = 0; c < Is; ++c) acc += moeref_bf16_to_f64(W->sh_down[(int64_t)r * Is + c]) * hs[c];
        s[r] = acc;
      }
    }
    for (int r = 0; r < H; ++r) {
      double acc = 0.0;
      for (int j = 0; j < k; ++j) acc += (double)topk_w[t * k + j] * o[(t * k + j) * H + r];
      acc += s[r];
      if (residual) acc += (double)residual[t * H + r];
      y[t * H + r] = (float)acc;
    }
    free(hs);
    free(s);
    free(xt);
  }
  free(o);
  return rc;
}

/* ------------------------------------------------------------ whole layer
 * route, then the expert FFN with the router's fp32 weights. */
int moeref_layer_forward(const moeref_desc* desc, const moeref_weights* W, const void* x, int x_dtype, int T,
                         const float* residual, float* y, int32_t* topk_idx, float* topk_w) {
  if (!desc || !W) return REF_ERR_ARG;
  if (T == 0) return REF_OK;
  int rc = moeref_route(desc->hidden, desc->n_experts, desc->top_k, W->router_w, W->router_bias, x, x_dtype, T,
                        topk_idx, topk_w, NULL);
  if (rc) return rc;
  return moeref_expert_ffn(desc, W, x, x_dtype, T, topk_idx, topk_w, residual, y);
}

/* ------------------------------------------------------------- quantisers
 * Float weights -> the two block formats, without an importance matrix. The
 * pages say the routed experts are quantized (IQ2_XXS for up/gate, Q2_K for
 * down) and that the project's own 2-bit files were made with an imatrix
 * ("ds4 : un MoE de 284 milliards sur un Mac de 128 Go", « Comment un 284B
 * tient »); they give no algorithm. These are this project's plain rules:
 * round-to-nearest for Q2K and an exhaustive codebook search for IQ2. Every
 * decision (a scale byte, a code, a codebook row) is taken in fp32 with the
 * operations below in the order written, each rounded to nearest even and
 * none fused, so that another implementation can reproduce the codes bit for
 * bit. Parity: pinned by hand-worked blocks, reconstruction bounds and a
 * brute-force optimality check of the IQ2 search. */

/* fp32 -> IEEE binary16, round to nearest even; finite inputs below 65520. */
uint16_t moeref_f32_to_f16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
  uint32_t a = u & 0x7FFFFFFFu;
  if (a >= 0x477FF000u) return sign | 0x7C00u; /* rounds to inf */
  if (a < 0x33000001u) return sign;             /* below half the smallest subnormal: +-0 */
  int e = (int)(a >> 23) - 127;
  uint32_t m = (a & 0x7FFFFFu) | 0x800000u;    /* 24-bit significand */
  int shift;                                    /* bits dropped from m */
  uint32_t base;
  if (e < -14) { /* subnormal half: value = m * 2^(e-23) = k * 2^-24 with k = m * 2^(e+1) */
    shift = -1 - e;
    base = 0;
  } else {
    shift = 13;
    base = (uint32_t)(e + 15) << 10;
    m &= 0x7FFFFFu; /* drop the implicit bit: the mantissa field */
  }
  uint32_t q = m >> shift, rem = m & ((1u << shift) - 1u), half = 1u << (shift - 1);
  if (rem > half || (rem == half && (q & 1u))) q += 1; /* a carry into the exponent is correct rounding */
  return (uint16_t)(sign | (base + q));
}

static float f16_to_f32(uint16_t h) { return (float)moeref_f16_to_f64(h); }

static float clampf_(float v, float lo, float hi) { return v < lo ? lo : (v > hi ? hi : v); }

/* Q2K round-to-nearest, per 256-weight block:
 *   sub-block s (16 weights): lo_s = min(0, min w), hi_s = max w,
 *     step_s = (hi_s - lo_s) / 3, off_s = -lo_s;
 *   d = fp16(max_s step_s / 15), dmin = fp16(max_s off_s / 15);
 *   sc_s = clamp(rint(step_s / d), 0, 15) (0 if d == 0),
 *   m_s = clamp(rint(off_s / dmin), 0, 15) (0 if dmin == 0);
 *   q = clamp(rint((w + dmin * m_s) / (d * sc_s)), 0, 3) (0 if d * sc_s == 0). */
void moeref_quantize_q2k(const float* w, int64_t nblocks, uint8_t* codes, uint32_t* dd) {
#pragma omp parallel for schedule(static)
  for (int64_t b = 0; b < nblocks; ++b) {
    const float* x = w + b * QK;
    uint8_t* q = codes + b * Q2K_BYTES;
    float step[16], off[16], smax = 0.f, omax = 0.f;
    for (int s = 0; s < 16; ++s) {
      float lo = 0.f, hi = x[16 * s];
      for (int i = 0; i < 16; ++i) {
        if (x[16 * s + i] < lo) lo = x[16 * s + i];
        if (x[16 * s + i] > hi) hi = x[16 * s + i];
      }
      step[s] = (hi - lo) / 3.0f;
      off[s] = -lo;
      if (step[s] > smax) smax = step[s];
      if (off[s] > omax) omax = off[s];
    }
    uint16_t d16 = moeref_f32_to_f16(smax / 15.0f), m16 = moeref_f32_to_f16(omax / 15.0f);
    float df = f16_to_f32(d16), mf = f16_to_f32(m16);
    dd[b] = (uint32_t)d16 | ((uint32_t)m16 << 16);
    memset(q, 0, Q2K_BYTES);
    for (int s = 0; s < 16; ++s) {
      int sc = df > 0.f ? (int)clampf_(rintf(step[s] / df), 0.f, 15.f) : 0;
      int m = mf > 0.f ? (int)clampf_(rintf(off[s] / mf), 0.f, 15.f) : 0;
      q[s] = (uint8_t)(sc | (m << 4));
      float st = df * (float)sc, of = mf * (float)m;
      for (int i = 0; i < 16; ++i) {
        int v = st > 0.f ? (int)clampf_(rintf((x[16 * s + i] + of) / st), 0.f, 3.f) : 0;
        int k = 16 * s + i;
        q[16 + k / 4] |= (uint8_t)(v << (2 * (k % 4)));
      }
    }
  }
}

/* IQ2 codebook search, per 256-weight block:
 *   d = fp16(max |w| * 8 / (31 * 43)) (the largest magnitude the format holds
 *   is d * 31 * 43 / 8); with d == 0 every code is 0;
 *   sub-block s (32 weights): ls = clamp(rint((max|w| * 8 / (d * 43) - 1) / 2), 0, 15),
 *   c = d * (2 ls + 1) / 8;
 *   group j (8 weights): element signs follow w (w < 0 is negative); if their
 *   count is odd, the element of smallest |w| (lowest e on ties) is flipped,
 *   since the format's eighth sign is the parity of the other seven. For every
 *   codebook row r the error sum_e (|w_e| -+ c * grid[r][e])^2 is formed in
 *   fp32 with e ascending (the flipped element takes +); the row of least error
 *   wins, the lower row on ties. */
void moeref_quantize_iq2(const float* w, int64_t nblocks, uint8_t* codes, uint16_t* d) {
  uint8_t grid[256 * 8];
  moeref_grid(grid);
#pragma omp parallel for schedule(static)
  for (int64_t b = 0; b < nblocks; ++b) {
    const float* x = w + b * QK;
    uint8_t* q = codes + b * IQ2_BYTES;
    float amax = 0.f;
    for (int i = 0; i < QK; ++i) amax = fabsf(x[i]) > amax ? fabsf(x[i]) : amax;
    uint16_t d16 = moeref_f32_to_f16(amax * 8.0f / 1333.0f);
    float df = f16_to_f32(d16);
    d[b] = d16;
    memset(q, 0, IQ2_BYTES);
    if (!(df > 0.f)) continue;
    for (int s = 0; s < 8; ++s) {
      float smax = 0.f;
      for (int i = 0; i < 32; ++i) smax = fabsf(x[32 * s + i]) > smax ? fabsf(x[32 * s + i]) : smax;
      int ls = (int)clampf_(rintf((smax * 8.0f / (df * 43.0f) - 1.0f) / 2.0f), 0.f, 15.f);
      float c = df * (float)(2 * ls + 1) / 8.0f;
      uint32_t v = (uint32_t)ls << 28;
      for (int j = 0; j < 4; ++j) {
        const float* g = x + 32 * s + 8 * j;
        int neg[8], nneg = 0, flip = -1;
        float a[8];
        for (int e = 0; e < 8; ++e) {
          a[e] = fabsf(g[e]);
          neg[e] = g[e] < 0.f;
          nneg += neg[e];
        }
        if (nneg & 1) {
          flip = 0;
          for (int e = 1; e < 8; ++e)
            if (a[e] < a[flip]) flip = e;
        }
        int best = 0;
        float best_err = 0.f;
        for (int r = 0; r < 256; ++r) {
          float err = 0.f;
          for (int e = 0; e < 8; ++e) {
            float t = c * (float)grid[r * 8 + e];
            float diff = e == flip ? a[e] + t : a[e] - t;
            err = err + diff * diff;
          }
          if (r == 0 || err < best_err) {
            best = r;
            best_err = err;
          }
        }
        q[8 * s + j] = (uint8_t)best;
        for (int e = 0; e < 7; ++e) v |= (uint32_t)(neg[e] ^ (e == flip)) << (7 * j + e);
      }
      q[8 * s + 4] = (uint8_t)(v & 0xFF);
      q[8 * s + 5] = (uint8_t)((v >> 8) & 0xFF);
      q[8 * s + 6] = (uint8_t)((v >> 16) & 0xFF);
      q[8 * s + 7] = (uint8_t)(v >> 24);
    }
  }
}
