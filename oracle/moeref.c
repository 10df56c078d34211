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
} moeref_weights;

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
  if (((int64_t)H * I) % QK) return REF_ERR_SHAPE;
  if (T == 0) return REF_OK;
  if (!x || !topk_idx || !topk_w || !y || !W->gate_codes || !W->gate_d || !W->up_codes || !W->up_d ||
      !W->down_codes || !W->down_dd)
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
    dequant_matrix_iq2(W->gate_codes, W->gate_d, e, I, H, wg);
    dequant_matrix_iq2(W->up_codes, W->up_d, e, I, H, wu);
    dequant_matrix_q2k(W->down_codes, W->down_dd, e, H, I, wd);
    /* the assignments of expert e (and, with OpenMP, their rows) are
       independent; each dot product is the same sequential loop */
    double* hh = (double*)malloc(sizeof(double) * (size_t)na * I);
    double* xa = (double*)malloc(sizeof(double) * (size_t)na * H); /* exact widening of x_t */
    if (!hh || !xa) { free(hh); free(xa); free(mine); free(o); free(wg); free(wu); free(wd); return REF_ERR_NOMEM; }
    for (int64_t i = 0; i < na; ++i)
      for (int c = 0; c < H; ++c) xa[i * H + c] = act_in(x, x_dtype, (mine[i] / k) * H + c);
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
