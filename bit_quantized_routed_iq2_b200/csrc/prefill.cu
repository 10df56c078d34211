// prefill.cu - the many-token path: a grouped GEMM per routed expert on the
// 5th-generation tensor cores (tcgen05.mma kind::f16, accumulators in TMEM),
// with the 2-bit expert tiles dequantised into shared memory by dedicated
// warps, and the unquantized shared expert as a dense GEMM on the same engine.
//
// Sources: "ds4 : analyse pratique pour un usage documenté", section « Support
// de modèles et choix de quantification » (routed up/gate IQ2_XXS, down Q2_K;
// shared expert unquantized); "Un modèle de 284 milliards de paramètres tourne
// désormais sur un Mac de 128 Go. Qui y perd ?", section « Comment un modèle de
// 284 milliards de paramètres tient sur une seule machine » (each token uses a
// few routed experts). The weight formats are the library's own (see dequant.cuh).
//
// Weights are the M operand (128 rows per tile) and the tokens routed to an
// expert are the N operand (up to 128 per tile), so one dequantised weight tile
// is multiplied by all of the expert's tokens. Per CTA (one per SM, 768
// threads):
//   warps 0-3   epilogue: TMEM -> registers -> SwiGLU / scaling -> global
//   warp 4      producer: TMA loads of the token tiles (and bf16 weight tiles)
//   warp 5      TMEM allocation; one lane issues the MMAs and commits
//   warp 6      dequantising kinds: TMA loads of the code blocks (their own ring)
//   warps 8-23  dequantisers: 2-bit codes -> fp16 weight tiles (128-byte swizzle),
//               each thread one sub-block of one row per stage
// Stages of (A tiles, B tile) circulate through full/empty mbarriers; the MMA
// completion (tcgen05.commit) frees a stage. Two accumulator buffers in TMEM
// let the epilogue of one tile overlap the MMAs of the next. Every wait is
// bounded: a time-out records MOE_ERR_TIMEOUT, all roles stop, and the CTA
// drains its in-flight copies and MMAs before freeing TMEM.
//
// Precision: routed weights enter the MMA as fp16. IQ2 values are the fp16
// rounding of s * grid with s = fp16(d*(2ls+1)*2^10/8), the sign applied
// exactly afterwards, which keeps them clear of fp16
// subnormals for the scales this library's generator and real checkpoints use
// (|d| in [2^-24, 2^5]); the 2^10 is taken out in the fp32 epilogue. Q2K values
// q*d*sc - dmin*m are formed in fp32 per sub-block and rounded once to fp16.
// Routed activations enter as fp16(x * 2^-e) with one power-of-2 exponent e per
// token (largest element just below 2^13), h as fp16(h * 2^(-2e-12)), and the
// down outputs leave as fp16(o * 2^(-2e-12)) (h and o scale with x squared);
// the epilogues and the combine undo the exponents exactly, so activations of
// any magnitude stay inside the fp16 range (a chained residual stream grows
// layer by layer). The shared expert
// takes bf16 x and bf16 hi + lo parts of h.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "decode.cuh"
#include "kernels.cuh"
#include "profile.cuh"
#include "ptx.cuh"
#include "tc.cuh"

namespace moe {
namespace {

constexpr int kTcThreads = 768;
constexpr int kEpiWarps = 4;     // warps 0-3
constexpr int kProdWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kCodeWarp = 6;    // dequantising kinds: issues the code-block ring
constexpr int kDqWarp0 = 8;      // warps 8-23
constexpr int kDqWarps = 16;
constexpr int kMT = 128;         // weight rows per tile (MMA M)
constexpr int kNT = 128;         // max tokens per tile (MMA N)
constexpr int kKS = 64;          // K per stage: 128 bytes of fp16 per row
constexpr int kTile = 128 * 128; // one 128-row x 128-byte operand tile
constexpr int kTmemCols = 512;   // two accumulator buffers of (gate, up) x 128 columns
constexpr int kCStages = 3;  // code-block ring of the dequantising kinds (one entry per 256-weight block)

__device__ const Iq2Codebook d_codebook_tc = kCodebook;

// A tile source and epilogue kind.
enum TcKind : int {
  TC_IQ2_PAIR = 0,   // routed gate+up: dequantised IQ2 pair, SwiGLU, fp16 h out
  TC_Q2K = 1,        // routed down: dequantised Q2K, fp32 out
  TC_BF16_PAIR = 2,  // shared gate+up: bf16 tiles by TMA, SwiGLU, bf16 hi/lo h out
  TC_BF16 = 3,       // shared down: bf16 tiles by TMA, fp32 out
  TC_Q4_PAIR = 4,    // routed gate+up: dequantised Q4-style pair, SwiGLU, fp16 h out
  TC_Q4 = 5,         // routed down: dequantised Q4-style blocks, fp16 out
};
// Kind predicates: weights dequantised by the SMs; two weight matrices (gate and up) per tile; the routed
// gate/up epilogue (SwiGLU, fp16 h); the routed down epilogue (fp16 expert outputs).
constexpr bool tc_dq(int K) { return K == TC_IQ2_PAIR || K == TC_Q2K || K == TC_Q4_PAIR || K == TC_Q4; }
constexpr bool tc_two(int K) { return K == TC_IQ2_PAIR || K == TC_BF16_PAIR || K == TC_Q4_PAIR; }
constexpr bool tc_hout(int K) { return K == TC_IQ2_PAIR || K == TC_Q4_PAIR; }
constexpr bool tc_oout(int K) { return K == TC_Q2K || K == TC_Q4; }

struct TcPair {
  int e, p0, n, pad;  // expert (weight block), first B row, rows of B used
};

struct TcArgs {
  int n_experts;  // weight blocks (experts) the tiles may name
  int b_rows;     // rows of one B plane (bound of every tile)
  int rows_e;    // weight rows per expert
  int K;         // reduction length of one plane
  int mt;        // 128-row tiles per expert
  int planes;    // B planes summed along K (bf16 hi/lo parts), A re-read per plane
  const uint8_t* c0;
  const uint16_t* d0;
  const uint8_t* c1;
  const uint16_t* d1;
  const uint32_t* dd;
  const TcPair* pairs;     // tile list (expert, first B row, rows), or null for dense tiles
  const int32_t* npairs;
  int dense_rows;          // with pairs == null: tiles of 128 rows over this many B rows, expert 0
  const float* bias;       // TC_BF16 only: added per weight row (router bias), may be null
  const int32_t* row_exp;  // routed kinds: power-of-2 exponent e of each B row (see the epilogues)
  void* out;
  int ldo;        // output row stride in elements
  int out_rows;   // rows of one output plane (bf16 hi/lo output)
  float oscale;
  int* err;
  int clear_err;  // CTA 0 clears *err at start (first kernel of a call)
};

// Memory plan per kernel kind.
// Dequantising kinds: the fp16 weight tiles (A) go from registers into TMEM
// (tcgen05.st) and the MMA reads A from there, so shared memory carries only
// the TMA ring of token tiles (B), a ring of code blocks (the code bytes of one
// 256-weight block of the tile's rows, one TMA box per matrix and block) and
// the replicated lookup tables:
// IQ2 level selectors (8 bytes, 16 copies), IQ2 signs as fp16 +-1 pairs (16
// bytes, 8 copies), Q2K selectors (4 bytes, 32 copies); every copy serves the
// lanes of one load phase, so lookups are free of bank conflicts.
// bf16 kinds: A and B tiles both arrive by TMA into one ring of stages.
// TMEM (512 columns): A stages at columns [0, 256) for the dequantising kinds,
// accumulators above them; the bf16 kinds double-buffer the accumulators over
// all 512 columns.
template <int KIND>
struct TcLayout {
  static constexpr bool dq = tc_dq(KIND);
  static constexpr bool pair = tc_two(KIND);
  static constexpr int stages = dq ? (KIND == TC_Q4_PAIR ? 7 : 8) : (pair ? 4 : 6);  // shared-memory ring
  static constexpr size_t stage_bytes = dq ? kTile : (pair ? 3 : 2) * kTile;
  // code bytes of one 256-weight block for the tile's 128 rows: IQ2 64 bytes per row of gate and of up,
  // Q2K the whole 80-byte block, Q4-style 128 code bytes per row (of gate and of up)
  static constexpr size_t code_bytes = KIND == TC_IQ2_PAIR ? 2 * 128 * 64
                                       : KIND == TC_Q2K    ? 128 * 80
                                       : KIND == TC_Q4_PAIR ? 2 * 128 * 128
                                       : KIND == TC_Q4      ? 128 * 128
                                                            : 0;
  static constexpr size_t code_off = stages * stage_bytes;
  static constexpr size_t b_off = dq ? 0 : (pair ? 2 : 1) * kTile;      // B tile inside a stage
  static constexpr int a_stages = tc_hout(KIND) ? 4 : 8;                 // TMEM A ring (dq kinds)
  static constexpr uint32_t a_cols = pair ? 64 : 32;                     // TMEM columns per A stage
  static constexpr int acc_bufs = tc_hout(KIND) ? 1 : 2;
  static constexpr uint32_t acc_base = dq ? 256 : 0;
  static constexpr uint32_t acc_stride = tc_oout(KIND) ? 128 : 256;     // columns per accumulator buffer
  static constexpr size_t tabs = code_off + (dq ? kCStages * code_bytes : 0);
  static constexpr size_t tab_bytes =
      KIND == TC_IQ2_PAIR ? (256 * 128 + 128 * 128) : (KIND == TC_Q2K ? 256 * 128 : 0);
  static constexpr size_t bars = tabs + tab_bytes;
  static constexpr size_t total = bars + 1024;
  static_assert(total <= 227 * 1024, "shared memory plan too large");
};

// fp16 grid levels; scaled per sub-block into prmt source bytes with the low
// bytes at 0..2 and the high bytes at 3..5, so level L is the byte pair (L, 3 + L).
constexpr uint32_t kHalf8And25 = 0x4E404800u;   // fp16 pair (8, 25)
constexpr uint32_t kHalf43Twice = 0x51605160u;  // fp16 pair (43, 43)

__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity, int* err, volatile int* abort_flag) {
  if (*abort_flag) return false;
  if (mbar_wait_bounded(bar, parity, err, ERR_TIMEOUT)) return true;
  *abort_flag = 1;
  return false;
}

// The same with sleeps between polls, for waits whose latency matters little.
__device__ __forceinline__ bool tc_wait_sleepy(uint64_t* bar, uint32_t parity, int* err, volatile int* abort_flag,
                                               unsigned max_ns = 2048) {
  if (*abort_flag) return false;
  if (mbar_wait_bounded_sleepy(bar, parity, err, ERR_TIMEOUT, max_ns)) return true;
  *abort_flag = 1;
  return false;
}

// The same for all 32 lanes of a warp, with one outcome for the whole warp.
__device__ __forceinline__ bool tc_wait_warp(uint64_t* bar, uint32_t parity, int* err, volatile int* abort_flag) {
  const bool ok = tc_wait(bar, parity, err, abort_flag);
  return __all_sync(0xffffffffu, ok) != 0;
}

__device__ __forceinline__ uint32_t hmul2_u(uint32_t a, uint32_t b) {
  __half2 r = __hmul2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t f2_to_h2(float lo, float hi) {
  __half2 r = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&r);
}
__device__ __forceinline__ uint4 lds128s(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ uint2 lds64s(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds16s(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds32s(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}

// One IQ2 sub-block of a row (32 weights: an 8-byte record of four grid
// index bytes and a word holding four 7-bit sign fields and the 4-bit scale)
// -> 16 words of fp16 pairs in K order. The three scaled levels s*8, s*25,
// s*43 are rounded to fp16 once and laid out as prmt source bytes (low bytes
// at 0..2, high bytes at 3..5, the byte positions the level selectors
// expect); per group of 8 the grid row gives four prmt selectors and the sign
// field four fp16 pairs of +-1 that multiply exactly, so each weight is the
// fp16 rounding of (+-level) * s. Shifts are written as multiplications so
// that the compiler may place them on the multiply-add pipe beside the prmt work.
__device__ __forceinline__ void dq_iq2_sub(uint2 rec, float dsc, uint32_t tabL, uint32_t tabS, uint32_t (&o)[16]) {
  const uint32_t idx = rec.x, v = rec.y;
  const float sf = dsc * static_cast<float>(2 * __umulhi(v, 16u) + 1);  // v >> 28 = ls
  const uint32_t s2 = f2_to_h2(sf, sf);
  const uint32_t t01 = hmul2_u(kHalf8And25, s2), t2 = hmul2_u(kHalf43Twice, s2);
  const uint32_t srcA = prmt(t01, t2, 0x1420u), srcB = prmt(t01, t2, 0x0053u);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    // byte e of idx at bits 7..14 (x 128-byte entries), sign field e likewise
    const uint32_t gsh = e == 0 ? idx * 128u : __umulhi(idx, 1u << (39 - 8 * e));
    const uint32_t ssh = e == 0 ? v * 128u : (e == 1 ? v : __umulhi(v, 1u << (39 - 7 * e)));
    const uint2 L = lds64s(tabL + (gsh & 0x7F80u));
    const uint4 S = lds128s(tabS + (ssh & 0x3F80u));
    o[4 * e + 0] = hmul2_u(prmt(srcA, srcB, L.x), S.x);
    o[4 * e + 1] = hmul2_u(prmt(srcA, srcB, __umulhi(L.x, 0x10000u)), S.y);
    o[4 * e + 2] = hmul2_u(prmt(srcA, srcB, L.y), S.z);
    o[4 * e + 3] = hmul2_u(prmt(srcA, srcB, __umulhi(L.y, 0x10000u)), S.w);
  }
}

// One Q2K sub-block of a row (16 weights, four per byte of `w`: weight 4b+i at
// bits 8b+2i) with scale byte `scb` (sc | m << 4) -> 8 words of fp16 pairs in
// K order. The four values d*sc*q - dmin*m, q = 0..3, are the prmt source bytes.
__device__ __forceinline__ void dq_q2k_sub(uint32_t w, uint32_t scb, float d, float dmin, uint32_t tabQ,
                                           uint32_t (&o)[8]) {
  const float A = d * static_cast<float>(scb & 15u), B = dmin * static_cast<float>(scb >> 4);
  // q = 0 is evaluated as (d*sc)*0 - dmin*m, not -dmin*m: a zero weight then has the sign IEEE
  // arithmetic gives the rule's expression (it follows the signs of d and dmin)
  const uint32_t tlo = f2_to_h2(__fsub_rn(__fmul_rn(A, 0.f), B), A - B), thi = f2_to_h2(2.f * A - B, 3.f * A - B);
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    const uint32_t ent = b == 0 ? w * 128u : __umulhi(w, 1u << (39 - 8 * b));  // byte b at bits 7..14
    const uint32_t sel = lds32s(tabQ + (ent & 0x7F80u));                       // tabQ includes lane * 4
    o[2 * b] = prmt(tlo, thi, sel);
    o[2 * b + 1] = prmt(tlo, thi, __umulhi(sel, 0x10000u));
  }
}

__device__ __forceinline__ uint32_t hsub2_u(uint32_t a, uint32_t b) {
  __half2 r = __hsub2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}

// One Q4-style block of a row (32 weights: element 2i in the low nibble of
// code byte i, 2i+1 in the high nibble; w = d * (q - 8)) with s2 = the fp16
// pair (s, s), s = fp16(d * 2^10) -> 16 words of fp16 pairs in K order. The
// pair (1024 + q0, 1024 + q1) is built from its bits (0x6400 | q), so
// q - 8 = (1024 + q) - 1032 is exact in fp16; each weight is then the fp16
// rounding of s * (q - 8). The 2^10 keeps small scales clear of fp16
// subnormals and is taken out in the fp32 epilogue.
__device__ __forceinline__ void dq_q4_block(uint4 c, uint32_t s2, uint32_t (&o)[16]) {
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
  constexpr uint32_t kHalf1032Twice = 0x64086408u;  // fp16 pair (1032, 1032)
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t lo = w[i] & 0x0F0F0F0Fu, hi = (w[i] >> 4) & 0x0F0F0F0Fu;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      // bytes: low nibble of byte b (element 2b) at byte 0, its high nibble (element 2b + 1) at byte 2
      const uint32_t pr = (prmt(lo, hi, static_cast<uint32_t>(b | ((4 + b) << 8))) & 0x00FF00FFu) | 0x64006400u;
      o[4 * i + b] = hmul2_u(hsub2_u(pr, kHalf1032Twice), s2);
    }
  }
}

// The dequantisation tables of the dequantising kinds, at `tabs` (see
// TcLayout): IQ2 level selectors (16 copies of 8 bytes per grid row), IQ2 signs
// as fp16 +-1 pairs (8 copies of 16 bytes per sign field), Q2K selectors (32
// copies of 4 bytes per code byte).
template <int KIND>
__device__ __forceinline__ void fill_dq_tables(uint8_t* tabs, int tid, int nthr) {
  if (KIND == TC_IQ2_PAIR) {
    for (int i = tid; i < 256 * 16 * 2; i += nthr) {  // (row, copy, word): two prmt selectors per word
      const int ent = i >> 5, w = i & 1;
      uint32_t word = 0;
      for (int h = 0; h < 2; ++h) {
        const int e0 = 4 * w + 2 * h;
        uint32_t lv[2];
        for (int q = 0; q < 2; ++q) {
          const uint32_t v = d_codebook_tc.val[ent][e0 + q];
          lv[q] = v == 8 ? 0u : (v == 25 ? 1u : 2u);
        }
        const uint32_t sel = lv[0] | ((3 + lv[0]) << 4) | (lv[1] << 8) | ((3 + lv[1]) << 12);
        word |= sel << (16 * h);
      }
      reinterpret_cast<uint32_t*>(tabs)[i] = word;
    }
    for (int i = tid; i < 128 * 8 * 4; i += nthr) {  // (sign field, copy, word)
      const int ent = i >> 5, w = i & 3;
      uint32_t par = 0;
      for (int b = 0; b < 7; ++b) par ^= (ent >> b) & 1;
      const uint32_t s0 = (2 * w < 7) ? ((ent >> (2 * w)) & 1) : par;
      const uint32_t s1 = (2 * w + 1 < 7) ? ((ent >> (2 * w + 1)) & 1) : par;
      // fp16 pair of +-1 (0x3C00 / 0xBC00)
      reinterpret_cast<uint32_t*>(tabs + 256 * 128)[i] = 0x3C003C00u | (s0 << 15) | (s1 << 31);
    }
  } else if (KIND == TC_Q2K) {
    for (int i = tid; i < 256 * 32; i += nthr) {  // (byte of four 2-bit codes, copy) -> two selectors
      const int byte = i >> 5;
      uint32_t sel = 0;
      for (int q = 0; q < 4; ++q) {
        const uint32_t c = (byte >> (2 * q)) & 3u;
        sel |= ((2 * c) | ((2 * c + 1) << 4)) << (8 * q);
      }
      reinterpret_cast<uint32_t*>(tabs)[i] = sel;
    }
  }
}

// One lane of the (converged) warp returns true, the same lane every time.
__device__ __forceinline__ bool elect_one() {
  uint32_t p;
  asm volatile("{\n .reg .pred P;\n elect.sync _|P, 0xffffffff;\n selp.u32 %0, 1, 0, P;\n}\n" : "=r"(p));
  return p != 0;
}

// silu(g) * u with the fast exponential and division: relative error near
// 1e-6, far below the fp16 rounding that follows; g -> -inf gives -0.
__device__ __forceinline__ float silu_mul_fast(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }

// x * 2^k as two exact power-of-2 multiplications (each factor a normal
// float), the same value as ldexpf for results in the normal range; k is
// clamped to [-252, 252], beyond which every finite fp32 x under- or overflows.
__device__ __forceinline__ float mul_pow2(float x, int k) {
  k = max(-252, min(252, k));
  const int k1 = k >> 1, k2 = k - k1;
  return x * __int_as_float((k1 + 127) << 23) * __int_as_float((k2 + 127) << 23);
}

// Tile i of the list; a tile outside the operands' bounds comes back with
// n = 0 (every role then skips it) and records MOE_ERR_INVALID_ARG.
__device__ __forceinline__ TcPair tc_pair(const TcArgs& a, int i) {
  TcPair p;
  if (a.pairs) {
    p = a.pairs[i];
  } else {
    p.e = 0;
    p.p0 = i * kNT;
    p.n = min(kNT, a.dense_rows - i * kNT);
    p.pad = 0;
  }
  if (p.e < 0 || p.e >= a.n_experts || p.p0 < 0 || p.n < 1 || p.n > kNT || p.p0 + p.n > a.b_rows) {
    if (a.err) atomicCAS(a.err, 0, ERR_ARG);
    p.n = 0;
  }
  return p;
}

// Tensor maps of one launch: the B operand in boxes of 32, 64, 96 and 128 rows (a tile loads the smallest box
// that covers its rows, so the TMA moves no rows of other tiles), and the A weight or code planes.
struct alignas(64) TcMaps {
  CUtensorMap b[4];
  CUtensorMap a0, a1;
};

template <int KIND>
__global__ void __launch_bounds__(kTcThreads, 1) tc_gemm_kernel(const __grid_constant__ TcMaps tm, TcArgs a) {
  constexpr bool PAIR = tc_two(KIND);
  constexpr bool DQ = tc_dq(KIND);
  constexpr bool Q4K = (KIND == TC_Q4_PAIR || KIND == TC_Q4);
  constexpr bool BF16 = (KIND == TC_BF16_PAIR || KIND == TC_BF16);
  using L = TcLayout<KIND>;
  constexpr int kStages = L::stages;
  constexpr int kAStages = L::a_stages;
  constexpr int kAccBufs = L::acc_bufs;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint64_t* fullB = reinterpret_cast<uint64_t*>(smem + L::bars);  // [kStages] shared-memory ring
  uint64_t* emptyB = fullB + kStages;
  uint64_t* fullA = emptyB + kStages;  // [kAStages] TMEM A ring (dequantising kinds)
  uint64_t* emptyA = fullA + kAStages;
  uint64_t* fullC = emptyA + kAStages;  // [kCStages] code-block ring (dequantising kinds)
  uint64_t* emptyC = fullC + kCStages;
  uint64_t* accf = emptyC + kCStages;  // [kAccBufs]
  uint64_t* acce = accf + kAccBufs;    // [kAccBufs]
  uint64_t* drain = acce + kAccBufs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t sbase = smem_addr(smem);

  if ((sbase & 1023u) != 0) {  // the swizzled tiles need 1024-byte alignment
    if (tid == 0) atomicCAS(a.err, 0, ERR_CUDA);
    return;
  }
  if (tid == 0 && blockIdx.x == 0 && a.clear_err) *a.err = 0;
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&fullB[s], 1);
      mbar_init(&emptyB[s], 1);
    }
    for (int s = 0; s < kAStages; ++s) {
      mbar_init(&fullA[s], kDqWarps / 2);  // one group of eight warps fills a stage
      mbar_init(&emptyA[s], 1);
    }
    for (int c = 0; c < kCStages; ++c) {
      mbar_init(&fullC[c], 1);
      mbar_init(&emptyC[c], kDqWarps);  // every dequantising warp reads every block
    }
    for (int b = 0; b < kAccBufs; ++b) {
      mbar_init(&accf[b], 1);
      mbar_init(&acce[b], kEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  // dequantisation tables, replicated per load phase (see TcLayout); the
  // replica of this lane is folded into the table bases (entries 128 bytes apart)
  const uint32_t tabL = sbase + L::tabs + (lane & 15) * 8, tabS = sbase + L::tabs + 256 * 128 + (lane & 7) * 16,
                 tabQ = sbase + L::tabs + lane * 4;
  fill_dq_tables<KIND>(smem + L::tabs, tid, kTcThreads);
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int npairs = a.pairs ? *a.npairs : (a.dense_rows + kNT - 1) / kNT;
  const int nunits = npairs * a.mt;
  const int nks = a.planes * (a.K / kKS);
  const int ks_plane = a.K / kKS;

  if (warp == kProdWarp) {
    if (lane == 0) {
      for (int i = 0; i < 4; ++i) prefetch_tmap(&tm.b[i]);
      int s = 0;
      uint32_t ph = 0;
      int issued = 0;
      for (int u = blockIdx.x; u < nunits && !*abort_flag; u += gridDim.x) {
        const TcPair pr = tc_pair(a, u / a.mt);
        const int m0 = (u % a.mt) * kMT;
        if (pr.n == 0) continue;
        const int bi = (pr.n - 1) >> 5;                                    // B box of 32 (bi + 1) rows
        const uint32_t btx = 32u * 128u * static_cast<uint32_t>(bi + 1);  // its bytes (rows of 64 x 2 bytes)
        for (int ks = 0; ks < nks; ++ks) {
          if (!tc_wait_sleepy(&emptyB[s], ph ^ 1u, a.err, abort_flag, 256)) break;  // the ring runs ahead
          uint8_t* st = smem + s * L::stage_bytes;
          const int kx = (ks % ks_plane) * kKS, pl = ks / ks_plane;
          if (BF16) {
            mbar_arrive_expect_tx(&fullB[s], static_cast<uint32_t>(L::b_off) + btx);
            // the weight maps are 3-D like every map of this file (one plane)
            tma_load_3d(st, &tm.a0, kx, pr.e * a.rows_e + m0, 0, &fullB[s]);
            if (PAIR) tma_load_3d(st + kTile, &tm.a1, kx, pr.e * a.rows_e + m0, 0, &fullB[s]);
          } else {
            mbar_arrive_expect_tx(&fullB[s], btx);
          }
          tma_load_3d(st + L::b_off, &tm.b[bi], kx, pr.p0, pl, &fullB[s]);
          ++issued;
          if (++s == kStages) { s = 0; ph ^= 1u; }
        }
      }
      if (*abort_flag) {  // let every copy issued into a stage land before the CTA can exit
        for (int i = 0; i < kStages && i < issued; ++i) {
          if (--s < 0) { s = kStages - 1; ph ^= 1u; }
          mbar_wait_bounded(&fullB[s], ph, nullptr, 0);
        }
      }
    }
  } else if (DQ && warp == kCodeWarp) {
    // the code-block ring has its own issuing lane, so a code entry that the dequantising warps release
    // late never holds back the token tiles, which then run the whole B ring ahead of the MMAs
    if (lane == 0) {
      prefetch_tmap(&tm.a0);
      int c = 0, issued_c = 0;
      uint32_t pc = 0;
      for (int u = blockIdx.x; u < nunits && !*abort_flag; u += gridDim.x) {
        const TcPair pr = tc_pair(a, u / a.mt);
        const int m0 = (u % a.mt) * kMT;
        if (pr.n == 0) continue;
        const int wrow = pr.e * a.rows_e + m0;
        for (int b = 0; b < nks / 4; ++b) {  // one entry per 256-weight block: its code bytes for four stages
          if (!tc_wait_sleepy(&emptyC[c], pc ^ 1u, a.err, abort_flag, 256)) break;
          uint8_t* ce = smem + L::code_off + c * L::code_bytes;
          mbar_arrive_expect_tx(&fullC[c], L::code_bytes);
          if (KIND == TC_IQ2_PAIR) {
            tma_load_2d(ce, &tm.a0, 64 * b, wrow, &fullC[c]);
            tma_load_2d(ce + 128 * 64, &tm.a1, 64 * b, wrow, &fullC[c]);
          } else if (KIND == TC_Q4_PAIR) {
            tma_load_2d(ce, &tm.a0, 128 * b, wrow, &fullC[c]);
            tma_load_2d(ce + 128 * 128, &tm.a1, 128 * b, wrow, &fullC[c]);
          } else if (KIND == TC_Q4) {
            tma_load_2d(ce, &tm.a0, 128 * b, wrow, &fullC[c]);
          } else {
            tma_load_2d(ce, &tm.a0, 80 * b, wrow, &fullC[c]);
          }
          ++issued_c;
          if (++c == kCStages) { c = 0; pc ^= 1u; }
        }
      }
      if (*abort_flag) {  // let every issued code copy land before the CTA can exit
        for (int i = 0; i < kCStages && i < issued_c; ++i) {
          if (--c < 0) { c = kCStages - 1; pc ^= 1u; }
          mbar_wait_bounded(&fullC[c], pc, nullptr, 0);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // the whole warp runs the loop (waits and operand arithmetic stay warp-uniform)
    // and one elected lane issues the MMAs and their commits
    const uint32_t idesc = umma_idesc_f16(kMT, 16, BF16);  // N patched per tile
    const uint32_t tm = __shfl_sync(0xffffffffu, tmem, 0);
    int s = 0, sa = 0;
    uint32_t ph = 0, pha = 0;
    int t = 0;
    // the abort flag is read once per lane, so its test is made warp-uniform
    for (int u = blockIdx.x; u < nunits && !__any_sync(0xffffffffu, *abort_flag != 0); u += gridDim.x) {
      const TcPair pr = tc_pair(a, u / a.mt);
      if (pr.n == 0) continue;
      const int n16 = (pr.n + 15) & ~15;
      const uint32_t id = (idesc & ~(0x3Fu << 17)) | (static_cast<uint32_t>(n16 >> 3) << 17);
      const int buf = t % kAccBufs;
      if (!tc_wait_warp(&acce[buf], ((t / kAccBufs) & 1) ^ 1u, a.err, abort_flag)) break;
      tc_fence_after();
      const uint32_t d0 = tm + L::acc_base + buf * L::acc_stride, d1 = d0 + 128;
      bool ok = true;
      for (int ks = 0; ks < nks; ++ks) {
        if (!tc_wait_warp(&fullB[s], ph, a.err, abort_flag)) { ok = false; break; }
        if (DQ && !tc_wait_warp(&fullA[sa], pha, a.err, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t st = sbase + s * L::stage_bytes;
        const uint64_t db = umma_desc_sw128(st + L::b_off);
        if (DQ) {
          const uint32_t at = tm + sa * L::a_cols;  // gate (or the single matrix), up at +32
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < kKS / 16; ++kk) {
              const uint32_t acc = (ks | kk) ? 1u : 0u;
              umma_f16_ts(d0, at + 8 * kk, db + 2 * kk, id, acc);  // 16 fp16 = 8 columns of A per step
              if (PAIR) umma_f16_ts(d1, at + 32 + 8 * kk, db + 2 * kk, id, acc);
            }
            umma_commit(&emptyA[sa]);
            umma_commit(&emptyB[s]);
          }
          __syncwarp();
          if (++sa == kAStages) { sa = 0; pha ^= 1u; }
        } else {
          const uint64_t da0 = umma_desc_sw128(st), da1 = umma_desc_sw128(st + kTile);
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < kKS / 16; ++kk) {
              const uint32_t acc = (ks | kk) ? 1u : 0u;
              umma_f16(d0, da0 + 2 * kk, db + 2 * kk, id, acc);  // +32 bytes along K per step
              if (PAIR) umma_f16(d1, da1 + 2 * kk, db + 2 * kk, id, acc);
            }
            umma_commit(&emptyB[s]);
          }
          __syncwarp();
        }
        if (++s == kStages) { s = 0; ph ^= 1u; }
      }
      if (!ok) break;
      if (elect_one()) umma_commit(&accf[buf]);
      __syncwarp();
      ++t;
    }
    // drain: every MMA issued by this warp completes before TMEM is freed
    if (elect_one()) umma_commit(drain);
    __syncwarp();
    mbar_wait_bounded(drain, 0, nullptr, 0);
  } else if (DQ && warp >= kDqWarp0) {
    // sixteen warps in two groups of eight: group g fills the stages ks = g (mod 2),
    // so the two groups' latencies overlap. Warp w may write TMEM lanes
    // 32*(w%4)..+31, so the row is 32*(w%4) + lane; the two warps of a lane
    // quarter in a group split the stage's weights of their rows, each thread
    // turning two sub-blocks of one row into fp16, from the code-block ring the
    // producer fills (one entry per 256-weight block, released by all sixteen warps)
    const int grp = (warp - kDqWarp0) >> 3, part = ((warp - kDqWarp0) >> 2) & 1;
    const int quarter = warp & 3;
    const int r = 32 * quarter + lane;
    const uint32_t tlane = static_cast<uint32_t>(32 * quarter) << 16;
    long long gs = grp;  // global stage index (over this CTA's tiles) of this group's next stage
    int cb = 0;          // code-block ring position and phase
    uint32_t pcb = 0;
    const int nblk = nks / 4;
    // per-block scales of this row (IQ2 d, Q2K d | dmin << 16), loaded one block
    // ahead along the sequence of this CTA's tiles (the next tile's first block
    // is requested during the last block of the current one)
    auto next_tile = [&](int uu) {
      while (uu < nunits && tc_pair(a, uu / a.mt).n == 0) uu += gridDim.x;
      return uu;
    };
    auto row_of = [&](int uu) -> size_t {
      return static_cast<size_t>(tc_pair(a, uu / a.mt).e) * a.rows_e + (uu % a.mt) * kMT + r;
    };
    auto ldscale = [&](size_t grow, int b) -> uint32_t {
      if (KIND == TC_IQ2_PAIR) return static_cast<uint32_t>(__ldg((part ? a.d1 : a.d0) + grow * nblk + b));
      return __ldg(a.dd + grow * nblk + b);
    };
    // Q4-style kinds: the fp16 d of the stage's two 32-weight blocks of this row (one word), loaded one
    // stage of this group ahead
    auto ldq4 = [&](size_t grow, int ks_) -> uint32_t {
      const uint16_t* dp = (KIND == TC_Q4_PAIR && part) ? a.d1 : a.d0;
      return __ldg(reinterpret_cast<const uint32_t*>(dp + grow * (a.K / 32)) + ks_);
    };
    int u = next_tile(blockIdx.x);
    uint32_t dq1 = (!Q4K && u < nunits) ? ldscale(row_of(u), 0) : 0u;
    uint32_t q4n = (Q4K && u < nunits) ? ldq4(row_of(u), grp) : 0u;
    while (u < nunits) {
      const int un = next_tile(u + gridDim.x);
      const size_t grow = row_of(u);
      const size_t grow_n = un < nunits ? row_of(un) : 0;
      bool ok = true;
      uint32_t dq0 = 0;
      for (int ks = grp; ks < nks && ok; ks += 2, gs += 2) {  // nks is a multiple of 4
        const int q = ks & 3;
        if (q == grp && !tc_wait_warp(&fullC[cb], pcb, a.err, abort_flag)) {  // the block's code bytes
          ok = false;
          break;
        }
        if (!Q4K && (ks & 3) == grp) {  // the group's first stage of a block
          const int b = ks >> 2;
          dq0 = dq1;
          dq1 = b + 1 < nblk ? ldscale(grow, b + 1) : (un < nunits ? ldscale(grow_n, 0) : 0u);
        }
        uint32_t q4d = 0;
        if (Q4K) {
          q4d = q4n;
          q4n = ks + 2 < nks ? ldq4(grow, ks + 2) : (un < nunits ? ldq4(grow_n, grp) : 0u);
        }
        // A free TMEM A slot is needed only for the stores. The Q4-style kinds decode into registers first,
        // so their longer decode overlaps the MMAs still reading the slot (6 % faster gate/up); the 2-bit kinds
        // wait first (decoding first was no faster for them, within the run-to-run spread of ~2 %).
        const int sa = static_cast<int>(gs % kAStages);
        const uint32_t pha = static_cast<uint32_t>((gs / kAStages) & 1);
        if (!Q4K && !tc_wait_warp(&emptyA[sa], pha ^ 1u, a.err, abort_flag)) {
          ok = false;
          break;
        }
        const uint32_t ce = sbase + L::code_off + cb * L::code_bytes;
        uint32_t o0[16], o1[16];
        if (KIND == TC_IQ2_PAIR) {
          // part = matrix; the row's two 8-byte records of this stage (32 weights each)
          const uint4 rec = lds128s(ce + part * (128 * 64) + r * 64 + 16 * q);
          const float dsc = half_bits_to_float(static_cast<uint16_t>(dq0)) * 128.0f;  // d / 8 * 2^10
          dq_iq2_sub(make_uint2(rec.x, rec.y), dsc, tabL, tabS, o0);
          dq_iq2_sub(make_uint2(rec.z, rec.w), dsc, tabL, tabS, o1);
        } else if (KIND == TC_Q4_PAIR) {
          // part = matrix; the row's 64 weights of this stage: two 32-weight blocks, 32 code bytes
          const uint32_t cq = ce + part * (128 * 128) + r * 128 + 32 * q;
          const uint4 c0 = lds128s(cq), c1 = lds128s(cq + 16);
          const float s0 = half_bits_to_float(static_cast<uint16_t>(q4d & 0xFFFFu)) * 1024.0f;
          const float s1 = half_bits_to_float(static_cast<uint16_t>(q4d >> 16)) * 1024.0f;
          dq_q4_block(c0, f2_to_h2(s0, s0), o0);
          dq_q4_block(c1, f2_to_h2(s1, s1), o1);
        } else if (KIND == TC_Q4) {
          // part = half of the stage's 64 weights = block 2 * ks + part (16 code bytes)
          const uint4 c0 = lds128s(ce + r * 128 + 32 * q + 16 * part);
          const float s0 = half_bits_to_float(static_cast<uint16_t>(part ? q4d >> 16 : q4d & 0xFFFFu)) * 1024.0f;
          dq_q4_block(c0, f2_to_h2(s0, s0), o0);
        } else {
          // part = half of the stage's 64 weights = sub-blocks 4 * (ks % 4) + 2 * part, +1 of the block
          const uint2 w = lds64s(ce + r * 80 + 16 + 16 * q + 8 * part);
          const uint32_t scb = lds16s(ce + r * 80 + 4 * q + 2 * part);
          const float d = half_bits_to_float(static_cast<uint16_t>(dq0 & 0xFFFFu));
          const float dmin = half_bits_to_float(static_cast<uint16_t>(dq0 >> 16));
          uint32_t q0[8], q1[8];
          dq_q2k_sub(w.x, scb & 0xFFu, d, dmin, tabQ, q0);
          dq_q2k_sub(w.y, scb >> 8, d, dmin, tabQ, q1);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            o0[i] = q0[i];
            o0[8 + i] = q1[i];
          }
        }
        if (Q4K && !tc_wait_warp(&emptyA[sa], pha ^ 1u, a.err, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (tc_two(KIND)) {  // gate (or up) stage of the pair: 32 columns
          const uint32_t tc = tmem + tlane + part * 32 + sa * L::a_cols;
          tmem_st16(tc, o0);
          tmem_st16(tc + 16, o1);
        } else {  // half of a single matrix's stage: 16 columns
          tmem_st16(tmem + tlane + part * 16 + sa * L::a_cols, o0);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&fullA[sa]);
        if (q == grp + 2) {  // this group's last stage of the block: the code entry is free for this warp
          if (lane == 0) mbar_arrive(&emptyC[cb]);
          if (++cb == kCStages) { cb = 0; pcb ^= 1u; }
        }
      }
      if (!ok) break;
      u = un;
    }
  } else if (warp < kEpiWarps) {
    const int r = 32 * warp + lane;  // TMEM lane = weight row of the tile
    int t = 0;
    for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
      const TcPair pr = tc_pair(a, u / a.mt);
      const int m0 = (u % a.mt) * kMT;
      if (pr.n == 0) continue;
      const int buf = t % kAccBufs;
      // the tile's per-row exponents (lane n % 32 of word n / 32), loaded before the wait
      int ex4[4] = {0, 0, 0, 0};
      if (tc_hout(KIND)) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (32 * i + lane < pr.n) ex4[i] = __ldg(a.row_exp + pr.p0 + 32 * i + lane);
      }
      // the epilogue waits out a whole tile of MMAs: it sleeps between polls
      const bool got = tc_wait_sleepy(&accf[buf], (t / kAccBufs) & 1, a.err, abort_flag, kAccBufs > 1 ? 2048 : 256);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const uint32_t tl = tmem + L::acc_base + buf * L::acc_stride + (static_cast<uint32_t>(32 * warp) << 16);
      const int row = m0 + r;
      for (int c0 = 0; c0 < pr.n; c0 += 16) {
        uint32_t g[16], v[16];
        tmem_ld16(tl + c0, g);
        if (PAIR) tmem_ld16(tl + 128 + c0, v);
        const int exw = (c0 < 64) ? (c0 < 32 ? ex4[0] : ex4[1]) : (c0 < 96 ? ex4[2] : ex4[3]);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int n = c0 + j;
          if (n >= pr.n) break;
          const size_t orow = static_cast<size_t>(pr.p0 + n);
          if (tc_hout(KIND)) {
            // B row = x * 2^-e: g, u come back as exact fp32 rescalings; h leaves as
            // fp16(h * 2^(-2e-12)), the scale that keeps it inside the fp16 range
            const int ex = __shfl_sync(0xffffffffu, exw, (c0 & 31) + j);
            float gs = __uint_as_float(g[j]) * a.oscale, us = __uint_as_float(v[j]) * a.oscale;
            float h;
            if (ex >= -60 && ex <= 55) {  // both factors are normal floats: build them from exponent bits
              const float up = __int_as_float((ex + 127) << 23), down = __int_as_float((127 - 12 - 2 * ex) << 23);
              h = silu_mul_fast(gs * up, us * up) * down;
            } else {
              h = mul_pow2(silu_mul_fast(mul_pow2(gs, ex), mul_pow2(us, ex)), -2 * ex - 12);
            }
            reinterpret_cast<__half*>(a.out)[orow * a.ldo + row] = __float2half_rn(h);
          } else if (KIND == TC_BF16_PAIR) {
            const float h = silu_mul_fast(__uint_as_float(g[j]), __uint_as_float(v[j]));
            const __nv_bfloat16 hi = __float2bfloat16_rn(h);
            const __nv_bfloat16 lo = __float2bfloat16_rn(h - __bfloat162float(hi));
            reinterpret_cast<__nv_bfloat16*>(a.out)[orow * a.ldo + row] = hi;
            reinterpret_cast<__nv_bfloat16*>(a.out)[(static_cast<size_t>(a.out_rows) + orow) * a.ldo + row] = lo;
          } else if (tc_oout(KIND)) {  // routed expert outputs, combined later in slot order
            // B row = h * 2^(-2e-12), so the accumulator is o * 2^(-2e-12) (h and o are
            // quadratic in x); it is stored as is and the combine applies 2^(2e+12)
            reinterpret_cast<__half*>(a.out)[orow * a.ldo + row] = __float2half_rn(__uint_as_float(g[j]) * a.oscale);
          } else {
            const float bv = (KIND == TC_BF16 && a.bias) ? a.bias[row] : 0.f;
            reinterpret_cast<float*>(a.out)[orow * a.ldo + row] = __uint_as_float(g[j]) * a.oscale + bv;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acce[buf]);
      ++t;
    }
  }
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace
}  // namespace moe

namespace moe {
namespace {

// Power-of-2 exponent per token: e = floor(log2 max|x_t|) - 12 (0 for a zero
// row), so x * 2^-e lies below 2^13 in magnitude and well inside fp16.
template <typename XT>
__global__ void __launch_bounds__(256) token_exp_kernel(const XT* __restrict__ x, int T, int H,
                                                        int32_t* __restrict__ texp) {
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (t >= T) return;
  float m = 0.f;
  for (int i = lane; i < H; i += 32) {
    float v;
    if constexpr (sizeof(XT) == 4) v = reinterpret_cast<const float*>(x)[static_cast<size_t>(t) * H + i];
    else v = __uint_as_float(static_cast<uint32_t>(reinterpret_cast<const uint16_t*>(x)[static_cast<size_t>(t) * H + i]) << 16);
    m = fmaxf(m, fabsf(v));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) texp[t] = m > 0.f ? floor_log2_pos(m) - 12 : 0;
}

// Expert-sorted fp16 copy of the activations for the routed B operand, and the
// tile lists: routed (expert, first assignment, count) tiles of up to 128
// assignments, and shared tiles of up to 128 tokens. Block 0 also clears the
// call's status word.
template <typename XT>
__global__ void __launch_bounds__(256) prefill_prep_kernel(const XT* __restrict__ x, int T, int H, int k,
                                                           const int32_t* __restrict__ perm, __half* __restrict__ xp,
                                                           const int32_t* __restrict__ offsets,
                                                           const int32_t* __restrict__ active, int E,
                                                           TcPair* __restrict__ pairs, int32_t* __restrict__ npairs,
                                                           TcPair* __restrict__ spairs, int32_t* __restrict__ nspairs,
                                                           const int32_t* __restrict__ texp,
                                                           int32_t* __restrict__ aexp, int* __restrict__ err_word) {
  const int nA = T * k;
  if (blockIdx.x == 0 && threadIdx.x < 32) {
    const int lane = threadIdx.x;
    if (lane == 0 && err_word) *err_word = 0;
    const int nact = active[E];
    int base = 0;
    for (int s0 = 0; s0 < nact; s0 += 32) {
      const int s = s0 + lane;
      int e = 0, p0 = 0, ne = 0;
      if (s < nact) {
        e = active[s];
        p0 = offsets[e];
        ne = offsets[e + 1] - p0;
      }
      const int nt = (ne + kNT - 1) / kNT;
      int incl = nt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      for (int j = 0; j < nt; ++j) {
        TcPair pr;
        pr.e = e;
        pr.p0 = p0 + j * kNT;
        pr.n = min(kNT, ne - j * kNT);
        pr.pad = 0;
        pairs[base + incl - nt + j] = pr;
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) *npairs = base;
    const int ns = (T + kNT - 1) / kNT;
    for (int j = lane; j < ns; j += 32) {
      TcPair pr;
      pr.e = 0;
      pr.p0 = j * kNT;
      pr.n = min(kNT, T - j * kNT);
      pr.pad = 0;
      spairs[j] = pr;
    }
    if (lane == 0) *nspairs = ns;
  }
  const int per = H / 8;
  const size_t n8 = static_cast<size_t>(nA) * per;
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int p = static_cast<int>(i / per), c = static_cast<int>(i % per);
    const int tok = perm[p] / k;
    const int ex = texp[tok];
    if (c == 0) aexp[p] = ex;
    const size_t src = static_cast<size_t>(tok) * H + c * 8;
    float v[8];
    if constexpr (sizeof(XT) == 4) {
      const float4 a0 = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(x) + src);
      const float4 a1 = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(x) + src + 4);
      v[0] = a0.x; v[1] = a0.y; v[2] = a0.z; v[3] = a0.w; v[4] = a1.x; v[5] = a1.y; v[6] = a1.z; v[7] = a1.w;
    } else {
      const uint4 w = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(x) + src);
      v[0] = __uint_as_float(w.x << 16); v[1] = __uint_as_float(w.x & 0xFFFF0000u);
      v[2] = __uint_as_float(w.y << 16); v[3] = __uint_as_float(w.y & 0xFFFF0000u);
      v[4] = __uint_as_float(w.z << 16); v[5] = __uint_as_float(w.z & 0xFFFF0000u);
      v[6] = __uint_as_float(w.w << 16); v[7] = __uint_as_float(w.w & 0xFFFF0000u);
    }
    if (ex >= -127 && ex <= 126) {  // 2^-ex is a normal float: one rounding, the value ldexpf gives
      const float sc = __int_as_float((127 - ex) << 23);
#pragma unroll
      for (int q = 0; q < 8; ++q) v[q] *= sc;
    } else {
#pragma unroll
      for (int q = 0; q < 8; ++q) v[q] = ldexpf(v[q], -ex);
    }
    uint4 o;
    o.x = f2_to_h2(v[0], v[1]);
    o.y = f2_to_h2(v[2], v[3]);
    o.z = f2_to_h2(v[4], v[5]);
    o.w = f2_to_h2(v[6], v[7]);
    *reinterpret_cast<uint4*>(xp + static_cast<size_t>(p) * H + c * 8) = o;
  }
}

// fp32 activations as two bf16 parts [2][T][H] for the shared expert.
__global__ void __launch_bounds__(256) bf16_parts_kernel(const float* __restrict__ x, size_t n,
                                                         __nv_bfloat16* __restrict__ xb) {
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const float v = x[i];
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    xb[i] = hi;
    xb[n + i] = __float2bfloat16_rn(v - __bfloat162float(hi));
  }
}

// y[t][h] = sum_j w[t][j] o[inv[t*k+j]][h] (j ascending) + s[t][h] (+ residual),
// with the routed expert outputs stored as fp16 o * 2^(-2e-12) of their token
// (relative rounding 2^-11, an order below the 2e-3 bound) to halve the
// traffic of this pass; w * 2^(2e+12) is exact.
__global__ void __launch_bounds__(256) prefill_combine_kernel(int T, int H, int k, const float* __restrict__ topk_w,
                                                              const int32_t* __restrict__ inv,
                                                              const __half* __restrict__ o,
                                                              const int32_t* __restrict__ texp, const float* s,
                                                              const float* residual, float* y) {
  const size_t n4 = static_cast<size_t>(T) * H / 4;
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int t = static_cast<int>((i * 4) / H), h = static_cast<int>((i * 4) % H);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    const float tsc = ldexpf(1.0f, 2 * texp[t] + 12);  // the routed outputs arrive as o * 2^(-2e-12)
    for (int j = 0; j < k; ++j) {
      const float w = topk_w[t * k + j] * tsc;
      const uint2 hv = *reinterpret_cast<const uint2*>(o + static_cast<size_t>(inv[t * k + j]) * H + h);
      const float2 v01 = __half22float2(*reinterpret_cast<const __half2*>(&hv.x));
      const float2 v23 = __half22float2(*reinterpret_cast<const __half2*>(&hv.y));
      acc.x = fmaf(w, v01.x, acc.x);
      acc.y = fmaf(w, v01.y, acc.y);
      acc.z = fmaf(w, v23.x, acc.z);
      acc.w = fmaf(w, v23.y, acc.w);
    }
    if (s) {
      const float4 v = *reinterpret_cast<const float4*>(s + i * 4);
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    if (residual) {
      const float4 v = *reinterpret_cast<const float4*>(residual + i * 4);
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    *reinterpret_cast<float4*>(y + i * 4) = acc;
  }
}

PFN_cuTensorMapEncodeTiled_v12000 tc_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// [planes][rows][K] 16-bit elements, box 64 (K) x box_rows rows x 1 plane, 128-byte swizzle.
bool tc_map(CUtensorMap* m, const void* base, bool bf16, uint64_t K, uint64_t rows, uint64_t planes,
            uint32_t box_rows = 128) {
  auto fn = tc_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {K, rows, planes};
  const cuuint64_t strides[2] = {K * 2, K * 2 * rows};
  const cuuint32_t box[3] = {64, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
                        const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D map over a plane of code bytes: rows of `row_bytes`, boxes of `box_bytes` x 128 rows.
bool code_map(CUtensorMap* m, const void* base, uint64_t row_bytes, uint64_t rows, uint32_t box_bytes) {
  auto fn = tc_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {row_bytes, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_bytes, 128};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The four B maps (boxes of 32, 64, 96, 128 rows) over one B plane set.
bool tc_bmaps(TcMaps* m, const void* base, bool bf16, uint64_t K, uint64_t rows, uint64_t planes) {
  for (int i = 0; i < 4; ++i)
    if (!tc_map(&m->b[i], base, bf16, K, rows, planes, 32u * (i + 1))) return false;
  return true;
}

template <int KIND>
int launch_tc(const TcMaps& tm, const TcArgs& a, int sms, cudaStream_t st) {
  const size_t smem = TcLayout<KIND>::total;
  cudaFuncSetAttribute(tc_gemm_kernel<KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  tc_gemm_kernel<KIND><<<sms, kTcThreads, smem, st>>>(tm, a);
  return cudaGetLastError() == cudaSuccess ? OK : ERR_CUDA;
}

struct PrefillWs {
  __half* xp;
  __half* hh;
  __half* o;  // routed expert outputs [T*k][H], fp16
  __nv_bfloat16* xb;
  __nv_bfloat16* hs;
  float* s;
  TcPair* pairs;
  TcPair* spairs;
  int32_t* counts;
  int32_t* texp;  // per token
  int32_t* aexp;  // per assignment
  size_t bytes;
};

PrefillWs carve_prefill(const LayerShape& sh, int T, char* base) {
  const size_t nA = static_cast<size_t>(T) * sh.k;
  PrefillWs w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* q = base ? base + off : nullptr;
    off += align_up(bytes > 0 ? bytes : 1, 1024);
    return q;
  };
  w.xp = reinterpret_cast<__half*>(take(nA * sh.H * 2));
  w.hh = reinterpret_cast<__half*>(take(nA * sh.I * 2));
  w.o = reinterpret_cast<__half*>(take(nA * sh.H * 2));
  w.xb = reinterpret_cast<__nv_bfloat16*>(take(static_cast<size_t>(T) * sh.H * 2 * 2));
  w.hs = reinterpret_cast<__nv_bfloat16*>(take(static_cast<size_t>(T) * (sh.Is > 0 ? sh.Is : 1) * 2 * 2));
  w.s = reinterpret_cast<float*>(take(static_cast<size_t>(T) * sh.H * 4));
  w.pairs = reinterpret_cast<TcPair*>(take((static_cast<size_t>(sh.E) + nA / kNT + 1) * sizeof(TcPair)));
  w.spairs = reinterpret_cast<TcPair*>(take((static_cast<size_t>(T) / kNT + 1) * sizeof(TcPair)));
  w.counts = reinterpret_cast<int32_t*>(take(64));
  w.texp = reinterpret_cast<int32_t*>(take(static_cast<size_t>(T) * 4));
  w.aexp = reinterpret_cast<int32_t*>(take(nA * 4));
  w.bytes = off;
  return w;
}

// The grouped GEMM's dequantisers run on their own, for exact checks: every
// 32-weight IQ2 sub-block (dq_iq2_sub, scale d / 8 * 2^10) and every 16-weight
// Q2K sub-block (dq_q2k_sub) to the fp16 words the kernel stores into TMEM,
// weights in K order. Each lane reads its own replica of the tables.
__global__ void __launch_bounds__(256) debug_tc_iq2_kernel(const uint8_t* __restrict__ codes,
                                                           const uint16_t* __restrict__ d, int64_t nsub,
                                                           uint32_t* __restrict__ out) {
  extern __shared__ __align__(1024) uint8_t smem[];
  fill_dq_tables<TC_IQ2_PAIR>(smem, threadIdx.x, blockDim.x);
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const uint32_t sbase = smem_addr(smem);
  const uint32_t tabL = sbase + (lane & 15) * 8, tabS = sbase + 256 * 128 + (lane & 7) * 16;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nsub;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint2 rec = *reinterpret_cast<const uint2*>(codes + 8 * i);
    const float dsc = half_bits_to_float(d[i / 8]) * 128.0f;  // d / 8 * 2^10, as the GEMM's dequantisers
    uint32_t o[16];
    dq_iq2_sub(rec, dsc, tabL, tabS, o);
    uint4* dst = reinterpret_cast<uint4*>(out + 16 * i);
#pragma unroll
    for (int q = 0; q < 4; ++q) dst[q] = make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
  }
}

__global__ void __launch_bounds__(256) debug_tc_q2k_kernel(const uint8_t* __restrict__ codes,
                                                           const uint32_t* __restrict__ dd, int64_t nsub,
                                                           uint32_t* __restrict__ out) {
  extern __shared__ __align__(1024) uint8_t smem[];
  fill_dq_tables<TC_Q2K>(smem, threadIdx.x, blockDim.x);
  __syncthreads();
  const uint32_t tabQ = smem_addr(smem) + (threadIdx.x & 31) * 4;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nsub;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint8_t* blk = codes + (i / 16) * 80;
    const int sb = static_cast<int>(i % 16);
    const uint32_t w = *reinterpret_cast<const uint32_t*>(blk + 16 + 4 * sb);
    const uint32_t ddv = dd[i / 16];
    uint32_t o[8];
    dq_q2k_sub(w, blk[sb], half_bits_to_float(static_cast<uint16_t>(ddv & 0xFFFFu)),
               half_bits_to_float(static_cast<uint16_t>(ddv >> 16)), tabQ, o);
    uint4* dst = reinterpret_cast<uint4*>(out + 8 * i);
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

}  // namespace

// Router logits for many bf16 tokens on the same tensor-core GEMM: weights
// Wr [E][H] (bf16, by TMA) are the M operand, tokens the N operand, the bias is
// added in the epilogue: logits[t][e] = sum_h Wr[e][h] x[t][h] + bias[e].
bool router_tc_supported(int T, int H, int E) {
  return T > 64 && H % kKS == 0 && E % kMT == 0 && tc_encode_fn() != nullptr;
}

int launch_router_tc(const uint16_t* Wr, const float* bias, const uint16_t* x, int T, int H, int E, float* logits,
                     int* err, int sms, cudaStream_t st) {
  TcMaps tm;
  if (!tc_bmaps(&tm, x, true, H, T, 1) || !tc_map(&tm.a0, Wr, true, H, E, 1)) return ERR_CUDA;
  tm.a1 = tm.a0;
  TcArgs a{};
  a.n_experts = 1; a.b_rows = T;
  a.rows_e = E; a.K = H; a.mt = E / kMT; a.planes = 1;
  a.dense_rows = T; a.bias = bias; a.out = logits; a.ldo = E; a.out_rows = T;
  a.oscale = 1.0f; a.err = err; a.clear_err = 1;
  return launch_tc<TC_BF16>(tm, a, sms, st);
}

bool prefill_path_supported(const LayerShape& s, int T) {
  if (T < 1 || s.H % 256 != 0 || s.I % 256 != 0 || s.H % kMT != 0 || s.I % kMT != 0) return false;
  if (s.Is > 0 && (s.Is % kMT != 0 || s.Is % kKS != 0)) return false;
  return tc_encode_fn() != nullptr;
}

size_t prefill_workspace_bytes(const LayerShape& s, int T) { return carve_prefill(s, T, nullptr).bytes; }

int launch_ffn_prefill(const LayerShape& sh, const WeightPtrs& w, const void* x, int x_dtype, int T,
                       const Routing& r, const float* residual, float* y, void* ws, int* err, bool clear_status,
                       int sms, cudaStream_t st, const MxPlanes* q4) {
  const PrefillWs pw = carve_prefill(sh, T, static_cast<char*>(ws));
  const int nA = T * sh.k;
  int rc = OK;
  {
    ProfScope ps(MOE_K_PREP, st);
    const int grid = std::max(1, std::min(sms * 4, (nA * (sh.H / 8) + 255) / 256));
    if (x_dtype == 0)
      token_exp_kernel<float><<<(T + 7) / 8, 256, 0, st>>>(static_cast<const float*>(x), T, sh.H, pw.texp);
    else
      token_exp_kernel<uint16_t><<<(T + 7) / 8, 256, 0, st>>>(static_cast<const uint16_t*>(x), T, sh.H, pw.texp);
    if (x_dtype == 0)
      prefill_prep_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float*>(x), T, sh.H, sh.k, r.perm, pw.xp,
                                                       r.offsets, r.active, sh.E, pw.pairs, pw.counts, pw.spairs,
                                                       pw.counts + 1, pw.texp, pw.aexp, clear_status ? err : nullptr);
    else
      prefill_prep_kernel<uint16_t><<<grid, 256, 0, st>>>(static_cast<const uint16_t*>(x), T, sh.H, sh.k, r.perm,
                                                          pw.xp, r.offsets, r.active, sh.E, pw.pairs, pw.counts,
                                                          pw.spairs, pw.counts + 1, pw.texp, pw.aexp,
                                                          clear_status ? err : nullptr);
    if (sh.Is > 0 && x_dtype == 0) {
      const size_t n = static_cast<size_t>(T) * sh.H;
      bf16_parts_kernel<<<sms * 4, 256, 0, st>>>(static_cast<const float*>(x), n, pw.xb);
    }
  }
  TcMaps tm;
  // routed gate/up: A = IQ2 gate/up rows (dequantised), B = expert-sorted fp16 activations
  {
    ProfScope ps(MOE_K_PREFILL_GATEUP, st);
    const uint64_t wrows = static_cast<uint64_t>(sh.E) * sh.I;
    // IQ2: 64 code bytes per 256 weights; Q4-style: 128
    const uint8_t* gc = q4 ? q4->gate_codes : w.gate_codes;
    const uint8_t* uc = q4 ? q4->up_codes : w.up_codes;
    const uint32_t cb = q4 ? 128 : 64;
    if (!tc_bmaps(&tm, pw.xp, false, sh.H, nA, 1) || !code_map(&tm.a0, gc, sh.H / 256 * cb, wrows, cb) ||
        !code_map(&tm.a1, uc, sh.H / 256 * cb, wrows, cb))
      return ERR_CUDA;
    TcArgs a{};
    a.n_experts = sh.E; a.b_rows = nA;
    a.rows_e = sh.I; a.K = sh.H; a.mt = sh.I / kMT; a.planes = 1;
    a.c0 = gc; a.c1 = uc;
    a.d0 = q4 ? static_cast<const uint16_t*>(q4->gate_scales) : w.gate_d;
    a.d1 = q4 ? static_cast<const uint16_t*>(q4->up_scales) : w.up_d;
    a.pairs = pw.pairs; a.npairs = pw.counts; a.out = pw.hh; a.ldo = sh.I; a.out_rows = nA;
    a.oscale = 1.0f / 1024.0f; a.err = err; a.row_exp = pw.aexp;
    rc |= q4 ? launch_tc<TC_Q4_PAIR>(tm, a, sms, st) : launch_tc<TC_IQ2_PAIR>(tm, a, sms, st);
  }
  if (sh.Is > 0) {
    ProfScope ps(MOE_K_SHARED_GATEUP, st);
    const int planes = x_dtype == 0 ? 2 : 1;
    const void* xsrc = x_dtype == 0 ? static_cast<const void*>(pw.xb) : x;
    if (!tc_bmaps(&tm, xsrc, true, sh.H, T, planes) || !tc_map(&tm.a0, w.sh_gate, true, sh.H, sh.Is, 1) ||
        !tc_map(&tm.a1, w.sh_up, true, sh.H, sh.Is, 1))
      return ERR_CUDA;
    TcArgs a{};
    a.n_experts = 1; a.b_rows = T;
    a.rows_e = sh.Is; a.K = sh.H; a.mt = sh.Is / kMT; a.planes = planes;
    a.dense_rows = T; a.out = pw.hs; a.ldo = sh.Is; a.out_rows = T;
    a.oscale = 1.0f; a.err = err;
    rc |= launch_tc<TC_BF16_PAIR>(tm, a, sms, st);
  }
  {
    ProfScope ps(MOE_K_PREFILL_DOWN, st);
    // Q2K: 80 code bytes per 256 weights; Q4-style: 128
    const uint8_t* dc = q4 ? q4->down_codes : w.down_codes;
    const uint32_t cb = q4 ? 128 : 80;
    if (!tc_bmaps(&tm, pw.hh, false, sh.I, nA, 1) ||
        !code_map(&tm.a0, dc, static_cast<uint64_t>(sh.I / 256) * cb, static_cast<uint64_t>(sh.E) * sh.H, cb))
      return ERR_CUDA;
    tm.a1 = tm.a0;
    TcArgs a{};
    a.n_experts = sh.E; a.b_rows = nA;
    a.rows_e = sh.H; a.K = sh.I; a.mt = sh.H / kMT; a.planes = 1;
    a.c0 = dc; a.dd = w.down_dd;
    if (q4) a.d0 = static_cast<const uint16_t*>(q4->down_scales);
    a.pairs = pw.pairs; a.npairs = pw.counts; a.out = pw.o; a.ldo = sh.H; a.out_rows = nA;
    a.oscale = q4 ? 1.0f / 1024.0f : 1.0f; a.err = err; a.row_exp = pw.aexp;
    rc |= q4 ? launch_tc<TC_Q4>(tm, a, sms, st) : launch_tc<TC_Q2K>(tm, a, sms, st);
  }
  if (sh.Is > 0) {
    ProfScope ps(MOE_K_SHARED_DOWN, st);
    if (!tc_bmaps(&tm, pw.hs, true, sh.Is, T, 2) || !tc_map(&tm.a0, w.sh_down, true, sh.Is, sh.H, 1)) return ERR_CUDA;
    tm.a1 = tm.a0;
    TcArgs a{};
    a.n_experts = 1; a.b_rows = T;
    a.rows_e = sh.H; a.K = sh.Is; a.mt = sh.H / kMT; a.planes = 2;
    a.dense_rows = T; a.out = pw.s; a.ldo = sh.H; a.out_rows = T;
    a.oscale = 1.0f; a.err = err;
    rc |= launch_tc<TC_BF16>(tm, a, sms, st);
  }
  {
    ProfScope ps(MOE_K_COMBINE, st);
    const int grid = std::max(1, std::min(sms * 8, static_cast<int>((static_cast<size_t>(T) * sh.H / 4 + 255) / 256)));
    prefill_combine_kernel<<<grid, 256, 0, st>>>(T, sh.H, sh.k, r.topk_w, r.inv, pw.o, pw.texp, sh.Is > 0 ? pw.s : nullptr,
                                                 residual, y);
  }
  if (rc != OK) return ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? OK : ERR_CUDA;
}

// The shared expert alone on the tensor-core GEMM for T tokens: s = Wsd (silu(Wsg x) * (Wsu x)), fp32 [T][H].
// Workspace: bf16 parts of x (fp32 inputs) and of h.
size_t prefill_shared_workspace_bytes(const LayerShape& sh, int T) {
  return align_up(static_cast<size_t>(T) * sh.H * 2 * 2, 1024) +
         align_up(static_cast<size_t>(T) * (sh.Is > 0 ? sh.Is : 1) * 2 * 2, 1024);
}

int launch_prefill_shared(const LayerShape& sh, const uint16_t* wg, const uint16_t* wu, const uint16_t* wd,
                          const void* x, int x_dtype, int T, void* ws, float* s_out, int* err, int sms,
                          cudaStream_t st) {
  __nv_bfloat16* xb = static_cast<__nv_bfloat16*>(ws);
  __nv_bfloat16* hs = reinterpret_cast<__nv_bfloat16*>(static_cast<char*>(ws) +
                                                       align_up(static_cast<size_t>(T) * sh.H * 2 * 2, 1024));
  int rc = OK;
  if (x_dtype == 0) {
    ProfScope ps(MOE_K_PREP, st);
    bf16_parts_kernel<<<sms * 4, 256, 0, st>>>(static_cast<const float*>(x), static_cast<size_t>(T) * sh.H, xb);
  }
  TcMaps tm;
  {
    ProfScope ps(MOE_K_SHARED_GATEUP, st);
    const int planes = x_dtype == 0 ? 2 : 1;
    const void* xsrc = x_dtype == 0 ? static_cast<const void*>(xb) : x;
    if (!tc_bmaps(&tm, xsrc, true, sh.H, T, planes) || !tc_map(&tm.a0, wg, true, sh.H, sh.Is, 1) ||
        !tc_map(&tm.a1, wu, true, sh.H, sh.Is, 1))
      return ERR_CUDA;
    TcArgs a{};
    a.n_experts = 1; a.b_rows = T;
    a.rows_e = sh.Is; a.K = sh.H; a.mt = sh.Is / kMT; a.planes = planes;
    a.dense_rows = T; a.out = hs; a.ldo = sh.Is; a.out_rows = T;
    a.oscale = 1.0f; a.err = err;
    rc |= launch_tc<TC_BF16_PAIR>(tm, a, sms, st);
  }
  {
    ProfScope ps(MOE_K_SHARED_DOWN, st);
    if (!tc_bmaps(&tm, hs, true, sh.Is, T, 2) || !tc_map(&tm.a0, wd, true, sh.Is, sh.H, 1)) return ERR_CUDA;
    tm.a1 = tm.a0;
    TcArgs a{};
    a.n_experts = 1; a.b_rows = T;
    a.rows_e = sh.H; a.K = sh.Is; a.mt = sh.H / kMT; a.planes = 2;
    a.dense_rows = T; a.out = s_out; a.ldo = sh.H; a.out_rows = T;
    a.oscale = 1.0f; a.err = err;
    rc |= launch_tc<TC_BF16>(tm, a, sms, st);
  }
  if (rc != OK) return ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? OK : ERR_CUDA;
}

}  // namespace moe

namespace moe {
int launch_debug_tc_iq2(const uint8_t* codes, const uint16_t* d, int64_t nblocks, uint16_t* out, cudaStream_t st) {
  const int64_t nsub = nblocks * 8;
  const int grid = static_cast<int>(std::min<int64_t>((nsub + 255) / 256, 4096));
  constexpr int smem = 256 * 128 + 128 * 128;
  cudaFuncSetAttribute(debug_tc_iq2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  debug_tc_iq2_kernel<<<grid, 256, smem, st>>>(codes, d, nsub, reinterpret_cast<uint32_t*>(out));
  return cudaGetLastError() == cudaSuccess ? OK : ERR_CUDA;
}

int launch_debug_tc_q2k(const uint8_t* codes, const uint32_t* dd, int64_t nblocks, uint16_t* out, cudaStream_t st) {
  const int64_t nsub = nblocks * 16;
  const int grid = static_cast<int>(std::min<int64_t>((nsub + 255) / 256, 4096));
  constexpr int smem = 256 * 128;
  debug_tc_q2k_kernel<<<grid, 256, smem, st>>>(codes, dd, nsub, reinterpret_cast<uint32_t*>(out));
  return cudaGetLastError() == cudaSuccess ? OK : ERR_CUDA;
}
}  // namespace moe
