// mxfp4.cu - decode GEMVs for the block-32 routed-expert formats: MXFP4
// (moe_layer_forward_mxfp4) and the Q4-style format (moe_layer_forward_q4);
// the h quantiser that feeds their down projections; the debug decoders.
//
// Source: "ds4 : analyse pratique pour un usage documenté", section « Support
// de modèles et choix de quantification » (an MXFP4 file keeps the routed
// expert weights as published; CUDA Blackwell runs native FP4 matrix
// instructions for batched expert work). Element and scale encodings: OCP
// Microscaling Formats (MX) v1.0 (32 FP4 E2M1 elements, one E8M0 scale).
//
// Operands. Twice an E2M1 value is an integer in [-12, 12], so a block's
// elements enter the same int8 m16n8k32 MMAs as the 2-bit formats, against
// the two int8 digits of the 14-bit activation code; the block's integer dot
// products are exact and are scaled by 2^(E - 128) (the power of two of the
// block, the factor 2 taken back) in fp32. An element code c (sign bit 3,
// magnitude index c & 7) becomes its int8 byte by three byte permutes per four
// elements: one picks from the positive magnitudes, one from the negative
// ones, and one picks between the two by the sign bit.
//
// Work split. A unit is (expert, matrix, 256 rows, one 256-element part kp of
// the reduction axis): one TMA box of 256 rows x 128 code bytes (128-byte
// swizzle) = 8 blocks per row. Each CTA serves one part kp (CTA b takes
// kp = b mod KP) and walks the units of that part with the other CTAs of the
// part, so it stages only that 256-column slice of the activations of every
// token (gate/up) or assignment (down). Lane mapping (lane = 4g + tig): rows g
// and g + 8 of the warp's 16; in round cc (0, 1) the lane owns block 4cc + tig
// of the unit, whole; MMA j takes that block's elements 8j..8j+7 (one 32-bit
// word of nibbles per row). MMA columns are (owner tig, digit hi/lo), so the
// accumulators of lane tig hold exactly its own block: one exact power-of-two
// scale per block and row. Tokens of a unit are taken four at a time, each
// reusing the decoded A operands of the round.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "decode.cuh"
#include "kernels.cuh"
#include "profile.cuh"
#include "ptx.cuh"

namespace moe {
namespace {

constexpr int kMxCW = 16;                     // consumer warps (16 rows each)
constexpr int kMxThreads = (kMxCW + 1) * 32;  // + one producer warp
constexpr int kMxRows = 16 * kMxCW;           // 256 rows per box
constexpr int kMxBoxW = 128;                  // code bytes per box row: 256 elements, 8 blocks
constexpr int kMxBox = kMxRows * kMxBoxW;     // 32 KB
constexpr int kMxPart = 256;                  // elements of the reduction axis per unit
constexpr int kMxZero = 1024;
constexpr int kMxTok = 4;                     // tokens per pass over a unit's decoded operands

// Ring position: stage index and phase parity.
struct RingPos {
  int s;
  uint32_t ph;
  __device__ __forceinline__ void next(int S) {
    if (++s == S) {
      s = 0;
      ph ^= 1u;
    }
  }
};

// Shared-memory loads at 32-bit shared-window addresses (volatile: they stay after the mbarrier wait).
__device__ __forceinline__ uint4 ld_s128_mx(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ float ld_sf_mx(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}

// The two block-32 formats of this file: MXFP4 (E2M1 elements, E8M0 scale
// byte per block) and the Q4-style format (unsigned 4-bit codes q, fp16 scale
// d per block, w = d (q - 8)). Both decode a 4-bit code c by its low three bits
// from one of two 8-entry byte tables, chosen by bit 3:
//   MXFP4: bit 3 = sign; int8 = 2 * E2M1 value (0 1 2 3 4 6 8 12, negated)
//   Q4:    bit 3 = q >= 8; int8 = q - 8 (-8 .. -1, 0 .. 7)
enum BlkFmt : int { FMT_MXFP4 = 0, FMT_Q4 = 1 };
template <int FMT> struct BlkTab;
template <> struct BlkTab<FMT_MXFP4> {
  static constexpr uint32_t t0 = 0x03020100u, t1 = 0x0C080604u;  // bit 3 clear: 0 1 2 3 | 4 6 8 12
  static constexpr uint32_t u0 = 0xFDFEFF00u, u1 = 0xF4F8FAFCu;  // bit 3 set:  0 -1 -2 -3 | -4 -6 -8 -12
};
template <> struct BlkTab<FMT_Q4> {
  static constexpr uint32_t t0 = 0xFBFAF9F8u, t1 = 0xFFFEFDFCu;  // q 0..7:  -8 .. -1
  static constexpr uint32_t u0 = 0x03020100u, u1 = 0x07060504u;  // q 8..15:  0 .. 7
};

// Eight codes (one 32-bit word, element i in nibble i) -> two int8x4 operand
// registers: elements 0..3 and 4..7.
template <int FMT>
__device__ __forceinline__ void blk_decode8(uint32_t w, uint32_t& lo, uint32_t& hi) {
  using TB = BlkTab<FMT>;
  const uint32_t mag = w & 0x77777777u;
  // byte i of the result comes from byte i of the first pick (selector i) or of the second (i + 4)
  const uint32_t sel = ((w >> 1) & 0x44444444u) | 0x32103210u;
  const uint32_t maghi = __umulhi(mag, 0x10000u), selhi = __umulhi(sel, 0x10000u);
  lo = prmt(prmt(TB::t0, TB::t1, mag), prmt(TB::u0, TB::u1, mag), sel);
  hi = prmt(prmt(TB::t0, TB::t1, maghi), prmt(TB::u0, TB::u1, maghi), selhi);
}

// 2^(E - 128) exactly, for every byte E (subnormal for E < 2).
__device__ __forceinline__ float mx_pow2(uint32_t E) {
  return E >= 2u ? __uint_as_float((E - 1u) << 23) : __uint_as_float(0x00200000u << E);
}

// Mixed-radix walk over units v = v0, v0 + dv, ...: v = (slot * M + m) * rbs + rb.
struct UnitIt {
  int rb, m, slot, drb, dm, dslot;
  __device__ __forceinline__ void init(int v0, int dv, int rbs, int M) {
    rb = v0 % rbs;
    int q = v0 / rbs;
    m = q % M;
    slot = q / M;
    drb = dv % rbs;
    q = dv / rbs;
    dm = q % M;
    dslot = q / M;
  }
  __device__ __forceinline__ void next(int rbs, int M) {
    rb += drb;
    int c = rb >= rbs ? 1 : 0;
    rb -= c * rbs;
    m += dm + c;
    c = m >= M ? 1 : 0;
    m -= c * M;
    slot += dslot + c;
  }
};

struct MxArgs {
  int K, R, E, k, KP, S, pair, nrows, nA;
  const void* sc0;      // scale planes [E][R][K/32]: E8M0 bytes (MXFP4) or fp16 (Q4); gate or the single
  const void* sc1;      // matrix, and up
  const int8_t* ad;     // activation digits [nrows][2][K], natural order
  const float* as;      // their scales [nrows][K/256] (2^s / 8)
  const int32_t* offsets;
  const int32_t* active;
  const int32_t* perm;
  float* part;          // pair: [nA][2][KP][R]; single: [nA][KP][R]
  size_t part_n;
  int* err;
};

struct MxPlan {
  size_t meta, zero, act, as, ring, bars, total;
};
__host__ __device__ inline MxPlan mx_plan(int E, int nA, int nrows, int S) {
  MxPlan p;
  p.meta = 0;
  p.zero = align_up(static_cast<size_t>(2 * (E + 1) + nA) * 4, 128);
  p.act = p.zero + kMxZero;
  p.as = p.act + static_cast<size_t>(nrows) * 2 * kMxPart;
  p.ring = align_up(p.as + align_up(static_cast<size_t>(nrows) * 4, 128), 1024);
  p.bars = p.ring + static_cast<size_t>(S) * kMxBox;
  p.total = p.bars + 2 * static_cast<size_t>(S) * 8;
  return p;
}

template <int FMT>
__global__ void __launch_bounds__(kMxThreads, 1) mx_gemv_kernel(const __grid_constant__ CUtensorMap tm0,
                                                               const __grid_constant__ CUtensorMap tm1, MxArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  pdl_trigger();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int K = a.K, R = a.R, S = a.S, KP = a.KP, M = a.pair ? 2 : 1, rbs = R / kMxRows;
  const MxPlan pl = mx_plan(a.E, a.nA, a.nrows, S);
  int32_t* off = reinterpret_cast<int32_t*>(smem + pl.meta);
  int32_t* act = off + (a.E + 1);
  int32_t* arow = act + (a.E + 1);  // activation row of each expert-sorted assignment
  int8_t* zero = reinterpret_cast<int8_t*>(smem + pl.zero);
  int8_t* acts = reinterpret_cast<int8_t*>(smem + pl.act);
  float* ass = reinterpret_cast<float*>(smem + pl.as);
  uint8_t* ring = smem + pl.ring;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + pl.bars);
  uint64_t* empty = full + S;
  // this CTA's part of the reduction axis and its place among the CTAs of that part
  const int kpc = static_cast<int>(blockIdx.x % KP), kib = static_cast<int>(blockIdx.x / KP);
  const int kG = static_cast<int>((gridDim.x - kpc + KP - 1) / KP);

  if ((smem_addr(ring) & 1023u) != 0) {  // the 128-byte swizzle assumes 1024-byte aligned boxes
    if (tid == 0) atomicCAS(a.err, 0, ERR_CUDA);
    return;
  }
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kMxCW);
    }
    fence_barrier_init();
  }
  for (int i = tid; i < kMxZero / 16; i += kMxThreads) reinterpret_cast<uint4*>(zero)[i] = make_uint4(0, 0, 0, 0);
  pdl_wait();  // routing and activations come from the kernels before this one
  for (int i = tid; i <= a.E; i += kMxThreads) {
    off[i] = a.offsets[i];
    act[i] = a.active[i];
  }
  for (int i = tid; i < a.nA; i += kMxThreads) arow[i] = a.pair ? a.perm[i] / a.k : i;
  __syncthreads();
  const int nact = act[a.E];

  if (warp == kMxCW) {  // producer
    if (lane == 0) {
      prefetch_tmap(&tm0);
      if (a.pair) prefetch_tmap(&tm1);
      const uint64_t pol = l2_policy_evict_first();  // expert codes are read once per step
      RingPos rp{0, 0u};
      UnitIt it;
      it.init(kib, kG, rbs, M);
      for (; it.slot < nact; it.next(rbs, M)) {
        const int e = act[it.slot];
        if (!mbar_wait_bounded(&empty[rp.s], rp.ph ^ 1u, a.err, ERR_TIMEOUT)) return;
        mbar_arrive_expect_tx(&full[rp.s], kMxBox);
        tma_load_2d_hint(ring + rp.s * kMxBox, it.m ? &tm1 : &tm0, kpc * kMxBoxW, e * R + it.rb * kMxRows,
                         &full[rp.s], pol);
        rp.next(S);
      }
    }
    return;
  }

  // consumers: the 256-column slice [kpc 256, kpc 256 + 256) of every activation row, in the x_off layout of a
  // 256-column matrix, and its scale; asynchronously, while the first boxes are in flight
  for (int i = tid; i < a.nrows * 32; i += kMxCW * 32) {
    const int row = i >> 5, d = (i >> 4) & 1, c = i & 15;
    cp_async16(smem_addr(acts + x_off(kMxPart, row, d, 16 * c)),
               a.ad + (static_cast<size_t>(row) * 2 + d) * K + static_cast<size_t>(kpc) * kMxPart + 16 * c);
  }
  for (int i = tid; i < a.nrows; i += kMxCW * 32) ass[i] = a.as[static_cast<size_t>(i) * (K / kMxPart) + kpc] * 8.f;
  cp_async_wait_all();
  named_barrier(1, kMxCW * 32);

  const int g = lane >> 2, tig = lane & 3;
  const bool bact = (g >> 1) == tig;  // this lane carries B: digit g & 1 of its column's block
  const int row_l = 16 * warp + g;
  // this lane's block of round cc in a stage, rows g and g + 8 (128-byte swizzle: chunk ^ (row & 7))
  const uint32_t rec0 = smem_addr(ring) + static_cast<uint32_t>(row_l) * kMxBoxW;
  const uint32_t ch0 = static_cast<uint32_t>(tig ^ (row_l & 7)), ch1 = static_cast<uint32_t>((4 + tig) ^ (row_l & 7));
  // B of round cc for activation row r: block 4cc + tig of the slice (non-carrying lanes read zeros)
  const uint32_t acts_s = smem_addr(acts), zero_s = smem_addr(zero);
  const uint32_t ass_s = smem_addr(ass);
  const int spr = K / 32;  // scale bytes per row
  RingPos rp{0, 0u};
  // this CTA's units v = kib, kib + kG, ... as a mixed-radix counter (rb fastest, then m, then slot)
  UnitIt it;
  it.init(kib, kG, rbs, M);
  // the scales of a unit, rows g and g + 8 (MXFP4: 8 bytes per row; Q4: 8 fp16 per row), loaded one unit
  // ahead so that their latency is hidden behind the previous unit
  auto ldsc = [&](const UnitIt& u, uint4& s0v, uint4& s8v) {
    const int eu = act[u.slot];
    const size_t sidx = (static_cast<size_t>(eu) * R + u.rb * kMxRows + row_l) * spr + kpc * 8;
    if (FMT == FMT_MXFP4) {
      const uint8_t* scp = static_cast<const uint8_t*>(u.m ? a.sc1 : a.sc0) + sidx;
      const uint2 v0 = __ldg(reinterpret_cast<const uint2*>(scp));
      const uint2 v8 = __ldg(reinterpret_cast<const uint2*>(scp + 8 * static_cast<size_t>(spr)));
      s0v = make_uint4(v0.x, v0.y, 0u, 0u);
      s8v = make_uint4(v8.x, v8.y, 0u, 0u);
    } else {
      const uint16_t* scp = static_cast<const uint16_t*>(u.m ? a.sc1 : a.sc0) + sidx;
      s0v = __ldg(reinterpret_cast<const uint4*>(scp));
      s8v = __ldg(reinterpret_cast<const uint4*>(scp + 8 * static_cast<size_t>(spr)));
    }
  };
  uint4 nsg0 = make_uint4(0u, 0u, 0u, 0u), nsg8 = nsg0;
  if (it.slot < nact) ldsc(it, nsg0, nsg8);
  while (it.slot < nact) {
    const int rb = it.rb, m = it.m;
    const int e = act[it.slot];
    const int p0 = off[e], ne = off[e + 1] - p0;
    const uint4 sg0 = nsg0, sg8 = nsg8;
    it.next(rbs, M);
    if (it.slot < nact) ldsc(it, nsg0, nsg8);
    if (!mbar_wait_bounded(&full[rp.s], rp.ph, a.err, ERR_TIMEOUT)) return;
    const uint32_t st = rec0 + static_cast<uint32_t>(rp.s) * kMxBox;
    const uint4 ra0 = ld_s128_mx(st + 16u * ch0), rb0 = ld_s128_mx(st + 8u * kMxBoxW + 16u * ch0);
    const uint4 ra1 = ld_s128_mx(st + 16u * ch1), rb1 = ld_s128_mx(st + 8u * kMxBoxW + 16u * ch1);
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[rp.s]);  // the codes are in registers: the stage is free
    rp.next(S);
    const uint32_t wa[2][4] = {{ra0.x, ra0.y, ra0.z, ra0.w}, {ra1.x, ra1.y, ra1.z, ra1.w}};
    const uint32_t wb[2][4] = {{rb0.x, rb0.y, rb0.z, rb0.w}, {rb1.x, rb1.y, rb1.z, rb1.w}};
    // the scale factors of this lane's blocks (tig and 4 + tig), rows g and g + 8: MXFP4 2^(E - 128)
    // (the elements enter doubled), Q4 d
    float s0[2], s8[2];
    if (FMT == FMT_MXFP4) {
      s0[0] = mx_pow2((sg0.x >> (8 * tig)) & 0xFFu);
      s0[1] = mx_pow2((sg0.y >> (8 * tig)) & 0xFFu);
      s8[0] = mx_pow2((sg8.x >> (8 * tig)) & 0xFFu);
      s8[1] = mx_pow2((sg8.y >> (8 * tig)) & 0xFFu);
    } else {
      // fp16 of block b is half b & 1 of word b >> 1: blocks tig (words 0, 1) and 4 + tig (words 2, 3)
      const bool hw = (tig >> 1) != 0;
      const uint32_t sh = 16u * (tig & 1);
      s0[0] = half_bits_to_float(static_cast<uint16_t>((hw ? sg0.y : sg0.x) >> sh));
      s0[1] = half_bits_to_float(static_cast<uint16_t>((hw ? sg0.w : sg0.z) >> sh));
      s8[0] = half_bits_to_float(static_cast<uint16_t>((hw ? sg8.y : sg8.x) >> sh));
      s8[1] = half_bits_to_float(static_cast<uint16_t>((hw ? sg8.w : sg8.z) >> sh));
    }
    for (int t0 = 0; t0 < ne; t0 += kMxTok) {
      float f0[kMxTok], f1[kMxTok];
      int ar[kMxTok];
#pragma unroll
      for (int t = 0; t < kMxTok; ++t) {
        f0[t] = f1[t] = 0.f;
        ar[t] = t0 + t < ne ? arow[p0 + t0 + t] : -1;
      }
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t A[4][4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          blk_decode8<FMT>(wa[cc][j], A[j][0], A[j][2]);  // row g: elements 8j..8j+3, 8j+4..8j+7
          blk_decode8<FMT>(wb[cc][j], A[j][1], A[j][3]);  // row g + 8
        }
#pragma unroll
        for (int t = 0; t < kMxTok; ++t) {
          if (ar[t] < 0) break;
          const uint32_t xb = bact ? acts_s + static_cast<uint32_t>(x_off(kMxPart, ar[t], g & 1, (4 * cc + tig) * 32))
                                   : zero_s;
          const uint4 bx0 = ld_s128_mx(xb), bx1 = ld_s128_mx(xb ^ 16u);
          const uint32_t bv[8] = {bx0.x, bx0.y, bx0.z, bx0.w, bx1.x, bx1.y, bx1.z, bx1.w};
          int acc[4];
          mma_s8s8_zero(acc, A[0][0], A[0][1], A[0][2], A[0][3], bv[0], bv[1]);
          mma_s8s8(acc, A[1][0], A[1][1], A[1][2], A[1][3], bv[2], bv[3]);
          mma_s8s8(acc, A[2][0], A[2][1], A[2][2], A[2][3], bv[4], bv[5]);
          mma_s8s8(acc, A[3][0], A[3][1], A[3][2], A[3][3], bv[6], bv[7]);
          // this lane's columns: its own block, digits hi and lo, rows g and g + 8
          f0[t] = fmaf(static_cast<float>(acc[0] * 128 + acc[1]), s0[cc], f0[t]);
          f1[t] = fmaf(static_cast<float>(acc[2] * 128 + acc[3]), s8[cc], f1[t]);
        }
      }
#pragma unroll
      for (int t = 0; t < kMxTok; ++t) {
        if (ar[t] < 0) break;
        const float xsv = ld_sf_mx(ass_s + 4u * static_cast<uint32_t>(ar[t]));
        float v0 = f0[t] * xsv, v1 = f1[t] * xsv;
        // the four lanes of a quad hold the four blocks of each round: add them in a fixed order
        v0 += __shfl_xor_sync(0xffffffffu, v0, 1);
        v0 += __shfl_xor_sync(0xffffffffu, v0, 2);
        v1 += __shfl_xor_sync(0xffffffffu, v1, 1);
        v1 += __shfl_xor_sync(0xffffffffu, v1, 2);
        if (tig == 0) {
          const int p = p0 + t0 + t;
          const size_t o = (a.pair ? (static_cast<size_t>(p) * 2 + m) : static_cast<size_t>(p)) * KP * R +
                           static_cast<size_t>(kpc) * R + rb * kMxRows + row_l;
          if (o + 8 < a.part_n) {
            a.part[o] = v0;
            a.part[o + 8] = v1;
          }
        }
      }
    }
  }
}

// h for MXFP4 down projections: per assignment p and 256-element block sb of I,
// g and u are the sums of the KP gate/up part rows (warp w adds parts w, w+8,
// ... in order, then the warps' sums in warp order), h = silu(g) * u, and h is
// written as the activation digits of x_digits_kernel (14-bit code, natural
// order [nA][2][I], scale 2^(s-3) per block).
__global__ void __launch_bounds__(256) mx_hquant_kernel(int I, int KP, const float* __restrict__ gu,
                                                        int8_t* __restrict__ hd, float* __restrict__ hs) {
  __shared__ float4 red[8][4][32];
  pdl_trigger();
  pdl_wait();
  const int p = blockIdx.x, sb = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float* g = gu + static_cast<size_t>(p) * 2 * KP * I + sb * 256 + lane * 8;
  const float* u = g + static_cast<size_t>(KP) * I;
  float4 s4[4] = {make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f),
                  make_float4(0.f, 0.f, 0.f, 0.f)};
  for (int kp = warp; kp < KP; kp += 8) {
    const float4 v0 = __ldcg(reinterpret_cast<const float4*>(g + static_cast<size_t>(kp) * I));
    const float4 v1 = __ldcg(reinterpret_cast<const float4*>(g + static_cast<size_t>(kp) * I + 4));
    const float4 v2 = __ldcg(reinterpret_cast<const float4*>(u + static_cast<size_t>(kp) * I));
    const float4 v3 = __ldcg(reinterpret_cast<const float4*>(u + static_cast<size_t>(kp) * I + 4));
    s4[0].x += v0.x; s4[0].y += v0.y; s4[0].z += v0.z; s4[0].w += v0.w;
    s4[1].x += v1.x; s4[1].y += v1.y; s4[1].z += v1.z; s4[1].w += v1.w;
    s4[2].x += v2.x; s4[2].y += v2.y; s4[2].z += v2.z; s4[2].w += v2.w;
    s4[3].x += v3.x; s4[3].y += v3.y; s4[3].z += v3.z; s4[3].w += v3.w;
  }
#pragma unroll
  for (int q = 0; q < 4; ++q) red[warp][q][lane] = s4[q];
  __syncthreads();
  if (warp != 0) return;
  float gv[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f}, uv[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int w = 0; w < 8; ++w) {
    const float4 ra = red[w][0][lane], rb = red[w][1][lane], rc = red[w][2][lane], rd = red[w][3][lane];
    gv[0] += ra.x; gv[1] += ra.y; gv[2] += ra.z; gv[3] += ra.w; gv[4] += rb.x; gv[5] += rb.y; gv[6] += rb.z; gv[7] += rb.w;
    uv[0] += rc.x; uv[1] += rc.y; uv[2] += rc.z; uv[3] += rc.w; uv[4] += rd.x; uv[5] += rd.y; uv[6] += rd.z; uv[7] += rd.w;
  }
  float h[8], mx = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    h[i] = silu_mul(gv[i], uv[i]);
    mx = fmaxf(mx, fabsf(h[i]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  const int s = mx > 0.f ? floor_log2_pos(mx) - 12 : 0;  // 14-bit code, |q| <= 8192
  uint32_t hw[2] = {0, 0}, lw[2] = {0, 0};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    int hi = 0, lo = 0;
    if (mx > 0.f) split_digits(h[i], s, hi, lo);
    hw[i / 4] |= (static_cast<uint32_t>(hi) & 0xFFu) << (8 * (i % 4));
    lw[i / 4] |= (static_cast<uint32_t>(lo) & 0xFFu) << (8 * (i % 4));
  }
  int8_t* row = hd + static_cast<size_t>(p) * 2 * I + sb * 256 + lane * 8;
  *reinterpret_cast<uint2*>(row) = make_uint2(hw[0], hw[1]);
  *reinterpret_cast<uint2*>(row + I) = make_uint2(lw[0], lw[1]);
  if (lane == 0) hs[static_cast<size_t>(p) * (I / 256) + sb] = mx > 0.f ? ldexpf(1.0f, s - 3) : 0.f;
}

// Debug decoder: one thread per block, the kernels' element decoding.
template <int FMT>
__global__ void mx_dequant_kernel(const uint8_t* __restrict__ codes, const void* __restrict__ scales, int64_t nb,
                                  float* __restrict__ out) {
  for (int64_t b = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; b < nb;
       b += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float sc = FMT == FMT_MXFP4 ? mx_pow2(static_cast<const uint8_t*>(scales)[b])
                                      : half_bits_to_float(static_cast<const uint16_t*>(scales)[b]);
    for (int w = 0; w < 4; ++w) {
      const uint32_t word = *reinterpret_cast<const uint32_t*>(codes + b * 16 + 4 * w);
      uint32_t lo, hi;
      blk_decode8<FMT>(word, lo, hi);
      for (int i = 0; i < 8; ++i) {
        const int8_t v = static_cast<int8_t>(((i < 4 ? lo : hi) >> (8 * (i & 3))) & 0xFFu);
        out[b * 32 + 8 * w + i] = static_cast<float>(v) * sc;
      }
    }
  }
}

PFN_cuTensorMapEncodeTiled_v12000 mx_encode_fn() {
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

// codes [rows][row_bytes] with boxes of 256 rows x 128 bytes, 128-byte swizzle
bool mx_map(CUtensorMap* m, const void* base, uint64_t row_bytes, uint64_t rows) {
  auto fn = mx_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {row_bytes, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {kMxBoxW, kMxRows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr size_t kMxBudget = 227 * 1024;

}  // namespace

bool mx_path_supported(const LayerShape& s, int T) {
  return s.H % 512 == 0 && s.I % 512 == 0 && T >= 1 && T <= 16 && s.E <= 1024 &&
         static_cast<size_t>(T) * s.k <= 256 && mx_encode_fn() != nullptr &&
         mx_plan(s.E, T * s.k, T * s.k, 2).total <= kMxBudget;
}

int mx_parts(int K) { return K / kMxPart; }

// One MXFP4 GEMV launch: pair = gate + up over the token rows of x digits (partials [nA][2][KP][R]),
// else the single (down) matrix over the assignment rows of h digits (partials [nA][KP][R]).
int launch_mx_gemv(int fmt, bool pair, int K, int R, int E, int k, int T, const uint8_t* codes0, const void* sc0,
                   const uint8_t* codes1, const void* sc1, const int8_t* ad, const float* as,
                   const Routing& r, float* part, int* err, int sms, cudaStream_t st) {
  const int nA = T * k, nrows = pair ? T : nA;
  CUtensorMap t0, t1;
  const uint64_t rows = static_cast<uint64_t>(E) * R;
  if (!mx_map(&t0, codes0, static_cast<uint64_t>(K) / 2, rows)) return ERR_CUDA;
  if (pair ? !mx_map(&t1, codes1, static_cast<uint64_t>(K) / 2, rows) : false) return ERR_CUDA;
  if (!pair) t1 = t0;
  MxArgs a{};
  a.K = K; a.R = R; a.E = E; a.k = k; a.KP = K / kMxPart; a.pair = pair ? 1 : 0; a.nrows = nrows; a.nA = nA;
  a.sc0 = sc0; a.sc1 = pair ? sc1 : sc0; a.ad = ad; a.as = as;
  a.offsets = r.offsets; a.active = r.active; a.perm = r.perm;
  a.part = part; a.part_n = static_cast<size_t>(nA) * (pair ? 2 : 1) * a.KP * R; a.err = err;
  int S = 2;
  while (S < 6 && mx_plan(E, nA, nrows, S + 1).total <= kMxBudget) ++S;
  const size_t smem = mx_plan(E, nA, nrows, S).total;
  if (smem > kMxBudget) return ERR_SHAPE;
  a.S = S;
  const int slots = std::min(nA, E);
  const int units = slots * (pair ? 2 : 1) * (R / kMxRows) * a.KP;
  const int grid = std::max(a.KP, std::min(units, sms));
  if (fmt == FMT_MXFP4) {
    cudaFuncSetAttribute(mx_gemv_kernel<FMT_MXFP4>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    launch_pdl(mx_gemv_kernel<FMT_MXFP4>, dim3(grid), dim3(kMxThreads), smem, st, t0, t1, a);
  } else if (fmt == FMT_Q4) {
    cudaFuncSetAttribute(mx_gemv_kernel<FMT_Q4>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    launch_pdl(mx_gemv_kernel<FMT_Q4>, dim3(grid), dim3(kMxThreads), smem, st, t0, t1, a);
  } else {
    return ERR_ARG;
  }
  return cudaGetLastError() == cudaSuccess ? OK : ERR_CUDA;
}

int launch_mx_hquant(int I, int KP, int nA, const float* gu, int8_t* hd, float* hs, cudaStream_t st) {
  launch_pdl(mx_hquant_kernel, dim3(nA, I / 256), dim3(256), 0, st, I, KP, gu, hd, hs);
  return cudaGetLastError() == cudaSuccess ? OK : ERR_CUDA;
}

int launch_mx_dequant(int fmt, const uint8_t* codes, const void* scales, int64_t nb, float* out, cudaStream_t st) {
  if (nb <= 0) return OK;
  const int grid = static_cast<int>(std::min<int64_t>((nb + 255) / 256, 4096));
  if (fmt == FMT_MXFP4)
    mx_dequant_kernel<FMT_MXFP4><<<grid, 256, 0, st>>>(codes, scales, nb, out);
  else if (fmt == FMT_Q4)
    mx_dequant_kernel<FMT_Q4><<<grid, 256, 0, st>>>(codes, scales, nb, out);
  else
    return ERR_ARG;
  return cudaGetLastError() == cudaSuccess ? OK : ERR_CUDA;
}

}  // namespace moe
