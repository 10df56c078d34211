// gemv_tma.cu - decode dequant-GEMVs of the routed experts fed by 2-D TMA
// tensor-map loads, with warp specialisation: one producer warp streams boxes
// of code rows into a ring of shared-memory stages (full/empty mbarriers, all
// waits bounded), sixteen consumer warps each own 16 rows and turn the codes
// into int8 MMA operands. No block-wide barrier inside the main loop.
//
// Sources: "ds4 : analyse pratique pour un usage documenté", section « Support
// de modèles et choix de quantification » (up/gate IQ2_XXS, down Q2_K). The
// operand construction and the integer accumulation are those of decode.cuh.
//
// Work is split into equal units so that every SM gets the same number: a
// gate/up unit is (expert, gate or up, 256 rows, NB boxes of 512 of H) and a
// down unit is (expert, 256 rows of H, NB blocks of 256 of I), NB = 1 for a
// single token and 2 otherwise (fewer partial sums to keep). Each unit writes
// partial sums that the next kernel adds up in a fixed order.
//
// Routing metadata (offsets, active experts, token of each assignment) is
// copied to shared memory once per CTA; units are walked with a mixed-radix
// counter (no integer division in the loop), and the per-row fp16 scales of
// the next unit are loaded one unit ahead, so no dependent global load sits
// on the critical path of a unit.
//
// When the activations fit, they are staged in shared memory with rows padded
// by 32 bytes, and the zero operand region is placed 64 bytes further, so the
// hi-digit row, the lo-digit row and the zeros that one MMA's B operand reads
// fall in different banks.
//
// gate/up boxes: 256 rows x 128 code bytes (16 sub-blocks), 128-byte swizzle,
//   so the eight rows a quad column reads together land in eight different
//   16-byte bank groups. down boxes: 256 rows x 80 code bytes (one block),
//   dense; the 80-byte pitch maps eight consecutive rows to eight different
//   16-byte bank groups as well.
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

__device__ const Iq2SelTables d_sel_tables2 = make_sel_tables();

constexpr int kCW = 16;                      // consumer warps (16 rows each)
constexpr int kThreadsT = (kCW + 1) * 32;    // + one producer warp
constexpr int kBoxRows = 16 * kCW;           // 256 rows per box
constexpr int kGuW = 128;                    // code bytes per gate/up box row (512 weights)
constexpr int kGuBox = kBoxRows * kGuW;      // 32 KB
constexpr int kDnW = 80;                     // one Q2K-style block per down box row
constexpr int kDnBox = kBoxRows * kDnW;      // 20 KB
// Selector tables, each entry replicated for the 32 lanes: grid row i at byte
// 256*i + 4*lane, sign field s at byte 256*s + 128 + 4*lane (interleaved, so
// that one prmt turns a grid index byte into its table address).
constexpr int kTabBytes = 256 * 256;
constexpr int kZeroBytes = 1024;             // zero operand region for idle MMA columns
constexpr int kRowPad = 32;                  // padding of a staged activation row
constexpr int kMaxExpertsTma = 1024;
constexpr int kMaxNB = 2;

// Zero operand for the variants that read activations from global memory.
__device__ __align__(128) const int8_t g_zero_operand[kZeroBytes] = {};

__device__ __forceinline__ uint32_t rotr(uint32_t v, uint32_t n) { return __funnelshift_r(v, v, n); }

__device__ __forceinline__ uint4 lds128(const uint8_t* p) { return *reinterpret_cast<const uint4*>(p); }

// Loads from shared memory at 32-bit shared-window addresses. They are volatile
// so that they stay after the mbarrier wait that makes the data visible.
__device__ __forceinline__ uint4 ld_s128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ uint2 ld_s64(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t ld_s32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t ld_s8(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u8 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ float ld_sf(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
  return v;
}

__host__ __device__ inline size_t meta_bytes(int E, int nA, bool with_tok) {
  return align_up(static_cast<size_t>(2 * (E + 1) + (with_tok ? nA : 0)) * 4, 128);
}

// Routing metadata in shared memory.
struct MetaSmem {
  int32_t* off;  // [E+1]
  int32_t* act;  // [E+1], act[E] = number of active experts
  int32_t* tok;  // [T*k] token of each expert-sorted assignment (gate/up only)
};

__device__ __forceinline__ void load_meta(const MetaSmem& m, const int32_t* offsets, const int32_t* active,
                                          const int32_t* perm, int E, int nA, int k, int tid, int nthr) {
  for (int i = tid; i <= E; i += nthr) {
    m.off[i] = offsets[i];
    m.act[i] = active[i];
  }
  if (m.tok)
    for (int i = tid; i < nA; i += nthr) m.tok[i] = perm[i] / k;
}

// Copy rows of `row_bytes` (a multiple of 16) from global memory into shared
// memory with a row pitch of row_bytes + kRowPad.
__device__ __forceinline__ void stage_rows(int8_t* dst, const int8_t* src, int rows, int row_bytes, int tid,
                                           int nthr) {
  const int per = row_bytes / 16;
  for (int i = tid; i < rows * per; i += nthr) {
    const int r = i / per, cidx = i - r * per;
    *reinterpret_cast<uint4*>(dst + static_cast<size_t>(r) * (row_bytes + kRowPad) + cidx * 16) =
        reinterpret_cast<const uint4*>(src)[i];
  }
}

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

// ===========================================================================
// gate/up
// ===========================================================================
struct GuTmaArgs {
  int H, I, E, k, T, KP, NB, S;
  const uint16_t* gate_d;
  const uint16_t* up_d;
  const int8_t* xd;
  const float* xs;
  const int32_t* offsets;
  const int32_t* perm;
  const int32_t* active;
  float* gpart;  // [T*k][2][KP][I]
  int* err;
};

// Unit u = ((slot * 2 + m) * rbs + rb) * KP + kp, walked in steps of gridDim.x.
struct GuIter {
  int kp, rb, m, slot, dkp, drb, dm, dslot;
  __device__ __forceinline__ void init(int u0, int G, int KP, int rbs) {
    kp = u0 % KP;
    int r = u0 / KP;
    rb = r % rbs;
    r /= rbs;
    m = r & 1;
    slot = r >> 1;
    dkp = G % KP;
    r = G / KP;
    drb = r % rbs;
    r /= rbs;
    dm = r & 1;
    dslot = r >> 1;
  }
  __device__ __forceinline__ void next(int KP, int rbs) {
    kp += dkp;
    int c = kp >= KP ? 1 : 0;
    kp -= c * KP;
    rb += drb + c;
    c = rb >= rbs ? 1 : 0;
    rb -= c * rbs;
    m += dm + c;
    c = m >= 2 ? 1 : 0;
    m -= 2 * c;
    slot += dslot + c;
  }
};

struct GuUnit {
  int e, m, rb, kp, p0, ne;
};

__device__ __forceinline__ GuUnit gu_unit_of(const GuIter& t, const MetaSmem& ms) {
  GuUnit w;
  w.kp = t.kp;
  w.rb = t.rb;
  w.m = t.m;
  w.e = ms.act[t.slot];
  w.p0 = ms.off[w.e];
  w.ne = ms.off[w.e + 1] - w.p0;
  return w;
}

struct GuCtx {
  const char* tab;      // interleaved level and sign tables (start of dynamic shared memory)
  const uint8_t* ring;
  uint64_t* full;
  uint64_t* empty;
  const int8_t* xdig;   // rows (token, digit hi/lo) of H digits, pitch xpitch
  const float* xscl;    // [T][H/256] 2^s / 8
  const int8_t* zero;   // 128-byte aligned zero region
  const int32_t* tok;
  uint32_t ring_s, x_s, xs_s, zero_s;  // shared-window addresses (staged variant)
  int xpitch, warp, lane, g, tig, S;
  uint32_t lane4, sel_idx, rot_sig, sgn_lane;
};

// Selector word (level nibbles | sign bits) of grid group `tig` of one 8-byte
// sub-block record -> two int8x4 A registers.
__device__ __forceinline__ void iq2_operand(const GuCtx& c, uint2 rec, uint32_t& lo, uint32_t& hi) {
  const uint32_t al = prmt(rec.x, c.lane4, c.sel_idx);                  // 256 * index byte + 4 * lane
  const uint32_t as = (rotr(rec.y, c.rot_sig) & 0x7F00u) | c.sgn_lane;  // 256 * sign field + 128 + 4 * lane
  // level codes sit in bits 0-1 of each nibble and signs in bit 2: the sum is the union
  const uint32_t sel = *reinterpret_cast<const uint32_t*>(c.tab + al) + *reinterpret_cast<const uint32_t*>(c.tab + as);
  lo = prmt(kPosBytes, kNegBytes, sel);
  hi = prmt(kPosBytes, kNegBytes, __umulhi(sel, 0x10000u));
}

// The eight records (four sub-blocks x rows g, g+8) of chunk pair cc.
__device__ __forceinline__ void gu_records(const uint8_t* rg, int cc, int g, uint2 (&rec)[4][2]) {
  const uint4 a0 = lds128(rg + (((2 * cc) ^ g) << 4));
  const uint4 a1 = lds128(rg + (((2 * cc + 1) ^ g) << 4));
  const uint4 b0 = lds128(rg + 1024 + (((2 * cc) ^ g) << 4));
  const uint4 b1 = lds128(rg + 1024 + (((2 * cc + 1) ^ g) << 4));
  rec[0][0] = make_uint2(a0.x, a0.y); rec[1][0] = make_uint2(a0.z, a0.w);
  rec[2][0] = make_uint2(a1.x, a1.y); rec[3][0] = make_uint2(a1.z, a1.w);
  rec[0][1] = make_uint2(b0.x, b0.y); rec[1][1] = make_uint2(b0.z, b0.w);
  rec[2][1] = make_uint2(b1.x, b1.y); rec[3][1] = make_uint2(b1.z, b1.w);
}

// 2*ls+1 of sub-block sb (0..15) of the row at rg (swizzled 128-byte row).
__device__ __forceinline__ int gu_odd(const uint8_t* rg, int sb, int g) {
  const uint32_t b = rg[(((sb >> 1) ^ g) << 4) + (sb & 1) * 8 + 7];
  return static_cast<int>((b >> 3) | 1u);
}

__device__ __forceinline__ float half_lo(uint32_t w) { return half_bits_to_float(static_cast<uint16_t>(w & 0xFFFFu)); }
__device__ __forceinline__ float half_hi(uint32_t w) { return half_bits_to_float(static_cast<uint16_t>(w >> 16)); }

// One unit whose expert holds a single assignment (every decode step with one
// token), activations staged in shared memory. MMA columns: (sub-block slot
// 0..3) x (digit hi, lo); the B operand of an idle column comes from the zero
// region, so no select is needed. All shared-memory addresses are 32-bit and
// the 128-byte swizzle is applied with one XOR per 16-byte chunk: with
// rgg = row base + 16*g, logical chunk L of row g sits at rgg ^ (16*L).
__device__ __forceinline__ bool gu_unit_one(const GuTmaArgs& a, const GuCtx& c, RingPos& rp, const GuUnit& w,
                                            const uint32_t (&dp)[kMaxNB][2]) {
  const int H = a.H, I = a.I, NB = a.NB;
  const int g = c.g, tig = c.tig;
  const int tok = c.tok[w.p0];
  const int row_l = 16 * c.warp + g;
  const uint32_t xrow = c.x_s + (tok * 2 + (g & 1)) * c.xpitch + w.kp * NB * 512 + 8 * tig;
  const uint32_t zrow = c.zero_s + ((64 * (tok & 1) + 64) & 127) + 8 * tig;
  const uint32_t xsc = c.xs_s + (tok * (H / 256) + 2 * NB * w.kp) * 4;
  const uint32_t lsoff = ((((tig >> 1) ^ g)) << 4) + (tig & 1) * 8 + 7;
  float f0 = 0.f, f1 = 0.f;
#pragma unroll 1
  for (int j = 0; j < NB; ++j) {
    uint32_t bp[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) bp[u] = ((g >> 1) == u) ? xrow + j * 512 : zrow;
    if (!mbar_wait_bounded(&c.full[rp.s], rp.ph, a.err, ERR_TIMEOUT)) return false;
    const uint32_t rg = c.ring_s + rp.s * kGuBox + row_l * kGuW;
    const int s = rp.s;
    rp.next(c.S);
    const uint32_t rgg = rg + 16 * g, lsa = rg + lsoff;
    int i0 = 0, i1 = 0;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      const uint4 a0 = ld_s128(rgg ^ (32 * cc));
      const uint4 a1 = ld_s128(rgg ^ (32 * cc + 16));
      const uint4 b0 = ld_s128((rgg + 1024) ^ (32 * cc));
      const uint4 b1 = ld_s128((rgg + 1024) ^ (32 * cc + 16));
      uint2 bv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) bv[u] = ld_s64(bp[u] + (4 * cc + u) * 32);
      const uint32_t l0 = ld_s8(lsa ^ (32 * cc)), l1 = ld_s8((lsa + 1024) ^ (32 * cc));
      const uint2 rec[4][2] = {{make_uint2(a0.x, a0.y), make_uint2(b0.x, b0.y)},
                               {make_uint2(a0.z, a0.w), make_uint2(b0.z, b0.w)},
                               {make_uint2(a1.x, a1.y), make_uint2(b1.x, b1.y)},
                               {make_uint2(a1.z, a1.w), make_uint2(b1.z, b1.w)}};
      int acc[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        uint32_t r0lo, r0hi, r1lo, r1hi;
        iq2_operand(c, rec[u][0], r0lo, r0hi);
        iq2_operand(c, rec[u][1], r1lo, r1hi);
        if (u == 0)
          mma_s8s8_zero(acc, r0lo, r1lo, r0hi, r1hi, bv[u].x, bv[u].y);
        else
          mma_s8s8(acc, r0lo, r1lo, r0hi, r1hi, bv[u].x, bv[u].y);
      }
      // this thread's columns are sub-block 4cc+tig, digits hi and lo
      i0 += (acc[0] * 128 + acc[1]) * static_cast<int>((l0 >> 3) | 1u);
      i1 += (acc[2] * 128 + acc[3]) * static_cast<int>((l1 >> 3) | 1u);
      if (cc & 1) {
        const int sb = cc >> 1;
        const float xsv = ld_sf(xsc + (2 * j + sb) * 4);
        const uint32_t w0 = j ? dp[1][0] : dp[0][0], w1 = j ? dp[1][1] : dp[0][1];
        const float d0 = sb ? half_hi(w0) : half_lo(w0);
        const float d1 = sb ? half_hi(w1) : half_lo(w1);
        f0 = fmaf(static_cast<float>(i0), d0 * xsv, f0);
        f1 = fmaf(static_cast<float>(i1), d1 * xsv, f1);
        i0 = i1 = 0;
      }
    }
    __syncwarp();
    if (c.lane == 0) mbar_arrive(&c.empty[s]);
  }
  // the four lanes of a quad hold four different sub-blocks of the same rows
  f0 += __shfl_xor_sync(0xffffffffu, f0, 1);
  f0 += __shfl_xor_sync(0xffffffffu, f0, 2);
  f1 += __shfl_xor_sync(0xffffffffu, f1, 1);
  f1 += __shfl_xor_sync(0xffffffffu, f1, 2);
  if (tig == 0) {
    float* out = a.gpart + ((static_cast<size_t>(w.p0) * 2 + w.m) * a.KP + w.kp) * I + w.rb * kBoxRows + row_l;
    out[0] = f0;
    out[8] = f1;
  }
  return true;
}

// One unit whose expert holds 2..4*MAXQ assignments. TPG tokens share one set
// of MMA columns (TPG tokens x 4/TPG sub-block slots x 2 digits); MAXQ column
// sets reuse the same A operands.
template <int TPG, int MAXQ>
__device__ __forceinline__ bool gu_unit_multi(const GuTmaArgs& a, const GuCtx& c, RingPos& rp, const GuUnit& w,
                                              const uint32_t (&dp)[kMaxNB][2]) {
  constexpr int SPS = 4 / TPG;
  const int H = a.H, I = a.I, ne = w.ne, p0 = w.p0;
  const int ngroups = (ne + TPG - 1) / TPG;
  const int g = c.g, tig = c.tig;
  const int tslot_b = (g >> 1) % TPG, sslot_b = (g >> 1) / TPG, dig_b = g & 1;
  const int tslot_c = tig % TPG, sslot_c = tig / TPG;
  const int row_l = 16 * c.warp + g;
  const int8_t* xb[MAXQ];
  const float* xsc[MAXQ];
  bool bon[MAXQ];
#pragma unroll
  for (int q = 0; q < MAXQ; ++q) {
    const int tb = q * TPG + tslot_b, tc = q * TPG + tslot_c;
    bon[q] = q < ngroups && tb < ne;
    xb[q] = bon[q] ? c.xdig + (c.tok[p0 + tb] * 2 + dig_b) * c.xpitch + 8 * tig + (w.kp * a.NB * 16 + sslot_b) * 32
                   : c.zero + 8 * tig;
    xsc[q] = (q < ngroups && tc < ne) ? c.xscl + c.tok[p0 + tc] * (H / 256) + 2 * a.NB * w.kp : nullptr;
  }
  int acc[MAXQ][4];
  int iacc[MAXQ][2];
  float facc[MAXQ][2];
#pragma unroll
  for (int q = 0; q < MAXQ; ++q) {
    iacc[q][0] = iacc[q][1] = 0;
    facc[q][0] = facc[q][1] = 0.f;
  }
#pragma unroll 1
  for (int j = 0; j < a.NB; ++j) {
    if (!mbar_wait_bounded(&c.full[rp.s], rp.ph, a.err, ERR_TIMEOUT)) return false;
    const int s = rp.s;
    rp.next(c.S);
    const uint8_t* rg = c.ring + s * kGuBox + row_l * kGuW;
    const uint32_t dj0 = j ? dp[1][0] : dp[0][0], dj1 = j ? dp[1][1] : dp[0][1];
#pragma unroll 1
    for (int cc = 0; cc < 4; ++cc) {
      uint2 rec[4][2];
      gu_records(rg, cc, g, rec);
      uint32_t af[4][2][2];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        iq2_operand(c, rec[u][0], af[u][0][0], af[u][0][1]);
        iq2_operand(c, rec[u][1], af[u][1][0], af[u][1][1]);
      }
#pragma unroll
      for (int q = 0; q < MAXQ; ++q) {
        if (q >= ngroups) break;
#pragma unroll
        for (int jj = 0; jj < TPG; ++jj) {
          // column set jj covers sub-blocks 4cc + jj*SPS .. +SPS-1
          const int8_t* xp = bon[q] ? xb[q] + j * 512 : xb[q];
          const uint2 bl = *reinterpret_cast<const uint2*>(xp + (4 * cc + jj * SPS) * 32);
#pragma unroll
          for (int sl = 0; sl < SPS; ++sl) {
            const int u = jj * SPS + sl;
            const bool on = sl == sslot_b;
            const uint32_t b0 = on ? bl.x : 0u, b1 = on ? bl.y : 0u;
            if (sl == 0)
              mma_s8s8_zero(acc[q], af[u][0][0], af[u][1][0], af[u][0][1], af[u][1][1], b0, b1);
            else
              mma_s8s8(acc[q], af[u][0][0], af[u][1][0], af[u][0][1], af[u][1][1], b0, b1);
          }
          const int sbi = 4 * cc + jj * SPS + sslot_c;
          const int odd0 = gu_odd(rg, sbi, g), odd1 = gu_odd(rg + 1024, sbi, g);
          iacc[q][0] += (acc[q][0] * 128 + acc[q][1]) * odd0;
          iacc[q][1] += (acc[q][2] * 128 + acc[q][3]) * odd1;
        }
      }
      if (cc & 1) {
        const int sb = cc >> 1;
        const float d0 = sb ? half_hi(dj0) : half_lo(dj0);
        const float d1 = sb ? half_hi(dj1) : half_lo(dj1);
#pragma unroll
        for (int q = 0; q < MAXQ; ++q) {
          const float xsv = xsc[q] ? xsc[q][2 * j + sb] : 0.f;
          facc[q][0] = fmaf(static_cast<float>(iacc[q][0]), d0 * xsv, facc[q][0]);
          facc[q][1] = fmaf(static_cast<float>(iacc[q][1]), d1 * xsv, facc[q][1]);
          iacc[q][0] = iacc[q][1] = 0;
        }
      }
    }
    __syncwarp();
    if (c.lane == 0) mbar_arrive(&c.empty[s]);
  }
  // quad lanes holding the same token (TPG < 4) hold partial sums of different sub-blocks
#pragma unroll
  for (int q = 0; q < MAXQ; ++q)
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      float v = facc[q][r];
      if (TPG == 2) v += __shfl_xor_sync(0xffffffffu, v, 2);
      facc[q][r] = v;
    }
  const bool owner = (TPG == 4) || (tig < TPG);
#pragma unroll
  for (int q = 0; q < MAXQ; ++q) {
    const int t = q * TPG + tslot_c;
    if (q < ngroups && owner && t < ne) {
      float* out = a.gpart + ((static_cast<size_t>(p0 + t) * 2 + w.m) * a.KP + w.kp) * I + w.rb * kBoxRows + row_l;
      out[0] = facc[q][0];
      out[8] = facc[q][1];
    }
  }
  return true;
}


// Shared-memory plan of the gate/up kernel (host and device agree on it); the
// selector tables come first, at a fixed shared address, so lookups need no
// base add.
struct GuPlan {
  size_t tab, meta, zero, x, xs, ring, bars, total;
};
__host__ __device__ inline GuPlan gu_plan(int E, int T, int k, int H, bool xs_in, int S) {
  GuPlan p;
  p.tab = 0;
  p.meta = kTabBytes;
  p.zero = p.meta + meta_bytes(E, T * k, true);
  p.x = p.zero + kZeroBytes;
  p.xs = p.x + (xs_in ? align_up(static_cast<size_t>(T) * 2 * (H + kRowPad), 128) : 0);
  const size_t end = p.xs + (xs_in ? align_up(static_cast<size_t>(T) * (H / 256) * 4, 128) : 0);
  p.ring = align_up(end, 1024);
  p.bars = p.ring + static_cast<size_t>(S) * kGuBox;
  p.total = p.bars + 2 * static_cast<size_t>(S) * 8;
  return p;
}

template <int MAXQ, bool XS>
__global__ void __launch_bounds__(kThreadsT, 1) gateup_tma_kernel(const __grid_constant__ CUtensorMap tm_gate,
                                                                  const __grid_constant__ CUtensorMap tm_up,
                                                                  GuTmaArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  pdl_trigger();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = a.H, I = a.I, T = a.T, S = a.S, NB = a.NB;
  const int nA = T * a.k;
  const GuPlan pl = gu_plan(a.E, T, a.k, H, XS, S);
  MetaSmem ms;
  ms.off = reinterpret_cast<int32_t*>(smem + pl.meta);
  ms.act = ms.off + (a.E + 1);
  ms.tok = ms.act + (a.E + 1);
  int8_t* zero = reinterpret_cast<int8_t*>(smem + pl.zero);
  int8_t* xsm = reinterpret_cast<int8_t*>(smem + pl.x);
  float* xssm = reinterpret_cast<float*>(smem + pl.xs);
  uint8_t* ring = smem + pl.ring;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + pl.bars);
  uint64_t* empty = full + S;
  const int rbs = I / kBoxRows;

  if ((smem_addr(ring) & 1023u) != 0) {  // the 128-byte swizzle pattern assumes 1024-byte aligned boxes
    if (tid == 0) atomicCAS(a.err, 0, ERR_CUDA);
    return;
  }
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kCW);
    }
    fence_barrier_init();
  }
  for (int i = tid; i < kTabBytes / 4; i += kThreadsT) {
    const int ent = i >> 6;
    reinterpret_cast<uint32_t*>(smem + pl.tab)[i] =
        (i & 32) == 0 ? d_sel_tables2.level[ent] : (ent < 128 ? d_sel_tables2.sign[ent] : 0u);
  }
  for (int i = tid; i < kZeroBytes / 16; i += kThreadsT) reinterpret_cast<uint4*>(zero)[i] = make_uint4(0, 0, 0, 0);
  pdl_wait();  // routing and activations come from the kernels before this one
  load_meta(ms, a.offsets, a.active, a.perm, a.E, nA, a.k, tid, kThreadsT);
  if (XS) {
    stage_rows(xsm, a.xd, T * 2, H, tid, kThreadsT);
    for (int i = tid; i < T * (H / 256); i += kThreadsT) xssm[i] = a.xs[i];
  }
  __syncthreads();
  const int nact = ms.act[a.E];

  if (warp == kCW) {  // producer
    if (lane == 0) {
      prefetch_tmap(&tm_gate);
      prefetch_tmap(&tm_up);
      RingPos rp{0, 0u};
      GuIter t;
      t.init(blockIdx.x, gridDim.x, a.KP, rbs);
      for (; t.slot < nact; t.next(a.KP, rbs)) {
        const int e = ms.act[t.slot];
        for (int j = 0; j < NB; ++j) {
          if (!mbar_wait_bounded(&empty[rp.s], rp.ph ^ 1u, a.err, ERR_TIMEOUT)) return;
          mbar_arrive_expect_tx(&full[rp.s], kGuBox);
          tma_load_2d(ring + rp.s * kGuBox, t.m ? &tm_up : &tm_gate, (t.kp * NB + j) * kGuW, e * I + t.rb * kBoxRows,
                      &full[rp.s]);
          rp.next(S);
        }
      }
    }
    return;
  }

  GuCtx c;
  c.tab = reinterpret_cast<const char*>(smem + pl.tab);
  c.ring = ring;
  c.full = full;
  c.empty = empty;
  if (XS) {
    c.xdig = xsm;
    c.xscl = xssm;
    c.zero = zero;
    c.xpitch = H + kRowPad;
  } else {
    c.xdig = a.xd;
    c.xscl = a.xs;
    c.zero = g_zero_operand;
    c.xpitch = H;
  }
  c.ring_s = smem_addr(ring);
  c.x_s = smem_addr(xsm);
  c.xs_s = smem_addr(xssm);
  c.zero_s = smem_addr(zero);
  c.tok = ms.tok;
  c.warp = warp;
  c.lane = lane;
  c.g = lane >> 2;
  c.tig = lane & 3;
  c.S = S;
  c.lane4 = static_cast<uint32_t>(lane) << 2;
  c.sel_idx = 0x5504u | (static_cast<uint32_t>(c.tig) << 4);  // bytes: lane4, index byte tig, 0, 0
  c.rot_sig = (7u * c.tig - 8u) & 31u;                          // sign field tig to bits 8..14
  c.sgn_lane = 128u + c.lane4;
  const int row_l = 16 * warp + c.g;
  const int dstride = H / 256;
  // per-row fp16 scales of a unit: for box j the pair of super-blocks 2(kp*NB+j), +1
  auto dload = [&](const GuUnit& w, uint32_t (&d)[kMaxNB][2]) {
    const uint16_t* dpl = w.m ? a.up_d : a.gate_d;
    const size_t row = static_cast<size_t>(w.e) * I + w.rb * kBoxRows + row_l;
    const uint16_t* r0 = dpl + row * dstride + 2 * w.kp * NB;
    d[0][0] = __ldg(reinterpret_cast<const uint32_t*>(r0));
    d[0][1] = __ldg(reinterpret_cast<const uint32_t*>(r0 + 8 * dstride));
    if (NB > 1) {
      d[1][0] = __ldg(reinterpret_cast<const uint32_t*>(r0 + 2));
      d[1][1] = __ldg(reinterpret_cast<const uint32_t*>(r0 + 8 * dstride + 2));
    }
  };
  RingPos rp{0, 0u};
  GuIter t;
  t.init(blockIdx.x, gridDim.x, a.KP, rbs);
  uint32_t nd[kMaxNB][2] = {};
  GuUnit nw{};
  if (t.slot < nact) {
    nw = gu_unit_of(t, ms);
    dload(nw, nd);
  }
  while (t.slot < nact) {
    const GuUnit w = nw;
    uint32_t d[kMaxNB][2];
#pragma unroll
    for (int j = 0; j < kMaxNB; ++j) d[j][0] = nd[j][0], d[j][1] = nd[j][1];
    t.next(a.KP, rbs);
    if (t.slot < nact) {
      nw = gu_unit_of(t, ms);
      dload(nw, nd);
    }
    bool ok;
    if (XS && (MAXQ == 1 || w.ne == 1)) ok = gu_unit_one(a, c, rp, w, d);
    else if (w.ne == 1) ok = gu_unit_multi<4, 1>(a, c, rp, w, d);
    else if (w.ne == 2) ok = gu_unit_multi<2, 1>(a, c, rp, w, d);
    else ok = gu_unit_multi<4, (MAXQ > 1 ? MAXQ : 1)>(a, c, rp, w, d);
    if (!ok) return;
  }
}

// ===========================================================================
// down
// ===========================================================================
struct DnTmaArgs {
  int H, I, E, k, T, DP, NB, S;
  const uint32_t* dd;
  const int8_t* hd;
  const float* hsc;
  const int32_t* hq;
  const int32_t* offsets;
  const int32_t* active;
  float* opart;  // [T*k][DP][H]
  int* err;
  int hss;
};

// Unit u = (slot * rbs + rb) * DP + dp, walked in steps of gridDim.x.
struct DnIter {
  int dp, rb, slot, ddp, drb, dslot;
  __device__ __forceinline__ void init(int u0, int G, int DP, int rbs) {
    dp = u0 % DP;
    int r = u0 / DP;
    rb = r % rbs;
    slot = r / rbs;
    ddp = G % DP;
    r = G / DP;
    drb = r % rbs;
    dslot = r / rbs;
  }
  __device__ __forceinline__ void next(int DP, int rbs) {
    dp += ddp;
    int c = dp >= DP ? 1 : 0;
    dp -= c * DP;
    rb += drb + c;
    c = rb >= rbs ? 1 : 0;
    rb -= c * rbs;
    slot += dslot + c;
  }
};

struct DnUnit {
  int e, rb, dp, p0, ne;
};

__device__ __forceinline__ DnUnit dn_unit_of(const DnIter& t, const MetaSmem& ms) {
  DnUnit w;
  w.dp = t.dp;
  w.rb = t.rb;
  w.e = ms.act[t.slot];
  w.p0 = ms.off[w.e];
  w.ne = ms.off[w.e + 1] - w.p0;
  return w;
}

struct DnCtx {
  const uint8_t* ring;
  uint64_t* full;
  uint64_t* empty;
  const int8_t* hd;    // rows (assignment, digit) of I digits in MMA k order, pitch hpitch
  const float* hsc;    // [T*k][hss]
  const int32_t* hq;   // [T*k][I/16]
  const int8_t* zero;  // 128-byte aligned zero region
  uint32_t ring_s, hd_s, hsc_s, hq_s, zero_s;  // shared-window addresses (staged variant)
  int hpitch, warp, lane, g, tig, S;
};

__device__ __forceinline__ float dn_block(uint32_t dd, float e2, int iA, int iM) {
  return e2 * fmaf(half_lo(dd), static_cast<float>(iA), -half_hi(dd) * static_cast<float>(iM));
}

// One down unit for an expert with one assignment. MMA columns:
// (pair slot 0..1) x (half 0..1) x (digit hi, lo); idle column halves read the
// zero region.
// One down unit for an expert with one assignment, h staged in shared memory.
// MMA columns: (pair slot 0..1) x (half 0..1) x (digit hi, lo); idle column
// halves read the zero region. All shared-memory addresses are 32-bit with
// compile-time offsets.
__device__ __forceinline__ bool dn_unit_one(const DnTmaArgs& a, const DnCtx& c, RingPos& rp, const DnUnit& w,
                                            const uint32_t (&dd)[kMaxNB][2]) {
  const int H = a.H, I = a.I, NB = a.NB;
  const int g = c.g, tig = c.tig;
  const int row_l = 16 * c.warp + g;
  const uint32_t sh = 2 * tig;
  const int sl_b = g >> 2, hb = (g >> 1) & 1, dig_b = g & 1;
  const uint32_t hrow = c.hd_s + (w.p0 * 2 + dig_b) * c.hpitch + w.dp * NB * 256 + 8 * tig;
  const uint32_t zrow = c.zero_s + ((64 * (w.p0 & 1) + 64) & 127) + 8 * tig;
  const uint32_t hqr = c.hq_s + (w.p0 * (I / 16) + w.dp * NB * 16 + tig) * 4;
  const uint32_t e2p = c.hsc_s + (w.p0 * a.hss + w.dp * NB) * 4;
  float f0 = 0.f, f1 = 0.f;
#pragma unroll 1
  for (int j = 0; j < NB; ++j) {
    uint32_t bp0[2], bp1[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      bp0[u] = (sl_b == u && hb == 0) ? hrow + j * 256 : zrow;
      bp1[u] = (sl_b == u && hb == 1) ? hrow + j * 256 + 4 : zrow + 4;
    }
    if (!mbar_wait_bounded(&c.full[rp.s], rp.ph, a.err, ERR_TIMEOUT)) return false;
    const uint32_t rA = c.ring_s + rp.s * kDnBox + row_l * kDnW, rB = rA + 8 * kDnW;
    const int s = rp.s;
    rp.next(c.S);
    int iA0 = 0, iA1 = 0, iM0 = 0, iM1 = 0;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {  // 16 q bytes = four sub-blocks = two MMAs
      const uint4 qa = ld_s128(rA + 16 + 16 * cc);
      const uint4 qb = ld_s128(rB + 16 + 16 * cc);
      uint32_t bv0[2], bv1[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        bv0[u] = ld_s32(bp0[u] + (2 * cc + u) * 32);
        bv1[u] = ld_s32(bp1[u] + (2 * cc + u) * 32);
      }
      // this thread's columns: sub-block 4cc + tig (pair 2cc + tig/2, half tig&1)
      const uint32_t scA = ld_s8(rA + 4 * cc + tig), scB = ld_s8(rB + 4 * cc + tig);
      const int hqv = static_cast<int>(ld_s32(hqr + (j * 16 + 4 * cc) * 4));
      int acc[4];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const uint32_t wa0 = u ? qa.z : qa.x, wa1 = u ? qa.w : qa.y;
        const uint32_t wb0 = u ? qb.z : qb.x, wb1 = u ? qb.w : qb.y;
        const uint32_t a0 = (wa0 >> sh) & 0x03030303u, a1 = (wb0 >> sh) & 0x03030303u;
        const uint32_t a2 = (wa1 >> sh) & 0x03030303u, a3 = (wb1 >> sh) & 0x03030303u;
        if (u == 0) mma_u8s8_zero(acc, a0, a1, a2, a3, bv0[u], bv1[u]);
        else mma_u8s8(acc, a0, a1, a2, a3, bv0[u], bv1[u]);
      }
      iA0 += (acc[0] * 128 + acc[1]) * static_cast<int>(scA & 15u);
      iA1 += (acc[2] * 128 + acc[3]) * static_cast<int>(scB & 15u);
      iM0 += static_cast<int>(scA >> 4) * hqv;
      iM1 += static_cast<int>(scB >> 4) * hqv;
    }
    const float e2 = ld_sf(e2p + j * 4);
    __syncwarp();
    if (c.lane == 0) mbar_arrive(&c.empty[s]);
    const uint32_t dA = j ? dd[1][0] : dd[0][0], dB = j ? dd[1][1] : dd[0][1];
    f0 += dn_block(dA, e2, iA0, iM0);
    f1 += dn_block(dB, e2, iA1, iM1);
  }
  f0 += __shfl_xor_sync(0xffffffffu, f0, 1);
  f0 += __shfl_xor_sync(0xffffffffu, f0, 2);
  f1 += __shfl_xor_sync(0xffffffffu, f1, 1);
  f1 += __shfl_xor_sync(0xffffffffu, f1, 2);
  if (tig == 0) {
    float* out = a.opart + (static_cast<size_t>(w.p0) * a.DP + w.dp) * H + w.rb * kBoxRows + row_l;
    out[0] = f0;
    out[8] = f1;
  }
  return true;
}

// One down unit for an expert with 2..2*MAXQ assignments. MMA columns:
// (token slot 0..1) x (half 0..1) x (digit hi, lo).
template <int MAXQ>
__device__ __forceinline__ bool dn_unit_multi(const DnTmaArgs& a, const DnCtx& c, RingPos& rp, const DnUnit& w,
                                              const uint32_t (&dd)[kMaxNB][2]) {
  const int H = a.H, I = a.I, ne = w.ne, p0 = w.p0;
  const int g = c.g, tig = c.tig;
  const int ngroups = (ne + 1) / 2;
  const int dig_b = g & 1, hb = (g >> 1) & 1, sl_b = g >> 2;
  const int hc = tig & 1, sl_c = tig >> 1;
  const uint32_t sh = 2 * tig;
  const int row_l = 16 * c.warp + g;
  const int8_t* hrow[MAXQ];
  bool b0on[MAXQ], b1on[MAXQ];
  const int32_t* hq_ptr[MAXQ];
  const float* e2p[MAXQ];
#pragma unroll
  for (int q = 0; q < MAXQ; ++q) {
    const int tb = 2 * q + sl_b, tc = 2 * q + sl_c;
    const bool on = q < ngroups && tb < ne;
    hrow[q] = c.hd + ((p0 + (on ? tb : 0)) * 2 + dig_b) * c.hpitch + w.dp * a.NB * 256 + 8 * tig;
    b0on[q] = on && hb == 0;
    b1on[q] = on && hb == 1;
    const bool cv = q < ngroups && tc < ne;
    hq_ptr[q] = c.hq + (p0 + (cv ? tc : 0)) * (I / 16) + w.dp * a.NB * 16 + hc;
    e2p[q] = cv ? c.hsc + (p0 + tc) * a.hss + w.dp * a.NB : nullptr;
  }
  const int8_t* zrow = c.zero + 8 * tig;
  float facc[MAXQ][2];
#pragma unroll
  for (int q = 0; q < MAXQ; ++q) facc[q][0] = facc[q][1] = 0.f;
#pragma unroll 1
  for (int j = 0; j < a.NB; ++j) {
    int acc[4];
    int iA[MAXQ][2], iM[MAXQ][2];
#pragma unroll
    for (int q = 0; q < MAXQ; ++q) iA[q][0] = iA[q][1] = iM[q][0] = iM[q][1] = 0;
    if (!mbar_wait_bounded(&c.full[rp.s], rp.ph, a.err, ERR_TIMEOUT)) return false;
    const int s = rp.s;
    rp.next(c.S);
    const uint8_t* rA = c.ring + s * kDnBox + row_l * kDnW;
    const uint8_t* rB = rA + 8 * kDnW;
#pragma unroll 1
    for (int cc = 0; cc < 4; ++cc) {
      const uint4 qa = lds128(rA + 16 + 16 * cc);
      const uint4 qb = lds128(rB + 16 + 16 * cc);
      uint32_t af[2][4];
      af[0][0] = (qa.x >> sh) & 0x03030303u; af[0][1] = (qb.x >> sh) & 0x03030303u;
      af[0][2] = (qa.y >> sh) & 0x03030303u; af[0][3] = (qb.y >> sh) & 0x03030303u;
      af[1][0] = (qa.z >> sh) & 0x03030303u; af[1][1] = (qb.z >> sh) & 0x03030303u;
      af[1][2] = (qa.w >> sh) & 0x03030303u; af[1][3] = (qb.w >> sh) & 0x03030303u;
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int pr = 2 * cc + u;
        // this thread's columns: sub-block 2*pr + hc of token 2q + sl_c
        const int sub = 2 * pr + hc;
        const uint32_t scA = rA[sub], scB = rB[sub];
#pragma unroll
        for (int q = 0; q < MAXQ; ++q) {
          if (q >= ngroups) break;
          const int8_t* p0b = b0on[q] ? hrow[q] + j * 256 : zrow;
          const int8_t* p1b = b1on[q] ? hrow[q] + j * 256 + 4 : zrow + 4;
          const uint32_t b0 = *reinterpret_cast<const uint32_t*>(p0b + pr * 32);
          const uint32_t b1 = *reinterpret_cast<const uint32_t*>(p1b + pr * 32);
          mma_u8s8_zero(acc, af[u][0], af[u][1], af[u][2], af[u][3], b0, b1);
          const int hqv = hq_ptr[q][j * 16 + 2 * pr];
          iA[q][0] += (acc[0] * 128 + acc[1]) * static_cast<int>(scA & 15u);
          iA[q][1] += (acc[2] * 128 + acc[3]) * static_cast<int>(scB & 15u);
          iM[q][0] += static_cast<int>(scA >> 4) * hqv;
          iM[q][1] += static_cast<int>(scB >> 4) * hqv;
        }
      }
    }
    __syncwarp();
    if (c.lane == 0) mbar_arrive(&c.empty[s]);
    const uint32_t dA = j ? dd[1][0] : dd[0][0], dB = j ? dd[1][1] : dd[0][1];
#pragma unroll
    for (int q = 0; q < MAXQ; ++q) {
      const float e2 = e2p[q] ? e2p[q][j] : 0.f;
      facc[q][0] += dn_block(dA, e2, iA[q][0], iM[q][0]);
      facc[q][1] += dn_block(dB, e2, iA[q][1], iM[q][1]);
    }
  }
#pragma unroll
  for (int q = 0; q < MAXQ; ++q) {
    if (q >= ngroups) break;
    float f0 = facc[q][0], f1 = facc[q][1];
    f0 += __shfl_xor_sync(0xffffffffu, f0, 1);
    f1 += __shfl_xor_sync(0xffffffffu, f1, 1);
    const int t = 2 * q + sl_c;
    if (hc == 0 && t < ne) {
      float* out = a.opart + (static_cast<size_t>(p0 + t) * a.DP + w.dp) * H + w.rb * kBoxRows + row_l;
      out[0] = f0;
      out[8] = f1;
    }
  }
  return true;
}

// Shared-memory plan of the down kernel.
struct DnPlan {
  size_t meta, zero, hd, hsc, hq, ring, bars, total;
};
__host__ __device__ inline DnPlan dn_plan(int E, int nA, int I, int hss, bool hs_in, int S) {
  DnPlan p;
  p.meta = 0;
  p.zero = meta_bytes(E, nA, false);
  p.hd = p.zero + kZeroBytes;
  p.hsc = p.hd + (hs_in ? align_up(static_cast<size_t>(nA) * 2 * (I + kRowPad), 128) : 0);
  p.hq = p.hsc + (hs_in ? align_up(static_cast<size_t>(nA) * hss * 4, 128) : 0);
  const size_t end = p.hq + (hs_in ? align_up(static_cast<size_t>(nA) * (I / 16) * 4, 128) : 0);
  p.ring = align_up(end, 1024);
  p.bars = p.ring + static_cast<size_t>(S) * kDnBox;
  p.total = p.bars + 2 * static_cast<size_t>(S) * 8;
  return p;
}

template <int MAXQ, bool HS>
__global__ void __launch_bounds__(kThreadsT, 1) down_tma_kernel(const __grid_constant__ CUtensorMap tm_down,
                                                                DnTmaArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  pdl_trigger();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = a.H, I = a.I, S = a.S, NB = a.NB;
  const int nA = a.T * a.k;
  const DnPlan pl = dn_plan(a.E, nA, I, a.hss, HS, S);
  MetaSmem ms;
  ms.off = reinterpret_cast<int32_t*>(smem + pl.meta);
  ms.act = ms.off + (a.E + 1);
  ms.tok = nullptr;
  int8_t* zero = reinterpret_cast<int8_t*>(smem + pl.zero);
  int8_t* hd_s = reinterpret_cast<int8_t*>(smem + pl.hd);
  float* hsc_s = reinterpret_cast<float*>(smem + pl.hsc);
  int32_t* hq_s = reinterpret_cast<int32_t*>(smem + pl.hq);
  uint8_t* ring = smem + pl.ring;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + pl.bars);
  uint64_t* empty = full + S;
  const int rbs = H / kBoxRows;

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kCW);
    }
    fence_barrier_init();
  }
  for (int i = tid; i < kZeroBytes / 16; i += kThreadsT) reinterpret_cast<uint4*>(zero)[i] = make_uint4(0, 0, 0, 0);
  pdl_wait();  // routing and h come from the kernels before this one
  load_meta(ms, a.offsets, a.active, nullptr, a.E, nA, a.k, tid, kThreadsT);
  if (HS) {
    stage_rows(hd_s, a.hd, nA * 2, I, tid, kThreadsT);
    for (int i = tid; i < nA * a.hss; i += kThreadsT) hsc_s[i] = a.hsc[i];
    for (int i = tid; i < nA * (I / 16); i += kThreadsT) hq_s[i] = a.hq[i];
  }
  __syncthreads();
  const int nact = ms.act[a.E];

  if (warp == kCW) {  // producer
    if (lane == 0) {
      prefetch_tmap(&tm_down);
      RingPos rp{0, 0u};
      DnIter t;
      t.init(blockIdx.x, gridDim.x, a.DP, rbs);
      for (; t.slot < nact; t.next(a.DP, rbs)) {
        const int e = ms.act[t.slot];
        for (int j = 0; j < NB; ++j) {
          if (!mbar_wait_bounded(&empty[rp.s], rp.ph ^ 1u, a.err, ERR_TIMEOUT)) return;
          mbar_arrive_expect_tx(&full[rp.s], kDnBox);
          tma_load_2d(ring + rp.s * kDnBox, &tm_down, (t.dp * NB + j) * kDnW, e * H + t.rb * kBoxRows, &full[rp.s]);
          rp.next(S);
        }
      }
    }
    return;
  }
  DnCtx c;
  c.ring = ring;
  c.ring_s = smem_addr(ring);
  c.full = full;
  c.empty = empty;
  if (HS) {
    c.hd = hd_s;
    c.hsc = hsc_s;
    c.hq = hq_s;
    c.zero = zero;
    c.hpitch = I + kRowPad;
    c.hd_s = smem_addr(hd_s);
    c.hsc_s = smem_addr(hsc_s);
    c.hq_s = smem_addr(hq_s);
    c.zero_s = smem_addr(zero);
  } else {
    c.hd = a.hd;
    c.hsc = a.hsc;
    c.hq = a.hq;
    c.zero = g_zero_operand;
    c.hpitch = I;
  }
  c.warp = warp;
  c.lane = lane;
  c.g = lane >> 2;
  c.tig = lane & 3;
  c.S = S;
  const int row_l = 16 * warp + c.g;
  const int nblk = I / 256;
  auto ddload = [&](const DnUnit& w, uint32_t (&d)[kMaxNB][2]) {
    const size_t row = static_cast<size_t>(w.e) * H + w.rb * kBoxRows + row_l;
    const uint32_t* r0 = a.dd + row * nblk + w.dp * NB;
    d[0][0] = __ldg(r0);
    d[0][1] = __ldg(r0 + 8 * nblk);
    if (NB > 1) {
      d[1][0] = __ldg(r0 + 1);
      d[1][1] = __ldg(r0 + 8 * nblk + 1);
    }
  };
  RingPos rp{0, 0u};
  DnIter t;
  t.init(blockIdx.x, gridDim.x, a.DP, rbs);
  uint32_t nd[kMaxNB][2] = {};
  DnUnit nw{};
  if (t.slot < nact) {
    nw = dn_unit_of(t, ms);
    ddload(nw, nd);
  }
  while (t.slot < nact) {
    const DnUnit w = nw;
    uint32_t d[kMaxNB][2];
#pragma unroll
    for (int j = 0; j < kMaxNB; ++j) d[j][0] = nd[j][0], d[j][1] = nd[j][1];
    t.next(a.DP, rbs);
    if (t.slot < nact) {
      nw = dn_unit_of(t, ms);
      ddload(nw, nd);
    }
    bool ok;
    if (HS && (MAXQ == 1 || w.ne == 1)) ok = dn_unit_one(a, c, rp, w, d);
    else ok = dn_unit_multi<(MAXQ > 1 ? MAXQ : 1)>(a, c, rp, w, d);
    if (!ok) return;
  }
}

// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// 2-D byte tensor [rows][row_bytes] with a box of box_rows x box_bytes.
bool make_map(CUtensorMap* m, const void* base, uint64_t row_bytes, uint64_t rows, uint32_t box_bytes,
              uint32_t box_rows, bool swizzle128) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {row_bytes, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_bytes, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

constexpr size_t kBudget = 227 * 1024;

int nb_for(int T) { return T == 1 ? 1 : 2; }

template <typename K>
void launch_k(K kern, int grid, size_t smem, cudaStream_t st, const CUtensorMap& m0, const CUtensorMap& m1,
              const GuTmaArgs& a) {
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  launch_pdl(kern, dim3(grid), dim3(kThreadsT), smem, st, m0, m1, a);
}

template <typename K>
void launch_k(K kern, int grid, size_t smem, cudaStream_t st, const CUtensorMap& m0, const DnTmaArgs& a) {
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  launch_pdl(kern, dim3(grid), dim3(kThreadsT), smem, st, m0, a);
}

}  // namespace

bool tma_path_supported(const LayerShape& s, int T) {
  return s.H % 1024 == 0 && s.I % 512 == 0 && T >= 1 && T <= 16 && s.E <= kMaxExpertsTma &&
         encode_fn() != nullptr;
}
// A gate/up unit covers NB*512 of H and a down unit NB*256 of I, so the
// reduction axis is always split into this many parts.
int tma_gu_parts(const LayerShape& s, int T) { return s.H / (512 * nb_for(T)); }
int tma_dn_parts(const LayerShape& s, int T) { return s.I / (256 * nb_for(T)); }

int launch_gateup_tma(const LayerShape& sh, const uint8_t* gate_codes, const uint16_t* gate_d,
                      const uint8_t* up_codes, const uint16_t* up_d, const int8_t* xd, const float* xs, int T,
                      const Routing& r, float* gpart, int* err, int sms, cudaStream_t st) {
  CUtensorMap tg, tu;
  const uint64_t rb = sh.H / 4, rows = static_cast<uint64_t>(sh.E) * sh.I;
  if (!make_map(&tg, gate_codes, rb, rows, kGuW, kBoxRows, true) ||
      !make_map(&tu, up_codes, rb, rows, kGuW, kBoxRows, true))
    return ERR_CUDA;
  GuTmaArgs a{};
  a.H = sh.H; a.I = sh.I; a.E = sh.E; a.k = sh.k; a.T = T;
  a.NB = nb_for(T); a.KP = tma_gu_parts(sh, T);
  a.gate_d = gate_d; a.up_d = up_d; a.xd = xd; a.xs = xs;
  a.offsets = r.offsets; a.perm = r.perm; a.active = r.active; a.gpart = gpart; a.err = err;
  // stage the activations when that still leaves three ring stages
  const size_t budget = kBudget;
  const bool xs_in = gu_plan(sh.E, T, sh.k, sh.H, true, 3).total <= budget;
  int S = 2;
  while (S < 6 && gu_plan(sh.E, T, sh.k, sh.H, xs_in, S + 1).total <= budget) ++S;
  if (gu_plan(sh.E, T, sh.k, sh.H, xs_in, S).total > budget) return ERR_SHAPE;
  a.S = S;
  const size_t smem = gu_plan(sh.E, T, sh.k, sh.H, xs_in, S).total;
  const size_t nA = static_cast<size_t>(T) * sh.k;
  const int slots = static_cast<int>(std::min<size_t>(nA, static_cast<size_t>(sh.E)));
  const int units = slots * 2 * (sh.I / kBoxRows) * a.KP;
  const int grid = std::max(1, std::min(units, sms));
  if (T == 1) {  // one token: the single-assignment variant with staged activations
    if (!xs_in) return ERR_SHAPE;
    launch_k(gateup_tma_kernel<1, true>, grid, smem, st, tg, tu, a);
  } else if (xs_in) {  // at most 16 tokens per expert: four groups of four
    launch_k(gateup_tma_kernel<4, true>, grid, smem, st, tg, tu, a);
  } else {
    launch_k(gateup_tma_kernel<4, false>, grid, smem, st, tg, tu, a);
  }
  return cudaGetLastError() == cudaSuccess ? OK : ERR_CUDA;
}

int launch_down_tma(const LayerShape& sh, const uint8_t* down_codes, const uint32_t* down_dd, const int8_t* hd,
                    const float* hsc, const int32_t* hq, int hss, int T, const Routing& r, float* opart, int* err,
                    int sms, cudaStream_t st) {
  CUtensorMap td;
  const uint64_t rb = static_cast<uint64_t>(sh.I / 256) * kDnW, rows = static_cast<uint64_t>(sh.E) * sh.H;
  if (!make_map(&td, down_codes, rb, rows, kDnW, kBoxRows, false)) return ERR_CUDA;
  DnTmaArgs a{};
  a.H = sh.H; a.I = sh.I; a.E = sh.E; a.k = sh.k; a.T = T; a.hss = hss;
  a.NB = nb_for(T); a.DP = tma_dn_parts(sh, T);
  a.dd = down_dd; a.hd = hd; a.hsc = hsc; a.hq = hq;
  a.offsets = r.offsets; a.active = r.active; a.opart = opart; a.err = err;
  const int nA = T * sh.k;
  const bool hs_in = dn_plan(sh.E, nA, sh.I, hss, true, 4).total <= kBudget;
  int S = 2;
  while (S < 8 && dn_plan(sh.E, nA, sh.I, hss, hs_in, S + 1).total <= kBudget) ++S;
  if (dn_plan(sh.E, nA, sh.I, hss, hs_in, S).total > kBudget) return ERR_SHAPE;
  a.S = S;
  const size_t smem = dn_plan(sh.E, nA, sh.I, hss, hs_in, S).total;
  const int slots = std::min(nA, sh.E);
  const int units = slots * (sh.H / kBoxRows) * a.DP;
  const int grid = std::max(1, std::min(units, sms));
  if (T == 1) {  // one token: the single-assignment variant with h staged
    if (!hs_in) return ERR_SHAPE;
    launch_k(down_tma_kernel<1, true>, grid, smem, st, td, a);
  } else if (hs_in) {  // at most 16 tokens per expert: eight groups of two
    launch_k(down_tma_kernel<8, true>, grid, smem, st, td, a);
  } else {
    launch_k(down_tma_kernel<8, false>, grid, smem, st, td, a);
  }
  return cudaGetLastError() == cudaSuccess ? OK : ERR_CUDA;
}

}  // namespace moe
