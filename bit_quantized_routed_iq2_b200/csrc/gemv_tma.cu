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


constexpr int kCW = 16;                      // consumer warps (16 rows each)
constexpr int kThreadsT = (kCW + 1) * 32;    // + one producer warp
constexpr int kBoxRows = 16 * kCW;           // 256 rows per box
constexpr int kGuW = 128;                    // code bytes per gate/up box row (512 weights)
constexpr int kGuBox = kBoxRows * kGuW;      // 32 KB
// Selector tables, each entry replicated for the 32 lanes: grid row i at byte
// 256*i + 4*lane, sign field s at byte 256*s + 128 + 4*lane (interleaved, so
// that one prmt turns a grid index byte into its table address).
constexpr int kTabBytes = 256 * 256;
constexpr int kZeroBytes = 1024;             // zero operand region for idle MMA columns
constexpr int kMaxExpertsTma = 1024;
constexpr int kMaxNB = 2;

// Zero operand for the variants that read activations from global memory.
__device__ __align__(128) const int8_t g_zero_operand[kZeroBytes] = {};

__device__ __forceinline__ uint32_t rotr(uint32_t v, uint32_t n) { return __funnelshift_r(v, v, n); }

// Bounds-checked build (-DMOE_BOUNDS_CHECK, a separate library): every
// shared-memory load of these kernels checks that it lies inside the CTA's
// dynamic shared memory and is aligned, every partial-sum store and TMA box
// that it stays inside its buffer; a violation is counted in
// g_bounds_violations (read by moe_debug_bounds_violations) and the access is
// skipped (a load returns zeros). Nothing traps. The normal build compiles the
// checks away.
#ifdef MOE_BOUNDS_CHECK
__device__ unsigned long long g_bounds_violations = 0;
__device__ __forceinline__ bool bc_fail() {
  atomicAdd(&g_bounds_violations, 1ull);
  return false;
}
__device__ __forceinline__ bool smem_ok(uint32_t a, uint32_t bytes) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint32_t size;
  asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(size));
  const uint32_t base = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  return (a >= base && a - base + bytes <= size && (a & (bytes - 1)) == 0) ? true : bc_fail();
}
__device__ __forceinline__ bool index_ok(size_t i, size_t n) { return i < n ? true : bc_fail(); }
#define MOE_SMEM_GUARD(a, n, zero) \
  if (!smem_ok((a), (n))) return zero;
#else
__device__ __forceinline__ bool index_ok(size_t, size_t) { return true; }
#define MOE_SMEM_GUARD(a, n, zero)
#endif

__device__ __forceinline__ uint4 lds128(const uint8_t* p) {
  MOE_SMEM_GUARD(static_cast<uint32_t>(__cvta_generic_to_shared(p)), 16, make_uint4(0u, 0u, 0u, 0u))
  return *reinterpret_cast<const uint4*>(p);
}

// Loads from shared memory at 32-bit shared-window addresses. They are volatile
// so that they stay after the mbarrier wait that makes the data visible.
__device__ __forceinline__ uint4 ld_s128(uint32_t a) {
  MOE_SMEM_GUARD(a, 16, make_uint4(0u, 0u, 0u, 0u))
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ uint2 ld_s64(uint32_t a) {
  MOE_SMEM_GUARD(a, 8, make_uint2(0u, 0u))
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t ld_s32(uint32_t a) {
  MOE_SMEM_GUARD(a, 4, 0u)
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ float ld_sf(uint32_t a) {
  MOE_SMEM_GUARD(a, 4, 0.f)
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
  int no_produce;           // fault injection (test aid): the producer issues no loads
  int one;                  // 1, opaque to the compiler (keeps an integer add on the multiply-add pipe)
  long long wait_limit;     // bound of every mbarrier wait, in SM cycles
  const uint16_t* gate_d;
  const uint16_t* up_d;
  const int8_t* xd;
  const float* xs;
  const int32_t* offsets;
  const int32_t* perm;
  const int32_t* active;
  float* gpart;  // [T*k][2][KP][I]
  size_t gpart_n;  // its length in floats (bounds-checked build)
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


// The selector tables as they sit at the start of dynamic shared memory: row
// i (256 bytes) holds the level word of grid row i at bytes 0..127 and the
// sign word of sign field i mod 128 at bytes 128..255, each replicated for the
// 32 lanes. Built at compile time; a kernel brings the 64 KB in with one bulk
// asynchronous copy instead of thousands of dependent loads.
struct SelRep {
  uint32_t w[kTabBytes / 4];
};
constexpr SelRep make_sel_rep() {
  const Iq2SelTables t = make_sel_tables();
  SelRep r{};
  for (int i = 0; i < kTabBytes / 4; ++i) {
    const int ent = i >> 6;
    r.w[i] = (i & 32) == 0 ? t.level[ent] : t.sign[ent & 127];
  }
  return r;
}
// (not const: it must live in global memory, the source of a bulk copy)
__device__ __align__(128) SelRep g_sel_rep = make_sel_rep();

// Word-by-word copy of the same tables (the debug kernel's path).
__device__ __forceinline__ void fill_sel_tables(uint32_t* tab, int tid, int nthr) {
  for (int i = tid; i < kTabBytes / 4; i += nthr) tab[i] = g_sel_rep.w[i];
}

// Word of the selector tables at byte offset `off` of dynamic shared memory
// (the tables sit at its start, so the base folds into the load).
__device__ __forceinline__ uint32_t tab_ld(uint32_t off) {
  extern __shared__ __align__(1024) uint8_t smem[];
  MOE_SMEM_GUARD(static_cast<uint32_t>(__cvta_generic_to_shared(smem + off)), 4, 0u)
  return *reinterpret_cast<const uint32_t*>(smem + off);
}

// Two int8x4 A registers (elements 0..3 and 4..7) of one IQ2 group from its
// selector word: level code of element e in bits 4e..4e+1, sign in bit 4e+2.
// The 16-bit shift for the upper half is a multiply-high (FMA pipe).
__device__ __forceinline__ void iq2_pair(uint32_t sel, uint32_t& lo, uint32_t& hi) {
  lo = prmt(kPosBytes, kNegBytes, sel);
  hi = prmt(kPosBytes, kNegBytes, __umulhi(sel, 0x10000u));
}

// The int8 A operands (elements 0..3, 4..7 = level * sign) of group JJ of one
// 8-byte IQ2 sub-block record: the grid index byte JJ and the sign field JJ
// become table offsets by one prmt each (byte 1 = table row, byte 0 = this
// lane's replica), the two table words add up to the prmt selector word. The
// sign field is moved to bits 8..15 by a multiply (FMA pipe); its bit 15 is a
// neighbour's bit, which the sign table ignores by repeating every 128 rows.
template <int JJ>
__device__ __forceinline__ void iq2_group_int8(uint2 rec, uint32_t lane4, uint32_t sgn_lane, uint32_t one,
                                               uint32_t& lo, uint32_t& hi) {
  const uint32_t sf = JJ == 0 ? rec.y : (JJ == 1 ? rec.y * 2u : __umulhi(rec.y, JJ == 2 ? (1u << 26) : (1u << 19)));
  const uint32_t lv = tab_ld(prmt(rec.x, lane4, 0x5504u | (JJ << 4)));
  const uint32_t sg = tab_ld(prmt(sf, sgn_lane, JJ ? 0x5514u : 0x5504u));
  iq2_pair(lv * one + sg, lo, hi);  // level codes and sign bits are disjoint: the sum is the union
}

// 2*ls + 1 of an IQ2 sub-block record (ls = bits 28..31 of its sign word).
__device__ __forceinline__ int iq2_odd(uint2 rec) { return 2 * static_cast<int>(__umulhi(rec.y, 16u)) + 1; }

// The four 2-bit codes at bit pair `sh` / 2 of each byte of a Q2K code word, as
// uint8 A operand bytes (the down GEMV's K order takes weights 4i + tig).
__device__ __forceinline__ uint32_t q2k_quad(uint32_t w, uint32_t sh) { return (w >> sh) & 0x03030303u; }

// One unit whose expert holds a single assignment (every unit of a one-token
// step; single-token experts of a batch), activations staged in shared memory.
//
// Lane mapping (m16n8k32, lane = 4g + tig): the lane builds A for rows g and
// g+8 of the warp's 16. In round cc (0..3) of a 512-weight box it owns
// sub-block 2cc + (tig & 1) of block tig >> 1 of the box, whole: its four MMAs
// j = 0..3 take groups j of that sub-block, one 8-weight group per row each.
// So every lane reads its own two 8-byte sub-block records (no lane reads
// another's), takes the 2ls+1 scale from them and needs one fp16 d per row.
// MMA columns are (owner tig, digit hi/lo): B is non-zero only on the lanes
// with g >> 1 == tig, which load the x digits of their column's sub-block; the
// accumulator registers of lane tig then hold exactly its own sub-block.
// Shared-memory traffic per round and warp: two conflict-free 8-byte record
// loads per lane (the 128-byte swizzle spreads the 16 rows' chunks), two
// 16-byte B loads on eight lanes, sixteen selector-table loads.
template <bool XS>
__device__ __forceinline__ bool gu_unit_one(const GuTmaArgs& a, const GuCtx& c, RingPos& rp, const GuUnit& w,
                                            const uint32_t (&dp)[kMaxNB][2]) {
  const int I = a.I, NB = a.NB;
  const int g = c.g, tig = c.tig, bb = tig >> 1, hf = tig & 1;
  const int tok = c.tok[w.p0];
  const bool bact = (g >> 1) == tig;  // this lane carries B (digit g & 1 of its column's sub-block)
  const uint32_t one = static_cast<uint32_t>(a.one);
  // sub-block record of round 0 for row g, relative to the row's base: chunk (cc | 4bb) ^ g, half hf
  const uint32_t roff = (((static_cast<uint32_t>(g) ^ (4u * bb)) << 4) | (8u * hf));
  const uint32_t rowb = static_cast<uint32_t>(16 * c.warp + g) * kGuW;
  float f0 = 0.f, f1 = 0.f;
#pragma unroll 1
  for (int j = 0; j < NB; ++j) {
    const int kblk = j * 2 + bb;  // this lane's block of the staged slice
    // B source: the staged slice (x_off layout; chunk 1 of a sub-block is the XOR-16 neighbour of chunk 0)
    const uint32_t xb0 = c.x_s + x_off(c.xpitch, tok, g & 1, kblk * 256 + hf * 32);
    const uint32_t xb1 = xb0 ^ 16u;
    if (!mbar_wait_bounded(&c.full[rp.s], rp.ph, a.err, ERR_TIMEOUT, a.wait_limit)) return false;
    const uint32_t r0 = c.ring_s + rp.s * kGuBox + rowb + roff;
    const int s = rp.s;
    rp.next(c.S);
    int i0 = 0, i1 = 0;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      const uint2 ra = ld_s64(r0 ^ (16u * cc));          // row g
      const uint2 rb = ld_s64((r0 ^ (16u * cc)) + 1024);  // row g + 8
      uint4 bx0 = make_uint4(0u, 0u, 0u, 0u), bx1 = make_uint4(0u, 0u, 0u, 0u);
      if (bact) {
        bx0 = ld_s128(xb0 + 128u * cc);
        bx1 = ld_s128(xb1 + 128u * cc);
      }
      const uint32_t bv[8] = {bx0.x, bx0.y, bx0.z, bx0.w, bx1.x, bx1.y, bx1.z, bx1.w};
      int acc[4];
#define MOE_GU_GROUP(JJ)                                                                  \
  {                                                                                       \
    uint32_t a0, a1, a2, a3;                                                              \
    iq2_group_int8<JJ>(ra, c.lane4, c.sgn_lane, one, a0, a2);                            \
    iq2_group_int8<JJ>(rb, c.lane4, c.sgn_lane, one, a1, a3);                            \
    if (JJ == 0) mma_s8s8_zero(acc, a0, a1, a2, a3, bv[2 * JJ], bv[2 * JJ + 1]);          \
    else mma_s8s8(acc, a0, a1, a2, a3, bv[2 * JJ], bv[2 * JJ + 1]);                       \
  }
      MOE_GU_GROUP(0) MOE_GU_GROUP(1) MOE_GU_GROUP(2) MOE_GU_GROUP(3)
#undef MOE_GU_GROUP
      // this lane's columns: its own sub-block, digits hi and lo, rows g and g + 8
      i0 += (acc[0] * 128 + acc[1]) * iq2_odd(ra);
      i1 += (acc[2] * 128 + acc[3]) * iq2_odd(rb);
    }
    __syncwarp();
    if (c.lane == 0) mbar_arrive(&c.empty[s]);
    const float xsv = ld_sf(c.xs_s + (tok * (c.xpitch / 256) + kblk) * 4);
    const uint32_t w0 = j ? dp[1][0] : dp[0][0], w1 = j ? dp[1][1] : dp[0][1];
    const float d0 = bb ? half_hi(w0) : half_lo(w0);
    const float d1 = bb ? half_hi(w1) : half_lo(w1);
    f0 = fmaf(static_cast<float>(i0), d0 * xsv, f0);
    f1 = fmaf(static_cast<float>(i1), d1 * xsv, f1);
  }
  // the four lanes of a quad hold the four sub-block columns of rows g, g + 8
  f0 += __shfl_xor_sync(0xffffffffu, f0, 1);
  f0 += __shfl_xor_sync(0xffffffffu, f0, 2);
  f1 += __shfl_xor_sync(0xffffffffu, f1, 1);
  f1 += __shfl_xor_sync(0xffffffffu, f1, 2);
  if (tig == 0) {
    const size_t o = ((static_cast<size_t>(w.p0) * 2 + w.m) * a.KP + w.kp) * I + w.rb * kBoxRows + 16 * c.warp + g;
    if (index_ok(o + 8, a.gpart_n)) {
      a.gpart[o] = f0;
      a.gpart[o + 8] = f1;
    }
  }
  return true;
}

// One unit whose expert holds 2..4*MAXQ assignments. TPG tokens share one set
// of MMA columns (TPG tokens x 4/TPG sub-block slots x 2 digits); MAXQ column
// sets reuse the same A operands.
template <int TPG, int MAXQ, bool XS>
__device__ __forceinline__ bool gu_unit_multi(const GuTmaArgs& a, const GuCtx& c, RingPos& rp, const GuUnit& w,
                                              const uint32_t (&dp)[kMaxNB][2]) {
  constexpr int SPS = 4 / TPG;
  const int I = a.I, ne = w.ne, p0 = w.p0;
  const int ngroups = (ne + TPG - 1) / TPG;
  const int g = c.g, tig = c.tig;
  const int tslot_b = (g >> 1) % TPG, sslot_b = (g >> 1) / TPG, dig_b = g & 1;
  const int tslot_c = tig % TPG, sslot_c = tig / TPG;
  const int row_l = 16 * c.warp + g;
  // B of column set q: digit dig_b of token tb = q*TPG + tslot_b, elements e0 + 32*(sub-block) of the box
  int xtok[MAXQ];
  const float* xsc[MAXQ];
  bool bon[MAXQ];
#pragma unroll
  for (int q = 0; q < MAXQ; ++q) {
    const int tb = q * TPG + tslot_b, tc = q * TPG + tslot_c;
    bon[q] = q < ngroups && tb < ne;
    xtok[q] = bon[q] ? c.tok[p0 + tb] : 0;
    xsc[q] = (q < ngroups && tc < ne) ? c.xscl + c.tok[p0 + tc] * (c.xpitch / 256) : nullptr;
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
    if (!mbar_wait_bounded(&c.full[rp.s], rp.ph, a.err, ERR_TIMEOUT, a.wait_limit)) return false;
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
      // 2 ls + 1 of the sub-block of each column set, rows g and g + 8 (the same for every token group)
      int odd0[TPG], odd1[TPG];
#pragma unroll
      for (int jj = 0; jj < TPG; ++jj) {
        const int sbi = 4 * cc + jj * SPS + sslot_c;
        odd0[jj] = gu_odd(rg, sbi, g);
        odd1[jj] = gu_odd(rg + 1024, sbi, g);
      }
#pragma unroll
      for (int q = 0; q < MAXQ; ++q) {
        if (q >= ngroups) break;
#pragma unroll
        for (int jj = 0; jj < TPG; ++jj) {
          // column set jj covers sub-blocks 4cc + jj*SPS .. +SPS-1 of box j of the staged slice
          const int e = j * 512 + (4 * cc + jj * SPS + sslot_b) * 32 + 8 * tig;
          const int8_t* xp = bon[q] ? c.xdig + x_off(c.xpitch, xtok[q], dig_b, e) : c.zero + 8 * tig;
          const uint2 bl = *reinterpret_cast<const uint2*>(xp);
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
          iacc[q][0] += (acc[q][0] * 128 + acc[q][1]) * odd0[jj];
          iacc[q][1] += (acc[q][2] * 128 + acc[q][3]) * odd1[jj];
        }
      }
      {  // every four sub-blocks: with 14-bit activation digits a longer int32 sum could overflow
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
      const size_t o = ((static_cast<size_t>(p0 + t) * 2 + w.m) * a.KP + w.kp) * I + w.rb * kBoxRows + row_l;
      if (index_ok(o + 8, a.gpart_n)) {
        a.gpart[o] = facc[q][0];
        a.gpart[o + 8] = facc[q][1];
      }
    }
  }
  return true;
}


// The consumer loop of the one-token kernel (every expert holds one
// assignment, the activations are staged). The lane mapping and the operand
// construction are those of gu_unit_one; everything that depends only on the
// lane is computed once, the B operand is loaded unconditionally (lanes that
// carry no activations read the zero region, so no register is zeroed and no
// branch is taken per round), and the two fp16 row scales of a unit are
// loaded before its data wait and first used after its MMAs, so their latency
// never stalls the warp.
__device__ __forceinline__ void gu_consume_t1(const GuTmaArgs& a, const MetaSmem& ms, uint64_t* full, uint64_t* empty,
                                              uint32_t ring_s, uint32_t x_s, uint32_t xs_s, uint32_t zero_s, int warp,
                                              int lane) {
  const int H = a.H, I = a.I, KP = a.KP, S = a.S, rbs = I / kBoxRows;
  const int nact = ms.act[a.E];
  const int g = lane >> 2, tig = lane & 3, bb = tig >> 1, hf = tig & 1;
  const uint32_t lane4 = static_cast<uint32_t>(lane) << 2, sgn_lane = 128u + lane4;
  const uint32_t one = static_cast<uint32_t>(a.one);
  // this lane's round-0 record of row g (chunk (4bb) ^ g, half hf) inside stage 0
  const uint32_t ring_lane = ring_s + static_cast<uint32_t>(16 * warp + g) * kGuW +
                             (((static_cast<uint32_t>(g) ^ (4u * bb)) << 4) | (8u * hf));
  // B: the x digits of this lane's column (block 2kp + bb of the x_off layout: kp steps 1024 bytes), or zeros
  const bool bact = (g >> 1) == tig;
  const uint32_t xb_base = bact ? x_s + static_cast<uint32_t>(x_off(H, 0, g & 1, bb * 256 + hf * 32)) : zero_s;
  const uint32_t xb_step = bact ? 1024u : 0u;
  const uint32_t xs_lane = xs_s + 4u * bb;  // + 8 kp: the 2^s / 8 of block 2kp + bb
  const int row_l = 16 * warp + g;
  const int dstride = H / 256;
  RingPos rp{0, 0u};
  GuIter t;
  t.init(blockIdx.x, gridDim.x, KP, rbs);
  for (; t.slot < nact; t.next(KP, rbs)) {
    const int e = ms.act[t.slot];
    const uint16_t* dr = (t.m ? a.up_d : a.gate_d) +
                         (static_cast<size_t>(e) * I + t.rb * kBoxRows + row_l) * dstride + 2 * t.kp;
    const uint32_t dw0 = __ldg(reinterpret_cast<const uint32_t*>(dr));                 // row g: blocks 2kp, 2kp+1
    const uint32_t dw1 = __ldg(reinterpret_cast<const uint32_t*>(dr + 8 * dstride));  // row g + 8
    const uint32_t xb0 = xb_base + static_cast<uint32_t>(t.kp) * xb_step, xb1 = xb0 ^ 16u;
    if (!mbar_wait_bounded(&full[rp.s], rp.ph, a.err, ERR_TIMEOUT, a.wait_limit)) return;
    const uint32_t r0 = ring_lane + static_cast<uint32_t>(rp.s) * kGuBox;
    const int s = rp.s;
    rp.next(S);
    int i0 = 0, i1 = 0;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      const uint2 ra = ld_s64(r0 ^ (16u * cc));          // row g
      const uint2 rb = ld_s64((r0 ^ (16u * cc)) + 1024);  // row g + 8
      const uint4 bx0 = ld_s128(xb0 + 128u * cc);
      const uint4 bx1 = ld_s128(xb1 + 128u * cc);
      const uint32_t bv[8] = {bx0.x, bx0.y, bx0.z, bx0.w, bx1.x, bx1.y, bx1.z, bx1.w};
      int acc[4];
#define MOE_GU_GROUP(JJ)                                                                  \
  {                                                                                       \
    uint32_t a0, a1, a2, a3;                                                              \
    iq2_group_int8<JJ>(ra, lane4, sgn_lane, one, a0, a2);                                \
    iq2_group_int8<JJ>(rb, lane4, sgn_lane, one, a1, a3);                                \
    if (JJ == 0) mma_s8s8_zero(acc, a0, a1, a2, a3, bv[2 * JJ], bv[2 * JJ + 1]);          \
    else mma_s8s8(acc, a0, a1, a2, a3, bv[2 * JJ], bv[2 * JJ + 1]);                       \
  }
      MOE_GU_GROUP(0) MOE_GU_GROUP(1) MOE_GU_GROUP(2) MOE_GU_GROUP(3)
#undef MOE_GU_GROUP
      i0 += (acc[0] * 128 + acc[1]) * iq2_odd(ra);
      i1 += (acc[2] * 128 + acc[3]) * iq2_odd(rb);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    const float xsv = ld_sf(xs_lane + 8u * static_cast<uint32_t>(t.kp));
    const float d0 = bb ? half_hi(dw0) : half_lo(dw0);
    const float d1 = bb ? half_hi(dw1) : half_lo(dw1);
    float f0 = static_cast<float>(i0) * (d0 * xsv);
    float f1 = static_cast<float>(i1) * (d1 * xsv);
    f0 += __shfl_xor_sync(0xffffffffu, f0, 1);
    f0 += __shfl_xor_sync(0xffffffffu, f0, 2);
    f1 += __shfl_xor_sync(0xffffffffu, f1, 1);
    f1 += __shfl_xor_sync(0xffffffffu, f1, 2);
    if (tig == 0) {
      const size_t o = ((static_cast<size_t>(ms.off[e]) * 2 + t.m) * KP + t.kp) * I + t.rb * kBoxRows + row_l;
      if (index_ok(o + 8, a.gpart_n)) {
        a.gpart[o] = f0;
        a.gpart[o + 8] = f1;
      }
    }
  }
}

// Shared-memory plan of the gate/up kernel (host and device agree on it); the
// selector tables come first, at a fixed shared address, so lookups need no
// base add.
struct GuPlan {
  size_t tab, meta, zero, x, xs, ring, bars, total;
};
// Hx: the activation columns staged per CTA (all of H for one token; for more
// tokens the CTA's fixed NB*512-column slice).
__host__ __device__ inline GuPlan gu_plan(int E, int T, int k, int Hx, bool xs_in, int S) {
  GuPlan p;
  p.tab = 0;
  p.meta = kTabBytes;
  p.zero = p.meta + meta_bytes(E, T * k, true);
  p.x = p.zero + kZeroBytes;
  p.xs = p.x + (xs_in ? align_up(static_cast<size_t>(T) * 2 * Hx, 128) : 0);
  const size_t end = p.xs + (xs_in ? align_up(static_cast<size_t>(T) * (Hx / 256) * 4, 128) : 0);
  p.ring = align_up(end, 1024);
  p.bars = p.ring + static_cast<size_t>(S) * kGuBox;
  p.total = p.bars + (2 * static_cast<size_t>(S) + 1) * 8;  // full[S], empty[S], the table copy
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
  // staged activation columns: all of H for one token; otherwise the CTA serves one fixed part kpc of H
  // (units walked over (slot, m, rb) by the CTAs of that part) and stages that NB*512-column slice only
  const int Hx = MAXQ == 1 ? H : NB * 512;
  const int kpc = MAXQ == 1 ? 0 : static_cast<int>(blockIdx.x % a.KP);
  const int kib = MAXQ == 1 ? static_cast<int>(blockIdx.x) : static_cast<int>(blockIdx.x / a.KP);
  const int kG = MAXQ == 1 ? static_cast<int>(gridDim.x) : static_cast<int>((gridDim.x - kpc + a.KP - 1) / a.KP);
  const GuPlan pl = gu_plan(a.E, T, a.k, Hx, XS, S);
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
  uint64_t* tabbar = empty + S;
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kCW);
    }
    mbar_init(tabbar, 1);
    fence_barrier_init();
    // the selector tables: one 64 KB bulk copy, in flight while the rest of the prologue runs
    mbar_arrive_expect_tx(tabbar, kTabBytes);
    bulk_copy_g2s(smem + pl.tab, &g_sel_rep, kTabBytes, tabbar);
  }
  for (int i = tid; i < kZeroBytes / 16; i += kThreadsT) reinterpret_cast<uint4*>(zero)[i] = make_uint4(0, 0, 0, 0);
  pdl_wait();  // routing and activations come from the kernels before this one
  load_meta(ms, a.offsets, a.active, a.perm, a.E, nA, a.k, tid, kThreadsT);
  __syncthreads();  // barriers, zero region and routing metadata are in place: the producer may start
  const int nact = ms.act[a.E];

  if (warp == kCW) {  // producer
    if (lane == 0 && !a.no_produce) {
      prefetch_tmap(&tm_gate);
      prefetch_tmap(&tm_up);
      const uint64_t pol = l2_policy_evict_first();  // expert codes are read once per step
      RingPos rp{0, 0u};
      GuIter t;
      t.init(kib, kG, MAXQ == 1 ? a.KP : 1, rbs);
      for (; t.slot < nact; t.next(MAXQ == 1 ? a.KP : 1, rbs)) {
        const int e = ms.act[t.slot];
        const int kp = MAXQ == 1 ? t.kp : kpc;
        for (int j = 0; j < NB; ++j) {
          if (!mbar_wait_bounded(&empty[rp.s], rp.ph ^ 1u, a.err, ERR_TIMEOUT, a.wait_limit)) return;
          mbar_arrive_expect_tx(&full[rp.s], kGuBox);
          index_ok(static_cast<size_t>(e) * I + t.rb * kBoxRows + kBoxRows - 1, static_cast<size_t>(a.E) * I);
          index_ok(static_cast<size_t>(kp * NB + j) * kGuW + kGuW - 1, static_cast<size_t>(H) / 4);
          tma_load_2d_hint(ring + rp.s * kGuBox, t.m ? &tm_up : &tm_gate, (kp * NB + j) * kGuW,
                           e * I + t.rb * kBoxRows, &full[rp.s], pol);
          rp.next(S);
        }
      }
    }
    return;
  }

  // consumers: stage the activations while the first boxes are in flight
  if (XS) {  // columns [kpc Hx, kpc Hx + Hx) of the [T][2][H] digits -> the x_off layout of an Hx-column
             // matrix, 16 bytes at a time, asynchronously; their 2^s/8 scales likewise
    const int per = Hx / 16;
    for (int i = tid; i < T * 2 * per; i += kCW * 32) {
      const int row = i / per, e = (i - row * per) * 16;
      cp_async16(smem_addr(xsm + x_off(Hx, row >> 1, row & 1, e)),
                 a.xd + static_cast<size_t>(row) * H + static_cast<size_t>(kpc) * Hx + e);
    }
    const int bpr = Hx / 256;
    for (int i = tid; i < T * bpr; i += kCW * 32) {
      const int tt = i / bpr;
      xssm[i] = a.xs[tt * (H / 256) + kpc * bpr + (i - tt * bpr)];
    }
    cp_async_wait_all();
  }
  named_barrier(1, kCW * 32);
  // the table copy must have landed before the first lookup (the producer never reads it)
  if (!mbar_wait_bounded(tabbar, 0, a.err, ERR_TIMEOUT, a.wait_limit)) return;
  if (MAXQ == 1) {  // one token
    gu_consume_t1(a, ms, full, empty, smem_addr(ring), smem_addr(xsm), smem_addr(xssm), smem_addr(zero), warp, lane);
    return;
  }
  GuCtx c;
  c.tab = reinterpret_cast<const char*>(smem + pl.tab);
  c.ring = ring;
  c.full = full;
  c.empty = empty;
  c.xdig = xsm;  // the staged slice (x_off layout of an Hx-column matrix)
  c.xscl = xssm;
  c.zero = zero;
  c.xpitch = Hx;
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
  t.init(kib, kG, 1, rbs);
  uint32_t nd[kMaxNB][2] = {};
  GuUnit nw{};
  if (t.slot < nact) {
    nw = gu_unit_of(t, ms);
    nw.kp = kpc;
    dload(nw, nd);
  }
  while (t.slot < nact) {
    const GuUnit w = nw;
    uint32_t d[kMaxNB][2];
#pragma unroll
    for (int j = 0; j < kMaxNB; ++j) d[j][0] = nd[j][0], d[j][1] = nd[j][1];
    t.next(1, rbs);
    if (t.slot < nact) {
      nw = gu_unit_of(t, ms);
      nw.kp = kpc;
      dload(nw, nd);
    }
    bool ok;
    if (MAXQ == 1 || w.ne == 1) ok = gu_unit_one<XS>(a, c, rp, w, d);
    else if (w.ne == 2) ok = gu_unit_multi<2, 1, XS>(a, c, rp, w, d);
    else ok = gu_unit_multi<4, (MAXQ > 1 ? MAXQ : 1), XS>(a, c, rp, w, d);
    if (!ok) return;
  }
}

// ===========================================================================
// down
// ===========================================================================
// A down box is one Q2K block of 256 rows, brought in as two TMA boxes of the
// same rows: the 64 q bytes with the 64-byte swizzle (rows 64 bytes apart,
// 16-byte chunk c of row R at c ^ ((R >> 1) & 3)) and the 16 scale bytes dense.
constexpr int kDnQBytes = kBoxRows * 64;             // 16 KB
constexpr int kDnSBytes = kBoxRows * 16;             // 4 KB
constexpr int kDnStage = kDnQBytes + kDnSBytes;      // 20 KB, a multiple of 1024


struct DnTmaArgs {
  int H, I, E, k, T, DP, NB, S;
  const uint32_t* dd;
  const int8_t* hd;
  const float* hsc;
  const int32_t* hq;
  const int32_t* offsets;
  const int32_t* active;
  float* opart;  // [T*k][DP][H]
  size_t opart_n;  // its length in floats (bounds-checked build)
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
  const int8_t* hd;    // h digits (h_off layout), staged or global
  const float* hsc;    // [T*k][hss]
  const int32_t* hq;   // [T*k][I/16]
  const int8_t* zero;  // 128-byte aligned zero region
  uint32_t ring_s, hd_s, hsc_s, hq_s;  // shared-window addresses (staged variant)
  int warp, lane, g, tig, S;
  int hI, hqp, hsp;  // h_off pitch, hq and hsc entries per assignment (staged slice or global)
};

__device__ __forceinline__ float dn_block(uint32_t dd, float e2, int iA, int iM) {
  return e2 * fmaf(half_lo(dd), static_cast<float>(iA), -half_hi(dd) * static_cast<float>(iM));
}

// Q2K A operands of one 16-weight sub-block word for one row: bit pair r of
// its four bytes (weights 4i + r) -> uint8 bytes. The shifts are multiplies
// (FMA pipe), the masks LOP3s.
__device__ __forceinline__ void q2k_sub4(uint32_t w, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  r0 = w & 0x03030303u;
  r1 = __umulhi(w, 1u << 30) & 0x03030303u;
  r2 = __umulhi(w, 1u << 28) & 0x03030303u;
  r3 = __umulhi(w, 1u << 26) & 0x03030303u;
}

// One down unit whose expert holds a single assignment.
//
// Lane mapping (m16n8k32, lane = 4g + tig): rows g and g+8 of the warp's 16; in
// round cc (0..3) the lane owns sub-block 4*tig + cc of the block, whole: two
// MMAs take its bit pairs (0, 1) and (2, 3). Its four q words are one 16-byte
// chunk per row and its four scale bytes one word per row, loaded once per
// box, after which the stage is released. MMA columns are (owner tig, digit
// hi/lo); B is non-zero on the lanes with g >> 1 == tig (one 16-byte load of
// h digits per round), so the accumulators of lane tig hold its own sub-block.
template <bool HS>
__device__ __forceinline__ bool dn_unit_one(const DnTmaArgs& a, const DnCtx& c, RingPos& rp, const DnUnit& w,
                                            const uint32_t (&dd)[kMaxNB][2]) {
  const int H = a.H, NB = a.NB;
  const int g = c.g, tig = c.tig;
  const bool bact = (g >> 1) == tig;
  const int row = 16 * c.warp + g;
  const uint32_t qoff = static_cast<uint32_t>(row) * 64 + 16u * (static_cast<uint32_t>(tig) ^ ((g >> 1) & 3));
  const uint32_t soff = kDnQBytes + static_cast<uint32_t>(row) * 16 + 4u * tig;
  float f0 = 0.f, f1 = 0.f;
#pragma unroll 1
  for (int j = 0; j < NB; ++j) {
    const int blk = (HS ? 0 : w.dp * NB) + j;  // block of the staged slice, or of I
    const int hb = h_off(c.hI, w.p0, g & 1, blk * 256 + 64 * tig);  // sub-block 4 tig, round 0
    const int hqi = w.p0 * c.hqp + blk * 16 + 4 * tig;
    int4 hq4;
    float e2;
    if (HS) {
      const uint4 v = ld_s128(c.hq_s + hqi * 4);
      hq4 = make_int4(static_cast<int>(v.x), static_cast<int>(v.y), static_cast<int>(v.z), static_cast<int>(v.w));
      e2 = ld_sf(c.hsc_s + (w.p0 * c.hsp + blk) * 4);
    } else {
      hq4 = __ldcg(reinterpret_cast<const int4*>(c.hq + hqi));
      e2 = __ldcg(c.hsc + w.p0 * c.hsp + blk);
    }
    if (!mbar_wait_bounded(&c.full[rp.s], rp.ph, a.err, ERR_TIMEOUT)) return false;
    const uint32_t st = c.ring_s + rp.s * kDnStage;
    const uint4 qa = ld_s128(st + qoff), qb = ld_s128(st + qoff + 8 * 64);
    const uint32_t sa = ld_s32(st + soff), sb = ld_s32(st + soff + 8 * 16);
    __syncwarp();
    if (c.lane == 0) mbar_arrive(&c.empty[rp.s]);  // the codes are in registers: the stage is free
    rp.next(c.S);
    const uint32_t wa[4] = {qa.x, qa.y, qa.z, qa.w}, wb[4] = {qb.x, qb.y, qb.z, qb.w};
    const int hqv[4] = {hq4.x, hq4.y, hq4.z, hq4.w};
    int iA0 = 0, iA1 = 0, iM0 = 0, iM1 = 0;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      uint4 bh = make_uint4(0u, 0u, 0u, 0u);
      if (bact) {
        if (HS) bh = ld_s128(c.hd_s + hb + 128 * cc);
        else bh = __ldcg(reinterpret_cast<const uint4*>(c.hd + hb + 128 * cc));
      }
      uint32_t x0, x1, x2, x3, y0, y1, y2, y3;
      q2k_sub4(wa[cc], x0, x1, x2, x3);
      q2k_sub4(wb[cc], y0, y1, y2, y3);
      int acc[4];
      mma_u8s8_zero(acc, x0, y0, x1, y1, bh.x, bh.y);
      mma_u8s8(acc, x2, y2, x3, y3, bh.z, bh.w);
      const uint32_t ba = cc ? __umulhi(sa, 1u << (32 - 8 * cc)) : sa;  // scale byte cc at bits 0..7
      const uint32_t bb = cc ? __umulhi(sb, 1u << (32 - 8 * cc)) : sb;
      iA0 += (acc[0] * 128 + acc[1]) * static_cast<int>(ba & 15u);
      iA1 += (acc[2] * 128 + acc[3]) * static_cast<int>(bb & 15u);
      iM0 += static_cast<int>((ba >> 4) & 15u) * hqv[cc];
      iM1 += static_cast<int>((bb >> 4) & 15u) * hqv[cc];
    }
    const uint32_t dA = j ? dd[1][0] : dd[0][0], dB = j ? dd[1][1] : dd[0][1];
    f0 += dn_block(dA, e2, iA0, iM0);
    f1 += dn_block(dB, e2, iA1, iM1);
  }
  // the four lanes of a quad hold the four quarters of the block of rows g, g + 8
  f0 += __shfl_xor_sync(0xffffffffu, f0, 1);
  f0 += __shfl_xor_sync(0xffffffffu, f0, 2);
  f1 += __shfl_xor_sync(0xffffffffu, f1, 1);
  f1 += __shfl_xor_sync(0xffffffffu, f1, 2);
  if (tig == 0) {
    const size_t o = (static_cast<size_t>(w.p0) * a.DP + w.dp) * H + w.rb * kBoxRows + row;
    if (index_ok(o + 8, a.opart_n)) {
      a.opart[o] = f0;
      a.opart[o + 8] = f1;
    }
  }
  return true;
}

// One down unit for an expert with 2..2*MAXQ assignments, taken four at a time.
// Each sub-block's 4-bit scale sc is folded into its uint8 A operand: sc * q is
// at most 45, so the 32-bit product of the four q bytes with sc carries nothing
// from byte to byte. An MMA then spans two whole sub-blocks (K 0..15: sub-block
// 2pr, K 16..31: 2pr + 1, lane tig bit pair tig of their bytes) and its
// accumulators sum sc * q * h over the whole block, with no scaling per MMA.
// MMA columns: (assignment slot 0..3) x (digit hi, lo), so lane tig's
// accumulators hold slot tig's two digits for rows g and g + 8. The min term
// sums m * (per-16 sum of h) over the block's sub-blocks per row and slot.
template <int MAXQ, bool HS>
__device__ __forceinline__ bool dn_unit_multi(const DnTmaArgs& a, const DnCtx& c, RingPos& rp, const DnUnit& w,
                                              const uint32_t (&dd)[kMaxNB][2]) {
  constexpr int G = (2 * MAXQ + 3) / 4;  // groups of four assignments
  const int H = a.H, ne = w.ne, p0 = w.p0;
  const int bb0 = HS ? 0 : w.dp * a.NB;  // first block of the unit in the staged slice, or in I
  const int g = c.g, tig = c.tig;
  const int ngroups = (ne + 3) / 4;
  const int dig_b = g & 1, sl_b = g >> 1;  // this lane's B column: slot sl_b, digit dig_b
  const uint32_t sh = 2 * tig;
  const int row = 16 * c.warp + g;
  int pb[G];                // assignment of this lane's B column per group (-1: zero column)
  const int32_t* hq_ptr[G]; // per-16 sums of the assignment in slot tig
  const float* e2p[G];
#pragma unroll
  for (int q = 0; q < G; ++q) {
    const int tb = 4 * q + sl_b, tc = 4 * q + tig;
    pb[q] = (q < ngroups && tb < ne) ? p0 + tb : -1;
    const bool cv = q < ngroups && tc < ne;
    hq_ptr[q] = c.hq + (p0 + (cv ? tc : 0)) * c.hqp + bb0 * 16;
    e2p[q] = cv ? c.hsc + (p0 + tc) * c.hsp + bb0 : nullptr;
  }
  float facc[G][2];
#pragma unroll
  for (int q = 0; q < G; ++q) facc[q][0] = facc[q][1] = 0.f;
  const uint32_t qoff = static_cast<uint32_t>(row) * 64;
  const uint32_t qsw = static_cast<uint32_t>((g >> 1) & 3);
#pragma unroll 1
  for (int j = 0; j < a.NB; ++j) {
    int acc[G][4], iM[G][2];
#pragma unroll
    for (int q = 0; q < G; ++q) {
      acc[q][0] = acc[q][1] = acc[q][2] = acc[q][3] = 0;
      iM[q][0] = iM[q][1] = 0;
    }
    if (!mbar_wait_bounded(&c.full[rp.s], rp.ph, a.err, ERR_TIMEOUT)) return false;
    const int s = rp.s;
    rp.next(c.S);
    const uint8_t* st = c.ring + s * kDnStage;
    const uint8_t* sA = st + kDnQBytes + row * 16;  // scale bytes (sc | m << 4) of the 16 sub-blocks, row g
    const uint8_t* sB = sA + 8 * 16;                // row g + 8
    const int blk = bb0 + j;
#pragma unroll 1
    for (int cc = 0; cc < 4; ++cc) {  // logical 16-byte chunk cc of the q bytes: sub-blocks 4cc .. 4cc + 3
      const uint4 qa = lds128(st + qoff + 16 * (cc ^ qsw));
      const uint4 qb = lds128(st + qoff + 8 * 64 + 16 * (cc ^ qsw));
      const uint32_t wa = *reinterpret_cast<const uint32_t*>(sA + 4 * cc);
      const uint32_t wb = *reinterpret_cast<const uint32_t*>(sB + 4 * cc);
      uint32_t af[2][4];
      af[0][0] = q2k_quad(qa.x, sh) * (wa & 15u);
      af[0][1] = q2k_quad(qb.x, sh) * (wb & 15u);
      af[0][2] = q2k_quad(qa.y, sh) * ((wa >> 8) & 15u);
      af[0][3] = q2k_quad(qb.y, sh) * ((wb >> 8) & 15u);
      af[1][0] = q2k_quad(qa.z, sh) * ((wa >> 16) & 15u);
      af[1][1] = q2k_quad(qb.z, sh) * ((wb >> 16) & 15u);
      af[1][2] = q2k_quad(qa.w, sh) * ((wa >> 24) & 15u);
      af[1][3] = q2k_quad(qb.w, sh) * ((wb >> 24) & 15u);
      const int ma[4] = {static_cast<int>((wa >> 4) & 15u), static_cast<int>((wa >> 12) & 15u),
                         static_cast<int>((wa >> 20) & 15u), static_cast<int>(wa >> 28)};
      const int mb[4] = {static_cast<int>((wb >> 4) & 15u), static_cast<int>((wb >> 12) & 15u),
                         static_cast<int>((wb >> 20) & 15u), static_cast<int>(wb >> 28)};
#pragma unroll
      for (int q = 0; q < G; ++q) {
        if (q >= ngroups) break;
        const int4 hv = *reinterpret_cast<const int4*>(hq_ptr[q] + j * 16 + 4 * cc);
        iM[q][0] += ma[0] * hv.x + ma[1] * hv.y + ma[2] * hv.z + ma[3] * hv.w;
        iM[q][1] += mb[0] * hv.x + mb[1] * hv.y + mb[2] * hv.z + mb[3] * hv.w;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          uint32_t b0 = 0u, b1 = 0u;
          if (pb[q] >= 0) {  // bit pair tig of sub-blocks 4cc + 2u and 4cc + 2u + 1 (elements tig + 4i)
            const int e0 = blk * 256 + (4 * cc + 2 * u) * 16 + tig;
            b0 = *reinterpret_cast<const uint32_t*>(c.hd + h_off(c.hI, pb[q], dig_b, e0));
            b1 = *reinterpret_cast<const uint32_t*>(c.hd + h_off(c.hI, pb[q], dig_b, e0 + 16));
          }
          mma_u8s8(acc[q], af[u][0], af[u][1], af[u][2], af[u][3], b0, b1);
        }
      }
    }
    __syncwarp();
    if (c.lane == 0) mbar_arrive(&c.empty[s]);
    const uint32_t dA = j ? dd[1][0] : dd[0][0], dB = j ? dd[1][1] : dd[0][1];
#pragma unroll
    for (int q = 0; q < G; ++q) {
      const float e2 = e2p[q] ? e2p[q][j] : 0.f;
      facc[q][0] += dn_block(dA, e2, acc[q][0] * 128 + acc[q][1], iM[q][0]);
      facc[q][1] += dn_block(dB, e2, acc[q][2] * 128 + acc[q][3], iM[q][1]);
    }
  }
#pragma unroll
  for (int q = 0; q < G; ++q) {
    const int t = 4 * q + tig;
    if (q < ngroups && t < ne) {
      const size_t o = (static_cast<size_t>(p0 + t) * a.DP + w.dp) * H + w.rb * kBoxRows + row;
      if (index_ok(o + 8, a.opart_n)) {
        a.opart[o] = facc[q][0];
        a.opart[o + 8] = facc[q][1];
      }
    }
  }
  return true;
}

// The consumer loop of the one-token down kernel (every expert holds one
// assignment, h staged). Lane mapping and operands are those of dn_unit_one;
// lane-only addresses are computed once, B is loaded unconditionally (lanes
// without h read the zero region), and the two Q2K block scale words of a unit
// are loaded before its data wait and first used after its MMAs.
__device__ __forceinline__ void dn_consume_t1(const DnTmaArgs& a, const MetaSmem& ms, uint64_t* full, uint64_t* empty,
                                              uint32_t ring_s, uint32_t hd_s, uint32_t hsc_s, uint32_t hq_s,
                                              uint32_t zero_s, int warp, int lane) {
  const int H = a.H, I = a.I, DP = a.DP, S = a.S, rbs = H / kBoxRows, nblk = I / 256;
  const int nact = ms.act[a.E];
  const int g = lane >> 2, tig = lane & 3;
  const bool bact = (g >> 1) == tig;
  const int row = 16 * warp + g;
  const uint32_t qoff = static_cast<uint32_t>(row) * 64 + 16u * (static_cast<uint32_t>(tig) ^ ((g >> 1) & 3));
  const uint32_t soff = kDnQBytes + static_cast<uint32_t>(row) * 16 + 4u * tig;
  RingPos rp{0, 0u};
  DnIter t;
  t.init(blockIdx.x, gridDim.x, DP, rbs);
  for (; t.slot < nact; t.next(DP, rbs)) {
    const int e = ms.act[t.slot];
    const int p0 = ms.off[e];
    const int blk = t.dp;
    const uint32_t* dr = a.dd + (static_cast<size_t>(e) * H + t.rb * kBoxRows + row) * nblk + blk;
    const uint32_t dA = __ldg(dr), dB = __ldg(dr + 8 * nblk);
    // sub-block 4 tig of block blk, round 0 (rounds step 128 bytes; the zero region covers them too)
    const uint32_t hb = bact ? hd_s + static_cast<uint32_t>(h_off(I, p0, g & 1, blk * 256 + 64 * tig)) : zero_s;
    const uint4 hqv = ld_s128(hq_s + 4u * static_cast<uint32_t>(p0 * (I / 16) + blk * 16 + 4 * tig));
    const float e2 = ld_sf(hsc_s + 4u * static_cast<uint32_t>(p0 * a.hss + blk));
    if (!mbar_wait_bounded(&full[rp.s], rp.ph, a.err, ERR_TIMEOUT)) return;
    const uint32_t st = ring_s + static_cast<uint32_t>(rp.s) * kDnStage;
    const uint4 qa = ld_s128(st + qoff), qb = ld_s128(st + qoff + 8 * 64);
    const uint32_t sa = ld_s32(st + soff), sb = ld_s32(st + soff + 8 * 16);
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[rp.s]);  // the codes are in registers: the stage is free
    rp.next(S);
    const uint32_t wa[4] = {qa.x, qa.y, qa.z, qa.w}, wb[4] = {qb.x, qb.y, qb.z, qb.w};
    const int hq[4] = {static_cast<int>(hqv.x), static_cast<int>(hqv.y), static_cast<int>(hqv.z),
                       static_cast<int>(hqv.w)};
    int iA0 = 0, iA1 = 0, iM0 = 0, iM1 = 0;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      const uint4 bh = ld_s128(hb + 128u * cc);
      uint32_t x0, x1, x2, x3, y0, y1, y2, y3;
      q2k_sub4(wa[cc], x0, x1, x2, x3);
      q2k_sub4(wb[cc], y0, y1, y2, y3);
      int acc[4];
      mma_u8s8_zero(acc, x0, y0, x1, y1, bh.x, bh.y);
      mma_u8s8(acc, x2, y2, x3, y3, bh.z, bh.w);
      const uint32_t ba = cc ? __umulhi(sa, 1u << (32 - 8 * cc)) : sa;  // scale byte cc at bits 0..7
      const uint32_t bs = cc ? __umulhi(sb, 1u << (32 - 8 * cc)) : sb;
      iA0 += (acc[0] * 128 + acc[1]) * static_cast<int>(ba & 15u);
      iA1 += (acc[2] * 128 + acc[3]) * static_cast<int>(bs & 15u);
      iM0 += static_cast<int>((ba >> 4) & 15u) * hq[cc];
      iM1 += static_cast<int>((bs >> 4) & 15u) * hq[cc];
    }
    float f0 = dn_block(dA, e2, iA0, iM0);
    float f1 = dn_block(dB, e2, iA1, iM1);
    f0 += __shfl_xor_sync(0xffffffffu, f0, 1);
    f0 += __shfl_xor_sync(0xffffffffu, f0, 2);
    f1 += __shfl_xor_sync(0xffffffffu, f1, 1);
    f1 += __shfl_xor_sync(0xffffffffu, f1, 2);
    if (tig == 0) {
      const size_t o = (static_cast<size_t>(p0) * DP + blk) * H + t.rb * kBoxRows + row;
      if (index_ok(o + 8, a.opart_n)) {
        a.opart[o] = f0;
        a.opart[o + 8] = f1;
      }
    }
  }
}

// Shared-memory plan of the down kernel.
struct DnPlan {
  size_t meta, zero, hd, hsc, hq, ring, bars, total;
};
// Ix, hssx: the h columns and scale entries staged per assignment (all of I for
// one token; for more tokens the CTA's fixed NB*256-column slice, NB scales).
__host__ __device__ inline DnPlan dn_plan(int E, int nA, int Ix, int hssx, bool hs_in, int S) {
  DnPlan p;
  p.meta = 0;
  p.zero = meta_bytes(E, nA, false);
  p.hd = p.zero + kZeroBytes;
  p.hsc = p.hd + (hs_in ? align_up(static_cast<size_t>(nA) * 2 * Ix, 128) : 0);
  p.hq = p.hsc + (hs_in ? align_up(static_cast<size_t>(nA) * hssx * 4, 128) : 0);
  const size_t end = p.hq + (hs_in ? align_up(static_cast<size_t>(nA) * (Ix / 16) * 4, 128) : 0);
  p.ring = align_up(end, 1024);
  p.bars = p.ring + static_cast<size_t>(S) * kDnStage;
  p.total = p.bars + 2 * static_cast<size_t>(S) * 8;
  return p;
}

template <int MAXQ, bool HS>
__global__ void __launch_bounds__(kThreadsT, 1) down_tma_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                                const __grid_constant__ CUtensorMap tm_s,
                                                                DnTmaArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  pdl_trigger();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = a.H, I = a.I, S = a.S, NB = a.NB;
  const int nA = a.T * a.k;
  // staged h: all of I for one token; for more tokens (HS) the CTA serves one fixed part dpc of I (units
  // walked over (slot, rb) by the CTAs of that part) and stages that NB*256-column slice of every assignment
  const bool slice = MAXQ > 1 && HS;
  const int Ix = slice ? NB * 256 : I, hssx = slice ? NB : a.hss;
  const int dpc = slice ? static_cast<int>(blockIdx.x % a.DP) : 0;
  const int dib = slice ? static_cast<int>(blockIdx.x / a.DP) : static_cast<int>(blockIdx.x);
  const int dG = slice ? static_cast<int>((gridDim.x - dpc + a.DP - 1) / a.DP) : static_cast<int>(gridDim.x);
  const DnPlan pl = dn_plan(a.E, nA, Ix, hssx, HS, S);
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

  if ((smem_addr(ring) & 1023u) != 0) {  // the swizzled q boxes assume 1024-byte aligned stages
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
  for (int i = tid; i < kZeroBytes / 16; i += kThreadsT) reinterpret_cast<uint4*>(zero)[i] = make_uint4(0, 0, 0, 0);
  pdl_wait();  // routing and h come from the kernels before this one
  load_meta(ms, a.offsets, a.active, nullptr, a.E, nA, a.k, tid, kThreadsT);
  __syncthreads();  // barriers, zero region and routing metadata are in place: the producer may start
  const int nact = ms.act[a.E];

  if (warp == kCW) {  // producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_s);
      const uint64_t pol = l2_policy_evict_first();  // expert codes are read once per step
      RingPos rp{0, 0u};
      DnIter t;
      t.init(dib, dG, slice ? 1 : a.DP, rbs);
      for (; t.slot < nact; t.next(slice ? 1 : a.DP, rbs)) {
        const int e = ms.act[t.slot];
        const int dp = slice ? dpc : t.dp;
        for (int j = 0; j < NB; ++j) {
          if (!mbar_wait_bounded(&empty[rp.s], rp.ph ^ 1u, a.err, ERR_TIMEOUT)) return;
          mbar_arrive_expect_tx(&full[rp.s], kDnStage);
          const int x0 = (dp * NB + j) * 80, y0 = e * H + t.rb * kBoxRows;
          index_ok(static_cast<size_t>(y0) + kBoxRows - 1, static_cast<size_t>(a.E) * H);
          index_ok(static_cast<size_t>(x0) + 79, static_cast<size_t>(I / 256) * 80);
          uint8_t* st = ring + rp.s * kDnStage;
          tma_load_2d_hint(st, &tm_q, x0 + 16, y0, &full[rp.s], pol);
          tma_load_2d_hint(st + kDnQBytes, &tm_s, x0, y0, &full[rp.s], pol);
          rp.next(S);
        }
      }
    }
    return;
  }
  // consumers: stage h while the first boxes are in flight (the h_off layout is the same in global and
  // shared memory; I % 256 == 0 makes both byte counts multiples of 16)
  if (HS) {  // per assignment: h digits of blocks [dpc NB, dpc NB + NB) (contiguous in the h_off layout, here
             // and in the slice), their per-16 sums and their scales; with slice == false all of them
    const int hc = Ix / 8, qc = Ix / 64;  // 16-byte chunks per assignment: h digits, per-16 sums
    for (int i = tid; i < nA * hc; i += kCW * 32) {
      const int pp = i / hc, cidx = i - pp * hc;
      cp_async16(smem_addr(hd_s) + 16u * i,
                 a.hd + static_cast<size_t>(pp) * 2 * I + static_cast<size_t>(dpc) * NB * 512 + 16 * cidx);
    }
    for (int i = tid; i < nA * qc; i += kCW * 32) {
      const int pp = i / qc, cidx = i - pp * qc;
      cp_async16(smem_addr(hq_s) + 16u * i, a.hq + static_cast<size_t>(pp) * (I / 16) + dpc * NB * 16 + 4 * cidx);
    }
    for (int i = tid; i < nA * hssx; i += kCW * 32) {
      const int pp = i / hssx;
      hsc_s[i] = a.hsc[static_cast<size_t>(pp) * a.hss + dpc * NB + (i - pp * hssx)];
    }
    cp_async_wait_all();
  }
  named_barrier(1, kCW * 32);
  if (MAXQ == 1) {  // one token
    dn_consume_t1(a, ms, full, empty, smem_addr(ring), smem_addr(hd_s), smem_addr(hsc_s), smem_addr(hq_s),
                  smem_addr(zero), warp, lane);
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
    c.hd_s = smem_addr(hd_s);
    c.hsc_s = smem_addr(hsc_s);
    c.hq_s = smem_addr(hq_s);
  } else {
    c.hd = a.hd;
    c.hsc = a.hsc;
    c.hq = a.hq;
  }
  c.zero = zero;
  c.warp = warp;
  c.lane = lane;
  c.g = lane >> 2;
  c.tig = lane & 3;
  c.S = S;
  c.hI = HS ? Ix : I;
  c.hqp = (HS ? Ix : I) / 16;
  c.hsp = HS ? hssx : a.hss;
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
  t.init(dib, dG, slice ? 1 : a.DP, rbs);
  uint32_t nd[kMaxNB][2] = {};
  DnUnit nw{};
  if (t.slot < nact) {
    nw = dn_unit_of(t, ms);
    if (slice) nw.dp = dpc;
    ddload(nw, nd);
  }
  while (t.slot < nact) {
    const DnUnit w = nw;
    uint32_t d[kMaxNB][2];
#pragma unroll
    for (int j = 0; j < kMaxNB; ++j) d[j][0] = nd[j][0], d[j][1] = nd[j][1];
    t.next(slice ? 1 : a.DP, rbs);
    if (t.slot < nact) {
      nw = dn_unit_of(t, ms);
      if (slice) nw.dp = dpc;
      ddload(nw, nd);
    }
    bool ok;
    if (MAXQ == 1 || w.ne == 1) ok = dn_unit_one<HS>(a, c, rp, w, d);
    else ok = dn_unit_multi<(MAXQ > 1 ? MAXQ : 1), HS>(a, c, rp, w, d);
    if (!ok) return;
  }
}

// ---------------------------------------------------------------------------
// The decode GEMVs' operand builders run on their own, for exact checks: per
// IQ2 sub-block record the int8 A bytes (level * sign) of its four groups and
// 2ls + 1; per Q2K sub-block sc * q of its 16 weights (from the uint8 q bytes of
// q2k_quad) and m. Every lane uses its own table replica, as in the GEMV.
__global__ void __launch_bounds__(256) debug_gemv_iq2_kernel(const uint8_t* __restrict__ codes, int64_t nsub,
                                                             int8_t* __restrict__ w, uint8_t* __restrict__ odd,
                                                             uint32_t one) {
  extern __shared__ __align__(1024) uint8_t smem[];
  fill_sel_tables(reinterpret_cast<uint32_t*>(smem), threadIdx.x, blockDim.x);
  __syncthreads();
  const uint32_t lane = threadIdx.x & 31, lane4 = 4u * lane, sgn_lane = 128u + 4u * lane;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nsub;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint2 rec = *reinterpret_cast<const uint2*>(codes + 8 * i);
    uint32_t o[8];
    iq2_group_int8<0>(rec, lane4, sgn_lane, one, o[0], o[1]);
    iq2_group_int8<1>(rec, lane4, sgn_lane, one, o[2], o[3]);
    iq2_group_int8<2>(rec, lane4, sgn_lane, one, o[4], o[5]);
    iq2_group_int8<3>(rec, lane4, sgn_lane, one, o[6], o[7]);
    uint4* dst = reinterpret_cast<uint4*>(w + 32 * i);
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    odd[i] = static_cast<uint8_t>(iq2_odd(rec));
  }
}

__global__ void __launch_bounds__(256) debug_gemv_q2k_kernel(const uint8_t* __restrict__ codes, int64_t nsub,
                                                             int16_t* __restrict__ scq, uint8_t* __restrict__ m) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nsub;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint8_t* blk = codes + (i / 16) * 80;
    const int sb = static_cast<int>(i % 16);
    const uint32_t word = *reinterpret_cast<const uint32_t*>(blk + 16 + 4 * sb);
    const uint32_t scb = blk[sb];
    for (int r = 0; r < 4; ++r) {
      const uint32_t quad = q2k_quad(word, 2u * r);  // weights 4i + r of the sub-block, i = 0..3
      for (int b = 0; b < 4; ++b)
        scq[16 * i + 4 * b + r] = static_cast<int16_t>(static_cast<int>((quad >> (8 * b)) & 0xFFu) * (scb & 15u));
    }
    m[i] = static_cast<uint8_t>(scb >> 4);
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
              uint32_t box_rows, CUtensorMapSwizzle swizzle) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {row_bytes, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_bytes, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

constexpr size_t kBudget = 227 * 1024;

// Fault injection (moe_debug_inject): read at each gate/up launch.
int g_inject_mode = 0;
long long g_inject_limit = 0;

int nb_for(int T) { return T == 1 ? 1 : 2; }

template <typename K>
void launch_k(K kern, int grid, size_t smem, cudaStream_t st, const CUtensorMap& m0, const CUtensorMap& m1,
              const GuTmaArgs& a) {
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  launch_pdl(kern, dim3(grid), dim3(kThreadsT), smem, st, m0, m1, a);
}

template <typename K>
void launch_k(K kern, int grid, size_t smem, cudaStream_t st, const CUtensorMap& m0, const CUtensorMap& m1,
              const DnTmaArgs& a) {
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  launch_pdl(kern, dim3(grid), dim3(kThreadsT), smem, st, m0, m1, a);
}

}  // namespace

int launch_debug_gemv_iq2(const uint8_t* codes, int64_t nblocks, int8_t* w, uint8_t* odd, cudaStream_t st) {
  const int64_t nsub = nblocks * 8;
  const int grid = static_cast<int>(std::min<int64_t>((nsub + 255) / 256, 4096));
  cudaFuncSetAttribute(debug_gemv_iq2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kTabBytes);
  debug_gemv_iq2_kernel<<<grid, 256, kTabBytes, st>>>(codes, nsub, w, odd, 1u);
  return cudaGetLastError() == cudaSuccess ? OK : ERR_CUDA;
}

int launch_debug_gemv_q2k(const uint8_t* codes, int64_t nblocks, int16_t* scq, uint8_t* m, cudaStream_t st) {
  const int64_t nsub = nblocks * 16;
  const int grid = static_cast<int>(std::min<int64_t>((nsub + 255) / 256, 4096));
  debug_gemv_q2k_kernel<<<grid, 256, 0, st>>>(codes, nsub, scq, m);
  return cudaGetLastError() == cudaSuccess ? OK : ERR_CUDA;
}

int read_bounds_violations(unsigned long long* out) {
#ifdef MOE_BOUNDS_CHECK
  const unsigned long long zero = 0;
  if (cudaMemcpyFromSymbol(out, g_bounds_violations, sizeof(*out)) != cudaSuccess ||
      cudaMemcpyToSymbol(g_bounds_violations, &zero, sizeof(zero)) != cudaSuccess)
    return ERR_CUDA;
  return OK;
#else
  *out = 0;
  return ERR_SHAPE;  // not a bounds-checked build
#endif
}

void set_debug_inject(int mode, long long wait_limit) {
  g_inject_mode = mode;
  g_inject_limit = wait_limit;
}

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
  if (!make_map(&tg, gate_codes, rb, rows, kGuW, kBoxRows, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&tu, up_codes, rb, rows, kGuW, kBoxRows, CU_TENSOR_MAP_SWIZZLE_128B))
    return ERR_CUDA;
  GuTmaArgs a{};
  a.H = sh.H; a.I = sh.I; a.E = sh.E; a.k = sh.k; a.T = T;
  a.NB = nb_for(T); a.KP = tma_gu_parts(sh, T);
  a.gate_d = gate_d; a.up_d = up_d; a.xd = xd; a.xs = xs;
  a.offsets = r.offsets; a.perm = r.perm; a.active = r.active; a.gpart = gpart; a.err = err;
  a.gpart_n = static_cast<size_t>(T) * sh.k * 2 * a.KP * sh.I;
  a.no_produce = g_inject_mode == 1;
  a.one = 1;
  a.wait_limit = g_inject_mode ? g_inject_limit : kDefaultWaitCycles;
  // stage the activations when that still leaves three ring stages
  const size_t budget = kBudget;
  const int Hx = T == 1 ? sh.H : a.NB * 512;  // staged activation columns per CTA (see the kernel)
  const bool xs_in = gu_plan(sh.E, T, sh.k, Hx, true, 3).total <= budget;
  int S = 2;
  while (S < 6 && gu_plan(sh.E, T, sh.k, Hx, xs_in, S + 1).total <= budget) ++S;
  if (!xs_in || gu_plan(sh.E, T, sh.k, Hx, xs_in, S).total > budget) return ERR_SHAPE;
  a.S = S;
  const size_t smem = gu_plan(sh.E, T, sh.k, Hx, xs_in, S).total;
  const size_t nA = static_cast<size_t>(T) * sh.k;
  const int slots = static_cast<int>(std::min<size_t>(nA, static_cast<size_t>(sh.E)));
  const int units = slots * 2 * (sh.I / kBoxRows) * a.KP;
  const int grid = std::max(1, std::min(units, sms));
  if (T == 1)  // one token: the single-assignment variant with staged activations
    launch_k(gateup_tma_kernel<1, true>, grid, smem, st, tg, tu, a);
  else  // at most 16 tokens per expert: four groups of four, each CTA on one part of H
    launch_k(gateup_tma_kernel<4, true>, grid, smem, st, tg, tu, a);
  return cudaGetLastError() == cudaSuccess ? OK : ERR_CUDA;
}

int launch_down_tma(const LayerShape& sh, const uint8_t* down_codes, const uint32_t* down_dd, const int8_t* hd,
                    const float* hsc, const int32_t* hq, int hss, int T, const Routing& r, float* opart, int* err,
                    int sms, cudaStream_t st) {
  CUtensorMap tq, ts;
  const uint64_t rb = static_cast<uint64_t>(sh.I / 256) * 80, rows = static_cast<uint64_t>(sh.E) * sh.H;
  if (!make_map(&tq, down_codes, rb, rows, 64, kBoxRows, CU_TENSOR_MAP_SWIZZLE_64B) ||
      !make_map(&ts, down_codes, rb, rows, 16, kBoxRows, CU_TENSOR_MAP_SWIZZLE_NONE))
    return ERR_CUDA;
  DnTmaArgs a{};
  a.H = sh.H; a.I = sh.I; a.E = sh.E; a.k = sh.k; a.T = T; a.hss = hss;
  a.NB = nb_for(T); a.DP = tma_dn_parts(sh, T);
  a.dd = down_dd; a.hd = hd; a.hsc = hsc; a.hq = hq;
  a.offsets = r.offsets; a.active = r.active; a.opart = opart; a.err = err;
  const int nA = T * sh.k;
  a.opart_n = static_cast<size_t>(nA) * a.DP * sh.H;
  // staged h per assignment: all of I for one token, a slice of NB*256 columns for more (see the kernel)
  const int Ix = T == 1 ? sh.I : a.NB * 256, hssx = T == 1 ? hss : a.NB;
  const bool hs_in = dn_plan(sh.E, nA, Ix, hssx, true, 3).total <= kBudget;
  int S = 2;
  while (S < 8 && dn_plan(sh.E, nA, Ix, hssx, hs_in, S + 1).total <= kBudget) ++S;
  if (dn_plan(sh.E, nA, Ix, hssx, hs_in, S).total > kBudget) return ERR_SHAPE;
  a.S = S;
  const size_t smem = dn_plan(sh.E, nA, Ix, hssx, hs_in, S).total;
  const int slots = std::min(nA, sh.E);
  const int units = slots * (sh.H / kBoxRows) * a.DP;
  const int grid = std::max(1, std::min(units, sms));
  if (T == 1) {  // one token: the single-assignment variant with h staged
    if (!hs_in) return ERR_SHAPE;
    launch_k(down_tma_kernel<1, true>, grid, smem, st, tq, ts, a);
  } else if (hs_in) {  // at most 16 tokens per expert: eight groups of two
    launch_k(down_tma_kernel<8, true>, grid, smem, st, tq, ts, a);
  } else {
    launch_k(down_tma_kernel<8, false>, grid, smem, st, tq, ts, a);
  }
  return cudaGetLastError() == cudaSuccess ? OK : ERR_CUDA;
}

}  // namespace moe
