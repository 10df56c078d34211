// gemv_tma.cu - decode dequant-GEMVs of the routed experts fed by 2-D TMA
// tensor-map loads, with warp specialisation: one producer warp streams boxes
// of code rows into a ring of shared-memory stages (full/empty mbarriers, all
// waits bounded), eight consumer warps each own 16 rows and turn the codes into
// int8 MMA operands. No block-wide barrier inside the main loop.
//
// Sources: "ds4 : analyse pratique pour un usage documenté", section « Support
// de modèles et choix de quantification » (up/gate IQ2_XXS, down Q2_K). The
// operand construction and the integer accumulation are those of decode.cuh.
//
// Work is split into units small enough to balance over all SMs: a gate/up
// unit is (expert, gate or up, 128 rows, 1024-wide part of H) and a down unit
// is (expert, 128 rows of H, 512-wide part of I). Each unit writes partial
// sums that the next kernel adds up in a fixed order.
//
// gate/up boxes: 128 rows x 128 code bytes (16 sub-blocks), 128-byte swizzle,
//   so the eight rows a warp reads together land in eight different 16-byte
//   bank groups. down boxes: 128 rows x 160 code bytes (two blocks), dense; the
//   160-byte pitch makes the eight-row reads two-way conflicted at most.
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

constexpr int kCW = 8;                       // consumer warps (16 rows each)
constexpr int kThreadsT = (kCW + 1) * 32;    // + one producer warp
constexpr int kBoxRows = 16 * kCW;           // 128 rows per box
constexpr int kGuBox = kBoxRows * 128;       // bytes per gate/up box
constexpr int kDnBox = kBoxRows * 160;       // bytes per down box
constexpr uint32_t kLvlOff = 0;              // replicated level table (32 KB)
constexpr uint32_t kSgnOff = 32768;          // replicated sign table (16 KB)
constexpr uint32_t kXOff = 49152;            // activation digits when staged

__device__ __forceinline__ uint32_t rotr(uint32_t v, uint32_t n) { return __funnelshift_r(v, v, n); }

struct GuTmaArgs {
  int H, I, E, k, T, KP, S, x_in_smem;
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

struct GuCtx {
  const uint8_t* ring;
  uint64_t* full;
  uint64_t* empty;
  const int8_t* xdig;
  const float* xscl;
  int warp, lane, g, tig, S;
  uint32_t lane4, rot_idx, rot_sig;
};

// One unit (two boxes) for TPG tokens per MMA column group, up to MAXQ groups.
// Returns false on a timed-out wait.
template <int TPG, int MAXQ>
__device__ __forceinline__ bool gu_unit(const GuTmaArgs& a, const uint8_t* smem, const GuCtx& c, int& it, int e,
                                        int m, int rb, int kp, int p0, int ne) {
  constexpr int SPS = 4 / TPG;
  const int H = a.H, I = a.I;
  const int ngroups = (ne + TPG - 1) / TPG;
  const int g = c.g, tig = c.tig;
  const int tslot_b = (g >> 1) % TPG, sslot_b = (g >> 1) / TPG, dig_b = g & 1;
  const int tslot_c = tig % TPG, sslot_c = tig / TPG;
  const int row_l = 16 * c.warp + g;  // row within the box (and +8)
  const size_t row_g = static_cast<size_t>(e) * I + rb * kBoxRows + row_l;
  // d of the part's four super-blocks for rows g and g+8
  const uint16_t* dpl = m ? a.up_d : a.gate_d;
  const uint2 dq0 = *reinterpret_cast<const uint2*>(dpl + row_g * (H / 256) + kp * 4);
  const uint2 dq1 = *reinterpret_cast<const uint2*>(dpl + (row_g + 8) * (H / 256) + kp * 4);
  const int8_t* xb[MAXQ];
  bool bval[MAXQ];
  const float* xsc[MAXQ];
#pragma unroll
  for (int q = 0; q < MAXQ; ++q) {
    const int tb = q * TPG + tslot_b, tc = q * TPG + tslot_c;
    bval[q] = q < ngroups && tb < ne;
    const int tok = bval[q] ? a.perm[p0 + tb] / a.k : 0;
    xb[q] = c.xdig + (static_cast<size_t>(tok) * 2 + dig_b) * H + 8 * tig + (kp * 32 + sslot_b) * 32;
    xsc[q] = (q < ngroups && tc < ne) ? c.xscl + static_cast<size_t>(a.perm[p0 + tc] / a.k) * (H / 256) + kp * 4
                                      : nullptr;
  }
  int acc[MAXQ][2][4];
  int iacc[MAXQ][2];
  float facc[MAXQ][2];
#pragma unroll
  for (int q = 0; q < MAXQ; ++q) {
#pragma unroll
    for (int h = 0; h < 2; ++h) acc[q][h][0] = acc[q][h][1] = acc[q][h][2] = acc[q][h][3] = 0;
    iacc[q][0] = iacc[q][1] = 0;
    facc[q][0] = facc[q][1] = 0.f;
  }
#pragma unroll 1
  for (int j = 0; j < 2; ++j, ++it) {
    const int s = it % c.S;
    if (!mbar_wait_bounded(&c.full[s], (it / c.S) & 1u, a.err, ERR_TIMEOUT)) return false;
    const uint8_t* st = c.ring + s * kGuBox;
    const uint8_t* rg = st + row_l * 128;
    const uint8_t* rg8 = rg + 8 * 128;
#pragma unroll 1
    for (int cc = 0; cc < 4; ++cc) {
      uint2 rec[4][2];
      {
        const uint4 a0 = *reinterpret_cast<const uint4*>(rg + (((2 * cc) ^ g) << 4));
        const uint4 a1 = *reinterpret_cast<const uint4*>(rg + (((2 * cc + 1) ^ g) << 4));
        const uint4 b0 = *reinterpret_cast<const uint4*>(rg8 + (((2 * cc) ^ g) << 4));
        const uint4 b1 = *reinterpret_cast<const uint4*>(rg8 + (((2 * cc + 1) ^ g) << 4));
        rec[0][0] = make_uint2(a0.x, a0.y); rec[1][0] = make_uint2(a0.z, a0.w);
        rec[2][0] = make_uint2(a1.x, a1.y); rec[3][0] = make_uint2(a1.z, a1.w);
        rec[0][1] = make_uint2(b0.x, b0.y); rec[1][1] = make_uint2(b0.z, b0.w);
        rec[2][1] = make_uint2(b1.x, b1.y); rec[3][1] = make_uint2(b1.z, b1.w);
      }
      uint32_t af[4][2][2];
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const uint32_t al = (rotr(rec[u][r].x, c.rot_idx) & 0x7F80u) | c.lane4;
          const uint32_t as = (rotr(rec[u][r].y, c.rot_sig) & 0x3F80u) | c.lane4;
          const uint32_t sel = *reinterpret_cast<const uint32_t*>(smem + kLvlOff + al) |
                               *reinterpret_cast<const uint32_t*>(smem + kSgnOff + as);
          af[u][r][0] = prmt(kPosBytes, kNegBytes, sel);
          af[u][r][1] = prmt(kPosBytes, kNegBytes, sel >> 16);
        }
      const int sbo = j * 16 + 4 * cc;  // sub-block offset inside the part
#pragma unroll
      for (int q = 0; q < MAXQ; ++q) {
        if (q >= ngroups) break;
        uint2 bl[TPG];
#pragma unroll
        for (int jj = 0; jj < TPG; ++jj)
          bl[jj] = bval[q] ? *reinterpret_cast<const uint2*>(xb[q] + (sbo + jj * SPS) * 32) : make_uint2(0u, 0u);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int jj = u / SPS, slot = u % SPS;
          const bool on = slot == sslot_b;
          mma_s8s8(acc[q][u & 1], af[u][0][0], af[u][1][0], af[u][0][1], af[u][1][1], on ? bl[jj].x : 0u,
                   on ? bl[jj].y : 0u);
          if (slot == SPS - 1) {
            uint32_t v0 = rec[jj * SPS][0].y, v1 = rec[jj * SPS][1].y;
#pragma unroll
            for (int w = 1; w < SPS; ++w)
              if (sslot_c == w) { v0 = rec[jj * SPS + w][0].y; v1 = rec[jj * SPS + w][1].y; }
            const int odd0 = static_cast<int>((v0 >> 27) | 1u), odd1 = static_cast<int>((v1 >> 27) | 1u);
            iacc[q][0] += ((acc[q][0][0] + acc[q][1][0]) * 128 + acc[q][0][1] + acc[q][1][1]) * odd0;
            iacc[q][1] += ((acc[q][0][2] + acc[q][1][2]) * 128 + acc[q][0][3] + acc[q][1][3]) * odd1;
#pragma unroll
            for (int h = 0; h < 2; ++h) acc[q][h][0] = acc[q][h][1] = acc[q][h][2] = acc[q][h][3] = 0;
          }
        }
      }
      if (cc & 1) {
        // super-block done: d (per row) and 2^s/8 (per token)
        const int sbl = j * 2 + (cc >> 1);
        const uint32_t w0 = sbl < 2 ? dq0.x : dq0.y, w1 = sbl < 2 ? dq1.x : dq1.y;
        const float d0 = half_bits_to_float(static_cast<uint16_t>((sbl & 1) ? (w0 >> 16) : (w0 & 0xFFFFu)));
        const float d1 = half_bits_to_float(static_cast<uint16_t>((sbl & 1) ? (w1 >> 16) : (w1 & 0xFFFFu)));
#pragma unroll
        for (int q = 0; q < MAXQ; ++q) {
          const float xsv = xsc[q] ? xsc[q][sbl] : 0.f;
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
      if (TPG == 1) {
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
      } else if (TPG == 2) {
        v += __shfl_xor_sync(0xffffffffu, v, 2);
      }
      facc[q][r] = v;
    }
  const bool owner = (TPG == 4) || (tig < TPG);
#pragma unroll
  for (int q = 0; q < MAXQ; ++q) {
    const int tok = q * TPG + tslot_c;
    if (q < ngroups && owner && tok < ne) {
      float* out = a.gpart + ((static_cast<size_t>(p0 + tok) * 2 + m) * a.KP + kp) * I + rb * kBoxRows + row_l;
      out[0] = facc[q][0];
      out[8] = facc[q][1];
    }
  }
  return true;
}

template <int MAXQ>
__global__ void __launch_bounds__(kThreadsT, 1) gateup_tma_kernel(const __grid_constant__ CUtensorMap tm_gate,
                                                                  const __grid_constant__ CUtensorMap tm_up,
                                                                  GuTmaArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = a.H, I = a.I, T = a.T, S = a.S;
  const size_t xb_bytes = a.x_in_smem ? align_up(static_cast<size_t>(T) * 2 * H, 128) : 0;
  const size_t xs_bytes = a.x_in_smem ? align_up(static_cast<size_t>(T) * (H / 256) * 4, 128) : 0;
  int8_t* xsm = reinterpret_cast<int8_t*>(smem + kXOff);
  float* xssm = reinterpret_cast<float*>(smem + kXOff + xb_bytes);
  uint8_t* ring = smem + align_up(kXOff + xb_bytes + xs_bytes, 1024);
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + static_cast<size_t>(S) * kGuBox);
  uint64_t* empty = full + S;
  const int rbs = I / kBoxRows;
  const int nunits = a.active[a.E] * 2 * rbs * a.KP;

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
  for (int i = tid; i < 256 * 32; i += kThreadsT)
    reinterpret_cast<uint32_t*>(smem + kLvlOff)[i] = d_sel_tables2.level[i >> 5];
  for (int i = tid; i < 128 * 32; i += kThreadsT)
    reinterpret_cast<uint32_t*>(smem + kSgnOff)[i] = d_sel_tables2.sign[i >> 5];
  if (a.x_in_smem) {
    const int nx = T * 2 * H / 16;
    for (int i = tid; i < nx; i += kThreadsT) reinterpret_cast<uint4*>(xsm)[i] = reinterpret_cast<const uint4*>(a.xd)[i];
    for (int i = tid; i < T * (H / 256); i += kThreadsT) xssm[i] = a.xs[i];
  }
  __syncthreads();

  if (warp == kCW) {  // producer
    if (lane == 0) {
      prefetch_tmap(&tm_gate);
      prefetch_tmap(&tm_up);
      int it = 0;
      for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
        const int kp = u % a.KP;
        const int rest = u / a.KP;
        const int rb = rest % rbs, m = (rest / rbs) & 1, slot = rest / rbs / 2;
        const int e = a.active[slot];
        for (int j = 0; j < 2; ++j, ++it) {
          const int s = it % S;
          if (!mbar_wait_bounded(&empty[s], ((it / S) & 1u) ^ 1u, a.err, ERR_TIMEOUT)) return;
          mbar_arrive_expect_tx(&full[s], kGuBox);
          tma_load_2d(ring + static_cast<size_t>(s) * kGuBox, m ? &tm_up : &tm_gate, kp * 256 + j * 128,
                      e * I + rb * kBoxRows, &full[s]);
        }
      }
    }
    return;
  }

  GuCtx c;
  c.ring = ring;
  c.full = full;
  c.empty = empty;
  c.xdig = a.x_in_smem ? xsm : a.xd;
  c.xscl = a.x_in_smem ? xssm : a.xs;
  c.warp = warp;
  c.lane = lane;
  c.g = lane >> 2;
  c.tig = lane & 3;
  c.S = S;
  c.lane4 = static_cast<uint32_t>(lane) << 2;
  c.rot_idx = (8u * c.tig - 7u) & 31u;
  c.rot_sig = (7u * c.tig - 7u) & 31u;
  int it = 0;
  for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
    const int kp = u % a.KP;
    const int rest = u / a.KP;
    const int rb = rest % rbs, m = (rest / rbs) & 1, slot = rest / rbs / 2;
    const int e = a.active[slot];
    const int p0 = a.offsets[e], ne = a.offsets[e + 1] - p0;
    bool ok;
    if (MAXQ == 1 || ne == 1) ok = gu_unit<1, 1>(a, smem, c, it, e, m, rb, kp, p0, ne);
    else if (ne == 2) ok = gu_unit<2, 1>(a, smem, c, it, e, m, rb, kp, p0, ne);
    else ok = gu_unit<4, (MAXQ > 1 ? MAXQ : 1)>(a, smem, c, it, e, m, rb, kp, p0, ne);
    if (!ok) return;
  }
}

// ---------------------------------------------------------------------------
struct DnTmaArgs {
  int H, I, E, k, T, DP, S, h_in_smem;
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

template <int TPG, int MAXQ>
__device__ __forceinline__ bool dn_unit(const DnTmaArgs& a, const uint8_t* ring, uint64_t* full, uint64_t* empty,
                                        const int8_t* hd, const float* hsc, const int32_t* hq, int warp, int lane,
                                        int& it, int e, int rb, int dp, int p0, int ne) {
  constexpr int SPP = TPG == 1 ? 2 : 1;  // sub-block pairs per column set
  const int H = a.H, I = a.I, S = a.S;
  const int g = lane >> 2, tig = lane & 3;
  const int ngroups = (ne + TPG - 1) / TPG;
  const int dig_b = g & 1, hb = (g >> 1) & 1, sl_b = g >> 2;
  const int hc = tig & 1, sl_c = tig >> 1;
  const uint32_t sh = 2 * tig;
  const int row_l = 16 * warp + g;
  const size_t row_g = static_cast<size_t>(e) * H + rb * kBoxRows + row_l;
  const int nblk = I / 256;
  const uint2 ddA = *reinterpret_cast<const uint2*>(a.dd + row_g * nblk + dp * 2);
  const uint2 ddB = *reinterpret_cast<const uint2*>(a.dd + (row_g + 8) * nblk + dp * 2);
  const int8_t* hb_ptr[MAXQ];
  bool hb_on[MAXQ];
  const float* sc_ptr[MAXQ];
  const int32_t* hq_ptr[MAXQ];
#pragma unroll
  for (int q = 0; q < MAXQ; ++q) {
    const int tb = q * TPG + (TPG == 1 ? 0 : sl_b);
    const int tc = q * TPG + (TPG == 1 ? 0 : sl_c);
    hb_on[q] = q < ngroups && tb < ne;
    hb_ptr[q] = hd + (static_cast<size_t>(p0 + (hb_on[q] ? tb : 0)) * 2 + dig_b) * I + 8 * tig + dp * 512;
    const bool cv = q < ngroups && tc < ne;
    sc_ptr[q] = cv ? hsc + static_cast<size_t>(p0 + tc) * a.hss + dp * 2 : nullptr;
    hq_ptr[q] = cv ? hq + static_cast<size_t>(p0 + tc) * (I / 16) + dp * 32 : nullptr;
  }
  int acc[MAXQ][4];
  int iA[MAXQ][2], iM[MAXQ][2];
  float facc[MAXQ][2];
#pragma unroll
  for (int q = 0; q < MAXQ; ++q) {
    acc[q][0] = acc[q][1] = acc[q][2] = acc[q][3] = 0;
    iA[q][0] = iA[q][1] = iM[q][0] = iM[q][1] = 0;
    facc[q][0] = facc[q][1] = 0.f;
  }
  const int s = it % S;
  if (!mbar_wait_bounded(&full[s], (it / S) & 1u, a.err, ERR_TIMEOUT)) return false;
  const uint8_t* rA = ring + static_cast<size_t>(s) * kDnBox + row_l * 160;
  const uint8_t* rB = rA + 8 * 160;
#pragma unroll 1
  for (int cc = 0; cc < 4; ++cc) {  // chunks of four sub-block pairs; 16 pairs = two blocks
    uint32_t af[4][4];
#pragma unroll
    for (int u2 = 0; u2 < 2; ++u2) {
      const int pr = 4 * cc + 2 * u2;
      const int off = (pr >> 3) * 80 + 16 + 8 * (pr & 7);
      const uint4 qa = *reinterpret_cast<const uint4*>(rA + off);
      const uint4 qb = *reinterpret_cast<const uint4*>(rB + off);
      af[2 * u2][0] = (qa.x >> sh) & 0x03030303u;
      af[2 * u2][1] = (qb.x >> sh) & 0x03030303u;
      af[2 * u2][2] = (qa.y >> sh) & 0x03030303u;
      af[2 * u2][3] = (qb.y >> sh) & 0x03030303u;
      af[2 * u2 + 1][0] = (qa.z >> sh) & 0x03030303u;
      af[2 * u2 + 1][1] = (qb.z >> sh) & 0x03030303u;
      af[2 * u2 + 1][2] = (qa.w >> sh) & 0x03030303u;
      af[2 * u2 + 1][3] = (qb.w >> sh) & 0x03030303u;
    }
#pragma unroll
    for (int q = 0; q < MAXQ; ++q) {
      if (q >= ngroups) break;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int pr = 4 * cc + u, slot = u % SPP;
        uint2 bv = make_uint2(0u, 0u);
        if (hb_on[q] && (SPP == 1 || slot == sl_b)) {
          bv = *reinterpret_cast<const uint2*>(hb_ptr[q] + pr * 32);
          if (hb) bv.x = 0u; else bv.y = 0u;
        }
        mma_u8s8(acc[q], af[u][0], af[u][1], af[u][2], af[u][3], bv.x, bv.y);
        if (slot == SPP - 1) {
          const int sub = 2 * (pr - (SPP - 1) + (TPG == 1 ? sl_c : 0)) + hc;  // sub-block inside the two blocks
          const int bb = sub >> 4, si = sub & 15;
          const uint32_t scA = rA[bb * 80 + si], scB = rB[bb * 80 + si];
          if (hq_ptr[q]) {
            const int hqv = hq_ptr[q][sub];
            iA[q][0] += (acc[q][0] * 128 + acc[q][1]) * static_cast<int>(scA & 15u);
            iA[q][1] += (acc[q][2] * 128 + acc[q][3]) * static_cast<int>(scB & 15u);
            iM[q][0] += static_cast<int>(scA >> 4) * hqv;
            iM[q][1] += static_cast<int>(scB >> 4) * hqv;
          }
          acc[q][0] = acc[q][1] = acc[q][2] = acc[q][3] = 0;
        }
      }
    }
    if (cc & 1) {
      // block (super-block) done: 2^e * (d * A - dmin * M)
      const int bl = cc >> 1;
      const uint32_t wA = bl ? ddA.y : ddA.x, wB = bl ? ddB.y : ddB.x;
      const float dA = half_bits_to_float(static_cast<uint16_t>(wA & 0xFFFFu));
      const float nA = half_bits_to_float(static_cast<uint16_t>(wA >> 16));
      const float dB = half_bits_to_float(static_cast<uint16_t>(wB & 0xFFFFu));
      const float nB = half_bits_to_float(static_cast<uint16_t>(wB >> 16));
#pragma unroll
      for (int q = 0; q < MAXQ; ++q) {
        const float e2 = sc_ptr[q] ? sc_ptr[q][bl] : 0.f;
        facc[q][0] = fmaf(e2, fmaf(dA, static_cast<float>(iA[q][0]), -nA * static_cast<float>(iM[q][0])), facc[q][0]);
        facc[q][1] = fmaf(e2, fmaf(dB, static_cast<float>(iA[q][1]), -nB * static_cast<float>(iM[q][1])), facc[q][1]);
        iA[q][0] = iA[q][1] = iM[q][0] = iM[q][1] = 0;
      }
    }
  }
  __syncwarp();
  if (lane == 0) mbar_arrive(&empty[s]);
  ++it;
#pragma unroll
  for (int q = 0; q < MAXQ; ++q)
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      float v = facc[q][r];
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      if (TPG == 1) v += __shfl_xor_sync(0xffffffffu, v, 2);
      facc[q][r] = v;
    }
  const bool owner = TPG == 1 ? (tig == 0) : (hc == 0);
#pragma unroll
  for (int q = 0; q < MAXQ; ++q) {
    const int tok = q * TPG + (TPG == 1 ? 0 : sl_c);
    if (q < ngroups && owner && tok < ne) {
      float* out = a.opart + (static_cast<size_t>(p0 + tok) * a.DP + dp) * H + rb * kBoxRows + row_l;
      out[0] = facc[q][0];
      out[8] = facc[q][1];
    }
  }
  return true;
}

template <int MAXQ>
__global__ void __launch_bounds__(kThreadsT, 1) down_tma_kernel(const __grid_constant__ CUtensorMap tm_down,
                                                                DnTmaArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = a.H, I = a.I, S = a.S;
  const int nA = a.T * a.k;
  const size_t hd_bytes = a.h_in_smem ? align_up(static_cast<size_t>(nA) * 2 * I, 128) : 0;
  const size_t hsc_bytes = a.h_in_smem ? align_up(static_cast<size_t>(nA) * a.hss * 4, 128) : 0;
  const size_t hq_bytes = a.h_in_smem ? align_up(static_cast<size_t>(nA) * (I / 16) * 4, 128) : 0;
  int8_t* hd_s = reinterpret_cast<int8_t*>(smem);
  float* hsc_s = reinterpret_cast<float*>(smem + hd_bytes);
  int32_t* hq_s = reinterpret_cast<int32_t*>(smem + hd_bytes + hsc_bytes);
  uint8_t* ring = smem + align_up(hd_bytes + hsc_bytes + hq_bytes, 1024);
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + static_cast<size_t>(S) * kDnBox);
  uint64_t* empty = full + S;
  const int rbs = H / kBoxRows;
  const int nunits = a.active[a.E] * rbs * a.DP;

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kCW);
    }
    fence_barrier_init();
  }
  if (a.h_in_smem) {
    for (int i = tid; i < nA * 2 * I / 16; i += kThreadsT)
      reinterpret_cast<uint4*>(hd_s)[i] = reinterpret_cast<const uint4*>(a.hd)[i];
    for (int i = tid; i < nA * a.hss; i += kThreadsT) hsc_s[i] = a.hsc[i];
    for (int i = tid; i < nA * (I / 16); i += kThreadsT) hq_s[i] = a.hq[i];
  }
  __syncthreads();

  if (warp == kCW) {  // producer
    if (lane == 0) {
      prefetch_tmap(&tm_down);
      int it = 0;
      for (int u = blockIdx.x; u < nunits; u += gridDim.x, ++it) {
        const int dp = u % a.DP;
        const int rest = u / a.DP;
        const int rb = rest % rbs, slot = rest / rbs;
        const int e = a.active[slot];
        const int s = it % S;
        if (!mbar_wait_bounded(&empty[s], ((it / S) & 1u) ^ 1u, a.err, ERR_TIMEOUT)) return;
        mbar_arrive_expect_tx(&full[s], kDnBox);
        tma_load_2d(ring + static_cast<size_t>(s) * kDnBox, &tm_down, dp * 160, e * H + rb * kBoxRows, &full[s]);
      }
    }
    return;
  }
  const int8_t* hd = a.h_in_smem ? hd_s : a.hd;
  const float* hsc = a.h_in_smem ? hsc_s : a.hsc;
  const int32_t* hq = a.h_in_smem ? hq_s : a.hq;
  int it = 0;
  for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
    const int dp = u % a.DP;
    const int rest = u / a.DP;
    const int rb = rest % rbs, slot = rest / rbs;
    const int e = a.active[slot];
    const int p0 = a.offsets[e], ne = a.offsets[e + 1] - p0;
    bool ok;
    if (MAXQ == 1 || ne == 1) ok = dn_unit<1, 1>(a, ring, full, empty, hd, hsc, hq, warp, lane, it, e, rb, dp, p0, ne);
    else ok = dn_unit<2, (MAXQ > 1 ? MAXQ : 1)>(a, ring, full, empty, hd, hsc, hq, warp, lane, it, e, rb, dp, p0, ne);
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

}  // namespace

bool tma_path_supported(const LayerShape& s, int T) {
  return s.H % 1024 == 0 && s.I % 512 == 0 && T <= 16 && encode_fn() != nullptr;
}
// A gate/up unit covers 1024 of H and a down unit 512 of I, so the reduction
// axis is always split into this many parts.
int tma_gu_parts(const LayerShape& s, int) { return s.H / 1024; }
int tma_dn_parts(const LayerShape& s, int) { return s.I / 512; }

int launch_gateup_tma(const LayerShape& sh, const uint8_t* gate_codes, const uint16_t* gate_d,
                      const uint8_t* up_codes, const uint16_t* up_d, const int8_t* xd, const float* xs, int T,
                      const Routing& r, float* gpart, int* err, int sms, cudaStream_t st) {
  CUtensorMap tg, tu;
  const uint64_t rb = sh.H / 4, rows = static_cast<uint64_t>(sh.E) * sh.I;
  if (!make_map(&tg, gate_codes, rb, rows, 128, kBoxRows, true) || !make_map(&tu, up_codes, rb, rows, 128, kBoxRows, true))
    return ERR_CUDA;
  GuTmaArgs a{};
  a.H = sh.H; a.I = sh.I; a.E = sh.E; a.k = sh.k; a.T = T; a.KP = tma_gu_parts(sh, T);
  a.gate_d = gate_d; a.up_d = up_d; a.xd = xd; a.xs = xs;
  a.offsets = r.offsets; a.perm = r.perm; a.active = r.active; a.gpart = gpart; a.err = err;
  const size_t xbytes = align_up(static_cast<size_t>(T) * 2 * sh.H, 128) + align_up(static_cast<size_t>(T) * (sh.H / 256) * 4, 128);
  a.x_in_smem = (kXOff + xbytes + 4 * kGuBox + 1024 <= kBudget) ? 1 : 0;
  const size_t ring_off = align_up(kXOff + (a.x_in_smem ? xbytes : 0), 1024);
  int S = static_cast<int>((kBudget - ring_off - 256) / kGuBox);
  S = std::max(2, std::min(S, 10));
  a.S = S;
  const size_t smem = ring_off + static_cast<size_t>(S) * kGuBox + 2 * S * 8;
  const int slots = static_cast<int>(std::min<size_t>(static_cast<size_t>(T) * sh.k, static_cast<size_t>(sh.E)));
  const int units = slots * 2 * (sh.I / kBoxRows) * a.KP;
  const int grid = std::max(1, std::min(units, sms));
  if (T == 1) {
    cudaFuncSetAttribute(gateup_tma_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    gateup_tma_kernel<1><<<grid, kThreadsT, smem, st>>>(tg, tu, a);
  } else {  // at most 16 tokens per expert: four groups of four
    cudaFuncSetAttribute(gateup_tma_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    gateup_tma_kernel<4><<<grid, kThreadsT, smem, st>>>(tg, tu, a);
  }
  return cudaGetLastError() == cudaSuccess ? OK : ERR_CUDA;
}

int launch_down_tma(const LayerShape& sh, const uint8_t* down_codes, const uint32_t* down_dd, const int8_t* hd,
                    const float* hsc, const int32_t* hq, int hss, int T, const Routing& r, float* opart, int* err,
                    int sms, cudaStream_t st) {
  CUtensorMap td;
  const uint64_t rb = static_cast<uint64_t>(sh.I / 256) * 80, rows = static_cast<uint64_t>(sh.E) * sh.H;
  if (!make_map(&td, down_codes, rb, rows, 160, kBoxRows, false)) return ERR_CUDA;
  DnTmaArgs a{};
  a.H = sh.H; a.I = sh.I; a.E = sh.E; a.k = sh.k; a.T = T; a.DP = tma_dn_parts(sh, T); a.hss = hss;
  a.dd = down_dd; a.hd = hd; a.hsc = hsc; a.hq = hq;
  a.offsets = r.offsets; a.active = r.active; a.opart = opart; a.err = err;
  const size_t nA = static_cast<size_t>(T) * sh.k;
  const size_t hbytes = align_up(nA * 2 * sh.I, 128) + align_up(nA * hss * 4, 128) + align_up(nA * (sh.I / 16) * 4, 128);
  a.h_in_smem = (hbytes + 4 * kDnBox + 1024 <= kBudget) ? 1 : 0;
  const size_t ring_off = align_up(a.h_in_smem ? hbytes : 0, 1024);
  int S = static_cast<int>((kBudget - ring_off - 256) / kDnBox);
  S = std::max(2, std::min(S, 8));
  a.S = S;
  const size_t smem = ring_off + static_cast<size_t>(S) * kDnBox + 2 * S * 8;
  const int slots = static_cast<int>(std::min<size_t>(nA, static_cast<size_t>(sh.E)));
  const int units = slots * (sh.H / kBoxRows) * a.DP;
  const int grid = std::max(1, std::min(units, sms));
  if (T == 1) {
    cudaFuncSetAttribute(down_tma_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    down_tma_kernel<1><<<grid, kThreadsT, smem, st>>>(td, a);
  } else {
    // at most 16 tokens per expert: eight groups of two
    cudaFuncSetAttribute(down_tma_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    down_tma_kernel<8><<<grid, kThreadsT, smem, st>>>(td, a);
  }
  return cudaGetLastError() == cudaSuccess ? OK : ERR_CUDA;
}

}  // namespace moe
