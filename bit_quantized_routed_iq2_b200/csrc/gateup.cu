// gateup.cu - gate/up dequant-GEMV of the routed experts (IQ2-style codes) on
// int8 warp MMAs (m16n8k32).
//
// Source of the format split: "ds4 : analyse pratique pour un usage documenté",
// section « Support de modèles et choix de quantification » (up/gate in
// IQ2_XXS). The activation/weight layout is the library's specification.
//
// Tile = (active expert, gate or up, 16 rows of I), all tokens of the expert.
// A persistent grid walks the tiles; one warp issues bulk copies of the tile's
// 16 code rows (one copy per row, rows padded by 16 bytes so the eight rows a
// warp reads together fall in distinct banks) and its d plane into a ring of
// stages guarded by mbarriers. The 8 warps split the reduction axis (H/256
// sub-blocks each) and walk it four sub-blocks at a time. The selector tables
// sit at fixed offsets of shared memory, replicated 32x (one copy per lane) so
// the random codebook lookups never conflict on a bank; a table address is one
// funnel rotate of the code word plus one LOP3.
// Output: g and u per (assignment, row) in fp32; SwiGLU follows in hquant.
#include <algorithm>

#include "decode.cuh"
#include "profile.cuh"
#include "ptx.cuh"

namespace moe {
namespace {

__device__ const Iq2SelTables d_sel_tables = make_sel_tables();

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr uint32_t kLvlOff = 0;      // 256 entries x 32 lanes x 4 bytes
constexpr uint32_t kSgnOff = 32768;  // 128 entries x 32 lanes x 4 bytes
constexpr uint32_t kXOff = 49152;    // activation digits when staged

size_t stage_bytes(int H) {
  return static_cast<size_t>(16) * (H / 4 + 16) + align_up(static_cast<size_t>(16) * (H / 128), 16);
}
size_t x_bytes(int T, int H) {
  return align_up(static_cast<size_t>(T) * 2 * H, 128) + align_up(static_cast<size_t>(T) * (H / 256) * 4, 128);
}
size_t red_bytes(int maxq) { return static_cast<size_t>(kWarps) * 16 * (4 * maxq) * 4; }

__device__ __forceinline__ uint32_t rotr(uint32_t v, uint32_t n) { return __funnelshift_r(v, v, n); }

template <int MAXQ>
__global__ void __launch_bounds__(kThreads, 1) gateup_kernel(GateupArgs a) {
  constexpr int TOKMAX = 4 * MAXQ;  // tokens per pass
  extern __shared__ __align__(1024) uint8_t smem[];
  const int H = a.H, I = a.I, S = a.stages, T = a.T;
  const int row_bytes = H / 4, rs = H / 4 + 16, dbytes = H / 128;
  const size_t sbytes = static_cast<size_t>(16) * rs + align_up(static_cast<size_t>(16) * dbytes, 16);
  const size_t xb_bytes = a.x_in_smem ? align_up(static_cast<size_t>(T) * 2 * H, 128) : 0;
  const size_t xs_bytes = a.x_in_smem ? align_up(static_cast<size_t>(T) * (H / 256) * 4, 128) : 0;
  int8_t* xsm = reinterpret_cast<int8_t*>(smem + kXOff);
  float* xssm = reinterpret_cast<float*>(smem + kXOff + xb_bytes);
  uint8_t* ring = smem + kXOff + xb_bytes + xs_bytes;
  float* red = reinterpret_cast<float*>(ring + S * sbytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(red + kWarps * 16 * TOKMAX);
  int* flag = reinterpret_cast<int*>(bars + 8);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, tig = lane & 3;
  const int tiles_per_e = (I / 16) * 2;
  const int ntiles = a.active[a.E] * tiles_per_e;

  if (tid == 0) {
    for (int s = 0; s < S; ++s) mbar_init(&bars[s], 1);
    fence_barrier_init();
  }
  auto issue = [&](int tile, int s) {
    const int e = a.active[tile / tiles_per_e];
    const int rem = tile % tiles_per_e;
    const int r0 = (rem >> 1) * 16, m = rem & 1;
    uint8_t* st = ring + s * sbytes;
    fence_proxy_async_smem();  // earlier generic reads of this stage come before the async writes
    if (lane == 0) mbar_arrive_expect_tx(&bars[s], 16u * row_bytes + 16u * dbytes);
    __syncwarp();
    const size_t rowg = static_cast<size_t>(e) * I + r0;
    const uint8_t* codes = m ? a.up_codes : a.gate_codes;
    const uint16_t* dpl = m ? a.up_d : a.gate_d;
    if (lane < 16) bulk_copy_g2s(st + lane * rs, codes + (rowg + lane) * row_bytes, row_bytes, &bars[s]);
    if (lane == 16) bulk_copy_g2s(st + 16 * rs, dpl + rowg * (H / 256), 16 * dbytes, &bars[s]);
  };
  __syncthreads();
  if (warp == 0)
    for (int s = 0; s < S; ++s) {
      const int tile = blockIdx.x + s * gridDim.x;
      if (tile < ntiles) issue(tile, s);
    }
  // replicated selector tables: word (entry * 32 + lane)
  for (int i = tid; i < 256 * 32; i += kThreads)
    reinterpret_cast<uint32_t*>(smem + kLvlOff)[i] = d_sel_tables.level[i >> 5];
  for (int i = tid; i < 128 * 32; i += kThreads)
    reinterpret_cast<uint32_t*>(smem + kSgnOff)[i] = d_sel_tables.sign[i >> 5];
  if (a.x_in_smem) {
    const int nx = T * 2 * H / 16;
    for (int i = tid; i < nx; i += kThreads) reinterpret_cast<uint4*>(xsm)[i] = reinterpret_cast<const uint4*>(a.xd)[i];
    for (int i = tid; i < T * (H / 256); i += kThreads) xssm[i] = a.xs[i];
  }
  __syncthreads();
  const int8_t* xdig = a.x_in_smem ? xsm : a.xd;
  const float* xscl = a.x_in_smem ? xssm : a.xs;

  const int nsb = H / 256;  // sub-blocks (of 32) per warp
  const int sb0 = warp * nsb;
  const bool wide = (nsb & 1) == 0;  // 16-byte record loads (two sub-blocks) stay aligned
  const uint32_t lane4 = static_cast<uint32_t>(lane) << 2;
  const uint32_t rot_idx = (8u * tig - 7u) & 31u;  // brings byte tig of the index word to bits 7..14
  const uint32_t rot_sig = (7u * tig - 7u) & 31u;  // brings sign field tig to bits 7..13

  int it = 0;
  for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
    const int s = it % S;
    const uint32_t parity = (it / S) & 1u;
    if (tid == 0) *flag = mbar_wait_bounded(&bars[s], parity, a.err, ERR_TIMEOUT) ? 1 : 0;
    __syncthreads();
    if (*flag == 0) return;
    mbar_try_wait(&bars[s], parity);  // completes at once; orders the bulk-copied bytes for this thread

    const int e = a.active[tile / tiles_per_e];
    const int rem = tile % tiles_per_e;
    const int r0 = (rem >> 1) * 16, mat = rem & 1;
    const int p0 = a.offsets[e], ne = a.offsets[e + 1] - p0;
    const uint8_t* st = ring + s * sbytes;
    const uint8_t* row_g = st + g * rs;
    const uint8_t* row_g8 = st + (g + 8) * rs;
    const uint16_t* dtab = reinterpret_cast<const uint16_t*>(st + 16 * rs);

    const int tpg = ne == 1 ? 1 : (ne == 2 ? 2 : 4);
    const int sps = 4 / tpg;
    const int ngroups = (ne + tpg - 1) / tpg;
    const int tslot_b = (g >> 1) % tpg, sslot_b = (g >> 1) / tpg, dig_b = g & 1;
    const int tslot_c = tig % tpg, sslot_c = tig / tpg;

    for (int pass0 = 0; pass0 < ngroups; pass0 += MAXQ) {
      const int8_t* xb[MAXQ];
      const float* xsc[MAXQ];
#pragma unroll
      for (int q = 0; q < MAXQ; ++q) {
        const int grp = pass0 + q;
        const int tb = grp * tpg + tslot_b, tc = grp * tpg + tslot_c;
        xb[q] = (grp < ngroups && tb < ne)
                    ? xdig + (static_cast<size_t>(a.perm[p0 + tb] / a.k) * 2 + dig_b) * H + 8 * tig
                    : nullptr;
        xsc[q] = (grp < ngroups && tc < ne) ? xscl + static_cast<size_t>(a.perm[p0 + tc] / a.k) * (H / 256)
                                            : nullptr;
      }
      int acc[MAXQ][4];
      int iacc[MAXQ][2];
      float facc[MAXQ][2];
#pragma unroll
      for (int q = 0; q < MAXQ; ++q) {
        acc[q][0] = acc[q][1] = acc[q][2] = acc[q][3] = 0;
        iacc[q][0] = iacc[q][1] = 0;
        facc[q][0] = facc[q][1] = 0.f;
      }
      uint32_t vcap0 = 0, vcap1 = 0;  // v of this thread's flush sub-block, rows g and g+8
      int set_start = sb0;
      for (int c = 0; c < nsb; c += 4) {
        const int nu = min(4, nsb - c);
        uint2 rec[4][2];
        if (wide) {
#pragma unroll
          for (int u2 = 0; u2 < 2; ++u2) {
            uint4 r0v = make_uint4(0u, 0u, 0u, 0u), r1v = make_uint4(0u, 0u, 0u, 0u);
            if (2 * u2 < nu) {
              r0v = *reinterpret_cast<const uint4*>(row_g + (sb0 + c + 2 * u2) * 8);
              r1v = *reinterpret_cast<const uint4*>(row_g8 + (sb0 + c + 2 * u2) * 8);
            }
            rec[2 * u2][0] = make_uint2(r0v.x, r0v.y);
            rec[2 * u2 + 1][0] = make_uint2(r0v.z, r0v.w);
            rec[2 * u2][1] = make_uint2(r1v.x, r1v.y);
            rec[2 * u2 + 1][1] = make_uint2(r1v.z, r1v.w);
          }
        } else {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            rec[u][0] = u < nu ? *reinterpret_cast<const uint2*>(row_g + (sb0 + c + u) * 8) : make_uint2(0u, 0u);
            rec[u][1] = u < nu ? *reinterpret_cast<const uint2*>(row_g8 + (sb0 + c + u) * 8) : make_uint2(0u, 0u);
          }
        }
        uint32_t af[4][2][2];  // [u][row g / g+8][elements 0-3 / 4-7]
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const uint32_t al = (rotr(rec[u][r].x, rot_idx) & 0x7F80u) | lane4;
            const uint32_t as = (rotr(rec[u][r].y, rot_sig) & 0x3F80u) | lane4;
            const uint32_t sel = *reinterpret_cast<const uint32_t*>(smem + kLvlOff + al) |
                                 *reinterpret_cast<const uint32_t*>(smem + kSgnOff + as);
            af[u][r][0] = prmt(kPosBytes, kNegBytes, sel);
            af[u][r][1] = prmt(kPosBytes, kNegBytes, sel >> 16);
          }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (u >= nu) break;
          const int sb = sb0 + c + u;
          const int slot = sb - set_start;
          if (slot == sslot_c) {
            vcap0 = rec[u][0].y;
            vcap1 = rec[u][1].y;
          }
#pragma unroll
          for (int q = 0; q < MAXQ; ++q) {
            if (pass0 + q >= ngroups) break;
            uint2 b = make_uint2(0u, 0u);
            if (slot == sslot_b && xb[q]) b = *reinterpret_cast<const uint2*>(xb[q] + sb * 32);
            mma_s8s8(acc[q], af[u][0][0], af[u][1][0], af[u][0][1], af[u][1][1], b.x, b.y);
          }
          const bool sb_end = ((sb + 1) & 7) == 0 || sb + 1 == sb0 + nsb;
          if (slot == sps - 1 || sb_end) {
            // flush the set: (2ls+1) * (128 hi + lo) into the int32 super-block sums
            const int odd0 = static_cast<int>((vcap0 >> 27) | 1u);
            const int odd1 = static_cast<int>((vcap1 >> 27) | 1u);
#pragma unroll
            for (int q = 0; q < MAXQ; ++q) {
              iacc[q][0] += (acc[q][0] * 128 + acc[q][1]) * odd0;
              iacc[q][1] += (acc[q][2] * 128 + acc[q][3]) * odd1;
              acc[q][0] = acc[q][1] = acc[q][2] = acc[q][3] = 0;
            }
            vcap0 = vcap1 = 0;
            set_start = sb + 1;
            if (sb_end) {
              // super-block done: scale by d (per row) and 2^s/8 (per token)
              const int SBi = sb >> 3;
              const float d0 = half_bits_to_float(dtab[g * (H / 256) + SBi]);
              const float d1 = half_bits_to_float(dtab[(g + 8) * (H / 256) + SBi]);
#pragma unroll
              for (int q = 0; q < MAXQ; ++q) {
                const float xsv = xsc[q] ? xsc[q][SBi] : 0.f;
                facc[q][0] = fmaf(static_cast<float>(iacc[q][0]), d0 * xsv, facc[q][0]);
                facc[q][1] = fmaf(static_cast<float>(iacc[q][1]), d1 * xsv, facc[q][1]);
                iacc[q][0] = iacc[q][1] = 0;
              }
            }
          }
        }
      }
      // combine the quad lanes holding the same token (tpg < 4), then across warps
#pragma unroll
      for (int q = 0; q < MAXQ; ++q)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          float v = facc[q][r];
          if (tpg == 1) {
            v += __shfl_xor_sync(0xffffffffu, v, 1);
            v += __shfl_xor_sync(0xffffffffu, v, 2);
          } else if (tpg == 2) {
            v += __shfl_xor_sync(0xffffffffu, v, 2);
          }
          facc[q][r] = v;
        }
#pragma unroll
      for (int q = 0; q < MAXQ; ++q) {
        const int tok = q * tpg + tslot_c;
        const bool owner = (tpg == 4) || (tig < tpg);
        if (pass0 + q < ngroups && owner) {
          red[(warp * 16 + g) * TOKMAX + tok] = facc[q][0];
          red[(warp * 16 + g + 8) * TOKMAX + tok] = facc[q][1];
        }
      }
      __syncthreads();
      for (int i = tid; i < TOKMAX * 16; i += kThreads) {
        const int row = i & 15, tok = i >> 4;
        const int tglob = pass0 * tpg + tok;
        if (tok < MAXQ * tpg && tglob < ne) {
          float v = 0.f;
#pragma unroll
          for (int w = 0; w < kWarps; ++w) v += red[(w * 16 + row) * TOKMAX + tok];
          a.gu[(static_cast<size_t>(p0 + tglob) * 2 + mat) * I + r0 + row] = v;
        }
      }
      __syncthreads();
    }
    // stage s is free: prefetch the tile S steps ahead into it
    if (warp == 0) {
      const int nt = tile + S * gridDim.x;
      if (nt < ntiles) issue(nt, s);
    }
  }
}

// ---------------------------------------------------------------------------
// Aligned layout (H % 1024 == 0): each warp's range of sub-blocks starts on a
// multiple of four, so a chunk of four sub-blocks is exactly a whole number of
// column sets and every set/flush decision below is fixed at compile time.
// TPG = tokens sharing one MMA (1, 2 or 4); sub-blocks per set = 4 / TPG.
struct TileCtx {
  const uint8_t* row_g;
  const uint8_t* row_g8;
  const uint16_t* dtab;
  const int8_t* xdig;
  const float* xscl;
  float* red;
  int p0, ne, sb0, nsb, warp, g, tig;
  uint32_t lane4, rot_idx, rot_sig;
};

template <int TPG, int MAXQ>
__device__ __forceinline__ void gu_tile_aligned(const GateupArgs& a, const uint8_t* smem, const TileCtx& t,
                                                float (&facc)[4][2], int pass0) {
  constexpr int SPS = 4 / TPG;
  const int H = a.H;
  const int ngroups = (t.ne + TPG - 1) / TPG;
  const int tslot_b = (t.g >> 1) % TPG, sslot_b = (t.g >> 1) / TPG, dig_b = t.g & 1;
  const int tslot_c = t.tig % TPG, sslot_c = t.tig / TPG;
  const int8_t* xb[MAXQ];
  const float* xsc[MAXQ];
  bool bval[MAXQ];
#pragma unroll
  for (int q = 0; q < MAXQ; ++q) {
    const int grp = pass0 + q;
    const int tb = grp * TPG + tslot_b, tc = grp * TPG + tslot_c;
    bval[q] = grp < ngroups && tb < t.ne;
    xb[q] = t.xdig + (static_cast<size_t>(bval[q] ? a.perm[t.p0 + tb] / a.k : 0) * 2 + dig_b) * H + 8 * t.tig +
            (t.sb0 + sslot_b) * 32;
    xsc[q] = (grp < ngroups && tc < t.ne) ? t.xscl + static_cast<size_t>(a.perm[t.p0 + tc] / a.k) * (H / 256)
                                          : nullptr;
  }
  int acc[MAXQ][2][4];
  int iacc[MAXQ][2];
#pragma unroll
  for (int q = 0; q < MAXQ; ++q) {
#pragma unroll
    for (int h = 0; h < 2; ++h) acc[q][h][0] = acc[q][h][1] = acc[q][h][2] = acc[q][h][3] = 0;
    iacc[q][0] = iacc[q][1] = 0;
  }
  for (int c = 0; c < t.nsb; c += 4) {
    const int sbc = t.sb0 + c;
    uint2 rec[4][2];
    {
      const uint4 a0 = *reinterpret_cast<const uint4*>(t.row_g + sbc * 8);
      const uint4 a1 = *reinterpret_cast<const uint4*>(t.row_g + sbc * 8 + 16);
      const uint4 b0 = *reinterpret_cast<const uint4*>(t.row_g8 + sbc * 8);
      const uint4 b1 = *reinterpret_cast<const uint4*>(t.row_g8 + sbc * 8 + 16);
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
        const uint32_t al = (rotr(rec[u][r].x, t.rot_idx) & 0x7F80u) | t.lane4;
        const uint32_t as = (rotr(rec[u][r].y, t.rot_sig) & 0x3F80u) | t.lane4;
        const uint32_t sel = *reinterpret_cast<const uint32_t*>(smem + kLvlOff + al) |
                             *reinterpret_cast<const uint32_t*>(smem + kSgnOff + as);
        af[u][r][0] = prmt(kPosBytes, kNegBytes, sel);
        af[u][r][1] = prmt(kPosBytes, kNegBytes, sel >> 16);
      }
#pragma unroll
    for (int q = 0; q < MAXQ; ++q) {
      if (pass0 + q >= ngroups) break;
      uint2 bl[TPG];
#pragma unroll
      for (int j = 0; j < TPG; ++j)
        bl[j] = bval[q] ? *reinterpret_cast<const uint2*>(xb[q] + (c + j * SPS) * 32) : make_uint2(0u, 0u);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = u / SPS, slot = u % SPS;
        const bool on = slot == sslot_b;
        mma_s8s8(acc[q][u & 1], af[u][0][0], af[u][1][0], af[u][0][1], af[u][1][1], on ? bl[j].x : 0u,
                 on ? bl[j].y : 0u);
        if (slot == SPS - 1) {
          // set j done: this thread owns sub-block j*SPS + sslot_c for rows g and g+8
          uint32_t v0 = rec[j * SPS][0].y, v1 = rec[j * SPS][1].y;
#pragma unroll
          for (int w = 1; w < SPS; ++w)
            if (sslot_c == w) { v0 = rec[j * SPS + w][0].y; v1 = rec[j * SPS + w][1].y; }
          const int odd0 = static_cast<int>((v0 >> 27) | 1u), odd1 = static_cast<int>((v1 >> 27) | 1u);
          const int c0 = acc[q][0][0] + acc[q][1][0], c1 = acc[q][0][1] + acc[q][1][1];
          const int c2 = acc[q][0][2] + acc[q][1][2], c3 = acc[q][0][3] + acc[q][1][3];
          iacc[q][0] += (c0 * 128 + c1) * odd0;
          iacc[q][1] += (c2 * 128 + c3) * odd1;
#pragma unroll
          for (int h = 0; h < 2; ++h) acc[q][h][0] = acc[q][h][1] = acc[q][h][2] = acc[q][h][3] = 0;
        }
      }
    }
    if (((sbc + 4) & 7) == 0 || c + 4 == t.nsb) {
      // super-block done: scale by d (per row) and 2^s/8 (per token)
      const int SBi = (sbc + 3) >> 3;
      const float d0 = half_bits_to_float(t.dtab[t.g * (H / 256) + SBi]);
      const float d1 = half_bits_to_float(t.dtab[(t.g + 8) * (H / 256) + SBi]);
#pragma unroll
      for (int q = 0; q < MAXQ; ++q) {
        const float xsv = xsc[q] ? xsc[q][SBi] : 0.f;
        facc[q][0] = fmaf(static_cast<float>(iacc[q][0]), d0 * xsv, facc[q][0]);
        facc[q][1] = fmaf(static_cast<float>(iacc[q][1]), d1 * xsv, facc[q][1]);
        iacc[q][0] = iacc[q][1] = 0;
      }
    }
  }
  // combine the quad lanes holding the same token (TPG < 4), then across warps
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
  constexpr int TOKMAX = 16;
#pragma unroll
  for (int q = 0; q < MAXQ; ++q) {
    const int tok = q * TPG + tslot_c;
    const bool owner = (TPG == 4) || (t.tig < TPG);
    if (pass0 + q < ngroups && owner) {
      t.red[(t.warp * 16 + t.g) * TOKMAX + tok] = facc[q][0];
      t.red[(t.warp * 16 + t.g + 8) * TOKMAX + tok] = facc[q][1];
    }
  }
}

template <bool SINGLE>
__global__ void __launch_bounds__(kThreads, 1) gateup_aligned_kernel(GateupArgs a) {
  constexpr int TOKMAX = 16;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int H = a.H, I = a.I, S = a.stages, T = a.T;
  const int row_bytes = H / 4, rs = H / 4 + 16, dbytes = H / 128;
  const size_t sbytes = static_cast<size_t>(16) * rs + align_up(static_cast<size_t>(16) * dbytes, 16);
  const size_t xb_bytes = a.x_in_smem ? align_up(static_cast<size_t>(T) * 2 * H, 128) : 0;
  const size_t xs_bytes = a.x_in_smem ? align_up(static_cast<size_t>(T) * (H / 256) * 4, 128) : 0;
  int8_t* xsm = reinterpret_cast<int8_t*>(smem + kXOff);
  float* xssm = reinterpret_cast<float*>(smem + kXOff + xb_bytes);
  uint8_t* ring = smem + kXOff + xb_bytes + xs_bytes;
  float* red = reinterpret_cast<float*>(ring + S * sbytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(red + kWarps * 16 * TOKMAX);
  int* flag = reinterpret_cast<int*>(bars + 8);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, tig = lane & 3;
  const int tiles_per_e = (I / 16) * 2;
  const int ntiles = a.active[a.E] * tiles_per_e;

  if (tid == 0) {
    for (int s = 0; s < S; ++s) mbar_init(&bars[s], 1);
    fence_barrier_init();
  }
  auto issue = [&](int tile, int s) {
    const int e = a.active[tile / tiles_per_e];
    const int rem = tile % tiles_per_e;
    const int r0 = (rem >> 1) * 16, m = rem & 1;
    uint8_t* st = ring + s * sbytes;
    fence_proxy_async_smem();
    if (lane == 0) mbar_arrive_expect_tx(&bars[s], 16u * row_bytes + 16u * dbytes);
    __syncwarp();
    const size_t rowg = static_cast<size_t>(e) * I + r0;
    const uint8_t* codes = m ? a.up_codes : a.gate_codes;
    const uint16_t* dpl = m ? a.up_d : a.gate_d;
    if (lane < 16) bulk_copy_g2s(st + lane * rs, codes + (rowg + lane) * row_bytes, row_bytes, &bars[s]);
    if (lane == 16) bulk_copy_g2s(st + 16 * rs, dpl + rowg * (H / 256), 16 * dbytes, &bars[s]);
  };
  __syncthreads();
  if (warp == 0)
    for (int s = 0; s < S; ++s) {
      const int tile = blockIdx.x + s * gridDim.x;
      if (tile < ntiles) issue(tile, s);
    }
  for (int i = tid; i < 256 * 32; i += kThreads)
    reinterpret_cast<uint32_t*>(smem + kLvlOff)[i] = d_sel_tables.level[i >> 5];
  for (int i = tid; i < 128 * 32; i += kThreads)
    reinterpret_cast<uint32_t*>(smem + kSgnOff)[i] = d_sel_tables.sign[i >> 5];
  if (a.x_in_smem) {
    const int nx = T * 2 * H / 16;
    for (int i = tid; i < nx; i += kThreads) reinterpret_cast<uint4*>(xsm)[i] = reinterpret_cast<const uint4*>(a.xd)[i];
    for (int i = tid; i < T * (H / 256); i += kThreads) xssm[i] = a.xs[i];
  }
  __syncthreads();

  TileCtx t{};
  t.xdig = a.x_in_smem ? xsm : a.xd;
  t.xscl = a.x_in_smem ? xssm : a.xs;
  t.red = red;
  t.nsb = H / 256;
  t.sb0 = warp * t.nsb;
  t.warp = warp;
  t.g = g;
  t.tig = tig;
  t.lane4 = static_cast<uint32_t>(lane) << 2;
  t.rot_idx = (8u * tig - 7u) & 31u;
  t.rot_sig = (7u * tig - 7u) & 31u;

  int it = 0;
  for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
    const int s = it % S;
    const uint32_t parity = (it / S) & 1u;
    if (tid == 0) *flag = mbar_wait_bounded(&bars[s], parity, a.err, ERR_TIMEOUT) ? 1 : 0;
    __syncthreads();
    if (*flag == 0) return;
    mbar_try_wait(&bars[s], parity);

    const int e = a.active[tile / tiles_per_e];
    const int rem = tile % tiles_per_e;
    const int r0 = (rem >> 1) * 16, mat = rem & 1;
    t.p0 = a.offsets[e];
    t.ne = a.offsets[e + 1] - t.p0;
    const uint8_t* st = ring + s * sbytes;
    t.row_g = st + g * rs;
    t.row_g8 = st + (g + 8) * rs;
    t.dtab = reinterpret_cast<const uint16_t*>(st + 16 * rs);
    const int tpg = (SINGLE || t.ne == 1) ? 1 : (t.ne == 2 ? 2 : 4);
    const int ngroups = (t.ne + tpg - 1) / tpg;
    const int maxq = tpg == 4 ? 4 : 1;
    for (int pass0 = 0; pass0 < ngroups; pass0 += maxq) {
      float facc[4][2] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
      if (SINGLE || tpg == 1) gu_tile_aligned<1, 1>(a, smem, t, facc, pass0);
      else if (tpg == 2) gu_tile_aligned<2, 1>(a, smem, t, facc, pass0);
      else gu_tile_aligned<4, 4>(a, smem, t, facc, pass0);
      __syncthreads();
      for (int i = tid; i < TOKMAX * 16; i += kThreads) {
        const int row = i & 15, tok = i >> 4;
        const int tglob = pass0 * tpg + tok;
        if (tok < maxq * tpg && tglob < t.ne) {
          float v = 0.f;
#pragma unroll
          for (int w = 0; w < kWarps; ++w) v += red[(w * 16 + row) * TOKMAX + tok];
          a.gu[(static_cast<size_t>(t.p0 + tglob) * 2 + mat) * I + r0 + row] = v;
        }
      }
      __syncthreads();
    }
    if (warp == 0) {
      const int nt = tile + S * gridDim.x;
      if (nt < ntiles) issue(nt, s);
    }
  }
}

}  // namespace

int launch_gateup(const GateupArgs& a0, int slots, int sms, cudaStream_t st) {
  GateupArgs a = a0;
  const bool aligned = a.H % 1024 == 0;
  const int maxq = (a.T == 1 && !aligned) ? 1 : 4;
  const size_t sb = stage_bytes(a.H);
  const size_t budget = 227 * 1024;
  auto fixed = [&](bool xin) {
    return static_cast<size_t>(kXOff) + (xin ? x_bytes(a.T, a.H) : 0) + red_bytes(maxq) + 16 * 8 + 64;
  };
  a.x_in_smem = a.T <= 4 ? 1 : 0;
  int stages = budget > fixed(a.x_in_smem) ? static_cast<int>((budget - fixed(a.x_in_smem)) / sb) : 0;
  if (stages < 3 && a.x_in_smem) {  // keep the ring deep: read activations from global memory instead
    a.x_in_smem = 0;
    stages = static_cast<int>((budget - fixed(false)) / sb);
  }
  stages = std::max(1, std::min(stages, 6));
  a.stages = stages;
  const size_t smem = stages * sb + fixed(a.x_in_smem);
  const int tiles = slots * (a.I / 16) * 2;
  const int grid = std::max(1, std::min(tiles, sms));
  if (aligned) {
    if (a.T == 1) {
      cudaFuncSetAttribute(gateup_aligned_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem));
      gateup_aligned_kernel<true><<<grid, kThreads, smem, st>>>(a);
    } else {
      cudaFuncSetAttribute(gateup_aligned_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem));
      gateup_aligned_kernel<false><<<grid, kThreads, smem, st>>>(a);
    }
  } else if (maxq == 1) {
    cudaFuncSetAttribute(gateup_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    gateup_kernel<1><<<grid, kThreads, smem, st>>>(a);
  } else {
    cudaFuncSetAttribute(gateup_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    gateup_kernel<4><<<grid, kThreads, smem, st>>>(a);
  }
  return cudaGetLastError() == cudaSuccess ? OK : ERR_CUDA;
}

}  // namespace moe
