// down_gemv.cu - down dequant-GEMV of the routed experts (Q2K-style codes) on
// unsigned x signed int8 warp MMAs (m16n8k32), one output row per assignment.
//
// Source of the format split: "ds4 : analyse pratique pour un usage documenté",
// section « Support de modèles et choix de quantification » (down in Q2_K).
// The value w = d*sc*q - dmin*m is the library's specification of that format.
// With h_k = 2^e Q_k (Q = 128 hi + lo, one e per 256-element block of h), one
// super-block of a row contributes
//   2^e * ( d * sum_s sc_s (sum_k q_k Q_k)  -  dmin * sum_s m_s (sum_k Q_k) )
// where both sums over the 16 sub-blocks s are exact int32: the first from the
// MMA, the second from the per-16 sums of Q written by the h quantiser.
//
// Tile = (active expert, 64 rows of H). Each stage holds the tile's 64 code rows
// (padded by 16 bytes), their d|dmin words and the h digits, scales and sums of
// up to 4 of the expert's assignments, all brought in by bulk copies. 8 warps =
// 4 groups of 16 rows x 2 halves of I; one MMA covers a pair of sub-blocks
// (A, B); the 8 columns hold (half, slot or token, digit). The per-tile body is
// compiled separately for one token (two pairs per column set) and for token
// pairs (one pair per set), so every set decision is fixed at compile time.
#include <algorithm>

#include "decode.cuh"
#include "profile.cuh"
#include "ptx.cuh"

namespace moe {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kRows = 64;
constexpr int kStageTok = 4;  // assignments whose h data ride along in each stage
constexpr int kTokMax = 8;    // assignments per pass (4 groups of 2)

// per-assignment stride (floats) of the 256-block scales of h, padded to 16 bytes
__host__ __device__ inline int hsc_stride(int I) { return ((I / 256) + 3) & ~3; }
__host__ __device__ inline size_t hdata_bytes(int I) {
  return static_cast<size_t>(kStageTok) * (2 * I + hsc_stride(I) * 4 + (I / 16) * 4);
}
__host__ __device__ inline size_t stage_bytes(int I) {
  return static_cast<size_t>(kRows) * (I / 256 * 80 + 16) + static_cast<size_t>(kRows) * (I / 256) * 4 +
         hdata_bytes(I);
}
constexpr size_t kFixed = static_cast<size_t>(kWarps) * 16 * kTokMax * 4 + 16 * 8 + 64;

struct DnCtx {
  const uint8_t* rowA;  // code row of this thread's first row (rows rA, rB = rA + 8)
  const uint8_t* rowB;
  const uint32_t* ddt;
  const int8_t* hd_s;
  const float* hsc_s;
  const int32_t* hq_s;
  float* red;
  int p0, ne, pr0, npair, nblk, rA, rB, warp, g, tig, hss;
};

// One pass over this warp's half of I for up to MAXQ column groups of TPG
// assignments each; leaves per-(row, assignment) partial sums in red.
template <int TPG, int MAXQ>
__device__ __forceinline__ void dn_tile(const DownArgs& a, const DnCtx& t, int pass0) {
  constexpr int SPP = TPG == 1 ? 2 : 1;  // sub-block pairs per column set
  const int I = a.I;
  const int ngroups = (t.ne + TPG - 1) / TPG;
  const int dig_b = t.g & 1, hb = (t.g >> 1) & 1, sl_b = t.g >> 2;  // B column: digit, half, slot/token
  const int hc = t.tig & 1, sl_c = t.tig >> 1;                      // owned C columns: half, slot/token
  const uint32_t sh = 2 * t.tig;

  const int8_t* hb_ptr[MAXQ];
  bool hb_on[MAXQ];
  const float* sc_ptr[MAXQ];
  const int32_t* hq_ptr[MAXQ];
#pragma unroll
  for (int q = 0; q < MAXQ; ++q) {
    const int grp = pass0 + q;
    const int tb = grp * TPG + (TPG == 1 ? 0 : sl_b);
    const int tc = grp * TPG + (TPG == 1 ? 0 : sl_c);
    hb_on[q] = grp < ngroups && tb < t.ne;
    const int tbs = hb_on[q] ? tb : 0;
    hb_ptr[q] = (tbs < kStageTok ? t.hd_s + (static_cast<size_t>(tbs) * 2 + dig_b) * I
                                 : a.hd + (static_cast<size_t>(t.p0 + tbs) * 2 + dig_b) * I) +
                8 * t.tig + t.pr0 * 32;
    sc_ptr[q] = nullptr;
    hq_ptr[q] = nullptr;
    if (grp < ngroups && tc < t.ne) {
      sc_ptr[q] = tc < kStageTok ? t.hsc_s + tc * t.hss : a.hsc + static_cast<size_t>(t.p0 + tc) * t.hss;
      hq_ptr[q] = tc < kStageTok ? t.hq_s + tc * (I / 16) : a.hq + static_cast<size_t>(t.p0 + tc) * (I / 16);
    }
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
  for (int c = 0; c < t.npair; c += 4) {
    const int prc = t.pr0 + c;
    // q words of pairs (prc .. prc+3) for rows A and B (two 16-byte loads per row)
    uint32_t af[4][4];
#pragma unroll
    for (int u2 = 0; u2 < 2; ++u2) {
      const int pr = prc + 2 * u2;
      const int off = (pr >> 3) * 80 + 16 + 8 * (pr & 7);
      const uint4 qa = *reinterpret_cast<const uint4*>(t.rowA + off);
      const uint4 qb = *reinterpret_cast<const uint4*>(t.rowB + off);
      af[2 * u2][0] = (qa.x >> sh) & 0x03030303u;  // row A, sub-block A of the pair
      af[2 * u2][1] = (qb.x >> sh) & 0x03030303u;  // row B, sub-block A
      af[2 * u2][2] = (qa.y >> sh) & 0x03030303u;  // row A, sub-block B
      af[2 * u2][3] = (qb.y >> sh) & 0x03030303u;
      af[2 * u2 + 1][0] = (qa.z >> sh) & 0x03030303u;
      af[2 * u2 + 1][1] = (qb.z >> sh) & 0x03030303u;
      af[2 * u2 + 1][2] = (qa.w >> sh) & 0x03030303u;
      af[2 * u2 + 1][3] = (qb.w >> sh) & 0x03030303u;
    }
#pragma unroll
    for (int q = 0; q < MAXQ; ++q) {
      if (pass0 + q >= ngroups) break;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int slot = u % SPP;
        uint2 bv = make_uint2(0u, 0u);
        if (hb_on[q] && (SPP == 1 || slot == sl_b)) {
          bv = *reinterpret_cast<const uint2*>(hb_ptr[q] + (c + u) * 32);
          if (hb) bv.x = 0u; else bv.y = 0u;
        }
        mma_u8s8(acc[q], af[u][0], af[u][1], af[u][2], af[u][3], bv.x, bv.y);
        if (slot == SPP - 1) {
          // set done: this thread owns sub-block 2*(first pair of set + slot_c) + hc for rows A and B
          const int sub = 2 * (prc + u - (SPP - 1) + (TPG == 1 ? sl_c : 0)) + hc;
          const int bb = sub >> 4, si = sub & 15;
          const uint32_t scA = t.rowA[bb * 80 + si], scB = t.rowB[bb * 80 + si];
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
    if (((prc + 4) & 7) == 0 || c + 4 == t.npair) {
      // super-block (8 pairs) done: 2^e * (d * A - dmin * M)
      const int SBi = (prc + 3) >> 3;
      const uint32_t wA = t.ddt[t.rA * t.nblk + SBi], wB = t.ddt[t.rB * t.nblk + SBi];
      const float dA = half_bits_to_float(static_cast<uint16_t>(wA & 0xFFFFu));
      const float nA = half_bits_to_float(static_cast<uint16_t>(wA >> 16));
      const float dB = half_bits_to_float(static_cast<uint16_t>(wB & 0xFFFFu));
      const float nB = half_bits_to_float(static_cast<uint16_t>(wB >> 16));
#pragma unroll
      for (int q = 0; q < MAXQ; ++q) {
        const float e2 = sc_ptr[q] ? sc_ptr[q][SBi] : 0.f;
        facc[q][0] = fmaf(e2, fmaf(dA, static_cast<float>(iA[q][0]), -nA * static_cast<float>(iM[q][0])), facc[q][0]);
        facc[q][1] = fmaf(e2, fmaf(dB, static_cast<float>(iA[q][1]), -nB * static_cast<float>(iM[q][1])), facc[q][1]);
        iA[q][0] = iA[q][1] = iM[q][0] = iM[q][1] = 0;
      }
    }
  }
  // reduce lanes holding the same assignment (TPG 1: all 4 tig; TPG 2: tig pairs 0/1 and 2/3)
#pragma unroll
  for (int q = 0; q < MAXQ; ++q)
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      float v = facc[q][r];
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      if (TPG == 1) v += __shfl_xor_sync(0xffffffffu, v, 2);
      facc[q][r] = v;
    }
#pragma unroll
  for (int q = 0; q < MAXQ; ++q) {
    const int tok = q * TPG + (TPG == 1 ? 0 : sl_c);
    const bool owner = TPG == 1 ? (t.tig == 0) : (hc == 0);
    if (pass0 + q < ngroups && owner) {
      t.red[(t.warp * 16 + t.g) * kTokMax + tok] = facc[q][0];
      t.red[(t.warp * 16 + t.g + 8) * kTokMax + tok] = facc[q][1];
    }
  }
}

template <bool SINGLE>
__global__ void __launch_bounds__(kThreads, 1) down_kernel(DownArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int H = a.H, I = a.I, S = a.stages;
  const int nblk = I / 256;
  const int row_bytes = nblk * 80, rs = row_bytes + 16;
  const size_t sbytes = stage_bytes(I);
  const size_t hoff = static_cast<size_t>(kRows) * rs + static_cast<size_t>(kRows) * nblk * 4;
  const int hss = hsc_stride(I);
  uint8_t* ring = smem;
  float* red = reinterpret_cast<float*>(smem + S * sbytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(red + kWarps * 16 * kTokMax);
  int* flag = reinterpret_cast<int*>(bars + 8);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, tig = lane & 3;
  const int tiles_per_e = H / kRows;
  const int ntiles = a.active[a.E] * tiles_per_e;

  if (tid == 0) {
    for (int s = 0; s < S; ++s) mbar_init(&bars[s], 1);
    fence_barrier_init();
  }
  __syncthreads();

  auto issue = [&](int tile, int s) {
    const int e = a.active[tile / tiles_per_e];
    const int r0 = (tile % tiles_per_e) * kRows;
    const int p0 = a.offsets[e];
    const int nst = min(a.offsets[e + 1] - p0, kStageTok);
    uint8_t* st = ring + s * sbytes;
    fence_proxy_async_smem();
    const uint32_t hbytes = static_cast<uint32_t>(nst) * (2 * I + hss * 4 + (I / 16) * 4);
    if (lane == 0) mbar_arrive_expect_tx(&bars[s], kRows * row_bytes + kRows * nblk * 4 + hbytes);
    __syncwarp();
    const size_t rowg = static_cast<size_t>(e) * H + r0;
    bulk_copy_g2s(st + lane * rs, a.codes + (rowg + lane) * row_bytes, row_bytes, &bars[s]);
    bulk_copy_g2s(st + (lane + 32) * rs, a.codes + (rowg + lane + 32) * row_bytes, row_bytes, &bars[s]);
    uint8_t* hs = st + hoff;
    if (lane == 0) bulk_copy_g2s(st + kRows * rs, a.dd + rowg * nblk, kRows * nblk * 4, &bars[s]);
    if (lane == 1) bulk_copy_g2s(hs, a.hd + static_cast<size_t>(p0) * 2 * I, nst * 2 * I, &bars[s]);
    if (lane == 2)
      bulk_copy_g2s(hs + kStageTok * 2 * I, a.hsc + static_cast<size_t>(p0) * hss, nst * hss * 4, &bars[s]);
    if (lane == 3)
      bulk_copy_g2s(hs + kStageTok * (2 * I + hss * 4), a.hq + static_cast<size_t>(p0) * (I / 16),
                    nst * (I / 16) * 4, &bars[s]);
  };

  if (warp == 0)
    for (int s = 0; s < S; ++s) {
      const int tile = blockIdx.x + s * gridDim.x;
      if (tile < ntiles) issue(tile, s);
    }

  DnCtx t{};
  t.red = red;
  t.npair = I / 64;  // sub-block pairs per half of I (a multiple of 4)
  t.pr0 = (warp >> 2) * t.npair;
  t.nblk = nblk;
  t.rA = (warp & 3) * 16 + g;
  t.rB = t.rA + 8;
  t.warp = warp;
  t.g = g;
  t.tig = tig;
  t.hss = hss;

  int it = 0;
  for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
    const int s = it % S;
    const uint32_t parity = (it / S) & 1u;
    if (tid == 0) *flag = mbar_wait_bounded(&bars[s], parity, a.err, ERR_TIMEOUT) ? 1 : 0;
    __syncthreads();
    if (*flag == 0) return;
    mbar_try_wait(&bars[s], parity);

    const int e = a.active[tile / tiles_per_e];
    const int r0 = (tile % tiles_per_e) * kRows;
    t.p0 = a.offsets[e];
    t.ne = a.offsets[e + 1] - t.p0;
    const uint8_t* st = ring + s * sbytes;
    t.rowA = st + t.rA * rs;
    t.rowB = st + t.rB * rs;
    t.ddt = reinterpret_cast<const uint32_t*>(st + kRows * rs);
    t.hd_s = reinterpret_cast<const int8_t*>(st + hoff);
    t.hsc_s = reinterpret_cast<const float*>(st + hoff + kStageTok * 2 * I);
    t.hq_s = reinterpret_cast<const int32_t*>(st + hoff + kStageTok * (2 * I + hss * 4));

    const int tpg = (SINGLE || t.ne == 1) ? 1 : 2;
    const int ngroups = (t.ne + tpg - 1) / tpg;
    const int maxq = tpg == 1 ? 1 : 4;
    for (int pass0 = 0; pass0 < ngroups; pass0 += maxq) {
      if (SINGLE || tpg == 1) dn_tile<1, 1>(a, t, pass0);
      else dn_tile<2, 4>(a, t, pass0);
      __syncthreads();
      for (int i = tid; i < kRows * kTokMax; i += kThreads) {
        const int row = i & 63, tok = i >> 6;  // 64 rows x 8 assignments
        const int tglob = pass0 * tpg + tok;
        if (tok < maxq * tpg && tglob < t.ne) {
          const int rg = row >> 4, r16 = row & 15;
          const float v = red[(rg * 16 + r16) * kTokMax + tok] + red[((rg + 4) * 16 + r16) * kTokMax + tok];
          a.o[static_cast<size_t>(t.p0 + tglob) * H + r0 + row] = v;
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

int launch_down(const DownArgs& a0, int slots, int T, int sms, cudaStream_t st) {
  DownArgs a = a0;
  const size_t sb = stage_bytes(a.I);
  const size_t budget = 227 * 1024;
  int stages = static_cast<int>((budget - kFixed) / sb);
  stages = std::max(1, std::min(stages, 6));
  a.stages = stages;
  const size_t smem = stages * sb + kFixed;
  const int tiles = slots * (a.H / kRows);
  const int grid = std::max(1, std::min(tiles, sms));
  if (T == 1) {
    cudaFuncSetAttribute(down_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    down_kernel<true><<<grid, kThreads, smem, st>>>(a);
  } else {
    cudaFuncSetAttribute(down_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    down_kernel<false><<<grid, kThreads, smem, st>>>(a);
  }
  return cudaGetLastError() == cudaSuccess ? OK : ERR_CUDA;
}

}  // namespace moe
