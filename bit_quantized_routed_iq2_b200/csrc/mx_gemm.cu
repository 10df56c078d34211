// mx_gemm.cu - MXFP4 routed experts for many tokens: a grouped GEMM on the
// block-scaled 5th-generation tensor cores (tcgen05.mma kind::mxf8f6f4 with
// block_scale). The FP4 E2M1 weights and their E8M0 block scales are the M
// operand exactly as stored; the tokens routed to an expert are the N operand,
// their activations quantised to MXFP8 (E4M3 elements, one E8M0 scale per 32);
// accumulators are fp32 in TMEM.
//
// Sources: "ds4 : analyse pratique pour un usage documenté", section « Support
// de modèles et choix de quantification » (an MXFP4 file of the routed experts,
// run on CUDA with native FP4 matrix instructions on Blackwell for batched
// expert work); the formats are those of the OCP Microscaling Formats (MX)
// v1.0 specification (MXFP4 for the weights, MXFP8 E4M3 for the activations,
// both with 32-element blocks and E8M0 scales). The activation format is this
// library's reading: the block-scaled FP4 instruction needs an MX operand on
// both sides, and FP8 keeps the activations' rounding at 2^-4 relative.
//
// No dequantisation runs on the SMs: TMA brings the FP4 code bytes into shared
// memory in the unpacked layout the MMA reads (each 8 bytes of packed codes
// followed by 8 bytes of padding: 128 elements per 128-byte row), and the
// tensor core applies both operands' scales per 32-element block of K. Per CTA
// (one per SM, 224 threads):
//   warps 0-3  epilogue: TMEM -> registers; gate/up: SwiGLU, then h quantised
//              to MXFP8 (a warp holds 32 consecutive rows of one token, exactly
//              one block); down: fp32 expert outputs
//   warp 4     producer: TMA loads of the weight tiles (gate and up, or down)
//              and of the token tile, 128 elements of K per stage
//   warp 5     TMEM allocation; one lane copies the stage's scale factors into
//              TMEM (tcgen05.cp) and issues the MMAs
//   warp 6     scale builder: reads 16 scale bytes per row (four stages) of the
//              weight and token rows and writes, per stage, the 512-byte chunks
//              the scale copy takes (row r0 + 32 r1 of a 128-row chunk at byte
//              16 r0 + 4 r1, its four block scales in K order)
// Every wait is bounded: a time-out records MOE_ERR_TIMEOUT, all roles stop,
// and the CTA drains its in-flight copies and MMAs before freeing TMEM.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
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

constexpr int kMgThreads = 224;
constexpr int kMgEpiWarps = 4;  // warps 0-3
constexpr int kMgProdWarp = 4;
constexpr int kMgMmaWarp = 5;
constexpr int kMgSfWarp = 6;
constexpr int kMgMT = 128;  // weight rows per tile (MMA M)
constexpr int kMgNT = 112;  // max tokens per tile (MMA N): two buffers of gate+up accumulators fit in TMEM
constexpr int kMgKS = 128;  // K elements per stage
constexpr int kMgTile = 128 * 128;         // one 128-row x 128-byte shared-memory operand tile
constexpr uint32_t kMgFp4BoxTx = 128 * 64;  // bytes a 128 x 128 FP4 box moves (packed in global memory)
constexpr int kMgTmemCols = 512;
constexpr uint32_t kMgSfCol = 448;  // scale-factor columns: two sets of 16 above the accumulators

struct MgTile {
  int e, p0, n, pad;  // expert, first B row, rows of B used
};

struct MgArgs {
  int n_experts;  // experts the tiles may name
  int b_rows;     // rows of the B operand (assignments)
  int rows_e;     // weight rows per expert
  int K;          // reduction length
  int mt;         // 128-row tiles per expert
  const uint8_t* sa0;  // E8M0 scales of the weight rows [E * rows_e][K/32] (gate, or down)
  const uint8_t* sa1;  // up (pair kind)
  const uint8_t* sb;   // E8M0 scales of the B rows [b_rows][K/32]
  const MgTile* tiles;
  const int32_t* ntiles;
  void* out;     // pair: h E4M3 codes [b_rows][rows_e]; single: fp32 [b_rows][rows_e]
  uint8_t* osc;  // pair: h E8M0 scales [b_rows][rows_e / 32]
  int* err;
};

template <bool PAIR>
struct MgLayout {
  static constexpr int stages = PAIR ? 4 : 6;
  static constexpr size_t stage_bytes = (PAIR ? 3 : 2) * kMgTile;  // A tile(s), then the B tile
  static constexpr size_t b_off = (PAIR ? 2 : 1) * kMgTile;
  static constexpr size_t sf_off = stages * stage_bytes;
  static constexpr size_t sf_slot = (PAIR ? 3 : 2) * 512;  // scale chunks of one stage: A (gate, up), B
  static constexpr size_t bars = sf_off + stages * sf_slot;
  static constexpr size_t total = bars + 1024;
  static constexpr uint32_t acc_stride = PAIR ? 2 * kMgNT : kMgNT;  // TMEM columns per accumulator buffer
  static_assert(total <= 227 * 1024, "shared memory plan too large");
  static_assert(2 * acc_stride <= kMgSfCol, "accumulators overlap the scale-factor columns");
};

__device__ __forceinline__ bool mg_wait(uint64_t* bar, uint32_t parity, int* err, volatile int* abort_flag) {
  if (*abort_flag) return false;
  if (mbar_wait_bounded(bar, parity, err, ERR_TIMEOUT)) return true;
  *abort_flag = 1;
  return false;
}
__device__ __forceinline__ bool mg_wait_sleepy(uint64_t* bar, uint32_t parity, int* err, volatile int* abort_flag,
                                               unsigned max_ns) {
  if (*abort_flag) return false;
  if (mbar_wait_bounded_sleepy(bar, parity, err, ERR_TIMEOUT, max_ns)) return true;
  *abort_flag = 1;
  return false;
}
__device__ __forceinline__ bool mg_wait_warp(uint64_t* bar, uint32_t parity, int* err, volatile int* abort_flag) {
  const bool ok = mg_wait(bar, parity, err, abort_flag);
  return __all_sync(0xffffffffu, ok) != 0;
}

__device__ __forceinline__ bool mg_elect_one() {
  uint32_t p;
  asm volatile("{\n .reg .pred P;\n elect.sync _|P, 0xffffffff;\n selp.u32 %0, 1, 0, P;\n}\n" : "=r"(p));
  return p != 0;
}

__device__ __forceinline__ void sts128(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(x), "r"(y), "r"(z), "r"(w) : "memory");
}

__device__ __forceinline__ uint32_t word_of(const uint4& v, int q) {
  return q == 0 ? v.x : (q == 1 ? v.y : (q == 2 ? v.z : v.w));
}

// MXFP8 block exponent of a block whose largest magnitude has fp32 bits `amax_bits`:
// X = floor(log2 amax) - 8 (8 = the E4M3 emax), clamped to [-127, 127]; -127 for a zero
// block. A zero or subnormal amax has exponent field 0 and lands on the clamp.
__device__ __forceinline__ int mx8_exponent(uint32_t amax_bits) {
  const int ef = static_cast<int>(amax_bits >> 23);
  return max(-127, min(127, ef - 127 - 8));
}
// v * 2^-X (exact: 2^-X is a normal float for X in [-127, 126]) rounded to E4M3, nearest even, saturating.
__device__ __forceinline__ uint32_t mx8_code(float v, int X) {
  return static_cast<uint32_t>(
      __nv_cvt_float_to_fp8(v * __int_as_float((127 - X) << 23), __NV_SATFINITE, __NV_E4M3));
}

__device__ __forceinline__ float silu_mul(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }

__device__ __forceinline__ MgTile mg_tile(const MgArgs& a, int i) {
  MgTile t = a.tiles[i];
  if (t.e < 0 || t.e >= a.n_experts || t.p0 < 0 || t.n < 1 || t.n > kMgNT || t.p0 + t.n > a.b_rows) {
    if (a.err) atomicCAS(a.err, 0, ERR_ARG);
    t.n = 0;
  }
  return t;
}

template <bool PAIR>
__global__ void __launch_bounds__(kMgThreads, 1) mx_gemm_kernel(const __grid_constant__ CUtensorMap tm_b,
                                                                const __grid_constant__ CUtensorMap tm_a0,
                                                                const __grid_constant__ CUtensorMap tm_a1,
                                                                MgArgs a) {
  using L = MgLayout<PAIR>;
  constexpr int kStages = L::stages;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint64_t* fullB = reinterpret_cast<uint64_t*>(smem + L::bars);  // operand tiles landed
  uint64_t* emptyB = fullB + kStages;                             // stage free again (MMA commit)
  uint64_t* sfF = emptyB + kStages;                               // scale chunks of the stage written
  uint64_t* accf = sfF + kStages;                                 // [2] accumulator buffer complete
  uint64_t* acce = accf + 2;                                      // [2] accumulator buffer read out
  uint64_t* drain = acce + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t sbase = smem_addr(smem);

  if ((sbase & 1023u) != 0) {  // the swizzled tiles need 1024-byte alignment
    if (tid == 0) atomicCAS(a.err, 0, ERR_CUDA);
    return;
  }
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&fullB[s], 1);
      mbar_init(&emptyB[s], 1);
      mbar_init(&sfF[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accf[b], 1);
      mbar_init(&acce[b], kMgEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMgMmaWarp) {
    tmem_alloc(tmem_slot, kMgTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int nunits = *a.ntiles * a.mt;
  const int nks = a.K / kMgKS;

  if (warp == kMgProdWarp) {
    if (lane == 0) {
      prefetch_tmap(&tm_b);
      prefetch_tmap(&tm_a0);
      if (PAIR) prefetch_tmap(&tm_a1);
      int s = 0, issued = 0;
      uint32_t ph = 0;
      for (int u = blockIdx.x; u < nunits && !*abort_flag; u += gridDim.x) {
        const MgTile t = mg_tile(a, u / a.mt);
        if (t.n == 0) continue;
        const int wrow = t.e * a.rows_e + (u % a.mt) * kMgMT;
        for (int ks = 0; ks < nks; ++ks) {
          if (!mg_wait_sleepy(&emptyB[s], ph ^ 1u, a.err, abort_flag, 256)) break;  // the ring runs ahead
          uint8_t* st = smem + s * L::stage_bytes;
          mbar_arrive_expect_tx(&fullB[s], (PAIR ? 2 : 1) * kMgFp4BoxTx + kMgTile);
          tma_load_2d(st, &tm_a0, ks * kMgKS, wrow, &fullB[s]);
          if (PAIR) tma_load_2d(st + kMgTile, &tm_a1, ks * kMgKS, wrow, &fullB[s]);
          tma_load_2d(st + L::b_off, &tm_b, ks * kMgKS, t.p0, &fullB[s]);
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
  } else if (warp == kMgSfWarp) {
    // per 512 elements of K, 16 scale bytes of each row: rows r0 + 32 r1 of the weight tile (and of the
    // token tile) for this lane r0, then per stage q of the four the 32-bit word q of each. The next
    // 512 elements' bytes (of this tile or of the CTA's next one) are loaded before this one's are written.
    const size_t ldk = static_cast<size_t>(a.K / 32);
    const int nsup = a.K / (4 * kMgKS);
    auto next_unit = [&](int uu) {
      while (uu < nunits && mg_tile(a, uu / a.mt).n == 0) uu += gridDim.x;
      return uu;
    };
    auto load_sup = [&](int uu, int j, uint4 (&ga)[4], uint4 (&ua)[4], uint4 (&gb)[4]) {
      const MgTile t = a.tiles[uu / a.mt];  // validated by next_unit
      const size_t wrow = static_cast<size_t>(t.e) * a.rows_e + (uu % a.mt) * kMgMT + lane;
#pragma unroll
      for (int r1 = 0; r1 < 4; ++r1) {
        ga[r1] = __ldg(reinterpret_cast<const uint4*>(a.sa0 + (wrow + 32 * r1) * ldk) + j);
        if (PAIR) ua[r1] = __ldg(reinterpret_cast<const uint4*>(a.sa1 + (wrow + 32 * r1) * ldk) + j);
        const int brow = min(t.p0 + lane + 32 * r1, a.b_rows - 1);  // rows past the tile: any valid row
        gb[r1] = __ldg(reinterpret_cast<const uint4*>(a.sb + static_cast<size_t>(brow) * ldk) + j);
      }
    };
    int s = 0;
    uint32_t ph = 0;
    int u = next_unit(blockIdx.x), j = 0;
    uint4 ga[4], ua[4], gb[4];
    if (u < nunits) load_sup(u, 0, ga, ua, gb);
    bool ok = true;
    while (u < nunits && ok) {
      int un = u, jn = j + 1;
      if (jn == nsup) {
        jn = 0;
        un = next_unit(u + gridDim.x);
      }
      uint4 na[4], nu[4], nb[4];
      if (un < nunits) load_sup(un, jn, na, nu, nb);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (!mg_wait_warp(&emptyB[s], ph ^ 1u, a.err, abort_flag)) {
          ok = false;
          break;
        }
        const uint32_t ch = sbase + L::sf_off + s * L::sf_slot + 16 * lane;
        sts128(ch, word_of(ga[0], q), word_of(ga[1], q), word_of(ga[2], q), word_of(ga[3], q));
        if (PAIR) sts128(ch + 512, word_of(ua[0], q), word_of(ua[1], q), word_of(ua[2], q), word_of(ua[3], q));
        sts128(ch + (PAIR ? 1024 : 512), word_of(gb[0], q), word_of(gb[1], q), word_of(gb[2], q),
               word_of(gb[3], q));
        fence_proxy_async_smem();  // the chunks are read by the tensor core's copy
        __syncwarp();
        if (lane == 0) mbar_arrive(&sfF[s]);
        if (++s == kStages) { s = 0; ph ^= 1u; }
      }
#pragma unroll
      for (int r1 = 0; r1 < 4; ++r1) {
        ga[r1] = na[r1];
        if (PAIR) ua[r1] = nu[r1];
        gb[r1] = nb[r1];
      }
      u = un;
      j = jn;
    }
  } else if (warp == kMgMmaWarp) {
    // the whole warp runs the loop (waits stay warp-uniform); one elected lane copies and issues
    const uint32_t idesc0 = umma_idesc_mx_e2m1_e4m3(kMgMT, 16);
    int s = 0, t = 0;
    uint32_t ph = 0;
    for (int u = blockIdx.x; u < nunits && !__any_sync(0xffffffffu, *abort_flag != 0); u += gridDim.x) {
      const MgTile tl = mg_tile(a, u / a.mt);
      if (tl.n == 0) continue;
      const int n16 = (tl.n + 15) & ~15;
      const uint32_t idn = (idesc0 & ~(0x3Fu << 17)) | (static_cast<uint32_t>(n16 >> 3) << 17);
      const int buf = t & 1;
      if (!mg_wait_warp(&acce[buf], ((t >> 1) & 1) ^ 1u, a.err, abort_flag)) break;
      tc_fence_after();
      const uint32_t d0 = tmem + buf * L::acc_stride, d1 = d0 + kMgNT;
      bool ok = true;
      for (int ks = 0; ks < nks; ++ks) {
        if (!mg_wait_warp(&fullB[s], ph, a.err, abort_flag) || !mg_wait_warp(&sfF[s], ph, a.err, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t st = sbase + s * L::stage_bytes;
        const uint32_t ch = sbase + L::sf_off + s * L::sf_slot;
        const uint32_t sfa0 = tmem + kMgSfCol + 16 * (s & 1), sfa1 = sfa0 + 4, sfb = sfa0 + (PAIR ? 8 : 4);
        if (mg_elect_one()) {
          tmem_cp_32x128_x4(sfa0, umma_desc_rows16(ch));
          if (PAIR) tmem_cp_32x128_x4(sfa1, umma_desc_rows16(ch + 512));
          tmem_cp_32x128_x4(sfb, umma_desc_rows16(ch + (PAIR ? 1024 : 512)));
          const uint64_t da0 = umma_desc_sw128(st), da1 = umma_desc_sw128(st + kMgTile);
          const uint64_t db = umma_desc_sw128(st + L::b_off);
#pragma unroll
          for (uint32_t kk = 0; kk < kMgKS / 32; ++kk) {  // 32 elements = 32 bytes of each tile per step
            const uint32_t acc = (ks | kk) ? 1u : 0u;
            const uint32_t id = umma_idesc_sf_ids(idn, kk, kk);
            umma_mx(d0, da0 + 2 * kk, db + 2 * kk, id, sfa0 | (kk << 30), sfb | (kk << 30), acc);
            if (PAIR) umma_mx(d1, da1 + 2 * kk, db + 2 * kk, id, sfa1 | (kk << 30), sfb | (kk << 30), acc);
          }
          umma_commit(&emptyB[s]);
        }
        __syncwarp();
        if (++s == kStages) { s = 0; ph ^= 1u; }
      }
      if (!ok) break;
      if (mg_elect_one()) umma_commit(&accf[buf]);
      __syncwarp();
      ++t;
    }
    // drain: every MMA issued by this warp completes before TMEM is freed
    if (mg_elect_one()) umma_commit(drain);
    __syncwarp();
    mbar_wait_bounded(drain, 0, nullptr, 0);
  } else if (warp < kMgEpiWarps) {
    int t = 0;
    for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
      const MgTile tl = mg_tile(a, u / a.mt);
      if (tl.n == 0) continue;
      const int buf = t & 1;
      const bool got = mg_wait_sleepy(&accf[buf], (t >> 1) & 1, a.err, abort_flag, 1024);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const uint32_t tb = tmem + buf * L::acc_stride + (static_cast<uint32_t>(32 * warp) << 16);
      const int row0 = (u % a.mt) * kMgMT + 32 * warp;  // this warp's 32 rows: one MX block of h
      const int row = row0 + lane;
      for (int c0 = 0; c0 < tl.n; c0 += 16) {
        uint32_t g[16], v[16];
        tmem_ld16(tb + c0, g);
        if (PAIR) tmem_ld16(tb + kMgNT + c0, v);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int n = c0 + j;
          if (n >= tl.n) break;
          const size_t p = static_cast<size_t>(tl.p0 + n);
          if (PAIR) {
            const float h = silu_mul(__uint_as_float(g[j]), __uint_as_float(v[j]));
            const int X = mx8_exponent(__reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(h))));
            static_cast<uint8_t*>(a.out)[p * a.rows_e + row] = static_cast<uint8_t>(mx8_code(h, X));
            if (lane == 0) a.osc[p * (a.rows_e / 32) + row0 / 32] = static_cast<uint8_t>(X + 127);
          } else {
            static_cast<float*>(a.out)[p * a.rows_e + row] = __uint_as_float(g[j]);
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
  if (warp == kMgMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kMgTmemCols);
  }
}

// The routed B operand: each assignment's activations (expert-sorted by the
// permutation) as MXFP8, E4M3 codes [nA][H] and E8M0 scales [nA][H/32]; and
// the tile list (expert, first assignment, count) of up to kMgNT assignments.
// Block 0 also clears the call's status word.
template <typename XT>
__global__ void __launch_bounds__(256) mx8_prep_kernel(const XT* __restrict__ x, int T, int H, int k,
                                                       const int32_t* __restrict__ perm, uint8_t* __restrict__ xq,
                                                       uint8_t* __restrict__ xsc, const int32_t* __restrict__ offsets,
                                                       const int32_t* __restrict__ active, int E,
                                                       MgTile* __restrict__ tiles, int32_t* __restrict__ ntiles,
                                                       int* __restrict__ err_word) {
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
      const int nt = (ne + kMgNT - 1) / kMgNT;
      int incl = nt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      for (int j = 0; j < nt; ++j) {
        MgTile tl;
        tl.e = e;
        tl.p0 = p0 + j * kMgNT;
        tl.n = min(kMgNT, ne - j * kMgNT);
        tl.pad = 0;
        tiles[base + incl - nt + j] = tl;
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) *ntiles = base;
  }
  const int nb = H / 32;
  const size_t nblk = static_cast<size_t>(nA) * nb;
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nblk;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int p = static_cast<int>(i / nb), b = static_cast<int>(i % nb);
    const size_t src = static_cast<size_t>(perm[p] / k) * H + 32 * b;
    float v[32];
    if constexpr (sizeof(XT) == 4) {
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float4 f = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(x) + src + 4 * q);
        v[4 * q] = f.x; v[4 * q + 1] = f.y; v[4 * q + 2] = f.z; v[4 * q + 3] = f.w;
      }
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 w = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(x) + src + 8 * q);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          v[8 * q + 2 * r] = __uint_as_float(ws[r] << 16);
          v[8 * q + 2 * r + 1] = __uint_as_float(ws[r] & 0xFFFF0000u);
        }
      }
    }
    float m = 0.f;
#pragma unroll
    for (int q = 0; q < 32; ++q) m = fmaxf(m, fabsf(v[q]));
    const int X = mx8_exponent(__float_as_uint(m));
    uint32_t wds[8];
#pragma unroll
    for (int q = 0; q < 8; ++q)
      wds[q] = mx8_code(v[4 * q], X) | (mx8_code(v[4 * q + 1], X) << 8) | (mx8_code(v[4 * q + 2], X) << 16) |
               (mx8_code(v[4 * q + 3], X) << 24);
    uint4* dst = reinterpret_cast<uint4*>(xq + static_cast<size_t>(p) * H + 32 * b);
    dst[0] = make_uint4(wds[0], wds[1], wds[2], wds[3]);
    dst[1] = make_uint4(wds[4], wds[5], wds[6], wds[7]);
    xsc[static_cast<size_t>(p) * nb + b] = static_cast<uint8_t>(X + 127);
  }
}

// y[t][h] = sum_j w[t][j] o[inv[t*k+j]][h] (j ascending) + s[t][h] (+ residual).
__global__ void __launch_bounds__(256) mx_combine_kernel(int T, int H, int k, const float* __restrict__ topk_w,
                                                         const int32_t* __restrict__ inv, const float* __restrict__ o,
                                                         const float* s, const float* residual, float* y) {
  const size_t n4 = static_cast<size_t>(T) * H / 4;
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int t = static_cast<int>((i * 4) / H), h = static_cast<int>((i * 4) % H);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
      const float w = topk_w[t * k + j];
      const float4 v = *reinterpret_cast<const float4*>(o + static_cast<size_t>(inv[t * k + j]) * H + h);
      acc.x = fmaf(w, v.x, acc.x);
      acc.y = fmaf(w, v.y, acc.y);
      acc.z = fmaf(w, v.z, acc.z);
      acc.w = fmaf(w, v.w, acc.w);
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

PFN_cuTensorMapEncodeTiled_v12000 mg_encode_fn() {
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

// FP4 codes [rows][K/2] bytes as K 4-bit elements per row, boxes of 128 elements x 128 rows landing
// unpacked (8 bytes of codes, 8 bytes of padding) in 128-byte swizzled rows. The base must be 32-byte
// aligned and the row pitch K/2 a multiple of 32.
bool fp4_map(CUtensorMap* m, const void* base, uint64_t K, uint64_t rows) {
  auto fn = mg_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {K, rows};
  const cuuint64_t strides[1] = {K / 2};
  const cuuint32_t box[2] = {128, 128};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// E4M3 codes [rows][K] bytes, boxes of 128 bytes x 128 rows, 128-byte swizzle.
bool e4m3_map(CUtensorMap* m, const void* base, uint64_t K, uint64_t rows) {
  auto fn = mg_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {K, rows};
  const cuuint64_t strides[1] = {K};
  const cuuint32_t box[2] = {128, 128};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool PAIR>
int launch_mg(const CUtensorMap& mb, const CUtensorMap& ma0, const CUtensorMap& ma1, const MgArgs& a, int sms,
              cudaStream_t st) {
  const size_t smem = MgLayout<PAIR>::total;
  cudaFuncSetAttribute(mx_gemm_kernel<PAIR>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  mx_gemm_kernel<PAIR><<<sms, kMgThreads, smem, st>>>(mb, ma0, ma1, a);
  return cudaGetLastError() == cudaSuccess ? OK : ERR_CUDA;
}

struct MgWs {
  uint8_t* xq;   // [nA][H] E4M3
  uint8_t* xsc;  // [nA][H/32]
  uint8_t* hq;   // [nA][I]
  uint8_t* hsc;  // [nA][I/32]
  float* o;      // [nA][H]
  float* s;      // [T][H] shared expert
  MgTile* tiles;
  int32_t* ntiles;
  void* shared_ws;
  size_t bytes;
};

MgWs carve_mg(const LayerShape& sh, int T, char* base) {
  const size_t nA = static_cast<size_t>(T) * sh.k;
  MgWs w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* q = base ? base + off : nullptr;
    off += align_up(bytes > 0 ? bytes : 1, 1024);
    return q;
  };
  w.xq = reinterpret_cast<uint8_t*>(take(nA * sh.H));
  w.xsc = reinterpret_cast<uint8_t*>(take(nA * sh.H / 32));
  w.hq = reinterpret_cast<uint8_t*>(take(nA * sh.I));
  w.hsc = reinterpret_cast<uint8_t*>(take(nA * sh.I / 32));
  w.o = reinterpret_cast<float*>(take(nA * sh.H * 4));
  w.s = reinterpret_cast<float*>(take(static_cast<size_t>(T) * sh.H * 4));
  w.tiles = reinterpret_cast<MgTile*>(take((static_cast<size_t>(sh.E) + nA / kMgNT + 1) * sizeof(MgTile)));
  w.ntiles = reinterpret_cast<int32_t*>(take(64));
  w.shared_ws = take(sh.Is > 0 ? prefill_shared_workspace_bytes(sh, T) : 0);
  w.bytes = off;
  return w;
}

}  // namespace

bool mx_prefill_supported(const LayerShape& s, int T) {
  if (T <= kPrefillMinT || s.H % 512 != 0 || s.I % 512 != 0) return false;
  if (static_cast<long long>(s.E) * std::max(s.H, s.I) >= (1ll << 31)) return false;
  if (static_cast<long long>(T) * s.k >= (1ll << 31) / std::max(s.H, s.I)) return false;
  if (s.Is > 0 && (s.Is % 128 != 0 || s.Is % 64 != 0)) return false;
  return mg_encode_fn() != nullptr;
}

size_t mx_prefill_workspace_bytes(const LayerShape& s, int T) { return carve_mg(s, T, nullptr).bytes; }

int launch_ffn_mx_prefill(const LayerShape& sh, const WeightPtrs& shw, const MxPlanes& w, const void* x, int x_dtype,
                          int T, const Routing& r, const float* residual, float* y, void* ws, int* err,
                          bool clear_status, int sms, cudaStream_t st) {
  if (w.fmt != 0) return ERR_SHAPE;  // the block-scaled instruction takes MXFP4; Q4-style blocks stop at 16 tokens
  const void* codes[] = {w.gate_codes, w.up_codes, w.down_codes};
  for (const void* c : codes)
    if (reinterpret_cast<uintptr_t>(c) % 32 != 0) return ERR_ARG;  // the unpacking TMA copy needs 32-byte bases
  const MgWs mw = carve_mg(sh, T, static_cast<char*>(ws));
  const int nA = T * sh.k;
  int rc = OK;
  {
    ProfScope ps(MOE_K_PREP, st);
    const int grid = std::max(1, std::min(sms * 4, (nA * (sh.H / 32) + 255) / 256));
    if (x_dtype == 0)
      mx8_prep_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float*>(x), T, sh.H, sh.k, r.perm, mw.xq, mw.xsc,
                                                   r.offsets, r.active, sh.E, mw.tiles, mw.ntiles,
                                                   clear_status ? err : nullptr);
    else
      mx8_prep_kernel<uint16_t><<<grid, 256, 0, st>>>(static_cast<const uint16_t*>(x), T, sh.H, sh.k, r.perm, mw.xq,
                                                      mw.xsc, r.offsets, r.active, sh.E, mw.tiles, mw.ntiles,
                                                      clear_status ? err : nullptr);
  }
  if (sh.Is > 0)
    rc |= launch_prefill_shared(sh, shw.sh_gate, shw.sh_up, shw.sh_down, x, x_dtype, T, mw.shared_ws, mw.s, err, sms,
                                st);
  CUtensorMap mb, ma0, ma1;
  {
    ProfScope ps(MOE_K_PREFILL_GATEUP, st);
    const uint64_t wrows = static_cast<uint64_t>(sh.E) * sh.I;
    if (!e4m3_map(&mb, mw.xq, sh.H, nA) || !fp4_map(&ma0, w.gate_codes, sh.H, wrows) ||
        !fp4_map(&ma1, w.up_codes, sh.H, wrows))
      return ERR_CUDA;
    MgArgs a{};
    a.n_experts = sh.E; a.b_rows = nA; a.rows_e = sh.I; a.K = sh.H; a.mt = sh.I / kMgMT;
    a.sa0 = static_cast<const uint8_t*>(w.gate_scales);
    a.sa1 = static_cast<const uint8_t*>(w.up_scales);
    a.sb = mw.xsc;
    a.tiles = mw.tiles; a.ntiles = mw.ntiles;
    a.out = mw.hq; a.osc = mw.hsc; a.err = err;
    rc |= launch_mg<true>(mb, ma0, ma1, a, sms, st);
  }
  {
    ProfScope ps(MOE_K_PREFILL_DOWN, st);
    if (!e4m3_map(&mb, mw.hq, sh.I, nA) ||
        !fp4_map(&ma0, w.down_codes, sh.I, static_cast<uint64_t>(sh.E) * sh.H))
      return ERR_CUDA;
    MgArgs a{};
    a.n_experts = sh.E; a.b_rows = nA; a.rows_e = sh.H; a.K = sh.I; a.mt = sh.H / kMgMT;
    a.sa0 = static_cast<const uint8_t*>(w.down_scales);
    a.sb = mw.hsc;
    a.tiles = mw.tiles; a.ntiles = mw.ntiles;
    a.out = mw.o; a.err = err;
    rc |= launch_mg<false>(mb, ma0, ma0, a, sms, st);
  }
  {
    ProfScope ps(MOE_K_COMBINE, st);
    const int grid = std::max(1, std::min(sms * 8, static_cast<int>((static_cast<size_t>(T) * sh.H / 4 + 255) / 256)));
    mx_combine_kernel<<<grid, 256, 0, st>>>(T, sh.H, sh.k, r.topk_w, r.inv, mw.o, sh.Is > 0 ? mw.s : nullptr,
                                            residual, y);
  }
  if (rc != OK) return ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? OK : ERR_CUDA;
}

}  // namespace moe
