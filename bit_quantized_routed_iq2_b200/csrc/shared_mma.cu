// shared_mma.cu - the unquantized shared expert for up to 32 tokens on bf16
// warp MMAs (m16n8k16, fp32 accumulation), and the weighted combine fused into
// the epilogue of its down projection.
//
// Source: "ds4 : analyse pratique pour un usage documenté", section « Support de
// modèles et choix de quantification » (the shared expert stays unquantized).
// The combine is the library's specification: y[t] = sum_j w[t][j] o[(t,j)]
// (j ascending) + s[t] (+ residual[t]).
//
// Layout of the work: a CTA owns 16 weight rows and KS warps split the
// reduction axis K; every warp streams its slice of the 16 rows with 16-byte
// loads (two steps of 32 columns in flight) and multiplies them by the
// activations as MMA B columns. One 16-byte load of a row feeds two MMAs: the
// K order inside a 32-column step is permuted identically for A and B (thread
// tig holds physical columns 8*tig .. 8*tig+7), which leaves the dot products
// unchanged. The KS partial tiles are added in warp order in shared memory.
//
// B columns are (token, part): bf16 activations are one part; fp32 values are
// split exactly enough into two bf16 parts (hi = rn(v), lo = rn(v - hi)) whose
// columns are added after the MMA, so the products keep ~16 mantissa bits.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace moe {
namespace {

__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 ldg16(const uint16_t* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }

__device__ __forceinline__ float silu_mul_f(float g, float u) { return g / (1.0f + expf(-g)) * u; }

__device__ __forceinline__ uint16_t bf16_rn_bits(float v) { return __bfloat16_as_ushort(__float2bfloat16_rn(v)); }
__device__ __forceinline__ float bf16_bits_f(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }

constexpr int kRows = 16;

// Accumulate D[r][c] += sum_{k in [kbeg, kend)} W_m[r0 + r][k] * B[c][k] for
// NM weight matrices sharing the B columns. B column c of group q is
// (token, part) = ((8q + c) / P, (8q + c) % P).
template <int NM, int NG, int U = (NG == 1 ? 4 : 2)>
__device__ __forceinline__ void skinny_mainloop(const uint16_t* const (&W)[NM], int K, int r0, const uint16_t* xb,
                                                int P, int T, int kbeg, int kend, float (&acc)[NM][NG][4]) {
  const int lane = threadIdx.x & 31, g = lane >> 2, tig = lane & 3;
  const uint16_t* arow[NM][2];
#pragma unroll
  for (int m = 0; m < NM; ++m) {
    arow[m][0] = W[m] + static_cast<size_t>(r0 + g) * K + 8 * tig;
    arow[m][1] = W[m] + static_cast<size_t>(r0 + g + 8) * K + 8 * tig;
  }
  const uint16_t* brow[NG];
  bool bval[NG];
#pragma unroll
  for (int q = 0; q < NG; ++q) {
    const int col = 8 * q + g, tok = col / P, part = col - tok * P;
    bval[q] = tok < T;
    brow[q] = xb + (static_cast<size_t>(part) * T + (bval[q] ? tok : 0)) * K + 8 * tig;
  }
#pragma unroll
  for (int m = 0; m < NM; ++m)
#pragma unroll
    for (int q = 0; q < NG; ++q) acc[m][q][0] = acc[m][q][1] = acc[m][q][2] = acc[m][q][3] = 0.f;
  // U steps of 32 columns in flight per warp
  for (int k0 = kbeg; k0 < kend; k0 += 32 * U) {
    uint4 av[U][NM][2];
    uint4 bv[U][NG];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int k = k0 + 32 * u;
      const bool in = k < kend;
#pragma unroll
      for (int m = 0; m < NM; ++m) {
        av[u][m][0] = in ? ldg16(arow[m][0] + k) : make_uint4(0, 0, 0, 0);
        av[u][m][1] = in ? ldg16(arow[m][1] + k) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int q = 0; q < NG; ++q) bv[u][q] = (in && bval[q]) ? ldg16(brow[q] + k) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int m = 0; m < NM; ++m)
#pragma unroll
        for (int q = 0; q < NG; ++q) {
          mma_bf16(acc[m][q], av[u][m][0].x, av[u][m][1].x, av[u][m][0].y, av[u][m][1].y, bv[u][q].x, bv[u][q].y);
          mma_bf16(acc[m][q], av[u][m][0].z, av[u][m][1].z, av[u][m][0].w, av[u][m][1].w, bv[u][q].z, bv[u][q].w);
        }
  }
}

// The same for a warp whose K slice is exactly one step of 32 * U columns, in
// two halves: skinny_load_a fetches the weight slice (constants of the layer),
// skinny_finish loads the B columns and multiplies. A kernel can issue the
// first half before it waits for the kernels that produce B.
template <int NM, int U>
__device__ __forceinline__ void skinny_load_a(const uint16_t* const (&W)[NM], int K, int r0, int kbeg,
                                              uint4 (&av)[U][NM][2]) {
  const int lane = threadIdx.x & 31, g = lane >> 2, tig = lane & 3;
#pragma unroll
  for (int m = 0; m < NM; ++m) {
    const uint16_t* a0 = W[m] + static_cast<size_t>(r0 + g) * K + 8 * tig + kbeg;
    const uint16_t* a1 = W[m] + static_cast<size_t>(r0 + g + 8) * K + 8 * tig + kbeg;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      av[u][m][0] = ldg16(a0 + 32 * u);
      av[u][m][1] = ldg16(a1 + 32 * u);
    }
  }
}

template <int NM, int NG, int U>
__device__ __forceinline__ void skinny_finish(const uint4 (&av)[U][NM][2], int K, const uint16_t* xb, int P, int T,
                                              int kbeg, float (&acc)[NM][NG][4]) {
  const int lane = threadIdx.x & 31, g = lane >> 2, tig = lane & 3;
  uint4 bv[U][NG];
#pragma unroll
  for (int q = 0; q < NG; ++q) {
    const int col = 8 * q + g, tok = col / P, part = col - tok * P;
    const uint16_t* brow = xb + (static_cast<size_t>(part) * T + (tok < T ? tok : 0)) * K + 8 * tig + kbeg;
#pragma unroll
    for (int u = 0; u < U; ++u) bv[u][q] = tok < T ? ldg16(brow + 32 * u) : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int m = 0; m < NM; ++m)
#pragma unroll
    for (int q = 0; q < NG; ++q) acc[m][q][0] = acc[m][q][1] = acc[m][q][2] = acc[m][q][3] = 0.f;
#pragma unroll
  for (int u = 0; u < U; ++u)
#pragma unroll
    for (int m = 0; m < NM; ++m)
#pragma unroll
      for (int q = 0; q < NG; ++q) {
        mma_bf16(acc[m][q], av[u][m][0].x, av[u][m][1].x, av[u][m][0].y, av[u][m][1].y, bv[u][q].x, bv[u][q].y);
        mma_bf16(acc[m][q], av[u][m][0].z, av[u][m][1].z, av[u][m][0].w, av[u][m][1].w, bv[u][q].z, bv[u][q].w);
      }
}

// Store a warp's partial tiles: red[warp][m][col][row].
template <int NM, int NG>
__device__ __forceinline__ void skinny_store(float* red, const float (&acc)[NM][NG][4]) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tig = lane & 3;
  float* base = red + static_cast<size_t>(warp) * NM * NG * 8 * kRows;
#pragma unroll
  for (int m = 0; m < NM; ++m)
#pragma unroll
    for (int q = 0; q < NG; ++q) {
      float* p = base + (m * NG * 8 + 8 * q + 2 * tig) * kRows;
      p[g] = acc[m][q][0];
      p[kRows + g] = acc[m][q][1];
      p[g + 8] = acc[m][q][2];
      p[kRows + g + 8] = acc[m][q][3];
    }
}

// Sum over warps (in order) and parts of matrix m, row r, token t.
template <int NM, int NG>
__device__ __forceinline__ float skinny_value(const float* red, int KS, int m, int r, int t, int P) {
  float v = 0.f;
  for (int part = 0; part < P; ++part) {
    const int col = t * P + part;
    float s = 0.f;
    for (int w = 0; w < KS; ++w) s += red[(static_cast<size_t>(w) * NM * NG * 8 + m * NG * 8 + col) * kRows + r];
    v += s;
  }
  return v;
}

template <int NG>
constexpr int ks_max() {
  return NG <= 2 ? 16 : (NG == 4 ? 8 : 4);
}

// h = silu(Wg x) * (Wu x) for 16 rows per CTA; written as two bf16 parts
// hb[part][t][Is] for the down projection (and as fp32 when hs is given).
template <int NG>
__global__ void __launch_bounds__(512) shared_gateup_mma_kernel(int H, int Is, const uint16_t* __restrict__ wg,
                                                                const uint16_t* __restrict__ wu,
                                                                const uint16_t* __restrict__ xb, int P, int T,
                                                                int KS, uint16_t* __restrict__ hb) {
  __shared__ __align__(16) float red[ks_max<NG>() * 2 * NG * 8 * kRows];
  const int warp = threadIdx.x >> 5;
  const int r0 = blockIdx.x * kRows;
  const int span = H / KS;
  float acc[2][NG][4];
  const uint16_t* const W[2] = {wg, wu};
  skinny_mainloop<2, NG>(W, H, r0, xb, P, T, warp * span, (warp + 1) * span, acc);
  skinny_store<2, NG>(red, acc);
  __syncthreads();
  for (int i = threadIdx.x; i < kRows * T; i += blockDim.x) {
    const int r = i % kRows, t = i / kRows;
    const float gv = skinny_value<2, NG>(red, KS, 0, r, t, P);
    const float uv = skinny_value<2, NG>(red, KS, 1, r, t, P);
    const float h = silu_mul_f(gv, uv);
    const uint16_t hi = bf16_rn_bits(h);
    const uint16_t lo = bf16_rn_bits(h - bf16_bits_f(hi));
    hb[static_cast<size_t>(t) * Is + r0 + r] = hi;
    hb[(static_cast<size_t>(T) + t) * Is + r0 + r] = lo;
  }
}

// y[t][r] = sum_j w[t][j] sum_dp o[inv[t*k+j]][dp][r] + (Wsd h_t)[r] (+ residual),
// 16 rows of H per CTA; h arrives as two bf16 parts. After the weight stream,
// all threads gather the routed partial rows (one (row, token, slot) each,
// parts added in order; the first slot index is loaded before the stream) into
// shared memory; each output then adds its k slots in slot order.
template <int NG>
__global__ void __launch_bounds__(512) shared_down_combine_mma_kernel(
    int H, int Is, const uint16_t* __restrict__ wd, const uint16_t* __restrict__ hb, int T, int KS, int k,
    const float* __restrict__ topk_w, const int32_t* __restrict__ inv, const float* __restrict__ obuf, int DP,
    const float* residual, float* y) {
  __shared__ __align__(16) float red[ks_max<NG>() * NG * 8 * kRows];
  extern __shared__ float osum[];  // [T*k][kRows]
  constexpr int U = NG == 1 ? 4 : 2;
  pdl_trigger();
  const int warp = threadIdx.x >> 5;
  const int r0 = blockIdx.x * kRows;
  const int nitems = kRows * T * k;
  const int span = Is / KS;
  float acc[1][NG][4];
  const uint16_t* const W[1] = {wd};
  if (span == 32 * U) {
    // the weight slice is a constant of the layer: it streams in while the kernels before this one finish
    uint4 av[U][1][2];
    skinny_load_a<1, U>(W, Is, r0, warp * span, av);
    pdl_wait();  // h, the routed partials and the routing come from the kernels before this one
    skinny_finish<1, NG, U>(av, Is, hb, 2, T, warp * span, acc);
  } else {
    pdl_wait();
    skinny_mainloop<1, NG>(W, Is, r0, hb, 2, T, warp * span, (warp + 1) * span, acc);
  }
  // the assignment rows of this thread's first gather item
  const int a0 = threadIdx.x < nitems ? inv[threadIdx.x / kRows] : 0;
  skinny_store<1, NG>(red, acc);
  for (int i = threadIdx.x; i < nitems; i += blockDim.x) {
    const int r = i % kRows, a = i / kRows;
    const float* o = obuf + static_cast<size_t>(i < static_cast<int>(blockDim.x) ? a0 : inv[a]) * DP * H + r0 + r;
    float sacc = 0.f;
    for (int dp = 0; dp < DP; ++dp) sacc += o[static_cast<size_t>(dp) * H];
    osum[i] = sacc;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kRows * T; i += blockDim.x) {
    const int r = i % kRows, t = i / kRows;
    const int row = r0 + r;
    float v = 0.f;
    for (int j = 0; j < k; ++j) v = fmaf(topk_w[t * k + j], osum[(t * k + j) * kRows + r], v);
    v += skinny_value<1, NG>(red, KS, 0, r, t, 2);
    if (residual) v += residual[static_cast<size_t>(t) * H + row];
    y[static_cast<size_t>(t) * H + row] = v;
  }
}

int pick_ks(int K, int ksmax) {
  for (int ks = ksmax; ks >= 1; ks >>= 1)
    if (K % (32 * ks) == 0) return ks;
  return 0;
}

int groups_for(int cols) { return cols <= 8 ? 1 : cols <= 16 ? 2 : cols <= 32 ? 4 : cols <= 64 ? 8 : 0; }

int ksmax_for(int ng) { return ng <= 2 ? 16 : (ng == 4 ? 8 : 4); }

}  // namespace

bool shared_mma_supported(int H, int Is, int T, int x_parts, int k) {
  if (Is <= 0 || H % kRows != 0 || Is % kRows != 0 || T < 1) return false;
  if (static_cast<size_t>(kRows) * T * k * sizeof(float) > 48 * 1024 - 16 * 1024) return false;
  const int ng_gu = groups_for(T * x_parts), ng_dn = groups_for(2 * T);
  if (ng_gu == 0 || ng_gu > 4 || ng_dn == 0) return false;
  return pick_ks(H, ksmax_for(ng_gu)) > 0 && pick_ks(Is, ksmax_for(ng_dn)) > 0;
}

int launch_shared_gateup_mma(int H, int Is, const uint16_t* wg, const uint16_t* wu, const uint16_t* xb, int P,
                             int T, uint16_t* hb, cudaStream_t st) {
  const int ng = groups_for(T * P);
  const int ks = pick_ks(H, ksmax_for(ng));
  if (ks == 0) return ERR_SHAPE;
  const dim3 grid(Is / kRows), block(32 * ks);
  switch (ng) {
    case 1: shared_gateup_mma_kernel<1><<<grid, block, 0, st>>>(H, Is, wg, wu, xb, P, T, ks, hb); break;
    case 2: shared_gateup_mma_kernel<2><<<grid, block, 0, st>>>(H, Is, wg, wu, xb, P, T, ks, hb); break;
    case 4: shared_gateup_mma_kernel<4><<<grid, block, 0, st>>>(H, Is, wg, wu, xb, P, T, ks, hb); break;
    default: return ERR_SHAPE;
  }
  return cudaGetLastError() == cudaSuccess ? OK : ERR_CUDA;
}

int launch_shared_down_combine_mma(int H, int Is, const uint16_t* wd, const uint16_t* hb, int T, int k,
                                   const float* topk_w, const int32_t* inv, const float* obuf, int DP,
                                   const float* residual, float* y, cudaStream_t st) {
  const int ng = groups_for(2 * T);
  const int ks = pick_ks(Is, ksmax_for(ng));
  if (ks == 0) return ERR_SHAPE;
  const dim3 grid(H / kRows), block(32 * ks);
  const size_t dyn = static_cast<size_t>(kRows) * T * k * sizeof(float);
  switch (ng) {
    case 1:
      launch_pdl(shared_down_combine_mma_kernel<1>, grid, block, dyn, st, H, Is, wd, hb, T, ks, k, topk_w, inv, obuf,
                 DP, residual, y);
      break;
    case 2:
      launch_pdl(shared_down_combine_mma_kernel<2>, grid, block, dyn, st, H, Is, wd, hb, T, ks, k, topk_w, inv, obuf,
                 DP, residual, y);
      break;
    case 4:
      launch_pdl(shared_down_combine_mma_kernel<4>, grid, block, dyn, st, H, Is, wd, hb, T, ks, k, topk_w, inv, obuf,
                 DP, residual, y);
      break;
    case 8:
      launch_pdl(shared_down_combine_mma_kernel<8>, grid, block, dyn, st, H, Is, wd, hb, T, ks, k, topk_w, inv, obuf,
                 DP, residual, y);
      break;
    default: return ERR_SHAPE;
  }
  return cudaGetLastError() == cudaSuccess ? OK : ERR_CUDA;
}

}  // namespace moe
