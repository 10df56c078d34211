// decode.cu - the routed-expert FFN path built on int8 warp MMAs: activation
// digits, the gate/up and down dequant-GEMVs (gateup.cu, down.cu), the
// unquantized shared expert and the weighted combine.
//
// Sources: "ds4 : analyse pratique pour un usage documenté", section « Support de
// modèles et choix de quantification » (routed experts in 2-bit: up/gate IQ2_XXS,
// down Q2_K; shared experts unquantized) and "Un modèle de 284 milliards de
// paramètres tourne désormais sur un Mac de 128 Go. Qui y perd ?", section
// « Comment un modèle de 284 milliards de paramètres tient sur une seule
// machine » (the routed experts hold most of the bytes, so decode is bound by
// HBM bandwidth).
#include <cuda_bf16.h>

#include <algorithm>

#include <map>
#include <mutex>

#include "decode.cuh"
#include "kernels.cuh"
#include "profile.cuh"
#include "ptx.cuh"

namespace moe {

// x [T][H] -> xd [T][2][H] int8 digits (plane 0 hi, plane 1 lo) and
// xs [T][H/256] = 2^s / 8 per 256-element block (the 1/8 of the IQ2 scale is
// folded in). With qbits = 14 the block maximum maps into [2^12, 2^13), so
// |q| <= 8192 and hi = (q + 64) >> 7 stays within [-64, 64]; the TMA-fed GEMVs
// keep every int32 partial sum of such digits below 2^31 (four 32-weight
// sub-blocks at most before each conversion to fp32). The other GEMVs take
// qbits = 13 (|q| <= 4096), for which their longer integer sums are sized. One warp per 256-element block, 8 elements per lane. Block (0,0)
// also clears the call's device status word.
// For fp32 x it also writes two bf16 parts xb[part][T][H] (hi = rn(v),
// lo = rn(v - hi)) for the bf16 MMAs of the shared expert.
template <typename XT>
__global__ void __launch_bounds__(256) x_digits_kernel(const XT* __restrict__ x, int T, int H,
                                                       int8_t* __restrict__ xd, float* __restrict__ xs,
                                                       uint16_t* __restrict__ xb, int* __restrict__ err_word,
                                                       int qbits) {
  pdl_trigger();
  pdl_wait();
  if (err_word && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *err_word = 0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x;
  const int blk = blockIdx.y * 8 + warp;
  if (t >= T || blk * 256 >= H) return;
  const size_t base = static_cast<size_t>(t) * H + blk * 256 + lane * 8;
  float v[8];
  if constexpr (sizeof(XT) == 4) {
    const float4 a = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(x) + base);
    const float4 b = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(x) + base + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
    const uint4 a = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(x) + base);
    v[0] = __uint_as_float(a.x << 16); v[1] = __uint_as_float(a.x & 0xFFFF0000u);
    v[2] = __uint_as_float(a.y << 16); v[3] = __uint_as_float(a.y & 0xFFFF0000u);
    v[4] = __uint_as_float(a.z << 16); v[5] = __uint_as_float(a.z & 0xFFFF0000u);
    v[6] = __uint_as_float(a.w << 16); v[7] = __uint_as_float(a.w & 0xFFFF0000u);
  }
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(v[i]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  const int s = m > 0.f ? floor_log2_pos(m) - (qbits - 2) : 0;
  uint32_t hw[2] = {0, 0}, lw[2] = {0, 0};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    int hi = 0, lo = 0;
    if (m > 0.f) split_digits(v[i], s, hi, lo);
    hw[i / 4] |= (static_cast<uint32_t>(hi) & 0xFFu) << (8 * (i % 4));
    lw[i / 4] |= (static_cast<uint32_t>(lo) & 0xFFu) << (8 * (i % 4));
  }
  int8_t* row = xd + static_cast<size_t>(t) * 2 * H + blk * 256 + lane * 8;
  *reinterpret_cast<uint2*>(row) = make_uint2(hw[0], hw[1]);
  *reinterpret_cast<uint2*>(row + H) = make_uint2(lw[0], lw[1]);
  if (lane == 0) xs[static_cast<size_t>(t) * (H / 256) + blk] = m > 0.f ? ldexpf(1.0f, s - 3) : 0.f;
  if (sizeof(XT) == 4 && xb) {
    uint32_t hp[4], lp[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t h0 = __bfloat16_as_ushort(__float2bfloat16_rn(v[2 * i]));
      const uint32_t h1 = __bfloat16_as_ushort(__float2bfloat16_rn(v[2 * i + 1]));
      const uint32_t l0 = __bfloat16_as_ushort(__float2bfloat16_rn(v[2 * i] - __uint_as_float(h0 << 16)));
      const uint32_t l1 = __bfloat16_as_ushort(__float2bfloat16_rn(v[2 * i + 1] - __uint_as_float(h1 << 16)));
      hp[i] = h0 | (h1 << 16);
      lp[i] = l0 | (l1 << 16);
    }
    *reinterpret_cast<uint4*>(xb + base) = make_uint4(hp[0], hp[1], hp[2], hp[3]);
    *reinterpret_cast<uint4*>(xb + static_cast<size_t>(T) * H + base) = make_uint4(lp[0], lp[1], lp[2], lp[3]);
  }
}

// ------------------------------------------------------------ L2 prefetch
// Up to four ranges (16-byte aligned; sizes rounded down to 16 bytes, at most
// 2^32 - 16 each) brought into L2 with the evict_last policy, in chunks of
// 64 KB spread over the grid. Only L2 state changes; nothing is written.
struct PrefetchRanges {
  const uint8_t* p[4];
  uint64_t n[4];
};
__global__ void __launch_bounds__(128) l2_prefetch_kernel(PrefetchRanges r) {
  constexpr uint64_t kChunk = 64 * 1024;
  const uint64_t pol = l2_policy_evict_last();
  const uint64_t tid = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const uint64_t nthr = static_cast<uint64_t>(gridDim.x) * blockDim.x;
  for (int i = 0; i < 4; ++i) {
    const uint64_t n = r.n[i] & ~uint64_t(15);
    for (uint64_t off = tid * kChunk; off < n; off += nthr * kChunk) {
      const uint64_t len = n - off < kChunk ? n - off : kChunk;
      bulk_prefetch_l2(r.p[i] + off, static_cast<uint32_t>(len), pol);
    }
  }
}

int launch_l2_prefetch(const void* const* ptrs, const size_t* bytes, int n, cudaStream_t st) {
  PrefetchRanges r{};
  for (int i = 0; i < 4; ++i) {
    r.p[i] = i < n ? static_cast<const uint8_t*>(ptrs[i]) : nullptr;
    r.n[i] = (i < n && ptrs[i]) ? bytes[i] : 0;
  }
  l2_prefetch_kernel<<<148, 128, 0, st>>>(r);
  return cudaGetLastError() == cudaSuccess ? OK : ERR_CUDA;
}

// ------------------------------------------------------------ shared expert
__device__ __forceinline__ void bf16x8_to_f32(const uint4 w, float (&f)[8]) {
  f[0] = __uint_as_float(w.x << 16); f[1] = __uint_as_float(w.x & 0xFFFF0000u);
  f[2] = __uint_as_float(w.y << 16); f[3] = __uint_as_float(w.y & 0xFFFF0000u);
  f[4] = __uint_as_float(w.z << 16); f[5] = __uint_as_float(w.z & 0xFFFF0000u);
  f[6] = __uint_as_float(w.w << 16); f[7] = __uint_as_float(w.w & 0xFFFF0000u);
}

// hs[t][r] = silu(Wsg x_t)[r] * (Wsu x_t)[r] with bf16 weights: one warp per row
// pair (gate r, up r); activations staged in shared memory (fp32) in chunks of
// 2048; each lane keeps four 16-byte weight loads of each matrix in flight.
template <typename XT, int TMAX>
__global__ void __launch_bounds__(256) shared_gateup_kernel(int H, int Is, const uint16_t* __restrict__ sg,
                                                            const uint16_t* __restrict__ su,
                                                            const XT* __restrict__ x, int T,
                                                            float* __restrict__ hs) {
  constexpr int CH = 2048;
  __shared__ __align__(16) float xs[TMAX][CH];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + warp;
  for (int t0 = 0; t0 < T; t0 += TMAX) {
    const int nt = min(TMAX, T - t0);
    float ag[TMAX], au[TMAX];
#pragma unroll
    for (int t = 0; t < TMAX; ++t) ag[t] = au[t] = 0.f;
    for (int c0 = 0; c0 < H; c0 += CH) {
      __syncthreads();
      for (int i = threadIdx.x; i < TMAX * CH; i += 256) {
        const int t = i / CH, c = i % CH;
        float v = 0.f;
        if (t < nt && c0 + c < H) {
          const size_t idx = static_cast<size_t>(t0 + t) * H + c0 + c;
          if constexpr (sizeof(XT) == 4) v = reinterpret_cast<const float*>(x)[idx];
          else v = bf16_bits_to_float(reinterpret_cast<const uint16_t*>(x)[idx]);
        }
        xs[t][c] = v;
      }
      __syncthreads();
      if (row < Is) {
        const int lim = min(CH, H - c0);
        for (int cb = lane * 8; cb < lim; cb += 4 * 256) {
          uint4 wg[4], wu[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int c = cb + j * 256;
            if (c < lim) {
              wg[j] = *reinterpret_cast<const uint4*>(sg + static_cast<size_t>(row) * H + c0 + c);
              wu[j] = *reinterpret_cast<const uint4*>(su + static_cast<size_t>(row) * H + c0 + c);
            } else {
              wg[j] = wu[j] = make_uint4(0u, 0u, 0u, 0u);
            }
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int c = cb + j * 256;
            if (c >= lim) break;
            float g8[8], u8[8];
            bf16x8_to_f32(wg[j], g8);
            bf16x8_to_f32(wu[j], u8);
#pragma unroll
            for (int t = 0; t < TMAX; ++t) {
              if (t >= nt) break;
              const float4 xa = *reinterpret_cast<const float4*>(&xs[t][c]);
              const float4 xb = *reinterpret_cast<const float4*>(&xs[t][c + 4]);
              const float xv[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                ag[t] = fmaf(g8[i], xv[i], ag[t]);
                au[t] = fmaf(u8[i], xv[i], au[t]);
              }
            }
          }
        }
      }
    }
    if (row < Is) {
#pragma unroll
      for (int t = 0; t < TMAX; ++t) {
        float gg = ag[t], uu = au[t];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          gg += __shfl_xor_sync(0xffffffffu, gg, o);
          uu += __shfl_xor_sync(0xffffffffu, uu, o);
        }
        if (lane == 0 && t < nt) hs[static_cast<size_t>(t0 + t) * Is + row] = silu_mul(gg, uu);
      }
    }
  }
}

// Same for few tokens (T <= TMAX): no shared-memory staging and no block-wide
// barrier; activations come from global memory (L1-resident, the same for every
// warp), four 16-byte weight loads of each matrix per lane are in flight. One
// warp per row, any number of warps per CTA: launched with small CTAs and no
// shared memory, it fits beside the routed GEMVs on the same SMs.
template <typename XT, int TMAX>
__global__ void __launch_bounds__(256) shared_gateup_direct_kernel(int H, int Is, const uint16_t* __restrict__ sg,
                                                                   const uint16_t* __restrict__ su,
                                                                   const XT* __restrict__ x, int T,
                                                                   float* __restrict__ hs) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + warp;
  if (row >= Is) return;
  float ag[TMAX], au[TMAX];
#pragma unroll
  for (int t = 0; t < TMAX; ++t) ag[t] = au[t] = 0.f;
  const uint16_t* gr = sg + static_cast<size_t>(row) * H;
  const uint16_t* ur = su + static_cast<size_t>(row) * H;
  for (int cb = lane * 8; cb < H; cb += 4 * 256) {
    uint4 wg[4], wu[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = cb + j * 256;
      wg[j] = c < H ? *reinterpret_cast<const uint4*>(gr + c) : make_uint4(0u, 0u, 0u, 0u);
      wu[j] = c < H ? *reinterpret_cast<const uint4*>(ur + c) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = cb + j * 256;
      if (c >= H) break;
      float g8[8], u8[8];
      bf16x8_to_f32(wg[j], g8);
      bf16x8_to_f32(wu[j], u8);
#pragma unroll
      for (int t = 0; t < TMAX; ++t) {
        if (t >= T) break;
        float xv[8];
        if constexpr (sizeof(XT) == 4) {
          const float4 xa = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(x) + static_cast<size_t>(t) * H + c);
          const float4 xb = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(x) + static_cast<size_t>(t) * H + c + 4);
          xv[0] = xa.x; xv[1] = xa.y; xv[2] = xa.z; xv[3] = xa.w; xv[4] = xb.x; xv[5] = xb.y; xv[6] = xb.z; xv[7] = xb.w;
        } else {
          bf16x8_to_f32(*reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(x) + static_cast<size_t>(t) * H + c), xv);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          ag[t] = fmaf(g8[i], xv[i], ag[t]);
          au[t] = fmaf(u8[i], xv[i], au[t]);
        }
      }
    }
  }
#pragma unroll
  for (int t = 0; t < TMAX; ++t) {
    float gg = ag[t], uu = au[t];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      gg += __shfl_xor_sync(0xffffffffu, gg, o);
      uu += __shfl_xor_sync(0xffffffffu, uu, o);
    }
    if (lane == 0 && t < T) hs[static_cast<size_t>(t) * Is + row] = silu_mul(gg, uu);
  }
}

// y[t][r] = sum_j w[t][j] o[inv[t*k+j]][r] (j ascending) + (Wsd hs_t)[r] + residual[t][r],
// where o of an assignment is the sum of its DP partial rows (parts in order).
// One warp per output row r, all tokens; the row's weights are loaded up front.
// With k = 0 it is the shared expert's down projection alone.
template <int TMAX>
__global__ void __launch_bounds__(256) shared_down_combine_kernel(int H, int Is, int k, const uint16_t* __restrict__ sd,
                                                                  const float* __restrict__ hs, int T,
                                                                  const float* __restrict__ topk_w,
                                                                  const int32_t* __restrict__ inv,
                                                                  const float* __restrict__ obuf, int DP,
                                                                  const float* residual, float* y) {
  constexpr int WMAX = 8;  // 16-byte weight loads per lane kept in registers (Is <= 2048)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + warp;
  if (row >= H) return;
  const int nw = (Is + 255) / 256;
  uint4 wv[WMAX];
  const bool in_regs = nw <= WMAX;
  if (in_regs) {
#pragma unroll
    for (int j = 0; j < WMAX; ++j) {
      const int c = lane * 8 + j * 256;
      wv[j] = (j < nw && c < Is) ? *reinterpret_cast<const uint4*>(sd + static_cast<size_t>(row) * Is + c)
                                 : make_uint4(0u, 0u, 0u, 0u);
    }
  }
  for (int t0 = 0; t0 < T; t0 += TMAX) {
    const int nt = min(TMAX, T - t0);
    float acc[TMAX];
#pragma unroll
    for (int t = 0; t < TMAX; ++t) acc[t] = 0.f;
    auto dot8 = [&](const uint4 w, int c) {
      float w8[8];
      bf16x8_to_f32(w, w8);
#pragma unroll
      for (int t = 0; t < TMAX; ++t) {
        if (t >= nt) break;
        const float4 ha = *reinterpret_cast<const float4*>(hs + static_cast<size_t>(t0 + t) * Is + c);
        const float4 hb = *reinterpret_cast<const float4*>(hs + static_cast<size_t>(t0 + t) * Is + c + 4);
        float s = acc[t];
        s = fmaf(w8[0], ha.x, s); s = fmaf(w8[1], ha.y, s); s = fmaf(w8[2], ha.z, s); s = fmaf(w8[3], ha.w, s);
        s = fmaf(w8[4], hb.x, s); s = fmaf(w8[5], hb.y, s); s = fmaf(w8[6], hb.z, s); s = fmaf(w8[7], hb.w, s);
        acc[t] = s;
      }
    };
    if (in_regs) {
#pragma unroll
      for (int j = 0; j < WMAX; ++j) {
        const int c = lane * 8 + j * 256;
        if (j >= nw || c >= Is) break;
        dot8(wv[j], c);
      }
    } else {
      for (int c = lane * 8; c < Is; c += 256)
        dot8(*reinterpret_cast<const uint4*>(sd + static_cast<size_t>(row) * Is + c), c);
    }
#pragma unroll
    for (int t = 0; t < TMAX; ++t) {
      float s = acc[t];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      acc[t] = s;
    }
    // routed part: lane i takes (slot i / DP, part i % DP); fixed shuffle tree
#pragma unroll
    for (int t = 0; t < TMAX; ++t) {
      if (t >= nt) break;
      const int tt = t0 + t;
      float v = 0.f;
      for (int i = lane; i < k * DP; i += 32) {
        const int aidx = tt * k + i / DP;
        v = fmaf(topk_w[aidx], obuf[(static_cast<size_t>(inv[aidx]) * DP + i % DP) * H + row], v);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) {
        v += acc[t];
        if (residual) v += residual[static_cast<size_t>(tt) * H + row];
        y[static_cast<size_t>(tt) * H + row] = v;
      }
    }
  }
}

// y[t][r] = sum_j w[t][j] o[inv[t*k+j]][r] (j ascending) + ys[t][r] + residual[t][r],
// where o of an assignment is the sum of its DP partial rows (parts in order)
// and ys the shared expert's output computed beforehand. One thread per (t, r);
// the assignments are taken eight at a time with all their routing words, then
// all their partial rows, requested before any is added, so a thread waits for
// memory once per eight assignments rather than twice per assignment. With yb,
// the same value rounded to bf16 (nearest, ties to even) is stored there too:
// the next layer's input.
__global__ void __launch_bounds__(256) combine_routed_kernel(int H, int k, const float* __restrict__ topk_w,
                                                             const int32_t* __restrict__ inv,
                                                             const float* __restrict__ obuf, int DP,
                                                             const float* __restrict__ ys, const float* residual,
                                                             float* y, uint16_t* __restrict__ yb) {
  constexpr int JC = 8, DC = 8;
  pdl_trigger();
  pdl_wait();  // the routed partials come from the kernel before this one
  const int r = blockIdx.x * blockDim.x + threadIdx.x, t = blockIdx.y;
  if (r >= H) return;
  float v = 0.f;
  for (int j0 = 0; j0 < k; j0 += JC) {
    const float* o[JC];
    float wj[JC];
#pragma unroll
    for (int j = 0; j < JC; ++j) {
      const int a = t * k + j0 + j;
      const bool in = j0 + j < k;
      o[j] = in ? obuf + static_cast<size_t>(inv[a]) * DP * H + r : nullptr;
      wj[j] = in ? topk_w[a] : 0.f;
    }
    float sacc[JC];
#pragma unroll
    for (int j = 0; j < JC; ++j) sacc[j] = 0.f;
    for (int d0 = 0; d0 < DP; d0 += DC) {
      float pv[JC][DC];
#pragma unroll
      for (int j = 0; j < JC; ++j)
#pragma unroll
        for (int d = 0; d < DC; ++d)
          pv[j][d] = (o[j] && d0 + d < DP) ? o[j][static_cast<size_t>(d0 + d) * H] : 0.f;
#pragma unroll
      for (int j = 0; j < JC; ++j)
#pragma unroll
        for (int d = 0; d < DC; ++d)
          if (d0 + d < DP) sacc[j] += pv[j][d];
    }
#pragma unroll
    for (int j = 0; j < JC; ++j)
      if (j0 + j < k) v = fmaf(wj[j], sacc[j], v);
  }
  const size_t i = static_cast<size_t>(t) * H + r;
  v += ys[i];
  if (residual) v += residual[i];
  y[i] = v;
  if (yb) yb[i] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

// yb[i] = bf16(y[i]) (nearest, ties to even) for the paths whose last kernel
// does not write the bf16 copy itself; n a multiple of 4, both 16-byte aligned.
__global__ void __launch_bounds__(256) y_to_bf16_kernel(const float* __restrict__ y, uint16_t* __restrict__ yb,
                                                        size_t n4) {
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const float4 v = reinterpret_cast<const float4*>(y)[i];
    const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(v.x)) |
                        (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v.y))) << 16);
    const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(v.z)) |
                        (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v.w))) << 16);
    reinterpret_cast<uint2*>(yb)[i] = make_uint2(lo, hi);
  }
}

// ------------------------------------------------------------ launcher
namespace {
int num_sms() {
  static int sms = 0;
  if (sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
  }
  return sms;
}
}  // namespace

bool fast_path_supported(const LayerShape& s) { return s.I % 256 == 0 && s.H % 256 == 0; }

namespace {
int hsc_stride(int I) { return ((I / 256) + 3) & ~3; }
}  // namespace

// h = silu(g) * u for assignment blockIdx.x, 256-element block blockIdx.y:
// g and u arrive as KP partial sums each ([p][2][KP][I]); warp w adds parts
// w, w + 8, ... in order, the eight warp sums are added in warp order (a fixed
// order: results are identical run to run), and warp 0 quantises the block
// (hquant_finish_warp).
template <bool kHOff>
__global__ void __launch_bounds__(256) hquant_kernel(int I, int KP, const float* __restrict__ gu,
                                                     int8_t* __restrict__ hd, float* __restrict__ hsc,
                                                     int32_t* __restrict__ hq, int hss) {
  __shared__ float4 red[8][4][32];  // [warp][g lo, g hi, u lo, u hi][lane]
  pdl_trigger();
  pdl_wait();
  const int p = blockIdx.x, sb = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float* g = gu + static_cast<size_t>(p) * 2 * KP * I + sb * 256 + lane * 8;
  const float* u = g + static_cast<size_t>(KP) * I;
  float4 s[4] = {make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f),
                 make_float4(0.f, 0.f, 0.f, 0.f)};
  for (int kp = warp; kp < KP; kp += 8) {
    const float4 v0 = __ldcg(reinterpret_cast<const float4*>(g + static_cast<size_t>(kp) * I));
    const float4 v1 = __ldcg(reinterpret_cast<const float4*>(g + static_cast<size_t>(kp) * I + 4));
    const float4 v2 = __ldcg(reinterpret_cast<const float4*>(u + static_cast<size_t>(kp) * I));
    const float4 v3 = __ldcg(reinterpret_cast<const float4*>(u + static_cast<size_t>(kp) * I + 4));
    s[0].x += v0.x; s[0].y += v0.y; s[0].z += v0.z; s[0].w += v0.w;
    s[1].x += v1.x; s[1].y += v1.y; s[1].z += v1.z; s[1].w += v1.w;
    s[2].x += v2.x; s[2].y += v2.y; s[2].z += v2.z; s[2].w += v2.w;
    s[3].x += v3.x; s[3].y += v3.y; s[3].z += v3.z; s[3].w += v3.w;
  }
#pragma unroll
  for (int q = 0; q < 4; ++q) red[warp][q][lane] = s[q];
  __syncthreads();
  if (warp != 0) return;
  float gv[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f}, uv[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int w = 0; w < 8; ++w) {
    const float4 a = red[w][0][lane], b = red[w][1][lane], c = red[w][2][lane], d = red[w][3][lane];
    gv[0] += a.x; gv[1] += a.y; gv[2] += a.z; gv[3] += a.w; gv[4] += b.x; gv[5] += b.y; gv[6] += b.z; gv[7] += b.w;
    uv[0] += c.x; uv[1] += c.y; uv[2] += c.z; uv[3] += c.w; uv[4] += d.x; uv[5] += d.y; uv[6] += d.z; uv[7] += d.w;
  }
  hquant_finish_warp<kHOff>(I, p, sb, gv, uv, hd, hsc, hq, hss, lane);
}

// The TMA-fed GEMVs (gemv_tma.cu) serve shapes with H % 1024 == 0 and
// I % 512 == 0 for up to kTmaMaxT tokens; they write KP (gate/up) and DP
// (down) partial sums per assignment.
namespace {
constexpr int kTmaMaxT = 16;
bool tma_shape(const LayerShape& s, int T) { return s.H % 1024 == 0 && s.I % 512 == 0 && T <= kTmaMaxT; }

struct FastWs {
  int8_t* xd;
  float* xs;
  float* gu;
  int8_t* hd;
  float* hsc;
  int32_t* hq;
  float* obuf;
  float* hsh;
  float* ysh;    // the shared expert's output [T][H] (computed on the side stream)
  uint16_t* xb;  // bf16 parts of fp32 x [2][T][H]
  uint16_t* hb;  // bf16 parts of the shared intermediate [2][T][Is]
  size_t bytes;
};

FastWs carve_fast(const LayerShape& s, int T, int KP, int DP, char* base) {
  const size_t nA = static_cast<size_t>(T) * s.k;
  FastWs w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* q = base ? base + off : nullptr;
    off += align_up(bytes > 0 ? bytes : 1, 256);
    return q;
  };
  w.xd = reinterpret_cast<int8_t*>(take(static_cast<size_t>(T) * 2 * s.H));
  w.xs = reinterpret_cast<float*>(take(static_cast<size_t>(T) * (s.H / 256) * 4));
  w.gu = reinterpret_cast<float*>(take(nA * 2 * KP * s.I * 4));
  w.hd = reinterpret_cast<int8_t*>(take(nA * 2 * s.I));
  w.hsc = reinterpret_cast<float*>(take(nA * hsc_stride(s.I) * 4));
  w.hq = reinterpret_cast<int32_t*>(take(nA * (s.I / 16) * 4));
  w.obuf = reinterpret_cast<float*>(take(nA * DP * s.H * 4));
  w.hsh = reinterpret_cast<float*>(take(static_cast<size_t>(T) * (s.Is > 0 ? s.Is : 1) * 4));
  w.ysh = reinterpret_cast<float*>(take(static_cast<size_t>(T) * s.H * 4));
  w.xb = reinterpret_cast<uint16_t*>(take(static_cast<size_t>(T) * 2 * s.H * 2));
  w.hb = reinterpret_cast<uint16_t*>(take(static_cast<size_t>(T) * 2 * (s.Is > 0 ? s.Is : 1) * 2));
  w.bytes = off;
  return w;
}
}  // namespace

size_t fast_ffn_workspace_bytes(const LayerShape& s, int T) {
  size_t b = carve_fast(s, T, 1, 1, nullptr).bytes;
  if (s.H % 1024 == 0 && s.I % 512 == 0) {
    const int Tt = std::min(T, kTmaMaxT);  // keeps the size monotone in T
    b = std::max(b, carve_fast(s, Tt, tma_gu_parts(s, Tt), tma_dn_parts(s, Tt), nullptr).bytes);
  }
  return b;
}

// Token counts up to which the side stream runs the shared expert as warp-per-row GEMVs.
constexpr int kSharedDirectMaxT = 4;

// Side stream and fork/join events per (device, caller stream), created on first use.
struct SideCtx {
  cudaStream_t st = nullptr;
  // fork: caller -> side; digits: x digits ready; join: shared h ready
  cudaEvent_t fork = nullptr, digits = nullptr, join = nullptr;
};
static SideCtx* side_ctx(cudaStream_t st) {
  static std::mutex mu;
  static std::map<std::pair<int, cudaStream_t>, SideCtx> table;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  SideCtx& c = table[{dev, st}];
  if (!c.st) {
    if (cudaStreamCreateWithFlags(&c.st, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&c.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&c.digits, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&c.join, cudaEventDisableTiming) != cudaSuccess) {
      table.erase({dev, st});
      return nullptr;
    }
  }
  return &c;
}

bool shared_early_ok(const LayerShape& s, int x_dtype, int T) {
  return x_dtype == 1 && s.Is > 0 && !use_prefill(s, T) && fast_path_supported(s) &&
         shared_mma_supported(s.H, s.Is, T, 1, s.k);
}

void join_shared_early(cudaStream_t st) {
  if (SideCtx* c = side_ctx(st)) cudaStreamWaitEvent(st, c->join, 0);
}

int launch_shared_early(const LayerShape& s, const WeightPtrs& w, const void* x, int T, void* ws, cudaStream_t st,
                        int KP, int DP) {
  SideCtx* c = side_ctx(st);
  if (!c) return ERR_CUDA;
  const bool tma = tma_shape(s, T) && tma_path_supported(s, T);
  if (KP <= 0) {  // the layout of launch_ffn_fast
    KP = tma ? tma_gu_parts(s, T) : 1;
    DP = tma ? tma_dn_parts(s, T) : 1;
  }
  const FastWs fw = carve_fast(s, T, KP, DP, static_cast<char*>(ws));
  if (cudaEventRecord(c->fork, st) != cudaSuccess || cudaStreamWaitEvent(c->st, c->fork, 0) != cudaSuccess)
    return ERR_CUDA;
  // the activation digits of the routed GEMVs do not depend on routing either
  {
    ProfScope ps(MOE_K_PREP, c->st);
    dim3 g(T, (s.H / 256 + 7) / 8);
    x_digits_kernel<uint16_t><<<g, 256, 0, c->st>>>(static_cast<const uint16_t*>(x), T, s.H, fw.xd, fw.xs, nullptr,
                                                    nullptr, tma ? 14 : 13);
  }
  if (cudaEventRecord(c->digits, c->st) != cudaSuccess) return ERR_CUDA;
  // the whole shared expert follows on the side stream, into ysh. For a few tokens its GEMVs run in CTAs of
  // four warps without shared memory, which fit on the SMs beside the routed GEMVs (compute-bound at these
  // sizes) and use the HBM bandwidth those leave; for more tokens the tensor-core kernels.
  const uint16_t* xb = static_cast<const uint16_t*>(x);
  int rc = OK;
  if (T <= kSharedDirectMaxT) {
    {
      ProfScope ps(MOE_K_SHARED_GATEUP, c->st);
      const int grid = (s.Is + 3) / 4;
      if (T == 1)
        shared_gateup_direct_kernel<uint16_t, 1><<<grid, 128, 0, c->st>>>(s.H, s.Is, w.sh_gate, w.sh_up, xb, T, fw.hsh);
      else
        shared_gateup_direct_kernel<uint16_t, 4><<<grid, 128, 0, c->st>>>(s.H, s.Is, w.sh_gate, w.sh_up, xb, T, fw.hsh);
    }
    {
      ProfScope ps(MOE_K_SHARED_DOWN, c->st);
      const int grid = (s.H + 3) / 4;
      if (T == 1)
        shared_down_combine_kernel<1><<<grid, 128, 0, c->st>>>(s.H, s.Is, 0, w.sh_down, fw.hsh, T, nullptr, nullptr,
                                                               nullptr, 1, nullptr, fw.ysh);
      else
        shared_down_combine_kernel<4><<<grid, 128, 0, c->st>>>(s.H, s.Is, 0, w.sh_down, fw.hsh, T, nullptr, nullptr,
                                                               nullptr, 1, nullptr, fw.ysh);
    }
  } else {
    {
      ProfScope ps(MOE_K_SHARED_GATEUP, c->st);
      rc = launch_shared_gateup_mma(s.H, s.Is, w.sh_gate, w.sh_up, xb, 1, T, fw.hb, c->st);
    }
    {
      ProfScope ps(MOE_K_SHARED_DOWN, c->st);
      rc |= launch_shared_down_combine_mma(s.H, s.Is, w.sh_down, fw.hb, T, 0, nullptr, nullptr, nullptr, 1, nullptr,
                                           fw.ysh, c->st);
    }
  }
  if (cudaEventRecord(c->join, c->st) != cudaSuccess) return ERR_CUDA;
  return rc != OK ? ERR_CUDA : (cudaGetLastError() == cudaSuccess ? OK : ERR_CUDA);
}

int launch_ffn_fast(const LayerShape& s, const WeightPtrs& w, const void* x, int x_dtype, int T, const Routing& r,
                    const float* residual, float* y, void* ws, int* err, bool clear_status, cudaStream_t st,
                    bool shared_early, uint16_t* y_bf16) {
  const size_t nA = static_cast<size_t>(T) * s.k;
  const bool tma = tma_shape(s, T) && tma_path_supported(s, T);
  const int KP = tma ? tma_gu_parts(s, T) : 1, DP = tma ? tma_dn_parts(s, T) : 1;
  const FastWs fw = carve_fast(s, T, KP, DP, static_cast<char*>(ws));
  int8_t* xd = fw.xd;
  float* xs = fw.xs;
  float* gu = fw.gu;
  int8_t* hd = fw.hd;
  float* hsc = fw.hsc;
  int32_t* hq = fw.hq;
  float* obuf = fw.obuf;
  float* hsh = fw.hsh;

  const int sms = num_sms();
  const int slots = static_cast<int>(std::min<size_t>(nA, static_cast<size_t>(s.E)));
  int rc = OK;
  if (shared_early) {  // the digits come from the side stream (launch_shared_early)
    SideCtx* c = side_ctx(st);
    if (!c || cudaStreamWaitEvent(st, c->digits, 0) != cudaSuccess) return ERR_CUDA;
  } else {
    ProfScope ps(MOE_K_PREP, st);
    dim3 g(T, (s.H / 256 + 7) / 8);
    const int qbits = tma ? 14 : 13;
    if (x_dtype == 0)
      launch_pdl(x_digits_kernel<float>, g, dim3(256), 0, st, static_cast<const float*>(x), T, s.H, xd, xs, fw.xb,
                 clear_status ? err : nullptr, qbits);
    else
      launch_pdl(x_digits_kernel<uint16_t>, g, dim3(256), 0, st, static_cast<const uint16_t*>(x), T, s.H, xd, xs,
                 static_cast<uint16_t*>(nullptr), clear_status ? err : nullptr, qbits);
  }
  // bf16 activations feed the shared expert's MMAs as one part, fp32 as two
  const int xparts = x_dtype == 0 ? 2 : 1;
  const uint16_t* xbp = x_dtype == 0 ? fw.xb : static_cast<const uint16_t*>(x);
  const bool sh_mma = s.Is > 0 && shared_mma_supported(s.H, s.Is, T, xparts, s.k);
  if (tma) {
    ProfScope ps(MOE_K_GATEUP, st);
    rc |= launch_gateup_tma(s, w.gate_codes, w.gate_d, w.up_codes, w.up_d, xd, xs, T, r, gu, err, sms, st);
  } else {
    GateupArgs ga{};
    ga.H = s.H; ga.I = s.I; ga.E = s.E; ga.k = s.k; ga.T = T;
    ga.gate_codes = w.gate_codes; ga.gate_d = w.gate_d; ga.up_codes = w.up_codes; ga.up_d = w.up_d;
    ga.xd = xd; ga.xs = xs; ga.offsets = r.offsets; ga.perm = r.perm; ga.active = r.active;
    ga.gu = gu; ga.err = err;
    ProfScope ps(MOE_K_GATEUP, st);
    rc |= launch_gateup(ga, slots, sms, st);
  }
  if (sh_mma && shared_early) {
    // launched before routing on the side stream (launch_shared_early)
  } else if (sh_mma) {
    ProfScope ps(MOE_K_SHARED_GATEUP, st);
    rc |= launch_shared_gateup_mma(s.H, s.Is, w.sh_gate, w.sh_up, xbp, xparts, T, fw.hb, st);
  } else if (s.Is > 0) {
    ProfScope ps(MOE_K_SHARED_GATEUP, st);
    const int grid = (s.Is + 7) / 8;
    if (T <= 4) {
      if (x_dtype == 0)
        shared_gateup_direct_kernel<float, 4><<<grid, 256, 0, st>>>(s.H, s.Is, w.sh_gate, w.sh_up,
                                                                    static_cast<const float*>(x), T, hsh);
      else
        shared_gateup_direct_kernel<uint16_t, 4><<<grid, 256, 0, st>>>(s.H, s.Is, w.sh_gate, w.sh_up,
                                                                       static_cast<const uint16_t*>(x), T, hsh);
    } else if (x_dtype == 0) {
      shared_gateup_kernel<float, 4><<<grid, 256, 0, st>>>(s.H, s.Is, w.sh_gate, w.sh_up,
                                                           static_cast<const float*>(x), T, hsh);
    } else {
      shared_gateup_kernel<uint16_t, 4><<<grid, 256, 0, st>>>(s.H, s.Is, w.sh_gate, w.sh_up,
                                                              static_cast<const uint16_t*>(x), T, hsh);
    }
  }
  {
    ProfScope ps(MOE_K_HQUANT, st);
    const dim3 hg(static_cast<unsigned>(nA), static_cast<unsigned>(s.I / 256));
    if (tma)
      launch_pdl(hquant_kernel<true>, hg, dim3(256), 0, st, s.I, KP, static_cast<const float*>(gu), hd, hsc, hq,
                 hsc_stride(s.I));
    else
      launch_pdl(hquant_kernel<false>, hg, dim3(256), 0, st, s.I, KP, static_cast<const float*>(gu), hd, hsc, hq,
                 hsc_stride(s.I));
  }
  if (tma) {
    ProfScope ps(MOE_K_DOWN, st);
    rc |= launch_down_tma(s, w.down_codes, w.down_dd, hd, hsc, hq, hsc_stride(s.I), T, r, obuf, err, sms, st);
  } else {
    DownArgs da{};
    da.H = s.H; da.I = s.I; da.E = s.E; da.k = s.k;
    da.codes = w.down_codes; da.dd = w.down_dd; da.hd = hd; da.hsc = hsc; da.hq = hq;
    da.offsets = r.offsets; da.active = r.active; da.o = obuf; da.err = err;
    ProfScope ps(MOE_K_DOWN, st);
    rc |= launch_down(da, slots, T, sms, st);
  }
  if (shared_early) {  // the shared output is ready in ysh once the side stream joins
    SideCtx* c = side_ctx(st);
    if (!c || cudaStreamWaitEvent(st, c->join, 0) != cudaSuccess) return ERR_CUDA;
    ProfScope ps(MOE_K_COMBINE, st);
    launch_pdl(combine_routed_kernel, dim3((s.H + 255) / 256, T), dim3(256), 0, st, s.H, s.k,
               static_cast<const float*>(r.topk_w), static_cast<const int32_t*>(r.inv),
               static_cast<const float*>(obuf), DP, static_cast<const float*>(fw.ysh), residual, y, y_bf16);
  } else if (sh_mma) {
    ProfScope ps(MOE_K_COMBINE, st);
    rc |= launch_shared_down_combine_mma(s.H, s.Is, w.sh_down, fw.hb, T, s.k, r.topk_w, r.inv, obuf, DP, residual, y,
                                         st);
  } else {
    ProfScope ps(MOE_K_COMBINE, st);
    const int grid = (s.H + 7) / 8;
    shared_down_combine_kernel<8><<<grid, 256, 0, st>>>(s.H, s.Is, s.k, s.Is > 0 ? w.sh_down : nullptr, hsh, T,
                                                        r.topk_w, r.inv, obuf, DP, residual, y);
  }
  if (y_bf16 && !shared_early) rc |= launch_y_to_bf16(y, y_bf16, static_cast<size_t>(T) * s.H, st);
  if (rc != OK) return ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? OK : ERR_CUDA;
}

int launch_y_to_bf16(const float* y, uint16_t* yb, size_t n, cudaStream_t st) {
  const size_t n4 = n / 4;
  if (n4 == 0) return OK;
  ProfScope ps(MOE_K_COMBINE, st);
  const int grid = static_cast<int>(std::min<size_t>((n4 + 255) / 256, static_cast<size_t>(num_sms()) * 8));
  y_to_bf16_kernel<<<grid, 256, 0, st>>>(y, yb, n4);
  return cudaGetLastError() == cudaSuccess ? OK : ERR_CUDA;
}


// ------------------------------------------------------------ block-32 experts
// The same step as launch_ffn_fast (digits, gate/up, h, down, shared expert,
// combine) with the block-32 GEMVs of mxfp4.cu (MXFP4 or Q4-style): gate/up and
// down in 256-element parts of their reduction axes, h re-quantised as
// activation digits.
size_t mx_ffn_workspace_bytes(const LayerShape& s, int T, int fmt) {
  // one workspace serves every T up to the given one: the GEMV step up to 16 tokens, the grouped GEMM above
  const size_t dec = carve_fast(s, std::min(T, kPrefillMinT), mx_parts(s.H), mx_parts(s.I), nullptr).bytes;
  if (T <= kPrefillMinT) return dec;
  if (fmt == 0) return mx_prefill_supported(s, T) ? std::max(dec, mx_prefill_workspace_bytes(s, T)) : dec;
  return prefill_path_supported(s, T) ? std::max(dec, prefill_workspace_bytes(s, T)) : dec;
}

int launch_ffn_mxfp4(const LayerShape& s, const WeightPtrs& shw, const MxPlanes& w, const void* x, int x_dtype,
                     int T, const Routing& r, const float* residual, float* y, void* ws, int* err, bool clear_status,
                     cudaStream_t st, bool shared_early) {
  if (T > kPrefillMinT) {  // many tokens: MXFP4 on the block-scaled grouped GEMM, Q4-style on the dequantising one
    if (shared_early) return ERR_ARG;
    if (w.fmt == 0)
      return launch_ffn_mx_prefill(s, shw, w, x, x_dtype, T, r, residual, y, ws, err, clear_status, num_sms(), st);
    return launch_ffn_prefill(s, shw, x, x_dtype, T, r, residual, y, ws, err, clear_status, num_sms(), st, &w);
  }
  const int nA = T * s.k;
  const int KP = mx_parts(s.H), DP = mx_parts(s.I);
  const FastWs fw = carve_fast(s, T, KP, DP, static_cast<char*>(ws));
  const int sms = num_sms();
  int rc = OK;
  if (shared_early) {  // the digits come from the side stream (launch_shared_early with this layout)
    SideCtx* c = side_ctx(st);
    if (!c || cudaStreamWaitEvent(st, c->digits, 0) != cudaSuccess) return ERR_CUDA;
  } else {
    ProfScope ps(MOE_K_PREP, st);
    dim3 g(T, (s.H / 256 + 7) / 8);
    if (x_dtype == 0)
      launch_pdl(x_digits_kernel<float>, g, dim3(256), 0, st, static_cast<const float*>(x), T, s.H, fw.xd, fw.xs,
                 fw.xb, clear_status ? err : nullptr, 14);
    else
      launch_pdl(x_digits_kernel<uint16_t>, g, dim3(256), 0, st, static_cast<const uint16_t*>(x), T, s.H, fw.xd,
                 fw.xs, static_cast<uint16_t*>(nullptr), clear_status ? err : nullptr, 14);
  }
  {
    ProfScope ps(MOE_K_GATEUP, st);
    rc |= launch_mx_gemv(w.fmt, true, s.H, s.I, s.E, s.k, T, w.gate_codes, w.gate_scales, w.up_codes, w.up_scales,
                         fw.xd, fw.xs, r, fw.gu, err, sms, st);
  }
  {
    ProfScope ps(MOE_K_HQUANT, st);
    rc |= launch_mx_hquant(s.I, KP, nA, fw.gu, fw.hd, fw.hsc, st);
  }
  {
    ProfScope ps(MOE_K_DOWN, st);
    rc |= launch_mx_gemv(w.fmt, false, s.I, s.H, s.E, s.k, T, w.down_codes, w.down_scales, nullptr, nullptr, fw.hd,
                         fw.hsc, r, fw.obuf, err, sms, st);
  }
  if (shared_early) {  // the shared output is ready in ysh once the side stream joins
    SideCtx* c = side_ctx(st);
    if (!c || cudaStreamWaitEvent(st, c->join, 0) != cudaSuccess) return ERR_CUDA;
    ProfScope ps(MOE_K_COMBINE, st);
    launch_pdl(combine_routed_kernel, dim3((s.H + 255) / 256, T), dim3(256), 0, st, s.H, s.k,
               static_cast<const float*>(r.topk_w), static_cast<const int32_t*>(r.inv),
               static_cast<const float*>(fw.obuf), DP, static_cast<const float*>(fw.ysh), residual, y,
               static_cast<uint16_t*>(nullptr));
  } else {
    // the shared expert here, then its down projection fused with the combine
    const int xparts = x_dtype == 0 ? 2 : 1;
    const uint16_t* xbp = x_dtype == 0 ? fw.xb : static_cast<const uint16_t*>(x);
    if (s.Is > 0 && shared_mma_supported(s.H, s.Is, T, xparts, s.k)) {
      {
        ProfScope ps(MOE_K_SHARED_GATEUP, st);
        rc |= launch_shared_gateup_mma(s.H, s.Is, shw.sh_gate, shw.sh_up, xbp, xparts, T, fw.hb, st);
      }
      ProfScope ps(MOE_K_COMBINE, st);
      rc |= launch_shared_down_combine_mma(s.H, s.Is, shw.sh_down, fw.hb, T, s.k, r.topk_w, r.inv, fw.obuf, DP,
                                           residual, y, st);
    } else {
      if (s.Is > 0) {
        ProfScope ps(MOE_K_SHARED_GATEUP, st);
        const int grid = (s.Is + 7) / 8;
        if (x_dtype == 0)
          shared_gateup_direct_kernel<float, 4><<<grid, 256, 0, st>>>(s.H, s.Is, shw.sh_gate, shw.sh_up,
                                                                      static_cast<const float*>(x), T, fw.hsh);
        else
          shared_gateup_direct_kernel<uint16_t, 4><<<grid, 256, 0, st>>>(s.H, s.Is, shw.sh_gate, shw.sh_up,
                                                                         static_cast<const uint16_t*>(x), T, fw.hsh);
      }
      ProfScope ps(MOE_K_COMBINE, st);
      shared_down_combine_kernel<8><<<(s.H + 7) / 8, 256, 0, st>>>(s.H, s.Is, s.k, s.Is > 0 ? shw.sh_down : nullptr,
                                                                   fw.hsh, T, r.topk_w, r.inv, fw.obuf, DP,
                                                                   residual, y);
    }
  }
  if (rc != OK) return ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? OK : ERR_CUDA;
}

}  // namespace moe
