// quant.cu - float weights -> the library's 2-bit block formats on the GPU:
// round-to-nearest for the Q2K-style format, an exhaustive codebook search
// for the IQ2-style format, no importance matrix.
//
// Source: the routed experts are quantized, up/gate in IQ2_XXS and down in
// Q2_K ("ds4 : analyse pratique pour un usage documenté", section « Support de
// modèles et choix de quantification »); the project's files were made with an
// importance matrix ("ds4 : un MoE de 284 milliards sur un Mac de 128 Go",
// section « Comment un 284B tient »). The pages give no quantisation algorithm;
// the rules below are this library's own. Every decision (scale, code,
// codebook row) is taken in fp32 with round-to-nearest-even operations that
// are never fused (the __f*_rn intrinsics), in the order the rule states, so
// that any correct implementation of the rule produces the same bytes.
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.cuh"

namespace moe {
namespace {

__device__ const Iq2Codebook d_codebook_q = kCodebook;

__device__ __forceinline__ float clamp_(float v, float lo, float hi) { return fminf(fmaxf(v, lo), hi); }
__device__ __forceinline__ uint16_t f16_rn(float v) { return __half_as_ushort(__float2half_rn(v)); }
__device__ __forceinline__ float f16_f(uint16_t h) { return __half2float(__ushort_as_half(h)); }

// Q2K: one 16-lane half warp per 256-weight block, lane s = sub-block s.
//   lo_s = min(0, min w), hi_s = max w, step_s = (hi_s - lo_s) / 3, off_s = -lo_s;
//   d = fp16(max step / 15), dmin = fp16(max off / 15);
//   sc = clamp(rint(step / d), 0, 15), m = clamp(rint(off / dmin), 0, 15);
//   q = clamp(rint((w + dmin m) / (d sc)), 0, 3).
__global__ void __launch_bounds__(256) quantize_q2k_kernel(const float* __restrict__ w, int64_t nblocks,
                                                           uint8_t* __restrict__ codes, uint32_t* __restrict__ dd) {
  const int lane = threadIdx.x & 31, s = lane & 15;
  const int64_t b = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 4;
  const bool live = b < nblocks;
  const float* x = w + (live ? b : 0) * 256 + 16 * s;
  float v[16];
#pragma unroll
  for (int i = 0; i < 16; i += 4) {
    const float4 t = live ? *reinterpret_cast<const float4*>(x + i) : make_float4(0.f, 0.f, 0.f, 0.f);
    v[i] = t.x; v[i + 1] = t.y; v[i + 2] = t.z; v[i + 3] = t.w;
  }
  // strict comparisons, as the rule is written: a zero of either sign never replaces +0
  float lo = 0.f, hi = v[0];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    lo = v[i] < lo ? v[i] : lo;
    hi = v[i] > hi ? v[i] : hi;
  }
  const float step = __fdiv_rn(__fsub_rn(hi, lo), 3.0f), off = -lo;
  float smax = step > 0.f ? step : 0.f, omax = off > 0.f ? off : 0.f;
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) {  // within the half warp (the maximum is exact in any order)
    const float so = __shfl_xor_sync(0xffffffffu, smax, o), oo = __shfl_xor_sync(0xffffffffu, omax, o);
    smax = so > smax ? so : smax;
    omax = oo > omax ? oo : omax;
  }
  const uint16_t d16 = f16_rn(__fdiv_rn(smax, 15.0f)), m16 = f16_rn(__fdiv_rn(omax, 15.0f));
  const float df = f16_f(d16), mf = f16_f(m16);
  const int sc = df > 0.f ? static_cast<int>(clamp_(rintf(__fdiv_rn(step, df)), 0.f, 15.f)) : 0;
  const int m = mf > 0.f ? static_cast<int>(clamp_(rintf(__fdiv_rn(off, mf)), 0.f, 15.f)) : 0;
  const float st = __fmul_rn(df, static_cast<float>(sc)), of = __fmul_rn(mf, static_cast<float>(m));
  uint32_t qw = 0;  // the sub-block's four q bytes
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int q = st > 0.f ? static_cast<int>(clamp_(rintf(__fdiv_rn(__fadd_rn(v[i], of), st)), 0.f, 3.f)) : 0;
    qw |= static_cast<uint32_t>(q) << (2 * i);  // weight 4j + r at bit 8j + 2r = 2i
  }
  if (!live) return;
  uint8_t* c = codes + b * 80;
  c[s] = static_cast<uint8_t>(sc | (m << 4));
  *reinterpret_cast<uint32_t*>(c + 16 + 4 * s) = qw;
  if (s == 0) dd[b] = static_cast<uint32_t>(d16) | (static_cast<uint32_t>(m16) << 16);
}

// IQ2: one CTA of 8 warps per 256-weight block, warp s = sub-block s.
//   d = fp16(max|w| * 8 / 1333); ls = clamp(rint((max_s|w| * 8 / (d * 43) - 1) / 2), 0, 15);
//   c = d * (2 ls + 1) / 8; per group of 8: signs of w, the smallest |w| flipped
//   when their count is odd; the codebook row of least error
//   sum_e (|w_e| -+ c * grid[r][e])^2 (e ascending), the lower row on ties.
// The 256 rows of a group are split over the lanes (rows l, l + 32, ...); the
// warp minimum is taken on the error's bit pattern (errors are >= 0, so the
// order of the bits is the order of the values), then on the row index.
__global__ void __launch_bounds__(256) quantize_iq2_kernel(const float* __restrict__ w, int64_t nblocks,
                                                           uint8_t* __restrict__ codes, uint16_t* __restrict__ dout) {
  __shared__ float wmax[8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t b = blockIdx.x;
  const float* x = w + b * 256 + 32 * warp;
  const float wl = x[lane];  // this lane's weight of the sub-block
  float smax = fabsf(wl);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, o));
  if (lane == 0) wmax[warp] = smax;
  __syncthreads();
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) amax = fmaxf(amax, wmax[i]);
  const uint16_t d16 = f16_rn(__fdiv_rn(__fmul_rn(amax, 8.0f), 1333.0f));
  const float df = f16_f(d16);
  uint8_t* q = codes + b * 64 + 8 * warp;
  if (warp == 0 && lane == 0) dout[b] = d16;
  if (!(df > 0.f)) {
    if (lane < 8) q[lane] = 0;
    return;
  }
  const float r1 = __fdiv_rn(__fmul_rn(smax, 8.0f), __fmul_rn(df, 43.0f));
  const int ls = static_cast<int>(clamp_(rintf(__fdiv_rn(__fsub_rn(r1, 1.0f), 2.0f)), 0.f, 15.f));
  const float c = __fdiv_rn(__fmul_rn(df, static_cast<float>(2 * ls + 1)), 8.0f);
  uint32_t v = static_cast<uint32_t>(ls) << 28;
  uint32_t rows = 0;  // the four chosen rows, byte j = group j
  for (int j = 0; j < 4; ++j) {
    float a[8];
    int nneg = 0;
    uint32_t negm = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float we = __shfl_sync(0xffffffffu, wl, 8 * j + e);
      a[e] = fabsf(we);
      const bool ng = we < 0.f;
      nneg += ng ? 1 : 0;
      negm |= (ng ? 1u : 0u) << e;
    }
    int flip = -1;
    if (nneg & 1) {
      flip = 0;
#pragma unroll
      for (int e = 1; e < 8; ++e)
        if (a[e] < a[flip]) flip = e;
    }
    uint32_t best_bits = 0xFFFFFFFFu, best_row = 0xFFFFFFFFu;
    for (int i = 0; i < 8; ++i) {
      const int r = lane + 32 * i;
      float err = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float t = __fmul_rn(c, static_cast<float>(d_codebook_q.val[r][e]));
        const float diff = e == flip ? __fadd_rn(a[e], t) : __fsub_rn(a[e], t);
        err = __fadd_rn(err, __fmul_rn(diff, diff));
      }
      const uint32_t eb = __float_as_uint(err);
      if (eb < best_bits) {  // rows ascend within the lane: the first least error is the lowest row
        best_bits = eb;
        best_row = static_cast<uint32_t>(r);
      }
    }
    const uint32_t mbits = __reduce_min_sync(0xffffffffu, best_bits);
    const uint32_t row = __reduce_min_sync(0xffffffffu, best_bits == mbits ? best_row : 0xFFFFFFFFu);
    rows |= row << (8 * j);
    const uint32_t sig = (negm ^ (flip >= 0 ? (1u << flip) : 0u)) & 127u;
    v |= sig << (7 * j);
  }
  if (lane == 0) *reinterpret_cast<uint2*>(q) = make_uint2(rows, v);
}

}  // namespace

int launch_quantize_q2k(const float* w, int64_t nblocks, uint8_t* codes, uint32_t* dd, cudaStream_t st) {
  const int64_t threads = nblocks * 16;
  quantize_q2k_kernel<<<static_cast<unsigned>((threads + 255) / 256), 256, 0, st>>>(w, nblocks, codes, dd);
  return cudaGetLastError() == cudaSuccess ? OK : ERR_CUDA;
}

int launch_quantize_iq2(const float* w, int64_t nblocks, uint8_t* codes, uint16_t* d, cudaStream_t st) {
  quantize_iq2_kernel<<<static_cast<unsigned>(nblocks), 256, 0, st>>>(w, nblocks, codes, d);
  return cudaGetLastError() == cudaSuccess ? OK : ERR_CUDA;
}

}  // namespace moe
