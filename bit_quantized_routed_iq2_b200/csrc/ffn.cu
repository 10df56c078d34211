// ffn.cu - routed expert FFN (gate/up dequant-GEMV, SwiGLU, down dequant-GEMV),
// the unquantized shared expert and the weighted combine.
//
// Sources: "ds4 : analyse pratique pour un usage documenté", section « Support de
// modèles et choix de quantification » (routed experts 2-bit: up/gate IQ2_XXS,
// down Q2_K; shared experts unquantized). The expert function (SwiGLU, weighted
// sum of the chosen experts plus the shared expert) is the library's
// specification.
//
// This file holds the straightforward CUDA-core path: one warp per output row,
// lanes striding over 8-weight groups along the reduction axis. It is the path
// for shapes the tuned kernels do not cover and the baseline they are measured
// against.
#include <algorithm>

#include "common.cuh"
#include "dequant.cuh"
#include "kernels.cuh"
#include "profile.cuh"

namespace moe {

namespace {

template <typename XT>
__device__ __forceinline__ float load_act(const XT* x, size_t i) {
  if constexpr (sizeof(XT) == 4) return reinterpret_cast<const float*>(x)[i];
  else return bf16_bits_to_float(reinterpret_cast<const uint16_t*>(x)[i]);
}

// 8 IQ2-style weights starting at flattened index f (multiple of 8) of a matrix.
__device__ __forceinline__ void iq2_decode8(const uint32_t* s_grid, const uint8_t* codes, const uint16_t* d,
                                            size_t f, float w[8]) {
  const size_t blk = f / QK;
  const int pos = static_cast<int>(f % QK);
  const int s = pos >> 5, j = (pos >> 3) & 3;
  const uint8_t* c = codes + blk * IQ2_BYTES + 8 * s;
  const uint32_t v = *reinterpret_cast<const uint32_t*>(c + 4);
  const float scale = iq2_scale(half_bits_to_float(d[blk]), v);
  iq2_group(s_grid, c[j], (v >> (7 * j)) & 127u, scale, w);
}

// 8 Q2K-style weights starting at flattened index f (multiple of 8).
__device__ __forceinline__ void q2k_decode8(const uint8_t* codes, const uint32_t* dd, size_t f, float w[8]) {
  const size_t blk = f / QK;
  const int pos = static_cast<int>(f % QK);
  const uint8_t* c = codes + blk * Q2K_BYTES;
  const uint32_t sm = c[pos >> 4];
  const uint32_t pd = dd[blk];
  const float dv = half_bits_to_float(static_cast<uint16_t>(pd & 0xFFFFu));
  const float dm = half_bits_to_float(static_cast<uint16_t>(pd >> 16));
  const uint32_t qb = static_cast<uint32_t>(c[16 + pos / 4]) | static_cast<uint32_t>(c[16 + pos / 4 + 1]) << 8;
#pragma unroll
  for (int i = 0; i < 8; ++i) w[i] = q2k_value(dv, dm, sm & 15u, sm >> 4, (qb >> (2 * i)) & 3u);
}

__device__ __forceinline__ float warp_sum(float a) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
  return a;
}

// gate/up for every assignment of one active expert and 32 rows of I.
template <typename XT>
__global__ void __launch_bounds__(256) gateup_simple_kernel(LayerShape s, const uint8_t* __restrict__ gate_codes,
                                                            const uint16_t* __restrict__ gate_d,
                                                            const uint8_t* __restrict__ up_codes,
                                                            const uint16_t* __restrict__ up_d,
                                                            const XT* __restrict__ x, Routing r,
                                                            float* __restrict__ hbuf) {
  __shared__ uint32_t s_grid[512];
  load_grid_smem(s_grid);
  __syncthreads();
  const int slot = blockIdx.x;
  if (slot >= r.active[s.E]) return;
  const int e = r.active[slot];
  const int p0 = r.offsets[e], p1 = r.offsets[e + 1];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t nb = static_cast<size_t>(s.I) * s.H / QK;
  const uint8_t* gc = gate_codes + e * nb * IQ2_BYTES;
  const uint8_t* uc = up_codes + e * nb * IQ2_BYTES;
  const uint16_t* gd = gate_d + e * nb;
  const uint16_t* ud = up_d + e * nb;
  for (int i = 0; i < 4; ++i) {
    const int row = blockIdx.y * 32 + warp * 4 + i;
    if (row >= s.I) break;
    for (int p = p0; p < p1; ++p) {
      const size_t t = static_cast<size_t>(r.perm[p] / s.k);
      float g = 0.f, u = 0.f;
      for (int grp = lane; grp < s.H / 8; grp += 32) {
        const size_t f = static_cast<size_t>(row) * s.H + 8 * grp;
        float wg[8], wu[8];
        iq2_decode8(s_grid, gc, gd, f, wg);
        iq2_decode8(s_grid, uc, ud, f, wu);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float xv = load_act(x, t * s.H + 8 * grp + q);
          g = fmaf(wg[q], xv, g);
          u = fmaf(wu[q], xv, u);
        }
      }
      g = warp_sum(g);
      u = warp_sum(u);
      if (lane == 0) hbuf[static_cast<size_t>(p) * s.I + row] = silu_mul(g, u);
    }
  }
}

// down for every assignment of one active expert and 32 rows of H.
__global__ void __launch_bounds__(256) down_simple_kernel(LayerShape s, const uint8_t* __restrict__ down_codes,
                                                          const uint32_t* __restrict__ down_dd, Routing r,
                                                          const float* __restrict__ hbuf, float* __restrict__ obuf) {
  const int slot = blockIdx.x;
  if (slot >= r.active[s.E]) return;
  const int e = r.active[slot];
  const int p0 = r.offsets[e], p1 = r.offsets[e + 1];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t nb = static_cast<size_t>(s.I) * s.H / QK;
  const uint8_t* dc = down_codes + e * nb * Q2K_BYTES;
  const uint32_t* ddd = down_dd + e * nb;
  for (int i = 0; i < 4; ++i) {
    const int row = blockIdx.y * 32 + warp * 4 + i;
    if (row >= s.H) break;
    for (int p = p0; p < p1; ++p) {
      const float* h = hbuf + static_cast<size_t>(p) * s.I;
      float acc = 0.f;
      for (int grp = lane; grp < s.I / 8; grp += 32) {
        const size_t f = static_cast<size_t>(row) * s.I + 8 * grp;
        float w[8];
        q2k_decode8(dc, ddd, f, w);
#pragma unroll
        for (int q = 0; q < 8; ++q) acc = fmaf(w[q], h[8 * grp + q], acc);
      }
      acc = warp_sum(acc);
      if (lane == 0) obuf[static_cast<size_t>(p) * s.H + row] = acc;
    }
  }
}

// Shared expert gate/up: hs[t][row] = silu(Wsg x_t)[row] * (Wsu x_t)[row].
template <typename XT>
__global__ void __launch_bounds__(256) shared_gateup_simple_kernel(LayerShape s, const uint16_t* __restrict__ sg,
                                                                   const uint16_t* __restrict__ su,
                                                                   const XT* __restrict__ x, int T,
                                                                   float* __restrict__ hs) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = 0; i < 4; ++i) {
    const int row = blockIdx.x * 32 + warp * 4 + i;
    if (row >= s.Is) break;
    for (int t = 0; t < T; ++t) {
      float g = 0.f, u = 0.f;
      for (int c = lane; c < s.H; c += 32) {
        const float xv = load_act(x, static_cast<size_t>(t) * s.H + c);
        g = fmaf(bf16_bits_to_float(sg[static_cast<size_t>(row) * s.H + c]), xv, g);
        u = fmaf(bf16_bits_to_float(su[static_cast<size_t>(row) * s.H + c]), xv, u);
      }
      g = warp_sum(g);
      u = warp_sum(u);
      if (lane == 0) hs[static_cast<size_t>(t) * s.Is + row] = silu_mul(g, u);
    }
  }
}

__global__ void __launch_bounds__(256) shared_down_simple_kernel(LayerShape s, const uint16_t* __restrict__ sd,
                                                                 const float* __restrict__ hs, int T,
                                                                 float* __restrict__ sbuf) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = 0; i < 4; ++i) {
    const int row = blockIdx.x * 32 + warp * 4 + i;
    if (row >= s.H) break;
    for (int t = 0; t < T; ++t) {
      float acc = 0.f;
      for (int c = lane; c < s.Is; c += 32)
        acc = fmaf(bf16_bits_to_float(sd[static_cast<size_t>(row) * s.Is + c]), hs[static_cast<size_t>(t) * s.Is + c],
                   acc);
      acc = warp_sum(acc);
      if (lane == 0) sbuf[static_cast<size_t>(t) * s.H + row] = acc;
    }
  }
}

// y[t][r] = sum_j w[t][j] * o[inv[t*k+j]][r] (j ascending) + s[t][r] + residual[t][r].
__global__ void __launch_bounds__(256) combine_kernel(LayerShape s, Routing r, const float* __restrict__ obuf,
                                                      const float* __restrict__ sbuf, const float* residual,
                                                      float* y, int T) {
  const int t = blockIdx.x;
  const int row = blockIdx.y * 256 + threadIdx.x;
  if (t >= T || row >= s.H) return;
  float acc = 0.f;
  for (int j = 0; j < s.k; ++j) {
    const int a = t * s.k + j;
    acc = fmaf(r.topk_w[a], obuf[static_cast<size_t>(r.inv[a]) * s.H + row], acc);
  }
  if (sbuf) acc += sbuf[static_cast<size_t>(t) * s.H + row];
  if (residual) acc += residual[static_cast<size_t>(t) * s.H + row];
  y[static_cast<size_t>(t) * s.H + row] = acc;
}

// ----------------------------------------------------------- debug dequant
__global__ void debug_dequant_iq2_kernel(const uint8_t* __restrict__ codes, const uint16_t* __restrict__ d,
                                         int64_t nblocks, float* __restrict__ out) {
  __shared__ uint32_t s_grid[512];
  load_grid_smem(s_grid);
  __syncthreads();
  const int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;  // group id
  if (g >= nblocks * 32) return;
  float w[8];
  iq2_decode8(s_grid, codes, d, static_cast<size_t>(g) * 8, w);
  float4* o = reinterpret_cast<float4*>(out + g * 8);
  o[0] = make_float4(w[0], w[1], w[2], w[3]);
  o[1] = make_float4(w[4], w[5], w[6], w[7]);
}

__global__ void debug_dequant_q2k_kernel(const uint8_t* __restrict__ codes, const uint32_t* __restrict__ dd,
                                         int64_t nblocks, float* __restrict__ out) {
  const int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (g >= nblocks * 32) return;
  float w[8];
  q2k_decode8(codes, dd, static_cast<size_t>(g) * 8, w);
  float4* o = reinterpret_cast<float4*>(out + g * 8);
  o[0] = make_float4(w[0], w[1], w[2], w[3]);
  o[1] = make_float4(w[4], w[5], w[6], w[7]);
}

}  // namespace

// Workspace of the CUDA-core FFN stage: h [T*k][I], o [T*k][H], shared h [T][Is], s [T][H].
static size_t simple_ffn_workspace_bytes(const LayerShape& s, int T) {
  const size_t nA = static_cast<size_t>(T) * s.k;
  size_t b = 0;
  b += align_up(nA * s.I * 4, 256);
  b += align_up(nA * s.H * 4, 256);
  b += align_up(static_cast<size_t>(T) * (s.Is > 0 ? s.Is : 1) * 4, 256);
  b += align_up(static_cast<size_t>(T) * s.H * 4, 256);
  return b;
}

// Token counts above the decode GEMVs' range go through the tensor-core grouped
// GEMM (prefill.cu) when the shape allows it.
bool use_prefill(const LayerShape& s, int T) { return T > kPrefillMinT && prefill_path_supported(s, T); }

size_t ffn_workspace_bytes(const LayerShape& s, int T) {
  size_t b = fast_path_supported(s) ? fast_ffn_workspace_bytes(s, T) : simple_ffn_workspace_bytes(s, T);
  if (use_prefill(s, T)) b = std::max(b, prefill_workspace_bytes(s, T));
  return b;
}

static int launch_ffn_simple(const LayerShape& s, const WeightPtrs& w, const void* x, int x_dtype, int T,
                             const Routing& r, const float* residual, float* y, void* ws, cudaStream_t st) {
  const size_t nA = static_cast<size_t>(T) * s.k;
  char* p = static_cast<char*>(ws);
  float* hbuf = reinterpret_cast<float*>(p);
  p += align_up(nA * s.I * 4, 256);
  float* obuf = reinterpret_cast<float*>(p);
  p += align_up(nA * s.H * 4, 256);
  float* hs = reinterpret_cast<float*>(p);
  p += align_up(static_cast<size_t>(T) * (s.Is > 0 ? s.Is : 1) * 4, 256);
  float* sbuf = reinterpret_cast<float*>(p);

  const int slots = static_cast<int>(nA < static_cast<size_t>(s.E) ? nA : s.E);
  dim3 g1(slots, (s.I + 31) / 32);
  {
    ProfScope ps(MOE_K_GATEUP, st);
    if (x_dtype == 0)
      gateup_simple_kernel<float><<<g1, 256, 0, st>>>(s, w.gate_codes, w.gate_d, w.up_codes, w.up_d,
                                                      static_cast<const float*>(x), r, hbuf);
    else
      gateup_simple_kernel<uint16_t><<<g1, 256, 0, st>>>(s, w.gate_codes, w.gate_d, w.up_codes, w.up_d,
                                                         static_cast<const uint16_t*>(x), r, hbuf);
  }
  dim3 g2(slots, (s.H + 31) / 32);
  {
    ProfScope ps(MOE_K_DOWN, st);
    down_simple_kernel<<<g2, 256, 0, st>>>(s, w.down_codes, w.down_dd, r, hbuf, obuf);
  }
  if (s.Is > 0) {
    {
      ProfScope ps(MOE_K_SHARED_GATEUP, st);
      if (x_dtype == 0)
        shared_gateup_simple_kernel<float><<<(s.Is + 31) / 32, 256, 0, st>>>(s, w.sh_gate, w.sh_up,
                                                                           static_cast<const float*>(x), T, hs);
      else
        shared_gateup_simple_kernel<uint16_t><<<(s.Is + 31) / 32, 256, 0, st>>>(
            s, w.sh_gate, w.sh_up, static_cast<const uint16_t*>(x), T, hs);
    }
    ProfScope ps(MOE_K_SHARED_DOWN, st);
    shared_down_simple_kernel<<<(s.H + 31) / 32, 256, 0, st>>>(s, w.sh_down, hs, T, sbuf);
  }
  dim3 g3(T, (s.H + 255) / 256);
  {
    ProfScope ps(MOE_K_COMBINE, st);
    combine_kernel<<<g3, 256, 0, st>>>(s, r, obuf, s.Is > 0 ? sbuf : nullptr, residual, y, T);
  }
  return cudaGetLastError() == cudaSuccess ? OK : ERR_CUDA;
}

int launch_ffn(const LayerShape& s, const WeightPtrs& w, const void* x, int x_dtype, int T, const Routing& r,
               const float* residual, float* y, void* ws, int* err, bool clear_status, cudaStream_t st,
               bool shared_early, uint16_t* y_bf16) {
  if (fast_path_supported(s) && !use_prefill(s, T))
    return launch_ffn_fast(s, w, x, x_dtype, T, r, residual, y, ws, err, clear_status, st, shared_early, y_bf16);
  int rc;
  if (use_prefill(s, T)) {
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    rc = launch_ffn_prefill(s, w, x, x_dtype, T, r, residual, y, ws, err, clear_status, sms > 0 ? sms : 148, st);
  } else {
    // the plain kernels have no bounded waits and never write the status word: clear it here, as the first
    // kernel of every other path does
    if (clear_status && err && cudaMemsetAsync(err, 0, sizeof(int), st) != cudaSuccess) return ERR_CUDA;
    rc = launch_ffn_simple(s, w, x, x_dtype, T, r, residual, y, ws, st);
  }
  if (rc == OK && y_bf16) rc = launch_y_to_bf16(y, y_bf16, static_cast<size_t>(T) * s.H, st);
  return rc;
}

int launch_debug_dequant_iq2(const uint8_t* codes, const uint16_t* d, int64_t nblocks, float* out, cudaStream_t st) {
  const int64_t groups = nblocks * 32;
  debug_dequant_iq2_kernel<<<static_cast<unsigned>((groups + 255) / 256), 256, 0, st>>>(codes, d, nblocks, out);
  return cudaGetLastError() == cudaSuccess ? OK : ERR_CUDA;
}

int launch_debug_dequant_q2k(const uint8_t* codes, const uint32_t* dd, int64_t nblocks, float* out,
                             cudaStream_t st) {
  const int64_t groups = nblocks * 32;
  debug_dequant_q2k_kernel<<<static_cast<unsigned>((groups + 255) / 256), 256, 0, st>>>(codes, dd, nblocks, out);
  return cudaGetLastError() == cudaSuccess ? OK : ERR_CUDA;
}

}  // namespace moe
