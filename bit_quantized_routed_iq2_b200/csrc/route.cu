// route.cu - router logits, top-k with renormalised weights, and the stable
// token-to-expert permutation (histogram, scan, scatter).
//
// The router is unquantized ("ds4 : analyse pratique pour un usage documenté",
// section « Support de modèles et choix de quantification ») and picks a few
// experts per token ("Un modèle de 284 milliards de paramètres tourne désormais
// sur un Mac de 128 Go. Qui y perd ?", section « Comment un modèle de 284
// milliards de paramètres tient sur une seule machine »). Its function here is
// the library's specification: logits = x . Wr (+ bias), top-k by logit (ties
// to the lower index), weights = softmax over the chosen k.
#include "common.cuh"
#include "kernels.cuh"
#include "profile.cuh"

namespace moe {

// ---------------------------------------------------------------------------
// Logits: l[t][e] = sum_h x[t][h] * Wr[e][h] (+ b[e]), fp32 accumulation of the
// exact bf16 x bf16 (or fp32 x bf16) products. One warp per expert, TT tokens
// per CTA; lanes read 16-byte slices of the expert's row (coalesced) and the
// tokens' activations from shared memory. The lane partial sums are combined by
// a fixed shuffle tree, so results are deterministic.
template <typename XT, int TT>
__global__ void __launch_bounds__(256) router_logits_kernel(const uint16_t* __restrict__ Wr,
                                                            const float* __restrict__ bias,
                                                            const XT* __restrict__ x, int T, int H, int E,
                                                            float* __restrict__ logits) {
  constexpr int CH = 1024;  // activation chunk (elements of H) staged in smem
  __shared__ float xs[TT][CH];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * TT;
  const int e = blockIdx.y * 8 + warp;
  float acc[TT];
#pragma unroll
  for (int i = 0; i < TT; ++i) acc[i] = 0.f;
  for (int h0 = 0; h0 < H; h0 += CH) {
    __syncthreads();
    for (int i = threadIdx.x; i < TT * CH; i += blockDim.x) {
      int tt = i / CH, hh = i % CH;
      float v = 0.f;
      if (t0 + tt < T && h0 + hh < H) {
        if constexpr (sizeof(XT) == 4) v = reinterpret_cast<const float*>(x)[(size_t)(t0 + tt) * H + h0 + hh];
        else v = bf16_bits_to_float(reinterpret_cast<const uint16_t*>(x)[(size_t)(t0 + tt) * H + h0 + hh]);
      }
      xs[tt][hh] = v;
    }
    __syncthreads();
    if (e < E) {
      const int lim = min(CH, H - h0);
      for (int c = lane * 8; c < lim; c += 256) {
        uint4 wv = *reinterpret_cast<const uint4*>(Wr + (size_t)e * H + h0 + c);
        float w8[8];
        w8[0] = __uint_as_float(wv.x << 16); w8[1] = __uint_as_float(wv.x & 0xFFFF0000u);
        w8[2] = __uint_as_float(wv.y << 16); w8[3] = __uint_as_float(wv.y & 0xFFFF0000u);
        w8[4] = __uint_as_float(wv.z << 16); w8[5] = __uint_as_float(wv.z & 0xFFFF0000u);
        w8[6] = __uint_as_float(wv.w << 16); w8[7] = __uint_as_float(wv.w & 0xFFFF0000u);
#pragma unroll
        for (int tt = 0; tt < TT; ++tt) {
          const float4 xa = *reinterpret_cast<const float4*>(&xs[tt][c]);
          const float4 xb = *reinterpret_cast<const float4*>(&xs[tt][c + 4]);
          float a = acc[tt];
          a = fmaf(w8[0], xa.x, a); a = fmaf(w8[1], xa.y, a); a = fmaf(w8[2], xa.z, a); a = fmaf(w8[3], xa.w, a);
          a = fmaf(w8[4], xb.x, a); a = fmaf(w8[5], xb.y, a); a = fmaf(w8[6], xb.z, a); a = fmaf(w8[7], xb.w, a);
          acc[tt] = a;
        }
      }
    }
  }
  if (e >= E) return;
#pragma unroll
  for (int tt = 0; tt < TT; ++tt) {
    float a = acc[tt];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
    if (lane == 0 && t0 + tt < T) logits[(size_t)(t0 + tt) * E + e] = a + (bias ? bias[e] : 0.f);
  }
}

// ---------------------------------------------------------------------------
// Top-k: one warp per token. k rounds of a warp argmax over the logits held in
// shared memory (ties to the lower expert index); the winner is removed by
// writing -inf. Weights: exp(l_j - l_0) / sum_i exp(l_i - l_0), summed in slot
// order by lane 0.
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ logits, int T, int E, int k,
                                                   int32_t* __restrict__ topk_idx, float* __restrict__ topk_w) {
  extern __shared__ float sl[];  // [8 warps][E]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + warp;
  if (t >= T) return;
  float* l = sl + (size_t)warp * E;
  for (int e = lane; e < E; e += 32) l[e] = logits[(size_t)t * E + e];
  __syncwarp();
  float chosen[16];
  int chosen_idx[16];
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    for (int e = lane; e < E; e += 32) {
      float v = l[e];
      if (v > bv || (v == bv && e < bi)) { bv = v; bi = e; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
    }
    chosen[j] = bv;
    chosen_idx[j] = bi;
    if (lane == 0) l[bi] = -INFINITY;
    __syncwarp();
  }
  if (lane == 0) {
    float z = 0.f;
    for (int j = 0; j < k; ++j) z += expf(chosen[j] - chosen[0]);
    for (int j = 0; j < k; ++j) {
      topk_idx[(size_t)t * k + j] = chosen_idx[j];
      topk_w[(size_t)t * k + j] = expf(chosen[j] - chosen[0]) / z;
    }
  }
}

// ---------------------------------------------------------------------------
// Block-wide exclusive scan over 1024 threads (one value each).
__device__ __forceinline__ int block_exclusive_scan_1024(int v, int* warp_sums, int* total) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int s = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int n = __shfl_up_sync(0xffffffffu, s, o);
    if (lane >= o) s += n;
  }
  if (lane == 31) warp_sums[warp] = s;
  __syncthreads();
  if (warp == 0) {
    int w = warp_sums[lane];
    int ws = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int n = __shfl_up_sync(0xffffffffu, ws, o);
      if (lane >= o) ws += n;
    }
    warp_sums[lane] = ws - w;  // exclusive
    if (lane == 31) *total = ws;
  }
  __syncthreads();
  int r = s - v + warp_sums[warp];
  __syncthreads();
  return r;
}

// Histogram + exclusive scan + stable scatter in one CTA of 1024 threads, plus
// the compacted list of experts that received at least one assignment.
// Stability: assignments are consumed in rounds of 1024 consecutive ids; within
// a round the rank of an assignment among those routed to the same expert is
// (#earlier warps' matches, from a per-warp count table) + (#earlier lanes'
// matches in its own warp, from __match_any_sync). All integer, deterministic.
__global__ void __launch_bounds__(1024) permute_kernel(const int32_t* __restrict__ topk_idx, int n, int E,
                                                       int32_t* __restrict__ offsets, int32_t* __restrict__ perm,
                                                       int32_t* __restrict__ inv, int32_t* __restrict__ active) {
  extern __shared__ uint8_t smem_raw[];
  uint16_t* cnt = reinterpret_cast<uint16_t*>(smem_raw);  // [32][E] per-round per-warp counts
  int* run = reinterpret_cast<int*>(cnt + 32 * E);        // [E] assignments placed so far
  int* off = run + E;                                     // [E] offsets
  int* rt = off + E;                                      // [E] this round's totals
  __shared__ int warp_sums[32];
  __shared__ int total;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  for (int e = tid; e < E; e += 1024) run[e] = 0;
  for (int i = tid; i < 32 * E; i += 1024) cnt[i] = 0;
  __syncthreads();
  for (int a = tid; a < n; a += 1024) atomicAdd(&run[topk_idx[a]], 1);  // histogram (integer)
  __syncthreads();
  {
    const int c = tid < E ? run[tid] : 0;
    const int ex = block_exclusive_scan_1024(c, warp_sums, &total);
    if (tid < E) { off[tid] = ex; offsets[tid] = ex; }
    if (tid == 0) offsets[E] = n;
    const int flag = (tid < E && c > 0) ? 1 : 0;
    const int pos = block_exclusive_scan_1024(flag, warp_sums, &total);
    if (flag) active[pos] = tid;
    if (tid == 0) active[E] = total;
  }
  for (int e = tid; e < E; e += 1024) run[e] = 0;
  __syncthreads();
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int base = 0; base < n; base += 1024) {
    const int a = base + tid;
    const bool valid = a < n;
    const int e = valid ? topk_idx[a] : E;  // E is a sentinel, never a real expert
    const unsigned m = __match_any_sync(0xffffffffu, e);
    const int rank_w = __popc(m & lt_mask);
    if (valid && rank_w == 0) cnt[warp * E + e] = (uint16_t)__popc(m);
    __syncthreads();
    for (int ee = tid; ee < E; ee += 1024) {  // exclusive prefix over warps, in place
      int s = 0;
      for (int w = 0; w < 32; ++w) {
        const int c = cnt[w * E + ee];
        cnt[w * E + ee] = (uint16_t)s;
        s += c;
      }
      rt[ee] = s;
    }
    __syncthreads();
    if (valid) {
      const int p = off[e] + run[e] + cnt[warp * E + e] + rank_w;
      perm[p] = a;
      inv[a] = p;
    }
    __syncthreads();
    for (int ee = tid; ee < E; ee += 1024) {
      run[ee] += rt[ee];
      for (int w = 0; w < 32; ++w) cnt[w * E + ee] = 0;
    }
    __syncthreads();
  }
}

// Active-expert list from caller-provided offsets (used by moe_expert_ffn).
__global__ void __launch_bounds__(1024) active_from_offsets_kernel(const int32_t* __restrict__ offsets, int E,
                                                                   int32_t* __restrict__ active) {
  __shared__ int warp_sums[32];
  __shared__ int total;
  const int tid = threadIdx.x;
  int flag = (tid < E && offsets[tid + 1] > offsets[tid]) ? 1 : 0;
  int pos = block_exclusive_scan_1024(flag, warp_sums, &total);
  if (flag) active[pos] = tid;
  if (tid == 0) active[E] = total;
}

// ---------------------------------------------------------------------------
int launch_route(const uint16_t* Wr, const float* bias, const void* x, int x_dtype, int T, int H, int E, int k,
                 float* logits, int32_t* topk_idx, float* topk_w, int32_t* offsets, int32_t* perm, int32_t* inv,
                 int32_t* active, cudaStream_t st) {
  constexpr int TT = 8;
  dim3 g1((T + TT - 1) / TT, (E + 7) / 8);
  {
    ProfScope ps(MOE_K_ROUTER_LOGITS, st);
    if (x_dtype == 0)
      router_logits_kernel<float, TT><<<g1, 256, 0, st>>>(Wr, bias, static_cast<const float*>(x), T, H, E, logits);
    else
      router_logits_kernel<uint16_t, TT><<<g1, 256, 0, st>>>(Wr, bias, static_cast<const uint16_t*>(x), T, H, E,
                                                             logits);
  }
  {
    ProfScope ps(MOE_K_TOPK, st);
    topk_kernel<<<(T + 7) / 8, 256, 8 * E * sizeof(float), st>>>(logits, T, E, k, topk_idx, topk_w);
  }
  const size_t psmem = 32 * E * sizeof(uint16_t) + 3 * E * sizeof(int);
  if (psmem > 48 * 1024)
    cudaFuncSetAttribute(permute_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)psmem);
  {
    ProfScope ps(MOE_K_PERMUTE, st);
    permute_kernel<<<1, 1024, psmem, st>>>(topk_idx, T * k, E, offsets, perm, inv, active);
  }
  return cudaGetLastError() == cudaSuccess ? OK : ERR_CUDA;
}

int launch_active_from_offsets(const int32_t* offsets, int E, int32_t* active, cudaStream_t st) {
  ProfScope ps(MOE_K_ACTIVE, st);
  active_from_offsets_kernel<<<1, 1024, 0, st>>>(offsets, E, active);
  return cudaGetLastError() == cudaSuccess ? OK : ERR_CUDA;
}

}  // namespace moe
