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
#include "ptx.cuh"
#include "profile.cuh"

namespace moe {

__device__ __forceinline__ void bf16x8(const uint4 w, float (&f)[8]) {
  f[0] = __uint_as_float(w.x << 16); f[1] = __uint_as_float(w.x & 0xFFFF0000u);
  f[2] = __uint_as_float(w.y << 16); f[3] = __uint_as_float(w.y & 0xFFFF0000u);
  f[4] = __uint_as_float(w.z << 16); f[5] = __uint_as_float(w.z & 0xFFFF0000u);
  f[6] = __uint_as_float(w.w << 16); f[7] = __uint_as_float(w.w & 0xFFFF0000u);
}

template <typename XT>
__device__ __forceinline__ void load_x8(const XT* x, size_t i, float (&f)[8]) {
  if constexpr (sizeof(XT) == 4) {
    const float4 a = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(x) + i);
    const float4 b = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(x) + i + 4);
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
  } else {
    bf16x8(*reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(x) + i), f);
  }
}

// ---------------------------------------------------------------------------
// Logits for few tokens: one CTA per (expert, group of TT tokens), 128 threads,
// each thread holding all of its 16-byte slices of the expert's router row in
// flight at once. Partial sums combine in a fixed order (deterministic).
template <typename XT, int TT>
__global__ void __launch_bounds__(128) router_logits_small_kernel(const uint16_t* __restrict__ Wr,
                                                                  const float* __restrict__ bias,
                                                                  const XT* __restrict__ x, int T, int H, int E,
                                                                  float* __restrict__ logits, int* clear_word) {
  constexpr int MAXJ = 16;  // H <= 16 * 1024
  __shared__ float part[4][TT];
  const int e = blockIdx.y;
  const int t0 = blockIdx.x * TT;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nj = H / 1024 + ((H % 1024) ? 1 : 0);
  pdl_trigger();
  uint4 wv[MAXJ];
#pragma unroll
  for (int j = 0; j < MAXJ; ++j) {
    const int c = tid * 8 + j * 1024;
    wv[j] = (j < nj && c < H) ? *reinterpret_cast<const uint4*>(Wr + static_cast<size_t>(e) * H + c)
                              : make_uint4(0u, 0u, 0u, 0u);
  }
  // the router weights are constants; x and the logits belong to the step
  pdl_wait();
  if (clear_word && blockIdx.x == 0 && blockIdx.y == 0 && tid == 0) *clear_word = 0;  // first kernel of a call
  float acc[TT];
#pragma unroll
  for (int t = 0; t < TT; ++t) acc[t] = 0.f;
  if constexpr (TT == 1 && sizeof(XT) == 2) {  // one bf16 token: all activation slices in flight at once
    uint4 xv[MAXJ];
#pragma unroll
    for (int j = 0; j < MAXJ; ++j) {
      const int c = tid * 8 + j * 1024;
      xv[j] = (j < nj && c < H && t0 < T)
                  ? *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(x) + static_cast<size_t>(t0) * H + c)
                  : make_uint4(0u, 0u, 0u, 0u);
    }
    float a = 0.f;
#pragma unroll
    for (int j = 0; j < MAXJ; ++j) {
      const int c = tid * 8 + j * 1024;
      if (j >= nj || c >= H) break;
      float w8[8], x8[8];
      bf16x8(wv[j], w8);
      bf16x8(xv[j], x8);
#pragma unroll
      for (int i = 0; i < 8; ++i) a = fmaf(w8[i], x8[i], a);
    }
    acc[0] = a;
  } else {
#pragma unroll
  for (int j = 0; j < MAXJ; ++j) {
    const int c = tid * 8 + j * 1024;
    if (j >= nj || c >= H) break;
    float w8[8];
    bf16x8(wv[j], w8);
#pragma unroll
    for (int t = 0; t < TT; ++t) {
      if (t0 + t >= T) break;
      float x8[8];
      load_x8(x, static_cast<size_t>(t0 + t) * H + c, x8);
      float a = acc[t];
#pragma unroll
      for (int i = 0; i < 8; ++i) a = fmaf(w8[i], x8[i], a);
      acc[t] = a;
    }
  }
  }
#pragma unroll
  for (int t = 0; t < TT; ++t) {
    float a = acc[t];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
    if (lane == 0) part[warp][t] = a;
  }
  __syncthreads();
  if (tid < TT && t0 + tid < T) {
    const float v = ((part[0][tid] + part[1][tid]) + (part[2][tid] + part[3][tid])) + (bias ? bias[e] : 0.f);
    logits[static_cast<size_t>(t0 + tid) * E + e] = v;
  }
}

// Logits for many tokens: one warp per expert, TT tokens per CTA, activations
// staged in shared memory in chunks.
template <typename XT, int TT>
__global__ void __launch_bounds__(256) router_logits_kernel(const uint16_t* __restrict__ Wr,
                                                            const float* __restrict__ bias,
                                                            const XT* __restrict__ x, int T, int H, int E,
                                                            float* __restrict__ logits) {
  constexpr int CH = 1024;
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
      const int tt = i / CH, hh = i % CH;
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
        float w8[8];
        bf16x8(*reinterpret_cast<const uint4*>(Wr + (size_t)e * H + h0 + c), w8);
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
// Top-k of one token by one warp: lane l holds the logits of experts l, l+32,
// ... in registers (EPL per lane); k rounds of a warp argmax (ties to the lower
// expert index) with a per-lane bitmask of taken entries. Weights:
// exp(l_j - l_0) / sum_i exp(l_i - l_0), summed in slot order by lane 0.
template <int EPL>
__device__ __forceinline__ void topk_warp(const float* __restrict__ lrow, int E, int k, int32_t* idx_out,
                                          float* w_out, int32_t* idx_smem) {
  const int lane = threadIdx.x & 31;
  float l[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    const int e = lane + 32 * i;
    const float v = e < E ? lrow[e] : -INFINITY;
    l[i] = v == v ? v : -INFINITY;  // a NaN logit ranks last, so every index stays valid
  }
  uint32_t taken = 0;
  float chosen[16];
  int chosen_idx[16];
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !((taken >> i) & 1u) && (l[i] > bv || (l[i] == bv && e < bi))) {
        bv = l[i];
        bi = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
    }
    chosen[j] = bv;
    chosen_idx[j] = bi;
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
  }
  if (lane == 0) {
    float z = 0.f;
    for (int j = 0; j < k; ++j) z += expf(chosen[j] - chosen[0]);
    for (int j = 0; j < k; ++j) {
      idx_out[j] = chosen_idx[j];
      w_out[j] = expf(chosen[j] - chosen[0]) / z;
      if (idx_smem) idx_smem[j] = chosen_idx[j];
    }
  }
}

template <int EPL>
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ logits, int T, int E, int k,
                                                   int32_t* __restrict__ topk_idx, float* __restrict__ topk_w) {
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (t >= T) return;
  topk_warp<EPL>(logits + static_cast<size_t>(t) * E, E, k, topk_idx + static_cast<size_t>(t) * k,
                 topk_w + static_cast<size_t>(t) * k, nullptr);
}

// ---------------------------------------------------------------------------
// Block-wide exclusive scan over 1024 threads (one value each).
__device__ __forceinline__ int block_exclusive_scan_1024(int v, int* warp_sums, int* total) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int s = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, s, o);
    if (lane >= o) s += n;
  }
  if (lane == 31) warp_sums[warp] = s;
  __syncthreads();
  if (warp == 0) {
    const int w = warp_sums[lane];
    int ws = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, ws, o);
      if (lane >= o) ws += n;
    }
    warp_sums[lane] = ws - w;  // exclusive
    if (lane == 31) *total = ws;
  }
  __syncthreads();
  const int r = s - v + warp_sums[warp];
  __syncthreads();
  return r;
}

// Histogram + exclusive scan + stable scatter by one CTA of 1024 threads, plus
// the compacted list of experts that received at least one assignment.
// Stability: assignments are consumed in rounds of 1024 consecutive ids; within
// a round the rank of an assignment among those routed to the same expert is
// (#earlier warps' matches, from a per-warp count table) + (#earlier lanes'
// matches in its own warp, from __match_any_sync). All integer, deterministic.
// smem: 32*E u16 + 3*E int.
__device__ void permute_block(const int32_t* topk_idx, int n, int E, int32_t* __restrict__ offsets,
                              int32_t* __restrict__ perm, int32_t* __restrict__ inv, int32_t* __restrict__ active,
                              uint8_t* smem_raw) {
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
    if (valid && rank_w == 0) cnt[warp * E + e] = static_cast<uint16_t>(__popc(m));
    __syncthreads();
    for (int ee = tid; ee < E; ee += 1024) {  // exclusive prefix over warps, in place
      int s = 0;
      for (int w = 0; w < 32; ++w) {
        const int c = cnt[w * E + ee];
        cnt[w * E + ee] = static_cast<uint16_t>(s);
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

__global__ void __launch_bounds__(1024) permute_kernel(const int32_t* __restrict__ topk_idx, int n, int E,
                                                       int32_t* __restrict__ offsets, int32_t* __restrict__ perm,
                                                       int32_t* __restrict__ inv, int32_t* __restrict__ active) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  permute_block(topk_idx, n, E, offsets, perm, inv, active, smem_raw);
}

// Decode routing in one launch (T*k <= 1024, T <= 32): warp t takes the top-k
// of token t, then the CTA builds the permutation from shared memory.
template <int EPL>
__global__ void __launch_bounds__(1024) topk_permute_kernel(const float* __restrict__ logits, int T, int E, int k,
                                                            int32_t* __restrict__ topk_idx,
                                                            float* __restrict__ topk_w,
                                                            int32_t* __restrict__ offsets,
                                                            int32_t* __restrict__ perm, int32_t* __restrict__ inv,
                                                            int32_t* __restrict__ active) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  int32_t* idx_s = reinterpret_cast<int32_t*>(smem_raw);  // [T*k] <= 1024
  uint8_t* pbuf = smem_raw + 1024 * sizeof(int32_t);
  const int warp = threadIdx.x >> 5;
  if (warp < T)
    topk_warp<EPL>(logits + static_cast<size_t>(warp) * E, E, k, topk_idx + static_cast<size_t>(warp) * k,
                   topk_w + static_cast<size_t>(warp) * k, idx_s + warp * k);
  __syncthreads();
  permute_block(idx_s, T * k, E, offsets, perm, inv, active, pbuf);
}

// Decode routing for few assignments (T*k <= 1024, T <= 32, E <= 1024) in one
// CTA: warp t takes the top-k of token t; then an integer histogram (shared
// atomics, order-independent), one exclusive scan for the offsets, one for the
// active-expert list, and the stable rank of each assignment among the earlier
// ones routed to the same expert by direct counting.
template <int EPL>
__global__ void __launch_bounds__(1024) topk_permute_small_kernel(const float* __restrict__ logits, int T, int E,
                                                                  int k, int32_t* __restrict__ topk_idx,
                                                                  float* __restrict__ topk_w,
                                                                  int32_t* __restrict__ offsets,
                                                                  int32_t* __restrict__ perm, int32_t* __restrict__ inv,
                                                                  int32_t* __restrict__ active) {
  __shared__ int idx_s[1024];
  __shared__ int cnt[1024];
  __shared__ int warp_sums[32];
  __shared__ int total;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int n = T * k;
  pdl_trigger();
  pdl_wait();
  if (tid < E) cnt[tid] = 0;
  if (warp < T)
    topk_warp<EPL>(logits + static_cast<size_t>(warp) * E, E, k, topk_idx + static_cast<size_t>(warp) * k,
                   topk_w + static_cast<size_t>(warp) * k, idx_s + warp * k);
  __syncthreads();
  const int e = tid < n ? idx_s[tid] : 0;
  if (tid < n) atomicAdd(&cnt[e], 1);
  __syncthreads();
  const int c = tid < E ? cnt[tid] : 0;
  const int ex = block_exclusive_scan_1024(c, warp_sums, &total);
  if (tid < E) {
    offsets[tid] = ex;
    cnt[tid] = ex;  // becomes the offset table (each thread rewrites only its own entry)
  }
  if (tid == 0) offsets[E] = n;
  const int flag = (tid < E && c > 0) ? 1 : 0;
  const int pos = block_exclusive_scan_1024(flag, warp_sums, &total);
  if (flag) active[pos] = tid;
  if (tid == 0) active[E] = total;
  if (tid < n) {
    int rank = 0;
    for (int b = 0; b < tid; ++b) rank += idx_s[b] == e ? 1 : 0;
    const int p = cnt[e] + rank;
    perm[p] = tid;
    inv[tid] = p;
  }
}

// Decode routing for at most 32 assignments (T*k <= 32, E <= 32*EPL) in one
// warp: the top-k of each token in turn, then (lane j = assignment j) the
// offsets as counts of smaller expert indices, the stable rank among equal
// experts by match, and the active list by ballot prefix sums. Same outputs
// as topk_permute_small_kernel, without block barriers or shared atomics.
template <int EPL>
__global__ void __launch_bounds__(32) topk_permute_warp_kernel(const float* __restrict__ logits, int T, int E, int k,
                                                               int32_t* __restrict__ topk_idx,
                                                               float* __restrict__ topk_w,
                                                               int32_t* __restrict__ offsets,
                                                               int32_t* __restrict__ perm, int32_t* __restrict__ inv,
                                                               int32_t* __restrict__ active) {
  __shared__ int idx_s[32];
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x;
  const int n = T * k;
  for (int t = 0; t < T; ++t)
    topk_warp<EPL>(logits + static_cast<size_t>(t) * E, E, k, topk_idx + static_cast<size_t>(t) * k,
                   topk_w + static_cast<size_t>(t) * k, idx_s + t * k);
  __syncwarp();
  const int e = lane < n ? idx_s[lane] : 0x7fffffff;  // above every expert index
  // assignment j: position = (assignments with a smaller expert) + (earlier ones with the same expert)
  int below = 0;
  for (int j = 0; j < n; ++j) below += __shfl_sync(0xffffffffu, e, j) < e ? 1 : 0;
  const unsigned same = __match_any_sync(0xffffffffu, e);
  const int p = below + __popc(same & ((1u << lane) - 1u));
  if (lane < n) {
    perm[p] = lane;
    inv[lane] = p;
  }
  // offsets[x] for x = 0..E and the ascending list of experts with at least one assignment
  int nact = 0;
  for (int base = 0; base <= E; base += 32) {
    const int x = base + lane;
    int lt = 0, eq = 0;
    for (int j = 0; j < n; ++j) {
      const int ej = __shfl_sync(0xffffffffu, e, j);
      lt += ej < x ? 1 : 0;
      eq += ej == x ? 1 : 0;
    }
    if (x <= E) offsets[x] = x == E ? n : lt;
    const bool has = x < E && eq > 0;
    const unsigned m = __ballot_sync(0xffffffffu, has);
    if (has) active[nact + __popc(m & ((1u << lane) - 1u))] = x;
    nact += __popc(m);
  }
  if (lane == 0) active[E] = nact;
}

// The same outputs for T * k <= 32, k <= 32 and T * ceil(E / 32) <= 32 by one
// CTA of T * ceil(E / 32) warps. Order: larger logit first, equal logits by
// lower expert index (NaN ranks as -inf, padding after every expert). Warp w of
// token t sorts experts 32w..32w+31 with a bitonic network of shuffles; its
// first min(k, 32) are the only ones that can be among the token's k, and
// among those candidates each counts the ones ranked above it: the k with a
// count below k write themselves into their slot. The weights are summed in
// slot order by one thread per token, as in topk_warp. The permutation is
// computed in parallel from the chosen experts in shared memory: assignment j
// goes to (assignments with a smaller expert) + (earlier ones with the same
// expert), offsets[x] counts the assignments below x, and the first assignment
// of each distinct expert writes it into the active list at the number of
// distinct experts below it.
__device__ __forceinline__ bool ranks_before(float av, int ai, float bv, int bi) {
  return av > bv || (av == bv && ai < bi);
}

__global__ void __launch_bounds__(1024) topk_permute_sort_kernel(const float* __restrict__ logits, int T, int E, int k,
                                                                 int32_t* __restrict__ topk_idx,
                                                                 float* __restrict__ topk_w,
                                                                 int32_t* __restrict__ offsets,
                                                                 int32_t* __restrict__ perm,
                                                                 int32_t* __restrict__ inv,
                                                                 int32_t* __restrict__ active) {
  __shared__ float cand_v[1024];
  __shared__ int cand_i[1024];
  __shared__ int sel[32];
  __shared__ float chosen[32];
  __shared__ float ex[32];
  __shared__ int first[32];
  pdl_trigger();
  pdl_wait();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int W = (E + 31) / 32, kc = k < 32 ? k : 32, n = T * k;
  const int t = warp / W, e = (warp - t * W) * 32 + lane;
  float v = -INFINITY;
  int idx = E + lane;  // padding ranks after every expert
  if (e < E) {
    const float l = logits[static_cast<size_t>(t) * E + e];
    v = l == l ? l : -INFINITY;
    idx = e;
  }
  // bitonic sort of the warp's 32 keys into rank order
#pragma unroll
  for (int kk = 2; kk <= 32; kk <<= 1) {
#pragma unroll
    for (int j = kk >> 1; j > 0; j >>= 1) {
      const float pv = __shfl_xor_sync(0xffffffffu, v, j);
      const int pi = __shfl_xor_sync(0xffffffffu, idx, j);
      const bool p_first = ranks_before(pv, pi, v, idx);
      const bool lower = (lane & j) == 0, fwd = (lane & kk) == 0;
      // in a forward block the lower lane keeps the key that ranks first
      if (lower == fwd ? p_first : !p_first) {
        v = pv;
        idx = pi;
      }
    }
  }
  const int wt = warp - t * W;  // warp within the token
  if (lane < kc) {
    cand_v[t * W * kc + wt * kc + lane] = v;
    cand_i[t * W * kc + wt * kc + lane] = idx;
  }
  __syncthreads();
  {
    const int nc = W * kc;  // candidates of a token
    const int ct = tid / nc, c = tid - ct * nc;
    if (ct < T) {
      const float* cv = cand_v + ct * nc;
      const int* ci = cand_i + ct * nc;
      const float mv = cv[c];
      const int mi = ci[c];
      int rank = 0;
#pragma unroll 8
      for (int j = 0; j < nc; ++j) rank += ranks_before(cv[j], ci[j], mv, mi) ? 1 : 0;
      if (rank < k) {
        sel[ct * k + rank] = mi;
        chosen[ct * k + rank] = mv;
      }
    }
  }
  __syncthreads();
  // exp(l_j - l_0) of every chosen slot at once; then each slot's thread forms its token's sum in slot
  // order (the same sum in every thread of the token) and writes its own weight
  if (tid < n) ex[tid] = expf(chosen[tid] - chosen[(tid / k) * k]);
  __syncthreads();
  if (tid < n) {
    const int t0 = (tid / k) * k;
    float z = 0.f;
    for (int j = 0; j < k; ++j) z += ex[t0 + j];
    topk_idx[tid] = sel[tid];
    topk_w[tid] = ex[tid] / z;
  }
  if (tid < n) {
    const int ej = sel[tid];
    int below = 0, fst = 1;
#pragma unroll 8
    for (int j = 0; j < n; ++j) {
      const int ei = sel[j];
      below += (ei < ej || (ei == ej && j < tid)) ? 1 : 0;
      if (ei == ej && j < tid) fst = 0;
    }
    perm[below] = tid;
    inv[tid] = below;
    first[tid] = fst;
  }
  __syncthreads();
  for (int x = tid; x <= E; x += blockDim.x) {
    int lt = 0;
#pragma unroll 8
    for (int j = 0; j < n; ++j) lt += sel[j] < x ? 1 : 0;
    offsets[x] = x == E ? n : lt;
  }
  if (tid < n && first[tid]) {
    const int ej = sel[tid];
    int pos = 0;
#pragma unroll 8
    for (int j = 0; j < n; ++j) pos += (first[j] && sel[j] < ej) ? 1 : 0;
    active[pos] = ej;
  }
  if (tid == 0) {
    int nact = 0;
#pragma unroll 8
    for (int j = 0; j < n; ++j) nact += first[j];
    active[E] = nact;
  }
}

// Active-expert list from caller-provided offsets (used by moe_expert_ffn).
__global__ void __launch_bounds__(1024) active_from_offsets_kernel(const int32_t* __restrict__ offsets, int E,
                                                                   int32_t* __restrict__ active) {
  __shared__ int warp_sums[32];
  __shared__ int total;
  const int tid = threadIdx.x;
  const int flag = (tid < E && offsets[tid + 1] > offsets[tid]) ? 1 : 0;
  const int pos = block_exclusive_scan_1024(flag, warp_sums, &total);
  if (flag) active[pos] = tid;
  if (tid == 0) active[E] = total;
}

// ---------------------------------------------------------------------------
template <typename K>
static void set_smem(K kernel, size_t bytes) {
  if (bytes > 48 * 1024) cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

int launch_route(const uint16_t* Wr, const float* bias, const void* x, int x_dtype, int T, int H, int E, int k,
                 float* logits, int32_t* topk_idx, float* topk_w, int32_t* offsets, int32_t* perm, int32_t* inv,
                 int32_t* active, int* err, cudaStream_t st, bool clear_status) {
  {
    ProfScope ps(MOE_K_ROUTER_LOGITS, st);
    if (x_dtype == 1 && router_tc_supported(T, H, E)) {
      int dev = 0, sms = 0;
      cudaGetDevice(&dev);
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
      const int rc = launch_router_tc(Wr, bias, static_cast<const uint16_t*>(x), T, H, E, logits, err,
                                      sms > 0 ? sms : 148, st);
      if (rc != OK) return rc;
    } else if (T == 1 && x_dtype == 1) {
      launch_pdl(router_logits_small_kernel<uint16_t, 1>, dim3(1, E), dim3(128), 0, st, Wr, bias,
                 static_cast<const uint16_t*>(x), T, H, E, logits, clear_status ? err : nullptr);
    } else if (T <= 64) {
      constexpr int TT = 4;
      dim3 g((T + TT - 1) / TT, E);
      if (x_dtype == 0)
        launch_pdl(router_logits_small_kernel<float, TT>, g, dim3(128), 0, st, Wr, bias,
                   static_cast<const float*>(x), T, H, E, logits, clear_status ? err : nullptr);
      else
        launch_pdl(router_logits_small_kernel<uint16_t, TT>, g, dim3(128), 0, st, Wr, bias,
                   static_cast<const uint16_t*>(x), T, H, E, logits, clear_status ? err : nullptr);
    } else {
      constexpr int TT = 8;
      dim3 g((T + TT - 1) / TT, (E + 7) / 8);
      if (x_dtype == 0)
        router_logits_kernel<float, TT><<<g, 256, 0, st>>>(Wr, bias, static_cast<const float*>(x), T, H, E, logits);
      else
        router_logits_kernel<uint16_t, TT><<<g, 256, 0, st>>>(Wr, bias, static_cast<const uint16_t*>(x), T, H, E,
                                                              logits);
    }
  }
  const size_t psmem = 32 * E * sizeof(uint16_t) + 3 * E * sizeof(int);
  if (T * k <= 32 && k <= 32 && T * ((E + 31) / 32) <= 32) {
    ProfScope ps(MOE_K_PERMUTE, st);
    launch_pdl(topk_permute_sort_kernel, dim3(1), dim3(32 * T * ((E + 31) / 32)), 0, st, logits, T, E, k, topk_idx,
               topk_w, offsets, perm, inv, active);
  } else if (T * k <= 32 && E <= 256) {
    ProfScope ps(MOE_K_PERMUTE, st);
    launch_pdl(topk_permute_warp_kernel<8>, dim3(1), dim3(32), 0, st, logits, T, E, k, topk_idx, topk_w, offsets,
               perm, inv, active);
  } else if (T * k <= 1024 && T <= 32 && E <= 1024) {
    ProfScope ps(MOE_K_PERMUTE, st);
    if (E <= 256)
      launch_pdl(topk_permute_small_kernel<8>, dim3(1), dim3(1024), 0, st, logits, T, E, k, topk_idx, topk_w,
                 offsets, perm, inv, active);
    else
      launch_pdl(topk_permute_small_kernel<32>, dim3(1), dim3(1024), 0, st, logits, T, E, k, topk_idx, topk_w,
                 offsets, perm, inv, active);
  } else if (T * k <= 1024 && T <= 32) {
    ProfScope ps(MOE_K_PERMUTE, st);
    const size_t sm = 1024 * sizeof(int32_t) + psmem;
    if (E <= 256) {
      set_smem(topk_permute_kernel<8>, sm);
      topk_permute_kernel<8><<<1, 1024, sm, st>>>(logits, T, E, k, topk_idx, topk_w, offsets, perm, inv, active);
    } else {
      set_smem(topk_permute_kernel<32>, sm);
      topk_permute_kernel<32><<<1, 1024, sm, st>>>(logits, T, E, k, topk_idx, topk_w, offsets, perm, inv, active);
    }
  } else {
    {
      ProfScope ps(MOE_K_TOPK, st);
      if (E <= 256)
        topk_kernel<8><<<(T + 7) / 8, 256, 0, st>>>(logits, T, E, k, topk_idx, topk_w);
      else
        topk_kernel<32><<<(T + 7) / 8, 256, 0, st>>>(logits, T, E, k, topk_idx, topk_w);
    }
    ProfScope ps(MOE_K_PERMUTE, st);
    set_smem(permute_kernel, psmem);
    permute_kernel<<<1, 1024, psmem, st>>>(topk_idx, T * k, E, offsets, perm, inv, active);
  }
  return cudaGetLastError() == cudaSuccess ? OK : ERR_CUDA;
}

// ids[a] = map[ids[a]] for the n assignments (expert ids -> cache slot ids).
__global__ void __launch_bounds__(256) remap_ids_kernel(int32_t* __restrict__ ids, int n,
                                                        const int32_t* __restrict__ map) {
  const int a = blockIdx.x * blockDim.x + threadIdx.x;
  if (a < n) ids[a] = map[ids[a]];
}

int launch_remap_permute(int32_t* ids, int n, const int32_t* map, int E, int32_t* offsets, int32_t* perm,
                         int32_t* inv, int32_t* active, cudaStream_t st) {
  ProfScope ps(MOE_K_PERMUTE, st);
  remap_ids_kernel<<<(n + 255) / 256, 256, 0, st>>>(ids, n, map);
  const size_t psmem = 32 * E * sizeof(uint16_t) + 3 * E * sizeof(int);
  set_smem(permute_kernel, psmem);
  permute_kernel<<<1, 1024, psmem, st>>>(ids, n, E, offsets, perm, inv, active);
  return cudaGetLastError() == cudaSuccess ? OK : ERR_CUDA;
}

int launch_active_from_offsets(const int32_t* offsets, int E, int32_t* active, cudaStream_t st) {
  ProfScope ps(MOE_K_ACTIVE, st);
  active_from_offsets_kernel<<<1, 1024, 0, st>>>(offsets, E, active);
  return cudaGetLastError() == cudaSuccess ? OK : ERR_CUDA;
}

}  // namespace moe
