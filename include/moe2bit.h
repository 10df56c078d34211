/*
 * moe2bit.h - C ABI of the routed 2-bit MoE FFN layer for NVIDIA B200 (sm_100a).
 *
 * One hot path: for each token, router logits -> top-k experts with
 * renormalised weights -> per expert a SwiGLU FFN whose gate/up weights are in
 * an IQ2_XXS-style 2-bit codebook format and whose down weights are in a
 * Q2_K-style 2-bit format -> weighted combine plus an unquantized shared
 * expert (plus an optional residual).
 *
 * Sources (the ds4 engine pages):
 *   [Q] "ds4 : analyse pratique pour un usage documenté" (hysenlabs.com),
 *       section « Support de modèles et choix de quantification »: only routed
 *       MoE experts are quantized, up/gate in IQ2_XXS and down in Q2_K; shared
 *       experts, projections and routing stay unquantized.
 *   [W] "antirez/ds4 - Moteur local d'inférence DeepSeek V4 Flash pour Metal"
 *       (news.hada.io), section « Poids du modèle »: the same split.
 *   [R] "Un modèle de 284 milliards de paramètres tourne désormais sur un Mac
 *       de 128 Go. Qui y perd ?" (tiblogics.com), section « Comment un modèle de
 *       284 milliards de paramètres tient sur une seule machine »: a router picks
 *       a few experts per token; routed experts hold most of the weights.
 * The pages give no bit layout, no router function and no layer shapes; the
 * layouts, the router function (softmax over the chosen top-k) and the
 * numerics below are this library's specification.
 *
 * Conventions for every call:
 *   - Pointers marked "device" must be device-accessible memory of the current
 *     CUDA device; "host" pointers are ordinary host memory. All buffers are
 *     owned by the caller. The library never allocates or frees device memory
 *     and never synchronises (moe_read_status, a host query, is the one
 *     exception). Work is ordered on `stream`: it starts after the
 *     work already enqueued there and finishes before anything enqueued later.
 *     The whole-layer calls (moe_layer_forward and its variants) may run part
 *     of it on a side stream that they fork from `stream` and join back with
 *     events (created once per device and caller stream, kept for the life of
 *     the process); this is safe inside CUDA graph capture.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *   - Argument and shape errors are detected on the host before anything is
 *     enqueued and are returned as a status; nothing is launched in that case.
 *     A failed launch returns MOE_ERR_CUDA (the CUDA error is left queryable by
 *     cudaGetLastError). Faults in device code surface at the caller's next
 *     synchronisation. No C++ exception crosses this interface.
 *   - Supported shapes: hidden % 256 == 0; inter % 256 == 0 or 256 % inter == 0;
 *     1 <= top_k <= min(n_experts, 16); 1 <= n_experts <= 1024;
 *     shared_inter % 8 == 0 (0 = no shared expert); hidden <= 16384;
 *     inter <= 16384; T >= 0 (T == 0 enqueues nothing and returns MOE_OK).
 *     Anything else returns MOE_ERR_UNSUPPORTED_SHAPE.
 *   - Device pointers must be 16-byte aligned (weights, activations, outputs,
 *     workspace); otherwise MOE_ERR_INVALID_ARG.
 */
#ifndef MOE2BIT_H
#define MOE2BIT_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,         /* null pointer, misaligned pointer, bad dtype */
  MOE_ERR_UNSUPPORTED_SHAPE = 2,   /* shape outside the supported set above */
  MOE_ERR_WORKSPACE_TOO_SMALL = 3, /* ws_bytes < moe_workspace_size(...) */
  MOE_ERR_CUDA = 4,                /* a CUDA runtime call or launch failed */
  MOE_ERR_TIMEOUT = 5              /* a bounded device-side wait gave up */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

/* Layer shape. T (tokens) is passed per call. */
typedef struct {
  int32_t hidden;       /* H: model width, reduction length of gate/up */
  int32_t inter;        /* I: routed expert intermediate width */
  int32_t n_experts;    /* E: routed experts */
  int32_t top_k;        /* k: experts per token */
  int32_t shared_inter; /* I_s: shared expert intermediate width, 0 = none */
} moe_layer_desc;

/*
 * Weights of one layer, all device pointers, read only.
 *
 * Routed expert planes (structure of arrays; blocks run along the reduction
 * axis over the row-major flattened [rows][K] matrix of each expert, so for
 * K < 256 one 256-weight block spans 256/K rows):
 *
 * IQ2-style (gate, up; matrix [I][H] per expert, K = H), per 256-weight block:
 *   codes: 64 bytes. Sub-block s (weights 32s..32s+31) is bytes 8s..8s+7:
 *          bytes 8s+j (j = 0..3) = codebook row of group j (weights 32s+8j..+7);
 *          bytes 8s+4..8s+7 = little-endian u32 v with sign field sigma_j in
 *          bits 7j..7j+6 (bit e set => element e negative, e = 0..6) and the
 *          4-bit scale ls in bits 28..31; element 7 is negative iff
 *          popcount(sigma_j) is odd.
 *   d:     one IEEE fp16 per block.
 *   value: w[32s + 8j + e] = d * (2*ls + 1) * grid[row][e] * sign_e / 8, where
 *          grid is the library's 256 x 8 codebook over {8, 25, 43}: splitmix64
 *          seeded 0x4951325F47524944, c = (next() >> 32) mod 6561, duplicates
 *          rejected, 256 rows in acceptance order, element e = base-3 digit e of
 *          c (least significant first) mapped 0->8, 1->25, 2->43.
 *   plane shapes: codes [E][I*H/256][64] u8, d [E][I*H/256] u16.
 *
 * Q2K-style (down; matrix [H][I] per expert, K = I), per 256-weight block:
 *   codes: 80 bytes. Byte s (0..15) = sub-block s (weights 16s..16s+15) scale
 *          byte, sc = low nibble, m = high nibble. Byte 16+i holds weights
 *          4i..4i+3, weight 4i+r in bits 2r..2r+1 (q = 0..3).
 *   dd:    one u32 per block: fp16 d in bits 0..15, fp16 dmin in bits 16..31.
 *   value: w = d * sc * q - dmin * m.
 *   plane shapes: codes [E][H*I/256][80] u8, dd [E][H*I/256] u32.
 *
 * Router and shared expert (unquantized per [Q], [W]): bf16 bit patterns.
 */
typedef struct {
  const uint16_t* router_w;    /* bf16 [E][H] */
  const float* router_bias;    /* fp32 [E], or NULL; added to the logits */
  const uint8_t* gate_codes;   /* IQ2-style codes [E][I*H/256][64] */
  const uint16_t* gate_d;      /* fp16 [E][I*H/256] */
  const uint8_t* up_codes;     /* IQ2-style codes [E][I*H/256][64] */
  const uint16_t* up_d;        /* fp16 [E][I*H/256] */
  const uint8_t* down_codes;   /* Q2K-style codes [E][H*I/256][80] */
  const uint32_t* down_dd;     /* u32 [E][H*I/256] = fp16 d | fp16 dmin << 16 */
  const uint16_t* sh_gate;     /* bf16 [I_s][H] (unused when I_s == 0) */
  const uint16_t* sh_up;       /* bf16 [I_s][H] */
  const uint16_t* sh_down;     /* bf16 [H][I_s] */
} moe_layer_weights;

/*
 * Workspace bytes needed by moe_route / moe_expert_ffn / moe_layer_forward for
 * any T <= max_tokens. Host only; touches no device. `bytes` is a host pointer.
 */
MOE_API moe_status moe_workspace_size(const moe_layer_desc* desc, int32_t max_tokens, size_t* bytes);

/*
 * Router and permutation ([R]: the router selects a few experts per token; [Q]:
 * it is unquantized).
 *   logits l[t][e] = sum_h x[t][h] * router_w[e][h] (+ router_bias[e]), fp32
 *   accumulation of exact products;
 *   topk_idx[t][j] = the k largest logits, j = 0 the largest, ties to the lower
 *   expert index;
 *   topk_w[t][j] = exp(l_j - l_0) / sum_i exp(l_i - l_0) over the chosen k
 *   (softmax over all experts renormalised over the chosen ones);
 *   assignment a = t*k + j; offsets[e] = number of assignments to experts < e
 *   (offsets[E] = T*k); perm[offsets[e] + r] = the r-th smallest a routed to e;
 *   inv[perm[p]] = p.
 * x: device [T][H] in `x_dtype`. Outputs (device): topk_idx [T][k] i32,
 * topk_w [T][k] f32, offsets [E+1] i32, perm [T*k] i32, inv [T*k] i32.
 * ws: device workspace of ws_bytes >= moe_workspace_size(desc, T).
 */
MOE_API moe_status moe_route(const moe_layer_desc* desc, const uint16_t* router_w, const float* router_bias,
                     const void* x, moe_dtype x_dtype, int32_t T, int32_t* topk_idx, float* topk_w,
                     int32_t* offsets, int32_t* perm, int32_t* inv, void* ws, size_t ws_bytes, void* stream);

/*
 * Routed experts, shared expert and combine, given a routing (from moe_route
 * or the caller's own; topk_w need not sum to one):
 *   for each assignment a = t*k + j, with e the expert whose range
 *   [offsets[e], offsets[e+1]) holds inv[a]:
 *     g = Wg_e x_t, u = Wu_e x_t, h = silu(g) * u (silu(z) = z / (1 + e^-z)),
 *     o_a = Wd_e h;
 *   s_t = Wsd (silu(Wsg x_t) * (Wsu x_t))   (absent when I_s == 0);
 *   y[t] = sum_{j ascending} topk_w[t][j] * o_{t*k+j} + s_t (+ residual[t]).
 * Accumulation is fp32 (exact integer partial sums inside each 2-bit block);
 * outputs are fp32 and are deterministic run to run.
 * x: device [T][H]; residual: device fp32 [T][H] or NULL (may alias y);
 * y: device fp32 [T][H].
 */
MOE_API moe_status moe_expert_ffn(const moe_layer_desc* desc, const moe_layer_weights* w, const void* x,
                          moe_dtype x_dtype, int32_t T, const float* topk_w, const int32_t* offsets,
                          const int32_t* perm, const int32_t* inv, const float* residual, float* y, void* ws,
                          size_t ws_bytes, void* stream);

/*
 * The whole layer: moe_route then moe_expert_ffn, with the routing kept in the
 * workspace. Same argument meanings as above. For bf16 x on the decode path
 * (T <= 16) the shared expert's gate/up and the activation digits, which do not
 * depend on routing, run on a side stream forked from `stream` before the
 * router and joined back before the combine.
 */
MOE_API moe_status moe_layer_forward(const moe_layer_desc* desc, const moe_layer_weights* w, const void* x,
                             moe_dtype x_dtype, int32_t T, const float* residual, float* y, void* ws,
                             size_t ws_bytes, void* stream);

/*
 * moe_layer_forward that also hands the next layer its input: besides the fp32
 * y (the residual stream), y_next[t][h] = bf16(y[t][h]), rounded to nearest
 * with ties to even. Chained layers keep the residual stream in fp32 and take
 * its bf16 rounding as their input (the pages chain the MoE layers without
 * naming the formats; this is the library's reading), and with this call that
 * rounding is the library's own work rather than a cast by the caller.
 * Same arguments, workspace and results as moe_layer_forward, plus
 * y_next: device bf16 [T][H] (uint16 bit patterns), 16-byte aligned, required
 * (MOE_ERR_INVALID_ARG when NULL and T > 0), overlapping none of x, y,
 * residual or the workspace (MOE_ERR_INVALID_ARG otherwise; a chain of layers
 * alternates two input buffers). On the decode path with bf16 x and a shared
 * expert (T <= 16, the shared expert on the side stream) the routed combine
 * kernel stores both outputs; on the other paths a cast kernel runs after the
 * combine.
 */
MOE_API moe_status moe_layer_forward_next(const moe_layer_desc* desc, const moe_layer_weights* w, const void* x,
                                          moe_dtype x_dtype, int32_t T, const float* residual, float* y,
                                          uint16_t* y_next, void* ws, size_t ws_bytes, void* stream);

/*
 * The whole layer without any caller-provided scratch: same arguments and
 * results as moe_layer_forward, minus `ws` / `ws_bytes`. (The ds4 pages have
 * no counterpart of this call; it exists for callers of this library that
 * cannot allocate device memory themselves, e.g. a plugin whose host engine
 * hands out no workspace, or a serving loop that must not allocate after
 * start-up because cudaMalloc may synchronise the device.)
 *   - Scratch is a fixed device array of MOE_NOALLOC_SCRATCH_BYTES inside the
 *     library, present on every GPU that loads the library until the process
 *     exits. Calls whose workspace need (moe_workspace_size) exceeds it return
 *     MOE_ERR_WORKSPACE_TOO_SMALL before anything is enqueued; the size covers
 *     a 32-token decode batch at H=7168, I=2048, E=256, k=8, I_s=2048.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current). Under lazy module
 *     loading (the CUDA default) that first lookup is also when the driver
 *     loads the library's module and commits the array's memory. The first
 *     decode-path call (bf16 x, T <= 16) for each device and caller stream
 *     also creates the side stream and three events described under
 *     moe_layer_forward; they are kept, one set per distinct caller stream,
 *     until the process exits. So make the first call for each device and
 *     each caller stream during start-up, outside any stream capture; later
 *     calls create nothing and allocate nothing.
 *   - Every call on a device shares the one array and leaves its contents
 *     behind; the library clears whatever must start at zero itself. Calls
 *     that overlap on the GPU (other streams, other host threads) race on the
 *     array: serialise them.
 *   - The device status of the last call is read with
 *     moe_read_status_noalloc.
 */
#define MOE_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)
MOE_API moe_status moe_layer_forward_noalloc(const moe_layer_desc* desc, const moe_layer_weights* w,
                                             const void* x, moe_dtype x_dtype, int32_t T, const float* residual,
                                             float* y, void* stream);

/*
 * Prefetch of the weights a layer reads before (and regardless of) routing:
 * the router and the shared expert ([Q]: both unquantized) are brought into
 * L2 with an evict-last policy, so that a moe_layer_forward of this layer
 * issued later finds them there. Meant for a chain of layers: while layer l
 * runs, prefetch layer l+1 on another stream (the routed experts of l+1 are
 * unknown until its router has run; they stream with an evict-first policy
 * and do not displace the prefetched lines). Changes only cache state; reads
 * E*H*2 + 3*I_s*H*2 bytes from HBM. Asynchronous on `stream`; capturable.
 * MOE_ERR_INVALID_ARG for a null router or (I_s > 0) null shared weights.
 */
MOE_API moe_status moe_prefetch_layer(const moe_layer_desc* desc, const moe_layer_weights* weights, void* stream);

/*
 * Device-side status of the last call that used workspace `ws` (moe_route,
 * moe_expert_ffn or moe_layer_forward). Every call's first kernel clears a
 * status word at the head of its workspace; a kernel that gives up a bounded
 * wait (about two seconds, or the limit set by moe_debug_inject) records
 * MOE_ERR_TIMEOUT there and returns, and a kernel that finds an inconsistent
 * launch (a misaligned shared-memory window, a tile outside its operand)
 * records MOE_ERR_CUDA or MOE_ERR_INVALID_ARG. The first code recorded wins;
 * the outputs of a call with a non-zero status are undefined.
 * This call enqueues a 4-byte device-to-host copy on `stream` and waits for
 * `stream` (it is the one call of this interface that synchronises); it
 * writes the word to *status (host pointer). Returns MOE_ERR_INVALID_ARG for
 * a null or misaligned `ws` or a null `status`, MOE_ERR_CUDA if the copy fails.
 */
MOE_API moe_status moe_read_status(const void* ws, int32_t* status, void* stream);

/* The same for moe_layer_forward_noalloc: reads the status word at the head
 * of the library's scratch array on the current device. */
MOE_API moe_status moe_read_status_noalloc(int32_t* status, void* stream);

/*
 * Fault injection, a test aid (process-wide, not thread-safe; mode 0 = off).
 * Mode 1: the decode gate/up GEMV's producer warp issues no weight loads, so
 * its consumer warps wait on shared-memory barriers that never complete; with
 * `wait_limit_cycles` as their bound they give up, record MOE_ERR_TIMEOUT in
 * the call's status word and return. Nothing faults, traps or hangs; later
 * kernels of the call run on undefined partial sums. The following call with
 * mode 0 behaves normally again.
 * Returns MOE_ERR_INVALID_ARG for an unknown mode or a negative limit.
 */
MOE_API moe_status moe_debug_inject(int32_t mode, int64_t wait_limit_cycles);

/*
 * Expert cache: the routed experts of one layer live in host memory and the
 * GPU keeps `n_slots` of them ("ds4 : analyse pratique pour un usage
 * documenté", section « Exécuter des modèles plus grands que la RAM avec le
 * streaming SSD »: non-routed weights stay resident while routed experts are
 * kept in a cache and loaded on a miss; here host memory plays the SSD's part
 * and HBM the cache's).
 *   moe_cache_bytes: device bytes of the slot memory for n_slots
 *     (1 <= n_slots <= n_experts): the six routed planes of n_slots experts
 *     plus an expert -> slot map.
 *   moe_cache_create: `host_pool` names the routed planes of all E experts in
 *     the layout of moe_layer_weights, in page-locked host memory
 *     (cudaHostAlloc / cudaHostRegister) that stays valid and unchanged for the
 *     life of the cache; its router and shared fields are ignored. `slot_mem`
 *     is caller-owned device memory of slot_mem_bytes >= moe_cache_bytes on the
 *     current device. Creates a host object (the one host allocation of this
 *     interface); destroy it with moe_cache_destroy. inter % 256 == 0 required.
 *   moe_layer_forward_cached: the whole layer (same meaning and results as
 *     moe_layer_forward, bit for bit) with the routed planes taken from the
 *     cache: it routes, waits for the routing (this call synchronises `stream`
 *     once and cannot be captured in a CUDA graph), keeps the experts already
 *     in a slot (hits), copies each missing expert from the host pool into an
 *     empty slot or the least recently used slot that this call does not need
 *     (cudaMemcpyAsync on `stream`), maps the routing to slot ids and runs the
 *     expert FFN over the slots. `weights` supplies the device router and
 *     shared expert (its routed fields are ignored). Returns
 *     MOE_ERR_WORKSPACE_TOO_SMALL, after the routing only, when one call needs
 *     more distinct experts than there are slots (at most min(E, T * k)).
 *     Not thread-safe per cache; calls on one cache must use one device.
 *   moe_cache_read_stats: calls, hits and misses (experts), bytes copied.
 */
typedef struct moe_expert_cache moe_expert_cache;
typedef struct {
  int64_t calls;
  int64_t hits;
  int64_t misses;
  int64_t bytes_copied;
} moe_cache_stats;
MOE_API moe_status moe_cache_bytes(const moe_layer_desc* desc, int32_t n_slots, size_t* bytes);
MOE_API moe_status moe_cache_create(const moe_layer_desc* desc, const moe_layer_weights* host_pool, int32_t n_slots,
                                    void* slot_mem, size_t slot_mem_bytes, moe_expert_cache** out);
MOE_API moe_status moe_cache_destroy(moe_expert_cache* cache);
MOE_API moe_status moe_cache_read_stats(const moe_expert_cache* cache, moe_cache_stats* stats);
MOE_API moe_status moe_layer_forward_cached(moe_expert_cache* cache, const moe_layer_weights* weights, const void* x,
                                            moe_dtype x_dtype, int32_t T, const float* residual, float* y, void* ws,
                                            size_t ws_bytes, void* stream);

/*
 * Bounds-checked build, a test aid standing in for a memory checker: the
 * library can be built a second time with -DMOE_BOUNDS_CHECK
 * (libmoe2bit_bc.so). In that build every shared-memory load of the decode
 * GEMVs checks its address against the CTA's dynamic shared memory and its
 * alignment, and every partial-sum store and TMA box its buffer; a violation
 * is counted and the access skipped (loads return zeros), nothing traps.
 *   moe_debug_bounds_check_build: 1 in that build, 0 otherwise.
 *   moe_debug_bounds_violations: the count since the last read (then reset to
 *     0), after the caller's synchronisation; MOE_ERR_UNSUPPORTED_SHAPE with
 *     *count = 0 from a normal build.
 */
MOE_API int32_t moe_debug_bounds_check_build(void);
MOE_API moe_status moe_debug_bounds_violations(uint64_t* count);

/* Static, NUL-terminated name of a status code. */
MOE_API const char* moe_status_string(moe_status s);

/*
 * Block-dequantisation unit exposed for testing: decodes `nblocks` consecutive
 * 256-weight blocks to fp32 (device out [nblocks*256]). The result is exact:
 * IQ2-style values have at most 22 significant bits and Q2K-style values are a
 * single correctly rounded fp32 subtraction of two exact products.
 */
MOE_API moe_status moe_debug_dequant_iq2(const uint8_t* codes, const uint16_t* d, int64_t nblocks, float* out,
                                 void* stream);
MOE_API moe_status moe_debug_dequant_q2k(const uint8_t* codes, const uint32_t* dd, int64_t nblocks, float* out,
                                 void* stream);

/*
 * Quantisers: float weights -> the block formats above, without an importance
 * matrix ([Q]: the routed experts are quantized, up/gate IQ2_XXS-style, down
 * Q2_K-style; the pages give no algorithm, these plain rules are the
 * library's). `w` holds nblocks * 256 fp32 weights (device, 16-byte aligned),
 * blocks along the flattened array exactly as the planes above (for a
 * [rows][K] matrix with K % 256 == 0, block i is row i / (K/256)). Outputs are
 * device planes of nblocks entries. Decisions are taken in fp32 with
 * round-to-nearest-even operations, never fused, in the order written, so the
 * bytes are reproducible by any correct implementation of the rule.
 *   moe_quantize_q2k: per 16-weight sub-block lo = min(0, min w), hi = max w,
 *     step = (hi - lo) / 3, off = -lo; d = fp16(max step / 15),
 *     dmin = fp16(max off / 15); sc = clamp(rint(step / d), 0, 15),
 *     m = clamp(rint(off / dmin), 0, 15) (0 when the divisor is 0);
 *     q = clamp(rint((w + dmin * m) / (d * sc)), 0, 3) (0 when d * sc is 0).
 *   moe_quantize_iq2: d = fp16(max |w| * 8 / 1333); per 32-weight sub-block
 *     ls = clamp(rint((max |w| * 8 / (d * 43) - 1) / 2), 0, 15),
 *     c = d * (2 ls + 1) / 8; per group of 8 the signs of w, with the element
 *     of smallest |w| (lowest index on ties) flipped when the count of negatives
 *     is odd; the codebook row minimising sum_e (|w_e| -+ c * grid[row][e])^2
 *     (e ascending; + for the flipped element), the lower row on ties. A block
 *     whose d rounds to 0 gets all-zero codes.
 * Weights must be finite with every scale below 65504 (fp16). Asynchronous on
 * `stream`; MOE_ERR_INVALID_ARG for null or misaligned pointers or a negative
 * count.
 */
MOE_API moe_status moe_quantize_q2k(const float* w, int64_t nblocks, uint8_t* codes, uint32_t* dd, void* stream);
MOE_API moe_status moe_quantize_iq2(const float* w, int64_t nblocks, uint8_t* codes, uint16_t* d, void* stream);

/*
 * The layer's own operand builders exposed for exact tests (same device
 * functions and lookup tables as the hot kernels; every lane of a warp uses
 * its own table replica, as in the kernels). `nblocks` 256-weight blocks.
 *
 * Decode GEMVs (int8 MMA operands):
 *   moe_debug_gemv_operands_iq2: w[256 b + 32 s + 8 j + e] = level * sign of
 *     weight e of group j of sub-block s (int8, device out [nblocks*256]) and
 *     odd[8 b + s] = 2 ls + 1 (u8, device out [nblocks*8]); the weight is then
 *     d * odd * w / 8.
 *   moe_debug_gemv_operands_q2k: scq[256 b + i] = sc * q of weight i (int16,
 *     device out [nblocks*256]) and m[16 b + s] (u8, [nblocks*16]); the weight
 *     is then d * scq - dmin * m.
 * Grouped GEMM (fp16 operands stored into tensor memory, weights in K order):
 *   moe_debug_tc_operands_iq2: out[256 b + i] = fp16 bits of
 *     sign * fp16(fp16(d * (2 ls + 1) * 2^10 / 8) * level), i.e. the weight
 *     times 2^10 with one rounding of the scale and one of the product.
 *   moe_debug_tc_operands_q2k: out[256 b + i] = fp16 bits of the weight's fp32
 *     value d * sc * q - dmin * m rounded to fp16.
 * codes: device, 16-byte aligned (IQ2) / any (Q2K); d, dd: device planes.
 */
MOE_API moe_status moe_debug_gemv_operands_iq2(const uint8_t* codes, int64_t nblocks, int8_t* w, uint8_t* odd,
                                               void* stream);
MOE_API moe_status moe_debug_gemv_operands_q2k(const uint8_t* codes, int64_t nblocks, int16_t* scq, uint8_t* m,
                                               void* stream);
MOE_API moe_status moe_debug_tc_operands_iq2(const uint8_t* codes, const uint16_t* d, int64_t nblocks, uint16_t* out,
                                             void* stream);
MOE_API moe_status moe_debug_tc_operands_q2k(const uint8_t* codes, const uint32_t* dd, int64_t nblocks,
                                             uint16_t* out, void* stream);

/*
 * Kernel timing, a profiling aid (off by default; not thread-safe). While
 * enabled, every launch of the library records a pair of CUDA events on its
 * stream around the kernel (ids below). moe_profile_read waits for the recorded
 * events, writes per-kernel total milliseconds and launch counts into the host
 * arrays (MOE_K_COUNT entries each) and clears the record. Enabling creates a
 * fixed pool of events (no device memory); disabling destroys it.
 */
typedef enum {
  MOE_K_ROUTER_LOGITS = 0,
  MOE_K_TOPK = 1,
  MOE_K_PERMUTE = 2,
  MOE_K_ACTIVE = 3,
  MOE_K_GATEUP = 4,
  MOE_K_DOWN = 5,
  MOE_K_SHARED_GATEUP = 6,
  MOE_K_SHARED_DOWN = 7,
  MOE_K_COMBINE = 8,
  MOE_K_PREP = 9,
  MOE_K_PREFILL_GATEUP = 10,
  MOE_K_PREFILL_DOWN = 11,
  MOE_K_HQUANT = 12,
  MOE_K_COUNT = 16
} moe_kernel_id;
MOE_API moe_status moe_profile_enable(int32_t on);
MOE_API moe_status moe_profile_read(float* total_ms, int32_t* launches);

/*
 * MXFP4 routed experts (second expert format).
 *
 * [Q] names an MXFP4 file that keeps the routed expert weights as published
 * (no requantisation), running on CUDA with native FP4 matrix instructions on
 * Blackwell for batched expert work. The pages give no bit layout; the element
 * and scale encodings below are those of the OCP Microscaling Formats (MX) v1.0
 * specification (MXFP4: blocks of 32 FP4 E2M1 elements sharing one E8M0 scale),
 * and the packing into planes is this library's.
 *
 * All three routed matrices of a layer are MXFP4. A matrix [rows][K] (K = H for
 * gate and up, K = I for down; K % 32 == 0) is two planes:
 *   codes  [rows][K/2] bytes: element 2i of a row in bits 0..3 of byte i,
 *          element 2i+1 in bits 4..7;
 *   scales [rows][K/32] bytes: E8M0 exponent E of block b (elements 32b..32b+31).
 * Element code c: sign = bit 3, magnitude m(c & 7) = 0, 0.5, 1, 1.5, 2, 3, 4, 6.
 * Weight: w = (-1)^sign * m * 2^(E - 127), exact in fp32 for E in [1, 254].
 * E = 255 (the format's NaN) and E = 0 are outside what this library supports
 * (the results for them are unspecified; nothing checks the scale bytes).
 * The router and the shared expert are the bf16 ones of moe_layer_weights.
 */
typedef struct {
  const uint16_t* router_w;     /* bf16 [E][H] */
  const float* router_bias;     /* fp32 [E], or NULL */
  const uint8_t* gate_codes;    /* [E][I][H/2] */
  const uint8_t* gate_scales;   /* [E][I][H/32] */
  const uint8_t* up_codes;      /* [E][I][H/2] */
  const uint8_t* up_scales;     /* [E][I][H/32] */
  const uint8_t* down_codes;    /* [E][H][I/2] */
  const uint8_t* down_scales;   /* [E][H][I/32] */
  const uint16_t* sh_gate;      /* bf16 [I_s][H] (unused when I_s == 0) */
  const uint16_t* sh_up;        /* bf16 [I_s][H] */
  const uint16_t* sh_down;      /* bf16 [H][I_s] */
} moe_mxfp4_weights;

/*
 * moe_workspace_size_mxfp4: workspace bytes of moe_layer_forward_mxfp4 for any
 * T <= max_tokens (host only); MOE_ERR_UNSUPPORTED_SHAPE for shapes the MXFP4
 * path does not serve (see below).
 *
 * The layer forward of moe_layer_forward with MXFP4 routed experts: the same
 * routing, shared expert, combine, residual and output, with the gate, up and
 * down projections of each assignment taken over the decoded MXFP4 weights.
 * T == 0 enqueues nothing. Shapes, in addition to those of the common
 * conventions: hidden % 512 == 0, inter % 512 == 0; for 1 <= T <= 16 also
 * n_experts <= 1024; above 16 tokens I_s % 128 == 0 (or I_s == 0); otherwise
 * MOE_ERR_UNSUPPORTED_SHAPE. Every pointer of `w` (the shared-expert ones when
 * I_s > 0) is a 16-byte aligned device pointer, else MOE_ERR_INVALID_ARG; above
 * 16 tokens the three code planes are 32-byte aligned (the copy that unpacks
 * them requires it), else MOE_ERR_INVALID_ARG. Workspace:
 * ws_bytes >= moe_workspace_size_mxfp4(desc, T), else
 * MOE_ERR_WORKSPACE_TOO_SMALL. Stream, side stream, status word
 * (moe_read_status) and errors as moe_layer_forward.
 * Numerics, 1 <= T <= 16 (dequant-GEMVs): activations enter the integer
 * products as two signed digits of a 14-bit fixed-point code per 256-element
 * block (as in moe_layer_forward's decode path), the decoded elements times 2
 * are exact int8 values, every block of 32 is scaled exactly by its power of
 * two; accumulation in fp32 per block and across blocks.
 * Numerics, T > 16 (grouped GEMM on the block-scaled tensor cores, FP4 x FP8):
 * the routed experts' activations x, and h = silu(g) * u, are quantised to
 * MXFP8 before their contraction: per block of 32 consecutive elements along
 * the reduction axis the E8M0 exponent X = floor(log2 max|v|) - 8 (clamped to
 * [-127, 127], -127 for a zero block) and elements v / 2^X rounded to FP8 E4M3
 * (nearest even, saturating at 448). Products of the FP4 and FP8 elements and
 * both block scales are exact; accumulation is fp32 in the tensor core. The
 * shared expert runs in bf16 (two bf16 parts for fp32 activations) as in
 * moe_layer_forward's many-token path.
 */
MOE_API moe_status moe_workspace_size_mxfp4(const moe_layer_desc* desc, int32_t max_tokens, size_t* bytes);
MOE_API moe_status moe_layer_forward_mxfp4(const moe_layer_desc* desc, const moe_mxfp4_weights* w, const void* x,
                                           moe_dtype x_dtype, int32_t T, const float* residual, float* y, void* ws,
                                           size_t ws_bytes, void* stream);

/*
 * Decode n_blocks consecutive MXFP4 blocks (codes: device [n_blocks][16] bytes,
 * scales: device [n_blocks] E8M0 bytes) into out: device fp32 [n_blocks][32],
 * with the GPU path's element decoding (2 * element as int8, times 2^(E - 128)).
 * Stream-ordered; MOE_ERR_INVALID_ARG for null pointers or n_blocks < 0.
 */
MOE_API moe_status moe_debug_dequant_mxfp4(const uint8_t* codes, const uint8_t* scales, int64_t n_blocks, float* out,
                                           void* stream);

/*
 * Q4-style routed experts (third expert format).
 *
 * The pages name 4-bit routed-expert variants ([R]: Q4 models; [W]: routed
 * expert checkpoints shared between the 2-bit and 4-bit variants) without a
 * layout. This library's Q4-style block: 32 weights along the reduction axis,
 * one fp16 scale d and 32 unsigned 4-bit codes q; w = d * (q - 8). A matrix
 * [rows][K] (K % 32 == 0) is two planes:
 *   codes [rows][K/2] bytes: element 2i in bits 0..3 of byte i, 2i+1 in bits 4..7;
 *   d     [rows][K/32] fp16.
 * moe_layer_forward_q4 is moe_layer_forward_mxfp4 with these planes: the same
 * routing, shared expert, combine, shapes (hidden % 512 == 0, inter % 512 ==
 * 0; n_experts <= 1024 up to 16 tokens; I_s % 128 == 0 or I_s == 0 above),
 * 16-byte alignment (no 32-byte rule), status and errors; its workspace is
 * moe_workspace_size_q4 (it differs from the MXFP4 one above 16 tokens).
 * Numerics, 1 <= T <= 16: the elements enter the integer products as the exact
 * int8 q - 8 and every block is scaled by its d in fp32 (activations as in
 * moe_layer_forward_mxfp4's GEMVs). T > 16: the many-token path of
 * moe_layer_forward (fp16 weight tiles on the tensor cores, fp32
 * accumulation), each weight entering as fp16(fp16(d * 2^10) * (q - 8)), the
 * 2^10 removed in fp32; activations and h as in moe_layer_forward's many-token
 * path.
 */
typedef struct {
  const uint16_t* router_w;     /* bf16 [E][H] */
  const float* router_bias;     /* fp32 [E], or NULL */
  const uint8_t* gate_codes;    /* [E][I][H/2] */
  const uint16_t* gate_d;       /* fp16 [E][I][H/32] */
  const uint8_t* up_codes;      /* [E][I][H/2] */
  const uint16_t* up_d;         /* fp16 [E][I][H/32] */
  const uint8_t* down_codes;    /* [E][H][I/2] */
  const uint16_t* down_d;       /* fp16 [E][H][I/32] */
  const uint16_t* sh_gate;      /* bf16 [I_s][H] (unused when I_s == 0) */
  const uint16_t* sh_up;        /* bf16 [I_s][H] */
  const uint16_t* sh_down;      /* bf16 [H][I_s] */
} moe_q4_weights;

MOE_API moe_status moe_workspace_size_q4(const moe_layer_desc* desc, int32_t max_tokens, size_t* bytes);
MOE_API moe_status moe_layer_forward_q4(const moe_layer_desc* desc, const moe_q4_weights* w, const void* x,
                                        moe_dtype x_dtype, int32_t T, const float* residual, float* y, void* ws,
                                        size_t ws_bytes, void* stream);

/*
 * Decode n_blocks consecutive Q4-style blocks (codes: device [n_blocks][16]
 * bytes, d: device fp16 [n_blocks]) into out: device fp32 [n_blocks][32], with
 * the GPU path's decoding (int8 q - 8 times d). Stream-ordered;
 * MOE_ERR_INVALID_ARG for null pointers or n_blocks < 0.
 */
MOE_API moe_status moe_debug_dequant_q4(const uint8_t* codes, const uint16_t* d, int64_t n_blocks, float* out,
                                        void* stream);

/* Host copy of the library's compiled-in 256 x 8 IQ2 codebook (row-major,
 * values in {8, 25, 43}). `out` is a host pointer to 2048 bytes. */
MOE_API void moe_debug_grid(uint8_t* out);

#ifdef __cplusplus
}
#endif

#endif /* MOE2BIT_H */
