// kernels.cuh - launchers shared between the translation units of the library.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace moe {

struct LayerShape {
  int H, I, E, k, Is;
};

struct WeightPtrs {
  const uint16_t* router_w;
  const float* router_bias;
  const uint8_t* gate_codes;
  const uint16_t* gate_d;
  const uint8_t* up_codes;
  const uint16_t* up_d;
  const uint8_t* down_codes;
  const uint32_t* down_dd;
  const uint16_t* sh_gate;
  const uint16_t* sh_up;
  const uint16_t* sh_down;
};

// Routing state produced by the router/permutation step (device pointers).
struct Routing {
  const float* topk_w;    // [T][k]
  const int32_t* offsets; // [E+1]
  const int32_t* perm;    // [T*k]
  const int32_t* inv;     // [T*k]
  const int32_t* active;  // [E+1]: compacted active experts, active[E] = count
};

int launch_route(const uint16_t* Wr, const float* bias, const void* x, int x_dtype, int T, int H, int E, int k,
                 float* logits, int32_t* topk_idx, float* topk_w, int32_t* offsets, int32_t* perm, int32_t* inv,
                 int32_t* active, int* err, cudaStream_t st,
                 bool clear_status = false);
int launch_active_from_offsets(const int32_t* offsets, int E, int32_t* active, cudaStream_t st);
// ids <- map[ids] (n entries), then the stable permutation of the n ids over E values.
int launch_remap_permute(int32_t* ids, int n, const int32_t* map, int E, int32_t* offsets, int32_t* perm,
                         int32_t* inv, int32_t* active, cudaStream_t st);

// Workspace needed by the FFN stage for T tokens (bytes) and the launcher.
size_t ffn_workspace_bytes(const LayerShape& s, int T);
// clear_status: the FFN's first kernel clears *err (false when an earlier
// kernel of the same call already did). y_bf16 (optional, [T][H]): also store
// bf16(y), rounded to nearest even, by the combine kernel where it can, else by
// a cast kernel after it.
int launch_ffn(const LayerShape& s, const WeightPtrs& w, const void* x, int x_dtype, int T, const Routing& r,
               const float* residual, float* y, void* ws, int* err, bool clear_status, cudaStream_t st,
               bool shared_early = false, uint16_t* y_bf16 = nullptr);
// yb = bf16(y) elementwise (nearest, ties to even); n a multiple of 4, both 16-byte aligned (decode.cu).
int launch_y_to_bf16(const float* y, uint16_t* yb, size_t n, cudaStream_t st);

// L2 prefetch (evict_last) of up to four device ranges (decode.cu).
int launch_l2_prefetch(const void* const* ptrs, const size_t* bytes, int n, cudaStream_t st);

// Tensor-core dequant-GEMV path (decode.cu): shapes with H % 256 == 0 and I % 256 == 0.
bool fast_path_supported(const LayerShape& s);
// true when launch_ffn takes the tensor-core grouped GEMM for T tokens
bool use_prefill(const LayerShape& s, int T);
size_t fast_ffn_workspace_bytes(const LayerShape& s, int T);
int launch_ffn_fast(const LayerShape& s, const WeightPtrs& w, const void* x, int x_dtype, int T, const Routing& r,
                    const float* residual, float* y, void* ws, int* err, bool clear_status, cudaStream_t st,
                    bool shared_early = false, uint16_t* y_bf16 = nullptr);

// TMA-fed GEMVs (gemv_tma.cu).
bool tma_path_supported(const LayerShape& s, int T);
int tma_gu_parts(const LayerShape& s, int T);
int tma_dn_parts(const LayerShape& s, int T);
int launch_gateup_tma(const LayerShape& sh, const uint8_t* gate_codes, const uint16_t* gate_d,
                      const uint8_t* up_codes, const uint16_t* up_d, const int8_t* xd, const float* xs, int T,
                      const Routing& r, float* gpart, int* err, int sms, cudaStream_t st);
// MXFP4 routed experts (mxfp4.cu; the step in decode.cu).
struct MxPlanes {
  int fmt;  // 0 = MXFP4, 1 = Q4-style
  const uint8_t* gate_codes;
  const void* gate_scales;
  const uint8_t* up_codes;
  const void* up_scales;
  const uint8_t* down_codes;
  const void* down_scales;
};
// fmt: 0 = MXFP4, 1 = Q4-style (the many-token step differs: block-scaled GEMM or the dequantising one)
size_t mx_ffn_workspace_bytes(const LayerShape& s, int T, int fmt);
int launch_ffn_mxfp4(const LayerShape& s, const WeightPtrs& shw, const MxPlanes& w, const void* x, int x_dtype,
                     int T, const Routing& r, const float* residual, float* y, void* ws, int* err, bool clear_status,
                     cudaStream_t st, bool shared_early);
bool mx_path_supported(const LayerShape& s, int T);
int mx_parts(int K);
// fmt: 0 = MXFP4 (E8M0 byte scales), 1 = Q4-style (fp16 scales)
int launch_mx_gemv(int fmt, bool pair, int K, int R, int E, int k, int T, const uint8_t* codes0, const void* sc0,
                   const uint8_t* codes1, const void* sc1, const int8_t* ad, const float* as, const Routing& r,
                   float* part, int* err, int sms, cudaStream_t st);
int launch_mx_hquant(int I, int KP, int nA, const float* gu, int8_t* hd, float* hs, cudaStream_t st);
int launch_mx_dequant(int fmt, const uint8_t* codes, const void* scales, int64_t nb, float* out, cudaStream_t st);

int launch_down_tma(const LayerShape& sh, const uint8_t* down_codes, const uint32_t* down_dd, const int8_t* hd,
                    const float* hsc, const int32_t* hq, int hss, int T, const Routing& r, float* opart, int* err,
                    int sms, cudaStream_t st);

// Shared expert on bf16 warp MMAs for up to 32 tokens (shared_mma.cu). xb holds
// P bf16 parts of x as [P][T][H]; hb receives h as two parts [2][T][Is].
bool shared_mma_supported(int H, int Is, int T, int x_parts, int k);
// Shared expert ahead of routing: for bf16 activations on the decode path the
// shared gate/up runs on a side stream forked from `st` before the router, and
// the decode path's combine waits for it. Returns true when it was launched.
bool shared_early_ok(const LayerShape& s, int x_dtype, int T);
// KP, DP: the part counts of the caller's workspace layout (<= 0: those of launch_ffn_fast).
int launch_shared_early(const LayerShape& s, const WeightPtrs& w, const void* x, int T, void* ffn_ws, cudaStream_t st,
                        int KP = -1, int DP = -1);
// Joins the side stream back into `st` (the error path of a call that forked it).
void join_shared_early(cudaStream_t st);
int launch_shared_gateup_mma(int H, int Is, const uint16_t* wg, const uint16_t* wu, const uint16_t* xb, int P,
                             int T, uint16_t* hb, cudaStream_t st);
int launch_shared_down_combine_mma(int H, int Is, const uint16_t* wd, const uint16_t* hb, int T, int k,
                                   const float* topk_w, const int32_t* inv, const float* obuf, int DP,
                                   const float* residual, float* y, cudaStream_t st);

// Router logits on the tensor cores for many bf16 tokens (prefill.cu).
bool router_tc_supported(int T, int H, int E);
int launch_router_tc(const uint16_t* Wr, const float* bias, const uint16_t* x, int T, int H, int E, float* logits,
                     int* err, int sms, cudaStream_t st);

// Tensor-core grouped GEMM for many tokens (prefill.cu). Up to 16 tokens the
// int8 dequant-GEMVs are faster (an 8-layer chain of 16-token steps measured
// 9.3 ms on the GEMVs against 10.3 ms on the grouped GEMM).
constexpr int kPrefillMinT = 16;
bool prefill_path_supported(const LayerShape& s, int T);
size_t prefill_workspace_bytes(const LayerShape& s, int T);
// q4: Q4-style routed experts (codes and fp16 d planes) in place of the IQ2 / Q2K planes of `w`.
int launch_ffn_prefill(const LayerShape& s, const WeightPtrs& w, const void* x, int x_dtype, int T, const Routing& r,
                       const float* residual, float* y, void* ws, int* err, bool clear_status, int sms,
                       cudaStream_t st, const MxPlanes* q4 = nullptr);

// The shared expert alone on the tensor-core GEMM (prefill.cu): s_out = fp32 [T][H].
size_t prefill_shared_workspace_bytes(const LayerShape& s, int T);
int launch_prefill_shared(const LayerShape& s, const uint16_t* wg, const uint16_t* wu, const uint16_t* wd,
                          const void* x, int x_dtype, int T, void* ws, float* s_out, int* err, int sms,
                          cudaStream_t st);

// MXFP4 routed experts for more than 16 tokens (mx_gemm.cu): a grouped GEMM on the block-scaled
// tensor cores, FP4 weights x MXFP8 activations.
bool mx_prefill_supported(const LayerShape& s, int T);
size_t mx_prefill_workspace_bytes(const LayerShape& s, int T);
int launch_ffn_mx_prefill(const LayerShape& s, const WeightPtrs& shw, const MxPlanes& w, const void* x, int x_dtype,
                          int T, const Routing& r, const float* residual, float* y, void* ws, int* err,
                          bool clear_status, int sms, cudaStream_t st);

// Copies the device status word at `word` to *out after the work enqueued on `st` (synchronises `st`).
int read_status_word(const int* word, int32_t* out, cudaStream_t st);

// Test aid: fault injection into the decode gate/up GEMV (mode 1: its producer issues no loads, so its
// consumers' bounded waits run out after `wait_limit` cycles). Mode 0 restores normal operation.
void set_debug_inject(int mode, long long wait_limit);

// Violations counted by the bounds-checked build of the decode GEMVs since the
// last read (then reset); ERR_SHAPE from a normal build.
int read_bounds_violations(unsigned long long* out);

// Float weights -> block formats (quant.cu).
int launch_quantize_q2k(const float* w, int64_t nblocks, uint8_t* codes, uint32_t* dd, cudaStream_t st);
int launch_quantize_iq2(const float* w, int64_t nblocks, uint8_t* codes, uint16_t* d, cudaStream_t st);

// The hot paths' own operand builders, run on their own (gemv_tma.cu, prefill.cu).
int launch_debug_gemv_iq2(const uint8_t* codes, int64_t nblocks, int8_t* w, uint8_t* odd, cudaStream_t st);
int launch_debug_gemv_q2k(const uint8_t* codes, int64_t nblocks, int16_t* scq, uint8_t* m, cudaStream_t st);
int launch_debug_tc_iq2(const uint8_t* codes, const uint16_t* d, int64_t nblocks, uint16_t* out, cudaStream_t st);
int launch_debug_tc_q2k(const uint8_t* codes, const uint32_t* dd, int64_t nblocks, uint16_t* out, cudaStream_t st);

int launch_debug_dequant_iq2(const uint8_t* codes, const uint16_t* d, int64_t nblocks, float* out, cudaStream_t st);
int launch_debug_dequant_q2k(const uint8_t* codes, const uint32_t* dd, int64_t nblocks, float* out,
                             cudaStream_t st);

}  // namespace moe
