// api.cu - the C ABI declared in include/moe2bit.h: argument validation,
// workspace carving and the launch sequence of each entry point.
#include <cstring>

#include "../../include/moe2bit.h"
#include "common.cuh"
#include "kernels.cuh"

namespace moe {
namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape check shared by every entry point.
moe_status check_desc(const moe_layer_desc* d) {
  if (!d) return MOE_ERR_INVALID_ARG;
  const int H = d->hidden, I = d->inter, E = d->n_experts, k = d->top_k, Is = d->shared_inter;
  if (H <= 0 || I <= 0 || E <= 0 || k <= 0 || Is < 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (H % QK != 0 || H > 16384) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!(I % QK == 0 || (QK % I == 0 && I >= 8)) || I > 16384) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (E > 1024 || k > E || k > 16) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (Is % 8 != 0 || Is > 16384) return MOE_ERR_UNSUPPORTED_SHAPE;
  return MOE_OK;
}

moe_status check_tokens(const moe_layer_desc* d, int32_t T) {
  if (T < 0) return MOE_ERR_INVALID_ARG;
  if (static_cast<int64_t>(T) * d->top_k > (1 << 24)) return MOE_ERR_UNSUPPORTED_SHAPE;
  return MOE_OK;
}

LayerShape shape_of(const moe_layer_desc* d) {
  return LayerShape{d->hidden, d->inter, d->n_experts, d->top_k, d->shared_inter};
}

// Routing part of the workspace.
struct RouteWs {
  int* status;  // device status word (MOE_ERR_TIMEOUT from a bounded wait), cleared by each call
  float* logits;
  int32_t* topk_idx;
  float* topk_w;
  int32_t* offsets;
  int32_t* perm;
  int32_t* inv;
  int32_t* active;
  char* ffn;
  size_t bytes;
};

RouteWs carve(const moe_layer_desc* d, int32_t T, void* base) {
  const size_t nA = static_cast<size_t>(T) * d->top_k, E = d->n_experts;
  char* p = static_cast<char*>(base);
  RouteWs w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* q = p ? p + off : nullptr;
    off += align_up(bytes > 0 ? bytes : 1, 256);
    return q;
  };
  w.status = reinterpret_cast<int*>(take(16));
  w.logits = reinterpret_cast<float*>(take(static_cast<size_t>(T) * E * 4));
  w.topk_idx = reinterpret_cast<int32_t*>(take(nA * 4));
  w.topk_w = reinterpret_cast<float*>(take(nA * 4));
  w.offsets = reinterpret_cast<int32_t*>(take((E + 1) * 4));
  w.perm = reinterpret_cast<int32_t*>(take(nA * 4));
  w.inv = reinterpret_cast<int32_t*>(take(nA * 4));
  w.active = reinterpret_cast<int32_t*>(take((E + 1) * 4));
  w.ffn = take(ffn_workspace_bytes(shape_of(d), T));
  w.bytes = off;
  return w;
}

WeightPtrs weights_of(const moe_layer_weights* w) {
  return WeightPtrs{w->router_w, w->router_bias, w->gate_codes, w->gate_d,    w->up_codes, w->up_d,
                    w->down_codes, w->down_dd,   w->sh_gate,    w->sh_up,     w->sh_down};
}

moe_status check_expert_weights(const moe_layer_desc* d, const moe_layer_weights* w) {
  if (!w) return MOE_ERR_INVALID_ARG;
  const void* req[] = {w->gate_codes, w->gate_d, w->up_codes, w->up_d, w->down_codes, w->down_dd};
  for (const void* p : req)
    if (!p || !aligned16(p)) return MOE_ERR_INVALID_ARG;
  if (d->shared_inter > 0) {
    const void* sh[] = {w->sh_gate, w->sh_up, w->sh_down};
    for (const void* p : sh)
      if (!p || !aligned16(p)) return MOE_ERR_INVALID_ARG;
  }
  return MOE_OK;
}

moe_status to_status(int rc) { return static_cast<moe_status>(rc); }

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "MOE_ERR_UNSUPPORTED_SHAPE";
    case MOE_ERR_WORKSPACE_TOO_SMALL: return "MOE_ERR_WORKSPACE_TOO_SMALL";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
  }
  return "MOE_UNKNOWN_STATUS";
}

moe_status moe_workspace_size(const moe_layer_desc* desc, int32_t max_tokens, size_t* bytes) {
  moe_status st = check_desc(desc);
  if (st != MOE_OK) return st;
  if (!bytes) return MOE_ERR_INVALID_ARG;
  if ((st = check_tokens(desc, max_tokens)) != MOE_OK) return st;
  *bytes = carve(desc, max_tokens, nullptr).bytes;
  return MOE_OK;
}

moe_status moe_route(const moe_layer_desc* desc, const uint16_t* router_w, const float* router_bias, const void* x,
                     moe_dtype x_dtype, int32_t T, int32_t* topk_idx, float* topk_w, int32_t* offsets,
                     int32_t* perm, int32_t* inv, void* ws, size_t ws_bytes, void* stream) {
  moe_status st = check_desc(desc);
  if (st != MOE_OK) return st;
  if ((st = check_tokens(desc, T)) != MOE_OK) return st;
  if (x_dtype != MOE_F32 && x_dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  const void* req[] = {router_w, x, topk_idx, topk_w, offsets, perm, inv, ws};
  for (const void* p : req)
    if (!p || !aligned16(p)) return MOE_ERR_INVALID_ARG;
  if (router_bias && !aligned16(router_bias)) return MOE_ERR_INVALID_ARG;
  RouteWs w = carve(desc, T, ws);
  if (ws_bytes < w.bytes) return MOE_ERR_WORKSPACE_TOO_SMALL;
  return to_status(launch_route(router_w, router_bias, x, x_dtype, T, desc->hidden, desc->n_experts,
                                desc->top_k, w.logits, topk_idx, topk_w, offsets, perm, inv, w.active, w.status,
                                static_cast<cudaStream_t>(stream)));
}

moe_status moe_expert_ffn(const moe_layer_desc* desc, const moe_layer_weights* weights, const void* x,
                          moe_dtype x_dtype, int32_t T, const float* topk_w, const int32_t* offsets,
                          const int32_t* perm, const int32_t* inv, const float* residual, float* y, void* ws,
                          size_t ws_bytes, void* stream) {
  moe_status st = check_desc(desc);
  if (st != MOE_OK) return st;
  if ((st = check_tokens(desc, T)) != MOE_OK) return st;
  if (x_dtype != MOE_F32 && x_dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if ((st = check_expert_weights(desc, weights)) != MOE_OK) return st;
  const void* req[] = {x, topk_w, offsets, perm, inv, y, ws};
  for (const void* p : req)
    if (!p || !aligned16(p)) return MOE_ERR_INVALID_ARG;
  if (residual && !aligned16(residual)) return MOE_ERR_INVALID_ARG;
  RouteWs w = carve(desc, T, ws);
  if (ws_bytes < w.bytes) return MOE_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int rc = launch_active_from_offsets(offsets, desc->n_experts, w.active, s);
  if (rc != OK) return to_status(rc);
  Routing r{topk_w, offsets, perm, inv, w.active};
  return to_status(
      launch_ffn(shape_of(desc), weights_of(weights), x, x_dtype, T, r, residual, y, w.ffn, w.status, true, s));
}

moe_status moe_layer_forward(const moe_layer_desc* desc, const moe_layer_weights* weights, const void* x,
                             moe_dtype x_dtype, int32_t T, const float* residual, float* y, void* ws,
                             size_t ws_bytes, void* stream) {
  moe_status st = check_desc(desc);
  if (st != MOE_OK) return st;
  if ((st = check_tokens(desc, T)) != MOE_OK) return st;
  if (x_dtype != MOE_F32 && x_dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if ((st = check_expert_weights(desc, weights)) != MOE_OK) return st;
  if (!weights->router_w || !aligned16(weights->router_w)) return MOE_ERR_INVALID_ARG;
  if (weights->router_bias && !aligned16(weights->router_bias)) return MOE_ERR_INVALID_ARG;
  const void* req[] = {x, y, ws};
  for (const void* p : req)
    if (!p || !aligned16(p)) return MOE_ERR_INVALID_ARG;
  if (residual && !aligned16(residual)) return MOE_ERR_INVALID_ARG;
  RouteWs w = carve(desc, T, ws);
  if (ws_bytes < w.bytes) return MOE_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the shared expert does not depend on routing: its gate/up starts first, on a side stream
  const bool early = shared_early_ok(shape_of(desc), x_dtype, T);
  if (early) {
    const int rc0 = launch_shared_early(shape_of(desc), weights_of(weights), x, T, w.ffn, s);
    if (rc0 != OK) return to_status(rc0);
  }
  int rc = launch_route(weights->router_w, weights->router_bias, x, x_dtype, T, desc->hidden, desc->n_experts,
                        desc->top_k, w.logits, w.topk_idx, w.topk_w, w.offsets, w.perm, w.inv, w.active, w.status,
                        s, early);
  if (rc != OK) {
    if (early) join_shared_early(s);  // leave no forked work unjoined (graph capture requires it)
    return to_status(rc);
  }
  Routing r{w.topk_w, w.offsets, w.perm, w.inv, w.active};
  // the status word is cleared by the first kernel on the caller's stream: the router when the shared
  // expert and the digits run ahead on the side stream, the tensor-core router for many bf16 tokens
  const bool routed_clears = x_dtype == MOE_BF16 && router_tc_supported(T, desc->hidden, desc->n_experts);
  return to_status(launch_ffn(shape_of(desc), weights_of(weights), x, x_dtype, T, r, residual, y, w.ffn, w.status,
                              !routed_clears && !early, s, early));
}

moe_status moe_debug_dequant_iq2(const uint8_t* codes, const uint16_t* d, int64_t nblocks, float* out,
                                 void* stream) {
  if (nblocks < 0) return MOE_ERR_INVALID_ARG;
  if (nblocks == 0) return MOE_OK;
  if (!codes || !d || !out || !aligned16(codes) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  return to_status(launch_debug_dequant_iq2(codes, d, nblocks, out, static_cast<cudaStream_t>(stream)));
}

moe_status moe_debug_dequant_q2k(const uint8_t* codes, const uint32_t* dd, int64_t nblocks, float* out,
                                 void* stream) {
  if (nblocks < 0) return MOE_ERR_INVALID_ARG;
  if (nblocks == 0) return MOE_OK;
  if (!codes || !dd || !out || !aligned16(codes) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  return to_status(launch_debug_dequant_q2k(codes, dd, nblocks, out, static_cast<cudaStream_t>(stream)));
}

void moe_debug_grid(uint8_t* out) {
  if (!out) return;
  for (int r = 0; r < 256; ++r)
    for (int e = 0; e < 8; ++e) out[r * 8 + e] = kCodebook.val[r][e];
}

}  // extern "C"
