// api.cu - the C ABI declared in include/moe2bit.h: argument validation,
// workspace carving and the launch sequence of each entry point.
#include <cstring>
#include <initializer_list>
#include <vector>

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

// ffn_bytes: the FFN part of the workspace (default: that of the IQ2 / Q2K layer forward).
RouteWs carve(const moe_layer_desc* d, int32_t T, void* base, size_t ffn_bytes = SIZE_MAX) {
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
  w.ffn = take(ffn_bytes == SIZE_MAX ? ffn_workspace_bytes(shape_of(d), T) : ffn_bytes);
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

// Planes of one routed expert (per-matrix block count nb = I * H / 256).
struct ExpertPlaneBytes {
  size_t gate_codes, gate_d, up_codes, up_d, down_codes, down_dd;
};
ExpertPlaneBytes expert_plane_bytes(const moe_layer_desc* d) {
  const size_t nb = static_cast<size_t>(d->inter) * d->hidden / QK;
  return {nb * IQ2_BYTES, nb * 2, nb * IQ2_BYTES, nb * 2, nb * Q2K_BYTES, nb * 4};
}

}  // namespace

int read_status_word(const int* word, int32_t* out, cudaStream_t st) {
  int32_t v = 0;
  if (cudaMemcpyAsync(&v, word, sizeof(v), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return ERR_CUDA;
  *out = v;
  return OK;
}

}  // namespace moe

using namespace moe;

// Host-side state of an expert cache (see moe_cache_create in the header).
struct moe_expert_cache {
  moe_layer_desc desc;
  int n_slots;
  int device;
  ExpertPlaneBytes pb;
  const uint8_t* host[6];  // routed planes of all experts in pinned host memory
  uint8_t* slot[6];        // the same planes for n_slots experts in device memory
  int32_t* d_map;          // device [E]: slot of each expert resident for the current call
  std::vector<int> slot_of, expert_in;
  std::vector<uint64_t> last_use;
  std::vector<int32_t> h_active, h_map;
  uint64_t tick;
  moe_cache_stats stats;
};

namespace {
size_t cache_carve(const moe_layer_desc* d, int n_slots, uint8_t* base, uint8_t* (&slot)[6], int32_t** map) {
  const ExpertPlaneBytes pb = expert_plane_bytes(d);
  const size_t per[6] = {pb.gate_codes, pb.gate_d, pb.up_codes, pb.up_d, pb.down_codes, pb.down_dd};
  size_t off = 0;
  for (int i = 0; i < 6; ++i) {
    slot[i] = base ? base + off : nullptr;
    off += align_up(per[i] * n_slots, 256);
  }
  *map = base ? reinterpret_cast<int32_t*>(base + off) : nullptr;
  off += align_up(static_cast<size_t>(d->n_experts) * 4, 256);
  return off;
}
}  // namespace

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

}  // extern "C"

namespace {
bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
  return pa < pb + nb && pb < pa + na;
}

moe_status layer_forward_impl(const moe_layer_desc* desc, const moe_layer_weights* weights, const void* x,
                              moe_dtype x_dtype, int32_t T, const float* residual, float* y, uint16_t* y_next,
                              void* ws, size_t ws_bytes, void* stream) {
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
  if (y_next) {  // written while x, y and the residual are still read: no overlap with any of them
    const size_t n = static_cast<size_t>(T) * desc->hidden;
    const size_t xb = n * (x_dtype == MOE_F32 ? 4 : 2);
    if (!aligned16(y_next) || overlaps(y_next, 2 * n, x, xb) || overlaps(y_next, 2 * n, y, 4 * n) ||
        (residual && overlaps(y_next, 2 * n, residual, 4 * n)))
      return MOE_ERR_INVALID_ARG;
  }
  RouteWs w = carve(desc, T, ws);
  if (ws_bytes < w.bytes) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if (y_next && overlaps(y_next, static_cast<size_t>(T) * desc->hidden * 2, ws, w.bytes)) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the shared expert does not depend on routing: its gate/up starts first, on a side stream. Once the
  // fork may have been recorded, every return joins the side stream back (a capture in progress needs
  // every forked stream joined; joining twice is harmless).
  const bool early = shared_early_ok(shape_of(desc), x_dtype, T);
  int rc = OK;
  if (early) rc = launch_shared_early(shape_of(desc), weights_of(weights), x, T, w.ffn, s);
  if (rc == OK)
    rc = launch_route(weights->router_w, weights->router_bias, x, x_dtype, T, desc->hidden, desc->n_experts,
                      desc->top_k, w.logits, w.topk_idx, w.topk_w, w.offsets, w.perm, w.inv, w.active, w.status, s,
                      early);
  if (rc == OK) {
    Routing r{w.topk_w, w.offsets, w.perm, w.inv, w.active};
    // the status word is cleared by the first kernel on the caller's stream: the router when the shared
    // expert and the digits run ahead on the side stream, the tensor-core router for many bf16 tokens
    const bool routed_clears = x_dtype == MOE_BF16 && router_tc_supported(T, desc->hidden, desc->n_experts);
    rc = launch_ffn(shape_of(desc), weights_of(weights), x, x_dtype, T, r, residual, y, w.ffn, w.status,
                    !routed_clears && !early, s, early, y_next);
  }
  if (rc != OK && early) join_shared_early(s);
  return to_status(rc);
}
}  // namespace

extern "C" {

moe_status moe_layer_forward(const moe_layer_desc* desc, const moe_layer_weights* weights, const void* x,
                             moe_dtype x_dtype, int32_t T, const float* residual, float* y, void* ws,
                             size_t ws_bytes, void* stream) {
  return layer_forward_impl(desc, weights, x, x_dtype, T, residual, y, nullptr, ws, ws_bytes, stream);
}

moe_status moe_layer_forward_next(const moe_layer_desc* desc, const moe_layer_weights* weights, const void* x,
                                  moe_dtype x_dtype, int32_t T, const float* residual, float* y, uint16_t* y_next,
                                  void* ws, size_t ws_bytes, void* stream) {
  if (!y_next && T > 0) return MOE_ERR_INVALID_ARG;
  return layer_forward_impl(desc, weights, x, x_dtype, T, residual, y, y_next, ws, ws_bytes, stream);
}

moe_status moe_prefetch_layer(const moe_layer_desc* desc, const moe_layer_weights* weights, void* stream) {
  moe_status st = check_desc(desc);
  if (st != MOE_OK) return st;
  if (!weights || !weights->router_w || !aligned16(weights->router_w)) return MOE_ERR_INVALID_ARG;
  const size_t H = desc->hidden, Is = desc->shared_inter, E = desc->n_experts;
  const void* pp[4] = {weights->router_w, Is ? weights->sh_gate : nullptr, Is ? weights->sh_up : nullptr,
                       Is ? weights->sh_down : nullptr};
  const size_t nn[4] = {E * H * 2, Is * H * 2, Is * H * 2, Is * H * 2};
  for (int i = 1; i < 4; ++i)
    if (Is && (!pp[i] || !aligned16(pp[i]))) return MOE_ERR_INVALID_ARG;
  return to_status(launch_l2_prefetch(pp, nn, 4, static_cast<cudaStream_t>(stream)));
}

moe_status moe_read_status(const void* ws, int32_t* status, void* stream) {
  if (!ws || !status || !aligned16(ws)) return MOE_ERR_INVALID_ARG;
  return to_status(read_status_word(static_cast<const int*>(ws), status, static_cast<cudaStream_t>(stream)));
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

moe_status moe_debug_gemv_operands_iq2(const uint8_t* codes, int64_t nblocks, int8_t* w, uint8_t* odd,
                                       void* stream) {
  if (nblocks < 0) return MOE_ERR_INVALID_ARG;
  if (nblocks == 0) return MOE_OK;
  if (!codes || !w || !odd || !aligned16(codes) || !aligned16(w)) return MOE_ERR_INVALID_ARG;
  return to_status(launch_debug_gemv_iq2(codes, nblocks, w, odd, static_cast<cudaStream_t>(stream)));
}

moe_status moe_debug_gemv_operands_q2k(const uint8_t* codes, int64_t nblocks, int16_t* scq, uint8_t* m,
                                       void* stream) {
  if (nblocks < 0) return MOE_ERR_INVALID_ARG;
  if (nblocks == 0) return MOE_OK;
  if (!codes || !scq || !m || !aligned16(codes)) return MOE_ERR_INVALID_ARG;
  return to_status(launch_debug_gemv_q2k(codes, nblocks, scq, m, static_cast<cudaStream_t>(stream)));
}

moe_status moe_debug_tc_operands_iq2(const uint8_t* codes, const uint16_t* d, int64_t nblocks, uint16_t* out,
                                     void* stream) {
  if (nblocks < 0) return MOE_ERR_INVALID_ARG;
  if (nblocks == 0) return MOE_OK;
  if (!codes || !d || !out || !aligned16(codes) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  return to_status(launch_debug_tc_iq2(codes, d, nblocks, out, static_cast<cudaStream_t>(stream)));
}

moe_status moe_debug_tc_operands_q2k(const uint8_t* codes, const uint32_t* dd, int64_t nblocks, uint16_t* out,
                                     void* stream) {
  if (nblocks < 0) return MOE_ERR_INVALID_ARG;
  if (nblocks == 0) return MOE_OK;
  if (!codes || !dd || !out || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  return to_status(launch_debug_tc_q2k(codes, dd, nblocks, out, static_cast<cudaStream_t>(stream)));
}

moe_status moe_quantize_q2k(const float* w, int64_t nblocks, uint8_t* codes, uint32_t* dd, void* stream) {
  if (nblocks < 0) return MOE_ERR_INVALID_ARG;
  if (nblocks == 0) return MOE_OK;
  if (!w || !codes || !dd || !aligned16(w) || !aligned16(codes)) return MOE_ERR_INVALID_ARG;
  if (nblocks > (int64_t(1) << 31) / 16) return MOE_ERR_UNSUPPORTED_SHAPE;
  return to_status(launch_quantize_q2k(w, nblocks, codes, dd, static_cast<cudaStream_t>(stream)));
}

moe_status moe_quantize_iq2(const float* w, int64_t nblocks, uint8_t* codes, uint16_t* d, void* stream) {
  if (nblocks < 0) return MOE_ERR_INVALID_ARG;
  if (nblocks == 0) return MOE_OK;
  if (!w || !codes || !d || !aligned16(w) || !aligned16(codes)) return MOE_ERR_INVALID_ARG;
  if (nblocks > 0x7FFFFFFF) return MOE_ERR_UNSUPPORTED_SHAPE;
  return to_status(launch_quantize_iq2(w, nblocks, codes, d, static_cast<cudaStream_t>(stream)));
}

int32_t moe_debug_bounds_check_build(void) {
#ifdef MOE_BOUNDS_CHECK
  return 1;
#else
  return 0;
#endif
}

moe_status moe_debug_bounds_violations(uint64_t* count) {
  if (!count) return MOE_ERR_INVALID_ARG;
  unsigned long long v = 0;
  const int rc = read_bounds_violations(&v);
  *count = v;
  return to_status(rc);
}

moe_status moe_debug_inject(int32_t mode, int64_t wait_limit_cycles) {
  if (mode < 0 || mode > 1 || wait_limit_cycles < 0) return MOE_ERR_INVALID_ARG;
  set_debug_inject(mode, mode ? static_cast<long long>(wait_limit_cycles) : 0ll);
  return MOE_OK;
}

void moe_debug_grid(uint8_t* out) {
  if (!out) return;
  for (int r = 0; r < 256; ++r)
    for (int e = 0; e < 8; ++e) out[r * 8 + e] = kCodebook.val[r][e];
}


moe_status moe_cache_bytes(const moe_layer_desc* desc, int32_t n_slots, size_t* bytes) {
  moe_status st = check_desc(desc);
  if (st != MOE_OK) return st;
  if (!bytes || n_slots < 1 || n_slots > desc->n_experts) return MOE_ERR_INVALID_ARG;
  uint8_t* slot[6];
  int32_t* map;
  *bytes = cache_carve(desc, n_slots, nullptr, slot, &map);
  return MOE_OK;
}

moe_status moe_cache_create(const moe_layer_desc* desc, const moe_layer_weights* host_pool, int32_t n_slots,
                            void* slot_mem, size_t slot_mem_bytes, moe_expert_cache** out) {
  moe_status st = check_desc(desc);
  if (st != MOE_OK) return st;
  if (!out || !host_pool || !slot_mem || !aligned16(slot_mem)) return MOE_ERR_INVALID_ARG;
  if (desc->inter % QK != 0) return MOE_ERR_UNSUPPORTED_SHAPE;  // the cached path serves the GEMV/GEMM kernels
  size_t need = 0;
  if ((st = moe_cache_bytes(desc, n_slots, &need)) != MOE_OK) return st;
  if (slot_mem_bytes < need) return MOE_ERR_WORKSPACE_TOO_SMALL;
  const void* hp[6] = {host_pool->gate_codes, host_pool->gate_d, host_pool->up_codes,
                       host_pool->up_d,       host_pool->down_codes, host_pool->down_dd};
  for (const void* p : hp)
    if (!p) return MOE_ERR_INVALID_ARG;
  moe_expert_cache* c = new (std::nothrow) moe_expert_cache();
  if (!c) return MOE_ERR_CUDA;
  c->desc = *desc;
  c->n_slots = n_slots;
  if (cudaGetDevice(&c->device) != cudaSuccess) {
    delete c;
    return MOE_ERR_CUDA;
  }
  c->pb = expert_plane_bytes(desc);
  for (int i = 0; i < 6; ++i) c->host[i] = static_cast<const uint8_t*>(hp[i]);
  cache_carve(desc, n_slots, static_cast<uint8_t*>(slot_mem), c->slot, &c->d_map);
  c->slot_of.assign(desc->n_experts, -1);
  c->expert_in.assign(n_slots, -1);
  c->last_use.assign(n_slots, 0);
  c->h_active.assign(desc->n_experts + 1, 0);
  c->h_map.assign(desc->n_experts, 0);
  c->tick = 0;
  c->stats = moe_cache_stats{0, 0, 0, 0};
  *out = c;
  return MOE_OK;
}

moe_status moe_cache_destroy(moe_expert_cache* cache) {
  delete cache;
  return MOE_OK;
}

moe_status moe_cache_read_stats(const moe_expert_cache* cache, moe_cache_stats* stats) {
  if (!cache || !stats) return MOE_ERR_INVALID_ARG;
  *stats = cache->stats;
  return MOE_OK;
}

moe_status moe_layer_forward_cached(moe_expert_cache* cache, const moe_layer_weights* weights, const void* x,
                                    moe_dtype x_dtype, int32_t T, const float* residual, float* y, void* ws,
                                    size_t ws_bytes, void* stream) {
  if (!cache) return MOE_ERR_INVALID_ARG;
  const moe_layer_desc* desc = &cache->desc;
  moe_status st = check_tokens(desc, T);
  if (st != MOE_OK) return st;
  if (x_dtype != MOE_F32 && x_dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!weights || !weights->router_w || !aligned16(weights->router_w)) return MOE_ERR_INVALID_ARG;
  if (weights->router_bias && !aligned16(weights->router_bias)) return MOE_ERR_INVALID_ARG;
  if (desc->shared_inter > 0) {
    const void* sh[] = {weights->sh_gate, weights->sh_up, weights->sh_down};
    for (const void* p : sh)
      if (!p || !aligned16(p)) return MOE_ERR_INVALID_ARG;
  }
  const void* req[] = {x, y, ws};
  for (const void* p : req)
    if (!p || !aligned16(p)) return MOE_ERR_INVALID_ARG;
  if (residual && !aligned16(residual)) return MOE_ERR_INVALID_ARG;
  RouteWs w = carve(desc, T, ws);
  if (ws_bytes < w.bytes) return MOE_ERR_WORKSPACE_TOO_SMALL;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != cache->device) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int E = desc->n_experts, k = desc->top_k, S = cache->n_slots;
  // the shared expert runs as in moe_layer_forward (side stream, step 5), so the outputs agree bit for bit;
  // then the router is the first kernel on the caller's stream and clears the status word
  const bool early = shared_early_ok(shape_of(desc), x_dtype, T);
  // 1. routing by expert
  int rc = launch_route(weights->router_w, weights->router_bias, x, x_dtype, T, desc->hidden, E, k, w.logits,
                        w.topk_idx, w.topk_w, w.offsets, w.perm, w.inv, w.active, w.status, s, early);
  if (rc != OK) return to_status(rc);
  // 2. the experts this call needs (a copy to pageable host memory returns once the routing is done)
  if (cudaMemcpyAsync(cache->h_active.data(), w.active, (E + 1) * sizeof(int32_t), cudaMemcpyDeviceToHost, s) !=
          cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return MOE_ERR_CUDA;
  const int nact = cache->h_active[E];
  if (nact < 0 || nact > E) return MOE_ERR_CUDA;
  if (nact > S) return MOE_ERR_WORKSPACE_TOO_SMALL;  // the slots cannot hold every expert of this call
  // 3. hits keep their slot; each miss takes an empty slot or the least recently used one not needed now
  const uint64_t now = ++cache->tick;
  for (int i = 0; i < nact; ++i) {
    const int e = cache->h_active[i];
    if (e < 0 || e >= E) return MOE_ERR_CUDA;
    if (cache->slot_of[e] >= 0) {
      cache->last_use[cache->slot_of[e]] = now;
      ++cache->stats.hits;
    }
  }
  const size_t per[6] = {cache->pb.gate_codes, cache->pb.gate_d, cache->pb.up_codes,
                         cache->pb.up_d,       cache->pb.down_codes, cache->pb.down_dd};
  for (int i = 0; i < nact; ++i) {
    const int e = cache->h_active[i];
    if (cache->slot_of[e] >= 0) continue;
    int victim = -1;
    for (int q = 0; q < S; ++q) {
      if (cache->expert_in[q] < 0) {
        victim = q;
        break;
      }
      if (cache->last_use[q] < now && (victim < 0 || cache->last_use[q] < cache->last_use[victim])) victim = q;
    }
    if (victim < 0) return MOE_ERR_CUDA;  // cannot happen: nact <= S
    if (cache->expert_in[victim] >= 0) cache->slot_of[cache->expert_in[victim]] = -1;
    for (int pl = 0; pl < 6; ++pl) {
      if (cudaMemcpyAsync(cache->slot[pl] + per[pl] * victim, cache->host[pl] + per[pl] * e, per[pl],
                          cudaMemcpyHostToDevice, s) != cudaSuccess)
        return MOE_ERR_CUDA;
      cache->stats.bytes_copied += static_cast<int64_t>(per[pl]);
    }
    cache->expert_in[victim] = e;
    cache->slot_of[e] = victim;
    cache->last_use[victim] = now;
    ++cache->stats.misses;
  }
  ++cache->stats.calls;
  // 4. routing by slot: the expert -> slot map, then the permutation over the slots
  for (int e = 0; e < E; ++e) cache->h_map[e] = cache->slot_of[e] >= 0 ? cache->slot_of[e] : 0;
  if (cudaMemcpyAsync(cache->d_map, cache->h_map.data(), E * sizeof(int32_t), cudaMemcpyHostToDevice, s) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  rc = launch_remap_permute(w.topk_idx, T * k, cache->d_map, S, w.offsets, w.perm, w.inv, w.active, s);
  if (rc != OK) return to_status(rc);
  // 5. the expert FFN over the slots (the same kernels as the resident layer)
  moe_layer_desc sd = *desc;
  sd.n_experts = S;
  WeightPtrs wp = weights_of(weights);
  wp.gate_codes = cache->slot[0];
  wp.gate_d = reinterpret_cast<const uint16_t*>(cache->slot[1]);
  wp.up_codes = cache->slot[2];
  wp.up_d = reinterpret_cast<const uint16_t*>(cache->slot[3]);
  wp.down_codes = cache->slot[4];
  wp.down_dd = reinterpret_cast<const uint32_t*>(cache->slot[5]);
  Routing r{w.topk_w, w.offsets, w.perm, w.inv, w.active};
  const bool routed_clears = x_dtype == MOE_BF16 && router_tc_supported(T, desc->hidden, E);
  // the FFN's workspace part is sized for E experts, which covers S <= E slots (its layout does not depend on E)
  if (early) rc = launch_shared_early(shape_of(desc), wp, x, T, w.ffn, s);
  if (rc == OK)
    rc = launch_ffn(shape_of(&sd), wp, x, x_dtype, T, r, residual, y, w.ffn, w.status, !routed_clears && !early, s,
                    early);
  if (rc != OK && early) join_shared_early(s);
  return to_status(rc);
}


// ------------------------------------------------------------ MXFP4 experts
namespace {
// fmt 0 = MXFP4 (GEMVs up to 16 tokens, the block-scaled grouped GEMM above), 1 = Q4-style (GEMVs up to 16
// tokens, the dequantising grouped GEMM above)
moe_status check_mx(const moe_layer_desc* desc, int32_t T, int fmt) {
  moe_status st = check_desc(desc);
  if (st != MOE_OK) return st;
  if ((st = check_tokens(desc, T)) != MOE_OK) return st;
  const LayerShape sh = shape_of(desc);
  const bool ok = T <= kPrefillMinT ? mx_path_supported(sh, T)
                                     : (fmt == 0 ? mx_prefill_supported(sh, T) : prefill_path_supported(sh, T));
  if (T > 0 && !ok) return MOE_ERR_UNSUPPORTED_SHAPE;
  return MOE_OK;
}

moe_status blk32_workspace_size(const moe_layer_desc* desc, int32_t max_tokens, int fmt, size_t* bytes) {
  moe_status st = check_mx(desc, max_tokens, fmt);
  if (st != MOE_OK) return st;
  if (!bytes) return MOE_ERR_INVALID_ARG;
  *bytes = carve(desc, max_tokens, nullptr, mx_ffn_workspace_bytes(shape_of(desc), max_tokens, fmt)).bytes;
  return MOE_OK;
}
}  // namespace

moe_status moe_workspace_size_mxfp4(const moe_layer_desc* desc, int32_t max_tokens, size_t* bytes) {
  return blk32_workspace_size(desc, max_tokens, 0, bytes);
}

namespace {
// The layer forward over block-32 routed experts (MXFP4 or Q4-style): `planes` holds the three code planes
// and the three scale planes (their element type per `mp.fmt`), `shw` the router and the shared expert.
moe_status blk32_forward(const moe_layer_desc* desc, const WeightPtrs& shw, const MxPlanes& mp, const void* x,
                         moe_dtype x_dtype, int32_t T, const float* residual, float* y, void* ws, size_t ws_bytes,
                         void* stream) {
  moe_status st = check_mx(desc, T, mp.fmt);
  if (st != MOE_OK) return st;
  if (x_dtype != MOE_F32 && x_dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  const void* planes[] = {shw.router_w, mp.gate_codes, mp.gate_scales, mp.up_codes,
                          mp.up_scales, mp.down_codes, mp.down_scales};
  for (const void* p : planes)
    if (!p || !aligned16(p)) return MOE_ERR_INVALID_ARG;
  if (T > kPrefillMinT && mp.fmt == 0)  // the block-scaled GEMM's unpacking copy of the FP4 codes needs 32-byte bases
    for (const void* p : {static_cast<const void*>(mp.gate_codes), static_cast<const void*>(mp.up_codes),
                          static_cast<const void*>(mp.down_codes)})
      if (reinterpret_cast<uintptr_t>(p) % 32 != 0) return MOE_ERR_INVALID_ARG;
  if (shw.router_bias && !aligned16(shw.router_bias)) return MOE_ERR_INVALID_ARG;
  if (desc->shared_inter > 0) {
    const void* sh[] = {shw.sh_gate, shw.sh_up, shw.sh_down};
    for (const void* p : sh)
      if (!p || !aligned16(p)) return MOE_ERR_INVALID_ARG;
  }
  const void* req[] = {x, y, ws};
  for (const void* p : req)
    if (!p || !aligned16(p)) return MOE_ERR_INVALID_ARG;
  if (residual && !aligned16(residual)) return MOE_ERR_INVALID_ARG;
  const LayerShape sh = shape_of(desc);
  RouteWs w = carve(desc, T, ws, mx_ffn_workspace_bytes(sh, T, mp.fmt));
  if (ws_bytes < w.bytes) return MOE_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // as moe_layer_forward: the shared expert and the digits start first on the side stream (with this
  // path's workspace layout); every return after the fork joins it back
  const bool early = T <= kPrefillMinT && shared_early_ok(sh, x_dtype, T);
  int rc = OK;
  if (early) rc = launch_shared_early(sh, shw, x, T, w.ffn, s, mx_parts(sh.H), mx_parts(sh.I));
  if (rc == OK)
    rc = launch_route(shw.router_w, shw.router_bias, x, x_dtype, T, desc->hidden, desc->n_experts, desc->top_k,
                      w.logits, w.topk_idx, w.topk_w, w.offsets, w.perm, w.inv, w.active, w.status, s, early);
  if (rc == OK) {
    Routing r{w.topk_w, w.offsets, w.perm, w.inv, w.active};
    const bool routed_clears = x_dtype == MOE_BF16 && router_tc_supported(T, desc->hidden, desc->n_experts);
    rc = launch_ffn_mxfp4(sh, shw, mp, x, x_dtype, T, r, residual, y, w.ffn, w.status, !routed_clears && !early, s,
                          early);
  }
  if (rc != OK && early) join_shared_early(s);
  return to_status(rc);
}

WeightPtrs blk32_shared(const uint16_t* router_w, const float* router_bias, const uint16_t* sh_gate,
                        const uint16_t* sh_up, const uint16_t* sh_down) {
  WeightPtrs shw{};  // router and shared expert (the routed fields are unused on this path)
  shw.router_w = router_w;
  shw.router_bias = router_bias;
  shw.sh_gate = sh_gate;
  shw.sh_up = sh_up;
  shw.sh_down = sh_down;
  return shw;
}
}  // namespace

moe_status moe_layer_forward_mxfp4(const moe_layer_desc* desc, const moe_mxfp4_weights* weights, const void* x,
                                   moe_dtype x_dtype, int32_t T, const float* residual, float* y, void* ws,
                                   size_t ws_bytes, void* stream) {
  if (!weights) return T == 0 && check_mx(desc, T, 0) == MOE_OK ? MOE_OK : MOE_ERR_INVALID_ARG;
  const MxPlanes mp{0, weights->gate_codes, weights->gate_scales, weights->up_codes,
                    weights->up_scales, weights->down_codes, weights->down_scales};
  return blk32_forward(desc,
                       blk32_shared(weights->router_w, weights->router_bias, weights->sh_gate, weights->sh_up,
                                    weights->sh_down),
                       mp, x, x_dtype, T, residual, y, ws, ws_bytes, stream);
}

moe_status moe_workspace_size_q4(const moe_layer_desc* desc, int32_t max_tokens, size_t* bytes) {
  return blk32_workspace_size(desc, max_tokens, 1, bytes);
}

moe_status moe_layer_forward_q4(const moe_layer_desc* desc, const moe_q4_weights* weights, const void* x,
                                moe_dtype x_dtype, int32_t T, const float* residual, float* y, void* ws,
                                size_t ws_bytes, void* stream) {
  if (!weights) return T == 0 && check_mx(desc, T, 1) == MOE_OK ? MOE_OK : MOE_ERR_INVALID_ARG;
  const MxPlanes mp{1, weights->gate_codes, weights->gate_d, weights->up_codes,
                    weights->up_d, weights->down_codes, weights->down_d};
  return blk32_forward(desc,
                       blk32_shared(weights->router_w, weights->router_bias, weights->sh_gate, weights->sh_up,
                                    weights->sh_down),
                       mp, x, x_dtype, T, residual, y, ws, ws_bytes, stream);
}

moe_status moe_debug_dequant_q4(const uint8_t* codes, const uint16_t* d, int64_t n_blocks, float* out,
                                void* stream) {
  if (!codes || !d || !out || n_blocks < 0) return MOE_ERR_INVALID_ARG;
  return to_status(launch_mx_dequant(1, codes, d, n_blocks, out, static_cast<cudaStream_t>(stream)));
}

moe_status moe_debug_dequant_mxfp4(const uint8_t* codes, const uint8_t* scales, int64_t n_blocks, float* out,
                                   void* stream) {
  if (!codes || !scales || !out || n_blocks < 0) return MOE_ERR_INVALID_ARG;
  return to_status(launch_mx_dequant(0, codes, scales, n_blocks, out, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
