// noalloc.cu - moe_layer_forward_noalloc: the whole layer with the scratch
// memory taken from a fixed array that is part of the library image itself.
//
// Who needs this: callers that cannot obtain device memory on their own, such
// as a plugin invoked by a host engine that hands out no workspace, or a
// serving loop that must not allocate after start-up (cudaMalloc may
// synchronise the device and stall every stream). They still pass inputs and
// outputs; only the scratch moves into the library.
//
// The array below lives in device memory on every GPU that loads the library,
// from module load until process exit. Host code cannot use its name as a
// device address (the name denotes a host-side shadow), so the address is
// looked up with cudaGetSymbolAddress once per device, with that device
// current, and cached.
#include <atomic>
#include <mutex>

#include "../../include/moe2bit.h"

static constexpr size_t kNoallocScratchBytes = size_t(32) << 20;  // MOE_NOALLOC_SCRATCH_BYTES in the header
static_assert(kNoallocScratchBytes == MOE_NOALLOC_SCRATCH_BYTES, "header and library disagree on the size");

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

namespace {

constexpr int kMaxDevices = 64;
std::atomic<void*> g_scratch_addr[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device (set-up on the
// first call per device). Returns MOE_ERR_CUDA if the runtime refuses.
moe_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
  void* p = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (!p) {
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    p = g_scratch_addr[dev].load(std::memory_order_relaxed);
    if (!p) {
      if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return MOE_ERR_CUDA;
      g_scratch_addr[dev].store(p, std::memory_order_release);
    }
  }
  *out = p;
  return MOE_OK;
}

}  // namespace

extern "C" {

moe_status moe_layer_forward_noalloc(const moe_layer_desc* desc, const moe_layer_weights* w, const void* x,
                                     moe_dtype x_dtype, int32_t T, const float* residual, float* y,
                                     void* stream) {
  size_t need = 0;
  moe_status st = moe_workspace_size(desc, T < 0 ? 0 : T, &need);
  if (st != MOE_OK) return st;
  if (T < 0) return MOE_ERR_INVALID_ARG;
  if (need > kNoallocScratchBytes) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if (T == 0) return MOE_OK;
  void* scratch = nullptr;
  if ((st = scratch_address(&scratch)) != MOE_OK) return st;
  return moe_layer_forward(desc, w, x, x_dtype, T, residual, y, scratch, kNoallocScratchBytes, stream);
}

moe_status moe_read_status_noalloc(int32_t* status, void* stream) {
  if (!status) return MOE_ERR_INVALID_ARG;
  void* scratch = nullptr;
  moe_status st = scratch_address(&scratch);
  if (st != MOE_OK) return st;
  return moe_read_status(scratch, status, stream);
}

}  // extern "C"
