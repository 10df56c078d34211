// profile.cuh - hooks around each launch for the optional kernel timing.
#pragma once
#include <cuda_runtime.h>

#include "../../include/moe2bit.h"

namespace moe {
void prof_start(int kid, cudaStream_t st);
void prof_stop(int kid, cudaStream_t st);

// Records start/stop events around the launches in its scope when timing is on.
struct ProfScope {
  int kid;
  cudaStream_t st;
  ProfScope(int k, cudaStream_t s) : kid(k), st(s) { prof_start(kid, st); }
  ~ProfScope() { prof_stop(kid, st); }
};
}  // namespace moe
