// profile.cu - optional per-kernel CUDA-event timing of the library's launches.
#include <vector>

#include "../../include/moe2bit.h"
#include "profile.cuh"

namespace moe {

namespace {
struct Record {
  int kid;
  int ev;  // index of the start event; stop is ev + 1
};
struct ProfState {
  bool on = false;
  std::vector<cudaEvent_t> pool;
  std::vector<Record> recs;
  int open_kid = -1;
};
ProfState g_prof;
constexpr int kPoolEvents = 16384;
}  // namespace

void prof_start(int kid, cudaStream_t st) {
  if (!g_prof.on) return;
  const size_t ev = g_prof.recs.size() * 2;
  if (ev + 2 > g_prof.pool.size()) return;
  cudaEventRecord(g_prof.pool[ev], st);
  g_prof.recs.push_back(Record{kid, static_cast<int>(ev)});
}

void prof_stop(int kid, cudaStream_t st) {
  if (!g_prof.on || g_prof.recs.empty()) return;
  const Record& r = g_prof.recs.back();
  if (r.kid != kid) return;
  cudaEventRecord(g_prof.pool[r.ev + 1], st);
}

}  // namespace moe

using namespace moe;

extern "C" {

moe_status moe_profile_enable(int32_t on) {
  if (on && !g_prof.on) {
    g_prof.pool.resize(kPoolEvents);
    for (auto& e : g_prof.pool)
      if (cudaEventCreate(&e) != cudaSuccess) return MOE_ERR_CUDA;
    g_prof.recs.clear();
    g_prof.on = true;
  } else if (!on && g_prof.on) {
    for (auto& e : g_prof.pool) cudaEventDestroy(e);
    g_prof.pool.clear();
    g_prof.recs.clear();
    g_prof.on = false;
  }
  return MOE_OK;
}

moe_status moe_profile_read(float* total_ms, int32_t* launches) {
  if (!total_ms || !launches) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < MOE_K_COUNT; ++i) {
    total_ms[i] = 0.f;
    launches[i] = 0;
  }
  moe_status st = MOE_OK;
  for (const Record& r : g_prof.recs) {
    float ms = 0.f;
    if (cudaEventSynchronize(g_prof.pool[r.ev + 1]) != cudaSuccess ||
        cudaEventElapsedTime(&ms, g_prof.pool[r.ev], g_prof.pool[r.ev + 1]) != cudaSuccess) {
      st = MOE_ERR_CUDA;
      continue;
    }
    if (r.kid >= 0 && r.kid < MOE_K_COUNT) {
      total_ms[r.kid] += ms;
      launches[r.kid] += 1;
    }
  }
  g_prof.recs.clear();
  return st;
}

}  // extern "C"
