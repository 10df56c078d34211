// common.cuh - formats, compile-time codebook and small device helpers of the
// routed 2-bit MoE FFN library (sm_100a).
//
// Block formats (library specification; the ds4 pages name only "IQ2_XXS" for
// up/gate and "Q2_K" for down: "ds4 : analyse pratique pour un usage
// documenté", section « Support de modèles et choix de quantification »):
//   IQ2-style, 256 weights: 64 code bytes + fp16 d. Sub-block s = bytes 8s..8s+7;
//     bytes 8s+j = codebook row of group j; u32 v = bytes 8s+4..8s+7 holds the
//     7-bit sign field of group j at bits 7j.. and the scale ls at bits 28..31;
//     element 7 of a group is negative iff its sign field has odd popcount.
//     w = d * (2 ls + 1) * grid[row][e] * sign / 8.
//   Q2K-style, 256 weights: 80 code bytes + u32 (fp16 d | fp16 dmin << 16).
//     Byte s < 16: sc | m << 4 of sub-block s (16 weights); byte 16+i holds
//     weights 4i..4i+3 at bits 2r. w = d * sc * q - dmin * m.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace moe {

constexpr int QK = 256;
constexpr int IQ2_BYTES = 64;
constexpr int Q2K_BYTES = 80;

// ---------------------------------------------------------------------------
// The IQ2 codebook, generated at compile time from its definition: splitmix64
// (Steele, Lea, Flood 2014) seeded 0x4951325F47524944; c = (next() >> 32) mod
// 6561, duplicates rejected, 256 rows in acceptance order; element e = base-3
// digit e of c (least significant first) mapped 0 -> 8, 1 -> 25, 2 -> 43.
struct Iq2Codebook {
  uint16_t code[256];  // c of each row (base-3 word, < 6561)
  uint8_t val[256][8]; // magnitudes
};

constexpr uint64_t splitmix64_step(uint64_t& state) {
  state += 0x9E3779B97F4A7C15ull;
  uint64_t z = state;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

constexpr Iq2Codebook make_iq2_codebook() {
  Iq2Codebook cb{};
  uint64_t st = 0x4951325F47524944ull;
  int n = 0;
  while (n < 256) {
    uint32_t c = static_cast<uint32_t>((splitmix64_step(st) >> 32) % 6561u);
    bool seen = false;
    for (int i = 0; i < n; ++i) seen = seen || cb.code[i] == c;
    if (!seen) cb.code[n++] = static_cast<uint16_t>(c);
  }
  const uint8_t level[3] = {8, 25, 43};
  for (int r = 0; r < 256; ++r) {
    uint32_t c = cb.code[r];
    for (int e = 0; e < 8; ++e) {
      cb.val[r][e] = level[c % 3];
      c /= 3;
    }
  }
  return cb;
}

inline constexpr Iq2Codebook kCodebook = make_iq2_codebook();

// ---------------------------------------------------------------------------
// Status (mirrors moe_status of the public header).
enum Status : int { OK = 0, ERR_ARG = 1, ERR_SHAPE = 2, ERR_WS = 3, ERR_CUDA = 4, ERR_TIMEOUT = 5 };

__device__ __forceinline__ float half_bits_to_float(uint16_t h) {
  float f;
  asm("{ .reg .f16 t; mov.b16 t, %1; cvt.f32.f16 %0, t; }" : "=f"(f) : "h"(h));
  return f;
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }

__device__ __forceinline__ float silu_mul(float g, float u) { return g / (1.0f + __expf(-g)) * u; }

__host__ __device__ constexpr inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace moe
