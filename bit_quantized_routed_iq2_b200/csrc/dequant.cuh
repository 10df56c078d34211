// dequant.cuh - block-dequantisation unit (device functions) for the two 2-bit
// formats of the routed experts: IQ2-style (gate/up) and Q2K-style (down).
//
// Exactness: every IQ2-style value d * (2ls+1) * g / 8 has at most 11 + 5 + 6
// significant bits, so each fp32 product below is exact; a Q2K-style value is
// d*sc*q (exact, <= 17 bits) minus dmin*m (exact, <= 15 bits), one rounding,
// which fmaf or a plain subtraction give identically. The decoded fp32 values
// are therefore bit-identical to the format's definition.
#pragma once
#include "common.cuh"

namespace moe {

// Codebook magnitudes for device use (row-major 256 x 8 bytes), from the
// compile-time generator in common.cuh.
struct GridBytes {
  uint32_t w[512];
};
constexpr GridBytes make_grid_bytes() {
  GridBytes g{};
  for (int r = 0; r < 256; ++r)
    for (int e = 0; e < 8; ++e) g.w[r * 2 + e / 4] |= static_cast<uint32_t>(kCodebook.val[r][e]) << (8 * (e % 4));
  return g;
}
__device__ const GridBytes d_grid_bytes = make_grid_bytes();

// Copy the 2 KB codebook into shared memory (call with all threads, then sync).
__device__ __forceinline__ void load_grid_smem(uint32_t* s_grid) {
  for (int i = threadIdx.x; i < 512; i += blockDim.x) s_grid[i] = d_grid_bytes.w[i];
}

// IQ2-style group: `idx` = codebook row, `sigma` = 7-bit sign field, `scale` =
// d * (2ls+1) / 8 (exact). Writes the 8 weights.
__device__ __forceinline__ void iq2_group(const uint32_t* s_grid, uint32_t idx, uint32_t sigma, float scale,
                                          float out[8]) {
  const uint32_t lo = s_grid[idx * 2], hi = s_grid[idx * 2 + 1];
  const uint32_t signs = sigma | ((__popc(sigma) & 1u) << 7);
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float mag = static_cast<float>(((e < 4 ? lo : hi) >> (8 * (e & 3))) & 0xFFu);
    const float v = scale * mag;
    out[e] = ((signs >> e) & 1u) ? -v : v;
  }
}

// Scale of IQ2 sub-block with code word v: d * (2ls+1) / 8, exact.
__device__ __forceinline__ float iq2_scale(float d, uint32_t v) {
  return d * static_cast<float>(2 * (v >> 28) + 1) * 0.125f;
}

// Q2K-style weight from its fields.
__device__ __forceinline__ float q2k_value(float d, float dmin, uint32_t sc, uint32_t m, uint32_t q) {
  return fmaf(d, static_cast<float>(sc * q), -(dmin * static_cast<float>(m)));
}

}  // namespace moe
