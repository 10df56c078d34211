// decode.cuh - shared pieces of the tensor-core dequant-GEMV path (decode.cu,
// gateup.cu, down.cu): PRMT tables for the IQ2-style codes, the activation digit
// split, and the argument blocks of the kernels.
//
// Arithmetic (exact integer inner products):
//   IQ2 weights enter the MMA as int8 values +-{8, 25, 43}: a PRMT from two
//   registers holding those six bytes, driven by a selector built from the
//   codebook row (2-bit level codes) OR the sign field (bit 2 of each nibble).
//   Q2K weights enter as uint8 q in 0..3.
//   Activations enter as two int8 digits per element: with a power-of-two scale
//   2^s per 256-element block, q = rint(x / 2^s) in [-4096, 4096],
//   q = 128 hi + lo with hi in [-32, 32], lo in [-64, 63]. Products and
//   per-block sums are exact in int32; the block scales (d, 2ls+1, sc, m, 2^s)
//   are applied after, sc and m as integers, d and 2^s in fp32.
//   "Column packing": with one or two tokens per expert, the 8 columns of the
//   m16n8k32 MMA hold (sub-block slot, token, digit) instead of 8 tokens, so that
//   several sub-blocks with different scales share one accumulator set.
#pragma once
#include "common.cuh"

namespace moe {

// ------------------------------------------------------------ PRMT tables
struct Iq2SelTables {
  uint32_t level[256];  // nibble e = level code (0, 1, 2) of codebook element e
  uint32_t sign[128];   // nibble e bit 2 = sign of element e (element 7 from parity)
};
constexpr Iq2SelTables make_sel_tables() {
  Iq2SelTables t{};
  for (int r = 0; r < 256; ++r) {
    uint32_t w = 0;
    for (int e = 0; e < 8; ++e) {
      const uint32_t v = kCodebook.val[r][e];
      const uint32_t code = v == 8 ? 0u : (v == 25 ? 1u : 2u);
      w |= code << (4 * e);
    }
    t.level[r] = w;
  }
  for (int s = 0; s < 128; ++s) {
    uint32_t w = 0, par = 0;
    for (int e = 0; e < 7; ++e) {
      const uint32_t b = (s >> e) & 1u;
      par ^= b;
      w |= b << (4 * e + 2);
    }
    w |= par << (4 * 7 + 2);
    t.sign[s] = w;
  }
  return t;
}

constexpr uint32_t kPosBytes = 0x002B1908u;  // bytes 8, 25, 43, 0
constexpr uint32_t kNegBytes = 0x00D5E7F8u;  // bytes -8, -25, -43, 0

__device__ __forceinline__ int floor_log2_pos(float m) {
  const uint32_t b = __float_as_uint(m);
  const int e = static_cast<int>((b >> 23) & 0xFFu);
  if (e) return e - 127;
  return -149 + (31 - __clz(b & 0x7FFFFFu));
}

// Split x = 2^s * (128 hi + lo) (up to the rounding of q = rint(x / 2^s)).
__device__ __forceinline__ void split_digits(float x, int s, int& hi, int& lo) {
  const int q = __float2int_rn(ldexpf(x, -s));
  hi = (q + 64) >> 7;
  lo = q - (hi << 7);
}

// ------------------------------------------------------------ gate/up
struct GateupArgs {
  int H, I, E, k, T;
  const uint8_t* gate_codes;
  const uint16_t* gate_d;
  const uint8_t* up_codes;
  const uint16_t* up_d;
  const int8_t* xd;   // [T][2][H] activation digits
  const float* xs;    // [T][H/256] 2^s / 8
  const int32_t* offsets;
  const int32_t* perm;
  const int32_t* active;
  float* gu;     // [T*k][2][I] gate (plane 0) and up (plane 1) outputs per assignment
  int* err;
  int stages;
  int x_in_smem;  // 1: all T tokens' digits staged in shared memory once per CTA
};

// ------------------------------------------------------------ down
struct DownArgs {
  int H, I, E, k;
  const uint8_t* codes;
  const uint32_t* dd;
  const int8_t* hd;   // [T*k][2][I] digits of h, interleaved per 32-block for the MMA
  const float* hsc;   // [T*k][round_up(I/256, 4)] 2^s of each 256-block of h
  const int32_t* hq;  // [T*k][I/16] sum of q over each 16-block of h
  const int32_t* offsets;
  const int32_t* active;
  float* o;  // [T*k][H]
  int* err;
  int stages;
};

int launch_gateup(const GateupArgs& a, int slots, int sms, cudaStream_t st);
int launch_down(const DownArgs& a, int slots, int T, int sms, cudaStream_t st);

}  // namespace moe
