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

// Offset of digit d of element e (a multiple of 8) of token t in the staged
// activations: per token 2*H bytes; block b (256 elements) takes 512 bytes, its
// sub-block s (32 elements) 64 bytes, digit d at +32d, and the two 16-element
// halves c of the sub-block at +16*(c ^ (b & 1)). The half swap on odd blocks
// makes the B loads of the one-token unit below conflict-free.
__host__ __device__ __forceinline__ int x_off(int H, int t, int d, int e) {
  const int b = e >> 8;
  return t * 2 * H + b * 512 + ((e >> 5) & 7) * 64 + d * 32 + 16 * (((e >> 4) & 1) ^ (b & 1)) + (e & 15);
}

// Offset of digit d of element e (of I) of assignment p in the h digits (global
// and staged alike): per assignment 2*I bytes; block b (256 elements) takes 512
// bytes; its 16-element sub-block S = 4t + c (t = S >> 2, c = S & 3) takes 16
// bytes per digit at c*128 + t*32 + d*16, element 4i + r at byte 4r + i. So one
// 16-byte load gives a lane the four bytes of each bit pair r of its sub-block
// (the K order of q2k_quad), and the eight lanes that carry B in the one-token
// unit hit eight different 16-byte bank groups.
__host__ __device__ __forceinline__ int h_off(int I, int p, int d, int e) {
  const int S = (e >> 4) & 15, j = e & 15;
  return p * 2 * I + (e >> 8) * 512 + (S & 3) * 128 + (S >> 2) * 32 + d * 16 + 4 * (j & 3) + (j >> 2);
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


// Second half of the h quantiser, by one warp (8 elements per lane, lane l
// holding elements 8l .. 8l+7 of the 256-element block sb of assignment p):
// h = silu(g) * u from the summed gate/up rows, split into int8 digits with
// one power-of-two scale per block and stored in the order the down MMA reads
// them (kHOff: the h_off layout of the TMA-fed down GEMV; otherwise rows of I
// per digit where, inside each 32-element block, element j of sub-block half
// sub goes to byte 8*(j%4) + 4*sub + j/4), with the exact integer sum of
// q = 128 hi + lo per 16-element sub-block (the min term of the Q2K-style down
// projection).
template <bool kHOff>
__device__ __forceinline__ void hquant_finish_warp(int I, int p, int sb, const float (&gv)[8], const float (&uv)[8],
                                                   int8_t* __restrict__ hd, float* __restrict__ hsc,
                                                   int32_t* __restrict__ hq, int hss, int lane) {
  const int base = sb * 256 + lane * 8;
  float h[8], m = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    h[i] = silu_mul(gv[i], uv[i]);
    m = fmaxf(m, fabsf(h[i]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  // the TMA-fed down GEMV takes 14-bit digits (|q| <= 8192), the other one 13-bit (see x_digits_kernel)
  const int e = m > 0.f ? floor_log2_pos(m) - (kHOff ? 12 : 11) : 0;
  int qs = 0;
  int8_t* hi_row = hd + static_cast<size_t>(p) * 2 * I;
  int8_t* lo_row = hi_row + I;
  const int blk32 = base >> 5, jj0 = base & 31;  // this lane's 8 elements sit in one 32-block
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    int hi = 0, lo = 0;
    if (m > 0.f) split_digits(h[i], e, hi, lo);
    qs += hi * 128 + lo;
    if (kHOff) {
      hd[h_off(I, p, 0, base + i)] = static_cast<int8_t>(hi);
      hd[h_off(I, p, 1, base + i)] = static_cast<int8_t>(lo);
    } else {
      const int jj = jj0 + i, sub = jj >> 4, j = jj & 15;
      const int pos = blk32 * 32 + 8 * (j & 3) + 4 * sub + (j >> 2);
      hi_row[pos] = static_cast<int8_t>(hi);
      lo_row[pos] = static_cast<int8_t>(lo);
    }
  }
  qs += __shfl_xor_sync(0xffffffffu, qs, 1);  // lanes 2i, 2i+1 hold one 16-element sub-block
  if ((lane & 1) == 0) hq[static_cast<size_t>(p) * (I / 16) + sb * 16 + (lane >> 1)] = qs;
  if (lane == 0) hsc[static_cast<size_t>(p) * hss + sb] = m > 0.f ? ldexpf(1.0f, e) : 0.f;
}

}  // namespace moe
