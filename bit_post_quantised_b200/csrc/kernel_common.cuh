// kernel_common.cuh -- device helpers shared by the ternary MMA kernels:
// the 2-bit code expansion to bf16 and the shared-memory matrix descriptor.
#pragma once
#include <cstdint>

namespace tern {

// ------------------------------------------------------------------ decode
__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Expands one 32-bit code word (16 consecutive k: even k in bits 2j of the
// low half-word, odd k in bits 16+2j) into eight bf16x2 words, pair j = (k0 +
// 2j, k0 + 2j + 1).  For the code u at bits [2j, 2j+1] of each half-word:
// masking keeps u, XOR-ing with the bf16 pattern of (2^(7-2j) + 2) flips u's
// top bit (u ^ 2 = t + 2 for the two's-complement t) and supplies an exponent
// that makes bit 2j the units bit, giving the bf16 value 2^(7-2j) + t + 2.
// Subtracting the same constant leaves exactly t.  Three pairs share one
// shift, so a word costs 2 shifts + 8 LOP3 + 8 bf16x2 subtracts.
__device__ __forceinline__ void decode_word(uint32_t w, uint32_t* out) {
  constexpr uint32_t M0 = 0x00030003u, M1 = 0x000C000Cu, M2 = 0x00300030u;
  constexpr uint32_t C0 = 0x43024302u;  // bf16 130 = 128 + 2
  constexpr uint32_t C1 = 0x42084208u;  // bf16 34  = 32 + 2
  constexpr uint32_t C2 = 0x41204120u;  // bf16 10  = 8 + 2
  const uint32_t w1 = w >> 6, w2 = w >> 12;
  out[0] = bf16x2_sub((w & M0) ^ C0, C0);
  out[1] = bf16x2_sub((w & M1) ^ C1, C1);
  out[2] = bf16x2_sub((w & M2) ^ C2, C2);
  out[3] = bf16x2_sub((w1 & M0) ^ C0, C0);
  out[4] = bf16x2_sub((w1 & M1) ^ C1, C1);
  out[5] = bf16x2_sub((w1 & M2) ^ C2, C2);
  out[6] = bf16x2_sub((w2 & M0) ^ C0, C0);
  out[7] = bf16x2_sub((w2 & M1) ^ C1, C1);
}

// bf16x2 of 2t for the code pair J (k and k + 1) of a code word: shifted so
// that the two bits of each half-word's code land on bits 15 and 14, a
// two's-complement code is exactly the bf16 2t (0x4000 = 2, 0xC000 = -2,
// 0 = 0), so a pair costs one shift and one AND (none for J = 7).  Sums of
// 2t products are halved, exactly, with the scale.
template <int J>
__device__ __forceinline__ uint32_t code_pair_2t(uint32_t w) {
  return (J == 7 ? w : (w << (14 - 2 * J))) & 0xC000C000u;
}

// The eight bf16x2 pairs of 2t of one code word, pair j = (k0 + 2j, k0 + 2j + 1).
__device__ __forceinline__ void decode_word_2t(uint32_t w, uint32_t* out) {
  out[0] = code_pair_2t<0>(w);
  out[1] = code_pair_2t<1>(w);
  out[2] = code_pair_2t<2>(w);
  out[3] = code_pair_2t<3>(w);
  out[4] = code_pair_2t<4>(w);
  out[5] = code_pair_2t<5>(w);
  out[6] = code_pair_2t<6>(w);
  out[7] = code_pair_2t<7>(w);
}

// Shared-memory matrix descriptor of a K-major bf16 tile written by TMA with
// 128-byte swizzle: rows of 128 bytes, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= uint64_t((saddr & 0x3FFFFu) >> 4);  // start address
  d |= uint64_t(1) << 16;                   // leading byte offset (unused when swizzled)
  d |= uint64_t(1024 >> 4) << 32;           // stride byte offset: next 8-row group
  d |= uint64_t(1) << 46;                   // descriptor version for sm_100
  d |= uint64_t(2) << 61;                   // SWIZZLE_128B
  return d;
}

// Epilogue activations (the values of tern_act in tern.h).
constexpr int kActNone = 0;
constexpr int kActGeluTanh = 1;

// The tanh form of GELU, g(v) = 0.5 v (1 + tanh(u)), u = sqrt(2/pi) (v +
// 0.044715 v^3), evaluated as v / (1 + e^(-2u)) (the same function, since
// 0.5 (1 + tanh(u)) = 1 / (1 + e^(-2u))): no cancellation for large negative
// v, where 1 + tanh(u) would lose its digits.  fp32, a few ulp.
__device__ __forceinline__ float gelu_tanh(float v) {
  const float u = 0.7978845608028654f * fmaf(0.044715f * v, v * v, v);
  // e^(-2u) overflows to +inf for u < -44: the quotient is then 0 (as the
  // true value, |g| < 1e-37, rounds to in bf16).
  return __fdividef(v, 1.0f + __expf(-2.0f * u));
}

// y = v or act(v) for output channel n, given the problem's activation and
// its first activated column.
__device__ __forceinline__ float apply_act(float v, int act, int n, int act_col0) {
  return (act == kActGeluTanh && n >= act_col0) ? gelu_tanh(v) : v;
}

// The whole epilogue after v = acc * s + b, in fp32 (one rounding follows):
// a = act(v) on the activated columns, then residual[m, n] + gate[n] * a
// where a residual is given (gate 1 where none is).
__device__ __forceinline__ float epilogue_value(float v, int act, int n, int act_col0, const uint16_t* residual,
                                                size_t mn, float gate) {
  const float a = apply_act(v, act, n, act_col0);
  return residual ? fmaf(gate, a, __uint_as_float(uint32_t(residual[mn]) << 16)) : gate * a;
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(uint32_t(b) << 16);
}

}  // namespace tern
