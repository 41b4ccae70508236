// adaln.cu -- FLUX.1's adaLN modulation of layer-normalised activations, in
// one pass over HBM.
//
// Page "1.58-bit FLUX" (arXiv 2412.18653) quantises every linear of FLUX.1's
// blocks (Section 3.1) and keeps the activations in 16 bits (Section 4); it
// does not describe the operations between the linears.  Each block feeds its
// first linears with its token rows layer-normalised (no affine) and
// modulated by two rows of its adaLN modulation output (the M = 1 linears of
// the modulation layers):
//   out[m,k] = (x[m,k] - mean_m) / sqrt(var_m + eps) * (1 + scale[g,k]) + shift[g,k],
// g = m / tokens_per_row.  Unfused that is a normalisation, a multiply and an
// add, each reading and writing the activations.  Here one warp owns one
// row and holds it in registers (16-byte loads, all issued before the first
// is used), takes the mean and then the variance about the mean in fp32, and
// writes the modulated row rounded once to bf16: x is read once and out
// written once.  out may be x itself (the warp has read its whole row before
// it stores).  At 64 registers four 8-warp CTAs fit an SM, so the 4608 rows
// of a FLUX.1 single block's stream run in one wave.
#include "internal.h"
#include "kernel_common.cuh"
#include "ptx.cuh"

namespace tern {

namespace {

constexpr int kAdaRows = 8;  // rows (warps) per CTA

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
// The same conversions written as byte permutes, for the passes after the
// first: the compiler then recomputes them from the packed row instead of
// keeping every converted value live between passes (twice the registers).
__device__ __forceinline__ float bf16_lo_p(uint32_t w) {
  uint32_t d;
  asm("prmt.b32 %0, %1, 0, 0x1044;" : "=r"(d) : "r"(w));
  return __uint_as_float(d);
}
__device__ __forceinline__ float bf16_hi_p(uint32_t w) {
  uint32_t d;
  asm("prmt.b32 %0, %1, 0, 0x3244;" : "=r"(d) : "r"(w));
  return __uint_as_float(d);
}
__device__ __forceinline__ float bf16_lo_q(uint32_t w) {
  uint32_t d;
  asm("prmt.b32 %0, 0, %1, 0x5400;" : "=r"(d) : "r"(w));
  return __uint_as_float(d);
}
__device__ __forceinline__ float bf16_hi_q(uint32_t w) {
  uint32_t d;
  asm("prmt.b32 %0, 0, %1, 0x7600;" : "=r"(d) : "r"(w));
  return __uint_as_float(d);
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

// Read-only 16-byte load kept in program order (asm volatile): the scale and
// shift groups are loaded one step at a time (L1 hits after the first warp of
// a CTA) instead of all hoisted ahead of the loop, which would hold 8 NV
// registers and halve the CTAs per SM.
__device__ __forceinline__ uint4 ld_nc_v4_ordered(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

// (v - mean) * rstd * (1 + s) + h for the two values of a word.
__device__ __forceinline__ uint32_t modulate2(uint32_t xv, uint32_t sv, uint32_t hv, float mean, float rstd) {
  const float a = (bf16_lo_q(xv) - mean) * rstd, b = (bf16_hi_q(xv) - mean) * rstd;
  return pack2(fmaf(a, 1.f + bf16_lo(sv), bf16_lo(hv)), fmaf(b, 1.f + bf16_hi(sv), bf16_hi(hv)));
}

// NV 16-byte groups per lane: k = 8i .. 8i + 7 for i = lane + 32 t, t < NV
// (K <= 256 NV).  x and out are not __restrict__: they may be one buffer.
template <int NV>
__global__ void __launch_bounds__(kAdaRows * 32, 4)
    adaln_modulate_kernel(const uint16_t* x, int M, int K, const uint16_t* __restrict__ scale,
                          const uint16_t* __restrict__ shift, int mod_ld, int tokens_per_row, float eps,
                          uint16_t* out) {
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m = blockIdx.x * kAdaRows + warp;
  if (m >= M) return;
  const uint4* row = reinterpret_cast<const uint4*>(x + size_t(m) * K);
  const int n8 = K >> 3;
  uint4 v[NV];
#pragma unroll
  for (int t = 0; t < NV; ++t) {
    const int i = lane + 32 * t;
    v[t] = i < n8 ? row[i] : make_uint4(0u, 0u, 0u, 0u);
  }
  // ---- mean (absent groups are zeros and add nothing)
  float sum = 0.f;
#pragma unroll
  for (int t = 0; t < NV; ++t) {
    const float a = (bf16_lo(v[t].x) + bf16_hi(v[t].x)) + (bf16_lo(v[t].y) + bf16_hi(v[t].y));
    const float b = (bf16_lo(v[t].z) + bf16_hi(v[t].z)) + (bf16_lo(v[t].w) + bf16_hi(v[t].w));
    sum += a + b;
  }
  const float mean = warp_sum(sum) / float(K);
  // ---- biased variance about the mean
  float sq = 0.f;
#pragma unroll
  for (int t = 0; t < NV; ++t) {
    if (lane + 32 * t < n8) {
      const uint32_t w[4] = {v[t].x, v[t].y, v[t].z, v[t].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float a = bf16_lo_p(w[e]) - mean, b = bf16_hi_p(w[e]) - mean;
        sq = fmaf(a, a, fmaf(b, b, sq));
      }
    }
  }
  const float rstd = rsqrtf(warp_sum(sq) / float(K) + eps);
  // ---- modulate and store
  const int g = m / tokens_per_row;
  const uint4* sc = reinterpret_cast<const uint4*>(scale + size_t(g) * mod_ld);
  const uint4* sh = reinterpret_cast<const uint4*>(shift + size_t(g) * mod_ld);
  uint4* orow = reinterpret_cast<uint4*>(out + size_t(m) * K);
#pragma unroll
  for (int t = 0; t < NV; ++t) {
    const int i = lane + 32 * t;
    if (i < n8) {
      const uint4 s = ld_nc_v4_ordered(sc + i), h = ld_nc_v4_ordered(sh + i);
      uint4 o;
      o.x = modulate2(v[t].x, s.x, h.x, mean, rstd);
      o.y = modulate2(v[t].y, s.y, h.y, mean, rstd);
      o.z = modulate2(v[t].z, s.z, h.z, mean, rstd);
      o.w = modulate2(v[t].w, s.w, h.w, mean, rstd);
      orow[i] = o;
    }
  }
}

template <int NV>
cudaError_t launch_nv(const uint16_t* x, int M, int K, const uint16_t* scale, const uint16_t* shift, int mod_ld,
                      int tokens_per_row, float eps, uint16_t* out, cudaStream_t stream) {
  const int grid = (M + kAdaRows - 1) / kAdaRows;
  return launch_pdl(adaln_modulate_kernel<NV>, dim3(grid), dim3(kAdaRows * 32), 0, stream, 1, x, M, K, scale, shift,
                    mod_ld, tokens_per_row, eps, out);
}

}  // namespace

cudaError_t launch_adaln_modulate(const __nv_bfloat16* x, int M, int K, const __nv_bfloat16* scale,
                                  const __nv_bfloat16* shift, int mod_ld, int tokens_per_row, float eps,
                                  __nv_bfloat16* out, cudaStream_t stream) {
  const uint16_t* xs = reinterpret_cast<const uint16_t*>(x);
  const uint16_t* ss = reinterpret_cast<const uint16_t*>(scale);
  const uint16_t* hs = reinterpret_cast<const uint16_t*>(shift);
  uint16_t* os = reinterpret_cast<uint16_t*>(out);
  if (K <= 256) return launch_nv<1>(xs, M, K, ss, hs, mod_ld, tokens_per_row, eps, os, stream);
  if (K <= 512) return launch_nv<2>(xs, M, K, ss, hs, mod_ld, tokens_per_row, eps, os, stream);
  if (K <= 1024) return launch_nv<4>(xs, M, K, ss, hs, mod_ld, tokens_per_row, eps, os, stream);
  if (K <= 2048) return launch_nv<8>(xs, M, K, ss, hs, mod_ld, tokens_per_row, eps, os, stream);
  if (K <= 3072) return launch_nv<12>(xs, M, K, ss, hs, mod_ld, tokens_per_row, eps, os, stream);
  if (K <= kAdaMaxK) return launch_nv<16>(xs, M, K, ss, hs, mod_ld, tokens_per_row, eps, os, stream);
  return cudaErrorInvalidValue;
}

}  // namespace tern
