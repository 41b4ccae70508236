// quantize_pack.cu -- absmean ternarisation and 2-bit packing, plus the
// dequantise helper and the bounded-wait self test.
//
// Page "1.58-bit FLUX" (arXiv 2412.18653), Section 1: weights restricted to
// {-1, 0, +1} "akin to BitNet b1.58", stored as 2-bit signed integers.  The
// absmean rule of BitNet b1.58, per output channel n:
//   s_n = mean_k |W[n,k]| + eps,   T[n,k] = RoundClip(W[n,k] / s_n, -1, +1).
// With round-to-nearest-even, RoundClip gives +-1 exactly when
// |W[n,k]| / s_n > 1/2, i.e. |W[n,k]| > s_n / 2.  For a bf16 W that holds
// exactly when |W| exceeds s_n / 2 truncated to bf16, so the kernel decides
// every code exactly for the fp32 s_n it stores (two bf16x2 compares per
// pair of values).
//
// One warp owns one row.  It sums |w| over 16-byte loads: eight values in
// fp32 (a pairwise tree, error <= 3 ulp of the group), the groups in fp64,
// then s_n = fp32(sum / K + eps) is rounded once.  It then forms the 2-bit
// codes and writes them in the tile-interleaved layout: the lane that read
// k = 8L..8L+7 builds half of the 32-bit word for 16 consecutive k, its
// neighbour lane the other half.  Rows of up to 4096 values stay in
// registers between the two steps; longer rows are read twice (the second
// time from L2).  When N is not a multiple of 128 a second small kernel
// completes the last slab with zero-code rows (no scale), which the linear
// kernels never store.
#include "internal.h"
#include "ptx.cuh"

namespace tern {

namespace {

constexpr int kRowsPerCta = 8;

__device__ __forceinline__ float lo_bf16(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi_bf16(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ float abs_sum8(const uint4& v) {
  const float a = fabsf(lo_bf16(v.x)) + fabsf(hi_bf16(v.x));
  const float b = fabsf(lo_bf16(v.y)) + fabsf(hi_bf16(v.y));
  const float c = fabsf(lo_bf16(v.z)) + fabsf(hi_bf16(v.z));
  const float d = fabsf(lo_bf16(v.w)) + fabsf(hi_bf16(v.w));
  return (a + b) + (c + d);
}


// Codes of the two bf16 values of a 32-bit word (k in the low half, k + 1 in
// the high half) at bits 0-1 and 16-17, given the bf16 threshold thr16 =
// s/2 truncated to bf16 (the top 16 bits of s/2 halved toward zero in fp32:
// exact for normal s, and still the truncation for subnormal s, where the
// halving drops a bit).  For a bf16 magnitude m (15 bits), m > thr16 exactly
// when |w| > s/2 (|w| is a bf16).  Per half, 0x8000 + thr16 - m stays in [1, 0xFFFF], so its
// bit 15 is clear exactly when m > thr16, with no borrow into the other half.
__device__ __forceinline__ uint32_t code_pair(uint32_t w, uint32_t thr_pair) {
  const uint32_t mag = w & 0x7FFF7FFFu;
  const uint32_t nz = (~((thr_pair | 0x80008000u) - mag) >> 15) & 0x00010001u;
  const uint32_t neg = (w >> 15) & 0x00010001u;
  return nz | ((nz & neg) << 1);
}

// The codes of a lane's eight values (one 16-byte group: k = 8i .. 8i + 7)
// ORed into their places in the 16-k code word, from two bf16x2 compares per
// 32-bit word: w > t and w < -t, t = s/2 rounded down to bf16 (thr_pos; thr_neg
// is -t).  For a bf16 w, w > t exactly when w > s/2 (t <= s/2 < the next bf16
// above t), so the compares decide every code exactly, like code_pair, with
// two compares and two LOP3s per word instead of ten integer operations.  A
// compare writes 0xFFFF into each half where it holds; the code bits of the
// word's two values go to bits (2p, 2p + 1) of each half, p = the pair's index
// in the 16-k word, through the masks k1 (0x00010001 << 2p: sign-free bit) and
// k3 (0x00030003 << 2p: both bits, -1 = 0b11).  Needs t normal (the compare
// may treat subnormal operands as zero); the caller takes code_pair otherwise.
__device__ __forceinline__ uint32_t bf16x2_gt_mask(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("set.gt.u32.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t bf16x2_lt_mask(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("set.lt.u32.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
struct CodeMasks {
  uint32_t k1[4], k3[4];
  __device__ __forceinline__ explicit CodeMasks(int j0) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      k1[e] = 0x00010001u << (2 * (j0 + e));
      k3[e] = 0x00030003u << (2 * (j0 + e));
    }
  }
};
__device__ __forceinline__ uint32_t group_codes(const uint4& v, uint32_t thr_pos, uint32_t thr_neg,
                                                const CodeMasks& m) {
  const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
  uint32_t word = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    word |= bf16x2_gt_mask(w4[e], thr_pos) & m.k1[e];
    word |= bf16x2_lt_mask(w4[e], thr_neg) & m.k3[e];
  }
  return word;
}
// The same word through code_pair (any threshold).
__device__ __forceinline__ uint32_t group_codes_int(const uint4& v, uint32_t thr_pair, int j0) {
  const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
  uint32_t word = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e) word |= code_pair(w4[e], thr_pair) << (2 * (j0 + e));
  return word;
}

// The padding rows n = N .. Np - 1 of the last 128-channel slab (N % 128
// != 0): their code words are zero and they have no scale.  One thread per
// 32-bit word (word w of a row holds k = 16w .. 16w + 15).
__global__ void zero_pad_rows_kernel(uint8_t* __restrict__ packed, int N, int K) {
  pdl_wait();
  pdl_trigger();
  const int words = K >> 4;
  const int pad_rows = ((N + 127) & ~127) - N;
  const long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (i >= (long long)pad_rows * words) return;
  const int n = N + int(i / words), w = int(i % words);
  uint8_t* slab = packed + size_t(n >> 7) * size_t(K >> 6) * 2048 + size_t(n & 127) * 16;
  *reinterpret_cast<uint32_t*>(slab + size_t(w >> 2) * 2048 + (w & 3) * 4) = 0u;
}

// Same computation with the row held in registers, so W is read from HBM
// once: a lane keeps its NV 16-byte groups (k = 8i .. 8i + 7, i = lane +
// 32 t) from the mean through the codes.  All NV loads are issued before the
// first is used.  For K <= 256 NV.
template <int NV>
__global__ void __launch_bounds__(kRowsPerCta * 32)
    quantize_pack_regs_kernel(const uint16_t* __restrict__ W, int N, int K, float eps,
                              uint8_t* __restrict__ packed, float* __restrict__ scales) {
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = blockIdx.x * kRowsPerCta + warp;
  if (n >= N) return;
  const uint4* row = reinterpret_cast<const uint4*>(W + size_t(n) * K);
  const int n8 = K >> 3;
  uint4 v[NV];
#pragma unroll
  for (int t = 0; t < NV; ++t) {
    const int i = lane + 32 * t;
    v[t] = i < n8 ? __ldg(row + i) : make_uint4(0u, 0u, 0u, 0u);
  }
  // ---- mean magnitude: groups of eight in fp32, groups summed in fp64
  double acc = 0.0;
#pragma unroll
  for (int t = 0; t < NV; ++t) acc += double(abs_sum8(v[t]));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  const float s = float(acc / double(K) + double(eps));
  if (lane == 0) scales[n] = s;
  const uint32_t thr16 = __float_as_uint(__fmul_rz(0.5f, s)) >> 16;  // trunc(s / 2), exact for any s
  const uint32_t thr_pair = thr16 | (thr16 << 16);
  const bool normal_thr = thr16 >= 0x0080u;  // t is a normal bf16 (uniform over the warp)

  // ---- codes
  uint8_t* slab = packed + size_t(n >> 7) * size_t(K >> 6) * 2048 + size_t(n & 127) * 16;
  const int j0 = (lane & 1) * 4;  // pair index of k = 8i inside its 16-k word (i has lane's parity)
  const CodeMasks cm(j0);
#pragma unroll
  for (int t = 0; t < NV; ++t) {
    const int i = lane + 32 * t;
    uint32_t word = normal_thr ? group_codes(v[t], thr_pair, thr_pair | 0x80008000u, cm)
                               : group_codes_int(v[t], thr_pair, j0);
    word |= __shfl_xor_sync(0xffffffffu, word, 1);
    if (i < n8 && (i & 1) == 0)
      *reinterpret_cast<uint32_t*>(slab + size_t(i >> 3) * 2048 + ((i & 7) >> 1) * 4) = word;
  }
}

// Rows longer than 4096 values: the same steps over segments of 4096 values
// (16 groups of eight per lane, all loads of a segment in flight), the mean
// over every segment first, then the codes segment by segment, re-reading
// the row (from L2: a warp's row is at most 2 MiB / 64 = 32 KiB here).
__global__ void __launch_bounds__(kRowsPerCta * 32)
    quantize_pack_long_kernel(const uint16_t* __restrict__ W, int N, int K, float eps,
                              uint8_t* __restrict__ packed, float* __restrict__ scales) {
  pdl_wait();
  pdl_trigger();
  constexpr int NV = 16;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = blockIdx.x * kRowsPerCta + warp;
  if (n >= N) return;
  const uint4* row = reinterpret_cast<const uint4*>(W + size_t(n) * K);
  const int n8 = K >> 3;
  double acc = 0.0;
  for (int base = 0; base < n8; base += 32 * NV) {
    uint4 v[NV];
#pragma unroll
    for (int t = 0; t < NV; ++t) {
      const int i = base + lane + 32 * t;
      v[t] = i < n8 ? __ldg(row + i) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int t = 0; t < NV; ++t) acc += double(abs_sum8(v[t]));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  const float s = float(acc / double(K) + double(eps));
  if (lane == 0) scales[n] = s;
  const uint32_t thr16 = __float_as_uint(__fmul_rz(0.5f, s)) >> 16;  // trunc(s / 2), exact for any s
  const uint32_t thr_pair = thr16 | (thr16 << 16);
  const bool normal_thr = thr16 >= 0x0080u;
  uint8_t* slab = packed + size_t(n >> 7) * size_t(K >> 6) * 2048 + size_t(n & 127) * 16;
  const int j0 = (lane & 1) * 4;
  const CodeMasks cm(j0);
  for (int base = 0; base < n8; base += 32 * NV) {
    uint4 v[NV];
#pragma unroll
    for (int t = 0; t < NV; ++t) {
      const int i = base + lane + 32 * t;
      v[t] = i < n8 ? __ldg(row + i) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int t = 0; t < NV; ++t) {
      const int i = base + lane + 32 * t;
      uint32_t word = normal_thr ? group_codes(v[t], thr_pair, thr_pair | 0x80008000u, cm)
                                 : group_codes_int(v[t], thr_pair, j0);
      word |= __shfl_xor_sync(0xffffffffu, word, 1);
      if (i < n8 && (i & 1) == 0)
        *reinterpret_cast<uint32_t*>(slab + size_t(i >> 3) * 2048 + ((i & 7) >> 1) * 4) = word;
    }
  }
}

// ---- dequantise: one thread per 16-byte group (row n, 64-wide chunk c)
__global__ void dequantize_kernel(const uint8_t* __restrict__ packed, const float* __restrict__ scales,
                                  int N, int K, __nv_bfloat16* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  const size_t groups = size_t(N) * (K >> 6);
  const size_t g = size_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (g >= groups) return;
  const int kc_total = K >> 6;
  // groups are enumerated in memory order: tile-slab, chunk, row
  const size_t slab = g / (size_t(kc_total) * 128);
  const size_t rem = g - slab * size_t(kc_total) * 128;
  const int c = int(rem / 128);
  const int r = int(rem % 128);
  const int n = int(slab) * 128 + r;
  const uint4 v = *reinterpret_cast<const uint4*>(packed + g * 16);
  const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
  const float s = scales[n];
  __nv_bfloat16* dst = out + size_t(n) * K + size_t(c) * 64;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t o[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int t_even = int((w4[q] >> (2 * j)) & 3u), t_odd = int((w4[q] >> (16 + 2 * j)) & 3u);
      const float fe = float(t_even == 3 ? -1 : t_even), fo = float(t_odd == 3 ? -1 : t_odd);
      const __nv_bfloat162 p = __floats2bfloat162_rn(fe * s, fo * s);
      o[j] = *reinterpret_cast<const uint32_t*>(&p);
    }
    uint4* d = reinterpret_cast<uint4*>(dst + q * 16);
    d[0] = make_uint4(o[0], o[1], o[2], o[3]);
    d[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

// ---- a wait that nothing will ever satisfy; must end by its limit
__global__ void wait_selftest_kernel(unsigned long long limit_ns, unsigned int* status) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, limit_ns, status);
}

}  // namespace

cudaError_t launch_quantize_pack(const __nv_bfloat16* W, int N, int K, float eps, uint8_t* packed,
                                 float* scales, cudaStream_t stream) {
  const int grid = (N + kRowsPerCta - 1) / kRowsPerCta;
  const uint16_t* w = reinterpret_cast<const uint16_t*>(W);
  // Rows of up to 4096 values stay in registers (one read of W); longer rows
  // are read twice, the second time mostly from L2.
  const dim3 g(grid), b(kRowsPerCta * 32);
  cudaError_t e;
  if (K <= 32 * 8 * 4)
    e = launch_pdl(quantize_pack_regs_kernel<4>, g, b, 0, stream, 1, w, N, K, eps, packed, scales);
  else if (K <= 32 * 8 * 8)
    e = launch_pdl(quantize_pack_regs_kernel<8>, g, b, 0, stream, 1, w, N, K, eps, packed, scales);
  else if (K <= 32 * 8 * 12)
    e = launch_pdl(quantize_pack_regs_kernel<12>, g, b, 0, stream, 1, w, N, K, eps, packed, scales);
  else if (K <= 32 * 8 * 16)
    e = launch_pdl(quantize_pack_regs_kernel<16>, g, b, 0, stream, 1, w, N, K, eps, packed, scales);
  else
    e = launch_pdl(quantize_pack_long_kernel, g, b, 0, stream, 1, w, N, K, eps, packed, scales);
  if (e != cudaSuccess || N % 128 == 0) return e;
  const long long n_words = (long long)(((N + 127) & ~127) - N) * (K >> 4);
  return launch_pdl(zero_pad_rows_kernel, dim3(unsigned((n_words + 255) / 256)), dim3(256), 0, stream, 1, packed, N,
                    K);
}

cudaError_t launch_dequantize(const uint8_t* packed, const float* scales, int N, int K,
                              __nv_bfloat16* out, cudaStream_t stream) {
  const size_t groups = size_t(N) * (K >> 6);
  const int threads = 256;
  const size_t grid = (groups + threads - 1) / threads;
  return launch_pdl(dequantize_kernel, dim3(unsigned(grid)), dim3(threads), 0, stream, 1, packed, scales, N, K, out);
}

cudaError_t launch_wait_selftest(unsigned long long limit_ns, unsigned int* status,
                                 cudaStream_t stream) {
  wait_selftest_kernel<<<1, 32, 0, stream>>>(limit_ns, status);
  return cudaGetLastError();
}

}  // namespace tern
