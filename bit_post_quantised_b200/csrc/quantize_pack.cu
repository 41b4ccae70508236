// quantize_pack.cu -- absmean ternarisation and 2-bit packing, plus the
// dequantise helper and the bounded-wait self test.
//
// Page "1.58-bit FLUX" (arXiv 2412.18653), Section 1: weights restricted to
// {-1, 0, +1} "akin to BitNet b1.58", stored as 2-bit signed integers.  The
// absmean rule of BitNet b1.58, per output channel n:
//   s_n = mean_k |W[n,k]| + eps,   T[n,k] = RoundClip(W[n,k] / s_n, -1, +1).
// With round-to-nearest-even, RoundClip gives +-1 exactly when
// |W[n,k]| / s_n > 1/2, i.e. |W[n,k]| > s_n / 2; s_n / 2 is exact in fp32, so
// the kernel decides every code exactly for the fp32 s_n it stores.
//
// One warp owns one row.  Pass 1 streams the row with 16-byte loads and sums
// |w|: eight values in fp32 (a pairwise tree, error <= 3 ulp of the group),
// the groups in fp64, then s_n = fp32(sum / K + eps) is rounded once.  Pass 2
// re-reads the row (now in L1/L2), forms the 2-bit codes and writes them in
// the tile-interleaved layout: the lane that read k = 8L..8L+7 builds half
// of the 32-bit word for 16 consecutive k, its neighbour lane the other half.
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

// 2-bit two's-complement code of one bf16 value given the fp32 threshold
// s/2 (as bits, non-negative): 01 for +1, 11 for -1, 00 for 0.  Magnitudes of
// non-negative floats order like their bit patterns.
__device__ __forceinline__ uint32_t code_of(uint32_t b16, uint32_t half_s_bits) {
  const uint32_t nz = ((b16 & 0x7FFFu) << 16) > half_s_bits ? 1u : 0u;
  const uint32_t neg = b16 >> 15;
  return nz | ((nz & neg) << 1);
}

__global__ void __launch_bounds__(kRowsPerCta * 32)
    quantize_pack_kernel(const uint16_t* __restrict__ W, int N, int K, float eps,
                         uint8_t* __restrict__ packed, float* __restrict__ scales) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = blockIdx.x * kRowsPerCta + warp;
  if (n >= N) return;
  const uint4* row = reinterpret_cast<const uint4*>(W + size_t(n) * K);
  const int n8 = K >> 3;  // 16-byte groups of 8 values; K % 64 == 0 -> n8 % 8 == 0

  // ---- pass 1: mean magnitude
  double acc = 0.0;
#pragma unroll 4
  for (int i = lane; i < n8; i += 32) acc += double(abs_sum8(__ldg(row + i)));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  const float s = float(acc / double(K) + double(eps));
  if (lane == 0) scales[n] = s;
  const uint32_t half_s = __float_as_uint(0.5f * s);

  // ---- pass 2: codes
  uint8_t* slab = packed + size_t(n >> 7) * size_t(K >> 6) * 2048 + size_t(n & 127) * 16;
  for (int base = 0; base < n8; base += 32) {
    const int i = base + lane;  // this lane's 8 values are k = 8i .. 8i+7
    uint32_t word = 0;
    if (i < n8) {
      const uint4 v = __ldg(row + i);
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
      const int j0 = (i & 1) * 4;  // pair index of k = 8i inside its 16-k word
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        // k = 8i + 2e (even) and 8i + 2e + 1 (odd): pair j0 + e
        word |= code_of(w4[e] & 0xFFFFu, half_s) << (2 * (j0 + e));
        word |= code_of(w4[e] >> 16, half_s) << (16 + 2 * (j0 + e));
      }
    }
    word |= __shfl_xor_sync(0xffffffffu, word, 1);
    if (i < n8 && (i & 1) == 0) {
      const int chunk = i >> 3;          // 64-wide k chunk
      const int wsel = (i & 7) >> 1;     // word inside the 16-byte group
      *reinterpret_cast<uint32_t*>(slab + size_t(chunk) * 2048 + wsel * 4) = word;
    }
  }
}

// ---- dequantise: one thread per 16-byte group (row n, 64-wide chunk c)
__global__ void dequantize_kernel(const uint8_t* __restrict__ packed, const float* __restrict__ scales,
                                  int N, int K, __nv_bfloat16* __restrict__ out) {
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
  quantize_pack_kernel<<<grid, kRowsPerCta * 32, 0, stream>>>(reinterpret_cast<const uint16_t*>(W), N,
                                                             K, eps, packed, scales);
  return cudaGetLastError();
}

cudaError_t launch_dequantize(const uint8_t* packed, const float* scales, int N, int K,
                              __nv_bfloat16* out, cudaStream_t stream) {
  const size_t groups = size_t(N) * (K >> 6);
  const int threads = 256;
  const size_t grid = (groups + threads - 1) / threads;
  dequantize_kernel<<<unsigned(grid), threads, 0, stream>>>(packed, scales, N, K, out);
  return cudaGetLastError();
}

cudaError_t launch_wait_selftest(unsigned long long limit_ns, unsigned int* status,
                                 cudaStream_t stream) {
  wait_selftest_kernel<<<1, 32, 0, stream>>>(limit_ns, status);
  return cudaGetLastError();
}

}  // namespace tern
