// ternary_fp8.cu -- the ternary linear with FP8 (E4M3) activations:
//   xq[m, :] = E4M3(x[m, :] / a_m),  a_m = max_k |x[m, k]| / 448,
//   y[m, n]  = a_m * s_n * sum_k xq[m, k] * T[n, k] + b_n.
//
// Page "1.58-bit FLUX" (arXiv 2412.18653), Section 4: the method leaves the
// activations unquantised and names their quantisation as the step that would
// turn the 2-bit weights into a latency gain; the pages fix no format.  Here
// the activations are E4M3 with one fp32 scale per token row, while the
// ternary weights stay exact (+-1 and 0 are E4M3 values), so the tensor cores
// run kind::f8f6f4 at twice the bf16 rate.
//
// Two kernels:
//   * quantize_act_e4m3_kernel: one warp per token row; the row's absolute
//     maximum, a_m = max / 448 and x / a_m in fp32 with IEEE division, each
//     rounded to E4M3 to nearest even with saturation (cvt.rn.satfinite).
//     Inside every 16-element group of k the two halves are interleaved:
//     byte 2i holds k = i and byte 2i + 1 holds k = 8 + i (i < 8).  That is
//     the k order in which the weight expansion below is cheapest; the MMA
//     sums over k, so the same order on both operands changes nothing.
//   * ternary_fp8_pair_kernel: the CTA-pair tile kernel of the bf16 path
//     (256 channels x 256 tokens per pair, tcgen05 cta_group::2, weights
//     decoded into TMEM as the A operand) with 128-k stages of one 2-D TMA box
//     of E4M3 x (128 tokens x 128 bytes per CTA) and 4 KiB of codes, four
//     K = 32 MMAs per stage.  A code shifted so its two bits land on bits 7
//     and 6 of a byte is the E4M3 value 2t (0x40 = 2, 0xC0 = -2, 0 = 0; the
//     unused pattern 10 reads as -0): one shift and one AND yield four bytes,
//     the codes of k = 2q, 8 + 2q, 2q + 1 and 9 + 2q of a 16-k word for
//     q = 0..3 -- exactly four consecutive bytes of the interleaved x.  The
//     epilogue scales the fp32 accumulator by a_m * s_n / 2.
// Every wait is bounded and reports a timeout in the status word; no TMA
// multicast is used (the pair's commits arrive in both CTAs).
#include "internal.h"
#include "kernel_common.cuh"
#include "ptx.cuh"

namespace tern {

namespace {

constexpr float kE4M3Max = 448.0f;

__device__ __forceinline__ uint16_t e4m3x2(float hi, float lo) {
  uint16_t d;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
  return d;
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float (&f)[8]) {
  f[0] = __uint_as_float(v.x << 16);
  f[1] = __uint_as_float(v.x & 0xFFFF0000u);
  f[2] = __uint_as_float(v.y << 16);
  f[3] = __uint_as_float(v.y & 0xFFFF0000u);
  f[4] = __uint_as_float(v.z << 16);
  f[5] = __uint_as_float(v.z & 0xFFFF0000u);
  f[6] = __uint_as_float(v.w << 16);
  f[7] = __uint_as_float(v.w & 0xFFFF0000u);
}

}  // namespace

// One warp per token row, eight rows per CTA.  K % 64 == 0; x, xq 16-byte
// aligned rows.
__global__ void __launch_bounds__(256) quantize_act_e4m3_kernel(const uint16_t* __restrict__ x, int M, int K,
                                                                 uint8_t* __restrict__ xq, float* __restrict__ a) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= M) return;
  const uint16_t* xr = x + size_t(row) * K;
  const int groups = K >> 4;  // 16-element groups of the row
  float mx = 0.f;
  for (int g = lane; g < groups; g += 32) {
    const uint4 v0 = *reinterpret_cast<const uint4*>(xr + 16 * g);
    const uint4 v1 = *reinterpret_cast<const uint4*>(xr + 16 * g + 8);
    float f0[8], f1[8];
    bf16x8_to_f32(v0, f0);
    bf16x8_to_f32(v1, f1);
#pragma unroll
    for (int i = 0; i < 8; ++i) mx = fmaxf(mx, fmaxf(fabsf(f0[i]), fabsf(f1[i])));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  const float am = mx > 0.f ? __fdiv_rn(mx, kE4M3Max) : 1.0f;
  if (lane == 0) a[row] = am;
  uint8_t* qr = xq + size_t(row) * K;
  for (int g = lane; g < groups; g += 32) {  // the row again, mostly from L1/L2
    const uint4 v0 = *reinterpret_cast<const uint4*>(xr + 16 * g);
    const uint4 v1 = *reinterpret_cast<const uint4*>(xr + 16 * g + 8);
    float f0[8], f1[8];
    bf16x8_to_f32(v0, f0);
    bf16x8_to_f32(v1, f1);
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      // bytes 4j .. 4j + 3 = k 2j, 8 + 2j, 2j + 1, 9 + 2j
      const uint16_t lo = e4m3x2(__fdiv_rn(f1[2 * j], am), __fdiv_rn(f0[2 * j], am));
      const uint16_t hi = e4m3x2(__fdiv_rn(f1[2 * j + 1], am), __fdiv_rn(f0[2 * j + 1], am));
      w[j] = uint32_t(lo) | (uint32_t(hi) << 16);
    }
    *reinterpret_cast<uint4*>(qr + 16 * g) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

namespace {

struct F8Cfg {
  static constexpr int kTokPair = 256;            // UMMA N: tokens per pair tile
  static constexpr int kTokCta = 128;             // x rows each CTA loads
  static constexpr int kBK = 128;                 // k per stage
  static constexpr int kXBytes = kTokCta * 128;   // 128 rows x 128 E4M3, 128-byte swizzle
  static constexpr int kCSub = 128 * 16;          // codes of 128 channels x 64 k
  static constexpr int kCBytes = 2 * kCSub;
  static constexpr int kStageBytes = kXBytes + kCBytes;  // 20 KiB
  static constexpr int kStages = 10;
  static constexpr int kASlots = 8;               // decoded-weight slots in TMEM
  static constexpr int kACols = kBK / 4;          // 32-bit TMEM columns per slot (four E4M3)
  static constexpr int kDCols = kTokPair;         // one fp32 accumulator
  static constexpr int kACol0 = kDCols;
  static constexpr int kTmemCols = 512;
  static constexpr int kDecWarps = 4;
  static constexpr int kEpiWarps = 16;
  static constexpr int kEpiCols = kTokPair / (kEpiWarps / 4);  // 64 tokens per epilogue warp
  static constexpr int kEpiWarp0 = 2 + kDecWarps;
  static constexpr int kThreads = (2 + kDecWarps + kEpiWarps) * 32;
  static constexpr int kSmemBytes = kStages * kStageBytes + 1024;
  // kind::f8f6f4: D fp32 (bits 4-5 = 1), A and B E4M3 (0), K-major, N = 256,
  // M = 256 (the pair).
  static constexpr uint32_t kIdesc = (1u << 4) | (uint32_t(kTokPair >> 3) << 17) | (uint32_t(256 >> 4) << 24);
  static_assert(kStageBytes % 1024 == 0, "stages stay 1024-byte aligned for the swizzle");
  static_assert(kACol0 + kASlots * kACols <= kTmemCols, "TMEM columns");
  static_assert(kSmemBytes <= 220 * 1024, "shared memory");
};

// Four (or, for a 64-k tail, two) K = 32 MMAs of one stage and two commits,
// issued by the lane elect.sync picks in the converged MMA warp.  A: the
// stage's TMEM slot, step j at a + 8 j; B: the stage's x box, step j adds 32
// bytes (2 in the descriptor's address field).
template <int NMMA>
__device__ __forceinline__ void mma_stage_f8(uint32_t d, uint32_t a, uint64_t desc, uint32_t idesc, uint32_t acc,
                                             uint32_t bar0, uint32_t bar1) {
  static_assert(NMMA == 2 || NMMA == 4, "a stage is one or two 64-k halves");
  const uint16_t both = 0x3;
  if constexpr (NMMA == 4)
    asm volatile(
        "{\n\t.reg .pred p, q, t;\n\t.reg .b64 e1, e2, e3;\n\t.reg .b32 a1, a2, a3;\n\t"
        "elect.sync _|p, 0xffffffff;\n\t"
        "setp.ne.b32 q, %4, 0;\n\tsetp.eq.b32 t, 0, 0;\n\t"
        "add.s64 e1, %2, 2;\n\tadd.s64 e2, %2, 4;\n\tadd.s64 e3, %2, 6;\n\t"
        "add.u32 a1, %1, 8;\n\tadd.u32 a2, %1, 16;\n\tadd.u32 a3, %1, 24;\n\t"
        "@p tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], [%1], %2, %3, q;\n\t"
        "@p tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], [a1], e1, %3, t;\n\t"
        "@p tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], [a2], e2, %3, t;\n\t"
        "@p tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], [a3], e3, %3, t;\n\t"
        "@p tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%5], %7;\n\t"
        "@p tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%6], %7;\n\t}"
        ::"r"(d), "r"(a), "l"(desc), "r"(idesc), "r"(acc), "r"(bar0), "r"(bar1), "h"(both)
        : "memory");
  else
    asm volatile(
        "{\n\t.reg .pred p, q, t;\n\t.reg .b64 e1;\n\t.reg .b32 a1;\n\t"
        "elect.sync _|p, 0xffffffff;\n\t"
        "setp.ne.b32 q, %4, 0;\n\tsetp.eq.b32 t, 0, 0;\n\t"
        "add.s64 e1, %2, 2;\n\tadd.u32 a1, %1, 8;\n\t"
        "@p tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], [%1], %2, %3, q;\n\t"
        "@p tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], [a1], e1, %3, t;\n\t"
        "@p tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%5], %7;\n\t"
        "@p tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%6], %7;\n\t}"
        ::"r"(d), "r"(a), "l"(desc), "r"(idesc), "r"(acc), "r"(bar0), "r"(bar1), "h"(both)
        : "memory");
}

// The E4M3 bytes of 2t for the 16 codes of one code word, as four 32-bit
// TMEM columns: column q holds k = 2q, 8 + 2q, 2q + 1, 9 + 2q of the word's
// 16 k (the code of k sits at bits 16 (k % 2) + 2 ((k % 16) / 2)); shifting
// the word left by 6 - 2q puts the codes of k = 2q, 2q + 1, 8 + 2q, 9 + 2q on
// bits 7-6 of bytes 0, 2, 1, 3.
__device__ __forceinline__ void decode_word_e4m3(uint32_t w, uint32_t* out) {
  out[0] = (w << 6) & 0xC0C0C0C0u;
  out[1] = (w << 4) & 0xC0C0C0C0u;
  out[2] = (w << 2) & 0xC0C0C0C0u;
  out[3] = w & 0xC0C0C0C0u;
}

__device__ __forceinline__ uint32_t pack_bf16x2_rn(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

// One lane waits (bounded) and the warp barrier orders the others after it.
__device__ __forceinline__ bool warp_wait_f8(uint32_t bar, uint32_t parity, uint64_t lim, unsigned int* st,
                                             int lane) {
  bool ok = true;
  if (lane == 0) ok = mbar_wait(bar, parity, lim, st);
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp();
  return ok;
}

}  // namespace

// Clusters of two CTAs (one per SM of a TPC).  Work unit u = one pair tile:
// m_tile = local / n_tiles, n_tile = local % n_tiles of problem p (n_tiles =
// N / 256).  The problem's tmap_x is the 2-D E4M3 map {K bytes, M rows} with
// box {128, 128}; `ws` carries the per-token scales a (fp32 [M]).
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(F8Cfg::kThreads, 1)
    ternary_fp8_pair_kernel(const __grid_constant__ Batch batch) {
  using C = F8Cfg;
  constexpr int S = C::kStages;
  constexpr int A = C::kASlots;

  __shared__ __align__(8) uint64_t full_bar[S];   // TMA of stage s landed (this CTA)
  __shared__ __align__(8) uint64_t empty_bar[S];  // MMAs reading stage s done (both CTAs)
  __shared__ __align__(8) uint64_t afull_bar[A];  // leader: slot a decoded in both CTAs
  __shared__ __align__(8) uint64_t aempty_bar[A]; // MMAs reading slot a done (both CTAs)
  __shared__ __align__(8) uint64_t accfull_bar;   // a tile's last MMA is done (both CTAs)
  __shared__ __align__(8) uint64_t accempty_bar;  // leader: both CTAs' epilogues read the accumulator
  __shared__ __align__(8) uint64_t drain_bar;     // leader: every MMA issued is done
  __shared__ uint32_t tmem_base_sh;
  extern __shared__ uint8_t dyn_smem[];

  const uint64_t lim = batch.wait_limit_ns;
  unsigned int* const st = batch.status;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t smem_base = (smem_u32(dyn_smem) + 1023u) & ~1023u;
  const uint8_t* const smem_gen = dyn_smem + (smem_base - smem_u32(dyn_smem));
  const int u0 = int(cluster_id_x()), ustep = int(nclusters_x()), units = batch.total_units;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    for (int a = 0; a < A; ++a) {
      mbar_init(smem_u32(&afull_bar[a]), 2 * C::kDecWarps);
      mbar_init(smem_u32(&aempty_bar[a]), 1);
    }
    mbar_init(smem_u32(&accfull_bar), 1);
    mbar_init(smem_u32(&accempty_bar), 2 * C::kEpiWarps);
    mbar_init(smem_u32(&drain_bar), 1);
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc_2sm(smem_u32(&tmem_base_sh), C::kTmemCols);
    tmem_relinquish_2sm();
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers exist and TMEM is allocated
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  auto unit_problem = [&](int u, int* m_tile, int* n_tile) -> const Problem& {
    int pi = 0;
    while (pi + 1 < batch.count && u >= batch.p[pi + 1].unit_begin) ++pi;
    const Problem& P = batch.p[pi];
    const int local = u - P.unit_begin;
    *m_tile = local / P.n_tiles;
    *n_tile = local - *m_tile * P.n_tiles;
    return P;
  };

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer (one lane)
    if (lane == 0) {
      for (int pi = 0; pi < batch.count; ++pi) prefetch_tensormap(&batch.p[pi].tmap_x);
      int it = 0;
      bool ok = true;
      for (int u = u0; u < units && ok; u += ustep) {
        int mt, nt;
        const Problem& P = unit_problem(u, &mt, &nt);
        const int kc_total = P.K >> 6;
        const uint8_t* codes = P.packed + size_t(2 * nt + int(rank)) * kc_total * C::kCSub;
        const int row = mt * C::kTokPair + int(rank) * C::kTokCta;
        for (int kc = 0; kc < kc_total; kc += 2, ++it) {
          const int s = it % S;
          ok = mbar_wait(smem_u32(&empty_bar[s]), ((it / S) & 1) ^ 1, lim, st);
          if (!ok) break;
          const int nsub = min(2, kc_total - kc);
          const uint32_t stage = smem_base + s * C::kStageBytes;
          const uint32_t fb = smem_u32(&full_bar[s]);
          // 128 k of E4M3 x (zero past K and past M) and the stage's codes.
          mbar_arrive_expect_tx(fb, C::kXBytes + nsub * C::kCSub);
          tma_load_2d(stage, &P.tmap_x, kc * 64, row, fb);
          tma_load_bulk(stage + C::kXBytes, codes + size_t(kc) * C::kCSub, nsub * C::kCSub, fb);
        }
      }
      // No copy may still be landing in shared memory when the CTA exits.
      for (int i = it > S ? it - S : 0; i < it; ++i) mbar_wait(smem_u32(&full_bar[i % S]), (i / S) & 1, lim, st);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------ MMA issuer (leader)
    const uint32_t tmem_u = __shfl_sync(0xffffffffu, tmem, 0);
    if (rank == 0) {
      int it = 0, lt = 0;
      bool ok = true;
      for (int u = u0; u < units && ok; u += ustep, ++lt) {
        int mt, nt;
        const int kc_total = unit_problem(u, &mt, &nt).K >> 6;
        ok = warp_wait_f8(smem_u32(&accempty_bar), (lt & 1) ^ 1, lim, st, lane);
        if (!ok) break;
        tc_fence_after();
        for (int kc = 0; kc < kc_total; kc += 2, ++it) {
          const int s = it % S, a = it % A;
          ok = warp_wait_f8(smem_u32(&afull_bar[a]), (it / A) & 1, lim, st, lane);
          if (!ok) break;
          tc_fence_after();
          const uint32_t a_tmem = tmem_u + C::kACol0 + a * C::kACols;
          const uint64_t desc = sw128_kmajor_desc(smem_base + s * C::kStageBytes);
          const uint32_t bar0 = smem_u32(&empty_bar[s]), bar1 = smem_u32(&aempty_bar[a]);
          if (kc + 1 < kc_total)
            mma_stage_f8<4>(tmem_u, a_tmem, desc, C::kIdesc, kc != 0, bar0, bar1);
          else
            mma_stage_f8<2>(tmem_u, a_tmem, desc, C::kIdesc, kc != 0, bar0, bar1);
        }
        if (ok) mma_commit_2sm_multicast_elected(smem_u32(&accfull_bar), 0x3);
        __syncwarp();
      }
      mma_commit_2sm_elected(smem_u32(&drain_bar));
      __syncwarp();
      warp_wait_f8(smem_u32(&drain_bar), 0, lim, st, lane);
    }
  } else if (warp < C::kEpiWarp0) {
    // ------------------------------------------------------ decoders
    // One thread per channel row: the stage's 32 code bytes become the 32
    // TMEM columns (128 E4M3 bytes) of the row's slot.
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = uint32_t(quarter * 32) << 16;
    const uint32_t afull_leader0 = mapa_shared(smem_u32(&afull_bar[0]), 0);
    int it = 0;
    bool ok = true;
    for (int u = u0; u < units && ok; u += ustep) {
      int mt, nt;
      const int kc_total = unit_problem(u, &mt, &nt).K >> 6;
      for (int kc = 0; kc < kc_total; kc += 2, ++it) {
        const int s = it % S, a = it % A;
        bool got = true;
        if (lane == 0) {
          got = mbar_wait(smem_u32(&full_bar[s]), (it / S) & 1, lim, st);
          got = got && mbar_wait(smem_u32(&aempty_bar[a]), ((it / A) & 1) ^ 1, lim, st);
        }
        ok = __shfl_sync(0xffffffffu, got, 0);
        __syncwarp();
        if (!ok) break;
        tc_fence_after();
        const uint8_t* cp = smem_gen + s * C::kStageBytes + C::kXBytes + r * 16;
        uint32_t t[32];
        const uint4 v0 = *reinterpret_cast<const uint4*>(cp);
        decode_word_e4m3(v0.x, t + 0);
        decode_word_e4m3(v0.y, t + 4);
        decode_word_e4m3(v0.z, t + 8);
        decode_word_e4m3(v0.w, t + 12);
        if (kc + 1 < kc_total) {
          const uint4 v1 = *reinterpret_cast<const uint4*>(cp + C::kCSub);
          decode_word_e4m3(v1.x, t + 16);
          decode_word_e4m3(v1.y, t + 20);
          decode_word_e4m3(v1.z, t + 24);
          decode_word_e4m3(v1.w, t + 28);
        } else {
#pragma unroll
          for (int i = 16; i < 32; ++i) t[i] = 0u;  // never read: the tail stage issues two MMAs
        }
        tmem_st32(tmem + lane_off + C::kACol0 + a * C::kACols, t);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(afull_leader0 + a * 8);
      }
    }
  } else {
    // ------------------------------------------------------ epilogue
    constexpr int kCols = C::kEpiCols;
    const int ew = warp - C::kEpiWarp0;
    const int quarter = warp & 3;
    const int part = ew >> 2;  // token columns [kCols * part, kCols * part + kCols)
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = uint32_t(quarter * 32) << 16;
    const uint32_t accempty_leader = mapa_shared(smem_u32(&accempty_bar), 0);
    int lt = 0;
    for (int u = u0; u < units; u += ustep, ++lt) {
      int mt, nt;
      const Problem& P = unit_problem(u, &mt, &nt);
      const int n = nt * 256 + int(rank) * 128 + r;
      const float sc = 0.5f * P.scales[n];  // A held 2t
      const float bi = P.bias ? bf16_bits_to_float(reinterpret_cast<const uint16_t*>(P.bias)[n]) : 0.f;
      const int row0 = mt * C::kTokPair + part * kCols;
      const int rows = min(kCols, P.M - row0);
      // This warp's 64 token scales, two per lane (zero past M).
      const float* ascale = P.ws;
      const float alo = lane < rows ? ascale[row0 + lane] : 0.f;
      const float ahi = lane + 32 < rows ? ascale[row0 + 32 + lane] : 0.f;
      if (!warp_wait_f8(smem_u32(&accfull_bar), lt & 1, lim, st, lane)) break;
      tc_fence_after();
      // y = acc * (a_m s_n / 2) + b_n, packed to bf16x2 while the
      // accumulator is read; it is released before the stores.
      uint32_t out[kCols / 2];
#pragma unroll
      for (int c0 = 0; c0 < kCols; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_off + part * kCols + c0, v);
        tmem_wait_ld();
        const float ah = c0 == 0 ? alo : ahi;
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const float a0 = __shfl_sync(0xffffffffu, ah, j);
          const float a1 = __shfl_sync(0xffffffffu, ah, j + 1);
          out[(c0 + j) / 2] = pack_bf16x2_rn(fmaf(__uint_as_float(v[j]), sc * a0, bi),
                                             fmaf(__uint_as_float(v[j + 1]), sc * a1, bi));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(accempty_leader);  // the next tile's MMAs may start
      uint16_t* yp = reinterpret_cast<uint16_t*>(P.y) + size_t(row0) * P.N + n;
#pragma unroll
      for (int c = 0; c < kCols; ++c)
        if (c < rows) yp[size_t(c) * P.N] = uint16_t(out[c >> 1] >> ((c & 1) * 16));
    }
  }

  // ------------------------------------------------------ teardown
  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_2sm(tmem, C::kTmemCols);
  }
}

cudaError_t launch_quantize_act_e4m3(const __nv_bfloat16* x, int M, int K, uint8_t* xq, float* a,
                                     cudaStream_t stream) {
  if (M <= 0) return cudaSuccess;
  quantize_act_e4m3_kernel<<<(M + 7) / 8, 256, 0, stream>>>(reinterpret_cast<const uint16_t*>(x), M, K, xq, a);
  return cudaGetLastError();
}

cudaError_t launch_ternary_fp8(const Batch& batch, int pairs, cudaStream_t stream) {
  using C = F8Cfg;
  static unsigned long long configured = 0;  // one bit per device ordinal
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64) return cudaErrorInvalidDevice;
  if (!(__atomic_load_n(&configured, __ATOMIC_ACQUIRE) & (1ull << dev))) {
    e = cudaFuncSetAttribute(ternary_fp8_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    __atomic_fetch_or(&configured, 1ull << dev, __ATOMIC_RELEASE);
  }
  ternary_fp8_pair_kernel<<<2 * pairs, C::kThreads, C::kSmemBytes, stream>>>(batch);
  return cudaGetLastError();
}

}  // namespace tern
