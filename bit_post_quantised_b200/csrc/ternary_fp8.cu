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
//     maximum, a_m = max / 448 (IEEE fp32 division) and x / a_m rounded to
//     fp32 exactly as IEEE division would (an fp64 multiply by the fp64
//     reciprocal; the kernel states why that is exact for bf16 x), then to
//     E4M3 to nearest even with saturation (cvt.rn.satfinite).
//     Inside every 16-element group of k the two halves are interleaved:
//     byte 2i holds k = i and byte 2i + 1 holds k = 8 + i (i < 8).  That is
//     the k order in which the weight expansion below is cheapest; the MMA
//     sums over k, so the same order on both operands changes nothing.
//   * ternary_fp8_pair_kernel: the CTA-pair tile kernel of the bf16 path
//     (256 channels x 256 tokens per pair, tcgen05 cta_group::2, weights
//     decoded into TMEM as the A operand) with 256-k stages of two 2-D TMA
//     boxes of E4M3 x (128 tokens x 128 bytes each per CTA) and 8 KiB of
//     codes, eight K = 32 MMAs per stage (1024 tensor cycles between two
//     barrier handshakes, as in a bf16 stage).  A code shifted so its two bits land on bits 7
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

// One warp per token row, eight rows per CTA (four CTAs per SM for K <= 3072,
// so the 4096 rows of a FLUX image stream run in one wave).  K % 64 == 0; x,
// xq 16-byte aligned rows.  NV > 0: the row is held in registers (lane l keeps the
// 16-element groups l, l + 32, ..., NV per lane, K <= 512 NV), so x is read
// once; NV == 0: any K, the row is read twice (the second time mostly from
// L2).
template <int NV>
__global__ void __launch_bounds__(256, NV > 6 ? 2 : 4) quantize_act_e4m3_kernel(const uint16_t* __restrict__ x, int M, int K,
                                                                 uint8_t* __restrict__ xq, float* __restrict__ a) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= M) return;
  const uint16_t* xr = x + size_t(row) * K;
  uint8_t* qr = xq + size_t(row) * K;
  const int groups = K >> 4;  // 16-element groups of the row
  // x / a_m rounded to fp32 as IEEE division would, from one fp64 multiply
  // by the fp64 reciprocal r = RN64(1 / a_m).  x is a bf16 (8 significant
  // bits) and a_m an fp32 (24), so x / a_m is never exactly halfway between
  // two fp32 numbers, and when it is not, it lies at least 2^-49 (relative)
  // from such a midpoint; RN64(x r) is within 2^-52 (relative) of x / a_m,
  // so rounding it to fp32 gives RN32(x / a_m).  (Where x / a_m falls into
  // the fp32 subnormals the E4M3 code is a signed zero either way.)
  auto q32 = [](float v, double r) { return __double2float_rn(double(v) * r); };
  // bytes 4j .. 4j + 3 of a group's output = k 2j, 8 + 2j, 2j + 1, 9 + 2j
  auto emit = [&](int g, const uint4& v0, const uint4& v1, double r) {
    float f0[8], f1[8];
    bf16x8_to_f32(v0, f0);
    bf16x8_to_f32(v1, f1);
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint16_t lo = e4m3x2(q32(f1[2 * j], r), q32(f0[2 * j], r));
      const uint16_t hi = e4m3x2(q32(f1[2 * j + 1], r), q32(f0[2 * j + 1], r));
      w[j] = uint32_t(lo) | (uint32_t(hi) << 16);
    }
    *reinterpret_cast<uint4*>(qr + 16 * g) = make_uint4(w[0], w[1], w[2], w[3]);
  };
  auto absmax8 = [](const uint4& v) {
    // |bf16| as bits: clear the sign; the largest magnitude has the largest bits
    const uint32_t m = 0x7FFF7FFFu;
    const uint32_t a0 = max(max((v.x & m) & 0xFFFFu, (v.x & m) >> 16), max((v.y & m) & 0xFFFFu, (v.y & m) >> 16));
    const uint32_t a1 = max(max((v.z & m) & 0xFFFFu, (v.z & m) >> 16), max((v.w & m) & 0xFFFFu, (v.w & m) >> 16));
    return max(a0, a1);
  };
  uint32_t mb = 0;  // the bits of the largest magnitude so far (bf16 magnitudes order as integers)
  if constexpr (NV > 0) {
    uint4 v[NV][2];
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int g = lane + 32 * i;
      if (g < groups) {
        v[i][0] = *reinterpret_cast<const uint4*>(xr + 16 * g);
        v[i][1] = *reinterpret_cast<const uint4*>(xr + 16 * g + 8);
      } else {
        v[i][0] = v[i][1] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
#pragma unroll
    for (int i = 0; i < NV; ++i) mb = max(mb, max(absmax8(v[i][0]), absmax8(v[i][1])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mb = max(mb, __shfl_xor_sync(0xffffffffu, mb, o));
    const float mx = __uint_as_float(mb << 16);
    const float am = mx > 0.f ? __fdiv_rn(mx, kE4M3Max) : 1.0f;
    if (lane == 0) a[row] = am;
    const double r = 1.0 / double(am);
#pragma unroll
    for (int i = 0; i < NV; ++i)
      if (lane + 32 * i < groups) emit(lane + 32 * i, v[i][0], v[i][1], r);
  } else {
    for (int g = lane; g < groups; g += 32)
      mb = max(mb, max(absmax8(*reinterpret_cast<const uint4*>(xr + 16 * g)),
                       absmax8(*reinterpret_cast<const uint4*>(xr + 16 * g + 8))));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mb = max(mb, __shfl_xor_sync(0xffffffffu, mb, o));
    const float mx = __uint_as_float(mb << 16);
    const float am = mx > 0.f ? __fdiv_rn(mx, kE4M3Max) : 1.0f;
    if (lane == 0) a[row] = am;
    const double r = 1.0 / double(am);
    for (int g = lane; g < groups; g += 32)  // the row again, mostly from L2
      emit(g, *reinterpret_cast<const uint4*>(xr + 16 * g), *reinterpret_cast<const uint4*>(xr + 16 * g + 8), r);
  }
}

namespace {

struct F8Cfg {
  static constexpr int kTokPair = 256;            // UMMA N: tokens per pair tile
  static constexpr int kTokCta = 128;             // x rows each CTA loads
  static constexpr int kChunks = 4;               // 64-k chunks per stage: 256 k
  static constexpr int kXBox = kTokCta * 128;     // 128 rows x 128 E4M3 bytes, 128-byte swizzle
  static constexpr int kXBytes = 2 * kXBox;       // two boxes: k 0-127 and 128-255 of the stage
  static constexpr int kCSub = 128 * 16;          // codes of 128 channels x 64 k
  static constexpr int kCBytes = kChunks * kCSub;
  static constexpr int kStageBytes = kXBytes + kCBytes;  // 40 KiB
  static constexpr int kStages = 5;
  static constexpr int kASlots = 4;               // decoded-weight slots in TMEM, one stage each
  static constexpr int kACols = kChunks * 16;     // 32-bit TMEM columns per slot (four E4M3)
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

// The K = 32 MMAs of one stage (2 per 64-k chunk: NMMA = 2, 4, 6 or 8) and two
// commits, issued by the lane elect.sync picks in the converged MMA warp, as
// one block (uniform operands; per-MMA arithmetic in a single-lane branch
// measured several times slower on the bf16 kernels).  A: the stage's TMEM
// slot, MMA j at a + 8 j.  B: the stage's two x boxes; MMA j reads 32 bytes
// at 32 (j % 4) of box j / 4 (descriptor address units of 16 bytes: + 2 per
// MMA, + 1024 for the second 16 KiB box).
#define F8_MMA(AR, ER, P) "@p tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], [" AR "], " ER ", %3, " P ";\n\t"
#define F8_COMMITS                                                                                       \
  "@p tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%5], %7;\n\t" \
  "@p tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%6], %7;\n\t}"
#define F8_PROLOGUE                                                                              \
  "{\n\t.reg .pred p, q, t;\n\t.reg .b64 e1, e2, e3, e4, e5, e6, e7;\n\t"                     \
  ".reg .b32 a1, a2, a3, a4, a5, a6, a7;\n\t"                                                   \
  "elect.sync _|p, 0xffffffff;\n\tsetp.ne.b32 q, %4, 0;\n\tsetp.eq.b32 t, 0, 0;\n\t"           \
  "add.s64 e1, %2, 2;\n\tadd.s64 e2, %2, 4;\n\tadd.s64 e3, %2, 6;\n\tadd.s64 e4, %2, 1024;\n\t" \
  "add.s64 e5, %2, 1026;\n\tadd.s64 e6, %2, 1028;\n\tadd.s64 e7, %2, 1030;\n\t"                \
  "add.u32 a1, %1, 8;\n\tadd.u32 a2, %1, 16;\n\tadd.u32 a3, %1, 24;\n\tadd.u32 a4, %1, 32;\n\t" \
  "add.u32 a5, %1, 40;\n\tadd.u32 a6, %1, 48;\n\tadd.u32 a7, %1, 56;\n\t"
#define F8_M01 F8_MMA("%1", "%2", "q") F8_MMA("a1", "e1", "t")
#define F8_M23 F8_MMA("a2", "e2", "t") F8_MMA("a3", "e3", "t")
#define F8_M45 F8_MMA("a4", "e4", "t") F8_MMA("a5", "e5", "t")
#define F8_M67 F8_MMA("a6", "e6", "t") F8_MMA("a7", "e7", "t")
#define F8_ARGS                                                                                  \
  ::"r"(d), "r"(a), "l"(desc), "r"(idesc), "r"(acc), "r"(bar0), "r"(bar1), "h"(both) : "memory"

template <int NMMA>
__device__ __forceinline__ void mma_stage_f8(uint32_t d, uint32_t a, uint64_t desc, uint32_t idesc, uint32_t acc,
                                             uint32_t bar0, uint32_t bar1) {
  static_assert(NMMA == 2 || NMMA == 4 || NMMA == 6 || NMMA == 8, "two MMAs per 64-k chunk");
  const uint16_t both = 0x3;
  if constexpr (NMMA == 8)
    asm volatile(F8_PROLOGUE F8_M01 F8_M23 F8_M45 F8_M67 F8_COMMITS F8_ARGS);
  else if constexpr (NMMA == 6)
    asm volatile(F8_PROLOGUE F8_M01 F8_M23 F8_M45 F8_COMMITS F8_ARGS);
  else if constexpr (NMMA == 4)
    asm volatile(F8_PROLOGUE F8_M01 F8_M23 F8_COMMITS F8_ARGS);
  else
    asm volatile(F8_PROLOGUE F8_M01 F8_COMMITS F8_ARGS);
}
#undef F8_MMA
#undef F8_COMMITS
#undef F8_PROLOGUE
#undef F8_M01
#undef F8_M23
#undef F8_M45
#undef F8_M67
#undef F8_ARGS

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
  pdl_wait();
  pdl_trigger();
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
    // ------------------------------------------------------ TMA producer
    // Stage it is issued by lane it % S (each lane owns one ring slot): one
    // thread issues a copy only every ~280 SM cycles, and a stage is three
    // copies.
    if (lane == 0)
      for (int pi = 0; pi < batch.count; ++pi) prefetch_tensormap(&batch.p[pi].tmap_x);
    __syncwarp();
    if (lane < S) {
      int it = 0;
      bool ok = true;
      for (int u = u0; u < units && ok; u += ustep) {
        int mt, nt;
        const Problem& P = unit_problem(u, &mt, &nt);
        const int kc_total = P.K >> 6;
        const uint8_t* codes = P.packed + size_t(2 * nt + int(rank)) * kc_total * C::kCSub;
        const int row = mt * C::kTokPair + int(rank) * C::kTokCta;
        for (int kc = 0; kc < kc_total; kc += C::kChunks, ++it) {
          if (it % S != lane) continue;
          const int s = lane;
          ok = mbar_wait(smem_u32(&empty_bar[s]), ((it / S) & 1) ^ 1, lim, st);
          if (!ok) break;
          const int nch = min(C::kChunks, kc_total - kc);
          const uint32_t stage = smem_base + s * C::kStageBytes;
          const uint32_t fb = smem_u32(&full_bar[s]);
          // 256 k of E4M3 x as two 128-byte-wide boxes (zero past K and past
          // M) and the stage's codes, one block.
          mbar_arrive_expect_tx(fb, C::kXBytes + nch * C::kCSub);
          tma_load_2d(stage, &P.tmap_x, kc * 64, row, fb);
          tma_load_2d(stage + C::kXBox, &P.tmap_x, kc * 64 + 128, row, fb);
          tma_load_bulk(stage + C::kXBytes, codes + size_t(kc) * C::kCSub, nch * C::kCSub, fb);
        }
      }
      // No copy this lane issued may still be landing when the CTA exits.
      if (it > lane) {
        const int last = lane + ((it - 1 - lane) / S) * S;  // this lane's last stage
        mbar_wait(smem_u32(&full_bar[lane]), (last / S) & 1, lim, st);
      }
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
        for (int kc = 0; kc < kc_total; kc += C::kChunks, ++it) {
          const int s = it % S, a = it % A;
          ok = warp_wait_f8(smem_u32(&afull_bar[a]), (it / A) & 1, lim, st, lane);
          if (!ok) break;
          tc_fence_after();
          const uint32_t a_tmem = tmem_u + C::kACol0 + a * C::kACols;
          const uint64_t desc = sw128_kmajor_desc(smem_base + s * C::kStageBytes);
          const uint32_t bar0 = smem_u32(&empty_bar[s]), bar1 = smem_u32(&aempty_bar[a]);
          const int nch = min(C::kChunks, kc_total - kc);
          if (nch == 4)
            mma_stage_f8<8>(tmem_u, a_tmem, desc, C::kIdesc, kc != 0, bar0, bar1);
          else if (nch == 3)
            mma_stage_f8<6>(tmem_u, a_tmem, desc, C::kIdesc, kc != 0, bar0, bar1);
          else if (nch == 2)
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
      for (int kc = 0; kc < kc_total; kc += C::kChunks, ++it) {
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
        const uint32_t dst = tmem + lane_off + C::kACol0 + a * C::kACols;
        // Two 128-k halves of the stage, 32 columns each (a half past K is
        // not written: its MMAs are not issued).
#pragma unroll
        for (int h = 0; h < 2; ++h)
          if (kc + 2 * h < kc_total) {
            uint32_t t[32];
            const uint4 v0 = *reinterpret_cast<const uint4*>(cp + (2 * h) * C::kCSub);
            decode_word_e4m3(v0.x, t + 0);
            decode_word_e4m3(v0.y, t + 4);
            decode_word_e4m3(v0.z, t + 8);
            decode_word_e4m3(v0.w, t + 12);
            if (kc + 2 * h + 1 < kc_total) {
              const uint4 v1 = *reinterpret_cast<const uint4*>(cp + (2 * h + 1) * C::kCSub);
              decode_word_e4m3(v1.x, t + 16);
              decode_word_e4m3(v1.y, t + 20);
              decode_word_e4m3(v1.z, t + 24);
              decode_word_e4m3(v1.w, t + 28);
            } else {
#pragma unroll
              for (int i = 16; i < 32; ++i) t[i] = 0u;  // past K: never read
            }
            tmem_st32(dst + 32 * h, t);
          }
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
      // The accumulator goes to registers and is released at once (the next
      // tile's MMAs wait for it); y = acc * (a_m s_n / 2) + b_n comes after.
      float f[kCols];
#pragma unroll
      for (int c0 = 0; c0 < kCols; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_off + part * kCols + c0, v);
        tmem_wait_ld();  // the registers hold the values only after the wait
#pragma unroll
        for (int j = 0; j < 32; ++j) f[c0 + j] = __uint_as_float(v[j]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(accempty_leader);  // the next tile's MMAs may start
      uint16_t* yp = reinterpret_cast<uint16_t*>(P.y) + size_t(row0) * P.ldy + n;
#pragma unroll
      for (int c = 0; c < kCols; ++c) {
        const float am = __shfl_sync(0xffffffffu, c < 32 ? alo : ahi, c & 31);
        const float y = fmaf(f[c], sc * am, bi);
        if (c < rows) yp[size_t(c) * P.ldy] = __bfloat16_as_ushort(__float2bfloat16_rn(y));
      }
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
  const uint16_t* xb = reinterpret_cast<const uint16_t*>(x);
  const dim3 grid((M + 7) / 8);
  const dim3 b(256);
  if (K <= 512 * 2) return launch_pdl(quantize_act_e4m3_kernel<2>, grid, b, 0, stream, 1, xb, M, K, xq, a);
  if (K <= 512 * 4) return launch_pdl(quantize_act_e4m3_kernel<4>, grid, b, 0, stream, 1, xb, M, K, xq, a);
  if (K <= 512 * 6) return launch_pdl(quantize_act_e4m3_kernel<6>, grid, b, 0, stream, 1, xb, M, K, xq, a);
  if (K <= 512 * 8) return launch_pdl(quantize_act_e4m3_kernel<8>, grid, b, 0, stream, 1, xb, M, K, xq, a);
  return launch_pdl(quantize_act_e4m3_kernel<0>, grid, b, 0, stream, 1, xb, M, K, xq, a);
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
  return launch_pdl(ternary_fp8_pair_kernel, dim3(2 * pairs), dim3(C::kThreads), C::kSmemBytes, stream, 1, batch);
}

}  // namespace tern
