// ternary_mma2.cu -- the large-M ternary linear y = (x . T^T) * s + b on
// pairs of SMs (tcgen05 cta_group::2).
//
// Page "1.58-bit FLUX" (arXiv 2412.18653): Section 1 (weights in {-1,0,+1},
// stored as 2-bit signed integers), Section 4 (activations stay 16-bit).
//
// A cluster of two CTAs (one per SM) owns a 256-channel x 256-token tile of
// y, held transposed in TMEM: D[channel, token].  One UMMA instruction of the
// pair is M = 256 channels (the 128 decoded weight rows in each CTA's TMEM are
// its half of A), N = 256 tokens (128 rows of x in each CTA's shared memory
// are its half of B), K = 16; each CTA's TMEM receives its own 128 channel
// rows of the fp32 accumulator.  One instruction is 128 tensor cycles per
// SM, and every x byte brought from L2 feeds 256 channels.
//
// Per CTA, per 128-wide k stage (36 KiB of shared memory, 6 stages; the last
// stage of a row holds 64 k when K % 128 == 64):
//   * warp 0 (producer): tiled TMA copies of its 128 x-rows (one 64 k x 128
//     row box per 64 k, 128-byte swizzle) and one bulk copy of its codes
//     (128 channels x 128 k, contiguous in the tile-interleaved layout), all
//     completing on full[s].
//   * warps 2-5 (decoders): one thread per channel row waits for the stage
//     and for TMEM slot a (4 slots of 64 columns) to be free, expands its
//     code bytes into bf16x2 TMEM columns (tcgen05.st), then one lane per warp
//     arrives on the leader CTA's afull[a].  The arrival also vouches for
//     that CTA's x rows of the stage, which the decoder waited for.
//   * warp 1 of the leader CTA (rank 0): waits afull[a] (eight arrivals, four
//     from each CTA), issues the eight MMAs of the stage and commits, with
//     one arrival in both CTAs, to empty[s] (shared-memory stage free) and
//     aempty[a] (TMEM slot free).  Eight MMAs (1024 tensor cycles) between
//     two waits of the issuing thread keep the tensor pipe fed; a wait every
//     four MMAs measurably starves it.
//   * warps 6-13 (epilogue): after the tile's last MMA, tcgen05.ld of the
//     accumulator into registers, release to the leader at once (so the next
//     tile's MMAs start), then y = acc * s + b rounded to bf16 and stored.
// Work is persistent: cluster c takes tiles c, c + #clusters, ...  No TMA
// multicast is used: every copy reads this GPU's global memory into the
// issuing CTA's own shared memory.
#include "internal.h"
#include "kernel_common.cuh"
#include "ptx.cuh"

namespace tern {

namespace {

struct Cfg2 {
  static constexpr int kTokPair = 256;            // UMMA N: tokens per tile
  static constexpr int kTokCta = 128;             // x rows each CTA loads
  static constexpr int kBK = 128;                 // k per stage
  static constexpr int kXBox = kTokCta * 128;     // one 64 k x 128 row box, 128-byte swizzle
  static constexpr int kXBytes = 2 * kXBox;
  static constexpr int kCSub = 128 * 16;          // codes of 128 channels x 64 k
  static constexpr int kCBytes = 2 * kCSub;
  static constexpr int kStageBytes = kXBytes + kCBytes;
  static constexpr int kStages = 6;
  static constexpr int kASlots = 4;               // decoded-weight slots in TMEM
  static constexpr int kACols = kBK / 2;          // 32-bit TMEM columns per slot (bf16x2)
  static constexpr int kDCols = kTokPair;         // the accumulator
  static constexpr int kACol0 = kDCols;
  static constexpr int kTmemCols = 512;
  static constexpr int kDecWarps = 4;
  static constexpr int kEpiWarps = 8;             // two per TMEM lane quarter, 128 columns each
  static constexpr int kEpiWarp0 = 2 + kDecWarps;
  static constexpr int kThreads = (2 + kDecWarps + kEpiWarps) * 32;
  static constexpr int kSmemBytes = kStages * kStageBytes + 1024;
  // kind::f16, D fp32, A/B bf16 K-major, N = 256, M = 256 (the pair).
  static constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) |
                                     (uint32_t(kTokPair >> 3) << 17) | (uint32_t(256 >> 4) << 24);
  static_assert(kStageBytes % 1024 == 0, "stages stay 1024-byte aligned for the swizzle");
  static_assert(kACol0 + kASlots * kACols <= kTmemCols, "TMEM columns");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

struct Tile2 {
  const Problem* P;
  int m_tile, n_tile;
};

__device__ __forceinline__ Tile2 tile_of(const Batch& batch, int u) {
  int pi = 0;
  while (pi + 1 < batch.count && u >= batch.p[pi + 1].unit_begin) ++pi;
  Tile2 t;
  t.P = &batch.p[pi];
  const int local = u - t.P->unit_begin;
  t.m_tile = local / t.P->n_tiles;
  t.n_tile = local - t.m_tile * t.P->n_tiles;
  return t;
}

// fp32 pair -> bf16x2 (round to nearest even), lo in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

}  // namespace

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Cfg2::kThreads, 1)
    ternary_mma2_kernel(const __grid_constant__ Batch batch) {
  using C = Cfg2;
  constexpr int S = C::kStages;
  constexpr int A = C::kASlots;

  __shared__ __align__(8) uint64_t full_bar[S];   // TMA of stage s landed (this CTA)
  __shared__ __align__(8) uint64_t empty_bar[S];  // MMAs reading stage s done (both CTAs)
  __shared__ __align__(8) uint64_t afull_bar[A];  // leader: slot a decoded in both CTAs
  __shared__ __align__(8) uint64_t aempty_bar[A]; // MMAs reading slot a done (both CTAs)
  __shared__ __align__(8) uint64_t accfull_bar;   // the tile's last MMA is done (both CTAs)
  __shared__ __align__(8) uint64_t accempty_bar;  // leader: both epilogues drained TMEM
  __shared__ __align__(8) uint64_t drain_bar;     // leader: every MMA issued is done
  __shared__ uint32_t tmem_base_sh;
  extern __shared__ uint8_t dyn_smem[];

  const uint64_t lim = batch.wait_limit_ns;
  unsigned int* const st = batch.status;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t smem_base = (smem_u32(dyn_smem) + 1023u) & ~1023u;
  uint8_t* const smem_gen = dyn_smem + (smem_base - smem_u32(dyn_smem));
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

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0)
      for (int pi = 0; pi < batch.count; ++pi) prefetch_tensormap(&batch.p[pi].tmap_x);
    int it = 0;
    bool ok = true;
    for (int u = u0; u < units && ok; u += ustep) {
      const Tile2 t = tile_of(batch, u);
      const int kc_total = t.P->K >> 6;  // 64-wide k chunks
      const uint8_t* codes = t.P->packed + size_t(t.n_tile * 2 + int(rank)) * kc_total * C::kCSub;
      const int row = t.m_tile * C::kTokPair + int(rank) * C::kTokCta;
      for (int kc = 0; kc < kc_total; kc += 2, ++it) {
        const int s = it % S;
        const int nsub = min(2, kc_total - kc);
        ok = __shfl_sync(0xffffffffu, mbar_wait(smem_u32(&empty_bar[s]), ((it / S) & 1) ^ 1, lim, st), 0);
        if (!ok) break;
        if (lane == 0) {
          const uint32_t stage = smem_base + s * C::kStageBytes;
          const uint32_t fb = smem_u32(&full_bar[s]);
          mbar_arrive_expect_tx(fb, nsub * (C::kXBox + C::kCSub));
          tma_load_2d(stage, &t.P->tmap_x, kc * 64, row, fb);
          if (nsub == 2) tma_load_2d(stage + C::kXBox, &t.P->tmap_x, kc * 64 + 64, row, fb);
          tma_load_bulk(stage + C::kXBytes, codes + size_t(kc) * C::kCSub, nsub * C::kCSub, fb);
        }
        __syncwarp();
      }
    }
    // No copy may still be landing in shared memory when the CTA exits.
    for (int i = it > S ? it - S : 0; i < it; ++i)
      mbar_wait(smem_u32(&full_bar[i % S]), (i / S) & 1, lim, st);
  } else if (warp == 1) {
    // ------------------------------------------------------ MMA issuer (leader)
    if (rank == 0) {
      int it = 0, lt = 0;
      bool ok = true;
      for (int u = u0; u < units && ok; u += ustep, ++lt) {
        const int kc_total = tile_of(batch, u).P->K >> 6;
        ok = __shfl_sync(0xffffffffu, mbar_wait(smem_u32(&accempty_bar), (lt & 1) ^ 1, lim, st), 0);
        if (!ok) break;
        tc_fence_after();
        for (int kc = 0; kc < kc_total; kc += 2, ++it) {
          const int s = it % S, a = it % A;
          const int nmma = kc + 1 < kc_total ? 8 : 4;
          ok = __shfl_sync(0xffffffffu, mbar_wait(smem_u32(&afull_bar[a]), (it / A) & 1, lim, st), 0);
          if (!ok) break;
          tc_fence_after();
          if (lane == 0) {
            const uint32_t stage = smem_base + s * C::kStageBytes;
            const uint32_t a_tmem = tmem + C::kACol0 + a * C::kACols;
#pragma unroll
            for (int j = 0; j < 8; ++j)
              if (j < nmma)
                mma_bf16_ts_2sm(tmem, a_tmem + j * 8,
                                sw128_kmajor_desc(stage + (j >> 2) * C::kXBox + (j & 3) * 32), C::kIdesc,
                                (kc | j) != 0);
            mma_commit_2sm_multicast(smem_u32(&empty_bar[s]), 0x3);
            mma_commit_2sm_multicast(smem_u32(&aempty_bar[a]), 0x3);
          }
          __syncwarp();
        }
        if (ok && lane == 0) mma_commit_2sm_multicast(smem_u32(&accfull_bar), 0x3);
        __syncwarp();
      }
      if (lane == 0) mma_commit_2sm(smem_u32(&drain_bar));
      __syncwarp();
      mbar_wait(smem_u32(&drain_bar), 0, lim, st);
    }
  } else if (warp < C::kEpiWarp0) {
    // ------------------------------------------------------ decoders
    const int quarter = warp & 3;  // TMEM lanes this warp may touch
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = uint32_t(quarter * 32) << 16;
    const uint32_t afull_leader0 = mapa_shared(smem_u32(&afull_bar[0]), 0);
    int it = 0;
    bool ok = true;
    for (int u = u0; u < units && ok; u += ustep) {
      const int kc_total = tile_of(batch, u).P->K >> 6;
      for (int kc = 0; kc < kc_total; kc += 2, ++it) {
        const int s = it % S, a = it % A;
        bool got = mbar_wait(smem_u32(&full_bar[s]), (it / S) & 1, lim, st);
        got = got && mbar_wait(smem_u32(&aempty_bar[a]), ((it / A) & 1) ^ 1, lim, st);
        ok = __all_sync(0xffffffffu, got);
        if (!ok) break;
        tc_fence_after();
        const uint8_t* cp = smem_gen + s * C::kStageBytes + C::kXBytes + r * 16;
        const uint32_t dst = tmem + lane_off + C::kACol0 + a * C::kACols;
        uint32_t t[32];
        const uint4 v0 = *reinterpret_cast<const uint4*>(cp);
        decode_word(v0.x, t + 0);
        decode_word(v0.y, t + 8);
        decode_word(v0.z, t + 16);
        decode_word(v0.w, t + 24);
        tmem_st32(dst, t);
        if (kc + 1 < kc_total) {
          const uint4 v1 = *reinterpret_cast<const uint4*>(cp + C::kCSub);
          decode_word(v1.x, t + 0);
          decode_word(v1.y, t + 8);
          decode_word(v1.z, t + 16);
          decode_word(v1.w, t + 24);
          tmem_st32(dst + 32, t);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(afull_leader0 + a * 8);
      }
    }
  } else {
    // ------------------------------------------------------ epilogue
    const int ew = warp - C::kEpiWarp0;
    const int quarter = warp & 3;
    const int half = ew >> 2;  // token columns [128 * half, 128 * half + 128)
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = uint32_t(quarter * 32) << 16;
    const uint32_t accempty_leader = mapa_shared(smem_u32(&accempty_bar), 0);
    int lt = 0;
    for (int u = u0; u < units; u += ustep, ++lt) {
      const Tile2 t = tile_of(batch, u);
      const Problem& P = *t.P;
      const int n = t.n_tile * 256 + int(rank) * 128 + r;
      const float sc = P.scales[n];
      const float bi = P.bias ? bf16_bits_to_float(reinterpret_cast<const uint16_t*>(P.bias)[n]) : 0.f;
      if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&accfull_bar), lt & 1, lim, st))) break;
      tc_fence_after();
      uint32_t out[64];  // bf16x2: tokens (2c, 2c + 1) of this half
#pragma unroll
      for (int c0 = 0; c0 < 128; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_off + half * 128 + c0, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j)
          out[c0 / 2 + j] = pack_bf16x2(fmaf(__uint_as_float(v[2 * j]), sc, bi),
                                        fmaf(__uint_as_float(v[2 * j + 1]), sc, bi));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(accempty_leader);
      const int row0 = t.m_tile * C::kTokPair + half * 128;
      const int rows = min(128, P.M - row0);
      uint16_t* yp = reinterpret_cast<uint16_t*>(P.y) + size_t(row0) * P.N + n;
#pragma unroll
      for (int c = 0; c < 128; ++c)
        if (c < rows) yp[size_t(c) * P.N] = uint16_t(out[c >> 1] >> ((c & 1) * 16));
    }
  }

  // ------------------------------------------------------ teardown
  // No CTA may leave while the pair's MMAs or remote arrivals still touch it.
  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_2sm(tmem, C::kTmemCols);
  }
}

int smem_bytes_2sm() { return Cfg2::kSmemBytes; }

static cudaError_t configure_2sm() {
  static unsigned long long configured = 0;  // one bit per device ordinal
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64) return cudaErrorInvalidDevice;
  if (!(__atomic_load_n(&configured, __ATOMIC_ACQUIRE) & (1ull << dev))) {
    e = cudaFuncSetAttribute(ternary_mma2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Cfg2::kSmemBytes);
    if (e != cudaSuccess) return e;
    __atomic_fetch_or(&configured, 1ull << dev, __ATOMIC_RELEASE);
  }
  return cudaSuccess;
}

cudaError_t launch_ternary_mma2(const Batch& batch, int clusters, cudaStream_t stream) {
  cudaError_t e = configure_2sm();
  if (e != cudaSuccess) return e;
  ternary_mma2_kernel<<<2 * clusters, Cfg2::kThreads, Cfg2::kSmemBytes, stream>>>(batch);
  return cudaGetLastError();
}

int max_active_clusters_2sm() {
  if (configure_2sm() != cudaSuccess) return 0;
  int n = 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * 148);
  cfg.blockDim = dim3(Cfg2::kThreads);
  cfg.dynamicSmemBytes = Cfg2::kSmemBytes;
  if (cudaOccupancyMaxActiveClusters(&n, ternary_mma2_kernel, &cfg) != cudaSuccess) return 0;
  return n;
}

}  // namespace tern
