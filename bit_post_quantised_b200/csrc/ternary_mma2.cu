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
// Per CTA, per 128-wide k stage (36 KiB of shared memory, 6 stages, 4 with a
// residual epilogue; the last stage of a row holds 64 k when K % 128 == 64):
//   * warp 0 (producer): one 3-D TMA copy of its 128 x-rows x 128 k (two
//     64-k chunks, 128-byte swizzle) and one bulk copy of its codes (128
//     channels x 128 k, contiguous in the tile-interleaved layout), both
//     completing on full[s]; consecutive stages are issued by different
//     lanes, because one thread issues a copy only every ~280 cycles.
//   * warps 2-5 (decoders): one thread per channel row waits for the stage
//     and for TMEM slot a (4 slots of 64 columns) to be free, expands its
//     code bytes into bf16x2 TMEM columns (tcgen05.st), then one lane per warp
//     arrives on the leader CTA's afull[a].  The arrival also vouches for
//     that CTA's x rows of the stage, which the decoder waited for.
//   * warp 1 of the leader CTA (rank 0): waits afull[a] (eight arrivals, four
//     from each CTA), issues the eight MMAs of the stage and commits, with
//     one arrival in both CTAs, to empty[s] (shared-memory stage free) and
//     aempty[a] (TMEM slot free).  The whole warp computes the operands and
//     its elected lane issues the stage as one block, so the operands stay
//     uniform.  Eight MMAs (1024 tensor cycles) between two waits of the
//     issuing thread keep the tensor pipe fed; a wait every four MMAs
//     measurably starves it.
//   * warps 6-21 (epilogue, 64 tokens each): after the tile's last MMA,
//     tcgen05.ld of the accumulator into registers, release to the leader at
//     once (the single accumulator holds up the next tile's MMAs until
//     then), then y = acc * s + b rounded to bf16 and stored.  A residual
//     epilogue copies each warp's residual slice into shared memory while
//     the tile's MMAs run, so after the release it reads shared memory only.
// The 64-token tiles (16 < M <= 64) run on single CTAs (cta_group::1, 128
// channels x 64 tokens) with the same roles, eight decoder warps (two
// groups of four taking alternate stages), eight epilogue warps, two
// accumulators and 256-k stages (40 KiB, 5 stages, 4 with a residual
// epilogue; 3 TMEM slots of 128 columns): sixteen MMAs per handshake
// instead of eight.
// Work is persistent: cluster c takes tiles c, c + #clusters, ...  No TMA
// multicast is used: every copy reads this GPU's global memory into the
// issuing CTA's own shared memory.
#include <algorithm>

#include "internal.h"
#include "kernel_common.cuh"
#include "ptx.cuh"

namespace tern {

namespace {

// TOK = UMMA N = tokens per tile.  PAIR: a cluster of two CTAs shares each
// MMA (cta_group::2, M = 256 channels, each CTA loads TOK / 2 x rows) -- used
// for TOK = 256, where one instruction is long enough to hide its issue cost.
// !PAIR: one CTA per tile (cta_group::1, M = 128 channels, all TOK x rows),
// used for TOK = 64, where a pair instruction would take as long as at
// N = 256 but do a quarter of the work.
// EPI == 2 (residual or gate epilogues) trades two x stages for a shared
// memory slice per epilogue warp where each tile's residual lands while its
// MMAs run (4 stages keep the tensor pipe as busy as 6 on the plain layer).
// EPI == 3 keeps 6: its normalising epilogue holds the accumulator long
// enough that the deeper pipeline pays (4 stages: +18 us on QKV).
template <int TOK, bool PAIR, int EPI = 0>
struct Cfg2 {
  static constexpr int kTokPair = TOK;
  static constexpr int kTokCta = PAIR ? TOK / 2 : TOK;  // x rows each CTA loads
  static constexpr int kChCta = 128;              // channels (TMEM lanes) per CTA
  static constexpr int kChTile = PAIR ? 256 : 128;  // channels per tile
  // 64-k chunks per stage.  Every stage costs its handshakes (copy landed,
  // slot decoded, MMAs done: several hundred cycles, measured) however many
  // MMAs it feeds, and an N = 64 MMA is short, so the 64-token tiles take
  // 256 k per stage; the pair tiles' N = 256 MMAs hide them at 128 k.
  static constexpr int kChunks = TOK >= 256 ? 2 : 4;
  static constexpr int kBK = 64 * kChunks;        // k per stage
  static constexpr int kXBox = kTokCta * 128;     // one 64 k x kTokCta row box, 128-byte swizzle
  static constexpr int kXBytes = kChunks * kXBox;
  static constexpr int kCSub = 128 * 16;          // codes of 128 channels x 64 k
  static constexpr int kCBytes = kChunks * kCSub;
  static constexpr int kStageBytes = kXBytes + kCBytes;
  static constexpr bool kResStaged = EPI == 2;
  static constexpr int kStages = TOK >= 256 ? (kResStaged ? 4 : 6) : (kResStaged ? 4 : 5);
  static constexpr int kACols = kBK / 2;          // 32-bit TMEM columns per slot (bf16x2)
  static constexpr int kDCols = TOK;              // one accumulator
  // Two accumulators (the epilogue of a tile overlaps the next tile's MMAs)
  // where TMEM has room next to the A slots; one at N = 256.
  static constexpr int kAccBufs = TOK >= 256 ? 1 : 2;
  static constexpr int kACol0 = kAccBufs * kDCols;
  static constexpr int kTmemCols = 512;
  // Decoded-weight slots in TMEM: what the accumulators leave, at most four
  // (4 x 128 k at N = 256, 3 x 256 k at N = 64).
  static constexpr int kASlots = (kTmemCols - kACol0) / kACols < 4 ? (kTmemCols - kACol0) / kACols : 4;
  // A narrow tile makes the MMAs of a stage short, so decoding needs more warps.
  static constexpr int kDecWarps = TOK >= 256 ? 4 : 8;
  // Epilogue warps: kEpiWarps / 4 per TMEM lane quarter, each draining
  // kEpiCols accumulator columns.  The single accumulator of the 256-token
  // tile is released sooner with more of them.
  static constexpr int kEpiWarps = TOK >= 256 ? 16 : 8;
  static constexpr int kEpiCols = TOK / (kEpiWarps / 4);
  static constexpr int kEpiWarp0 = 2 + kDecWarps;
  static constexpr int kThreads = (2 + kDecWarps + kEpiWarps) * 32;
  // Residual slice of one epilogue warp: its kEpiCols tokens x 32 channels, bf16.
  static constexpr int kResWarpBytes = kEpiCols * 64;
  static constexpr int kResBytes = kResStaged ? kEpiWarps * kResWarpBytes : 0;
  static constexpr int kSmemBytes = kStages * kStageBytes + kResBytes + 1024;
  static constexpr int kCtas = PAIR ? 2 : 1;      // CTAs sharing one MMA
  // kind::f16, D fp32, A/B bf16 K-major, N = TOK, M = 128 per CTA of the MMA.
  static constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) |
                                     (uint32_t(TOK >> 3) << 17) | (uint32_t((128 * kCtas) >> 4) << 24);
  static_assert(TOK % 64 == 0 && TOK >= 64 && TOK <= 256, "UMMA N; 32-column epilogue loads per half");
  static_assert(kStageBytes % 1024 == 0, "stages stay 1024-byte aligned for the swizzle");
  static_assert(kACol0 + kASlots * kACols <= kTmemCols, "TMEM columns");
  static_assert(kSmemBytes + 6 * 1024 <= 227 * 1024, "shared memory, with the static barriers and norm sums");
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

// The tcgen05 forms of a one-CTA tile (cta_group::1) or a CTA-pair tile
// (cta_group::2: the leader's commits arrive in both CTAs, the other CTA's
// warps arrive on the leader's barriers).  The commits are called by the whole
// converged MMA warp and issued by its elected lane, like the MMAs.
template <bool PAIR>
struct Tc;
template <>
struct Tc<true> {
  static __device__ __forceinline__ void alloc(uint32_t dst, uint32_t n) { tmem_alloc_2sm(dst, n); }
  static __device__ __forceinline__ void relinquish() { tmem_relinquish_2sm(); }
  static __device__ __forceinline__ void dealloc(uint32_t t, uint32_t n) { tmem_dealloc_2sm(t, n); }
  static __device__ __forceinline__ void commit_all(uint32_t bar) { mma_commit_2sm_multicast_elected(bar, 0x3); }
  static __device__ __forceinline__ void commit_local(uint32_t bar) { mma_commit_2sm_elected(bar); }
  static __device__ __forceinline__ uint32_t leader_addr(uint32_t bar) { return mapa_shared(bar, 0); }
  static __device__ __forceinline__ void arrive_leader(uint32_t addr) { mbar_arrive_cluster(addr); }
  static __device__ __forceinline__ void sync_all() { cluster_sync(); }
};
template <>
struct Tc<false> {
  static __device__ __forceinline__ void alloc(uint32_t dst, uint32_t n) { tmem_alloc(dst, n); }
  static __device__ __forceinline__ void relinquish() { tmem_relinquish(); }
  static __device__ __forceinline__ void dealloc(uint32_t t, uint32_t n) { tmem_dealloc(t, n); }
  static __device__ __forceinline__ void commit_all(uint32_t bar) { mma_commit_elected(bar); }
  static __device__ __forceinline__ void commit_local(uint32_t bar) { mma_commit_elected(bar); }
  static __device__ __forceinline__ uint32_t leader_addr(uint32_t bar) { return bar; }
  static __device__ __forceinline__ void arrive_leader(uint32_t addr) { mbar_arrive(addr); }
  static __device__ __forceinline__ void sync_all() { __syncthreads(); }
};

// Sums a[i] over the 32 lanes of the warp for every i and leaves the sum for
// i = lane * (N / 32) + j in a[j], j < N / 32 (the other entries are dead).
// Five butterfly steps, each halving the entries a lane keeps: N - N/32
// shuffles in all.
template <int N>
__device__ __forceinline__ void warp_reduce_scatter(float (&a)[N], int lane) {
  static_assert(N >= 32 && (N & (N - 1)) == 0, "N");
#pragma unroll
  for (int step = 0; step < 5; ++step) {
    const int o = 16 >> step, half = (N >> step) / 2;
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int j = 0; j < half; ++j) {
      const float send = up ? a[j] : a[j + half];
      const float keep = up ? a[j + half] : a[j];
      a[j] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
}

// EPI: the fused epilogues a launch needs -- 0 none, 1 activations only, 2
// residual or gate as well, 3 RMS normalisation of 128-channel groups as
// well.  Each level is its own instantiation, so a richer epilogue cannot
// cost a plainer launch registers.
template <int TOK, bool PAIR, int EPI>
__device__ __forceinline__ void tile_kernel_body(const Batch& batch) {
  using C = Cfg2<TOK, PAIR, EPI>;
  using T = Tc<PAIR>;
  constexpr int S = C::kStages;
  constexpr int A = C::kASlots;
  constexpr int AB = C::kAccBufs;

  __shared__ __align__(8) uint64_t full_bar[S];      // TMA of stage s landed (this CTA)
  __shared__ __align__(8) uint64_t empty_bar[S];     // MMAs reading stage s done (both CTAs)
  __shared__ __align__(8) uint64_t afull_bar[A];     // leader: slot a decoded in both CTAs
  __shared__ __align__(8) uint64_t aempty_bar[A];    // MMAs reading slot a done (both CTAs)
  __shared__ __align__(8) uint64_t accfull_bar[AB];  // a tile's last MMA is done (both CTAs)
  __shared__ __align__(8) uint64_t accempty_bar[AB]; // leader: both epilogues drained TMEM
  __shared__ __align__(8) uint64_t drain_bar;        // leader: every MMA issued is done
  __shared__ uint32_t tmem_base_sh;
  // RMS normalisation (EPI == 3): per 64-token column group ("half") of the
  // epilogue, each lane quarter's partial sums of squares, the inverse RMS per
  // token, and two barriers (partials written, inverses written).
  constexpr int kHalves = C::kEpiWarps / 4;
  __shared__ float norm_part[EPI == 3 ? kHalves * 4 * C::kEpiCols : 1];
  __shared__ float norm_inv[EPI == 3 ? kHalves * C::kEpiCols : 1];
  __shared__ __align__(8) uint64_t norm_bar[EPI == 3 ? 2 * kHalves : 1];
  // EPI == 2: per epilogue warp, its residual slice of the tile has landed.
  __shared__ __align__(8) uint64_t res_bar[C::kResStaged ? C::kEpiWarps : 1];
  extern __shared__ uint8_t dyn_smem[];

  const uint64_t lim = batch.wait_limit_ns;
  unsigned int* const st = batch.status;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const uint32_t smem_base = (smem_u32(dyn_smem) + 1023u) & ~1023u;
  uint8_t* const smem_gen = dyn_smem + (smem_base - smem_u32(dyn_smem));
  const int u0 = PAIR ? int(cluster_id_x()) : int(blockIdx.x);
  const int ustep = PAIR ? int(nclusters_x()) : int(gridDim.x);
  const int units = batch.total_units;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    for (int a = 0; a < A; ++a) {
      mbar_init(smem_u32(&afull_bar[a]), C::kCtas * 4);  // one decoder warp per lane quarter per CTA
      mbar_init(smem_u32(&aempty_bar[a]), 1);
    }
    for (int b = 0; b < AB; ++b) {
      mbar_init(smem_u32(&accfull_bar[b]), 1);
      mbar_init(smem_u32(&accempty_bar[b]), C::kCtas * C::kEpiWarps);
    }
    mbar_init(smem_u32(&drain_bar), 1);
    if constexpr (EPI == 3)
      for (int h = 0; h < 2 * kHalves; ++h) mbar_init(smem_u32(&norm_bar[h]), 4);
    if constexpr (C::kResStaged)
      for (int w = 0; w < C::kEpiWarps; ++w) mbar_init(smem_u32(&res_bar[w]), 1);
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    T::alloc(smem_u32(&tmem_base_sh), C::kTmemCols);
    T::relinquish();
  }
  tc_fence_before();
  T::sync_all();  // (both CTAs') barriers exist and TMEM is allocated
  // The previous kernel of the stream may still be running (programmatic
  // dependent launch): the producer first asks L2 for the codes of its first
  // stages (a hint: a write by that kernel still reaches the readers through
  // L2), then every thread waits for it before touching global memory.
  if (warp == 0 && lane == 0 && u0 < units) {
    const Tile2 t = tile_of(batch, u0);
    const int kc_total = t.P->K >> 6;
    const uint8_t* codes = t.P->packed + size_t(t.n_tile * C::kCtas + int(rank)) * kc_total * C::kCSub;
    prefetch_l2_bulk(codes, uint32_t(min(kc_total, S * C::kChunks)) * C::kCSub);
  }
  pdl_wait();
  pdl_trigger();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    // Stage it is issued by lane it % L: one thread issues a bulk or tensor
    // copy only every ~280 SM cycles (measured: one lane streaming 4 KiB
    // copies reaches 4.1 TB/s, four lanes 7.1), which at two copies per stage
    // would pace the short stages of the 64-token tiles.  Each lane owns the
    // ring slots s = lane, lane + L, ... (S % L == 0), so a slot's phases are
    // waited for by one thread, in order.
    constexpr int L = S % 4 == 0 ? 4 : S % 3 == 0 ? 3 : S % 2 == 0 ? 2 : 1;
    if (lane == 0)
      for (int pi = 0; pi < batch.count; ++pi) prefetch_tensormap(&batch.p[pi].tmap_x);
    __syncwarp();
    if (lane < L) {
      int it = 0;
      bool ok = true;
      for (int u = u0; u < units && ok; u += ustep) {
        const Tile2 t = tile_of(batch, u);
        const int kc_total = t.P->K >> 6;  // 64-wide k chunks
        const uint8_t* codes =
            t.P->packed + size_t(t.n_tile * C::kCtas + int(rank)) * kc_total * C::kCSub;
        const int row = t.m_tile * C::kTokPair + int(rank) * C::kTokCta;
        for (int kc = 0; kc < kc_total; kc += C::kChunks, ++it) {
          if (it % L != lane) continue;
          const int s = it % S;
          ok = mbar_wait(smem_u32(&empty_bar[s]), ((it / S) & 1) ^ 1, lim, st);
          if (!ok) break;
          const int nsub = min(C::kChunks, kc_total - kc);
          const uint32_t stage = smem_base + s * C::kStageBytes;
          const uint32_t fb = smem_u32(&full_bar[s]);
          // One 3-D box brings all 64-k chunks of x of the stage (those past
          // K read as zero); the codes of the stage are one contiguous block.
          mbar_arrive_expect_tx(fb, C::kXBytes + nsub * C::kCSub);
          tma_load_3d(stage, &t.P->tmap_x, 0, row, kc, fb);
          tma_load_bulk(stage + C::kXBytes, codes + size_t(kc) * C::kCSub, nsub * C::kCSub, fb);
        }
      }
      // No copy this lane issued may still be landing in shared memory when
      // the CTA exits.
      for (int i = it > S ? it - S : 0; i < it; ++i)
        if (i % L == lane) mbar_wait(smem_u32(&full_bar[i % S]), (i / S) & 1, lim, st);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------ MMA issuer (leader)
    const uint32_t tmem_u = __shfl_sync(0xffffffffu, tmem, 0);  // warp-uniform TMEM base
    if (rank == 0) {  // the leader issues for the pair
      int it = 0, lt = 0;
      bool ok = true;
      for (int u = u0; u < units && ok; u += ustep, ++lt) {
        const int kc_total = tile_of(batch, u).P->K >> 6;
        const int ab = lt % AB;
        ok = __shfl_sync(0xffffffffu, mbar_wait(smem_u32(&accempty_bar[ab]), ((lt / AB) & 1) ^ 1, lim, st), 0);
        if (!ok) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_u + ab * C::kDCols;
        for (int kc = 0; kc < kc_total; kc += C::kChunks, ++it) {
          const int s = it % S, a = it % A;
          ok = __shfl_sync(0xffffffffu, mbar_wait(smem_u32(&afull_bar[a]), (it / A) & 1, lim, st), 0);
          if (!ok) break;
          tc_fence_after();
          // The whole warp computes the (uniform) operands; one lane issues.
          uint32_t a_tmem = tmem_u + C::kACol0 + a * C::kACols;
          uint64_t desc = sw128_kmajor_desc(smem_base + s * C::kStageBytes);
          const uint32_t bar0 = smem_u32(&empty_bar[s]), bar1 = smem_u32(&aempty_bar[a]);
          constexpr uint64_t kChunk2 = uint64_t(C::kXBox >> 4);  // next 64-k chunk of x, 16-byte units
          int left = kc_total - kc;  // 64-k chunks this stage still holds
          uint32_t acc = kc != 0;
          if constexpr (C::kChunks == 4) {
            // 256-k stage: the first 128 k (when the stage has more) without
            // a commit, then the rest with the stage's two commits.
            if (left > 2) {
              mma_stage_open<PAIR>(d_tmem, a_tmem, desc, C::kIdesc, acc, kChunk2);
              a_tmem += 64;
              desc += 2 * kChunk2;
              acc = 1;
              left -= 2;
            }
          }
          if (left >= 2)
            mma_stage<8, PAIR>(d_tmem, a_tmem, desc, C::kIdesc, acc, bar0, bar1, kChunk2);
          else
            mma_stage<4, PAIR>(d_tmem, a_tmem, desc, C::kIdesc, acc, bar0, bar1, kChunk2);
        }
        if (ok) T::commit_all(smem_u32(&accfull_bar[ab]));  // converged warp: the issuing lane
        __syncwarp();
      }
      T::commit_local(smem_u32(&drain_bar));
      __syncwarp();
      mbar_wait(smem_u32(&drain_bar), 0, lim, st);
    }
  } else if (warp < C::kEpiWarp0) {
    // ------------------------------------------------------ decoders
    // Each thread expands every 64-k chunk of its channel row of a stage.
    // With eight decoder warps, warps 2-5 take the even stages and warps 6-9
    // the odd ones: a stage's decode is a chain of latencies (two barrier
    // polls of ~200 cycles each even when the phase is complete, shared
    // loads, tcgen05.st and its wait), so two stages in flight double the
    // rate at which slots fill; splitting one stage's chunks over both
    // groups instead left every stage paying the whole chain.
    constexpr int kGroups = C::kDecWarps / 4;
    const int group = (warp - 2) >> 2;
    const int quarter = warp & 3;  // TMEM lanes this warp may touch
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = uint32_t(quarter * 32) << 16;
    const uint32_t afull_leader0 = T::leader_addr(smem_u32(&afull_bar[0]));
    int it = 0;
    bool ok = true;
    for (int u = u0; u < units && ok; u += ustep) {
      const int kc_total = tile_of(batch, u).P->K >> 6;
      for (int kc = 0; kc < kc_total; kc += C::kChunks, ++it) {
        if (kGroups > 1 && it % kGroups != group) continue;
        const int s = it % S, a = it % A;
        ok = __all_sync(0xffffffffu, mbar_wait_both(smem_u32(&full_bar[s]), (it / S) & 1, smem_u32(&aempty_bar[a]),
                                                    ((it / A) & 1) ^ 1, lim, st));
        if (!ok) break;
        tc_fence_after();
        const uint8_t* cp = smem_gen + s * C::kStageBytes + C::kXBytes + r * 16;
        const uint32_t dst = tmem + lane_off + C::kACol0 + a * C::kACols;
#pragma unroll
        for (int sub = 0; sub < C::kChunks; ++sub) {
          if (kc + sub < kc_total) {
            uint32_t t[32];
            const uint4 v = *reinterpret_cast<const uint4*>(cp + sub * C::kCSub);
            decode_word_2t(v.x, t + 0);  // A holds 2t: the epilogue halves the scale
            decode_word_2t(v.y, t + 8);
            decode_word_2t(v.z, t + 16);
            decode_word_2t(v.w, t + 24);
            tmem_st32(dst + sub * 32, t);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) T::arrive_leader(afull_leader0 + a * 8);
      }
    }
  } else {
    // ------------------------------------------------------ epilogue
    constexpr int kCols = C::kEpiCols;
    const int ew = warp - C::kEpiWarp0;
    const int quarter = warp & 3;
    const int half = ew >> 2;  // token columns [kCols * half, kCols * half + kCols) ("half" of 2 or 4)
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = uint32_t(quarter * 32) << 16;
    const uint32_t accempty_leader0 = T::leader_addr(smem_u32(&accempty_bar[0]));
    int lt = 0;
    int norm_it = 0;  // normalised tiles so far (the phase of norm_bar)
    int res_it = 0;   // residual slices staged so far (the phase of res_bar[ew])
    for (int u = u0; u < units; u += ustep, ++lt) {
      const Tile2 t = tile_of(batch, u);
      const Problem& P = *t.P;
      const int ab = lt % AB;
      const int n = t.n_tile * C::kChTile + int(rank) * C::kChCta + r;
      const float sc = 0.5f * P.scales[n];  // A held 2t
      const float bi = P.bias ? bf16_bits_to_float(reinterpret_cast<const uint16_t*>(P.bias)[n]) : 0.f;
      // Per tile (the same for every warp of the CTA): a tile whose 128
      // channels get no epilogue step (no residual or gate, no activation
      // or normalisation on them: the v columns of a QKV with q/k norm, the
      // attention columns of a single block's fused projection) takes the
      // plain epilogue, and one with only an activation the activation
      // epilogue, whatever else the launch carries.
      bool plain = true, act_only = false;
      if constexpr (EPI > 0) {
        const int n0 = n - r;  // the CTA's first channel
        act_only = !P.residual && !P.gate && !(n0 >= P.norm_col0 && n0 < P.norm_col1);
        plain = act_only && (P.act == kActNone || n0 + 127 < P.act_col0);
      }
      // Residual, gate and activation ("early", EPI == 2): this warp's slice
      // of the tile's residual (its 32 channels of kCols tokens, 64 bytes per
      // token) is copied into shared memory while the tile's MMAs run; after
      // the release the epilogue reads shared memory only.  (Read from global
      // memory after the release, the residual's round trips and the
      // registers they need made the epilogue longer than the next tile's
      // MMAs.)
      bool early = false, staged = false;
      float gt = 1.f;
      if constexpr (EPI >= 2) {
        const bool normed = EPI == 3 && n - r >= P.norm_col0 && n - r < P.norm_col1;
        const uint16_t* res = reinterpret_cast<const uint16_t*>(P.residual);
        early = C::kResStaged && !plain && !normed && (reinterpret_cast<uintptr_t>(res) & 15) == 0;
        const int row0 = t.m_tile * C::kTokPair + half * kCols;
        const int rows = max(0, min(kCols, P.M - row0));
        if (early) {
          if (P.gate) gt = bf16_bits_to_float(reinterpret_cast<const uint16_t*>(P.gate)[n]);
          if (res) {
            // The warp read its previous slice before its last release.
            fence_proxy_async_smem();
            const uint32_t bar = smem_u32(&res_bar[ew]);
            const uint32_t dst = smem_base + C::kStages * C::kStageBytes + ew * C::kResWarpBytes;
            // 16-byte aligned: res is, N is a multiple of 128 and n - lane of 32
            const uint8_t* src = reinterpret_cast<const uint8_t*>(res + size_t(row0) * P.ldy + (n - lane));
            if (lane == 0) mbar_arrive_expect_tx(bar, uint32_t(rows) * 64u);
            __syncwarp();
            for (int c = lane; c < rows; c += 32) tma_load_bulk(dst + c * 64, src + size_t(c) * P.ldy * 2, 64, bar);
            staged = true;
          }
        } else if (res) {
          // Otherwise bring the residual rows into L2, so the loads after the
          // release do not wait for HBM.
          for (int c = 0; c < rows; ++c) prefetch_l2(res + size_t(row0 + c) * P.ldy + n);
        }
      }
      if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&accfull_bar[ab]), (lt / AB) & 1, lim, st))) {
        if (staged) mbar_wait(smem_u32(&res_bar[ew]), res_it & 1, lim, st);  // no copy may land after exit
        break;
      }
      tc_fence_after();
      if (C::kResStaged && early) {
        // y = residual + gate * act(acc * s + b), one rounding.  The
        // accumulator is released as soon as acc * s + b is in registers; the
        // activation and the residual slice (from shared memory) come after.
        float f[kCols];
#pragma unroll
        for (int c0 = 0; c0 < kCols; c0 += 32) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_off + ab * C::kDCols + half * kCols + c0, v);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) f[c0 + j] = fmaf(__uint_as_float(v[j]), sc, bi);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) T::arrive_leader(accempty_leader0 + ab * 8);
        if (P.act != kActNone) {
          const int act = P.act, act_col0 = P.act_col0;
#pragma unroll
          for (int c = 0; c < kCols; ++c) f[c] = apply_act(f[c], act, n, act_col0);
        }
        uint32_t out[kCols / 2];  // bf16x2: tokens (2i, 2i + 1) of this lane's channel
        if (staged) {
          const bool ok_r = mbar_wait(smem_u32(&res_bar[ew]), res_it & 1, lim, st);
          ++res_it;
          if (!__all_sync(0xffffffffu, ok_r)) break;
          // Tokens past M read stale shared memory; they are not stored.
          const uint16_t* sres =
              reinterpret_cast<const uint16_t*>(smem_gen + C::kStages * C::kStageBytes + ew * C::kResWarpBytes) + lane;
#pragma unroll
          for (int i = 0; i < kCols / 2; ++i)
            out[i] = pack_bf16x2(fmaf(gt, f[2 * i], bf16_bits_to_float(sres[2 * i * 32])),
                                 fmaf(gt, f[2 * i + 1], bf16_bits_to_float(sres[(2 * i + 1) * 32])));
        } else {
#pragma unroll
          for (int i = 0; i < kCols / 2; ++i) out[i] = pack_bf16x2(fmaf(gt, f[2 * i], 0.f), fmaf(gt, f[2 * i + 1], 0.f));
        }
        // Two channels of one token per word (lane l: channels 2(l % 16) and
        // 2(l % 16) + 1 of token 2i + l / 16) for 4-byte stores.
        const int row0 = t.m_tile * C::kTokPair + half * kCols;
        const int rows = min(kCols, P.M - row0);
        const int ld = P.ldy;
        uint16_t* yp = reinterpret_cast<uint16_t*>(P.y) + size_t(row0) * P.ldy + (n - lane) + 2 * (lane & 15);
        const uint32_t sel = (lane >> 4) ? 0x7632u : 0x5410u;
#pragma unroll
        for (int i = 0; i < kCols / 2; ++i) {
          const uint32_t a = __shfl_sync(0xffffffffu, out[i], 2 * (lane & 15));
          const uint32_t b = __shfl_sync(0xffffffffu, out[i], 2 * (lane & 15) + 1);
          const int c = 2 * i + (lane >> 4);
          if (c < rows) *reinterpret_cast<uint32_t*>(yp + c * ld) = __byte_perm(a, b, sel);
        }
      } else if (plain || EPI == 1 || act_only) {
        uint32_t out[kCols / 2];  // bf16x2: tokens (2c, 2c + 1) of this half
        if (plain) {
#pragma unroll
          for (int c0 = 0; c0 < kCols; c0 += 32) {
            uint32_t v[32];
            tmem_ld32(tmem + lane_off + ab * C::kDCols + half * kCols + c0, v);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j)
              out[c0 / 2 + j] = pack_bf16x2(fmaf(__uint_as_float(v[2 * j]), sc, bi),
                                            fmaf(__uint_as_float(v[2 * j + 1]), sc, bi));
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) T::arrive_leader(accempty_leader0 + ab * 8);
        } else {
          // Activation only: its transcendentals run after the accumulator
          // is released, overlapping the next tile's MMAs; y stays fp32 until
          // then.
          float f[kCols];
#pragma unroll
          for (int c0 = 0; c0 < kCols; c0 += 32) {
            uint32_t v[32];
            tmem_ld32(tmem + lane_off + ab * C::kDCols + half * kCols + c0, v);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) f[c0 + j] = fmaf(__uint_as_float(v[j]), sc, bi);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) T::arrive_leader(accempty_leader0 + ab * 8);
#pragma unroll
          for (int j = 0; j < kCols / 2; ++j)
            out[j] = pack_bf16x2(apply_act(f[2 * j], P.act, n, P.act_col0),
                                 apply_act(f[2 * j + 1], P.act, n, P.act_col0));
        }
        const int row0 = t.m_tile * C::kTokPair + half * kCols;
        const int rows = min(kCols, P.M - row0);
        uint16_t* yp = reinterpret_cast<uint16_t*>(P.y) + size_t(row0) * P.ldy + n;
#pragma unroll
        for (int c = 0; c < kCols; ++c)
          if (c < rows) yp[size_t(c) * P.ldy] = uint16_t(out[c >> 1] >> ((c & 1) * 16));
      } else if (EPI == 3 && n - r >= P.norm_col0 && n - r < P.norm_col1 && !P.residual && !P.gate &&
                 (P.act == kActNone || n - r + 127 < P.act_col0)) {
        // RMS normalisation with nothing else on these channels (FLUX's q/k
        // norm; the CTA's 128 channels are one group and the condition is
        // the same for every warp of the CTA).  y = acc * s + b is rounded
        // to bf16 as it leaves TMEM -- as the unfused layer stores q and k in
        // bf16 and normalises those -- so the accumulator is released after
        // one read, like the plain epilogue's; the sums of squares of the
        // rounded values, their exchange across the four lane quarters and
        // the scaling all run after the release, overlapping the next
        // tile's MMAs.  Two bf16 roundings: within 3 * 2^-9 relative.
        uint32_t out[kCols / 2];  // bf16x2: tokens (2i, 2i + 1) of this lane's channel
#pragma unroll
        for (int c0 = 0; c0 < kCols; c0 += 32) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_off + ab * C::kDCols + half * kCols + c0, v);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j)
            out[c0 / 2 + j] = pack_bf16x2(fmaf(__uint_as_float(v[2 * j]), sc, bi),
                                          fmaf(__uint_as_float(v[2 * j + 1]), sc, bi));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) T::arrive_leader(accempty_leader0 + ab * 8);
        const float w = P.norm_weight ? bf16_bits_to_float(reinterpret_cast<const uint16_t*>(P.norm_weight)[n]) : 1.f;
#pragma unroll
        for (int c0 = 0; c0 < kCols; c0 += 32) {
          float sq[32];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float lo = __uint_as_float(out[c0 / 2 + j] << 16), hi = __uint_as_float(out[c0 / 2 + j] & 0xFFFF0000u);
            sq[2 * j] = lo * lo;
            sq[2 * j + 1] = hi * hi;
          }
          warp_reduce_scatter<32>(sq, lane);  // token c0 + lane, this warp's 32 channels
          norm_part[(half * 4 + quarter) * kCols + c0 + lane] = sq[0];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&norm_bar[2 * half]));
        bool ok_n = mbar_wait(smem_u32(&norm_bar[2 * half]), norm_it & 1, lim, st);
        if (quarter == 0 && ok_n)
          for (int c = lane; c < kCols; c += 32) {
            const float tot = (norm_part[(half * 4 + 0) * kCols + c] + norm_part[(half * 4 + 1) * kCols + c]) +
                              (norm_part[(half * 4 + 2) * kCols + c] + norm_part[(half * 4 + 3) * kCols + c]);
            norm_inv[half * kCols + c] = rsqrtf(tot * (1.0f / 128.0f) + P.norm_eps);
          }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&norm_bar[2 * half + 1]));
        ok_n = mbar_wait(smem_u32(&norm_bar[2 * half + 1]), norm_it & 1, lim, st) && ok_n;
        ++norm_it;
        if (!__all_sync(0xffffffffu, ok_n)) break;
        const int row0 = t.m_tile * C::kTokPair + half * kCols;
        const int rows = min(kCols, P.M - row0);
        // Rotary (cos, sin) of this lane's channel pair, kRG token rows at a
        // time: the rows come from L2, so a group's loads go out together.
        // The two lanes of a pair split the rows (the even lane loads the
        // even rows, the odd lane the odd ones) and swap them by shuffle.
        constexpr int kRG = 8;
        static_assert(kCols % kRG == 0, "rotary row groups");
        const float2* rcs = reinterpret_cast<const float2*>(P.rope);
        const int pair = (n & 127) >> 1;
        float2 cs[kRG / 2];  // rows c0 + 2i + (lane & 1)
        auto load_cs = [&](int c0) {
#pragma unroll
          for (int i = 0; i < kRG / 2; ++i) {
            const int m = row0 + c0 + 2 * i + (lane & 1);
            cs[i] = m < P.M ? __ldg(rcs + size_t(m) * 64 + pair) : make_float2(1.f, 0.f);
          }
        };
        // Rotary embedding (the same for the whole problem): channel pair
        // (2p, 2p + 1) of the group turns by the angle of pair p of its row;
        // the partner channel is the neighbouring lane.  Even channel:
        // a cos - b sin, odd: a cos + b sin (b the partner's value).
        const float sgn = (n & 1) ? 1.f : -1.f;
        uint16_t* yp = reinterpret_cast<uint16_t*>(P.y) + size_t(row0) * P.ldy + n;
#pragma unroll
        for (int g = 0; g < kCols; g += kRG) {
          if (rcs) load_cs(g);
#pragma unroll
          for (int j = g / 2; j < (g + kRG) / 2; ++j) {
            const float lo = __uint_as_float(out[j] << 16), hi = __uint_as_float(out[j] & 0xFFFF0000u);
            float a0 = lo * (norm_inv[half * kCols + 2 * j] * w), a1 = hi * (norm_inv[half * kCols + 2 * j + 1] * w);
            if (rcs) {
              const float b0 = __shfl_xor_sync(0xffffffffu, a0, 1), b1 = __shfl_xor_sync(0xffffffffu, a1, 1);
              const float2 mine = cs[j - g / 2];  // row 2j + (lane & 1)
              const float2 other = make_float2(__shfl_xor_sync(0xffffffffu, mine.x, 1),
                                               __shfl_xor_sync(0xffffffffu, mine.y, 1));
              const float2 c0 = (lane & 1) ? other : mine, c1 = (lane & 1) ? mine : other;
              a0 = fmaf(a0, c0.x, sgn * b0 * c0.y);
              a1 = fmaf(a1, c1.x, sgn * b1 * c1.y);
            }
            out[j] = pack_bf16x2(a0, a1);
          }
#pragma unroll
          for (int c = g; c < g + kRG; ++c)
            if (c < rows) yp[size_t(c) * P.ldy] = uint16_t(out[c >> 1] >> ((c & 1) * 16));
        }
      } else if (EPI == 3 && n - r >= P.norm_col0 && n - r < P.norm_col1) {
        // RMS normalisation combined with an activation, a residual or a
        // gate on the same channels: fp32 throughout with one rounding.  The
        // per-token sums of squares need all four lane quarters, so the
        // accumulator is held (read twice from TMEM) until the normalised,
        // activated and combined values are stored; registers hold 32
        // columns at a time.
        constexpr int kChunk = 32;
        const int row0 = t.m_tile * C::kTokPair + half * kCols;
        const int rows = min(kCols, P.M - row0);
        bool ok_n = true;
#pragma unroll
        for (int c0 = 0; c0 < kCols; c0 += kChunk) {
          uint32_t v[kChunk];
          tmem_ld32(tmem + lane_off + ab * C::kDCols + half * kCols + c0, v);
          tmem_wait_ld();
          float sq[kChunk];
#pragma unroll
          for (int j = 0; j < kChunk; ++j) {
            const float y = fmaf(__uint_as_float(v[j]), sc, bi);
            sq[j] = y * y;
          }
          warp_reduce_scatter<kChunk>(sq, lane);  // token c0 + lane, this warp's 32 channels
          norm_part[(half * 4 + quarter) * kCols + c0 + lane] = sq[0];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&norm_bar[2 * half]));
        ok_n = mbar_wait(smem_u32(&norm_bar[2 * half]), norm_it & 1, lim, st);
        if (quarter == 0 && ok_n)
          for (int c = lane; c < kCols; c += 32) {
            const float tot = (norm_part[(half * 4 + 0) * kCols + c] + norm_part[(half * 4 + 1) * kCols + c]) +
                              (norm_part[(half * 4 + 2) * kCols + c] + norm_part[(half * 4 + 3) * kCols + c]);
            norm_inv[half * kCols + c] = rsqrtf(tot * (1.0f / 128.0f) + P.norm_eps);
          }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&norm_bar[2 * half + 1]));
        ok_n = mbar_wait(smem_u32(&norm_bar[2 * half + 1]), norm_it & 1, lim, st) && ok_n;
        ++norm_it;
        if (!__all_sync(0xffffffffu, ok_n)) break;
        const float w = P.norm_weight ? bf16_bits_to_float(reinterpret_cast<const uint16_t*>(P.norm_weight)[n]) : 1.f;
        const int act = P.act, act_col0 = P.act_col0, ld = P.ldy;  // c * ld < 2^28
        const uint16_t* res = reinterpret_cast<const uint16_t*>(P.residual);
        const uint16_t* rp = res ? res + size_t(row0) * P.ldy + n : nullptr;
        const float gt = P.gate ? bf16_bits_to_float(reinterpret_cast<const uint16_t*>(P.gate)[n]) : 1.f;
        uint32_t out[kCols / 2];  // the finished values, bf16x2; stored after the release
#pragma unroll
        for (int c0 = 0; c0 < kCols; c0 += 16) {
          uint32_t v[16];
          tmem_ld16(tmem + lane_off + ab * C::kDCols + half * kCols + c0, v);
          tmem_wait_ld();
#pragma unroll
          for (int g0 = 0; g0 < 16; g0 += 8) {
            float rv[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int c = c0 + g0 + j;
              rv[j] = (rp && c < rows) ? bf16_bits_to_float(rp[c * ld]) : 0.f;
            }
#pragma unroll
            for (int j = 0; j < 8; j += 2) {
              const int c = c0 + g0 + j;
              const float y0 = fmaf(__uint_as_float(v[g0 + j]), sc, bi) * (norm_inv[half * kCols + c] * w);
              const float y1 = fmaf(__uint_as_float(v[g0 + j + 1]), sc, bi) * (norm_inv[half * kCols + c + 1] * w);
              out[c / 2] = pack_bf16x2(fmaf(gt, apply_act(y0, act, n, act_col0), rv[j]),
                                       fmaf(gt, apply_act(y1, act, n, act_col0), rv[j + 1]));
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) T::arrive_leader(accempty_leader0 + ab * 8);
        uint16_t* yp = reinterpret_cast<uint16_t*>(P.y) + size_t(row0) * P.ldy + n;
#pragma unroll
        for (int c = 0; c < kCols; ++c)
          if (c < rows) yp[size_t(c) * P.ldy] = uint16_t(out[c >> 1] >> ((c & 1) * 16));
      } else {
        // Residual and gate (with or without the activation): fp32 until the
        // store, everything after the release.
        float f[kCols];
#pragma unroll
        for (int c0 = 0; c0 < kCols; c0 += 32) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_off + ab * C::kDCols + half * kCols + c0, v);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) f[c0 + j] = fmaf(__uint_as_float(v[j]), sc, bi);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) T::arrive_leader(accempty_leader0 + ab * 8);
        const int row0 = t.m_tile * C::kTokPair + half * kCols;
        const int rows = min(kCols, P.M - row0);
        const int act = P.act, act_col0 = P.act_col0, ld = P.ldy;  // c * ld < 2^28
        uint16_t* yp = reinterpret_cast<uint16_t*>(P.y) + size_t(row0) * P.ldy + n;
        const uint16_t* res = reinterpret_cast<const uint16_t*>(P.residual);
        const uint16_t* rp = res ? res + size_t(row0) * P.ldy + n : nullptr;
        const float gt = P.gate ? bf16_bits_to_float(reinterpret_cast<const uint16_t*>(P.gate)[n]) : 1.f;
#pragma unroll
        for (int c = 0; c < kCols; ++c) f[c] = apply_act(f[c], act, n, act_col0);
#pragma unroll
        for (int c0 = 0; c0 < kCols; c0 += 8) {
          // The residual may be y itself: a group's loads all go out before
          // its stores (an element's load precedes its own store; the others
          // are different addresses), so they are not serialised one by one.
          float rv[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) rv[j] = (rp && c0 + j < rows) ? bf16_bits_to_float(rp[(c0 + j) * ld]) : 0.f;
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if (c0 + j < rows) yp[(c0 + j) * ld] = __bfloat16_as_ushort(__float2bfloat16_rn(fmaf(gt, f[c0 + j], rv[j])));
        }
      }
    }
  }

  // ------------------------------------------------------ teardown
  // No CTA may leave while the pair's MMAs or remote arrivals still touch it.
  tc_fence_before();
  T::sync_all();
  if (warp == 1) {
    tc_fence_after();
    T::dealloc(tmem, C::kTmemCols);
  }
}

// Pair tiles run as clusters of two CTAs; single-CTA tiles without clusters.
template <int TOK, int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Cfg2<TOK, true, EPI>::kThreads, 1)
    ternary_pair_kernel(const __grid_constant__ Batch batch) {
  tile_kernel_body<TOK, true, EPI>(batch);
}
template <int TOK, int EPI>
__global__ void __launch_bounds__(Cfg2<TOK, false, EPI>::kThreads, 1)
    ternary_tile_kernel(const __grid_constant__ Batch batch) {
  tile_kernel_body<TOK, false, EPI>(batch);
}
template <int TOK, bool PAIR, int EPI>
constexpr auto tile_kernel() {
  if constexpr (PAIR) return ternary_pair_kernel<TOK, EPI>;
  else return ternary_tile_kernel<TOK, EPI>;
}

template <int TOK, bool PAIR, int EPI>
static cudaError_t configure_tile() {
  static unsigned long long configured = 0;  // one bit per device ordinal
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64) return cudaErrorInvalidDevice;
  if (!(__atomic_load_n(&configured, __ATOMIC_ACQUIRE) & (1ull << dev))) {
    e = cudaFuncSetAttribute(tile_kernel<TOK, PAIR, EPI>(), cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Cfg2<TOK, PAIR, EPI>::kSmemBytes);
    if (e != cudaSuccess) return e;
    __atomic_fetch_or(&configured, 1ull << dev, __ATOMIC_RELEASE);
  }
  return cudaSuccess;
}

// `ctas_or_pairs` CTAs (one-CTA tiles) or clusters of two (pair tiles).
template <int TOK, bool PAIR, int EPI>
static cudaError_t launch_tile(const Batch& batch, int ctas_or_pairs, cudaStream_t stream) {
  using C = Cfg2<TOK, PAIR, EPI>;
  cudaError_t e = configure_tile<TOK, PAIR, EPI>();
  if (e != cudaSuccess) return e;
  return launch_pdl(tile_kernel<TOK, PAIR, EPI>(), dim3(C::kCtas * ctas_or_pairs), dim3(C::kThreads), C::kSmemBytes,
                    stream, 1, batch);
}

cudaError_t launch_ternary_mma2(int tok, bool pair, const Batch& batch, int ctas_or_pairs, cudaStream_t stream) {
  int epi = 0;
  for (int i = 0; i < batch.count; ++i) {
    if (batch.p[i].norm_col0 != batch.p[i].norm_col1) epi = 3;
    else if (batch.p[i].residual || batch.p[i].gate) epi = std::max(epi, 2);
    else if (batch.p[i].act != kActNone) epi = std::max(epi, 1);
  }
  if (pair && tok == 256) {
    if (epi == 3) return launch_tile<256, true, 3>(batch, ctas_or_pairs, stream);
    if (epi == 2) return launch_tile<256, true, 2>(batch, ctas_or_pairs, stream);
    if (epi == 1) return launch_tile<256, true, 1>(batch, ctas_or_pairs, stream);
    return launch_tile<256, true, 0>(batch, ctas_or_pairs, stream);
  }
  if (!pair && tok == 64) {
    if (epi == 3) return launch_tile<64, false, 3>(batch, ctas_or_pairs, stream);
    if (epi == 2) return launch_tile<64, false, 2>(batch, ctas_or_pairs, stream);
    if (epi == 1) return launch_tile<64, false, 1>(batch, ctas_or_pairs, stream);
    return launch_tile<64, false, 0>(batch, ctas_or_pairs, stream);
  }
  return cudaErrorInvalidValue;
}

int x_chunks_2sm(int tok) { return tok == 256 ? Cfg2<256, true>::kChunks : Cfg2<64, false>::kChunks; }

int max_active_clusters_2sm() {
  if (configure_tile<256, true, 0>() != cudaSuccess || configure_tile<256, true, 1>() != cudaSuccess ||
      configure_tile<256, true, 2>() != cudaSuccess || configure_tile<256, true, 3>() != cudaSuccess ||
      configure_tile<64, false, 0>() != cudaSuccess || configure_tile<64, false, 1>() != cudaSuccess ||
      configure_tile<64, false, 2>() != cudaSuccess || configure_tile<64, false, 3>() != cudaSuccess)
    return 0;
  int n = 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * 148);
  cfg.blockDim = dim3(Cfg2<256, true>::kThreads);
  cfg.dynamicSmemBytes = Cfg2<256, true>::kSmemBytes;
  if (cudaOccupancyMaxActiveClusters(&n, ternary_pair_kernel<256, 0>, &cfg) != cudaSuccess) return 0;
  return n;
}

}  // namespace tern
