// ternary_gemv.cu -- the small-M (M <= 16) ternary linear y = (x . T^T) * s + b,
// bound by the HBM stream of packed codes.
//
// Page "1.58-bit FLUX" (arXiv 2412.18653): Section 1 (weights in {-1,0,+1},
// stored as 2-bit signed integers), Section 4 (activations stay 16-bit); the
// adaLN modulation layers of every block are such products with one token
// row per image.
//
// With a handful of tokens every code byte is used by at most 16 multiply-
// adds, so the kernel's job is to stream the N*K/4 code bytes at HBM speed and
// spend as few instructions per weight as possible.  The tensor cores of
// tcgen05 read their operands as bf16 from shared memory or TMEM, which caps
// them at about 64 weights per SM clock -- below the ~90 weights per clock
// that HBM delivers as 2-bit codes.  So this kernel expands codes in
// registers and feeds the warp-level tensor-core instruction (mma.sync
// m16n8k16, bf16 in, fp32 accumulate), whose A operand comes from registers:
//   * A = 16 channels x 16 k of weights.  A code (two's complement: +1 = 01,
//     -1 = 11, 0 = 00) shifted so that its two bits land on bits 14 and 15 of
//     a bf16 is the bf16 value 2t exactly (0x4000 = 2, 0xC000 = -2, 0 = 0),
//     so one shift and one AND expand a (k, k+1) pair; the sum is halved at
//     the end (exact).
//   * The k order inside each 64-k chunk is permuted so that the lane that
//     loads code word c of a row (one 32-bit shared-memory load, the 32 lanes
//     of a warp reading 128 contiguous bytes) holds exactly its A-fragment
//     pairs: MMA q (q = 0..3) of the chunk takes pairs 2q and 2q+1 of every
//     word, i.e. k = 16c + 4q .. 16c + 4q + 3 for the lane with c = lane % 4,
//     and B = x is read in the same permuted order (8 contiguous bytes).
//   * B = x^T for 8 tokens per n8 block (NT blocks: M <= 8 NT).
// One CTA owns 128 channels (one tile-interleaved slab: each 64-k chunk is a
// contiguous 2 KiB block) over a range of k.  Its eight consumer warps own 16
// channels each and take every chunk of their rows.  A producer lane streams
// stages of sixteen chunks (M <= 8; eight for M <= 16) into a four- (six-)
// stage ring with two copies per stage: one bulk copy of the codes (32 or 16
// KiB) and one 3-D TMA box of the matching x rows (k-in-chunk x token x chunk,
// 128-byte swizzle, 8 NT token rows; rows past M read as zero, and their MMA
// columns are never stored).  When there
// are too few slabs to fill the SMs, the k range is split over a cluster of
// CTAs, whose partial sums are added in rank order through distributed shared
// memory (deterministic, no global scratch).  No TMA multicast is used.
#include "internal.h"
#include "kernel_common.cuh"
#include "ptx.cuh"

namespace tern {

namespace {

template <int NT>
struct GemvCfg {
  static constexpr int kGroups = 8;                  // 16-channel groups per 128-channel slab
  // One consumer warp per group: it takes every chunk of its 16 rows, so no
  // warp ever waits for another (two warps per SM sub-partition already keep
  // the expansion and the MMAs at full rate).
  static constexpr int kWarps = kGroups;
  static constexpr int kThreads = (kWarps + 1) * 32;  // + one producer warp
  // 64-k chunks per stage: 16 (32 KiB of codes) where shared memory allows,
  // so the per-stage handshake is paid half as often.
  static constexpr int kChunks = NT == 1 ? 16 : 8;
  static constexpr int kStages = NT == 1 ? 4 : 6;
  static constexpr int kCodeBytes = kChunks * 2048;
  static constexpr int kXChunk = 8 * NT * 128;          // 8 NT token rows x 64 bf16 (rows >= M read as 0)
  static constexpr int kXBytes = kChunks * kXChunk;
  static constexpr int kStageBytes = kCodeBytes + kXBytes;
  static constexpr int kSmemBytes = kStages * kStageBytes + 1024;
  static_assert(kStageBytes % 1024 == 0 && kCodeBytes % 1024 == 0, "swizzled x boxes stay 1024-aligned");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};


__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

}  // namespace

// Grid (splits, G), cluster (splits, 1, 1).  Work unit u = one 128-channel
// slab of one problem of the batch (u < total_units); the CTAs with
// blockIdx.y = g take units g, g + G, ...  (persistent: the producer streams
// the next unit's codes while the consumers finish the current one).
// blockIdx.x, the rank in the cluster, picks the k range of every unit
// (chunks_per_split 64-k chunks).  The x tensor map is 3-D {64 k, M tokens,
// K / 64 chunks} with box {64, min(M, 8 NT), kChunks}.
// The fields of a batch problem that the GEMV reads at every unit, copied
// once to shared memory: reading them from the parameter block with a runtime
// problem index measured ~0.5 us per unit boundary (each CTA walks several
// units of a batch), shared-memory reads a few cycles.
struct GemvProb {
  const uint8_t* packed;
  const float* scales;
  const uint16_t* bias;
  __nv_bfloat16* y;
  int unit_begin, M, N, K, chunks_per_split;
  int act, act_col0;  // epilogue activation and its first column
  int ldy;            // elements between rows of y and of the residual
  const uint16_t* residual;  // [M, N] or null
  const uint16_t* gate;      // [N] or null
};

__device__ __forceinline__ int unit_problem(const GemvProb* probs, int count, int u, int* slab) {
  int pi = 0;
  while (pi + 1 < count && u >= probs[pi + 1].unit_begin) ++pi;
  *slab = u - probs[pi].unit_begin;
  return pi;
}

template <int NT>
__global__ void __launch_bounds__(GemvCfg<NT>::kThreads, 1)
    ternary_gemv_kernel(const __grid_constant__ Batch batch) {
  using C = GemvCfg<NT>;
  constexpr int S = C::kStages;

  __shared__ __align__(8) uint64_t full_bar[S];   // codes and x of stage s landed
  __shared__ __align__(8) uint64_t empty_bar[S];  // all consumer warps are done with stage s
  __shared__ __align__(16) float part[C::kWarps * 32 * NT * 4];  // this CTA's sums, for rank 0
  __shared__ GemvProb probs[kMaxProblems];
  extern __shared__ uint8_t dyn_smem[];

  const uint64_t lim = batch.wait_limit_ns;
  unsigned int* const st = batch.status;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t smem_base = (smem_u32(dyn_smem) + 1023u) & ~1023u;
  const uint8_t* const smem_gen = dyn_smem + (smem_base - smem_u32(dyn_smem));
  const int splits = gridDim.x, rank = blockIdx.x;
  const int u0 = blockIdx.y, ustep = gridDim.y, units = batch.total_units;
  // With K split over a cluster the producer only joins the per-unit cluster
  // rendezvous after its whole stream, so each CTA must own a single unit.
  // (The host never launches otherwise; the test is uniform over the grid,
  // so every CTA leaves here and the host reads TERN_ERR_LAUNCH_CONFIG.)
  if (splits > 1 && ustep < units) {
    pdl_wait();
    if (threadIdx.x == 0) atomicOr(st, kStatusLaunchConfig);
    return;
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), C::kWarps);
    }
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (threadIdx.x < batch.count) {
    const Problem& q = batch.p[threadIdx.x];
    GemvProb& g = probs[threadIdx.x];
    g.packed = q.packed;
    g.scales = q.scales;
    g.bias = reinterpret_cast<const uint16_t*>(q.bias);
    g.y = q.y;
    g.unit_begin = q.unit_begin;
    g.M = q.M;
    g.N = q.N;
    g.K = q.K;
    g.chunks_per_split = q.chunks_per_split;
    g.act = q.act;
    g.act_col0 = q.act_col0;
    g.ldy = q.ldy;
    g.residual = reinterpret_cast<const uint16_t*>(q.residual);
    g.gate = reinterpret_cast<const uint16_t*>(q.gate);
  }
  const int nprob = batch.count;
  __syncthreads();
  // The previous kernel of the stream may still be running (programmatic
  // dependent launch): the producer first asks L2 for the codes of its first
  // stages (a hint: a write by that kernel still reaches the readers through
  // L2), then every thread waits for it before touching global memory.
  if (warp == C::kWarps && lane == 0 && u0 < units) {
    int slab;
    const GemvProb& P = probs[unit_problem(probs, nprob, u0, &slab)];
    const int kc_total = P.K >> 6;
    const int kc0 = rank * P.chunks_per_split;
    const int nk = max(0, min(kc_total, kc0 + P.chunks_per_split) - kc0);
    if (nk > 0)
      prefetch_l2_bulk(P.packed + (size_t(slab) * kc_total + kc0) * 2048, uint32_t(min(nk, S * C::kChunks)) * 2048u);
  }
  pdl_wait();
  pdl_trigger();
  const int grp = warp;  // 16-channel group of a consumer warp

  if (warp == C::kWarps) {
    // ------------------------------------------------------ producer
    if (lane == 0)
      for (int pi = 0; pi < batch.count; ++pi) prefetch_tensormap(&batch.p[pi].tmap_x);
    int it = 0;
    bool ok = true;
    for (int u = u0; u < units && ok; u += ustep) {
      int slab;
      const int pi = unit_problem(probs, nprob, u, &slab);
      const GemvProb& P = probs[pi];
      const int kc_total = P.K >> 6;
      const int kc0 = rank * P.chunks_per_split;
      const int nk = max(0, min(kc_total, kc0 + P.chunks_per_split) - kc0);
      const uint8_t* codes = P.packed + (size_t(slab) * kc_total + kc0) * 2048;
      for (int i = 0; i * C::kChunks < nk; ++i, ++it) {
        const int s = it % S;
        if (it >= S &&
            !__shfl_sync(0xffffffffu, mbar_wait(smem_u32(&empty_bar[s]), ((it / S) & 1) ^ 1, lim, st), 0)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          const int nch = min(C::kChunks, nk - i * C::kChunks);
          const uint32_t stage = smem_base + s * C::kStageBytes;
          const uint32_t fb = smem_u32(&full_bar[s]);
          mbar_arrive_expect_tx(fb, nch * 2048 + C::kXBytes);
          tma_load_bulk(stage, codes + size_t(i) * C::kCodeBytes, nch * 2048, fb);
          tma_load_3d(stage + C::kCodeBytes, &batch.p[pi].tmap_x, 0, 0, kc0 + i * C::kChunks, fb);
        }
        __syncwarp();
      }
    }
    // No copy may still be landing in shared memory when the CTA exits.
    for (int i = max(0, it - S); i < it; ++i) mbar_wait(smem_u32(&full_bar[i % S]), (i / S) & 1, lim, st);
  }

  // Consumers walk the same units; all threads (producer included) meet at
  // the per-unit cluster rendezvous when K is split.
  const int g = lane >> 2, c = lane & 3;
  // This lane's two 16-byte x pieces of a chunk: row g (and 8 + g, ... for
  // the next n8 blocks), k = 16c .. 16c + 15, XOR-swizzled by the row (each
  // chunk of the box is 8 NT rows of 128 bytes, so the swizzle row is g).
  const uint32_t xoff_a = uint32_t(g * 128) + ((uint32_t(2 * c) ^ uint32_t(g)) << 4);
  const uint32_t xoff_b = uint32_t(g * 128) + ((uint32_t(2 * c + 1) ^ uint32_t(g)) << 4);
  int it = 0;
  bool ok = true;
  for (int u = u0; u < units; u += ustep) {
    int slab;
    const GemvProb& P = probs[unit_problem(probs, nprob, u, &slab)];
    float d[NT][4];  // D fragments: channels (g, g + 8) x tokens (2c, 2c + 1) of each n8 block
#pragma unroll
    for (int nb = 0; nb < NT; ++nb)
#pragma unroll
      for (int e = 0; e < 4; ++e) d[nb][e] = 0.f;
    const int n_out = slab * 128 + grp * 16 + g;
    // N % 16 == 0: a 16-channel group is wholly inside N or wholly padding
    // (zero codes; its sums are computed like the others and not stored).
    const bool live = slab * 128 + grp * 16 < P.N;
    if (warp < C::kWarps) {
      // Scale and bias of this lane's two output channels, loaded now and used
      // after the stream (only rank 0 stores).
      float s0 = 0.f, s1 = 0.f, b0 = 0.f, b1 = 0.f, g0 = 1.f, g1 = 1.f;
      if (rank == 0 && live) {
        s0 = 0.5f * P.scales[n_out];  // codes expand to 2t
        s1 = 0.5f * P.scales[n_out + 8];
        const uint16_t* bias = P.bias;
        if (bias) {
          b0 = bf16_bits_to_float(bias[n_out]);
          b1 = bf16_bits_to_float(bias[n_out + 8]);
        }
        if (P.gate) {
          g0 = bf16_bits_to_float(P.gate[n_out]);
          g1 = bf16_bits_to_float(P.gate[n_out + 8]);
        }
      }
      const int kc_total = P.K >> 6;
      const int nk = max(0, min(kc_total, (rank + 1) * P.chunks_per_split) - rank * P.chunks_per_split);
      float acc[4][NT][4];  // one accumulator per MMA position q: four independent chains
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int nb = 0; nb < NT; ++nb)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[q][nb][e] = 0.f;
      for (int i = 0; ok && i * C::kChunks < nk; ++i, ++it) {
        const int s = it % S;
        if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&full_bar[s]), (it / S) & 1, lim, st))) {
          ok = false;
          break;
        }
        const int nch = min(C::kChunks, nk - i * C::kChunks);
        // Word c of rows 16 grp + g and 16 grp + g + 8 of each chunk: 128
        // contiguous bytes per warp load.
        const uint32_t* cw =
            reinterpret_cast<const uint32_t*>(smem_gen + s * C::kStageBytes) + grp * 64 + lane;
        const uint8_t* xgen = smem_gen + s * C::kStageBytes + C::kCodeBytes;
        auto chunk = [&](int j) {
          const uint32_t a = cw[j * 512], b = cw[j * 512 + 32];
#pragma unroll
          for (int nb = 0; nb < NT; ++nb) {
            // Every lane loads its x piece: rows past M are zeros that the TMA
            // box filled in, and plain (non-volatile, unpredicated) loads let
            // the compiler schedule them ahead of the MMAs (measured 7 %
            // faster at M = 16 than skipping the absent rows behind a branch).
            const uint4 xa = *reinterpret_cast<const uint4*>(xgen + j * C::kXChunk + nb * 1024 + xoff_a);
            const uint4 xb = *reinterpret_cast<const uint4*>(xgen + j * C::kXChunk + nb * 1024 + xoff_b);
            mma_16816(acc[0][nb], code_pair_2t<0>(a), code_pair_2t<0>(b), code_pair_2t<1>(a), code_pair_2t<1>(b),
                      xa.x, xa.y);
            mma_16816(acc[1][nb], code_pair_2t<2>(a), code_pair_2t<2>(b), code_pair_2t<3>(a), code_pair_2t<3>(b),
                      xa.z, xa.w);
            mma_16816(acc[2][nb], code_pair_2t<4>(a), code_pair_2t<4>(b), code_pair_2t<5>(a), code_pair_2t<5>(b),
                      xb.x, xb.y);
            mma_16816(acc[3][nb], code_pair_2t<6>(a), code_pair_2t<6>(b), code_pair_2t<7>(a), code_pair_2t<7>(b),
                      xb.z, xb.w);
          }
        };
        if (nch == C::kChunks) {  // every stage but a row's last: no bounds tests
#pragma unroll
          for (int j = 0; j < C::kChunks; ++j) chunk(j);
        } else {
#pragma unroll 1
          for (int j = 0; j < nch; ++j) chunk(j);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&empty_bar[s]));
      }
#pragma unroll
      for (int nb = 0; nb < NT; ++nb)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          d[nb][e] = (acc[0][nb][e] + acc[1][nb][e]) + (acc[2][nb][e] + acc[3][nb][e]);
      if (splits > 1) {
        float* mine = &part[(grp * 32 + lane) * NT * 4];
#pragma unroll
        for (int nb = 0; nb < NT; ++nb)
#pragma unroll
          for (int e = 0; e < 4; ++e) mine[nb * 4 + e] = d[nb][e];  // this CTA's sums, for rank 0
      }
      if (splits > 1) cluster_sync();  // every rank's partial sums are in its shared memory
      if (rank == 0) {
        if (splits > 1) {
          const uint32_t mine = smem_u32(&part[(grp * 32 + lane) * NT * 4]);
          for (int r = 1; r < splits; ++r)  // rank order: deterministic
#pragma unroll
            for (int nb = 0; nb < NT; ++nb)
#pragma unroll
              for (int e = 0; e < 4; ++e)
                d[nb][e] += ld_shared_cluster_f32(mapa_shared(mine + uint32_t(nb * 4 + e) * 4, uint32_t(r)));
        }
        // This lane's outputs: tokens t0 = 8 nb + 2c (+1), channels n_out
        // (+8).  The residual may be y itself, so every residual value is
        // read before the first store.
        float rv[NT][4];
#pragma unroll
        for (int nb = 0; nb < NT; ++nb)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int t = 8 * nb + 2 * c + (e & 1);
            const int nn = n_out + (e >> 1) * 8;
            rv[nb][e] = (P.residual && live && t < P.M) ? bf16_bits_to_float(P.residual[size_t(t) * P.ldy + nn]) : 0.f;
          }
#pragma unroll
        for (int nb = 0; nb < NT; ++nb)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int t = 8 * nb + 2 * c + (e & 1);
            const int nn = n_out + (e >> 1) * 8;
            if (live && t < P.M) {
              const float v = fmaf(d[nb][e], e >> 1 ? s1 : s0, e >> 1 ? b1 : b0);
              const float a = apply_act(v, P.act, nn, P.act_col0);
              P.y[size_t(t) * P.ldy + nn] = __float2bfloat16_rn(fmaf(e >> 1 ? g1 : g0, a, rv[nb][e]));
            }
          }
      }
      if (splits > 1) cluster_sync_relaxed();  // rank 0 has read every partial before they change
    } else if (splits > 1) {
      cluster_sync();  // the producer warp takes part in every cluster rendezvous
      cluster_sync_relaxed();
    }
  }
}

// Grid (splits, ctas): with splits > 1 one CTA per unit (ctas = units).
template <int NT>
static cudaError_t launch_nt(const Batch& batch, int splits, int ctas, cudaStream_t stream) {
  using C = GemvCfg<NT>;
  static unsigned long long configured = 0;  // one bit per device ordinal
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64) return cudaErrorInvalidDevice;
  if (!(__atomic_load_n(&configured, __ATOMIC_ACQUIRE) & (1ull << dev))) {
    e = cudaFuncSetAttribute(ternary_gemv_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    __atomic_fetch_or(&configured, 1ull << dev, __ATOMIC_RELEASE);
  }
  return launch_pdl(ternary_gemv_kernel<NT>, dim3(unsigned(splits), unsigned(ctas), 1), dim3(C::kThreads),
                    C::kSmemBytes, stream, unsigned(splits), batch);
}

cudaError_t launch_ternary_gemv(int nt, const Batch& batch, int splits, int ctas, cudaStream_t stream) {
  if (splits < 1 || splits > 8 || ctas < 1 || ctas > 65535 || (splits > 1 && ctas < batch.total_units))
    return cudaErrorInvalidValue;
  switch (nt) {
    case 1: return launch_nt<1>(batch, splits, ctas, stream);
    case 2: return launch_nt<2>(batch, splits, ctas, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace tern
