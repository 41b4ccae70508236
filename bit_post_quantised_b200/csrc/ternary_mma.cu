// ternary_mma.cu -- the ternary linear layer y = (x . T^T) * s + b on the
// 5th-generation tensor cores (tcgen05) of sm_100a.
//
// Page "1.58-bit FLUX" (arXiv 2412.18653): Section 1 (weights in {-1,0,+1},
// stored as 2-bit signed integers), Section 4 (activations stay 16-bit).
//
// One CTA computes a 128-channel x TOK-token tile of y (transposed in TMEM):
//   D[channel, token] = sum_k T[channel, k] * x[token, k]
// with UMMA M = 128 (channels), N = TOK (tokens), K = 16 per instruction.
//   * warp 0 (one lane): TMA producer.  Per 64-wide k stage it issues a tiled
//     2-D copy of the x tile (TOK rows x 128 bytes, 128-byte swizzle) and an
//     untiled 2 KiB bulk copy of the codes of 128 channels x 64 k, which the
//     tile-interleaved layout keeps contiguous.  Both complete on one mbarrier.
//   * decoder warps: one thread per channel row (two per row with 8 warps)
//     reads its 16 (8) code bytes from shared memory, expands them in
//     registers to bf16 (+-1 and 0 are exact), and writes them with
//     tcgen05.st straight into a TMEM slot, which is the UMMA A operand.
//     Decoded weights therefore never touch shared memory.
//   * warp 1 (one lane): issues tcgen05.mma (A from TMEM, B = x from shared
//     memory) into the fp32 accumulator in TMEM and commits to mbarriers that
//     free the shared-memory stage and the TMEM slot.
//   * epilogue (decoder warps): tcgen05.ld of the accumulator, one channel per
//     thread, y = acc * s + b, round to bf16, store.  When K is split across
//     CTAs (few tokens), each split stores fp32 partials and the last CTA of a
//     tile to arrive sums them in split order and writes y.
// No TMA multicast is used anywhere, so the kernel is legal on every GPU of a
// multi-GPU node.
#include "internal.h"
#include "kernel_common.cuh"
#include "ptx.cuh"

namespace tern {

// ------------------------------------------------------------------ kernel
template <int TOK>
__global__ void __launch_bounds__(TileCfg<TOK>::kThreads, 1)
    ternary_mma_kernel(const __grid_constant__ Batch batch) {
  using C = TileCfg<TOK>;
  constexpr int S = C::kStages;
  constexpr int A = C::kASlots;
  constexpr int kDecThreads = C::kDecWarps * 32;
  constexpr int kHalves = C::kDecWarps / 4;  // decoder warps per TMEM lane quarter

  __shared__ __align__(8) uint64_t full_bar[S];
  __shared__ __align__(8) uint64_t empty_bar[S];
  __shared__ __align__(8) uint64_t afull_bar[A];
  __shared__ __align__(8) uint64_t aempty_bar[A];
  __shared__ __align__(8) uint64_t acc_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int last_sh;
  extern __shared__ uint8_t dyn_smem[];

  // ---- which problem and tile
  const int cta = blockIdx.x;
  int pi = 0;
  while (pi + 1 < batch.count && cta >= batch.p[pi + 1].unit_begin) ++pi;
  const Problem& P = batch.p[pi];
  const int local = cta - P.unit_begin;
  const int tiles = P.n_tiles * P.m_tiles;
  const int split = local / tiles;
  const int tile = local - split * tiles;
  const int m_tile = tile / P.n_tiles;
  const int n_tile = tile - m_tile * P.n_tiles;
  const int kc_total = P.K >> 6;
  const int kc_begin = split * P.chunks_per_split;
  const int kc_end = min(kc_total, kc_begin + P.chunks_per_split);
  const int nk = kc_end - kc_begin;
  const int row0 = m_tile * TOK;
  const uint64_t lim = batch.wait_limit_ns;
  unsigned int* const st = batch.status;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t smem_base = (smem_u32(dyn_smem) + 1023u) & ~1023u;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    for (int a = 0; a < A; ++a) {
      mbar_init(smem_u32(&afull_bar[a]), kDecThreads);
      mbar_init(smem_u32(&aempty_bar[a]), 1);
    }
    mbar_init(smem_u32(&acc_bar), 1);
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) prefetch_tensormap(&P.tmap_x);
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_base_sh), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  pdl_wait();
  pdl_trigger();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint8_t* codes = P.packed + (size_t(n_tile) * kc_total + kc_begin) * 2048;
      int issued = 0;
      for (int i = 0; i < nk; ++i) {
        const int s = i % S;
        if (!mbar_wait(smem_u32(&empty_bar[s]), ((i / S) & 1) ^ 1, lim, st)) break;
        const uint32_t stage = smem_base + s * C::kStageBytes;
        const uint32_t fb = smem_u32(&full_bar[s]);
        mbar_arrive_expect_tx(fb, C::kStageBytes);
        tma_load_2d(stage, &P.tmap_x, (kc_begin + i) * 64, row0, fb);
        tma_load_bulk(stage + C::kXBytes, codes + size_t(i) * 2048, C::kCBytes, fb);
        ++issued;
      }
      // No copy may still be landing in shared memory when the CTA exits.
      for (int i = issued > S ? issued - S : 0; i < issued; ++i)
        mbar_wait(smem_u32(&full_bar[i % S]), (i / S) & 1, lim, st);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------ MMA issuer
    if (lane == 0) {
      for (int i = 0; i < nk; ++i) {
        const int s = i % S, a = i % A;
        if (!mbar_wait(smem_u32(&full_bar[s]), (i / S) & 1, lim, st)) break;
        if (!mbar_wait(smem_u32(&afull_bar[a]), (i / A) & 1, lim, st)) break;
        tc_fence_after();
        const uint32_t xaddr = smem_base + s * C::kStageBytes;
        const uint32_t a_tmem = tmem + C::kDCols + a * C::kACols;
#pragma unroll
        for (int j = 0; j < C::kBK / 16; ++j)
          mma_bf16_ts(tmem, a_tmem + j * 8, sw128_kmajor_desc(xaddr + j * 32), C::kIdesc,
                      (i | j) != 0);
        mma_commit(smem_u32(&empty_bar[s]));
        mma_commit(smem_u32(&aempty_bar[a]));
      }
      mma_commit(smem_u32(&acc_bar));
      // Every MMA this thread issued is complete before TMEM is released.
      mbar_wait(smem_u32(&acc_bar), 0, lim, st);
    }
  } else {
    // ------------------------------------------------------ decoders
    const int dw = warp - 2;
    const int quarter = warp & 3;  // TMEM lanes this warp may touch
    const int half = dw >> 2;
    const int r = quarter * 32 + lane;  // channel row inside the tile
    const uint32_t lane_off = uint32_t(quarter * 32) << 16;
    for (int i = 0; i < nk; ++i) {
      const int s = i % S, a = i % A;
      if (!mbar_wait(smem_u32(&full_bar[s]), (i / S) & 1, lim, st)) break;
      if (!mbar_wait(smem_u32(&aempty_bar[a]), ((i / A) & 1) ^ 1, lim, st)) break;
      tc_fence_after();
      const uint8_t* cp = dyn_smem + (smem_base - smem_u32(dyn_smem)) + s * C::kStageBytes +
                          C::kXBytes + r * 16;
      const uint32_t dst = tmem + lane_off + C::kDCols + a * C::kACols;
      if constexpr (kHalves == 1) {
        const uint4 v = *reinterpret_cast<const uint4*>(cp);
        uint32_t t[32];
        decode_word(v.x, t + 0);
        decode_word(v.y, t + 8);
        decode_word(v.z, t + 16);
        decode_word(v.w, t + 24);
        tmem_st32(dst, t);
      } else {
        const uint2 v = *reinterpret_cast<const uint2*>(cp + half * 8);
        uint32_t t[16];
        decode_word(v.x, t + 0);
        decode_word(v.y, t + 8);
        tmem_st16(dst + half * 16, t);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(&afull_bar[a]));
    }

    // ------------------------------------------------------ epilogue
    mbar_wait(smem_u32(&acc_bar), 0, lim, st);
    tc_fence_after();
    constexpr int kColsPerHalf = (TOK / kHalves) < 16 ? 16 : (TOK / kHalves);
    const int col_begin = half * kColsPerHalf;
    const int col_end = min(TOK, col_begin + kColsPerHalf);
    const int n = n_tile * 128 + r;
    const int M = P.M, N = P.N;
    const size_t ld = size_t(P.ldy);  // elements between rows of y and of the residual
    const bool live = n < N;  // channels past N (the last slab's zero-code rows) are not stored
    const uint16_t* res = reinterpret_cast<const uint16_t*>(P.residual);
    if (P.splits == 1) {
      const float sc = live ? P.scales[n] : 0.f;
      const float gt = P.gate && live ? bf16_bits_to_float(reinterpret_cast<const uint16_t*>(P.gate)[n]) : 1.f;
      const float bi = P.bias && live ? bf16_bits_to_float(reinterpret_cast<const uint16_t*>(P.bias)[n]) : 0.f;
      for (int c0 = col_begin; c0 < col_end; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(tmem + lane_off + c0, v);
        tmem_wait_ld();
        float rv[16];  // residual loads of the group first (it may be y itself)
#pragma unroll
        for (int j = 0; j < 16; ++j)
          rv[j] = (res && live && row0 + c0 + j < M) ? bf16_bits_to_float(res[size_t(row0 + c0 + j) * ld + n]) : 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int m = row0 + c0 + j;
          if (live && m < M)
            P.y[size_t(m) * ld + n] = __float2bfloat16_rn(
                fmaf(gt, apply_act(fmaf(__uint_as_float(v[j]), sc, bi), P.act, n, P.act_col0), rv[j]));
        }
      }
    } else {
      float* part = P.ws + (size_t(split) * tiles + tile) * TOK * 128;
      for (int c0 = col_begin; c0 < col_end; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(tmem + lane_off + c0, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) __stcg(part + (c0 + j) * 128 + r, __uint_as_float(v[j]));
      }
      __threadfence();
      named_barrier_sync(1, kDecThreads);
      if (dw == 0 && lane == 0) {
        const int prev = atomicAdd(P.counters + tile, 1);
        last_sh = (prev == P.splits - 1);
      }
      named_barrier_sync(1, kDecThreads);
      if (last_sh) {
        __threadfence();
        if (live) {
          const float sc = P.scales[n];
          const float bi =
              P.bias ? bf16_bits_to_float(reinterpret_cast<const uint16_t*>(P.bias)[n]) : 0.f;
          const float gt = P.gate ? bf16_bits_to_float(reinterpret_cast<const uint16_t*>(P.gate)[n]) : 1.f;
          for (int c = col_begin; c < col_end; ++c) {
            const int m = row0 + c;
            if (m >= M) break;
            float acc = 0.f;
            for (int sp = 0; sp < P.splits; ++sp)
              acc += __ldcg(P.ws + ((size_t(sp) * tiles + tile) * TOK + c) * 128 + r);
            P.y[size_t(m) * ld + n] = __float2bfloat16_rn(
                epilogue_value(fmaf(acc, sc, bi), P.act, n, P.act_col0, res, size_t(m) * ld + n, gt));
          }
        }
        if (dw == 0 && lane == 0) P.counters[tile] = 0;  // ready for the next launch
      }
    }
  }

  // ------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int TOK>
static cudaError_t launch_tok(const Batch& batch, cudaStream_t stream) {
  using C = TileCfg<TOK>;
  static unsigned long long configured = 0;  // one bit per device ordinal
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64) return cudaErrorInvalidDevice;
  if (!(__atomic_load_n(&configured, __ATOMIC_ACQUIRE) & (1ull << dev))) {
    e = cudaFuncSetAttribute(ternary_mma_kernel<TOK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::kSmemBytes);
    if (e != cudaSuccess) return e;
    __atomic_fetch_or(&configured, 1ull << dev, __ATOMIC_RELEASE);
  }
  return launch_pdl(ternary_mma_kernel<TOK>, dim3(batch.total_units), dim3(C::kThreads), C::kSmemBytes, stream, 1,
                    batch);
}

int smem_bytes_for_tok(int tok) {
  switch (tok) {
    case 32: return TileCfg<32>::kSmemBytes;
    case 64: return TileCfg<64>::kSmemBytes;
    case 128: return TileCfg<128>::kSmemBytes;
    default: return -1;
  }
}

cudaError_t launch_ternary_mma(int tok, const Batch& batch, cudaStream_t stream) {
  switch (tok) {
    case 32: return launch_tok<32>(batch, stream);
    case 64: return launch_tok<64>(batch, stream);
    case 128: return launch_tok<128>(batch, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace tern
