// internal.h -- structures shared by the host API (tern_api.cu) and the
// kernels.  Not part of the public ABI.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace tern {

// One ternary linear problem as the grouped tcgen05 kernel sees it.
struct alignas(64) Problem {
  CUtensorMap tmap_x;       // x [M, K] bf16, box {64 k, TOK rows}, 128-byte swizzle
  const uint8_t* packed;    // tile-interleaved codes
  const float* scales;      // [N]
  const __nv_bfloat16* bias;  // [N] or null
  __nv_bfloat16* y;         // [M, N]
  union {
    float* ws;              // ternary_mma: split-K partials [splits][tiles][TOK][128] (splits > 1);
                            // ternary_fp8: the E4M3 row scales a [M]
    const float* rope;      // ternary_mma2: (cos, sin) per token row and channel pair [M][64][2], or null
  };
  int* counters;            // one arrival counter per output tile (splits > 1), zero at rest
  int M, N, K;
  int n_tiles, m_tiles, splits;
  int chunks_per_split;     // 64-wide k chunks per split
  int unit_begin;            // first work unit (CTA, or 2-SM tile) of this problem
  int act;                   // epilogue activation (kActNone / kActGeluTanh)
  int act_col0;              // first output column the activation applies to
  const __nv_bfloat16* residual;  // [M, N] or null: y = residual + gate * act(v)
  const __nv_bfloat16* gate;      // [N] or null (gate 1)
  int norm_col0, norm_col1;       // RMS-normalised columns (128-column groups), empty if equal
  float norm_eps;
  int ldy;                        // elements between rows of y (and of the residual), >= N
  const __nv_bfloat16* norm_weight;  // [N] or null (weight 1)
};
static_assert(sizeof(Problem) == 256, "Problem layout");

// Launches `kernel` with programmatic dependent launch allowed (see
// pdl_wait in ptx.cuh: the kernel may be scheduled while the previous one of
// the stream drains, and waits for it before touching global memory) and,
// for cluster_x > 1, a cluster of cluster_x CTAs along x.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              unsigned cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

constexpr int kMaxProblems = 15;  // keeps the kernel parameter block under 4 KiB

struct Batch {
  Problem p[kMaxProblems];
  int count;
  int total_units;
  unsigned long long wait_limit_ns;
  unsigned int* status;     // per-device status word (bounded waits report here)
};
static_assert(sizeof(Batch) <= 4096, "kernel parameter block");

// Token-tile sizes (UMMA N) with a compiled kernel.
constexpr int kTokTiles[] = {32, 64, 128};

// Per-tile geometry, shared by host (launch) and device (kernel).
template <int TOK>
struct TileCfg {
  static constexpr int kCh = 128;                 // output channels per CTA (UMMA M)
  static constexpr int kBK = 64;                  // k per pipeline stage
  static constexpr int kXBytes = TOK * 128;       // TOK rows x 64 bf16, 128-byte swizzled
  static constexpr int kCBytes = kCh * 16;        // 128 rows x 16 bytes of codes
  static constexpr int kStageBytes = kXBytes + kCBytes;
  // Stage counts also size shared memory so that at most two CTAs fit on an
  // SM: two CTAs use all 512 TMEM columns.
  static constexpr int kStages = TOK <= 16 ? 20 : TOK <= 32 ? 14 : TOK <= 64 ? 8 : 5;
  static constexpr int kASlots = 4;               // decoded-weight slots in TMEM
  static constexpr int kACols = kBK / 2;          // 32-bit TMEM columns per slot (bf16x2)
  static constexpr int kDCols = TOK < 32 ? 32 : TOK;
  static constexpr int kTmemCols = (kDCols + kASlots * kACols) <= 256 ? 256 : 512;
  static constexpr int kDecWarps = TOK <= 64 ? 8 : 4;
  static constexpr int kThreads = (2 + kDecWarps) * 32;
  static constexpr int kSmemBytes = kStages * kStageBytes + 1024;
  // Instruction descriptor, kind::f16: D fp32, A bf16, B bf16, both K-major,
  // N = TOK, M = 128.
  static constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) |
                                     (uint32_t(TOK >> 3) << 17) | (uint32_t(128 >> 4) << 24);
  static_assert(TOK % 16 == 0 && TOK >= 16 && TOK <= 256, "UMMA N for M=128");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
  static_assert(3 * (kSmemBytes + 1024) > 228 * 1024, "a third CTA per SM would exceed TMEM");
};

cudaError_t launch_ternary_mma(int tok, const Batch& batch, cudaStream_t stream);
cudaError_t launch_quantize_pack(const __nv_bfloat16* W, int N, int K, float eps, uint8_t* packed,
                                 float* scales, cudaStream_t stream);
cudaError_t launch_dequantize(const uint8_t* packed, const float* scales, int N, int K,
                              __nv_bfloat16* out, cudaStream_t stream);
cudaError_t launch_wait_selftest(unsigned long long limit_ns, unsigned int* status,
                                 cudaStream_t stream);
// adaLN modulation of layer-normalised token rows (one warp per row, the row
// in registers): K % 8 == 0, K <= kAdaMaxK, 16-byte aligned rows, scale and
// shift rows mod_ld elements apart.
constexpr int kAdaMaxK = 4096;
cudaError_t launch_adaln_modulate(const __nv_bfloat16* x, int M, int K, const __nv_bfloat16* scale,
                                  const __nv_bfloat16* shift, int mod_ld, int tokens_per_row, float eps,
                                  __nv_bfloat16* out, cudaStream_t stream);
int smem_bytes_for_tok(int tok);
// Persistent tcgen05 tile kernel: tok-token tiles of 256 channels on CTA pairs
// (pair, cta_group::2; tok 256 for M > 64) or of 128 channels on single CTAs
// (!pair; tok 64 for 16 < M <= 64).  Problems use n_tiles = N / (256 or 128),
// m_tiles = ceil(M / tok), splits = 1 and a 3-D x tensor map {64 k, M,
// K / 64} whose box is {64, tok / 2 or tok rows, x_chunks_2sm(tok) chunks}
// (the 64-k chunks of one pipeline stage); ctas_or_pairs work units run at
// once.
cudaError_t launch_ternary_mma2(int tok, bool pair, const Batch& batch, int ctas_or_pairs, cudaStream_t stream);
int max_active_clusters_2sm();
int x_chunks_2sm(int tok);
// Small-M kernel (M <= 8 nt tokens, nt in {1, 2}), persistent over work
// units (problem, 128-channel slab): grid (splits, ctas) with clusters of
// `splits` CTAs along k (splits > 1 needs ctas == total_units); problems use
// n_tiles = N / 128 slabs, unit_begin = first slab in the launch,
// chunks_per_split 64-k chunks per CTA and a 3-D x tensor map {64 k, M,
// K / 64} whose box is {64, min(M, 8 nt), 16 (nt = 1) or 8 chunks}.
cudaError_t launch_ternary_gemv(int nt, const Batch& batch, int splits, int ctas, cudaStream_t stream);
// FP8 (E4M3) activations: per-token absmax quantisation of x (one warp per
// row, k interleaved inside 16-element groups), and the CTA-pair tile kernel
// with kind::f8f6f4 MMAs (one problem: N % 256 == 0, tmap_x = the 2-D E4M3 map
// {K, M} with box {128, 128}, ws = the per-token scales).
cudaError_t launch_quantize_act_e4m3(const __nv_bfloat16* x, int M, int K, uint8_t* xq, float* a,
                                     cudaStream_t stream);
cudaError_t launch_ternary_fp8(const Batch& batch, int pairs, cudaStream_t stream);


}  // namespace tern
