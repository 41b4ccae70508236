/*
 * tern.h -- C ABI of libtern, the B200 (sm_100a) ternary linear layer of
 * "1.58-bit FLUX" (arXiv 2412.18653).
 *
 * The method (page "1.58-bit FLUX", HTML v1):
 *   Section 1 -- the weights of every linear layer of the vision transformer
 *     take only the values {-1, 0, +1} ("akin to BitNet b1.58") and are stored
 *     as 2-bit signed integers instead of 16-bit numbers.
 *   Section 3.1 -- all linear layers of the double- and single-stream
 *     transformer blocks are quantised that way.
 *   Section 4 -- activations are not quantised: x and y stay 16-bit (bf16).
 * With the absmean quantiser of BitNet b1.58 per output channel n,
 *     s_n = mean_k |W[n,k]| + eps,   T[n,k] = RoundClip(W[n,k] / s_n, -1, +1),
 * the layer computes
 *     y[m,n] = s_n * sum_k x[m,k] * T[n,k] + b_n     (fp32 accumulation).
 *
 * Conventions for every call:
 *   - Every tensor is caller-owned DEVICE memory on the current CUDA device,
 *     dense and row-major.  The library never frees or keeps a caller pointer.
 *   - bf16 tensors are passed as `const void*` / `void*` (IEEE bfloat16).
 *   - Calls are asynchronous and stream-ordered on `stream` (NULL = the legacy
 *     default stream).  A host-detectable error returns at once with nothing
 *     launched.  Errors found on the device (a bounded wait that ran out) are
 *     reported later by tern_get_device_status().
 *   - Shapes: N % 16 == 0, K % 64 == 0, N, K >= 1; M >= 0 (M == 0 is a
 *     no-op, and x and y may then be NULL).  Pointers to bf16/packed data must
 *     be 16-byte aligned, `scales` 4-byte aligned.  Outputs must not overlap
 *     inputs.
 *
 * Packed weight layout ("tile-interleaved", Np*K/4 bytes with Np = N rounded
 * up to a multiple of 128, four codes per byte; the Np - N padding channels
 * hold zero codes and are never stored):
 *   a code is the 2-bit two's complement integer (+1 -> 01, 0 -> 00,
 *   -1 -> 11; 10 never occurs).  Codes are grouped in 16-byte groups, one per
 *   (row n, 64-wide chunk c = k/64), the group at byte offset
 *       ((n/128) * (K/64) + c) * 2048 + (n % 128) * 16,
 *   so the 128 rows x 64 k of one tile are one contiguous 2 KiB block and the
 *   K-chunks of a 128-row slab follow each other.  Inside a group, the
 *   little-endian 32-bit word w = (k % 64) / 16 holds 16 consecutive k; with
 *   j = (k % 16) / 2 and h = k % 2 the code of k sits at bits 16*h + 2*j.
 *   (Even k fill the low half-word and odd k the high half-word, so one
 *   shift-and-mask yields a bf16x2 pair.)
 */
#ifndef TERN_H
#define TERN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TERN_API __attribute__((visibility("default")))
#else
#define TERN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same handle as cudaStream_t / CUstream; NULL is the legacy default stream. */
typedef struct CUstream_st* tern_stream_t;

typedef enum {
  TERN_OK = 0,
  TERN_ERR_INVALID_ARG = -1,      /* null pointer, negative size, overlap, bad eps */
  TERN_ERR_UNSUPPORTED_SHAPE = -2, /* N % 16, K % 64, or a size beyond the limits */
  TERN_ERR_MISALIGNED = -3,       /* a pointer breaks the alignment rule above */
  TERN_ERR_CUDA = -4,             /* a CUDA runtime call or launch failed */
  TERN_ERR_TIMEOUT = -5,          /* a bounded device wait ran out (device status) */
  TERN_ERR_NO_DEVICE = -6,        /* the current device is not an sm_100 GPU */
  TERN_ERR_LAUNCH_CONFIG = -7     /* a kernel found its launch configuration inconsistent
                                     with its arguments and computed nothing: a defect of
                                     the library's host code, not of the caller's data
                                     (device status) */
} tern_status;

/* Bytes of the packed codes of an N x K ternary matrix: Np*K/4, Np = N rounded
 * up to a multiple of 128 (N*K/4 when N % 128 == 0).  Returns 0 for a shape
 * the layout does not support (N % 16, K % 64, or non-positive).  The four
 * 2-bit codes per byte follow page "1.58-bit FLUX", Section 1 (weights
 * "stored using 2-bit signed integers"); the padding to whole 128-channel
 * slabs is this library's layout choice, not on the pages. */
TERN_API size_t tern_packed_bytes(int64_t N, int64_t K);

/*
 * Absmean ternarisation and packing (page "1.58-bit FLUX", Section 1; the
 * BitNet b1.58 absmean rule it points to).
 *   W_bf16  [N, K] bf16, read only.
 *   eps     >= 0 and finite, added to the mean magnitude: s_n = mean|W_n| + eps.
 *   packed  [tern_packed_bytes(N, K)] bytes, written in the tile-interleaved layout above.
 *   scales  [N] fp32, written: s_n (the dequantised weight is T[n,k] * s_n).
 * The mean is accumulated at better than fp32 precision and rounded once to
 * fp32; a code is +-1 exactly when |W[n,k]| > s_n / 2 (fp32 s_n), else 0,
 * which is RoundClip with ties to even.  An all-zero row gets s_n = eps and
 * all-zero codes.
 */
TERN_API tern_status tern_quantize_pack(const void* W_bf16, int64_t N, int64_t K, float eps, void* packed,
                               float* scales, tern_stream_t stream);

/*
 * Ternary linear layer y = (x . T^T) * s + b (page "1.58-bit FLUX",
 * Sections 1 and 4).
 *   x_bf16  [M, K] bf16 activations.
 *   packed  [tern_packed_bytes(N, K)] codes from tern_quantize_pack (tile-interleaved layout).
 *   scales  [N] fp32 per-output-channel scales.
 *   bias    [N] bf16, or NULL for no bias.
 *   y_bf16  [M, N] bf16 output, overwritten (round to nearest even).
 * Products are exact (T is +-1/0), sums are fp32, then y = fp32 sum * s + b.
 * M <= 16 runs on a register-fed GEMV kernel; N % 256 == 0 with M > 16 on
 * CTA pairs; neither needs scratch.  The remaining case, 16 < M <= 64 with
 * N % 256 != 0, splits K across CTAs and uses a library-owned fp32 workspace
 * per (device, stream), allocated on the first such call; make that first
 * call outside CUDA stream capture.  Calls on the same stream are ordered;
 * calls on different streams use different workspaces.
 */
TERN_API tern_status tern_linear(const void* x_bf16, int64_t M, int64_t K, const void* packed,
                        const float* scales, const void* bias_bf16, int64_t N, void* y_bf16,
                        tern_stream_t stream);

/*
 * tern_linear without any device allocation, for callers that cannot call
 * cudaMalloc: code that runs while a CUDA graph is being captured in global
 * mode, engines that own all device memory in a preplanned arena or a
 * memory budget, and latency-critical loops where an allocation (which may
 * synchronise the device) is not allowed.  The paper has no counterpart: this
 * is an interface choice of this library.
 *   Arguments, layouts and results are those of tern_linear, and the tile and
 *   split choice is the same, so y matches tern_linear's bit for bit.
 *   Scratch: the path for 16 < M <= 64 with N % 256 != 0 splits K and keeps its
 *   fp32 partial sums and per-tile counters in one static device array of
 *   10 MiB + 4 KiB inside this library (held on every GPU that loads the
 *   library until the process exits).  That covers every shape on a 148-SM
 *   B200; a shape that would need more returns TERN_ERR_UNSUPPORTED_SHAPE
 *   with the sizes in tern_last_error().  Other M need no scratch.
 *   Set-up: the first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture.
 *   Sharing: every call on a device uses the same array, which keeps the last
 *   call's contents (the counters are cleared on the stream before each
 *   launch).  Calls whose kernels may overlap on the GPU -- on different
 *   streams, or from different host threads -- race on it: order them on one
 *   stream, or use tern_linear.
 */
TERN_API tern_status tern_linear_noalloc(const void* x_bf16, int64_t M, int64_t K, const void* packed,
                                const float* scales, const void* bias_bf16, int64_t N, void* y_bf16,
                                tern_stream_t stream);

/* Activations a fused epilogue applies (tern_linear_act, tern_linear_batch_act). */
typedef enum {
  TERN_ACT_NONE = 0,      /* the plain layer */
  TERN_ACT_GELU_TANH = 1  /* g(v) = 0.5 v (1 + tanh(sqrt(2/pi) (v + 0.044715 v^3))) */
} tern_act;

/*
 * tern_linear with an activation fused into the kernel's epilogue:
 *     y[m,n] = act(s_n * sum_k x[m,k] * T[n,k] + b_n)   for n >= act_col0,
 *     y[m,n] =     s_n * sum_k x[m,k] * T[n,k] + b_n    for n <  act_col0,
 * with act applied to the fp32 value before its one rounding to bf16.
 *   act       a tern_act value; TERN_ACT_NONE gives exactly tern_linear.
 *   act_col0  first activated output column, 0 <= act_col0 <= N (FLUX's
 *             single blocks compute q, k, v and the MLP's first projection in
 *             one linear and activate only the MLP part).
 * Other arguments, routing and errors as tern_linear; an unknown act or an
 * act_col0 outside [0, N] returns TERN_ERR_INVALID_ARG.  The pages quantise
 * every linear of FLUX's transformer blocks (Section 3.1) but do not describe
 * the operations between them: fusing the activation of FLUX.1's MLP into its
 * first linear is an interface choice of this library, saving one read and
 * one write of that linear's output.
 */
TERN_API tern_status tern_linear_act(const void* x_bf16, int64_t M, int64_t K, const void* packed,
                            const float* scales, const void* bias_bf16, int64_t N, int act,
                            int64_t act_col0, void* y_bf16, tern_stream_t stream);

/* One independent linear problem of a batch (same meaning as tern_linear). */
typedef struct {
  const void* x;      /* [M, K] bf16 */
  const void* packed; /* [tern_packed_bytes(N, K)] codes */
  const float* scales; /* [N] fp32 */
  const void* bias;   /* [N] bf16 or NULL */
  void* y;            /* [M, N] bf16 */
  int64_t M, N, K;
} tern_linear_args;

/*
 * A fused epilogue.  With v = s_n * sum_k x[m,k] * T[n,k] + b_n in fp32
 * (RMS-normalised first on the normalised columns, see norm_col0 below):
 *     a = act(v) for n >= act_col0, else v;
 *     y[m,n] = residual[m,n] + gate[n] * a     (residual NULL: 0; gate NULL: 1),
 * in fp32, then one rounding to bf16.  All zero is the plain layer.
 *   act, act_col0  as tern_linear_act.
 *   residual       [M, N] bf16, row-major, or NULL.  It may be y itself (an
 *                  in-place update of a residual stream); any other overlap
 *                  with y is TERN_ERR_INVALID_ARG.  2-byte aligned.
 *   gate           [N] bf16 or NULL, 2-byte aligned, not overlapping y.
 * FLUX.1's blocks add their attention output projection and their MLP's
 * second linear to the residual stream scaled by an adaLN-Zero gate taken
 * from the modulation GEMV's output; with residual = y = the stream and gate
 * = that slice, the update happens inside the linear's epilogue.  The pages
 * describe no operation between the quantised linears (Section 3.1): this is
 * an interface choice of this library.
 */
typedef struct {
  int act;              /* tern_act */
  int64_t act_col0;     /* first activated output column */
  const void* residual; /* [M, N] bf16 or NULL */
  const void* gate;     /* [N] bf16 or NULL */
  /* RMS normalisation over groups of 128 consecutive output columns (one
   * attention head of FLUX.1's q or k) on columns [norm_col0, norm_col1),
   * both multiples of 128 (equal: none), applied first, to v itself:
   *     v <- v / sqrt(mean over the token's group of v^2 + norm_eps) * norm_weight[n].
   * Where a normalised group has no activation, residual or gate on its
   * columns (FLUX.1's q/k norm), v is rounded to bf16 before it is
   * normalised, as the unfused layer stores q and k in bf16 and normalises
   * those: two roundings, within 3 * 2^-9 relative; otherwise fp32 and one
   * rounding as above.
   * Only where the layer runs on the tcgen05 tile kernels (N % 256 == 0 and
   * M > 16); elsewhere a requested normalisation is TERN_ERR_UNSUPPORTED_SHAPE. */
  int64_t norm_col0, norm_col1;
  const void* norm_weight; /* [N] bf16 or NULL (weight 1) */
  float norm_eps;          /* > 0 and finite when a normalisation is requested */
  /* Rotary position embedding of the normalised columns (FLUX.1 rotates q
   * and k after their RMS norm), or NULL: fp32 (cos, sin) pairs, 64 per
   * token row (row m at rope_cs + 128 m, 8-byte aligned, read only): channels
   * (2j, 2j + 1) of every normalised 128-column group of row m become
   *     (a cos - b sin, a sin + b cos),  (cos, sin) = pair j of row m,
   * applied to the normalised fp32 values before the one rounding (the
   * value before the normalisation was rounded to bf16, so a rotated value
   * is within 3 * 2^-9 of (|a| + |b|) of the exact one).  Only
   * with a normalisation and with no activation, residual or gate on the
   * normalised columns (TERN_ERR_INVALID_ARG otherwise). */
  const float* rope_cs;
} tern_epilogue;

/* tern_linear of *args with the fused epilogue *epilogue (NULL: none). */
TERN_API tern_status tern_linear_epilogue(const tern_linear_args* args, const tern_epilogue* epilogue,
                                 tern_stream_t stream);

/* tern_linear_batch with epilogues[i] for problem i (epilogues NULL: none). */
TERN_API tern_status tern_linear_batch_epilogue(const tern_linear_args* args, const tern_epilogue* epilogues,
                                       int count, tern_stream_t stream);

/*
 * Several independent ternary linears (for instance the per-stream adaLN
 * modulation GEMVs and projections of one FLUX block) with as few launches as
 * possible.  Each problem is the layer of page "1.58-bit FLUX", Sections 1
 * and 3.1 (every linear of both block types is ternary); batching them is not
 * on the pages -- it is an interface choice of this library, made because a
 * FLUX forward has 76 small modulation GEMVs whose launches would otherwise
 * dominate their run time.  Problems with similar M share one grouped launch (M <= 8, M <= 16,
 * then the tcgen05 kernels).  `args` is host memory, read before the call
 * returns.  Every problem is validated before anything is launched; on an
 * error nothing runs.  count == 0 is a no-op.  Problems may share inputs
 * (x, codes, scales, bias, gate), but no problem's y may overlap any buffer
 * of another problem (TERN_ERR_INVALID_ARG): they run concurrently.  Batched problems need no
 * workspace (only the single-call path for 16 < M <= 64 splits K into one).
 */
TERN_API tern_status tern_linear_batch(const tern_linear_args* args, int count, tern_stream_t stream);

/*
 * Row-strided x and y (page "1.58-bit FLUX", Sections 1 and 3.1: the same
 * ternary layer; strides are this library's interface choice, so that a
 * linear can read a column slice of a wider activation and write its output
 * into a slice of a concatenation buffer -- e.g. the attention and MLP parts
 * of a single FLUX block feeding its output projection -- without a copy).
 * x[m, k] is at x + m*ldx + k and y[m, n] at y + m*ldy + n (elements); the
 * residual of an epilogue has y's layout (rows ldy apart; it may be y
 * itself).  ldx >= K, ldy >= N, both multiples of 8 (16 bytes) and <= 2^30;
 * x and y 16-byte aligned.  y may share a parent tensor with x or with
 * another problem's buffers as long as no element is shared: regions with
 * equal strides are checked element-exactly, regions with different strides
 * must not intersect at all.  Everything else is as tern_linear_epilogue /
 * tern_linear_batch_epilogue (ldx = K, ldy = N gives exactly those calls).
 */
typedef struct {
  tern_linear_args linear;
  int64_t ldx; /* elements between rows of x */
  int64_t ldy; /* elements between rows of y (and of the residual) */
} tern_linear_strided_args;

TERN_API tern_status tern_linear_strided(const tern_linear_strided_args* args, const tern_epilogue* epilogue,
                                         tern_stream_t stream);
TERN_API tern_status tern_linear_batch_strided(const tern_linear_strided_args* args, const tern_epilogue* epilogues,
                                               int count, tern_stream_t stream);

/* One problem of tern_linear_batch_act: a linear and its epilogue activation. */
typedef struct {
  tern_linear_args linear;
  int act;          /* tern_act */
  int64_t act_col0; /* first activated output column */
} tern_linear_act_args;

/* tern_linear_batch with a per-problem epilogue activation (as tern_linear_act). */
TERN_API tern_status tern_linear_batch_act(const tern_linear_act_args* args, int count, tern_stream_t stream);

/*
 * Expands packed codes to the dequantised bf16 weight W'[n,k] = T[n,k] * s_n
 * ([N, K] row-major).  Not on the inference path: it feeds dense reference
 * GEMMs for comparison.
 */
TERN_API tern_status tern_dequantize(const void* packed, const float* scales, int64_t N, int64_t K,
                            void* W_bf16_out, tern_stream_t stream);

/*
 * adaLN modulation of layer-normalised activations, one pass.  FLUX.1's
 * blocks feed their first linears (QKV, MLP up; the fused projection of a
 * single block) with their token rows layer-normalised without affine and
 * modulated by a shift and a scale row of the block's adaLN modulation
 * output.  The pages quantise those linears (page "1.58-bit FLUX", Section
 * 3.1) and keep activations in 16 bits (Section 4) but do not describe this
 * step; it is an interface choice of this library.  Per token row m, with
 * g = m / tokens_per_row:
 *     out[m,k] = (x[m,k] - mean_m) / sqrt(var_m + eps) * (1 + scale[g,k]) + shift[g,k],
 * mean_m and the biased variance var_m over k in fp32, then one rounding to bf16.
 *   x, out          [M, K] bf16, row-major, 16-byte aligned.  out may be x
 *                   itself (in place); any other overlap is TERN_ERR_INVALID_ARG.
 *   scale, shift    ceil(M / tokens_per_row) rows of K bf16, row g at
 *                   scale + g * mod_ld (mod_ld >= K elements; e.g. slices of
 *                   the [B, 6 * hidden] modulation output with mod_ld =
 *                   6 * hidden), 16-byte aligned, mod_ld % 8 == 0, not
 *                   overlapping out.
 *   eps             >= 0 and finite (FLUX.1: 1e-6).
 *   M >= 0 (0: nothing launched, no pointer used), tokens_per_row >= 1, K % 8 == 0 and
 *   8 <= K <= 4096, else TERN_ERR_UNSUPPORTED_SHAPE.
 */
TERN_API tern_status tern_adaln_modulate(const void* x, int64_t M, int64_t K, const void* scale, const void* shift,
                                int64_t mod_ld, int64_t tokens_per_row, float eps, void* out,
                                tern_stream_t stream);

/*
 * FP8 (E4M3) activations for the ternary linear (page "1.58-bit FLUX",
 * Section 4: the method keeps activations at 16 bits and names quantising them
 * as the step that would turn the 2-bit weights into a latency gain; the pages
 * fix no format, so this is one reading of it).  Per token row m:
 *     a_m = max_k |x[m,k]| / 448   (fp32, IEEE division; 1 for an all-zero row)
 *     xq[m,k] = E4M3(x[m,k] / a_m) (fp32 IEEE division, round to nearest even,
 *                                  saturating at +-448; subnormals kept)
 * and the layer  y[m,n] = a_m * s_n * sum_k xq[m,k] * T[n,k] + b_n  with fp32
 * accumulation (the ternary weights are exact E4M3 values), rounded once to
 * bf16.  The only new error against tern_linear is the activation rounding
 * (at most 2^-4 relative per element).
 *
 * tern_quantize_act_e4m3: x [M, K] bf16 (16-byte aligned) -> xq [M, K] bytes
 * (16-byte aligned) and a [M] fp32 (4-byte aligned), all device memory owned
 * by the caller; K % 64 == 0.  Layout of xq: row-major, but inside every group
 * of 16 consecutive k the two halves are interleaved -- byte 16g + 2i holds
 * E4M3 of k = 16g + i and byte 16g + 2i + 1 holds k = 16g + 8 + i (i < 8) --
 * the order tern_linear_e4m3's kernel expands the weights in.  One launch.
 */
TERN_API tern_status tern_quantize_act_e4m3(const void* x_bf16, int64_t M, int64_t K, void* xq, float* a,
                                            tern_stream_t stream);

/* The layer on E4M3 activations from tern_quantize_act_e4m3: xq [M, K] in its
 * interleaved layout and a [M]; packed, scales, bias and y as tern_linear.
 * N % 256 == 0 (CTA-pair tiles of 256 channels; TERN_ERR_UNSUPPORTED_SHAPE
 * otherwise), K % 64 == 0, M >= 0.  y must not overlap an input.  One launch;
 * no workspace. */
TERN_API tern_status tern_linear_e4m3(const void* xq, const float* a, int64_t M, int64_t K, const void* packed,
                                      const float* scales, const void* bias_bf16, int64_t N, void* y_bf16,
                                      tern_stream_t stream);

/* Synchronises `stream`, then returns and clears the device status word of the
 * current device: TERN_ERR_TIMEOUT if any kernel's bounded wait ran out since
 * the last call, else TERN_ERR_LAUNCH_CONFIG if a kernel refused an
 * inconsistent launch configuration, TERN_OK otherwise (TERN_ERR_CUDA if the
 * sync itself failed). */
TERN_API tern_status tern_get_device_status(tern_stream_t stream);

/* Wall-time limit of every device-side wait, in nanoseconds (default 1e9).
 * Values below 1000 are clamped to 1000. */
TERN_API void tern_set_wait_limit_ns(uint64_t limit_ns);

/* Launches one tiny kernel whose wait on an mbarrier nothing ever arrives at
 * must run out after `limit_ns`; it exists so tests can see a device-side
 * timeout reported through tern_get_device_status() without faulting or
 * hanging the GPU. */
TERN_API tern_status tern_selftest_wait_timeout(uint64_t limit_ns, tern_stream_t stream);

/* Static description of a status code. */
TERN_API const char* tern_status_string(tern_status status);

/* Detail of the last failure on the calling host thread ("" if none). */
TERN_API const char* tern_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* TERN_H */
