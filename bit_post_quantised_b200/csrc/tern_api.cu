// tern_api.cu -- host side of the libtern C ABI (include/tern.h): argument
// checks, tile/split choice, TMA tensor maps, the per-(device, stream)
// split-K workspace, and the device status word.
//
// Page "1.58-bit FLUX" (arXiv 2412.18653): Section 1 defines the ternary
// weights and their 2-bit storage, Section 4 the unquantised 16-bit
// activations; this file only routes calls to the kernels that compute them.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <utility>
#include <vector>

#include "internal.h"
#include "kernel_common.cuh"
#include "ptx.cuh"
#include "tern.h"

namespace tern {
namespace {

__device__ unsigned int g_status_word = 0;  // one instance per device

thread_local std::string t_last_error;
std::atomic<unsigned long long> g_wait_limit_ns{1000000000ull};

tern_status fail(tern_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return s;
}

tern_status cuda_fail(cudaError_t e, const char* what) {
  return fail(TERN_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// ------------------------------------------------------------ device state
struct DeviceState {
  bool checked = false;
  bool supported = false;
  int sms = 0;
  int clusters_2sm = 0;  // CTA pairs of the 2-SM kernel resident at once
  unsigned int* status = nullptr;
};

constexpr int kMaxDevices = 64;
std::mutex g_mu;
DeviceState g_dev[kMaxDevices];

tern_status current_device(int* dev_out, DeviceState** st_out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(TERN_ERR_NO_DEVICE, "device ordinal %d", dev);
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState& d = g_dev[dev];
  if (!d.checked) {
    int major = 0, minor = 0, sms = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute");
    d.supported = (major == 10 && minor == 0);
    d.sms = sms;
    if (d.supported) {
      e = cudaGetSymbolAddress(reinterpret_cast<void**>(&d.status), g_status_word);
      if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(status word)");
      d.clusters_2sm = max_active_clusters_2sm();
    }
    d.checked = true;
  }
  if (!d.supported)
    return fail(TERN_ERR_NO_DEVICE, "device %d is not an sm_100 (B200-class) GPU", dev);
  *dev_out = dev;
  *st_out = &d;
  return TERN_OK;
}

// ------------------------------------------------------------ tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledFn>(nullptr);
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// x [M, K] bf16 row-major; box = 64 k x tok rows; 128-byte swizzle; rows past
// M read as zero.
tern_status make_x_map(CUtensorMap* map, const void* x, int64_t M, int64_t K, int64_t ldx, int tok) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(TERN_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  const cuuint64_t dims[2] = {cuuint64_t(K), cuuint64_t(M)};
  const cuuint64_t strides[1] = {cuuint64_t(ldx) * 2};
  const cuuint32_t box[2] = {64, cuuint32_t(tok)};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(TERN_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
  return TERN_OK;
}

// x [M, K] bf16 row-major viewed as 3-D {64 k, M tokens, K / 64 chunks}: box
// {64, rows, chunks} lands as [chunk][token][64 k] with 128-byte swizzle, so
// one copy brings several 64-k chunks; tokens past M and chunks past K read
// as zero.
tern_status make_x_map_chunks(CUtensorMap* map, const void* x, int64_t M, int64_t K, int64_t ldx, int rows,
                              int chunks) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(TERN_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  const cuuint64_t dims[3] = {64, cuuint64_t(M), cuuint64_t(K / 64)};
  const cuuint64_t strides[2] = {cuuint64_t(ldx) * 2, 128};
  const cuuint32_t box[3] = {64, cuuint32_t(rows), cuuint32_t(chunks)};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(x), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(TERN_ERR_CUDA, "cuTensorMapEncodeTiled (3-D x) failed (%d)", int(r));
  return TERN_OK;
}

// E4M3 x [M, K] bytes row-major: box = 128 k x 128 rows, 128-byte swizzle;
// columns past K and rows past M read as zero.
tern_status make_xq_map(CUtensorMap* map, const void* xq, int64_t M, int64_t K) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(TERN_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  const cuuint64_t dims[2] = {cuuint64_t(K), cuuint64_t(M)};
  const cuuint64_t strides[1] = {cuuint64_t(K)};
  const cuuint32_t box[2] = {128, 128};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(xq), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(TERN_ERR_CUDA, "cuTensorMapEncodeTiled (E4M3 x) failed (%d)", int(r));
  return TERN_OK;
}

// ------------------------------------------------------------ workspace
struct Workspace {
  float* ws = nullptr;
  size_t ws_bytes = 0;
  int* counters = nullptr;
  size_t n_counters = 0;
};
std::map<std::pair<int, cudaStream_t>, Workspace> g_ws;

tern_status get_workspace(int dev, cudaStream_t stream, size_t ws_bytes, size_t n_counters,
                          float** ws, int** counters) {
  std::lock_guard<std::mutex> lock(g_mu);
  Workspace& w = g_ws[{dev, stream}];
  cudaError_t e;
  if (w.ws_bytes < ws_bytes || w.n_counters < n_counters) {
    // Kernels queued on this stream may still use the old buffers.
    if ((e = cudaStreamSynchronize(stream)) != cudaSuccess) return cuda_fail(e, "workspace sync");
    const size_t nb = std::max(ws_bytes, w.ws_bytes), nc = std::max(n_counters, w.n_counters);
    if (w.ws) cudaFree(w.ws);
    if (w.counters) cudaFree(w.counters);
    w = Workspace{};
    if ((e = cudaMalloc(&w.ws, nb)) != cudaSuccess) return cuda_fail(e, "workspace cudaMalloc");
    if ((e = cudaMalloc(&w.counters, nc * sizeof(int))) != cudaSuccess) {
      cudaFree(w.ws);
      w = Workspace{};
      return cuda_fail(e, "counter cudaMalloc");
    }
    if ((e = cudaMemset(w.counters, 0, nc * sizeof(int))) != cudaSuccess)
      return cuda_fail(e, "counter cudaMemset");
    w.ws_bytes = nb;
    w.n_counters = nc;
  }
  *ws = w.ws;
  *counters = w.counters;
  return TERN_OK;
}

// ------------------------------------------------------------ validation
bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  if (!a || !b || na == 0 || nb == 0) return false;
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

constexpr int64_t kMaxN = int64_t(1) << 20;
constexpr int64_t kMaxK = int64_t(1) << 20;
constexpr int64_t kMaxM = int64_t(1) << 26;

// 128-channel slabs of the tiled layout: N rounds up, the padding channels
// hold zero codes and are never stored.
int64_t n_slabs(int64_t N) { return (N + 127) / 128; }
size_t packed_size(int64_t N, int64_t K) { return size_t(n_slabs(N)) * 128 * size_t(K) / 4; }

// One problem with its row strides in elements: x rows ldx apart, y (and the
// residual) rows ldy apart.  The dense entry points pass ldx = K, ldy = N.
struct LinArgs : tern_linear_args {
  int64_t ldx = 0, ldy = 0;
};
LinArgs dense_args(const tern_linear_args& a) {
  LinArgs l;
  static_cast<tern_linear_args&>(l) = a;
  l.ldx = a.K;
  l.ldy = a.N;
  return l;
}

// Whether two row-strided byte regions (rows, bytes per row, bytes between
// rows) share a byte.  Exact when the strides are equal (two views of one
// parent tensor, e.g. column slices of a concatenation buffer); otherwise
// any intersection of their spans counts.
bool regions_overlap(const void* a, int64_t ra, size_t wa, size_t lda, const void* b, int64_t rb, size_t wb,
                     size_t ldb) {
  if (!a || !b || ra <= 0 || rb <= 0 || wa == 0 || wb == 0) return false;
  const size_t na = size_t(ra - 1) * lda + wa, nb = size_t(rb - 1) * ldb + wb;
  if (!overlaps(a, na, b, nb)) return false;
  if (lda != ldb || ra == 1 || rb == 1) return true;  // conservative
  uintptr_t pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
  if (pa > pb) {
    std::swap(pa, pb);
    std::swap(ra, rb);
    std::swap(wa, wb);
  }
  const size_t d = size_t(pb - pa), q = d / lda, rem = d % lda;
  // b's row r starts in a's row q + r at byte rem and may run into row q + r + 1.
  if (rem < wa && int64_t(q) < ra) return true;
  return rem + wb > lda && int64_t(q) + 1 < ra;
}

tern_status check_nk(int64_t N, int64_t K) {
  if (N < 0 || K < 0) return fail(TERN_ERR_INVALID_ARG, "negative size N=%lld K=%lld", (long long)N, (long long)K);
  if (N == 0 || K == 0 || N % 16 != 0 || K % 64 != 0)
    return fail(TERN_ERR_UNSUPPORTED_SHAPE, "need N %% 16 == 0 and K %% 64 == 0, got N=%lld K=%lld",
                (long long)N, (long long)K);
  if (N > kMaxN || K > kMaxK)
    return fail(TERN_ERR_UNSUPPORTED_SHAPE, "N or K above 2^20 (N=%lld K=%lld)", (long long)N, (long long)K);
  return TERN_OK;
}

tern_status check_linear(const LinArgs& a) {
  tern_status s = check_nk(a.N, a.K);
  if (s != TERN_OK) return s;
  if (a.M < 0) return fail(TERN_ERR_INVALID_ARG, "negative M=%lld", (long long)a.M);
  if (a.M > kMaxM) return fail(TERN_ERR_UNSUPPORTED_SHAPE, "M above 2^26 (M=%lld)", (long long)a.M);
  if (a.ldx < a.K || a.ldy < a.N || a.ldx % 8 != 0 || a.ldy % 8 != 0 || a.ldx > (int64_t(1) << 30) ||
      a.ldy > (int64_t(1) << 30))
    return fail(TERN_ERR_INVALID_ARG, "row strides need ldx >= K, ldy >= N, both multiples of 8 and <= 2^30 "
                "(ldx=%lld K=%lld ldy=%lld N=%lld)", (long long)a.ldx, (long long)a.K, (long long)a.ldy,
                (long long)a.N);
  if (!a.packed || !a.scales || (a.M > 0 && (!a.x || !a.y)))
    return fail(TERN_ERR_INVALID_ARG, "null x, packed, scales or y");
  if (!aligned(a.x, 16) || !aligned(a.packed, 16) || !aligned(a.y, 16) || !aligned(a.scales, 4) ||
      (a.bias && !aligned(a.bias, 2)))
    return fail(TERN_ERR_MISALIGNED, "x, packed and y need 16-byte, scales 4-byte, bias 2-byte alignment");
  const size_t yw = size_t(a.N) * 2, yld = size_t(a.ldy) * 2;
  if (regions_overlap(a.y, a.M, yw, yld, a.x, a.M, size_t(a.K) * 2, size_t(a.ldx) * 2) ||
      regions_overlap(a.y, a.M, yw, yld, a.packed, 1, packed_size(a.N, a.K), packed_size(a.N, a.K)) ||
      regions_overlap(a.y, a.M, yw, yld, a.scales, 1, size_t(a.N) * 4, size_t(a.N) * 4) ||
      regions_overlap(a.y, a.M, yw, yld, a.bias, a.bias ? 1 : 0, size_t(a.N) * 2, size_t(a.N) * 2))
    return fail(TERN_ERR_INVALID_ARG, "y overlaps an input");
  return TERN_OK;
}

static_assert(kActNone == TERN_ACT_NONE && kActGeluTanh == TERN_ACT_GELU_TANH, "kernel and ABI activation codes");

// (The epilogue of one problem is a tern_epilogue; all zero is the plain layer.)

tern_status check_epilogue(const tern_epilogue& e, const LinArgs& a) {
  if (e.act != TERN_ACT_NONE && e.act != TERN_ACT_GELU_TANH)
    return fail(TERN_ERR_INVALID_ARG, "unknown activation %d", e.act);
  if (e.act_col0 < 0 || e.act_col0 > a.N)
    return fail(TERN_ERR_INVALID_ARG, "act_col0=%lld outside [0, N=%lld]", (long long)e.act_col0, (long long)a.N);
  if (!aligned(e.residual, 2) || !aligned(e.gate, 2))
    return fail(TERN_ERR_MISALIGNED, "residual and gate need 2-byte alignment");
  const size_t yw = size_t(a.N) * 2, yld = size_t(a.ldy) * 2;
  // The residual has y's layout (rows ldy apart) and may be y itself (an
  // in-place update: each element is read before the same thread writes
  // it); any other overlap with y would race.
  if (e.residual && e.residual != a.y && regions_overlap(e.residual, a.M, yw, yld, a.y, a.M, yw, yld))
    return fail(TERN_ERR_INVALID_ARG, "residual overlaps y without being y");
  if (regions_overlap(e.gate, e.gate ? 1 : 0, yw, yw, a.y, a.M, yw, yld))
    return fail(TERN_ERR_INVALID_ARG, "gate overlaps y");
  if (e.norm_col0 < 0 || e.norm_col1 < e.norm_col0 || e.norm_col1 > a.N || e.norm_col0 % 128 || e.norm_col1 % 128)
    return fail(TERN_ERR_INVALID_ARG, "norm columns [%lld, %lld) must be 128-aligned within [0, N=%lld]",
                (long long)e.norm_col0, (long long)e.norm_col1, (long long)a.N);
  if (e.norm_col0 != e.norm_col1) {
    if (!(e.norm_eps > 0.f) || !std::isfinite(e.norm_eps))
      return fail(TERN_ERR_INVALID_ARG, "norm_eps must be finite and > 0");
    if (!aligned(e.norm_weight, 2)) return fail(TERN_ERR_MISALIGNED, "norm_weight needs 2-byte alignment");
    if (regions_overlap(e.norm_weight, e.norm_weight ? 1 : 0, yw, yw, a.y, a.M, yw, yld))
      return fail(TERN_ERR_INVALID_ARG, "norm_weight overlaps y");
  }
  if (e.rope_cs) {
    if (e.norm_col0 == e.norm_col1)
      return fail(TERN_ERR_INVALID_ARG, "the rotary embedding applies to normalised columns: none requested");
    if (e.residual || e.gate || (e.act != TERN_ACT_NONE && e.act_col0 < e.norm_col1))
      return fail(TERN_ERR_INVALID_ARG, "the rotary embedding needs no activation, residual or gate on the "
                                        "normalised columns");
    if (!aligned(e.rope_cs, 8)) return fail(TERN_ERR_MISALIGNED, "rope_cs needs 8-byte alignment");
    const size_t rw = 64 * 2 * sizeof(float);
    if (regions_overlap(e.rope_cs, a.M, rw, rw, a.y, a.M, yw, yld))
      return fail(TERN_ERR_INVALID_ARG, "rope_cs overlaps y");
  }
  return TERN_OK;
}

// The RMS normalisation exists only in the tcgen05 tile kernels: N % 256 ==
// 0 and M > 16 (checked without a device), and the device able to run the
// CTA-pair kernel for M > 64 (ptok from pair_tok; checked once it is known).
tern_status check_norm_route(const tern_epilogue& e, const tern_linear_args& a, int ptok = -1) {
  if (e.norm_col0 == e.norm_col1 || a.M == 0) return TERN_OK;
  if (a.N % 256 != 0 || a.M <= 16 || ptok == 0)
    return fail(TERN_ERR_UNSUPPORTED_SHAPE,
                "the RMS-normalising epilogue needs N %% 256 == 0 and M > 16 (M=%lld N=%lld)", (long long)a.M,
                (long long)a.N);
  return TERN_OK;
}

void set_epilogue(Problem* p, const tern_epilogue* epis, int i) {
  if (!epis) return;  // the Problem was zeroed: plain layer
  p->act = epis[i].act;
  p->act_col0 = int(epis[i].act_col0);
  p->residual = static_cast<const __nv_bfloat16*>(epis[i].residual);
  p->gate = static_cast<const __nv_bfloat16*>(epis[i].gate);
  p->norm_col0 = int(epis[i].norm_col0);
  p->norm_col1 = int(epis[i].norm_col1);
  p->norm_eps = epis[i].norm_eps;
  p->norm_weight = static_cast<const __nv_bfloat16*>(epis[i].norm_weight);
  // Shares its slot with the split-K workspace of the fallback kernel, which
  // never carries a normalisation (and so never a rotation): set only when
  // given.
  if (epis[i].rope_cs) p->rope = epis[i].rope_cs;
}

// Up to 16 tokens run on the register-fed GEMV kernel, in n8 blocks.
constexpr int64_t kGemvMaxM = 16;
int gemv_nt(int64_t M) { return M <= 8 ? 1 : 2; }

// Token tile of the single-SM tcgen05 kernel for 16 < M (or N % 256 != 0).
int pick_tok(int64_t M) {
  if (M <= 32) return 32;
  if (M <= 64) return 64;
  return 128;
}

// Fills everything of a Problem except unit_begin; returns its CTA count.
tern_status fill_problem(const LinArgs& a, int tok, int splits_wanted, Problem* p,
                         int64_t* ctas) {
  std::memset(static_cast<void*>(p), 0, sizeof(Problem));
  tern_status s = make_x_map(&p->tmap_x, a.x, a.M, a.K, a.ldx, tok);
  if (s != TERN_OK) return s;
  p->packed = static_cast<const uint8_t*>(a.packed);
  p->scales = a.scales;
  p->bias = static_cast<const __nv_bfloat16*>(a.bias);
  p->y = static_cast<__nv_bfloat16*>(a.y);
  p->M = int(a.M);
  p->N = int(a.N);
  p->K = int(a.K);
  p->ldy = int(a.ldy);
  p->n_tiles = int(n_slabs(a.N));
  p->m_tiles = int((a.M + tok - 1) / tok);
  const int kc_total = int(a.K / 64);
  int splits = std::max(1, std::min(splits_wanted, kc_total));
  const int per = (kc_total + splits - 1) / splits;
  splits = (kc_total + per - 1) / per;  // no empty split
  p->splits = splits;
  p->chunks_per_split = per;
  *ctas = int64_t(p->n_tiles) * p->m_tiles * splits;
  if (*ctas > (int64_t(1) << 31) - 1) return fail(TERN_ERR_UNSUPPORTED_SHAPE, "too many tiles");
  return TERN_OK;
}

// Token tile of the persistent tcgen05 tile kernel for this problem, or 0
// when it does not apply: N must tile into 256-channel pairs (every FLUX
// linear does), and M <= 16 goes to the GEMV kernel.  M > 64 runs 256-token
// tiles on CTA pairs (needs the device to co-schedule pairs), 16 < M <= 64
// 64-token tiles on single CTAs.
int pair_tok(const tern_linear_args& a, const DeviceState* ds) {
  if (a.N % 256 != 0 || a.M <= 16) return 0;
  if (a.M <= 64) return 64;
  return ds->clusters_2sm > 0 ? 256 : 0;
}
bool tok_is_pair(int tok) { return tok == 256; }

// Fills a Problem for the pair-tile kernel except unit_begin; returns its tiles.
tern_status fill_problem_2sm(const LinArgs& a, int tok, Problem* p, int64_t* tiles) {
  std::memset(static_cast<void*>(p), 0, sizeof(Problem));
  const bool pair = tok_is_pair(tok);
  tern_status s = make_x_map_chunks(&p->tmap_x, a.x, a.M, a.K, a.ldx, pair ? tok / 2 : tok, x_chunks_2sm(tok));
  if (s != TERN_OK) return s;
  p->packed = static_cast<const uint8_t*>(a.packed);
  p->scales = a.scales;
  p->bias = static_cast<const __nv_bfloat16*>(a.bias);
  p->y = static_cast<__nv_bfloat16*>(a.y);
  p->M = int(a.M);
  p->N = int(a.N);
  p->K = int(a.K);
  p->ldy = int(a.ldy);
  p->n_tiles = int(a.N / (pair ? 256 : 128));
  p->m_tiles = int((a.M + tok - 1) / tok);
  p->splits = 1;
  p->chunks_per_split = int(a.K / 64);
  *tiles = int64_t(p->n_tiles) * p->m_tiles;
  if (*tiles > (int64_t(1) << 31) - 1) return fail(TERN_ERR_UNSUPPORTED_SHAPE, "too many tiles");
  return TERN_OK;
}

// Launches the problems `idx_in` of `args` (all with pair_tok == tok) on the
// pair-tile kernel, up to kMaxProblems per launch.  The kernel hands tile u
// of a launch to CTA (pair) u mod #resident, in problem order; problems go in
// by decreasing K (a tile's cost), so the long tiles are dealt out first and
// spread evenly (a FLUX double block's batch, whose MLP-down tiles take four
// times the others: the busiest pair holds 36 instead of 39 tile-units for
// an even share of 35).
tern_status launch_2sm_group(const LinArgs* args, const tern_epilogue* epis, const std::vector<int>& idx_in, int tok,
                             Batch& batch, const DeviceState* ds, cudaStream_t cs) {
  std::vector<int> idx(idx_in);
  std::stable_sort(idx.begin(), idx.end(), [&](int a, int b) { return args[a].K > args[b].K; });
  for (size_t g0 = 0; g0 < idx.size(); g0 += kMaxProblems) {
    std::memset(static_cast<void*>(&batch), 0, sizeof batch);
    int64_t total = 0;
    int n = 0;
    for (size_t g = g0; g < idx.size() && n < kMaxProblems; ++g, ++n) {
      int64_t tiles = 0;
      tern_status s = fill_problem_2sm(args[idx[g]], tok, &batch.p[n], &tiles);
      if (s != TERN_OK) return s;
      set_epilogue(&batch.p[n], epis, idx[g]);
      batch.p[n].unit_begin = int(total);
      total += tiles;
      if (total > (int64_t(1) << 31) - 1) return fail(TERN_ERR_UNSUPPORTED_SHAPE, "batch too large");
    }
    batch.count = n;
    batch.total_units = int(total);
    batch.wait_limit_ns = g_wait_limit_ns.load();
    batch.status = ds->status;
    const bool pair = tok_is_pair(tok);
    const int64_t resident = pair ? ds->clusters_2sm : ds->sms;
    cudaError_t e = launch_ternary_mma2(tok, pair, batch, int(std::min<int64_t>(total, resident)), cs);
    if (e != cudaSuccess) return cuda_fail(e, "ternary_mma2 launch");
  }
  return TERN_OK;
}

// Launches the problems `idx` of `args` (all with M <= 8 nt) on the GEMV
// kernel, up to kMaxProblems per launch.  K is split over a cluster of up to
// eight CTAs when the launch has fewer 128-channel slabs than the GPU has SMs.
tern_status launch_gemv_group(const LinArgs* args, const tern_epilogue* epis, const std::vector<int>& idx, int nt,
                              Batch& batch, const DeviceState* ds, cudaStream_t cs) {
  for (size_t g0 = 0; g0 < idx.size(); g0 += kMaxProblems) {
    std::memset(static_cast<void*>(&batch), 0, sizeof batch);
    int64_t slabs = 0;
    int64_t min_chunks = int64_t(1) << 40;
    int n = 0;
    for (size_t g = g0; g < idx.size() && n < kMaxProblems; ++g, ++n) {
      const LinArgs& a = args[idx[g]];
      Problem* p = &batch.p[n];
      tern_status s = make_x_map_chunks(&p->tmap_x, a.x, a.M, a.K, a.ldx, 8 * nt, nt == 1 ? 16 : 8);
      if (s != TERN_OK) return s;
      p->packed = static_cast<const uint8_t*>(a.packed);
      p->scales = a.scales;
      p->bias = static_cast<const __nv_bfloat16*>(a.bias);
      p->y = static_cast<__nv_bfloat16*>(a.y);
      p->M = int(a.M);
      p->N = int(a.N);
      p->K = int(a.K);
      p->ldy = int(a.ldy);
      p->n_tiles = int(n_slabs(a.N));
      p->m_tiles = 1;
      set_epilogue(p, epis, idx[g]);
      p->unit_begin = int(slabs);
      slabs += n_slabs(a.N);
      min_chunks = std::min<int64_t>(min_chunks, a.K / 64);
    }
    if (slabs > 65535) return fail(TERN_ERR_UNSUPPORTED_SHAPE, "more than 65535 slabs of 128 channels in one launch");
    const int splits = int(std::max<int64_t>(1, std::min<int64_t>({8, ds->sms / slabs, min_chunks})));
    for (int i = 0; i < n; ++i) {
      batch.p[i].splits = splits;
      batch.p[i].chunks_per_split = (batch.p[i].K / 64 + splits - 1) / splits;
    }
    batch.count = n;
    batch.total_units = int(slabs);
    batch.wait_limit_ns = g_wait_limit_ns.load();
    batch.status = ds->status;
    // splits > 1: one CTA per slab; otherwise persistent CTAs, one per SM at most.
    const int ctas = splits > 1 ? int(slabs) : int(std::min<int64_t>(slabs, ds->sms));
    cudaError_t e = launch_ternary_gemv(nt, batch, splits, ctas, cs);
    if (e != cudaSuccess) return cuda_fail(e, "ternary_gemv launch");
  }
  return TERN_OK;
}

int ctas_per_sm(int tok) {
  const int smem = smem_bytes_for_tok(tok);
  const int by_smem = (228 * 1024) / (smem + 1024);
  const int by_tmem = 2;  // each CTA allocates 256 of the 512 TMEM columns (tok <= 128)
  return std::max(1, std::min(by_smem, by_tmem));
}

// K splits of the single-CTA fallback kernel for one problem: with few tokens
// (tok <= 64), enough splits that every SM streams codes, at least 4 chunks
// of 64 k per split, at most 16.
int fallback_splits(int64_t M, int64_t N, int64_t K, int tok, const DeviceState* ds) {
  if (tok > 64) return 1;
  const int64_t tiles = n_slabs(N) * ((M + tok - 1) / tok);
  const int64_t target = int64_t(ds->sms) * ctas_per_sm(tok);
  int splits = 1;
  if (tiles < target) splits = int(std::min<int64_t>(target / tiles, std::max<int64_t>(1, K / 64 / 4)));
  return std::max(1, std::min(splits, 16));
}

}  // namespace
}  // namespace tern

using namespace tern;

extern "C" {

size_t tern_packed_bytes(int64_t N, int64_t K) {
  if (N <= 0 || K <= 0 || N % 16 != 0 || K % 64 != 0 || N > kMaxN || K > kMaxK) return 0;
  return packed_size(N, K);
}

tern_status tern_quantize_pack(const void* W_bf16, int64_t N, int64_t K, float eps, void* packed,
                               float* scales, tern_stream_t stream) {
  tern_status s = check_nk(N, K);
  if (s != TERN_OK) return s;
  if (!W_bf16 || !packed || !scales) return fail(TERN_ERR_INVALID_ARG, "null W, packed or scales");
  if (!(eps >= 0.f) || !std::isfinite(eps)) return fail(TERN_ERR_INVALID_ARG, "eps must be finite and >= 0");
  if (!aligned(W_bf16, 16) || !aligned(packed, 16) || !aligned(scales, 4))
    return fail(TERN_ERR_MISALIGNED, "W and packed need 16-byte, scales 4-byte alignment");
  const size_t wb = size_t(N) * size_t(K) * 2, pb = packed_size(N, K), sb = size_t(N) * 4;
  if (overlaps(packed, pb, W_bf16, wb) || overlaps(scales, sb, W_bf16, wb) || overlaps(packed, pb, scales, sb))
    return fail(TERN_ERR_INVALID_ARG, "outputs overlap each other or W");
  int dev;
  DeviceState* ds;
  if ((s = current_device(&dev, &ds)) != TERN_OK) return s;
  cudaError_t e = launch_quantize_pack(static_cast<const __nv_bfloat16*>(W_bf16), int(N), int(K), eps,
                                       static_cast<uint8_t*>(packed), scales,
                                       reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "quantize_pack launch");
  return TERN_OK;
}

tern_status tern_adaln_modulate(const void* x, int64_t M, int64_t K, const void* scale, const void* shift,
                                int64_t mod_ld, int64_t tokens_per_row, float eps, void* out,
                                tern_stream_t stream) {
  if (M < 0 || K < 0 || mod_ld < 0) return fail(TERN_ERR_INVALID_ARG, "negative size");
  if (K < 8 || K % 8 != 0 || K > kAdaMaxK || M > int64_t(INT32_MAX) || tokens_per_row < 1 ||
      tokens_per_row > int64_t(INT32_MAX) || mod_ld < K || mod_ld % 8 != 0 || mod_ld > int64_t(INT32_MAX))
    return fail(TERN_ERR_UNSUPPORTED_SHAPE, "adaln_modulate: M=%lld K=%lld mod_ld=%lld tokens_per_row=%lld",
                (long long)M, (long long)K, (long long)mod_ld, (long long)tokens_per_row);
  if (!(eps >= 0.f) || !std::isfinite(eps)) return fail(TERN_ERR_INVALID_ARG, "eps must be finite and >= 0");
  if (M == 0) return TERN_OK;  // no row: the pointers are not used
  if (!x || !scale || !shift || !out) return fail(TERN_ERR_INVALID_ARG, "null x, scale, shift or out");
  if (!aligned(x, 16) || !aligned(scale, 16) || !aligned(shift, 16) || !aligned(out, 16))
    return fail(TERN_ERR_MISALIGNED, "x, scale, shift and out need 16-byte alignment");
  const size_t xb = size_t(M) * size_t(K) * 2;
  const int64_t G = (M + tokens_per_row - 1) / tokens_per_row;
  const size_t mb = (size_t(G - 1) * size_t(mod_ld) + size_t(K)) * 2;
  if (out != x && overlaps(out, xb, x, xb)) return fail(TERN_ERR_INVALID_ARG, "out overlaps x without being x");
  if (overlaps(out, xb, scale, mb) || overlaps(out, xb, shift, mb))
    return fail(TERN_ERR_INVALID_ARG, "out overlaps scale or shift");
  int dev;
  DeviceState* ds;
  tern_status s;
  if ((s = current_device(&dev, &ds)) != TERN_OK) return s;
  cudaError_t e = launch_adaln_modulate(static_cast<const __nv_bfloat16*>(x), int(M), int(K),
                                        static_cast<const __nv_bfloat16*>(scale),
                                        static_cast<const __nv_bfloat16*>(shift), int(mod_ld), int(tokens_per_row),
                                        eps, static_cast<__nv_bfloat16*>(out), reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "adaln_modulate launch");
  return TERN_OK;
}

}  // extern "C"

namespace tern {
namespace {

tern_status linear_impl(const LinArgs& a, const tern_epilogue& epi, tern_stream_t stream) {
  const int64_t M = a.M, N = a.N, K = a.K;
  tern_status s = check_linear(a);
  if (s != TERN_OK) return s;
  if ((s = check_epilogue(epi, a)) != TERN_OK) return s;
  if ((s = check_norm_route(epi, a)) != TERN_OK) return s;
  if (M == 0) return TERN_OK;
  int dev;
  DeviceState* ds;
  if ((s = current_device(&dev, &ds)) != TERN_OK) return s;
  if ((s = check_norm_route(epi, a, pair_tok(a, ds))) != TERN_OK) return s;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);

  if (M <= kGemvMaxM) {
    static Batch batch_g;  // built under the lock below; ~4 KiB, copied into the launch
    static std::mutex batch_g_mu;
    std::lock_guard<std::mutex> lock(batch_g_mu);
    return launch_gemv_group(&a, &epi, std::vector<int>{0}, gemv_nt(M), batch_g, ds, cs);
  }
  if (const int ptok = pair_tok(a, ds)) {
    static Batch batch2;  // built under the lock below; ~4 KiB, copied into the launch
    static std::mutex batch2_mu;
    std::lock_guard<std::mutex> lock(batch2_mu);
    return launch_2sm_group(&a, &epi, std::vector<int>{0}, ptok, batch2, ds, cs);
  }
  const int tok = pick_tok(M);
  const int splits = fallback_splits(M, N, K, tok, ds);
  const int64_t tiles = n_slabs(N) * ((M + tok - 1) / tok);
  static Batch batch;  // built under the lock below; ~4 KiB, copied into the launch
  static std::mutex batch_mu;
  std::lock_guard<std::mutex> lock(batch_mu);
  std::memset(static_cast<void*>(&batch), 0, sizeof batch);
  int64_t ctas = 0;
  if ((s = fill_problem(a, tok, splits, &batch.p[0], &ctas)) != TERN_OK) return s;
  Problem& p = batch.p[0];
  set_epilogue(&p, &epi, 0);
  if (p.splits > 1) {
    const size_t ws_bytes = size_t(p.splits) * size_t(tiles) * tok * 128 * sizeof(float);
    if ((s = get_workspace(dev, cs, ws_bytes, size_t(tiles), &p.ws, &p.counters)) != TERN_OK) return s;
  }
  p.unit_begin = 0;
  batch.count = 1;
  batch.total_units = int(ctas);
  batch.wait_limit_ns = g_wait_limit_ns.load();
  batch.status = ds->status;
  cudaError_t e = launch_ternary_mma(tok, batch, cs);
  if (e != cudaSuccess) return cuda_fail(e, "ternary_mma launch");
  return TERN_OK;
}

tern_status batch_impl(const LinArgs* args, const tern_epilogue* epis, int count, tern_stream_t stream) {
  for (int i = 0; i < count; ++i) {
    tern_status s = check_linear(args[i]);
    if (s == TERN_OK && epis) s = check_epilogue(epis[i], args[i]);
    if (s == TERN_OK && epis) s = check_norm_route(epis[i], args[i]);
    if (s != TERN_OK) {
      t_last_error = "problem " + std::to_string(i) + ": " + t_last_error;
      return s;
    }
  }
  if (count == 0) return TERN_OK;
  // Problems of one launch run concurrently: no problem's y may overlap any
  // buffer of another problem (its inputs, its residual or its y).
  for (int i = 0; i < count; ++i) {
    const LinArgs& a = args[i];
    if (a.M == 0) continue;
    const size_t wa = size_t(a.N) * 2, lda = size_t(a.ldy) * 2;
    for (int j = 0; j < count; ++j) {
      const LinArgs& b = args[j];
      if (j == i || b.M == 0) continue;
      const size_t wb = size_t(b.N) * 2, ldb = size_t(b.ldy) * 2;
      const void* res = epis ? epis[j].residual : nullptr;
      const void* gate = epis ? epis[j].gate : nullptr;
      const void* nw = epis ? epis[j].norm_weight : nullptr;
      const size_t pb = packed_size(b.N, b.K);
      if (regions_overlap(a.y, a.M, wa, lda, b.y, b.M, wb, ldb) ||
          regions_overlap(a.y, a.M, wa, lda, b.x, b.M, size_t(b.K) * 2, size_t(b.ldx) * 2) ||
          regions_overlap(a.y, a.M, wa, lda, b.packed, 1, pb, pb) ||
          regions_overlap(a.y, a.M, wa, lda, b.scales, 1, size_t(b.N) * 4, size_t(b.N) * 4) ||
          regions_overlap(a.y, a.M, wa, lda, b.bias, b.bias ? 1 : 0, wb, wb) ||
          regions_overlap(a.y, a.M, wa, lda, res, res ? b.M : 0, wb, ldb) ||
          regions_overlap(a.y, a.M, wa, lda, gate, gate ? 1 : 0, wb, wb) ||
          regions_overlap(a.y, a.M, wa, lda, nw, nw ? 1 : 0, wb, wb))
        return fail(TERN_ERR_INVALID_ARG, "problem %d's y overlaps a buffer of problem %d", i, j);
    }
  }
  int dev;
  DeviceState* ds;
  tern_status s = current_device(&dev, &ds);
  if (s != TERN_OK) return s;
  for (int i = 0; epis && i < count; ++i)
    if ((s = check_norm_route(epis[i], args[i], pair_tok(args[i], ds))) != TERN_OK) {
      t_last_error = "problem " + std::to_string(i) + ": " + t_last_error;
      return s;
    }
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);

  static Batch batch;
  static std::mutex batch_mu;
  std::lock_guard<std::mutex> lock(batch_mu);
  for (int nt : {1, 2}) {
    std::vector<int> group;
    for (int i = 0; i < count; ++i)
      if (args[i].M > 0 && args[i].M <= kGemvMaxM && gemv_nt(args[i].M) == nt) group.push_back(i);
    if ((s = launch_gemv_group(args, epis, group, nt, batch, ds, cs)) != TERN_OK) return s;
  }
  for (int ptok : {64, 256}) {
    std::vector<int> group;
    for (int i = 0; i < count; ++i)
      if (args[i].M > 0 && pair_tok(args[i], ds) == ptok) group.push_back(i);
    if ((s = launch_2sm_group(args, epis, group, ptok, batch, ds, cs)) != TERN_OK) return s;
  }
  for (int tok : kTokTiles) {
    std::vector<int> group;
    for (int i = 0; i < count; ++i)
      if (args[i].M > kGemvMaxM && !pair_tok(args[i], ds) && pick_tok(args[i].M) == tok) group.push_back(i);
    for (size_t g0 = 0; g0 < group.size(); g0 += kMaxProblems) {
      std::memset(static_cast<void*>(&batch), 0, sizeof batch);
      int64_t total = 0;
      int n = 0;
      for (size_t g = g0; g < group.size() && n < kMaxProblems; ++g, ++n) {
        int64_t ctas = 0;
        if ((s = fill_problem(args[group[g]], tok, 1, &batch.p[n], &ctas)) != TERN_OK) return s;
        set_epilogue(&batch.p[n], epis, group[g]);
        batch.p[n].unit_begin = int(total);
        total += ctas;
        if (total > (int64_t(1) << 31) - 1) return fail(TERN_ERR_UNSUPPORTED_SHAPE, "batch too large");
      }
      batch.count = n;
      batch.total_units = int(total);
      batch.wait_limit_ns = g_wait_limit_ns.load();
      batch.status = ds->status;
      cudaError_t e = launch_ternary_mma(tok, batch, cs);
      if (e != cudaSuccess) return cuda_fail(e, "ternary_mma batch launch");
    }
  }
  return TERN_OK;
}

}  // namespace
}  // namespace tern

extern "C" {

tern_status tern_linear(const void* x_bf16, int64_t M, int64_t K, const void* packed,
                        const float* scales, const void* bias_bf16, int64_t N, void* y_bf16,
                        tern_stream_t stream) {
  return linear_impl(dense_args(tern_linear_args{x_bf16, packed, scales, bias_bf16, y_bf16, M, N, K}), tern_epilogue{},
                     stream);
}

tern_status tern_linear_act(const void* x_bf16, int64_t M, int64_t K, const void* packed,
                            const float* scales, const void* bias_bf16, int64_t N, int act, int64_t act_col0,
                            void* y_bf16, tern_stream_t stream) {
  tern_epilogue spec{};
  spec.act = act;
  spec.act_col0 = act_col0;
  return linear_impl(dense_args(tern_linear_args{x_bf16, packed, scales, bias_bf16, y_bf16, M, N, K}), spec, stream);
}

tern_status tern_linear_batch(const tern_linear_args* args, int count, tern_stream_t stream) {
  if (count < 0 || (count > 0 && !args)) return fail(TERN_ERR_INVALID_ARG, "bad count or null args");
  std::vector<LinArgs> lin(size_t(std::max(count, 0)));
  for (int i = 0; i < count; ++i) lin[i] = dense_args(args[i]);
  return batch_impl(lin.data(), nullptr, count, stream);
}

tern_status tern_linear_batch_act(const tern_linear_act_args* args, int count, tern_stream_t stream) {
  if (count < 0 || (count > 0 && !args)) return fail(TERN_ERR_INVALID_ARG, "bad count or null args");
  std::vector<LinArgs> lin(size_t(std::max(count, 0)));
  std::vector<tern_epilogue> epis(size_t(std::max(count, 0)));
  for (int i = 0; i < count; ++i) {
    lin[i] = dense_args(args[i].linear);
    epis[i] = tern_epilogue{};
    epis[i].act = args[i].act;
    epis[i].act_col0 = args[i].act_col0;
  }
  return batch_impl(lin.data(), epis.data(), count, stream);
}

tern_status tern_linear_epilogue(const tern_linear_args* args, const tern_epilogue* epilogue, tern_stream_t stream) {
  if (!args) return fail(TERN_ERR_INVALID_ARG, "null args");
  return linear_impl(dense_args(*args), epilogue ? *epilogue : tern_epilogue{}, stream);
}

tern_status tern_linear_batch_epilogue(const tern_linear_args* args, const tern_epilogue* epilogues, int count,
                                       tern_stream_t stream) {
  if (count < 0 || (count > 0 && !args)) return fail(TERN_ERR_INVALID_ARG, "bad count or null args");
  std::vector<LinArgs> lin(size_t(std::max(count, 0)));
  for (int i = 0; i < count; ++i) lin[i] = dense_args(args[i]);
  return batch_impl(lin.data(), epilogues, count, stream);
}

namespace {
LinArgs strided_args(const tern_linear_strided_args& a) {
  LinArgs l = dense_args(a.linear);
  l.ldx = a.ldx;
  l.ldy = a.ldy;
  return l;
}
}  // namespace

tern_status tern_linear_strided(const tern_linear_strided_args* args, const tern_epilogue* epilogue,
                                tern_stream_t stream) {
  if (!args) return fail(TERN_ERR_INVALID_ARG, "null args");
  return linear_impl(strided_args(*args), epilogue ? *epilogue : tern_epilogue{}, stream);
}

tern_status tern_linear_batch_strided(const tern_linear_strided_args* args, const tern_epilogue* epilogues,
                                      int count, tern_stream_t stream) {
  if (count < 0 || (count > 0 && !args)) return fail(TERN_ERR_INVALID_ARG, "bad count or null args");
  std::vector<LinArgs> lin(size_t(std::max(count, 0)));
  for (int i = 0; i < count; ++i) lin[i] = strided_args(args[i]);
  return batch_impl(lin.data(), epilogues, count, stream);
}

tern_status tern_dequantize(const void* packed, const float* scales, int64_t N, int64_t K,
                            void* W_bf16_out, tern_stream_t stream) {
  tern_status s = check_nk(N, K);
  if (s != TERN_OK) return s;
  if (!packed || !scales || !W_bf16_out) return fail(TERN_ERR_INVALID_ARG, "null pointer");
  if (!aligned(packed, 16) || !aligned(W_bf16_out, 16) || !aligned(scales, 4))
    return fail(TERN_ERR_MISALIGNED, "packed and output need 16-byte, scales 4-byte alignment");
  if (overlaps(W_bf16_out, size_t(N) * size_t(K) * 2, packed, packed_size(N, K)) ||
      overlaps(W_bf16_out, size_t(N) * size_t(K) * 2, scales, size_t(N) * 4))
    return fail(TERN_ERR_INVALID_ARG, "output overlaps an input");
  int dev;
  DeviceState* ds;
  if ((s = current_device(&dev, &ds)) != TERN_OK) return s;
  cudaError_t e = launch_dequantize(static_cast<const uint8_t*>(packed), scales, int(N), int(K),
                                    static_cast<__nv_bfloat16*>(W_bf16_out),
                                    reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "dequantize launch");
  return TERN_OK;
}

tern_status tern_quantize_act_e4m3(const void* x_bf16, int64_t M, int64_t K, void* xq, float* a,
                                   tern_stream_t stream) {
  if (M < 0 || K < 0) return fail(TERN_ERR_INVALID_ARG, "negative size M=%lld K=%lld", (long long)M, (long long)K);
  if (K == 0 || K % 64 != 0 || K > kMaxK || M > kMaxM)
    return fail(TERN_ERR_UNSUPPORTED_SHAPE, "quantize_act_e4m3: need K %% 64 == 0, K <= 2^20, M <= 2^26 (M=%lld K=%lld)",
                (long long)M, (long long)K);
  if (M == 0) return TERN_OK;
  if (!x_bf16 || !xq || !a) return fail(TERN_ERR_INVALID_ARG, "null x, xq or a");
  if (!aligned(x_bf16, 16) || !aligned(xq, 16) || !aligned(a, 4))
    return fail(TERN_ERR_MISALIGNED, "x and xq need 16-byte, a 4-byte alignment");
  const size_t xb = size_t(M) * size_t(K) * 2, qb = size_t(M) * size_t(K), ab = size_t(M) * 4;
  if (overlaps(xq, qb, x_bf16, xb) || overlaps(a, ab, x_bf16, xb) || overlaps(a, ab, xq, qb))
    return fail(TERN_ERR_INVALID_ARG, "outputs overlap each other or x");
  int dev;
  DeviceState* ds;
  tern_status s;
  if ((s = current_device(&dev, &ds)) != TERN_OK) return s;
  cudaError_t e = launch_quantize_act_e4m3(static_cast<const __nv_bfloat16*>(x_bf16), int(M), int(K),
                                           static_cast<uint8_t*>(xq), a, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "quantize_act_e4m3 launch");
  return TERN_OK;
}

tern_status tern_linear_e4m3(const void* xq, const float* a, int64_t M, int64_t K, const void* packed,
                             const float* scales, const void* bias_bf16, int64_t N, void* y_bf16,
                             tern_stream_t stream) {
  tern_status s = check_nk(N, K);
  if (s != TERN_OK) return s;
  if (N % 256 != 0) return fail(TERN_ERR_UNSUPPORTED_SHAPE, "linear_e4m3: need N %% 256 == 0, got N=%lld", (long long)N);
  if (M < 0) return fail(TERN_ERR_INVALID_ARG, "negative M=%lld", (long long)M);
  if (M > kMaxM) return fail(TERN_ERR_UNSUPPORTED_SHAPE, "M above 2^26 (M=%lld)", (long long)M);
  if (M == 0) return TERN_OK;
  if (!xq || !a || !packed || !scales || !y_bf16) return fail(TERN_ERR_INVALID_ARG, "null xq, a, packed, scales or y");
  if (!aligned(xq, 16) || !aligned(packed, 16) || !aligned(y_bf16, 16) || !aligned(scales, 4) || !aligned(a, 4) ||
      (bias_bf16 && !aligned(bias_bf16, 2)))
    return fail(TERN_ERR_MISALIGNED, "xq, packed and y need 16-byte, a and scales 4-byte, bias 2-byte alignment");
  const size_t yb = size_t(M) * size_t(N) * 2;
  if (overlaps(y_bf16, yb, xq, size_t(M) * size_t(K)) || overlaps(y_bf16, yb, a, size_t(M) * 4) ||
      overlaps(y_bf16, yb, packed, packed_size(N, K)) || overlaps(y_bf16, yb, scales, size_t(N) * 4) ||
      overlaps(y_bf16, yb, bias_bf16, bias_bf16 ? size_t(N) * 2 : 0))
    return fail(TERN_ERR_INVALID_ARG, "y overlaps an input");
  int dev;
  DeviceState* ds;
  if ((s = current_device(&dev, &ds)) != TERN_OK) return s;
  if (ds->clusters_2sm <= 0) return fail(TERN_ERR_NO_DEVICE, "the device cannot co-schedule CTA pairs");
  static Batch batch;  // built under the lock below; ~4 KiB, copied into the launch
  static std::mutex batch_mu;
  std::lock_guard<std::mutex> lock(batch_mu);
  std::memset(static_cast<void*>(&batch), 0, sizeof batch);
  Problem& p = batch.p[0];
  if ((s = make_xq_map(&p.tmap_x, xq, M, K)) != TERN_OK) return s;
  p.packed = static_cast<const uint8_t*>(packed);
  p.scales = scales;
  p.bias = static_cast<const __nv_bfloat16*>(bias_bf16);
  p.y = static_cast<__nv_bfloat16*>(y_bf16);
  p.ws = const_cast<float*>(a);  // the per-token scales
  p.M = int(M);
  p.N = int(N);
  p.K = int(K);
  p.ldy = int(N);
  p.n_tiles = int(N / 256);
  p.m_tiles = int((M + 255) / 256);
  p.splits = 1;
  p.chunks_per_split = int(K / 64);
  const int64_t tiles = int64_t(p.n_tiles) * p.m_tiles;
  if (tiles > (int64_t(1) << 31) - 1) return fail(TERN_ERR_UNSUPPORTED_SHAPE, "too many tiles");
  batch.count = 1;
  batch.total_units = int(tiles);
  batch.wait_limit_ns = g_wait_limit_ns.load();
  batch.status = ds->status;
  cudaError_t e = launch_ternary_fp8(batch, int(std::min<int64_t>(tiles, ds->clusters_2sm)),
                                     reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "ternary_fp8 launch");
  return TERN_OK;
}

tern_status tern_get_device_status(tern_stream_t stream) {
  int dev;
  DeviceState* ds;
  tern_status s = current_device(&dev, &ds);
  if (s != TERN_OK) return s;
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  unsigned int word = 0;
  if ((e = cudaMemcpy(&word, ds->status, sizeof word, cudaMemcpyDeviceToHost)) != cudaSuccess)
    return cuda_fail(e, "status read");
  if ((e = cudaMemset(ds->status, 0, sizeof word)) != cudaSuccess) return cuda_fail(e, "status clear");
  if (word & kStatusTimeout) {
    // A CTA that gave up may have left a split-K arrival counter non-zero;
    // zero them all so later calls start clean.
    std::lock_guard<std::mutex> lock(g_mu);
    for (auto& kv : g_ws)
      if (kv.first.first == dev && kv.second.counters) {
        if ((e = cudaDeviceSynchronize()) != cudaSuccess) return cuda_fail(e, "sync");
        if ((e = cudaMemset(kv.second.counters, 0, kv.second.n_counters * sizeof(int))) != cudaSuccess)
          return cuda_fail(e, "counter reset");
      }
    return fail(TERN_ERR_TIMEOUT, "a device-side wait ran out of time");
  }
  if (word & kStatusLaunchConfig)
    return fail(TERN_ERR_LAUNCH_CONFIG, "a kernel found its launch configuration inconsistent and computed nothing");
  return TERN_OK;
}

void tern_set_wait_limit_ns(uint64_t limit_ns) {
  g_wait_limit_ns.store(std::max<uint64_t>(limit_ns, 1000));
}

tern_status tern_selftest_wait_timeout(uint64_t limit_ns, tern_stream_t stream) {
  int dev;
  DeviceState* ds;
  tern_status s = current_device(&dev, &ds);
  if (s != TERN_OK) return s;
  if (limit_ns < 1000 || limit_ns > 10000000000ull)
    return fail(TERN_ERR_INVALID_ARG, "limit_ns must lie in [1e3, 1e10]");
  cudaError_t e = launch_wait_selftest(limit_ns, ds->status, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "selftest launch");
  return TERN_OK;
}

const char* tern_status_string(tern_status status) {
  switch (status) {
    case TERN_OK: return "ok";
    case TERN_ERR_INVALID_ARG: return "invalid argument";
    case TERN_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case TERN_ERR_MISALIGNED: return "misaligned pointer";
    case TERN_ERR_CUDA: return "CUDA error";
    case TERN_ERR_TIMEOUT: return "device wait timed out";
    case TERN_ERR_NO_DEVICE: return "no supported device";
    case TERN_ERR_LAUNCH_CONFIG: return "inconsistent kernel launch configuration";
  }
  return "unknown status";
}

const char* tern_last_error(void) { return t_last_error.c_str(); }

}  // extern "C"

// ---------------------------------------------------------------------------
// tern_linear_noalloc: the same ternary linear with its scratch in a fixed
// device array of this library, for callers that must not allocate device
// memory (see include/tern.h).  Only the split-K path of small M needs
// scratch (fp32 partial sums and per-tile arrival counters); here they live
// in g_noalloc_scratch instead of the per-(device, stream) workspace that
// tern_linear allocates on first use.
namespace tern {
namespace {

constexpr size_t kNoAllocPartialBytes = size_t(10) << 20;  // fp32 split-K partials
constexpr size_t kNoAllocCounters = 1024;                  // arrival counters (int)
constexpr size_t kNoAllocScratchBytes = kNoAllocPartialBytes + kNoAllocCounters * sizeof(int);

// One copy per GPU that loads the library, kept until the process exits.
// Host code must not use this name as a device address: the address comes
// from cudaGetSymbolAddress below, once per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

unsigned char* g_noalloc_ptr[kMaxDevices] = {};  // device address of the array, per device

// The device address of g_noalloc_scratch on `dev` (the current device),
// looked up on the first call for that device.
tern_status noalloc_scratch(int dev, unsigned char** out) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(no-alloc scratch)");
    g_noalloc_ptr[dev] = static_cast<unsigned char*>(p);
  }
  *out = g_noalloc_ptr[dev];
  return TERN_OK;
}

}  // namespace
}  // namespace tern

extern "C" tern_status tern_linear_noalloc(const void* x_bf16, int64_t M, int64_t K, const void* packed,
                                           const float* scales, const void* bias_bf16, int64_t N,
                                           void* y_bf16, tern_stream_t stream) {
  const LinArgs a = dense_args(tern_linear_args{x_bf16, packed, scales, bias_bf16, y_bf16, M, N, K});
  tern_status s = check_linear(a);
  if (s != TERN_OK) return s;
  if (M == 0) return TERN_OK;
  int dev;
  DeviceState* ds;
  if ((s = current_device(&dev, &ds)) != TERN_OK) return s;
  unsigned char* scratch = nullptr;
  if ((s = noalloc_scratch(dev, &scratch)) != TERN_OK) return s;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);

  static Batch batch;  // built under the lock below, copied into the launch
  static std::mutex batch_mu;
  std::lock_guard<std::mutex> lock(batch_mu);
  // Neither the small-M GEMV nor the pair-tile kernel needs scratch.
  if (M <= kGemvMaxM) return launch_gemv_group(&a, nullptr, std::vector<int>{0}, gemv_nt(M), batch, ds, cs);
  if (const int ptok = pair_tok(a, ds))
    return launch_2sm_group(&a, nullptr, std::vector<int>{0}, ptok, batch, ds, cs);

  // Same tile and split choice as tern_linear, so the two give identical y.
  const int tok = pick_tok(M);
  const int splits = fallback_splits(M, N, K, tok, ds);
  const int64_t tiles = n_slabs(N) * ((M + tok - 1) / tok);
  std::memset(static_cast<void*>(&batch), 0, sizeof batch);
  int64_t ctas = 0;
  if ((s = fill_problem(a, tok, splits, &batch.p[0], &ctas)) != TERN_OK) return s;
  Problem& p = batch.p[0];
  if (p.splits > 1) {
    const size_t need = size_t(p.splits) * size_t(tiles) * tok * 128 * sizeof(float);
    if (need > kNoAllocPartialBytes || size_t(tiles) > kNoAllocCounters)
      return fail(TERN_ERR_UNSUPPORTED_SHAPE,
                  "M=%lld N=%lld K=%lld needs %zu bytes of split-K partials and %lld counters; the "
                  "static scratch holds %zu bytes and %zu counters",
                  (long long)M, (long long)N, (long long)K, need, (long long)tiles, kNoAllocPartialBytes,
                  kNoAllocCounters);
    p.ws = reinterpret_cast<float*>(scratch);
    p.counters = reinterpret_cast<int*>(scratch + kNoAllocPartialBytes);
    // The array keeps whatever the previous call (or a timed-out one) left:
    // the arrival counters must start at zero.  The kernel resets each
    // counter it used, but a launch that failed or timed out may not have;
    // this clear on every call is what covers that case, so it stays even
    // though it is redundant after a clean launch.
    cudaError_t e = cudaMemsetAsync(p.counters, 0, size_t(tiles) * sizeof(int), cs);
    if (e != cudaSuccess) return cuda_fail(e, "no-alloc counter clear");
  }
  p.unit_begin = 0;
  batch.count = 1;
  batch.total_units = int(ctas);
  batch.wait_limit_ns = g_wait_limit_ns.load();
  batch.status = ds->status;
  cudaError_t e = launch_ternary_mma(tok, batch, cs);
  if (e != cudaSuccess) return cuda_fail(e, "ternary_mma launch (no-alloc)");
  return TERN_OK;
}
