"""fp64 CPU oracle for the ternary linear layer of "1.58-bit FLUX".

TEST INFRASTRUCTURE ONLY.  The test suite, the smoke check and the
benchmark's CPU-baseline leg are the only users; the product library never
imports, links or runs anything here.  The arithmetic lives in
``tern_oracle.c`` (plain C, IEEE double), which shares no code with the CUDA
library.  This module builds it with gcc on first use and marshals numpy
arrays through ctypes.

Functions (each follows page "1.58-bit FLUX", arXiv 2412.18653 HTML v1):

* ``quantize(W_bits, eps)`` -- absmean ternarisation per output channel
  (Section 1: weights in {-1, 0, +1}, "akin to BitNet b1.58"):
  ``s = mean|W| + eps``, ``T = RoundClip(W / s, -1, 1)``, ties to even.
* ``ternarize(W_bits, s)`` -- the same RoundClip with given scales, used to
  compare codes "given the scales" of another implementation.
* ``near_threshold(W_bits, s, band)`` -- elements with ``| |w|/s - 0.5 | <
  band``; the rounding decision there is not fixed by the scale's precision.
* ``pack_canonical / unpack_canonical`` -- 2-bit signed codes, four per byte,
  row-major (Section 1: "stored using 2-bit signed integers").
* ``pack_tiled / unpack_tiled`` -- the tile-interleaved device layout.
* ``linear(x_bits, T, s, b_bits)`` -- ``y = s * (x @ T^T) + b`` in double
  (Section 4: activations are not quantised).
* ``gelu_tanh(y, col0)``, ``linear_act(...)`` -- the tanh form of GELU on
  output columns [col0, N), the activation a fused epilogue of the MLP's
  first linear applies.  The pages quantise every linear of FLUX's blocks
  (Section 3.1) but do not describe the operations between them; this is
  FLUX.1's MLP activation, written from its definition.
* ``rms_norm_groups``, ``rotate_pairs``, ``linear_epilogue(...)`` -- the
  fused epilogues of FLUX.1's blocks: q/k RMS normalisation per head and
  their rotary embedding, the activation, and the gated residual update.
* ``adaln_modulate(x_bits, scale_bits, shift_bits, eps, tokens_per_row)`` --
  layer normalisation of each token row (no affine) modulated by a row of
  the adaLN modulation output: ``(x - mean) / sqrt(var + eps) * (1 + scale)
  + shift``, what FLUX.1's blocks feed to their first linears.  Like the
  epilogues, an operation between the quantised linears that the pages do
  not describe (Section 3.1), written from that model's definition.
* ``fp8_e4m3_rne``, ``fp8_e4m3_bits``, ``quantize_act_e4m3``,
  ``linear_act_e4m3`` -- the
  activation quantisation the pages name as the missing latency lever
  (Section 4): x per token row to FP8 E4M3 with an absmax scale, against the
  same exact ternary weights.  The pages fix no format or granularity; this
  is one reading, for a kernel that does not exist yet.

bf16 tensors are passed as their raw uint16 bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tern_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

_i64 = ctypes.c_int64
_ptr = ctypes.c_void_p


def build(force: bool = False) -> str:
    """Compile tern_oracle.c into liboracle.so (gcc, -O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fopenmp", "-fno-fast-math", "-fPIC", "-shared",
             _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.oracle_absmean_scales.argtypes = [_ptr, _i64, _i64, ctypes.c_double, _ptr]
        lib.oracle_ternarize.argtypes = [_ptr, _i64, _i64, _ptr, _ptr]
        lib.oracle_near_threshold.argtypes = [_ptr, _i64, _i64, _ptr, ctypes.c_double, _ptr]
        lib.oracle_near_threshold.restype = _i64
        lib.oracle_quantize.argtypes = [_ptr, _i64, _i64, ctypes.c_double, _ptr, _ptr]
        lib.oracle_pack_canonical.argtypes = [_ptr, _i64, _i64, _ptr]
        lib.oracle_unpack_canonical.argtypes = [_ptr, _i64, _i64, _ptr]
        lib.oracle_unpack_canonical.restype = ctypes.c_int
        lib.oracle_pack_tiled.argtypes = [_ptr, _i64, _i64, _ptr]
        lib.oracle_pack_tiled.restype = ctypes.c_int
        lib.oracle_unpack_tiled.argtypes = [_ptr, _i64, _i64, _ptr]
        lib.oracle_unpack_tiled.restype = ctypes.c_int
        lib.oracle_linear.argtypes = [_ptr, _i64, _i64, _ptr, _ptr, _ptr, _i64, _ptr]
        lib.oracle_gelu_tanh.argtypes = [_ptr, _i64, _i64, _i64]
        lib.oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    """Threads the oracle's parallel loop uses (OMP_NUM_THREADS or all cores)."""
    return int(_load().oracle_num_threads())


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float64 (for test-side use)."""
    u = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def absmean_scales(W_bits: np.ndarray, eps: float) -> np.ndarray:
    W_bits = _c(W_bits, np.uint16)
    N, K = W_bits.shape
    s = np.empty(N, np.float64)
    _load().oracle_absmean_scales(_p(W_bits), N, K, float(eps), _p(s))
    return s


def ternarize(W_bits: np.ndarray, s: np.ndarray) -> np.ndarray:
    W_bits = _c(W_bits, np.uint16)
    s = _c(s, np.float64)
    N, K = W_bits.shape
    T = np.empty((N, K), np.int8)
    _load().oracle_ternarize(_p(W_bits), N, K, _p(s), _p(T))
    return T


def near_threshold(W_bits: np.ndarray, s: np.ndarray, band: float = 1e-6):
    """Returns (count, boolean mask [N,K])."""
    W_bits = _c(W_bits, np.uint16)
    s = _c(s, np.float64)
    N, K = W_bits.shape
    mask = np.empty((N, K), np.uint8)
    cnt = _load().oracle_near_threshold(_p(W_bits), N, K, _p(s), float(band), _p(mask))
    return int(cnt), mask.astype(bool)


def quantize(W_bits: np.ndarray, eps: float):
    """Returns (T int8 [N,K], s float64 [N])."""
    W_bits = _c(W_bits, np.uint16)
    N, K = W_bits.shape
    T = np.empty((N, K), np.int8)
    s = np.empty(N, np.float64)
    _load().oracle_quantize(_p(W_bits), N, K, float(eps), _p(T), _p(s))
    return T, s


def pack_canonical(T: np.ndarray) -> np.ndarray:
    T = _c(T, np.int8)
    N, K = T.shape
    if K % 4:
        raise ValueError("K must be a multiple of 4")
    P = np.empty(N * K // 4, np.uint8)
    _load().oracle_pack_canonical(_p(T), N, K, _p(P))
    return P


def unpack_canonical(P: np.ndarray, N: int, K: int):
    """Returns (T, number of invalid codes)."""
    P = _c(P, np.uint8)
    T = np.empty((N, K), np.int8)
    bad = _load().oracle_unpack_canonical(_p(P), N, K, _p(T))
    return T, int(bad)


def tiled_bytes(N: int, K: int) -> int:
    """Size of the tiled layout: N rounded up to whole 128-channel slabs."""
    return -(-N // 128) * 128 * K // 4


def pack_tiled(T: np.ndarray) -> np.ndarray:
    """Tiled device layout of T [N, K] (N % 16 == 0, K % 64 == 0); channels
    past N up to the next multiple of 128 hold zero codes."""
    T = _c(T, np.int8)
    N, K = T.shape
    P = np.empty(tiled_bytes(N, K), np.uint8)
    if _load().oracle_pack_tiled(_p(T), N, K, _p(P)) != 0:
        raise ValueError("tiled layout needs N % 16 == 0 and K % 64 == 0")
    return P


def unpack_tiled(P: np.ndarray, N: int, K: int):
    """Returns (T, number of invalid codes)."""
    P = _c(P, np.uint8)
    if P.size < tiled_bytes(N, K):
        raise ValueError("packed buffer smaller than the tiled layout")
    T = np.empty((N, K), np.int8)
    bad = _load().oracle_unpack_tiled(_p(P), N, K, _p(T))
    if bad < 0:
        raise ValueError("tiled layout needs N % 16 == 0 and K % 64 == 0")
    return T, int(bad)


def linear(x_bits: np.ndarray, T: np.ndarray, s: np.ndarray, b_bits=None) -> np.ndarray:
    """y[m,n] = s_n * sum_k x[m,k] T[n,k] + b_n in float64, shape [M,N]."""
    x_bits = _c(x_bits, np.uint16)
    T = _c(T, np.int8)
    s = _c(s, np.float64)
    M, K = x_bits.shape
    N, K2 = T.shape
    if K2 != K or s.shape != (N,):
        raise ValueError("shape mismatch")
    bp = None
    if b_bits is not None:
        b_bits = _c(b_bits, np.uint16)
        if b_bits.shape != (N,):
            raise ValueError("bias shape mismatch")
        bp = _p(b_bits)
    y = np.empty((M, N), np.float64)
    _load().oracle_linear(_p(x_bits), M, K, _p(T), _p(s), bp, N, _p(y))
    return y


ACT_NONE = 0
ACT_GELU_TANH = 1


def gelu_tanh(y: np.ndarray, col0: int = 0) -> np.ndarray:
    """The tanh form of GELU on columns [col0, N) of a float64 [M, N] array
    (a new array; columns below col0 unchanged):
    g(v) = 0.5 v (1 + tanh(sqrt(2/pi) (v + 0.044715 v^3)))."""
    y = np.array(y, dtype=np.float64, order="C", copy=True)
    if y.ndim != 2:
        raise ValueError("y must be [M, N]")
    M, N = y.shape
    if not 0 <= col0 <= N:
        raise ValueError("col0 out of range")
    _load().oracle_gelu_tanh(_p(y), M, N, col0)
    return y


def linear_act(x_bits: np.ndarray, T: np.ndarray, s: np.ndarray, b_bits=None, act: int = ACT_NONE,
               col0: int = 0) -> np.ndarray:
    """``linear`` followed by the activation ``act`` on output columns
    [col0, N): the layer with a fused epilogue, in float64."""
    y = linear(x_bits, T, s, b_bits)
    if act == ACT_NONE:
        return y
    if act == ACT_GELU_TANH:
        return gelu_tanh(y, col0)
    raise ValueError("unknown activation")


def rms_norm_groups(y: np.ndarray, col0: int, col1: int, eps: float, w_bits=None, group: int = 128) -> np.ndarray:
    """RMS normalisation of every token row over each group of `group`
    consecutive columns in [col0, col1): v / sqrt(mean(v^2) + eps) * w[n]
    (w bf16 bit patterns [N], absent = 1); other columns unchanged.  FLUX.1
    normalises q and k per attention head (128 channels) this way."""
    y = np.array(y, dtype=np.float64, order="C", copy=True)
    M, N = y.shape
    if not (0 <= col0 <= col1 <= N and col0 % group == 0 and col1 % group == 0):
        raise ValueError("norm columns must be group-aligned within [0, N]")
    w = np.ones(N) if w_bits is None else bf16_bits_to_f64(_c(w_bits, np.uint16))
    for g0 in range(col0, col1, group):
        blk = y[:, g0:g0 + group]
        inv = 1.0 / np.sqrt(np.mean(blk * blk, axis=1, keepdims=True) + eps)
        y[:, g0:g0 + group] = blk * inv * w[None, g0:g0 + group]
    return y


def rotate_pairs(y: np.ndarray, col0: int, col1: int, cs: np.ndarray, group: int = 128) -> np.ndarray:
    """Rotary embedding of columns [col0, col1) of y [M, N]: in every group of
    `group` columns, channels (2j, 2j + 1) of row m become (a cos - b sin,
    a sin + b cos) with (cos, sin) = cs[m, j] (cs [M, group / 2, 2])."""
    y = np.array(y, dtype=np.float64, order="C", copy=True)
    cs = np.asarray(cs, dtype=np.float64)
    c, sn = cs[:, :, 0], cs[:, :, 1]
    for g0 in range(col0, col1, group):
        a = y[:, g0:g0 + group:2].copy()
        b = y[:, g0 + 1:g0 + group:2].copy()
        y[:, g0:g0 + group:2] = a * c - b * sn
        y[:, g0 + 1:g0 + group:2] = a * sn + b * c
    return y


def linear_epilogue(x_bits: np.ndarray, T: np.ndarray, s: np.ndarray, b_bits=None, act: int = ACT_NONE,
                    col0: int = 0, residual_bits=None, gate_bits=None, norm_cols=(0, 0), norm_w_bits=None,
                    norm_eps: float = 0.0, rope_cs=None) -> np.ndarray:
    """The layer with a fused epilogue, in float64: v = linear(...),
    RMS-normalised per 128-column group on norm_cols, a = act(v) on columns
    [col0, N), then residual + gate * a (residual [M, N] and gate [N] are bf16
    bit patterns; absent residual = 0, absent gate = 1).  FLUX.1 normalises
    q and k per head and adds its attention and MLP outputs to the residual
    stream scaled by an adaLN-Zero gate; the pages describe no operation
    between the quantised linears, so this follows that model's definition.
    rope_cs [M, 64, 2]: the rotary embedding of the normalised columns'
    channel pairs after the normalisation (FLUX.1 rotates q and k there)."""
    v = linear(x_bits, T, s, b_bits)
    if norm_cols[1] > norm_cols[0]:
        v = rms_norm_groups(v, norm_cols[0], norm_cols[1], norm_eps, norm_w_bits)
        if rope_cs is not None:
            v = rotate_pairs(v, norm_cols[0], norm_cols[1], rope_cs)
    if act == ACT_GELU_TANH:
        a = gelu_tanh(v, col0)
    elif act == ACT_NONE:
        a = v
    else:
        raise ValueError("unknown activation")
    if gate_bits is not None:
        g = bf16_bits_to_f64(_c(gate_bits, np.uint16))
        if g.shape != (a.shape[1],):
            raise ValueError("gate shape mismatch")
        a = a * g[None, :]
    if residual_bits is not None:
        r = bf16_bits_to_f64(_c(residual_bits, np.uint16))
        if r.shape != a.shape:
            raise ValueError("residual shape mismatch")
        a = r + a
    return a


def adaln_modulate(x_bits: np.ndarray, scale_bits: np.ndarray, shift_bits: np.ndarray, eps: float,
                   tokens_per_row=None) -> np.ndarray:
    """Layer normalisation of every token row of x [M, K] (mean and biased
    variance over K, no affine), then the adaLN modulation with row g =
    m // tokens_per_row of scale and shift [G, K]:
        out[m, k] = (x[m, k] - mean_m) / sqrt(var_m + eps) * (1 + scale[g, k]) + shift[g, k],
    in float64 over the exact bf16 inputs.  tokens_per_row None: every row
    uses scale[0] and shift[0]."""
    x = bf16_bits_to_f64(_c(x_bits, np.uint16))
    if x.ndim != 2:
        raise ValueError("x must be [M, K]")
    M, K = x.shape
    T = M if tokens_per_row is None else int(tokens_per_row)
    if T < 1:
        raise ValueError("tokens_per_row must be >= 1")
    G = max(1, -(-M // T))
    sc = bf16_bits_to_f64(_c(scale_bits, np.uint16)).reshape(-1, K)
    sh = bf16_bits_to_f64(_c(shift_bits, np.uint16)).reshape(-1, K)
    if sc.shape[0] < G or sh.shape[0] < G:
        raise ValueError("scale and shift need one row per group of tokens_per_row tokens")
    mean = x.mean(axis=1, keepdims=True)
    var = ((x - mean) ** 2).mean(axis=1, keepdims=True)
    v = (x - mean) / np.sqrt(var + eps)
    g = np.arange(M) // T
    return v * (1.0 + sc[g]) + sh[g]


E4M3_MAX = 448.0


def fp8_e4m3_rne(v) -> np.ndarray:
    """Nearest FP8 E4M3 value of each float64 (1 sign, 4 exponent bits with
    bias 7, 3 mantissa bits, subnormals down to 2^-9, no infinities), ties to
    even, magnitudes above 448 saturated to 448 (the finite-saturating
    conversion), as float64."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    _, ex = np.frexp(a)  # a = m 2^ex, 0.5 <= m < 1, so floor(log2 a) = ex - 1 exactly
    e = np.maximum(ex - 1, -6)  # below 2^-6 the spacing stays 2^-9
    q = np.ldexp(1.0, e - 3)  # spacing of the binade: 3 mantissa bits
    r = np.minimum(np.round(a / q) * q, E4M3_MAX)  # a / q is exact; np.round ties to even
    return np.copysign(r, v)


def quantize_act_e4m3(x_bits: np.ndarray):
    """Per token row m: a_m = max_k |x[m,k]| / 448 and v = x / a_m, both
    divisions in fp32 (the precision a kernel would decide in), then
    xq = E4M3(v).  A zero row gets a_m = 1 and zero codes.  Returns
    (xq [M, K] as float64 values, a [M] float64)."""
    x = bf16_bits_to_f64(_c(x_bits, np.uint16)).astype(np.float32)
    if x.ndim != 2:
        raise ValueError("x must be [M, K]")
    amax = np.max(np.abs(x), axis=1)
    a = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    v = (x / a[:, None]).astype(np.float32)
    return fp8_e4m3_rne(v.astype(np.float64)), a.astype(np.float64)


def linear_act_e4m3(x_bits: np.ndarray, T: np.ndarray, s: np.ndarray, b_bits=None) -> np.ndarray:
    """y[m,n] = a_m s_n sum_k xq[m,k] T[n,k] + b_n in float64 with the
    E4M3-quantised activations of ``quantize_act_e4m3``."""
    xq, a = quantize_act_e4m3(x_bits)
    T = _c(T, np.int8)
    s = _c(s, np.float64)
    if T.shape[1] != xq.shape[1] or s.shape != (T.shape[0],):
        raise ValueError("shape mismatch")
    acc = xq @ T.astype(np.float64).T  # exact: multiples of 2^-9 below 2^33
    y = acc * a[:, None] * s[None, :]
    if b_bits is not None:
        y = y + bf16_bits_to_f64(_c(b_bits, np.uint16))[None, :]
    return y


def fp8_e4m3_bits(v) -> np.ndarray:
    """The E4M3 byte of each value that is already an E4M3 value (as
    returned by ``fp8_e4m3_rne``): sign bit 7, biased exponent bits 3-6
    (bias 7; 0 for subnormals), mantissa bits 0-2.  -0 encodes as 0x80."""
    v = np.asarray(v, dtype=np.float64)
    if np.any(fp8_e4m3_rne(v) != v):
        raise ValueError("value not representable in E4M3")
    a = np.abs(v)
    _, ex = np.frexp(a)
    e = ex - 1  # floor(log2 a) for a > 0
    normal = a >= 2.0 ** -6
    exp_field = np.where(normal, e + 7, 0)
    mant = np.where(normal, a / np.ldexp(1.0, e) - 1.0, a / 2.0 ** -6) * 8.0
    bits = (np.signbit(v).astype(np.int64) << 7) | (exp_field.astype(np.int64) << 3) | mant.astype(np.int64)
    return bits.astype(np.uint8)
