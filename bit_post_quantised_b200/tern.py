"""Python binding of libtern (include/tern.h): argument marshalling only.

Every step of the ternary linear path runs in the library's sm_100a kernels;
this module only turns torch tensors into pointers, sizes and the current
CUDA stream, calls the C ABI, and raises on a non-OK status.  There is no
fallback: if libtern.so is missing or the device is not an sm_100 GPU, the
calls fail loudly.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libtern.so")
_lib = None

TERN_OK = 0
STATUS_NAMES = {0: "TERN_OK", -1: "TERN_ERR_INVALID_ARG", -2: "TERN_ERR_UNSUPPORTED_SHAPE",
                -3: "TERN_ERR_MISALIGNED", -4: "TERN_ERR_CUDA", -5: "TERN_ERR_TIMEOUT",
                -6: "TERN_ERR_NO_DEVICE", -7: "TERN_ERR_LAUNCH_CONFIG"}

EXPORTED = ("tern_packed_bytes", "tern_quantize_pack", "tern_linear", "tern_linear_noalloc",
            "tern_linear_act", "tern_linear_epilogue", "tern_linear_batch", "tern_linear_batch_act",
            "tern_linear_batch_epilogue", "tern_linear_strided", "tern_linear_batch_strided",
            "tern_adaln_modulate", "tern_quantize_act_e4m3", "tern_linear_e4m3",
            "tern_dequantize", "tern_get_device_status", "tern_set_wait_limit_ns",
            "tern_selftest_wait_timeout", "tern_status_string", "tern_last_error")


class TernError(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {detail}")
        self.status = status


class LinearArgs(ctypes.Structure):
    """Mirror of tern_linear_args."""
    _fields_ = [("x", ctypes.c_void_p), ("packed", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("bias", ctypes.c_void_p), ("y", ctypes.c_void_p),
                ("M", ctypes.c_int64), ("N", ctypes.c_int64), ("K", ctypes.c_int64)]


class LinearActArgs(ctypes.Structure):
    """Mirror of tern_linear_act_args."""
    _fields_ = [("linear", LinearArgs), ("act", ctypes.c_int), ("act_col0", ctypes.c_int64)]


class LinearStridedArgs(ctypes.Structure):
    """Mirror of tern_linear_strided_args."""
    _fields_ = [("linear", LinearArgs), ("ldx", ctypes.c_int64), ("ldy", ctypes.c_int64)]


class Epilogue(ctypes.Structure):
    """Mirror of tern_epilogue."""
    _fields_ = [("act", ctypes.c_int), ("act_col0", ctypes.c_int64), ("residual", ctypes.c_void_p),
                ("gate", ctypes.c_void_p), ("norm_col0", ctypes.c_int64), ("norm_col1", ctypes.c_int64),
                ("norm_weight", ctypes.c_void_p), ("norm_eps", ctypes.c_float), ("rope_cs", ctypes.c_void_p)]


ACT_NONE = 0       # tern_act values
ACT_GELU_TANH = 1


def library_path() -> str:
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    """Loads libtern.so (raising if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise ImportError(f"libtern.so not found at {_LIB_PATH}; build it with "
                              "bit_post_quantised_b200._build.build()")
        L = ctypes.CDLL(_LIB_PATH)
        i64, vp, st = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int
        L.tern_packed_bytes.argtypes = [i64, i64]
        L.tern_packed_bytes.restype = ctypes.c_size_t
        L.tern_quantize_pack.argtypes = [vp, i64, i64, ctypes.c_float, vp, vp, vp]
        L.tern_quantize_pack.restype = st
        L.tern_linear.argtypes = [vp, i64, i64, vp, vp, vp, i64, vp, vp]
        L.tern_linear.restype = st
        L.tern_linear_noalloc.argtypes = [vp, i64, i64, vp, vp, vp, i64, vp, vp]
        L.tern_linear_noalloc.restype = st
        L.tern_linear_batch.argtypes = [ctypes.POINTER(LinearArgs), ctypes.c_int, vp]
        L.tern_linear_act.argtypes = [vp, i64, i64, vp, vp, vp, i64, ctypes.c_int, i64, vp, vp]
        L.tern_linear_act.restype = st
        L.tern_linear_batch_act.argtypes = [ctypes.POINTER(LinearActArgs), ctypes.c_int, vp]
        L.tern_linear_batch_act.restype = st
        L.tern_linear_epilogue.argtypes = [ctypes.POINTER(LinearArgs), ctypes.POINTER(Epilogue), vp]
        L.tern_linear_epilogue.restype = st
        L.tern_linear_batch_epilogue.argtypes = [ctypes.POINTER(LinearArgs), ctypes.POINTER(Epilogue), ctypes.c_int,
                                                 vp]
        L.tern_linear_batch_epilogue.restype = st
        L.tern_linear_strided.argtypes = [ctypes.POINTER(LinearStridedArgs), ctypes.POINTER(Epilogue), vp]
        L.tern_linear_strided.restype = st
        L.tern_linear_batch_strided.argtypes = [ctypes.POINTER(LinearStridedArgs), ctypes.POINTER(Epilogue),
                                                ctypes.c_int, vp]
        L.tern_linear_batch_strided.restype = st
        L.tern_linear_batch.restype = st
        L.tern_adaln_modulate.argtypes = [vp, i64, i64, vp, vp, i64, i64, ctypes.c_float, vp, vp]
        L.tern_adaln_modulate.restype = st
        L.tern_quantize_act_e4m3.argtypes = [vp, i64, i64, vp, vp, vp]
        L.tern_quantize_act_e4m3.restype = st
        L.tern_linear_e4m3.argtypes = [vp, vp, i64, i64, vp, vp, vp, i64, vp, vp]
        L.tern_linear_e4m3.restype = st
        L.tern_dequantize.argtypes = [vp, vp, i64, i64, vp, vp]
        L.tern_dequantize.restype = st
        L.tern_get_device_status.argtypes = [vp]
        L.tern_get_device_status.restype = st
        L.tern_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
        L.tern_set_wait_limit_ns.restype = None
        L.tern_selftest_wait_timeout.argtypes = [ctypes.c_uint64, vp]
        L.tern_selftest_wait_timeout.restype = st
        L.tern_status_string.argtypes = [st]
        L.tern_status_string.restype = ctypes.c_char_p
        L.tern_last_error.argtypes = []
        L.tern_last_error.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _check(status: int) -> None:
    if status != TERN_OK:
        raise TernError(status, lib().tern_last_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _empty(*shape, dtype, device, stream=None) -> torch.Tensor:
    """An output buffer allocated on the stream the call launches on, so that
    the caching allocator orders its reuse after that stream's work."""
    if stream is None:
        return torch.empty(*shape, dtype=dtype, device=device)
    with torch.cuda.stream(stream):
        return torch.empty(*shape, dtype=dtype, device=device)


def packed_bytes(N: int, K: int) -> int:
    return int(lib().tern_packed_bytes(N, K))


def quantize_pack(W: torch.Tensor, eps: float = 1e-5, packed: Optional[torch.Tensor] = None,
                  scales: Optional[torch.Tensor] = None, stream=None):
    """tern_quantize_pack: W bf16 [N,K] -> (packed uint8 [N*K/4], scales fp32 [N])."""
    N, K = W.shape
    if packed is None:
        packed = _empty(max(packed_bytes(N, K), 1), dtype=torch.uint8, device=W.device, stream=stream)
    if scales is None:
        scales = _empty(N, dtype=torch.float32, device=W.device, stream=stream)
    _check(lib().tern_quantize_pack(_ptr(W), N, K, float(eps), _ptr(packed), _ptr(scales),
                                    _stream(stream)))
    return packed, scales


def adaln_modulate(x: torch.Tensor, scale: torch.Tensor, shift: torch.Tensor, eps: float = 1e-6,
                   tokens_per_row: Optional[int] = None, mod_ld: Optional[int] = None,
                   out: Optional[torch.Tensor] = None, stream=None):
    """tern_adaln_modulate: out = LayerNorm(x) * (1 + scale[g]) + shift[g] per
    token row, g = row // tokens_per_row (default: every row uses row 0).
    scale and shift are bf16 with rows mod_ld elements apart (default: their
    own row stride), e.g. slices of the modulation output; out may be x."""
    M, K = x.shape
    T = M if tokens_per_row is None else int(tokens_per_row)
    if scale.stride(-1) != 1 or shift.stride(-1) != 1:
        raise ValueError("scale and shift rows must be contiguous")
    if mod_ld is None:
        mod_ld = scale.stride(0) if scale.dim() == 2 else K
        if shift.dim() == 2 and shift.stride(0) != mod_ld:
            raise ValueError("scale and shift rows must be the same distance apart")
    G = -(-M // max(T, 1)) if M else 0
    for name, t in (("scale", scale), ("shift", shift)):
        rows = t.shape[0] if t.dim() == 2 else 1
        if t.shape[-1] < K or (G and (G - 1) * int(mod_ld) + K > (rows - 1) * int(mod_ld) + t.shape[-1]):
            raise ValueError(f"{name} holds fewer than the {G} modulation rows of {K} values that "
                             f"{M} rows at {T} tokens per row need")
    if out is None:
        out = _empty(*x.shape, dtype=x.dtype, device=x.device, stream=stream)
    _check(lib().tern_adaln_modulate(_ptr(x), M, K, _ptr(scale), _ptr(shift), int(mod_ld), max(T, 1), float(eps),
                                     _ptr(out), _stream(stream)))
    return out


def _dense(*ts) -> None:
    """The dense entry points take row-major tensors without gaps; a view
    with a row stride goes through linear_strided / linear_batch_strided."""
    for t in ts:
        if t is not None and not t.is_contiguous():
            raise ValueError("x, y and residual must be dense row-major here; row-strided views go through "
                             "linear_strided / linear_batch_strided")


def linear(x: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor,
           bias: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None, stream=None):
    """tern_linear: y = (x . T^T) * s + b, x bf16 [M,K] -> y bf16 [M,N]."""
    M, K = x.shape
    N = scales.shape[0]
    if out is None:
        out = _empty(M, N, dtype=torch.bfloat16, device=x.device, stream=stream)
    _dense(x, out)
    _check(lib().tern_linear(_ptr(x), M, K, _ptr(packed), _ptr(scales), _ptr(bias), N, _ptr(out),
                             _stream(stream)))
    return out


def linear_noalloc(x: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor,
                   bias: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                   stream=None):
    """tern_linear_noalloc: tern_linear with its split-K scratch in the library's
    static device array (no device allocation by the library; `out` must be
    given by callers that cannot allocate)."""
    M, K = x.shape
    N = scales.shape[0]
    if out is None:
        out = _empty(M, N, dtype=torch.bfloat16, device=x.device, stream=stream)
    _dense(x, out)
    _check(lib().tern_linear_noalloc(_ptr(x), M, K, _ptr(packed), _ptr(scales), _ptr(bias), N,
                                     _ptr(out), _stream(stream)))
    return out


def linear_batch(problems: Sequence[dict], stream=None) -> None:
    """tern_linear_batch over dicts with keys x, packed, scales, bias (or None), y."""
    arr = (LinearArgs * max(1, len(problems)))()
    for i, p in enumerate(problems):
        _dense(p["x"], p["y"])
        M, K = p["x"].shape
        N = p["scales"].shape[0]
        arr[i] = LinearArgs(p["x"].data_ptr(), p["packed"].data_ptr(), p["scales"].data_ptr(),
                            None if p.get("bias") is None else p["bias"].data_ptr(),
                            p["y"].data_ptr(), M, N, K)
    _check(lib().tern_linear_batch(arr, len(problems), _stream(stream)))


def linear_act(x: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor,
               bias: Optional[torch.Tensor] = None, act: int = ACT_GELU_TANH, act_col0: int = 0,
               out: Optional[torch.Tensor] = None, stream=None):
    """tern_linear_act: the linear with `act` fused into its epilogue on
    output columns [act_col0, N)."""
    M, K = x.shape
    N = scales.shape[0]
    if out is None:
        out = _empty(M, N, dtype=torch.bfloat16, device=x.device, stream=stream)
    _dense(x, out)
    _check(lib().tern_linear_act(_ptr(x), M, K, _ptr(packed), _ptr(scales), _ptr(bias), N, act, act_col0,
                                 _ptr(out), _stream(stream)))
    return out


def linear_batch_act(problems: Sequence[dict], stream=None) -> None:
    """tern_linear_batch_act over dicts as linear_batch's plus act (default
    none) and act_col0 (default 0)."""
    arr = (LinearActArgs * max(1, len(problems)))()
    for i, p in enumerate(problems):
        _dense(p["x"], p["y"])
        M, K = p["x"].shape
        N = p["scales"].shape[0]
        arr[i] = LinearActArgs(LinearArgs(p["x"].data_ptr(), p["packed"].data_ptr(), p["scales"].data_ptr(),
                                          None if p.get("bias") is None else p["bias"].data_ptr(),
                                          p["y"].data_ptr(), M, N, K),
                               p.get("act", ACT_NONE), p.get("act_col0", 0))
    _check(lib().tern_linear_batch_act(arr, len(problems), _stream(stream)))


def _linear_args(p: dict) -> LinearArgs:
    _dense(p["x"], p["y"])
    M, K = p["x"].shape
    N = p["scales"].shape[0]
    return LinearArgs(p["x"].data_ptr(), p["packed"].data_ptr(), p["scales"].data_ptr(),
                      None if p.get("bias") is None else p["bias"].data_ptr(), p["y"].data_ptr(), M, N, K)


def _epilogue(p: dict, strided: bool = False) -> Epilogue:
    if not strided:
        _dense(p.get("residual"))
    rope = p.get("rope_cs")
    if rope is not None and (rope.dtype != torch.float32 or not rope.is_contiguous() or rope.shape[-2:] != (64, 2)
                             or rope.shape[0] < p["y"].shape[0]):
        raise ValueError("rope_cs must be contiguous fp32 [>= M, 64, 2] (cos, sin) pairs")
    return Epilogue(p.get("act", ACT_NONE), p.get("act_col0", 0), _ptr(p.get("residual")), _ptr(p.get("gate")),
                    p.get("norm_col0", 0), p.get("norm_col1", 0), _ptr(p.get("norm_weight")),
                    p.get("norm_eps", 0.0), _ptr(rope))


def linear_epilogue(x: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor,
                    bias: Optional[torch.Tensor] = None, act: int = ACT_NONE, act_col0: int = 0,
                    residual: Optional[torch.Tensor] = None, gate: Optional[torch.Tensor] = None,
                    norm_cols=(0, 0), norm_weight: Optional[torch.Tensor] = None, norm_eps: float = 0.0,
                    out: Optional[torch.Tensor] = None, stream=None, rope_cs: Optional[torch.Tensor] = None):
    """tern_linear_epilogue: y = residual + gate * act(norm(x . T^T * s + b))
    (see tern_epilogue); `out` may be `residual` itself for an in-place
    update; norm_cols = (first, end) of the RMS-normalised columns; rope_cs
    fp32 [M, 64, 2] (cos, sin) rotates the normalised columns' channel pairs."""
    M, K = x.shape
    N = scales.shape[0]
    if out is None:
        out = _empty(M, N, dtype=torch.bfloat16, device=x.device, stream=stream)
    a = _linear_args(dict(x=x, packed=packed, scales=scales, bias=bias, y=out))
    e = _epilogue(dict(act=act, act_col0=act_col0, residual=residual, gate=gate, norm_col0=norm_cols[0],
                       norm_col1=norm_cols[1], norm_weight=norm_weight, norm_eps=norm_eps, rope_cs=rope_cs, y=out))
    _check(lib().tern_linear_epilogue(ctypes.byref(a), ctypes.byref(e), _stream(stream)))
    return out


def linear_batch_epilogue(problems: Sequence[dict], stream=None) -> None:
    """tern_linear_batch_epilogue over dicts as linear_batch's plus the
    optional keys act, act_col0, residual, gate, norm_col0, norm_col1,
    norm_weight, norm_eps and rope_cs."""
    n = max(1, len(problems))
    args, epis = (LinearArgs * n)(), (Epilogue * n)()
    for i, p in enumerate(problems):
        args[i] = _linear_args(p)
        epis[i] = _epilogue(p)
    _check(lib().tern_linear_batch_epilogue(args, epis, len(problems), _stream(stream)))


def quantize_act_e4m3(x: torch.Tensor, xq: Optional[torch.Tensor] = None, a: Optional[torch.Tensor] = None,
                      stream=None):
    """tern_quantize_act_e4m3: x bf16 [M,K] -> (xq uint8 [M,K] E4M3 bytes in the
    interleaved k order of include/tern.h, a fp32 [M] per-token scales)."""
    M, K = x.shape
    if xq is None:
        xq = _empty(M, K, dtype=torch.uint8, device=x.device, stream=stream)
    if a is None:
        a = _empty(M, dtype=torch.float32, device=x.device, stream=stream)
    _check(lib().tern_quantize_act_e4m3(_ptr(x), M, K, _ptr(xq), _ptr(a), _stream(stream)))
    return xq, a


def linear_e4m3(xq: torch.Tensor, a: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor,
                bias: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None, stream=None):
    """tern_linear_e4m3: y = a_m * s_n * sum_k xq[m,k] T[n,k] + b_n -> bf16 [M,N]."""
    M, K = xq.shape
    N = scales.shape[0]
    if out is None:
        out = _empty(M, N, dtype=torch.bfloat16, device=xq.device, stream=stream)
    _check(lib().tern_linear_e4m3(_ptr(xq), _ptr(a), M, K, _ptr(packed), _ptr(scales), _ptr(bias), N, _ptr(out),
                                  _stream(stream)))
    return out


def _strided_args(p: dict) -> LinearStridedArgs:
    x, y = p["x"], p["y"]
    if x.stride(1) != 1 or y.stride(1) != 1:
        raise ValueError("x and y rows must be contiguous (stride 1 along the last dimension)")
    M, K = x.shape
    N = p["scales"].shape[0]
    lin = LinearArgs(x.data_ptr(), p["packed"].data_ptr(), p["scales"].data_ptr(),
                     None if p.get("bias") is None else p["bias"].data_ptr(), y.data_ptr(), M, N, K)
    return LinearStridedArgs(lin, x.stride(0), y.stride(0))


def linear_strided(x: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor, bias: Optional[torch.Tensor],
                   out: torch.Tensor, stream=None, **epilogue):
    """tern_linear_strided: x and out may be row-strided views (for instance
    column slices of wider tensors); their row strides are passed as ldx and
    ldy.  Keyword arguments are the epilogue's (act, act_col0, residual,
    gate, norm_col0, norm_col1, norm_weight, norm_eps); a residual has out's
    row stride."""
    a = _strided_args(dict(x=x, packed=packed, scales=scales, bias=bias, y=out))
    e = _epilogue(dict(epilogue, y=out), strided=True)
    _check(lib().tern_linear_strided(ctypes.byref(a), ctypes.byref(e), _stream(stream)))
    return out


def linear_batch_strided(problems: Sequence[dict], stream=None) -> None:
    """tern_linear_batch_strided over dicts as linear_batch_epilogue's, with x
    and y possibly row-strided views."""
    n = max(1, len(problems))
    args, epis = (LinearStridedArgs * n)(), (Epilogue * n)()
    for i, p in enumerate(problems):
        args[i] = _strided_args(p)
        epis[i] = _epilogue(p, strided=True)
    _check(lib().tern_linear_batch_strided(args, epis, len(problems), _stream(stream)))


def dequantize(packed: torch.Tensor, scales: torch.Tensor, K: int, out: Optional[torch.Tensor] = None,
               stream=None) -> torch.Tensor:
    """tern_dequantize: codes -> bf16 [N,K] with W'[n,k] = T[n,k] * s_n."""
    N = scales.shape[0]
    if out is None:
        out = _empty(N, K, dtype=torch.bfloat16, device=scales.device, stream=stream)
    _check(lib().tern_dequantize(_ptr(packed), _ptr(scales), N, K, _ptr(out), _stream(stream)))
    return out


def device_status(stream=None) -> int:
    """tern_get_device_status (synchronises the stream); returns the raw status."""
    return int(lib().tern_get_device_status(_stream(stream)))


def set_wait_limit_ns(limit_ns: int) -> None:
    lib().tern_set_wait_limit_ns(int(limit_ns))


def selftest_wait_timeout(limit_ns: int, stream=None) -> None:
    _check(lib().tern_selftest_wait_timeout(int(limit_ns), _stream(stream)))


def status_string(status: int) -> str:
    return lib().tern_status_string(int(status)).decode()
