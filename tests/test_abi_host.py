"""Host-side checks of the C ABI that need no GPU.

The library must load, export every entry point include/tern.h declares, and
reject every invalid call on the host with the documented status before
anything is launched.  Pointers here are fake addresses: every call below is
invalid in at least one way, so nothing is ever dereferenced or launched.
"""
from __future__ import annotations

import ctypes
import os
import re
import subprocess
import sys

import pytest
import torch

from bit_post_quantised_b200 import _build, tern

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

OK, INVALID, SHAPE, MISALIGNED = 0, -1, -2, -3


@pytest.fixture(scope="module")
def L():
    _build.build()
    return tern.lib()


def declared_entry_points():
    text = open(os.path.join(ROOT, "include", "tern.h")).read()
    return re.findall(r"^TERN_API\s+[^;(]*?\b(tern_\w+)\s*\(", text, flags=re.M)


def test_header_declares_the_boundary():
    names = declared_entry_points()
    for required in ("tern_quantize_pack", "tern_linear", "tern_linear_batch"):
        assert required in names
    assert set(names) == set(tern.EXPORTED)


def test_library_exports_every_declared_symbol(L):
    out = subprocess.check_output(["nm", "-D", "--defined-only", tern.library_path()], text=True)
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    for name in declared_entry_points():
        assert name in exported, name
        assert hasattr(L, name)


def test_packed_bytes(L):
    assert tern.packed_bytes(9216, 3072) == 9216 * 3072 // 4
    assert tern.packed_bytes(128, 64) == 2048
    # N % 16 == 0 but not % 128: whole 128-channel slabs (FLUX.1's 64-channel final projection)
    assert tern.packed_bytes(64, 3072) == 128 * 3072 // 4
    assert tern.packed_bytes(208, 128) == 256 * 128 // 4
    for N, K in [(0, 64), (128, 0), (100, 64), (8, 64), (128, 48), (-128, 64), (1 << 21, 64)]:
        assert tern.packed_bytes(N, K) == 0


def test_status_strings(L):
    assert tern.status_string(0) == "ok"
    assert "timed out" in tern.status_string(-5)
    assert "launch configuration" in tern.status_string(-7)
    assert tern.status_string(123) == "unknown status"


F = 0x7F0000000000  # a fake, 256-byte aligned address that is never dereferenced


def call_linear(L, x=F, M=16, K=256, packed=F + 0x100000, scales=F + 0x200000, bias=None, N=256,
                y=F + 0x300000):
    return L.tern_linear(ctypes.c_void_p(x), M, K, ctypes.c_void_p(packed), ctypes.c_void_p(scales),
                         None if bias is None else ctypes.c_void_p(bias), N, ctypes.c_void_p(y), None)


@pytest.mark.parametrize("kw,expected", [
    (dict(N=100), SHAPE), (dict(K=100), SHAPE), (dict(N=0), SHAPE), (dict(K=0), SHAPE),
    (dict(N=-128), INVALID), (dict(M=-1), INVALID), (dict(N=1 << 21), SHAPE), (dict(M=1 << 27), SHAPE),
    (dict(x=0), INVALID), (dict(packed=0), INVALID), (dict(scales=0), INVALID), (dict(y=0), INVALID),
    (dict(x=F + 2), MISALIGNED), (dict(packed=F + 0x100008), MISALIGNED), (dict(y=F + 0x300004), MISALIGNED),
    (dict(scales=F + 0x200002), MISALIGNED), (dict(bias=F + 0x400001), MISALIGNED),
    (dict(y=F), INVALID),                 # y aliases x
    (dict(y=F + 0x100000), INVALID),      # y aliases packed
    (dict(bias=F + 0x300010), INVALID),   # bias inside y
])
def test_linear_rejects_on_host(L, kw, expected):
    assert call_linear(L, **kw) == expected
    assert L.tern_last_error().decode() != ""


def test_quantize_rejects_on_host(L):
    q = lambda W=F, N=256, K=256, eps=1e-5, P=F + 0x1000000, S=F + 0x2000000: L.tern_quantize_pack(
        ctypes.c_void_p(W), N, K, eps, ctypes.c_void_p(P), ctypes.c_void_p(S), None)
    assert q(N=200) == SHAPE
    assert q(K=32) == SHAPE
    assert q(W=0) == INVALID
    assert q(eps=-1.0) == INVALID
    assert q(eps=float("nan")) == INVALID
    assert q(eps=float("inf")) == INVALID
    assert q(W=F + 8) == MISALIGNED
    assert q(S=F + 0x2000001) == MISALIGNED
    assert q(P=F + 0x10) == INVALID  # packed overlaps W


def test_batch_rejects_on_host(L):
    arr = (tern.LinearArgs * 2)()
    arr[0] = tern.LinearArgs(F, F + 0x100000, F + 0x200000, None, F + 0x300000, 16, 256, 256)
    arr[1] = tern.LinearArgs(F, F + 0x100000, F + 0x200000, None, F + 0x300000, 16, 100, 256)
    assert L.tern_linear_batch(arr, 2, None) == SHAPE
    assert "problem 1" in L.tern_last_error().decode()
    assert L.tern_linear_batch(arr, -1, None) == INVALID
    assert L.tern_linear_batch(None, 3, None) == INVALID


def test_dequantize_rejects_on_host(L):
    d = lambda P=F, S=F + 0x100000, N=256, K=256, O=F + 0x200000: L.tern_dequantize(
        ctypes.c_void_p(P), ctypes.c_void_p(S), N, K, ctypes.c_void_p(O), None)
    assert d(N=12) == SHAPE
    assert d(P=0) == INVALID
    assert d(O=F + 2) == MISALIGNED
    assert d(O=F) == INVALID


def test_selftest_rejects_bad_limit_without_gpu(L):
    # no GPU here: the device check fails before any launch
    import torch
    if torch.cuda.is_available():
        pytest.skip("host-only check")
    assert L.tern_selftest_wait_timeout(10, None) != OK


def test_binding_fails_loudly_without_library(tmp_path):
    code = ("import bit_post_quantised_b200.tern as t; t._LIB_PATH = '/nonexistent/libtern.so'\n"
            "try:\n    t.packed_bytes(128, 64)\nexcept ImportError as e:\n    print('LOUD', e)\n")
    out = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True)
    assert "LOUD" in out.stdout, out.stderr


def test_linear_with_no_tokens_is_a_host_noop(L):
    assert call_linear(L, M=0, x=0, y=0) == OK


def test_linear_act_rejects_on_host(L):
    """Unknown activations and activated-column starts outside [0, N] are
    refused before any device work; the other checks are tern_linear's."""
    def call(act, col0, N=256, y=F + 0x300000):
        return L.tern_linear_act(ctypes.c_void_p(F), 16, 256, ctypes.c_void_p(F + 0x100000),
                                 ctypes.c_void_p(F + 0x200000), None, N, act, col0, ctypes.c_void_p(y), None)
    assert call(7, 0) == INVALID
    assert call(-1, 0) == INVALID
    assert call(tern.ACT_GELU_TANH, -1) == INVALID
    assert call(tern.ACT_GELU_TANH, 257) == INVALID
    assert call(tern.ACT_GELU_TANH, 0, N=100) == SHAPE
    assert call(tern.ACT_GELU_TANH, 0, y=F + 0x300004) == MISALIGNED
    # M = 0 is a no-op that still validates the activation
    assert L.tern_linear_act(None, 0, 256, ctypes.c_void_p(F), ctypes.c_void_p(F + 0x100000), None, 256,
                             tern.ACT_GELU_TANH, 256, None, None) == 0
    assert L.tern_linear_act(None, 0, 256, ctypes.c_void_p(F), ctypes.c_void_p(F + 0x100000), None, 256,
                             5, 0, None, None) == INVALID


def test_batch_act_rejects_on_host(L):
    arr = (tern.LinearActArgs * 2)()
    ok = tern.LinearArgs(F, F + 0x100000, F + 0x200000, None, F + 0x300000, 16, 256, 256)
    arr[0] = tern.LinearActArgs(ok, tern.ACT_GELU_TANH, 128)
    arr[1] = tern.LinearActArgs(ok, tern.ACT_GELU_TANH, 300)
    assert L.tern_linear_batch_act(arr, 2, None) == INVALID
    assert b"problem 1" in L.tern_last_error()
    assert L.tern_linear_batch_act(arr, 0, None) == 0
    assert L.tern_linear_batch_act(None, 1, None) == INVALID


def test_epilogue_rejects_on_host(L):
    """Residual and gate checks of tern_linear_epilogue, before any device work."""
    a = tern.LinearArgs(F, F + 0x100000, F + 0x200000, None, F + 0x300000, 16, 256, 256)
    y_bytes = 16 * 256 * 2

    def call(**kw):
        e = tern.Epilogue(kw.get("act", 0), kw.get("col0", 0), kw.get("residual"), kw.get("gate"))
        return L.tern_linear_epilogue(ctypes.byref(a), ctypes.byref(e), None)
    assert call(residual=F + 0x300000 + 2) == INVALID        # partial overlap with y
    assert call(residual=F + 0x300000 - y_bytes + 2) == INVALID
    assert call(residual=F + 0x500001) == MISALIGNED
    assert call(gate=F + 0x500001) == MISALIGNED
    assert call(gate=F + 0x300000 + 64) == INVALID           # gate inside y
    assert call(act=3) == INVALID
    assert L.tern_linear_epilogue(None, None, None) == INVALID
    assert L.tern_linear_batch_epilogue(None, None, 2, None) == INVALID
    assert L.tern_linear_batch_epilogue(None, None, 0, None) == 0


def test_norm_epilogue_rejects_on_host(L):
    """The RMS-normalising epilogue: 128-aligned column bounds within [0, N],
    eps > 0, and only shapes that run on the tcgen05 tile kernels."""
    def call(M=40, N=256, c0=0, c1=128, eps=1e-6, w=None):
        a = tern.LinearArgs(F, F + 0x100000, F + 0x200000, None, F + 0x300000, M, N, 256)
        e = tern.Epilogue(0, 0, None, None, c0, c1, w, eps)
        return L.tern_linear_epilogue(ctypes.byref(a), ctypes.byref(e), None)
    assert call(c0=64) == INVALID
    assert call(c1=384) == INVALID
    assert call(c0=128, c1=0) == INVALID
    assert call(eps=0.0) == INVALID
    assert call(eps=float("nan")) == INVALID
    assert call(w=F + 0x500001) == MISALIGNED
    assert call(M=16) == SHAPE            # would run on the GEMV
    assert call(N=384, c1=128) == SHAPE   # would run on the fallback kernel


def test_rope_epilogue_rejects_on_host(L):
    """The rotary table: only with a normalisation, no activation, residual or
    gate on the normalised columns, 8-byte aligned, not overlapping y."""
    def call(c1=256, act=0, col0=0, residual=None, gate=None, rope=F + 0x600000):
        a = tern.LinearArgs(F, F + 0x100000, F + 0x200000, None, F + 0x300000, 40, 512, 256)
        e = tern.Epilogue(act, col0, residual, gate, 0, c1, None, 1e-6, rope)
        return L.tern_linear_epilogue(ctypes.byref(a), ctypes.byref(e), None)
    assert call(c1=0) == INVALID                     # nothing normalised
    assert call(act=1, col0=128) == INVALID          # GELU on normalised columns
    assert call(residual=F + 0x700000) == INVALID
    assert call(gate=F + 0x700000) == INVALID
    assert call(rope=F + 0x600004) == MISALIGNED
    assert call(rope=F + 0x300000 + 512) == INVALID  # inside y
    assert call(act=1, col0=256, rope=F + 0x600004) == MISALIGNED  # GELU past the normalised columns is fine


def test_adaln_rejects_on_host(L):
    """tern_adaln_modulate's shape, alignment and overlap checks, before any
    device work; M = 0 is a successful no-op."""
    x, sc, sh, out = F, F + 0x100000, F + 0x200000, F + 0x300000

    def call(M=16, K=256, scale=sc, shift=sh, ld=256, T=16, eps=1e-6, o=out, xx=x):
        return L.tern_adaln_modulate(xx, M, K, scale, shift, ld, T, eps, o, None)
    assert call(K=100) == SHAPE            # K % 8
    assert call(K=8192, ld=8192) == SHAPE  # longer than a row in registers
    assert call(ld=200) == SHAPE           # mod_ld < K
    assert call(ld=260) == SHAPE           # mod_ld % 8
    assert call(T=0) == SHAPE
    assert call(M=-1) == INVALID
    assert call(eps=-1.0) == INVALID and call(eps=float("inf")) == INVALID
    assert call(xx=None) == INVALID and call(scale=None) == INVALID
    assert call(xx=x + 8) == MISALIGNED and call(shift=sh + 2) == MISALIGNED and call(o=out + 4) == MISALIGNED
    assert call(o=x + 16) == INVALID       # partial overlap with x
    assert call(o=sc - 16 * 256 * 2 + 16) == INVALID  # out runs into scale
    assert call(M=0) == 0


def test_batch_rejects_cross_problem_overlaps_on_host(L):
    """Problems of a batch run concurrently: one problem's y may not overlap
    another problem's x, codes, residual or y (all rejected before any
    device work)."""
    M, N, K = 16, 256, 256
    yb = M * N * 2

    def args(x1=F + 0x400000, y1=F + 0x500000, p1=F + 0x100000):
        arr = (tern.LinearArgs * 2)()
        arr[0] = tern.LinearArgs(F, F + 0x100000, F + 0x200000, None, F + 0x300000, M, N, K)
        arr[1] = tern.LinearArgs(x1, p1, F + 0x200000, None, y1, M, N, K)
        return arr
    assert L.tern_linear_batch(args(y1=F + 0x300000 + yb - 64), 2, None) == INVALID  # y1 runs into y0
    assert L.tern_linear_batch(args(x1=F + 0x300000), 2, None) == INVALID  # x1 is y0
    assert L.tern_linear_batch(args(p1=F + 0x500000 - 0x100), 2, None) == INVALID  # codes 1 overlap y1 (own check)
    eps = (tern.Epilogue * 2)()
    eps[1] = tern.Epilogue(0, 0, F + 0x300000, None)  # problem 1's residual is problem 0's y
    assert L.tern_linear_batch_epilogue(args(), eps, 2, None) == INVALID


def test_adaln_binding_checks_row_layout():
    """The binding passes scale and shift as rows mod_ld apart: rows that are
    not contiguous, or scale and shift rows spaced differently, are refused
    before the library is called."""
    x = torch.zeros(4, 64, dtype=torch.bfloat16)
    mod = torch.zeros(2, 6 * 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        tern.adaln_modulate(x, mod[:, 64:128].t().contiguous().t(), mod[:, :64])  # columns strided
    with pytest.raises(ValueError):
        tern.adaln_modulate(x, mod[:, 64:128], torch.zeros(2, 64, dtype=torch.bfloat16))  # 384 vs 64 apart


def test_quantize_act_e4m3_rejects_on_host(L):
    q = lambda x=F, M=16, K=256, xq=F + 0x1000000, a=F + 0x2000000: L.tern_quantize_act_e4m3(
        ctypes.c_void_p(x), M, K, ctypes.c_void_p(xq), ctypes.c_void_p(a), None)
    assert q(K=100) == SHAPE
    assert q(K=0) == SHAPE
    assert q(M=-1) == INVALID
    assert q(M=1 << 27) == SHAPE
    assert q(x=0) == INVALID
    assert q(a=0) == INVALID
    assert q(x=F + 2) == MISALIGNED
    assert q(xq=F + 0x1000008) == MISALIGNED
    assert q(a=F + 0x2000002) == MISALIGNED
    assert q(xq=F + 0x100) == INVALID   # xq overlaps x
    assert q(a=F + 0x1000010) == INVALID  # a overlaps xq
    assert q(M=0, x=0, xq=0, a=0) == OK  # empty: nothing to do, nothing checked


def test_linear_e4m3_rejects_on_host(L):
    f = lambda xq=F, a=F + 0x80000, M=16, K=256, P=F + 0x100000, S=F + 0x200000, b=None, N=256, y=F + 0x300000: \
        L.tern_linear_e4m3(ctypes.c_void_p(xq), ctypes.c_void_p(a), M, K, ctypes.c_void_p(P), ctypes.c_void_p(S),
                           None if b is None else ctypes.c_void_p(b), N, ctypes.c_void_p(y), None)
    assert f(N=128) == SHAPE      # the FP8 kernel tiles 256 channels per CTA pair
    assert f(N=100) == SHAPE
    assert f(K=96) == SHAPE
    assert f(M=-1) == INVALID
    assert f(a=0) == INVALID
    assert f(xq=0) == INVALID
    assert f(xq=F + 4) == MISALIGNED
    assert f(a=F + 0x80002) == MISALIGNED
    assert f(y=F + 0x300008) == MISALIGNED
    assert f(y=F) == INVALID          # y aliases xq
    assert f(y=F + 0x80000) == INVALID  # y aliases a
    assert f(M=0, xq=0, a=0, y=0) == OK


PASSES = "passes"  # accepted by every host-side check


def _no_gpu() -> bool:
    return not torch.cuda.is_available()


def call_strided(L, x=F, ldx=256, M=16, K=256, packed=F + 0x1000000, scales=F + 0x2000000, bias=None, N=256,
                 y=F + 0x3000000, ldy=256, residual=None):
    a = tern.LinearStridedArgs(tern.LinearArgs(x, packed, scales, bias, y, M, N, K), ldx, ldy)
    e = tern.Epilogue(0, 0, residual, None, 0, 0, None, 0.0)
    return L.tern_linear_strided(ctypes.byref(a), ctypes.byref(e), None)


@pytest.mark.parametrize("kw,expected", [
    (dict(ldx=128), INVALID), (dict(ldy=200), INVALID), (dict(ldx=260), INVALID), (dict(ldy=268), INVALID),
    (dict(ldx=(1 << 30) + 8), INVALID),
    # y rows interleaved with x rows of one parent tensor (equal strides, disjoint columns): passes the host checks
    (dict(x=F, y=F + 512, ldx=512, ldy=512, N=256), PASSES),
    # ... but the columns overlap by one 16-byte group
    (dict(x=F, y=F + 496, ldx=512, ldy=512, N=256), INVALID),
    # different strides whose spans intersect: rejected
    (dict(x=F, y=F + 512, ldx=512, ldy=768, N=256), INVALID),
    # a residual with y's stride in the other half of each row of y's parent: fine; inside y's columns: not
    (dict(y=F + 0x3000000, ldy=512, residual=F + 0x3000000 + 512), PASSES),
    (dict(y=F + 0x3000000, ldy=512, residual=F + 0x3000000 + 256), INVALID),
])
def test_strided_linear_checks_on_host(L, kw, expected):
    if expected == PASSES:
        # The fake pointers must never reach a launch: only where no GPU can
        # run one does the call get past the host checks (to the device query).
        if not _no_gpu():
            pytest.skip("a call that passes the host checks would launch on this machine's GPU")
        assert call_strided(L, **kw) in (-4, -6)  # TERN_ERR_CUDA / TERN_ERR_NO_DEVICE from the device query
    else:
        assert call_strided(L, **kw) == expected


@pytest.mark.parametrize("T,rows", [(1000, 2), (2303, 2), (4607, 1), (1, 4607)])
def test_adaln_binding_checks_modulation_rows(T, rows):
    """The binding refuses scale/shift views with fewer modulation rows than
    ceil(M / tokens_per_row) before anything reaches the library (the C ABI
    sees only pointers and cannot).  Host tensors: nothing is launched."""
    M, K = 4608, 3072
    x = torch.zeros(M, K, dtype=torch.bfloat16)
    mod = torch.zeros(rows, 6 * K, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="modulation rows"):
        tern.adaln_modulate(x, mod[:, K:2 * K], mod[:, :K], 1e-6, tokens_per_row=T)


C_CLIENT = r"""
#include <stdio.h>
#include <string.h>
#include "tern.h"

int main(void) {
  /* host-only calls: no device memory is touched */
  size_t bytes = tern_packed_bytes(9216, 3072);
  uintptr_t f = (uintptr_t)0x7F0000000000ull;  /* never dereferenced */
  tern_status s = tern_linear((const void*)f, 16, 100, (const void*)(f + 0x100000),
                              (const float*)(f + 0x200000), NULL, 256, (void*)(f + 0x300000), NULL);
  printf("%zu %d %s|%s\n", bytes, (int)s, tern_status_string(s), tern_last_error());
  return (bytes == (size_t)9216 * 3072 / 4 && s == TERN_ERR_UNSUPPORTED_SHAPE) ? 0 : 1;
}
"""


def test_header_compiles_as_c_and_links(tmp_path, L):
    """A plain C99 client of include/tern.h, built with gcc against libtern.so
    (no CUDA headers, no C++): the boundary is usable from C.  It calls only
    host-side paths (the packed size and a shape the library refuses before
    any CUDA call)."""
    src = tmp_path / "client.c"
    src.write_text(C_CLIENT)
    exe = tmp_path / "client"
    libdir = os.path.dirname(tern.library_path())
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I",
                           os.path.join(ROOT, "include"), str(src), "-o", str(exe), "-L", libdir, "-ltern",
                           f"-Wl,-rpath,{libdir}"])
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout + out.stderr
    bytes_, status, rest = out.stdout.split(" ", 2)
    assert int(bytes_) == 9216 * 3072 // 4 and int(status) == -2
    assert "K" in rest.split("|", 1)[1]  # the message names the failing dimension
