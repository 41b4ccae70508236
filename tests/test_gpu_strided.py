"""Row-strided x and y (tern_linear_strided / tern_linear_batch_strided)
through the C ABI on the GPU, against the fp64 oracle.

Page "1.58-bit FLUX" (arXiv 2412.18653), Sections 1 and 3.1: the same ternary
layer; only where x is read from and y written to changes.  x is a column
slice of a wider activation, y a column slice of a wider output (a
concatenation buffer), and the elements of the parent tensors outside the
slices are canaries that must come back untouched.  Every kernel class is
covered: the M <= 16 GEMV (one and two 8-token blocks), the 64-token tcgen05
tiles, the CTA-pair tiles, and the single-CTA fallback (N % 256 != 0) with and
without split K; with the fused epilogues (GELU, in-place gated residual with
y's stride).  Bar: |y - y_ref| <= 8e-3 |y_ref| + 1e-3 rms(y_ref).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from bit_post_quantised_b200 import tern, workloads

pytestmark = pytest.mark.gpu

EPS = workloads.EPS
Y_RTOL = 8e-3
Y_RMS = 1e-3
CANARY = 7.0


def bits(t: torch.Tensor) -> np.ndarray:
    return workloads.bf16_bits(t.detach().cpu().contiguous())


def rand_bf16(shape, std, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * std).to(torch.bfloat16)


def check_y(y_gpu, y_ref):
    y = y_gpu.detach().cpu().double().numpy()
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    err = np.abs(y - y_ref)
    bad = err > Y_RTOL * np.abs(y_ref) + Y_RMS * rms
    assert not bad.any(), f"{int(bad.sum())} of {bad.size} out of tolerance; worst {err.max():.3e}"


def make_case(M, N, K, seed, x_pad=64, x_off=32, y_pad=128, y_off=64):
    W = rand_bf16((N, K), 0.02, seed)
    b = rand_bf16((N,), 0.01, seed + 2)
    packed, scales = tern.quantize_pack(W.cuda(), EPS)
    T, bad = oracle.unpack_tiled(packed.cpu().numpy(), N, K)
    assert bad == 0
    xbig = rand_bf16((M, K + x_pad), 1.0, seed + 1).cuda()
    x = xbig[:, x_off:x_off + K]
    ybig = torch.full((M, N + y_pad), CANARY, dtype=torch.bfloat16, device="cuda")
    y = ybig[:, y_off:y_off + N]
    return dict(x=x, packed=packed, scales=scales, bias=b.cuda(), y=y), (T, scales.cpu().double().numpy(), b), ybig, y_off


def canaries_intact(ybig, y_off, N):
    c = ybig.cpu()
    assert (c[:, :y_off] == CANARY).all() and (c[:, y_off + N:] == CANARY).all(), "wrote outside the y slice"


@pytest.mark.parametrize("M,N,K", [
    (1, 384, 320),      # GEMV, one 8-token block
    (12, 256, 448),     # GEMV, two 8-token blocks
    (40, 512, 256),     # 64-token tcgen05 tiles
    (300, 512, 192),    # CTA-pair tiles
    (70, 384, 128),     # fallback tiles (N % 256 != 0)
    (40, 384, 1024),    # fallback with split K
])
def test_strided_linear_matches_oracle(M, N, K):
    p, (T, s, b), ybig, y_off = make_case(M, N, K, seed=M + N + K)
    tern.linear_strided(p["x"], p["packed"], p["scales"], p["bias"], p["y"])
    torch.cuda.synchronize()
    assert tern.device_status() == 0
    check_y(p["y"], oracle.linear(bits(p["x"]), T, s, bits(b)))
    canaries_intact(ybig, y_off, N)


@pytest.mark.parametrize("M,N,K", [(5, 256, 192), (40, 512, 256), (300, 512, 192), (70, 384, 128)])
def test_strided_epilogue_residual_in_place_and_gelu(M, N, K):
    """GELU on the upper half of the columns and the gated residual update in
    place: the residual is the y slice itself (rows ldy apart)."""
    p, (T, s, b), ybig, y_off = make_case(M, N, K, seed=3 * M + N)
    r = rand_bf16((M, N), 1.0, M + N + 5)
    p["y"].copy_(r.cuda())
    g = rand_bf16((N,), 0.5, N + 9).cuda()
    col0 = N // 2
    tern.linear_strided(p["x"], p["packed"], p["scales"], p["bias"], p["y"], act=tern.ACT_GELU_TANH,
                        act_col0=col0, residual=p["y"], gate=g)
    torch.cuda.synchronize()
    assert tern.device_status() == 0
    ref = oracle.linear_epilogue(bits(p["x"]), T, s, bits(b), oracle.ACT_GELU_TANH, col0, bits(r), bits(g))
    check_y(p["y"], ref)
    canaries_intact(ybig, y_off, N)


def test_strided_batch_writes_a_concatenation_buffer():
    """A single FLUX block's output projection reads concat(attention, MLP):
    here one batch writes the two parts side by side into one [M, 3*128+512]
    buffer (two problems whose y are column slices of the same parent, rows
    equally strided), plus a GEMV and a pair-tile problem with their own
    strided x; each against the oracle."""
    M = 300
    parent = torch.full((M, 384 + 512 + 64), CANARY, dtype=torch.bfloat16, device="cuda")
    cases = []
    # attention-like part: columns [0, 384) ; MLP-like part with GELU: [384, 896)
    for i, (N, K, c0, act) in enumerate([(384, 256, 0, tern.ACT_NONE), (512, 192, 384, tern.ACT_GELU_TANH)]):
        W = rand_bf16((N, K), 0.02, 40 + i)
        packed, scales = tern.quantize_pack(W.cuda(), EPS)
        T, _ = oracle.unpack_tiled(packed.cpu().numpy(), N, K)
        xbig = rand_bf16((M, K + 64), 1.0, 50 + i).cuda()
        b = rand_bf16((N,), 0.01, 60 + i)
        p = dict(x=xbig[:, 64:], packed=packed, scales=scales, bias=b.cuda(), y=parent[:, c0:c0 + N], act=act)
        cases.append((p, T, scales.cpu().double().numpy(), b, act))
    # a GEMV problem and a pair-tile problem with strided x, dense y
    for i, (Mi, N, K) in enumerate([(3, 256, 192), (260, 256, 128)]):
        W = rand_bf16((N, K), 0.02, 70 + i)
        packed, scales = tern.quantize_pack(W.cuda(), EPS)
        T, _ = oracle.unpack_tiled(packed.cpu().numpy(), N, K)
        xbig = rand_bf16((Mi, K + 128), 1.0, 80 + i).cuda()
        b = rand_bf16((N,), 0.01, 90 + i)
        y = torch.empty(Mi, N, dtype=torch.bfloat16, device="cuda")
        p = dict(x=xbig[:, 128:], packed=packed, scales=scales, bias=b.cuda(), y=y, act=tern.ACT_NONE)
        cases.append((p, T, scales.cpu().double().numpy(), b, tern.ACT_NONE))
    tern.linear_batch_strided([c[0] for c in cases])
    torch.cuda.synchronize()
    assert tern.device_status() == 0
    for p, T, s, b, act in cases:
        ref = oracle.linear_act(bits(p["x"]), T, s, bits(b), act, 0)
        check_y(p["y"], ref)
    assert (parent[:, 896:].cpu() == CANARY).all()


def test_strided_with_dense_strides_is_the_plain_layer():
    """ldx = K and ldy = N: bit for bit tern_linear."""
    M, N, K = 300, 512, 256
    W = rand_bf16((N, K), 0.02, 1).cuda()
    x = rand_bf16((M, K), 1.0, 2).cuda()
    packed, scales = tern.quantize_pack(W, EPS)
    y1 = tern.linear(x, packed, scales)
    y2 = torch.empty_like(y1)
    tern.linear_strided(x, packed, scales, None, y2)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
