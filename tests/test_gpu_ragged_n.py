"""Output widths N with N % 16 == 0 but N % 128 != 0 (FLUX.1's final
projection has N = 64), through the C ABI on the GPU against the fp64 oracle.

The packed layout keeps whole 128-channel slabs: the channels past N hold zero
codes and no scale, and no kernel stores them.  M <= 16 runs on the GEMV
kernel, M > 16 on the general tile kernel (split-K for M <= 64).  Same bars
as the other parity tests: codes bit-exact given the GPU's scales (near the
rounding threshold counted), the padding bytes zero, y within
8e-3 |y_ref| + 1e-3 rms(y_ref).
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


def bits(t: torch.Tensor) -> np.ndarray:
    return workloads.bf16_bits(t.detach().cpu())


def rand_bf16(shape, std, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * std).to(torch.bfloat16)


def quantize_checked(W: torch.Tensor):
    """GPU quantise/pack of W [N, K] with its codes checked against the oracle;
    returns (packed, scales, T) with T the codes the GPU wrote."""
    N, K = W.shape
    packed, scales = tern.quantize_pack(W.cuda(), EPS)
    torch.cuda.synchronize()
    assert tern.device_status() == 0
    P = packed.cpu().numpy()
    assert P.size == tern.packed_bytes(N, K) == oracle.tiled_bytes(N, K)
    s_gpu = scales.cpu().double().numpy()
    s_ref = oracle.absmean_scales(bits(W), EPS)
    assert np.max(np.abs(s_gpu - s_ref) / s_ref) <= 1e-6
    T, bad = oracle.unpack_tiled(P, N, K)
    assert bad == 0
    _, near = oracle.near_threshold(bits(W), s_gpu, 1e-6)
    assert not np.any((T != oracle.ternarize(bits(W), s_gpu)) & ~near)
    # every byte, the padding channels' zeros included
    assert np.array_equal(P, oracle.pack_tiled(T))
    return packed, scales, T


def check_y(y: torch.Tensor, y_ref: np.ndarray):
    a = y.detach().cpu().double().numpy()
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    bad = np.abs(a - y_ref) > Y_RTOL * np.abs(y_ref) + Y_RMS * rms
    assert not bad.any(), f"{int(bad.sum())} of {bad.size} outputs out of tolerance"


@pytest.mark.parametrize("N,K", [(16, 64), (64, 3072), (208, 256), (400, 1024)])
def test_quantize_ragged_n_bit_exact_with_zero_padding(N, K):
    quantize_checked(rand_bf16((N, K), 0.02, seed=N + K))


@pytest.mark.parametrize("M,N,K", [(1, 64, 3072), (5, 208, 256), (16, 64, 512), (17, 64, 3072), (40, 208, 1024),
                                   (64, 400, 256), (300, 64, 3072), (257, 208, 512)])
def test_linear_ragged_n(M, N, K):
    W = rand_bf16((N, K), 0.02, seed=3 * N + K)
    x = rand_bf16((M, K), 1.0, seed=M + 1)
    b = rand_bf16((N,), 0.01, seed=N + 2)
    packed, scales, T = quantize_checked(W)
    # y wider than N by a guard band: nothing past row M, column N may change
    guard = torch.full((M + 1, N), 7.0, dtype=torch.bfloat16, device="cuda")
    y = guard[:M]
    tern.linear(x.cuda(), packed, scales, b.cuda(), out=y)
    torch.cuda.synchronize()
    assert tern.device_status() == 0
    check_y(y, oracle.linear(bits(x), T, scales.cpu().double().numpy(), bits(b)))
    assert torch.all(guard[M] == 7.0)


@pytest.mark.parametrize("M", [4, 40, 300])
def test_linear_ragged_n_fused_epilogue(M):
    """GELU on the upper columns and a gated residual update in place at
    N = 208."""
    N, K, col0 = 208, 512, 96
    W = rand_bf16((N, K), 0.02, seed=M + 40)
    x = rand_bf16((M, K), 1.0, seed=M + 41)
    b = rand_bf16((N,), 0.01, seed=M + 42)
    r = rand_bf16((M, N), 0.5, seed=M + 43)
    g = rand_bf16((N,), 0.3, seed=M + 44)
    packed, scales, T = quantize_checked(W)
    ref = oracle.linear_epilogue(bits(x), T, scales.cpu().double().numpy(), bits(b), oracle.ACT_GELU_TANH, col0,
                                 bits(r), bits(g))
    rd = r.cuda()
    tern.linear_epilogue(x.cuda(), packed, scales, b.cuda(), act=tern.ACT_GELU_TANH, act_col0=col0, residual=rd,
                         gate=g.cuda(), out=rd)
    torch.cuda.synchronize()
    assert tern.device_status() == 0
    check_y(rd, ref)


def test_flux_final_projection_sampled():
    """FLUX.1's final projection at 1024x1024: 4096 tokens x 3072 -> 64
    channels; the oracle on 128 sampled rows."""
    M, N, K = 4096, 64, 3072
    W = rand_bf16((N, K), 0.02, seed=61)
    x = rand_bf16((M, K), 1.0, seed=62)
    b = rand_bf16((N,), 0.01, seed=63)
    packed, scales, T = quantize_checked(W)
    y = tern.linear(x.cuda(), packed, scales, b.cuda())
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(64).choice(M, 128, replace=False))
    ref = oracle.linear(bits(x[torch.from_numpy(rows)]), T, scales.cpu().double().numpy(), bits(b))
    check_y(y.cpu()[torch.from_numpy(rows)], ref)


def test_batch_mixes_ragged_and_whole_slab_widths():
    cases = [(3, 64, 256), (3, 256, 256), (48, 208, 512), (48, 384, 512)]
    probs, refs = [], []
    for i, (M, N, K) in enumerate(cases):
        W = rand_bf16((N, K), 0.02, seed=70 + i)
        x = rand_bf16((M, K), 1.0, seed=80 + i)
        b = rand_bf16((N,), 0.01, seed=90 + i)
        packed, scales, T = quantize_checked(W)
        probs.append(dict(x=x.cuda(), packed=packed, scales=scales, bias=b.cuda(),
                          y=torch.empty(M, N, dtype=torch.bfloat16, device="cuda")))
        refs.append(oracle.linear(bits(x), T, scales.cpu().double().numpy(), bits(b)))
    tern.linear_batch(probs)
    torch.cuda.synchronize()
    assert tern.device_status() == 0
    for p, ref in zip(probs, refs):
        check_y(p["y"], ref)
