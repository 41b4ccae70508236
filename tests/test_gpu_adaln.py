"""tern_adaln_modulate against the fp64 oracle, through the C ABI on the GPU.

out = (x - mean) / sqrt(var + eps) * (1 + scale[g]) + shift[g] per token
row, g = row // tokens_per_row, rounded once to bf16.  Bar: one round to
nearest bf16 is within 2^-8 of the value, the fp32 statistics add ~1e-6
relative, so |out - ref| <= 4e-3 |ref| + 1e-4 rms(ref).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from bit_post_quantised_b200 import tern, workloads

pytestmark = pytest.mark.gpu

RTOL = 4e-3
ARMS = 1e-4
EPS = 1e-6


def rand_bf16(shape, mean, std, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * std + mean).to(torch.bfloat16)


def bits(t: torch.Tensor) -> np.ndarray:
    return workloads.bf16_bits(t.cpu().contiguous())


def assert_close(out: torch.Tensor, ref: np.ndarray):
    a = out.double().cpu().numpy()
    rms = float(np.sqrt(np.mean(ref ** 2)))
    bad = np.abs(a - ref) > RTOL * np.abs(ref) + ARMS * rms
    assert not bad.any(), f"{int(bad.sum())} of {bad.size} outputs out of tolerance"


@pytest.mark.parametrize("M,K,T", [(1, 3072, 1), (37, 256, 37), (300, 3072, 300), (64, 4096, 16), (5, 8, 5),
                                   (17, 1000, 5), (129, 2048, 43), (8, 3064, 3)])
def test_adaln_modulate_matches_oracle(M, K, T):
    G = -(-M // T)
    x = rand_bf16((M, K), 0.3, 2.0, seed=M * 7 + K)
    sc = rand_bf16((G, K), 0.0, 0.1, seed=M + K + 1)
    sh = rand_bf16((G, K), 0.0, 0.5, seed=M + K + 2)
    out = tern.adaln_modulate(x.cuda(), sc.cuda(), sh.cuda(), EPS, tokens_per_row=T)
    torch.cuda.synchronize()
    assert tern.device_status() == 0
    assert_close(out, oracle.adaln_modulate(bits(x), bits(sc), bits(sh), EPS, T))


def test_adaln_modulate_in_place_and_modulation_slices():
    """out = x, with shift and scale read as slices of a [2, 6K] modulation
    output (rows 6K elements apart); tokens 0..M/2-1 use row 0."""
    M, K = 96, 3072
    x = rand_bf16((M, K), -0.2, 1.5, seed=5)
    mod = rand_bf16((2, 6 * K), 0.0, 0.2, seed=6)
    ref = oracle.adaln_modulate(bits(x), bits(mod[:, K:2 * K]), bits(mod[:, :K]), EPS, M // 2)
    xd, modd = x.cuda(), mod.cuda()
    got = tern.adaln_modulate(xd, modd[:, K:2 * K], modd[:, :K], EPS, tokens_per_row=M // 2, out=xd)
    torch.cuda.synchronize()
    assert got.data_ptr() == xd.data_ptr()
    assert_close(xd, ref)


def test_adaln_modulate_constant_rows_give_the_shift():
    """A constant row has zero variance: its normalised values are exactly 0,
    so the output is the shift row, bit for bit."""
    M, K = 12, 512
    x = rand_bf16((M, K), 0.0, 1.0, seed=8)
    x[3] = 1.5
    x[7] = -0.25
    sc = rand_bf16((1, K), 0.0, 0.3, seed=9)
    sh = rand_bf16((1, K), 0.0, 0.7, seed=10)
    out = tern.adaln_modulate(x.cuda(), sc.cuda(), sh.cuda(), EPS).cpu()
    for r in (3, 7):
        assert torch.equal(out[r], sh[0])
    assert_close(out, oracle.adaln_modulate(bits(x), bits(sc), bits(sh), EPS))


def test_adaln_modulate_flux_image_stream_full():
    """FLUX.1's double-block image stream at 1024x1024 (4096 tokens x 3072),
    two images' modulation rows; the oracle on every row."""
    M, K, T = 4096, 3072, 2048
    x = rand_bf16((M, K), 0.0, 1.0, seed=21).cuda()
    mod = rand_bf16((2, 6 * K), 0.0, 0.1, seed=22).cuda()
    out = tern.adaln_modulate(x, mod[:, K:2 * K], mod[:, :K], EPS, tokens_per_row=T)
    torch.cuda.synchronize()
    assert tern.device_status() == 0
    ref = oracle.adaln_modulate(bits(x.cpu()), bits(mod.cpu()[:, K:2 * K]), bits(mod.cpu()[:, :K]), EPS, T)
    assert_close(out.cpu(), ref)


def test_adaln_modulate_empty_is_a_no_op():
    x = torch.empty(0, 256, dtype=torch.bfloat16, device="cuda")
    sc = torch.zeros(1, 256, dtype=torch.bfloat16, device="cuda")
    out = tern.adaln_modulate(x, sc, sc, EPS, tokens_per_row=1)
    assert out.shape == (0, 256)
