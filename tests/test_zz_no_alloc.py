"""tern_linear_noalloc against tern_linear, through the C ABI on the GPU.

tern_linear_noalloc serves callers that cannot allocate device memory (code
running under global-mode CUDA graph capture, engines that own all device
memory in a preplanned arena, latency-critical loops where an allocation could
synchronise the device).  Its split-K scratch is a static device array of the
library instead of a workspace allocated on first use.  It must give the same
y as tern_linear bit for bit (the same kernels with the same tile and split
choice; the last CTA of a tile adds the split partial sums in split order),
on two calls in a row (the second one finds the first one's partial sums and
counters in the shared array), whether this file runs alone in a fresh
process or after every other test.  This file is named so that pytest
collects it last.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from bit_post_quantised_b200 import tern

pytestmark = pytest.mark.gpu

Y_RTOL = 8e-3
Y_RMS = 1e-3


def rand_bf16(shape, std, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * std).to(torch.bfloat16)


def make_case(M, N, K, seed):
    W = rand_bf16((N, K), 0.02, seed).cuda()
    x = rand_bf16((M, K), 1.0, seed + 1).cuda()
    b = rand_bf16((N,), 0.01, seed + 2).cuda()
    packed, scales = tern.quantize_pack(W)
    return x, packed, scales, b


def assert_close(y, y_ref):
    a = y.double().cpu().numpy()
    r = y_ref.double().cpu().numpy()
    rms = float(np.sqrt(np.mean(r ** 2)))
    bad = np.abs(a - r) > Y_RTOL * np.abs(r) + Y_RMS * rms
    assert not bad.any(), f"{int(bad.sum())} of {bad.size} outputs out of tolerance"


# 16 < M <= 64 with N % 256 != 0 takes the split-K path whose scratch lives in
# the static array; M <= 16 (the GEMV kernel) and N % 256 == 0 (the pair-tile
# kernels) need no scratch.
@pytest.mark.parametrize("M,N,K", [(1, 18432, 3072), (40, 384, 1024), (64, 640, 3072), (24, 1152, 3072),
                                   (300, 512, 256)])
def test_noalloc_matches_linear_on_two_calls(M, N, K):
    x, packed, scales, b = make_case(M, N, K, seed=M + N + K)
    y_ref = tern.linear(x, packed, scales, b)
    for call in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        tern.linear_noalloc(x, packed, scales, b, out=y)
        torch.cuda.synchronize()
        assert tern.device_status() == 0
        assert_close(y, y_ref)
        assert torch.equal(y, y_ref)


def test_noalloc_back_to_back_different_shapes():
    """A call that leaves partial sums of another shape in the array, then a
    second shape, each checked against tern_linear."""
    cases = [make_case(33, 1152, 3072, seed=1), make_case(64, 640, 1536, seed=2)]
    refs = [tern.linear(*c) for c in cases]
    outs = [tern.linear_noalloc(*c) for c in cases]
    torch.cuda.synchronize()
    assert tern.device_status() == 0
    for y, r in zip(outs, refs):
        assert_close(y, r)
        assert torch.equal(y, r)
