"""Whole FLUX.1-dev blocks at full size, through the C ABI on the GPU, against
the fp64 oracle.

Page "1.58-bit FLUX" (arXiv 2412.18653), Section 3.1: every linear layer of
the double-stream and single-stream transformer blocks is ternary.  One block
of each type is built at the sizes of one 1024x1024 image (4096 image tokens,
512 text tokens, hidden 3072, MLP 12288) and run as ONE
tern_linear_batch_epilogue launch group per block, exactly as the benchmark's
whole-stack forward runs it: the M = 1 adaLN modulation GEMVs, the QKV
projections, the attention output projections and the MLPs of both streams
(single block: modulation, the fused 3072 -> 21504 projection, the
15360 -> 3072 output projection), with FLUX.1's epilogues fused:

  * GELU (tanh form) on the MLP's first linear, and from column 9216 of a
    single block's fused projection;
  * the in-place gated residual update on every output projection;
  * optionally the per-head RMS normalisation of q and k (columns
    [0, 6144) of each QKV projection).

Every problem of the batch is checked element by element against
oracle.linear_epilogue on the GPU-produced codes and scales (which are
themselves checked against the oracle's quantisation): all token rows of the
text stream and of the M = 1 GEMVs, 512 seeded rows (first and last included)
of the 4096- and 4608-token problems, every output channel.  Bar:
|y - y_ref| <= 8e-3 |y_ref| + 1e-3 rms(y_ref), per problem.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from bit_post_quantised_b200 import tern, workloads

pytestmark = pytest.mark.gpu

EPS = workloads.EPS
SCALE_RTOL = 1e-6
BAND = 1e-6
Y_RTOL = 8e-3
Y_RMS = 1e-3
NORM_EPS = 1e-6
ROWS_CHECKED = 512


def bits(t: torch.Tensor) -> np.ndarray:
    return workloads.bf16_bits(t.detach().cpu())


def rand_bf16(shape, std, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * std).to(torch.bfloat16)


def quantize_checked(W_cpu: torch.Tensor):
    """GPU quantise/pack of W, checked against the oracle: scales within 1e-6
    relative, codes bit-exact given the GPU's scales away from the rounding
    threshold.  Returns the device buffers and the codes and scales the oracle
    linear takes."""
    packed, scales = tern.quantize_pack(W_cpu.cuda(), EPS)
    torch.cuda.synchronize()
    assert tern.device_status() == 0
    N, K = W_cpu.shape
    Wb = bits(W_cpu)
    s_gpu = scales.cpu().double().numpy()
    s_ref = oracle.absmean_scales(Wb, EPS)
    assert (np.abs(s_gpu - s_ref) / s_ref).max() <= SCALE_RTOL
    T, bad = oracle.unpack_tiled(packed.cpu().numpy(), N, K)
    assert bad == 0
    _, near = oracle.near_threshold(Wb, s_gpu, BAND)
    assert not np.any((T != oracle.ternarize(Wb, s_gpu)) & ~near)
    return packed, scales, T, s_gpu


def check_y(y_gpu: torch.Tensor, y_ref: np.ndarray, what: str):
    y = y_gpu.detach().cpu().double().numpy()
    assert y.shape == y_ref.shape, what
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    err = np.abs(y - y_ref)
    bad = err > Y_RTOL * np.abs(y_ref) + Y_RMS * rms
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} outputs out of tolerance; worst err "
                           f"{err.max():.3e} at {np.unravel_index(err.argmax(), err.shape)}")


def checked_rows(M: int, seed: int) -> np.ndarray:
    if M <= ROWS_CHECKED:
        return np.arange(M)
    rows = np.sort(np.random.default_rng(seed).choice(M, ROWS_CHECKED, replace=False))
    rows[0], rows[-1] = 0, M - 1
    return np.unique(rows)


@pytest.mark.parametrize("qk_norm", [False, True], ids=["bench_epilogues", "with_qk_norm"])
@pytest.mark.parametrize("block", ["double0", "single0"])
def test_flux_block_batch_epilogue(block, qk_norm):
    layers = workloads.block_layers(block)
    assert len(layers) == (10 if block.startswith("double") else 3)
    probs, refs = [], []
    for L in layers:
        x, W, b = workloads.make_inputs(L)
        packed, scales, T, s = quantize_checked(W)
        del W
        e = workloads.block_epilogue(L.name, qk_norm)
        act = {"gelu_tanh": tern.ACT_GELU_TANH}.get(e.get("act"), tern.ACT_NONE)
        p = dict(x=x.cuda(), packed=packed, scales=scales, bias=b.cuda(), act=act, act_col0=e.get("act_col0", 0))
        r = g = w = None
        if e.get("gated_residual"):
            r = rand_bf16((L.M, L.N), 1.0, L.seed + 7)
            g = rand_bf16((L.N,), 0.5, L.seed + 8)
            p["y"] = p["residual"] = r.cuda()  # the residual stream, updated in place
            p["gate"] = g.cuda()
        else:
            p["y"] = torch.full((L.M, L.N), float("nan"), dtype=torch.bfloat16, device="cuda")
        cols = e.get("norm_cols", (0, 0))
        if cols[1] > cols[0]:
            w = (torch.rand(L.N, generator=torch.Generator().manual_seed(L.seed + 9)) + 0.5).to(torch.bfloat16)
            p.update(norm_col0=cols[0], norm_col1=cols[1], norm_weight=w.cuda(), norm_eps=NORM_EPS)
        probs.append(p)
        rows = checked_rows(L.M, L.seed)
        refs.append((L, rows, x, T, s, b, act, e.get("act_col0", 0), r, g, cols, w))
    tern.linear_batch_epilogue(probs)
    torch.cuda.synchronize()
    assert tern.device_status() == 0
    for p, (L, rows, x, T, s, b, act, col0, r, g, cols, w) in zip(probs, refs):
        y_ref = oracle.linear_epilogue(bits(x[rows]), T, s, bits(b), act, col0,
                                       None if r is None else bits(r[rows]), None if g is None else bits(g),
                                       cols, None if w is None else bits(w), NORM_EPS)
        check_y(p["y"][torch.from_numpy(rows).cuda()], y_ref, L.name)
