"""Host-side pieces of the FLUX.1 forward (bit_post_quantised_b200.flux) on
the CPU, against the fp64 block oracle's own forms: the rotary angles' cos /
sin table the q/k epilogue reads, torch's rotary embedding of the dense
path, the sinusoidal timestep embedding, the token positions, and the
dense-bf16 twin of the blocks as a whole."""
from __future__ import annotations

import math

import numpy as np
import torch

from oracle import flux as OF
from bit_post_quantised_b200 import flux, workloads


def test_rope_table_matches_the_oracle_angles():
    ids = workloads.flux_inputs(workloads.FLUX_SMALL)[3]
    big = torch.cat([ids, torch.tensor([[0.0, 63.0, 63.0], [0.0, 17.0, 40.0]])])
    cos, sin = flux.rope_cos_sin(big)
    ang = OF.rope_angles(big.numpy())
    assert cos.dtype == torch.float32 and cos.shape == (big.shape[0], 64)
    assert np.abs(cos.double().numpy() - np.cos(ang)).max() <= 2e-7
    assert np.abs(sin.double().numpy() - np.sin(ang)).max() <= 2e-7


def test_torch_rope_matches_the_oracle():
    """The dense path's rotary embedding (fp32, one bf16 rounding) against the
    oracle's fp64 rotation rounded once: equal but for rounding flips."""
    g = torch.Generator().manual_seed(3)
    L, H = 40, 2
    x = (torch.randn(L, H, 128, generator=g) * 2).to(torch.bfloat16)
    ids = torch.stack([torch.zeros(L), torch.randint(0, 64, (L,), generator=g).float(),
                       torch.randint(0, 64, (L,), generator=g).float()], dim=1)
    cos, sin = flux.rope_cos_sin(ids)
    got = flux.apply_rope(x, cos, sin).double().numpy()
    want = OF.bf16(OF.apply_rope(x.double().numpy().transpose(1, 0, 2), OF.rope_angles(ids.numpy()))
                   .transpose(1, 0, 2))
    rel = np.abs(got - want) / np.maximum(np.abs(want), 1e-3)
    assert (got != want).mean() < 0.01 and rel.max() <= 2.0 ** -7


def test_timestep_embedding_closed_form():
    e = flux.timestep_embedding(0.0, "cpu").float()[0]
    assert torch.equal(e[:128], torch.ones(128)) and torch.equal(e[128:], torch.zeros(128))
    t = 0.37
    e = flux.timestep_embedding(t, "cpu").double()[0].numpy()
    f = np.exp(-math.log(10000.0) * np.arange(128) / 128)
    want = np.concatenate([np.cos(1000 * t * f), np.sin(1000 * t * f)])
    assert np.abs(e - want).max() <= 2.0 ** -8 * 1.01  # bf16 rounding of values in [-1, 1]


def test_token_positions():
    cfg = workloads.FLUX_SMALL
    ids = workloads.flux_inputs(cfg)[3]
    assert ids.shape == (cfg.txt_tokens + cfg.img_tokens, 3)
    assert not ids[:cfg.txt_tokens].any()
    img = ids[cfg.txt_tokens:]
    assert torch.equal(img[:, 0], torch.zeros(cfg.img_tokens))
    assert torch.equal(img[cfg.img_w + 3], torch.tensor([0.0, 1.0, 3.0]))  # row 1, column 3


def test_dense_twin_matches_the_block_oracle():
    """flux.dense_forward (the bf16 model with dense weights that the forward
    is timed against) on the CPU, one double and one single block of the
    small config, with weights bf16(T * s) from the oracle's quantisation,
    against the fp64 block oracle on the same T and s.  The scales are taken
    8x larger than the seeded weights give, so that the blocks' updates
    outweigh the residual streams they are added to (with the seeded scales
    the gates keep them near 1 % of the stream, below what the bf16 stream
    resolves).  The dense twin rounds to bf16 after each unfused torch
    operation and its weights carry one more rounding: rms 2^-6 of the
    output; a missing q/k norm weight, swapped position axes or a dropped
    projection each exceed it."""
    import types

    import oracle

    cfg = workloads.FLUX_SMALL
    C = cfg.hidden
    dense, params = {}, {}
    for kind in ("double", "single"):
        w = workloads.flux_block_weights(cfg, kind, 0)
        d, p = {}, {}
        for name, N, K in workloads.flux_block_shapes(cfg, kind):
            W, b = w[name]
            T, s = oracle.quantize(workloads.bf16_bits(W), workloads.EPS)
            s = 8.0 * s
            d[name] = (torch.from_numpy(T * s[:, None]).to(torch.bfloat16), b)
            p[name] = (T, s, workloads.bf16_bits(b))
        for st in (("img.", "txt.") if kind == "double" else ("",)):
            N = 3 * C if kind == "double" else 3 * C + cfg.mlp
            d[st + "norm_w"] = flux._qk_norm_weight(w[st + "q_norm"], w[st + "k_norm"], C, N)
            p[st + "q_norm"] = workloads.bf16_bits(w[st + "q_norm"])
            p[st + "k_norm"] = workloads.bf16_bits(w[st + "k_norm"])
        dense[(kind, 0)], params[kind] = d, p
    img, txt, vec, ids = workloads.flux_inputs(cfg)
    out = flux.dense_forward(types.SimpleNamespace(cfg=cfg), dense, img, txt, vec, ids, 1, 1)
    f = lambda t: OF.from_bits(workloads.bf16_bits(t))  # noqa: E731
    ang = OF.rope_angles(ids.numpy())
    oi, ot = OF.double_block(f(img), f(txt), f(vec), params["double"], ang)
    ref = OF.single_block(np.concatenate([ot, oi]), f(vec), params["single"], ang)
    x0 = np.concatenate([f(txt), f(img)])
    rms = float(np.sqrt(np.mean(ref ** 2)))
    assert float(np.sqrt(np.mean((ref - x0) ** 2))) > 0.5 * rms  # the update dominates
    assert out.shape == (cfg.txt_tokens + cfg.img_tokens, C)
    assert float(np.sqrt(np.mean((out.double().numpy() - ref) ** 2))) <= 2.0 ** -6 * rms


def test_parameter_count_matches_the_pages():
    """The synthetic transformer's parameters (ternary block linears, their
    biases and q/k norm weights, and the bf16 input/output layers and
    embedders) add up to the 11.9B the pages give for FLUX.1-dev, and the
    ternary weights to the 99.5 % they quantise ("1.58-bit FLUX", Abstract
    and Section 1): a check of every layer shape of the forward."""
    cfg = workloads.FluxConfig()
    blocks = [s for kind, n in (("double", cfg.n_double), ("single", cfg.n_single))
              for _ in range(n) for s in workloads.flux_block_shapes(cfg, kind)]
    ternary = sum(N * K for _, N, K in blocks)
    biases = sum(N for _, N, _ in blocks)
    norms = (4 * cfg.n_double + 2 * cfg.n_single) * workloads.HEAD_DIM
    io = sum(W.numel() + b.numel() for W, b in workloads.flux_io_weights(cfg).values())
    total = ternary + biases + norms + io
    assert abs(total / 1e9 - 11.9) < 0.05
    assert abs(ternary / total - 0.995) < 2e-3
