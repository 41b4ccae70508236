"""Host-side pieces of the FLUX.1 forward (bit_post_quantised_b200.flux) on
the CPU, against the fp64 block oracle's own forms: the rotary angles' cos /
sin table the q/k epilogue reads, torch's rotary embedding of the dense
path, the sinusoidal timestep embedding, and the token positions."""
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
