"""FLUX.1 blocks on the ternary linear layer (bit_post_quantised_b200.flux),
on the GPU, against the fp64 block oracle (oracle/flux.py).

Small config (hidden 256 = two heads, MLP 1024, 8 x 8 image tokens + 24
text tokens, one double and one single block): every linear runs through
the C ABI with its fused epilogue, and every kernel class takes part (M = 1
modulation GEMVs, the 64-token tiles for the 24- and 64-token streams, CTA
pairs for the 88-token single block, the strided second linear).  The oracle
uses the GPU's own codes and scales, and rounds to bf16 wherever the GPU
path stores bf16, so the two differ only where a rounding decision flips (a
value within fp32 error of a bf16 rounding boundary: one unit in the last
place, 2^-8 relative) and in the attention kernel's bf16 probabilities
(2^-9 relative each).  Bar: about eight such units stacking up at one
element, two in the rms: |out - ref| <= 2^-5 (|ref| + rms(ref)) and
rms(out - ref) <= 2^-7 rms(ref).

Full size (hidden 3072, 4096 + 512 tokens), one double and one single
block against the same blocks in bf16 with dense weights (cuBLAS, torch's
unfused operations): a consistency check of the fused path at full size,
rms(out - dense) <= 2^-5 rms(dense) (the dense path rounds to bf16 after
each unfused operation and uses T*s rounded to bf16 as its weights); and
the whole transformer (the unquantised input layers and embedders, the
blocks, the final layer) the same way.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from oracle import flux as OF
from bit_post_quantised_b200 import flux, tern, workloads

pytestmark = pytest.mark.gpu


def oracle_params(model, weights, cfg, kind):
    q = model.blocks[(kind, 0)]
    p = {}
    for name, N, K in workloads.flux_block_shapes(cfg, kind):
        packed, scales, b = q[name]
        T, bad = oracle.unpack_tiled(packed.cpu().numpy(), N, K)
        assert bad == 0
        p[name] = (T, scales.cpu().double().numpy(), workloads.bf16_bits(b.cpu()))
    for key, v in weights[(kind, 0)].items():
        if key.endswith("_norm"):
            p[key] = workloads.bf16_bits(v)
    return p


def check(out: torch.Tensor, ref: np.ndarray):
    a = out.double().cpu().numpy()
    rms = float(np.sqrt(np.mean(ref ** 2)))
    d = np.abs(a - ref)
    bad = d > 2.0 ** -5 * (np.abs(ref) + rms)
    assert not bad.any(), f"{int(bad.sum())} of {bad.size} outside the bar; worst {d.max() / rms:.3e} rms"
    assert np.sqrt(np.mean(d ** 2)) <= 2.0 ** -7 * rms, f"rms diff {np.sqrt(np.mean(d ** 2)) / rms:.3e}"


@pytest.fixture(scope="module")
def small():
    cfg = workloads.FLUX_SMALL
    weights = {(k, 0): workloads.flux_block_weights(cfg, k, 0) for k in ("double", "single")}
    model = flux.TernaryFlux(cfg, weights, device="cuda")
    img, txt, vec, ids = workloads.flux_inputs(cfg)
    f = lambda t: OF.from_bits(workloads.bf16_bits(t))  # noqa: E731
    ref_in = (f(img), f(txt), f(vec), OF.rope_angles(ids.numpy()))
    return cfg, weights, model, (img.cuda(), txt.cuda(), vec.cuda(), ids), ref_in


@pytest.fixture(scope="module")
def small_strong():
    """The small config with every ternary weight 8x larger (exact in bf16,
    the same codes, 8x the scales): the blocks' updates then outweigh the
    residual streams, so a wrong update cannot hide under the streams' bf16
    rounding (with the seeded weights the gates keep the updates near 1 % of
    the stream)."""
    cfg = workloads.FLUX_SMALL
    weights = {}
    for k in ("double", "single"):
        w = workloads.flux_block_weights(cfg, k, 0)
        for name, _, _ in workloads.flux_block_shapes(cfg, k):
            W, b = w[name]
            w[name] = (W * 8, b)
        weights[(k, 0)] = w
    model = flux.TernaryFlux(cfg, weights, device="cuda")
    img, txt, vec, ids = workloads.flux_inputs(cfg)
    f = lambda t: OF.from_bits(workloads.bf16_bits(t))  # noqa: E731
    ref_in = (f(img), f(txt), f(vec), OF.rope_angles(ids.numpy()))
    return cfg, weights, model, (img.cuda(), txt.cuda(), vec.cuda(), ids), ref_in


def test_blocks_with_dominant_updates_match_oracle(small_strong):
    cfg, weights, model, (img, txt, vec, ids), (i64, t64, v64, ang) = small_strong
    out = model.forward(img, txt, vec, ids)
    torch.cuda.synchronize()
    assert tern.device_status() == 0
    oi, ot = OF.double_block(i64, t64, v64, oracle_params(model, weights, cfg, "double"), ang)
    ref = OF.single_block(np.concatenate([ot, oi]), v64, oracle_params(model, weights, cfg, "single"), ang)
    x0 = np.concatenate([t64, i64])
    assert np.sqrt(np.mean((ref - x0) ** 2)) > 0.5 * np.sqrt(np.mean(ref ** 2))  # the update dominates
    check(out, ref)


def test_double_block_matches_oracle(small):
    cfg, weights, model, (img, txt, vec, ids), (i64, t64, v64, ang) = small
    out = model.forward(img, txt, vec, ids, n_double=1, n_single=0)
    torch.cuda.synchronize()
    assert tern.device_status() == 0
    oi, ot = OF.double_block(i64, t64, v64, oracle_params(model, weights, cfg, "double"), ang)
    check(out, np.concatenate([ot, oi]))
    assert torch.equal(img.cpu(), workloads.flux_inputs(cfg)[0])  # inputs untouched


def test_double_then_single_block_matches_oracle(small):
    cfg, weights, model, (img, txt, vec, ids), (i64, t64, v64, ang) = small
    out = model.forward(img, txt, vec, ids)
    torch.cuda.synchronize()
    assert tern.device_status() == 0
    oi, ot = OF.double_block(i64, t64, v64, oracle_params(model, weights, cfg, "double"), ang)
    ref = OF.single_block(np.concatenate([ot, oi]), v64, oracle_params(model, weights, cfg, "single"), ang)
    check(out, ref)


def test_forward_on_a_side_stream_matches(small):
    """A model given its own stream (construction and forward on it, torch
    operations included) gives the same bits as on the current stream."""
    cfg, weights, model, (img, txt, vec, ids), _ = small
    ref = model.forward(img, txt, vec, ids)
    s = torch.cuda.Stream()
    side = flux.TernaryFlux(cfg, weights, device="cuda", stream=s)
    out = side.forward(img, txt, vec, ids)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    assert tern.device_status() == 0
    assert torch.equal(out, ref)


def test_full_size_blocks_agree_with_dense_bf16():
    cfg = workloads.FluxConfig(n_double=1, n_single=1)
    model = flux.TernaryFlux(cfg, device="cuda")
    img, txt, vec, ids = (t.cuda() for t in workloads.flux_inputs(cfg))
    out = model.forward(img, txt, vec, ids)
    dense = flux.dense_forward(model, flux.dense_weights(model), img, txt, vec, ids)
    torch.cuda.synchronize()
    assert tern.device_status() == 0
    assert torch.isfinite(out.float()).all()
    d = (out.float() - dense.float()).pow(2).mean().sqrt().item()
    r = dense.float().pow(2).mean().sqrt().item()
    assert d <= 2.0 ** -5 * r, f"rms diff {d / r:.3e}"


def test_whole_model_agrees_with_dense_bf16():
    """Input projections, time/guidance/pooled-text embedders, one double and
    one single block, the final layer: [4096, 64] out, against the same model
    with the blocks in dense bf16."""
    cfg = workloads.FluxConfig(n_double=1, n_single=1)
    model = flux.TernaryFlux(cfg, device="cuda")
    io = {k: (W.cuda(), b.cuda()) for k, (W, b) in workloads.flux_io_weights(cfg).items()}
    img, txt, pooled, t, g, ids = workloads.flux_model_inputs(cfg)
    args = (img.cuda(), txt.cuda(), pooled.cuda(), t, g, ids.cuda())
    out = flux.model_forward(model, io, *args)
    ref = flux.dense_model_forward(model, flux.dense_weights(model), io, *args)
    torch.cuda.synchronize()
    assert tern.device_status() == 0
    assert out.shape == (cfg.img_tokens, cfg.in_channels) and torch.isfinite(out.float()).all()
    d = (out.float() - ref.float()).pow(2).mean().sqrt().item()
    r = ref.float().pow(2).mean().sqrt().item()
    assert d <= 2.0 ** -5 * r, f"rms diff {d / r:.3e}"
