"""Pins of the FLUX.1 block oracle (oracle/flux.py) against facts that do not
come from the oracle itself: torch's bf16 rounding, closed forms of the
rotary embedding and of softmax attention, and structural identities of the
blocks (zero gates leave the residual streams untouched; with all positions
equal, swapping the two streams' roles swaps their outputs; a zero second
linear adds gate * bias).  CPU only."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from oracle import flux as OF
from bit_post_quantised_b200 import workloads

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(1)
    v = rng.standard_normal(200000) * np.exp(rng.uniform(-90, 80, 200000))
    v = v.astype(np.float32).astype(np.float64)  # exact in fp32: torch rounds once
    ties = np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 2 ** -130 * 1.5, 255.5 * 2 ** -7])
    for x in (v, ties.astype(np.float32).astype(np.float64)):
        want = torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).double().numpy()
        assert np.array_equal(OF.bf16(x), want)
    assert OF.bf16(1 + 2 ** -8) == 1.0 and OF.bf16(1 + 3 * 2 ** -8) == 1 + 2 ** -6  # ties to even


def test_rope_angles_axis_layout():
    ids = np.array([[3.0, 5.0, 7.0]])
    a = OF.rope_angles(ids)
    assert a.shape == (1, 64)
    # pair 0 of every axis turns by the position itself (omega = 1)
    assert a[0, 0] == 3.0 and a[0, 8] == 5.0 and a[0, 36] == 7.0
    # last pair of the first axis: 3 * 10000^(-14/16)
    assert np.isclose(a[0, 7], 3.0 * 10000.0 ** (-14 / 16), rtol=1e-15)
    assert np.isclose(a[0, 35], 5.0 * 10000.0 ** (-54 / 56), rtol=1e-15)


def test_apply_rope_rotations():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((2, 5, 128))
    zero = np.zeros((5, 64))
    assert np.array_equal(OF.apply_rope(x, zero), x)
    quarter = np.full((5, 64), np.pi / 2)
    y = OF.apply_rope(x, quarter)
    assert np.allclose(y[..., 0::2], -x[..., 1::2], atol=1e-15) and np.allclose(y[..., 1::2], x[..., 0::2], atol=1e-15)
    ang = rng.uniform(-40, 40, (5, 64))
    assert np.allclose(np.linalg.norm(OF.apply_rope(x, ang), axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)
    # relative positions: <R(m) q, R(n) k> depends on m - n only
    ids = np.array([[0, 2.0, 9.0], [0, 5.0, 1.0], [0, 12.0, 19.0], [0, 15.0, 11.0]])
    A = OF.rope_angles(ids)
    q, k = rng.standard_normal(128), rng.standard_normal(128)
    rot = lambda v, a: OF.apply_rope(v[None, None, :], a[None, :])[0, 0]  # noqa: E731
    d1 = rot(q, A[0]) @ rot(k, A[1])
    d2 = rot(q, A[2]) @ rot(k, A[3])  # both positions shifted by (10, 10)
    assert np.isclose(d1, d2, rtol=1e-12)


def test_attention_closed_forms():
    rng = np.random.default_rng(3)
    q = rng.standard_normal((2, 4, 128))
    k1 = rng.standard_normal((2, 1, 128))
    v1 = rng.standard_normal((2, 1, 128))
    assert np.allclose(OF.attention(q, k1, v1), np.broadcast_to(v1, (2, 4, 128)), atol=1e-15)  # one key
    k = np.repeat(k1, 6, axis=1)
    v = rng.standard_normal((2, 6, 128))
    assert np.allclose(OF.attention(q, k, v), v.mean(axis=1, keepdims=True), atol=1e-14)  # equal keys: the mean
    kk = rng.standard_normal((2, 6, 128))
    perm = rng.permutation(6)
    assert np.allclose(OF.attention(q, kk, v), OF.attention(q, kk[:, perm], v[:, perm]), atol=1e-14)
    # a key aligned with the query and scaled far up takes all the weight
    ks = kk.copy()
    ks[:, 2] = q[:, 0] * 50
    assert np.allclose(OF.attention(q[:, :1], ks, v), v[:, 2:3], atol=1e-12)


def _params(cfg, kind, zero_gates=False, zero_linear2=False):
    """Oracle parameters from the seeded bf16 weights, quantised by the
    oracle's own absmean rule (these pins exercise the block wiring)."""
    w = workloads.flux_block_weights(cfg, kind, 0)
    C = cfg.hidden
    p = {}
    for name, N, K in workloads.flux_block_shapes(cfg, kind):
        W, b = w[name]
        T, s = oracle.quantize(workloads.bf16_bits(W), workloads.EPS)
        bb = workloads.bf16_bits(b).copy()
        if zero_gates and name.endswith("mod"):
            gate_rows = [range(2 * C, 3 * C), range(5 * C, 6 * C)] if kind == "double" else [range(2 * C, 3 * C)]
            for r in gate_rows:
                T[list(r)] = 0
                bb[list(r)] = 0
        if zero_linear2 and name == "linear2":
            T = np.zeros_like(T)
        p[name] = (T, s, bb)
    for key in w:
        if key.endswith("_norm"):
            p[key] = workloads.bf16_bits(w[key])
    return p


def _inputs(cfg):
    img, txt, vec, ids = workloads.flux_inputs(cfg)
    f = lambda t: OF.from_bits(workloads.bf16_bits(t))  # noqa: E731
    return f(img), f(txt), f(vec), ids.numpy()


def test_double_block_zero_gates_keep_the_streams():
    cfg = workloads.FLUX_SMALL
    img, txt, vec, ids = _inputs(cfg)
    p = _params(cfg, "double", zero_gates=True)
    oi, ot = OF.double_block(img, txt, vec, p, OF.rope_angles(ids))
    assert np.array_equal(oi, img) and np.array_equal(ot, txt)
    q = _params(cfg, "double")
    oi, ot = OF.double_block(img, txt, vec, q, OF.rope_angles(ids))
    assert not np.array_equal(oi, img) and np.isfinite(oi).all() and np.isfinite(ot).all()


def test_double_block_swapping_the_streams_swaps_the_outputs():
    """All positions equal (rotary embedding the same for every token) and
    both streams given the same parameters: attention then treats the token
    set without order, so the block's text/image bookkeeping (which rows of
    the joint attention go back to which stream) is the only difference."""
    cfg = workloads.FLUX_SMALL
    img, txt, vec, _ = _inputs(cfg)
    p = _params(cfg, "double")
    for name in ("mod", "qkv", "proj", "mlp_up", "mlp_down", "q_norm", "k_norm"):
        p["txt." + name] = p["img." + name]
    ids0 = np.zeros((img.shape[0] + txt.shape[0], 3))
    a_img, a_txt = OF.double_block(img, txt, vec, p, OF.rope_angles(ids0))
    b_img, b_txt = OF.double_block(txt, img, vec, p, OF.rope_angles(ids0))
    assert np.allclose(a_img, b_txt, rtol=0, atol=1e-2 * np.abs(a_img).max())
    assert np.allclose(a_txt, b_img, rtol=0, atol=1e-2 * np.abs(a_txt).max())


def test_single_block_zero_gate_and_zero_second_linear():
    cfg = workloads.FLUX_SMALL
    img, txt, vec, ids = _inputs(cfg)
    x = np.concatenate([txt, img])
    ang = OF.rope_angles(ids)
    assert np.array_equal(OF.single_block(x, vec, _params(cfg, "single", zero_gates=True), ang), x)
    # linear2's codes all zero: x + gate * bias, with the block's own gate
    p = _params(cfg, "single", zero_linear2=True)
    out = OF.single_block(x, vec, p, ang)
    C = cfg.hidden
    T, s, b = p["mod"]
    g = OF.bf16(oracle.linear(OF.bits(OF.bf16(OF.silu(vec))), T, s, b))[0, 2 * C:]
    want = OF.bf16(x + g[None, :] * OF.from_bits(p["linear2"][2])[None, :])
    assert np.array_equal(out, want)


def test_rotate_pairs_matches_the_pinned_rotary_embedding():
    """oracle.rotate_pairs (the fused epilogue's rotation of the normalised
    columns) against OF.apply_rope (pinned above) on two heads."""
    rng = np.random.default_rng(9)
    L = 7
    y = rng.standard_normal((L, 3 * 128))
    ids = np.stack([np.zeros(L), rng.integers(0, 60, L), rng.integers(0, 60, L)], axis=1).astype(float)
    ang = OF.rope_angles(ids)
    got = oracle.rotate_pairs(y, 0, 256, OF.cos_sin(ang))
    heads = y[:, :256].reshape(L, 2, 128).transpose(1, 0, 2)
    want = OF.apply_rope(heads, ang).transpose(1, 0, 2).reshape(L, 256)
    assert np.allclose(got[:, :256], want, rtol=0, atol=1e-14)
    assert np.array_equal(got[:, 256:], y[:, 256:])
