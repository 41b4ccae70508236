"""fp64 CPU oracle for FLUX.1's two transformer block types built on the
ternary linear layer of "1.58-bit FLUX" (arXiv 2412.18653).

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle``: the tests are its
only users, and it shares no code with the CUDA library.

The pages quantise every linear layer of FLUX.1's double-stream and
single-stream blocks (Section 3.1) and compare whole-model latency and
memory (Table 3); they describe nothing between the linears.  What sits
between them here is FLUX.1's block, written from that model's definition:
adaLN-Zero modulation of layer-normalised tokens, per-head RMS
normalisation of q and k, rotary position embedding over three position
axes, softmax attention over the text and image tokens together, the tanh
GELU MLP, and gated residual updates.

Every tensor that the GPU path keeps in bf16 between two operations is
rounded to bf16 here at the same point (``bf16``: round to nearest even from
float64), so the oracle is FLUX.1's sequence of operations with bf16
activations, each operation itself exact; where the GPU path fuses two
(q/k norm and rotary embedding in the projection's epilogue) there is one
rounding after both.  Linears go through
``oracle.linear`` / ``linear_act`` / ``linear_epilogue`` with the codes and
scales of the ternary weights.

Block parameters are dicts (see ``bit_post_quantised_b200.workloads``):
ternary linears as ``(T, s, b_bits)`` with T int8 [N, K], s float64 [N],
b bf16 bit patterns [N]; ``q_norm`` / ``k_norm`` bf16 bit patterns [128].
"""
from __future__ import annotations

import numpy as np

from . import (ACT_GELU_TANH, adaln_modulate, bf16_bits_to_f64, gelu_tanh, linear, linear_act, linear_epilogue,
               rms_norm_groups, rotate_pairs)

HEAD_DIM = 128
LN_EPS = 1e-6
QK_EPS = 1e-6
ROPE_THETA = 10000.0
ROPE_AXES = (16, 56, 56)


def bf16(v) -> np.ndarray:
    """Nearest bf16 value (ties to even) of every float64, as float64.  A
    finite v = m 2^e (0.5 <= |m| < 1) keeps 8 significant bits, quantum
    2^(e-8), never finer than the subnormal step 2^-133."""
    v = np.asarray(v, dtype=np.float64)
    _, e = np.frexp(v)
    q = np.ldexp(1.0, np.maximum(e - 8, -133))
    return np.rint(v / q) * q


def bits(v) -> np.ndarray:
    """bf16 bit patterns of float64 values that are already bf16 values."""
    f = np.ascontiguousarray(v, dtype=np.float64).astype(np.float32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def silu(v: np.ndarray) -> np.ndarray:
    return v / (1.0 + np.exp(-v))


def rope_angles(ids: np.ndarray, axes=ROPE_AXES, theta: float = ROPE_THETA) -> np.ndarray:
    """Rotation angles [L, HEAD_DIM / 2] of the token positions ids [L, len(axes)]:
    axis a with d_a channels owns d_a / 2 consecutive channel pairs, pair j
    of it turning by ids[:, a] * theta^(-2j / d_a)."""
    ids = np.asarray(ids, dtype=np.float64)
    parts = []
    for a, d in enumerate(axes):
        omega = theta ** (-np.arange(0, d, 2, dtype=np.float64) / d)
        parts.append(ids[:, a:a + 1] * omega[None, :])
    return np.concatenate(parts, axis=1)


def apply_rope(x: np.ndarray, angles: np.ndarray) -> np.ndarray:
    """Rotates channel pairs (2i, 2i + 1) of x [H, L, D] by angles [L, D / 2]:
    (a, b) -> (a cos - b sin, a sin + b cos)."""
    a, b = x[..., 0::2], x[..., 1::2]
    c, s = np.cos(angles)[None], np.sin(angles)[None]
    out = np.empty_like(x)
    out[..., 0::2] = a * c - b * s
    out[..., 1::2] = a * s + b * c
    return out


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """softmax(q k^T / sqrt(D)) v per head; q, k, v [H, L, D]."""
    z = np.einsum("hld,hmd->hlm", q, k) / np.sqrt(q.shape[-1])
    z = z - z.max(axis=-1, keepdims=True)
    p = np.exp(z)
    p = p / p.sum(axis=-1, keepdims=True)
    return np.einsum("hlm,hmd->hld", p, v)


def _heads(x: np.ndarray) -> np.ndarray:
    """[L, H * D] -> [H, L, D]."""
    L, C = x.shape
    return x.reshape(L, C // HEAD_DIM, HEAD_DIM).transpose(1, 0, 2)


def _tokens(x: np.ndarray) -> np.ndarray:
    """[H, L, D] -> [L, H * D]."""
    H, L, D = x.shape
    return x.transpose(1, 0, 2).reshape(L, H * D)


def _qk_norm_weight(q_norm, k_norm, hidden: int) -> np.ndarray:
    """bf16 bit patterns of the per-channel weight over the q and k columns
    [0, 2 hidden): each head's 128-channel RMS norm shares one 128-vector
    for q and one for k."""
    heads = hidden // HEAD_DIM
    return np.concatenate([np.tile(q_norm, heads), np.tile(k_norm, heads)])


def _lin(x, lin, **kw):
    T, s, b = lin
    return linear_epilogue(bits(x), T, s, b, **kw)


def cos_sin(angles: np.ndarray) -> np.ndarray:
    """(cos, sin) pairs [L, 64, 2] of rotation angles [L, 64]."""
    return np.stack([np.cos(angles), np.sin(angles)], axis=-1)


def _qk_normed(y: np.ndarray, q_norm, k_norm, hidden: int, angles: np.ndarray) -> np.ndarray:
    """q, k and v columns of a projection's bf16 output y, q and k normalised
    per head and then rotated (fp64, one rounding to bf16: the GPU path does
    both in the projection's epilogue)."""
    qk = rms_norm_groups(y[:, :2 * hidden], 0, 2 * hidden, QK_EPS, _qk_norm_weight(q_norm, k_norm, hidden))
    qk = rotate_pairs(qk, 0, 2 * hidden, cos_sin(angles))
    return np.concatenate([bf16(qk), y[:, 2 * hidden:3 * hidden]], axis=1)


def _attend(qkv: np.ndarray, hidden: int) -> np.ndarray:
    """Attention over all rows of qkv (q and k already rotated)."""
    q, k, v = _heads(qkv[:, :hidden]), _heads(qkv[:, hidden:2 * hidden]), _heads(qkv[:, 2 * hidden:])
    return bf16(_tokens(attention(q, k, v)))


def double_block(img: np.ndarray, txt: np.ndarray, vec: np.ndarray, p: dict, angles: np.ndarray):
    """FLUX.1's double-stream block.  img [Li, C], txt [Lt, C] and vec [1, C]
    are bf16 values in float64; angles [Lt + Li, 64] for the text tokens
    followed by the image tokens.  Returns (img, txt) as bf16 values."""
    hidden = img.shape[1]
    y = bf16(silu(vec))
    out = {}
    mods = {}
    for s, x in (("img", img), ("txt", txt)):
        m = bf16(_lin(y, p[s + ".mod"]))[0]
        mods[s] = [m[i * hidden:(i + 1) * hidden] for i in range(6)]  # shift1 scale1 gate1 shift2 scale2 gate2
    qkv = {}
    lt = txt.shape[0]
    for s, x, ang in (("img", img, angles[lt:]), ("txt", txt, angles[:lt])):
        sh1, sc1 = mods[s][0], mods[s][1]
        xm = bf16(adaln_modulate(bits(x), bits(sc1[None]), bits(sh1[None]), LN_EPS))
        qkv[s] = _qk_normed(bf16(_lin(xm, p[s + ".qkv"])), p[s + ".q_norm"], p[s + ".k_norm"], hidden, ang)
    att = _attend(np.concatenate([qkv["txt"], qkv["img"]], axis=0), hidden)
    for s, x, a in (("img", img, att[lt:]), ("txt", txt, att[:lt])):
        sh1, sc1, g1, sh2, sc2, g2 = mods[s]
        x1 = bf16(_lin(a, p[s + ".proj"], residual_bits=bits(x), gate_bits=bits(g1)))
        xm = bf16(adaln_modulate(bits(x1), bits(sc2[None]), bits(sh2[None]), LN_EPS))
        T, sc, b = p[s + ".mlp_up"]
        h = bf16(linear_act(bits(xm), T, sc, b, ACT_GELU_TANH, 0))
        out[s] = bf16(_lin(h, p[s + ".mlp_down"], residual_bits=bits(x1), gate_bits=bits(g2)))
    return out["img"], out["txt"]


def single_block(x: np.ndarray, vec: np.ndarray, p: dict, angles: np.ndarray) -> np.ndarray:
    """FLUX.1's single-stream block on x [L, C] (text tokens, then image
    tokens; bf16 values in float64).  One linear projects to q, k, v and the
    MLP's hidden layer; the second reads the attention output and the
    activated hidden layer side by side.  Returns x as bf16 values."""
    hidden = x.shape[1]
    m = bf16(_lin(bf16(silu(vec)), p["mod"]))[0]
    sh, sc, g = m[:hidden], m[hidden:2 * hidden], m[2 * hidden:]
    xm = bf16(adaln_modulate(bits(x), bits(sc[None]), bits(sh[None]), LN_EPS))
    T, s1, b1 = p["linear1"]
    z = linear(bits(xm), T, s1, b1)
    qkv = _qk_normed(bf16(z[:, :3 * hidden]), p["q_norm"], p["k_norm"], hidden, angles)
    mlp = bf16(gelu_tanh(z[:, 3 * hidden:]))
    att = _attend(qkv, hidden)
    return bf16(_lin(np.concatenate([att, mlp], axis=1), p["linear2"], residual_bits=bits(x), gate_bits=bits(g)))


def from_bits(b) -> np.ndarray:
    return bf16_bits_to_f64(np.asarray(b, dtype=np.uint16))
