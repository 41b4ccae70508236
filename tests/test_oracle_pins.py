"""Pins for the fp64 CPU oracle, each independent of the oracle's own code.

CPU only.  The oracle is checked against: a hand-worked example, exact
rational brute force, a library routine (numpy's dense float64 matmul of the
dequantised weights), hand-computed layout positions, invariants of the
method, and the storage figures printed on page "1.58-bit FLUX"
(arXiv 2412.18653): 7.7x smaller storage with 99.5% of the 11.9B
vision-transformer parameters quantised (Abstract; Section 1).
"""
from __future__ import annotations

import itertools
import os
import random
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from bit_post_quantised_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def to_bf16_bits(values) -> np.ndarray:
    """Bit patterns of values that must be exactly representable in bf16."""
    a = np.asarray(values, dtype=np.float32)
    bits = (a.view(np.uint32) >> 16).astype(np.uint16)
    back = (bits.astype(np.uint32) << 16).view(np.float32)
    assert np.array_equal(back, a), "value not exact in bf16"
    return bits


def read_hand_example():
    rows = {}
    with open(os.path.join(GOLDEN, "hand_worked_4x4.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            rows.setdefault(key, []).append(vals)
    return rows


# ---------------------------------------------------------------- hand-worked
def test_hand_worked_example():
    g = read_hand_example()
    eps = float(g["eps"][0][0])
    W = to_bf16_bits([[float(v) for v in r] for r in g["W"]])
    T_exp = np.array([[int(v) for v in r] for r in g["T"]], np.int8)
    s_exp = np.array([float(v) for v in g["s"][0]])
    gamma_exp = np.array([float(v) for v in g["gamma"][0]])

    T, s = oracle.quantize(W, eps)
    np.testing.assert_allclose(s, s_exp, rtol=1e-12, atol=0)
    np.testing.assert_allclose(s - eps, gamma_exp, rtol=1e-12, atol=1e-15)
    np.testing.assert_array_equal(T, T_exp)

    P = oracle.pack_canonical(T)
    assert [int(b) for b in P] == [int(v, 16) for v in g["bytes"][0]]

    x = to_bf16_bits([[float(v) for v in g["x"][0]]])
    b = to_bf16_bits([float(v) for v in g["b"][0]])
    y = oracle.linear(x, T, s, b)[0]
    np.testing.assert_allclose(y, [float(v) for v in g["y"][0]], rtol=1e-12)
    y_bf16 = torch.tensor(y, dtype=torch.float64).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(y_bf16, [float(v) for v in g["y_bf16"][0]])
    acc = oracle.linear(x, T, np.ones(4), None)[0]
    np.testing.assert_array_equal(acc, [float(v) for v in g["acc"][0]])


# ------------------------------------------------------- exact brute force
def exact_round_clip(w: Fraction, s: Fraction) -> int:
    """Nearest of {-1, 0, +1} to w/s; an exact tie goes to the even value 0."""
    if s == 0:
        return 0
    r = w / s
    best = min((abs(r - t), t != 0, t) for t in (-1, 0, 1))
    return best[2]


def bf16_grid_value(rng: random.Random) -> float:
    mant = rng.randint(-255, 255)
    exp = rng.randint(-14, -4)
    return float(mant) * 2.0 ** exp


@pytest.mark.parametrize("eps", [0.0, 1e-5, 0.25])
@pytest.mark.parametrize("seed", range(6))
def test_quantize_matches_exact_rational_brute_force(eps, seed):
    rng = random.Random(seed * 7 + int(eps * 1e6))
    N, K = rng.randint(1, 8), rng.randint(1, 8)
    vals = [[bf16_grid_value(rng) if rng.random() > 0.15 else 0.0 for _ in range(K)] for _ in range(N)]
    W = to_bf16_bits(vals)
    T, s = oracle.quantize(W, eps)
    e = Fraction(eps)
    for n in range(N):
        row = [Fraction(v) for v in vals[n]]
        s_exact = sum(abs(w) for w in row) / K + e
        assert abs(Fraction(s[n]) - s_exact) <= s_exact * Fraction(1, 10**15)
        for k in range(K):
            r = abs(row[k] / s_exact) if s_exact else Fraction(0)
            if r != Fraction(1, 2) and abs(r - Fraction(1, 2)) < Fraction(1, 10**12):
                continue  # a double rounding of s could decide this one either way
            assert T[n, k] == exact_round_clip(row[k], s_exact), (n, k, vals[n])


def test_round_half_to_even_ties():
    # eps = 0 makes the ratios exact: [1, 3] -> s = 2 -> r = [0.5, 1.5].
    W = to_bf16_bits([[1, 3, 0, 0], [-1, -3, 0, 0], [1, 1, 1, 5], [3, 1, 0, 0]])
    T, s = oracle.quantize(W, 0.0)
    np.testing.assert_array_equal(s, [1.0, 1.0, 2.0, 1.0])
    # row 0: s = 1 -> r = [1, 3, 0, 0] ; row 2: r = [0.5, 0.5, 0.5, 2.5]
    np.testing.assert_array_equal(T, [[1, 1, 0, 0], [-1, -1, 0, 0], [0, 0, 0, 1], [1, 1, 0, 0]])
    W2 = to_bf16_bits([[1, 3], [-1, -3], [3, 1]])
    T2, s2 = oracle.quantize(W2, 0.0)
    np.testing.assert_array_equal(s2, [2.0, 2.0, 2.0])
    np.testing.assert_array_equal(T2, [[0, 1], [0, -1], [1, 0]])


def test_linear_exact_over_every_code_row():
    """All 3^4 ternary rows against exact rational arithmetic."""
    rng = np.random.default_rng(5)
    rows = np.array(list(itertools.product((-1, 0, 1), repeat=4)), np.int8)  # N = 81
    N, K, M = rows.shape[0], 4, 3
    x_vals = [[bf16_grid_value(random.Random(int(v))) for v in rng.integers(0, 1 << 30, K)] for _ in range(M)]
    b_vals = [bf16_grid_value(random.Random(int(v))) for v in rng.integers(0, 1 << 30, N)]
    x = to_bf16_bits(x_vals)
    b = to_bf16_bits(b_vals)
    s = rng.uniform(0.01, 0.05, N)
    y = oracle.linear(x, rows, s, b)
    for m in range(M):
        for n in range(N):
            exact = Fraction(s[n]) * sum(Fraction(x_vals[m][k]) * int(rows[n, k]) for k in range(K)) + Fraction(b_vals[n])
            # a few double roundings, relative to the size of the terms summed
            size = Fraction(s[n]) * sum(abs(Fraction(v)) for v in x_vals[m]) + abs(Fraction(b_vals[n]))
            assert abs(Fraction(y[m, n]) - exact) <= size * Fraction(1, 10**15)


@pytest.mark.parametrize("M,K,N", [(5, 12, 7), (33, 200, 130), (1, 64, 3)])
def test_linear_equals_dense_matmul_of_dequantised_weight(M, K, N):
    """numpy's float64 matmul of T*s (scale before the sum) is the library check."""
    rng = np.random.default_rng(M * 1000 + N)
    x = workloads.bf16_bits(torch.randn(M, K, generator=torch.Generator().manual_seed(N)).to(torch.bfloat16))
    b = workloads.bf16_bits((0.1 * torch.randn(N, generator=torch.Generator().manual_seed(M))).to(torch.bfloat16))
    T = rng.integers(-1, 2, (N, K)).astype(np.int8)
    s = rng.uniform(0.001, 0.1, N)
    y = oracle.linear(x, T, s, b)
    xd = oracle.bf16_bits_to_f64(x)
    bd = oracle.bf16_bits_to_f64(b)
    y_lib = xd @ (T.astype(np.float64) * s[:, None]).T + bd
    np.testing.assert_allclose(y, y_lib, rtol=1e-12, atol=1e-13)
    y_nobias = oracle.linear(x, T, s, None)
    np.testing.assert_allclose(y_nobias, y_lib - bd, rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- packing
def two_bit_fields(P: np.ndarray) -> np.ndarray:
    return np.stack([(P >> sh) & 3 for sh in (0, 2, 4, 6)], axis=-1).ravel()


def test_canonical_pack_roundtrip_and_codes():
    rng = np.random.default_rng(0)
    T = rng.integers(-1, 2, (37, 48)).astype(np.int8)
    P = oracle.pack_canonical(T)
    assert P.size == 37 * 48 // 4
    fields = two_bit_fields(P)
    assert not np.any(fields == 2), "pattern 10 must never be written"
    # counts of each code equal the counts of each value
    assert np.sum(fields == 1) == np.sum(T == 1)
    assert np.sum(fields == 3) == np.sum(T == -1)
    U, bad = oracle.unpack_canonical(P, 37, 48)
    assert bad == 0
    np.testing.assert_array_equal(U, T)
    # a byte holding only the invalid pattern is reported
    _, bad = oracle.unpack_canonical(np.array([0b10], np.uint8), 1, 4)
    assert bad == 1


def test_canonical_single_rows():
    assert oracle.pack_canonical(np.array([[-1, -1, -1, -1]], np.int8))[0] == 0xFF
    assert oracle.pack_canonical(np.array([[0, 0, 1, 0]], np.int8))[0] == 0x10
    assert oracle.pack_canonical(np.array([[0, -1, 0, 0]], np.int8))[0] == 0x0C


def read_positions():
    out = []
    with open(os.path.join(GOLDEN, "tiled_positions.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                out.append(tuple(int(v) for v in line.split()))
    return out


@pytest.mark.parametrize("pos", read_positions())
def test_tiled_layout_hand_positions(pos):
    N, K, n, k, value, byte, shift = pos
    T = np.zeros((N, K), np.int8)
    T[n, k] = value
    P = oracle.pack_tiled(T)
    assert P.size == N * K // 4
    nz = np.nonzero(P)[0]
    assert list(nz) == [byte]
    assert P[byte] == ((value & 3) << shift)
    U, bad = oracle.unpack_tiled(P, N, K)
    assert bad == 0
    np.testing.assert_array_equal(U, T)


def test_tiled_layout_ragged_n_pads_whole_slabs():
    """N % 128 != 0 (N % 16 == 0): the layout keeps whole 128-channel slabs;
    an element of the first slab keeps its hand-computed position (which
    does not depend on N), the channels past N are zero bytes, and unpack
    inverts pack."""
    used = 0
    for N0, K, n, k, value, byte, shift in read_positions():
        if n >= 48:
            continue
        T = np.zeros((48, K), np.int8)
        T[n, k] = value
        P = oracle.pack_tiled(T)
        assert P.size == 128 * K // 4
        assert list(np.nonzero(P)[0]) == [byte] and P[byte] == ((value & 3) << shift)
        used += 1
    assert used >= 2
    rng = np.random.default_rng(4)
    N, K = 208, 128  # two slabs, the second 80 channels deep
    T = rng.integers(-1, 2, (N, K)).astype(np.int8)
    P = oracle.pack_tiled(T)
    assert P.size == 256 * K // 4
    for kc in range(K // 64):  # slab 1, chunk kc: rows 80..127 are padding
        g0 = (1 * (K // 64) + kc) * 2048
        assert not P[g0 + 80 * 16:g0 + 128 * 16].any()
    U, bad = oracle.unpack_tiled(P, N, K)
    assert bad == 0
    np.testing.assert_array_equal(U, T)
    with pytest.raises(ValueError):
        oracle.pack_tiled(np.zeros((40, 64), np.int8))


def test_tiled_is_a_permutation_of_canonical():
    rng = np.random.default_rng(1)
    N, K = 256, 192
    T = rng.integers(-1, 2, (N, K)).astype(np.int8)
    Pt = oracle.pack_tiled(T)
    Pc = oracle.pack_canonical(T)
    assert Pt.size == Pc.size == N * K // 4
    ft, fc = two_bit_fields(Pt), two_bit_fields(Pc)
    assert np.array_equal(np.bincount(ft, minlength=4), np.bincount(fc, minlength=4))
    U, bad = oracle.unpack_tiled(Pt, N, K)
    assert bad == 0
    np.testing.assert_array_equal(U, T)
    with pytest.raises(ValueError):
        oracle.pack_tiled(np.zeros((100, 64), np.int8))
    with pytest.raises(ValueError):
        oracle.pack_tiled(np.zeros((128, 48), np.int8))


# ------------------------------------------------------------- invariants
def random_W(N, K, seed, std=0.02):
    g = torch.Generator().manual_seed(seed)
    return workloads.bf16_bits((torch.randn(N, K, generator=g) * std).to(torch.bfloat16))


def test_quantizer_invariants():
    W = random_W(64, 96, 3)
    T, s = oracle.quantize(W, 1e-5)
    assert set(np.unique(T)) <= {-1, 0, 1}
    assert np.all(s > 0)
    # scaling by 2 is exact in bf16: with eps = 0 the scales double, codes stay
    Wd = oracle.bf16_bits_to_f64(W)
    W2 = to_bf16_bits((2.0 * Wd).astype(np.float32))
    T0, s0 = oracle.quantize(W, 0.0)
    T2, s2 = oracle.quantize(W2, 0.0)
    np.testing.assert_array_equal(s2, 2.0 * s0)
    np.testing.assert_array_equal(T2, T0)
    # negation flips every code and keeps the scale
    Wn = W ^ np.uint16(0x8000)
    Tn, sn = oracle.quantize(Wn, 1e-5)
    np.testing.assert_array_equal(sn, s)
    np.testing.assert_array_equal(Tn, -T)
    # a zero row: s = eps and all codes 0; with eps = 0 still all codes 0
    Z = np.zeros((2, 8), np.uint16)
    Tz, sz = oracle.quantize(Z, 1e-5)
    np.testing.assert_array_equal(sz, [1e-5, 1e-5])
    assert not Tz.any()
    Tz0, sz0 = oracle.quantize(Z, 0.0)
    assert not Tz0.any() and not sz0.any()
    # equal magnitudes: every code is the sign
    E = to_bf16_bits([[0.5, -0.5, 0.5, 0.5, -0.5, -0.5, 0.5, -0.5]])
    Te, _ = oracle.quantize(E, 1e-5)
    np.testing.assert_array_equal(Te[0], np.sign(oracle.bf16_bits_to_f64(E)[0]).astype(np.int8))


def test_given_scale_ternarize_and_near_threshold():
    # eps = 0, row [1, 3]: s = 2, r = [0.5, 1.5]; the 0.5 element sits on the threshold
    W = to_bf16_bits([[1, 3]])
    T, s = oracle.quantize(W, 0.0)
    assert s[0] == 2.0
    cnt, mask = oracle.near_threshold(W, s, 1e-6)
    assert cnt == 1 and mask[0, 0] and not mask[0, 1:].any()
    # a scale a hair off moves r off the threshold by ~1e-7: still counted
    s_off = s * (1 + 2e-7)
    cnt2, _ = oracle.near_threshold(W, s_off, 1e-6)
    assert cnt2 == 1
    # far from it: not counted
    cnt3, _ = oracle.near_threshold(W, s * 0.8, 1e-6)
    assert cnt3 == 0
    np.testing.assert_array_equal(oracle.ternarize(W, s * 0.8), [[1, 1]])
    np.testing.assert_array_equal(oracle.ternarize(W, s * 1.2), [[0, 1]])


# ------------------------------------------------- the pages' storage figure
def test_storage_ratio_matches_pages():
    """7.7x smaller storage with 99.5% of 11.9B parameters ternary (Abstract; Section 1)."""
    for N, K in [(256, 256), (9216, 3072)]:
        assert oracle.pack_canonical(np.zeros((N, K), np.int8)).nbytes * 8 == N * K * 2  # 2 bits each
    layers = workloads.flux_stack()
    assert len(layers) == 19 * 2 * 5 + 38 * 3
    p_ternary = sum(l.N * l.K for l in layers)
    channels = sum(l.N for l in layers)
    total = 11.9e9
    assert abs(p_ternary / total - 0.995) < 1e-3  # "99.5% of the 11.9B parameters"
    bits_bf16 = 16 * total
    bits_ternary = 2 * p_ternary + 32 * channels + 16 * (total - p_ternary)
    ratio = bits_bf16 / bits_ternary
    assert round(ratio, 1) == 7.7
    # without the per-channel scales and the 0.5% kept in 16 bit it would be 8x
    assert 16 / 2 == 8.0


# ------------------------------------------------- fused GELU epilogue (tanh form)
# Pins of oracle.gelu_tanh that do not retype its formula: an exact symmetry,
# the Taylor coefficients at 0 (which fix sqrt(2/pi) and 0.044715), the
# limits, and torch's own implementation of the same activation.

def test_gelu_tanh_symmetry_and_limits():
    rng = np.random.default_rng(7)
    v = rng.normal(0.0, 3.0, size=(4, 257))
    g, gm = oracle.gelu_tanh(v), oracle.gelu_tanh(-v)
    # g(v) - g(-v) = v: 0.5 v (1 + t) + 0.5 v (1 - t) with t odd in v
    assert np.allclose(g - gm, v, rtol=0, atol=1e-12)
    big = np.array([[10.0, 20.0, 40.0]])
    assert np.array_equal(oracle.gelu_tanh(big), big)
    assert np.all(np.abs(oracle.gelu_tanh(-big)) < 1e-15)
    assert oracle.gelu_tanh(np.zeros((1, 3))).tolist() == [[0.0, 0.0, 0.0]]


def test_gelu_tanh_taylor_coefficients_at_zero():
    # even part (g(h) + g(-h)) / 2 = (c/2) h^2 + (c a - c^3/3)/2 h^4 + O(h^6),
    # c = sqrt(2/pi), a = 0.044715
    c, a = np.sqrt(2.0 / np.pi), 0.044715
    h1, h2 = 1e-2, 2e-2
    e = lambda h: 0.5 * (oracle.gelu_tanh(np.array([[h]]))[0, 0] + oracle.gelu_tanh(np.array([[-h]]))[0, 0])
    # eliminate the h^4 term from two step sizes: c2 = (16 e(h1) - e(h2)) / (12 h1^2)
    c2 = (16 * e(h1) - e(h2)) / (12 * h1 * h1)
    assert abs(c2 - c / 2) < 1e-9
    # and the h^4 coefficient from the same two steps: e(h)/h^2 = c2 + c4 h^2 + O(h^4)
    c4 = (e(h2) / h2 ** 2 - e(h1) / h1 ** 2) / (h2 ** 2 - h1 ** 2)
    assert abs(c4 - 0.5 * (c * a - c ** 3 / 3)) < 1e-5


def test_gelu_tanh_matches_torch():
    v = torch.linspace(-12, 12, 4801, dtype=torch.float64).reshape(1, -1)
    ref = torch.nn.functional.gelu(v, approximate="tanh").numpy()
    assert np.allclose(oracle.gelu_tanh(v.numpy()), ref, rtol=1e-13, atol=1e-15)


def test_linear_act_touches_only_columns_from_col0():
    rng = np.random.default_rng(3)
    M, K, N = 3, 64, 256
    x = workloads.bf16_bits(torch.randn(M, K).to(torch.bfloat16))
    T = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    s = rng.uniform(0.01, 0.03, size=N)
    b = workloads.bf16_bits((torch.randn(N) * 0.01).to(torch.bfloat16))
    y = oracle.linear(x, T, s, b)
    ya = oracle.linear_act(x, T, s, b, oracle.ACT_GELU_TANH, 128)
    assert np.array_equal(ya[:, :128], y[:, :128])
    assert np.array_equal(ya[:, 128:], oracle.gelu_tanh(y[:, 128:]))
    assert np.array_equal(oracle.linear_act(x, T, s, b, oracle.ACT_NONE, 0), y)
    with pytest.raises(ValueError):
        oracle.linear_act(x, T, s, b, 7, 0)


def test_linear_epilogue_gate_and_residual_algebra():
    """residual + gate * a: gate 0 gives the residual exactly, no residual and
    no gate give linear_act, and the gated part scales linearly with gate."""
    rng = np.random.default_rng(4)
    M, K, N = 5, 128, 256
    x = workloads.bf16_bits(torch.randn(M, K).to(torch.bfloat16))
    T = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    s = rng.uniform(0.01, 0.03, size=N)
    b = workloads.bf16_bits((torch.randn(N) * 0.01).to(torch.bfloat16))
    r = workloads.bf16_bits(torch.randn(M, N).to(torch.bfloat16))
    g = workloads.bf16_bits((torch.rand(N) * 2 - 0.5).to(torch.bfloat16))
    zero = workloads.bf16_bits(torch.zeros(N, dtype=torch.bfloat16))
    two = workloads.bf16_bits(torch.full((N,), 2.0, dtype=torch.bfloat16))
    one = workloads.bf16_bits(torch.ones(N, dtype=torch.bfloat16))
    r64 = oracle.bf16_bits_to_f64(r)
    for act, col0 in ((oracle.ACT_NONE, 0), (oracle.ACT_GELU_TANH, 96)):
        a = oracle.linear_act(x, T, s, b, act, col0)
        assert np.array_equal(oracle.linear_epilogue(x, T, s, b, act, col0), a)
        assert np.array_equal(oracle.linear_epilogue(x, T, s, b, act, col0, r, zero), r64)
        y1 = oracle.linear_epilogue(x, T, s, b, act, col0, r, one)
        y2 = oracle.linear_epilogue(x, T, s, b, act, col0, r, two)
        assert np.allclose(y2 - r64, 2 * (y1 - r64), rtol=1e-14, atol=1e-14)
        yg = oracle.linear_epilogue(x, T, s, b, act, col0, None, g)
        assert np.allclose(yg, a * oracle.bf16_bits_to_f64(g)[None, :], rtol=1e-15, atol=0)


def test_rms_norm_groups_properties_and_torch():
    """Per-128-column RMS normalisation: unit mean square per group (eps 0),
    scale invariance, groups independent, columns outside untouched, and
    torch's rms_norm on each group."""
    rng = np.random.default_rng(9)
    y = rng.normal(0.0, 2.0, size=(6, 512))
    n = oracle.rms_norm_groups(y, 128, 384, 0.0)
    assert np.array_equal(n[:, :128], y[:, :128]) and np.array_equal(n[:, 384:], y[:, 384:])
    for g0 in (128, 256):
        assert np.allclose(np.mean(n[:, g0:g0 + 128] ** 2, axis=1), 1.0, rtol=1e-13)
    assert np.allclose(oracle.rms_norm_groups(3.5 * y, 128, 384, 0.0)[:, 128:384], n[:, 128:384], rtol=1e-13,
                       atol=1e-15)
    y2 = y.copy()
    y2[:, 128:256] *= 7.0
    assert np.array_equal(oracle.rms_norm_groups(y2, 128, 384, 0.0)[:, 256:384], n[:, 256:384])
    w = workloads.bf16_bits((torch.rand(512) + 0.5).to(torch.bfloat16))
    got = oracle.rms_norm_groups(y, 0, 512, 1e-6, w)
    wt = torch.from_numpy(oracle.bf16_bits_to_f64(w))
    for g0 in range(0, 512, 128):
        ref = torch.nn.functional.rms_norm(torch.from_numpy(y[:, g0:g0 + 128]), (128,), wt[g0:g0 + 128], 1e-6)
        assert np.allclose(got[:, g0:g0 + 128], ref.numpy(), rtol=1e-12, atol=1e-14)
    with pytest.raises(ValueError):
        oracle.rms_norm_groups(y, 64, 256, 1e-6)


def test_adaln_modulate_closed_form_and_torch():
    """adaLN modulation: a row of alternating +-a has mean 0 and variance a^2,
    so its normalised values are +-a / sqrt(a^2 + eps) exactly; with scale
    and shift the closed form (1 + scale) * that + shift (a sign slip, a
    dropped 1 + or a shift applied before the scale fails it).  With scale =
    shift = 0 it is torch's layer_norm without affine, in float64."""
    K = 16
    a, eps = 0.75, 1e-6
    row = np.array([a if k % 2 == 0 else -a for k in range(K)])
    sc = (np.arange(K) - 8) / 16.0  # bf16-exact
    sh = (3 * np.arange(K) - 20) / 32.0
    x_bits, sc_bits, sh_bits = to_bf16_bits(row[None, :]), to_bf16_bits(sc), to_bf16_bits(sh)
    got = oracle.adaln_modulate(x_bits, sc_bits, sh_bits, eps)
    sc64 = oracle.bf16_bits_to_f64(sc_bits)
    sh64 = oracle.bf16_bits_to_f64(sh_bits)
    n = np.where(np.arange(K) % 2 == 0, 1.0, -1.0) * a / np.sqrt(a * a + eps)
    assert np.allclose(got[0], n * (1.0 + sc64) + sh64, rtol=1e-14, atol=1e-15)

    rng = np.random.default_rng(11)
    x = torch.from_numpy(rng.normal(0.3, 2.0, size=(5, 384))).to(torch.bfloat16)
    xb = workloads.bf16_bits(x)
    zeros = np.zeros(384, np.uint16)
    got = oracle.adaln_modulate(xb, zeros, zeros, 1e-6)
    ref = torch.nn.functional.layer_norm(x.double(), (384,), eps=1e-6).numpy()
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-13)


def test_adaln_modulate_invariants_and_row_groups():
    """With eps = 0 the normalisation ignores a positive scale and an offset
    of the row; each token row takes modulation row m // tokens_per_row."""
    rng = np.random.default_rng(12)
    M, K, T = 6, 256, 4
    xv = rng.integers(-32, 33, size=(M, K)) / 8.0  # on a grid where 2x + 1 stays exact in bf16
    x_bits = to_bf16_bits(xv)
    sc_bits = workloads.bf16_bits((torch.rand(2, K) - 0.5).to(torch.bfloat16))
    sh_bits = workloads.bf16_bits((torch.rand(2, K) - 0.5).to(torch.bfloat16))
    base = oracle.adaln_modulate(x_bits, sc_bits, sh_bits, 0.0, T)
    moved_bits = to_bf16_bits(xv * 2.0 + 1.0)
    assert np.allclose(oracle.adaln_modulate(moved_bits, sc_bits, sh_bits, 0.0, T), base, rtol=1e-12, atol=1e-12)
    # rows 0..3 use modulation row 0, rows 4..5 row 1
    top = oracle.adaln_modulate(x_bits[:T], sc_bits[0], sh_bits[0], 0.0)
    bot = oracle.adaln_modulate(x_bits[T:], sc_bits[1], sh_bits[1], 0.0)
    assert np.array_equal(base[:T], top) and np.array_equal(base[T:], bot)
    # unit variance and zero mean of the normalised rows (scale = shift = 0)
    zeros = np.zeros(K, np.uint16)
    v = oracle.adaln_modulate(x_bits, zeros, zeros, 0.0)
    assert np.allclose(v.mean(axis=1), 0.0, atol=1e-13) and np.allclose(v.var(axis=1), 1.0, rtol=1e-12)
    with pytest.raises(ValueError):
        oracle.adaln_modulate(x_bits, sc_bits[:1], sh_bits[:1], 0.0, T)


def test_fp8_e4m3_rounding_against_torch_and_closed_forms():
    """E4M3 rounding: torch's float8_e4m3fn conversion (a library routine) on
    values up to 448 including subnormals and exact ties, the eight
    mantissas of [1, 2), ties to even, the extremes, and saturation."""
    rng = np.random.default_rng(13)
    v = np.concatenate([rng.uniform(-448, 448, 4000), rng.uniform(-0.02, 0.02, 2000),
                        rng.uniform(-2.0 ** -6, 2.0 ** -6, 1000)])
    # exact midpoints between neighbours in several binades (ties)
    for e in (-9, -7, -6, -3, 0, 4, 7):
        for m in range(8):
            lo = (8 + m) * 2.0 ** (e - 3) if e >= -6 else m * 2.0 ** -9
            v = np.append(v, [lo + 2.0 ** (max(e, -6) - 4), -(lo + 2.0 ** (max(e, -6) - 4))])
    v = v[np.abs(v) <= 448]
    ref = torch.from_numpy(v.astype(np.float32)).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(oracle.fp8_e4m3_rne(v.astype(np.float32).astype(np.float64)), ref)
    assert list(oracle.fp8_e4m3_rne(1 + np.arange(8) / 8.0)) == list(1 + np.arange(8) / 8.0)
    assert oracle.fp8_e4m3_rne(1.0625) == 1.0 and oracle.fp8_e4m3_rne(1.1875) == 1.25  # ties to even
    assert oracle.fp8_e4m3_rne(2.0 ** -9) == 2.0 ** -9 and oracle.fp8_e4m3_rne(2.0 ** -10) == 0.0
    assert oracle.fp8_e4m3_rne(448.0) == 448.0 and oracle.fp8_e4m3_rne(-1000.0) == -448.0


def test_act_e4m3_linear_lossless_on_grid_and_bounded_otherwise():
    """Rows whose values are E4M3 values times a power of two, with the
    largest magnitude 448 times that power, quantise without loss, so the
    linear equals the unquantised one exactly; otherwise each activation
    moves by at most 2^-4 of its magnitude (3 mantissa bits) or one
    subnormal step, and y by the matching bound.  The absmax element of a
    row maps to +-448."""
    rng = np.random.default_rng(14)
    M, K, N = 5, 128, 64
    grid = np.concatenate([(8 + np.arange(8)) * 2.0 ** (e - 3) for e in range(-6, 9)])
    grid = grid[grid <= 448]
    xq = rng.choice(grid, size=(M, K)) * rng.choice([-1.0, 1.0], size=(M, K))
    xq[:, 0] = 448.0
    x = xq * (2.0 ** -6)  # every value and the scale exact in bf16
    x_bits = to_bf16_bits(x)
    T = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    s = rng.uniform(0.01, 0.03, N)
    got = oracle.linear_act_e4m3(x_bits, T, s)
    assert np.array_equal(got, oracle.linear(x_bits, T, s))
    q, a = oracle.quantize_act_e4m3(x_bits)
    assert np.all(q[:, 0] == 448.0) and np.all(a == 2.0 ** -6)

    xr = torch.randn(M, K, generator=torch.Generator().manual_seed(15)).to(torch.bfloat16)
    xb = workloads.bf16_bits(xr)
    q, a = oracle.quantize_act_e4m3(xb)
    x64 = oracle.bf16_bits_to_f64(xb)
    assert np.all(np.max(np.abs(q), axis=1) == 448.0)
    err = np.abs(q * a[:, None] - x64)
    assert np.all(err <= 2.0 ** -4 * np.abs(x64) * (1 + 1e-6) + 2.0 ** -9 * a[:, None])
    y = oracle.linear_act_e4m3(xb, T, s)
    y_ref = oracle.linear(xb, T, s)
    bound = (err @ np.abs(T.astype(np.float64)).T) * s[None, :]
    assert np.all(np.abs(y - y_ref) <= bound * (1 + 1e-9) + 1e-12)


def test_fp8_e4m3_bytes_against_torch():
    """E4M3 encoding of every finite E4M3 value (all 254 non-NaN bytes,
    through torch's float8_e4m3fn), and the codes +1 -> 0x38, -1 -> 0xB8,
    0 -> 0x00 that ternary weights take in an FP8 MMA."""
    b = torch.arange(256, dtype=torch.uint8)
    b = b[(b & 0x7F) != 0x7F]  # the two NaN bytes
    vals = b.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(oracle.fp8_e4m3_bits(vals), b.numpy())
    assert list(oracle.fp8_e4m3_bits([1.0, -1.0, 0.0, 448.0, 2.0 ** -9])) == [0x38, 0xB8, 0x00, 0x7E, 0x01]
    with pytest.raises(ValueError):
        oracle.fp8_e4m3_bits([1.0625])
