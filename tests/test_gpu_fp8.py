"""FP8 (E4M3) activations through the C ABI on the GPU, against the fp64 oracle.

Page "1.58-bit FLUX" (arXiv 2412.18653), Section 4, names quantising the
activations as the step the method leaves out.  The reading tested here (the
oracle's quantize_act_e4m3 / linear_act_e4m3): per token row a_m = max|x| / 448
and x / a_m in fp32 with IEEE division, rounded to E4M3 to nearest even with
saturation; y = a_m * s_n * sum_k xq * T + b_n.

Bars:
  * a_m bit for bit, and every E4M3 byte of xq bit for bit: both sides decide
    the codes in the same precision (fp32), so nothing is near-threshold here.
    The GPU stores xq with the halves of every 16-element group interleaved
    (include/tern.h); the test undoes that with its own copy of the rule.
  * y: |y - y_ref| <= 8e-3 |y_ref| + 1e-3 rms(y_ref) against the oracle's own
    end-to-end E4M3 linear (it quantises x itself) on the GPU-produced ternary
    codes: the products are exact, the fp32 accumulation adds ~1e-6 relative
    and the single bf16 output rounding 2^-9, so the bf16 path's rule applies.
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


def natural_order(xq_dev: np.ndarray) -> np.ndarray:
    """Undo the interleaving of include/tern.h: byte 16g + 2i holds k = 16g + i,
    byte 16g + 2i + 1 holds k = 16g + 8 + i."""
    M, K = xq_dev.shape
    g = xq_dev.reshape(M, K // 16, 8, 2)
    return np.concatenate([g[..., 0], g[..., 1]], axis=2).reshape(M, K)


def check_act(x_cpu: torch.Tensor):
    xq, a = tern.quantize_act_e4m3(x_cpu.cuda())
    torch.cuda.synchronize()
    assert tern.device_status() == 0
    q_ref, a_ref = oracle.quantize_act_e4m3(bits(x_cpu))
    a_gpu = a.cpu().numpy().astype(np.float64)
    assert np.array_equal(a_gpu, a_ref), f"scales differ at rows {np.nonzero(a_gpu != a_ref)[0][:8]}"
    got = natural_order(xq.cpu().numpy())
    want = oracle.fp8_e4m3_bits(q_ref)
    bad = got != want
    assert not bad.any(), (f"{int(bad.sum())} of {bad.size} E4M3 bytes differ; first at "
                           f"{np.argwhere(bad)[0]}: {got[bad][0]:#04x} vs {want[bad][0]:#04x}")
    return xq, a


@pytest.mark.parametrize("M,K", [(1, 64), (7, 192), (33, 3072), (130, 1024), (4096, 3072), (64, 15360)])
def test_quantize_act_matches_oracle(M, K):
    check_act(rand_bf16((M, K), 1.0, M + K))


def test_quantize_act_special_rows():
    """A zero row (scale 1, zero codes), a row whose values sit on E4M3 rounding
    ties after scaling, tiny values that scale into E4M3 subnormals, huge
    values, a single non-zero element, and negative zeros."""
    K = 256
    x = rand_bf16((8, K), 1.0, 5)
    x[0] = 0
    # max 448 -> a = 1 exactly; 1.0625 (tie between 1 and 1.125 -> the even
    # mantissa, 1), 1.1875 (tie between 1.125 and 1.25 -> 1.25), -3.125 (tie
    # between -3 and -3.25 -> -3)
    x[1] = 0
    x[1, :4] = torch.tensor([448.0, 1.0625, 1.1875, -3.125])
    x[2] = (torch.randn(K, generator=torch.Generator().manual_seed(6)) * 1e-3).to(torch.bfloat16)
    x[2, 7] = 30.0  # others scale to ~1e-2 .. 1e-4: many E4M3 subnormals and zeros
    x[3] = (torch.randn(K, generator=torch.Generator().manual_seed(7)) * 1e30).to(torch.bfloat16)
    x[4] = 0
    x[4, 100] = -2.5
    x[5] = -0.0
    x[5, 3] = 1.0
    xq, a = check_act(x)
    assert a[0].item() == 1.0 and a[1].item() == 1.0
    nat = natural_order(xq.cpu().numpy())
    assert not nat[0].any()
    assert list(nat[1, :4]) == [0x7E, 0x38, 0x3A, 0xC4]  # 448, 1.0, 1.25, -3.0


def test_quantize_act_scales_across_the_exponent_range():
    """Rows whose magnitudes span bf16's exponent range (1e-38 .. 1e38, bf16
    subnormals included) and random mantissas, so that x / a_m and its fp32
    rounding are exercised far from 1: every byte must still match the
    oracle's fp32 division."""
    M, K = 512, 1024
    g = torch.Generator().manual_seed(31)
    mant = torch.rand(M, K, generator=g) * 2 - 1
    expo = torch.randint(-130, 127, (M, 1), generator=g).float()
    spread = torch.randint(-20, 1, (M, K), generator=g).float()
    x = (mant * torch.pow(2.0, (expo + spread).clamp(-133, 127))).to(torch.bfloat16)
    check_act(x)


def test_quantize_act_empty_is_a_no_op():
    x = torch.empty(0, 128, dtype=torch.bfloat16, device="cuda")
    xq, a = tern.quantize_act_e4m3(x)
    assert xq.shape == (0, 128) and a.shape == (0,)


def run_fp8_case(M, N, K, seed, with_bias=True, x_std=1.0, rows=None):
    W = rand_bf16((N, K), 0.02, seed)
    x = rand_bf16((M, K), x_std, seed + 1)
    b = rand_bf16((N,), 0.01, seed + 2) if with_bias else None
    packed, scales = tern.quantize_pack(W.cuda(), EPS)
    T, bad = oracle.unpack_tiled(packed.cpu().numpy(), N, K)
    assert bad == 0
    s = scales.cpu().double().numpy()
    xq, a = tern.quantize_act_e4m3(x.cuda())
    y = tern.linear_e4m3(xq, a, packed, scales, None if b is None else b.cuda())
    torch.cuda.synchronize()
    assert tern.device_status() == 0
    sel = np.arange(M) if rows is None else rows
    y_ref = oracle.linear_act_e4m3(bits(x[sel]), T, s, None if b is None else bits(b))
    yg = y.cpu()[torch.from_numpy(sel)].double().numpy()
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    err = np.abs(yg - y_ref)
    bad = err > Y_RTOL * np.abs(y_ref) + Y_RMS * rms
    assert not bad.any(), (f"{int(bad.sum())} of {bad.size} outputs out of tolerance; worst err {err.max():.3e} "
                           f"at {np.unravel_index(err.argmax(), err.shape)}")
    return y


@pytest.mark.parametrize("M,N,K", [(1, 256, 128), (17, 256, 64), (256, 256, 192), (300, 512, 192),
                                   (513, 768, 320), (2048, 2560, 192), (1000, 256, 3072)])
def test_linear_e4m3_matches_oracle(M, N, K):
    """Ragged token tails, a single 64-k stage, a 64-k tail stage, more tiles
    than CTA pairs."""
    run_fp8_case(M, N, K, seed=M + N + K)


def test_linear_e4m3_no_bias_and_zero_rows():
    y = run_fp8_case(130, 256, 256, seed=11, with_bias=False)
    assert torch.isfinite(y.float()).all()


def test_linear_e4m3_flux_qkv_full():
    """FLUX.1-dev double-block image-stream QKV at full size (4096 x 3072 ->
    9216), every output."""
    L = workloads.CONFIGS["qkv"]
    run_fp8_case(L.M, L.N, L.K, seed=L.seed)


def test_linear_e4m3_flux_mlp_down_sampled():
    """MLP down projection (4608 x 12288 -> 3072, x ~ N(0, 0.5)), 512 seeded rows."""
    L = workloads.CONFIGS["mlp_down"]
    rows = np.sort(np.random.default_rng(3).choice(L.M, 512, replace=False))
    rows[0], rows[-1] = 0, L.M - 1
    run_fp8_case(L.M, L.N, L.K, seed=L.seed, x_std=L.x_std, rows=np.unique(rows))


def test_linear_e4m3_close_to_bf16_path():
    """The E4M3 layer differs from the bf16 layer only by the activation
    rounding: relative difference well below the 2^-4 element bound."""
    M, N, K = 512, 512, 3072
    W = rand_bf16((N, K), 0.02, 21).cuda()
    x = rand_bf16((M, K), 1.0, 22).cuda()
    packed, scales = tern.quantize_pack(W, EPS)
    y16 = tern.linear(x, packed, scales).float()
    xq, a = tern.quantize_act_e4m3(x)
    y8 = tern.linear_e4m3(xq, a, packed, scales).float()
    rel = float((y8 - y16).norm() / y16.norm())
    assert rel < 0.03, rel


def test_linear_e4m3_m_zero_is_noop():
    W = rand_bf16((256, 128), 0.02, 1).cuda()
    packed, scales = tern.quantize_pack(W, EPS)
    xq = torch.empty(0, 128, dtype=torch.uint8, device="cuda")
    a = torch.empty(0, dtype=torch.float32, device="cuda")
    y = tern.linear_e4m3(xq, a, packed, scales)
    assert y.shape == (0, 256)
