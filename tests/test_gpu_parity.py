"""GPU parity: the sm_100a kernels behind the C ABI against the fp64 CPU oracle.

Rules (written here, checked element by element):
  * scales: |s_gpu - s_oracle| <= 1e-6 * s_oracle;
  * codes: bit-exact given the GPU's scales, except elements whose |w|/s lies
    within 1e-6 of the 0.5 rounding threshold, which are counted and reported;
  * linear: |y - y_ref| <= 8e-3 |y_ref| + 1e-3 rms(y_ref), with y_ref the
    oracle's fp64 linear on the GPU-produced codes and scales.  The bound
    covers bf16's 2^-9 relative output rounding plus fp32 accumulation.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from bit_post_quantised_b200 import tern, workloads

pytestmark = pytest.mark.gpu

SCALE_RTOL = 1e-6
BAND = 1e-6
Y_RTOL = 8e-3
Y_RMS = 1e-3
EPS = workloads.EPS


def bits(t: torch.Tensor) -> np.ndarray:
    return workloads.bf16_bits(t.detach().cpu())


def rand_bf16(shape, std, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * std).to(torch.bfloat16)


def quantize_on_gpu(W_cpu: torch.Tensor):
    W = W_cpu.cuda()
    packed, scales = tern.quantize_pack(W, EPS)
    torch.cuda.synchronize()
    assert tern.device_status() == 0
    return packed, scales


def check_quantize(W_cpu, packed, scales, report):
    N, K = W_cpu.shape
    Wb = bits(W_cpu)
    s_gpu = scales.cpu().double().numpy()
    s_ref = oracle.absmean_scales(Wb, EPS)
    rel = np.abs(s_gpu - s_ref) / s_ref
    assert rel.max() <= SCALE_RTOL, f"scale rel err {rel.max():.3e}"
    P = packed.cpu().numpy()
    assert P.size == N * K // 4
    T_gpu, bad = oracle.unpack_tiled(P, N, K)
    assert bad == 0, "pattern 10 written"
    T_ref = oracle.ternarize(Wb, s_gpu)
    near_cnt, near = oracle.near_threshold(Wb, s_gpu, BAND)
    diff = T_gpu != T_ref
    assert not np.any(diff & ~near), f"{int(np.sum(diff & ~near))} codes differ off the threshold"
    report["near_threshold"] = near_cnt
    report["near_flips"] = int(np.sum(diff & near))
    # end to end against the oracle's own quantisation: only threshold flips
    T_own, _ = oracle.quantize(Wb, EPS)
    near_own_cnt, near_own = oracle.near_threshold(Wb, s_ref, BAND)
    d2 = T_gpu != T_own
    assert not np.any(d2 & ~near_own)
    return T_gpu, s_gpu


def check_y(y_gpu: torch.Tensor, y_ref: np.ndarray):
    y = y_gpu.detach().cpu().double().numpy()
    assert y.shape == y_ref.shape
    rms = float(np.sqrt(np.mean(y_ref ** 2))) if y_ref.size else 0.0
    err = np.abs(y - y_ref)
    bound = Y_RTOL * np.abs(y_ref) + Y_RMS * rms
    bad = err > bound
    assert not bad.any(), (f"{int(bad.sum())} of {bad.size} outputs out of tolerance; "
                           f"worst err {err.max():.3e} at {np.unravel_index(err.argmax(), err.shape)}")
    return float((err / (np.abs(y_ref) + rms)).max()) if y_ref.size else 0.0


# ------------------------------------------------------------- quantise/pack
@pytest.mark.parametrize("N,K", [(128, 64), (256, 256), (384, 320), (128, 1024), (1280, 3072)])
def test_quantize_pack_small(N, K):
    W = rand_bf16((N, K), 0.02, N * 7 + K)
    packed, scales = quantize_on_gpu(W)
    check_quantize(W, packed, scales, {})


def test_quantize_pack_special_rows():
    """Zero rows, equal magnitudes, exact threshold ties, large and tiny values."""
    N, K = 128, 128
    W = rand_bf16((N, K), 0.02, 99)
    W[0] = 0
    W[1] = 0.5
    W[2, ::2] = -0.25
    W[2, 1::2] = 0.25
    W[3, :2] = torch.tensor([1.0, 3.0])  # mean 4/128, far above threshold
    W[3, 2:] = 0
    W[4] = torch.tensor([1e-30] * K)
    W[5, 0] = 1e4
    packed, scales = quantize_on_gpu(W)
    check_quantize(W, packed, scales, {})
    s = scales.cpu()
    assert s[0].item() == pytest.approx(EPS, rel=1e-7)
    T, _ = oracle.unpack_tiled(packed.cpu().numpy(), N, K)
    assert not T[0].any()
    assert (T[1] == 1).all()


def test_quantize_pack_tiny_thresholds_eps_zero():
    """eps = 0 and rows of tiny magnitudes, so that s_n / 2 falls below the
    smallest normal bf16 (the kernel then decides the codes with integer
    compares instead of bf16 ones), or right at it, or just above; bf16
    subnormal weights among them.  Codes must equal the oracle's |w| > s_n / 2
    for the GPU's s_n exactly; s_n as the oracle's mean."""
    N, K = 128, 192
    g = torch.Generator().manual_seed(17)
    W = torch.zeros(N, K)
    tiny = 2.0 ** -126  # smallest normal fp32 / bf16
    for n in range(N):
        mag = tiny * 2.0 ** (n % 12 - 8)  # s/2 from ~2^-135 (subnormal) to ~2^-124
        W[n] = torch.randn(K, generator=g) * mag
    W = W.to(torch.bfloat16)
    packed, scales = tern.quantize_pack(W.cuda(), 0.0)
    torch.cuda.synchronize()
    assert tern.device_status() == 0
    Wb = bits(W)
    s_gpu = scales.cpu().double().numpy()
    s_ref = oracle.absmean_scales(Wb, 0.0)
    # fp32 subnormal scales carry fewer digits: one rounding of the fp32 grid
    assert np.all(np.abs(s_gpu - s_ref) <= 1e-6 * s_ref + 2.0 ** -149)
    T_gpu, bad = oracle.unpack_tiled(packed.cpu().numpy(), N, K)
    assert bad == 0
    assert np.array_equal(T_gpu, oracle.ternarize(Wb, s_gpu))
    assert (T_gpu != 0).any(axis=1).all()  # every row has codes on both sides of the threshold


@pytest.mark.parametrize("N,K", [(9216, 3072), (12288, 3072), (3072, 12288), (21504, 3072), (3072, 15360),
                                 (18432, 3072)])
def test_quantize_pack_flux_shapes(N, K):
    """Every weight shape of the FLUX linear stack, in full."""
    W = rand_bf16((N, K), workloads.W_STD, 5000 + N + K)
    packed, scales = quantize_on_gpu(W)
    rep = {}
    check_quantize(W, packed, scales, rep)
    print(f"N={N} K={K}: near-threshold elements {rep['near_threshold']}, flips {rep['near_flips']}")


# ---------------------------------------------------------------- linear
def run_linear_case(M, N, K, seed, with_bias=True, x_std=1.0):
    W = rand_bf16((N, K), 0.02, seed)
    x = rand_bf16((M, K), x_std, seed + 1)
    b = rand_bf16((N,), 0.01, seed + 2) if with_bias else None
    packed, scales = quantize_on_gpu(W)
    T, s = check_quantize(W, packed, scales, {})
    y = tern.linear(x.cuda(), packed, scales, None if b is None else b.cuda())
    torch.cuda.synchronize()
    assert tern.device_status() == 0
    y_ref = oracle.linear(bits(x), T, s, None if b is None else bits(b))
    return check_y(y, y_ref)


@pytest.mark.parametrize("M", [1, 2, 3, 5, 8, 15, 16, 17, 31, 32, 33, 48, 63, 64, 65, 100, 127, 128, 129, 200, 300])
def test_linear_token_counts(M):
    run_linear_case(M, 384, 320, seed=M)


@pytest.mark.parametrize("N,K", [(128, 64), (128, 128), (256, 448), (512, 1024), (1024, 3072)])
@pytest.mark.parametrize("M", [1, 24, 64, 130])
def test_linear_shapes(M, N, K):
    run_linear_case(M, N, K, seed=N + K + M)


@pytest.mark.parametrize("M,N,K", [(65, 256, 64), (129, 512, 320), (255, 256, 128), (256, 512, 192),
                                   (257, 768, 320), (511, 256, 576), (513, 512, 64), (777, 1280, 448),
                                   (2048, 2560, 192)])
def test_linear_pair_tiles(M, N, K):
    """Large M with N % 256 == 0 runs on CTA pairs (256 x 256 tiles): ragged
    token tails, single-stage and many-stage K, more tiles than SM pairs."""
    run_linear_case(M, N, K, seed=M + N + K)


@pytest.mark.parametrize("M,N,K", [(17, 256, 64), (24, 768, 192), (31, 512, 3072), (32, 256, 448),
                                   (33, 1280, 320), (48, 256, 128), (64, 2560, 576), (40, 512, 256),
                                   (56, 256, 1280)])
def test_linear_pair_tiles_narrow(M, N, K):
    """16 < M <= 64 with N % 256 == 0 runs the 64-token tcgen05 tiles (one
    CTA per 128 channels, double-buffered accumulators, eight decoder warps,
    256-k stages): K covers every tail of a stage (64, 128 and 192 k left)
    and whole stages."""
    run_linear_case(M, N, K, seed=3 * M + N + K)


def test_linear_pair_tiles_many_token_tiles():
    """Token rows far past 2^16 with a single 256-wide channel slab: 128 token
    tiles queued on fewer CTA pairs, each pair looping over several."""
    run_linear_case(32768, 256, 128, seed=91)
    run_linear_case(20001, 512, 64, seed=92)


def test_linear_no_bias():
    run_linear_case(40, 256, 256, seed=3, with_bias=False)
    run_linear_case(257, 256, 256, seed=4, with_bias=False)


def test_linear_tiny_config():
    L = workloads.CONFIGS["tiny"]
    x, W, b = workloads.make_inputs(L)
    packed, scales = quantize_on_gpu(W)
    T, s = check_quantize(W, packed, scales, {})
    y = tern.linear(x.cuda(), packed, scales, b.cuda())
    y_ref = oracle.linear(bits(x), T, s, bits(b))
    check_y(y, y_ref)
    # end to end against the oracle's own quantisation
    T_own, s_own = oracle.quantize(bits(W), EPS)
    check_y(y, oracle.linear(bits(x), T_own, s_own, bits(b)))


def test_linear_deterministic_and_canaries():
    M, N, K = 33, 256, 512
    W = rand_bf16((N, K), 0.02, 11)
    x = rand_bf16((M, K), 1.0, 12).cuda()
    packed, scales = quantize_on_gpu(W)
    buf = torch.full((M * N + 4096,), 7.0, dtype=torch.bfloat16, device="cuda")
    y1 = buf[2048:2048 + M * N].view(M, N)
    tern.linear(x, packed, scales, None, out=y1)
    y2 = tern.linear(x, packed, scales, None)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2), "two runs differ"
    assert (buf[:2048] == 7.0).all() and (buf[2048 + M * N:] == 7.0).all(), "wrote outside y"


def test_linear_m_zero_is_noop():
    W = rand_bf16((128, 64), 0.02, 1)
    packed, scales = quantize_on_gpu(W)
    x = torch.empty(0, 64, dtype=torch.bfloat16, device="cuda")
    y = tern.linear(x, packed, scales)
    assert y.shape == (0, 128)


def test_linear_rejects_misaligned_pointer():
    W = rand_bf16((128, 64), 0.02, 1)
    packed, scales = quantize_on_gpu(W)
    xbuf = torch.zeros(4 * 64 + 8, dtype=torch.bfloat16, device="cuda")
    x = xbuf[1:1 + 4 * 64].view(4, 64)  # 2-byte offset
    with pytest.raises(tern.TernError) as e:
        tern.linear(x, packed, scales)
    assert e.value.status == -3


# ---------------------------------------------------------------- batch
def test_linear_batch_mixed_sizes():
    # one or more problems of each launch group: GEMV M <= 8 and M <= 16,
    # 64-token and 256-token CTA-pair tiles, and the single-CTA kernel for
    # N % 256 != 0
    cases = [(1, 256, 192), (16, 384, 256), (70, 128, 128), (300, 256, 320), (2, 512, 64), (130, 128, 576),
             (40, 512, 256), (9, 256, 128), (64, 256, 3072), (600, 512, 192), (257, 768, 320),
             (33, 384, 448)]
    probs, refs = [], []
    for i, (M, N, K) in enumerate(cases):
        W = rand_bf16((N, K), 0.02, 100 + i)
        x = rand_bf16((M, K), 1.0, 200 + i)
        b = rand_bf16((N,), 0.01, 300 + i) if i % 2 == 0 else None
        packed, scales = quantize_on_gpu(W)
        T, s = check_quantize(W, packed, scales, {})
        y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        probs.append(dict(x=x.cuda(), packed=packed, scales=scales, bias=None if b is None else b.cuda(), y=y))
        refs.append(oracle.linear(bits(x), T, s, None if b is None else bits(b)))
    tern.linear_batch(probs)
    torch.cuda.synchronize()
    assert tern.device_status() == 0
    for p, r in zip(probs, refs):
        check_y(p["y"], r)
    tern.linear_batch([])


def test_linear_batch_rejects_bad_problem_before_launch():
    W = rand_bf16((128, 64), 0.02, 1)
    packed, scales = quantize_on_gpu(W)
    x = rand_bf16((4, 64), 1.0, 2).cuda()
    y = torch.full((4, 128), 3.0, dtype=torch.bfloat16, device="cuda")
    bad_y = torch.empty(4, 128, dtype=torch.bfloat16, device="cuda")
    probs = [dict(x=x, packed=packed, scales=scales, bias=None, y=y),
             dict(x=x, packed=packed, scales=scales, bias=None, y=bad_y)]
    probs[1]["y"] = x  # aliasing input and output
    with pytest.raises(tern.TernError):
        tern.linear_batch(probs)
    torch.cuda.synchronize()
    assert (y == 3.0).all(), "nothing may run when one problem is invalid"


# ------------------------------------------------------------- full sizes
@pytest.mark.parametrize("name", ["qkv", "mlp_up", "mlp_down"])
def test_linear_flux_layers_full(name):
    """Full-size layers in the launch configuration the benchmark times; the
    oracle checks every token row against every output channel."""
    L = workloads.CONFIGS[name]
    x, W, b = workloads.make_inputs(L)
    packed, scales = quantize_on_gpu(W)
    T, s = check_quantize(W, packed, scales, {})
    y = tern.linear(x.cuda(), packed, scales, b.cuda())
    torch.cuda.synchronize()
    assert tern.device_status() == 0
    check_y(y, oracle.linear(bits(x), T, s, bits(b)))


@pytest.mark.parametrize("M", [1, 4, 16, 64])
@pytest.mark.parametrize("mult", [6, 3])
def test_linear_modulation_gemv_full(M, mult):
    """adaLN modulation GEMV sweep, every output against the oracle."""
    L = workloads.CONFIGS[f"mod{mult}_m{M}"]
    x, W, b = workloads.make_inputs(L)
    packed, scales = quantize_on_gpu(W)
    T, s = check_quantize(W, packed, scales, {})
    y = tern.linear(x.cuda(), packed, scales, b.cuda())
    torch.cuda.synchronize()
    assert tern.device_status() == 0
    check_y(y, oracle.linear(bits(x), T, s, bits(b)))


def test_dequantize_matches_codes_times_scales():
    N, K = 256, 192
    W = rand_bf16((N, K), 0.02, 77)
    packed, scales = quantize_on_gpu(W)
    Wd = tern.dequantize(packed, scales, K)
    T, _ = oracle.unpack_tiled(packed.cpu().numpy(), N, K)
    ref = (torch.from_numpy(T.astype(np.float32)) * scales.cpu()[:, None]).to(torch.bfloat16)
    assert torch.equal(Wd.cpu(), ref)


# ---------------------------------------------------------- failure detection
def test_device_wait_timeout_is_reported_and_context_survives():
    assert tern.device_status() == 0
    tern.selftest_wait_timeout(5_000_000)  # 5 ms wait that nothing satisfies
    assert tern.device_status() == -5
    assert tern.device_status() == 0  # cleared by the read
    run_linear_case(8, 128, 64, seed=5)  # the context is still usable


# ------------------------------------------------ fused activation epilogue
@pytest.mark.parametrize("M,N,K,col0", [
    (1, 384, 256, 0),        # GEMV, 8-token blocks
    (12, 256, 320, 128),     # GEMV, two 8-token blocks, activation on the upper half
    (40, 512, 256, 0),       # 64-token tcgen05 tiles
    (300, 512, 192, 256),    # CTA-pair tiles, activation on the second pair tile
    (300, 512, 192, 100),    # CTA-pair tiles, activation from inside a warp's channels
    (1024, 1024, 512, 0),    # several pair tiles per CTA pair
    (70, 384, 128, 0),       # single-CTA fallback (N % 256 != 0)
    (40, 384, 1024, 129),    # fallback with split K (partials summed by the last CTA)
])
def test_linear_act_gelu(M, N, K, col0):
    W = rand_bf16((N, K), 0.02, M + N)
    x = rand_bf16((M, K), 1.0, M + K)
    b = rand_bf16((N,), 0.01, N + K)
    packed, scales = quantize_on_gpu(W)
    T, s = check_quantize(W, packed, scales, {})
    y = tern.linear_act(x.cuda(), packed, scales, b.cuda(), tern.ACT_GELU_TANH, col0)
    torch.cuda.synchronize()
    assert tern.device_status() == 0
    y_ref = oracle.linear_act(bits(x), T, s, bits(b), oracle.ACT_GELU_TANH, col0)
    check_y(y, y_ref)
    # the columns below col0 are the plain layer, bit for bit
    y_plain = tern.linear(x.cuda(), packed, scales, b.cuda())
    torch.cuda.synchronize()
    assert torch.equal(y[:, :col0], y_plain[:, :col0])


def test_linear_act_none_is_linear():
    W = rand_bf16((512, 256), 0.02, 5)
    x = rand_bf16((300, 256), 1.0, 6).cuda()
    packed, scales = quantize_on_gpu(W)
    assert torch.equal(tern.linear_act(x, packed, scales, None, tern.ACT_NONE, 0),
                       tern.linear(x, packed, scales, None))


def test_linear_act_gelu_flux_mlp_up_full():
    """The MLP up projection of the FLUX stack with its GELU fused, at full size
    (4608 tokens), in the launch configuration of the layer; every output."""
    L = workloads.CONFIGS["mlp_up"]
    x, W, b = workloads.make_inputs(L)
    packed, scales = quantize_on_gpu(W)
    T, s = check_quantize(W, packed, scales, {})
    y = tern.linear_act(x.cuda(), packed, scales, b.cuda(), tern.ACT_GELU_TANH, 0)
    torch.cuda.synchronize()
    assert tern.device_status() == 0
    check_y(y, oracle.linear_act(bits(x), T, s, bits(b), oracle.ACT_GELU_TANH, 0))


def test_linear_batch_act_mixed():
    cases = [(1, 256, 192, tern.ACT_GELU_TANH, 0), (9, 384, 256, tern.ACT_NONE, 0),
             (40, 512, 256, tern.ACT_GELU_TANH, 256), (300, 256, 320, tern.ACT_GELU_TANH, 0),
             (70, 128, 128, tern.ACT_GELU_TANH, 64), (600, 512, 192, tern.ACT_NONE, 0)]
    probs, refs = [], []
    for i, (M, N, K, act, col0) in enumerate(cases):
        W = rand_bf16((N, K), 0.02, 400 + i)
        x = rand_bf16((M, K), 1.0, 500 + i)
        b = rand_bf16((N,), 0.01, 600 + i)
        packed, scales = quantize_on_gpu(W)
        T, s = check_quantize(W, packed, scales, {})
        y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        probs.append(dict(x=x.cuda(), packed=packed, scales=scales, bias=b.cuda(), y=y, act=act, act_col0=col0))
        refs.append(oracle.linear_act(bits(x), T, s, bits(b), act, col0))
    tern.linear_batch_act(probs)
    torch.cuda.synchronize()
    assert tern.device_status() == 0
    for p, r in zip(probs, refs):
        check_y(p["y"], r)


# --------------------------------------- fused gated residual (adaLN-Zero) epilogue
@pytest.mark.parametrize("M,N,K,act,col0,inplace", [
    (1, 384, 256, 0, 0, True),        # GEMV, in-place residual stream update
    (12, 256, 320, 1, 128, False),    # GEMV, GELU on half the channels + residual
    (40, 512, 256, 0, 0, True),       # 64-token tiles
    (300, 512, 192, 0, 0, True),      # CTA-pair tiles, in place
    (300, 512, 192, 1, 100, False),   # CTA-pair tiles, GELU + residual + gate
    (70, 384, 128, 0, 0, True),       # fallback
    (40, 384, 1024, 1, 0, False),     # fallback with split K
])
def test_linear_epilogue_gated_residual(M, N, K, act, col0, inplace):
    W = rand_bf16((N, K), 0.02, M + 3 * N)
    x = rand_bf16((M, K), 1.0, M + 5 * K)
    b = rand_bf16((N,), 0.01, N + 7)
    r = rand_bf16((M, N), 1.0, M * N + 1)
    g = rand_bf16((N,), 0.5, N + 11)
    packed, scales = quantize_on_gpu(W)
    T, s = check_quantize(W, packed, scales, {})
    rd = r.cuda()
    out = rd if inplace else torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    y = tern.linear_epilogue(x.cuda(), packed, scales, b.cuda(), act, col0, residual=rd, gate=g.cuda(), out=out)
    torch.cuda.synchronize()
    assert tern.device_status() == 0
    if inplace:
        assert y.data_ptr() == rd.data_ptr()
    y_ref = oracle.linear_epilogue(bits(x), T, s, bits(b), act, col0, bits(r), bits(g))
    check_y(y, y_ref)


def test_linear_batch_epilogue_mixed():
    """A batch holding every kernel class with different epilogues, some in place."""
    cases = [(1, 256, 192, dict(act=1)), (9, 384, 256, dict(res=True, gate=True, inplace=True)),
             (40, 512, 256, dict(res=True)), (300, 256, 320, dict(gate=True)),
             (70, 128, 128, dict(act=1, act_col0=64, res=True, gate=True)), (600, 512, 192, dict())]
    probs, refs = [], []
    for i, (M, N, K, e) in enumerate(cases):
        W = rand_bf16((N, K), 0.02, 700 + i)
        x = rand_bf16((M, K), 1.0, 800 + i)
        b = rand_bf16((N,), 0.01, 900 + i)
        r = rand_bf16((M, N), 1.0, 1000 + i) if e.get("res") else None
        g = rand_bf16((N,), 0.5, 1100 + i) if e.get("gate") else None
        packed, scales = quantize_on_gpu(W)
        T, s = check_quantize(W, packed, scales, {})
        rd = None if r is None else r.cuda()
        y = rd if e.get("inplace") else torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        probs.append(dict(x=x.cuda(), packed=packed, scales=scales, bias=b.cuda(), y=y, act=e.get("act", 0),
                          act_col0=e.get("act_col0", 0), residual=rd, gate=None if g is None else g.cuda()))
        refs.append(oracle.linear_epilogue(bits(x), T, s, bits(b), e.get("act", 0), e.get("act_col0", 0),
                                           None if r is None else bits(r), None if g is None else bits(g)))
    tern.linear_batch_epilogue(probs)
    torch.cuda.synchronize()
    assert tern.device_status() == 0
    for p, ref in zip(probs, refs):
        check_y(p["y"], ref)


# ------------------------------------------------ RMS normalisation of 128-channel groups
@pytest.mark.parametrize("M,N,K,cols,act,res", [
    (300, 512, 192, (0, 256), 0, False),      # CTA-pair tiles: the first pair tile normalised
    (300, 512, 192, (128, 384), 1, True),     # one CTA of each pair tile, with GELU and residual
    (1024, 1024, 512, (0, 768), 0, False),    # several tiles per CTA pair (barrier phases)
    (40, 512, 256, (128, 384), 0, False),     # 64-token tiles
    (64, 768, 320, (0, 768), 0, True),        # 64-token tiles, all normalised, residual in place
])
def test_linear_epilogue_rms_norm(M, N, K, cols, act, res):
    W = rand_bf16((N, K), 0.02, M + 13 * N)
    x = rand_bf16((M, K), 1.0, M + 17 * K)
    b = rand_bf16((N,), 0.01, N + 19)
    w = (torch.rand(N, generator=torch.Generator().manual_seed(N)) + 0.5).to(torch.bfloat16)
    r = rand_bf16((M, N), 1.0, M * N + 3) if res else None
    packed, scales = quantize_on_gpu(W)
    T, s = check_quantize(W, packed, scales, {})
    rd = None if r is None else r.cuda()
    out = rd if res else torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    y = tern.linear_epilogue(x.cuda(), packed, scales, b.cuda(), act, 0, residual=rd, norm_cols=cols,
                             norm_weight=w.cuda(), norm_eps=1e-6, out=out)
    torch.cuda.synchronize()
    assert tern.device_status() == 0
    y_ref = oracle.linear_epilogue(bits(x), T, s, bits(b), act, 0, None if r is None else bits(r), None, cols,
                                   bits(w), 1e-6)
    check_y(y, y_ref)


def test_linear_epilogue_rms_norm_flux_qkv_full():
    """The FLUX QKV projection with q and k normalised per 128-channel head
    (columns [0, 6144)), full size, every output."""
    L = workloads.CONFIGS["qkv"]
    x, W, b = workloads.make_inputs(L)
    packed, scales = quantize_on_gpu(W)
    T, s = check_quantize(W, packed, scales, {})
    w = (torch.rand(L.N, generator=torch.Generator().manual_seed(2)) + 0.5).to(torch.bfloat16)
    y = tern.linear_epilogue(x.cuda(), packed, scales, b.cuda(), norm_cols=(0, 2 * workloads.HIDDEN),
                             norm_weight=w.cuda(), norm_eps=1e-6)
    torch.cuda.synchronize()
    assert tern.device_status() == 0
    ref = oracle.linear_epilogue(bits(x), T, s, bits(b), 0, 0, None, None, (0, 2 * workloads.HIDDEN),
                                 bits(w), 1e-6)
    check_y(y, ref)


def check_y_rotated(y_gpu: torch.Tensor, y_ref: np.ndarray, cols):
    """check_y, with the bar on the rotated columns [cols) taken over both
    channels of each pair: the rotation mixes a channel with its partner,
    each carrying the bf16 rounding of the value before the normalisation
    (2^-9 relative), so the error scales with |a| + |b| of the pair, not
    with the rotated output alone."""
    y = y_gpu.detach().cpu().double().numpy()
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    mag = np.abs(y_ref).copy()
    c0, c1 = cols
    pair = np.abs(y_ref[:, c0:c1]).reshape(y_ref.shape[0], -1, 2).sum(axis=2)
    mag[:, c0:c1] = np.repeat(pair, 2, axis=1)
    err = np.abs(y - y_ref)
    bad = err > Y_RTOL * mag + Y_RMS * rms
    assert not bad.any(), (f"{int(bad.sum())} of {bad.size} outputs out of tolerance; "
                           f"worst err {err.max():.3e} at {np.unravel_index(err.argmax(), err.shape)}")


def rope_table(M, seed):
    """fp32 (cos, sin) pairs [M, 64, 2] of seeded angles in [-60, 60)."""
    a = torch.rand(M, 64, generator=torch.Generator().manual_seed(seed), dtype=torch.float64) * 120 - 60
    return torch.stack([torch.cos(a), torch.sin(a)], dim=-1).float()


@pytest.mark.parametrize("M,N,K,cols", [
    (300, 512, 192, (0, 512)),      # CTA-pair tiles, every column normalised and rotated
    (1024, 768, 320, (0, 512)),     # several tiles per pair, v-like columns untouched
    (40, 512, 256, (128, 384)),     # 64-token tiles
    (17, 256, 128, (0, 256)),       # 64-token tile, one token past the GEMV range
])
def test_linear_epilogue_rms_norm_rope(M, N, K, cols):
    """q/k norm followed by the rotary embedding of the normalised columns'
    channel pairs, one rounding; ragged token tails read no table row past M.
    The value before the normalisation is rounded to bf16 (the norm's
    two-rounding path), and the rotation mixes it with its partner channel:
    the bar covers both channels' magnitudes (check_y_rotated)."""
    W = rand_bf16((N, K), 0.02, M + 29 * N)
    x = rand_bf16((M, K), 1.0, M + 31 * K)
    b = rand_bf16((N,), 0.01, N + 37)
    w = (torch.rand(N, generator=torch.Generator().manual_seed(N + 1)) + 0.5).to(torch.bfloat16)
    cs = rope_table(M, M + N)
    packed, scales = quantize_on_gpu(W)
    T, s = check_quantize(W, packed, scales, {})
    y = tern.linear_epilogue(x.cuda(), packed, scales, b.cuda(), norm_cols=cols, norm_weight=w.cuda(),
                             norm_eps=1e-6, rope_cs=cs.cuda())
    torch.cuda.synchronize()
    assert tern.device_status() == 0
    ref = oracle.linear_epilogue(bits(x), T, s, bits(b), 0, 0, None, None, cols, bits(w), 1e-6,
                                 rope_cs=cs.double().numpy())
    check_y_rotated(y, ref, cols)


def test_linear_batch_epilogue_rope_row_offsets():
    """Two problems writing the halves of one buffer, each with its own rows
    of one rotary table (the caller offsets the table pointer)."""
    M1, M2, N, K = 96, 200, 512, 256
    cs = rope_table(M1 + M2, 7)
    buf = torch.empty(M1 + M2, N, dtype=torch.bfloat16, device="cuda")
    probs, refs = [], []
    for i, (r0, r1) in enumerate([(0, M1), (M1, M1 + M2)]):
        W = rand_bf16((N, K), 0.02, 1500 + i)
        x = rand_bf16((r1 - r0, K), 1.0, 1600 + i)
        b = rand_bf16((N,), 0.01, 1700 + i)
        packed, scales = quantize_on_gpu(W)
        T, s = check_quantize(W, packed, scales, {})
        probs.append(dict(x=x.cuda(), packed=packed, scales=scales, bias=b.cuda(), y=buf[r0:r1], norm_col0=0,
                          norm_col1=256, norm_eps=1e-6, rope_cs=cs[r0:r1].cuda()))
        refs.append(oracle.linear_epilogue(bits(x), T, s, bits(b), 0, 0, None, None, (0, 256), None, 1e-6,
                                           rope_cs=cs[r0:r1].double().numpy()))
    tern.linear_batch_epilogue(probs)
    torch.cuda.synchronize()
    assert tern.device_status() == 0
    for p, ref in zip(probs, refs):
        check_y_rotated(p["y"], ref, (0, 256))


def test_linear_batch_epilogue_with_norm():
    """A batch where one pair-tile problem normalises and the others do not:
    the whole launch runs the normalising kernel."""
    cases = [(300, 512, 192, (0, 256)), (600, 256, 320, (0, 0)), (40, 256, 256, (0, 256))]
    probs, refs = [], []
    for i, (M, N, K, cols) in enumerate(cases):
        W = rand_bf16((N, K), 0.02, 1200 + i)
        x = rand_bf16((M, K), 1.0, 1300 + i)
        b = rand_bf16((N,), 0.01, 1400 + i)
        packed, scales = quantize_on_gpu(W)
        T, s = check_quantize(W, packed, scales, {})
        y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        probs.append(dict(x=x.cuda(), packed=packed, scales=scales, bias=b.cuda(), y=y, norm_col0=cols[0],
                          norm_col1=cols[1], norm_eps=1e-6))
        refs.append(oracle.linear_epilogue(bits(x), T, s, bits(b), 0, 0, None, None, cols, None, 1e-6))
    tern.linear_batch_epilogue(probs)
    torch.cuda.synchronize()
    assert tern.device_status() == 0
    for p, ref in zip(probs, refs):
        check_y(p["y"], ref)
