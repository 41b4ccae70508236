"""Seeded synthetic inputs shaped like the linear layers of FLUX.1-dev at 1024x1024.

This module only draws random numbers and lists shapes; it holds none of the
ternary method's arithmetic, so the CUDA path and the CPU oracle can both be
fed from it without sharing any of the computation.

Shapes follow page "1.58-bit FLUX" (arXiv 2412.18653), Section 3.1: every
linear layer of the double-stream (FluxTransformerBlock) and single-stream
(FluxSingleTransformerBlock) blocks is ternary.  One 1024x1024 image gives
4096 image tokens; the text stream has 512 tokens, hidden size 3072, MLP
width 12288.  Distributions: x ~ N(0, 1) (N(0, 0.5) into the MLP down
projection), W ~ N(0, 0.02), bias ~ N(0, 0.01); every tensor is drawn in
fp32 from a seeded CPU generator and rounded to bf16.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import torch

HIDDEN = 3072
MLP = 12288
IMG_TOKENS = 4096
TXT_TOKENS = 512
N_DOUBLE = 19
N_SINGLE = 38
W_STD = 0.02
B_STD = 0.01
EPS = 1e-5


@dataclasses.dataclass(frozen=True)
class Layer:
    name: str
    M: int
    K: int
    N: int
    seed: int
    x_std: float = 1.0
    w_std: float = W_STD
    b_std: float = B_STD

    @property
    def flop(self) -> float:
        return 2.0 * self.M * self.N * self.K

    @property
    def packed_bytes(self) -> int:
        return self.N * self.K // 4

    @property
    def algorithmic_bytes(self) -> int:
        """codes + fp32 scales + bf16 bias + bf16 x + bf16 y."""
        return self.N * self.K // 4 + 4 * self.N + 2 * self.N + 2 * self.M * self.K + 2 * self.M * self.N


# The single-layer workloads.  "mod_*" is the adaLN modulation GEMV sweep.
CONFIGS = {
    "tiny": Layer("tiny", M=16, K=256, N=256, seed=0),
    "qkv": Layer("qkv", M=IMG_TOKENS, K=HIDDEN, N=3 * HIDDEN, seed=1),
    "mlp_up": Layer("mlp_up", M=IMG_TOKENS + TXT_TOKENS, K=HIDDEN, N=MLP, seed=2),
    "mlp_down": Layer("mlp_down", M=IMG_TOKENS + TXT_TOKENS, K=MLP, N=HIDDEN, seed=3, x_std=0.5),
}
for _m in (1, 4, 16, 64):
    CONFIGS[f"mod6_m{_m}"] = Layer(f"mod6_m{_m}", M=_m, K=HIDDEN, N=6 * HIDDEN, seed=4)
    CONFIGS[f"mod3_m{_m}"] = Layer(f"mod3_m{_m}", M=_m, K=HIDDEN, N=3 * HIDDEN, seed=4)


def flux_stack() -> List[Layer]:
    """Every ternary linear of one FLUX.1-dev transformer forward (one image)."""
    layers: List[Layer] = []
    idx = 0

    def add(name, M, K, N, x_std=1.0):
        nonlocal idx
        layers.append(Layer(name, M=M, K=K, N=N, seed=1000 + idx, x_std=x_std))
        idx += 1

    for b in range(N_DOUBLE):
        for stream, M in (("img", IMG_TOKENS), ("txt", TXT_TOKENS)):
            add(f"double{b}.{stream}.mod", 1, HIDDEN, 6 * HIDDEN)
            add(f"double{b}.{stream}.qkv", M, HIDDEN, 3 * HIDDEN)
            add(f"double{b}.{stream}.proj", M, HIDDEN, HIDDEN)
            add(f"double{b}.{stream}.mlp_up", M, HIDDEN, MLP)
            add(f"double{b}.{stream}.mlp_down", M, MLP, HIDDEN, x_std=0.5)
    for b in range(N_SINGLE):
        M = IMG_TOKENS + TXT_TOKENS
        add(f"single{b}.mod", 1, HIDDEN, 3 * HIDDEN)
        add(f"single{b}.qkv_mlp", M, HIDDEN, 3 * HIDDEN + MLP)
        add(f"single{b}.proj_out", M, HIDDEN + MLP, HIDDEN, x_std=0.5)
    return layers


def _normal(shape, std: float, gen: torch.Generator) -> torch.Tensor:
    return (torch.randn(shape, generator=gen, dtype=torch.float32) * std).to(torch.bfloat16)


def make_inputs(layer: Layer, M: Optional[int] = None):
    """Returns CPU bf16 tensors (x [M,K], W [N,K], b [N]) for a layer.

    W and b depend only on the seed; x is drawn after them so a smaller M
    gives the leading rows of the same stream only when the caller passes
    the same M.
    """
    gen = torch.Generator().manual_seed(layer.seed)
    W = _normal((layer.N, layer.K), layer.w_std, gen)
    b = _normal((layer.N,), layer.b_std, gen)
    x = _normal((layer.M if M is None else M, layer.K), layer.x_std, gen)
    return x, W, b


def bf16_bits(t: torch.Tensor):
    """Raw uint16 bit patterns of a CPU bf16 tensor, as a numpy array."""
    import numpy as np

    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def block_layers(block: str) -> List[Layer]:
    """The layers of one block of ``flux_stack()``, e.g. "double0" or "single7"."""
    return [L for L in flux_stack() if L.name.split(".")[0] == block]


def block_epilogue(name: str, qk_norm: bool = False) -> dict:
    """How one FLUX.1 block uses the output of its linear ``name``.

    The pages quantise every linear of both block types (Section 3.1) and
    describe nothing between them; this lists what FLUX.1's blocks do there,
    as plain data (no arithmetic):
      * act "gelu_tanh" from column act_col0: the MLP's first linear (all of
        its columns), or the MLP part of a single block's fused projection
        (after q, k and v: from column 3 * HIDDEN);
      * gated_residual: the attention and MLP output projections update the
        residual stream in place, scaled per channel by an adaLN-Zero gate;
      * norm_cols (only with qk_norm): per-head RMS normalisation of q and k,
        the first 2 * HIDDEN columns of a QKV projection.
    """
    e: dict = {}
    if name.endswith(".mlp_up"):
        e["act"], e["act_col0"] = "gelu_tanh", 0
    elif name.endswith(".qkv_mlp"):
        e["act"], e["act_col0"] = "gelu_tanh", 3 * HIDDEN
    elif name.endswith((".proj", ".mlp_down", ".proj_out")):
        e["gated_residual"] = True
    if qk_norm and name.endswith((".qkv", ".qkv_mlp")):
        e["norm_cols"] = (0, 2 * HIDDEN)
    return e


# --------------------------------------------------------------------- blocks
HEAD_DIM = 128
ROPE_AXES = (16, 56, 56)
NORM_W_STD = 0.1


@dataclasses.dataclass(frozen=True)
class FluxConfig:
    """A FLUX.1-shaped transformer: hidden width, MLP width, heads of 128,
    an image token grid (64 x 64 for a 1024 x 1024 image: 2 x 2 patches of
    its 128 x 128 latent), text tokens, and the block counts."""
    hidden: int = HIDDEN
    mlp: int = MLP
    img_h: int = 64
    img_w: int = 64
    txt_tokens: int = TXT_TOKENS
    n_double: int = N_DOUBLE
    n_single: int = N_SINGLE
    in_channels: int = 64
    context_dim: int = 4096
    seed: int = 77

    @property
    def img_tokens(self) -> int:
        return self.img_h * self.img_w

    @property
    def heads(self) -> int:
        return self.hidden // HEAD_DIM


FLUX_SMALL = FluxConfig(hidden=256, mlp=1024, img_h=8, img_w=8, txt_tokens=24, n_double=1, n_single=1,
                        in_channels=64, context_dim=256)


def flux_block_shapes(cfg: FluxConfig, kind: str):
    """(name, N, K) of every ternary linear of one block, "double" or "single"."""
    C, F = cfg.hidden, cfg.mlp
    if kind == "double":
        out = []
        for s in ("img", "txt"):
            out += [(f"{s}.mod", 6 * C, C), (f"{s}.qkv", 3 * C, C), (f"{s}.proj", C, C),
                    (f"{s}.mlp_up", F, C), (f"{s}.mlp_down", C, F)]
        return out
    return [("mod", 3 * C, C), ("linear1", 3 * C + F, C), ("linear2", C, C + F)]


def flux_block_weights(cfg: FluxConfig, kind: str, index: int, device=None):
    """Seeded bf16 parameters of one block: for every ternary linear
    (W [N, K] ~ N(0, 0.02), b [N] ~ N(0, 0.01)), and the q/k RMS norm weights
    ([128] ~ 1 + N(0, 0.1); per stream in a double block).  Drawn on
    `device` (CPU by default) from a generator seeded by the block."""
    dev = torch.device("cpu") if device is None else torch.device(device)
    gen = torch.Generator(device=dev).manual_seed(cfg.seed * 1000003 + (0 if kind == "double" else 500) + index)

    def normal(shape, std, mean=0.0):
        return (torch.randn(shape, generator=gen, device=dev) * std + mean).to(torch.bfloat16)

    p = {}
    for name, N, K in flux_block_shapes(cfg, kind):
        p[name] = (normal((N, K), W_STD), normal((N,), B_STD))
    for s in (("img.", "txt.") if kind == "double" else ("",)):
        p[s + "q_norm"] = normal((HEAD_DIM,), NORM_W_STD, 1.0)
        p[s + "k_norm"] = normal((HEAD_DIM,), NORM_W_STD, 1.0)
    return p


def flux_inputs(cfg: FluxConfig, seed: int = 5):
    """Seeded CPU inputs of the block stack: img [Li, C], txt [Lt, C], vec
    [1, C] (bf16, N(0, 1)) and the token positions ids [Lt + Li, 3] (text
    tokens at 0, image token (0, row, column)), text first."""
    gen = torch.Generator().manual_seed(seed)
    C = cfg.hidden
    img = _normal((cfg.img_tokens, C), 1.0, gen)
    txt = _normal((cfg.txt_tokens, C), 1.0, gen)
    vec = _normal((1, C), 1.0, gen)
    ids = torch.zeros(cfg.txt_tokens + cfg.img_tokens, 3)
    r = torch.arange(cfg.img_h).repeat_interleave(cfg.img_w)
    c = torch.arange(cfg.img_w).repeat(cfg.img_h)
    ids[cfg.txt_tokens:, 1] = r.float()
    ids[cfg.txt_tokens:, 2] = c.float()
    return img, txt, vec, ids


def flux_io_weights(cfg: FluxConfig, device=None):
    """Seeded bf16 parameters of the unquantised input and output layers of a
    FLUX.1-shaped transformer (the 0.5 % of parameters the pages leave in
    16 bits): image and text input projections, the time, guidance and
    pooled-text embedders (Linear -> SiLU -> Linear), the final adaLN
    modulation and output projection; each (W [N, K] ~ N(0, 0.02),
    b [N] ~ N(0, 0.01))."""
    dev = torch.device("cpu") if device is None else torch.device(device)
    gen = torch.Generator(device=dev).manual_seed(cfg.seed * 1000003 + 999)
    C = cfg.hidden

    def lin(N, K):
        W = (torch.randn((N, K), generator=gen, device=dev) * W_STD).to(torch.bfloat16)
        b = (torch.randn((N,), generator=gen, device=dev) * B_STD).to(torch.bfloat16)
        return W, b

    return {"img_in": lin(C, cfg.in_channels), "txt_in": lin(C, cfg.context_dim),
            "time_in.0": lin(C, 256), "time_in.1": lin(C, C), "guidance_in.0": lin(C, 256),
            "guidance_in.1": lin(C, C), "vector_in.0": lin(C, 768), "vector_in.1": lin(C, C),
            "final.mod": lin(2 * C, C), "final.out": lin(cfg.in_channels, C)}


def flux_model_inputs(cfg: FluxConfig, seed: int = 6):
    """Seeded CPU inputs of the whole transformer: packed image latents
    [Li, in_channels] and text encoder states [Lt, context_dim] (bf16,
    N(0, 1)), pooled text vector [1, 768], the timestep and guidance value
    (scalars in [0, 1) and [1, 5)), and the token positions as flux_inputs."""
    gen = torch.Generator().manual_seed(seed)
    img = _normal((cfg.img_tokens, cfg.in_channels), 1.0, gen)
    txt = _normal((cfg.txt_tokens, cfg.context_dim), 1.0, gen)
    pooled = _normal((1, 768), 1.0, gen)
    t = float(torch.rand(1, generator=gen))
    guidance = 1.0 + 4.0 * float(torch.rand(1, generator=gen))
    ids = flux_inputs(cfg)[3]
    return img, txt, pooled, t, guidance, ids
