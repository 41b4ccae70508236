"""FLUX.1's transformer blocks on the ternary linear layer: every linear of
both block types runs through the C ABI (batched, with the fused epilogues:
q/k norm and rotary embedding, GELU, gated residual); attention and SiLU are
torch operations around it.

Page "1.58-bit FLUX" (arXiv 2412.18653): Section 3.1 quantises every linear
layer of FLUX.1's double-stream and single-stream blocks, and Table 3
compares whole-model latency and memory against the bf16 model.  The pages
describe nothing between the linears; the block structure here is FLUX.1's
(adaLN-Zero modulation, q/k RMS norm per head, rotary embedding over
(text, row, column) positions, attention over text and image tokens
together, tanh GELU MLP, gated residual updates).

Per double block: the two streams' QKV projections write into one
[Lt + Li, 3C] buffer (text rows first) with q and k normalised and rotated
in the epilogue, so attention needs no concatenation; the output
projections and the MLP's second linears update the residual streams in
place through the gated-residual epilogue.  Per single block: the fused projection writes
[q | k | v | GELU(mlp)] (norm, rotation and activation in its epilogue); the
attention output overwrites the v columns, so the second linear reads
[attention | mlp] as one strided view of that buffer.  The adaLN modulation
vectors of every block depend only on vec: one batch of GEMVs computes them
all before the first block.

``dense_forward`` runs the same blocks with bf16 dense weights (the
dequantised ternary weights) through cuBLAS and torch's unfused operations:
the bf16 model that the pages compare against, for latency context.
"""
from __future__ import annotations

import contextlib
import math
from typing import Dict, Optional

import torch
import torch.nn.functional as F

from . import tern, workloads

HEAD_DIM = workloads.HEAD_DIM
LN_EPS = 1e-6
QK_EPS = 1e-6
ROPE_THETA = 10000.0


def rope_cos_sin(ids: torch.Tensor, axes=workloads.ROPE_AXES, theta: float = ROPE_THETA):
    """fp32 cos and sin [L, HEAD_DIM / 2] of the rotation angles of the token
    positions ids [L, 3]: axis a with d_a channels owns d_a / 2 consecutive
    channel pairs, pair j turning by ids[:, a] * theta^(-2j / d_a)."""
    parts = []
    for a, d in enumerate(axes):
        omega = theta ** (-torch.arange(0, d, 2, dtype=torch.float64, device=ids.device) / d)
        parts.append(ids[:, a:a + 1].double() * omega[None, :])
    ang = torch.cat(parts, dim=1)
    return torch.cos(ang).float(), torch.sin(ang).float()


def apply_rope(x: torch.Tensor, cos: torch.Tensor, sin: torch.Tensor) -> torch.Tensor:
    """x [L, H, D] bf16 (any strides with unit channel stride): channel pairs
    (2i, 2i + 1) turned by the angles of their token, in fp32, rounded to
    bf16; returns [L, H, D] contiguous."""
    xf = x.float().unflatten(-1, (-1, 2))
    a, b = xf[..., 0], xf[..., 1]
    c, s = cos[:, None, :], sin[:, None, :]
    return torch.stack((a * c - b * s, a * s + b * c), dim=-1).flatten(-2).to(torch.bfloat16)


def attention(qkv: torch.Tensor, hidden: int, cos=None, sin=None) -> torch.Tensor:
    """softmax(q k^T / sqrt(D)) v over all tokens of qkv [L, 3C] (q, k
    already normalised; rotated here when cos and sin are given, else
    already rotated); returns [H, L, D] bf16."""
    L = qkv.shape[0]
    H = hidden // HEAD_DIM
    q = qkv[:, :hidden].view(L, H, HEAD_DIM)
    k = qkv[:, hidden:2 * hidden].view(L, H, HEAD_DIM)
    if cos is not None:
        q, k = apply_rope(q, cos, sin), apply_rope(k, cos, sin)
    v = qkv[:, 2 * hidden:3 * hidden].view(L, H, HEAD_DIM)
    o = F.scaled_dot_product_attention(q.transpose(0, 1)[None], k.transpose(0, 1)[None], v.transpose(0, 1)[None])
    return o[0]


def _on(stream):
    """Makes `stream` current (when given), after the work already queued on
    the current stream (the caller's inputs), so that the torch operations
    between the library calls run on the stream those calls are given.  The
    results are then ready on `stream`."""
    if stream is None:
        return contextlib.nullcontext()
    stream.wait_stream(torch.cuda.current_stream(stream.device))
    return torch.cuda.stream(stream)


def _qk_norm_weight(q_norm: torch.Tensor, k_norm: torch.Tensor, hidden: int, N: int) -> torch.Tensor:
    """[N] bf16 epilogue weight: the per-head q and k norm weights over
    columns [0, 2C), 1 elsewhere (unused there)."""
    H = hidden // HEAD_DIM
    w = torch.ones(N, dtype=torch.bfloat16, device=q_norm.device)
    w[:hidden] = q_norm.repeat(H)
    w[hidden:2 * hidden] = k_norm.repeat(H)
    return w


class TernaryFlux:
    """The block stack of a FLUX.1-shaped transformer with ternary linears.

    ``weights`` maps ("double" | "single", index) to the bf16 parameters of
    ``workloads.flux_block_weights``; every linear is quantised with
    ``tern.quantize_pack`` at construction (eps = workloads.EPS) and only the
    codes, scales and biases are kept.  With ``stream`` given, construction
    and every forward run on it, the torch operations included, after the
    work queued before the call on the current stream; results are ready on
    ``stream``."""

    def __init__(self, cfg: workloads.FluxConfig, weights: Optional[Dict] = None, device="cuda", stream=None):
        self.cfg = cfg
        self.device = torch.device(device)
        self.stream = stream
        self.blocks = {}
        with _on(stream):
            self._quantize(weights)

    def _quantize(self, weights):
        cfg, stream = self.cfg, self.stream
        C, Fm = cfg.hidden, cfg.mlp
        for kind, n in (("double", cfg.n_double), ("single", cfg.n_single)):
            for i in range(n):
                p = (weights[(kind, i)] if weights is not None
                     else workloads.flux_block_weights(cfg, kind, i, device=self.device))
                q = {}
                for name, N, K in workloads.flux_block_shapes(cfg, kind):
                    W, b = p[name]
                    packed, scales = tern.quantize_pack(W.to(self.device), workloads.EPS, stream=stream)
                    q[name] = (packed, scales, b.to(self.device))
                for s in (("img.", "txt.") if kind == "double" else ("",)):
                    N = 3 * C if kind == "double" else 3 * C + Fm
                    q[s + "norm_w"] = _qk_norm_weight(p[s + "q_norm"].to(self.device), p[s + "k_norm"].to(self.device),
                                                      C, N)
                self.blocks[(kind, i)] = q

    def _lin(self, q, x, y, **epi):
        packed, scales, b = q
        return dict(x=x, packed=packed, scales=scales, bias=b, y=y, **epi)

    def modulations(self, vec: torch.Tensor):
        """Every block's adaLN modulation row from vec [1, C]: one batch of
        M = 1 GEMVs on SiLU(vec)."""
        y = F.silu(vec)
        probs, outs = [], {}
        for (kind, i), q in self.blocks.items():
            for s in (("img.", "txt.") if kind == "double" else ("",)):
                packed, scales, b = q[s + "mod"]
                out = torch.empty(1, scales.shape[0], dtype=torch.bfloat16, device=self.device)
                outs[(kind, i, s)] = out
                probs.append(dict(x=y, packed=packed, scales=scales, bias=b, y=out))
        for g in range(0, len(probs), 15):
            tern.linear_batch(probs[g:g + 15], stream=self.stream)
        return outs

    def double_block(self, i: int, img: torch.Tensor, txt: torch.Tensor, mods, cs, buf):
        """Updates img [Li, C] and txt [Lt, C] in place; cs [Lt + Li, 64, 2]
        the rotary (cos, sin) of every token row (text first)."""
        C = self.cfg.hidden
        q = self.blocks[("double", i)]
        Lt = txt.shape[0]
        qkv = buf["qkv"]
        probs = []
        for s, x, rows in (("img.", img, slice(Lt, None)), ("txt.", txt, slice(0, Lt))):
            m = mods[("double", i, s)]
            xm = buf[s + "xm"]
            tern.adaln_modulate(x, m[:, C:2 * C], m[:, :C], LN_EPS, out=xm, stream=self.stream)
            probs.append(self._lin(q[s + "qkv"], xm, qkv[rows], norm_col0=0, norm_col1=2 * C,
                                   norm_weight=q[s + "norm_w"], norm_eps=QK_EPS, rope_cs=cs[rows]))
        tern.linear_batch_epilogue(probs, stream=self.stream)
        o = attention(qkv, C)  # [H, L, D]; q and k rotated in the epilogue
        att = buf["att"]
        att.view(att.shape[0], -1, HEAD_DIM).copy_(o.transpose(0, 1))
        probs = []
        for s, x, rows in (("img.", img, slice(Lt, None)), ("txt.", txt, slice(0, Lt))):
            m = mods[("double", i, s)]
            probs.append(self._lin(q[s + "proj"], att[rows], x, residual=x, gate=m[0, 2 * C:3 * C]))
        tern.linear_batch_epilogue(probs, stream=self.stream)
        probs = []
        for s, x in (("img.", img), ("txt.", txt)):
            m = mods[("double", i, s)]
            xm = buf[s + "xm"]
            tern.adaln_modulate(x, m[:, 4 * C:5 * C], m[:, 3 * C:4 * C], LN_EPS, out=xm, stream=self.stream)
            probs.append(self._lin(q[s + "mlp_up"], xm, buf[s + "h"], act=tern.ACT_GELU_TANH, act_col0=0))
        tern.linear_batch_epilogue(probs, stream=self.stream)
        probs = [self._lin(q[s + "mlp_down"], buf[s + "h"], x, residual=x, gate=mods[("double", i, s)][0, 5 * C:])
                 for s, x in (("img.", img), ("txt.", txt))]
        tern.linear_batch_epilogue(probs, stream=self.stream)

    def single_block(self, i: int, x: torch.Tensor, mods, cs, buf):
        """Updates x [Lt + Li, C] in place."""
        C, Fm = self.cfg.hidden, self.cfg.mlp
        q = self.blocks[("single", i)]
        m = mods[("single", i, "")]
        xm, z = buf["xm"], buf["z"]
        tern.adaln_modulate(x, m[:, C:2 * C], m[:, :C], LN_EPS, out=xm, stream=self.stream)
        tern.linear_batch_epilogue([self._lin(q["linear1"], xm, z, act=tern.ACT_GELU_TANH, act_col0=3 * C,
                                              norm_col0=0, norm_col1=2 * C, norm_weight=q["norm_w"],
                                              norm_eps=QK_EPS, rope_cs=cs)], stream=self.stream)
        o = attention(z, C)
        z[:, 2 * C:3 * C].view(z.shape[0], -1, HEAD_DIM).copy_(o.transpose(0, 1))
        packed, scales, b = q["linear2"]
        tern.linear_strided(z[:, 2 * C:], packed, scales, b, x, stream=self.stream, residual=x, gate=m[0, 2 * C:])

    def buffers(self, Li: int, Lt: int):
        C, Fm = self.cfg.hidden, self.cfg.mlp
        e = lambda *shape: torch.empty(*shape, dtype=torch.bfloat16, device=self.device)  # noqa: E731
        return {"qkv": e(Lt + Li, 3 * C), "att": e(Lt + Li, C), "img.xm": e(Li, C), "txt.xm": e(Lt, C),
                "img.h": e(Li, Fm), "txt.h": e(Lt, Fm), "xm": e(Lt + Li, C), "z": e(Lt + Li, 3 * C + Fm)}

    def forward(self, img: torch.Tensor, txt: torch.Tensor, vec: torch.Tensor, ids: torch.Tensor,
                n_double: Optional[int] = None, n_single: Optional[int] = None) -> torch.Tensor:
        """All blocks on img [Li, C], txt [Lt, C], vec [1, C] (bf16 on the
        device), token positions ids [Lt + Li, 3]; returns the stream
        [Lt + Li, C] after the last single block (text rows first).  The
        inputs are not modified."""
        with _on(self.stream):
            return self._forward(img, txt, vec, ids, n_double, n_single)

    def _forward(self, img, txt, vec, ids, n_double, n_single):
        cfg = self.cfg
        nd = cfg.n_double if n_double is None else n_double
        ns = cfg.n_single if n_single is None else n_single
        Li, Lt = img.shape[0], txt.shape[0]
        cos, sin = rope_cos_sin(ids.to(self.device))
        cs = torch.stack([cos, sin], dim=-1).contiguous()  # [L, 64, 2], read by the q/k epilogues
        mods = self.modulations(vec)
        buf = self.buffers(Li, Lt)
        x = torch.empty(Lt + Li, cfg.hidden, dtype=torch.bfloat16, device=self.device)
        x[:Lt].copy_(txt)
        x[Lt:].copy_(img)
        img_s, txt_s = x[Lt:], x[:Lt]  # the streams live in their rows of x
        for i in range(nd):
            self.double_block(i, img_s, txt_s, mods, cs, buf)
        for i in range(ns):
            self.single_block(i, x, mods, cs, buf)
        return x


def timestep_embedding(t: float, device, dim: int = 256, max_period: float = 10000.0,
                       time_factor: float = 1000.0) -> torch.Tensor:
    """FLUX.1's sinusoidal embedding of a scalar (timestep or guidance) as
    [1, dim] bf16: cos and sin of 1000 t * max_period^(-j / (dim / 2))."""
    half = dim // 2
    freqs = torch.exp(-math.log(max_period) * torch.arange(half, dtype=torch.float32, device=device) / half)
    args = time_factor * t * freqs
    return torch.cat([torch.cos(args), torch.sin(args)])[None].to(torch.bfloat16)


def io_layers_in(io: Dict, img_lat, txt_ctx, pooled, t: float, guidance: float):
    """The unquantised input layers (bf16, cuBLAS): image and text
    projections, and vec = time + guidance + pooled-text embedders, each
    Linear -> SiLU -> Linear.  Returns img [Li, C], txt [Lt, C], vec [1, C]."""
    dev = img_lat.device

    def mlp(x, a, b):
        return F.linear(F.silu(F.linear(x, *io[a])), *io[b])

    vec = (mlp(timestep_embedding(t, dev), "time_in.0", "time_in.1")
           + mlp(timestep_embedding(guidance, dev), "guidance_in.0", "guidance_in.1")
           + mlp(pooled, "vector_in.0", "vector_in.1"))
    return F.linear(img_lat, *io["img_in"]), F.linear(txt_ctx, *io["txt_in"]), vec


def model_forward(model: "TernaryFlux", io: Dict, img_lat, txt_ctx, pooled, t: float, guidance: float, ids,
                  n_double=None, n_single=None) -> torch.Tensor:
    """The whole transformer: the bf16 input layers, every block through the
    library, and the final layer (adaLN modulation row from SiLU(vec) in
    bf16, layer norm and modulation of the image tokens by the library's
    adaLN pass, the bf16 output projection).  Returns [Li, in_channels]."""
    with _on(model.stream):
        img, txt, vec = io_layers_in(io, img_lat, txt_ctx, pooled, t, guidance)
        x = model.forward(img, txt, vec, ids, n_double, n_single)
        C = model.cfg.hidden
        mod = F.linear(F.silu(vec), *io["final.mod"])  # [shift | scale]
        h = tern.adaln_modulate(x[txt.shape[0]:], mod[:, C:], mod[:, :C], LN_EPS, stream=model.stream)
        return F.linear(h, *io["final.out"])


def dense_weights(model: TernaryFlux) -> Dict:
    """bf16 dense weights T * s of every ternary linear of `model` (what the
    bf16 model would hold), plus the biases and norm weights."""
    out = {}
    for key, q in model.blocks.items():
        d = {}
        for name, v in q.items():
            if name.endswith("norm_w"):
                d[name] = v
            else:
                packed, scales, b = v
                K = packed.numel() * 4 // scales.shape[0]
                d[name] = (tern.dequantize(packed, scales, K), b)
        out[key] = d
    return out


def dense_forward(model: TernaryFlux, dense: Dict, img, txt, vec, ids, n_double=None, n_single=None):
    """The same blocks in bf16 with dense weights, cuBLAS linears and torch's
    unfused operations (layer norm, modulation, RMS norm, GELU, residual)."""
    cfg = model.cfg
    C, H = cfg.hidden, cfg.heads
    nd = cfg.n_double if n_double is None else n_double
    ns = cfg.n_single if n_single is None else n_single
    Li, Lt = img.shape[0], txt.shape[0]
    cos, sin = rope_cos_sin(ids.to(img.device))
    y = F.silu(vec)

    def lin(w, x):
        return F.linear(x, w[0], w[1])

    def qk_norm(t, w):
        t = t.view(t.shape[0], H, HEAD_DIM)
        r = torch.rsqrt(t.float().pow(2).mean(-1, keepdim=True) + QK_EPS)
        return ((t.float() * r).to(torch.bfloat16) * w.view(H, HEAD_DIM)).view(t.shape[0], C)

    def modln(x, scale, shift):
        return F.layer_norm(x, (C,), eps=LN_EPS) * (1 + scale) + shift

    x = torch.cat([txt, img], dim=0)
    for i in range(nd):
        d = dense[("double", i)]
        streams = {"txt.": x[:Lt], "img.": x[Lt:]}
        mods, qkv = {}, []
        for s in ("txt.", "img."):
            m = lin(d[s + "mod"], y)[0]
            mods[s] = [m[j * C:(j + 1) * C] for j in range(6)]
            t = lin(d[s + "qkv"], modln(streams[s], mods[s][1], mods[s][0]))
            w = d[s + "norm_w"]
            qkv.append(torch.cat([qk_norm(t[:, :C], w[:C]), qk_norm(t[:, C:2 * C], w[C:2 * C]), t[:, 2 * C:]], 1))
        o = attention(torch.cat(qkv, 0), C, cos, sin).transpose(0, 1).reshape(Lt + Li, C)
        new = []
        for s, a in (("txt.", o[:Lt]), ("img.", o[Lt:])):
            sh1, sc1, g1, sh2, sc2, g2 = mods[s]
            h = streams[s] + g1 * lin(d[s + "proj"], a)
            h = h + g2 * lin(d[s + "mlp_down"], F.gelu(lin(d[s + "mlp_up"], modln(h, sc2, sh2)), approximate="tanh"))
            new.append(h)
        x = torch.cat(new, 0)
    for i in range(ns):
        d = dense[("single", i)]
        m = lin(d["mod"], y)[0]
        sh, sc, g = m[:C], m[C:2 * C], m[2 * C:]
        t = lin(d["linear1"], modln(x, sc, sh))
        w = d["norm_w"]
        qkv = torch.cat([qk_norm(t[:, :C], w[:C]), qk_norm(t[:, C:2 * C], w[C:2 * C]), t[:, 2 * C:3 * C]], 1)
        o = attention(qkv, C, cos, sin).transpose(0, 1).reshape(x.shape[0], C)
        x = x + g * lin(d["linear2"], torch.cat([o, F.gelu(t[:, 3 * C:], approximate="tanh")], 1))
    return x


def forward_flop(cfg: workloads.FluxConfig, n_double=None, n_single=None) -> Dict[str, float]:
    """Multiply-add FLOPs of one forward of the blocks: ternary linears and
    attention (q k^T and p v)."""
    nd = cfg.n_double if n_double is None else n_double
    ns = cfg.n_single if n_single is None else n_single
    Li, Lt, L = cfg.img_tokens, cfg.txt_tokens, cfg.img_tokens + cfg.txt_tokens
    lin = 0.0
    for kind, n in (("double", nd), ("single", ns)):
        for name, N, K in workloads.flux_block_shapes(cfg, kind):
            M = 1 if name.endswith("mod") else (Li if name.startswith("img") else Lt if name.startswith("txt") else L)
            lin += n * 2.0 * M * N * K
    att = (nd + ns) * 2 * 2.0 * L * L * cfg.hidden
    return {"linear": lin, "attention": att}


def dense_model_forward(model: TernaryFlux, dense: Dict, io: Dict, img_lat, txt_ctx, pooled, t: float,
                        guidance: float, ids, n_double=None, n_single=None) -> torch.Tensor:
    """model_forward with the blocks in dense bf16 (dense_forward) and the
    final layer norm and modulation from torch."""
    img, txt, vec = io_layers_in(io, img_lat, txt_ctx, pooled, t, guidance)
    x = dense_forward(model, dense, img, txt, vec, ids, n_double, n_single)
    C = model.cfg.hidden
    mod = F.linear(F.silu(vec), *io["final.mod"])
    h = F.layer_norm(x[txt.shape[0]:], (C,), eps=LN_EPS) * (1 + mod[:, C:]) + mod[:, :C]
    return F.linear(h, *io["final.out"])
