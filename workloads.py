"""Seeded synthetic workloads for the MATE token-mix core.

This module only describes shapes and draws random inputs. It holds none of
the method's arithmetic, so both the CUDA path (through its tests and the
bench) and the CPU oracle can be fed from it without sharing any code.

Shapes follow the five video-latent grids the token mix is measured on
(a tiny fp32 case and 256p/512p/768p grids of 17 s to 68 s). The pages give
no latent grid sizes, so these grids stand in for the pages' workloads; the
layer widths come from the LinGen paper review (xllm-io), "5.1 实验设置":
20 heads and embedding width 2560, with the Mamba2 head dimension 64 stated
under "MA-Branch", item 1.

Distributions (drawn on the host; the SSD inputs from a ``torch.Generator``
seeded with ``seed`` in the order x, dt_raw, A_raw, B, C, D, the attention
inputs q, k, v from a second generator seeded with ``seed + 1``, so that
either set can be drawn without the other):
    x ~ N(0, 1)
    dt = softplus(N(0, 1) - 4)
    A = -exp(U(0, ln 16))          (long-memory variant: divided by 256)
    B, C ~ N(0, 1) / sqrt(d_state)
    D ~ N(0, 1)
    q, k, v ~ N(0, 1)
Tensors the config marks bf16 (x, B, C, q, k, v) are cast to bf16 after the
draw; dt, A and D stay fp32.

`chunk` is the scan's tiling length, not part of the method: the output does
not depend on it beyond rounding. The bf16 grids use 512-token chunks (the
longest the tensor-core scan takes); the tiny fp32 case uses 32.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace
from typing import Dict, Optional, Tuple

import torch

# scan-mode codes shared by every layer of the stack
SR, SC, TR, TC = 0, 1, 2, 3
ZZ = 4  # the zigzag scan the pages compare RMS against (a comparison order, not an RMS mode)
MODE_NAMES = {SR: "spatial-row", SC: "spatial-column", TR: "temporal-row", TC: "temporal-column", ZZ: "zigzag"}


@dataclass(frozen=True)
class Config:
    name: str
    batch: int
    T: int
    H: int
    W: int
    # SSD (MA-branch)
    nheads: int
    headdim: int
    dstate: int
    ngroups: int
    chunk: int
    dtype: str                      # "f32" or "bf16" for x, B, C, q, k, v, out
    modes: Tuple[int, ...]          # RMS modes exercised by this config
    review: Optional[Tuple[int, int, int]]   # pooling kernel (pt, ph, pw) or None
    # TESA (TE-branch)
    attn_heads: int
    attn_dim: int
    Tw: int
    Sw: int
    shift: Tuple[int, int, int]
    variant: str = "default"        # "default" or "long_memory"

    @property
    def N(self) -> int:
        return self.T * self.H * self.W

    @property
    def tokens(self) -> int:
        return self.batch * self.N

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def with_(self, **kw) -> "Config":
        return replace(self, **kw)


CONFIGS: Dict[str, Config] = {
    "tiny": Config("tiny", 1, 4, 8, 8, 2, 16, 16, 1, 32, "f32", (SR, SC, TR, TC), (2, 4, 4),
                   2, 16, 2, 4, (1, 2, 2)),
    "256p-17s": Config("256p-17s", 1, 32, 16, 16, 80, 64, 64, 1, 512, "bf16", (SR,), None,
                       20, 128, 2, 8, (0, 0, 0)),
    "512p-17s": Config("512p-17s", 1, 32, 32, 32, 80, 64, 64, 1, 512, "bf16", (SR, SC, TR, TC),
                       (4, 8, 8), 20, 128, 2, 8, (1, 4, 4)),
    "512p-68s": Config("512p-68s", 1, 128, 32, 32, 80, 64, 64, 1, 512, "bf16", (TC,), (8, 8, 8),
                       20, 128, 2, 8, (1, 4, 4)),
    "768p-17s": Config("768p-17s", 2, 32, 48, 48, 80, 64, 64, 1, 512, "bf16", (SR, SC, TR, TC), None,
                       20, 128, 2, 8, (0, 0, 0)),
}

# the grid the headline throughput is quoted on (131,072 tokens)
HEADLINE = "512p-68s"


# model width of the MATE block ([Review] 5.1: embedding width 2560)
D_MODEL = 2560


def generate_compose(tokens: int, k_ma: int, k_te: int, d_model: int = D_MODEL, seed: int = 0,
                     dtype=torch.bfloat16) -> Dict[str, torch.Tensor]:
    """Inputs of the MATE composition on the host: the two branch outputs as
    rows (y_ma ~ N(0, 1), y_te ~ N(0, 1)) and random-init projections in the
    nn.Linear layout, w ~ N(0, 1 / (k_ma + k_te)) (so that out has unit scale),
    from a generator seeded with seed + 2 in the order y_ma, y_te, w_ma, w_te."""
    g = torch.Generator().manual_seed(seed + 2)
    scale = 1.0 / math.sqrt(max(k_ma + k_te, 1))
    y_ma = torch.randn(tokens, k_ma, generator=g)
    y_te = torch.randn(tokens, k_te, generator=g)
    w_ma = torch.randn(d_model, k_ma, generator=g) * scale
    w_te = torch.randn(d_model, k_te, generator=g) * scale
    return {k: v.to(dtype) for k, v in dict(y_ma=y_ma, y_te=y_te, w_ma=w_ma, w_te=w_te).items()}


def generate_gate_norm(tokens: int, channels: int, seed: int = 0) -> Dict[str, torch.Tensor]:
    """Inputs of the MA-branch output side on the host: the bi-SSD output y ~ N(0, 1) and the
    front-end's z ~ N(0, 1) as (tokens, channels) bf16 rows, and the norm weight
    w ~ 1 + N(0, 1) / 10 fp32 (an RMS norm weight starts at one), from a generator seeded with
    seed + 4 in the order y, z, w."""
    g = torch.Generator().manual_seed(seed + 4)
    y = torch.randn(tokens, channels, generator=g).to(torch.bfloat16)
    z = torch.randn(tokens, channels, generator=g).to(torch.bfloat16)
    w = 1.0 + torch.randn(channels, generator=g) / 10
    return {"y": y, "z": z, "w": w.float()}


def generate_frontend(cfg: Config, seed: int = 0, d_model: int = D_MODEL) -> Dict[str, torch.Tensor]:
    """Inputs of the MA-branch front-end for a grid: the block input u ~ N(0, 1)
    (batch, T, H, W, d_model) bf16, a random-init in_proj w_in ~ N(0, 1/d_model)
    (rows z, x, B, C, dt) bf16, conv taps and biases ~ U(-1/2, 1/2) fp32 (the
    uniform range of a width-4 conv's default init), and dt_bias = -4 fp32, so
    that dt = softplus(N(0, 1) - 4) as in the SSD inputs above. From a generator
    seeded with seed + 3 in the order u, w_in, conv_w, conv_b."""
    g = torch.Generator().manual_seed(seed + 3)
    d_inner = cfg.nheads * cfg.headdim
    dc = d_inner + 2 * cfg.ngroups * cfg.dstate
    u = torch.randn(cfg.batch, cfg.T, cfg.H, cfg.W, d_model, generator=g)
    w_in = torch.randn(d_inner + dc + cfg.nheads, d_model, generator=g) / math.sqrt(d_model)
    conv_w = torch.rand(dc, 4, generator=g) - 0.5
    conv_b = torch.rand(dc, generator=g) - 0.5
    dt_bias = torch.full((cfg.nheads,), -4.0)
    return {"u": u.to(torch.bfloat16), "w_in": w_in.to(torch.bfloat16), "conv_w": conv_w.float(),
            "conv_b": conv_b.float(), "dt_bias": dt_bias}


def generate_block(cfg: Config, seed: int = 0, d_model: int = D_MODEL) -> Dict[str, torch.Tensor]:
    """Input and random-init weights of one MATE token mixer on the host: the front-end's
    (generate_frontend: u, w_in, conv_w, conv_b, dt_bias), then, from a generator seeded
    with seed + 5 in this order, the SSD's A = -exp(U(0, ln 16)) and D ~ N(0, 1) (as in
    generate), the gated norm's weight 1 + N(0, 1) / 10, the TE-branch projections
    w_q, w_k, w_v ~ N(0, 1 / d_model) and the composition's w_ma, w_te ~ N(0, 1 / (k_ma + k_te))."""
    out = generate_frontend(cfg, seed=seed, d_model=d_model)
    g = torch.Generator().manual_seed(seed + 5)
    d_inner, te = cfg.nheads * cfg.headdim, cfg.attn_heads * cfg.attn_dim
    A = -torch.exp(torch.rand(cfg.nheads, generator=g) * math.log(16.0))
    D = torch.randn(cfg.nheads, generator=g)
    norm_w = 1.0 + torch.randn(d_inner, generator=g) / 10
    wq, wk, wv = (torch.randn(te, d_model, generator=g) / math.sqrt(d_model) for _ in range(3))
    scale = 1.0 / math.sqrt(d_inner + te)
    w_ma = torch.randn(d_model, d_inner, generator=g) * scale
    w_te = torch.randn(d_model, te, generator=g) * scale
    out.update(A=A.float(), D=D.float(), norm_w=norm_w.float(), w_q=wq.to(torch.bfloat16), w_k=wk.to(torch.bfloat16),
               w_v=wv.to(torch.bfloat16), w_ma=w_ma.to(torch.bfloat16), w_te=w_te.to(torch.bfloat16))
    return out


def sweep_configs():
    """N from 8k to 131k tokens at H=W=32 with the 131k grid's other settings."""
    base = CONFIGS[HEADLINE]
    return [base.with_(name=f"sweep-T{t}", T=t) for t in (8, 16, 32, 64, 128)]


def generate(cfg: Config, seed: int = 0, parts: Tuple[str, ...] = ("ssd", "attn")) -> Dict[str, torch.Tensor]:
    """Draw one batch of inputs on the host.

    The draw order within each stream is fixed, and the two streams are
    independent, so a config's SSD inputs do not depend on whether the
    attention inputs are drawn too.
    Returns CPU tensors in grid order (batch, T, H, W, ...).
    """
    g = torch.Generator().manual_seed(seed)
    b, T, H, W = cfg.batch, cfg.T, cfg.H, cfg.W
    out: Dict[str, torch.Tensor] = {}
    dt_ = cfg.torch_dtype
    if "ssd" in parts:
        x = torch.randn(b, T, H, W, cfg.nheads, cfg.headdim, generator=g)
        dt_raw = torch.randn(b, T, H, W, cfg.nheads, generator=g)
        a_raw = torch.rand(cfg.nheads, generator=g)
        Bm = torch.randn(b, T, H, W, cfg.ngroups, cfg.dstate, generator=g) / math.sqrt(cfg.dstate)
        Cm = torch.randn(b, T, H, W, cfg.ngroups, cfg.dstate, generator=g) / math.sqrt(cfg.dstate)
        D = torch.randn(cfg.nheads, generator=g)
        dt = torch.nn.functional.softplus(dt_raw - 4.0)
        A = -torch.exp(a_raw * math.log(16.0))
        if cfg.variant == "long_memory":
            A = A / 256.0
        out.update(x=x.to(dt_), dt=dt.float().contiguous(), A=A.float(), B=Bm.to(dt_), C=Cm.to(dt_),
                   D=D.float())
    if "attn" in parts:
        ga = torch.Generator().manual_seed(seed + 1)
        shape = (b, T, H, W, cfg.attn_heads, cfg.attn_dim)
        q = torch.randn(*shape, generator=ga)
        k = torch.randn(*shape, generator=ga)
        v = torch.randn(*shape, generator=ga)
        out.update(q=q.to(dt_), k=k.to(dt_), v=v.to(dt_))
    return out

