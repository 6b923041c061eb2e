"""Seeded synthetic workloads for ReLU linear attention.

This module only draws inputs and describes workload shapes. It holds none of
the attention arithmetic, so both the float64 oracle and the CUDA path can use
it without sharing any of the method's code.

Shapes follow the latent sizes of the SANA family:

* images: the F32C32P1 autoencoder turns a P x P image into (P/32)^2 tokens
  ("Sana: Efficient High-Resolution Image Synthesis with Linear Diffusion
  Transformers", section "模型架构", item 1); Sana-0.6B has 36 heads and
  Sana-1.6B 70 heads of width 32 (same page, "参数与分辨率策略").
* video: a latent grid of T x Hh x W tokens with 3D RoPE
  ("SANA-Video: Efficient Video Generation with Block Linear Diffusion
  Transformer", section "Stage 2"), and the block-causal loop of section 4.

Every tensor is drawn in float32 from the torch CPU generator with a fixed
seed, then rounded to bfloat16 once. The same bytes feed the oracle and the GPU.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional, Tuple

import torch

HEAD_DIM = 32


@dataclasses.dataclass(frozen=True)
class Workload:
    """One attention-layer workload.

    For non-causal configs ``N`` tokens per batch element; with RoPE the
    tokens form a ``T x Hh x W`` grid in (t, h, w) raster order.  For the
    block-causal config there are ``M`` blocks of ``T x Hh x W`` tokens, each
    applied ``steps`` times and then folded into the carried state once.
    """

    name: str
    B: int
    N: int
    H: int
    D: int = HEAD_DIM
    rope: bool = False
    T: int = 1
    Hh: int = 1
    W: int = 1
    rope_base: float = 10000.0
    eps: float = 1e-6
    outlier_frac: float = 0.0
    outlier_scale: float = 1.0
    M: int = 1  # blocks (block-causal only)
    steps: int = 0  # denoise passes per block (block-causal only)
    block_causal: bool = False

    @property
    def token_heads(self) -> int:
        return self.B * self.N * self.H

    @property
    def tensor_elems(self) -> int:
        return self.B * self.N * self.H * self.D


WORKLOADS: Dict[str, Workload] = {
    # Sana-0.6B, 512px image: 16x16 latent tokens, 36 heads.
    "sana0.6b_512px": Workload("sana0.6b_512px", B=1, N=256, H=36),
    # Sana-1.6B, 1024px image, batch 4: 32x32 latent tokens, 70 heads.
    "sana1.6b_1024px": Workload("sana1.6b_1024px", B=4, N=1024, H=70),
    # Sana-1.6B, 4096px image: 128x128 latent tokens, 1% of K entries x20.
    "sana1.6b_4k": Workload("sana1.6b_4k", B=1, N=16384, H=70,
                            outlier_frac=0.01, outlier_scale=20.0),
    # SANA-Video 480p layer: 21x30x52 latent grid, 3D RoPE.
    "sanavideo_480p": Workload("sanavideo_480p", B=1, N=21 * 30 * 52, H=70,
                               rope=True, T=21, Hh=30, W=52),
    # LongSANA: 12 blocks of 20x30x52 tokens, 4 denoise passes + 1 update.
    "longsana_block_causal": Workload("longsana_block_causal", B=1,
                                      N=20 * 30 * 52, H=70, rope=True,
                                      T=20, Hh=30, W=52, M=12, steps=4,
                                      block_causal=True),
}


def scaled(w: Workload, **changes) -> Workload:
    """A copy of ``w`` with some fields replaced (used for small test cases)."""
    return dataclasses.replace(w, **changes)


def _randn_bf16(shape: Tuple[int, ...], seed: int, outlier_frac: float = 0.0,
                outlier_scale: float = 1.0) -> torch.Tensor:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    x = torch.randn(shape, generator=g, dtype=torch.float32)
    if outlier_frac > 0.0:
        pick = torch.rand(shape, generator=g, dtype=torch.float32) < outlier_frac
        x = torch.where(pick, x * float(outlier_scale), x)
    return x.to(torch.bfloat16)


def make_qkv(w: Workload, seed: int = 0, block: Optional[int] = None,
             step: Optional[int] = None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Draw Q, K, V as contiguous bf16 CPU tensors of shape [B, N, H, D].

    Non-causal: Q/K/V use seeds ``seed + 0/1/2``.
    Block-causal: pass ``block`` = m and ``step`` = s (s = steps is the update
    pass); the seed is ``seed + 1000*m + 10*s + {0,1,2}``.
    Outliers (when the workload has them) are applied to K only.
    """
    shape = (w.B, w.N, w.H, w.D)
    base = int(seed)
    if block is not None:
        base += 1000 * int(block) + 10 * int(step or 0)
    q = _randn_bf16(shape, base + 0)
    k = _randn_bf16(shape, base + 1, w.outlier_frac, w.outlier_scale)
    v = _randn_bf16(shape, base + 2)
    return q, k, v


def make_tensor(shape: Tuple[int, ...], seed: int, dtype=torch.bfloat16) -> torch.Tensor:
    """A single seeded N(0,1) tensor, rounded once to ``dtype``."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return torch.randn(shape, generator=g, dtype=torch.float32).to(dtype)


def t_offset_of_block(w: Workload, m: int) -> int:
    """Global frame index of block m's first latent frame."""
    return int(m) * w.T


def hidden_width(w: Workload) -> int:
    """Model width of the DiT whose attention layer ``w`` describes: heads x
    head width (2240 for Sana-1.6B's 70 heads, 1152 for Sana-0.6B's 36)."""
    return int(w.H) * int(w.D)


def make_projection(w: Workload, C: int, seed: int = 0) -> Tuple[torch.Tensor, torch.Tensor,
                                                                  torch.Tensor]:
    """Token features and a random-init QKV projection, all bf16 CPU tensors.

    X [B, N, C] ~ N(0, 1); W [3 H D, C] ~ N(0, 1/C), so that each projected
    feature is about N(0, 1) like the attention inputs above; bias [3 H D] ~
    N(0, 0.1^2). Rows of W (and entries of the bias): all query features, then
    all key features, then all value features; head h owns rows
    [D h, D h + D) of each. Seeds ``seed + 0/1/2``. There are no trained
    weights: only the shapes and scales follow the model."""
    hd = w.H * w.D
    x = make_tensor((w.B, w.N, C), seed)
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) + 1)
    wt = (torch.randn((3 * hd, C), generator=g, dtype=torch.float32) / float(C) ** 0.5)
    g.manual_seed(int(seed) + 2)
    b = torch.randn((3 * hd,), generator=g, dtype=torch.float32) * 0.1
    return x, wt.to(torch.bfloat16), b.to(torch.bfloat16)
