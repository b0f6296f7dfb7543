"""Seeded synthetic Q/K/V generators shaped like Sana's latent token grids.

This module holds no linear-attention arithmetic: it only draws inputs. Both the
CUDA path and the fp64 oracle consume the tensors it returns, so neither side
regenerates a random stream on its own.

Token counts follow the AE-F32C32P1 autoencoder (downsampling 32, patch size 1),
which turns a 1024x1024 image into a 32x32 = 1,024-token grid and a 4096x4096
image into 128x128 = 16,384 tokens ("SANA: Efficient High-Resolution Image
Synthesis with Linear Diffusion Transformers", phd-frog.tistory.com/40, sections
2.1.2-2.1.3; "linear-diffusion-transformer-4k-efficient-generation",
blog.hotdry.top, section on DC-AE). Head counts and head size (C = H*d = 1152
with H = 36, C = 2240 with H = 70, d = 32) describe Sana-0.6B-like and
Sana-1.6B-like widths; the walk-through's section 5 gives 2240 channels for the
1.6B model. B = 2 is a classifier-free-guidance cond/uncond pair.

The block-causal workloads stand in for latent video: ``block`` tokens per
frame, 16 frames, after the video row of the token table in
"08_sana高效高分辨率生成" (papers-3lj.pages.dev), section "Linear Attention 的原理"
(4096x4096 x 16 frames = 1,048,576 tokens, i.e. 65,536 per frame; that table
counts 4,096 tokens per 1024x1024 frame). They draw the same tensors as the
sweep workloads of the same size (same seed and shape). The ``_elu1`` and ``_cos``
workloads draw the tensors of the 4096px one and use another feature map.

Recipe (all draws from one torch generator seeded per workload):
  1. Q, K, V drawn in that order with ``torch.randn`` in float32, each shaped
     (B, N, H, d).
  2. "half_normal_head_bias": Q, K, V are scaled by 0.5, then three per-head
     biases bQ, bK, bV of shape (1, 1, H, 1) are drawn (in that order) as
     0.1 * randn and added, still in float32.
  3. "tiny": rows n in NEG_ROWS of batch 0 are made all-negative in every head
     (Q <- -|Q|; an exact 0, which randn does not produce in practice, would
     become -1) so phi(Q) = 0 there and the eps path is exercised.
  4. Cast to bfloat16 (round to nearest even), except the fp32 "tiny" source,
     which the GPU sees through the same bf16 cast.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

NEG_ROWS = (0, 37, 74, 111, 148, 185, 222, 255)


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    N: int
    H: int
    d: int
    seed: int
    values: str = "normal"          # "normal" | "half_normal_head_bias"
    source: str = "bf16"            # "bf16" | "fp32" (tiny only)
    neg_rows: tuple = field(default=())
    eps: float = 1e-15
    description: str = ""
    block: int = 0                  # block-causal form: tokens per block (0 = not block-causal)
    feature: str = "relu"           # feature map phi: "relu" | "elu1" | "cos"

    @property
    def token_heads(self) -> int:
        return self.B * self.N * self.H

    def algorithmic_bytes(self, out_bytes: int) -> int:
        """One read each of Q, K, V (bf16) plus one write of O."""
        return self.token_heads * self.d * (3 * 2 + out_bytes)

    def flops(self) -> int:
        """4 d (d+1) per token-head: the state product and the apply product."""
        return self.token_heads * 4 * self.d * (self.d + 1)


def _sweep(n: int) -> Workload:
    return Workload(f"sweep_N{n}", 1, n, 36, 32, seed=4,
                    description=f"edge sweep, B=1, N={n}, H=36, d=32")


WORKLOADS: dict[str, Workload] = {
    "tiny": Workload("tiny", 1, 256, 4, 32, seed=0, source="fp32", neg_rows=NEG_ROWS,
                     description="16x16 latent, fp32 N(0,1), 8 all-negative query rows"),
    "1024px": Workload("1024px", 2, 1024, 36, 32, seed=1,
                       description="Sana-0.6B-like 1024px step: 32x32 latent, C=1152"),
    "2048px": Workload("2048px", 2, 4096, 70, 32, seed=2, values="half_normal_head_bias",
                       description="Sana-1.6B-like 2048px step: 64x64 latent, C=2240"),
    "4096px": Workload("4096px", 2, 16384, 70, 32, seed=3,
                       description="Sana-1.6B-like 4096px step: 128x128 latent, C=2240"),
    **{w.name: w for w in (_sweep(n) for n in (1024, 16384, 65536, 262144, 1048576))},
    "ragged_N16381": Workload("ragged_N16381", 1, 16381, 36, 32, seed=4,
                              description="ragged token count, B=1, H=36, d=32"),
    "d64": Workload("d64", 1, 16384, 18, 64, seed=4,
                    description="head size 64, B=1, N=16384, H=18"),
    "4096px_elu1": Workload("4096px_elu1", 2, 16384, 70, 32, seed=3, feature="elu1",
                            description="the 4096px step with phi = ELU+1"),
    "4096px_cos": Workload("4096px_cos", 2, 16384, 70, 32, seed=3, feature="cos",
                           description="the 4096px step with phi = cos"),
    "video16f_1024px": Workload("video16f_1024px", 1, 16 * 4096, 36, 32, seed=4, block=4096,
                                description="block-causal, 16 frames of 4,096 tokens, H=36, d=32"),
    "video16f_4096px": Workload("video16f_4096px", 1, 16 * 65536, 36, 32, seed=4, block=65536,
                                description="block-causal, 16 frames of 65,536 tokens, H=36, d=32"),
}


def make_inputs(w: Workload, device: str | torch.device = "cpu",
                generator_device: str = "cpu", keep_source: bool = False):
    """Draw (Q, K, V) for workload ``w``.

    Returns bf16 tensors of shape (B, N, H, d) on ``device``. With
    ``keep_source=True`` the "tiny" workload's fp32 tensors are returned as well,
    as a second triple. ``generator_device="cuda"`` draws with the CUDA
    generator instead (a different, equally seeded stream) for the largest sweep
    points, where a host draw would take minutes.
    """
    g = torch.Generator(device=generator_device)
    g.manual_seed(w.seed)
    shape = (w.B, w.N, w.H, w.d)

    def draw(s):
        return torch.randn(s, generator=g, dtype=torch.float32, device=generator_device)

    q, k, v = draw(shape), draw(shape), draw(shape)
    if w.values == "half_normal_head_bias":
        q, k, v = 0.5 * q, 0.5 * k, 0.5 * v
        bq, bk, bv = (0.1 * draw((1, 1, w.H, 1)) for _ in range(3))
        q, k, v = q + bq, k + bk, v + bv
    elif w.values != "normal":
        raise ValueError(f"unknown value recipe {w.values!r}")
    if w.neg_rows:
        rows = torch.tensor(w.neg_rows, device=generator_device)
        neg = -q[0, rows].abs()
        neg[neg == 0] = -1.0
        q[0, rows] = neg
    src = (q, k, v)
    bf = tuple(t.to(torch.bfloat16).to(device) for t in src)
    if keep_source:
        return bf, tuple(t.to(device) for t in src)
    return bf
