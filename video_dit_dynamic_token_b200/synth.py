"""Seeded synthetic inputs shaped like Wan2.2-A14B self-attention activations.

This module holds the input recipe only: it draws random Q, K, V tensors and
names the workloads. It contains none of the attention method's arithmetic
(no pooling, scoring, selection, quantisation or softmax), so both the CUDA
path and the CPU oracle may take their inputs from it.

Recipe (the pages name no dataset; these fields stand in for the post-RoPE
Q/K/V of a 14B video DiT at the token grids the pages quote, about 120K tokens
at the largest -- "Run Wan2.2-A14B on One RTX 5090: 720p Video in 3.8s",
"Why this matters"):

* one generator seeded with ``seed``; draws are fp32, in this fixed order:
  Q coarse, Q noise, K coarse, K noise, V;
* coarse field ``N(0,1)`` of shape ``[B*H, d, ceil(T/2), ceil(Hh/4), ceil(W/4)]``,
  trilinearly upsampled (``align_corners=False``) to ``(T, Hh, W)`` and flattened
  in raster order (t, h, w), w fastest;
* ``Q = 2*up + 0.5*N(0,1)``, the same for K with independent draws
  (``smooth=False`` drops the field: Q, K ~ N(0,1), no spatial locality);
* ``V ~ N(0,1)``; everything cast to bf16 (round to nearest even).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch
import torch.nn.functional as F


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    d: int
    grid: tuple  # (T, Hh, W) token grid
    keep: float
    modes: tuple

    @property
    def L(self) -> int:
        T, Hh, W = self.grid
        return T * Hh * W


# Token grids of the Wan2.2 latent at 480p / 720p and a ~120K-token case.
WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 64, (4, 16, 16), 0.25, ("bf16", "int8fp8")),
    "480p": Workload("480p", 1, 40, 128, (21, 30, 52), 0.2, ("int8fp8",)),
    "720p": Workload("720p", 1, 40, 128, (21, 45, 80), 0.1, ("int8fp8", "bf16")),
    "long": Workload("long", 1, 40, 128, (21, 60, 96), 0.1, ("int8fp8",)),
}
SWEEP_KEEPS = (0.05, 0.1, 0.2, 0.5, 1.0)


def _field(gen, BH, d, grid, device):
    T, Hh, W = grid
    coarse = torch.randn(BH, d, math.ceil(T / 2), math.ceil(Hh / 4), math.ceil(W / 4),
                         generator=gen, dtype=torch.float32, device=device)
    up = F.interpolate(coarse, size=(T, Hh, W), mode="trilinear", align_corners=False)
    return up.reshape(BH, d, T * Hh * W).transpose(1, 2)  # [BH, L, d]


def make_qkv(B, H, d, grid, seed=0, smooth=True, device="cpu", out_dtype=torch.bfloat16):
    """Return contiguous ``(Q, K, V)`` of shape ``[B, H, L, d]`` (bf16 by default)."""
    T, Hh, W = grid
    L = T * Hh * W
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    out = []
    for _ in range(2):  # Q then K
        if smooth:
            up = _field(gen, B * H, d, grid, device)
            noise = torch.randn(B * H, L, d, generator=gen, dtype=torch.float32, device=device)
            x = 2.0 * up + 0.5 * noise
            del noise, up
        else:
            x = torch.randn(B * H, L, d, generator=gen, dtype=torch.float32, device=device)
        out.append(x.to(out_dtype).reshape(B, H, L, d).contiguous())
        del x
    v = torch.randn(B * H, L, d, generator=gen, dtype=torch.float32, device=device)
    out.append(v.to(out_dtype).reshape(B, H, L, d).contiguous())
    return tuple(out)


def make_workload(name, seed=0, smooth=True, device="cpu"):
    w = WORKLOADS[name]
    return make_qkv(w.B, w.H, w.d, w.grid, seed=seed, smooth=smooth, device=device)


def random_qkv(B, H, L, d, seed=0, scale=1.0, device="cpu"):
    """Plain i.i.d. N(0, scale^2) bf16 Q, K, V of shape [B, H, L, d] (for odd shapes)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    return tuple((scale * torch.randn(B, H, L, d, generator=gen, device=device)).to(torch.bfloat16)
                 for _ in range(3))
