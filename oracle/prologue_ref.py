"""CPU oracle for the fused Q/K prologue: per-head RMSNorm, 3D RoPE, then the
block means and INT8 codes of the result; and for the K-smoothing variant of
the INT8 quantiser (plain numpy, fp64).

TEST INFRASTRUCTURE ONLY, like ``sparse_attn_ref``: only ``tests/`` use it; it
shares no code with the CUDA library.

What the pages fix: "600倍加速，720p视频实时生成！单卡也能带的动14B模型",
§高效推理算子 (last paragraph), and "Run Wan2.2-A14B on One RTX 5090: 720p
Video in 3.8s", §4: 3D RoPE and RMSNorm run as fused or parallel kernels, with
fewer dispatches, temporary tensors and memory round trips.  They give no
formula, so everything below is this library's reading:
  * RMSNorm over each head's d channels:  y = x / sqrt(mean_c x_c^2 + eps) * w[h, c]
    (a weight per head and channel; one vector for all heads is the case of
    equal rows);
  * 3D RoPE: the token at raster index n of a (T, Hh, W) grid (w fastest) has
    position (t, h, w) = (n div (Hh*W), (n div W) mod Hh, n mod W).  The head
    dimension is split into three contiguous parts of even sizes
    (d_t, d_h, d_w), by default (d - 4*floor(d/6), 2*floor(d/6), 2*floor(d/6));
    inside a part of size m that belongs to coordinate p, the channel pair
    (2i, 2i+1) is rotated by the angle p * theta^(-2i/m) (theta = 10000):
    (a, b) -> (a cos - b sin, a sin + b cos), the rotary embedding of RoFormer
    applied per axis;
  * the prologue's output tensor is the bf16 (round to nearest even) value of
    rope(rmsnorm(x)); the block means and the INT8 codes are those of that bf16
    tensor (``block_means`` and ``quant_qk_ref``).

Pins for every function live in ``tests/test_oracle_prologue.py``.
"""
from __future__ import annotations


import numpy as np

from .sparse_attn_ref import _f64, block_means, quant_qk_ref

ROPE_THETA = 10000.0


def rope3d_split(d: int) -> tuple[int, int, int]:
    """Default sizes of the (t, h, w) parts of a head dimension d."""
    q = d // 6
    return d - 4 * q, 2 * q, 2 * q


def token_positions(L: int, grid) -> np.ndarray:
    """[L, 3] integer (t, h, w) of the raster tokens 0..L-1 of grid (T, Hh, W)."""
    T, Hh, W = grid
    if L > T * Hh * W:
        raise ValueError("more tokens than grid positions")
    n = np.arange(L)
    return np.stack([n // (Hh * W), (n // W) % Hh, n % W], axis=1)


def qk_rmsnorm_ref(X, w, eps: float) -> np.ndarray:
    """y[b,h,t,c] = x / sqrt(mean_c x^2 + eps) * w[h, c]; X [B,H,L,d], w [H,d]."""
    x = _f64(X)
    w = _f64(w)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * w[None, :, None, :]


def rope3d_ref(X, grid, theta: float = ROPE_THETA, split=None) -> np.ndarray:
    """Rotate the channel pairs of each part by position * theta^(-2i/m)."""
    x = _f64(X)
    B, H, L, d = x.shape
    split = rope3d_split(d) if split is None else tuple(split)
    if sum(split) != d or any(m % 2 for m in split):
        raise ValueError("the three parts must be even and add up to d")
    pos = token_positions(L, grid)  # [L, 3]
    y = x.copy()
    c0 = 0
    for axis, m in enumerate(split):
        i = np.arange(m // 2)
        freq = theta ** (-2.0 * i / m)                     # [m/2]
        ang = pos[:, axis][:, None] * freq[None, :]        # [L, m/2]
        cs, sn = np.cos(ang), np.sin(ang)
        a = x[..., c0 + 2 * i]
        b = x[..., c0 + 2 * i + 1]
        y[..., c0 + 2 * i] = a * cs - b * sn
        y[..., c0 + 2 * i + 1] = a * sn + b * cs
        c0 += m
    return y


def bf16_round(x) -> np.ndarray:
    """Round fp64 values to the nearest bf16 (8 significant bits), ties to even."""
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    nz = x != 0
    e = np.floor(np.log2(np.abs(x[nz])))
    ulp = np.ldexp(1.0, (e - 7).astype(np.int64))
    out[nz] = np.rint(x[nz] / ulp) * ulp  # rint: half to even
    return out


def prologue_ref(X, w, eps: float, grid, theta: float = ROPE_THETA, split=None) -> dict:
    """The prologue of one tensor (Q or K): bf16 output Y, block means and INT8
    codes/scales of Y."""
    Y = bf16_round(rope3d_ref(qk_rmsnorm_ref(X, w, eps), grid, theta, split))
    codes, scales = quant_qk_ref(Y)
    return {"Y": Y, "means": block_means(Y), "codes": codes, "scales": scales}


# --------------------------------------------------------------------------
# K smoothing (a variant: not on the pages)
# --------------------------------------------------------------------------
# Subtracting one vector m from every key changes each score row by the constant
# q.m, which the softmax removes, so the attention is unchanged; quantising
# K - m instead of K shrinks the INT8 error when K has large channel offsets.
# This library's reading: m = the per-(b, h, channel) mean of K over all L
# tokens, taken in fp64 and rounded to fp32 once; the codes are those of
# fl32(K - m) by the INT8 rule of ``quant_qk_ref``.

def k_channel_mean_ref(K) -> np.ndarray:
    """fp32 [B,H,D]: fl32(mean over tokens of K), the mean taken in fp64."""
    return _f64(K).mean(axis=2).astype(np.float32)


def quant_k_smooth_ref(K, km) -> tuple:
    """INT8 codes and scales of fl32(K - km) (km fp32 [B,H,D])."""
    x = (_f64(K).astype(np.float32) - np.asarray(km, dtype=np.float32)[:, :, None, :]).astype(np.float32)
    return quant_qk_ref(x)
