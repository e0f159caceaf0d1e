"""CPU oracle for the Light-Ulysses exchange: FP8 row quantisation of the
fused Q/K/V payload and of the attention output, and the layout changes of the
sequence <-> head all-to-all (plain numpy).

TEST INFRASTRUCTURE ONLY, like ``sparse_attn_ref``: only ``tests/`` use it; it
shares no code with the CUDA library.

What the pages fix ("600倍加速，720p视频实时生成！单卡也能带的动14B模型",
§多卡路径; "Run Wan2.2-A14B on One RTX 5090: 720p Video in 3.8s", §4): Ulysses
sequence parallelism splits the token sequence over the GPUs and an all-to-all
moves the data between the sequence and head dimensions, so that each GPU
computes the attention of part of the heads; the exchanged data is FP8, Q, K
and V travel as one all-to-all payload, and the all-to-all runs per head
chunk, overlapped with the attention of the previous chunk.  Everything else
is this library's reading:
  * N ranks; rank r holds tokens [r*Lr, (r+1)*Lr) of every head (Lr = L / N,
    the sequence split in equal contiguous shards), in the layout [B, Lr, H, D];
  * after the exchange rank r holds heads [r*Hr, (r+1)*Hr) (Hr = H / N) of all
    L tokens, [B, Hr, L, D];
  * FP8: one scale per (token, head, tensor) row of D values, s = absmax/448
    (1 for an all-zero row), code = E4M3 round-to-nearest-even with
    saturation of fl32(x * fl32(448/absmax)); the receiver's value is
    bf16(fl32(decode(code) * s));
  * the payload a rank sends to rank n is [B, Hr, Lr, 3, D] codes (Q, K, V of
    rank n's heads, this rank's tokens) and [B, Hr, Lr, 3] fp32 scales; the
    output goes back the same way as [B, Hr, Lr, D] codes and [B, Hr, Lr]
    scales.

Pins live in ``tests/test_oracle_ulysses.py``.
"""
from __future__ import annotations

import numpy as np

from .prologue_ref import bf16_round
from .sparse_attn_ref import E4M3_MAX, _f32, e4m3_decode, e4m3_encode, e4m3_round


def fp8_rows_ref(X):
    """E4M3 codes (uint8, same shape) and fp32 scales (shape[:-1]) of the rows of X."""
    x = _f32(X)
    a = np.abs(x).max(axis=-1).astype(np.float32)
    nz = a > 0
    inv = np.where(nz, np.float32(E4M3_MAX) / np.where(nz, a, np.float32(1)), np.float32(0)).astype(np.float32)
    y = (x * inv[..., None]).astype(np.float32)
    codes = e4m3_encode(e4m3_round(y))
    scales = np.where(nz, a / np.float32(E4M3_MAX), np.float32(1)).astype(np.float32)
    return codes, scales


def fp8_rows_dequant_ref(codes, scales) -> np.ndarray:
    """bf16 (as fp64) of fl32(decode(code) * scale)."""
    v = (e4m3_decode(codes).astype(np.float32) * np.asarray(scales, dtype=np.float32)[..., None]).astype(np.float32)
    return bf16_round(v.astype(np.float64))


def pack_qkv_ref(q, k, v, N):
    """Send buffers of one rank: q, k, v [B, Lr, H, D] -> codes [N, B, Hr, Lr, 3, D],
    scales [N, B, Hr, Lr, 3]."""
    x = np.stack([_f32(q), _f32(k), _f32(v)], axis=3)        # [B, Lr, H, 3, D]
    B, Lr, H, _, D = x.shape
    Hr = H // N
    x = x.reshape(B, Lr, N, Hr, 3, D).transpose(2, 0, 3, 1, 4, 5)   # [N, B, Hr, Lr, 3, D]
    return fp8_rows_ref(x)


def all_to_all_ref(sends):
    """sends[r] is rank r's buffer with leading dimension N (slice n goes to rank
    n); returns the receive buffers: recv[r][n] = sends[n][r]."""
    N = len(sends)
    return [np.stack([sends[n][r] for n in range(N)]) for r in range(N)]


def unpack_qkv_ref(codes, scales):
    """Receive buffers [N, B, Hr, Lr, 3, D] -> q, k, v [B, Hr, L, D] (bf16 values
    as fp64), token n*Lr + t from source rank n."""
    y = fp8_rows_dequant_ref(codes, scales)                   # [N, B, Hr, Lr, 3, D]
    N, B, Hr, Lr, _, D = y.shape
    y = y.transpose(1, 2, 0, 3, 4, 5).reshape(B, Hr, N * Lr, 3, D)
    return y[..., 0, :], y[..., 1, :], y[..., 2, :]


def pack_o_ref(o, N):
    """o [B, Hr, L, D] -> codes [N, B, Hr, Lr, D], scales [N, B, Hr, Lr]
    (slice n holds the tokens of rank n)."""
    x = _f32(o)
    B, Hr, L, D = x.shape
    Lr = L // N
    x = x.reshape(B, Hr, N, Lr, D).transpose(2, 0, 1, 3, 4)
    return fp8_rows_ref(x)


def unpack_o_ref(codes, scales):
    """Receive buffers [N, B, Hr, Lr, D] -> o [B, Lr, H, D], head n*Hr + h from
    source rank n."""
    y = fp8_rows_dequant_ref(codes, scales)                   # [N, B, Hr, Lr, D]
    N, B, Hr, Lr, D = y.shape
    return y.transpose(1, 3, 0, 2, 4).reshape(B, Lr, N * Hr, D)
