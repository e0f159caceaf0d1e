"""Light-Ulysses: head-sharded sparse attention for sequence-sharded inputs.

"600倍加速，720p视频实时生成！单卡也能带的动14B模型", §多卡路径: each GPU holds a
contiguous part of the token sequence; an all-to-all moves Q, K and V (one FP8
payload) to head-sharded form, each GPU runs the attention of its heads, and a
second all-to-all (FP8 again) brings the output back to sequence-sharded form;
the exchange runs per head chunk, the next chunk in flight while the current
one computes.  Each exchange is one all-to-all with equal splits (NCCL on the
GPU) over one byte payload of N segments, each segment holding a
destination's FP8 codes and then their fp32 scales; the layout and the FP8
rule are those of the lx_ulysses_* calls (include/lx_sparse_attn.h).

The per-step operations are passed in as `UlyssesOps`; the default runs the
CUDA kernels and lx_sparse_attn.  Nothing here computes on the host.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass
from typing import Callable

import torch
import torch.distributed as dist

from . import _abi, _check, _ptr, _stream, bhld, lx_sparse_attn


# ---------------------------------------------------------------- payload layout
def segment_layout(B, hc, Lr, D, X):
    """(rows, byte offset of the scales, bytes) of one destination's segment:
    codes uint8 [B, hc, Lr, X, D], then from the 16-byte rounded code size the
    scales fp32 [B, hc, Lr, X], the segment rounded up to 16 bytes
    (lx_ulysses_segment_bytes gives the same size)."""
    rows = B * hc * Lr * X
    sc_off = (rows * D + 15) // 16 * 16
    return rows, sc_off, sc_off + (rows * 4 + 15) // 16 * 16


def new_payload(N, B, hc, Lr, D, X, device):
    return torch.empty((N, segment_layout(B, hc, Lr, D, X)[2]), dtype=torch.uint8, device=device)


def payload_views(payload, B, hc, Lr, D, X):
    """The codes [N, B, hc, Lr, (X,) D] and scales [N, B, hc, Lr, (X)] inside a
    payload [N, seg] (views, no copy; the X axis is dropped for X = 1)."""
    N = payload.shape[0]
    rows, sc_off, _ = segment_layout(B, hc, Lr, D, X)
    shape = (N, B, hc, Lr, X) if X > 1 else (N, B, hc, Lr)
    codes = payload[:, :rows * D].view(*shape, D)
    scales = payload[:, sc_off:sc_off + rows * 4].view(torch.float32).view(*shape)
    return codes, scales


# ---------------------------------------------------------------- CUDA operations
def pack_qkv(qv, kv, vv, N, h0, hc, payload, stream=None):
    """qv, kv, vv: [B, H, Lr, D] views of this rank's shard -> payload [N, seg]."""
    lib = _abi.load()
    q, k, v = bhld(qv), bhld(kv), bhld(vv)
    _check(lib.lx_ulysses_pack_qkv(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), N, h0, hc, _ptr(payload),
                                   _stream(stream)), "lx_ulysses_pack_qkv")


def unpack_qkv(payload, N, qh, kh, vh, stream=None):
    """Received payload [N, seg] -> q, k, v [B, hc, L, D]."""
    lib = _abi.load()
    q, k, v = bhld(qh), bhld(kh), bhld(vh)
    _check(lib.lx_ulysses_unpack_qkv(_ptr(payload), N, ctypes.byref(q), ctypes.byref(k), ctypes.byref(v),
                                     _stream(stream)), "lx_ulysses_unpack_qkv")


def pack_o(oh, N, payload, stream=None):
    """Attention output [B, hc, L, D] -> payload [N, seg] (segment n: rank n's tokens)."""
    lib = _abi.load()
    o = bhld(oh)
    _check(lib.lx_ulysses_pack_o(ctypes.byref(o), N, _ptr(payload), _stream(stream)), "lx_ulysses_pack_o")


def unpack_o(payload, N, h0, hc, outv, stream=None):
    """Received output payload -> heads of this rank's shard view outv [B, H, Lr, D]."""
    lib = _abi.load()
    o = bhld(outv)
    _check(lib.lx_ulysses_unpack_o(_ptr(payload), N, h0, hc, ctypes.byref(o), _stream(stream)),
           "lx_ulysses_unpack_o")


@dataclass
class UlyssesOps:
    pack_qkv: Callable = pack_qkv
    unpack_qkv: Callable = unpack_qkv
    pack_o: Callable = pack_o
    unpack_o: Callable = unpack_o
    attention: Callable = None   # (q, k, v [B, hc, L, D]) -> o [B, hc, L, D]


def head_chunks(Hr: int, n: int):
    """Split Hr heads into n nearly equal contiguous chunks (h0, hc)."""
    n = max(1, min(n, Hr))
    base, extra = divmod(Hr, n)
    out, h0 = [], 0
    for i in range(n):
        hc = base + (1 if i < extra else 0)
        out.append((h0, hc))
        h0 += hc
    return out


def _exchange(recv, send, group):
    if dist.is_initialized():
        return dist.all_to_all_single(recv, send, group=group, async_op=True)
    recv.copy_(send)
    return None


def ulysses_sparse_attn(q, k, v, keep, mode="int8fp8", group=None, n_chunks=2, ops: UlyssesOps | None = None):
    """q, k, v: this rank's shard [B, Lr, H, D] (bf16).  Returns the attention
    output of the shard's tokens over all heads, [B, Lr, H, D]."""
    ops = ops or UlyssesOps()
    attention = ops.attention or (lambda qh, kh, vh: lx_sparse_attn(qh, kh, vh, keep, mode)[0])
    N = dist.get_world_size(group) if dist.is_initialized() else 1
    B, Lr, H, D = q.shape
    if H % N:
        raise ValueError("the head count must be divisible by the number of ranks")
    Hr, L = H // N, N * Lr
    dev = q.device
    qv, kv, vv = (x.permute(0, 2, 1, 3) for x in (q, k, v))        # [B, H, Lr, D] views
    out = torch.empty_like(q)
    outv = out.permute(0, 2, 1, 3)
    chunks = head_chunks(Hr, n_chunks)

    def start_qkv(h0, hc):
        send = new_payload(N, B, hc, Lr, D, 3, dev)
        ops.pack_qkv(qv, kv, vv, N, h0, hc, send)
        recv = torch.empty_like(send)
        return recv, _exchange(recv, send, group), send

    pending_out = []
    nxt = start_qkv(*chunks[0])
    for i, (h0, hc) in enumerate(chunks):
        recv, work, _keep_alive = nxt
        if i + 1 < len(chunks):       # the next chunk's payload travels while this one computes
            nxt = start_qkv(*chunks[i + 1])
        if work is not None:
            work.wait()
        qh, kh, vh = (torch.empty((B, hc, L, D), dtype=torch.bfloat16, device=dev) for _ in range(3))
        ops.unpack_qkv(recv, N, qh, kh, vh)
        oh = attention(qh, kh, vh)
        send_o = new_payload(N, B, hc, Lr, D, 1, dev)
        ops.pack_o(oh, N, send_o)
        recv_o = torch.empty_like(send_o)
        pending_out.append((h0, hc, recv_o, _exchange(recv_o, send_o, group), send_o))
    for h0, hc, recv_o, work, _keep_alive in pending_out:
        if work is not None:
            work.wait()
        ops.unpack_o(recv_o, N, h0, hc, outv)
    return out
