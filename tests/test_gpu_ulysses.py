"""Light-Ulysses exchange kernels against the oracle, bit for bit: N virtual
ranks on one GPU, the all-to-all emulated by gathering segment r of every
rank's payload for rank r; and the whole ulysses_sparse_attn on a one-rank
NCCL group."""
import datetime
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
import video_dit_dynamic_token_b200 as lx
from video_dit_dynamic_token_b200 import ulysses
from gpu_util import to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _shards(N, B, Lr, H, D, seed):
    g = torch.Generator(device=DEV).manual_seed(seed)
    full = [(2 * torch.randn(B, N * Lr, H, D, generator=g, device=DEV)).to(torch.bfloat16) for _ in range(3)]
    return full, [[x[:, r * Lr:(r + 1) * Lr].contiguous() for x in full] for r in range(N)]


@pytest.mark.parametrize("N,B,Lr,H,D", [(4, 1, 96, 8, 128), (2, 2, 40, 6, 64), (1, 1, 130, 3, 128)])
def test_qkv_and_output_exchange_bit_exact(N, B, Lr, H, D):
    full, shards = _shards(N, B, Lr, H, D, seed=N + Lr)
    Hr = H // N
    chunks = ulysses.head_chunks(Hr, 2)
    for h0, hc in chunks:
        sends = []
        for r in range(N):
            qv, kv, vv = (x.permute(0, 2, 1, 3) for x in shards[r])
            pay = ulysses.new_payload(N, B, hc, Lr, D, 3, DEV)
            ulysses.pack_qkv(qv, kv, vv, N, h0, hc, pay)
            sends.append(pay)
            c, s = ulysses.payload_views(pay, B, hc, Lr, D, 3)
            heads = [n * Hr + h0 + j for n in range(N) for j in range(hc)]
            rc, rs = oracle.pack_qkv_ref(*(x[:, :, heads].cpu() for x in shards[r]), N)
            assert np.array_equal(to_np(c), rc) and np.array_equal(to_np(s), rs)
        for r in range(N):
            recv = torch.stack([sends[n][r] for n in range(N)])
            rc, rs = ulysses.payload_views(recv, B, hc, Lr, D, 3)
            qh, kh, vh = (torch.empty((B, hc, N * Lr, D), dtype=torch.bfloat16, device=DEV) for _ in range(3))
            ulysses.unpack_qkv(recv, N, qh, kh, vh)
            want = oracle.unpack_qkv_ref(to_np(rc), to_np(rs))
            for got, w in zip((qh, kh, vh), want):
                assert np.array_equal(to_np(got.float()).astype(np.float64), w)
            # the way back, with the received V standing in for the output
            pay_o = ulysses.new_payload(N, B, hc, Lr, D, 1, DEV)
            ulysses.pack_o(vh, N, pay_o)
            oc, os_ = ulysses.payload_views(pay_o, B, hc, Lr, D, 1)
            c2, s2 = oracle.pack_o_ref(vh.cpu(), N)
            assert np.array_equal(to_np(oc), c2) and np.array_equal(to_np(os_), s2)
            out = torch.zeros((B, Lr, H, D), dtype=torch.bfloat16, device=DEV)
            ulysses.unpack_o(pay_o, N, h0, hc, out.permute(0, 2, 1, 3))
            y = oracle.unpack_o_ref(c2, s2)                       # [B, Lr, N*hc, D]
            for n in range(N):
                for j in range(hc):
                    assert np.array_equal(to_np(out[:, :, n * Hr + h0 + j].float()).astype(np.float64),
                                          y[:, :, n * hc + j])


def test_ulysses_sparse_attn_one_rank_nccl():
    B, L, H, D, keep = 1, 4096, 4, 128, 0.2
    g = torch.Generator(device=DEV).manual_seed(5)
    q, k, v = ((1.5 * torch.randn(B, L, H, D, generator=g, device=DEV)).to(torch.bfloat16) for _ in range(3))
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        out = ulysses.ulysses_sparse_attn(q, k, v, keep, "int8fp8", n_chunks=2)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert lx.lx_last_device_status() == 0
    # the same steps called one by one (one chunk of all heads: the attention is per head)
    qv, kv, vv = (x.permute(0, 2, 1, 3) for x in (q, k, v))
    pay = ulysses.new_payload(1, B, H, L, D, 3, DEV)
    ulysses.pack_qkv(qv, kv, vv, 1, 0, H, pay)
    qh, kh, vh = (torch.empty((B, H, L, D), dtype=torch.bfloat16, device=DEV) for _ in range(3))
    ulysses.unpack_qkv(pay, 1, qh, kh, vh)
    oh, _ = lx.lx_sparse_attn(qh, kh, vh, keep, "int8fp8")
    pay_o = ulysses.new_payload(1, B, H, L, D, 1, DEV)
    ulysses.pack_o(oh, 1, pay_o)
    want = torch.empty_like(q)
    ulysses.unpack_o(pay_o, 1, 0, H, want.permute(0, 2, 1, 3))
    torch.cuda.synchronize()
    assert torch.equal(out, want)
