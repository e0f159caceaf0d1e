"""Light-Ulysses exchange logic on CPU: gloo ranks (world 2 and 4), the
payload steps given by the oracle and the attention by a per-head stand-in, so
that only the chunked all-to-all orchestration of ulysses_sparse_attn is under
test; the CUDA steps are tested on the GPU (tests/test_gpu_ulysses.py)."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _shards(world, B, Lr, H, D):
    g = np.random.default_rng(7)
    full = [g.standard_normal((B, world * Lr, H, D)).astype(np.float32) for _ in range(3)]
    return full, [[x[:, r * Lr:(r + 1) * Lr] for x in full] for r in range(world)]


def _oracle_ops():
    import oracle
    from video_dit_dynamic_token_b200.ulysses import UlyssesOps, payload_views

    def pack_qkv(qv, kv, vv, N, h0, hc, payload):
        # heads h0 .. h0+hc-1 of each destination's range, in destination order
        B, H, Lr, D = qv.shape
        Hr = H // N
        heads = [n * Hr + h0 + j for n in range(N) for j in range(hc)]
        sub = [x[:, heads].permute(0, 2, 1, 3).float().numpy() for x in (qv, kv, vv)]   # [B, Lr, N*hc, D]
        c, s = oracle.pack_qkv_ref(sub[0], sub[1], sub[2], N)
        codes, scales = payload_views(payload, B, hc, Lr, D, 3)
        codes.copy_(torch.from_numpy(c))
        scales.copy_(torch.from_numpy(s))

    def unpack_qkv(payload, N, qh, kh, vh):
        B, hc, L, D = qh.shape
        codes, scales = payload_views(payload, B, hc, L // N, D, 3)
        for dst, y in zip((qh, kh, vh), oracle.unpack_qkv_ref(codes.numpy(), scales.numpy())):
            dst.copy_(torch.from_numpy(y).to(torch.bfloat16))

    def pack_o(oh, N, payload):
        B, hc, L, D = oh.shape
        c, s = oracle.pack_o_ref(oh.float().numpy(), N)
        codes, scales = payload_views(payload, B, hc, L // N, D, 1)
        codes.copy_(torch.from_numpy(c))
        scales.copy_(torch.from_numpy(s))

    def unpack_o(payload, N, h0, hc, outv):
        B, H, Lr, D = outv.shape
        codes, scales = payload_views(payload, B, hc, Lr, D, 1)
        y = oracle.unpack_o_ref(codes.numpy(), scales.numpy())      # [B, Lr, N*hc, D]
        Hr = outv.shape[1] // N
        for n in range(N):
            for j in range(hc):
                outv[:, n * Hr + h0 + j] = torch.from_numpy(y[:, :, n * hc + j]).to(torch.bfloat16)

    return UlyssesOps(pack_qkv, unpack_qkv, pack_o, unpack_o,
                      attention=lambda qh, kh, vh: (vh.float() * 2 + qh.float()).to(torch.bfloat16))


def _worker(rank, world, port, n_chunks, out):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import datetime
    from video_dit_dynamic_token_b200.ulysses import ulysses_sparse_attn
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        B, Lr, H, D = 2, 3, 4 * world, 8
        _, shards = _shards(world, B, Lr, H, D)
        q, k, v = (torch.from_numpy(x).to(torch.bfloat16) for x in shards[rank])
        o = ulysses_sparse_attn(q, k, v, 0.5, ops=_oracle_ops(), n_chunks=n_chunks)
        out[rank] = o.float().numpy()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,n_chunks", [(2, 1), (2, 3), (4, 2)])
def test_exchange_round_trip_across_ranks(world, n_chunks):
    import oracle
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, port, n_chunks, out), nprocs=world, start_method="spawn", join=True)
        res = dict(out)
    B, Lr, H, D = 2, 3, 4 * world, 8
    full, _ = _shards(world, B, Lr, H, D)
    # what each head sees after the first exchange: one FP8 round trip of its
    # rows (bf16 inputs); then the stand-in attention; then one FP8 round trip back
    bf = [torch.from_numpy(x).to(torch.bfloat16).float().numpy() for x in full]
    rt = []
    for x in bf:
        c, s = oracle.fp8_rows_ref(x)
        rt.append(oracle.fp8_rows_dequant_ref(c, s))
    o_full = torch.from_numpy(rt[2] * 2 + rt[0]).float()
    o_full = o_full.to(torch.bfloat16).float().numpy()
    c, s = oracle.fp8_rows_ref(o_full)
    want = oracle.fp8_rows_dequant_ref(c, s)
    for r in range(world):
        assert np.array_equal(res[r], want[:, r * Lr:(r + 1) * Lr])


def test_head_chunks_cover_all_heads():
    sys.path.insert(0, ROOT)
    from video_dit_dynamic_token_b200.ulysses import head_chunks
    for Hr in (1, 2, 5, 10):
        for n in (1, 2, 3, 8):
            ch = head_chunks(Hr, n)
            assert sum(hc for _, hc in ch) == Hr and ch[0][0] == 0
            assert all(ch[i][0] + ch[i][1] == ch[i + 1][0] for i in range(len(ch) - 1))


def test_payload_layout_matches_the_library():
    """The host-side segment layout equals lx_ulysses_segment_bytes (a host
    call), and the code and scale views tile each segment without overlap."""
    sys.path.insert(0, ROOT)
    import ctypes
    from video_dit_dynamic_token_b200 import _abi
    from video_dit_dynamic_token_b200.ulysses import payload_views, segment_layout
    lib = _abi.load()
    for B, hc, Lr, D, X in [(1, 2, 96, 128, 3), (2, 3, 41, 64, 3), (1, 1, 7, 64, 1), (2, 5, 1, 128, 1)]:
        seg = ctypes.c_size_t(0)
        assert lib.lx_ulysses_segment_bytes(B, hc, Lr, D, X, ctypes.byref(seg)) == 0
        rows, sc_off, nbytes = segment_layout(B, hc, Lr, D, X)
        assert seg.value == nbytes and sc_off % 16 == 0 and nbytes % 16 == 0
        assert rows * D <= sc_off < sc_off + 4 * rows <= nbytes
        pay = torch.zeros((3, nbytes), dtype=torch.uint8)
        c, s = payload_views(pay, B, hc, Lr, D, X)
        c.fill_(1)
        s.view(torch.int32).fill_(0x01010101)   # no zero byte in any scale
        used = (pay != 0).sum(dim=1)
        assert used.tolist() == [rows * D + 4 * rows] * 3
    bad = ctypes.c_size_t(0)
    assert lib.lx_ulysses_segment_bytes(1, 1, 1, 96, 3, ctypes.byref(bad)) != 0
    assert lib.lx_ulysses_segment_bytes(1, 1, 1, 128, 2, ctypes.byref(bad)) != 0
