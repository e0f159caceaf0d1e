"""Fused Q/K prologue (per-head RMSNorm + 3D RoPE, then block means and INT8
codes of the bf16 result) against the prologue oracle.

The kernel takes y in fp32 and the oracle in fp64, so bf16(y) may differ by one
bf16 ulp where y lies within a few fp32 ulps of a bf16 rounding boundary (a
fraction of about 1e-4 of the elements), or by the fp32 rounding of the
rotation where it cancels (at most about 2^-20 of the row's largest value).
The bar: every Y element within one ulp plus that, with at most 1e-3 of them
differing; the block means within fp32
accumulation error plus the share of those flips; INT8 codes within one step
and rarely different; and, from the GPU alone, the fused means and codes equal
lx_pool_quantize_qk run on the GPU's own Y, bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import video_dit_dynamic_token_b200 as lx
from video_dit_dynamic_token_b200 import synth
from gpu_util import to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"
EPS = 1e-6


def _weights(H, d, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    return (1.0 + 0.2 * torch.randn(H, d, generator=g)).float()


def _bf16_ulp(x):
    a = np.abs(x)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, np.ldexp(1.0, (e - 7).astype(np.int64)), 2.0 ** -133)


def _check_tensor(out, X, w, grid, tag):
    r = oracle.prologue_ref(X.cpu(), w.numpy(), EPS, grid)
    Y = to_np(out["Y" + tag].float()).astype(np.float64)
    dY = np.abs(Y - r["Y"])
    # one bf16 ulp, plus the fp32 rounding of the rotation, which cancellation
    # can make large next to a small y: about 2^-24 of the pair's size, and a
    # pair's size is bounded by the row's largest value (RoPE keeps pair norms)
    rowmax = np.abs(r["Y"]).max(axis=-1, keepdims=True)
    tol = _bf16_ulp(r["Y"]) * 1.0000001 + 2.0 ** -20 * rowmax
    bad = dY > tol
    assert not bad.any(), [(tuple(i), Y[tuple(i)], r["Y"][tuple(i)]) for i in np.argwhere(bad)[:5]]
    frac = float((dY > 0).mean())
    assert frac <= 1e-3, frac
    # means: fp32 accumulation of the bf16 values, plus the flips' share
    m = to_np(out["m" + tag]).astype(np.float64)
    B, H, L, d = X.shape
    nB = oracle.n_blocks(L)
    flip = np.zeros((B, H, nB, d))
    for i in range(nB):
        rows = oracle.block_rows(i, L)
        flip[:, :, i] = dY[:, :, rows].sum(axis=2) / (rows.stop - rows.start)
    tol = 4e-6 * np.abs(r["means"]).max() + flip * 1.0000001
    assert np.all(np.abs(m - r["means"]) <= tol)
    if tag + "c" in out:
        c = to_np(out[tag + "c"]).astype(np.int32)
        dc = np.abs(c - r["codes"].astype(np.int32))
        assert dc.max() <= 1
        assert float((dc > 0).mean()) <= 2e-3
        s = to_np(out[tag + "s"]).astype(np.float64)
        assert np.all(np.abs(s - r["scales"]) <= 2.0 ** -7 * r["scales"])
    return frac


@pytest.mark.parametrize("D", [64, 128])
def test_rope_table_matches_fp64_angles(D):
    grid = (5, 9, 13)
    table = to_np(lx.lx_rope3d_table(grid, D)).astype(np.float64).reshape(-1, 2)
    dt, dh, dw = oracle.rope3d_split(D)
    want = []
    for n_pos, m in zip(grid, (dt, dh, dw)):
        i = np.arange(m // 2)
        ang = np.arange(n_pos)[:, None] * (10000.0 ** (-2.0 * i / m))[None, :]
        want.append(np.stack([np.cos(ang), np.sin(ang)], axis=-1).reshape(-1, 2))
    want = np.concatenate(want)
    assert table.shape == want.shape
    assert np.abs(table - want).max() <= 6e-8


@pytest.mark.parametrize("B,H,L,d,grid", [
    (1, 2, 1000, 128, (4, 16, 16)),    # ragged last block, L < T*Hh*W
    (2, 2, 640, 64, (2, 16, 20)),      # d = 64, B = 2
    (1, 3, 4096, 128, (4, 32, 32)),
    (1, 1, 65, 128, (1, 5, 13)),       # last block of one token
])
def test_prologue_parity(B, H, L, d, grid):
    Q, K, _ = synth.random_qkv(B, H, L, d, seed=L + d, scale=2.0, device=DEV)
    wq, wk = _weights(H, d, 1), _weights(H, d, 2)
    out = lx.lx_qk_prologue(Q, K, wq.to(DEV), wk.to(DEV), EPS, grid)
    torch.cuda.synchronize()
    assert lx.lx_last_device_status() == 0
    _check_tensor(out, Q, wq, grid, "q")
    _check_tensor(out, K, wk, grid, "k")


def test_prologue_fused_outputs_equal_block_pass_of_its_output():
    B, H, L, d, grid = 1, 2, 3000, 128, (3, 20, 50)
    Q, K, _ = synth.random_qkv(B, H, L, d, seed=5, scale=3.0, device=DEV)
    wq, wk = _weights(H, d, 3).to(DEV), _weights(H, d, 4).to(DEV)
    out = lx.lx_qk_prologue(Q, K, wq, wk, EPS, grid)
    mq, mk, qc, qs, kc, ks = lx.lx_pool_quantize_qk(out["Yq"], out["Yk"])
    torch.cuda.synchronize()
    for a, b in ((out["mq"], mq), (out["mk"], mk), (out["qc"], qc), (out["qs"], qs), (out["kc"], kc), (out["ks"], ks)):
        assert torch.equal(a, b)
    # the same means and codes without the Y outputs, and the same means without codes
    o2 = lx.lx_qk_prologue(Q, K, wq, wk, EPS, grid, with_y=False)
    o3 = lx.lx_qk_prologue(Q, K, wq, wk, EPS, grid, with_codes=False)
    torch.cuda.synchronize()
    for name in ("mq", "mk", "qc", "qs", "kc", "ks"):
        assert torch.equal(o2[name], out[name])
    for name in ("mq", "mk", "Yq", "Yk"):
        assert torch.equal(o3[name], out[name])


def test_prologue_strided_inputs():
    # Wan's [B, L, H, D] layout viewed as [B, H, L, D]
    g = torch.Generator(device=DEV).manual_seed(6)
    raw = (2 * torch.randn(1, 900, 2, 128, generator=g, device=DEV)).to(torch.bfloat16)
    X = raw.permute(0, 2, 1, 3)
    w = _weights(2, 128, 7)
    out = lx.lx_qk_prologue(X, X, w.to(DEV), w.to(DEV), EPS, (3, 15, 20))
    torch.cuda.synchronize()
    _check_tensor(out, X.contiguous(), w, (3, 15, 20), "q")


def test_prologue_720p_grid_sampled_heads():
    w = synth.WORKLOADS["720p"]
    Q, K, _ = synth.make_qkv(1, w.H, w.d, w.grid, seed=0, device=DEV)
    wq, wk = _weights(w.H, w.d, 8), _weights(w.H, w.d, 9)
    out = lx.lx_qk_prologue(Q, K, wq.to(DEV), wk.to(DEV), EPS, w.grid)
    torch.cuda.synchronize()
    assert lx.lx_last_device_status() == 0
    for h in (0, 23, 39):
        sub = {k: v[:, h:h + 1] for k, v in out.items()}
        _check_tensor(sub, Q[:, h:h + 1], wq[h:h + 1], w.grid, "q")
        _check_tensor(sub, K[:, h:h + 1], wk[h:h + 1], w.grid, "k")
