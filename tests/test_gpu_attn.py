"""Sparse attention parity (step a4): BF16 against the exact oracle, INT8/FP8
against the quantisation-simulating oracle, element by element."""
import numpy as np
import pytest
import torch

import oracle
import video_dit_dynamic_token_b200 as lx
from video_dit_dynamic_token_b200 import synth
from gpu_util import (TOL_BF16_MAXABS, TOL_I8_MAXABS, TOL_I8_RELL1, compare_rows, plan_from_oracle,
                      sample_blocks, to_np)

pytestmark = pytest.mark.gpu
DEV = "cuda"

SMALL = [
    (1, 2, 1024, 64, 0.25),     # tiny workload shape
    (1, 3, 1000, 128, 0.3),     # ragged last block, odd nB
    (1, 2, 4160, 128, 0.1),     # nB = 65: last pair holds one block
    (2, 2, 640, 64, 0.5),
    (1, 2, 64, 128, 0.5),       # nB = 1
    (1, 2, 40, 128, 0.5),       # one partial block
    (1, 2, 65, 64, 1.0),        # last block of one token
    (1, 2, 2048, 128, 1.0),     # dense
]


def _all_blocks(B, H, L):
    return [(b, h, i) for b in range(B) for h in range(H) for i in range(oracle.n_blocks(L))]


@pytest.mark.parametrize("B,H,L,d,keep", SMALL)
def test_attn_bf16_small(B, H, L, d, keep):
    Q, K, V = synth.random_qkv(B, H, L, d, seed=L + d, device=DEV)
    plan, ref = plan_from_oracle(Q.cpu(), K.cpu(), keep, DEV)
    O = lx.lx_attn_bf16(Q, K, V, plan)
    assert lx.lx_last_device_status() == 0
    R = oracle.attn_ref_exact(Q.cpu(), K.cpu(), V.cpu(), ref["idx"])
    mx, _ = compare_rows(O, R, L, _all_blocks(B, H, L))
    assert mx <= TOL_BF16_MAXABS, mx


@pytest.mark.parametrize("B,H,L,d,keep", SMALL)
def test_attn_int8fp8_small(B, H, L, d, keep):
    Q, K, V = synth.random_qkv(B, H, L, d, seed=L + d + 1, device=DEV)
    plan, ref = plan_from_oracle(Q.cpu(), K.cpu(), keep, DEV)
    O = lx.lx_sparse_attn_fwd(Q, K, V, plan, "int8fp8")
    assert lx.lx_last_device_status() == 0
    R = oracle.attn_ref_int8fp8(Q.cpu(), K.cpu(), V.cpu(), ref["idx"])
    mx, rl1 = compare_rows(O, R, L, _all_blocks(B, H, L))
    assert mx <= TOL_I8_MAXABS and rl1 <= TOL_I8_RELL1, (mx, rl1)


@pytest.mark.parametrize("mode", ["bf16", "int8fp8"])
def test_attn_tiny_workload_end_to_end(mode):
    """Plan and attention both from the library, oracle on the library's plan."""
    Q, K, V = synth.make_workload("tiny")
    Qd, Kd, Vd = Q.to(DEV), K.to(DEV), V.to(DEV)
    plan = lx.lx_sparse_attn_plan(Qd, Kd, 0.25)
    O = lx.lx_sparse_attn_fwd(Qd, Kd, Vd, plan, mode)
    assert lx.lx_last_device_status() == 0
    idx = to_np(plan.idx)
    R = (oracle.attn_ref_exact if mode == "bf16" else oracle.attn_ref_int8fp8)(Q, K, V, idx)
    mx, rl1 = compare_rows(O, R, Q.shape[2], _all_blocks(1, 2, 1024))
    if mode == "bf16":
        assert mx <= TOL_BF16_MAXABS
    else:
        assert mx <= TOL_I8_MAXABS and rl1 <= TOL_I8_RELL1, (mx, rl1)


def test_attn_strided_output_and_inputs():
    g = torch.Generator(device=DEV).manual_seed(4)
    raw = torch.randn(3, 1, 700, 2, 128, generator=g, device=DEV).to(torch.bfloat16)   # [3, B, L, H, D]
    Q, K, V = (raw[i].permute(0, 2, 1, 3) for i in range(3))                        # [B, H, L, D] views
    plan, ref = plan_from_oracle(Q.cpu(), K.cpu(), 0.4, DEV)
    out_raw = torch.zeros(1, 700, 2, 128, dtype=torch.bfloat16, device=DEV)
    O = out_raw.permute(0, 2, 1, 3)
    lx.lx_attn_bf16(Q, K, V, plan, out=O)
    assert lx.lx_last_device_status() == 0
    R = oracle.attn_ref_exact(Q.cpu(), K.cpu(), V.cpu(), ref["idx"])
    mx, _ = compare_rows(O, R, 700, _all_blocks(1, 2, 700))
    assert mx <= TOL_BF16_MAXABS


@pytest.mark.parametrize("name,mode", [("720p", "int8fp8"), ("720p", "bf16"), ("480p", "int8fp8"),
                                       ("long", "int8fp8")])
def test_attn_full_size_sampled(name, mode):
    """Full-size run in the configuration the benchmark times; the oracle checks
    a sample of query blocks (including the ragged last one) one by one."""
    w = synth.WORKLOADS[name]
    Q, K, V = synth.make_qkv(w.B, w.H, w.d, w.grid, seed=0, device=DEV)
    plan = lx.lx_sparse_attn_plan(Q, K, w.keep)
    O = lx.lx_sparse_attn_fwd(Q, K, V, plan, mode)
    assert lx.lx_last_device_status() == 0
    nB = plan.nB
    blocks = sample_blocks(w.B, w.H, nB, 12, seed=1, must=[(0, 0, 0), (0, w.H - 1, nB - 1), (0, 5, nB - 2)])
    idx = to_np(plan.idx)
    Qc, Kc, Vc = Q.cpu(), K.cpu(), V.cpu()
    if mode == "bf16":
        R = oracle.attn_ref_exact(Qc, Kc, Vc, idx, blocks=blocks)
        mx, _ = compare_rows(O, R, w.L, blocks)
        assert mx <= TOL_BF16_MAXABS, mx
    else:
        R = oracle.attn_ref_int8fp8(Qc, Kc, Vc, idx, blocks=blocks)
        mx, rl1 = compare_rows(O, R, w.L, blocks)
        assert mx <= TOL_I8_MAXABS and rl1 <= TOL_I8_RELL1, (mx, rl1)
    # every output row is finite
    assert torch.isfinite(O.float()).all()


def test_attn_720p_pure_noise_keep_sweep():
    w = synth.WORKLOADS["720p"]
    Q, K, V = synth.make_qkv(1, 2, w.d, w.grid, seed=2, smooth=False, device=DEV)
    for keep in (0.05, 0.5):
        plan = lx.lx_sparse_attn_plan(Q, K, keep)
        O8 = lx.lx_sparse_attn_fwd(Q, K, V, plan, "int8fp8")
        Ob = lx.lx_sparse_attn_fwd(Q, K, V, plan, "bf16")
        assert lx.lx_last_device_status() == 0
        blocks = sample_blocks(1, 2, plan.nB, 6, seed=3, must=[(0, 1, plan.nB - 1)])
        idx = to_np(plan.idx)
        R8 = oracle.attn_ref_int8fp8(Q.cpu(), K.cpu(), V.cpu(), idx, blocks=blocks)
        Rb = oracle.attn_ref_exact(Q.cpu(), K.cpu(), V.cpu(), idx, blocks=blocks)
        mx, rl1 = compare_rows(O8, R8, w.L, blocks)
        assert mx <= TOL_I8_MAXABS and rl1 <= TOL_I8_RELL1, (keep, mx, rl1)
        mx, _ = compare_rows(Ob, Rb, w.L, blocks)
        assert mx <= TOL_BF16_MAXABS, (keep, mx)


@pytest.mark.parametrize("qk_scale", [4.0, 6.0, 10.0])
def test_attn_int8fp8_large_qk_scales(qk_scale):
    # large Q/K magnitudes: the per-block score scale crosses the bound below
    # which the softmax folds the INT8 magic offset into its FMA constant, so
    # both the folded and the exact exponent paths run (V stays at scale 1)
    B, H, L, d, keep = 1, 2, 3000, 128, 0.2
    Q, K, _ = synth.random_qkv(B, H, L, d, seed=31, scale=qk_scale, device=DEV)
    _, _, V = synth.random_qkv(B, H, L, d, seed=32, device=DEV)
    plan, ref = plan_from_oracle(Q.cpu(), K.cpu(), keep, DEV)
    O = lx.lx_sparse_attn_fwd(Q, K, V, plan, "int8fp8")
    assert lx.lx_last_device_status() == 0
    R = oracle.attn_ref_int8fp8(Q.cpu(), K.cpu(), V.cpu(), ref["idx"])
    mx, rl1 = compare_rows(O, R, L, _all_blocks(B, H, L))
    assert mx <= TOL_I8_MAXABS and rl1 <= TOL_I8_RELL1, (mx, rl1)


@pytest.mark.parametrize("mode", ["int8fp8", "bf16"])
def test_one_call_equals_plan_then_forward(mode):
    B, H, L, d, keep = 1, 3, 5000, 128, 0.15
    Q, K, V = synth.random_qkv(B, H, L, d, seed=41, scale=1.5, device=DEV)
    plan = lx.lx_sparse_attn_plan(Q, K, keep)
    O1 = lx.lx_sparse_attn_fwd(Q, K, V, plan, mode)
    O2, plan2 = lx.lx_sparse_attn(Q, K, V, keep, mode)
    torch.cuda.synchronize()
    assert lx.lx_last_device_status() == 0
    assert torch.equal(plan.idx, plan2.idx) and torch.equal(plan.mask, plan2.mask)
    assert torch.equal(O1, O2)


@pytest.mark.parametrize("mode", ["int8fp8", "bf16"])
def test_attn_720p_whole_head(mode):
    """Every query block of one head at the 720p grid (1182 blocks, the ragged
    last one included), element by element, in the launch the benchmark times
    (all 40 heads in one call)."""
    w = synth.WORKLOADS["720p"]
    Q, K, V = synth.make_qkv(w.B, w.H, w.d, w.grid, seed=0, device=DEV)
    plan = lx.lx_sparse_attn_plan(Q, K, w.keep)
    O = lx.lx_sparse_attn_fwd(Q, K, V, plan, mode)
    assert lx.lx_last_device_status() == 0
    h = 23
    Qh, Kh, Vh = (x[:, h:h + 1].cpu() for x in (Q, K, V))
    idx = to_np(plan.idx)[:, h:h + 1]
    Oh = O[:, h:h + 1]
    del Q, K, V
    blocks = _all_blocks(1, 1, w.L)
    if mode == "bf16":
        R = oracle.attn_ref_exact(Qh, Kh, Vh, idx)
        mx, _ = compare_rows(Oh, R, w.L, blocks)
        assert mx <= TOL_BF16_MAXABS, mx
    else:
        R = oracle.attn_ref_int8fp8(Qh, Kh, Vh, idx)
        mx, rl1 = compare_rows(Oh, R, w.L, blocks)
        assert mx <= TOL_I8_MAXABS and rl1 <= TOL_I8_RELL1, (mx, rl1)
