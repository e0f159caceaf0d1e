"""Quantiser parity (step a3): INT8 Q/K and E4M3 V codes and scales, bit-exact."""
import numpy as np
import pytest
import torch

import oracle
import video_dit_dynamic_token_b200 as lx
from video_dit_dynamic_token_b200 import synth
from gpu_util import to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("B,H,L,d,scale", [(1, 2, 1024, 64, 1.0), (1, 3, 1000, 128, 3.0), (2, 1, 65, 128, 0.01),
                                           (1, 2, 1, 64, 1.0), (1, 1, 4096, 128, 40.0)])
def test_quant_qk_bit_exact(B, H, L, d, scale):
    Q, K, _ = synth.random_qkv(B, H, L, d, seed=L, scale=scale, device=DEV)
    qc, qs, kc, ks = lx.lx_quantize_qk(Q, K)
    torch.cuda.synchronize()
    for codes, sc, X in ((qc, qs, Q), (kc, ks, K)):
        rc, rs = oracle.quant_qk_ref(X)
        assert np.array_equal(to_np(codes), rc)
        assert np.array_equal(to_np(sc), rs)


@pytest.mark.parametrize("B,H,L,d,scale", [(1, 2, 1024, 64, 1.0), (1, 3, 1000, 128, 3.0), (2, 1, 65, 128, 1e-3),
                                           (1, 2, 1, 64, 1.0), (1, 1, 9000, 128, 100.0)])
def test_quant_v_bit_exact(B, H, L, d, scale):
    _, _, V = synth.random_qkv(B, H, L, d, seed=L + 1, scale=scale, device=DEV)
    vc, vs = lx.lx_quantize_v(V)
    torch.cuda.synchronize()
    rc, rs = oracle.quant_v_ref(V)
    assert np.array_equal(to_np(vc), rc)
    assert np.array_equal(to_np(vs), rs)


def test_quant_zero_block_and_channel():
    Q, K, V = synth.random_qkv(1, 1, 200, 128, seed=2, device=DEV)
    Q = Q.clone()
    Q[0, 0, 64:128] = 0
    V = V.clone()
    V[0, 0, :, 5] = 0
    qc, qs, _, _ = lx.lx_quantize_qk(Q, K)
    vc, vs = lx.lx_quantize_v(V)
    torch.cuda.synchronize()
    assert to_np(qs)[0, 0, 1] == 1.0 and np.all(to_np(qc)[0, 0, 64:128] == 0)
    assert to_np(vs)[0, 0, 5] == 1.0 and np.all(to_np(vc)[0, 0, :, 5] == 0)


def test_quant_full_720p_heads_subset():
    w = synth.WORKLOADS["720p"]
    Q, K, V = synth.make_qkv(1, w.H, w.d, w.grid, seed=0, device=DEV)
    qc, qs, kc, ks = lx.lx_quantize_qk(Q, K)
    vc, vs = lx.lx_quantize_v(V)
    torch.cuda.synchronize()
    for h in (0, 17, 39):
        rc, rs = oracle.quant_qk_ref(K[:, h:h + 1].cpu())
        assert np.array_equal(to_np(kc[:, h:h + 1]), rc) and np.array_equal(to_np(ks[:, h:h + 1]), rs)
        rc, rs = oracle.quant_v_ref(V[:, h:h + 1].cpu())
        assert np.array_equal(to_np(vc[:, h:h + 1]), rc) and np.array_equal(to_np(vs[:, h:h + 1]), rs)


@pytest.mark.parametrize("B,H,L,d,scale", [(1, 2, 1024, 64, 1.0), (1, 3, 1000, 128, 3.0), (2, 1, 65, 128, 0.01),
                                           (1, 2, 1, 64, 1.0), (1, 2, 4097, 128, 40.0)])
def test_pool_quantize_fused_equals_separate_calls(B, H, L, d, scale):
    # one read of Q/K for both outputs: identical to lx_pool_means + lx_quantize_qk,
    # and those agree with the oracle (means to fp32 rounding, codes bit-exact)
    Q, K, _ = synth.random_qkv(B, H, L, d, seed=L + 3, scale=scale, device=DEV)
    mq, mk, qc, qs, kc, ks = lx.lx_pool_quantize_qk(Q, K)
    pq, pk = lx.lx_pool_means(Q, K)
    sq, ssq, sk, ssk = lx.lx_quantize_qk(Q, K)
    torch.cuda.synchronize()
    for a, b in ((mq, pq), (mk, pk), (qc, sq), (qs, ssq), (kc, sk), (ks, ssk)):
        assert torch.equal(a, b)
    for m, codes, sc, X in ((mq, qc, qs, Q), (mk, kc, ks, K)):
        ref = oracle.block_means(X)
        assert np.abs(to_np(m) - ref).max() <= 2e-6 * max(1e-30, np.abs(ref).max())
        rc, rs = oracle.quant_qk_ref(X)
        assert np.array_equal(to_np(codes), rc)
        assert np.array_equal(to_np(sc), rs)


def test_pool_quantize_fused_strided_view():
    # Wan's [B, L, H, D] layout viewed as [B, H, L, D]: strided rows
    g = torch.Generator(device=DEV).manual_seed(4)
    raw = (torch.randn(1, 1000, 3, 128, generator=g, device=DEV) * 2).to(torch.bfloat16)
    Q = raw.permute(0, 2, 1, 3)
    mq, _, qc, qs, _, _ = lx.lx_pool_quantize_qk(Q, Q)
    torch.cuda.synchronize()
    Qc = Q.contiguous()
    ref = oracle.block_means(Qc)
    assert np.abs(to_np(mq) - ref).max() <= 2e-6 * np.abs(ref).max()
    rc, rs = oracle.quant_qk_ref(Qc)
    assert np.array_equal(to_np(qc), rc) and np.array_equal(to_np(qs), rs)
