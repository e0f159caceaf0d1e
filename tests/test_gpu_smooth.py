"""K smoothing (a variant): channel means, INT8 codes of K - m and the
INT8/FP8 attention on them, against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import video_dit_dynamic_token_b200 as lx
from video_dit_dynamic_token_b200 import synth
from gpu_util import TOL_I8_MAXABS, TOL_I8_RELL1, compare_rows, plan_from_oracle, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _offset_qkv(B, H, L, d, seed, offset):
    Q, K, V = synth.random_qkv(B, H, L, d, seed=seed, device=DEV)
    g = torch.Generator(device=DEV).manual_seed(seed + 1)
    off = offset * torch.randn(1, H, 1, d, generator=g, device=DEV)
    return Q, (K.float() + off).to(torch.bfloat16), V


@pytest.mark.parametrize("B,H,L,d", [(1, 2, 1000, 128), (2, 2, 1500, 64), (1, 3, 64, 128), (1, 1, 1, 64),
                                     (1, 2, 5000, 128)])
def test_channel_mean_and_smoothed_codes_bit_exact(B, H, L, d):
    Q, K, _ = _offset_qkv(B, H, L, d, seed=L + d, offset=4.0)
    qc, qs, kc, ks, km = lx.lx_quantize_qk_smooth(Q, K)
    torch.cuda.synchronize()
    km_ref = oracle.k_channel_mean_ref(K)
    assert np.array_equal(to_np(km), km_ref)
    rc, rs = oracle.quant_k_smooth_ref(K, km_ref)
    assert np.array_equal(to_np(kc), rc) and np.array_equal(to_np(ks), rs)
    rc, rs = oracle.quant_qk_ref(Q)
    assert np.array_equal(to_np(qc), rc) and np.array_equal(to_np(qs), rs)


def test_channel_mean_strided_and_repeatable():
    g = torch.Generator(device=DEV).manual_seed(3)
    raw = (3 + torch.randn(1, 2000, 2, 128, generator=g, device=DEV)).to(torch.bfloat16)
    K = raw.permute(0, 2, 1, 3)
    a = lx.lx_k_channel_mean(K)
    b = lx.lx_k_channel_mean(K)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert np.array_equal(to_np(a), oracle.k_channel_mean_ref(K.contiguous()))


@pytest.mark.parametrize("keep", [0.2, 1.0])
def test_attention_on_smoothed_codes(keep):
    B, H, L, d = 1, 2, 3000, 128
    Q, K, V = _offset_qkv(B, H, L, d, seed=21, offset=6.0)
    plan, ref = plan_from_oracle(Q.cpu(), K.cpu(), keep, DEV)
    qc, qs, kc, ks, km = lx.lx_quantize_qk_smooth(Q, K)
    vc, vs = lx.lx_quantize_v(V)
    O = lx.lx_attn_int8fp8(qc, qs, kc, ks, vc, vs, plan)
    assert lx.lx_last_device_status() == 0
    km_ref = oracle.k_channel_mean_ref(K)
    rqc, rqs = oracle.quant_qk_ref(Q)
    rkc, rks = oracle.quant_k_smooth_ref(K, km_ref)
    rvc, rvs = oracle.quant_v_ref(V)
    blocks = [(0, h, i) for h in range(H) for i in range(oracle.n_blocks(L))]
    R = oracle.attn_int8fp8_from_codes(rqc, rqs, rkc, rks, rvc, rvs, ref["idx"], L, blocks=blocks)
    mx, rl1 = compare_rows(O, R, L, blocks)
    assert mx <= TOL_I8_MAXABS and rl1 <= TOL_I8_RELL1, (mx, rl1)


def test_smoothing_reduces_error_on_offset_keys():
    B, H, L, d = 1, 2, 3000, 128
    Q, K, V = _offset_qkv(B, H, L, d, seed=22, offset=8.0)
    plan, ref = plan_from_oracle(Q.cpu(), K.cpu(), 0.3, DEV)
    vc, vs = lx.lx_quantize_v(V)
    qc, qs, kc, ks = lx.lx_quantize_qk(Q, K)
    O_plain = lx.lx_attn_int8fp8(qc, qs, kc, ks, vc, vs, plan)
    sqc, sqs, skc, sks, _ = lx.lx_quantize_qk_smooth(Q, K)
    O_smooth = lx.lx_attn_int8fp8(sqc, sqs, skc, sks, vc, vs, plan)
    torch.cuda.synchronize()
    blocks = [(0, h, i) for h in range(H) for i in range(0, oracle.n_blocks(L), 3)]
    R = oracle.attn_ref_exact(Q.cpu(), K.cpu(), V.cpu(), ref["idx"], blocks=blocks)
    _, e_plain = compare_rows(O_plain, R, L, blocks)
    _, e_smooth = compare_rows(O_smooth, R, L, blocks)
    assert e_smooth < 0.75 * e_plain, (e_plain, e_smooth)


def test_fused_means_and_smoothed_codes_equal_separate_calls():
    Q, K, _ = _offset_qkv(1, 2, 2500, 128, seed=23, offset=5.0)
    km = lx.lx_k_channel_mean(K)
    B, H, L, d = Q.shape
    nB = oracle.n_blocks(L)
    out = (torch.empty((B, H, nB, d), dtype=torch.float32, device=DEV),
           torch.empty((B, H, nB, d), dtype=torch.float32, device=DEV),
           torch.empty((B, H, L, d), dtype=torch.int8, device=DEV), torch.empty((B, H, nB), dtype=torch.float32, device=DEV),
           torch.empty((B, H, L, d), dtype=torch.int8, device=DEV), torch.empty((B, H, nB), dtype=torch.float32, device=DEV))
    lx.lx_pool_quantize_qk_smooth(Q, K, km, out)
    pq, pk = lx.lx_pool_means(Q, K)
    qc, qs, kc, ks, _ = lx.lx_quantize_qk_smooth(Q, K, km)
    torch.cuda.synchronize()
    for a, b in zip(out, (pq, pk, qc, qs, kc, ks)):
        assert torch.equal(a, b)
