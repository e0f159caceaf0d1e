"""Planner parity (steps a1 pool, a2 score + top-k) against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import video_dit_dynamic_token_b200 as lx
from video_dit_dynamic_token_b200 import synth
from gpu_util import check_plan, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _inputs(B, H, L, d, seed=0, smooth=False):
    if smooth:
        raise NotImplementedError
    return synth.random_qkv(B, H, L, d, seed=seed, device=DEV)


@pytest.mark.parametrize("B,H,L,d", [(1, 2, 1024, 64), (1, 3, 1000, 128), (2, 2, 65, 128), (1, 1, 1, 64),
                                     (1, 2, 130, 64)])
def test_pool_means(B, H, L, d):
    Q, K, _ = _inputs(B, H, L, d, seed=L)
    mq, mk = lx.lx_pool_means(Q, K)
    torch.cuda.synchronize()
    for got, X in ((mq, Q), (mk, K)):
        ref = oracle.block_means(X)
        err = np.abs(to_np(got) - ref).max() / max(1e-30, np.abs(ref).max())
        assert err < 2e-6, err


def test_pool_means_strided_view():
    # Wan's natural [B, L, H, D] layout, viewed as [B, H, L, D]
    g = torch.Generator(device=DEV).manual_seed(1)
    raw = torch.randn(2, 777, 3, 128, generator=g, device=DEV).to(torch.bfloat16)
    Q = raw.permute(0, 2, 1, 3)
    mq, mk = lx.lx_pool_means(Q, Q)
    torch.cuda.synchronize()
    ref = oracle.block_means(Q.contiguous())
    assert np.abs(to_np(mq) - ref).max() < 2e-6 * np.abs(ref).max()


@pytest.mark.parametrize("B,H,L,d,keep", [
    (1, 2, 1024, 64, 0.25),      # the tiny workload shape
    (1, 3, 1000, 128, 0.3),      # ragged last block
    (2, 2, 4160, 128, 0.1),      # nB = 65 (odd), B = 2
    (1, 2, 64, 128, 0.5),        # nB = 1
    (1, 2, 65, 64, 0.5),         # last block of one token
    (1, 1, 1, 64, 0.9),          # L = 1
    (1, 2, 3000, 128, 1.0),      # keep everything
    (1, 2, 3000, 128, 0.01),     # k = 1
])
def test_plan_parity_small(B, H, L, d, keep):
    Q, K, _ = _inputs(B, H, L, d, seed=L + 7)
    plan = lx.lx_sparse_attn_plan(Q, K, keep)
    assert lx.lx_last_device_status() == 0
    check_plan(plan.idx, plan.mask, Q.cpu(), K.cpu(), keep)


def test_plan_parity_tiny_workload():
    Q, K, _ = synth.make_workload("tiny")
    plan = lx.lx_sparse_attn_plan(Q.to(DEV), K.to(DEV), 0.25)
    assert lx.lx_last_device_status() == 0
    check_plan(plan.idx, plan.mask, Q, K, 0.25)


def test_plan_all_equal_scores_take_lowest_ids():
    # zero Q: every score is 0, so the k lowest key ids must be kept
    Q = torch.zeros(1, 1, 640, 128, dtype=torch.bfloat16, device=DEV)
    _, K, _ = _inputs(1, 1, 640, 128, seed=3)
    plan = lx.lx_sparse_attn_plan(Q, K, 0.3)
    k = plan.k
    assert np.array_equal(to_np(plan.idx)[0, 0], np.tile(np.arange(k), (10, 1)))


def test_plan_duplicate_key_blocks_tie_to_lower_index():
    Q, K, _ = _inputs(1, 1, 64 * 40, 128, seed=5)
    K = K.clone()
    K[0, 0, 64 * 30:64 * 31] = K[0, 0, 64 * 7:64 * 8]     # blocks 7 and 30 identical
    K[0, 0, 64 * 33:64 * 34] = K[0, 0, 64 * 7:64 * 8]     # and 33
    for keep in (0.05, 0.1, 0.2, 0.5):
        plan = lx.lx_sparse_attn_plan(Q, K, keep)
        check_plan(plan.idx, plan.mask, Q.cpu(), K.cpu(), keep)
        gi = to_np(plan.idx)[0, 0]
        for row in gi:   # a later duplicate is never kept without the earlier one
            s = set(row.tolist())
            assert not ((30 in s or 33 in s) and 7 not in s)
            assert not (33 in s and 30 not in s)


@pytest.mark.parametrize("name", ["480p", "720p", "long"])
def test_plan_parity_full_size(name):
    w = synth.WORKLOADS[name]
    Q, K, _ = synth.make_qkv(w.B, w.H, w.d, w.grid, seed=0, device=DEV)
    plan = lx.lx_sparse_attn_plan(Q, K, w.keep)
    assert lx.lx_last_device_status() == 0
    Qc, Kc = Q.cpu(), K.cpu()
    del Q, K
    # a flipped pair costs two bits; near-ties at the k-th place are rare
    check_plan(plan.idx, plan.mask, Qc, Kc, w.keep, max_exempt_frac=2e-3)


@pytest.mark.parametrize("keep", [0.05, 0.5, 1.0])
@pytest.mark.parametrize("smooth", [True, False])
def test_plan_parity_720p_keep_sweep(keep, smooth):
    w = synth.WORKLOADS["720p"]
    Q, K, _ = synth.make_qkv(1, 4, w.d, w.grid, seed=1, smooth=smooth, device=DEV)
    plan = lx.lx_sparse_attn_plan(Q, K, keep)
    assert lx.lx_last_device_status() == 0
    check_plan(plan.idx, plan.mask, Q.cpu(), K.cpu(), keep, max_exempt_frac=2e-3)


@pytest.mark.parametrize("keep", [0.1, 0.5])
def test_plan_large_tie_groups_take_lowest_ids(keep):
    # key blocks cycle through three patterns, so every score row holds only
    # three distinct values with ~100 members each: the bucket holding the k-th
    # score has far more members than the candidate buffer, and the exact
    # whole-row ranking must keep the lowest ids of the tied group.  Identical
    # key blocks give bit-identical means and scores on both sides, and the
    # three levels are far apart, so the ids must match the oracle exactly.
    nB, d = 300, 128
    Q, _, _ = _inputs(1, 2, 64 * nB, d, seed=11)
    g = torch.Generator(device=DEV).manual_seed(12)
    base = torch.randn(3, 2, 64, d, generator=g, device=DEV).to(torch.bfloat16)
    K = torch.stack([base[j % 3] for j in range(nB)], dim=1).reshape(2, nB * 64, d).unsqueeze(0)
    plan = lx.lx_sparse_attn_plan(Q, K, keep)
    assert lx.lx_last_device_status() == 0
    ref = oracle.plan_ref(Q.cpu(), K.cpu(), keep)
    assert np.array_equal(to_np(plan.idx), ref["idx"])
    check_plan(plan.idx, plan.mask, Q.cpu(), K.cpu(), keep)


def test_plan_narrow_score_range_with_large_offset():
    # all means near one common vector: the scores share a large offset and
    # differ by a small fraction of it
    B, H, L, d = 1, 2, 64 * 200, 128
    g = torch.Generator(device=DEV).manual_seed(13)
    Q = (1.0 + 0.1 * torch.randn(B, H, L, d, generator=g, device=DEV)).to(torch.bfloat16)
    K = (1.0 + 0.1 * torch.randn(B, H, L, d, generator=g, device=DEV)).to(torch.bfloat16)
    for keep in (0.1, 0.3):
        plan = lx.lx_sparse_attn_plan(Q, K, keep)
        assert lx.lx_last_device_status() == 0
        check_plan(plan.idx, plan.mask, Q.cpu(), K.cpu(), keep)


@pytest.mark.parametrize("smooth", [True, False])
def test_plan_parity_maximum_row_length(smooth):
    # nB = 2176, the longest score row the selection holds (17 chunks of 128),
    # on a grid of 2 heads; ragged last tile of the score GEMM (2176 = 17 * 128)
    grid = (17, 64, 128)    # 139264 tokens = 2176 blocks of 64
    Q, K, _ = synth.make_qkv(1, 2, 128, grid, seed=4, smooth=smooth, device=DEV)
    assert Q.shape[2] == 64 * 2176
    plan = lx.lx_sparse_attn_plan(Q, K, 0.1)
    assert lx.lx_last_device_status() == 0
    assert plan.nB == 2176
    check_plan(plan.idx, plan.mask, Q.cpu(), K.cpu(), 0.1)
