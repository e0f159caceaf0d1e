"""Failure detection on the device without faulting it: bounded waits that
run out report LX_ERR_TIMEOUT and leave the context usable; a malformed plan
is reported, not followed out of bounds."""
import numpy as np
import pytest
import torch

import video_dit_dynamic_token_b200 as lx
from video_dit_dynamic_token_b200 import synth
from video_dit_dynamic_token_b200._abi import LX_ERR_PLAN, LX_ERR_TIMEOUT

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_bounded_wait_times_out_and_context_survives():
    assert lx.lx_last_device_status() == 0
    lx.lx_debug_wait_timeout(50_000_000)        # 50 ms on a barrier nothing completes
    assert lx.lx_last_device_status() == LX_ERR_TIMEOUT
    assert lx.lx_last_device_status() == 0      # status word is cleared by the read
    x = torch.arange(10, device=DEV)
    assert int(x.sum()) == 45                   # the context still works
    Q, K, V = synth.random_qkv(1, 1, 256, 64, seed=0, device=DEV)
    plan = lx.lx_sparse_attn_plan(Q, K, 0.5)
    lx.lx_attn_bf16(Q, K, V, plan)
    assert lx.lx_last_device_status() == 0


def test_malformed_plan_is_reported():
    Q, K, V = synth.random_qkv(1, 1, 512, 128, seed=1, device=DEV)
    plan = lx.lx_sparse_attn_plan(Q, K, 0.5)
    bad = plan.idx.clone()
    bad[0, 0, 0] = torch.flip(bad[0, 0, 0], dims=[0])          # descending
    bad[0, 0, 1, 0] = 10_000                                     # out of range
    plan.idx = bad
    O = lx.lx_attn_bf16(Q, K, V, plan)
    assert lx.lx_last_device_status() == LX_ERR_PLAN
    assert torch.isfinite(O[0, 0, 128:].float()).all()           # other rows still computed
    assert lx.lx_last_device_status() == 0
