"""lx_quantize_v_noalloc: the V quantiser with its built-in scratch gives the same
codes and scales as lx_quantize_v with a caller buffer, call after call."""
import numpy as np
import pytest
import torch

import video_dit_dynamic_token_b200 as lx
from video_dit_dynamic_token_b200 import _abi, synth
from gpu_util import to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("B,H,L,d,scale", [(1, 3, 1000, 128, 3.0), (2, 2, 1024, 64, 0.5), (1, 40, 3000, 128, 20.0)])
def test_noalloc_matches_caller_scratch_twice(B, H, L, d, scale):
    _, _, V = synth.random_qkv(B, H, L, d, seed=L + 7, scale=scale, device=DEV)
    want_c, want_s = lx.lx_quantize_v(V)
    torch.cuda.synchronize()
    # two calls in a row: the second must not see the first one's absmax words
    for _ in range(2):
        got_c, got_s = lx.lx_quantize_v_noalloc(V)
        torch.cuda.synchronize()
        assert np.array_equal(to_np(got_c), to_np(want_c))
        assert np.array_equal(to_np(got_s), to_np(want_s))


def test_noalloc_after_larger_values_then_smaller():
    # a large-valued tensor followed by a small-valued one of the same shape: stale
    # absmax words from the first call would inflate the second call's scales
    _, _, Vbig = synth.random_qkv(1, 2, 500, 128, seed=3, scale=100.0, device=DEV)
    _, _, Vsmall = synth.random_qkv(1, 2, 500, 128, seed=4, scale=0.01, device=DEV)
    lx.lx_quantize_v_noalloc(Vbig)
    got_c, got_s = lx.lx_quantize_v_noalloc(Vsmall)
    want_c, want_s = lx.lx_quantize_v(Vsmall)
    torch.cuda.synchronize()
    assert np.array_equal(to_np(got_c), to_np(want_c))
    assert np.array_equal(to_np(got_s), to_np(want_s))


def test_noalloc_rejects_oversize():
    # B*H*D one head past the limit: rejected on the host, nothing launched
    d = 128
    H = _abi.LX_NOALLOC_AMAX_MAX // d + 1
    V = torch.zeros((1, H, 64, d), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(RuntimeError, match="workspace"):
        lx.lx_quantize_v_noalloc(V)
    torch.cuda.synchronize()
