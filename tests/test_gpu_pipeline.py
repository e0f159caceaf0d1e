"""HostPipeline: chunked host->device->host processing gives exactly the output
of one device-side plan + forward over all heads (heads are independent)."""
import pytest
import torch

import video_dit_dynamic_token_b200 as lx
from video_dit_dynamic_token_b200 import synth
from video_dit_dynamic_token_b200.pipeline import HostPipeline

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("mode", ["int8fp8", "bf16"])
@pytest.mark.parametrize("H,hc", [(5, 2), (4, 4), (3, 1)])
def test_pipeline_matches_device_call(mode, H, hc):
    B, L, d, keep = 1, 1000, 128, 0.25
    Q, K, V = synth.random_qkv(B, H, L, d, seed=H * 10 + hc, device=DEV)
    plan = lx.lx_sparse_attn_plan(Q, K, keep)
    want = lx.lx_sparse_attn_fwd(Q, K, V, plan, mode)
    torch.cuda.synchronize()
    hQ, hK, hV = (x.cpu().pin_memory() for x in (Q, K, V))
    hO = torch.empty(Q.shape, dtype=Q.dtype).pin_memory()
    pipe = HostPipeline(B, H, L, d, keep, mode, heads_per_chunk=hc, device=DEV)
    for _ in range(2):  # twice: the slots are reused across runs
        hO.zero_()
        pipe.run(hQ, hK, hV, hO)
        torch.cuda.synchronize()
        assert lx.lx_last_device_status() == 0
        assert torch.equal(hO, want.cpu())
