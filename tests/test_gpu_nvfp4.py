"""NVFP4 quantiser and block-scaled GEMM (tcgen05 kind::mxf4nvf4) against the
oracle (oracle/nvfp4_ref.py).

"Run Wan2.2-A14B on One RTX 5090: 720p Video in 3.8s", §2: E2M1 values with an
E4M3 scale per 16 elements and an FP32 global scale; FP32 accumulation, BF16
output, column bias fused in the epilogue.

Bars: codes, tiled scales and the global scale bit-exact; a GEMM whose fp32
sums are exact (small power-of-two scales) bit-exact; otherwise
|Y - y| <= 2^-8 |y| + 2^-13 mag, with y the exact result and mag = alpha *
sum_k |x_k w_k| (the accumulation error of an fp32 sum of K/16 block partial
sums is far below 2^-13 of mag; the bf16 rounding is below 2^-8 of |y|)."""
import numpy as np
import pytest
import torch

import oracle
from oracle import nvfp4_ref as nv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lx():
    import video_dit_dynamic_token_b200 as m
    return m


def _bf16(a, dev="cuda"):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).to(dev)


def _check_quant(lx, x_bf16, gscale=None):
    q = lx.lx_nvfp4_quantize(x_bf16, gscale=gscale)
    assert lx.lx_last_device_status() == 0
    xf = x_bf16.float().cpu().numpy()
    ref = nv.quant_nvfp4_ref(xf, None if gscale is None else float(gscale.item()))
    assert q.gscale.item() == float(ref["g"])
    assert np.array_equal(q.codes.cpu().numpy(), nv.pack_e2m1(ref["codes"]))
    assert np.array_equal(q.sf.cpu().numpy(), nv.sf_tiled(ref["sf"]))
    return q, ref


def test_quant_ragged_bit_exact(lx):
    rng = np.random.default_rng(10)
    R, K = 300, 320                       # three row tiles (the last ragged), five k-steps
    x = rng.standard_normal((R, K)) * np.exp(rng.uniform(-6, 6, (R, 1)))
    x[5, 16:32] = 0.0                     # an all-zero block
    x[7] = 0.0                            # an all-zero row
    _check_quant(lx, _bf16(x))


def test_quant_strided_rows(lx):
    rng = np.random.default_rng(11)
    big = _bf16(rng.standard_normal((130, 512)))
    _check_quant(lx, big[:, 128:448])     # row stride 512, K = 320


def test_quant_ties_and_given_scale(lx):
    row = [6, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5, -0.25, -0.75, -1.25, -1.75, -2.5, -3.5, -5, -0.1]
    x = np.tile(np.array(row * 4, np.float32), (3, 1))
    x[1] *= 0.5
    _check_quant(lx, _bf16(x), gscale=torch.ones(1, device="cuda"))


def test_quant_zero_tensor(lx):
    _check_quant(lx, torch.zeros((128, 64), dtype=torch.bfloat16, device="cuda"))


def _nv_from_parts(codes, sf, g, dev="cuda"):
    from video_dit_dynamic_token_b200 import NvFp4Tensor
    R, K = codes.shape
    return NvFp4Tensor(torch.from_numpy(nv.pack_e2m1(codes)).to(dev), torch.from_numpy(nv.sf_tiled(sf)).to(dev),
                       torch.tensor([g], dtype=torch.float32, device=dev), R, K)


@pytest.mark.parametrize("M,N,K", [(200, 384, 512), (128, 256, 256), (1, 128, 768), (517, 640, 1024)])
def test_gemm_exact_sums_bit_exact(lx, M, N, K):
    """Scales in {0.5, 1, 2, 4} and bias on a 1/16 grid make every fp32 sum exact,
    so Y must equal the bf16 rounding of the exact result bit for bit: this pins
    the nibble order, the swizzled k-steps and the scale of every (row, block)."""
    rng = np.random.default_rng(M * 7 + N + K)
    sf_codes = np.array([0x30, 0x38, 0x40, 0x48], np.uint8)
    xc = rng.integers(0, 16, (M, K)).astype(np.uint8)
    wc = rng.integers(0, 16, (N, K)).astype(np.uint8)
    xc[xc == 8] = 0
    wc[wc == 8] = 0
    xs = sf_codes[rng.integers(0, 4, (M, K // 16))]
    ws = sf_codes[rng.integers(0, 4, (N, K // 16))]
    bias = (rng.integers(-512, 512, N) / 16.0).astype(np.float32)
    xq, wq = {"codes": xc, "sf": xs, "g": np.float32(1)}, {"codes": wc, "sf": ws, "g": np.float32(1)}
    ref = nv.gemm_nvfp4_ref(xq, wq, bias)
    y = lx.lx_nvfp4_gemm(_nv_from_parts(xc, xs, 1.0), _nv_from_parts(wc, ws, 1.0),
                         torch.from_numpy(bias).cuda())
    assert lx.lx_last_device_status() == 0
    got = y.float().cpu().numpy().astype(np.float64)
    assert np.array_equal(got, ref["y_bf16"]), f"{np.count_nonzero(got != ref['y_bf16'])} outputs differ"


def _tol(ref):
    return 2.0 ** -8 * np.abs(ref["y"]) + 2.0 ** -13 * ref["mag"] + 1e-30


@pytest.mark.parametrize("M,N,K,with_bias", [(300, 512, 1024, True), (64, 128, 256, False)])
def test_gemm_quantised_random(lx, M, N, K, with_bias):
    rng = np.random.default_rng(M + N + K)
    X = _bf16(rng.standard_normal((M, K)))
    W = _bf16(rng.standard_normal((N, K)) * 0.05)
    bias = torch.from_numpy(rng.standard_normal(N).astype(np.float32)).cuda() if with_bias else None
    xq, xr = _check_quant(lx, X)
    wq, wr = _check_quant(lx, W)
    y = lx.lx_nvfp4_gemm(xq, wq, bias)
    assert lx.lx_last_device_status() == 0
    ref = nv.gemm_nvfp4_ref(xr, wr, None if bias is None else bias.cpu().numpy())
    got = y.float().cpu().numpy()
    assert np.all(np.abs(got - ref["y"]) <= _tol(ref))
    assert oracle.rel_l1_err(torch.from_numpy(got), ref["y"]) <= 4e-3


def test_gemm_output_stride_and_untouched_padding(lx):
    rng = np.random.default_rng(21)
    M, N, K = 130, 256, 512
    X, W = _bf16(rng.standard_normal((M, K))), _bf16(rng.standard_normal((N, K)))
    xq, xr = _check_quant(lx, X)
    wq, wr = _check_quant(lx, W)
    buf = torch.full((M, N + 64), 7.0, dtype=torch.bfloat16, device="cuda")
    lx.lx_nvfp4_gemm(xq, wq, None, out=buf[:, :N])
    assert lx.lx_last_device_status() == 0
    assert torch.all(buf[:, N:] == 7.0)
    ref = nv.gemm_nvfp4_ref(xr, wr)
    assert np.all(np.abs(buf[:, :N].float().cpu().numpy() - ref["y"]) <= _tol(ref))


def test_gemm_qkv_720p_sampled(lx):
    """The 720p fused QKV projection of the 14B model (M = 75600 tokens, K = 5120,
    N = 3 * 5120), in the launch the GEMM benchmark times, checked on sampled
    outputs: the oracle quantises the sampled rows with the global scales of the
    whole tensors."""
    M, N, K = 75600, 15360, 5120
    gen = torch.Generator(device="cuda").manual_seed(5)
    X = torch.randn((M, K), device="cuda", generator=gen).to(torch.bfloat16)
    W = (torch.randn((N, K), device="cuda", generator=gen) * 0.02).to(torch.bfloat16)
    bias = torch.randn(N, device="cuda", generator=gen) * 0.1
    xq = lx.lx_nvfp4_quantize(X)
    wq = lx.lx_nvfp4_quantize(W)
    y = lx.lx_nvfp4_gemm(xq, wq, bias)
    assert lx.lx_last_device_status() == 0
    gx = np.float32(np.float32(X.abs().max().float().item()) / np.float32(2688))
    gw = np.float32(np.float32(W.abs().max().float().item()) / np.float32(2688))
    assert xq.gscale.item() == gx and wq.gscale.item() == gw
    rng = np.random.default_rng(6)
    rows = np.concatenate([rng.choice(M, 14, replace=False), [0, M - 1]])
    cols = np.concatenate([rng.choice(N, 14, replace=False), [0, N - 1]])
    xr = nv.quant_nvfp4_ref(X[torch.from_numpy(rows).cuda()].float().cpu().numpy(), gx)
    wr = nv.quant_nvfp4_ref(W[torch.from_numpy(cols).cuda()].float().cpu().numpy(), gw)
    ref = nv.gemm_nvfp4_ref(xr, wr, bias[torch.from_numpy(cols).cuda()].cpu().numpy())
    got = y[torch.from_numpy(rows).cuda()][:, torch.from_numpy(cols).cuda()].float().cpu().numpy()
    assert np.all(np.abs(got - ref["y"]) <= _tol(ref))
    # the sampled rows' codes are those of the whole-tensor quantisation
    assert np.array_equal(xq.codes[torch.from_numpy(rows).cuda()].cpu().numpy(), nv.pack_e2m1(xr["codes"]))


def test_gemm_rejects_bad_shapes(lx):
    from video_dit_dynamic_token_b200 import LxError
    rng = np.random.default_rng(0)
    xq = lx.lx_nvfp4_quantize(_bf16(rng.standard_normal((64, 320))))
    wq = lx.lx_nvfp4_quantize(_bf16(rng.standard_normal((128, 320))))
    with pytest.raises(LxError):                      # K % 256 != 0
        lx.lx_nvfp4_gemm(xq, wq)
    wq2 = lx.lx_nvfp4_quantize(_bf16(rng.standard_normal((64, 256))))
    xq2 = lx.lx_nvfp4_quantize(_bf16(rng.standard_normal((64, 256))))
    with pytest.raises(LxError):                      # N % 128 != 0
        lx.lx_nvfp4_gemm(xq2, wq2)
