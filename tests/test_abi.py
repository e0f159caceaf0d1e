"""Host-side checks of the C-ABI library (no GPU needed, no compute calls).

The shared library must load, export every entry point the header declares,
and reject bad arguments on the host before anything is launched.
"""
import ctypes
import os
import re

import pytest

import oracle
from video_dit_dynamic_token_b200 import _abi, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _abi.load()


def _declared():
    names = []
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            src = open(os.path.join(ROOT, "include", f), encoding="utf-8").read()
            names += re.findall(r"^(?:lx_status|const char\*)\s+(lx_\w+)\(", src, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(_abi.SIGNATURES) == names


def test_status_strings(lib):
    for code in range(-7, 1):
        assert lib.lx_status_string(code)
    assert lib.lx_status_string(-6) == b"device wait timed out"


def _plan_size(lib, B, H, L, D, keep):
    k = ctypes.c_int64()
    a, b, c = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    st = lib.lx_plan_size(B, H, L, D, keep, ctypes.byref(k), ctypes.byref(a), ctypes.byref(b), ctypes.byref(c))
    return st, k.value, a.value, b.value, c.value


@pytest.mark.parametrize("L,keep", [(1024, 0.25), (32760, 0.2), (75600, 0.1), (120960, 0.1), (6400, 0.55),
                                    (21760, 0.55), (1, 0.3), (65, 1.0), (75600, 0.05), (75600, 0.5)])
def test_plan_size_matches_oracle_k(lib, L, keep):
    st, k, ib, mb, wb = _plan_size(lib, 1, 40, L, 128, keep)
    nB = oracle.n_blocks(L)
    assert st == 0
    assert k == oracle.keep_count(nB, keep)
    assert ib == 4 * 40 * nB * k
    assert mb == 4 * 40 * nB * ((nB + 31) // 32)
    # two fp32 block-mean arrays, then the fp32 scores with rows padded to 32 floats
    a256 = lambda n: (n + 255) // 256 * 256
    assert wb == 2 * a256(4 * 40 * nB * 128) + a256(4 * 40 * nB * ((nB + 31) // 32 * 32))


def test_plan_size_rejects(lib):
    assert _plan_size(lib, 1, 1, 100, 128, 0.0)[0] == _abi.LX_ERR_INVALID
    assert _plan_size(lib, 1, 1, 100, 128, 1.5)[0] == _abi.LX_ERR_INVALID
    assert _plan_size(lib, 0, 1, 100, 128, 0.5)[0] == _abi.LX_ERR_INVALID
    assert _plan_size(lib, 1, 1, 100, 96, 0.5)[0] == _abi.LX_ERR_UNSUPPORTED


def _view(ptr=0x10000, B=1, H=2, L=1000, D=128, sL=None):
    sL = D if sL is None else sL
    return _abi.LxBhld(ptr, B, H, L, D, H * L * sL, L * sL, sL)


def test_host_argument_errors_before_launch(lib):
    q = _view()
    s = ctypes.c_void_p(0)
    # misaligned pointer, bad stride, unsupported D, shape mismatch: all rejected on the host
    bad_ptr = _view(ptr=0x10008)
    assert lib.lx_pool_means(ctypes.byref(bad_ptr), ctypes.byref(q), 0x20000, 0x30000, s) == _abi.LX_ERR_ALIGN
    odd_stride = _view(sL=132)
    assert lib.lx_pool_means(ctypes.byref(odd_stride), ctypes.byref(odd_stride), 0x20000, 0x30000, s) == _abi.LX_ERR_ALIGN
    d96 = _view(D=96)
    assert lib.lx_pool_means(ctypes.byref(d96), ctypes.byref(d96), 0x20000, 0x30000, s) == _abi.LX_ERR_UNSUPPORTED
    other = _view(L=999)
    assert lib.lx_pool_means(ctypes.byref(q), ctypes.byref(other), 0x20000, 0x30000, s) == _abi.LX_ERR_INVALID
    assert lib.lx_pool_means(None, ctypes.byref(q), 0x20000, 0x30000, s) == _abi.LX_ERR_INVALID
    # the fused means + codes pass: every output required, each 16-byte aligned
    outs = [0x20000, 0x30000, 0x40000, 0x50000, 0x60000, 0x70000]
    for i in range(6):
        missing = list(outs)
        missing[i] = None
        assert lib.lx_pool_quantize_qk(ctypes.byref(q), ctypes.byref(q), *missing, s) == _abi.LX_ERR_INVALID
        odd = list(outs)
        odd[i] += 8
        assert lib.lx_pool_quantize_qk(ctypes.byref(q), ctypes.byref(q), *odd, s) == _abi.LX_ERR_ALIGN
    assert lib.lx_pool_quantize_qk(ctypes.byref(d96), ctypes.byref(d96), *outs, s) == _abi.LX_ERR_UNSUPPORTED
    # planner without enough workspace
    plan = _abi.LxPlan(0x40000, 0, 0, 0, 0, 0, 0, 0)
    assert lib.lx_sparse_attn_plan(ctypes.byref(q), ctypes.byref(q), 0.25, ctypes.byref(plan), 0x50000, 16, s) \
        == _abi.LX_ERR_WORKSPACE
    # planner beyond the selection kernel's row limit
    huge = _view(L=64 * 2177, H=1)
    _, _, _, _, wb = _plan_size(lib, 1, 1, 64 * 2177, 128, 0.1)
    assert lib.lx_sparse_attn_plan(ctypes.byref(huge), ctypes.byref(huge), 0.1, ctypes.byref(plan), 0x50000, wb, s) \
        == _abi.LX_ERR_UNSUPPORTED


def test_fwd_plan_and_workspace_checks(lib):
    q = _view()
    s = ctypes.c_void_p(0)
    nB = oracle.n_blocks(1000)
    good = _abi.LxPlan(0x40000, 0, 1, 2, 1000, nB, 4, 64)
    need = ctypes.c_size_t()
    assert lib.lx_fwd_workspace_size(ctypes.byref(q), _abi.LX_MODE_INT8FP8, ctypes.byref(need)) == 0
    assert need.value >= 3 * 2 * 1000 * 128
    assert lib.lx_fwd_workspace_size(ctypes.byref(q), _abi.LX_MODE_BF16, ctypes.byref(need)) == 0 and need.value == 0
    assert lib.lx_sparse_attn_fwd(ctypes.byref(q), ctypes.byref(q), ctypes.byref(q), ctypes.byref(good),
                                  _abi.LX_MODE_INT8FP8, ctypes.byref(q), 0x100000, 64, s) == _abi.LX_ERR_WORKSPACE
    for bad in (_abi.LxPlan(0x40000, 0, 1, 2, 1000, nB + 1, 4, 64),   # wrong nB
                _abi.LxPlan(0x40000, 0, 1, 2, 1000, nB, 0, 64),        # k = 0
                _abi.LxPlan(0x40000, 0, 1, 2, 1000, nB, nB + 1, 64),   # k > nB
                _abi.LxPlan(0x40000, 0, 1, 3, 1000, nB, 4, 64),        # wrong H
                _abi.LxPlan(0, 0, 1, 2, 1000, nB, 4, 64),              # no idx
                _abi.LxPlan(0x40000, 0, 1, 2, 1000, nB, 4, 32)):       # wrong block
        assert lib.lx_attn_bf16(ctypes.byref(q), ctypes.byref(q), ctypes.byref(q), ctypes.byref(bad),
                                ctypes.byref(q), s) == _abi.LX_ERR_INVALID
    assert lib.lx_sparse_attn_fwd(ctypes.byref(q), ctypes.byref(q), ctypes.byref(q), ctypes.byref(good), 7,
                                  ctypes.byref(q), 0x100000, 1 << 30, s) == _abi.LX_ERR_INVALID
    assert lib.lx_debug_wait_timeout(0, s) == _abi.LX_ERR_INVALID


def test_prologue_argument_errors_before_launch(lib):
    s = ctypes.c_void_p(0)
    q = _view(L=1000)
    good = _abi.LxRope3d(4, 16, 16, 44, 42, 42, 10000.0)
    n = ctypes.c_size_t()
    assert lib.lx_rope3d_table_size(ctypes.byref(good), 128, ctypes.byref(n)) == 0
    assert n.value == 8 * (4 * 22 + 16 * 21 + 16 * 21)
    for bad in (_abi.LxRope3d(4, 16, 16, 43, 43, 42, 10000.0),     # odd parts
                _abi.LxRope3d(4, 16, 16, 44, 42, 40, 10000.0),     # parts do not add up to D
                _abi.LxRope3d(4, 16, 16, 44, 42, 42, 0.0),         # theta
                _abi.LxRope3d(0, 16, 16, 44, 42, 42, 10000.0)):    # empty grid
        assert lib.lx_rope3d_table_size(ctypes.byref(bad), 128, ctypes.byref(n)) == _abi.LX_ERR_INVALID
    assert lib.lx_rope3d_table(ctypes.byref(good), 128, 0x20008, s) == _abi.LX_ERR_ALIGN
    p = [0x20000, 0x30000, 0x40000, 0x50000, 0x60000, 0x70000]   # mq mk qc qs kc ks
    call = lambda rope=good, yq=None, yk=None, outs=p, eps=1e-6, X=q: lib.lx_qk_prologue(
        ctypes.byref(X), ctypes.byref(X), 0x80000, 0x90000, eps, ctypes.byref(rope), 0xA0000,
        ctypes.byref(yq) if yq is not None else None, ctypes.byref(yk) if yk is not None else None, *outs, s)
    small = _abi.LxRope3d(3, 16, 16, 44, 42, 42, 10000.0)         # 768 positions < L = 1000
    assert call(rope=small) == _abi.LX_ERR_INVALID
    assert call(eps=-1.0) == _abi.LX_ERR_INVALID
    assert call(yq=q) == _abi.LX_ERR_INVALID                        # one output without the other
    assert call(outs=[0x20000, 0x30000, 0x40000, None, 0x60000, 0x70000]) == _abi.LX_ERR_INVALID
    assert call(outs=[None, 0x30000, 0x40000, 0x50000, 0x60000, 0x70000]) == _abi.LX_ERR_INVALID
    assert call(outs=[0x20008, 0x30000, 0x40000, 0x50000, 0x60000, 0x70000]) == _abi.LX_ERR_ALIGN


def test_smoothing_argument_errors_before_launch(lib):
    s = ctypes.c_void_p(0)
    k = _view(L=1000, H=2)
    n = ctypes.c_size_t()
    assert lib.lx_k_channel_mean_ws_size(ctypes.byref(k), ctypes.byref(n)) == 0
    assert n.value == 8 * 1 * 2 * 2 * 128            # ceil(1000 / 512) = 2 spans
    assert lib.lx_k_channel_mean(ctypes.byref(k), 0x20000, n.value - 8, 0x30000, s) == _abi.LX_ERR_WORKSPACE
    assert lib.lx_k_channel_mean(ctypes.byref(k), 0x20008, n.value, 0x30000, s) == _abi.LX_ERR_ALIGN
    assert lib.lx_k_channel_mean(ctypes.byref(k), 0x20000, n.value, None, s) == _abi.LX_ERR_INVALID
    outs = [0x40000, 0x50000, 0x60000, 0x70000]
    assert lib.lx_quantize_qk_smooth(ctypes.byref(k), ctypes.byref(k), None, *outs, s) == _abi.LX_ERR_INVALID
    assert lib.lx_quantize_qk_smooth(ctypes.byref(k), ctypes.byref(k), 0x30008, *outs, s) == _abi.LX_ERR_ALIGN
    other = _view(L=999, H=2)
    assert lib.lx_quantize_qk_smooth(ctypes.byref(k), ctypes.byref(other), 0x30000, *outs, s) == _abi.LX_ERR_INVALID


def test_nvfp4_sizes_and_argument_errors_before_launch(lib):
    s = ctypes.c_void_p(0)
    cb, sb = ctypes.c_size_t(), ctypes.c_size_t()
    assert lib.lx_nvfp4_sizes(300, 320, ctypes.byref(cb), ctypes.byref(sb)) == 0
    assert cb.value == 300 * 160
    assert sb.value == oracle.sf_tiled(__import__("numpy").zeros((300, 20), "uint8")).size   # 3 tiles x 5 k-steps x 512
    assert lib.lx_nvfp4_sizes(10, 96, ctypes.byref(cb), ctypes.byref(sb)) == _abi.LX_ERR_INVALID   # K % 64
    assert lib.lx_nvfp4_sizes(0, 64, ctypes.byref(cb), ctypes.byref(sb)) == _abi.LX_ERR_INVALID
    x, g, c, f = 0x10000, 0x20000, 0x30000, 0x40000
    assert lib.lx_nvfp4_quantize(x, 10, 128, 100, 1, g, c, f, s) == _abi.LX_ERR_INVALID          # ldx < K
    assert lib.lx_nvfp4_quantize(x, 10, 128, 132, 1, g, c, f, s) == _abi.LX_ERR_ALIGN            # ldx % 8
    assert lib.lx_nvfp4_quantize(x + 8, 10, 128, 128, 1, g, c, f, s) == _abi.LX_ERR_ALIGN
    assert lib.lx_nvfp4_quantize(None, 10, 128, 128, 1, g, c, f, s) == _abi.LX_ERR_INVALID
    args = (c, f, g, c, f, g, None)
    assert lib.lx_nvfp4_gemm(*args, 100, 256, 320, x, 256, s) == _abi.LX_ERR_INVALID             # K % 256
    assert lib.lx_nvfp4_gemm(*args, 100, 192, 256, x, 192, s) == _abi.LX_ERR_INVALID             # N % 128
    assert lib.lx_nvfp4_gemm(*args, 100, 256, 256, x, 200, s) == _abi.LX_ERR_INVALID             # ldy < N
    assert lib.lx_nvfp4_gemm(*args, 100, 256, 256, x, 260, s) == _abi.LX_ERR_ALIGN               # ldy % 8
    assert lib.lx_nvfp4_gemm(c, f, g + 2, c, f, g, None, 100, 256, 256, x, 256, s) == _abi.LX_ERR_ALIGN
    assert lib.lx_nvfp4_gemm(c, None, g, c, f, g, None, 100, 256, 256, x, 256, s) == _abi.LX_ERR_INVALID
    assert lib.lx_nvfp4_gemm(*args, 1 << 31, 256, 256, x, 256, s) == _abi.LX_ERR_UNSUPPORTED       # 32-bit rows
