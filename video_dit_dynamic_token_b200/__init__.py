"""Dynamic block-sparse, low-precision self-attention for video DiTs on B200.

Thin Python binding over the C-ABI library ``liblx_sparse_attn.so`` (see
``include/lx_sparse_attn.h``).  Functions carry the C names; they only marshal
arguments: torch allocates device memory and supplies the current stream, and
every step of the computation runs in the library's CUDA kernels.  There is no
CPU fallback -- a missing library raises.

Entry points: the planner (lx_pool_means, lx_score_topk, lx_sparse_attn_plan),
the quantisers (lx_quantize_qk, lx_pool_quantize_qk, lx_quantize_v), the
attention (lx_attn_bf16, lx_attn_int8fp8, lx_sparse_attn_fwd), plan and
forward in one call (lx_sparse_attn), the fused Q/K prologue (lx_rope3d_table,
lx_qk_prologue), K smoothing (lx_k_channel_mean, lx_quantize_qk_smooth,
lx_pool_quantize_qk_smooth), NVFP4 (lx_nvfp4_quantize, lx_nvfp4_gemm); the
host-to-host pipeline is in ``pipeline`` and the Light-Ulysses exchange in
``ulysses``.
"""
from __future__ import annotations

import ctypes
import math
from dataclasses import dataclass

import torch

from . import _abi
from ._abi import LX_BLOCK, LX_MODE_BF16, LX_MODE_INT8FP8, LxBhld, LxPlan  # noqa: F401

MODES = {"bf16": LX_MODE_BF16, "int8fp8": LX_MODE_INT8FP8}


class LxError(RuntimeError):
    def __init__(self, status: int, where: str):
        lib = _abi.load()
        super().__init__(f"{where}: {lib.lx_status_string(status).decode()} (status {status})")
        self.status = status


def _check(status: int, where: str):
    if status != 0:
        raise LxError(status, where)


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def bhld(t: torch.Tensor) -> LxBhld:
    """View of a bf16 [B,H,L,D] CUDA tensor whose last dim is contiguous."""
    if t.dtype != torch.bfloat16 or t.dim() != 4 or t.stride(3) != 1:
        raise ValueError("expected a bf16 [B,H,L,D] tensor with contiguous D")
    B, H, L, D = t.shape
    sB, sH, sL, _ = t.stride()
    return LxBhld(t.data_ptr(), B, H, L, D, sB, sH, sL)


@dataclass
class Plan:
    """Kept-block plan: idx int32 [B,H,nB,k] ascending, mask uint32-bits [B,H,nB,W]."""
    idx: torch.Tensor
    mask: torch.Tensor | None
    B: int
    H: int
    L: int
    nB: int
    k: int

    def c(self) -> LxPlan:
        return LxPlan(self.idx.data_ptr(), self.mask.data_ptr() if self.mask is not None else None,
                      self.B, self.H, self.L, self.nB, self.k, LX_BLOCK)


def lx_plan_size(B, H, L, D, keep):
    lib = _abi.load()
    k = ctypes.c_int64()
    ib, mb, wb = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib.lx_plan_size(B, H, L, D, float(keep), ctypes.byref(k), ctypes.byref(ib), ctypes.byref(mb),
                            ctypes.byref(wb)), "lx_plan_size")
    return k.value, ib.value, mb.value, wb.value


def empty_plan(B, H, L, D, keep, device, with_mask=True) -> Plan:
    k, _, _, _ = lx_plan_size(B, H, L, D, keep)
    nB = (L + LX_BLOCK - 1) // LX_BLOCK
    idx = torch.empty((B, H, nB, k), dtype=torch.int32, device=device)
    mask = torch.empty((B, H, nB, (nB + 31) // 32), dtype=torch.int32, device=device) if with_mask else None
    return Plan(idx, mask, B, H, L, nB, k)


def lx_pool_means(Q, K, out=None, stream=None):
    lib = _abi.load()
    B, H, L, D = Q.shape
    nB = (L + LX_BLOCK - 1) // LX_BLOCK
    if out is None:
        out = (torch.empty((B, H, nB, D), dtype=torch.float32, device=Q.device),
               torch.empty((B, H, nB, D), dtype=torch.float32, device=Q.device))
    q, k = bhld(Q), bhld(K)
    _check(lib.lx_pool_means(ctypes.byref(q), ctypes.byref(k), _ptr(out[0]), _ptr(out[1]), _stream(stream)),
           "lx_pool_means")
    return out


def score_ws_bytes(B, H, nB) -> int:
    """Scratch of lx_score_topk: the fp32 [B,H,nB,ldS] score matrix (ldS = nB
    rounded up to 32), 256-byte rounded."""
    ldS = (nB + 31) // 32 * 32
    return (4 * B * H * nB * ldS + 255) // 256 * 256


def lx_score_topk(mq, mk, L, keep, plan: Plan | None = None, ws=None, stream=None) -> Plan:
    lib = _abi.load()
    B, H, nB, D = mq.shape
    if plan is None:
        plan = empty_plan(B, H, L, D, keep, mq.device)
    if ws is None:
        ws = torch.empty(score_ws_bytes(B, H, nB), dtype=torch.uint8, device=mq.device)
    cp = plan.c()
    _check(lib.lx_score_topk(_ptr(mq), _ptr(mk), B, H, L, D, float(keep), ctypes.byref(cp), _ptr(ws), ws.numel(),
                             _stream(stream)), "lx_score_topk")
    return plan


def lx_sparse_attn_plan(Q, K, keep, plan: Plan | None = None, ws=None, stream=None, with_mask=True) -> Plan:
    lib = _abi.load()
    B, H, L, D = Q.shape
    _, _, _, wb = lx_plan_size(B, H, L, D, keep)
    if plan is None:
        plan = empty_plan(B, H, L, D, keep, Q.device, with_mask)
    if ws is None:
        ws = torch.empty(wb, dtype=torch.uint8, device=Q.device)
    q, k, cp = bhld(Q), bhld(K), plan.c()
    _check(lib.lx_sparse_attn_plan(ctypes.byref(q), ctypes.byref(k), float(keep), ctypes.byref(cp), _ptr(ws),
                                   ws.numel(), _stream(stream)), "lx_sparse_attn_plan")
    return plan


def lx_quantize_qk(Q, K, out=None, stream=None):
    lib = _abi.load()
    B, H, L, D = Q.shape
    nB = (L + LX_BLOCK - 1) // LX_BLOCK
    if out is None:
        dev = Q.device
        out = (torch.empty((B, H, L, D), dtype=torch.int8, device=dev),
               torch.empty((B, H, nB), dtype=torch.float32, device=dev),
               torch.empty((B, H, L, D), dtype=torch.int8, device=dev),
               torch.empty((B, H, nB), dtype=torch.float32, device=dev))
    qc, qs, kc, ks = out
    q, k = bhld(Q), bhld(K)
    _check(lib.lx_quantize_qk(ctypes.byref(q), ctypes.byref(k), _ptr(qc), _ptr(qs), _ptr(kc), _ptr(ks),
                              _stream(stream)), "lx_quantize_qk")
    return out


def lx_pool_quantize_qk(Q, K, out=None, stream=None):
    """Block means and INT8 codes of Q and K in one pass: (mq, mk, qc, qs, kc, ks)."""
    lib = _abi.load()
    B, H, L, D = Q.shape
    nB = (L + LX_BLOCK - 1) // LX_BLOCK
    if out is None:
        dev = Q.device
        out = (torch.empty((B, H, nB, D), dtype=torch.float32, device=dev),
               torch.empty((B, H, nB, D), dtype=torch.float32, device=dev),
               torch.empty((B, H, L, D), dtype=torch.int8, device=dev),
               torch.empty((B, H, nB), dtype=torch.float32, device=dev),
               torch.empty((B, H, L, D), dtype=torch.int8, device=dev),
               torch.empty((B, H, nB), dtype=torch.float32, device=dev))
    mq, mk, qc, qs, kc, ks = out
    q, k = bhld(Q), bhld(K)
    _check(lib.lx_pool_quantize_qk(ctypes.byref(q), ctypes.byref(k), _ptr(mq), _ptr(mk), _ptr(qc), _ptr(qs), _ptr(kc),
                                   _ptr(ks), _stream(stream)), "lx_pool_quantize_qk")
    return out


def rope3d_default_split(D):
    """The default (t, h, w) channel split of a head dimension D."""
    q = D // 6
    return D - 4 * q, 2 * q, 2 * q


def _rope(grid, D, theta, split):
    dt, dh, dw = rope3d_default_split(D) if split is None else split
    T, Hh, W = grid
    return _abi.LxRope3d(T, Hh, W, dt, dh, dw, float(theta))


def lx_rope3d_table(grid, D, theta=10000.0, split=None, device="cuda", stream=None):
    """The (cos, sin) table of the 3D RoPE of a (T, Hh, W) grid, fp32 on the device."""
    lib = _abi.load()
    r = _rope(grid, D, theta, split)
    n = ctypes.c_size_t()
    _check(lib.lx_rope3d_table_size(ctypes.byref(r), D, ctypes.byref(n)), "lx_rope3d_table_size")
    table = torch.empty(max(n.value // 4, 4), dtype=torch.float32, device=device)
    _check(lib.lx_rope3d_table(ctypes.byref(r), D, _ptr(table), _stream(stream)), "lx_rope3d_table")
    return table


def lx_qk_prologue(Q, K, wq, wk, eps, grid, theta=10000.0, split=None, table=None, with_y=True, with_codes=True,
                   stream=None):
    """Per-head RMSNorm + 3D RoPE of Q and K, with the block means and INT8 codes
    of the bf16 result, in one pass: dict(Yq, Yk, mq, mk, qc, qs, kc, ks)."""
    B, H, L, D = Q.shape
    nB = (L + LX_BLOCK - 1) // LX_BLOCK
    dev = Q.device
    if table is None:
        table = lx_rope3d_table(grid, D, theta, split, dev, stream)
    out = {"mq": torch.empty((B, H, nB, D), dtype=torch.float32, device=dev),
           "mk": torch.empty((B, H, nB, D), dtype=torch.float32, device=dev)}
    if with_y:
        out["Yq"] = torch.empty((B, H, L, D), dtype=torch.bfloat16, device=dev)
        out["Yk"] = torch.empty((B, H, L, D), dtype=torch.bfloat16, device=dev)
    if with_codes:
        out["qc"] = torch.empty((B, H, L, D), dtype=torch.int8, device=dev)
        out["qs"] = torch.empty((B, H, nB), dtype=torch.float32, device=dev)
        out["kc"] = torch.empty((B, H, L, D), dtype=torch.int8, device=dev)
        out["ks"] = torch.empty((B, H, nB), dtype=torch.float32, device=dev)
    lx_qk_prologue_into(Q, K, wq, wk, eps, grid, table, out["mq"], out["mk"], out.get("qc"), out.get("qs"),
                        out.get("kc"), out.get("ks"), out.get("Yq"), out.get("Yk"), theta, split, stream)
    return out


def lx_qk_prologue_into(Q, K, wq, wk, eps, grid, table, mq, mk, qc=None, qs=None, kc=None, ks=None, Yq=None, Yk=None,
                        theta=10000.0, split=None, stream=None):
    """lx_qk_prologue into caller buffers (no allocation): means, optional codes
    and optional bf16 outputs."""
    lib = _abi.load()
    D = Q.shape[-1]
    r = _rope(grid, D, theta, split)
    q, k = bhld(Q), bhld(K)
    yq = bhld(Yq) if Yq is not None else None
    yk = bhld(Yk) if Yk is not None else None
    _check(lib.lx_qk_prologue(ctypes.byref(q), ctypes.byref(k), _ptr(wq), _ptr(wk), float(eps), ctypes.byref(r),
                              _ptr(table), ctypes.byref(yq) if yq is not None else None,
                              ctypes.byref(yk) if yk is not None else None, _ptr(mq), _ptr(mk), _ptr(qc), _ptr(qs),
                              _ptr(kc), _ptr(ks), _stream(stream)), "lx_qk_prologue")


def lx_k_channel_mean(K, out=None, ws=None, stream=None):
    """Per-(b, h, channel) mean of K over all tokens (fp64 sums, fp32 result) [B,H,D]."""
    lib = _abi.load()
    B, H, L, D = K.shape
    k = bhld(K)
    if out is None:
        out = torch.empty((B, H, D), dtype=torch.float32, device=K.device)
    if ws is None:
        n = ctypes.c_size_t()
        _check(lib.lx_k_channel_mean_ws_size(ctypes.byref(k), ctypes.byref(n)), "lx_k_channel_mean_ws_size")
        ws = torch.empty(max(n.value, 16), dtype=torch.uint8, device=K.device)
    _check(lib.lx_k_channel_mean(ctypes.byref(k), _ptr(ws), ws.numel(), _ptr(out), _stream(stream)),
           "lx_k_channel_mean")
    return out


def lx_quantize_qk_smooth(Q, K, km=None, out=None, stream=None):
    """INT8 codes of Q and of K minus its channel means: (qc, qs, kc, ks, km)."""
    lib = _abi.load()
    B, H, L, D = Q.shape
    nB = (L + LX_BLOCK - 1) // LX_BLOCK
    if km is None:
        km = lx_k_channel_mean(K, stream=stream)
    if out is None:
        dev = Q.device
        out = (torch.empty((B, H, L, D), dtype=torch.int8, device=dev),
               torch.empty((B, H, nB), dtype=torch.float32, device=dev),
               torch.empty((B, H, L, D), dtype=torch.int8, device=dev),
               torch.empty((B, H, nB), dtype=torch.float32, device=dev))
    qc, qs, kc, ks = out
    q, k = bhld(Q), bhld(K)
    _check(lib.lx_quantize_qk_smooth(ctypes.byref(q), ctypes.byref(k), _ptr(km), _ptr(qc), _ptr(qs), _ptr(kc),
                                     _ptr(ks), _stream(stream)), "lx_quantize_qk_smooth")
    return qc, qs, kc, ks, km


def lx_pool_quantize_qk_smooth(Q, K, km, out, stream=None):
    """Block means of Q and K and INT8 codes of Q and K - km, into out = (mq, mk, qc, qs, kc, ks)."""
    lib = _abi.load()
    mq, mk, qc, qs, kc, ks = out
    q, k = bhld(Q), bhld(K)
    _check(lib.lx_pool_quantize_qk_smooth(ctypes.byref(q), ctypes.byref(k), _ptr(km), _ptr(mq), _ptr(mk), _ptr(qc),
                                          _ptr(qs), _ptr(kc), _ptr(ks), _stream(stream)), "lx_pool_quantize_qk_smooth")
    return out


def lx_quantize_v(V, out=None, amax_ws=None, stream=None):
    lib = _abi.load()
    B, H, L, D = V.shape
    if out is None:
        out = (torch.empty((B, H, L, D), dtype=torch.uint8, device=V.device),
               torch.empty((B, H, D), dtype=torch.float32, device=V.device))
    if amax_ws is None:
        amax_ws = torch.empty((B, H, D), dtype=torch.int32, device=V.device)
    v = bhld(V)
    _check(lib.lx_quantize_v(ctypes.byref(v), _ptr(out[0]), _ptr(out[1]), _ptr(amax_ws), _stream(stream)),
           "lx_quantize_v")
    return out


def lx_quantize_v_noalloc(V, out=None, stream=None):
    lib = _abi.load()
    B, H, L, D = V.shape
    if out is None:
        out = (torch.empty((B, H, L, D), dtype=torch.uint8, device=V.device),
               torch.empty((B, H, D), dtype=torch.float32, device=V.device))
    v = bhld(V)
    _check(lib.lx_quantize_v_noalloc(ctypes.byref(v), _ptr(out[0]), _ptr(out[1]), _stream(stream)),
           "lx_quantize_v_noalloc")
    return out


def lx_attn_bf16(Q, K, V, plan: Plan, out=None, stream=None):
    lib = _abi.load()
    if out is None:
        out = torch.empty_like(Q)
    q, k, v, o, cp = bhld(Q), bhld(K), bhld(V), bhld(out), plan.c()
    _check(lib.lx_attn_bf16(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), ctypes.byref(cp), ctypes.byref(o),
                            _stream(stream)), "lx_attn_bf16")
    return out


def lx_attn_int8fp8(qc, qs, kc, ks, vc, vs, plan: Plan, out=None, stream=None):
    lib = _abi.load()
    if out is None:
        out = torch.empty(qc.shape, dtype=torch.bfloat16, device=qc.device)
    o, cp = bhld(out), plan.c()
    _check(lib.lx_attn_int8fp8(_ptr(qc), _ptr(qs), _ptr(kc), _ptr(ks), _ptr(vc), _ptr(vs), ctypes.byref(cp),
                               ctypes.byref(o), _stream(stream)), "lx_attn_int8fp8")
    return out


def lx_fwd_workspace_size(Q, mode) -> int:
    lib = _abi.load()
    n = ctypes.c_size_t()
    q = bhld(Q)
    _check(lib.lx_fwd_workspace_size(ctypes.byref(q), MODES[mode], ctypes.byref(n)), "lx_fwd_workspace_size")
    return n.value


def lx_sparse_attn_fwd(Q, K, V, plan: Plan, mode="int8fp8", out=None, ws=None, stream=None):
    lib = _abi.load()
    if out is None:
        out = torch.empty_like(Q)
    if ws is None:
        n = lx_fwd_workspace_size(Q, mode)
        ws = torch.empty(max(n, 256), dtype=torch.uint8, device=Q.device)
    q, k, v, o, cp = bhld(Q), bhld(K), bhld(V), bhld(out), plan.c()
    _check(lib.lx_sparse_attn_fwd(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), ctypes.byref(cp), MODES[mode],
                                  ctypes.byref(o), _ptr(ws), ws.numel(), _stream(stream)), "lx_sparse_attn_fwd")
    return out


def lx_sparse_attn_ws_size(Q, keep, mode="int8fp8") -> int:
    lib = _abi.load()
    n = ctypes.c_size_t()
    q = bhld(Q)
    _check(lib.lx_sparse_attn_ws_size(ctypes.byref(q), float(keep), MODES[mode], ctypes.byref(n)),
           "lx_sparse_attn_ws_size")
    return n.value


def lx_sparse_attn(Q, K, V, keep, mode="int8fp8", plan: Plan | None = None, out=None, ws=None, stream=None):
    """Plan and forward in one call (Q and K read once for means and codes): (O, plan)."""
    lib = _abi.load()
    B, H, L, D = Q.shape
    if plan is None:
        plan = empty_plan(B, H, L, D, keep, Q.device)
    if out is None:
        out = torch.empty_like(Q)
    if ws is None:
        ws = torch.empty(max(lx_sparse_attn_ws_size(Q, keep, mode), 256), dtype=torch.uint8, device=Q.device)
    q, k, v, o, cp = bhld(Q), bhld(K), bhld(V), bhld(out), plan.c()
    _check(lib.lx_sparse_attn(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), float(keep), MODES[mode],
                              ctypes.byref(cp), ctypes.byref(o), _ptr(ws), ws.numel(), _stream(stream)),
           "lx_sparse_attn")
    return out, plan



# ---------------------------------------------------------------- NVFP4
@dataclass
class NvFp4Tensor:
    """An NVFP4 tensor [R, K] in the layouts of lx_nvfp4_quantize: codes uint8
    [R, K/2], tiled E4M3 scales (uint8, rows padded to 128), fp32 global scale [1]."""
    codes: torch.Tensor
    sf: torch.Tensor
    gscale: torch.Tensor
    R: int
    K: int


def lx_nvfp4_sizes(R, K):
    cb, sb = ctypes.c_size_t(), ctypes.c_size_t()
    _check(_abi.load().lx_nvfp4_sizes(int(R), int(K), ctypes.byref(cb), ctypes.byref(sb)), "lx_nvfp4_sizes")
    return cb.value, sb.value


def lx_nvfp4_quantize(x, gscale=None, out: NvFp4Tensor | None = None, stream=None) -> NvFp4Tensor:
    """x: bf16 [R, K] CUDA tensor with contiguous rows.  gscale None: the global
    scale is computed from x; else a CUDA fp32 tensor of one element used as given."""
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("expected a bf16 [R, K] tensor with contiguous rows")
    R, K = x.shape
    if out is None:
        cb, sb = lx_nvfp4_sizes(R, K)
        g = torch.empty(1, dtype=torch.float32, device=x.device)
        out = NvFp4Tensor(torch.empty((R, K // 2), dtype=torch.uint8, device=x.device),
                          torch.empty(sb, dtype=torch.uint8, device=x.device), g, R, K)
    compute = gscale is None
    if not compute:
        out.gscale.copy_(gscale.reshape(1))
    _check(_abi.load().lx_nvfp4_quantize(_ptr(x), R, K, x.stride(0), int(compute), _ptr(out.gscale), _ptr(out.codes),
                                         _ptr(out.sf), _stream(stream)), "lx_nvfp4_quantize")
    return out


def lx_nvfp4_gemm(xq: NvFp4Tensor, wq: NvFp4Tensor, bias=None, out=None, stream=None):
    """Y = X W^T + bias in bf16 [M, N] from NVFP4 X [M, K] and W [N, K]; bias fp32 [N] or None."""
    if xq.K != wq.K:
        raise ValueError("X and W differ in K")
    M, N, K = xq.R, wq.R, xq.K
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=xq.codes.device)
    if bias is not None and (bias.dtype != torch.float32 or not bias.is_contiguous()):
        raise ValueError("bias must be a contiguous fp32 tensor")
    _check(_abi.load().lx_nvfp4_gemm(_ptr(xq.codes), _ptr(xq.sf), _ptr(xq.gscale), _ptr(wq.codes), _ptr(wq.sf),
                                     _ptr(wq.gscale), _ptr(bias), M, N, K, _ptr(out), out.stride(0), _stream(stream)),
           "lx_nvfp4_gemm")
    return out


def nvfp4_gemm_flops(M, N, K) -> float:
    return 2.0 * M * N * K


def lx_last_device_status(stream=None) -> int:
    return _abi.load().lx_last_device_status(_stream(stream))


def lx_debug_wait_timeout(limit_ns: int, stream=None):
    _check(_abi.load().lx_debug_wait_timeout(int(limit_ns), _stream(stream)), "lx_debug_wait_timeout")


def keep_count(nB: int, keep: float) -> int:
    """k for a plan, from the library's own size query (nB blocks of 64)."""
    return lx_plan_size(1, 1, nB * LX_BLOCK, 64, keep)[0]


def effective_flops(B, H, L, D, keep) -> float:
    """4 L^2 D H B * k/nB: the attention work on the kept tiles only."""
    nB = math.ceil(L / LX_BLOCK)
    k = keep_count(nB, keep)
    return 4.0 * L * L * D * H * B * k / nB
