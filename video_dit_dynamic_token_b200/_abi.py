"""ctypes declarations of the C-ABI in include/lx_sparse_attn.h (marshalling only)."""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "liblx_sparse_attn.so")

LX_OK = 0
LX_ERR_INVALID = -1
LX_ERR_UNSUPPORTED = -2
LX_ERR_ALIGN = -3
LX_ERR_WORKSPACE = -4
LX_ERR_CUDA = -5
LX_ERR_TIMEOUT = -6
LX_ERR_PLAN = -7
LX_MODE_BF16 = 0
LX_MODE_INT8FP8 = 1
LX_BLOCK = 64
LX_NOALLOC_AMAX_MAX = 65536

# every entry point the header declares, with its ctypes signature
_c_i64, _c_sz, _vp, _dbl, _u64 = ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_double, ctypes.c_uint64


class LxBhld(ctypes.Structure):
    _fields_ = [("data", _vp), ("B", _c_i64), ("H", _c_i64), ("L", _c_i64), ("D", _c_i64),
                ("sB", _c_i64), ("sH", _c_i64), ("sL", _c_i64)]


class LxPlan(ctypes.Structure):
    _fields_ = [("idx", _vp), ("mask", _vp), ("B", _c_i64), ("H", _c_i64), ("L", _c_i64),
                ("nB", _c_i64), ("k", _c_i64), ("block", ctypes.c_int32)]


class LxRope3d(ctypes.Structure):
    _fields_ = [("T", _c_i64), ("Hh", _c_i64), ("W", _c_i64), ("dt", ctypes.c_int32), ("dh", ctypes.c_int32),
                ("dw", ctypes.c_int32), ("theta", _dbl)]


_P = ctypes.POINTER
SIGNATURES = {
    "lx_plan_size": [_c_i64, _c_i64, _c_i64, _c_i64, _dbl, _P(_c_i64), _P(_c_sz), _P(_c_sz), _P(_c_sz)],
    "lx_pool_means": [_P(LxBhld), _P(LxBhld), _vp, _vp, _vp],
    "lx_score_topk": [_vp, _vp, _c_i64, _c_i64, _c_i64, _c_i64, _dbl, _P(LxPlan), _vp, _c_sz, _vp],
    "lx_sparse_attn_plan": [_P(LxBhld), _P(LxBhld), _dbl, _P(LxPlan), _vp, _c_sz, _vp],
    "lx_quantize_qk": [_P(LxBhld), _P(LxBhld), _vp, _vp, _vp, _vp, _vp],
    "lx_pool_quantize_qk": [_P(LxBhld), _P(LxBhld), _vp, _vp, _vp, _vp, _vp, _vp, _vp],
    "lx_rope3d_table_size": [_P(LxRope3d), _c_i64, _P(_c_sz)],
    "lx_rope3d_table": [_P(LxRope3d), _c_i64, _vp, _vp],
    "lx_qk_prologue": [_P(LxBhld), _P(LxBhld), _vp, _vp, ctypes.c_float, _P(LxRope3d), _vp, _P(LxBhld), _P(LxBhld),
                       _vp, _vp, _vp, _vp, _vp, _vp, _vp],
    "lx_k_channel_mean_ws_size": [_P(LxBhld), _P(_c_sz)],
    "lx_k_channel_mean": [_P(LxBhld), _vp, _c_sz, _vp, _vp],
    "lx_quantize_qk_smooth": [_P(LxBhld), _P(LxBhld), _vp, _vp, _vp, _vp, _vp, _vp],
    "lx_pool_quantize_qk_smooth": [_P(LxBhld), _P(LxBhld), _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp],
    "lx_quantize_v": [_P(LxBhld), _vp, _vp, _vp, _vp],
    "lx_quantize_v_noalloc": [_P(LxBhld), _vp, _vp, _vp],
    "lx_attn_bf16": [_P(LxBhld), _P(LxBhld), _P(LxBhld), _P(LxPlan), _P(LxBhld), _vp],
    "lx_attn_int8fp8": [_vp, _vp, _vp, _vp, _vp, _vp, _P(LxPlan), _P(LxBhld), _vp],
    "lx_fwd_workspace_size": [_P(LxBhld), ctypes.c_int, _P(_c_sz)],
    "lx_sparse_attn_fwd": [_P(LxBhld), _P(LxBhld), _P(LxBhld), _P(LxPlan), ctypes.c_int, _P(LxBhld), _vp, _c_sz, _vp],
    "lx_sparse_attn_ws_size": [_P(LxBhld), _dbl, ctypes.c_int, _P(_c_sz)],
    "lx_sparse_attn": [_P(LxBhld), _P(LxBhld), _P(LxBhld), _dbl, ctypes.c_int, _P(LxPlan), _P(LxBhld), _vp, _c_sz, _vp],
    "lx_ulysses_segment_bytes": [_c_i64, _c_i64, _c_i64, _c_i64, _c_i64, _P(_c_sz)],
    "lx_ulysses_pack_qkv": [_P(LxBhld), _P(LxBhld), _P(LxBhld), _c_i64, _c_i64, _c_i64, _vp, _vp],
    "lx_ulysses_unpack_qkv": [_vp, _c_i64, _P(LxBhld), _P(LxBhld), _P(LxBhld), _vp],
    "lx_ulysses_pack_o": [_P(LxBhld), _c_i64, _vp, _vp],
    "lx_ulysses_unpack_o": [_vp, _c_i64, _c_i64, _c_i64, _P(LxBhld), _vp],
    "lx_nvfp4_sizes": [_c_i64, _c_i64, _P(_c_sz), _P(_c_sz)],
    "lx_nvfp4_quantize": [_vp, _c_i64, _c_i64, _c_i64, ctypes.c_int, _vp, _vp, _vp, _vp],
    "lx_nvfp4_gemm": [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_i64, _c_i64, _c_i64, _vp, _c_i64, _vp],
    "lx_last_device_status": [_vp],
    "lx_debug_wait_timeout": [_u64, _vp],
    "lx_status_string": [ctypes.c_int],
}

_lib = None


def load(path: str = LIB_PATH):
    """Load the CUDA library; raises (no fallback exists) when it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"CUDA library {path} is missing; build it with "
                          "`python -m video_dit_dynamic_token_b200.build`")
    lib = ctypes.CDLL(path)
    for name, args in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_char_p if name == "lx_status_string" else ctypes.c_int
    _lib = lib
    return lib
