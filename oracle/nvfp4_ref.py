"""CPU oracle for NVFP4 quantisation and the dual-NVFP4 block-scaled GEMM
(plain numpy, fp64 unless a step says fp32).

TEST INFRASTRUCTURE ONLY, like ``sparse_attn_ref``: only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg use it; it
shares no code with the CUDA library.

What the pages fix ("Run Wan2.2-A14B on One RTX 5090: 720p Video in 3.8s",
§2 "NVFP4 quantization-aware training"; "600倍加速，720p视频实时生成！单卡也能带
的动14B模型", §NVFP4量化感知训练 and §高效推理算子): an NVFP4 tensor holds E2M1
4-bit values, one FP8 E4M3 scale shared by each 16 consecutive elements, and
one FP32 scale for the whole tensor; the linear layers multiply NVFP4
activations by NVFP4 weights with FP32 accumulation and BF16 output, the column
bias added in the same kernel.  How the scales are chosen is not given; this
library's reading (the usual NVFP4 recipe, made exact in fp32 so that two
implementations agree bit for bit):
  * g   = fl32(amax / 2688) (2688 = 448 * 6: the largest E4M3 scale times the
          largest E2M1 value), g = 1 for an all-zero tensor;
  * ig6 = fl32(1 / fl32(6 * g));
  * per block of 16 along K: s = E4M3_rn_satfinite(fl32(amax_block * ig6));
  * inv = fl32(1 / fl32(s * g)) (0 when s = 0);
  * code = E2M1_rn_satfinite(fl32(x * inv)), ties to the even mantissa, and a
    value that rounds to zero is +0 (code 0) whatever its sign;
  * value = e2m1(code) * e4m3(s) * g.
The GEMM: Y[m, n] = bf16(fl32(acc[m, n] * fl32(g_x * g_w)) + bias[n]) with
acc = sum_k e2m1(a) e4m3(s_a) e2m1(w) e4m3(s_w) (exact here, fp32 on the GPU).

Pins live in ``tests/test_oracle_nvfp4.py``.
"""
from __future__ import annotations

import numpy as np

from .prologue_ref import bf16_round
from .sparse_attn_ref import E4M3_MAX, _f32, e4m3_decode, e4m3_encode, e4m3_round

E2M1_MAX = 6.0
NVFP4_BLOCK = 16            # elements per E4M3 scale
NVFP4_GS_DIV = E4M3_MAX * E2M1_MAX   # 2688


def e2m1_decode(codes) -> np.ndarray:
    """Value of 4-bit E2M1 codes from the bit fields: sign bit 3, exponent bits
    2..1 (bias 1), mantissa bit 0; exponent 0 is subnormal (m * 0.5)."""
    c = np.asarray(codes, dtype=np.int64) & 0xF
    s = np.where(c & 0x8, -1.0, 1.0)
    e = (c >> 1) & 0x3
    m = c & 0x1
    mag = np.where(e == 0, 0.5 * m, (1.0 + 0.5 * m) * np.ldexp(1.0, e - 1))
    return s * mag


def e2m1_round(y) -> np.ndarray:
    """Nearest E2M1 value of y, ties to the even mantissa, saturating at +-6.
    Within a binade of E2M1 the spacing is 0.5 below 2, 1 in [2, 4), 2 in [4, 6];
    rint on the exact quotient gives round-half-even (the mantissa is the
    parity of the quotient)."""
    y = np.asarray(y, dtype=np.float64)
    a = np.abs(y)
    step = np.where(a < 2.0, 0.5, np.where(a < 4.0, 1.0, 2.0))
    q = np.rint(a / step) * step
    q = np.minimum(q, E2M1_MAX)
    return np.copysign(q, y)


def e2m1_encode(v) -> np.ndarray:
    """4-bit codes (uint8) of E2M1 values already on the grid; zero is +0."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    e = np.where(a < 1.0, 0, np.floor(np.log2(np.maximum(a, 1.0))).astype(np.int64) + 1)
    m = np.where(e == 0, np.rint(a / 0.5), np.rint((a / np.ldexp(1.0, e - 1) - 1.0) * 2.0)).astype(np.int64)
    mag = (e << 1) | m
    sign = ((v < 0) & (mag != 0)).astype(np.int64) << 3
    return (mag | sign).astype(np.uint8)


def nvfp4_global_scale(X) -> np.float32:
    """g = fl32(amax / 2688), 1 for an all-zero tensor."""
    a = np.float32(np.abs(_f32(X)).max()) if np.asarray(X).size else np.float32(0)
    return np.float32(a / np.float32(NVFP4_GS_DIV)) if a > 0 else np.float32(1)


def quant_nvfp4_ref(X, g=None) -> dict:
    """NVFP4 codes of X [R, K] (K a multiple of 16), with the global scale g
    (computed from X when None).  Returns codes (uint8 [R, K], one 4-bit code
    each), sf (uint8 [R, K/16] E4M3 bit patterns) and g (fp32)."""
    x = _f32(X)
    R, K = x.shape
    if K % NVFP4_BLOCK:
        raise ValueError("K must be a multiple of 16")
    g = nvfp4_global_scale(x) if g is None else np.float32(g)
    ig6 = np.float32(np.float32(1) / np.float32(np.float32(6) * g))
    xb = x.reshape(R, K // NVFP4_BLOCK, NVFP4_BLOCK)
    amax_b = np.abs(xb).max(axis=-1).astype(np.float32)
    t = (amax_b * ig6).astype(np.float32)
    s = e4m3_round(t).astype(np.float32)                          # exact: E4M3 values are fp32 values
    sg = (s * g).astype(np.float32)
    nz = s > 0
    inv = np.where(nz, np.float32(1) / np.where(nz, sg, np.float32(1)), np.float32(0)).astype(np.float32)
    y = (xb * inv[..., None]).astype(np.float32)
    codes = e2m1_encode(e2m1_round(y)).reshape(R, K)
    return {"codes": codes, "sf": e4m3_encode(s), "g": g}


def dequant_nvfp4_ref(codes, sf, g) -> np.ndarray:
    """fp64 values e2m1(code) * e4m3(sf) * g of [R, K] codes and [R, K/16] scales."""
    c = e2m1_decode(codes)
    R, K = c.shape
    s = e4m3_decode(sf)
    return (c.reshape(R, K // NVFP4_BLOCK, NVFP4_BLOCK) * s[..., None]).reshape(R, K) * np.float64(np.float32(g))


def pack_e2m1(codes) -> np.ndarray:
    """[R, K] 4-bit codes -> [R, K/2] bytes, element 2i in the low nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def unpack_e2m1(packed) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty((p.shape[0], p.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = p & 0xF
    out[:, 1::2] = p >> 4
    return out


def sf_tiled(sf) -> np.ndarray:
    """Scale factors [R, K/16] -> the GEMM's tiled byte layout (1-D, R padded to
    a multiple of 128 with zero scales): for row r and block j, with tile
    t = r // 128, lane l = r % 32, column c = (r % 128) // 32, k-step
    ks = j // 4 and jj = j % 4, the byte sits at
    (t * KS + ks) * 512 + l * 16 + c * 4 + jj, KS = K / 64."""
    sf = np.asarray(sf, dtype=np.uint8)
    R, KB = sf.shape
    if KB % 4:
        raise ValueError("K must be a multiple of 64")
    KS = KB // 4
    T = (R + 127) // 128
    out = np.zeros(T * KS * 512, dtype=np.uint8)
    r = np.arange(R)[:, None]
    j = np.arange(KB)[None, :]
    off = ((r // 128) * KS + j // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + j % 4
    out[off] = sf
    return out


def gemm_nvfp4_ref(xq: dict, wq: dict, bias=None) -> dict:
    """Y = X W^T + bias from NVFP4 X [M, K] and W [N, K] (dicts of quant_nvfp4_ref).
    Returns 'y' (fp64 exact: acc * fl32(g_x g_w) + bias), 'y_bf16' (the bf16
    rounding of it) and 'mag' (fl32(g_x g_w) * sum_k |a_k w_k|, the scale of the
    fp32 accumulation error)."""
    a = dequant_nvfp4_ref(xq["codes"], xq["sf"], 1.0)
    w = dequant_nvfp4_ref(wq["codes"], wq["sf"], 1.0)
    alpha = np.float64(np.float32(np.float32(xq["g"]) * np.float32(wq["g"])))
    acc = a @ w.T
    y = acc * alpha
    if bias is not None:
        y = y + _f32(bias).astype(np.float64)[None, :]
    mag = (np.abs(a) @ np.abs(w).T) * alpha
    return {"y": y, "y_bf16": bf16_round(y), "mag": mag}
