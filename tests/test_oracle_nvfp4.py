"""Pins of the NVFP4 oracle (oracle/nvfp4_ref.py) against the format's
definition, brute force on small inputs and exact special cases.

"Run Wan2.2-A14B on One RTX 5090: 720p Video in 3.8s", §2: E2M1 values, an E4M3
scale per 16 elements, an FP32 global scale; FP32-accumulated GEMM with BF16
output and a fused column bias."""
import itertools

import numpy as np
import pytest

import oracle
from oracle import nvfp4_ref as nv

# The E2M1 grid of the OCP microscaling formats: magnitudes of codes 0..7.
E2M1_GRID = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_decode_all_codes():
    got = nv.e2m1_decode(np.arange(16))
    want = np.array(E2M1_GRID + [-v for v in E2M1_GRID])
    assert np.array_equal(got, want)


def _nearest_brute(y):
    """Nearest grid magnitude by scanning the 8 values; a tie goes to the even code."""
    a = min(abs(y), 6.0)
    best = None
    for code, v in enumerate(E2M1_GRID):
        d = abs(a - v)
        if best is None or d < best[0] - 1e-300 or (abs(d - best[0]) <= 0 and code % 2 == 0):
            best = (d, code, v)
    return np.copysign(best[2], y)


def test_e2m1_round_brute_force_and_ties():
    rng = np.random.default_rng(0)
    ys = list(rng.uniform(-8, 8, 4000)) + [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.75, -5.0, 6.0, 7.0,
                                           -100.0, 0.0, 1e-9]
    got = nv.e2m1_round(np.array(ys))
    want = np.array([_nearest_brute(y) for y in ys])
    assert np.array_equal(got, want)
    # ties resolve to the even mantissa (codes 0, 2, 4, 6)
    ties = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    for y, v in ties.items():
        assert nv.e2m1_round(y) == v


def test_e2m1_encode_decode_round_trip():
    vals = np.array(E2M1_GRID + [-v for v in E2M1_GRID[1:]])
    codes = nv.e2m1_encode(vals)
    assert np.array_equal(nv.e2m1_decode(codes), vals)
    assert nv.e2m1_encode(np.array([-0.0]))[0] == 0      # zero is always +0
    assert set(codes.tolist()) == set(range(16)) - {8}


def test_pack_nibble_order():
    codes = np.array([[1, 2, 3, 15]], dtype=np.uint8)
    p = nv.pack_e2m1(codes)
    assert p.tolist() == [[0x21, 0xF3]]
    assert np.array_equal(nv.unpack_e2m1(p), codes)


def test_sf_tiled_positions():
    R, KB = 200, 8                         # two row tiles, two k-steps
    sf = np.arange(R * KB, dtype=np.int64).reshape(R, KB) % 251 + 1
    t = nv.sf_tiled(sf.astype(np.uint8))
    assert t.size == 2 * 2 * 512
    # row 33, block 5: tile 0, lane 1, column 1, k-step 1, byte 1
    assert t[(0 * 2 + 1) * 512 + 1 * 16 + 1 * 4 + 1] == sf[33, 5]
    # row 130, block 2: tile 1, lane 2, column 0, k-step 0, byte 2
    assert t[(1 * 2 + 0) * 512 + 2 * 16 + 0 * 4 + 2] == sf[130, 2]
    # rows 200..255 of the last tile are padding with zero scales
    assert np.count_nonzero(t) == R * KB


def test_quant_exact_round_trip():
    """Values built from grid codes, E4M3 scales and a power-of-two global scale,
    with a +-6 in every block and 448 as the largest scale, quantise back to the
    same codes and scales."""
    rng = np.random.default_rng(1)
    R, K = 8, 64
    g0 = np.float32(2.0 ** -3)
    s_vals = nv.e4m3_round(rng.uniform(0.05, 400, (R, K // 16)))
    s_vals[0, 0] = 448.0
    c = rng.integers(0, 16, (R, K)).astype(np.uint8)
    c[:, ::16] = 7                          # a +6 in every block
    c[c == 8] = 0
    x = (nv.e2m1_decode(c).reshape(R, K // 16, 16) * s_vals[..., None]).reshape(R, K) * float(g0)
    q = nv.quant_nvfp4_ref(x.astype(np.float32))
    assert q["g"] == g0
    assert np.array_equal(q["codes"], c)
    assert np.array_equal(q["sf"], nv.e4m3_encode(s_vals))


def test_quant_error_bound_and_scale_range():
    rng = np.random.default_rng(2)
    x = (rng.standard_normal((64, 256)) * np.exp(rng.uniform(-4, 4, (64, 1)))).astype(np.float32)
    q = nv.quant_nvfp4_ref(x)
    s = oracle.e4m3_decode(q["sf"])
    assert s.max() <= 448.0 and s.min() >= 0.0
    # each block's largest element lands on +-6, +-4 or a neighbour of 6 after the E4M3 rounding of s
    deq = nv.dequant_nvfp4_ref(q["codes"], q["sf"], q["g"])
    xb = x.reshape(64, 16, 16).astype(np.float64)
    sg = (s * np.float64(q["g"]))[..., None]
    err = np.abs(deq.reshape(64, 16, 16) - xb)
    # within one E2M1 spacing of the scaled value (half a spacing plus the E4M3 rounding of s)
    y = np.abs(xb) / sg
    spacing = np.where(y < 2, 0.5, np.where(y < 4, 1.0, 2.0))
    assert np.all(err <= (0.5 * spacing + 1e-6 * y) * sg + 1e-30)


def test_quant_codes_brute_force():
    """Codes equal a scalar re-derivation of each step in fp32 on a small tensor."""
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((3, 32)) * 3).astype(np.float32)
    q = nv.quant_nvfp4_ref(x)
    amax = max(abs(float(v)) for v in x.ravel())
    g = np.float32(np.float32(amax) / np.float32(2688))
    assert q["g"] == g
    ig6 = np.float32(np.float32(1) / np.float32(np.float32(6) * g))
    for r, b in itertools.product(range(3), range(2)):
        blk = x[r, 16 * b:16 * b + 16]
        s = np.float32(nv.e4m3_round(np.float32(np.float32(np.abs(blk).max()) * ig6)))
        assert q["sf"][r, b] == nv.e4m3_encode(s)
        inv = np.float32(np.float32(1) / np.float32(s * g))
        for i in range(16):
            y = float(np.float32(blk[i] * inv))
            assert nv.e2m1_decode(q["codes"][r, 16 * b + i]) == _nearest_brute(y)


def test_quant_zero_tensor_and_zero_blocks():
    x = np.zeros((2, 32), np.float32)
    q = nv.quant_nvfp4_ref(x)
    assert q["g"] == 1.0 and not q["codes"].any() and not q["sf"].any()
    x[1, 20] = -3.0
    q = nv.quant_nvfp4_ref(x)
    assert q["sf"][0].tolist() == [0, 0] and q["sf"][1, 0] == 0
    assert nv.e2m1_decode(q["codes"][1, 20]) == -6.0


def test_gemm_brute_force():
    rng = np.random.default_rng(4)
    M, N, K = 3, 2, 32
    xq = nv.quant_nvfp4_ref(rng.standard_normal((M, K)).astype(np.float32))
    wq = nv.quant_nvfp4_ref(rng.standard_normal((N, K)).astype(np.float32))
    bias = rng.standard_normal(N).astype(np.float32)
    out = nv.gemm_nvfp4_ref(xq, wq, bias)
    alpha = float(np.float32(xq["g"] * wq["g"]))
    for m, n in itertools.product(range(M), range(N)):
        acc = 0.0
        for k in range(K):
            a = nv.e2m1_decode(xq["codes"][m, k]) * float(oracle.e4m3_decode(xq["sf"][m, k // 16]))
            w = nv.e2m1_decode(wq["codes"][n, k]) * float(oracle.e4m3_decode(wq["sf"][n, k // 16]))
            acc += a * w
        assert out["y"][m, n] == pytest.approx(acc * alpha + float(bias[n]), rel=1e-15, abs=1e-15)


def test_gemm_closed_form_ones():
    """All codes 1.0 (code 2) with unit scales: every output is K * g_x * g_w + bias."""
    M, N, K = 4, 3, 64
    ones = {"codes": np.full((M, K), 2, np.uint8), "sf": np.full((M, K // 16), 0x38, np.uint8), "g": np.float32(0.5)}
    w = {"codes": np.full((N, K), 2, np.uint8), "sf": np.full((N, K // 16), 0x38, np.uint8), "g": np.float32(0.25)}
    out = nv.gemm_nvfp4_ref(ones, w, np.array([1.0, -2.0, 0.5], np.float32))
    assert np.array_equal(out["y"], np.tile(np.array([K * 0.125 + 1.0, K * 0.125 - 2.0, K * 0.125 + 0.5]), (M, 1)))
