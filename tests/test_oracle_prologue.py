"""Pins of the prologue oracle (per-head RMSNorm, 3D RoPE, bf16 rounding)
against closed forms, invariants and torch's own cast; CPU only."""
import math

import numpy as np
import pytest
import torch

import oracle


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def test_rmsnorm_hand_example():
    # one head, d = 2, x = (3, 4): mean of squares 12.5
    x = np.array([[[[3.0, 4.0]]]])
    w = np.array([[2.0, 0.5]])
    y = oracle.qk_rmsnorm_ref(x, w, eps=0.0)
    r = math.sqrt(12.5)
    assert np.allclose(y[0, 0, 0], [2.0 * 3.0 / r, 0.5 * 4.0 / r], rtol=0, atol=1e-15)


def test_rmsnorm_unit_rms_and_scale_invariance():
    x = _rand((2, 3, 50, 64), 1)
    w = np.ones((3, 64))
    y = oracle.qk_rmsnorm_ref(x, w, eps=0.0)
    assert np.allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, atol=1e-13)
    y2 = oracle.qk_rmsnorm_ref(7.5 * x, w, eps=0.0)
    assert np.allclose(y, y2, atol=1e-13)
    # eps damps small rows: a zero row stays zero, a tiny row is not blown up to unit RMS
    z = np.zeros((1, 1, 1, 64))
    assert np.all(oracle.qk_rmsnorm_ref(z, np.ones((1, 64)), eps=1e-6) == 0)
    t = np.full((1, 1, 1, 64), 1e-6)
    assert np.sqrt(np.mean(oracle.qk_rmsnorm_ref(t, np.ones((1, 64)), eps=1e-6) ** 2)) < 2e-3


def test_rmsnorm_weights_per_head():
    x = _rand((1, 2, 4, 8), 2)
    w = np.stack([np.arange(1, 9, dtype=float), np.full(8, -1.0)])
    y = oracle.qk_rmsnorm_ref(x, w, eps=1e-6)
    base = oracle.qk_rmsnorm_ref(x, np.ones((2, 8)), eps=1e-6)
    assert np.allclose(y[:, 0], base[:, 0] * w[0], atol=1e-14)
    assert np.allclose(y[:, 1], -base[:, 1], atol=1e-14)


def test_split_and_positions():
    assert oracle.rope3d_split(128) == (44, 42, 42)
    assert oracle.rope3d_split(64) == (24, 20, 20)
    grid = (3, 4, 5)
    pos = oracle.token_positions(60, grid)
    n = 0
    for t in range(3):
        for h in range(4):
            for w in range(5):
                assert tuple(pos[n]) == (t, h, w)
                n += 1
    with pytest.raises(ValueError):
        oracle.token_positions(61, grid)


def test_rope_closed_form_one_pair_per_part():
    # d = 6 splits into three parts of one pair each, frequency theta^0 = 1, so
    # each pair turns by its own coordinate in radians
    grid = (2, 3, 4)
    L = 24
    x = _rand((1, 1, L, 6), 3)
    y = oracle.rope3d_ref(x, grid)
    for n in range(L):
        t, h, w = n // 12, (n // 4) % 3, n % 4
        for part, p in enumerate((t, h, w)):
            a, b = x[0, 0, n, 2 * part], x[0, 0, n, 2 * part + 1]
            want = (a * math.cos(p) - b * math.sin(p), a * math.sin(p) + b * math.cos(p))
            assert abs(y[0, 0, n, 2 * part] - want[0]) < 1e-14
            assert abs(y[0, 0, n, 2 * part + 1] - want[1]) < 1e-14


def test_rope_second_frequency():
    # a part of 4 channels: pair 0 turns by p, pair 1 by p * theta^(-1/2)
    x = np.zeros((1, 1, 8, 12))
    x[..., 2] = 1.0          # pair 1 of the time part (channels 2, 3), d_t = 12 - 8 = 4
    y = oracle.rope3d_ref(x, (8, 1, 1), split=(4, 4, 4))
    for t in range(8):
        ang = t * 10000.0 ** (-0.5)
        assert abs(y[0, 0, t, 2] - math.cos(ang)) < 1e-14 and abs(y[0, 0, t, 3] - math.sin(ang)) < 1e-14


def test_rope_identity_at_origin_and_norm_preserved():
    grid = (4, 6, 8)
    x = _rand((2, 2, 192, 128), 4)
    y = oracle.rope3d_ref(x, grid)
    assert np.allclose(y[:, :, 0], x[:, :, 0], atol=0)   # token 0 sits at (0, 0, 0)
    pair_x = x[..., 0::2] ** 2 + x[..., 1::2] ** 2
    pair_y = y[..., 0::2] ** 2 + y[..., 1::2] ** 2
    assert np.allclose(pair_x, pair_y, rtol=1e-12)


def test_rope_relative_position():
    # q . k after RoPE depends only on the position difference along each axis:
    # shifting both tokens by the same step along one axis keeps the product
    grid = (5, 5, 5)
    rng = np.random.default_rng(5)
    q, k = rng.standard_normal(128), rng.standard_normal(128)

    def dot(nq, nk):
        x = np.zeros((1, 1, 125, 128))
        x[0, 0, nq] += q
        y1 = oracle.rope3d_ref(x, grid)[0, 0, nq]
        x = np.zeros((1, 1, 125, 128))
        x[0, 0, nk] += k
        y2 = oracle.rope3d_ref(x, grid)[0, 0, nk]
        return float(y1 @ y2)

    idx = lambda t, h, w: t * 25 + h * 5 + w
    base = dot(idx(1, 2, 0), idx(0, 1, 3))
    assert abs(dot(idx(2, 2, 0), idx(1, 1, 3)) - base) < 1e-10      # t shifted
    assert abs(dot(idx(1, 4, 0), idx(0, 3, 3)) - base) < 1e-10      # h shifted
    assert abs(dot(idx(1, 2, 1), idx(0, 1, 4)) - base) < 1e-10      # w shifted
    assert abs(dot(idx(1, 2, 0), idx(0, 2, 3)) - base) > 1e-6       # a different offset


def test_bf16_round_matches_torch_cast():
    # fp32 values: torch's fp32 -> bf16 cast is round to nearest even
    x = (np.random.default_rng(6).standard_normal(200000) * np.exp(np.random.default_rng(7).uniform(-20, 20, 200000)))
    x = x.astype(np.float32)
    x[:4] = [0.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8)]   # exact ties
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = oracle.bf16_round(x.astype(np.float64))
    assert np.array_equal(got, want)


def test_prologue_composition_shapes():
    x = _rand((1, 2, 200, 64), 8, scale=3.0)
    w = 1.0 + 0.1 * _rand((2, 64), 9)
    r = oracle.prologue_ref(x, w, 1e-6, (2, 10, 10))
    assert r["Y"].shape == (1, 2, 200, 64) and r["means"].shape == (1, 2, 4, 64)
    assert r["codes"].dtype == np.int8 and r["scales"].shape == (1, 2, 4)
    # Y is bf16-representable
    assert np.array_equal(oracle.bf16_round(r["Y"]), r["Y"])


def test_k_channel_mean_and_zero_mean_after_shift():
    K = torch.from_numpy(_rand((1, 2, 300, 64), 10, scale=2.0) + 5.0).to(torch.bfloat16)
    km = oracle.k_channel_mean_ref(K)
    want = K.double().mean(dim=2).float().numpy()
    assert np.array_equal(km, want)
    Kd = K.double().numpy()
    assert np.abs((Kd - km[:, :, None, :].astype(np.float64)).mean(axis=2)).max() < 1e-6
    c = torch.full((1, 1, 70, 64), 1.25, dtype=torch.bfloat16)
    assert np.all(oracle.k_channel_mean_ref(c) == np.float32(1.25))


def test_smoothing_leaves_exact_attention_unchanged():
    # softmax over keys removes the per-row constant q.m
    rng = np.random.default_rng(11)
    B, H, L, d = 1, 2, 200, 64
    Q = torch.from_numpy(rng.standard_normal((B, H, L, d))).to(torch.bfloat16)
    K = torch.from_numpy(rng.standard_normal((B, H, L, d)) + rng.standard_normal((1, H, 1, d)) * 4).to(torch.bfloat16)
    V = torch.from_numpy(rng.standard_normal((B, H, L, d))).to(torch.bfloat16)
    idx = oracle.plan_ref(Q, K, 0.5)["idx"]
    km = oracle.k_channel_mean_ref(K).astype(np.float64)
    Ks = K.double().numpy() - km[:, :, None, :]
    O1 = oracle.attn_ref_exact(Q, K, V, idx)
    O2 = oracle.attn_ref_exact(Q, Ks, V, idx)
    assert np.abs(O1 - O2).max() < 1e-12


def test_smoothing_reduces_int8_error_on_offset_keys():
    # keys with a large common channel offset: the INT8 error of the smoothed
    # codes against the exact attention is much smaller
    rng = np.random.default_rng(12)
    B, H, L, d = 1, 1, 512, 64
    Q = torch.from_numpy(rng.standard_normal((B, H, L, d))).to(torch.bfloat16)
    off = rng.standard_normal((1, 1, 1, d)) * 8
    K = torch.from_numpy(rng.standard_normal((B, H, L, d)) + off).to(torch.bfloat16)
    V = torch.from_numpy(rng.standard_normal((B, H, L, d))).to(torch.bfloat16)
    idx = oracle.plan_ref(Q, K, 0.5)["idx"]
    R = oracle.attn_ref_exact(Q, K, V, idx)
    qc, sq = oracle.quant_qk_ref(Q)
    vc, sv = oracle.quant_v_ref(V)
    kc, sk = oracle.quant_qk_ref(K)
    ks_c, ks_s = oracle.quant_k_smooth_ref(K, oracle.k_channel_mean_ref(K))
    e_plain = oracle.rel_l1_err(oracle.attn_int8fp8_from_codes(qc, sq, kc, sk, vc, sv, idx, L), R)
    e_smooth = oracle.rel_l1_err(oracle.attn_int8fp8_from_codes(qc, sq, ks_c, ks_s, vc, sv, idx, L), R)
    assert e_smooth < 0.75 * e_plain, (e_plain, e_smooth)   # V and P keep their FP8 error


def test_quant_k_smooth_rule():
    # the codes are the INT8 rule applied to fl32(K - m): brute force on one block
    K = torch.from_numpy(_rand((1, 1, 64, 8), 13, scale=3.0) + 2.0).to(torch.bfloat16)
    km = oracle.k_channel_mean_ref(K)
    codes, scales = oracle.quant_k_smooth_ref(K, km)
    x = K.float().numpy()[0, 0] - km[0, 0][None, :]
    a = np.float32(np.abs(x).max())
    inv = np.float32(np.float32(127.0) / a)
    for t in range(64):
        for c in range(8):
            want = int(np.clip(np.rint(np.float32(x[t, c] * inv)), -127, 127))
            assert codes[0, 0, t, c] == want
    assert scales[0, 0, 0] == np.float32(a / np.float32(127.0))


def test_prologue_output_scalar_brute_force():
    """Y of a few rows re-derived with scalar loops: the RMS over the head's
    channels, the weight, then each channel pair turned by position * theta^(-2i/m)
    of its part (math.cos / math.sin), then the bf16 rounding of torch's cast."""
    d, grid, eps, theta = 64, (3, 4, 5), 1e-6, 10000.0
    x = _rand((1, 2, 60, d), 11, scale=2.0)
    w = 1.0 + 0.2 * _rand((2, d), 12)
    Y = oracle.prologue_ref(x, w, eps, grid, theta)["Y"]
    parts = (d - 4 * (d // 6), 2 * (d // 6), 2 * (d // 6))
    T, Hh, W = grid
    for h, t in [(0, 0), (1, 7), (0, 33), (1, 59)]:
        row = x[0, h, t].astype(np.float64)
        rms = math.sqrt(sum(v * v for v in row) / d + eps)
        y = [row[c] / rms * w[h, c] for c in range(d)]
        pos = (t // (Hh * W), (t // W) % Hh, t % W)
        out, c0 = list(y), 0
        for axis, m in enumerate(parts):
            for i in range(m // 2):
                ang = pos[axis] * theta ** (-2.0 * i / m)
                a, b = y[c0 + 2 * i], y[c0 + 2 * i + 1]
                out[c0 + 2 * i] = a * math.cos(ang) - b * math.sin(ang)
                out[c0 + 2 * i + 1] = a * math.sin(ang) + b * math.cos(ang)
            c0 += m
        want = torch.tensor(out, dtype=torch.float32).to(torch.bfloat16).double().numpy()
        got = Y[0, h, t]
        # torch rounds the fp32 value, the oracle the fp64 one: equal except where
        # the fp32 rounding lands on a bf16 tie, which one ulp covers
        ulp = np.ldexp(1.0, np.floor(np.log2(np.maximum(np.abs(want), 1e-30))).astype(int) - 7)
        assert np.all(np.abs(got - want) <= ulp)
        assert np.mean(got == want) > 0.95
