"""Pins of the Light-Ulysses exchange oracle: the FP8 row quantiser against
torch's E4M3 cast, its error bound, and the layout round trip of the
sequence -> head -> sequence exchange against a brute-force index map."""
import numpy as np
import pytest
import torch

import oracle


def _rand(shape, seed, scale=1.0):
    return (np.random.default_rng(seed).standard_normal(shape) * scale).astype(np.float32)


def test_fp8_rows_match_torch_cast():
    x = torch.from_numpy(_rand((3, 5, 7, 64), 1, scale=3.0)).to(torch.bfloat16)
    codes, scales = oracle.fp8_rows_ref(x)
    v = x.float()
    a = v.abs().amax(dim=-1)
    y = v * (torch.tensor(448.0) / a)[..., None]
    ref = y.clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codes, ref)
    assert np.array_equal(scales, (a / 448.0).numpy())


def test_fp8_rows_error_bound_and_zero_row():
    x = _rand((4, 100, 128), 2, scale=5.0)
    x[0, 0] = 0.0
    codes, scales = oracle.fp8_rows_ref(x)
    assert scales[0, 0] == 1.0 and np.all(codes[0, 0] == 0)
    y = oracle.fp8_rows_dequant_ref(codes, scales)
    # E4M3 keeps 3 mantissa bits (half-ulp 2^-4 relative) down to its normal
    # range, plus the bf16 rounding of the result; values below the E4M3 normal
    # range have an absolute error of at most half a subnormal step
    a = np.abs(x).max(axis=-1, keepdims=True)
    err = np.abs(y - x)
    bound = np.maximum(np.abs(x) * (2.0 ** -4 + 2.0 ** -8) * 1.001, a / 448.0 * 2.0 ** -10 * 1.001)
    assert np.all(err <= bound + 1e-30)


def _brute(q, k, v, N):
    """Index-by-index: what rank r should hold after the exchange."""
    B, Lr, H, D = q[0].shape
    Hr = H // N
    out = []
    for r in range(N):
        Q = np.zeros((B, Hr, N * Lr, D))
        K = np.zeros_like(Q)
        V = np.zeros_like(Q)
        for src in range(N):
            for h in range(Hr):
                for t in range(Lr):
                    for X, Y in ((q, Q), (k, K), (v, V)):
                        c, s = oracle.fp8_rows_ref(X[src][:, t, r * Hr + h, :])
                        Y[:, h, src * Lr + t, :] = oracle.fp8_rows_dequant_ref(c, s)
        out.append((Q, K, V))
    return out


@pytest.mark.parametrize("N", [1, 2, 4])
def test_exchange_layout_against_brute_force(N):
    B, Lr, H, D = 2, 3, 4, 8
    q = [_rand((B, Lr, H, D), 10 + r) for r in range(N)]
    k = [_rand((B, Lr, H, D), 20 + r) for r in range(N)]
    v = [_rand((B, Lr, H, D), 30 + r) for r in range(N)]
    sends = [oracle.pack_qkv_ref(q[r], k[r], v[r], N) for r in range(N)]
    recv_c = oracle.all_to_all_ref([s[0] for s in sends])
    recv_s = oracle.all_to_all_ref([s[1] for s in sends])
    want = _brute(q, k, v, N)
    for r in range(N):
        Q, K, V = oracle.unpack_qkv_ref(recv_c[r], recv_s[r])
        assert np.array_equal(Q, want[r][0]) and np.array_equal(K, want[r][1]) and np.array_equal(V, want[r][2])
    # the way back: head-sharded O -> sequence-sharded, each row one FP8 round trip
    o = [_rand((B, H // N, N * Lr, D), 40 + r) for r in range(N)]
    back = [oracle.pack_o_ref(o[r], N) for r in range(N)]
    rc = oracle.all_to_all_ref([b[0] for b in back])
    rs = oracle.all_to_all_ref([b[1] for b in back])
    for r in range(N):
        got = oracle.unpack_o_ref(rc[r], rs[r])                 # [B, Lr, H, D]
        for src in range(N):
            for h in range(H // N):
                for t in range(Lr):
                    c, s = oracle.fp8_rows_ref(o[src][:, h, r * Lr + t, :])
                    assert np.array_equal(got[:, t, src * (H // N) + h, :], oracle.fp8_rows_dequant_ref(c, s))


def test_dequant_is_bf16_of_the_fp32_product():
    """The receiver's value is bf16(fl32(decode(code) * scale)), with torch's fp32
    product and its round-to-nearest-even bf16 cast as the reference."""
    x = torch.from_numpy(_rand((6, 64), 3, scale=7.0)).to(torch.bfloat16)
    codes, scales = oracle.fp8_rows_ref(x)
    dec = torch.from_numpy(codes).view(torch.float8_e4m3fn).float()
    want = (dec * torch.from_numpy(scales)[:, None]).to(torch.bfloat16).double().numpy()
    assert np.array_equal(oracle.fp8_rows_dequant_ref(codes, scales), want)
