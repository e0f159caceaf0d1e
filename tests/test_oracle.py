"""Pins for the CPU oracle, each against something other than the oracle itself.

Pins: a textbook dense routine (torch fp64 SDPA) at keep=1, scalar brute force
on tiny inputs written independently of the oracle's vectorised forms, a
hand-worked planner example (tests/golden), invariants of softmax attention,
a constructed dominant-block case, torch's float8_e4m3fn cast, and the closed
form of the single-block INT8/FP8 case.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from video_dit_dynamic_token_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _sdpa64(Q, K, V):
    q, k, v = (torch.as_tensor(np.asarray(x, dtype=np.float64)) for x in (Q, K, V))
    return torch.nn.functional.scaled_dot_product_attention(q, k, v).numpy()


def _f64(x):
    return x.to(torch.float64).numpy() if hasattr(x, "to") else np.asarray(x, np.float64)


# ---------------------------------------------------------------- k rule
def test_keep_count_rule():
    # Values worked by hand from k = clamp(ceil(keep*nB - 1e-6), 1, nB).
    assert oracle.keep_count(16, 0.25) == 4
    assert oracle.keep_count(512, 0.2) == 103      # 102.4 -> 103
    assert oracle.keep_count(1182, 0.1) == 119     # 118.2 -> 119
    assert oracle.keep_count(1890, 0.1) == 189
    assert oracle.keep_count(100, 0.55) == 55      # fp64 0.55*100 = 55.00000000000001
    assert oracle.keep_count(340, 0.55) == 187     # fp64 0.55*340 = 187.00000000000003
    assert oracle.keep_count(1182, 0.05) == 60
    assert oracle.keep_count(1182, 1.0) == 1182
    assert oracle.keep_count(1, 0.01) == 1
    with pytest.raises(ValueError):
        oracle.keep_count(10, 0.0)


# ---------------------------------------------------------------- golden worked example
def _read_golden():
    rows = {}
    with open(os.path.join(GOLDEN, "plan_worked_example.txt"), encoding="utf-8") as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, rest = line.split(" ", 1)
            rows.setdefault(key, []).append(rest)
    return rows


def test_planner_worked_example():
    g = _read_golden()
    qv = [tuple(float(t) for t in p.split(",")) for p in g["q_vectors"][0].split()]
    kv = [tuple(float(t) for t in p.split(",")) for p in g["k_vectors"][0].split()]
    L = int(g["L"][0])
    Q = np.zeros((1, 1, L, 2))
    K = np.zeros((1, 1, L, 2))
    for i in range(3):
        Q[0, 0, i * 64:min(L, (i + 1) * 64)] = qv[i]
        K[0, 0, i * 64:min(L, (i + 1) * 64)] = kv[i]
    for rest in g["keep"]:
        head, *rows = rest.split("|")
        keep, _, k = head.split()
        p = oracle.plan_ref(Q, K, float(keep))
        assert p["k"] == int(k)
        for i, r in enumerate(rows):
            assert p["idx"][0, 0, i].tolist() == [int(t) for t in r.split()]


# ---------------------------------------------------------------- brute force
def _bf_means(x, L):
    nB = (L + 63) // 64
    d = len(x[0])
    out = []
    for i in range(nB):
        s = [0.0] * d
        n = 0
        for t in range(i * 64, min(L, i * 64 + 64)):
            n += 1
            for c in range(d):
                s[c] += x[t][c]
        out.append([v / n for v in s])
    return out


def _bf_plan(q, k, L, keep):
    mq, mk = _bf_means(q, L), _bf_means(k, L)
    nB = len(mq)
    d = len(q[0])
    kk = min(nB, max(1, math.ceil(keep * nB - 1e-6)))
    plan = []
    for i in range(nB):
        s = [sum(mq[i][c] * mk[j][c] for c in range(d)) / math.sqrt(d) for j in range(nB)]
        chosen = []
        for _ in range(kk):   # repeated selection: largest remaining, lowest index on ties
            best = None
            for j in range(nB):
                if j in chosen:
                    continue
                if best is None or s[j] > s[best]:
                    best = j
            chosen.append(best)
        plan.append(sorted(chosen))
    return plan


def _bf_attn_exact(q, k, v, L, plan):
    d = len(q[0])
    out = [[0.0] * d for _ in range(L)]
    for i, js in enumerate(plan):
        keys = [u for j in js for u in range(j * 64, min(L, j * 64 + 64))]
        for t in range(i * 64, min(L, i * 64 + 64)):
            s = [sum(q[t][c] * k[u][c] for c in range(d)) / math.sqrt(d) for u in keys]
            m = max(s)
            e = [math.exp(x - m) for x in s]
            z = sum(e)
            for c in range(d):
                out[t][c] = sum(e[n] * v[keys[n]][c] for n in range(len(keys))) / z
    return out


@pytest.mark.parametrize("L,d,keep,seed", [(256, 8, 0.5, 1), (200, 16, 0.34, 2), (130, 4, 0.67, 3)])
def test_plan_and_exact_attention_brute_force(L, d, keep, seed):
    Q, K, V = synth.random_qkv(1, 1, L, d, seed=seed)
    q, k, v = (_f64(x)[0, 0].tolist() for x in (Q, K, V))
    plan_bf = _bf_plan(q, k, L, keep)
    p = oracle.plan_ref(Q, K, keep)
    assert p["idx"][0, 0].tolist() == plan_bf
    O = oracle.attn_ref_exact(Q, K, V, p["idx"])
    O_bf = np.array(_bf_attn_exact(q, k, v, L, plan_bf))
    assert np.max(np.abs(O[0, 0] - O_bf)) < 1e-12


# ---- independent quantiser brute force: enumerate candidate codes, ties to even
def _bf_int8_code(y):
    best = None
    for c in range(-127, 128):
        dist = abs(c - y)
        if best is None or dist < best[0] or (dist == best[0] and c % 2 == 0):
            best = (dist, c)
    return best[1]


def _e4m3_table():
    vals = []
    for code in range(256):
        s = -1.0 if code & 0x80 else 1.0
        e = (code >> 3) & 0xF
        m = code & 7
        if e == 15 and m == 7:
            continue  # NaN
        val = s * (m / 8.0) * 2.0 ** -6 if e == 0 else s * (1 + m / 8.0) * 2.0 ** (e - 7)
        vals.append((val, code))
    return vals


E4M3_TABLE = _e4m3_table()


def _bf_e4m3(y):
    if y > 448.0:
        y = 448.0
    if y < -448.0:
        y = -448.0
    best = None
    for val, code in E4M3_TABLE:
        if math.copysign(1.0, val) != math.copysign(1.0, y) and val != 0.0:
            continue
        dist = abs(val - y)
        if best is None or dist < best[0] or (dist == best[0] and (code & 1) == 0):
            best = (dist, val, code)
    val, code = best[1], best[2]
    if val == 0.0:
        code = 0x80 if math.copysign(1.0, y) < 0 else 0x00
    return val, code


def test_int8_quantiser_brute_force():
    Q, _, _ = synth.random_qkv(1, 1, 150, 8, seed=5, scale=3.0)
    codes, scale = oracle.quant_qk_ref(Q)
    x = Q.to(torch.float32).numpy()[0, 0]
    for i in range(3):
        blk = x[i * 64:min(150, i * 64 + 64)]
        a = np.float32(np.abs(blk).max())
        assert scale[0, 0, i] == np.float32(a / np.float32(127))
        inv = np.float32(np.float32(127) / a)
        for t in range(blk.shape[0]):
            for c in range(8):
                y = float(np.float32(blk[t, c] * inv))
                assert codes[0, 0, i * 64 + t, c] == _bf_int8_code(y)


def test_int8_quantiser_idempotent_on_integers():
    # a block whose absmax is 127 and whose values are integers maps to itself
    rng = np.random.default_rng(0)
    x = rng.integers(-127, 128, size=(1, 1, 64, 16)).astype(np.float32)
    x[0, 0, 5, 3] = 127.0
    codes, scale = oracle.quant_qk_ref(x)
    assert scale[0, 0, 0] == 1.0
    assert np.array_equal(codes.astype(np.float32), x)


def test_int8_quantiser_zero_block():
    x = np.zeros((1, 1, 70, 4), np.float32)
    codes, scale = oracle.quant_qk_ref(x)
    assert np.all(codes == 0) and np.all(scale == 1.0)


def test_e4m3_round_brute_force():
    rng = np.random.default_rng(1)
    y = np.concatenate([rng.normal(0, 50, 3000), rng.uniform(-1e-2, 1e-2, 1000),
                        [0.0, -0.0, 448.0, -448.0, 460.0, 465.0, 1e9, 2 ** -10, 3 * 2 ** -11]])
    y = y.astype(np.float32).astype(np.float64)
    vals = oracle.e4m3_round(y)
    codes = oracle.e4m3_encode(vals)
    for n in range(len(y)):
        bv, bc = _bf_e4m3(float(y[n]))
        assert vals[n] == bv, (y[n], vals[n], bv)
        assert codes[n] == bc, (y[n], codes[n], bc)
    assert np.array_equal(oracle.e4m3_decode(codes), vals)


def test_e4m3_matches_torch_cast():
    # torch's float8_e4m3fn CPU cast (round to nearest even) is the library routine.
    g = torch.Generator().manual_seed(3)
    y = torch.cat([torch.randn(500_000, generator=g) * 40,
                   torch.randn(250_000, generator=g) * 0.01,
                   (torch.rand(250_000, generator=g) * 2 - 1) * 448]).clamp(-448, 448)
    ref = y.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    mine = oracle.e4m3_encode(oracle.e4m3_round(y.numpy().astype(np.float64)))
    assert np.array_equal(ref, mine)


def test_v_quantiser_against_torch():
    _, _, V = synth.random_qkv(1, 2, 333, 16, seed=7, scale=2.0)
    codes, scale = oracle.quant_v_ref(V)
    v = V.to(torch.float32)
    a = v.abs().amax(dim=2)                                   # [1,2,16]
    inv = (torch.tensor(448.0) / a)
    y = v * inv[:, :, None, :]
    ref = y.clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codes, ref)
    assert np.array_equal(scale, (a / 448.0).numpy())


# ---------------------------------------------------------------- textbook / invariants
@pytest.mark.parametrize("shape", [(1, 2, 1024, 64), (2, 1, 200, 16)])
def test_keep_one_equals_dense_attention(shape):
    B, H, L, d = shape
    Q, K, V = synth.random_qkv(B, H, L, d, seed=11)
    p = oracle.plan_ref(Q, K, 1.0)
    assert p["k"] == p["nB"]
    O = oracle.attn_ref_exact(Q, K, V, p["idx"])
    R = _sdpa64(_f64(Q), _f64(K), _f64(V))
    assert np.max(np.abs(O - R)) < 1e-12


def test_single_block_is_dense():
    Q, K, V = synth.random_qkv(1, 1, 50, 16, seed=12)
    p = oracle.plan_ref(Q, K, 0.01)
    assert p["nB"] == 1 and p["k"] == 1
    O = oracle.attn_ref_exact(Q, K, V, p["idx"])
    assert np.max(np.abs(O - _sdpa64(_f64(Q), _f64(K), _f64(V)))) < 1e-12


def test_rows_sum_to_one_and_constant_v():
    Q, K, _ = synth.make_workload("tiny")
    p = oracle.plan_ref(Q, K, 0.25)
    B, H, L, d = Q.shape
    ones = np.ones((B, H, L, d))
    O = oracle.attn_ref_exact(Q, K, ones, p["idx"])
    assert np.max(np.abs(O - 1.0)) < 1e-12          # softmax rows sum to 1
    c = np.linspace(-3, 5, d)[None, None, None, :] * ones
    O = oracle.attn_ref_exact(Q, K, c, p["idx"])
    assert np.max(np.abs(O - c)) < 1e-12


def test_exact_attention_matches_masked_sdpa():
    # the kept-block gather equals dense attention with a block mask (textbook routine)
    Q, K, V = synth.make_workload("tiny")
    p = oracle.plan_ref(Q, K, 0.25)
    B, H, L, d = Q.shape
    mask = np.zeros((B, H, L, L), dtype=bool)
    for b in range(B):
        for h in range(H):
            for i in range(p["nB"]):
                for j in p["idx"][b, h, i]:
                    mask[b, h, i * 64:(i + 1) * 64, j * 64:(j + 1) * 64] = True
    q, k, v = (torch.as_tensor(_f64(x)) for x in (Q, K, V))
    R = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=torch.as_tensor(mask)).numpy()
    O = oracle.attn_ref_exact(Q, K, V, p["idx"])
    assert np.max(np.abs(O - R)) < 1e-12


def test_plan_structure_and_scale_invariance():
    Q, K, _ = synth.make_workload("tiny")
    p = oracle.plan_ref(Q, K, 0.25)
    idx = p["idx"]
    assert idx.shape == (1, 2, 16, 4)
    assert np.all(np.diff(idx, axis=-1) > 0) and idx.min() >= 0 and idx.max() < 16
    # bitmask agrees with the id list
    m = p["mask"]
    for h in range(2):
        for i in range(16):
            bits = [j for j in range(16) if (int(m[0, h, i, j >> 5]) >> (j & 31)) & 1]
            assert bits == idx[0, h, i].tolist()
    for alpha in (2.0, 0.5, 8.0):        # exact scalings: the plan cannot change
        q2 = _f64(Q) * alpha
        assert np.array_equal(oracle.plan_ref(q2, K, 0.25)["idx"], idx)


def test_dominant_block_is_selected():
    rng = np.random.default_rng(4)
    L, d, nB = 512, 32, 8
    u = rng.normal(size=d)
    u /= np.linalg.norm(u)
    Q = rng.normal(0, 0.05, size=(1, 1, L, d))
    K = rng.normal(0, 0.05, size=(1, 1, L, d))
    i, jstar = 3, 6
    Q[0, 0, i * 64:(i + 1) * 64] += 4 * u
    K[0, 0, jstar * 64:(jstar + 1) * 64] += 4 * u
    p = oracle.plan_ref(Q, K, 1 / nB)
    assert p["k"] == 1 and p["idx"][0, 0, i].tolist() == [jstar]
    p = oracle.plan_ref(Q, K, 3 / nB)
    order = np.argsort(-p["scores"][0, 0, i], kind="stable")
    assert order[0] == jstar and jstar in p["idx"][0, 0, i]


def test_permuting_tokens_inside_a_key_block():
    Q, K, V = synth.random_qkv(1, 1, 256, 16, seed=9)
    p = oracle.plan_ref(Q, K, 0.5)
    O = oracle.attn_ref_exact(Q, K, V, p["idx"])
    perm = np.arange(256)
    perm[64:128] = 64 + np.random.default_rng(0).permutation(64)
    k2, v2 = _f64(K)[:, :, perm], _f64(V)[:, :, perm]
    O2 = oracle.attn_ref_exact(Q, k2, v2, p["idx"])
    assert np.max(np.abs(O - O2)) < 1e-12


# ---------------------------------------------------------------- INT8/FP8 attention
def _bf_int8fp8_online(qc, sq, kc, sk, vc, sv, idx, L):
    """Scalar online form of the P-quantisation protocol (rescales the running
    accumulator at each step instead of the closed-form weights)."""
    d = len(qc[0])
    out = [[0.0] * d for _ in range(L)]
    for i, js in enumerate(idx):
        for t in range(i * 64, min(L, i * 64 + 64)):
            m = -math.inf
            acc = [0.0] * d
            lsum = 0.0
            for j in js:
                keys = range(j * 64, min(L, j * 64 + 64))
                s = [sq[i] * sk[j] * sum(qc[t][c] * kc[u][c] for c in range(d)) / math.sqrt(d) for u in keys]
                m_new = max(m, max(s))
                alpha = math.exp(m - m_new) if m != -math.inf else 0.0
                acc = [a * alpha for a in acc]
                lsum *= alpha
                for n, u in enumerate(keys):
                    e = math.exp(s[n] - m_new)
                    lsum += e
                    pq = _bf_e4m3(448.0 * e)[0] / 448.0
                    for c in range(d):
                        acc[c] += pq * E4M3_VAL[vc[u][c]] * sv[c]
                m = m_new
            out[t] = [a / lsum for a in acc]
    return out


E4M3_VAL = {code: val for val, code in E4M3_TABLE}
E4M3_VAL[0x80] = -0.0


def test_int8fp8_attention_brute_force():
    L, d = 150, 8
    Q, K, V = synth.random_qkv(1, 1, L, d, seed=21, scale=1.5)
    p = oracle.plan_ref(Q, K, 0.67)
    qc, sq = oracle.quant_qk_ref(Q)
    kc, sk = oracle.quant_qk_ref(K)
    vc, sv = oracle.quant_v_ref(V)
    O = oracle.attn_int8fp8_from_codes(qc, sq, kc, sk, vc, sv, p["idx"], L)
    O_bf = _bf_int8fp8_online(qc[0, 0].astype(float).tolist(), sq[0, 0].astype(float).tolist(),
                              kc[0, 0].astype(float).tolist(), sk[0, 0].astype(float).tolist(),
                              vc[0, 0].tolist(), sv[0, 0].astype(float).tolist(), p["idx"][0, 0].tolist(), L)
    assert np.max(np.abs(O[0, 0] - np.array(O_bf))) < 1e-12
    # the composed helper quantises exactly as above
    assert np.array_equal(oracle.attn_ref_int8fp8(Q, K, V, p["idx"]), O)


def test_int8fp8_single_block_closed_form():
    # nB = 1: one step, m = row max, O = sum e4m3(448 e^{s-m})/448 Vdeq / sum e^{s-m}
    L, d = 64, 16
    Q, K, V = synth.random_qkv(1, 1, L, d, seed=22)
    qc, sq = oracle.quant_qk_ref(Q)
    kc, sk = oracle.quant_qk_ref(K)
    vc, sv = oracle.quant_v_ref(V)
    S = float(sq[0, 0, 0]) * float(sk[0, 0, 0]) * (qc[0, 0].astype(np.float64) @ kc[0, 0].astype(np.float64).T) / 4.0
    E = np.exp(S - S.max(axis=1, keepdims=True))
    Pq = np.vectorize(lambda x: _bf_e4m3(x)[0])(448.0 * E) / 448.0
    Vd = np.vectorize(lambda c: E4M3_VAL[int(c)])(vc[0, 0]) * sv[0, 0][None, :]
    R = (Pq @ Vd) / E.sum(axis=1, keepdims=True)
    O = oracle.attn_int8fp8_from_codes(qc, sq, kc, sk, vc, sv, np.zeros((1, 1, 1, 1), np.int32), L)
    assert np.max(np.abs(O[0, 0] - R)) < 1e-12


def test_int8fp8_close_to_exact_on_smooth_field():
    # not a pin of the protocol; records how far quantisation moves the result
    Q, K, V = synth.make_workload("tiny")
    p = oracle.plan_ref(Q, K, 0.25)
    O8 = oracle.attn_ref_int8fp8(Q, K, V, p["idx"])
    O = oracle.attn_ref_exact(Q, K, V, p["idx"])
    assert oracle.rel_l1_err(O8, O) < 0.08


# ---------------------------------------------------------------- threshold and error measures
def _kth_by_repeated_removal(row, k):
    """The k-th largest value of a list, found by removing the maximum k-1 times."""
    vals = [float(v) for v in row]
    for _ in range(k - 1):
        vals.remove(max(vals))
    return max(vals)


@pytest.mark.parametrize("k", [1, 2, 3, 5, 8])
def test_kth_threshold_against_repeated_removal(k):
    # Rows built with ties exactly at the k-th place, negative rows, and one
    # row of equal scores; the threshold is the k-th largest value counted with
    # multiplicity (the score the k-th kept block has).
    rows = np.array([
        [0.5, 3.0, 3.0, 1.0, -2.0, 3.0, 0.0, 7.0],
        [-1.0, -4.0, -0.5, -0.5, -9.0, -3.0, -0.5, -2.0],
        [2.0, 2.0, 2.0, 2.0, 2.0, 2.0, 2.0, 2.0],
        [1e-9, -1e-9, 0.0, 5.0, 5.0, 4.0, 4.0, 4.0],
    ])
    got = oracle.kth_threshold(rows, k)
    want = np.array([_kth_by_repeated_removal(r, k) for r in rows])
    assert np.array_equal(got, want)
    # the selection keeps exactly the blocks with a score above tau, plus the
    # lowest-index ones among those equal to tau
    sel = oracle.select_topk(rows, k)
    for r in range(rows.shape[0]):
        tau = want[r]
        assert np.all(rows[r][sel[r]] >= tau)
        assert np.sum(rows[r] > tau) <= k


def test_kth_threshold_ends_of_the_range():
    rng = np.random.default_rng(3)
    s = rng.standard_normal((2, 3, 5, 13))
    # k = 1 is the row maximum, k = nB the row minimum
    assert np.array_equal(oracle.kth_threshold(s, 1), s.max(axis=-1))
    assert np.array_equal(oracle.kth_threshold(s, 13), s.min(axis=-1))
    # a hand-computed row: sorted descending 9, 7, 7, 4, 1 -> k = 2, 3 give 7, k = 4 gives 4
    row = np.array([[4.0, 7.0, 1.0, 9.0, 7.0]])
    assert [float(oracle.kth_threshold(row, k)[0]) for k in (1, 2, 3, 4, 5)] == [9.0, 7.0, 7.0, 4.0, 1.0]


def test_error_measures_hand_computed():
    # Values worked by hand.  O - R = [0.5, -1, 0, 0.25, -0.125, 0.5]; |R| sums to
    # 1 + 2 + 0 + 4 + 0.5 + 0.5 = 8, so rel-L1 = (0.5 + 1 + 0 + 0.25 + 0.125 + 0.5) / 8
    # = 2.375 / 8 = 0.296875.  A reference entry of 0 contributes its error to the
    # numerator and nothing to the denominator; no element-wise ratio is taken.
    R = np.array([[1.0, -2.0, 0.0], [4.0, 0.5, -0.5]])
    O = np.array([[1.5, -3.0, 0.0], [4.25, 0.375, 0.0]])
    assert oracle.max_abs_err(O, R) == 1.0
    assert oracle.rel_l1_err(O, R) == 0.296875
    # symmetric in the sign of the error, exact zero for equal arrays
    assert oracle.max_abs_err(R, O) == 1.0
    assert oracle.max_abs_err(R, R) == 0.0 and oracle.rel_l1_err(R, R) == 0.0
    # the measure is over all elements, not per row: a row-wise mean of ratios
    # would give (1.5/3 + 0.875/5) / 2 = 0.3375 here
    assert oracle.rel_l1_err(O, R) != 0.3375
    # a large error at the single zero reference entry stays finite
    O2 = R.copy()
    O2[0, 2] = 3.0
    assert oracle.rel_l1_err(O2, R) == 3.0 / 8.0
    assert oracle.max_abs_err(O2, R) == 3.0


def test_error_measures_accept_torch_and_bf16():
    R = torch.tensor([[0.5, -1.5], [2.0, 0.0]], dtype=torch.float64)
    O = torch.tensor([[0.5, -1.0], [2.0, 0.25]], dtype=torch.bfloat16)
    # bf16 holds these values exactly: |O - R| = [0, 0.5, 0, 0.25], sum |R| = 4
    assert oracle.max_abs_err(O, R) == 0.5
    assert oracle.rel_l1_err(O, R) == 0.75 / 4.0
