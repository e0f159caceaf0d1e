"""CPU oracle for dynamic block-sparse, low-precision attention (plain numpy, fp64).

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` use it. It shares no code with the CUDA library and imports nothing
from it; it is written from the pages' description of the method and from this
library's fixed reading of the points the pages leave open (listed below).

What the pages fix (Dynamic Sparse SageAttention in LightX2V):
  * "600倍加速，720p视频实时生成！单卡也能带的动14B模型", §动态稀疏量化注意力:
    importance is estimated from block-level means of Q and K, the key blocks
    are chosen at run time, only the activated attention tiles are computed,
    and a chosen block stays dense inside; typical sparsity 80-90%.
  * same page, §高效推理算子: block relevance is judged from the current Q/K,
    about 10% of the attention blocks are kept, and the arithmetic is Q/K INT8
    with V FP8.
  * "Run Wan2.2-A14B on One RTX 5090: 720p Video in 3.8s", §3 Dynamic sparse
    attention: the same, in English (top 10-20% of blocks from Q/K block means).

Readings this library takes where the pages are silent (the pages give no
block size, score formula, selection rule or quantisation granularity):
  * blocks of 64 tokens; nB = ceil(L/64); the last block may be partial and
    then covers only its valid tokens;
  * block score s[i, j] = (mean of Q over query block i) . (mean of K over key
    block j) / sqrt(d);
  * per query block keep k = clamp(ceil(keep*nB - 1e-6), 1, nB) key blocks with
    the largest scores, ties going to the lower key-block index; the kept ids
    are listed in ascending order;
  * INT8 Q/K: symmetric, one scale per (b, h, 64-token block) = absmax/127,
    codes rint(x * (127/absmax)) clamped to [-127, 127]; the code decision is
    taken in fp32 (the precision the kernels use), the rest in fp64;
  * FP8 E4M3 V: one scale per (b, h, channel) = absmax over all L tokens / 448,
    codes = E4M3 round-to-nearest-even with saturation of v * (448/absmax),
    again decided in fp32;
  * an all-zero block or channel gets scale 1;
  * the INT8/FP8 attention quantises P to E4M3 with the fixed scale 448 against
    the running row maximum, one 64-key block at a time in ascending key-block
    order; the softmax denominator sums the unquantised probabilities
    (see ``attn_ref_int8fp8``).

Everything is fp64 unless stated. Pins for every function live in
``tests/test_oracle.py``.
"""
from __future__ import annotations

import math

import numpy as np

BLOCK = 64          # tokens per block (query and key)
K_EPS = 1e-6        # guards ceil(keep*nB) against fp error (0.55*100 is 55.00000000000001)
E4M3_MAX = 448.0    # largest finite E4M3 (fn) value
INT8_MAX = 127


# --------------------------------------------------------------------------
# small helpers
# --------------------------------------------------------------------------
def n_blocks(L: int) -> int:
    return (int(L) + BLOCK - 1) // BLOCK


def keep_count(nB: int, keep: float) -> int:
    """k = clamp(ceil(keep*nB - 1e-6), 1, nB), evaluated in fp64."""
    if not (0.0 < keep <= 1.0):
        raise ValueError("keep must be in (0, 1]")
    k = math.ceil(float(keep) * nB - K_EPS)
    return int(min(nB, max(1, k)))


def _f64(x):
    """bf16/fp32 torch tensor or numpy array -> numpy fp64 (exact for bf16)."""
    if hasattr(x, "detach"):
        import torch  # local: the oracle itself is numpy; torch only unwraps tensors
        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def _f32(x):
    if hasattr(x, "detach"):
        import torch
        return x.detach().to("cpu", torch.float32).numpy()
    return np.asarray(x, dtype=np.float32)


def block_rows(i: int, L: int) -> slice:
    return slice(i * BLOCK, min(L, (i + 1) * BLOCK))


# --------------------------------------------------------------------------
# (a1) pooling and (a2) scoring / selection
# --------------------------------------------------------------------------
def block_means(X) -> np.ndarray:
    """Mean of X over each 64-token block, valid tokens only.

    X: [B, H, L, d] -> [B, H, nB, d] (fp64).  Block-level means of Q and K are
    the importance estimate the pages describe ("600倍加速…", §动态稀疏量化注意力).
    """
    x = _f64(X)
    B, H, L, d = x.shape
    nB = n_blocks(L)
    M = np.empty((B, H, nB, d))
    for i in range(nB):
        r = block_rows(i, L)
        M[:, :, i, :] = x[:, :, r, :].sum(axis=2) / (r.stop - r.start)
    return M


def block_scores(Mq: np.ndarray, Mk: np.ndarray) -> np.ndarray:
    """s[b,h,i,j] = Mq[b,h,i,:] . Mk[b,h,j,:] / sqrt(d)  (fp64)."""
    d = Mq.shape[-1]
    return np.einsum("bhid,bhjd->bhij", Mq, Mk) / math.sqrt(d)


def select_topk(s: np.ndarray, k: int) -> np.ndarray:
    """Per row keep the k largest scores, ties to the lower index; ascending ids.

    Sorting by (-s, j) and taking the first k is the plain definition: a stable
    sort of -s keeps equal scores in index order.
    """
    order = np.argsort(-s, axis=-1, kind="stable")[..., :k]
    return np.sort(order, axis=-1).astype(np.int32)


def kth_threshold(s: np.ndarray, k: int) -> np.ndarray:
    """The k-th largest score of each row (the selection threshold tau)."""
    return -np.sort(-s, axis=-1)[..., k - 1]


def plan_mask(idx: np.ndarray, nB: int) -> np.ndarray:
    """Bitmask view of a plan: bit (j % 32) of word j // 32 is set iff j is kept."""
    W = (nB + 31) // 32
    flat_idx = idx.reshape(-1, idx.shape[-1]).astype(np.int64)
    flat_out = np.zeros((flat_idx.shape[0], W), dtype=np.uint32)
    rows = np.repeat(np.arange(flat_idx.shape[0]), flat_idx.shape[1])
    cols = flat_idx.reshape(-1)
    np.bitwise_or.at(flat_out, (rows, cols >> 5), (np.uint32(1) << (cols & 31).astype(np.uint32)))
    return flat_out.reshape(idx.shape[:-1] + (W,))


def plan_ref(Q, K, keep: float) -> dict:
    """Full planner: means, scores, top-k ids (ascending) and the bitmask."""
    Mq, Mk = block_means(Q), block_means(K)
    s = block_scores(Mq, Mk)
    nB = s.shape[-1]
    k = keep_count(nB, keep)
    idx = select_topk(s, k)
    return {"Mq": Mq, "Mk": Mk, "scores": s, "k": k, "nB": nB,
            "idx": idx, "mask": plan_mask(idx, nB), "tau": kth_threshold(s, k)}


# --------------------------------------------------------------------------
# (a3) quantisers
# --------------------------------------------------------------------------
def quant_qk_ref(X):
    """INT8 symmetric per-(b,h,64-token block) quantisation of Q or K.

    "600倍加速…", §高效推理算子: Q and K are INT8.  Scale granularity and rounding
    are this library's reading: scale = absmax/127, code = rint(x*(127/absmax))
    clamped to +-127, with the code decided in fp32 (127/absmax and the product
    each rounded to fp32) so the integer result is unique.
    Returns (codes int8 [B,H,L,d], scale fp32 [B,H,nB]).
    """
    x = _f32(X)
    B, H, L, d = x.shape
    nB = n_blocks(L)
    codes = np.zeros((B, H, L, d), dtype=np.int8)
    scale = np.ones((B, H, nB), dtype=np.float32)
    for i in range(nB):
        r = block_rows(i, L)
        blk = x[:, :, r, :]
        a = np.abs(blk).max(axis=(2, 3)).astype(np.float32)           # [B,H]
        nz = a > 0
        inv = np.where(nz, np.float32(INT8_MAX) / np.where(nz, a, np.float32(1)), np.float32(0))
        inv = inv.astype(np.float32)
        y = (blk * inv[:, :, None, None]).astype(np.float32)
        codes[:, :, r, :] = np.clip(np.rint(y), -INT8_MAX, INT8_MAX).astype(np.int8)
        scale[:, :, i] = np.where(nz, a / np.float32(INT8_MAX), np.float32(1)).astype(np.float32)
    return codes, scale


def e4m3_round(y) -> np.ndarray:
    """Round to the nearest E4M3 (fn) value, ties to even, saturating at +-448.

    E4M3: 1 sign, 4 exponent (bias 7), 3 mantissa bits; normals (1+m/8)*2^e for
    e in [-6, 8] (448 = 1.75*2^8 is the largest finite value), subnormals
    m/8 * 2^-6.  The spacing in the binade [2^e, 2^(e+1)) is 2^(e-3), and 2^-9
    below 2^-6; rint on the exact quotient gives round-half-even.
    """
    y = np.asarray(y, dtype=np.float64)
    a = np.abs(y)
    _, ex = np.frexp(a)                         # a = f*2^ex, f in [0.5, 1)
    e = np.maximum(ex - 1, -6)                  # binade exponent, clamped at subnormals
    step = np.ldexp(1.0, (e - 3).astype(np.int64))
    q = np.rint(a / step) * step
    q = np.minimum(q, E4M3_MAX)
    return np.copysign(q, y)


def e4m3_encode(v) -> np.ndarray:
    """Bit pattern (uint8) of E4M3 values that are already on the grid."""
    v = np.asarray(v, dtype=np.float64)
    sign = np.signbit(v).astype(np.uint8) << 7
    a = np.abs(v)
    _, ex = np.frexp(a)
    e = ex - 1
    normal = a >= 2.0 ** -6
    mant_n = np.where(normal, np.rint((a / np.ldexp(1.0, np.where(normal, e, 0)) - 1.0) * 8), 0)
    expf_n = np.where(normal, e + 7, 0)
    mant_s = np.rint(a / 2.0 ** -9)
    code = np.where(normal, (expf_n << 3) | mant_n.astype(np.int64), mant_s.astype(np.int64))
    return (code.astype(np.uint8) | sign).astype(np.uint8)


def e4m3_decode(codes) -> np.ndarray:
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    ef = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(ef == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.ldexp(1.0, ef - 7))
    val = np.where((ef == 0xF) & (m == 0x7), np.nan, val)
    return s * val


def quant_v_ref(V):
    """FP8 E4M3 per-(b,h,channel) quantisation of V.

    "600倍加速…", §高效推理算子: V is FP8.  Reading: scale = absmax over all L
    tokens of the channel / 448; code = E4M3_rne_satfinite(v * (448/absmax))
    with 448/absmax and the product rounded to fp32 (the kernels' precision).
    Returns (codes uint8 [B,H,L,d], scale fp32 [B,H,d]).
    """
    x = _f32(V)
    a = np.abs(x).max(axis=2).astype(np.float32)                       # [B,H,d]
    nz = a > 0
    inv = np.where(nz, np.float32(E4M3_MAX) / np.where(nz, a, np.float32(1)), np.float32(0))
    inv = inv.astype(np.float32)
    y = (x * inv[:, :, None, :]).astype(np.float32)
    codes = e4m3_encode(e4m3_round(y.astype(np.float64)))
    scale = np.where(nz, a / np.float32(E4M3_MAX), np.float32(1)).astype(np.float32)
    return codes, scale


# --------------------------------------------------------------------------
# (a4) attention over the kept blocks
# --------------------------------------------------------------------------
def _gather_keys(j_list, L):
    return np.concatenate([np.arange(j * BLOCK, min(L, (j + 1) * BLOCK)) for j in j_list])


def _blocks_iter(B, H, nB, blocks):
    if blocks is None:
        for b in range(B):
            for h in range(H):
                for i in range(nB):
                    yield b, h, i
    else:
        for bhi in blocks:
            yield tuple(int(t) for t in bhi)


def attn_ref_exact(Q, K, V, idx, blocks=None) -> np.ndarray:
    """Softmax attention of each query block over its kept key blocks (fp64).

    For query block i: G = valid tokens of the kept key blocks; S = Q_i G^T/sqrt(d);
    P = softmax(S) row-wise; O_i = P V_G.  Dense inside each kept tile
    ("600倍加速…", §动态稀疏量化注意力).  The plain definition, no online softmax.
    ``blocks``: optional iterable of (b, h, i) to compute; other rows stay 0.
    """
    B, H, L, d = Q.shape
    nB = n_blocks(L)
    O = np.zeros((B, H, L, d))
    cache = {}
    for b, h, i in _blocks_iter(B, H, nB, blocks):
        if (b, h) not in cache:
            cache.clear()
            cache[(b, h)] = (_f64(Q[b, h]), _f64(K[b, h]), _f64(V[b, h]))
        q, k, v = cache[(b, h)]
        r = block_rows(i, L)
        g = _gather_keys(idx[b, h, i], L)
        S = q[r] @ k[g].T / math.sqrt(d)
        S = S - S.max(axis=1, keepdims=True)
        P = np.exp(S)
        P /= P.sum(axis=1, keepdims=True)
        O[b, h, r] = P @ v[g]
    return O


def attn_int8fp8_from_codes(qc, sq, kc, sk, vc, sv, idx, L, blocks=None) -> np.ndarray:
    """INT8/FP8 attention of each query block, given the quantised operands.

    qc, kc: int8 codes [B,H,L,d]; sq, sk: fp32 [B,H,nB]; vc: E4M3 codes
    [B,H,L,d]; sv: fp32 [B,H,d]; idx: [B,H,nB,k] ascending.

    P-quantisation protocol (this library's reading of "FP8" for the P.V
    product; the pages fix only that the path is FP8).  For a query row and its
    kept blocks j_1 < ... < j_k, step c over one 64-key block:
        S_c   = sq_i * sk_{j_c} * (q_codes . k_codes) / sqrt(d)
        m_c   = max(m_{c-1}, max S_c)                 (m_0 = -inf)
        Pq_c  = E4M3(448 * exp(S_c - m_c)) / 448
        acc   = sum_c exp(m_c - m_k) * Pq_c . Vdeq_{j_c}
        l     = sum_c exp(m_c - m_k) * sum exp(S_c - m_c)   (unquantised)
        O     = acc / l,   Vdeq = code_value(V) * sv[channel].
    """
    B, H = qc.shape[:2]
    d = qc.shape[-1]
    nB = n_blocks(L)
    O = np.zeros((B, H, L, d))
    inv_sqrt_d = 1.0 / math.sqrt(d)
    for b, h, i in _blocks_iter(B, H, nB, blocks):
        r = block_rows(i, L)
        q = qc[b, h, r].astype(np.float64)                         # [R, d]
        js = [int(j) for j in idx[b, h, i]]
        R = q.shape[0]
        kk = len(js)
        S = np.full((R, kk, BLOCK), -np.inf)
        Vb = np.zeros((kk, BLOCK, d))
        for c, j in enumerate(js):
            g = np.arange(j * BLOCK, min(L, (j + 1) * BLOCK))
            kcode = kc[b, h, g].astype(np.float64)
            S[:, c, : len(g)] = (float(sq[b, h, i]) * float(sk[b, h, j]) * inv_sqrt_d) * (q @ kcode.T)
            Vb[c, : len(g)] = e4m3_decode(vc[b, h, g]) * sv[b, h].astype(np.float64)[None, :]
        m = np.maximum.accumulate(S.max(axis=2), axis=1)            # [R, k]
        E = np.exp(S - m[:, :, None])                              # exp(-inf) = 0
        Pq = e4m3_round(E4M3_MAX * E) / E4M3_MAX
        w = np.exp(m - m[:, -1:])                                  # exp(m_c - m_k)
        l = np.einsum("rc,rcu->r", w, E)
        acc = np.einsum("rc,rcu,cud->rd", w, Pq, Vb)
        O[b, h, r] = acc / l[:, None]
    return O


def attn_ref_int8fp8(Q, K, V, idx, blocks=None) -> np.ndarray:
    """Quantise Q, K, V as the kernels do, then run ``attn_int8fp8_from_codes``.

    Quantisation is per (b, h), so only the heads that ``blocks`` touches are
    quantised (all of them when ``blocks`` is None).
    """
    B, H, L, d = Q.shape
    nB = n_blocks(L)
    O = np.zeros((B, H, L, d))
    todo = {}
    for b, h, i in _blocks_iter(B, H, nB, blocks):
        todo.setdefault((b, h), []).append(i)
    for (b, h), rows in todo.items():
        qc, sq = quant_qk_ref(Q[b:b + 1, h:h + 1])
        kc, sk = quant_qk_ref(K[b:b + 1, h:h + 1])
        vc, sv = quant_v_ref(V[b:b + 1, h:h + 1])
        Oh = attn_int8fp8_from_codes(qc, sq, kc, sk, vc, sv, idx[b:b + 1, h:h + 1], L,
                                     blocks=[(0, 0, i) for i in rows])
        for i in rows:
            r = block_rows(i, L)
            O[b, h, r] = Oh[0, 0, r]
    return O


# --------------------------------------------------------------------------
# error measures used by the parity tests
# --------------------------------------------------------------------------
def max_abs_err(O, R) -> float:
    return float(np.max(np.abs(_f64(O) - _f64(R))))


def rel_l1_err(O, R) -> float:
    """Mean relative error read as sum|O - R| / sum|R| over all elements."""
    O, R = _f64(O), _f64(R)
    return float(np.abs(O - R).sum() / np.abs(R).sum())
