"""Helpers shared by the GPU parity tests (comparison logic only)."""
import numpy as np
import torch

import oracle

BAND_REL = 1e-5        # mask may differ only where the score is this close to the threshold
TOL_BF16_MAXABS = 2e-2
TOL_I8_MAXABS = 6e-2
TOL_I8_RELL1 = 1e-2


def to_np(t):
    return t.detach().cpu().numpy()


def bits_from_idx(idx, nB):
    sel = np.zeros(idx.shape[:-1] + (nB,), dtype=bool)
    np.put_along_axis(sel, idx.astype(np.int64), True, axis=-1)
    return sel


def bits_from_mask(mask_words, nB):
    m = mask_words.astype(np.uint32)
    j = np.arange(nB)
    return ((m[..., j >> 5] >> (j & 31).astype(np.uint32)) & 1).astype(bool)


def check_plan(gpu_idx, gpu_mask, Q, K, keep, heads=None, max_exempt_frac=None):
    """Compare a GPU plan with the oracle, head by head.

    Returns (exempt, outside_tau): the number of (row, key block) bits that
    differ from the oracle inside the tie band, and how many of those lie
    outside the pure tau-relative band |s - tau| <= 1e-5 |tau| (they are
    excused only by the row-scale floor of the band).  With
    `max_exempt_frac`, the exempt bits may be at most that fraction of the
    checked rows (plus 4), so that the band cannot hide a broad mismatch.
    """
    gi = to_np(gpu_idx)
    gm = to_np(gpu_mask) if gpu_mask is not None else None
    B, H, nB, k = gi.shape
    assert k == oracle.keep_count(nB, keep)
    # structural: strictly ascending, in range, mask agrees with idx
    assert np.all(gi >= 0) and np.all(gi < nB)
    assert np.all(np.diff(gi, axis=-1) > 0)
    exempt = outside_tau = rows = 0
    for b in range(B):
        for h in (range(H) if heads is None else heads):
            ref = oracle.plan_ref(Q[b:b + 1, h:h + 1], K[b:b + 1, h:h + 1], keep)
            s = ref["scores"][0, 0]
            tau = ref["tau"][0, 0][:, None]
            band = np.abs(s - tau) <= BAND_REL * np.maximum(np.abs(tau), np.abs(s).max(axis=-1, keepdims=True))
            tau_band = np.abs(s - tau) <= BAND_REL * np.abs(tau)
            want = bits_from_idx(ref["idx"][0, 0], nB)
            got = bits_from_idx(gi[b, h], nB)
            bad = (want != got) & ~band
            assert not bad.any(), f"mask mismatch outside the band at b={b} h={h}: {np.argwhere(bad)[:5]}"
            diff = (want != got) & band
            exempt += int(diff.sum())
            outside_tau += int((diff & ~tau_band).sum())
            rows += nB
            if gm is not None:
                assert np.array_equal(bits_from_mask(gm[b, h], nB), got)
    print(f"check_plan: {exempt} band-exempt bits over {rows} rows, {outside_tau} outside the pure tau band")
    if max_exempt_frac is not None:
        assert exempt <= max_exempt_frac * rows + 4, (exempt, rows)
    return exempt, outside_tau


def plan_from_oracle(Q, K, keep, device):
    """Oracle plan as a library Plan object (for attention tests independent of the planner)."""
    from video_dit_dynamic_token_b200 import Plan
    ref = oracle.plan_ref(Q, K, keep)
    B, H, L, D = Q.shape
    idx = torch.from_numpy(ref["idx"].astype(np.int32)).to(device)
    return Plan(idx, None, B, H, L, ref["nB"], ref["k"]), ref


def sample_blocks(B, H, nB, n, seed=0, must=()):
    rng = np.random.default_rng(seed)
    out = set(must)
    while len(out) < min(n, B * H * nB):
        out.add((int(rng.integers(B)), int(rng.integers(H)), int(rng.integers(nB))))
    return sorted(out)


def compare_rows(O_gpu, O_ref, L, blocks):
    """max-abs and rel-L1 restricted to the rows of the sampled query blocks."""
    og = O_gpu.detach().cpu().float().numpy().astype(np.float64)
    diffs, refs = [], []
    for b, h, i in blocks:
        r = slice(i * 64, min(L, (i + 1) * 64))
        diffs.append(np.abs(og[b, h, r] - O_ref[b, h, r]).ravel())
        refs.append(np.abs(O_ref[b, h, r]).ravel())
    d = np.concatenate(diffs)
    a = np.concatenate(refs)
    return float(d.max()), float(d.sum() / a.sum())
