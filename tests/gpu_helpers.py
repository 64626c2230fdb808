"""Comparison helpers for the GPU parity tests (CUDA path vs the fp64 oracle)."""
from __future__ import annotations

import numpy as np

import oracle

# Output tolerance against the fp64 oracle for unit-variance bf16 inputs with
# fp32 accumulation: bf16 rounding of O alone is up to 2^-9 of |O|.
MAX_ABS = 2e-2
MEAN_ABS = 2e-3


def _swap_within_tie(g, order, s, n, tol):
    """True when the set g holds n blocks and differs from the first n blocks of
    the oracle order only by exchanging blocks across a near-tie at that cut:
    every block the oracle keeps and g drops scores at most tol above every
    block g keeps and the oracle drops."""
    pref = set(order[:n].tolist())
    if len(g) != n:
        return False
    dropped, added = sorted(pref - g), sorted(g - pref)
    if not dropped:
        return True
    return float(s[dropped].max() - s[added].min()) <= tol


def lists_to_mask(gpu_idx, gpu_cnt, n_kb):
    """Boolean [n_qb, n_kb] mask of ascending kv lists (first cnt entries of each row)."""
    n_qb = gpu_cnt.shape[0]
    valid = np.arange(gpu_idx.shape[1])[None, :] < gpu_cnt[:, None]
    rows = np.repeat(np.arange(n_qb)[:, None], gpu_idx.shape[1], axis=1)[valid]
    mask = np.zeros((n_qb, n_kb), dtype=bool)
    mask[rows, gpu_idx[valid]] = True
    return mask


def compare_mask_rows(gpu_idx, gpu_cnt, s, k_frac, p, tol=oracle.NEAR_TIE_TOL, ora_mask=None):
    """Compare one head's GPU kv lists with the oracle decision on scores s.

    A row that differs is accepted only as a decision the fp32 GPU evaluation
    may take the other way:
      score tie   the same number of blocks, exchanged across the cut between
                  blocks whose scores differ by at most tol;
      cumsum tie  another length, at least K_sel, where every cumulative sum
                  between the two cuts lies within tol of p (so the fp32 sums
                  may cross p at either), and the kept set is that length's
                  prefix up to a score tie.
    Returns dict(exact, score_tie, cumsum_tie, bad)."""
    stats = {"exact": 0, "score_tie": 0, "cumsum_tie": 0, "bad": []}
    n_qb = s.shape[0]
    todo = range(n_qb)
    if ora_mask is not None:
        # rows equal to the oracle's mask need no tie analysis
        same = (lists_to_mask(gpu_idx, gpu_cnt, s.shape[1]) == ora_mask).all(axis=1)
        stats["exact"] = int(same.sum())
        todo = np.nonzero(~same)[0].tolist()
    for r in todo:
        g = set(gpu_idx[r, :gpu_cnt[r]].tolist())
        info = oracle.row_threshold_info(s[r], k_frac, p, tol)
        order, L = info["order"], info["L"]
        ora = set(order[:L].tolist())
        if g == ora:
            stats["exact"] += 1
            continue
        Lg = len(g)
        if Lg == L and _swap_within_tie(g, order, s[r], L, tol):
            stats["score_tie"] += 1
            continue
        # ranks whose cumulative sum decides between lengths L and Lg
        between = range(min(L, Lg) - 1, max(L, Lg) - 1)
        if Lg != L and Lg >= info["k_sel"] and min(L, Lg) >= 1 and \
                all(i in info["near_ranks"] for i in between) and \
                _swap_within_tie(g, order, s[r], Lg, tol):
            stats["cumsum_tie"] += 1
            continue
        stats["bad"].append((r, sorted(g - ora)[:8], sorted(ora - g)[:8], Lg, L))
    return stats


def assert_close(gpu, ref, what, max_abs=MAX_ABS, mean_abs=MEAN_ABS):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (what, gpu.shape, ref.shape)
    assert np.isfinite(gpu).all(), f"{what}: non-finite values"
    err = np.abs(gpu - ref)
    assert err.max() <= max_abs, f"{what}: max abs err {err.max():.3e} > {max_abs}"
    assert err.mean() <= mean_abs, f"{what}: mean abs err {err.mean():.3e} > {mean_abs}"
    return float(err.max()), float(err.mean())


def sample_blocks(n_qb, kv_cnt, rng, n_random=4):
    """Query blocks covering the first block, the ragged tail block, the
    densest and the sparsest block rows, and random others (at least 8 when
    the head has that many)."""
    blocks = {0, n_qb - 1, int(np.argmax(kv_cnt)), int(np.argmin(kv_cnt))}
    rest = [b for b in rng.permutation(n_qb).tolist() if b not in blocks]
    blocks |= set(rest[:max(n_random, 8 - len(blocks))])
    return sorted(blocks)


def sample_rows(n_qb, bq, N, kv_cnt, rng, n_random=4):
    """Every query row of the blocks sample_blocks picks, so that all four TMEM
    lane quadrants and both column halves of each sampled tile are compared."""
    blocks = sample_blocks(n_qb, kv_cnt, rng, n_random)
    return np.concatenate([np.arange(b * bq, min(N, (b + 1) * bq)) for b in blocks]).astype(np.int64)


def fp8_p_rounding_bound(q, k, v, mask, bq, bk, scale=None, rows=None):
    """Per-element bound on how far the low-bit attention may move from the
    oracle's (masked attention on the dequantised E4M3 inputs) through its own
    roundings: P rounded to E4M3 (within 2^-4 of P in the normal range, 2^-10
    absolute below it; P is normalised by the unrounded row sum), O rounded to
    bf16 (2^-9 relative), plus 1e-4 for fp32 accumulation.

    Inputs are one head's bf16 values as float64 [N, d]; returns [len(rows), d].
    """
    N, d = q.shape
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    qd, kd, vd = (c * s for c, s in (oracle.quantize_fp8_head(t) for t in (q, k, v)))
    rows = np.arange(N) if rows is None else np.asarray(rows, dtype=np.int64)
    bound = np.zeros((rows.shape[0], d))
    for qb in np.unique(rows // bq):
        at = np.nonzero(rows // bq == qb)[0]
        kept = np.nonzero(mask[qb])[0]
        if kept.shape[0] == 0:
            continue
        keys = np.concatenate([np.arange(kb * bk, min(N, (kb + 1) * bk)) for kb in kept])
        logits = scale * (qd[rows[at]] @ kd[keys].T)
        p = np.exp(logits - logits.max(axis=1, keepdims=True))
        l = p.sum(axis=1, keepdims=True)
        av = np.abs(vd[keys])
        o = np.abs(p @ vd[keys]) / l
        bound[at] = (2.0 ** -4 * (p @ av) + 2.0 ** -10 * av.sum(axis=0)[None, :]) / l + 2.0 ** -9 * o + 1e-4
    return bound


def assert_within_bound(gpu, ref, bound, what, mean_abs=MEAN_ABS, mean_frac=0.15):
    """Every element within its bound, and the mean error within mean_frac of
    the mean bound or mean_abs, whichever is larger: the bound assumes every
    rounding error points the same way, while rounding errors of independent
    weights largely cancel (a CPU simulation of the E4M3 rounding of P on
    unit-variance rows gives a mean error of 0.05 of the mean bound), so a
    systematic fault shows in the mean long before it reaches the bound."""
    gpu = np.asarray(gpu, dtype=np.float64)
    err = np.abs(gpu - np.asarray(ref, dtype=np.float64))
    assert np.isfinite(gpu).all(), f"{what}: non-finite values"
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    assert (err <= bound).all(), f"{what}: err {err[worst]:.3e} > bound {bound[worst]:.3e} at {worst}"
    lim = max(mean_abs, mean_frac * float(bound.mean()))
    assert err.mean() <= lim, f"{what}: mean abs err {err.mean():.3e} > {lim:.3e}"
    return float(err.max()), float(err.mean())
