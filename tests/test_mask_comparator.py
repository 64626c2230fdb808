"""Pins of the GPU-vs-oracle mask comparator (host logic, no GPU).

The comparator may excuse a differing row only as a near-tie that an fp32
evaluation can decide the other way: blocks exchanged across the cut whose
scores differ by at most the tolerance, or a length set by a cumulative sum
that lies within the tolerance of p at every rank between the two cuts. Each
case below plants a GPU row and checks the verdict, so an excuse that is too
wide (an off-by-one at the cut passed as a tie) fails here."""
import numpy as np

import oracle
from gpu_helpers import compare_mask_rows

TOL = oracle.NEAR_TIE_TOL


def _verdict(s_row, kept, k_frac, p):
    n = s_row.shape[0]
    idx = np.full((1, n), -1, dtype=np.int64)
    kept = sorted(kept)
    idx[0, :len(kept)] = kept
    st = compare_mask_rows(idx, np.array([len(kept)]), s_row[None, :], k_frac, p)
    for key in ("exact", "score_tie", "cumsum_tie"):
        if st[key]:
            return key
    assert len(st["bad"]) == 1
    return "bad"


def _oracle_prefix(s_row, n):
    return set(oracle.descending_order(s_row)[:n].tolist())


def _spread_row(seed=3, n=16):
    rng = np.random.default_rng(seed)
    return rng.permutation(np.linspace(3.0, -3.0, n))      # distinct, gaps of 0.4


def test_exact_row_and_off_by_one_at_the_cut_without_a_tie():
    s = _spread_row()
    k_frac, p = 0.25, 0.0                                  # Top-k only: L = 4
    _, L, _, _ = oracle.hybrid_row(s, k_frac, p)
    assert L == 4
    order = oracle.descending_order(s)
    ora = _oracle_prefix(s, L)
    assert _verdict(s, ora, k_frac, p) == "exact"
    assert _verdict(s, ora - {int(order[L - 1])}, k_frac, p) == "bad"     # one short
    assert _verdict(s, ora | {int(order[L])}, k_frac, p) == "bad"         # one extra
    swapped = (ora - {int(order[L - 1])}) | {int(order[L])}
    assert _verdict(s, swapped, k_frac, p) == "bad"                      # 0.4 apart


def test_exchange_across_a_score_tie_at_the_cut():
    s = np.array([9.0, 8.0, 7.0, 6.0 + 3e-7, 6.0, 1.0, 0.0, -1.0])
    k_frac, p = 0.5, 0.0                                   # L = 4: block 3 kept, block 4 not
    assert _verdict(s, {0, 1, 2, 3}, k_frac, p) == "exact"
    assert _verdict(s, {0, 1, 2, 4}, k_frac, p) == "score_tie"
    far = s.copy()
    far[3] = 6.001
    assert _verdict(far, {0, 1, 2, 4}, k_frac, p) == "bad"
    assert _verdict(s, {0, 1, 3, 4}, k_frac, p) == "bad"   # drops block 2, a whole unit above


def test_length_set_by_a_cumulative_sum_near_p():
    s = _spread_row(seed=11)
    order = oracle.descending_order(s)
    csum = np.cumsum(oracle.block_softmax(s)[order])
    k_frac = 1.0 / 16                                      # K_sel = 1: Top-p sets the length
    # p just below the sum of the first six: the oracle stops at six, an fp32
    # sum a little low would take a seventh
    p = float(csum[5] - 5e-8)
    _, L, _, m_p = oracle.hybrid_row(s, k_frac, p)
    assert L == m_p == 6
    assert _verdict(s, _oracle_prefix(s, 7), k_frac, p) == "cumsum_tie"
    assert _verdict(s, _oracle_prefix(s, 8), k_frac, p) == "bad"        # rank 6 is not near p
    assert _verdict(s, _oracle_prefix(s, 5), k_frac, p) == "bad"        # rank 4 is not near p
    # p just above it: the oracle needs seven, an fp32 sum a little high stops at six
    p = float(csum[5] + 5e-8)
    _, L, _, _ = oracle.hybrid_row(s, k_frac, p)
    assert L == 7
    assert _verdict(s, _oracle_prefix(s, 6), k_frac, p) == "cumsum_tie"
    assert _verdict(s, _oracle_prefix(s, 5), k_frac, p) == "bad"
    # a length near p but with a block other than the prefix's last one
    wrong = (_oracle_prefix(s, 6) - {int(order[2])}) | {int(order[9])}
    assert _verdict(s, wrong, k_frac, p) == "bad"


def test_cumsum_tie_never_goes_below_top_k():
    s = _spread_row(seed=5)
    order = oracle.descending_order(s)
    csum = np.cumsum(oracle.block_softmax(s)[order])
    p = float(csum[3] + 5e-8)                              # oracle Top-p length 5
    k_frac = 5.0 / 16                                      # K_sel = 5
    _, L, k_sel, _ = oracle.hybrid_row(s, k_frac, p)
    assert (L, k_sel) == (5, 5)
    assert _verdict(s, _oracle_prefix(s, 4), k_frac, p) == "bad"        # below K_sel


def test_fast_path_with_the_oracle_mask_gives_the_same_verdicts():
    """Given the oracle's mask, rows equal to it are counted exact without the
    tie analysis; every other row still gets it, so the verdicts match."""
    rng = np.random.default_rng(21)
    n_qb, n_kb, k_frac, p = 12, 40, 0.1, 0.8
    s = rng.standard_normal((n_qb, n_kb)) * 2.0
    s[3, 5] = s[3, int(oracle.descending_order(s[3])[0])]          # a tie with the top block
    ora = np.zeros((n_qb, n_kb), dtype=bool)
    for r in range(n_qb):
        ora[r] = oracle.hybrid_row(s[r], k_frac, p)[0]
    gpu = ora.copy()
    order = oracle.descending_order(s[7])
    L = int(ora[7].sum())
    gpu[7, order[L - 1]] = False                                   # one short: bad
    gpu[9, oracle.descending_order(s[9])[int(ora[9].sum())]] = True  # one extra: bad
    idx = np.full((n_qb, n_kb), -1, dtype=np.int64)
    cnt = gpu.sum(1)
    for r in range(n_qb):
        kept = np.nonzero(gpu[r])[0]
        idx[r, :kept.shape[0]] = kept
    slow = compare_mask_rows(idx, cnt, s, k_frac, p)
    fast = compare_mask_rows(idx, cnt, s, k_frac, p, ora_mask=ora)
    assert slow["exact"] == fast["exact"] == n_qb - 2
    assert [b[0] for b in slow["bad"]] == [b[0] for b in fast["bad"]] == [7, 9]
