"""Pins of the fp64 oracle against things other than itself.

Each test below ties one oracle function to brute force, a closed form, an
exhaustive search or a library routine (torch float64 SDPA), so that a dropped
term, a wrong index or a transposed operand in the oracle fails here.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_softmax_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.filterwarnings("ignore::UserWarning")


def _rng(seed):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- pooling
def test_pool_matches_brute_force_loops_with_partial_tail():
    x = _rng(0).standard_normal((37, 5))
    means, counts = oracle.pool_blocks(x, 8)
    assert means.shape == (5, 5) and counts.tolist() == [8, 8, 8, 8, 5]
    for blk in range(5):
        for c in range(5):
            acc, n = 0.0, 0
            for t in range(37):
                if t // 8 == blk:
                    acc += x[t, c]
                    n += 1
            assert abs(means[blk, c] - acc / n) < 1e-14


def test_pool_constant_blocks_and_token_sum_identity():
    x = np.repeat(np.arange(6, dtype=np.float64)[:, None] * 0.5, 10, axis=0)[:, :1].repeat(3, 1)
    x = x[:57]  # last block partial
    means, counts = oracle.pool_blocks(x, 10)
    assert np.allclose(means[:, 0], [0, 0.5, 1.0, 1.5, 2.0, 2.5])
    y = _rng(1).standard_normal((57, 4))
    m2, c2 = oracle.pool_blocks(y, 10)
    assert np.allclose((m2 * c2[:, None]).sum(0), y.sum(0), atol=1e-12)


# ---------------------------------------------------------------- scores + softmax
def test_block_scores_brute_force_and_softmax():
    qp = _rng(2).standard_normal((3, 4))
    kp = _rng(3).standard_normal((5, 4))
    s = oracle.block_scores(qp, kp, 0.5)
    for i in range(3):
        for j in range(5):
            assert abs(s[i, j] - 0.5 * sum(qp[i, c] * kp[j, c] for c in range(4))) < 1e-14
    P = oracle.block_softmax(s)
    for i in range(3):
        z = sum(math.exp(s[i, j]) for j in range(5))
        for j in range(5):
            assert abs(P[i, j] - math.exp(s[i, j]) / z) < 1e-15
    assert np.allclose(P.sum(1), 1.0)
    assert np.allclose(oracle.block_softmax(s + 123.0), P)


# ---------------------------------------------------------------- Top-k count
@pytest.mark.parametrize("k,n,want", [(0.10, 16, 2), (0.05, 512, 26), (0.03, 1182, 36),
                                      (0.05, 1182, 60), (0.05, 3840, 192), (0.1, 10, 1),
                                      (1.0, 77, 77), (1e-6, 50, 1), (0.5, 3, 2)])
def test_topk_count_closed_form(k, n, want):
    assert oracle.topk_count(k, n) == want


# ---------------------------------------------------------------- Top-p minimality
def _tiny_rows():
    wl = WORKLOADS["tiny"]
    x = make_inputs(wl, "cpu")
    rows = []
    for h in range(wl.H):
        out = oracle.build_mask(oracle.as_f64(x["q"][0, h]), oracle.as_f64(x["k"][0, h]),
                                wl.bq, wl.bk, wl.topk, wl.topp)
        rows += [(out["s"][r], out["mask"][r], out["m_p"][r], out["L"][r]) for r in range(out["s"].shape[0])]
    return wl, rows


def test_topp_minimal_by_exhaustive_subsets_on_tiny_workload():
    """Every row of the tiny workload has 16 key blocks: try all 2^16 subsets."""
    wl, rows = _tiny_rows()
    n = 16
    bits = ((np.arange(1 << n)[:, None] >> np.arange(n)[None, :]) & 1).astype(np.float64)
    sizes = bits.sum(1)
    for p in (wl.topp, 0.5, 0.99):
        for s_row, _, _, _ in rows:
            P = oracle.block_softmax(s_row)
            sums = bits @ P
            min_size = int(sizes[sums >= p - 0.0].min())
            order = oracle.descending_order(s_row)
            m_p = oracle.topp_count(P[order], p)
            # rounding of the running sum is allowed to differ only within the tie band
            if abs(np.cumsum(P[order])[m_p - 1] - p) > 1e-12 and (m_p < 2 or abs(np.cumsum(P[order])[m_p - 2] - p) > 1e-12):
                assert m_p == min_size
            assert P[order][:m_p].sum() >= p - 1e-12


def test_topp_count_from_the_low_end_of_the_order():
    """Top-p from the other end: the kept prefix of length m_p is the shortest
    one whose complement (the n - m_p lowest blocks) holds at most 1 - p of
    the mass, counted by accumulating from the last block of the order, on
    peaked, spread, near-uniform and sink rows."""
    rng = _rng(17)
    for trial in range(60):
        n = int(rng.choice([16, 100, 1182]))
        kind = trial % 4
        if kind == 0:
            s = rng.standard_normal(n) * 3.0
        elif kind == 1:
            s = rng.standard_normal(n) * 0.5
        elif kind == 2:
            s = rng.standard_normal(n) * 0.005                 # near-uniform
        else:
            s = rng.standard_normal(n) * 0.5
            s[rng.integers(n)] += 12.0                           # one sink block
        order = oracle.descending_order(s)
        P = oracle.block_softmax(s)[order]
        for p in (0.5, 0.85, 0.9, 0.99):
            m_p = oracle.topp_count(P, p)
            j = 0                                                # blocks droppable from the end
            while j < n - 1 and math.fsum(P[n - j - 1:]) <= 1.0 - p:
                j += 1
            t_keep = math.fsum(P[m_p:])
            t_more = math.fsum(P[m_p - 1:])
            near = abs(t_keep - (1.0 - p)) <= 1e-12 or abs(t_more - (1.0 - p)) <= 1e-12
            if not near:
                assert n - j == m_p, (trial, p, n - j, m_p)
            assert t_keep <= 1.0 - p + 1e-12
            assert m_p == 1 or t_more > 1.0 - p - 1e-12


def test_kept_set_from_the_low_end_with_ties():
    """On heavily tied rows, dropping the lowest blocks while their mass stays
    within 1 - p (ties at the last dropped score from the highest block index
    down) leaves exactly the oracle's kept set whenever that set is at least
    K_sel long: the order's tie rule (lower index first) seen from the other
    end."""
    rng = _rng(23)
    checked = 0
    for trial in range(200):
        n = int(rng.choice([40, 300]))
        s = np.round(rng.standard_normal(n) * 0.05, 2)          # many equal scores
        p = float(rng.choice([0.5, 0.8, 0.9]))
        k_frac = 0.05
        mask, L, k_sel, m_p = oracle.hybrid_row(s, k_frac, p)
        if m_p < k_sel:
            continue
        P = oracle.block_softmax(s)
        csum = np.cumsum(P[oracle.descending_order(s)])
        if np.any(np.abs(csum - p) <= 1e-12):
            continue                                             # a cumulative-sum tie: either end may round
        # ascending by score, equal scores by higher block index first
        low = sorted(range(n), key=lambda i: (s[i], -i))
        dropped, mass = [], 0.0
        for i in low:
            if mass + P[i] > 1.0 - p:
                break
            dropped.append(i)
            mass += P[i]
        kept = np.ones(n, dtype=bool)
        kept[dropped] = False
        assert (kept == mask).all(), (trial, n, p)
        checked += 1
    assert checked > 100


def test_hybrid_equals_union_of_rank_defined_sets():
    """Top-k and Top-p built from the rank definition, with deliberate ties."""
    rng = _rng(5)
    for trial in range(200):
        n = int(rng.integers(1, 12))
        s = np.round(rng.standard_normal(n) * 2, 1)   # rounding creates ties
        k = float(rng.uniform(0.01, 1.0))
        p = float(rng.uniform(0.0, 0.999))
        rank = np.array([sum(1 for j in range(n) if s[j] > s[i] or (s[j] == s[i] and j < i))
                         for i in range(n)])
        k_sel = oracle.topk_count(k, n)
        topk = {i for i in range(n) if rank[i] < k_sel}
        P = np.exp(s - s.max()); P /= P.sum()
        by_rank = P[np.argsort(rank)]
        m_p = next((m for m in range(1, n + 1) if by_rank[:m].sum() >= p), n)
        topp = {i for i in range(n) if rank[i] < m_p}
        mask, L, ks, mp = oracle.hybrid_row(s, k, p)
        assert set(np.nonzero(mask)[0].tolist()) == topk | topp
        assert ks == k_sel and L == max(k_sel, m_p)


def test_hybrid_special_cases():
    rng = _rng(6)
    s = rng.standard_normal(40)
    assert oracle.hybrid_row(s, 1.0, 0.5)[0].all()                       # k = 100%
    m, L, ks, mp = oracle.hybrid_row(s, 0.1, 0.0)                        # p = 0: Top-k only
    assert m.sum() == 4 and L == ks == 4
    assert oracle.hybrid_row(s, 1e-6, 1.0)[0].all()                       # p = 1: every block
    sink = np.full(40, -20.0); sink[7] = 20.0                             # one-hot sink row
    m, L, ks, mp = oracle.hybrid_row(sink, 0.05, 0.9)
    assert mp == 1 and L == ks == 2 and m[7] and m[0]                     # tie order: lowest index
    flat = np.zeros(16)                                                   # uniform row
    m, L, ks, mp = oracle.hybrid_row(flat, 0.1, 0.9)
    assert mp == 15 and L == 15 and m[:15].all() and not m[15]


def test_hybrid_worked_example_from_the_failure_modes():
    """SpargeAttention2 §1: Top-k misses mass on flat rows, Top-p collapses onto sinks."""
    flat = np.log(np.array([0.2, 0.2, 0.2, 0.2, 0.2]))
    m, L, ks, mp = oracle.hybrid_row(flat, 0.2, 0.7)
    assert ks == 1 and mp == 4 and L == 4           # Top-p rescues the flat row
    skew = np.log(np.array([0.91, 0.03, 0.03, 0.02, 0.01]))
    m, L, ks, mp = oracle.hybrid_row(skew, 0.4, 0.9)
    assert mp == 1 and ks == 2 and L == 2           # Top-k rescues the sink row
    assert m.tolist() == [True, True, False, False, False]


def test_kv_lists_round_trip():
    mask = _rng(7).random((9, 13)) < 0.3
    idx, cnt = oracle.kv_lists(mask)
    assert (oracle.mask_from_lists(idx, cnt, 13) == mask).all()
    for r in range(9):
        assert (np.diff(idx[r, :cnt[r]]) > 0).all()


# ---------------------------------------------------------------- attention
def _sdpa(q, k, v, mask=None, scale=None):
    t = lambda a: torch.from_numpy(a)[None, None]
    am = None if mask is None else torch.from_numpy(mask)[None, None]
    o = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), attn_mask=am, scale=scale)
    return o[0, 0].numpy()


def test_all_ones_mask_is_dense_attention_sdpa():
    rng = _rng(8)
    N, d = 100, 16
    q, k, v = (rng.standard_normal((N, d)) for _ in range(3))
    mask = np.ones((-(-N // 32), -(-N // 16)), dtype=bool)
    o, lse = oracle.masked_attention(q, k, v, mask, 32, 16)
    assert np.abs(o - _sdpa(q, k, v)).max() < 1e-12
    od, lsed = oracle.dense_attention(q, k, v)
    assert np.abs(o - od).max() < 1e-12
    ref_lse = torch.logsumexp(torch.from_numpy(q @ k.T / math.sqrt(d)), dim=1).numpy()
    assert np.abs(lse - ref_lse).max() < 1e-12


def test_block_mask_equals_sdpa_with_expanded_token_mask():
    rng = _rng(9)
    N, d, bq, bk = 70, 8, 16, 8
    q, k, v = (rng.standard_normal((N, d)) for _ in range(3))
    q *= 2.0
    mask = rng.random((-(-N // bq), -(-N // bk))) < 0.4
    mask[:, 0] = True
    tok = np.zeros((N, N), dtype=bool)
    for i in range(N):
        for j in range(N):
            tok[i, j] = mask[i // bq, j // bk]
    o, _ = oracle.masked_attention(q, k, v, mask, bq, bk, scale=0.3)
    assert np.abs(o - _sdpa(q, k, v, tok, scale=0.3)).max() < 1e-12


def test_attention_invariants():
    rng = _rng(10)
    N, d = 50, 8
    q, k = rng.standard_normal((N, d)), rng.standard_normal((N, d))
    v_const = np.tile(rng.standard_normal(d), (N, 1))
    mask = rng.random((4, 7)) < 0.5
    mask[:, 3] = True
    o, _ = oracle.masked_attention(q, k, v_const, mask, 16, 8)
    assert np.abs(o - v_const).max() < 1e-12
    v = rng.standard_normal((N, d))
    o, _ = oracle.masked_attention(q, k, v, mask, 16, 8)
    assert (np.abs(o) <= np.abs(v).max(0) + 1e-12).all()
    empty = np.zeros((4, 7), dtype=bool)
    o, lse = oracle.masked_attention(q, k, v, empty, 16, 8, rows=[0, 49])
    assert (o == 0).all() and np.isneginf(lse).all()


# ---------------------------------------------------------------- linear branch + blend
def test_phi_is_elu_plus_one():
    x = np.linspace(-30, 30, 1001)
    ref = torch.nn.functional.elu(torch.from_numpy(x)).numpy() + 1.0
    assert np.abs(oracle.phi(x) - ref).max() < 1e-15
    assert (oracle.phi(x) > 0).all()


def test_linear_branch_equals_quadratic_brute_force():
    rng = _rng(11)
    N, d = 40, 6
    q, k, v = (rng.standard_normal((N, d)) for _ in range(3))
    S, z = oracle.linear_state(k, v)
    o = oracle.linear_out(q, S, z)
    for i in range(N):
        num = np.zeros(d)
        den = 0.0
        for j in range(N):
            w = float(np.dot(oracle.phi(q[i]), oracle.phi(k[j])))
            num += w * v[j]
            den += w
        assert np.abs(o[i] - num / den).max() < 1e-12
    vc = np.tile(rng.standard_normal(d), (N, 1))
    S, z = oracle.linear_state(k, vc)
    assert np.abs(oracle.linear_out(q, S, z) - vc).max() < 1e-12


def test_blend_endpoints_and_midpoint():
    rng = _rng(12)
    a, b = rng.standard_normal((5, 4)), rng.standard_normal((5, 4))
    assert np.array_equal(oracle.blend(a, b, np.ones(4)), a)
    assert np.array_equal(oracle.blend(a, b, np.zeros(4)), b)
    assert np.allclose(oracle.blend(a, b, np.full(4, 0.5)), (a + b) / 2)


# ---------------------------------------------------------------- build_mask wiring
def _brute_force_mask(q, k, bq, bk, k_frac, p, scale):
    """The whole mask of one head from the definitions, by scalar loops only:
    block means over valid tokens (query blocks of bq tokens, key blocks of bk),
    s = scale * sum_c Qbar_c Kbar_c, P by exp and sum, ranks by counting
    (higher score first, equal scores lower index first), keep rank < max(K_sel, m_p)."""
    N, d = q.shape
    nq, nk = -(-N // bq), -(-N // bk)

    def means(x, b, n):
        out = []
        for blk in range(n):
            acc, cnt = [0.0] * d, 0
            for t in range(blk * b, min(N, (blk + 1) * b)):
                for c in range(d):
                    acc[c] += float(x[t, c])
                cnt += 1
            out.append([a / cnt for a in acc])
        return out

    qm, km = means(q, bq, nq), means(k, bk, nk)
    k_sel = min(nk, max(1, math.ceil(k_frac * nk - 1e-9)))
    mask = np.zeros((nq, nk), dtype=bool)
    for r in range(nq):
        s = [scale * sum(qm[r][c] * km[j][c] for c in range(d)) for j in range(nk)]
        top = max(s)
        e = [math.exp(x - top) for x in s]
        z = sum(e)
        P = [x / z for x in e]
        rank = [sum(1 for j in range(nk) if s[j] > s[i] or (s[j] == s[i] and j < i)) for i in range(nk)]
        by_rank = [P[i] for i in sorted(range(nk), key=lambda i: rank[i])]
        m_p, acc = nk, 0.0
        for m in range(1, nk + 1):
            acc += by_rank[m - 1]
            if acc >= p:
                m_p = m
                break
        L = max(k_sel, m_p)
        for i in range(nk):
            mask[r, i] = rank[i] < L
    return mask


@pytest.mark.parametrize("N,d,bq,bk,k_frac,p,seed", [
    (200, 8, 32, 16, 0.2, 0.7, 31),     # 7 query blocks (last 8 tokens), 13 key blocks (last 8)
    (700, 16, 128, 64, 0.2, 0.6, 32),   # the video geometry's 2:1 block ratio, both tails 60 tokens
    (130, 8, 16, 64, 0.34, 0.7, 33),    # key blocks wider than query blocks
])
def test_build_mask_wiring_by_brute_force(N, d, bq, bk, k_frac, p, seed):
    """build_mask's pooling sizes (Q by bq, K by bk), its default scale 1/sqrt(d)
    and its per-row selection, against scalar loops on ragged bq != bk shapes;
    the rows' cumulative sums are checked to stay clear of p so rounding order
    cannot decide them."""
    rng = _rng(seed)
    q = rng.standard_normal((N, d)) * 2.0 + rng.standard_normal(d)
    k = rng.standard_normal((N, d)) + rng.standard_normal(d)
    out = oracle.build_mask(q, k, bq, bk, k_frac, p)
    want = _brute_force_mask(q, k, bq, bk, k_frac, p, 1.0 / math.sqrt(d))
    assert out["mask"].shape == want.shape == (-(-N // bq), -(-N // bk))
    s = out["s"]
    for r in range(s.shape[0]):
        csum = np.cumsum(oracle.block_softmax(s[r])[oracle.descending_order(s[r])])
        assert np.abs(csum - p).min() > 1e-9
    assert (out["mask"] == want).all()
    # the mask depends on the scale: 1/d in place of 1/sqrt(d) changes some row here
    assert (_brute_force_mask(q, k, bq, bk, k_frac, p, 1.0 / d) != want).any()


# ---------------------------------------------------------------- golden regression
def test_tiny_workload_masks_match_golden():
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "tiny_kv_lists.txt")
    want = {}
    with open(path) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            h, r, cnt, idx = line.split(":")
            want[(int(h), int(r))] = (int(cnt), [int(t) for t in idx.split()])
    wl = WORKLOADS["tiny"]
    x = make_inputs(wl, "cpu")
    for h in range(wl.H):
        out = oracle.build_mask(oracle.as_f64(x["q"][0, h]), oracle.as_f64(x["k"][0, h]),
                                wl.bq, wl.bk, wl.topk, wl.topp)
        idx, cnt = oracle.kv_lists(out["mask"])
        for r in range(idx.shape[0]):
            assert want[(h, r)] == (int(cnt[r]), idx[r, :cnt[r]].tolist())


# ---------------------------------------------------------------- tile scoring (Veda §2.1, §2.3)
def test_trip_pool_by_brute_force_loops():
    x = _rng(41).standard_normal((37, 5))
    desc = oracle.trip_pool(x, 8)
    assert desc.shape == (5, 15)
    for blk in range(5):
        rows = [t for t in range(37) if t // 8 == blk]
        for c in range(5):
            vals = [x[t, c] for t in rows]
            assert abs(desc[blk, c] - sum(vals) / len(vals)) < 1e-14
            assert desc[blk, 5 + c] == max(vals)
            assert desc[blk, 10 + c] == min(vals)
    means, _ = oracle.pool_blocks(x, 8)
    assert np.array_equal(desc[:, :5], means)


def test_tile_max_heatmap_by_brute_force_probabilities():
    """logH against the full attention matrix built entry by entry (exp and
    row sums by scalar loops), max-pooled over ragged tiles."""
    rng = _rng(42)
    N, d, bq, bk = 45, 6, 16, 8
    q, k = rng.standard_normal((N, d)) * 1.5, rng.standard_normal((N, d))
    scale = 1.0 / math.sqrt(d)
    P = np.zeros((N, N))
    for i in range(N):
        w = [math.exp(scale * sum(q[i, c] * k[j, c] for c in range(d))) for j in range(N)]
        z = sum(w)
        for j in range(N):
            P[i, j] = w[j] / z
    want = np.zeros((-(-N // bq), -(-N // bk)))
    for qb in range(want.shape[0]):
        for kb in range(want.shape[1]):
            want[qb, kb] = math.log(P[qb * bq:(qb + 1) * bq, kb * bk:(kb + 1) * bk].max())
    got = oracle.tile_max_heatmap(q, k, bq, bk)
    assert np.abs(got - want).max() < 1e-12
    assert (got <= 1e-15).all()
    # every row of each query block holds a probability >= 1/N somewhere
    assert (got.max(axis=1) >= math.log(1.0 / N) - 1e-12).all()
    # the first pass alone: LSE against torch.logsumexp
    lse = oracle.full_attention_lse(q, k)
    ref = torch.logsumexp(torch.from_numpy(scale * q @ k.T), dim=1).numpy()
    assert np.abs(lse - ref).max() < 1e-12
    # a subset of query blocks (the sparse teacher): the same rows, -inf elsewhere
    part = oracle.tile_max_heatmap(q, k, bq, bk, q_blocks=[1])
    assert np.array_equal(part[1], got[1]) and np.isneginf(part[[0, 2]]).all()


def test_mask_from_scores_is_the_hybrid_rule_per_row():
    rng = _rng(43)
    s = rng.standard_normal((6, 20)) * 2.0
    m = oracle.mask_from_scores(s, 0.1, 0.7)
    for r in range(6):
        assert (m[r] == oracle.hybrid_row(s[r], 0.1, 0.7)[0]).all()
    # on a head's own block scores it reproduces build_mask
    q, k = rng.standard_normal((300, 8)) * 2, rng.standard_normal((300, 8))
    out = oracle.build_mask(q, k, 32, 16, 0.2, 0.8)
    assert (oracle.mask_from_scores(out["s"], 0.2, 0.8) == out["mask"]).all()


# ---------------------------------------------------------------- permuted layouts (Veda §2.2, SparsePR §2C)
@pytest.mark.parametrize("grid,tile", [((3, 4, 6), (1, 2, 3)), ((5, 7, 9), (2, 4, 4)), ((2, 8, 8), (1, 8, 8))])
def test_tile_permutation_by_coordinates(grid, tile):
    """A bijection of the raster tokens in which each tile's tokens are
    consecutive, tiles follow the tile grid's raster order, and tokens inside a
    tile follow the raster order; checked from each token's coordinates."""
    T, Hh, W = grid
    perm = oracle.tile_permutation(grid, tile)
    N = T * Hh * W
    assert sorted(perm.tolist()) == list(range(N))
    coords = [(r // (Hh * W), (r // W) % Hh, r % W) for r in perm.tolist()]
    tiles = [(t // tile[0], y // tile[1], x // tile[2]) for t, y, x in coords]
    nt = (-(-T // tile[0]), -(-Hh // tile[1]), -(-W // tile[2]))
    tile_rank = [(a * nt[1] + b) * nt[2] + c for a, b, c in tiles]
    assert tile_rank == sorted(tile_rank)                      # tiles contiguous, in raster order
    for i in range(1, N):
        if tile_rank[i] == tile_rank[i - 1]:
            assert perm[i] > perm[i - 1]                       # raster order inside a tile
    if all(g % p == 0 for g, p in zip(grid, tile)):            # full tiles: fixed-size runs
        size = tile[0] * tile[1] * tile[2]
        assert all(tile_rank[i] == i // size for i in range(N))


def test_permuted_dense_attention_is_equivariant():
    """Dense attention commutes with a permutation of the tokens (softmax over
    all keys), so un-permuting the permuted call's output gives the plain one."""
    rng = _rng(44)
    grid = (2, 3, 5)
    N, d = 30, 6
    q, k, v = (rng.standard_normal((N, d)) for _ in range(3))
    perm = oracle.tile_permutation(grid, (1, 2, 2))
    op, _ = oracle.dense_attention(oracle.permute_rows(q, perm), oracle.permute_rows(k, perm),
                                   oracle.permute_rows(v, perm))
    o, _ = oracle.dense_attention(q, k, v)
    assert np.abs(oracle.unpermute_rows(op, perm) - o).max() < 1e-12
    assert np.array_equal(oracle.unpermute_rows(oracle.permute_rows(q, perm), perm), q)


# ---------------------------------------------------------------- backward pass
def test_masked_attention_bwd_against_torch_autograd_of_sdpa():
    """The oracle's hand-derived gradients against float64 torch.autograd through
    scaled_dot_product_attention with the expanded token mask (ragged blocks,
    bq != bk; every query row keeps at least one block)."""
    rng = _rng(51)
    N, d, bq, bk = 70, 8, 16, 8
    q, k, v = (rng.standard_normal((N, d)) for _ in range(3))
    q *= 2.0
    mask = rng.random((-(-N // bq), -(-N // bk))) < 0.4
    mask[np.arange(mask.shape[0]), rng.integers(0, mask.shape[1], mask.shape[0])] = True
    dout = rng.standard_normal((N, d))
    tok = np.zeros((N, N), dtype=bool)
    for i in range(N):
        for j in range(N):
            tok[i, j] = mask[i // bq, j // bk]
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(tq[None, None], tk[None, None], tv[None, None],
                                                         attn_mask=torch.from_numpy(tok)[None, None])[0, 0]
    o.backward(torch.from_numpy(dout))
    dq, dk, dv = oracle.masked_attention_bwd(q, k, v, mask, bq, bk, dout)
    for got, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        assert np.abs(got - ref.numpy()).max() < 1e-10


def test_masked_attention_bwd_empty_rows_pass_no_gradient():
    rng = _rng(52)
    N, d = 40, 4
    q, k, v, dout = (rng.standard_normal((N, d)) for _ in range(4))
    mask = np.ones((3, 5), dtype=bool)
    mask[1] = False
    dq, dk, dv = oracle.masked_attention_bwd(q, k, v, mask, 16, 8, dout)
    assert (dq[16:32] == 0).all()
    dout2 = dout.copy()
    dout2[16:32] = 123.0                     # the empty rows' upstream gradient changes nothing
    _, dk2, dv2 = oracle.masked_attention_bwd(q, k, v, mask, 16, 8, dout2)
    assert np.array_equal(dk, dk2) and np.array_equal(dv, dv2)


def _central_diff(f, x, h=1e-6):
    g = np.zeros_like(x)
    for idx in np.ndindex(x.shape):
        xp, xm = x.copy(), x.copy()
        xp[idx] += h
        xm[idx] -= h
        g[idx] = (f(xp) - f(xm)) / (2 * h)
    return g


def test_linear_and_blend_bwd_by_finite_differences():
    """Linear-branch and blend gradients against central differences of the
    oracle's forward (a scalar loss <dout, O>), on inputs that straddle zero."""
    rng = _rng(53)
    N, d = 9, 4
    q, k, v = (rng.standard_normal((N, d)) for _ in range(3))
    dout = rng.standard_normal((N, d))
    dq, dk, dv = oracle.linear_bwd(q, k, v, dout)
    loss = lambda q_, k_, v_: float((dout * oracle.linear_out(q_, *oracle.linear_state(k_, v_))).sum())
    assert np.abs(dq - _central_diff(lambda x: loss(x, k, v), q)).max() < 1e-6
    assert np.abs(dk - _central_diff(lambda x: loss(q, x, v), k)).max() < 1e-6
    assert np.abs(dv - _central_diff(lambda x: loss(q, k, x), v)).max() < 1e-6
    o_s, o_l, al = rng.standard_normal((N, d)), rng.standard_normal((N, d)), rng.random(d)
    ds, dl, da = oracle.blend_bwd(o_s, o_l, al, dout)
    bl = lambda a_, s_, l_: float((dout * oracle.blend(s_, l_, a_)).sum())
    assert np.abs(da - _central_diff(lambda x: bl(x, o_s, o_l), al)).max() < 1e-6
    assert np.abs(ds - _central_diff(lambda x: bl(al, x, o_l), o_s)).max() < 1e-6
    assert np.abs(dl - _central_diff(lambda x: bl(al, o_s, x), o_l)).max() < 1e-6
    x = np.linspace(-3, 3, 61)
    assert np.abs(oracle.phi_grad(x) - _central_diff(lambda t: oracle.phi(t).sum(), x)).max() < 1e-6


# ---------------------------------------------------------------- low-bit forward
def _e4m3_table():
    """Every finite non-negative E4M3 value, from the format's fields: exponent
    field E (bias 7, E = 0 subnormal), mantissa field M; E = 15, M = 7 is NaN."""
    vals = {}
    for E in range(16):
        for M in range(8):
            if E == 15 and M == 7:
                continue
            v = (M / 8) * 2.0 ** -6 if E == 0 else (1 + M / 8) * 2.0 ** (E - 7)
            vals[v] = M
    return sorted(vals.items())


def test_e4m3_fixed_points_and_ties_to_even():
    table = _e4m3_table()
    assert len(table) == 127 and table[-1][0] == 448.0 and table[1][0] == 2.0 ** -9
    vals = np.array([v for v, _ in table])
    assert np.array_equal(oracle.e4m3_round(vals), vals)
    assert np.array_equal(oracle.e4m3_round(-vals[1:]), -vals[1:])
    for (a, ma), (b, mb) in zip(table[:-1], table[1:]):
        mid = (a + b) / 2
        want = a if ma % 2 == 0 else b              # exactly one neighbour has an even mantissa
        assert oracle.e4m3_round(mid) == want, (a, b)
        assert oracle.e4m3_round(np.nextafter(mid, 0)) == a
        assert oracle.e4m3_round(np.nextafter(mid, np.inf)) == b
    assert oracle.e4m3_round(449.0) == 448.0 and oracle.e4m3_round(1e9) == 448.0
    assert oracle.e4m3_round(-1e9) == -448.0 and np.isnan(oracle.e4m3_round(np.nan))


def test_e4m3_matches_torch_float8_conversion():
    """torch's float32 -> float8_e4m3fn cast (a library routine) below its
    overflow threshold, over random magnitudes from the subnormals up."""
    rng = _rng(60)
    mag = np.exp2(rng.uniform(-12, 8.85, 200000))
    x = (mag * rng.choice([-1.0, 1.0], mag.shape)).astype(np.float32)
    x = x[np.abs(x) < 464]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(oracle.e4m3_round(x.astype(np.float64)), ref)


def test_quantize_fp8_head_scale_and_codes():
    rng = _rng(61)
    x = rng.standard_normal((300, 16)).astype(np.float32)
    x[17, 3] = -5.25                                   # the largest magnitude
    codes, s = oracle.quantize_fp8_head(x)
    assert s == float(np.float32(5.25) / np.float32(448))
    assert codes[17, 3] == -448.0 and np.abs(codes).max() == 448.0
    deq = codes * s
    big = np.abs(x) >= 2.0 ** -6 * s
    assert (np.abs(deq - x)[big] <= 2.0 ** -4 * np.abs(x)[big] * (1 + 1e-6)).all()
    assert (np.abs(deq - x)[~big] <= 2.0 ** -10 * s * (1 + 1e-6)).all()
    z, s0 = oracle.quantize_fp8_head(np.zeros((5, 4)))
    assert s0 == 1.0 and (z == 0).all()


def test_fp8_attention_exact_on_representable_inputs():
    """Integers in [-7, 7] with 7 present quantise exactly (s = 7/448 = 2^-6 and
    every 64 n, |n| <= 7, is an E4M3 value), so the low-bit attention equals the
    masked attention of the inputs themselves."""
    rng = _rng(62)
    N, d, bq, bk = 90, 8, 16, 8
    q, k, v = (rng.integers(-7, 8, (N, d)).astype(np.float64) for _ in range(3))
    for t in (q, k, v):
        t[0, 0] = 7.0
    mask = rng.random((-(-N // bq), -(-N // bk))) < 0.5
    mask[2] = False
    o8, l8 = oracle.fp8_masked_attention(q, k, v, mask, bq, bk, scale=0.05)
    o, l = oracle.masked_attention(q, k, v, mask, bq, bk, scale=0.05)
    assert np.array_equal(o8, o) and np.array_equal(l8, l)
    assert (o8[32:48] == 0).all() and np.isneginf(l8[32:48]).all()


def test_fp8_attention_within_quantisation_error():
    """On unit-variance inputs the low-bit attention stays near the
    full-precision one (each operand within 2^-4 relative)."""
    rng = _rng(63)
    N, d = 256, 32
    q, k, v = (rng.standard_normal((N, d)) for _ in range(3))
    mask = np.ones((4, 4), dtype=bool)
    o8, _ = oracle.fp8_masked_attention(q, k, v, mask, 64, 64)
    o, _ = oracle.dense_attention(q, k, v)
    err = np.abs(o8 - o)
    assert 0 < err.max() < 0.05 and err.mean() < 0.01
