"""fp64 oracle: block pooling, hybrid Top-k ∪ Top-p block mask, masked softmax
attention, the elu+1 linear branch and the alpha blend.

TEST INFRASTRUCTURE: imported only by tests, the smoke check and the bench's
CPU-baseline leg. Written from the pages' definitions, in their order; numpy
matmul, exp and a stable sort are the only library steps.

Parity pins (tests/test_oracle_pins.py) tie each function to something other
than itself: brute force on tiny inputs, closed forms, exhaustive subset search
for Top-p minimality, the Top-p count from the low end of the order, and
torch's float64 scaled_dot_product_attention for dense and masked attention.
row_threshold_info, which the GPU comparison uses to recognise near-ties, is
pinned with planted rows in tests/test_mask_comparator.py. The E4M3 rounding
of the low-bit forward is pinned by the format's own table of values (fixed
points, ties to even, saturation) and by torch's float8_e4m3fn cast; the
low-bit attention by inputs that quantise exactly.
"""
from __future__ import annotations

import math

import numpy as np

# Near-tie band of the GPU comparison: blocks exchanged across the selection cut
# whose scores lie within this distance of each other, or a row length decided
# where the cumulative probability lies within it of p, may legitimately differ
# between an fp32 GPU evaluation and this fp64 one; such cases are reported.
NEAR_TIE_TOL = 1e-6


def as_f64(x) -> np.ndarray:
    """Exact conversion of a bf16/fp32 torch tensor or numpy array to float64."""
    if hasattr(x, "detach"):
        import torch
        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


# --------------------------------------------------------------------------
# Mask prediction: SLA2 提案手法 ① (mean pooling of Q and K per block) and
# SpargeAttention2 §2(1) (hybrid Top-k + Top-p per attention row).
# --------------------------------------------------------------------------

def pool_blocks(x: np.ndarray, b: int) -> tuple[np.ndarray, np.ndarray]:
    """Mean of the rows of x [N, d] over consecutive blocks of b tokens.

    The last block may be partial; it is averaged over its valid tokens only.
    Returns (means [ceil(N/b), d], counts [ceil(N/b)]).
    """
    N, d = x.shape
    n = -(-N // b)
    means = np.empty((n, d), dtype=np.float64)
    counts = np.empty(n, dtype=np.int64)
    for i in range(n):
        rows = x[i * b:min(N, (i + 1) * b)]
        counts[i] = rows.shape[0]
        means[i] = rows.sum(axis=0) / rows.shape[0]
    return means, counts


def block_scores(q_pool: np.ndarray, k_pool: np.ndarray, scale: float) -> np.ndarray:
    """s[qb, kb] = scale * <mean q of block qb, mean k of block kb>."""
    return scale * (q_pool @ k_pool.T)


def block_softmax(s: np.ndarray) -> np.ndarray:
    """Softmax of each row of block scores over all key blocks of that row."""
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / e.sum(axis=-1, keepdims=True)


def topk_count(k_frac: float, n_kb: int) -> int:
    """Number of blocks Top-k keeps in a row: ceil(k * n_kb), at least 1.

    The 1e-9 guard keeps exact products such as 0.1 * 10 from rounding up.
    """
    return int(min(n_kb, max(1, math.ceil(k_frac * n_kb - 1e-9))))


def descending_order(s_row: np.ndarray) -> np.ndarray:
    """Key blocks by score, largest first; equal scores keep the lower index first."""
    return np.argsort(-s_row, kind="stable")


def topp_count(p_sorted: np.ndarray, p: float) -> int:
    """Smallest m >= 1 whose m largest probabilities sum to at least p.

    p >= 1 asks for the whole distribution, i.e. every block. If rounding keeps
    the running sum below p, every block is taken.
    """
    n = p_sorted.shape[0]
    if p >= 1.0:
        return n
    csum = 0.0
    for m in range(1, n + 1):
        csum += p_sorted[m - 1]
        if csum >= p:
            return m
    return n


def topk_set(s_row: np.ndarray, k_frac: float) -> set:
    order = descending_order(s_row)
    return set(order[:topk_count(k_frac, s_row.shape[0])].tolist())


def topp_set(s_row: np.ndarray, p: float) -> set:
    order = descending_order(s_row)
    P = block_softmax(s_row)
    return set(order[:topp_count(P[order], p)].tolist())


def hybrid_row(s_row: np.ndarray, k_frac: float, p: float):
    """Hybrid mask of one query-block row: Top-k ∪ Top-p.

    Both sets are prefixes of the same descending order, so their union is the
    prefix of length L = max(K_sel, m_p). Returns (bool mask [n_kb], L, K_sel, m_p).
    """
    n = s_row.shape[0]
    order = descending_order(s_row)
    P = block_softmax(s_row)
    k_sel = topk_count(k_frac, n)
    m_p = topp_count(P[order], p)
    L = max(k_sel, m_p)
    mask = np.zeros(n, dtype=bool)
    mask[order[:L]] = True
    union = set(order[:k_sel].tolist()) | set(order[:m_p].tolist())
    assert union == set(np.nonzero(mask)[0].tolist())
    return mask, L, k_sel, m_p


def build_mask(q: np.ndarray, k: np.ndarray, bq: int, bk: int, k_frac: float, p: float,
               scale: float | None = None):
    """Block mask for one head from Q, K [N, d].

    Returns dict(mask [n_qb, n_kb] bool, s scores, P probabilities, L, k_sel, m_p).
    """
    d = q.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    qp, _ = pool_blocks(q, bq)
    kp, _ = pool_blocks(k, bk)
    s = block_scores(qp, kp, scale)
    n_qb, n_kb = s.shape
    mask = np.zeros((n_qb, n_kb), dtype=bool)
    L = np.zeros(n_qb, dtype=np.int64)
    ks = np.zeros(n_qb, dtype=np.int64)
    mp = np.zeros(n_qb, dtype=np.int64)
    for r in range(n_qb):
        mask[r], L[r], ks[r], mp[r] = hybrid_row(s[r], k_frac, p)
    return {"mask": mask, "s": s, "P": block_softmax(s), "L": L, "k_sel": ks, "m_p": mp,
            "q_pool": qp, "k_pool": kp}


def row_threshold_info(s_row: np.ndarray, k_frac: float, p: float, tol: float = NEAR_TIE_TOL):
    """Describe how close a row's decision is to a tie.

    Returns dict with the order, L, the cumulative sums, the blocks whose score is
    within tol of the last kept or first dropped score (score ties at the cut), and
    the ranks r where the cumulative sum up to r lies within tol of p (cumsum ties).
    """
    order = descending_order(s_row)
    P = block_softmax(s_row)[order]
    n = s_row.shape[0]
    _, L, k_sel, m_p = hybrid_row(s_row, k_frac, p)
    csum = np.cumsum(P)
    cut_scores = [s_row[order[L - 1]]]
    if L < n:
        cut_scores.append(s_row[order[L]])
    near_blocks = set()
    for c in cut_scores:
        near_blocks |= set(np.nonzero(np.abs(s_row - c) <= tol)[0].tolist())
    near_ranks = set(np.nonzero(np.abs(csum - p) <= tol)[0].tolist()) if p < 1.0 else set()
    return {"order": order, "L": L, "k_sel": k_sel, "m_p": m_p, "csum": csum,
            "near_blocks": near_blocks, "near_ranks": near_ranks}


def kv_lists(mask: np.ndarray):
    """Compacted form of a block mask: ascending kept key-block indices per row."""
    n_qb, n_kb = mask.shape
    kv_idx = np.full((n_qb, n_kb), -1, dtype=np.int64)
    kv_cnt = np.zeros(n_qb, dtype=np.int64)
    for r in range(n_qb):
        idx = np.nonzero(mask[r])[0]
        kv_cnt[r] = idx.shape[0]
        kv_idx[r, :idx.shape[0]] = idx
    return kv_idx, kv_cnt


def mask_from_lists(kv_idx: np.ndarray, kv_cnt: np.ndarray, n_kb: int) -> np.ndarray:
    n_qb = kv_cnt.shape[0]
    mask = np.zeros((n_qb, n_kb), dtype=bool)
    for r in range(n_qb):
        mask[r, kv_idx[r, :kv_cnt[r]]] = True
    return mask


# --------------------------------------------------------------------------
# Attention: SpargeAttention2 §2(3) — exact softmax attention restricted to the
# kept (query-block, key-block) tiles; masked tiles contribute nothing.
# --------------------------------------------------------------------------

def masked_attention(q, k, v, mask, bq, bk, scale=None, rows=None):
    """O[i] = sum_j softmax_j(scale * q_i . k_j) v_j over keys j in kept blocks.

    rows: iterable of query indices to evaluate (default: all). Returns
    (O [len(rows), d], LSE [len(rows)]); a row with no kept key gives O = 0 and
    LSE = -inf. Rows of one query block share that block's kept keys, so they
    are evaluated together: one logits matrix, then each row's own max,
    exponentials and sum.
    """
    N, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    rows = np.arange(N) if rows is None else np.asarray(list(rows), dtype=np.int64)
    out = np.zeros((rows.shape[0], d), dtype=np.float64)
    lse = np.full(rows.shape[0], -np.inf, dtype=np.float64)
    qb_of_row = rows // bq
    for qb in np.unique(qb_of_row):
        at = np.nonzero(qb_of_row == qb)[0]
        kept = np.nonzero(mask[qb])[0]
        if kept.shape[0] == 0:
            continue
        keys = np.concatenate([np.arange(kb * bk, min(N, (kb + 1) * bk)) for kb in kept])
        logits = scale * (q[rows[at]] @ k[keys].T)          # [rows of this block, kept keys]
        m = logits.max(axis=1, keepdims=True)
        w = np.exp(logits - m)
        z = w.sum(axis=1, keepdims=True)
        out[at] = (w @ v[keys]) / z
        lse[at] = m[:, 0] + np.log(z[:, 0])
    return out, lse


def dense_attention(q, k, v, scale=None):
    N, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    logits = scale * (q @ k.T)
    m = logits.max(axis=1, keepdims=True)
    w = np.exp(logits - m)
    z = w.sum(axis=1, keepdims=True)
    return (w @ v) / z, (m + np.log(z))[:, 0]


# --------------------------------------------------------------------------
# Linear branch (SALAD §2.1, SLA2 提案手法 ②): phi(x) = elu(x) + 1,
# O_l[i] = phi(q_i)^T S / phi(q_i)^T z with S = sum_j phi(k_j) v_j^T and
# z = sum_j phi(k_j) over all N keys; then O = alpha * O_s + (1 - alpha) * O_l.
# --------------------------------------------------------------------------

def phi(x: np.ndarray) -> np.ndarray:
    return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def linear_state(k: np.ndarray, v: np.ndarray):
    fk = phi(k)
    return fk.T @ v, fk.sum(axis=0)


def linear_out(q: np.ndarray, S: np.ndarray, z: np.ndarray) -> np.ndarray:
    fq = phi(q)
    return (fq @ S) / (fq @ z)[:, None]


def blend(o_s: np.ndarray, o_l: np.ndarray, alpha_h: np.ndarray) -> np.ndarray:
    return alpha_h[None, :] * o_s + (1.0 - alpha_h[None, :]) * o_l


# --------------------------------------------------------------------------
# Tile scoring from the full attention map (Veda §2.1 and §2.3): TripPool
# descriptors (mean, max and min of each block, per channel), and the
# reference heatmap that max-pools the full attention probabilities over each
# (query block, key block) tile, computed in two passes. Either kind of block
# score can feed the same hybrid Top-k ∪ Top-p selection.
# --------------------------------------------------------------------------

def trip_pool(x: np.ndarray, b: int) -> np.ndarray:
    """TripPool descriptor of each block of b tokens of x [N, d]: the mean, the
    maximum and the minimum over the block's valid tokens, per channel,
    concatenated as [mean | max | min] -> [ceil(N/b), 3d]."""
    N, d = x.shape
    n = -(-N // b)
    out = np.empty((n, 3 * d), dtype=np.float64)
    for i in range(n):
        rows = x[i * b:min(N, (i + 1) * b)]
        out[i, :d] = rows.sum(axis=0) / rows.shape[0]
        out[i, d:2 * d] = rows.max(axis=0)
        out[i, 2 * d:] = rows.min(axis=0)
    return out


def full_attention_lse(q: np.ndarray, k: np.ndarray, scale=None, rows=None) -> np.ndarray:
    """First pass: the natural-log log-sum-exp of each query row's logits
    scale * q_i . k_j over all N keys (the full softmax's normaliser)."""
    N, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    rows = np.arange(N) if rows is None else np.asarray(rows, dtype=np.int64)
    logits = scale * (q[rows] @ k.T)
    m = logits.max(axis=1, keepdims=True)
    return (m + np.log(np.exp(logits - m).sum(axis=1, keepdims=True)))[:, 0]


def tile_max_heatmap(q: np.ndarray, k: np.ndarray, bq: int, bk: int, scale=None, q_blocks=None):
    """Second pass: for each (query block, key block) tile, the log of the
    largest full-attention probability inside it,
        logH[qb, kb] = max over i in qb, j in kb of (scale * q_i . k_j - LSE_i),
    with LSE from the first pass (valid tokens only). q_blocks: the query
    blocks to evaluate (default all); the other rows are -inf."""
    N, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    n_qb, n_kb = -(-N // bq), -(-N // bk)
    q_blocks = range(n_qb) if q_blocks is None else q_blocks
    out = np.full((n_qb, n_kb), -np.inf, dtype=np.float64)
    for qb in q_blocks:
        rows = np.arange(qb * bq, min(N, (qb + 1) * bq))
        lse = full_attention_lse(q, k, scale, rows)
        logp = scale * (q[rows] @ k.T) - lse[:, None]            # [rows, N] log probabilities
        for kb in range(n_kb):
            out[qb, kb] = logp[:, kb * bk:min(N, (kb + 1) * bk)].max()
    return out


def mask_from_scores(s: np.ndarray, k_frac: float, p: float) -> np.ndarray:
    """The hybrid Top-k ∪ Top-p rule applied to each row of given block scores
    (softmax over the row, SpargeAttention2 §2(1)); with s = logH the row
    distribution is the max-pooled probabilities normalised over the row."""
    mask = np.zeros(s.shape, dtype=bool)
    for r in range(s.shape[0]):
        mask[r] = hybrid_row(s[r], k_frac, p)[0]
    return mask


# --------------------------------------------------------------------------
# Permuted token layouts (Veda §2.2: per-head tilings (p_t, p_h, p_w) of the
# latent grid; SparsePR §2C: tokens reordered into a contiguous group-major
# layout before the block-sparse call). Blocks of the sparse path are then
# runs of consecutive tokens of the permuted sequence.
# --------------------------------------------------------------------------

def tile_permutation(grid, tile) -> np.ndarray:
    """Token order that visits the (T, Hh, W) raster grid tile by tile: tiles
    of (p_t, p_h, p_w) tokens in raster order of the tile grid (edge tiles
    may be partial), tokens inside a tile in raster order. perm[i] is the
    raster index of the token placed at position i."""
    T, Hh, W = grid
    pt, ph, pw = tile
    perm = []
    for t0 in range(0, T, pt):
        for y0 in range(0, Hh, ph):
            for x0 in range(0, W, pw):
                for t in range(t0, min(T, t0 + pt)):
                    for y in range(y0, min(Hh, y0 + ph)):
                        for x in range(x0, min(W, x0 + pw)):
                            perm.append((t * Hh + y) * W + x)
    return np.asarray(perm, dtype=np.int64)


def permute_rows(x: np.ndarray, perm: np.ndarray) -> np.ndarray:
    """Rows of x in the permuted order: y[i] = x[perm[i]]."""
    return x[perm]


def unpermute_rows(y: np.ndarray, perm: np.ndarray) -> np.ndarray:
    """Inverse of permute_rows: x[perm[i]] = y[i]."""
    x = np.empty_like(y)
    x[perm] = y
    return x


# --------------------------------------------------------------------------
# Backward pass (SpargeAttention2 §2(2): the sparse attention is made
# trainable and fine-tuned by distillation, which needs gradients through the
# sparse path; SLA2 提案手法 ③: the backward pass runs in full precision).
# Gradients of the forward definitions above by the chain rule.
# --------------------------------------------------------------------------

def masked_attention_bwd(q, k, v, mask, bq, bk, dout, scale=None):
    """(dq, dk, dv) of O = masked_attention(q, k, v, mask) for the upstream
    gradient dout [N, d]. Per query block, with P the softmax of
    scale * q_i . k_j over the kept keys and O = P v:
        dv += P^T dout,  dP = dout v^T,  dS = P * (dP - rowsum(dout * O)),
        dq += scale * dS k,  dk += scale * dS^T q.
    Rows with no kept key have O = 0 and pass no gradient."""
    N, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for qb in range(mask.shape[0]):
        rows = np.arange(qb * bq, min(N, (qb + 1) * bq))
        kept = np.nonzero(mask[qb])[0]
        if kept.shape[0] == 0:
            continue
        keys = np.concatenate([np.arange(kb * bk, min(N, (kb + 1) * bk)) for kb in kept])
        logits = scale * (q[rows] @ k[keys].T)
        w = np.exp(logits - logits.max(axis=1, keepdims=True))
        P = w / w.sum(axis=1, keepdims=True)
        O = P @ v[keys]
        dP = dout[rows] @ v[keys].T
        dS = P * (dP - (dout[rows] * O).sum(axis=1, keepdims=True))
        dq[rows] += scale * (dS @ k[keys])
        dk[keys] += scale * (dS.T @ q[rows])          # keys of one row are distinct
        dv[keys] += P.T @ dout[rows]
    return dq, dk, dv


def phi_grad(x: np.ndarray) -> np.ndarray:
    """d phi / dx for phi = elu + 1: 1 above zero, e^x at or below."""
    return np.where(x > 0, 1.0, np.exp(np.minimum(x, 0.0)))


def linear_bwd(q, k, v, dout_l):
    """(dq, dk, dv) of O_l = phi(q) S / phi(q) . z with S = sum_j phi(k_j) v_j^T
    and z = sum_j phi(k_j), for the upstream gradient dout_l [N, d]:
        dnum = dout_l / den,  dden = -rowsum(dout_l * O_l) / den,
        dphi(q) = dnum S^T + dden z^T,  dS = phi(q)^T dnum,  dz = phi(q)^T dden,
        dphi(k) = v dS^T + dz,  dv = phi(k) dS,
    then dq = dphi(q) * phi'(q) and dk = dphi(k) * phi'(k)."""
    fq, fk = phi(q), phi(k)
    S, z = fk.T @ v, fk.sum(axis=0)
    den = fq @ z
    O = (fq @ S) / den[:, None]
    dnum = dout_l / den[:, None]
    dden = -(dout_l * O).sum(axis=1) / den
    dfq = dnum @ S.T + dden[:, None] * z[None, :]
    dS = fq.T @ dnum
    dz = fq.T @ dden
    dfk = v @ dS.T + dz[None, :]
    dv = fk @ dS
    return dfq * phi_grad(q), dfk * phi_grad(k), dv


def blend_bwd(o_s, o_l, alpha_h, dout):
    """(do_s, do_l, dalpha) of O = alpha * O_s + (1 - alpha) * O_l: alpha * dout,
    (1 - alpha) * dout, and the sum over tokens of dout * (O_s - O_l)."""
    return alpha_h[None, :] * dout, (1.0 - alpha_h[None, :]) * dout, (dout * (o_s - o_l)).sum(axis=0)


# --------------------------------------------------------------------------
# Low-bit forward (SLA2 提案手法 ③: the forward pass quantises queries, keys
# and values to a low-bit format and computes with them; the backward stays in
# full precision). The pages name neither the format nor the scale granularity.
# Reading: 8-bit floats in the E4M3 layout (1 sign bit, 4 exponent bits with
# bias 7, 3 mantissa bits, no infinities, largest finite value 448), one fp32
# scale per (batch, head) and tensor, s = amax / 448, codes = E4M3(x * r) with
# r = 448 / amax, both in fp32, the product rounded to fp32 and then to E4M3 by
# round-to-nearest-even with saturation at +-448. The low-bit attention is then
# the masked attention above on the dequantised tensors codes * s.
# --------------------------------------------------------------------------

E4M3_MAX = 448.0


def e4m3_round(x) -> np.ndarray:
    """Nearest E4M3 value (ties to even mantissa), saturated to +-448.

    Normal numbers 2^e * 1.mmm for e in [-6, 8] are spaced 2^(e-3) apart;
    below 2^-6 the subnormals m/8 * 2^-6 are spaced 2^-9 apart, and zero keeps
    its sign. NaN stays NaN.
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, ex = np.frexp(a)                      # a = f * 2^ex with f in [0.5, 1)
    e = np.maximum(ex - 1, -6)               # binade exponent, clamped to the subnormal range
    quantum = np.ldexp(1.0, e - 3)
    r = np.round(a / quantum) * quantum      # np.round: ties to even
    r = np.minimum(r, E4M3_MAX)
    return np.where(np.isnan(x), np.nan, np.copysign(r, x))


def quantize_fp8_head(x) -> tuple[np.ndarray, float]:
    """One (batch, head) slice [N, d] -> (E4M3 code values as float64, fp32 scale).

    s = amax / 448 and r = 448 / amax in fp32 (both 1 when the slice is all
    zeros); each code is the E4M3 rounding of the fp32 product x * r.
    """
    x32 = np.asarray(x, dtype=np.float32)
    amax = np.float32(np.max(np.abs(x32))) if x32.size else np.float32(0)
    if amax > 0:
        s = np.float32(amax) / np.float32(E4M3_MAX)
        r = np.float32(E4M3_MAX) / np.float32(amax)
    else:
        s = r = np.float32(1.0)
    codes = e4m3_round((x32 * r).astype(np.float64))
    return codes, float(s)


def fp8_masked_attention(q, k, v, mask, bq, bk, scale=None, rows=None):
    """Masked attention on the per-head E4M3 quantisations of q, k and v.

    Returns (O, LSE) as masked_attention does, computed in fp64 from the
    dequantised tensors codes * s.
    """
    qc, sq = quantize_fp8_head(q)
    kc, sk = quantize_fp8_head(k)
    vc, sv = quantize_fp8_head(v)
    return masked_attention(qc * sq, kc * sk, vc * sv, mask, bq, bk, scale=scale, rows=rows)
