"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Masks must equal the oracle's except at reported near-ties; attention, linear
branch and blend outputs computed on the oracle's own mask must stay within
max |err| <= 2e-2 and mean |err| <= 2e-3.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_softmax_b200.workloads import WORKLOADS, make_inputs, random_qkv
from gpu_helpers import MAX_ABS, MEAN_ABS, assert_close, compare_mask_rows, sample_rows

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _f64(t):
    return oracle.as_f64(t)


def _oracle_head_mask(q, k, b, h, bq, bk, topk, topp):
    return oracle.build_mask(_f64(q[b, h]), _f64(k[b, h]), bq, bk, topk, topp)


def _assert_same_lists(a, b):
    assert torch.equal(a["kv_cnt"], b["kv_cnt"])
    n = a["kv_idx"].shape[-1]
    valid = torch.arange(n, device=a["kv_idx"].device) < a["kv_cnt"].unsqueeze(-1)
    assert torch.equal(torch.where(valid, a["kv_idx"], -1), torch.where(valid, b["kv_idx"], -1))


def _check_masks(sa, q, k, bq, bk, topk, topp, heads):
    B, H, N, d = q.shape
    out = sa.sa_build_mask(q, k, bq, bk, topk, topp, want_mask=True, want_pools=True)
    # without the u8 mask the selection emits the kept list from its candidate
    # set instead of a full-row pass: the lists must be the same
    _assert_same_lists(out, sa.sa_build_mask(q, k, bq, bk, topk, topp))
    torch.cuda.synchronize()
    idx = out["kv_idx"].cpu().numpy()
    cnt = out["kv_cnt"].cpu().numpy()
    msk = out["mask"].cpu().numpy().astype(bool)
    totals = {"exact": 0, "score_tie": 0, "cumsum_tie": 0}
    ora_masks = {}
    for (b, h) in heads:
        ref = _oracle_head_mask(q, k, b, h, bq, bk, topk, topp)
        ora_masks[(b, h)] = ref
        # pooled means: fp32 sums of bf16 values
        assert_close(out["q_pool"][b, h].cpu().numpy(), ref["q_pool"], "q_pool", 1e-5, 1e-6)
        assert_close(out["k_pool"][b, h].cpu().numpy(), ref["k_pool"], "k_pool", 1e-5, 1e-6)
        st = compare_mask_rows(idx[b, h], cnt[b, h], ref["s"], topk, topp)
        assert not st["bad"], f"head {(b, h)}: rows differ beyond ties: {st['bad'][:3]}"
        for key in totals:
            totals[key] += st[key]
        # kv lists are ascending and agree with the uint8 mask
        for r in range(idx.shape[2]):
            row = idx[b, h, r, :cnt[b, h, r]]
            assert (np.diff(row) > 0).all()
            assert set(row.tolist()) == set(np.nonzero(msk[b, h, r])[0].tolist())
    return out, ora_masks, totals


def _oracle_attention_rows(q, k, v, mask, b, h, bq, bk, rows):
    return oracle.masked_attention(_f64(q[b, h]), _f64(k[b, h]), _f64(v[b, h]), mask, bq, bk, rows=rows)


# ------------------------------------------------------------------ tiny: everything, every row
def test_tiny_workload_full(cuda_lib):
    sa = cuda_lib
    wl = WORKLOADS["tiny"]
    x = make_inputs(wl, "cpu")
    q, k, v = (x[n].to(DEV) for n in ("q", "k", "v"))
    heads = [(0, h) for h in range(wl.H)]
    out, ora, totals = _check_masks(sa, q, k, wl.bq, wl.bk, wl.topk, wl.topp, heads)
    print("tiny mask rows:", totals)
    ext = torch.zeros(1, wl.H, wl.n_qb, wl.n_kb, dtype=torch.uint8)
    for (b, h), ref in ora.items():
        ext[b, h] = torch.from_numpy(ref["mask"].astype(np.uint8))
    o, lse = sa.sa_sparse_attn_fwd(q, k, v, wl.bq, wl.bk, ext_mask=ext.to(DEV), want_lse=True)
    o_list = sa.sa_sparse_attn_fwd(q, k, v, wl.bq, wl.bk, kv_idx=out["kv_idx"], kv_cnt=out["kv_cnt"])
    torch.cuda.synchronize()
    for (b, h), ref in ora.items():
        ro, rl = _oracle_attention_rows(q.cpu(), k.cpu(), v.cpu(), ref["mask"], b, h, wl.bq, wl.bk, None)
        assert_close(o[b, h].float().cpu().numpy(), ro, f"O head {h}")
        assert_close(lse[b, h].cpu().numpy(), rl, f"LSE head {h}", 1e-2, 1e-3)
        same = (out["mask"][b, h].cpu().numpy().astype(bool) == ref["mask"]).all(axis=1)
        rows_same = np.repeat(same, wl.bq)[:wl.N]
        assert torch.equal(o_list[b, h][torch.from_numpy(rows_same).to(DEV)],
                           o[b, h][torch.from_numpy(rows_same).to(DEV)])
    sa.sa_device_status()


def test_tiny_golden_lists(cuda_lib):
    """The GPU lists reproduce the stored oracle fixture for the tiny workload."""
    import os
    sa = cuda_lib
    wl = WORKLOADS["tiny"]
    x = make_inputs(wl, "cpu")
    out = sa.sa_build_mask(x["q"].to(DEV), x["k"].to(DEV), wl.bq, wl.bk, wl.topk, wl.topp)
    idx, cnt = out["kv_idx"].cpu().numpy(), out["kv_cnt"].cpu().numpy()
    path = os.path.join(os.path.dirname(__file__), "golden", "tiny_kv_lists.txt")
    mism = 0
    for line in open(path):
        if line.startswith("#"):
            continue
        h, r, c, rest = line.split(":")
        want = [int(t) for t in rest.split()]
        got = idx[0, int(h), int(r), :cnt[0, int(h), int(r)]].tolist()
        mism += got != want
    assert mism == 0


# ------------------------------------------------------------------ ragged / edge shapes
@pytest.mark.parametrize("N,d,bq,H", [(1, 64, 64, 1), (65, 128, 128, 2), (200, 128, 64, 1),
                                      (333, 64, 128, 3), (1000, 128, 128, 2), (4099, 128, 128, 1)])
def test_ragged_shapes(cuda_lib, N, d, bq, H):
    sa = cuda_lib
    bk = 64
    q, k, v = random_qkv(1, H, N, d, seed=N * 7 + d, device=DEV)
    q = (q.float() * 3.0).to(torch.bfloat16)  # sharper block scores
    heads = [(0, h) for h in range(H)]
    out, ora, _ = _check_masks(sa, q, k, bq, bk, 0.2, 0.8, heads)
    ext = torch.zeros(1, H, -(-N // bq), -(-N // bk), dtype=torch.uint8)
    for (b, h), ref in ora.items():
        ext[b, h] = torch.from_numpy(ref["mask"].astype(np.uint8))
    o, lse = sa.sa_sparse_attn_fwd(q, k, v, bq, bk, ext_mask=ext.to(DEV), want_lse=True)
    torch.cuda.synchronize()
    for (b, h), ref in ora.items():
        ro, rl = _oracle_attention_rows(q.cpu(), k.cpu(), v.cpu(), ref["mask"], b, h, bq, bk, None)
        assert_close(o[b, h].float().cpu().numpy(), ro, f"O N={N}")
        assert_close(lse[b, h].cpu().numpy(), rl, f"LSE N={N}", 1e-2, 1e-3)
    sa.sa_device_status()


def test_empty_rows_and_all_ones(cuda_lib):
    sa = cuda_lib
    N, d, bq, bk, H = 300, 128, 128, 64, 2
    q, k, v = random_qkv(1, H, N, d, seed=5, device=DEV)
    nqb, nkb = -(-N // bq), -(-N // bk)
    ext = torch.ones(1, H, nqb, nkb, dtype=torch.uint8)
    ext[0, 0, 1] = 0                              # a row with no kept block
    o, lse = sa.sa_sparse_attn_fwd(q, k, v, bq, bk, ext_mask=ext.to(DEV), want_lse=True)
    torch.cuda.synchronize()
    assert (o[0, 0, bq:2 * bq] == 0).all()
    assert torch.isneginf(lse[0, 0, bq:2 * bq]).all()
    ref, rl = oracle.dense_attention(_f64(q[0, 1]), _f64(k[0, 1]), _f64(v[0, 1]))
    assert_close(o[0, 1].float().cpu().numpy(), ref, "all-ones = dense")
    # k = 100% gives the all-ones mask through the builder too
    m = sa.sa_build_mask(q, k, bq, bk, 1.0, 0.5)
    assert (m["kv_cnt"] == nkb).all()
    m = sa.sa_build_mask(q, k, bq, bk, 0.01, 1.0)
    assert (m["kv_cnt"] == nkb).all()
    # dense entry point = all-ones mask
    od, ld = sa.sa_dense_attn_fwd(q, k, v, bq, want_lse=True)
    ref0, rl0 = oracle.dense_attention(_f64(q[0, 0]), _f64(k[0, 0]), _f64(v[0, 0]))
    assert_close(od[0, 0].float().cpu().numpy(), ref0, "dense entry point")
    assert_close(ld[0, 0].cpu().numpy(), rl0, "dense LSE", 1e-2, 1e-3)
    sa.sa_device_status()


def test_uniform_scores_tie_order(cuda_lib):
    """All-equal block scores: every block ties, lower index first."""
    sa = cuda_lib
    N, d, H = 1024, 64, 1
    q = torch.zeros(1, H, N, d, dtype=torch.bfloat16, device=DEV)
    _, k, v = random_qkv(1, H, N, d, seed=9, device=DEV)
    m = sa.sa_build_mask(q, k, 64, 64, 0.1, 0.5)
    cnt = m["kv_cnt"].cpu().numpy()
    idx = m["kv_idx"].cpu().numpy()
    # P = 1/16 each: the smallest m with m/16 >= 0.5 is 8 (exact in binary)
    assert (cnt == 8).all()
    assert (idx[0, 0, :, :8] == np.arange(8)).all()


# ------------------------------------------------------------------ both mask builders on small cases
@pytest.mark.parametrize("builder", ["matrix", "candidates"])
def test_each_mask_builder(cuda_lib, builder, monkeypatch):
    """The score-matrix and the candidate builder, forced, on cases the size
    rule would send to the other one: the tiny workload and ragged shapes
    against the oracle (every head), all-equal scores (every block ties),
    and a 1.3B-480p-shaped head group whose lists must also equal the other
    builder's except at reported near-ties."""
    sa = cuda_lib
    monkeypatch.setenv("SA_MASK_BUILDER", builder)
    wl = WORKLOADS["tiny"]
    x = make_inputs(wl, "cpu")
    _, _, totals = _check_masks(sa, x["q"].to(DEV), x["k"].to(DEV), wl.bq, wl.bk, wl.topk, wl.topp,
                                [(0, h) for h in range(wl.H)])
    print(builder, "tiny mask rows:", totals)
    for N, d, bq, H in [(200, 128, 64, 1), (4099, 128, 128, 2)]:
        q, k, _ = random_qkv(1, H, N, d, seed=N * 7 + d, device=DEV)
        q = (q.float() * 3.0).to(torch.bfloat16)
        _check_masks(sa, q, k, bq, 64, 0.2, 0.8, [(0, h) for h in range(H)])
    # all-equal scores: P = 1/16 each, Top-p 0.5 keeps the 8 lowest blocks
    q = torch.zeros(1, 1, 1024, 64, dtype=torch.bfloat16, device=DEV)
    _, k, _ = random_qkv(1, 1, 1024, 64, seed=9, device=DEV)
    m = sa.sa_build_mask(q, k, 64, 64, 0.1, 0.5)
    assert (m["kv_cnt"].cpu().numpy() == 8).all()
    assert (m["kv_idx"].cpu().numpy()[0, 0, :, :8] == np.arange(8)).all()
    # 4 heads of the 1.3B-480p geometry against the oracle
    wl = WORKLOADS["wan13b_480p"]
    x = make_inputs(wl, DEV)
    q, k = x["q"][:, :4].contiguous(), x["k"][:, :4].contiguous()
    _, _, totals = _check_masks(sa, q, k, wl.bq, wl.bk, wl.topk, wl.topp, [(0, 0), (0, 3)])
    print(builder, "1.3B-480p mask rows:", totals)
    sa.sa_device_status()


def test_candidate_hand_back_all_rows(cuda_lib, monkeypatch):
    """All-equal scores on 1,182-block rows under the candidate builder: every
    threshold count is 0 or 1,182, above the lists' capacity, so every row is
    handed back to the score-matrix selection. P = 1/1182 each, so Top-p 0.85
    keeps the smallest m with m/1182 >= 0.85, the 1005 lowest blocks."""
    sa = cuda_lib
    monkeypatch.setenv("SA_MASK_BUILDER", "candidates")
    N, d = 75600, 128
    q = torch.zeros(1, 1, N, d, dtype=torch.bfloat16, device=DEV)
    _, k, _ = random_qkv(1, 1, N, d, seed=11, device=DEV)
    m = sa.sa_build_mask(q, k, 128, 64, 0.03, 0.85, want_mask=True)
    cnt = m["kv_cnt"].cpu().numpy()
    idx = m["kv_idx"].cpu().numpy()
    want = math.ceil(0.85 * 1182 - 1e-9)
    assert want == 1005
    assert (cnt == want).all()
    assert (idx[0, 0, :, :want] == np.arange(want)).all()
    assert (m["mask"][0, 0, :, :want] == 1).all() and (m["mask"][0, 0, :, want:] == 0).all()
    sa.sa_device_status()


# ------------------------------------------------------------------ full-size workloads
FULL = ["wan13b_480p", "wan14b_720p", "sink_skew", "long_245k"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_workload(cuda_lib, name):
    """Full-size workloads: the mask of every head against the oracle, row by
    row; attention on the oracle's mask of every head, on every row of at
    least 8 sampled query blocks per head (first, ragged tail, densest,
    sparsest, random), O and LSE; with the linear branch, S and z of every
    head and the blended output on the same rows."""
    sa = cuda_lib
    wl = WORKLOADS[name]
    x = make_inputs(wl, DEV)
    q, k, v = x["q"], x["k"], x["v"]
    rng = np.random.default_rng(wl.seed)
    qc, kc, vc = q.cpu(), k.cpu(), v.cpu()
    out = sa.sa_build_mask(q, k, wl.bq, wl.bk, wl.topk, wl.topp, want_mask=True)
    _assert_same_lists(out, sa.sa_build_mask(q, k, wl.bq, wl.bk, wl.topk, wl.topp))
    torch.cuda.synchronize()
    idx, cnt = out["kv_idx"].cpu().numpy(), out["kv_cnt"].cpu().numpy()
    gmask = out["mask"].cpu().numpy().astype(bool)
    ext = torch.empty(wl.B, wl.H, wl.n_qb, wl.n_kb, dtype=torch.uint8)
    totals = {"exact": 0, "score_tie": 0, "cumsum_tie": 0}
    ora = {}
    for b in range(wl.B):
        for h in range(wl.H):
            ref = _oracle_head_mask(qc, kc, b, h, wl.bq, wl.bk, wl.topk, wl.topp)
            st = compare_mask_rows(idx[b, h], cnt[b, h], ref["s"], wl.topk, wl.topp, ora_mask=ref["mask"])
            assert not st["bad"], f"{name} head {h}: {st['bad'][:3]}"
            for kk in totals:
                totals[kk] += st[kk]
            ora[(b, h)] = (ref["mask"], (gmask[b, h] == ref["mask"]).all(1))
            ext[b, h] = torch.from_numpy(ref["mask"].astype(np.uint8))
    assert sum(totals.values()) == wl.B * wl.H * wl.n_qb
    density = float(cnt.sum()) / (wl.B * wl.H * wl.n_qb * wl.n_kb)
    print(f"{name}: mask rows {totals}, realised density {density:.4f}")
    # attention on the oracle's mask (every head), and on the GPU's own lists
    o, lse = sa.sa_sparse_attn_fwd(q, k, v, wl.bq, wl.bk, ext_mask=ext.to(DEV), want_lse=True)
    o_list = sa.sa_sparse_attn_fwd(q, k, v, wl.bq, wl.bk, kv_idx=out["kv_idx"], kv_cnt=out["kv_cnt"])
    torch.cuda.synchronize()
    rows_of = {}
    for (b, h), (mask, same) in ora.items():
        rows = sample_rows(wl.n_qb, wl.bq, wl.N, mask.sum(1), rng)
        rows_of[(b, h)] = rows
        ro, rl = _oracle_attention_rows(qc, kc, vc, mask, b, h, wl.bq, wl.bk, rows)
        sel = torch.from_numpy(rows).to(DEV)
        assert_close(o[b, h][sel].float().cpu().numpy(), ro, f"{name} O head {h}")
        assert_close(lse[b, h][sel].cpu().numpy(), rl, f"{name} LSE head {h}", 1e-2, 1e-3)
        # rows whose GPU mask equals the oracle's: the list path gives the same bits
        eq = rows[same[rows // wl.bq]]
        if eq.size:
            eq = torch.from_numpy(eq).to(DEV)
            assert torch.equal(o_list[b, h][eq], o[b, h][eq])
    if wl.linear:
        # the linear branch, then the sparse attention on the oracle's mask with
        # the blend in its epilogue (one rounding of O)
        alpha = x["alpha"]
        S, z, o_l = sa.sa_linear_branch(q, k, v, want_ol=True)
        ob = sa.sa_sparse_attn_fwd(q, k, v, wl.bq, wl.bk, ext_mask=ext.to(DEV), o_l=o_l, alpha=alpha)
        torch.cuda.synchronize()
        for (b, h), (mask, _) in ora.items():
            kS, kz = oracle.linear_state(_f64(kc[b, h]), _f64(vc[b, h]))
            # phi(k) is rounded to bf16 on the GPU: relative error ~4e-3 per term
            assert np.abs(S[b, h].cpu().numpy() - kS).max() <= 5e-3 * np.abs(kS).max()
            assert np.abs(z[b, h].cpu().numpy() - kz).max() <= 5e-3 * np.abs(kz).max()
            rows = rows_of[(b, h)]
            ro, _ = _oracle_attention_rows(qc, kc, vc, mask, b, h, wl.bq, wl.bk, rows)
            ol = oracle.linear_out(_f64(qc[b, h])[rows], kS, kz)
            ref = oracle.blend(ro, ol, alpha[h].double().cpu().numpy())
            assert_close(ob[b, h][torch.from_numpy(rows).to(DEV)].float().cpu().numpy(), ref, f"{name} blend head {h}")
    sa.sa_device_status()


# ------------------------------------------------------------------ several items per CTA, all rows
@pytest.mark.parametrize("ragged", [False, True])
def test_many_items_per_cta_all_rows(cuda_lib, ragged):
    """8 heads of 16384 (or 16344: ragged last query and key blocks) tokens in
    128-row query blocks: 1,024 work items, about 7 per persistent CTA, so the
    second Q slot, the wrap of the item ring and the hand-over of O between
    items all run. Every output row and LSE is compared with the oracle, on
    the GPU-built lists (odd kept counts among them) and on an external mask
    that empties runs of consecutive items (the zero-fill of skipped items)."""
    sa = cuda_lib
    B, H, d, bq, bk = 1, 8, 128, 128, 64
    N = 16344 if ragged else 16384
    q, k, v = random_qkv(B, H, N, d, seed=4242 + N, device=DEV)
    q = (q.float() * 2.0).to(torch.bfloat16)
    nqb, nkb = -(-N // bq), -(-N // bk)
    m = sa.sa_build_mask(q, k, bq, bk, 0.04, 0.6, want_mask=True)
    o1, l1 = sa.sa_sparse_attn_fwd(q, k, v, bq, bk, kv_idx=m["kv_idx"], kv_cnt=m["kv_cnt"], want_lse=True)
    gm = m["mask"].clone()
    cnt = m["kv_cnt"].cpu().numpy()
    assert (cnt % 2 == 1).any() and (cnt % 2 == 0).any()
    if ragged:
        assert gm[..., nkb - 1].any()              # the short last key block is kept somewhere
    ext = gm.clone()
    rng = np.random.default_rng(N)
    for h in range(H):
        for start in rng.choice(nqb - 4, size=3, replace=False):
            ext[0, h, start:start + 1 + (h % 4)] = 0     # 1-4 consecutive empty items
    ext[0, H - 1, nqb - 1] = 0                           # the very last item empty
    o2, l2 = sa.sa_sparse_attn_fwd(q, k, v, bq, bk, ext_mask=ext, want_lse=True)
    torch.cuda.synchronize()
    qc, kc, vc = q.cpu(), k.cpu(), v.cpu()
    for h in range(H):
        for mask_t, o, lse in ((gm, o1, l1), (ext, o2, l2)):
            mk = mask_t[0, h].cpu().numpy().astype(bool)
            ro, rl = _oracle_attention_rows(qc, kc, vc, mk, 0, h, bq, bk, None)
            assert_close(o[0, h].float().cpu().numpy(), ro, f"O head {h}")
            empty = ~mk.any(1)
            rows_empty = np.repeat(empty, bq)[:N]
            got_l = lse[0, h].cpu().numpy()
            assert np.isneginf(got_l[rows_empty]).all()
            assert (o[0, h].float().cpu().numpy()[rows_empty] == 0).all()
            assert_close(got_l[~rows_empty], rl[~rows_empty], f"LSE head {h}", 1e-2, 1e-3)
    sa.sa_device_status()


def test_linear_branch_small(cuda_lib):
    """O_l, the standalone blend (sa_blend, on a given bf16 O_s) and the blend
    in the sparse attention's epilogue (on the oracle's mask), with batch 2 so
    that alpha's row is the head's, not the flattened (batch, head)'s."""
    sa = cuda_lib
    for (N, d, B) in [(1000, 128, 2), (257, 64, 1)]:
        H = 2
        q, k, v = random_qkv(B, H, N, d, seed=N, device=DEV)
        S, z, ol = sa.sa_linear_branch(q, k, v, want_ol=True)
        alpha = torch.rand(H, d, device=DEV)
        os_ = torch.randn_like(q.float()).to(torch.bfloat16)
        ob = sa.sa_blend(os_, q, S, z, alpha)
        m = sa.sa_build_mask(q, k, 128, 64, 0.2, 0.8, want_mask=True)
        of = sa.sa_sparse_attn_fwd(q, k, v, 128, 64, kv_idx=m["kv_idx"], kv_cnt=m["kv_cnt"], o_l=ol, alpha=alpha)
        torch.cuda.synchronize()
        for b in range(B):
            for h in range(H):
                kS, kz = oracle.linear_state(_f64(k[b, h]), _f64(v[b, h]))
                ref_l = oracle.linear_out(_f64(q[b, h]), kS, kz)
                assert_close(ol[b, h].float().cpu().numpy(), ref_l, f"O_l N={N}")
                al = alpha[h].double().cpu().numpy()
                ref_b = oracle.blend(_f64(os_[b, h]), ref_l, al)
                assert_close(ob[b, h].float().cpu().numpy(), ref_b, f"blend N={N}")
                mk = m["mask"][b, h].cpu().numpy().astype(bool)
                ro, _ = oracle.masked_attention(_f64(q[b, h]), _f64(k[b, h]), _f64(v[b, h]), mk, 128, 64)
                assert_close(of[b, h].float().cpu().numpy(), oracle.blend(ro, ref_l, al), f"fused blend N={N}")
    sa.sa_device_status()


def test_public_api_host_pipeline(cuda_lib):
    """block_sparse_attention on pinned host tensors (heads in chunks through a
    three-stream copy/compute pipeline) against the same call on device
    tensors. Batch 2 checks the flattening of (batch, head) and alpha's rows."""
    sa = cuda_lib
    B, H, N, d = 2, 3, 4100, 128
    q, k, v = random_qkv(B, H, N, d, seed=77, device="cpu")
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    alpha = torch.rand(H, d)
    for al in (None, alpha):
        ref = sa.block_sparse_attention(q.to(DEV), k.to(DEV), v.to(DEV), 128, 64, 0.1, 0.9,
                                        alpha=None if al is None else al.to(DEV))
        got = sa.block_sparse_attention(qh, kh, vh, 128, 64, 0.1, 0.9, alpha=al, chunks=4)
        assert not got.is_cuda and got.shape == q.shape
        ref = ref.cpu()
        if al is None:
            assert torch.equal(got, ref)
        else:
            # the linear state's fixed-order partial sums depend on how many heads
            # one launch covers, so the blended output may differ in the last bits
            assert (got.float() - ref.float()).abs().max().item() <= 1e-2
