"""GPU parity of the tile-scoring entry points ("Veda" §2.1, §2.3) against the
fp64 oracle: TripPool descriptors, the two-pass max-pooled heatmap (all rows
and a sampled subset of query blocks) with its first-pass LSE, and the hybrid
selection from given block scores."""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_softmax_b200.workloads import WORKLOADS, make_inputs, random_qkv
from gpu_helpers import assert_close, compare_mask_rows

pytestmark = pytest.mark.gpu

DEV = "cuda"
f64 = oracle.as_f64


@pytest.mark.parametrize("N,d,bq", [(1024, 64, 64), (333, 128, 128), (200, 64, 128)])
def test_trip_pool(cuda_lib, N, d, bq):
    sa = cuda_lib
    q, k, _ = random_qkv(1, 2, N, d, seed=N + d, device=DEV)
    qd, kd = sa.sa_trip_pool(q, k, bq, 64)
    torch.cuda.synchronize()
    for h in range(2):
        for x, desc, b in ((q, qd, bq), (k, kd, 64)):
            ref = oracle.trip_pool(f64(x[0, h]), b)
            got = desc[0, h].cpu().numpy().astype(np.float64)
            assert np.abs(got[:, :d] - ref[:, :d]).max() <= 1e-5
            assert np.array_equal(got[:, d:], ref[:, d:])          # max and min are exact
    sa.sa_device_status()


@pytest.mark.parametrize("N,d,bq,scale_q", [(1024, 64, 64, 1.0), (333, 128, 128, 3.0), (4099, 128, 128, 2.0)])
def test_tile_heatmap_all_rows(cuda_lib, N, d, bq, scale_q):
    sa = cuda_lib
    q, k, _ = random_qkv(1, 2, N, d, seed=3 * N + d, device=DEV)
    q = (q.float() * scale_q).to(torch.bfloat16)
    heat, lse = sa.sa_tile_heatmap(q, k, bq, want_lse=True)
    torch.cuda.synchronize()
    for h in range(2):
        ref = oracle.tile_max_heatmap(f64(q[0, h]), f64(k[0, h]), bq, 64)
        got = heat[0, h].cpu().numpy().astype(np.float64)
        assert np.isfinite(got).all() and (got <= 0).all()
        assert np.abs(got - ref).max() <= 2e-3, np.abs(got - ref).max()
        rl = oracle.full_attention_lse(f64(q[0, h]), f64(k[0, h]))
        assert np.abs(lse[0, h].cpu().numpy() - rl).max() <= 1e-3
    # the hybrid selection from these scores, against the rule on the same fp32 values
    m = sa.sa_select_mask(heat, 0.1, 0.8, want_mask=True)
    torch.cuda.synchronize()
    idx, cnt = m["kv_idx"].cpu().numpy(), m["kv_cnt"].cpu().numpy()
    for h in range(2):
        s = heat[0, h].cpu().numpy().astype(np.float64)
        st = compare_mask_rows(idx[0, h], cnt[0, h], s, 0.1, 0.8, ora_mask=oracle.mask_from_scores(s, 0.1, 0.8))
        assert not st["bad"], st["bad"][:3]
    sa.sa_device_status()


def test_tile_heatmap_sampled_query_blocks(cuda_lib):
    """The sparse teacher: a random subset of the query blocks of a
    1.3B-480p-shaped pair of heads; the other rows are left untouched."""
    sa = cuda_lib
    wl = WORKLOADS["wan13b_480p"]
    x = make_inputs(wl, DEV)
    q, k = x["q"][:, :2].contiguous(), x["k"][:, :2].contiguous()
    rng = np.random.default_rng(7)
    nqb, nkb = wl.n_qb, wl.n_kb
    picks = {h: np.sort(rng.choice(nqb, size=6, replace=False)) for h in range(2)}
    picks[1][-1] = nqb - 1                                   # the ragged last query block
    rows = torch.tensor(np.concatenate([h * nqb + picks[h] for h in range(2)]), dtype=torch.int32, device=DEV)
    out = torch.full((1, 2, nqb, nkb), 7.0, device=DEV)
    sa.sa_tile_heatmap(q, k, wl.bq, rows=rows, out=out)
    torch.cuda.synchronize()
    got = out.cpu().numpy().astype(np.float64)
    for h in range(2):
        ref = oracle.tile_max_heatmap(f64(q[0, h]), f64(k[0, h]), wl.bq, 64, q_blocks=picks[h])
        assert np.abs(got[0, h, picks[h]] - ref[picks[h]]).max() <= 2e-3
        others = np.setdiff1d(np.arange(nqb), picks[h])
        assert (got[0, h, others] == 7.0).all()
    sa.sa_device_status()


def test_select_mask_on_block_scores(cuda_lib):
    """On a head's mean-pooled block scores the selection from scores gives
    the oracle's mask (up to reported near-ties), as sa_build_mask does."""
    sa = cuda_lib
    wl = WORKLOADS["tiny"]
    x = make_inputs(wl, "cpu")
    scores = np.stack([oracle.build_mask(f64(x["q"][0, h]), f64(x["k"][0, h]), wl.bq, wl.bk, wl.topk, wl.topp)["s"]
                       for h in range(wl.H)])[None]
    s32 = torch.from_numpy(scores.astype(np.float32)).to(DEV)
    m = sa.sa_select_mask(s32, wl.topk, wl.topp)
    torch.cuda.synchronize()
    for h in range(wl.H):
        s = s32[0, h].cpu().numpy().astype(np.float64)
        st = compare_mask_rows(m["kv_idx"][0, h].cpu().numpy(), m["kv_cnt"][0, h].cpu().numpy(), s, wl.topk, wl.topp)
        assert not st["bad"]
    sa.sa_device_status()
