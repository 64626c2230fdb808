"""GPU parity of the permuted token layouts ("Veda" §2.2 per-head tilings;
"SparsePR" §2C group-major layout): the tile-major orders against the oracle's,
the gather and scatter of token rows, and the whole sparse path run on
per-head permuted sequences against the oracle on the same permutation."""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_softmax_b200.workloads import random_qkv
from gpu_helpers import assert_close, compare_mask_rows

pytestmark = pytest.mark.gpu

DEV = "cuda"
f64 = oracle.as_f64


@pytest.mark.parametrize("grid,tiles", [
    ((21, 30, 52), [(1, 2, 32), (3, 5, 4), (1, 1, 64), (2, 4, 8)]),     # partial edge tiles
    ((30, 64, 128), [(1, 8, 8), (2, 4, 8)]),                              # full tiles of 64 tokens
    ((3, 5, 7), [(1, 1, 1), (3, 5, 7), (2, 2, 2)]),
])
def test_tile_permutation_matches_oracle(cuda_lib, grid, tiles):
    sa = cuda_lib
    perm = sa.sa_tile_permutation(grid, tiles).cpu().numpy()
    for h, tile in enumerate(tiles):
        assert np.array_equal(perm[h], oracle.tile_permutation(grid, tile))


def test_permute_and_scatter_back_rows(cuda_lib):
    sa = cuda_lib
    grid, tiles = (5, 6, 9), [(2, 4, 4), (1, 3, 8)]
    N = 5 * 6 * 9
    for d in (64, 128):
        x, _, _ = random_qkv(2, 2, N, d, seed=d, device=DEV)
        perm = sa.sa_tile_permutation(grid, tiles)
        y = sa.sa_permute_tokens(x, perm)
        back = sa.sa_permute_tokens(y, perm, inverse=True)
        torch.cuda.synchronize()
        pc = perm.cpu().numpy()
        for b in range(2):
            for h in range(2):
                assert torch.equal(y[b, h].cpu(), x[b, h].cpu()[torch.from_numpy(pc[h]).long()])
        assert torch.equal(back, x)


def test_sparse_path_on_permuted_heads(cuda_lib):
    """Mask, attention and the linear-branch blend on two heads with different
    tilings of a (6, 8, 10) grid (edge tiles partial): the GPU masks on the
    permuted tokens equal the oracle's, and the scattered-back output matches
    the oracle's masked attention (blended) on the same permutation."""
    sa = cuda_lib
    grid, tiles = (6, 8, 10), [(2, 4, 8), (1, 8, 8)]
    N, d, bq, bk, topk, topp = 480, 128, 128, 64, 0.2, 0.8
    q, k, v = random_qkv(1, 2, N, d, seed=55, device=DEV)
    q = (q.float() * 2.5).to(torch.bfloat16)
    alpha = torch.rand(2, d, device=DEV)
    perm = sa.sa_tile_permutation(grid, tiles)
    out = sa.block_sparse_attention(q, k, v, bq, bk, topk, topp, alpha=alpha, perm=perm)
    qp, kp = sa.sa_permute_tokens(q, perm), sa.sa_permute_tokens(k, perm)
    m = sa.sa_build_mask(qp, kp, bq, bk, topk, topp)
    torch.cuda.synchronize()
    pc = perm.cpu().numpy()
    for h in range(2):
        qh, kh, vh = (oracle.permute_rows(f64(t[0, h]), pc[h]) for t in (q, k, v))
        ref = oracle.build_mask(qh, kh, bq, bk, topk, topp)
        st = compare_mask_rows(m["kv_idx"][0, h].cpu().numpy(), m["kv_cnt"][0, h].cpu().numpy(), ref["s"], topk, topp)
        assert not st["bad"] and st["exact"] == ref["mask"].shape[0]
        ro, _ = oracle.masked_attention(qh, kh, vh, ref["mask"], bq, bk)
        S, z = oracle.linear_state(kh, vh)
        ob = oracle.blend(ro, oracle.linear_out(qh, S, z), alpha[h].double().cpu().numpy())
        assert_close(out[0, h].float().cpu().numpy(), oracle.unpermute_rows(ob, pc[h]), f"permuted path head {h}")
    sa.sa_device_status()
