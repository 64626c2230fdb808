"""GPU parity of the backward pass against the fp64 oracle: the sparse
attention's dq, dk, dv (tiny, ragged and several-items-per-CTA shapes, rows
with no kept block), the linear branch's (written and accumulated) and the
blend's. P and dS enter the tensor core as bf16 (relative rounding 2^-9 per
term, fp32 sums), so each gradient is compared relative to its own scale:
max |err| <= 2e-2 * max |ref| and mean |err| <= 2e-3 * max |ref|."""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_softmax_b200.workloads import WORKLOADS, make_inputs, random_qkv

pytestmark = pytest.mark.gpu

DEV = "cuda"
f64 = oracle.as_f64
REL_MAX, REL_MEAN = 2e-2, 2e-3


def _close_rel(got, ref, what):
    got = np.asarray(got, dtype=np.float64)
    scale = max(np.abs(ref).max(), 1e-30)
    err = np.abs(got - ref)
    print(f"{what}: max {err.max() / scale:.2e}, mean {err.mean() / scale:.2e} of max|ref| {scale:.3e}")
    assert np.isfinite(got).all(), what
    assert err.max() <= REL_MAX * scale, (what, err.max() / scale)
    assert err.mean() <= REL_MEAN * scale, (what, err.mean() / scale)


def _masks_from_lists(idx, cnt, nkb):
    B, H, nqb = cnt.shape
    out = np.zeros((B, H, nqb, nkb), dtype=bool)
    for b in range(B):
        for h in range(H):
            out[b, h] = oracle.mask_from_lists(idx[b, h], cnt[b, h], nkb)
    return out


def _check_sparse_bwd(sa, q, k, v, bq, bk, m, seed):
    B, H, N, d = q.shape
    o, lse = sa.sa_sparse_attn_fwd(q, k, v, bq, bk, kv_idx=m["kv_idx"], kv_cnt=m["kv_cnt"], want_lse=True)
    dout = torch.randn(q.shape, generator=torch.Generator(device=DEV).manual_seed(seed), device=DEV).to(torch.bfloat16)
    dq, dk, dv = sa.sa_sparse_attn_bwd(q, k, v, o, lse, dout, bq, bk, m["kv_idx"], m["kv_cnt"])
    torch.cuda.synchronize()
    masks = _masks_from_lists(m["kv_idx"].cpu().numpy(), m["kv_cnt"].cpu().numpy(), -(-N // bk))
    for b in range(B):
        for h in range(H):
            rq, rk, rv = oracle.masked_attention_bwd(f64(q[b, h]), f64(k[b, h]), f64(v[b, h]), masks[b, h], bq, bk,
                                                     f64(dout[b, h]))
            _close_rel(dq[b, h].cpu().numpy(), rq, f"dq {b},{h}")
            _close_rel(dk[b, h].cpu().numpy(), rk, f"dk {b},{h}")
            _close_rel(dv[b, h].cpu().numpy(), rv, f"dv {b},{h}")
    sa.sa_device_status()


def test_sparse_attention_bwd_tiny(cuda_lib):
    sa = cuda_lib
    wl = WORKLOADS["tiny"]
    x = make_inputs(wl, DEV)
    m = sa.sa_build_mask(x["q"], x["k"], wl.bq, wl.bk, wl.topk, wl.topp)
    _check_sparse_bwd(sa, x["q"], x["k"], x["v"], wl.bq, wl.bk, m, 1)


@pytest.mark.parametrize("N,d,bq,H", [(333, 128, 128, 2), (200, 64, 64, 1), (4099, 128, 128, 1), (16344, 128, 128, 2)])
def test_sparse_attention_bwd_shapes(cuda_lib, N, d, bq, H):
    """Ragged query and key blocks, one-block last tiles, and (16344 tokens)
    several items per CTA in both kernels."""
    sa = cuda_lib
    q, k, v = random_qkv(1, H, N, d, seed=N + 17, device=DEV)
    q = (q.float() * 2.0).to(torch.bfloat16)
    m = sa.sa_build_mask(q, k, bq, 64, 0.1, 0.7)
    _check_sparse_bwd(sa, q, k, v, bq, 64, m, N)


def test_sparse_attention_bwd_empty_rows(cuda_lib):
    """Query blocks with no kept block get dq = 0 and add nothing to dk, dv;
    key tiles no query block keeps get dk = dv = 0."""
    sa = cuda_lib
    N, d, bq, bk, H = 640, 128, 128, 64, 1
    q, k, v = random_qkv(1, H, N, d, seed=8, device=DEV)
    m = sa.sa_build_mask(q, k, bq, bk, 0.2, 0.5)
    cnt = m["kv_cnt"].clone()
    cnt[0, 0, 1] = 0
    cnt[0, 0, 3] = 0
    idx = m["kv_idx"].clone()
    # rows 0, 2, 4 keep only key blocks 0..3, so key tiles 2..4 (blocks 4..9) are kept by no row
    for r in (0, 2, 4):
        idx[0, 0, r, :4] = torch.arange(4, dtype=torch.int32, device=DEV)
        cnt[0, 0, r] = 4
    _check_sparse_bwd(sa, q, k, v, bq, bk, {"kv_idx": idx, "kv_cnt": cnt}, 3)


def test_linear_and_blend_bwd(cuda_lib):
    """Tiles of 128 tokens, one CTA per (tile, head): 8 and 3 tiles (ragged),
    and 128 tiles per head, where dz sums 128 partials and dS comes from the
    state kernel's split over many CTAs."""
    sa = cuda_lib
    for (N, d, B) in [(1000, 128, 2), (257, 64, 1), (16344, 128, 1)]:
        H = 2
        q, k, v = random_qkv(B, H, N, d, seed=N + 1, device=DEV)
        S, z, ol = sa.sa_linear_branch(q, k, v, want_ol=True)
        g = torch.Generator(device=DEV).manual_seed(N)
        dout = torch.randn(q.shape, generator=g, device=DEV).to(torch.bfloat16)
        dq, dk, dv = sa.sa_linear_bwd(q, k, v, S, z, dout)
        base = tuple(torch.ones_like(t) for t in (dq, dk, dv))
        acc = sa.sa_linear_bwd(q, k, v, S, z, dout, grads=tuple(t.clone() for t in base))
        o_s = torch.randn(q.shape, generator=g, device=DEV).to(torch.bfloat16)
        alpha = torch.rand(H, d, device=DEV)
        ds, dl, da = sa.sa_blend_bwd(o_s, ol, alpha, dout)
        torch.cuda.synchronize()
        dat = np.zeros((H, d))
        for b in range(B):
            for h in range(H):
                rq, rk, rv = oracle.linear_bwd(f64(q[b, h]), f64(k[b, h]), f64(v[b, h]), f64(dout[b, h]))
                for got, ref, nm in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")):
                    _close_rel(got[b, h].cpu().numpy(), ref, f"linear {nm} N={N}")
                for got, ref, nm in zip(acc, (rq, rk, rv), ("dq", "dk", "dv")):
                    _close_rel(got[b, h].cpu().numpy() - 1.0, ref, f"linear {nm} accumulated N={N}")
                rs, rl, ra = oracle.blend_bwd(f64(o_s[b, h]), f64(ol[b, h]), alpha[h].double().cpu().numpy(), f64(dout[b, h]))
                # do_s, do_l are bf16: one rounding, 2^-9 of each value
                assert np.abs(ds[b, h].float().cpu().numpy() - rs).max() <= 2 ** -8 * np.abs(rs).max()
                assert np.abs(dl[b, h].float().cpu().numpy() - rl).max() <= 2 ** -8 * np.abs(rl).max()
                dat[h] += ra
        _close_rel(da.cpu().numpy(), dat, f"dalpha N={N}")
    sa.sa_device_status()
