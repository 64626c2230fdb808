"""GPU parity of the low-bit forward (SLA2 提案手法 ③): per-head E4M3
quantisation against the oracle bit for bit, and the E4M3 sparse attention
against the oracle's masked attention on the dequantised inputs.

Tolerance: on top of the bf16 output rounding, the kernel rounds P to E4M3 for
the second product (within 2^-4 of each weight, 2^-10 absolute below 2^-6).
Each output element is held to the bound that follows from those roundings
(gpu_helpers.fp8_p_rounding_bound, computed from the oracle's dequantised
inputs), and the mean error to the bf16 path's 2e-3 or 0.15 of the mean
bound, whichever is larger (gpu_helpers.assert_within_bound). Over many kept keys the
P errors average out (a CPU simulation on unit-variance rows of a thousand
keys and more stays below 7.3e-3 max), but rows with one or two kept blocks
reach ~2e-2 and beyond.
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_softmax_b200.workloads import WORKLOADS, make_inputs, random_qkv
from gpu_helpers import assert_close, assert_within_bound, fp8_p_rounding_bound, sample_rows

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _f64(t):
    return oracle.as_f64(t)


def _codes_f64(x8):
    return x8.float().cpu().numpy().astype(np.float64)


def _lists_mask(m, b, h, n_kb):
    idx = m["kv_idx"][b, h].cpu().numpy()
    cnt = m["kv_cnt"][b, h].cpu().numpy()
    return oracle.mask_from_lists(idx, cnt, n_kb).astype(bool)


def test_quantize_matches_oracle_bit_for_bit(cuda_lib):
    sa = cuda_lib
    for (B, H, N, d) in [(2, 2, 777, 128), (1, 3, 130, 64)]:
        x = random_qkv(B, H, N, d, seed=N + d, device=DEV)[0]
        x[0, 1] = 0                                         # an all-zero head: scale 1, codes 0
        x[B - 1, 0, 5, 7] = 300.0                           # an outlier sets its head's scale
        x[B - 1, 0, 6, :4] = torch.tensor([1e-3, -2e-4, 3e-5, 0.0], dtype=torch.bfloat16)
        x8, sc = sa.sa_quantize_fp8(x)
        torch.cuda.synchronize()
        assert x8.dtype == torch.float8_e4m3fn and sc.shape == (B, H)
        for b in range(B):
            for h in range(H):
                codes, s = oracle.quantize_fp8_head(x[b, h].float().cpu().numpy())
                assert float(sc[b, h]) == s, (b, h, float(sc[b, h]), s)
                got = _codes_f64(x8[b, h])
                assert np.array_equal(got, codes), f"head {(b, h)}: {np.sum(got != codes)} codes differ"
        assert float(sc[0, 1]) == 1.0 and (x8[0, 1].float() == 0).all()
    sa.sa_device_status()


@pytest.mark.parametrize("N,bq", [(1000, 128), (257, 64), (4096, 128)])
def test_fp8_attention_all_rows(cuda_lib, N, bq):
    """Every row and LSE on the GPU-built lists (odd counts, the ragged last key
    block) and on an external mask with empty rows; with and without the blend."""
    sa = cuda_lib
    B, H, d, bk = 1, 3, 128, 64
    q, k, v = random_qkv(B, H, N, d, seed=7 * N + bq, device=DEV)
    nqb, nkb = -(-N // bq), -(-N // bk)
    m = sa.sa_build_mask(q, k, bq, bk, 0.1, 0.8, want_mask=True)
    (q8, qs), (k8, ks), (v8, vs) = (sa.sa_quantize_fp8(t) for t in (q, k, v))
    o1, l1 = sa.sa_sparse_attn_fp8_fwd(q8, k8, v8, qs, ks, vs, bq, bk, kv_idx=m["kv_idx"], kv_cnt=m["kv_cnt"],
                                       want_lse=True)
    ext = m["mask"].clone()
    ext[0, 0, 0] = 0
    ext[0, H - 1, nqb - 1] = 0
    o2, l2 = sa.sa_sparse_attn_fp8_fwd(q8, k8, v8, qs, ks, vs, bq, bk, ext_mask=ext, want_lse=True)
    o_l = random_qkv(B, H, N, d, seed=N + 99, device=DEV)[0]
    alpha = torch.rand(H, d, generator=torch.Generator().manual_seed(N)).to(DEV)
    o3 = sa.sa_sparse_attn_fp8_fwd(q8, k8, v8, qs, ks, vs, bq, bk, kv_idx=m["kv_idx"], kv_cnt=m["kv_cnt"],
                                   o_l=o_l, alpha=alpha)
    torch.cuda.synchronize()
    qc, kc, vc = q.cpu(), k.cpu(), v.cpu()
    for h in range(H):
        qh, kh, vh = _f64(qc[0, h]), _f64(kc[0, h]), _f64(vc[0, h])
        for mk, o, lse in ((_lists_mask(m, 0, h, nkb), o1, l1), (ext[0, h].cpu().numpy().astype(bool), o2, l2)):
            ro, rl = oracle.fp8_masked_attention(qh, kh, vh, mk, bq, bk)
            bound = fp8_p_rounding_bound(qh, kh, vh, mk, bq, bk)
            assert_within_bound(o[0, h].float().cpu().numpy(), ro, bound, f"O head {h}")
            empty = np.repeat(~mk.any(1), bq)[:N]
            got_l = lse[0, h].cpu().numpy()
            assert np.isneginf(got_l[empty]).all() and (o[0, h].float().cpu().numpy()[empty] == 0).all()
            assert_close(got_l[~empty], rl[~empty], f"LSE head {h}", 1e-2, 1e-3)
        mk = _lists_mask(m, 0, h, nkb)
        ro, _ = oracle.fp8_masked_attention(qh, kh, vh, mk, bq, bk)
        al = _f64(alpha[h].cpu())
        ref = oracle.blend(ro, _f64(o_l[0, h].cpu()), al)
        bound = al[None, :] * fp8_p_rounding_bound(qh, kh, vh, mk, bq, bk) + 2.0 ** -8 * np.abs(ref)
        assert_within_bound(o3[0, h].float().cpu().numpy(), ref, bound, f"blended O head {h}")
    sa.sa_device_status()


def test_fp8_many_items_per_cta_all_rows(cuda_lib):
    """1,024 work items (8 heads x 128 query blocks of a ragged 16,344-token
    sequence), about 7 per persistent CTA: the item ring with its per-item
    scale factors wraps several times. Every row is compared."""
    sa = cuda_lib
    B, H, N, d, bq, bk = 1, 8, 16344, 128, 128, 64
    q, k, v = random_qkv(B, H, N, d, seed=911, device=DEV)
    v[0, 3] *= 4                                        # heads with different scales
    k[0, 5] *= 0.25
    nkb = -(-N // bk)
    m = sa.sa_build_mask(q, k, bq, bk, 0.04, 0.6)
    (q8, qs), (k8, ks), (v8, vs) = (sa.sa_quantize_fp8(t) for t in (q, k, v))
    o, lse = sa.sa_sparse_attn_fp8_fwd(q8, k8, v8, qs, ks, vs, bq, bk, kv_idx=m["kv_idx"], kv_cnt=m["kv_cnt"],
                                       want_lse=True)
    torch.cuda.synchronize()
    qc, kc, vc = q.cpu(), k.cpu(), v.cpu()
    for h in range(H):
        mk = _lists_mask(m, 0, h, nkb)
        qh, kh, vh = _f64(qc[0, h]), _f64(kc[0, h]), _f64(vc[0, h])
        ro, rl = oracle.fp8_masked_attention(qh, kh, vh, mk, bq, bk)
        bound = fp8_p_rounding_bound(qh, kh, vh, mk, bq, bk)
        # head 3's values are 4x larger, and so are its errors
        assert_within_bound(o[0, h].float().cpu().numpy(), ro, bound, f"O head {h}", 8e-3 if h == 3 else 2e-3)
        assert_close(lse[0, h].cpu().numpy(), rl, f"LSE head {h}", 1e-2, 1e-3)
    sa.sa_device_status()


def test_fp8_full_size_sampled_rows(cuda_lib):
    """The 1.3B-480p-shaped workload at full size: quantiser and attention in
    the launch configuration the bench times; every head, all rows of 8+
    sampled query blocks each, against the oracle on the GPU's lists."""
    sa = cuda_lib
    wl = WORKLOADS["wan13b_480p"]
    x = make_inputs(wl, DEV)
    q, k, v = x["q"], x["k"], x["v"]
    m = sa.sa_build_mask(q, k, wl.bq, wl.bk, wl.topk, wl.topp)
    (q8, qs), (k8, ks), (v8, vs) = (sa.sa_quantize_fp8(t) for t in (q, k, v))
    o = sa.sa_sparse_attn_fp8_fwd(q8, k8, v8, qs, ks, vs, wl.bq, wl.bk, kv_idx=m["kv_idx"], kv_cnt=m["kv_cnt"])
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    qc, kc, vc = q.cpu(), k.cpu(), v.cpu()
    cnt = m["kv_cnt"].cpu().numpy()
    for h in range(wl.H):
        codes, s = oracle.quantize_fp8_head(qc[0, h].float().numpy())
        assert float(qs[0, h]) == s and np.array_equal(_codes_f64(q8[0, h]), codes)
        rows = sample_rows(wl.n_qb, wl.bq, wl.N, cnt[0, h], rng)
        mk = _lists_mask(m, 0, h, wl.n_kb)
        qh, kh, vh = _f64(qc[0, h]), _f64(kc[0, h]), _f64(vc[0, h])
        ro, _ = oracle.fp8_masked_attention(qh, kh, vh, mk, wl.bq, wl.bk, rows=rows)
        bound = fp8_p_rounding_bound(qh, kh, vh, mk, wl.bq, wl.bk, rows=rows)
        assert_within_bound(o[0, h, rows].float().cpu().numpy(), ro, bound, f"O head {h}")
    sa.sa_device_status()
