"""Host-side checks of the Python binding: tensors whose shape, element type,
layout or device the C ABI could not see behind a raw pointer are refused
with ValueError before the library is called (no GPU needed)."""
import pytest
import torch

import block_sparse_attention_softmax_b200 as sa

B, H, N, d = 1, 2, 200, 64


def _bf16(*shape):
    return torch.zeros(*shape, dtype=torch.bfloat16)


def _qkv():
    return _bf16(B, H, N, d), _bf16(B, H, N, d), _bf16(B, H, N, d)


def test_host_tensors_are_refused_by_device_calls():
    q, k, v = _qkv()
    with pytest.raises(ValueError, match="CUDA tensors"):
        sa.sa_build_mask(q, k, 64, 64, 0.1, 0.9)
    with pytest.raises(ValueError, match="CUDA tensors"):
        sa.sa_pool_blocks(q, k, 64, 64)
    with pytest.raises(ValueError, match="CUDA tensors"):
        sa.sa_dense_attn_fwd(q, k, v)


def test_operand_dtype_shape_and_layout():
    q, k, v = _qkv()
    with pytest.raises(ValueError, match="dtype"):
        sa.sa_build_mask(q.float(), k, 64, 64, 0.1, 0.9)
    with pytest.raises(ValueError, match="k: shape"):
        sa.sa_build_mask(q, _bf16(B, H, N + 1, d), 64, 64, 0.1, 0.9)
    with pytest.raises(ValueError, match="contiguous"):
        sa.sa_sparse_attn_fwd(q, k, v.transpose(2, 3).contiguous().transpose(2, 3), 64, 64,
                              ext_mask=torch.ones(B, H, 4, 4, dtype=torch.uint8))
    with pytest.raises(ValueError, match=r"\[B, H, N, d\]"):
        sa.sa_pool_blocks(q[0], k[0], 64, 64)


def test_mask_list_and_output_operands():
    q, k, v = _qkv()
    nqb = nkb = -(-N // 64)
    idx = torch.zeros(B, H, nqb, nkb, dtype=torch.int32)
    cnt = torch.zeros(B, H, nqb, dtype=torch.int32)
    with pytest.raises(ValueError, match="kv_idx: dtype"):
        sa.sa_sparse_attn_fwd(q, k, v, 64, 64, kv_idx=idx.long(), kv_cnt=cnt)
    with pytest.raises(ValueError, match="kv_cnt: shape"):
        sa.sa_sparse_attn_fwd(q, k, v, 64, 64, kv_idx=idx, kv_cnt=cnt[..., :-1])
    with pytest.raises(ValueError, match="ext_mask: shape"):
        sa.sa_sparse_attn_fwd(q, k, v, 64, 64, ext_mask=torch.ones(B, H, nqb, nkb - 1, dtype=torch.uint8))
    with pytest.raises(ValueError, match="out: dtype"):
        sa.sa_sparse_attn_fwd(q, k, v, 64, 64, kv_idx=idx, kv_cnt=cnt, out=torch.zeros(B, H, N, d))


def test_linear_and_blend_operands():
    q, k, v = _qkv()
    S = torch.zeros(B, H, d, d)
    z = torch.zeros(B, H, d)
    alpha = torch.zeros(H, d)
    with pytest.raises(ValueError, match="kv_state: shape"):
        sa.sa_blend(q, q, S[..., :-1], z, alpha)
    with pytest.raises(ValueError, match="ksum: dtype"):
        sa.sa_blend(q, q, S, z.double(), alpha)
    with pytest.raises(ValueError, match="alpha: shape"):
        sa.sa_blend(q, q, S, z, alpha[0])
    with pytest.raises(ValueError, match="q is required|q must be"):
        sa.sa_linear_branch(None, k, v, want_ol=True)
    with pytest.raises(ValueError, match="v: shape"):
        sa.sa_linear_branch(None, k, v[:, :1])


def test_public_call_checks_host_operands_first():
    q, k, v = _qkv()
    with pytest.raises(ValueError, match="alpha: shape"):
        sa.block_sparse_attention(q, k, v, 64, 64, alpha=torch.zeros(H + 1, d))
    with pytest.raises(ValueError, match="out: shape"):
        sa.block_sparse_attention(q, k, v, 64, 64, out=_bf16(B, H, N, d + 1))
    with pytest.raises(ValueError, match="v: dtype"):
        sa.block_sparse_attention(q, k, v.half(), 64, 64)
