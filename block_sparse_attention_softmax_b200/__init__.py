"""B200 block-sparse attention with a hybrid Top-k ∪ Top-p block mask.

The compute lives in libsa.so (CUDA kernels for sm_100a behind the C ABI of
include/sa.h). This package is its thin Python binding: the functions below
carry the C names, marshal torch tensors into pointers and sizes, allocate
outputs and workspaces with torch, and raise on any non-zero status. There is
no CPU fallback: without the built library or a CUDA device every call raises.
"""
from ._binding import (  # noqa: F401
    SAError, load, lib_path, sa_version, sa_status_string, sa_device_status,
    sa_pool_blocks, sa_build_mask, sa_sparse_attn_fwd, sa_dense_attn_fwd, sa_quantize_fp8, sa_sparse_attn_fp8_fwd,
    sa_linear_branch, sa_blend, block_sparse_attention, header_symbols,
    sa_sparse_attn_bwd, sa_linear_bwd, sa_blend_bwd, sa_trip_pool, sa_tile_heatmap, sa_select_mask, sa_tile_permutation, sa_permute_tokens,
    sa_diag_set_device_status, sa_diag_set_wait_limit, sa_diag_wait_timeout, sa_diag_exp2,
)
