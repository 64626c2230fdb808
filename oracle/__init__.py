"""CPU oracle for the block-sparse attention path (test infrastructure only).

This package is the slow, plain fp64 statement of what the CUDA path computes.
Only the test-suite, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import it; the product path never
does, and it shares no code with the CUDA kernels.

Pages followed (titles and sections):
  * "SpargeAttention2: 論文の技術的サマリー", §2(1) hybrid Top-k + Top-p masking,
    §2(2) trainable sparse attention (hence the backward pass), §2(3)
    block-sparse FlashAttention that skips masked tiles.
  * "SLA2" (ai-papers.net), 提案手法 ① mean pooling of queries and keys before
    scoring, ② O = alpha * O_s + (1 - alpha) * O_l, ③ a low-bit forward
    (queries, keys and values quantised) with a full-precision backward.
  * "SALAD", §2.1 a linear-attention branch in parallel with sparse attention.
  * "Veda", §2.1 TripPool descriptors and the reference mask from max-pooling
    the full attention map over tiles, §2.2 per-head tilings of the latent
    grid, §2.3 the two-pass heatmap.
  * "SparsePR", §2C tokens reordered into a group-major layout for the
    block-sparse call.

Every function works on one (batch, head) slice in float64 numpy arrays.
"""
from .sparse_attention import (  # noqa: F401
    as_f64, pool_blocks, block_scores, block_softmax, topk_count, descending_order,
    topp_count, topk_set, topp_set, hybrid_row, build_mask, kv_lists, mask_from_lists,
    masked_attention, dense_attention, phi, linear_state, linear_out, blend,
    row_threshold_info, NEAR_TIE_TOL, trip_pool, full_attention_lse, tile_max_heatmap,
    mask_from_scores, tile_permutation, permute_rows, unpermute_rows, masked_attention_bwd,
    phi_grad, linear_bwd, blend_bwd, E4M3_MAX, e4m3_round, quantize_fp8_head, fp8_masked_attention,
)
