/*
 * sa.h — C ABI of the B200 block-sparse attention library (libsa.so).
 *
 * The operation (pages: "SpargeAttention2: 論文の技術的サマリー" §2(1) and §2(3);
 * "SLA2" 提案手法 ① and ②; "SALAD" §2.1):
 *   1. Q and K are mean-pooled per head into query blocks of bq tokens and key
 *      blocks of bk tokens (SLA2 ①: mean pooling before scoring).
 *   2. Block scores s[qb,kb] = scale * <Qbar[qb], Kbar[kb]>; a softmax over kb
 *      turns each query-block row into probabilities P (SpargeAttention2 §2(1)
 *      needs a cumulative probability, which implies this softmax).
 *   3. Each row keeps Top-k ∪ Top-p: the ceil(k * n_kb) highest-scoring key
 *      blocks, united with the smallest set of highest-probability blocks whose
 *      probabilities sum to at least p (SpargeAttention2 §2(1)).
 *   4. FlashAttention-style attention over the kept (query-block, key-block)
 *      tiles only; masked tiles are skipped (SpargeAttention2 §2(3)).
 *   5. Optional linear branch phi(x) = elu(x) + 1 over all keys (SALAD §2.1)
 *      blended as O = alpha ⊙ O_s + (1 - alpha) ⊙ O_l (SLA2 ②).
 *
 * Conventions shared by every entry point
 *   - Tensors are device pointers, row-major and contiguous:
 *       Q, K, V, O      [B, H, N, d]  bf16 (passed as uint16_t bit patterns)
 *       q_pool          [B, H, n_qb, d] fp32,  n_qb = ceil(N / bq)
 *       k_pool          [B, H, n_kb, d] fp32,  n_kb = ceil(N / bk)
 *       kv_idx          [B, H, n_qb, n_kb] int32; row r holds kv_cnt[r] kept
 *                       key-block indices in ascending order; the remaining
 *                       entries of the row are left unspecified
 *       kv_cnt          [B, H, n_qb] int32
 *       mask            [B, H, n_qb, n_kb] uint8 (1 = kept)
 *       lse             [B, H, N] fp32, natural-log log-sum-exp of each row
 *       kv_state        [B, H, d, d] fp32, S = sum_j phi(k_j) v_j^T
 *       ksum            [B, H, d] fp32, z = sum_j phi(k_j)
 *       alpha           [H, d] fp32
 *   - Supported shapes: d in {64, 128}; bq in {64, 128}; bk = 64; N >= 1;
 *     1 <= B*H <= 65535; B*H*N*d < 2^40 and B*H*n_qb*n_kb < 2^34 (offsets
 *     are 64-bit); the mask builder also needs n_kb <= 16384 (N <= 1048576).
 *     Other values give SA_ERR_UNSUPPORTED; B, H or N below 1 give
 *     SA_ERR_INVALID_ARG.
 *   - Every device pointer must be 16-byte aligned (SA_ERR_ALIGN otherwise).
 *   - The caller owns every buffer. The library allocates no device memory; a
 *     call that needs scratch takes a caller-provided workspace whose size the
 *     matching *_workspace_size() function returns (0 means none needed).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Every call is
 *     asynchronous on it; argument errors are returned before anything is
 *     launched, launch errors as SA_ERR_CUDA.
 *   - Device-side waits are bounded. A wait that runs out records
 *     SA_ERR_DEVICE_TIMEOUT in a device status word, the kernel skips its
 *     remaining work and returns; sa_device_status() reads and clears it.
 *   - No exception or abort crosses this boundary. sa_last_error() returns a
 *     human-readable message for the last failing call on the calling thread.
 */
#ifndef SA_H_
#define SA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SA_OK                   0
#define SA_ERR_INVALID_ARG     -1
#define SA_ERR_UNSUPPORTED     -2
#define SA_ERR_ALIGN           -3
#define SA_ERR_CUDA            -4
#define SA_ERR_DEVICE_TIMEOUT  -5
#define SA_ERR_WORKSPACE       -6

/* Version of this ABI (major * 100 + minor). */
int sa_version(void);

/* Name of a status code ("SA_OK", "SA_ERR_INVALID_ARG", ...). Never NULL. */
const char* sa_status_string(int status);

/* Message describing the last failing call made by this thread ("" if none). */
const char* sa_last_error(void);

/* Synchronises `stream`, then returns and clears the device status word:
 * SA_OK, or SA_ERR_DEVICE_TIMEOUT if a bounded device-side wait ran out. */
int sa_device_status(void* stream);

/* Step 1 alone (SLA2 提案手法 ①): block means of Q and K over valid tokens.
 * The last block of a row may be partial and is averaged over its own tokens. */
int sa_pool_blocks(const uint16_t* q, const uint16_t* k, int B, int H, int N, int d,
                   int bq, int bk, float* q_pool, float* k_pool, void* stream);

/* Steps 1-3: hybrid Top-k ∪ Top-p block mask (SpargeAttention2 §2(1)).
 *   topk_frac  in (0, 1]: Top-k keeps K_sel = min(n_kb, max(1, ceil(k*n_kb - 1e-9)))
 *   topp       in [0, 1]: Top-p keeps the smallest m >= 1 such that the m most
 *              probable blocks sum to >= p; p >= 1 keeps every block
 *   scale      score scale; <= 0 selects 1/sqrt(d)
 * Order used by both rules: score descending, equal scores by lower block index.
 * The kept set of a row is therefore the first max(K_sel, m_p) blocks of that
 * order. Outputs kv_idx/kv_cnt (required) and, when non-NULL, the uint8 mask
 * and the pooled Q/K. Needs sa_build_mask_workspace_size() bytes of workspace.
 * Two exact implementations, chosen by problem size: up to 32 MiB of fp32
 * block scores, the scores are written and each row is selected from them;
 * above, the scores are reduced on the fly to per-row normalisers and
 * candidate lists (rows the lists cannot settle take the first way). The
 * environment variable SA_MASK_BUILDER=matrix or =candidates forces one. */
size_t sa_build_mask_workspace_size(int B, int H, int N, int d, int bq, int bk);
/* Kernel launches one sa_build_mask call of this shape makes (for launch
 * accounting); 0 for an invalid shape. */
int sa_build_mask_launches(int B, int H, int N, int d, int bq, int bk);
int sa_build_mask(const uint16_t* q, const uint16_t* k, int B, int H, int N, int d,
                  int bq, int bk, double topk_frac, double topp, double scale,
                  int32_t* kv_idx, int32_t* kv_cnt, uint8_t* mask_opt,
                  float* q_pool_opt, float* k_pool_opt,
                  void* workspace, size_t ws_bytes, void* stream);

/* Step 4 (SpargeAttention2 §2(3)): O_s[i] = sum over keys j of the kept key
 * blocks of softmax_j(scale * q_i . k_j) v_j, with fp32 online softmax and
 * bf16 tensor-core products; tiles not kept are never loaded or computed.
 * Exactly one of (kv_idx, kv_cnt) or ext_mask must be given. With ext_mask the
 * uint8 mask is first compacted into the workspace
 * (sa_sparse_attn_workspace_size(); 0 bytes are needed for the list form).
 * A row with no kept block outputs zeros and lse = -inf. lse_opt may be NULL.
 * scale <= 0 selects 1/sqrt(d). The lists are device data and are not
 * validated: a count outside [0, n_kb] is clamped into it, and an index
 * outside [0, n_kb) makes the result meaningless but cannot make an access
 * leave the caller's buffers (key and value tiles are fetched through tensor
 * maps, which bound every load by the tensor's extent). */
size_t sa_sparse_attn_workspace_size(int B, int H, int N, int d, int bq, int bk, int ext_mask);
int sa_sparse_attn_fwd(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                       int B, int H, int N, int d, int bq, int bk,
                       const int32_t* kv_idx, const int32_t* kv_cnt, const uint8_t* ext_mask,
                       double scale, uint16_t* o, float* lse_opt,
                       void* workspace, size_t ws_bytes, void* stream);

/* Steps 4 and 5b in one kernel (SpargeAttention2 §2(3); SLA2 提案手法 ②):
 * the sparse attention above, with its epilogue blending
 *   O = alpha ⊙ O_s + (1 - alpha) ⊙ O_l
 * while O_s is still fp32, so O is rounded to bf16 once. o_l [B, H, N, d]
 * bf16 is the linear branch's output (sa_linear_branch with o_l_opt), alpha
 * [H, d] fp32. Both are required; o must not overlap o_l (SA_ERR_INVALID_ARG).
 * lse_opt is the log-sum-exp of the sparse attention alone. Arguments,
 * workspace and errors otherwise as sa_sparse_attn_fwd. */
int sa_sparse_attn_blend_fwd(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                             int B, int H, int N, int d, int bq, int bk,
                             const int32_t* kv_idx, const int32_t* kv_cnt, const uint8_t* ext_mask,
                             double scale, const uint16_t* o_l, const float* alpha,
                             uint16_t* o, float* lse_opt,
                             void* workspace, size_t ws_bytes, void* stream);

/* Low-bit forward (SLA2 提案手法 ③: the forward pass computes with queries,
 * keys and values quantised to a low-bit format; the pages name neither the
 * format nor the scale granularity).
 *
 * sa_quantize_fp8: for each (batch, head) slice of x [B, H, N, d] bf16,
 *   amax = max |x|, scale = amax / 448 and r = 448 / amax in fp32 (both 1 for
 *   an all-zero slice), x8 = E4M3(x * r) with the product rounded to fp32 and
 *   then to E4M3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits; round
 *   to nearest even, saturating at +-448). Outputs: x8 [B, H, N, d] bytes,
 *   scale [B * H] fp32. d = 64 or 128; pointers 16-byte aligned. Launches a
 *   memset and three kernels on `stream`.
 *
 * sa_sparse_attn_fp8_fwd: the sparse attention of sa_sparse_attn_fwd on
 *   E4M3 inputs, O_s = softmax(scale * (s_q q8) . (s_k k8)) (s_v v8) over the
 *   kept tiles, with one fp32 scale per (batch, head) for each of q8, k8 and
 *   v8 (as sa_quantize_fp8 writes them; positive and finite). Both products
 *   run on E4M3 tensor-core operands with fp32 accumulation; the softmax is
 *   fp32 and P is rounded to E4M3 for the second product. d must be 128
 *   (SA_ERR_UNSUPPORTED otherwise). o_l_opt and alpha_opt (both or neither)
 *   blend the linear branch into the epilogue as sa_sparse_attn_blend_fwd
 *   does. Lists, mask, workspace, outputs and errors otherwise as
 *   sa_sparse_attn_fwd. */
int sa_quantize_fp8(const uint16_t* x, int B, int H, int N, int d, uint8_t* x8, float* scale,
                    void* stream);
int sa_sparse_attn_fp8_fwd(const uint8_t* q8, const uint8_t* k8, const uint8_t* v8,
                           const float* q_scale, const float* k_scale, const float* v_scale,
                           int B, int H, int N, int d, int bq, int bk,
                           const int32_t* kv_idx, const int32_t* kv_cnt, const uint8_t* ext_mask,
                           double scale, const uint16_t* o_l_opt, const float* alpha_opt,
                           uint16_t* o, float* lse_opt, void* workspace, size_t ws_bytes,
                           void* stream);

/* Dense attention through the same kernel, every tile kept (the comparison
 * point for the sparse speed-up). */
int sa_dense_attn_fwd(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                      int B, int H, int N, int d, int bq, double scale,
                      uint16_t* o, float* lse_opt, void* stream);

/* Step 5a (SALAD §2.1): kv_state = sum_j phi(k_j) v_j^T and ksum = sum_j phi(k_j)
 * over all N keys, phi(x) = elu(x) + 1 (phi(k) rounded to bf16, fp32 sums).
 * When o_l_opt is non-NULL also writes O_l[i] = phi(q_i)^T S / phi(q_i)^T z. */
size_t sa_linear_workspace_size(int B, int H, int N, int d);
int sa_linear_branch(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                     int B, int H, int N, int d, float* kv_state, float* ksum,
                     uint16_t* o_l_opt, void* workspace, size_t ws_bytes, void* stream);

/* Step 5b (SLA2 ②): O = alpha ⊙ O_s + (1 - alpha) ⊙ O_l with O_l computed from
 * q, kv_state and ksum inside the same kernel (the blend is its epilogue).
 * o may alias o_s. Needs sa_blend_workspace_size() bytes of workspace. */
size_t sa_blend_workspace_size(int B, int H, int N, int d);
int sa_blend(const uint16_t* o_s, const uint16_t* q, const float* kv_state, const float* ksum,
             const float* alpha, int B, int H, int N, int d, uint16_t* o,
             void* workspace, size_t ws_bytes, void* stream);

/* Backward pass ("SpargeAttention2" §2(2): the sparse attention is trainable and
 * fine-tuned by distillation, which needs gradients through the sparse path;
 * "SLA2" 提案手法 ③: the backward pass runs in full precision). Gradients are
 * fp32 [B, H, N, d]; upstream gradients are bf16 like the forward's outputs.
 *
 * sa_sparse_attn_bwd: gradients of O_s = sa_sparse_attn_fwd(q, k, v, lists)
 *   for dout = dL/dO_s, given the forward's o (O_s) and lse (its lse_opt):
 *     D = rowsum(dout * o),  dS = P * (dout v^T - D) over the kept tiles,
 *     dq = scale dS k,  dk = scale dS^T q,  dv = P^T dout,
 *   with P recomputed from lse. dq, dk and dv are written (every element: rows
 *   and keys that no kept tile reaches get zeros). The lists are the forward's
 *   (kv_idx, kv_cnt); the key-block to query-block lists that dk and dv need
 *   are built in the workspace (sa_sparse_attn_bwd_workspace_size()).
 *   Deterministic: every sum is owned by one CTA, in a fixed order.
 *
 * sa_linear_bwd: gradients of O_l = phi(q) S / phi(q) . z (the linear branch,
 *   kv_state = S and ksum = z from sa_linear_branch) for dout_l = dL/dO_l.
 *   accumulate != 0 adds into dq, dk, dv (for example onto the sparse
 *   attention's), else writes them. Deterministic (fixed-order partial sums).
 *
 * sa_blend_bwd: for O = alpha ⊙ o_s + (1 - alpha) ⊙ o_l and dout = dL/dO:
 *   do_s = alpha ⊙ dout and do_l = (1 - alpha) ⊙ dout (bf16 [B, H, N, d]),
 *   dalpha [H, d] fp32 = sum over batches and tokens of dout ⊙ (o_s - o_l). */
size_t sa_sparse_attn_bwd_workspace_size(int B, int H, int N, int d, int bq, int bk);
int sa_sparse_attn_bwd(const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint16_t* o,
                       const float* lse, const uint16_t* dout, int B, int H, int N, int d, int bq, int bk,
                       const int32_t* kv_idx, const int32_t* kv_cnt, double scale, float* dq, float* dk,
                       float* dv, void* workspace, size_t ws_bytes, void* stream);
size_t sa_linear_bwd_workspace_size(int B, int H, int N, int d);
int sa_linear_bwd(const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* kv_state,
                  const float* ksum, const uint16_t* dout_l, int B, int H, int N, int d, int accumulate,
                  float* dq, float* dk, float* dv, void* workspace, size_t ws_bytes, void* stream);
size_t sa_blend_bwd_workspace_size(int B, int H, int N, int d);
int sa_blend_bwd(const uint16_t* o_s, const uint16_t* o_l, const float* alpha, const uint16_t* dout,
                 int B, int H, int N, int d, uint16_t* do_s, uint16_t* do_l, float* dalpha,
                 void* workspace, size_t ws_bytes, void* stream);

/* Tile scoring from the full attention map ("Veda" §2.1 and §2.3).
 *
 * sa_trip_pool: TripPool descriptors of every query block (bq tokens) and key
 *   block (bk tokens): per channel the mean, the maximum and the minimum over
 *   the block's valid tokens, concatenated as [mean | max | min]:
 *     q_desc [B, H, n_qb, 3d] fp32,  k_desc [B, H, n_kb, 3d] fp32.
 *   The learned estimator that maps them to tile scores is not part of this
 *   library (it needs trained weights); its scores can be passed to
 *   sa_select_mask.
 *
 * sa_tile_heatmap: the reference tile scores, in two passes over every key
 *   tile of each evaluated query block: (1) the log-sum-exp of each query row
 *   over all N keys, (2) per (query block, key block) tile
 *     heat[qb, kb] = max over rows i of qb and keys j of kb of (scale q_i.k_j - LSE_i),
 *   the natural log of the largest full-attention probability in the tile
 *   (max pooling of the attention map over the tile; always <= 0).
 *   heat [B, H, n_qb, n_kb] fp32. rows_opt: device int32 list of n_rows
 *   query-block rows (b * H * n_qb + h * n_qb + qb) to evaluate, the sparse
 *   teacher of a random subset of query tiles; NULL evaluates every row (n_rows
 *   ignored). Rows not evaluated are left untouched. lse_opt [B, H, N] fp32
 *   (natural log) receives the first pass for the evaluated rows' tokens, or
 *   NULL. scale <= 0 selects 1/sqrt(d). Shape rules as sa_sparse_attn_fwd.
 *
 * sa_select_mask: the hybrid Top-k ∪ Top-p rule of sa_build_mask applied to
 *   given block scores (softmax over each row, the same order and ties):
 *   scores [B, H, n_qb, n_kb] fp32, finite; with scores = heat the row
 *   distribution is the max-pooled probabilities normalised over the row.
 *   Outputs as sa_build_mask (kv_idx, kv_cnt, optional uint8 mask). n_kb <= 16384. */
int sa_trip_pool(const uint16_t* q, const uint16_t* k, int B, int H, int N, int d, int bq, int bk,
                 float* q_desc, float* k_desc, void* stream);
int sa_tile_heatmap(const uint16_t* q, const uint16_t* k, int B, int H, int N, int d, int bq, int bk,
                    double scale, const int32_t* rows_opt, int n_rows, float* heat, float* lse_opt,
                    void* stream);
int sa_select_mask(const float* scores, int B, int H, int n_qb, int n_kb, double topk_frac, double topp,
                   int32_t* kv_idx, int32_t* kv_cnt, uint8_t* mask_opt, void* stream);

/* Permuted token layouts ("Veda" §2.2: a tiling (p_t, p_h, p_w) of the latent
 * grid chosen per head; "SparsePR" §2C: tokens reordered into a contiguous
 * group-major layout before the block-sparse call). The sparse path runs
 * unchanged on the permuted sequence, whose blocks are runs of consecutive
 * permuted tokens; the output is scattered back. Where a grid dimension is not
 * a multiple of the tile's, the edge tiles are partial and a block may span
 * two tiles.
 *
 * sa_tile_permutation: perm [H, N] int32 (device), N = T * Hh * W, for tokens
 *   flattened in raster order t-major over the (T, Hh, W) grid: perm[h, i] is
 *   the raster index of the token at position i of head h's order, which
 *   visits the tiles of tiles[3 h .. 3 h + 2] = (p_t, p_h, p_w) (a host array
 *   of H triples, each >= 1) in raster order of the tile grid and the tokens of
 *   a tile in raster order. 1 <= H <= 256.
 * sa_permute_tokens: rows of x [B, H, N, d] bf16 gathered into y in head h's
 *   order, y[b, h, i] = x[b, h, perm[h, i]] (inverse = 0), or scattered back,
 *   y[b, h, perm[h, i]] = x[b, h, i] (inverse = 1). perm must be a permutation
 *   of 0..N-1 for each head (it is not checked); y must not alias x. */
int sa_tile_permutation(int H, int T, int Hh, int W, const int32_t* tiles, int32_t* perm, void* stream);
int sa_permute_tokens(const uint16_t* x, const int32_t* perm, int B, int H, int N, int d, int inverse,
                      uint16_t* y, void* stream);

/* Mask builder that allocates nothing (no counterpart in the pages: it exists
 * for callers, not for the method). Some callers may not allocate device memory
 * when they call in: an inference engine's per-request callback that must not
 * allocate, or a service that plans its whole device memory budget at start-up
 * and cannot let a call grow it or synchronise the device to allocate. This
 * entry point computes exactly what sa_build_mask computes (same kernels, same
 * results) but keeps its scratch (pooled means and block scores) in a fixed
 * 32 MiB device array that is part of the library: every GPU that loads the
 * library holds those 32 MiB until the process exits. The caller still passes
 * the inputs and the outputs.
 *   - Problems whose scratch, as counted by sa_build_mask_workspace_size(), is
 *     above 32 MiB (33554432 bytes) are rejected with SA_ERR_UNSUPPORTED before
 *     anything is launched; about 12 heads of 32760 tokens at d = 128 fit.
 *   - The first call in each CUDA context looks up the array's device address
 *     (with that context current) and caches it under the context, so a new
 *     context (after cudaDeviceReset, or another context on the same device)
 *     gets its own lookup. Make that first call before any stream capture: a
 *     first call while `stream` is capturing returns SA_ERR_INVALID_ARG.
 *   - All calls share the one array and it keeps the last call's contents.
 *     Calls whose work overlaps on the GPU (for example on two streams without
 *     ordering between them) race on it; order them on one stream or with
 *     events. Nothing in the array needs to start at zero.
 *   - It calls no cudaMalloc, cudaFree or allocating library routine. */
int sa_build_mask_noalloc(const uint16_t* q, const uint16_t* k, int B, int H, int N, int d,
                          int bq, int bk, double topk_frac, double topp, double scale,
                          int32_t* kv_idx, int32_t* kv_cnt, uint8_t* mask_opt, void* stream);

/* Diagnostics (no counterpart in the pages). They exist so that tests can
 * reach the error-reporting path and the softmax's exponential helpers
 * directly, without causing a fault.
 *
 * sa_diag_set_device_status: writes `code` into the device status word that
 *   sa_device_status() reads and clears (synchronous; 0 clears it).
 * sa_diag_set_wait_limit: sets the bound, in SM clock cycles, of every
 *   device-side wait of the library's kernels (synchronous; <= 0 restores the
 *   default of 2e9 cycles, about a second). A lowered limit makes waits run
 *   out and the kernels stop early with SA_ERR_DEVICE_TIMEOUT: meant only for
 *   tests, which must restore it.
 * sa_diag_wait_timeout: launches one thread that waits on an mbarrier nothing
 *   arrives at, through the same bounded wait as the kernels; out[0] = 1 if
 *   the wait completed (never expected), out[1] = the CTA's abort flag after
 *   the wait. `out` is a device int[2]. The status word then reports the
 *   timeout.
 * sa_diag_exp2: y_poly[i] = the FMA-pipe polynomial 2^x[i] used for one
 *   column pair in four of the attention softmax (inputs clamped at -126, so
 *   values at or below 2^-125 for x <= -126), y_mufu[i] = ex2.approx(x[i]).
 *   Device float arrays of n elements, 16-byte aligned not required. */
int sa_diag_set_device_status(int code);
int sa_diag_set_wait_limit(long long cycles);
int sa_diag_wait_timeout(int* out, void* stream);
int sa_diag_exp2(const float* x, float* y_poly, float* y_mufu, int n, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SA_H_ */
