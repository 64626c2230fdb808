// sa_api.cu — the extern "C" boundary of libsa: argument validation, workspace
// carving, kernel dispatch and error reporting. Declarations and the contract
// of every entry point are in include/sa.h.
#include <math.h>
#include <stdarg.h>
#include <stdlib.h>
#include <stdio.h>
#include <string.h>

#include <string>

#include "../../include/sa.h"
#include "sa_internal.h"

namespace sa {

namespace {

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* where) {
  return fail(SA_ERR_CUDA, "%s: %s (%s)", where, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

constexpr int kMaxKeyBlocks = 16384;  // selection keeps one row of scores in shared memory

int check_shape(int B, int H, int N, int d, int bq, int bk) {
  if (B <= 0 || H <= 0 || N <= 0) return fail(SA_ERR_INVALID_ARG, "B, H and N must be positive (got %d, %d, %d)", B, H, N);
  if (d != 64 && d != 128) return fail(SA_ERR_UNSUPPORTED, "head dim %d unsupported (64 or 128)", d);
  if (bq != 64 && bq != 128) return fail(SA_ERR_UNSUPPORTED, "query block %d unsupported (64 or 128)", bq);
  if (bk != 64) return fail(SA_ERR_UNSUPPORTED, "key block %d unsupported (64)", bk);
  const long long BH = static_cast<long long>(B) * H;
  if (BH > 65535) return fail(SA_ERR_UNSUPPORTED, "B*H = %lld exceeds 65535", BH);
  if (BH * N * d >= (1LL << 40)) return fail(SA_ERR_UNSUPPORTED, "tensor too large");
  const long long nkb = (N + bk - 1) / bk, nqb = (N + bq - 1) / bq;
  if (BH * nqb * nkb >= (1LL << 34)) return fail(SA_ERR_UNSUPPORTED, "block mask too large");
  return SA_OK;
}

struct MaskWs {
  size_t q_pool, k_pool, q_sl, k_sl, q_ex, k_ex, s, st1, st2, rowinfo, cand_cnt, fb, fb_rows, tile_flag, total;
  long long s_ld;
};

// Workspace of the mask builder: pooled means (unless the caller takes them),
// their int8 slices and exponents, the score rows (candidate lists first,
// then the score rows of query tiles handed back to the full-row selection)
// and the per-row buffers of the candidate path.
MaskWs mask_ws(int B, int H, int N, int d, int bq, int bk, bool need_q, bool need_k) {
  const long long BH = static_cast<long long>(B) * H;
  const long long nqb = (N + bq - 1) / bq, nkb = (N + bk - 1) / bk;
  const long long rows = BH * nqb;
  MaskWs w{};
  w.s_ld = (nkb + 3) / 4 * 4;
  size_t off = 0;
  w.q_pool = off;
  if (need_q) off += round_up(static_cast<size_t>(BH * nqb * d) * 4, 256);
  w.k_pool = off;
  if (need_k) off += round_up(static_cast<size_t>(BH * nkb * d) * 4, 256);
  w.q_sl = off;
  off += round_up(static_cast<size_t>(BH * nqb * 4 * d), 256);
  w.k_sl = off;
  off += round_up(static_cast<size_t>(BH * nkb * 4 * d), 256);
  w.q_ex = off;
  off += round_up(static_cast<size_t>(BH * nqb) * 4, 256);
  w.k_ex = off;
  off += round_up(static_cast<size_t>(BH * nkb) * 4, 256);
  w.s = off;
  off += round_up(static_cast<size_t>(rows * cand_row_bytes(w.s_ld)), 256);
  w.st1 = off;
  off += round_up(static_cast<size_t>(rows) * 4 * kMaxKr * 16, 256);
  w.st2 = off;
  off += round_up(static_cast<size_t>(rows) * 4 * kMaxKr * 16, 256);
  w.rowinfo = off;
  off += round_up(static_cast<size_t>(rows) * 8, 256);
  w.cand_cnt = off;
  off += round_up(static_cast<size_t>(rows) * 8, 256);
  w.fb = off;
  off += 256;
  w.fb_rows = off;
  off += round_up(static_cast<size_t>(rows) * 4, 256);
  w.tile_flag = off;
  off += round_up(static_cast<size_t>(BH * ((nqb + kI8TileM - 1) / kI8TileM)) * 4, 256);
  w.total = off;
  return w;
}

// Which builder a shape takes: the score-matrix path while the fp32 scores
// fit in 32 MiB (cheap to write and re-read, three launches), else the
// candidate path. SA_MASK_BUILDER=matrix / =candidates forces one.
bool use_candidates(long long rows, long long s_ld) {
  const char* env = getenv("SA_MASK_BUILDER");
  if (env && strcmp(env, "matrix") == 0) return false;
  if (env && strcmp(env, "candidates") == 0) return true;
  return rows * s_ld * 4 > (32LL << 20);
}

// The launches of the mask builder, on carved workspace: pooling (with the
// int8 slices), then the score-matrix or the candidate path.
cudaError_t run_mask_builder(const void* q, const void* k, int BH, int N, int d, int bq, int bk,
                             int k_sel, double topp, double scale, int* kv_idx, int* kv_cnt,
                             uint8_t* mask_opt, float* qp, float* kp, char* ws, const MaskWs& w,
                             cudaStream_t st) {
  const int nqb = (N + bq - 1) / bq, nkb = (N + bk - 1) / bk;
  SliceOut sl{reinterpret_cast<int8_t*>(ws + w.q_sl), reinterpret_cast<int8_t*>(ws + w.k_sl),
              reinterpret_cast<int*>(ws + w.q_ex), reinterpret_cast<int*>(ws + w.k_ex)};
  float* s = reinterpret_cast<float*>(ws + w.s);
  CandWs cw{ws + w.st1, ws + w.st2, ws + w.rowinfo, reinterpret_cast<int*>(ws + w.cand_cnt),
            reinterpret_cast<int*>(ws + w.fb), reinterpret_cast<int*>(ws + w.fb_rows),
            reinterpret_cast<int*>(ws + w.tile_flag)};
  cudaError_t e = launch_pool(q, k, BH, N, d, bq, bk, qp, kp, st, &sl);
  if (e != cudaSuccess) return e;
  if (use_candidates(static_cast<long long>(BH) * nqb, w.s_ld))
    return launch_mask_cand(sl, BH, nqb, nkb, d, scale, k_sel, topp, s, w.s_ld, cw, kv_idx, kv_cnt, mask_opt, st);
  e = launch_scores_i8(sl, BH, nqb, nkb, d, scale, s, w.s_ld, st);
  if (e == cudaSuccess) e = launch_select(s, w.s_ld, BH * nqb, nkb, k_sel, topp, kv_idx, kv_cnt, mask_opt, st);
  return e;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

}  // namespace

CUresult encode_tensor_map_3d_bf16(CUtensorMap* map, const void* base, uint64_t inner,
                                   uint64_t rows, uint64_t planes, uint32_t box_inner,
                                   uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return CUDA_ERROR_NOT_SUPPORTED;
  const cuuint64_t dims[3] = {inner, rows, planes};
  const cuuint64_t strides[2] = {inner * 2, inner * rows * 2};
  const cuuint32_t box[3] = {box_inner, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

CUresult encode_tensor_map_3d_u8(CUtensorMap* map, const void* base, uint64_t inner,
                                 uint64_t rows, uint64_t planes, uint32_t box_inner,
                                 uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return CUDA_ERROR_NOT_SUPPORTED;
  const cuuint64_t dims[3] = {inner, rows, planes};
  const cuuint64_t strides[2] = {inner, inner * rows};
  const cuuint32_t box[3] = {box_inner, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

}  // namespace sa

using namespace sa;

extern "C" {

int sa_version(void) { return 100; }

const char* sa_status_string(int status) {
  switch (status) {
    case SA_OK: return "SA_OK";
    case SA_ERR_INVALID_ARG: return "SA_ERR_INVALID_ARG";
    case SA_ERR_UNSUPPORTED: return "SA_ERR_UNSUPPORTED";
    case SA_ERR_ALIGN: return "SA_ERR_ALIGN";
    case SA_ERR_CUDA: return "SA_ERR_CUDA";
    case SA_ERR_DEVICE_TIMEOUT: return "SA_ERR_DEVICE_TIMEOUT";
    case SA_ERR_WORKSPACE: return "SA_ERR_WORKSPACE";
    default: return "SA_ERR_UNKNOWN";
  }
}

const char* sa_last_error(void) { return g_last_error.c_str(); }

int sa_device_status(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "sa_device_status");
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "sa_device_status");
  if (v != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "sa_device_status (clearing the status word)");
    return fail(SA_ERR_DEVICE_TIMEOUT, "a bounded device-side wait ran out (code %d)", v);
  }
  return SA_OK;
}

int sa_pool_blocks(const uint16_t* q, const uint16_t* k, int B, int H, int N, int d, int bq,
                   int bk, float* q_pool, float* k_pool, void* stream) {
  int rc = check_shape(B, H, N, d, bq, bk);
  if (rc) return rc;
  if (!q || !k || !q_pool || !k_pool) return fail(SA_ERR_INVALID_ARG, "sa_pool_blocks: null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(q_pool) || !aligned16(k_pool))
    return fail(SA_ERR_ALIGN, "sa_pool_blocks: pointers must be 16-byte aligned");
  cudaError_t e = launch_pool(q, k, B * H, N, d, bq, bk, q_pool, k_pool, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SA_OK : cuda_fail(e, "sa_pool_blocks");
}

size_t sa_build_mask_workspace_size(int B, int H, int N, int d, int bq, int bk) {
  if (check_shape(B, H, N, d, bq, bk)) return 0;
  return mask_ws(B, H, N, d, bq, bk, true, true).total;
}

int sa_build_mask_launches(int B, int H, int N, int d, int bq, int bk) {
  if (check_shape(B, H, N, d, bq, bk)) return 0;
  const MaskWs w = mask_ws(B, H, N, d, bq, bk, true, true);
  const long long rows = static_cast<long long>(B) * H * ((N + bq - 1) / bq);
  // pooling, then statistics, candidates, selection and the two hand-back
  // launches, or scores and selection
  return use_candidates(rows, w.s_ld) ? 6 : 3;
}

int sa_build_mask(const uint16_t* q, const uint16_t* k, int B, int H, int N, int d, int bq, int bk,
                  double topk_frac, double topp, double scale, int32_t* kv_idx, int32_t* kv_cnt,
                  uint8_t* mask_opt, float* q_pool_opt, float* k_pool_opt, void* workspace,
                  size_t ws_bytes, void* stream) {
  int rc = check_shape(B, H, N, d, bq, bk);
  if (rc) return rc;
  if (!q || !k || !kv_idx || !kv_cnt) return fail(SA_ERR_INVALID_ARG, "sa_build_mask: null pointer");
  if (!(topk_frac > 0.0 && topk_frac <= 1.0)) return fail(SA_ERR_INVALID_ARG, "topk_frac %g outside (0, 1]", topk_frac);
  if (!(topp >= 0.0 && topp <= 1.0)) return fail(SA_ERR_INVALID_ARG, "topp %g outside [0, 1]", topp);
  if (!isfinite(scale)) return fail(SA_ERR_INVALID_ARG, "scale must be finite");
  const int nkb = (N + bk - 1) / bk;
  if (nkb > kMaxKeyBlocks) return fail(SA_ERR_UNSUPPORTED, "n_kb = %d exceeds %d", nkb, kMaxKeyBlocks);
  const void* ptrs[] = {q, k, kv_idx, kv_cnt, mask_opt, q_pool_opt, k_pool_opt, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(SA_ERR_ALIGN, "sa_build_mask: pointers must be 16-byte aligned");
  const MaskWs w = mask_ws(B, H, N, d, bq, bk, q_pool_opt == nullptr, k_pool_opt == nullptr);
  if (!workspace || ws_bytes < w.total)
    return fail(SA_ERR_WORKSPACE, "sa_build_mask: workspace of %zu bytes needed, %zu given", w.total, workspace ? ws_bytes : 0);
  if (scale <= 0.0) scale = 1.0 / sqrt(static_cast<double>(d));
  char* ws = static_cast<char*>(workspace);
  float* qp = q_pool_opt ? q_pool_opt : reinterpret_cast<float*>(ws + w.q_pool);
  float* kp = k_pool_opt ? k_pool_opt : reinterpret_cast<float*>(ws + w.k_pool);
  const int BH = B * H;
  const int k_sel = static_cast<int>(fmin(static_cast<double>(nkb), fmax(1.0, ceil(topk_frac * nkb - 1e-9))));
  cudaError_t e = run_mask_builder(q, k, BH, N, d, bq, bk, k_sel, topp, scale, kv_idx, kv_cnt, mask_opt,
                                   qp, kp, ws, w, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SA_OK : cuda_fail(e, "sa_build_mask");
}

size_t sa_sparse_attn_workspace_size(int B, int H, int N, int d, int bq, int bk, int ext_mask) {
  if (check_shape(B, H, N, d, bq, bk) || !ext_mask) return 0;
  const long long BH = static_cast<long long>(B) * H;
  const long long nqb = (N + bq - 1) / bq, nkb = (N + bk - 1) / bk;
  return round_up(static_cast<size_t>(BH * nqb * nkb) * 4, 256) + round_up(static_cast<size_t>(BH * nqb) * 4, 256);
}

namespace {

// Shared body of sa_sparse_attn_fwd and sa_sparse_attn_blend_fwd (o_l and
// alpha both null, or both given).
struct Fp8Scales {
  const float* q = nullptr;
  const float* k = nullptr;
  const float* v = nullptr;
};

int sparse_attn(const char* fn, const void* q, const void* k, const void* v, int B, int H,
                int N, int d, int bq, int bk, const int32_t* kv_idx, const int32_t* kv_cnt,
                const uint8_t* ext_mask, double scale, const uint16_t* o_l, const float* alpha,
                uint16_t* o, float* lse_opt, void* workspace, size_t ws_bytes, void* stream,
                const Fp8Scales* f8 = nullptr) {
  int rc = check_shape(B, H, N, d, bq, bk);
  if (rc) return rc;
  if (!q || !k || !v || !o) return fail(SA_ERR_INVALID_ARG, "%s: null tensor pointer", fn);
  if (f8) {
    if (d != 128) return fail(SA_ERR_UNSUPPORTED, "%s: the low-bit forward needs d = 128 (got %d)", fn, d);
    if (!f8->q || !f8->k || !f8->v) return fail(SA_ERR_INVALID_ARG, "%s: null scale pointer", fn);
    const void* sp[] = {f8->q, f8->k, f8->v};
    for (const void* p : sp)
      if (!aligned16(p)) return fail(SA_ERR_ALIGN, "%s: pointers must be 16-byte aligned", fn);
  }
  const bool lists = kv_idx && kv_cnt;
  if (lists == (ext_mask != nullptr) || (!lists && (kv_idx || kv_cnt)))
    return fail(SA_ERR_INVALID_ARG, "%s: give exactly one of (kv_idx, kv_cnt) or ext_mask", fn);
  if ((o_l == nullptr) != (alpha == nullptr)) return fail(SA_ERR_INVALID_ARG, "%s: o_l and alpha go together", fn);
  if (o_l) {
    // O is stored tile by tile while later tiles of O_l are still to be read
    const uintptr_t bytes = static_cast<uintptr_t>(B) * H * N * d * 2;
    const uintptr_t po = reinterpret_cast<uintptr_t>(o), pl = reinterpret_cast<uintptr_t>(o_l);
    if (po < pl + bytes && pl < po + bytes) return fail(SA_ERR_INVALID_ARG, "%s: o must not overlap o_l", fn);
  }
  if (!isfinite(scale)) return fail(SA_ERR_INVALID_ARG, "scale must be finite");
  const void* ptrs[] = {q, k, v, o, kv_idx, kv_cnt, lse_opt, workspace, o_l, alpha};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(SA_ERR_ALIGN, "%s: pointers must be 16-byte aligned", fn);
  if (scale <= 0.0) scale = 1.0 / sqrt(static_cast<double>(d));
  const int BH = B * H;
  const int nqb = (N + bq - 1) / bq, nkb = (N + bk - 1) / bk;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int* idx = kv_idx;
  const int* cnt = kv_cnt;
  if (!lists) {
    const size_t need = sa_sparse_attn_workspace_size(B, H, N, d, bq, bk, 1);
    if (!workspace || ws_bytes < need)
      return fail(SA_ERR_WORKSPACE, "%s: workspace of %zu bytes needed for ext_mask", fn, need);
    int* widx = static_cast<int*>(workspace);
    int* wcnt = reinterpret_cast<int*>(static_cast<char*>(workspace) + round_up(static_cast<size_t>(BH) * nqb * nkb * 4, 256));
    cudaError_t e = launch_compact_mask(ext_mask, BH * nqb, nkb, widx, wcnt, st);
    if (e != cudaSuccess) return cuda_fail(e, "mask compaction");
    idx = widx;
    cnt = wcnt;
  }
  AttnArgs a{q, k, v, o, lse_opt, idx, cnt, BH, N, d, bq, bk, nqb, nkb,
             static_cast<float>(scale * 1.4426950408889634), 0, o_l, alpha, H};
  if (f8) {
    a.fp8 = 1;
    a.q_scale = f8->q;
    a.k_scale = f8->k;
    a.v_scale = f8->v;
  }
  cudaError_t e = launch_sparse_attn(a, st);
  return e == cudaSuccess ? SA_OK : cuda_fail(e, fn);
}

}  // namespace

int sa_sparse_attn_fwd(const uint16_t* q, const uint16_t* k, const uint16_t* v, int B, int H,
                       int N, int d, int bq, int bk, const int32_t* kv_idx,
                       const int32_t* kv_cnt, const uint8_t* ext_mask, double scale, uint16_t* o,
                       float* lse_opt, void* workspace, size_t ws_bytes, void* stream) {
  return sparse_attn("sa_sparse_attn_fwd", q, k, v, B, H, N, d, bq, bk, kv_idx, kv_cnt, ext_mask, scale,
                     nullptr, nullptr, o, lse_opt, workspace, ws_bytes, stream);
}

int sa_sparse_attn_blend_fwd(const uint16_t* q, const uint16_t* k, const uint16_t* v, int B, int H,
                             int N, int d, int bq, int bk, const int32_t* kv_idx,
                             const int32_t* kv_cnt, const uint8_t* ext_mask, double scale,
                             const uint16_t* o_l, const float* alpha, uint16_t* o, float* lse_opt,
                             void* workspace, size_t ws_bytes, void* stream) {
  if (!o_l || !alpha) return fail(SA_ERR_INVALID_ARG, "sa_sparse_attn_blend_fwd: o_l and alpha are required");
  return sparse_attn("sa_sparse_attn_blend_fwd", q, k, v, B, H, N, d, bq, bk, kv_idx, kv_cnt, ext_mask,
                     scale, o_l, alpha, o, lse_opt, workspace, ws_bytes, stream);
}

int sa_quantize_fp8(const uint16_t* x, int B, int H, int N, int d, uint8_t* x8, float* scale, void* stream) {
  if (B <= 0 || H <= 0 || N <= 0) return fail(SA_ERR_INVALID_ARG, "B, H and N must be positive (got %d, %d, %d)", B, H, N);
  if (d != 64 && d != 128) return fail(SA_ERR_UNSUPPORTED, "head dim %d unsupported (64 or 128)", d);
  const long long BH = static_cast<long long>(B) * H;
  if (BH > 65535) return fail(SA_ERR_UNSUPPORTED, "B*H = %lld exceeds 65535", BH);
  if (BH * N * d >= (1LL << 40)) return fail(SA_ERR_UNSUPPORTED, "tensor too large");
  if (!x || !x8 || !scale) return fail(SA_ERR_INVALID_ARG, "sa_quantize_fp8: null pointer");
  if (!aligned16(x) || !aligned16(x8) || !aligned16(scale))
    return fail(SA_ERR_ALIGN, "sa_quantize_fp8: pointers must be 16-byte aligned");
  cudaError_t e = launch_quantize_fp8(x, BH, static_cast<long long>(N) * d, x8, scale, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SA_OK : cuda_fail(e, "sa_quantize_fp8");
}

int sa_sparse_attn_fp8_fwd(const uint8_t* q8, const uint8_t* k8, const uint8_t* v8, const float* q_scale,
                           const float* k_scale, const float* v_scale, int B, int H, int N, int d, int bq,
                           int bk, const int32_t* kv_idx, const int32_t* kv_cnt, const uint8_t* ext_mask,
                           double scale, const uint16_t* o_l_opt, const float* alpha_opt, uint16_t* o,
                           float* lse_opt, void* workspace, size_t ws_bytes, void* stream) {
  const Fp8Scales f8{q_scale, k_scale, v_scale};
  return sparse_attn("sa_sparse_attn_fp8_fwd", q8, k8, v8, B, H, N, d, bq, bk, kv_idx, kv_cnt, ext_mask, scale,
                     o_l_opt, alpha_opt, o, lse_opt, workspace, ws_bytes, stream, &f8);
}

int sa_dense_attn_fwd(const uint16_t* q, const uint16_t* k, const uint16_t* v, int B, int H, int N,
                      int d, int bq, double scale, uint16_t* o, float* lse_opt, void* stream) {
  int rc = check_shape(B, H, N, d, bq, 64);
  if (rc) return rc;
  if (!q || !k || !v || !o) return fail(SA_ERR_INVALID_ARG, "sa_dense_attn_fwd: null tensor pointer");
  if (!isfinite(scale)) return fail(SA_ERR_INVALID_ARG, "scale must be finite");
  const void* ptrs[] = {q, k, v, o, lse_opt};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(SA_ERR_ALIGN, "sa_dense_attn_fwd: pointers must be 16-byte aligned");
  if (scale <= 0.0) scale = 1.0 / sqrt(static_cast<double>(d));
  const int BH = B * H;
  const int nqb = (N + bq - 1) / bq, nkb = (N + 63) / 64;
  AttnArgs a{q, k, v, o, lse_opt, nullptr, nullptr, BH, N, d, bq, 64, nqb, nkb,
             static_cast<float>(scale * 1.4426950408889634), 1};
  cudaError_t e = launch_sparse_attn(a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SA_OK : cuda_fail(e, "sa_dense_attn_fwd");
}

size_t sa_linear_workspace_size(int B, int H, int N, int d) {
  if (check_shape(B, H, N, d, 64, 64)) return 0;
  return linear_state_ws_bytes(B * H, N, d);
}

int sa_linear_branch(const uint16_t* q, const uint16_t* k, const uint16_t* v, int B, int H, int N,
                     int d, float* kv_state, float* ksum, uint16_t* o_l_opt, void* workspace,
                     size_t ws_bytes, void* stream) {
  int rc = check_shape(B, H, N, d, 64, 64);
  if (rc) return rc;
  if (!k || !v || !kv_state || !ksum) return fail(SA_ERR_INVALID_ARG, "sa_linear_branch: null pointer");
  if (o_l_opt && !q) return fail(SA_ERR_INVALID_ARG, "sa_linear_branch: O_l needs q");
  const void* ptrs[] = {q, k, v, kv_state, ksum, o_l_opt, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(SA_ERR_ALIGN, "sa_linear_branch: pointers must be 16-byte aligned");
  const size_t need = linear_state_ws_bytes(B * H, N, d);
  if (!workspace || ws_bytes < need)
    return fail(SA_ERR_WORKSPACE, "sa_linear_branch: workspace of %zu bytes needed", need);
  LinearArgs a{q, k, v, nullptr, nullptr, kv_state, ksum, o_l_opt, B, H, N, d, workspace};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_linear_state(a, st);
  if (e == cudaSuccess && o_l_opt) e = launch_linear_out(a, st);
  return e == cudaSuccess ? SA_OK : cuda_fail(e, "sa_linear_branch");
}

size_t sa_blend_workspace_size(int B, int H, int N, int d) {
  if (check_shape(B, H, N, d, 64, 64)) return 0;
  return linear_out_ws_bytes(B * H, d);
}

int sa_blend(const uint16_t* o_s, const uint16_t* q, const float* kv_state, const float* ksum,
             const float* alpha, int B, int H, int N, int d, uint16_t* o, void* workspace,
             size_t ws_bytes, void* stream) {
  int rc = check_shape(B, H, N, d, 64, 64);
  if (rc) return rc;
  if (!o_s || !q || !kv_state || !ksum || !alpha || !o) return fail(SA_ERR_INVALID_ARG, "sa_blend: null pointer");
  const void* ptrs[] = {o_s, q, kv_state, ksum, alpha, o, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(SA_ERR_ALIGN, "sa_blend: pointers must be 16-byte aligned");
  const size_t need = linear_out_ws_bytes(B * H, d);
  if (need && (!workspace || ws_bytes < need)) return fail(SA_ERR_WORKSPACE, "sa_blend: workspace of %zu bytes needed", need);
  LinearArgs a{q, nullptr, nullptr, o_s, alpha, const_cast<float*>(kv_state), const_cast<float*>(ksum), o, B, H, N, d, workspace};
  cudaError_t e = launch_linear_out(a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SA_OK : cuda_fail(e, "sa_blend");
}

int sa_trip_pool(const uint16_t* q, const uint16_t* k, int B, int H, int N, int d, int bq, int bk,
                 float* q_desc, float* k_desc, void* stream) {
  int rc = check_shape(B, H, N, d, bq, bk);
  if (rc) return rc;
  if (!q || !k || !q_desc || !k_desc) return fail(SA_ERR_INVALID_ARG, "sa_trip_pool: null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(q_desc) || !aligned16(k_desc))
    return fail(SA_ERR_ALIGN, "sa_trip_pool: pointers must be 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_trip_pool(q, B * H, N, d, bq, q_desc, st);
  if (e == cudaSuccess) e = launch_trip_pool(k, B * H, N, d, bk, k_desc, st);
  return e == cudaSuccess ? SA_OK : cuda_fail(e, "sa_trip_pool");
}

int sa_tile_heatmap(const uint16_t* q, const uint16_t* k, int B, int H, int N, int d, int bq, int bk,
                    double scale, const int32_t* rows_opt, int n_rows, float* heat, float* lse_opt,
                    void* stream) {
  int rc = check_shape(B, H, N, d, bq, bk);
  if (rc) return rc;
  if (!q || !k || !heat) return fail(SA_ERR_INVALID_ARG, "sa_tile_heatmap: null pointer");
  if (!isfinite(scale)) return fail(SA_ERR_INVALID_ARG, "scale must be finite");
  const void* ptrs[] = {q, k, heat, lse_opt, rows_opt};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(SA_ERR_ALIGN, "sa_tile_heatmap: pointers must be 16-byte aligned");
  const long long all_rows = static_cast<long long>(B) * H * ((N + bq - 1) / bq);
  if (rows_opt && (n_rows < 0 || n_rows > all_rows))
    return fail(SA_ERR_INVALID_ARG, "sa_tile_heatmap: n_rows = %d outside [0, %lld]", n_rows, all_rows);
  if (all_rows > 0x7FFFFFFFLL) return fail(SA_ERR_UNSUPPORTED, "sa_tile_heatmap: too many query-block rows");
  if (scale <= 0.0) scale = 1.0 / sqrt(static_cast<double>(d));
  const int n_items = rows_opt ? n_rows : static_cast<int>(all_rows);
  cudaError_t e = launch_heat(q, k, B * H, N, d, bq, rows_opt, n_items, scale, heat, lse_opt,
                              static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SA_OK : cuda_fail(e, "sa_tile_heatmap");
}

int sa_select_mask(const float* scores, int B, int H, int n_qb, int n_kb, double topk_frac, double topp,
                   int32_t* kv_idx, int32_t* kv_cnt, uint8_t* mask_opt, void* stream) {
  if (B <= 0 || H <= 0 || n_qb <= 0 || n_kb <= 0)
    return fail(SA_ERR_INVALID_ARG, "sa_select_mask: B, H, n_qb and n_kb must be positive");
  if (n_kb > kMaxKeyBlocks) return fail(SA_ERR_UNSUPPORTED, "n_kb = %d exceeds %d", n_kb, kMaxKeyBlocks);
  const long long rows = static_cast<long long>(B) * H * n_qb;
  if (rows > 0x7FFFFFFFLL || rows * n_kb >= (1LL << 34)) return fail(SA_ERR_UNSUPPORTED, "sa_select_mask: too large");
  if (!scores || !kv_idx || !kv_cnt) return fail(SA_ERR_INVALID_ARG, "sa_select_mask: null pointer");
  if (!(topk_frac > 0.0 && topk_frac <= 1.0)) return fail(SA_ERR_INVALID_ARG, "topk_frac %g outside (0, 1]", topk_frac);
  if (!(topp >= 0.0 && topp <= 1.0)) return fail(SA_ERR_INVALID_ARG, "topp %g outside [0, 1]", topp);
  const void* ptrs[] = {scores, kv_idx, kv_cnt, mask_opt};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(SA_ERR_ALIGN, "sa_select_mask: pointers must be 16-byte aligned");
  const int k_sel = static_cast<int>(fmin(static_cast<double>(n_kb), fmax(1.0, ceil(topk_frac * n_kb - 1e-9))));
  cudaError_t e = launch_select(scores, n_kb, static_cast<int>(rows), n_kb, k_sel, topp, kv_idx, kv_cnt, mask_opt,
                                static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SA_OK : cuda_fail(e, "sa_select_mask");
}

int sa_tile_permutation(int H, int T, int Hh, int W, const int32_t* tiles, int32_t* perm, void* stream) {
  if (H < 1 || H > kMaxPermHeads) return fail(SA_ERR_INVALID_ARG, "sa_tile_permutation: H = %d outside [1, %d]", H, kMaxPermHeads);
  if (T < 1 || Hh < 1 || W < 1) return fail(SA_ERR_INVALID_ARG, "sa_tile_permutation: grid dimensions must be positive");
  if (static_cast<long long>(T) * Hh * W * H >= (1LL << 31)) return fail(SA_ERR_UNSUPPORTED, "sa_tile_permutation: grid too large");
  if (!tiles || !perm) return fail(SA_ERR_INVALID_ARG, "sa_tile_permutation: null pointer");
  if (!aligned16(perm)) return fail(SA_ERR_ALIGN, "sa_tile_permutation: perm must be 16-byte aligned");
  for (int h = 0; h < H; ++h)
    if (tiles[3 * h] < 1 || tiles[3 * h + 1] < 1 || tiles[3 * h + 2] < 1)
      return fail(SA_ERR_INVALID_ARG, "sa_tile_permutation: tile of head %d has a dimension below 1", h);
  cudaError_t e = launch_tile_perm(H, T, Hh, W, tiles, perm, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SA_OK : cuda_fail(e, "sa_tile_permutation");
}

int sa_permute_tokens(const uint16_t* x, const int32_t* perm, int B, int H, int N, int d, int inverse,
                      uint16_t* y, void* stream) {
  int rc = check_shape(B, H, N, d, 64, 64);
  if (rc) return rc;
  if (!x || !perm || !y) return fail(SA_ERR_INVALID_ARG, "sa_permute_tokens: null pointer");
  if (x == y) return fail(SA_ERR_INVALID_ARG, "sa_permute_tokens: y must not alias x");
  if (!aligned16(x) || !aligned16(y) || !aligned16(perm))
    return fail(SA_ERR_ALIGN, "sa_permute_tokens: pointers must be 16-byte aligned");
  cudaError_t e = launch_permute_rows(x, perm, B * H, H, N, d, inverse ? 1 : 0, y, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SA_OK : cuda_fail(e, "sa_permute_tokens");
}

size_t sa_sparse_attn_bwd_workspace_size(int B, int H, int N, int d, int bq, int bk) {
  if (check_shape(B, H, N, d, bq, bk)) return 0;
  return bwd_ws_bytes(B * H, N, (N + bq - 1) / bq, (N + bk - 1) / bk);
}

int sa_sparse_attn_bwd(const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint16_t* o,
                       const float* lse, const uint16_t* dout, int B, int H, int N, int d, int bq, int bk,
                       const int32_t* kv_idx, const int32_t* kv_cnt, double scale, float* dq, float* dk,
                       float* dv, void* workspace, size_t ws_bytes, void* stream) {
  int rc = check_shape(B, H, N, d, bq, bk);
  if (rc) return rc;
  if (!q || !k || !v || !o || !lse || !dout || !kv_idx || !kv_cnt || !dq || !dk || !dv)
    return fail(SA_ERR_INVALID_ARG, "sa_sparse_attn_bwd: null pointer");
  if (!isfinite(scale)) return fail(SA_ERR_INVALID_ARG, "scale must be finite");
  const void* ptrs[] = {q, k, v, o, lse, dout, kv_idx, kv_cnt, dq, dk, dv, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(SA_ERR_ALIGN, "sa_sparse_attn_bwd: pointers must be 16-byte aligned");
  const int nqb = (N + bq - 1) / bq, nkb = (N + bk - 1) / bk;
  const size_t need = bwd_ws_bytes(B * H, N, nqb, nkb);
  if (!workspace || ws_bytes < need)
    return fail(SA_ERR_WORKSPACE, "sa_sparse_attn_bwd: workspace of %zu bytes needed", need);
  if (scale <= 0.0) scale = 1.0 / sqrt(static_cast<double>(d));
  BwdArgs a{q, k, v, dout, lse, nullptr, kv_idx, kv_cnt, nullptr, nullptr, dq, dk, dv,
            B * H, N, bq, nqb, nkb, (nkb + 1) / 2, static_cast<float>(scale),
            static_cast<float>(scale * 1.4426950408889634)};
  cudaError_t e = launch_sparse_attn_bwd(a, d, o, workspace, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SA_OK : cuda_fail(e, "sa_sparse_attn_bwd");
}

size_t sa_linear_bwd_workspace_size(int B, int H, int N, int d) {
  if (check_shape(B, H, N, d, 64, 64)) return 0;
  return lin_bwd_ws_bytes(B * H, N, d);
}

int sa_linear_bwd(const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* kv_state, const float* ksum,
                  const uint16_t* dout_l, int B, int H, int N, int d, int accumulate, float* dq, float* dk, float* dv,
                  void* workspace, size_t ws_bytes, void* stream) {
  int rc = check_shape(B, H, N, d, 64, 64);
  if (rc) return rc;
  if (!q || !k || !v || !kv_state || !ksum || !dout_l || !dq || !dk || !dv)
    return fail(SA_ERR_INVALID_ARG, "sa_linear_bwd: null pointer");
  const void* ptrs[] = {q, k, v, kv_state, ksum, dout_l, dq, dk, dv, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(SA_ERR_ALIGN, "sa_linear_bwd: pointers must be 16-byte aligned");
  const size_t need = lin_bwd_ws_bytes(B * H, N, d);
  if (!workspace || ws_bytes < need) return fail(SA_ERR_WORKSPACE, "sa_linear_bwd: workspace of %zu bytes needed", need);
  cudaError_t e = launch_linear_bwd(q, k, v, kv_state, ksum, dout_l, B * H, N, d, dq, dk, dv, accumulate ? 1 : 0,
                                    workspace, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SA_OK : cuda_fail(e, "sa_linear_bwd");
}

size_t sa_blend_bwd_workspace_size(int B, int H, int N, int d) {
  if (check_shape(B, H, N, d, 64, 64)) return 0;
  return blend_bwd_ws_bytes(B * H, N, d);
}

int sa_blend_bwd(const uint16_t* o_s, const uint16_t* o_l, const float* alpha, const uint16_t* dout, int B, int H,
                 int N, int d, uint16_t* do_s, uint16_t* do_l, float* dalpha, void* workspace, size_t ws_bytes,
                 void* stream) {
  int rc = check_shape(B, H, N, d, 64, 64);
  if (rc) return rc;
  if (!o_s || !o_l || !alpha || !dout || !do_s || !do_l || !dalpha)
    return fail(SA_ERR_INVALID_ARG, "sa_blend_bwd: null pointer");
  const void* ptrs[] = {o_s, o_l, alpha, dout, do_s, do_l, dalpha, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(SA_ERR_ALIGN, "sa_blend_bwd: pointers must be 16-byte aligned");
  const size_t need = blend_bwd_ws_bytes(B * H, N, d);
  if (!workspace || ws_bytes < need) return fail(SA_ERR_WORKSPACE, "sa_blend_bwd: workspace of %zu bytes needed", need);
  cudaError_t e = launch_blend_bwd(o_s, o_l, alpha, dout, B, H, N, d, do_s, do_l, dalpha, workspace,
                                   static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SA_OK : cuda_fail(e, "sa_blend_bwd");
}

}  // extern "C"
