// noalloc.cu — sa_build_mask_noalloc: the hybrid Top-k ∪ Top-p mask builder
// with its scratch (pooled means and block scores) in a fixed device array
// that is part of the library image, for callers that may not allocate device
// memory at call time.
//
// The array is created when the library's device code is loaded on a GPU and
// stays allocated on every GPU that loads the library until the process exits.
// Host code cannot use the array's name as a device address, so the first call
// in each CUDA context looks the address up with cudaGetSymbolAddress (with
// that context's device current) and caches it under the context; later calls
// in that context reuse it. A new context (after cudaDeviceReset, or a caller
// that switches contexts) loads the module again, has its own copy of the
// array, and gets its own lookup.
//
// Included from libsa.cu after sa_api.cu (same translation unit), so it reuses
// that file's argument checks and error reporting.
#include <mutex>

namespace sa {

// Fixed scratch size. Enough for, e.g., B*H = 12 heads at N = 32760 tokens,
// d = 128 (about 17 MB of pooled means, slices, score rows and row buffers).
constexpr size_t kStaticScratchBytes = size_t(32) << 20;
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

namespace {

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  }
  return fn;
}

constexpr int kMaxContexts = 64;
std::mutex g_scratch_mutex;
CUcontext g_scratch_ctx[kMaxContexts] = {};
void* g_scratch_ptr[kMaxContexts] = {};
int g_scratch_n = 0;

// Device address of g_static_scratch in the current context (looked up once
// per context). The lookup may load the module, which must not happen inside
// a stream capture: a first call while `stream` captures is refused.
int static_scratch(cudaStream_t stream, void** out) {
  // also makes the device's primary context current if no context is
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  cudaError_t e = cudaStreamIsCapturing(stream, &cap);
  if (e != cudaSuccess) return cuda_fail(e, "sa_build_mask_noalloc (cudaStreamIsCapturing)");
  CtxGetCurrentFn get = ctx_get_current();
  CUcontext ctx = nullptr;
  if (!get || get(&ctx) != CUDA_SUCCESS || !ctx)
    return fail(SA_ERR_CUDA, "sa_build_mask_noalloc: no current CUDA context");
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  for (int i = 0; i < g_scratch_n; ++i)
    if (g_scratch_ctx[i] == ctx) {
      *out = g_scratch_ptr[i];
      return SA_OK;
    }
  if (cap != cudaStreamCaptureStatusNone)
    return fail(SA_ERR_INVALID_ARG,
                "sa_build_mask_noalloc: the first call in a CUDA context must come before any stream "
                "capture (it looks up the fixed scratch's address)");
  void* p = nullptr;
  e = cudaGetSymbolAddress(&p, g_static_scratch);
  if (e != cudaSuccess) return cuda_fail(e, "sa_build_mask_noalloc (cudaGetSymbolAddress)");
  const int slot = g_scratch_n < kMaxContexts ? g_scratch_n++ : kMaxContexts - 1;
  g_scratch_ctx[slot] = ctx;
  g_scratch_ptr[slot] = p;
  *out = p;
  return SA_OK;
}

}  // namespace
}  // namespace sa

extern "C" {

int sa_build_mask_noalloc(const uint16_t* q, const uint16_t* k, int B, int H, int N, int d, int bq,
                          int bk, double topk_frac, double topp, double scale, int32_t* kv_idx,
                          int32_t* kv_cnt, uint8_t* mask_opt, void* stream) {
  using namespace sa;
  int rc = check_shape(B, H, N, d, bq, bk);
  if (rc) return rc;
  if (!q || !k || !kv_idx || !kv_cnt) return fail(SA_ERR_INVALID_ARG, "sa_build_mask_noalloc: null pointer");
  if (!(topk_frac > 0.0 && topk_frac <= 1.0)) return fail(SA_ERR_INVALID_ARG, "topk_frac %g outside (0, 1]", topk_frac);
  if (!(topp >= 0.0 && topp <= 1.0)) return fail(SA_ERR_INVALID_ARG, "topp %g outside [0, 1]", topp);
  if (!isfinite(scale)) return fail(SA_ERR_INVALID_ARG, "scale must be finite");
  const int nkb = (N + bk - 1) / bk;
  if (nkb > kMaxKeyBlocks) return fail(SA_ERR_UNSUPPORTED, "n_kb = %d exceeds %d", nkb, kMaxKeyBlocks);
  const void* ptrs[] = {q, k, kv_idx, kv_cnt, mask_opt};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(SA_ERR_ALIGN, "sa_build_mask_noalloc: pointers must be 16-byte aligned");
  // Same scratch layout as sa_build_mask with internal pooled means.
  const MaskWs w = mask_ws(B, H, N, d, bq, bk, true, true);
  if (w.total > kStaticScratchBytes)
    return fail(SA_ERR_UNSUPPORTED,
                "sa_build_mask_noalloc: this problem needs %zu bytes of scratch; the fixed scratch holds %zu "
                "(use sa_build_mask with a caller workspace)", w.total, kStaticScratchBytes);
  void* scratch = nullptr;
  rc = static_scratch(static_cast<cudaStream_t>(stream), &scratch);
  if (rc) return rc;
  if (scale <= 0.0) scale = 1.0 / sqrt(static_cast<double>(d));
  // Nothing here must start at zero: every scratch byte that is read was
  // written earlier in this call.
  char* ws = static_cast<char*>(scratch);
  float* qp = reinterpret_cast<float*>(ws + w.q_pool);
  float* kp = reinterpret_cast<float*>(ws + w.k_pool);
  const int BH = B * H;
  const int k_sel = static_cast<int>(fmin(static_cast<double>(nkb), fmax(1.0, ceil(topk_frac * nkb - 1e-9))));
  cudaError_t e = run_mask_builder(q, k, BH, N, d, bq, bk, k_sel, topp, scale, kv_idx, kv_cnt, mask_opt,
                                   qp, kp, ws, w, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SA_OK : cuda_fail(e, "sa_build_mask_noalloc");
}

}  // extern "C"
