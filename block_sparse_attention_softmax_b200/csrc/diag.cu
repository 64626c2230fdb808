// diag.cu — diagnostic entry points. They let tests reach the library's
// error-reporting path and its device-side approximations directly, without
// a fault: set or read the device status word, shorten the bound of every
// device-side wait so that a wait runs out on purpose, and evaluate the
// exponential helpers the attention softmax uses on caller data.
//
// Included from libsa.cu after sa_api.cu (same translation unit), so it
// shares the status word, the wait limit and that file's error reporting.

namespace sa {

// Two-pass exponential evaluation: y_poly from the FMA-pipe polynomial
// (inputs taken in pairs, as the softmax does), y_mufu from ex2.approx.
__global__ void diag_exp2_kernel(const float* __restrict__ x, float* __restrict__ y_poly,
                                 float* __restrict__ y_mufu, int n) {
  const long long j = 2LL * (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x);
  if (j >= n) return;
  const bool two = j + 1 < n;
  const float x0 = x[j];
  const float x1 = two ? x[j + 1] : 0.f;
  float e0, e1;
  exp2_poly2(f2_make(x0, x1), e0, e1);
  y_poly[j] = e0;
  y_mufu[j] = fast_exp2(x0);
  if (two) {
    y_poly[j + 1] = e1;
    y_mufu[j + 1] = fast_exp2(x1);
  }
}

// One thread waits, through the library's bounded wait, on an mbarrier that
// nothing arrives at; the wait runs out after g_wait_limit cycles and records
// the timeout in the status word. The barrier expects one arrival, and the
// waiting thread is the only one, so the wait cannot complete.
__global__ void diag_wait_kernel(int* out) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  abort_flag = 0;
  mbar_init(&bar, 1);
  fence_barrier_init();
  const bool ok = mbar_wait(&bar, 0, &abort_flag);
  out[0] = ok ? 1 : 0;
  out[1] = abort_flag;
}

}  // namespace sa

extern "C" {

int sa_diag_set_device_status(int code) {
  using namespace sa;
  cudaError_t e = cudaMemcpyToSymbol(g_device_status, &code, sizeof(int));
  return e == cudaSuccess ? SA_OK : cuda_fail(e, "sa_diag_set_device_status");
}

int sa_diag_set_wait_limit(long long cycles) {
  using namespace sa;
  if (cycles <= 0) cycles = kWaitLimitCycles;
  cudaError_t e = cudaMemcpyToSymbol(g_wait_limit, &cycles, sizeof(long long));
  return e == cudaSuccess ? SA_OK : cuda_fail(e, "sa_diag_set_wait_limit");
}

int sa_diag_wait_timeout(int* out, void* stream) {
  using namespace sa;
  if (!out) return fail(SA_ERR_INVALID_ARG, "sa_diag_wait_timeout: null pointer");
  diag_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(out);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SA_OK : cuda_fail(e, "sa_diag_wait_timeout");
}

int sa_diag_exp2(const float* x, float* y_poly, float* y_mufu, int n, void* stream) {
  using namespace sa;
  if (n < 0) return fail(SA_ERR_INVALID_ARG, "sa_diag_exp2: n = %d", n);
  if (n == 0) return SA_OK;
  if (!x || !y_poly || !y_mufu) return fail(SA_ERR_INVALID_ARG, "sa_diag_exp2: null pointer");
  const int threads = 256;
  const long long pairs = (static_cast<long long>(n) + 1) / 2;
  const int blocks = static_cast<int>((pairs + threads - 1) / threads);
  diag_exp2_kernel<<<blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(x, y_poly, y_mufu, n);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SA_OK : cuda_fail(e, "sa_diag_exp2");
}

}  // extern "C"
