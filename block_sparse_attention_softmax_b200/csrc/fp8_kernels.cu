// fp8_kernels.cu — per-head E4M3 quantisation of bf16 queries, keys or values
// for the low-bit forward (page: "SLA2" 提案手法 ③, the forward pass runs on
// low-bit queries, keys and values; the pages name no format, and E4M3 is the
// 8-bit float both operands of a tcgen05 kind::f8f6f4 product take here).
//
// For each (batch, head) slice: amax = max |x|, s = amax / 448 and r = 448 / amax
// in fp32 (both 1 for an all-zero slice), code = E4M3(x * r) with the product
// rounded to fp32, then to E4M3 by round-to-nearest-even, saturating at +-448.
//
//   amax_kernel   grid (chunks, slices): max |x| over a chunk, combined per
//                 slice with an integer atomicMax on the float's bit pattern
//                 (for non-negative floats the two orders agree; max is order
//                 independent, so the result is deterministic)
//   quant_kernel  8 elements per thread, 16-byte loads and 8-byte stores
//   scale_kernel  s written over amax once every code is written
#include <algorithm>

#include "sa_internal.h"

namespace sa {

namespace q8 {
constexpr int kThreads = 256;
}

// |x| of the 8 bf16 values in w, folded into m (NaN inputs are skipped by fmaxf)
__device__ __forceinline__ float amax8(const uint4 w, float m) {
  const uint32_t v[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    m = fmaxf(m, fabsf(__uint_as_float(v[j] << 16)));
    m = fmaxf(m, fabsf(__uint_as_float(v[j] & 0xFFFF0000u)));
  }
  return m;
}

__global__ void __launch_bounds__(q8::kThreads) amax_kernel(const __nv_bfloat16* __restrict__ x,
                                                            long long vec_per_slice,
                                                            float* __restrict__ amax) {
  __shared__ float red[q8::kThreads / 32];
  const long long bh = blockIdx.y;
  const uint4* p = reinterpret_cast<const uint4*>(x) + bh * vec_per_slice;
  float m = 0.f;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < vec_per_slice;
       i += static_cast<long long>(gridDim.x) * blockDim.x)
    m = amax8(__ldg(p + i), m);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < q8::kThreads / 32; ++w) m = fmaxf(m, red[w]);
    atomicMax(reinterpret_cast<int*>(amax + bh), __float_as_int(m));
  }
}

__global__ void __launch_bounds__(q8::kThreads) quant_kernel(const __nv_bfloat16* __restrict__ x,
                                                             long long vec_per_slice, long long n_vec,
                                                             const float* __restrict__ amax,
                                                             uint8_t* __restrict__ x8) {
  const uint4* p = reinterpret_cast<const uint4*>(x);
  uint2* out = reinterpret_cast<uint2*>(x8);
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n_vec;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float a = __ldg(amax + i / vec_per_slice);
    const float r = a > 0.f ? 448.f / a : 1.f;
    const uint4 w = __ldg(p + i);
    const uint32_t v[4] = {w.x, w.y, w.z, w.w};
    uint32_t c[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
      c[j] = pack_e4m3x2(__uint_as_float(v[j] << 16) * r, __uint_as_float(v[j] & 0xFFFF0000u) * r);
    out[i] = make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
  }
}

__global__ void scale_kernel(int n, float* __restrict__ amax_to_scale) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float a = amax_to_scale[i];
  amax_to_scale[i] = a > 0.f ? a / 448.f : 1.f;
}

cudaError_t launch_quantize_fp8(const void* x, long long BH, long long per_slice, uint8_t* x8, float* scale,
                                cudaStream_t st) {
  const long long vps = per_slice / 8;
  cudaError_t e = cudaMemsetAsync(scale, 0, static_cast<size_t>(BH) * sizeof(float), st);
  if (e != cudaSuccess) return e;
  const long long gx = std::min<long long>(std::max<long long>((vps + q8::kThreads * 16 - 1) / (q8::kThreads * 16), 1), 1024);
  if (BH > 65535) return cudaErrorInvalidValue;
  amax_kernel<<<dim3(static_cast<unsigned>(gx), static_cast<unsigned>(BH)), q8::kThreads, 0, st>>>(
      static_cast<const __nv_bfloat16*>(x), vps, scale);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const long long n_vec = vps * BH;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long grid = std::min<long long>((n_vec + q8::kThreads - 1) / q8::kThreads, static_cast<long long>(sms) * 16);
  quant_kernel<<<static_cast<unsigned>(std::max<long long>(grid, 1)), q8::kThreads, 0, st>>>(
      static_cast<const __nv_bfloat16*>(x), vps, n_vec, scale, x8);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  scale_kernel<<<static_cast<unsigned>((BH + 255) / 256), 256, 0, st>>>(static_cast<int>(BH), scale);
  return cudaGetLastError();
}

}  // namespace sa
