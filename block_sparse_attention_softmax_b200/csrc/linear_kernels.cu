// linear_kernels.cu — the parallel linear-attention branch and the alpha blend
// (pages: "SALAD" §2.1, a linear-attention branch beside sparse attention over
// the same Q/K/V; "SLA2" 提案手法 ②, O = alpha ⊙ O_s + (1 - alpha) ⊙ O_l).
//
// phi(x) = elu(x) + 1. For each head:
//   state:  S = sum_j phi(k_j) v_j^T  [d, d],  z = sum_j phi(k_j)  [d]
//   output: O_l[i] = phi(q_i)^T S / phi(q_i)^T z
//   blend:  O[i]   = alpha ⊙ O_s[i] + (1 - alpha) ⊙ O_l[i]
// The state is summed over token splits into a fp32 workspace, then reduced in
// a fixed order, so results do not depend on scheduling.
#include "sa_internal.h"

namespace sa {

namespace {
constexpr int kLinThreads = 256;
constexpr int kLinTok = 32;      // tokens staged per step
constexpr int kSplitTokens = 512;

__device__ __forceinline__ float phi_f(float x) { return x > 0.f ? x + 1.f : expf(x); }

__device__ __forceinline__ float bf16_bits_to_f(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

int linear_splits(int BH, int N) {
  const int by_tokens = ceil_div(N, kSplitTokens);
  const int want = ceil_div(4 * 148, BH);
  return max(1, min(by_tokens, want));
}
}  // namespace

size_t linear_state_ws_bytes(int BH, int N, int d) {
  return static_cast<size_t>(BH) * linear_splits(BH, N) * (static_cast<size_t>(d) * d + d) * sizeof(float);
}

size_t linear_out_ws_bytes(int, int) { return 0; }

// Partial state of one token split. Thread (ti, tj) of a 16 x 16 grid owns
// rows [ti*D/16, +D/16) and columns [tj*D/16, +D/16) of S.
template <int D>
__global__ void __launch_bounds__(kLinThreads) linear_state_kernel(
    const uint16_t* __restrict__ k, const uint16_t* __restrict__ v, int N, int nsplit,
    float* __restrict__ part) {
  constexpr int R = D / 16;
  __shared__ float fk[kLinTok][D];
  __shared__ float vv[kLinTok][D];
  const int split = blockIdx.x, bh = blockIdx.y;
  const int per = ceil_div_dev(N, nsplit);
  const int t0 = split * per, t1 = min(N, t0 + per);
  const int ti = threadIdx.x / 16, tj = threadIdx.x % 16;
  float acc[R][R];
#pragma unroll
  for (int i = 0; i < R; ++i)
#pragma unroll
    for (int j = 0; j < R; ++j) acc[i][j] = 0.f;
  float zacc[R];
#pragma unroll
  for (int i = 0; i < R; ++i) zacc[i] = 0.f;
  const uint16_t* kb = k + static_cast<long long>(bh) * N * D;
  const uint16_t* vb = v + static_cast<long long>(bh) * N * D;
  for (int t = t0; t < t1; t += kLinTok) {
    __syncthreads();
    for (int e = threadIdx.x; e < kLinTok * D; e += blockDim.x) {
      const int r = e / D, c = e % D;
      const int tok = t + r;
      float a = 0.f, b = 0.f;
      if (tok < t1) {
        // phi(k) is rounded to bf16, as the tensor-core form of this branch does
        a = __bfloat162float(__float2bfloat16_rn(phi_f(bf16_bits_to_f(kb[static_cast<long long>(tok) * D + c]))));
        b = bf16_bits_to_f(vb[static_cast<long long>(tok) * D + c]);
      }
      fk[r][c] = a;
      vv[r][c] = b;
    }
    __syncthreads();
#pragma unroll 4
    for (int r = 0; r < kLinTok; ++r) {
      float av[R], bv[R];
#pragma unroll
      for (int i = 0; i < R; ++i) av[i] = fk[r][ti * R + i];
#pragma unroll
      for (int j = 0; j < R; ++j) bv[j] = vv[r][tj * R + j];
#pragma unroll
      for (int i = 0; i < R; ++i) {
#pragma unroll
        for (int j = 0; j < R; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        if (tj == 0) zacc[i] += av[i];
      }
    }
  }
  float* out = part + (static_cast<long long>(bh) * nsplit + split) * (D * D + D);
#pragma unroll
  for (int i = 0; i < R; ++i)
#pragma unroll
    for (int j = 0; j < R; ++j) out[(ti * R + i) * D + tj * R + j] = acc[i][j];
  if (tj == 0) {
#pragma unroll
    for (int i = 0; i < R; ++i) out[D * D + ti * R + i] = zacc[i];
  }
}

template <int D>
__global__ void linear_reduce_kernel(const float* __restrict__ part, int nsplit,
                                     float* __restrict__ kv_state, float* __restrict__ ksum) {
  const int bh = blockIdx.y;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= D * D + D) return;
  const float* p = part + static_cast<long long>(bh) * nsplit * (D * D + D) + e;
  float s = 0.f;
  for (int i = 0; i < nsplit; ++i) s += p[static_cast<long long>(i) * (D * D + D)];
  if (e < D * D) kv_state[static_cast<long long>(bh) * D * D + e] = s;
  else ksum[static_cast<long long>(bh) * D + (e - D * D)] = s;
}

// O_l (and the blend) for a tile of 64 tokens of one head. Thread (tr, tc) of a
// 16 x 16 grid computes tokens [tr*4, +4) and columns [tc*D/16, +D/16).
constexpr int kOutTok = 64;

template <int D>
__global__ void __launch_bounds__(kLinThreads) linear_out_kernel(
    const uint16_t* __restrict__ q, const float* __restrict__ kv_state,
    const float* __restrict__ ksum, const uint16_t* __restrict__ o_s,
    const float* __restrict__ alpha, int H, int N, uint16_t* __restrict__ o) {
  constexpr int C = D / 16;
  extern __shared__ float sm_lin[];
  float* S = sm_lin;                 // [D][D]
  float* z = S + D * D;              // [D]
  float* fq = z + D;                 // [kOutTok][D + 1]
  const int tile = blockIdx.x, bh = blockIdx.y;
  const int h = bh % H;
  const int tok0 = tile * kOutTok;
  const float* Sg = kv_state + static_cast<long long>(bh) * D * D;
  for (int e = threadIdx.x; e < D * D; e += blockDim.x) S[e] = Sg[e];
  for (int e = threadIdx.x; e < D; e += blockDim.x) z[e] = ksum[static_cast<long long>(bh) * D + e];
  const uint16_t* qb = q + static_cast<long long>(bh) * N * D;
  for (int e = threadIdx.x; e < kOutTok * D; e += blockDim.x) {
    const int r = e / D, c = e % D;
    const int tok = tok0 + r;
    float x = 0.f;
    if (tok < N) x = __bfloat162float(__float2bfloat16_rn(phi_f(bf16_bits_to_f(qb[static_cast<long long>(tok) * D + c]))));
    fq[r * (D + 1) + c] = x;
  }
  __syncthreads();
  const int tr = threadIdx.x / 16, tc = threadIdx.x % 16;
  float acc[4][C];
  float den[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    den[i] = 0.f;
#pragma unroll
    for (int j = 0; j < C; ++j) acc[i][j] = 0.f;
  }
  for (int c = 0; c < D; ++c) {
    float av[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) av[i] = fq[(tr * 4 + i) * (D + 1) + c];
    const float zc = z[c];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      den[i] = fmaf(av[i], zc, den[i]);
#pragma unroll
      for (int j = 0; j < C; ++j) acc[i][j] = fmaf(av[i], S[c * D + tc * C + j], acc[i][j]);
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int tok = tok0 + tr * 4 + i;
    if (tok >= N) continue;
    const long long base = (static_cast<long long>(bh) * N + tok) * D + tc * C;
    const float inv = 1.f / den[i];
#pragma unroll
    for (int j = 0; j < C; ++j) {
      float ol = acc[i][j] * inv;
      if (alpha) {
        const float al = alpha[static_cast<long long>(h) * D + tc * C + j];
        ol = al * bf16_bits_to_f(o_s[base + j]) + (1.f - al) * ol;
      }
      __nv_bfloat16 r = __float2bfloat16_rn(ol);
      o[base + j] = *reinterpret_cast<uint16_t*>(&r);
    }
  }
}

cudaError_t launch_linear_state(const LinearArgs& a, cudaStream_t st) {
  const int BH = a.B * a.H;
  const int ns = linear_splits(BH, a.N);
  float* part = static_cast<float*>(a.ws);
  dim3 g1(ns, BH);
  const auto* k = static_cast<const uint16_t*>(a.k);
  const auto* v = static_cast<const uint16_t*>(a.v);
  if (a.d == 128) linear_state_kernel<128><<<g1, kLinThreads, 0, st>>>(k, v, a.N, ns, part);
  else linear_state_kernel<64><<<g1, kLinThreads, 0, st>>>(k, v, a.N, ns, part);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int n = a.d * a.d + a.d;
  dim3 g2(ceil_div(n, 256), BH);
  if (a.d == 128) linear_reduce_kernel<128><<<g2, 256, 0, st>>>(part, ns, a.kv_state, a.ksum);
  else linear_reduce_kernel<64><<<g2, 256, 0, st>>>(part, ns, a.kv_state, a.ksum);
  return cudaGetLastError();
}

cudaError_t launch_linear_out(const LinearArgs& a, cudaStream_t st) {
  const int BH = a.B * a.H;
  dim3 grid(ceil_div(a.N, kOutTok), BH);
  const size_t smem = (static_cast<size_t>(a.d) * a.d + a.d + static_cast<size_t>(kOutTok) * (a.d + 1)) * sizeof(float);
  const auto* q = static_cast<const uint16_t*>(a.q);
  const auto* os = static_cast<const uint16_t*>(a.o_s);
  auto* o = static_cast<uint16_t*>(a.o);
  if (a.d == 128) {
    cudaFuncSetAttribute(linear_out_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    linear_out_kernel<128><<<grid, kLinThreads, smem, st>>>(q, a.kv_state, a.ksum, os, a.alpha, a.H, a.N, o);
  } else {
    cudaFuncSetAttribute(linear_out_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    linear_out_kernel<64><<<grid, kLinThreads, smem, st>>>(q, a.kv_state, a.ksum, os, a.alpha, a.H, a.N, o);
  }
  return cudaGetLastError();
}

}  // namespace sa
