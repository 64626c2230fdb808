// lin_bwd_kernels.cu — backward pass of the linear branch and of the alpha blend
// (pages: "SLA2" 提案手法 ② the blend O = alpha ⊙ O_s + (1 - alpha) ⊙ O_l and
// ③ full-precision backward; "SALAD" §2.1 the elu+1 linear attention).
//
// With phi = elu + 1, S = sum_j phi(k_j) v_j^T, z = sum_j phi(k_j), and per
// query num = phi(q) S, den = phi(q) . z, O_l = num / den:
//   dnum = dO_l / den,  dden = -(dO_l . O_l) / den
//   dq   = (S dnum + dden z) * phi'(q)
//   dS   = sum_i phi(q_i) dnum_i^T,  dz = sum_i dden_i phi(q_i)
//   dk   = (dS v + dz) * phi'(k),  dv = phi(k)^T dS
// These are O(N d^2) per head, small next to the sparse attention, and run on
// fp32 CUDA cores: lin_q_kernel (one warp per query token, S and z of the head
// in shared memory), lin_dsz_kernel (partial dS, dz over token chunks),
// lin_reduce_kernel (fixed-order sum of the partials: deterministic),
// lin_k_kernel (one warp per key token, dS and dz in shared memory).
// blend_bwd_kernel: dO_s = alpha dO, dO_l = (1 - alpha) dO and partial sums of
// dO (O_s - O_l) per head and chunk, reduced in a fixed order into dalpha.
#include "sa_internal.h"

namespace sa {

namespace linb {
constexpr int kChunk = 512;           // tokens per partial of dS, dz and dalpha
constexpr int kWarps = 8;
}

__device__ __forceinline__ float bf16_at(const __nv_bfloat16* p, long long i) { return __bfloat162float(p[i]); }
__device__ __forceinline__ float phi_f(float x) { return x > 0.f ? x + 1.f : __expf(x); }
__device__ __forceinline__ float phi_grad_f(float x) { return x > 0.f ? 1.f : __expf(x); }

// One warp per query token; lane l owns columns c = l + 32 j. Writes dq (or adds
// into it), dnum [BH, N, d] and dden [BH, N].
template <int D>
__global__ void __launch_bounds__(linb::kWarps * 32) lin_q_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ dol, const float* __restrict__ S,
    const float* __restrict__ z, int N, int tok_per_cta, float* __restrict__ dq, int accumulate,
    float* __restrict__ dnum, float* __restrict__ dden) {
  constexpr int J = D / 32;
  extern __shared__ float sm[];
  constexpr int LD = D + 1;              // padded row stride: row and column walks are both conflict-free
  float* sS = sm;                        // [D][LD]
  float* sz = sS + D * LD;               // [D]
  float* sv = sz + D;                    // [kWarps][2][D] per-warp vectors
  const int bh = blockIdx.y;
  for (int i = threadIdx.x; i < D * D; i += blockDim.x) sS[(i / D) * LD + i % D] = S[static_cast<long long>(bh) * D * D + i];
  for (int i = threadIdx.x; i < D; i += blockDim.x) sz[i] = z[static_cast<long long>(bh) * D + i];
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* fqv = sv + warp * 2 * D;
  float* dnv = fqv + D;
  const int t0 = blockIdx.x * tok_per_cta, t1 = min(N, t0 + tok_per_cta);
  for (int t = t0 + warp; t < t1; t += linb::kWarps) {
    const long long r = static_cast<long long>(bh) * N + t;
    float fq[J], qx[J], go[J];
    float den = 0.f;
#pragma unroll
    for (int j = 0; j < J; ++j) {
      const int c = lane + 32 * j;
      qx[j] = bf16_at(q, r * D + c);
      fq[j] = phi_f(qx[j]);
      go[j] = bf16_at(dol, r * D + c);
      fqv[c] = fq[j];
      den = fmaf(fq[j], sz[c], den);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) den += __shfl_xor_sync(0xFFFFFFFFu, den, off);
    __syncwarp();
    float num[J];
#pragma unroll
    for (int j = 0; j < J; ++j) num[j] = 0.f;
    for (int aa = 0; aa < D; ++aa) {
      const float f = fqv[aa];
#pragma unroll
      for (int j = 0; j < J; ++j) num[j] = fmaf(f, sS[aa * LD + lane + 32 * j], num[j]);
    }
    const float inv = 1.f / den;
    float dot = 0.f;
#pragma unroll
    for (int j = 0; j < J; ++j) dot = fmaf(go[j], num[j] * inv, dot);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xFFFFFFFFu, dot, off);
    const float dd = -dot * inv;
#pragma unroll
    for (int j = 0; j < J; ++j) {
      const int c = lane + 32 * j;
      const float dn = go[j] * inv;
      dnv[c] = dn;
      dnum[r * D + c] = dn;
    }
    if (lane == 0) dden[r] = dd;
    __syncwarp();
    // dfq[a] = sum_c S[a, c] dnum[c] + dden z[a]; lane owns rows a = lane + 32 j
#pragma unroll
    for (int j = 0; j < J; ++j) {
      const int aa = lane + 32 * j;
      float acc = dd * sz[aa];
      for (int c = 0; c < D; ++c) acc = fmaf(sS[aa * LD + c], dnv[c], acc);
      const float g = acc * phi_grad_f(qx[j]);
      dq[r * D + aa] = accumulate ? dq[r * D + aa] + g : g;
    }
    __syncwarp();
  }
}

// Partial dS (d x d) and dz over one chunk of tokens: thread i owns entries
// e = i, i + blockDim, ... of dS; phi(q) and dnum of each token are staged in
// shared memory.
template <int D>
__global__ void __launch_bounds__(256) lin_dsz_kernel(const __nv_bfloat16* __restrict__ q,
                                                      const float* __restrict__ dnum, const float* __restrict__ dden,
                                                      int N, int n_chunks, float* __restrict__ part) {
  __shared__ float fq[32][D];
  __shared__ float dn[32][D];
  __shared__ float ddv[32];
  const int bh = blockIdx.y, ch = blockIdx.x;
  const int t0 = ch * linb::kChunk, t1 = min(N, t0 + linb::kChunk);
  constexpr int E = D * D / 256;          // dS entries per thread
  float acc[E], accz = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  for (int tb = t0; tb < t1; tb += 32) {
    const int nt = min(32, t1 - tb);
    for (int i = threadIdx.x; i < 32 * D; i += 256) {
      const int tt = i / D, c = i % D;
      const long long r = static_cast<long long>(bh) * N + tb + tt;
      fq[tt][c] = tt < nt ? phi_f(bf16_at(q, r * D + c)) : 0.f;
      dn[tt][c] = tt < nt ? dnum[r * D + c] : 0.f;
    }
    if (threadIdx.x < 32) ddv[threadIdx.x] = threadIdx.x < nt ? dden[static_cast<long long>(bh) * N + tb + threadIdx.x] : 0.f;
    __syncthreads();
    for (int tt = 0; tt < nt; ++tt) {
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const int idx = threadIdx.x + 256 * e;
        acc[e] = fmaf(fq[tt][idx / D], dn[tt][idx % D], acc[e]);
      }
      if (threadIdx.x < D) accz = fmaf(ddv[tt], fq[tt][threadIdx.x], accz);
    }
    __syncthreads();
  }
  float* p = part + (static_cast<long long>(bh) * n_chunks + ch) * (D * D + D);
#pragma unroll
  for (int e = 0; e < E; ++e) p[threadIdx.x + 256 * e] = acc[e];
  if (threadIdx.x < D) p[D * D + threadIdx.x] = accz;
}

// Fixed-order sum of the chunk partials: out[bh][e] for e < len.
__global__ void lin_reduce_kernel(const float* __restrict__ part, int n_chunks, int len, float* __restrict__ out) {
  const int bh = blockIdx.y;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= len) return;
  float acc = 0.f;
  for (int c = 0; c < n_chunks; ++c) acc += part[(static_cast<long long>(bh) * n_chunks + c) * len + e];
  out[static_cast<long long>(bh) * len + e] = acc;
}

// One warp per key token: dk = (dS v + dz) * phi'(k), dv = phi(k)^T dS.
template <int D>
__global__ void __launch_bounds__(linb::kWarps * 32) lin_k_kernel(
    const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v, const float* __restrict__ dsz,
    int N, int tok_per_cta, float* __restrict__ dk, float* __restrict__ dv, int accumulate) {
  constexpr int J = D / 32;
  extern __shared__ float sm[];
  constexpr int LD = D + 1;               // padded row stride, as in lin_q_kernel
  float* sS = sm;                         // dS [D][LD]
  float* sz = sS + D * LD;                // dz [D]
  float* sv = sz + D;                     // [kWarps][2][D]
  const int bh = blockIdx.y;
  const float* src = dsz + static_cast<long long>(bh) * (D * D + D);
  for (int i = threadIdx.x; i < D * D; i += blockDim.x) sS[(i / D) * LD + i % D] = src[i];
  for (int i = threadIdx.x; i < D; i += blockDim.x) sz[i] = src[D * D + i];
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* vv = sv + warp * 2 * D;
  float* fk = vv + D;
  const int t0 = blockIdx.x * tok_per_cta, t1 = min(N, t0 + tok_per_cta);
  for (int t = t0 + warp; t < t1; t += linb::kWarps) {
    const long long r = static_cast<long long>(bh) * N + t;
    float kx[J];
#pragma unroll
    for (int j = 0; j < J; ++j) {
      const int c = lane + 32 * j;
      kx[j] = bf16_at(k, r * D + c);
      fk[c] = phi_f(kx[j]);
      vv[c] = bf16_at(v, r * D + c);
    }
    __syncwarp();
#pragma unroll
    for (int j = 0; j < J; ++j) {
      const int aa = lane + 32 * j;
      float gk = sz[aa], gv = 0.f;
      for (int c = 0; c < D; ++c) {
        gk = fmaf(sS[aa * LD + c], vv[c], gk);      // (dS v)[a]
        gv = fmaf(fk[c], sS[c * LD + aa], gv);      // (phi(k)^T dS)[a]
      }
      gk *= phi_grad_f(kx[j]);
      dk[r * D + aa] = accumulate ? dk[r * D + aa] + gk : gk;
      dv[r * D + aa] = accumulate ? dv[r * D + aa] + gv : gv;
    }
    __syncwarp();
  }
}

// dO_s = alpha dO, dO_l = (1 - alpha) dO, and per (head, chunk) partials of
// sum over tokens of dO (O_s - O_l); thread c of a CTA owns channel c.
template <int D>
__global__ void __launch_bounds__(D) blend_bwd_kernel(const __nv_bfloat16* __restrict__ o_s,
                                                      const __nv_bfloat16* __restrict__ o_l,
                                                      const float* __restrict__ alpha,
                                                      const __nv_bfloat16* __restrict__ dout, int H, int N,
                                                      int n_chunks, __nv_bfloat16* __restrict__ do_s,
                                                      __nv_bfloat16* __restrict__ do_l, float* __restrict__ part) {
  const int bh = blockIdx.y, ch = blockIdx.x, c = threadIdx.x;
  const float al = alpha[static_cast<long long>(bh % H) * D + c];
  const int t0 = ch * linb::kChunk, t1 = min(N, t0 + linb::kChunk);
  float acc = 0.f;
  for (int t = t0; t < t1; ++t) {
    const long long i = (static_cast<long long>(bh) * N + t) * D + c;
    const float g = __bfloat162float(dout[i]);
    acc = fmaf(g, __bfloat162float(o_s[i]) - __bfloat162float(o_l[i]), acc);
    do_s[i] = __float2bfloat16_rn(al * g);
    do_l[i] = __float2bfloat16_rn((1.f - al) * g);
  }
  part[(static_cast<long long>(bh) * n_chunks + ch) * D + c] = acc;
}

// dalpha[h][c] = sum over batches b and chunks of the partials of (b, h).
__global__ void blend_alpha_kernel(const float* __restrict__ part, int B, int H, int n_chunks, int D,
                                   float* __restrict__ dalpha) {
  const int h = blockIdx.x, c = threadIdx.x;
  float acc = 0.f;
  for (int b = 0; b < B; ++b)
    for (int ch = 0; ch < n_chunks; ++ch)
      acc += part[((static_cast<long long>(b) * H + h) * n_chunks + ch) * D + c];
  dalpha[static_cast<long long>(h) * D + c] = acc;
}

size_t lin_bwd_ws_bytes(int BH, int N, int d) {
  const long long nch = (N + linb::kChunk - 1) / linb::kChunk;
  auto up = [](long long x) { return static_cast<size_t>((x + 255) / 256 * 256); };
  return up(static_cast<long long>(BH) * N * d * 4) + up(static_cast<long long>(BH) * N * 4) +
         up(static_cast<long long>(BH) * nch * (d * d + d) * 4) + up(static_cast<long long>(BH) * (d * d + d) * 4);
}

size_t blend_bwd_ws_bytes(int BH, int N, int d) {
  const long long nch = (N + linb::kChunk - 1) / linb::kChunk;
  return static_cast<size_t>((BH * nch * d * 4 + 255) / 256 * 256);
}

template <int D>
static cudaError_t launch_lin_bwd_d(const void* q, const void* k, const void* v, const float* S, const float* z,
                                    const void* dol, int BH, int N, float* dq, float* dk, float* dv, int accumulate,
                                    char* ws, cudaStream_t st) {
  auto up = [](long long x) { return static_cast<size_t>((x + 255) / 256 * 256); };
  const int nch = (N + linb::kChunk - 1) / linb::kChunk;
  float* dnum = reinterpret_cast<float*>(ws);
  float* dden = reinterpret_cast<float*>(ws + up(static_cast<long long>(BH) * N * D * 4));
  float* part = reinterpret_cast<float*>(reinterpret_cast<char*>(dden) + up(static_cast<long long>(BH) * N * 4));
  float* dsz = reinterpret_cast<float*>(reinterpret_cast<char*>(part) + up(static_cast<long long>(BH) * nch * (D * D + D) * 4));
  const size_t smem = (D * (D + 1) + D + linb::kWarps * 2 * D) * 4;
  cudaError_t e = cudaFuncSetAttribute(lin_q_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(lin_k_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem))) != cudaSuccess) return e;
  const int tpc = 256;
  const dim3 gt((N + tpc - 1) / tpc, BH);
  lin_q_kernel<D><<<gt, linb::kWarps * 32, smem, st>>>(static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(dol),
                                                       S, z, N, tpc, dq, accumulate, dnum, dden);
  lin_dsz_kernel<D><<<dim3(nch, BH), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(q), dnum, dden, N, nch, part);
  lin_reduce_kernel<<<dim3((D * D + D + 255) / 256, BH), 256, 0, st>>>(part, nch, D * D + D, dsz);
  lin_k_kernel<D><<<gt, linb::kWarps * 32, smem, st>>>(static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v),
                                                       dsz, N, tpc, dk, dv, accumulate);
  return cudaGetLastError();
}

cudaError_t launch_linear_bwd(const void* q, const void* k, const void* v, const float* S, const float* z,
                              const void* dol, int BH, int N, int d, float* dq, float* dk, float* dv, int accumulate,
                              void* ws, cudaStream_t st) {
  char* w = static_cast<char*>(ws);
  return d == 128 ? launch_lin_bwd_d<128>(q, k, v, S, z, dol, BH, N, dq, dk, dv, accumulate, w, st)
                  : launch_lin_bwd_d<64>(q, k, v, S, z, dol, BH, N, dq, dk, dv, accumulate, w, st);
}

cudaError_t launch_blend_bwd(const void* o_s, const void* o_l, const float* alpha, const void* dout, int B, int H,
                             int N, int d, void* do_s, void* do_l, float* dalpha, void* ws, cudaStream_t st) {
  const int nch = (N + linb::kChunk - 1) / linb::kChunk;
  float* part = static_cast<float*>(ws);
  const dim3 g(nch, B * H);
  const auto* os = static_cast<const __nv_bfloat16*>(o_s);
  const auto* ol = static_cast<const __nv_bfloat16*>(o_l);
  const auto* go = static_cast<const __nv_bfloat16*>(dout);
  auto* ds = static_cast<__nv_bfloat16*>(do_s);
  auto* dl = static_cast<__nv_bfloat16*>(do_l);
  if (d == 128) blend_bwd_kernel<128><<<g, 128, 0, st>>>(os, ol, alpha, go, H, N, nch, ds, dl, part);
  else blend_bwd_kernel<64><<<g, 64, 0, st>>>(os, ol, alpha, go, H, N, nch, ds, dl, part);
  blend_alpha_kernel<<<H, d, 0, st>>>(part, B, H, nch, d, dalpha);
  return cudaGetLastError();
}

}  // namespace sa
