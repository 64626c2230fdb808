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
// Every product is a 128-token tile times a d x d matrix of the head, so each
// runs on the tensor core (bf16 operands, the d x d matrix split into bf16
// hi + lo parts as in the forward, fp32 accumulators in TMEM):
//   lin_bwd_q_kernel   per (128-token tile, head): num = phi(Q) S; then, from
//                      num, dO_l and den = phi(q) . z, the rows' dnum and dden;
//                      dq = (dnum S^T + dden z) * phi'(q) with phi'(q) =
//                      min(phi(q), 1); dnum (bf16) to global memory for the
//                      next step, and the tile's partial dz
//   dS = phi(Q)^T dnum the linear branch's state kernel run on (Q, dnum)
//   lin_reduce_kernel  dz = fixed-order sum of the tiles' partials
//   lin_bwd_k_kernel   per (128-token tile, head): dk = (V dS^T + dz) *
//                      phi'(k) and dv = phi(K) dS
// The d x d operand in shared memory serves as B both ways: its rows of 64
// bf16 are MN-major for X S and K-major for X S^T. Deterministic: every sum
// has one owner and a fixed order.
// blend_bwd_kernel: dO_s = alpha dO, dO_l = (1 - alpha) dO and partial sums of
// dO (O_s - O_l) per head and chunk, reduced in a fixed order into dalpha.
#include "sa_internal.h"

namespace sa {

namespace linb {
constexpr int kChunk = 512;           // tokens per partial of dalpha
constexpr int kThreads = 256;         // 8 warps: two per TMEM lane quadrant

template <int D>
struct BwdLayout {
  using O = lin::OutLayout<D>;                 // the d x d operand (hi, lo) at offset 0
  static constexpr uint32_t OFF_X = 2 * O::B_BYTES;                   // first token tile
  static constexpr uint32_t OFF_Y = OFF_X + O::T_BYTES;               // second token tile
  static constexpr uint32_t OFF_RED = OFF_Y + O::T_BYTES;             // [2 halves][128 rows] float2
  static constexpr uint32_t OFF_ROW = OFF_RED + 2 * 128 * 8;          // [128] per-row value
  static constexpr uint32_t OFF_VEC = OFF_ROW + 128 * 4;              // [D] z or dz
  static constexpr uint32_t OFF_PART = OFF_VEC + D * 4;               // [256] partial sums
  static constexpr uint32_t OFF_BAR = OFF_PART + 256 * 4;             // 4 mbarriers + TMEM slot
  // at least 80 KB, so that at most two CTAs (2 x 256 TMEM columns) share an SM
  static constexpr uint32_t SMEM = (OFF_BAR + 64 + 1024 > 80 * 1024) ? OFF_BAR + 64 + 1024 : 80 * 1024;
};

// 16-byte unit u (8 features) of token row r in a [128 tokens x D] tile with
// 128-byte swizzle, 64 features per chunk
template <int D>
__device__ __forceinline__ uint32_t tile_unit(int r, int u) {
  return (u >> 3) * lin::OutLayout<D>::T_CHUNK + r * 128 + (((u & 7) ^ (r & 7)) << 4);
}
}


// phi applied in place to a [128 x D] bf16 tile (all 256 threads). Two threads
// per row; thread h takes units 4h..4h+3 of the first 64-feature chunk and the
// other four of the second, so that a quarter-warp's eight 16-byte accesses
// fall in eight different bank groups of the swizzled rows.
template <int D>
__device__ __forceinline__ void phi_tile_inplace(uint8_t* tile, int tid) {
  constexpr int UPT = D / 16;                   // 16-byte units per thread: half a row
  const int r = tid >> 1, h = tid & 1;
#pragma unroll
  for (int j = 0; j < UPT; ++j) {
    const int c = j >> 2;
    uint4* p = reinterpret_cast<uint4*>(tile + linb::tile_unit<D>(r, c * 8 + (j & 3) + 4 * (h ^ c)));
    uint4 w = *p;
    uint32_t* x = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
    for (int e = 0; e < 4; ++e)
      x[e] = pack_bf16x2(lin::phi_f(__uint_as_float(x[e] << 16)), lin::phi_f(__uint_as_float(x[e] & 0xFFFF0000u)));
    *p = w;
  }
}

// D/2 fp32 accumulator columns [col0, col0 + D/2) of this thread's TMEM lane
template <int D>
__device__ __forceinline__ void tmem_ld_half(uint32_t taddr, float (&v)[D / 2]) {
  uint32_t r[32];
#pragma unroll
  for (int c = 0; c < D / 2; c += 32) {
    tmem_ld32_wait(taddr + c, r);
#pragma unroll
    for (int e = 0; e < 32; ++e) v[c + e] = __uint_as_float(r[e]);
  }
}

// the 8 bf16 of 16-byte unit u of row r as floats
template <int D>
__device__ __forceinline__ void unit_f32(const uint8_t* tile, int r, int u, float (&f)[8]) {
  const uint4 w = *reinterpret_cast<const uint4*>(tile + linb::tile_unit<D>(r, u));
  const uint32_t x[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    f[2 * e] = __uint_as_float(x[e] << 16);
    f[2 * e + 1] = __uint_as_float(x[e] & 0xFFFF0000u);
  }
}

// K-major view of the d x d operand: the product X M^T (its rows of 64 bf16 are
// the K extent; chunks of 64 columns are B_CHUNK apart)
template <int D>
__device__ __forceinline__ uint64_t head_desc_k(uint32_t base, int kk) {
  return sw128_desc(base + (kk >> 2) * lin::OutLayout<D>::B_CHUNK + (kk & 3) * 32u, 16, 1024);
}
// MN-major view: the product X M
template <int D>
__device__ __forceinline__ uint64_t head_desc_mn(uint32_t base, int kk) {
  return sw128_desc(base + kk * 2048u, lin::OutLayout<D>::B_CHUNK, 1024);
}
template <int D>
__device__ __forceinline__ uint64_t tile_desc(uint32_t base, int kk) {
  return sw128_desc(base + (kk >> 2) * lin::OutLayout<D>::T_CHUNK + (kk & 3) * 32u, 16, 1024);
}

// acc (+)= X M (mn = true) or X M^T, with M as hi + lo
template <int D>
__device__ __forceinline__ void issue_tile_by_head(uint32_t acc, uint32_t x, uint32_t m, bool mn) {
  const uint32_t idesc = idesc_bf16_f32(128, D, false, mn);
  const uint32_t mlo = m + lin::OutLayout<D>::B_BYTES;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint64_t a = tile_desc<D>(x, kk);
    umma_ss(acc, a, mn ? head_desc_mn<D>(m, kk) : head_desc_k<D>(m, kk), idesc, kk > 0 ? 1u : 0u);
    umma_ss(acc, a, mn ? head_desc_mn<D>(mlo, kk) : head_desc_k<D>(mlo, kk), idesc, 1u);
  }
}

// dq (and dnum, the tile's dz partial) for one (tile, head)
template <int D>
__global__ void __launch_bounds__(linb::kThreads, 1)
    lin_bwd_q_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                     const __grid_constant__ CUtensorMap tmDN, const float* __restrict__ S,
                     const float* __restrict__ z, int N, float* __restrict__ dq, int accumulate,
                     float* __restrict__ dz_part) {
  using L = linb::BwdLayout<D>;
  constexpr int HC = D / 2, HU = HC / 8;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = lin::align1k(smem_raw);
  uint8_t* sX = smem + L::OFF_X;              // Q, then phi(Q)
  uint8_t* sY = smem + L::OFF_Y;              // dO_l, then dnum
  float2* red = reinterpret_cast<float2*>(smem + L::OFF_RED);
  float* srow = reinterpret_cast<float*>(smem + L::OFF_ROW);      // dden per row
  float* sz = reinterpret_cast<float*>(smem + L::OFF_VEC);
  float* spart = reinterpret_cast<float*>(smem + L::OFF_PART);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);   // [0] loads, [1] num, [2] dq
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.y, tile = blockIdx.x, tok0 = tile * 128;
  if (tid == 0) {
    for (int i = 0; i < 3; ++i) mbar_init(&bars[i], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (tid == 0) {
    mbar_arrive_expect_tx(&bars[0], 2 * lin::OutLayout<D>::T_BYTES);
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      tma_load_3d(sX + c * lin::OutLayout<D>::T_CHUNK, &tmQ, &bars[0], c * 64, tok0, bh);
      tma_load_3d(sY + c * lin::OutLayout<D>::T_CHUNK, &tmDO, &bars[0], c * 64, tok0, bh);
    }
  }
  build_head_operand<D>(smem, S, bh, tid, linb::kThreads);
  for (int i = tid; i < D; i += linb::kThreads) sz[i] = z[static_cast<long long>(bh) * D + i];
  if (warp == 1) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *tmem_slot;
  bool ok = mbar_wait(&bars[0], 0, abort_flag);
  phi_tile_inplace<D>(sX, tid);
  fence_proxy_async_smem();
  __syncthreads();
  if (tid == 0) {
    tc_fence_after();
    if (ok) issue_tile_by_head<D>(tm, smem_u32(sX), smem_u32(smem), true);   // num = phi(Q) S
    tc_commit(&bars[1]);
  }
  // epilogue 1: this thread's row, half the columns
  const int quad = warp & 3, half = warp >> 2;
  const int r = quad * 32 + lane;
  const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
  ok = mbar_wait(&bars[1], 0, abort_flag) && ok;
  tc_fence_after();
  float acc[HC];
  tmem_ld_half<D>(tm + lane_addr + half * HC, acc);
  float pden = 0.f, pdot = 0.f;
#pragma unroll
  for (int j = 0; j < HU; ++j) {
    float fq[8], go[8];
    unit_f32<D>(sX, r, half * HU + j, fq);
    unit_f32<D>(sY, r, half * HU + j, go);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      pden = fmaf(fq[e], sz[(half * HU + j) * 8 + e], pden);
      pdot = fmaf(go[e], acc[j * 8 + e], pdot);
    }
  }
  red[half * 128 + r] = make_float2(pden, pdot);
  __syncthreads();
  const float2 r0 = red[r], r1 = red[128 + r];
  const float den = r0.x + r1.x;
  const float inv = 1.f / den;
  const float dden = -((r0.y + r1.y) * inv) * inv;   // -(dO . num / den) / den
#pragma unroll
  for (int j = 0; j < HU; ++j) {
    float go[8];
    unit_f32<D>(sY, r, half * HU + j, go);
    uint4 w;
    w.x = pack_bf16x2(go[0] * inv, go[1] * inv);
    w.y = pack_bf16x2(go[2] * inv, go[3] * inv);
    w.z = pack_bf16x2(go[4] * inv, go[5] * inv);
    w.w = pack_bf16x2(go[6] * inv, go[7] * inv);
    *reinterpret_cast<uint4*>(sY + linb::tile_unit<D>(r, half * HU + j)) = w;
  }
  if (half == 0) srow[r] = dden;          // rows past N have dO = 0, so dden = 0
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  if (tid == 0) {
    tc_fence_after();
    if (ok) issue_tile_by_head<D>(tm + 128, smem_u32(sY), smem_u32(smem), false);   // dnum S^T
    tc_commit(&bars[2]);
  } else if (tid == 32) {
#pragma unroll
    for (int c = 0; c < D / 64; ++c)
      tma_store_3d(&tmDN, sY + c * lin::OutLayout<D>::T_CHUNK, c * 64, tok0, bh);   // rows past N are clipped
    bulk_commit();
  }
  {
    // partial dz[a] = sum over the tile's rows of dden * phi(q)[a]: feature a,
    // a share of the rows per thread, shares added in a fixed order
    constexpr int TPF = linb::kThreads / D, RPT = 128 / TPF;
    const int a = tid % D, part = tid / D;
    float sacc = 0.f;
    for (int rr = part * RPT; rr < (part + 1) * RPT; ++rr) {
      const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(sX + linb::tile_unit<D>(rr, a >> 3)) + (a & 7);
      sacc = fmaf(srow[rr], __bfloat162float(*e), sacc);
    }
    spart[tid] = sacc;
  }
  ok = mbar_wait(&bars[2], 0, abort_flag) && ok;
  tc_fence_after();
  tmem_ld_half<D>(tm + 128 + lane_addr + half * HC, acc);
  const int tok = tok0 + r;
  if (tok < N) {
    float* dst = dq + (static_cast<long long>(bh) * N + tok) * D + half * HC;
#pragma unroll
    for (int j = 0; j < HU; ++j) {
      float fq[8];
      unit_f32<D>(sX, r, half * HU + j, fq);
      float g[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int c = (half * HU + j) * 8 + e;
        g[e] = (acc[j * 8 + e] + dden * sz[c]) * fminf(fq[e], 1.f);     // phi'(q) = min(phi(q), 1)
      }
      float4* d4 = reinterpret_cast<float4*>(dst + j * 8);
      if (accumulate) {
        const float4 o0 = d4[0], o1 = d4[1];
        g[0] += o0.x; g[1] += o0.y; g[2] += o0.z; g[3] += o0.w;
        g[4] += o1.x; g[5] += o1.y; g[6] += o1.z; g[7] += o1.w;
      }
      d4[0] = make_float4(g[0], g[1], g[2], g[3]);
      d4[1] = make_float4(g[4], g[5], g[6], g[7]);
    }
  }
  __syncthreads();
  if (tid < D) {
    float sacc = 0.f;
    for (int p2 = 0; p2 < linb::kThreads / D; ++p2) sacc += spart[p2 * D + tid];
    dz_part[(static_cast<long long>(bh) * gridDim.x + tile) * D + tid] = sacc;
  }
  if (tid == 32) bulk_wait_all();
  if (tid == 0) {
    // anything still in flight after a failed wait lands before the memory is released
    mbar_drain(&bars[0], 0);
    mbar_drain(&bars[1], 0);
    mbar_drain(&bars[2], 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tm, 256);
  }
}

// dk and dv for one (tile, head)
template <int D>
__global__ void __launch_bounds__(linb::kThreads, 1)
    lin_bwd_k_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const float* __restrict__ dS, const float* __restrict__ dz, int N, float* __restrict__ dk,
                     float* __restrict__ dv, int accumulate) {
  using L = linb::BwdLayout<D>;
  constexpr int HC = D / 2, HU = HC / 8;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = lin::align1k(smem_raw);
  uint8_t* sX = smem + L::OFF_X;              // K, then phi(K)
  uint8_t* sY = smem + L::OFF_Y;              // V
  float* sz = reinterpret_cast<float*>(smem + L::OFF_VEC);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);   // [0] loads, [1] products
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.y, tok0 = blockIdx.x * 128;
  if (tid == 0) {
    for (int i = 0; i < 2; ++i) mbar_init(&bars[i], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (tid == 0) {
    mbar_arrive_expect_tx(&bars[0], 2 * lin::OutLayout<D>::T_BYTES);
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      tma_load_3d(sX + c * lin::OutLayout<D>::T_CHUNK, &tmK, &bars[0], c * 64, tok0, bh);
      tma_load_3d(sY + c * lin::OutLayout<D>::T_CHUNK, &tmV, &bars[0], c * 64, tok0, bh);
    }
  }
  build_head_operand<D>(smem, dS, bh, tid, linb::kThreads);
  for (int i = tid; i < D; i += linb::kThreads) sz[i] = dz[static_cast<long long>(bh) * D + i];
  if (warp == 1) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *tmem_slot;
  bool ok = mbar_wait(&bars[0], 0, abort_flag);
  phi_tile_inplace<D>(sX, tid);
  fence_proxy_async_smem();
  __syncthreads();
  if (tid == 0) {
    tc_fence_after();
    if (ok) {
      issue_tile_by_head<D>(tm, smem_u32(sY), smem_u32(smem), false);        // V dS^T
      issue_tile_by_head<D>(tm + 128, smem_u32(sX), smem_u32(smem), true);   // phi(K) dS
    }
    tc_commit(&bars[1]);
  }
  const int quad = warp & 3, half = warp >> 2;
  const int r = quad * 32 + lane;
  const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
  ok = mbar_wait(&bars[1], 0, abort_flag) && ok;
  tc_fence_after();
  const int tok = tok0 + r;
  float acc[HC];
  tmem_ld_half<D>(tm + lane_addr + half * HC, acc);
  if (tok < N) {
    float* dst = dk + (static_cast<long long>(bh) * N + tok) * D + half * HC;
#pragma unroll
    for (int j = 0; j < HU; ++j) {
      float fk[8], g[8];
      unit_f32<D>(sX, r, half * HU + j, fk);
#pragma unroll
      for (int e = 0; e < 8; ++e) g[e] = (acc[j * 8 + e] + sz[(half * HU + j) * 8 + e]) * fminf(fk[e], 1.f);
      float4* d4 = reinterpret_cast<float4*>(dst + j * 8);
      if (accumulate) {
        const float4 o0 = d4[0], o1 = d4[1];
        g[0] += o0.x; g[1] += o0.y; g[2] += o0.z; g[3] += o0.w;
        g[4] += o1.x; g[5] += o1.y; g[6] += o1.z; g[7] += o1.w;
      }
      d4[0] = make_float4(g[0], g[1], g[2], g[3]);
      d4[1] = make_float4(g[4], g[5], g[6], g[7]);
    }
  }
  tmem_ld_half<D>(tm + 128 + lane_addr + half * HC, acc);
  if (tok < N) {
    float* dst = dv + (static_cast<long long>(bh) * N + tok) * D + half * HC;
#pragma unroll
    for (int j = 0; j < HU; ++j) {
      float g[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) g[e] = acc[j * 8 + e];
      float4* d4 = reinterpret_cast<float4*>(dst + j * 8);
      if (accumulate) {
        const float4 o0 = d4[0], o1 = d4[1];
        g[0] += o0.x; g[1] += o0.y; g[2] += o0.z; g[3] += o0.w;
        g[4] += o1.x; g[5] += o1.y; g[6] += o1.z; g[7] += o1.w;
      }
      d4[0] = make_float4(g[0], g[1], g[2], g[3]);
      d4[1] = make_float4(g[4], g[5], g[6], g[7]);
    }
  }
  if (tid == 0) {
    mbar_drain(&bars[0], 0);
    mbar_drain(&bars[1], 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tm, 256);
  }
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
  const long long nt = (N + 127) / 128;
  auto up = [](long long x) { return static_cast<size_t>((x + 255) / 256 * 256); };
  return up(static_cast<long long>(BH) * N * d * 2) + up(static_cast<long long>(BH) * nt * d * 4) +
         up(static_cast<long long>(BH) * d * d * 4) + 2 * up(static_cast<long long>(BH) * d * 4) +
         up(static_cast<long long>(linear_state_ws_bytes(BH, N, d)));
}

size_t blend_bwd_ws_bytes(int BH, int N, int d) {
  const long long nch = (N + linb::kChunk - 1) / linb::kChunk;
  return static_cast<size_t>((BH * nch * d * 4 + 255) / 256 * 256);
}

template <int D>
static cudaError_t launch_lin_bwd_d(const void* q, const void* k, const void* v, const float* S, const float* z,
                                    const void* dol, int BH, int N, float* dq, float* dk, float* dv, int accumulate,
                                    char* ws, cudaStream_t st) {
  using L = linb::BwdLayout<D>;
  auto up = [](long long x) { return static_cast<size_t>((x + 255) / 256 * 256); };
  const int nt = (N + 127) / 128;
  char* w = ws;
  void* dnum = w;                                       // [BH, N, d] bf16
  w += up(static_cast<long long>(BH) * N * D * 2);
  float* dz_part = reinterpret_cast<float*>(w);         // [BH, nt, d]
  w += up(static_cast<long long>(BH) * nt * D * 4);
  float* dS = reinterpret_cast<float*>(w);              // [BH, d, d]
  w += up(static_cast<long long>(BH) * D * D * 4);
  float* dz = reinterpret_cast<float*>(w);              // [BH, d]
  w += up(static_cast<long long>(BH) * D * 4);
  float* zq = reinterpret_cast<float*>(w);              // [BH, d] (sum of phi(q); unused)
  w += up(static_cast<long long>(BH) * D * 4);
  void* state_ws = w;
  CUtensorMap mq, mdo, mdn, mk, mv;
  if (encode_tensor_map_3d_bf16(&mq, q, D, N, BH, 64, 128) != CUDA_SUCCESS ||
      encode_tensor_map_3d_bf16(&mdo, dol, D, N, BH, 64, 128) != CUDA_SUCCESS ||
      encode_tensor_map_3d_bf16(&mdn, dnum, D, N, BH, 64, 128) != CUDA_SUCCESS ||
      encode_tensor_map_3d_bf16(&mk, k, D, N, BH, 64, 128) != CUDA_SUCCESS ||
      encode_tensor_map_3d_bf16(&mv, v, D, N, BH, 64, 128) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(lin_bwd_q_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM);
  if (e != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(lin_bwd_k_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM)) != cudaSuccess)
    return e;
  const dim3 grid(nt, BH);
  lin_bwd_q_kernel<D><<<grid, linb::kThreads, L::SMEM, st>>>(mq, mdo, mdn, S, z, N, dq, accumulate, dz_part);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // dS = phi(Q)^T dnum: the state kernel with (Q, dnum) in the places of (K, V)
  LinearArgs la{};
  la.k = q;
  la.v = dnum;
  la.kv_state = dS;
  la.ksum = zq;
  la.B = BH;
  la.H = 1;
  la.N = N;
  la.d = D;
  la.ws = state_ws;
  if ((e = launch_linear_state(la, st)) != cudaSuccess) return e;
  lin_reduce_kernel<<<dim3((D + 255) / 256, BH), 256, 0, st>>>(dz_part, nt, D, dz);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  lin_bwd_k_kernel<D><<<grid, linb::kThreads, L::SMEM, st>>>(mk, mv, dS, dz, N, dk, dv, accumulate);
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
