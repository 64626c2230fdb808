// mask_kernels.cu — block pooling, block scores and the hybrid Top-k ∪ Top-p
// selection (pages: "SLA2" 提案手法 ① mean pooling of Q and K;
// "SpargeAttention2" §2(1) hybrid Top-k + Top-p masking per attention row).
//
// Three kernels, all bound by memory or by a small amount of ALU work:
//   pool_kernel    Q, K [BH, N, d] bf16  ->  block means [BH, nb, d] fp32
//   score_kernel   means -> s[bh, qb, kb] = scale * <Qbar, Kbar> (fp32 partial
//                  sums of 32 products, combined in fp64, rounded once)
//   select_kernel  one query-block row per warp: radix select of the K_sel-th
//                  largest score (Top-k), a probability-mass search for the
//                  Top-p cut when Top-k alone does not reach p, and the
//                  ascending compacted index list.
#include "sa_internal.h"

namespace sa {

// ---------------------------------------------------------------- pooling
// One warp per token block. Each lane loads 16 B (8 bf16) per row it visits;
// d/8 lanes cover one row, so a warp reads 32*16 B per step.
template <int D>
__global__ void __launch_bounds__(256) pool_kernel(const __nv_bfloat16* __restrict__ q,
                                                   const __nv_bfloat16* __restrict__ k, int BH,
                                                   int N, int bq, int bk, int nqb, int nkb,
                                                   float* __restrict__ q_pool,
                                                   float* __restrict__ k_pool) {
  constexpr int LPR = D / 8;        // lanes per row
  constexpr int RPI = 32 / LPR;     // rows per warp step
  const int lane = threadIdx.x & 31;
  const long long warp = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long nq = static_cast<long long>(BH) * nqb;
  const long long total = nq + static_cast<long long>(BH) * nkb;
  if (warp >= total) return;
  const bool is_q = warp < nq;
  const long long w = is_q ? warp : warp - nq;
  const int nb = is_q ? nqb : nkb;
  const int b = is_q ? bq : bk;
  const int bh = static_cast<int>(w / nb);
  const int blk = static_cast<int>(w % nb);
  const __nv_bfloat16* src = (is_q ? q : k) + (static_cast<long long>(bh) * N + static_cast<long long>(blk) * b) * D;
  float* dst = (is_q ? q_pool : k_pool) + w * D;
  const int cnt = min(b, N - blk * b);
  const int r0 = lane / LPR;
  const int c8 = (lane % LPR) * 8;

  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  constexpr int UNROLL = 8;
  for (int r = r0; r < cnt; r += RPI * UNROLL) {
    uint4 v[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int rr = r + u * RPI;
      if (rr < cnt) {
        const uint4* p = reinterpret_cast<const uint4*>(src + static_cast<long long>(rr) * D + c8);
        asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(v[u].x), "=r"(v[u].y), "=r"(v[u].z), "=r"(v[u].w) : "l"(p));
      } else {
        v[u] = make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const uint32_t w4[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[2 * i] += __uint_as_float(w4[i] << 16);
        acc[2 * i + 1] += __uint_as_float(w4[i] & 0xFFFF0000u);
      }
    }
  }
#pragma unroll
  for (int off = LPR; off < 32; off <<= 1) {
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] += __shfl_xor_sync(0xFFFFFFFFu, acc[i], off);
  }
  if (r0 == 0) {
    const float fc = static_cast<float>(cnt);
    float4 a = make_float4(__fdiv_rn(acc[0], fc), __fdiv_rn(acc[1], fc), __fdiv_rn(acc[2], fc),
                           __fdiv_rn(acc[3], fc));
    float4 c = make_float4(__fdiv_rn(acc[4], fc), __fdiv_rn(acc[5], fc), __fdiv_rn(acc[6], fc),
                           __fdiv_rn(acc[7], fc));
    reinterpret_cast<float4*>(dst + c8)[0] = a;
    reinterpret_cast<float4*>(dst + c8)[1] = c;
  }
}

// ---------------------------------------------------------------- scores
// 64 x 64 tile of one head per CTA; thread (ty, tx) owns a 4 x 4 sub-tile.
// Products are summed in fp32 over 32 consecutive channels, the 32-channel
// partial sums in fp64, so the rounding error stays near 1e-7 of the score
// scale rather than the ~1e-6 of a 128-term fp32 sum.
constexpr int kScoreTile = 64;
constexpr int kScorePad = kScoreTile + 4;

template <int D>
__global__ void __launch_bounds__(256) score_kernel(const float* __restrict__ q_pool,
                                                    const float* __restrict__ k_pool, int nqb,
                                                    int nkb, double scale, float* __restrict__ s,
                                                    long long s_ld) {
  extern __shared__ float sm_score[];
  float* qs = sm_score;                  // [D][kScorePad], transposed
  float* ks = sm_score + D * kScorePad;  // [D][kScorePad]
  const int bh = blockIdx.z;
  const int qb0 = blockIdx.y * kScoreTile;
  const int kb0 = blockIdx.x * kScoreTile;
  const float* qp = q_pool + static_cast<long long>(bh) * nqb * D;
  const float* kp = k_pool + static_cast<long long>(bh) * nkb * D;
  for (int i = threadIdx.x; i < kScoreTile * (D / 4); i += blockDim.x) {
    const int r = i / (D / 4);
    const int c4 = (i % (D / 4)) * 4;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
    if (qb0 + r < nqb) a = *reinterpret_cast<const float4*>(qp + static_cast<long long>(qb0 + r) * D + c4);
    if (kb0 + r < nkb) b = *reinterpret_cast<const float4*>(kp + static_cast<long long>(kb0 + r) * D + c4);
    qs[(c4 + 0) * kScorePad + r] = a.x;
    qs[(c4 + 1) * kScorePad + r] = a.y;
    qs[(c4 + 2) * kScorePad + r] = a.z;
    qs[(c4 + 3) * kScorePad + r] = a.w;
    ks[(c4 + 0) * kScorePad + r] = b.x;
    ks[(c4 + 1) * kScorePad + r] = b.y;
    ks[(c4 + 2) * kScorePad + r] = b.z;
    ks[(c4 + 3) * kScorePad + r] = b.w;
  }
  __syncthreads();
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
  double acc64[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc64[i][j] = 0.0;
  for (int c0 = 0; c0 < D; c0 += 32) {
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll
    for (int c = c0; c < c0 + 32; ++c) {
      const float4 a = *reinterpret_cast<const float4*>(qs + c * kScorePad + ty * 4);
      const float4 b = *reinterpret_cast<const float4*>(ks + c * kScorePad + tx * 4);
      const float av[4] = {a.x, a.y, a.z, a.w};
      const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc64[i][j] += static_cast<double>(acc[i][j]);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int qb = qb0 + ty * 4 + i;
    if (qb >= nqb) continue;
    float* row = s + (static_cast<long long>(bh) * nqb + qb) * s_ld;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int kb = kb0 + tx * 4 + j;
      if (kb < nkb) row[kb] = __double2float_rn(acc64[i][j] * scale);
    }
  }
}

// ---------------------------------------------------------------- selection
// One warp per query-block row; rows of the grid are strided over the warps.
// Each warp keeps its row's keys and exponentials in its own slice of shared
// memory, so no block-wide barrier is ever needed.
//
//   keys    monotone uint32 image of the fp32 scores (larger score -> larger key)
//   e       exp(s - max) in fp32; Z and every probability mass in fp64
//   Top-k   4-pass radix select (8-bit digits, warp histogram with aggregated
//           atomics) of the K_sel-th largest key; ties at the cut are kept in
//           ascending block order (ballot prefix counts)
//   Top-p   only when the Top-k set holds less than p of the mass: bitwise
//           search for the largest key v with mass(key >= v) >= p * Z, then the
//           ties at v in block order until the mass is reached
//   output  the union is the longer of the two prefixes of the common order;
//           kept indices are written in ascending order (ballot compaction)
constexpr int kSelWarpsMax = 8;

__device__ __forceinline__ uint32_t score_key(float s) {
  const uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}
__device__ __forceinline__ int warp_sum_i(int v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

struct Cut {
  uint32_t key;    // threshold key value
  int above;       // elements strictly above the threshold
  int ties;        // elements equal to the threshold that are kept, lowest index first
};

// The `rank`-th largest key (1-based) of keys[0..n) and how many of its ties to keep.
__device__ Cut warp_select_rank(const uint32_t* keys, int n, int rank, uint32_t* hist) {
  const int lane = threadIdx.x & 31;
  uint32_t prefix = 0, pmask = 0;
  int need = rank, above = 0;
  for (int shift = 24; shift >= 0; shift -= 8) {
#pragma unroll
    for (int j = 0; j < 8; ++j) hist[lane * 8 + j] = 0;
    __syncwarp();
    for (int base = 0; base < n; base += 32) {
      const int i = base + lane;
      const uint32_t key = i < n ? keys[i] : 0u;
      const bool in = i < n && (key & pmask) == prefix;
      const uint32_t act = __ballot_sync(0xFFFFFFFFu, in);
      if (in) {
        const uint32_t dg = (key >> shift) & 255u;
        const uint32_t same = __match_any_sync(act, dg);
        if (lane == __ffs(same) - 1) atomicAdd(&hist[dg], static_cast<uint32_t>(__popc(same)));
      }
    }
    __syncwarp();
    // lane owns bins [8 lane, 8 lane + 8); suffix counts run from bin 255 down
    uint32_t c[8];
    uint32_t run = 0;
#pragma unroll
    for (int j = 7; j >= 0; --j) {
      run += hist[lane * 8 + j];
      c[j] = run;
    }
    uint32_t incl = run;  // inclusive suffix over lanes >= lane
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_down_sync(0xFFFFFFFFu, incl, o);
      if (lane + o < 32) incl += y;
    }
    const uint32_t higher = incl - run;   // elements in bins of higher lanes
    int hit = -1;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (static_cast<int>(higher + c[j]) >= need) hit = j;
    const uint32_t bal = __ballot_sync(0xFFFFFFFFu, hit >= 0);
    const int src = 31 - __clz(bal);
    const int hit_s = __shfl_sync(0xFFFFFFFFu, hit, src);
    uint32_t above_bin = 0;
    if (lane == src) above_bin = higher + (hit < 7 ? c[hit + 1] : 0u);
    above_bin = __shfl_sync(0xFFFFFFFFu, above_bin, src);
    need -= static_cast<int>(above_bin);
    above += static_cast<int>(above_bin);
    prefix |= static_cast<uint32_t>(src * 8 + hit_s) << shift;
    pmask |= 255u << shift;
    __syncwarp();
  }
  return Cut{prefix, above, need};
}

// Mass (fp64) of the elements whose key is >= v.
__device__ __forceinline__ double warp_mass_ge(const uint32_t* keys, const float* e, int n, uint32_t v) {
  const int lane = threadIdx.x & 31;
  double w = 0.0;
  for (int i = lane; i < n; i += 32)
    if (keys[i] >= v) w += static_cast<double>(e[i]);
  return warp_sum_d(w);
}

// Smallest m such that the m largest-key weights sum to >= target.
__device__ Cut warp_select_mass(const uint32_t* keys, const float* e, int n, double target) {
  const int lane = threadIdx.x & 31;
  uint32_t v = 0;
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = v | (1u << bit);
    if (warp_mass_ge(keys, e, n, cand) >= target) v = cand;
  }
  // strictly above v, and the ties at v
  int above = 0, nties = 0;
  double w_above = 0.0;
  float e_tie = 0.f;
  for (int i = lane; i < n; i += 32) {
    const uint32_t key = keys[i];
    if (key > v) {
      ++above;
      w_above += static_cast<double>(e[i]);
    } else if (key == v) {
      ++nties;
      e_tie = e[i];
    }
  }
  above = warp_sum_i(above);
  nties = warp_sum_i(nties);
  w_above = warp_sum_d(w_above);
  e_tie = warp_max(e_tie);            // every tie has the same weight
  int t = 0;
  double acc = w_above;
  while (acc < target && t < nties) {
    acc += static_cast<double>(e_tie);
    ++t;
  }
  if (acc < target) t = nties;        // rounding kept the total below the target
  if (above + t == 0) t = 1;
  return Cut{v, above, t};
}

__global__ void __launch_bounds__(kSelWarpsMax * 32) select_kernel(
    const float* __restrict__ s, long long s_ld, int n_rows, int nkb, int k_sel, double topp,
    int* __restrict__ kv_idx, int* __restrict__ kv_cnt, uint8_t* __restrict__ mask) {
  extern __shared__ __align__(16) uint8_t sm_sel[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wpc = blockDim.x >> 5;
  const size_t slice = static_cast<size_t>(nkb) * 8 + 256 * 4;
  uint32_t* keys = reinterpret_cast<uint32_t*>(sm_sel + warp * slice);
  float* e = reinterpret_cast<float*>(keys + nkb);
  uint32_t* hist = reinterpret_cast<uint32_t*>(e + nkb);
  const uint32_t lt = (1u << lane) - 1u;

  for (int row = blockIdx.x * wpc + warp; row < n_rows; row += gridDim.x * wpc) {
    const float* srow = s + static_cast<long long>(row) * s_ld;
    float mx = -INFINITY;
    for (int i = lane; i < nkb; i += 32) {
      const float v = __ldg(srow + i);
      keys[i] = score_key(v);
      e[i] = v;
      mx = fmaxf(mx, v);
    }
    mx = warp_max(mx);
    double z = 0.0;
    for (int i = lane; i < nkb; i += 32) {
      const float v = expf(e[i] - mx);
      e[i] = v;
      z += static_cast<double>(v);
    }
    z = warp_sum_d(z);
    __syncwarp();

    Cut cut{0u, 0, nkb};              // keep everything
    if (!(topp >= 1.0 || k_sel >= nkb)) {
      cut = warp_select_rank(keys, nkb, k_sel, hist);
      const double target = topp * z;
      // mass of the Top-k set (ties at the cut taken in block order)
      double wk = 0.0;
      int tie_before = 0;
      for (int base = 0; base < nkb; base += 32) {
        const int i = base + lane;
        const uint32_t key = i < nkb ? keys[i] : 0u;
        const bool tie = i < nkb && key == cut.key;
        const uint32_t tb = __ballot_sync(0xFFFFFFFFu, tie);
        const bool keep = i < nkb && (key > cut.key || (tie && tie_before + __popc(tb & lt) < cut.ties));
        if (keep) wk += static_cast<double>(e[i]);
        tie_before += __popc(tb);
      }
      wk = warp_sum_d(wk);
      if (wk < target) {
        const Cut cp = warp_select_mass(keys, e, nkb, target);
        if (cp.above + cp.ties > k_sel) cut = cp;
      }
    }

    // ascending compaction of the kept indices
    int* out = kv_idx + static_cast<long long>(row) * nkb;
    uint8_t* mrow = mask ? mask + static_cast<long long>(row) * nkb : nullptr;
    int written = 0, tie_before = 0;
    for (int base = 0; base < nkb; base += 32) {
      const int i = base + lane;
      const uint32_t key = i < nkb ? keys[i] : 0u;
      const bool tie = i < nkb && key == cut.key;
      const uint32_t tb = __ballot_sync(0xFFFFFFFFu, tie);
      const bool keep = i < nkb && (key > cut.key || (tie && tie_before + __popc(tb & lt) < cut.ties));
      const uint32_t kb = __ballot_sync(0xFFFFFFFFu, keep);
      if (keep) out[written + __popc(kb & lt)] = i;
      if (mrow && i < nkb) mrow[i] = keep ? 1 : 0;
      written += __popc(kb);
      tie_before += __popc(tb);
    }
    if (lane == 0) kv_cnt[row] = written;
    __syncwarp();
  }
}

// ---------------------------------------------------------------- uint8 mask -> lists
__global__ void __launch_bounds__(kSelWarpsMax * 32) compact_mask_kernel(
    const uint8_t* __restrict__ mask, int n_rows, int nkb, int* __restrict__ kv_idx,
    int* __restrict__ kv_cnt) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wpc = blockDim.x >> 5;
  const uint32_t lt = (1u << lane) - 1u;
  for (int row = blockIdx.x * wpc + warp; row < n_rows; row += gridDim.x * wpc) {
    const uint8_t* mrow = mask + static_cast<long long>(row) * nkb;
    int* out = kv_idx + static_cast<long long>(row) * nkb;
    int written = 0;
    for (int base = 0; base < nkb; base += 32) {
      const int i = base + lane;
      const bool keep = i < nkb && mrow[i] != 0;
      const uint32_t kb = __ballot_sync(0xFFFFFFFFu, keep);
      if (keep) out[written + __popc(kb & lt)] = i;
      written += __popc(kb);
    }
    if (lane == 0) kv_cnt[row] = written;
  }
}

// ---------------------------------------------------------------- launchers
cudaError_t launch_pool(const void* q, const void* k, int BH, int N, int d, int bq, int bk,
                        float* q_pool, float* k_pool, cudaStream_t st) {
  const int nqb = ceil_div(N, bq), nkb = ceil_div(N, bk);
  const long long warps = static_cast<long long>(BH) * (nqb + nkb);
  const long long blocks = (warps * 32 + 255) / 256;
  if (blocks > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  const auto* qq = static_cast<const __nv_bfloat16*>(q);
  const auto* kk = static_cast<const __nv_bfloat16*>(k);
  if (d == 128)
    pool_kernel<128><<<static_cast<unsigned>(blocks), 256, 0, st>>>(qq, kk, BH, N, bq, bk, nqb, nkb, q_pool, k_pool);
  else
    pool_kernel<64><<<static_cast<unsigned>(blocks), 256, 0, st>>>(qq, kk, BH, N, bq, bk, nqb, nkb, q_pool, k_pool);
  return cudaGetLastError();
}

cudaError_t launch_scores(const float* q_pool, const float* k_pool, int BH, int nqb, int nkb,
                          int d, double scale, float* s, long long s_ld, cudaStream_t st) {
  dim3 grid(ceil_div(nkb, kScoreTile), ceil_div(nqb, kScoreTile), BH);
  if (grid.y > 65535 || grid.z > 65535) return cudaErrorInvalidValue;
  const size_t smem = static_cast<size_t>(2) * d * kScorePad * sizeof(float);
  if (d == 128) {
    cudaFuncSetAttribute(score_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    score_kernel<128><<<grid, 256, smem, st>>>(q_pool, k_pool, nqb, nkb, scale, s, s_ld);
  } else {
    cudaFuncSetAttribute(score_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    score_kernel<64><<<grid, 256, smem, st>>>(q_pool, k_pool, nqb, nkb, scale, s, s_ld);
  }
  return cudaGetLastError();
}

cudaError_t launch_select(const float* s, long long s_ld, int n_rows, int nkb, int k_sel,
                          double topp, int* kv_idx, int* kv_cnt, uint8_t* mask,
                          cudaStream_t st) {
  const size_t slice = static_cast<size_t>(nkb) * 8 + 256 * 4;
  int wpc = static_cast<int>((200u * 1024u) / slice);
  wpc = wpc < 1 ? 1 : (wpc > kSelWarpsMax ? kSelWarpsMax : wpc);
  const size_t smem = slice * wpc;
  cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int want = (n_rows + wpc - 1) / wpc;
  const int per_sm = static_cast<int>((228u * 1024u) / (smem + 1024));
  const int cap = sms * (per_sm < 1 ? 1 : per_sm) * 2;
  const int grid = want < cap ? want : cap;
  select_kernel<<<grid, wpc * 32, smem, st>>>(s, s_ld, n_rows, nkb, k_sel, topp, kv_idx, kv_cnt, mask);
  return cudaGetLastError();
}

cudaError_t launch_compact_mask(const uint8_t* mask, int n_rows, int nkb, int* kv_idx,
                                int* kv_cnt, cudaStream_t st) {
  const int grid = (n_rows + kSelWarpsMax - 1) / kSelWarpsMax;
  compact_mask_kernel<<<grid < 65535 * 16 ? grid : 65535 * 16, kSelWarpsMax * 32, 0, st>>>(mask, n_rows, nkb, kv_idx, kv_cnt);
  return cudaGetLastError();
}

}  // namespace sa
