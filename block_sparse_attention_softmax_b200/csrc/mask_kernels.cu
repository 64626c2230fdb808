// mask_kernels.cu — block pooling, block scores and the hybrid Top-k ∪ Top-p
// selection (pages: "SLA2" 提案手法 ① mean pooling of Q and K;
// "SpargeAttention2" §2(1) hybrid Top-k + Top-p masking per attention row).
//
// Three kernels, all bound by memory or by a small amount of ALU work:
//   pool_kernel    Q, K [BH, N, d] bf16  ->  block means [BH, nb, d] fp32
//   score_kernel   means -> s[bh, qb, kb] = scale * <Qbar, Kbar> (fp32 partial
//                  sums of 16 products, combined in fp64, rounded once)
//   select_kernel  one query-block row per CTA: radix select of the K_sel-th
//                  largest score (Top-k), a probability-weighted radix select
//                  for the Top-p cut when Top-k alone does not reach p, and
//                  the ascending compacted index list.
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
// Products are summed in fp32 over 16 consecutive channels, the 16-channel
// partial sums in fp64, so the rounding error stays near 1e-8 of the score
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
  for (int c0 = 0; c0 < D; c0 += 16) {
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll
    for (int c = c0; c < c0 + 16; ++c) {
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
constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;

// Monotone map of an fp32 score to uint32: larger score -> larger key.
__device__ __forceinline__ uint32_t score_key(float s) {
  const uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct SelShared {
  uint32_t hist_c[256];
  double hist_w[256];
  double red_d[kSelWarps];
  float red_f[kSelWarps];
  int red_i[kSelWarps];
  int scan[kSelThreads];
  // results broadcast from warp 0
  uint32_t digit;
  uint32_t cnt_above;
  double w_above;
  int exhausted;
};

__device__ __forceinline__ float block_max_f(float v, SelShared& sh) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  if ((threadIdx.x & 31) == 0) sh.red_f[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = sh.red_f[0];
#pragma unroll
  for (int i = 1; i < kSelWarps; ++i) r = fmaxf(r, sh.red_f[i]);
  __syncthreads();
  return r;
}

__device__ __forceinline__ double block_sum_d(double v, SelShared& sh) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  if ((threadIdx.x & 31) == 0) sh.red_d[threadIdx.x >> 5] = v;
  __syncthreads();
  double r = 0.0;
#pragma unroll
  for (int i = 0; i < kSelWarps; ++i) r += sh.red_d[i];
  __syncthreads();
  return r;
}

// Exclusive prefix sum of one int per thread, in thread order; returns the
// block total through *total.
__device__ __forceinline__ int block_exclusive_scan(int v, SelShared& sh, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh.red_i[warp] = x;
  __syncthreads();
  int before = 0, all = 0;
#pragma unroll
  for (int i = 0; i < kSelWarps; ++i) {
    if (i < warp) before += sh.red_i[i];
    all += sh.red_i[i];
  }
  __syncthreads();
  *total = all;
  return before + x - v;
}

// One radix step over the elements whose key matches (prefix, pmask): builds
// the 256-bin histogram of the next digit (counts, and weights if weighted)
// and picks the digit holding the target. Unweighted: the bin holding the
// `need`-th largest element. Weighted: the first bin, from the top, at which
// w_above + (weight of bins >= it) reaches `target`.
template <bool WEIGHTED>
__device__ void radix_step(const uint32_t* keys, const float* e, int n, uint32_t prefix,
                           uint32_t pmask, int shift, uint32_t need, double w_above,
                           double target, SelShared& sh) {
  for (int i = threadIdx.x; i < 256; i += blockDim.x) {
    sh.hist_c[i] = 0;
    if (WEIGHTED) sh.hist_w[i] = 0.0;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const uint32_t key = keys[i];
    if ((key & pmask) == prefix) {
      const uint32_t dg = (key >> shift) & 255u;
      atomicAdd(&sh.hist_c[dg], 1u);
      if (WEIGHTED) atomicAdd(&sh.hist_w[dg], static_cast<double>(e[i]));
    }
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    // lane owns bins [8*lane, 8*lane + 8); suffix sums run from bin 255 down.
    uint32_t c[8];
    double w[8];
    uint32_t lc = 0;
    double lw = 0.0;
#pragma unroll
    for (int j = 7; j >= 0; --j) {
      lc += sh.hist_c[8 * lane + j];
      c[j] = lc;
      if (WEIGHTED) {
        lw += sh.hist_w[8 * lane + j];
        w[j] = lw;
      }
    }
    // inclusive suffix over lanes: add totals of higher lanes
    uint32_t hc = lc;
    double hw = lw;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t yc = __shfl_down_sync(0xFFFFFFFFu, hc, o);
      double yw = 0.0;
      if (WEIGHTED) yw = __shfl_down_sync(0xFFFFFFFFu, hw, o);
      if (lane + o < 32) {
        hc += yc;
        if (WEIGHTED) hw += yw;
      }
    }
    const uint32_t above_c = hc - lc;   // bins of higher lanes
    const double above_w = WEIGHTED ? hw - lw : 0.0;
    // largest bin j (in this lane) whose suffix reaches the target
    int hit = -1;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      bool ok;
      if (WEIGHTED) ok = (w_above + above_w + w[j] >= target) && (c[j] + above_c > 0);
      else ok = (c[j] + above_c >= need);
      if (ok) hit = j;
    }
    const uint32_t ballot = __ballot_sync(0xFFFFFFFFu, hit >= 0);
    if (ballot) {
      const int src = 31 - __clz(ballot);
      if (lane == src) {
        const int dg = 8 * lane + hit;
        // totals strictly above the chosen bin
        const uint32_t cnt_above = above_c + (hit < 7 ? c[hit + 1] : 0u);
        const double wt_above = WEIGHTED ? above_w + (hit < 7 ? w[hit + 1] : 0.0) : 0.0;
        sh.digit = static_cast<uint32_t>(dg);
        sh.cnt_above = cnt_above;
        sh.w_above = wt_above;
        sh.exhausted = 0;
      }
    } else {
      // Weighted only: rounding kept the bucket below the target; every element
      // of the bucket is needed, so continue into its lowest non-empty bin.
      const uint32_t nz = __ballot_sync(0xFFFFFFFFu, lc > 0);
      const int src = __ffs(nz) - 1;
      if (lane == src) {
        int j0 = 0;
        while (j0 < 7 && sh.hist_c[8 * lane + j0] == 0) ++j0;
        sh.digit = static_cast<uint32_t>(8 * lane + j0);
        sh.cnt_above = above_c + (j0 < 7 ? c[j0 + 1] : 0u);
        sh.w_above = above_w + (j0 < 7 ? w[j0 + 1] : 0.0);
        sh.exhausted = 1;
      }
    }
  }
  __syncthreads();
}

struct Cut {
  uint32_t key;    // threshold key value
  uint32_t above;  // elements strictly above the threshold
  uint32_t ties;   // elements equal to the threshold to keep, lowest index first
};

// The `rank`-th largest key (1-based) and the number of its ties to keep.
__device__ Cut select_rank(const uint32_t* keys, int n, uint32_t rank, SelShared& sh) {
  uint32_t prefix = 0, pmask = 0, need = rank, above = 0;
  for (int shift = 24; shift >= 0; shift -= 8) {
    radix_step<false>(keys, nullptr, n, prefix, pmask, shift, need, 0.0, 0.0, sh);
    const uint32_t dg = sh.digit, ca = sh.cnt_above;
    need -= ca;
    above += ca;
    prefix |= dg << shift;
    pmask |= 255u << shift;
    __syncthreads();
  }
  return Cut{prefix, above, need};
}

// Smallest m such that the m largest-key weights sum to >= target.
__device__ Cut select_mass(const uint32_t* keys, const float* e, int n, double target,
                           SelShared& sh) {
  uint32_t prefix = 0, pmask = 0, above = 0;
  double w_above = 0.0;
  int exhausted = 0;
  for (int shift = 24; shift >= 0; shift -= 8) {
    radix_step<true>(keys, e, n, prefix, pmask, shift, 0, w_above, target, sh);
    const uint32_t dg = sh.digit;
    above += sh.cnt_above;
    w_above += sh.w_above;
    exhausted |= sh.exhausted;
    prefix |= dg << shift;
    pmask |= 255u << shift;
    __syncthreads();
  }
  // Ties at the threshold: identical keys carry identical weights; take them in
  // index order until the running sum reaches the target.
  int n_ties = 0;
  float e_tie = 0.f;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    if (keys[i] == prefix) {
      ++n_ties;
      e_tie = e[i];
    }
  }
  int total;
  block_exclusive_scan(n_ties, sh, &total);
  const float ev = block_max_f(e_tie, sh);  // all ties share one weight
  uint32_t t = 0;
  if (exhausted) {
    t = static_cast<uint32_t>(total);
  } else {
    double acc = w_above;
    while (acc < target && t < static_cast<uint32_t>(total)) {
      acc += static_cast<double>(ev);
      ++t;
    }
    if (t == 0) t = 1;
  }
  __syncthreads();
  return Cut{prefix, above, t};
}

// Per-thread contiguous chunk [lo, hi) of the row, used where index order matters.
__device__ __forceinline__ void chunk_range(int n, int* lo, int* hi) {
  const int per = (n + blockDim.x - 1) / blockDim.x;
  *lo = min(n, static_cast<int>(threadIdx.x) * per);
  *hi = min(n, *lo + per);
}

// Marks kept elements (key > cut, or equal and among the first `ties` equal
// ones by index) in `flag`, and returns this thread's fp64 weight of them.
__device__ double mark_kept(const uint32_t* keys, const float* e, int n, Cut cut, uint8_t* flag,
                            SelShared& sh) {
  int lo, hi;
  chunk_range(n, &lo, &hi);
  int my_ties = 0;
  for (int i = lo; i < hi; ++i) my_ties += (keys[i] == cut.key);
  int total;
  int rank = block_exclusive_scan(my_ties, sh, &total);
  double w = 0.0;
  for (int i = lo; i < hi; ++i) {
    const uint32_t key = keys[i];
    bool keep = key > cut.key;
    if (key == cut.key) {
      keep = static_cast<uint32_t>(rank) < cut.ties;
      ++rank;
    }
    flag[i] = keep;
    if (keep && e) w += static_cast<double>(e[i]);
  }
  return w;
}

// One CTA per (bh, qb) row.
__global__ void __launch_bounds__(kSelThreads) select_kernel(
    const float* __restrict__ s, long long s_ld, int n_rows, int nkb, int k_sel, double topp,
    int* __restrict__ kv_idx, int* __restrict__ kv_cnt, uint8_t* __restrict__ mask) {
  extern __shared__ __align__(16) uint8_t sm_sel[];
  __shared__ SelShared sh;
  const int row = blockIdx.x;
  if (row >= n_rows) return;
  uint32_t* keys = reinterpret_cast<uint32_t*>(sm_sel);
  float* e = reinterpret_cast<float*>(sm_sel + static_cast<size_t>(nkb) * 4);
  uint8_t* flag = sm_sel + static_cast<size_t>(nkb) * 8;
  const float* srow = s + static_cast<long long>(row) * s_ld;

  float mx = -INFINITY;
  for (int i = threadIdx.x; i < nkb; i += blockDim.x) {
    const float v = srow[i];
    keys[i] = score_key(v);
    e[i] = v;
    mx = fmaxf(mx, v);
  }
  mx = block_max_f(mx, sh);  // contains __syncthreads
  double z = 0.0;
  for (int i = threadIdx.x; i < nkb; i += blockDim.x) {
    const float v = expf(e[i] - mx);
    e[i] = v;
    z += static_cast<double>(v);
  }
  z = block_sum_d(z, sh);

  if (topp >= 1.0 || k_sel >= nkb) {
    for (int i = threadIdx.x; i < nkb; i += blockDim.x) flag[i] = 1;
    __syncthreads();
  } else {
    const double target = topp * z;
    const Cut ck = select_rank(keys, nkb, static_cast<uint32_t>(k_sel), sh);
    double wk = mark_kept(keys, e, nkb, ck, flag, sh);
    wk = block_sum_d(wk, sh);
    if (wk < target) {
      const Cut cp = select_mass(keys, e, nkb, target, sh);
      const int m_p = static_cast<int>(cp.above + cp.ties);
      if (m_p > k_sel) {
        mark_kept(keys, nullptr, nkb, cp, flag, sh);
      }
    }
    __syncthreads();
  }

  // Ascending compaction of the kept indices.
  int lo, hi;
  chunk_range(nkb, &lo, &hi);
  int mine = 0;
  for (int i = lo; i < hi; ++i) mine += flag[i];
  int total;
  int pos = block_exclusive_scan(mine, sh, &total);
  int* out = kv_idx + static_cast<long long>(row) * nkb;
  for (int i = lo; i < hi; ++i)
    if (flag[i]) out[pos++] = i;
  if (mask) {
    uint8_t* mrow = mask + static_cast<long long>(row) * nkb;
    for (int i = threadIdx.x; i < nkb; i += blockDim.x) mrow[i] = flag[i];
  }
  if (threadIdx.x == 0) kv_cnt[row] = total;
}

// ---------------------------------------------------------------- uint8 mask -> lists
__global__ void __launch_bounds__(kSelThreads) compact_mask_kernel(
    const uint8_t* __restrict__ mask, int n_rows, int nkb, int* __restrict__ kv_idx,
    int* __restrict__ kv_cnt) {
  __shared__ SelShared sh;
  const int row = blockIdx.x;
  if (row >= n_rows) return;
  const uint8_t* mrow = mask + static_cast<long long>(row) * nkb;
  int lo, hi;
  chunk_range(nkb, &lo, &hi);
  int mine = 0;
  for (int i = lo; i < hi; ++i) mine += (mrow[i] != 0);
  int total;
  int pos = block_exclusive_scan(mine, sh, &total);
  int* out = kv_idx + static_cast<long long>(row) * nkb;
  for (int i = lo; i < hi; ++i)
    if (mrow[i]) out[pos++] = i;
  if (threadIdx.x == 0) kv_cnt[row] = total;
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
  const size_t smem = static_cast<size_t>(nkb) * 9 + 16;
  cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  select_kernel<<<n_rows, kSelThreads, smem, st>>>(s, s_ld, n_rows, nkb, k_sel, topp, kv_idx, kv_cnt, mask);
  return cudaGetLastError();
}

cudaError_t launch_compact_mask(const uint8_t* mask, int n_rows, int nkb, int* kv_idx,
                                int* kv_cnt, cudaStream_t st) {
  compact_mask_kernel<<<n_rows, kSelThreads, 0, st>>>(mask, n_rows, nkb, kv_idx, kv_cnt);
  return cudaGetLastError();
}

}  // namespace sa
