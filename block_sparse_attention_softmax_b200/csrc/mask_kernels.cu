// mask_kernels.cu — block pooling, block scores and the hybrid Top-k ∪ Top-p
// selection (pages: "SLA2" 提案手法 ① mean pooling of Q and K;
// "SpargeAttention2" §2(1) hybrid Top-k + Top-p masking per attention row).
//
//   pool_kernel        Q, K [BH, N, d] bf16 -> block means [BH, nb, d] fp32,
//                      and the same means as four signed 7-bit slices per
//                      element with a per-row power-of-two exponent
//   score_i8_kernel    scale * <Qbar, Kbar> on the int8 tensor cores from the
//                      slices (exact s32 slice products, combined in fp32 with
//                      one final rounding), in three modes: the fp32 score
//                      matrix; approximate per-row statistics; exact scores
//                      reduced to per-row normaliser partials and candidate
//                      lists
//   select_cand_kernel one query-block row per warp from its candidate lists:
//                      the K_sel-th largest score (Top-k), the Top-p cut when
//                      Top-k alone does not reach p, the ascending kept list
//   select_*_kernel    one row per warp from the score matrix: the same cuts by
//                      a short count search and an exact search among at most
//                      256 candidates, the row in registers (up to 1280 key
//                      blocks) or shared memory
// The score-matrix path (write mode, then select_fast / select_long) serves
// problems of up to 32 MiB of scores and the rows the candidate lists cannot
// settle; the candidate path (statistics, candidates, select_cand) the rest.
#include "sa_internal.h"

namespace sa {

// ---------------------------------------------------------------- pooling
// One warp per token block. Each lane loads 16 B (8 bf16) per row it visits;
// d/8 lanes cover one row, so a warp reads 32*16 B per step.
//
// With `sl` set, each block mean row x (fp32) is also written as four signed
// 7-bit slices for the integer tensor-core scores: with E the exponent for
// which max|x| < 2^E, y = x * 2^-E lies in (-1, 1) and
//   y = sum_{s=1..4} a_s 2^(-7 s) + r,  a_s = trunc of the running remainder
//   times 128, |a_s| <= 127, 0 <= |r| < 2^-28,
// computed exactly in fp32 (scaling by 128 and subtracting the integer part
// are exact). Row layout: slice s at bytes [s * d, (s + 1) * d); E in `ex`.

template <int D>
__global__ void __launch_bounds__(256) pool_kernel(const __nv_bfloat16* __restrict__ q,
                                                   const __nv_bfloat16* __restrict__ k, int BH,
                                                   int N, int bq, int bk, int nqb, int nkb,
                                                   float* __restrict__ q_pool,
                                                   float* __restrict__ k_pool, SliceOut sl) {
  constexpr int LPR = D / 8;        // lanes per row
  constexpr int RPI = 32 / LPR;     // rows per warp step
  grid_dep_trigger();               // the scoring kernel may begin its set-up
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
  const float fc = static_cast<float>(cnt);
  float mean[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) mean[i] = __fdiv_rn(acc[i], fc);
  if (r0 == 0) {
    reinterpret_cast<float4*>(dst + c8)[0] = make_float4(mean[0], mean[1], mean[2], mean[3]);
    reinterpret_cast<float4*>(dst + c8)[1] = make_float4(mean[4], mean[5], mean[6], mean[7]);
  }
  if (sl.q_sl) {
    float mx = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) mx = fmaxf(mx, fabsf(mean[i]));
#pragma unroll
    for (int off = 1; off < LPR; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
    int E = 0;
    if (mx > 0.f) frexpf(mx, &E);      // mx = m * 2^E with m in [0.5, 1): max|x| < 2^E
    if (r0 == 0) {
      int8_t* srow = (is_q ? sl.q_sl : sl.k_sl) + w * (4 * D);
      float y[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) y[i] = ldexpf(mean[i], -E);
#pragma unroll
      for (int sidx = 0; sidx < 4; ++sidx) {
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float t = y[i] * 128.f;
          const float a = truncf(t);
          y[i] = t - a;
          const uint32_t byte = static_cast<uint32_t>(static_cast<int>(a)) & 0xFFu;
          if (i < 4) lo |= byte << (8 * i);
          else hi |= byte << (8 * (i - 4));
        }
        *reinterpret_cast<uint2*>(srow + sidx * D + c8) = make_uint2(lo, hi);
      }
      if (lane == 0) (is_q ? sl.q_ex : sl.k_ex)[w] = E;
    }
  }
}

// ---------------------------------------------------------------- scores on the int8 tensor cores
// The block means arrive as four 7-bit slices per element (see pool_kernel):
// x = 2^E sum_s a_s 2^(-7 s) up to 2^(E-28). Then
//   <xq, xk> = 2^(Eq + Ek) sum_{s,t} 2^(-7 (s + t)) <a_s, b_t>,
// and every <a_s, b_t> (d products of |.| <= 127 values) is exact in the
// tensor core's s32 accumulator. Pairs are grouped by level L = s + t into
// four accumulators (L = 2..5; pairs with s + t > 5 weigh at most 2^-42 and
// are dropped), so that the score is
//   (acc2 + acc3 2^-7 + acc4 2^-14 + acc5 2^-21) * scale 2^(Eq - 14) * 2^Ek.
// Each accumulator is exact in fp32; the leading product is split exactly by
// an fma and the smaller terms are added before one final rounding
// (score_exact), so a score is within about half an ulp of the exact value:
// at most 5e-7 for scores below 16, inside the 1e-6 band within which the
// mask comparison treats a cut as a tie.
//
// Persistent CTAs over work items (head, 128 query blocks, a range of 64-key
// tiles): warp 0 loads the item's query slices (operand A, M = 128) and
// streams the key-slice tiles (operand B, N = 64) through a 3-stage ring by
// TMA (128-byte swizzled rows, one box per 128-byte column chunk; 6 stages
// in kScoreStats); warp 1 issues the MMAs of a key tile into one of two TMEM
// accumulator sets; the epilogue warps (per TMEM lane quadrant two warps of
// 32 key columns, or in kScoreCands four of 16, so that each thread owns one
// query-block row) consume the accumulators. Three modes:
//
//   kScoreWrite  exact scores, transposed through shared memory and written
//                as the fp32 score matrix with coalesced 128-byte stores;
//                with a query-tile filter, only the flagged tiles (the rows
//                the candidate selection handed back)
//   kScoreStats  the first slice pair only (one level, d / 32 MMAs), an
//                approximation of the score within about 2^-6 of
//                sum |q||k|: per row and item, its max, sum and sum of
//                squares, from which the candidate pass takes a reference
//                maximum and a threshold t
//   kScoreCands  exact scores as in kScoreWrite, never stored: per row and
//                item, the exact max and the partial normaliser
//                sum e^(s - m_ref) (fp32 pairwise over each 16-column
//                chunk, fp64 across chunks), and every score >= t (and, for
//                rows expected to need it, every score in [t_lo, t)) appended
//                to the row's lists (one atomic per thread, list and tile
//                reserves the slots; the entries are written two tiles later)
constexpr int kI8TileM = 128;
constexpr int kI8TileN = 64;
constexpr int kI8BStages = 3;
constexpr int kI8EpiWarps = 8;
constexpr int kMaxKr = 4;               // key ranges per row (bounds the partial arrays)

enum : int { kScoreWrite = 0, kScoreStats = 1, kScoreCands = 2 };

template <int D, int MODE>
struct I8Layout {
  static constexpr int ROW = 4 * D;                 // bytes per slice row
  static constexpr int NCH = MODE == kScoreStats ? 1 : ROW / 128;   // 128-byte chunks loaded
  static constexpr int LEVELS = MODE == kScoreStats ? 1 : 4;
  static constexpr int STAGES = MODE == kScoreStats ? 6 : kI8BStages;   // B ring depth
  // epilogue warps and the key columns of a tile each one reads: kScoreCands
  // splits a row's 64 columns over four warps (16 each) for more warps to
  // hide its latency, the other modes over two (32 each)
  static constexpr int EW = MODE == kScoreCands ? 16 : kI8EpiWarps;
  static constexpr int CW = 4 * kI8TileN / EW;
  static constexpr int THREADS = 32 * (2 + EW);
  static constexpr uint32_t A_CH = kI8TileM * 128;  // bytes of one A chunk
  static constexpr uint32_t B_CH = kI8TileN * 128;
  static constexpr uint32_t A_BYTES = NCH * A_CH;
  static constexpr uint32_t B_BYTES = NCH * B_CH;
  static constexpr uint32_t OFF_A = 0;
  static constexpr uint32_t OFF_B = OFF_A + A_BYTES;
  static constexpr uint32_t OFF_T = OFF_B + STAGES * B_BYTES;
  // kScoreWrite: [epi warps][32][33] fp32 transpose blocks
  static constexpr uint32_t T_BYTES = MODE == kScoreWrite ? EW * 32 * 33 * 4 : 0;
  // [epi warps][CW] fp32 column factors 2^Ek of the current tile
  static constexpr uint32_t OFF_C = OFF_T + T_BYTES;
  static constexpr uint32_t C_BYTES = EW * CW * 4;
  // kScoreCands: two tiles' scores, [2][CW columns][epilogue threads] fp32,
  // read back two tiles later for the candidates
  static constexpr uint32_t OFF_X = OFF_C + C_BYTES;
  static constexpr uint32_t X_BYTES = MODE == kScoreCands ? 2 * CW * EW * 32 * 4 : 0;
  static constexpr uint32_t OFF_BAR = OFF_X + X_BYTES;
  static constexpr uint32_t SMEM = OFF_BAR + 256 + 1024;
};

struct I8Work {
  int nqb, nkb, n_qt, n_kt, kr_tiles, n_kr, n_items;
};

// Partial results of one (row, key range, column half).
struct __align__(16) ZPart {
  double z;      // sum of e^(s - m_ref) over the part's columns
  float mx;      // exact max of the part's scores
  float pad;
};

// Buffers of the candidate selection (rows are bh * nqb + query block).
struct CandBufs {
  float4* st1;       // [rows][2 kMaxKr] approximate {max, sum, sum of squares, count}
  ZPart* st2;        // [rows][2 kMaxKr]
  float2* rowinfo;   // [rows] {m_ref, t}
  int* cand_cnt;     // [rows][2] scores >= t, and t_lo <= score < t (may exceed the capacities)
  uint2* cand;       // [rows][c_hi + c_lo] {key, key block}: the list >= t, then the list below
  int c_hi, c_lo;
  float zq;          // standard normal quantile with tail mass want / nkb (t)
  float zq_lo;       // the same for the wider list (t_lo)
  float p_lo;        // rows whose expected Top-k mass share is below this get the second list
  float zp;          // z with P(Z > z) = p (standard normal): the model's Top-p length is nkb Q(sd + zp)
  int all_cand;      // every key block is a candidate of the first list
  int* fb_cnt;       // rows handed back to the score-matrix path
  int* fb_rows;      // [rows]
  int* tile_flag;    // [BH * n_qt] query tiles holding such rows
  int n_tile_flags;
};

// Monotone uint32 image of an fp32 score (larger score -> larger key).
__device__ __forceinline__ uint32_t score_key(float s) {
  const uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Row constants of the exact score: c = scale 2^(Eq - 14) as an unevaluated
// fp32 pair ch + cl, and ch 2^-7, 2^-14, 2^-21 (exact scalings).
struct RowC {
  float ch, cl, ch7, ch14, ch21;
};

__device__ __forceinline__ RowC row_consts(double scale, int eq) {
  const double c = scale * __longlong_as_double(static_cast<long long>(eq - 14 + 1023) << 52);
  RowC r;
  r.ch = static_cast<float>(c);
  r.cl = static_cast<float>(c - static_cast<double>(r.ch));
  r.ch7 = r.ch * 0.0078125f;
  r.ch14 = r.ch * 6.103515625e-05f;
  r.ch21 = r.ch * 4.76837158203125e-07f;
  return r;
}

// 2^e as fp32 for a key-block exponent (clamped to the normal range; blocks
// beyond it have scores far below the tie band).
__device__ __forceinline__ float pow2f(int e) { return __int_as_float((min(max(e, -126), 127) + 127) << 23); }

// Score without the column factor: (acc2 + acc3 2^-7 + acc4 2^-14 + acc5 2^-21) c.
// Every accumulator is exact in fp32 (|acc_L| < 2^23); acc2 ch is split
// exactly into p + e by one fma, the remaining terms (each at most 2^-6 of
// the leading one) are summed in fp32 and the total rounds once, so the
// result is within about half an ulp of the exact value.
__device__ __forceinline__ float score_exact(uint32_t a2, uint32_t a3, uint32_t a4, uint32_t a5, const RowC& c) {
  const float f2 = static_cast<float>(static_cast<int>(a2));
  const float f3 = static_cast<float>(static_cast<int>(a3));
  const float f4 = static_cast<float>(static_cast<int>(a4));
  const float f5 = static_cast<float>(static_cast<int>(a5));
  const float p = f2 * c.ch;
  const float e = fmaf(f2, c.ch, -p);
  float t = f5 * c.ch21;
  t = fmaf(f4, c.ch14, t);
  t = fmaf(f3, c.ch7, t);
  t = fmaf(f2, c.cl, t);
  return p + (e + t);
}

// Candidates of one staged tile whose list slots are reserved.
struct CandPend {
  uint32_t h = 0u, l = 0u;   // columns in the first / second list
  int jh = 0, jl = 0;        // first reserved slot in each list
  int kc0 = 0;               // key block of column 0
  uint2* cl = nullptr;       // the row's lists
  const float* xb = nullptr; // the staged scores
};

// Writes the candidates of one staged tile (bits of `pend`, slots from j on;
// slots past cap are counted but not stored) and clears `pend`.
__device__ __forceinline__ void flush_cands(uint32_t pend, int j, int kc0, const float* xst, uint2* cl, int cap,
                                            int XS) {
  if (pend == 0u) return;
  uint32_t m = pend;
  while (m != 0u) {
    const int i = __ffs(m) - 1;
    m &= m - 1u;
    if (j < cap) cl[j] = make_uint2(score_key(xst[i * XS]), static_cast<uint32_t>(kc0 + i));
    ++j;
  }
}

// e^(x - m_ref) as computed for the normaliser and for every candidate mass.
__device__ __forceinline__ float cand_weight(float x, float mlog) {
  return fast_exp2(fmaf(x, 1.4426950408889634f, -mlog));
}

template <int D, int MODE>
__global__ void __launch_bounds__(I8Layout<D, MODE>::THREADS, 1) score_i8_kernel(const __grid_constant__ CUtensorMap tmA,
                                                                 const __grid_constant__ CUtensorMap tmB,
                                                                 const int* __restrict__ q_ex,
                                                                 const int* __restrict__ k_ex, I8Work wk,
                                                                 double scale, float* __restrict__ s,
                                                                 long long s_ld, CandBufs cb) {
  using L = I8Layout<D, MODE>;
  if constexpr (MODE == kScoreWrite) {
    // filtered launch with nothing handed back: leave before any setup
    grid_dep_wait();
    if (cb.fb_cnt && *reinterpret_cast<volatile const int*>(cb.fb_cnt) == 0) return;
  }
  extern __shared__ __align__(16) uint8_t smem_raw[];
  // 1024-byte aligned (swizzle atoms), derived from the shared array so that
  // accesses through it stay shared-memory instructions
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* a_full = bars;                        // item's query slices landed
  uint64_t* a_empty = bars + 1;                   // item's last MMA completed
  uint64_t* b_full = bars + 2;                    // [STAGES]
  uint64_t* b_empty = b_full + L::STAGES;        // [L::STAGES]
  uint64_t* acc_full = b_empty + L::STAGES;      // [2]
  uint64_t* acc_empty = acc_full + 2;             // [2] (epilogue warps)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr uint32_t kSet = L::LEVELS * kI8TileN;   // columns of one accumulator set
  constexpr uint32_t kAlloc = 2 * kSet;             // 128 or 512 columns

  if (threadIdx.x == 0) {
    mbar_init(a_full, 1);
    mbar_init(a_empty, 1);
    for (int i = 0; i < L::STAGES; ++i) {
      mbar_init(&b_full[i], 1);
      mbar_init(&b_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], L::EW);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kAlloc);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *tmem_slot;
  // set-up above overlaps the previous kernel's tail; inputs are read below
  if constexpr (MODE != kScoreWrite) grid_dep_wait();
  grid_dep_trigger();
  if constexpr (MODE == kScoreStats) {
    // clear the hand-back state of this call (read only by later launches)
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < cb.n_tile_flags; i += gridDim.x * blockDim.x)
      cb.tile_flag[i] = 0;
    if (blockIdx.x == 0 && threadIdx.x == 0) *cb.fb_cnt = 0;
  }

  // work item -> (head, query tile, key range, first and end key tile)
  auto decode = [&](int item, int& bh, int& qt, int& kr, int& kt0, int& kt1) {
    kr = item % wk.n_kr;
    const int rest = item / wk.n_kr;
    qt = rest % wk.n_qt;
    bh = rest / wk.n_qt;
    kt0 = kr * wk.kr_tiles;
    kt1 = min(wk.n_kt, kt0 + wk.kr_tiles);
  };
  // every role skips the same items (the flags do not change during the launch)
  auto skip = [&](int bh, int qt) -> bool {
    if constexpr (MODE == kScoreWrite) return cb.tile_flag != nullptr && cb.tile_flag[bh * wk.n_qt + qt] == 0;
    else return false;
  };
  // Items of this CTA: a contiguous range (consecutive items mostly share the
  // query tile, which then stays in shared memory), or for kScoreWrite a
  // stride of the grid (the few flagged tiles spread over the CTAs).
  constexpr bool kContig = MODE != kScoreWrite;
  const int per = kContig ? (wk.n_items + static_cast<int>(gridDim.x) - 1) / static_cast<int>(gridDim.x) : 1;
  const int it_begin = kContig ? static_cast<int>(blockIdx.x) * per : static_cast<int>(blockIdx.x);
  const int it_end = kContig ? min(wk.n_items, it_begin + per) : wk.n_items;
  const int it_step = kContig ? 1 : static_cast<int>(gridDim.x);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      int ic = 0, bt = 0, pbh = -1, pqt = -1;
      bool ok = true;
      for (int item = it_begin; ok && item < it_end; item += it_step) {
        int bh, qt, kr, kt0, kt1;
        decode(item, bh, qt, kr, kt0, kt1);
        if (skip(bh, qt)) continue;
        if (!kContig || bh != pbh || qt != pqt) {     // another query tile
          if (!(ok = mbar_wait(a_empty, (ic & 1) ^ 1, abort_flag))) break;
          mbar_arrive_expect_tx(a_full, L::A_BYTES);
#pragma unroll
          for (int c = 0; c < L::NCH; ++c)
            tma_load_3d(smem + L::OFF_A + c * L::A_CH, &tmA, a_full, c * 128, qt * kI8TileM, bh);
          ++ic;
          pbh = bh;
          pqt = qt;
        }
        for (int kt = kt0; kt < kt1; ++kt, ++bt) {
          const int st = bt % L::STAGES;
          if (!(ok = mbar_wait(&b_empty[st], ((bt / L::STAGES) & 1) ^ 1, abort_flag))) break;
          mbar_arrive_expect_tx(&b_full[st], L::B_BYTES);
#pragma unroll
          for (int c = 0; c < L::NCH; ++c)
            tma_load_3d(smem + L::OFF_B + st * L::B_BYTES + c * L::B_CH, &tmB, &b_full[st], c * 128, kt * kI8TileN, bh);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_s8_s32(kI8TileM, kI8TileN);
      const uint64_t a0 = sw128_desc(smem_u32(smem + L::OFF_A), 16, 1024);
      const uint64_t b00 = sw128_desc(smem_u32(smem + L::OFF_B), 16, 1024);
      // descriptor offset of a K step inside the chunked, swizzled tile
      auto off = [](int byte, uint32_t chunk_bytes) -> uint32_t {
        return (static_cast<uint32_t>(byte >> 7) * chunk_bytes + static_cast<uint32_t>(byte & 127)) >> 4;
      };
      int ic = 0, bt = 0, pbh = -1, pqt = -1;
      bool ok = true;
      for (int item = it_begin; ok && item < it_end; item += it_step) {
        int bh, qt, kr, kt0, kt1;
        decode(item, bh, qt, kr, kt0, kt1);
        if (skip(bh, qt)) continue;
        if (!kContig || bh != pbh || qt != pqt) {
          if (!(ok = mbar_wait(a_full, ic & 1, abort_flag))) break;
          ++ic;
          pbh = bh;
          pqt = qt;
        }
        for (int kt = kt0; kt < kt1; ++kt, ++bt) {
          const int st = bt % L::STAGES, ab = bt & 1;
          if (!(ok = mbar_wait(&b_full[st], (bt / L::STAGES) & 1, abort_flag))) break;
          if (!(ok = mbar_wait(&acc_empty[ab], ((bt >> 1) & 1) ^ 1, abort_flag))) break;
          tc_fence_after();
          const uint64_t b0 = b00 + ((st * L::B_BYTES) >> 4);
          const uint32_t acc = tm + ab * kSet;
          if constexpr (MODE == kScoreStats) {
            // slice 1 of both operands: level 2 only
#pragma unroll
            for (int j = 0; j < D / 32; ++j)
              umma_i8_ss(acc, a0 + off(32 * j, L::A_CH), b0 + off(32 * j, L::B_CH), idesc, j == 0 ? 0u : 1u);
          } else {
#pragma unroll
            for (int sa = 1; sa <= 4; ++sa)
#pragma unroll
              for (int tb = 1; sa + tb <= 5; ++tb)
#pragma unroll
                for (int j = 0; j < D / 32; ++j)
                  umma_i8_ss(acc + (sa + tb - 2) * kI8TileN, a0 + off(D * (sa - 1) + 32 * j, L::A_CH),
                             b0 + off(D * (tb - 1) + 32 * j, L::B_CH), idesc, (sa == 1 && j == 0) ? 0u : 1u);
          }
          tc_commit(&b_empty[st]);
          tc_commit(&acc_full[ab]);
        }
        // release the query tile unless the next item uses it too
        bool release = true;
        if (kContig && item + 1 < it_end) {
          int nbh, nqt, nkr, nk0, nk1;
          decode(item + 1, nbh, nqt, nkr, nk0, nk1);
          release = nbh != bh || nqt != qt;
        }
        if (ok && release) tc_commit(a_empty);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;                       // 0..7
    const int quad = warp & 3;                     // TMEM lane quadrant
    const int hc = ew >> 2;                        // key columns [32 hc, 32 hc + 32) of the tile
    const uint32_t la = tm + (static_cast<uint32_t>(quad * 32) << 16) + hc * 32;
    int bt = 0;
    bool ok = true;
    // kScoreCands: candidates of the last two tiles (p2 two tiles ago, p1 the
    // previous one), slots reserved, written two tiles later, when the
    // reserving atomics have returned
    CandPend p2, p1;
    for (int item = it_begin; ok && item < it_end; item += it_step) {
      int bh, qt, kr, kt0, kt1;
      decode(item, bh, qt, kr, kt0, kt1);
      if (skip(bh, qt)) continue;
      const int row0 = qt * kI8TileM + quad * 32;  // first query block of this warp's rows
      const int row = row0 + lane;
      const bool row_ok = row < wk.nqb;
      const long long grow = static_cast<long long>(bh) * wk.nqb + row;
      const int eq = row_ok ? __ldg(q_ex + grow) : 0;
      // this lane's key-block exponent in tile kt (0 past the row end)
      auto ld_ek = [&](int kt) -> int {
        const int kcol = kt * kI8TileN + hc * 32 + lane;
        return kcol < wk.nkb ? __ldg(k_ex + static_cast<long long>(bh) * wk.nkb + kcol) : 0;
      };
      if constexpr (MODE == kScoreWrite) {
        float* tbuf = reinterpret_cast<float*>(smem + L::OFF_T) + ew * 32 * 33;
        float* colf = reinterpret_cast<float*>(smem + L::OFF_C) + ew * 32;
        const RowC rc = row_consts(scale, eq);
        for (int kt = kt0; kt < kt1; ++kt, ++bt) {
          const int ab = bt & 1;
          const int kcol = kt * kI8TileN + hc * 32 + lane;   // this lane's key in the store phase
          const int ek_l = kcol < wk.nkb ? __ldg(k_ex + static_cast<long long>(bh) * wk.nkb + kcol) : 0;
          ok = __all_sync(0xFFFFFFFFu, mbar_wait(&acc_full[ab], (bt >> 1) & 1, abort_flag));   // warp-uniform
          if (!ok) break;
          tc_fence_after();
          uint32_t a2[32], a3[32], a4[32], a5[32];
          const uint32_t base = la + ab * kSet;
          tmem_ld16(base + 0 * kI8TileN, a2);
          tmem_ld16(base + 0 * kI8TileN + 16, a2 + 16);
          tmem_ld16(base + 1 * kI8TileN, a3);
          tmem_ld16(base + 1 * kI8TileN + 16, a3 + 16);
          tmem_ld16(base + 2 * kI8TileN, a4);
          tmem_ld16(base + 2 * kI8TileN + 16, a4 + 16);
          tmem_ld16(base + 3 * kI8TileN, a5);
          tmem_ld16(base + 3 * kI8TileN + 16, a5 + 16);
          tmem_wait_ld();
          reg_fence16(a2); reg_fence16(a2 + 16);
          reg_fence16(a3); reg_fence16(a3 + 16);
          reg_fence16(a4); reg_fence16(a4 + 16);
          reg_fence16(a5); reg_fence16(a5 + 16);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[ab]);    // accumulators are in registers
          colf[lane] = pow2f(ek_l);
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 32; ++i) tbuf[lane * 33 + i] = score_exact(a2[i], a3[i], a4[i], a5[i], rc) * colf[i];
          __syncwarp();
          // row r of this warp's 32 x 32 block: 32 consecutive keys
          if (kcol < wk.nkb) {
#pragma unroll 4
            for (int r = 0; r < 32; ++r)
              if (row0 + r < wk.nqb)
                s[(static_cast<long long>(bh) * wk.nqb + row0 + r) * s_ld + kcol] = tbuf[r * 33 + lane];
          }
          __syncwarp();
        }
      } else if constexpr (MODE == kScoreStats) {
        float* colf = reinterpret_cast<float*>(smem + L::OFF_C) + ew * 32;
        float vmax = -INFINITY, s0 = 0.f, s1 = 0.f, q0 = 0.f, q1 = 0.f;
        int nv = 0;
        int ek_next = kt0 < kt1 ? ld_ek(kt0) : 0;   // exponents one tile ahead
        for (int kt = kt0; kt < kt1; ++kt, ++bt) {
          const int ab = bt & 1;
          const int kc0 = kt * kI8TileN + hc * 32;
          const int ek = min(max(ek_next, -126), 127);
          if (kt + 1 < kt1) ek_next = ld_ek(kt + 1);
          ok = __all_sync(0xFFFFFFFFu, mbar_wait(&acc_full[ab], (bt >> 1) & 1, abort_flag));   // warp-uniform
          if (!ok) break;
          tc_fence_after();
          uint32_t a2[32];
          tmem_ld16(la + ab * kSet, a2);
          tmem_ld16(la + ab * kSet + 16, a2 + 16);
          tmem_wait_ld();
          reg_fence16(a2); reg_fence16(a2 + 16);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[ab]);
          colf[lane] = pow2f(ek);
          __syncwarp();
          const int nvalid = min(32, wk.nkb - kc0);
          if (nvalid >= 32) {
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              const float2 c = *reinterpret_cast<const float2*>(colf + i);
              const float v0 = static_cast<float>(static_cast<int>(a2[i])) * c.x;
              const float v1 = static_cast<float>(static_cast<int>(a2[i + 1])) * c.y;
              vmax = fmax3(vmax, v0, v1);
              s0 += v0;
              s1 += v1;
              q0 = fmaf(v0, v0, q0);
              q1 = fmaf(v1, v1, q1);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              if (i < nvalid) {
                const float v = static_cast<float>(static_cast<int>(a2[i])) * colf[i];
                vmax = fmaxf(vmax, v);
                s0 += v;
                q0 = fmaf(v, v, q0);
              }
            }
          }
          nv += max(nvalid, 0);
          __syncwarp();
        }
        if (ok && row_ok) {
          // approximate score = acc2 2^21 2^(Eq + Ek - 35) scale; 2^Ek applied above
          const float rowf = static_cast<float>(scale * __longlong_as_double(static_cast<long long>(eq - 14 + 1023) << 52));
          const float4 o = nv > 0 ? make_float4(vmax * rowf, (s0 + s1) * rowf, (q0 + q1) * rowf * rowf, static_cast<float>(nv))
                                  : make_float4(-INFINITY, 0.f, 0.f, 0.f);
          cb.st1[grow * (4 * kMaxKr) + kr * 2 + hc] = o;
          if (kr == 0 && hc == 0) *reinterpret_cast<int2*>(cb.cand_cnt + 2 * grow) = make_int2(0, 0);
        }
      } else {
        // ---------------------------------------------------------- kScoreCands
        // this warp: key columns [16 cq, 16 cq + 16) of each tile
        constexpr int CW = L::CW;
        const int cq = ew >> 2;
        const uint32_t lq = tm + (static_cast<uint32_t>(quad * 32) << 16) + cq * CW;
        float* colf = reinterpret_cast<float*>(smem + L::OFF_C) + ew * CW;
        // reference max and threshold from the row's approximate statistics
        // (the same arithmetic in every CTA that holds a part of the row)
        float m_ref = -INFINITY, t = INFINITY, tl = INFINITY;
        if (row_ok) {
          const float4* p = cb.st1 + grow * (4 * kMaxKr);
          float su = 0.f, sq = 0.f, n = 0.f;
          for (int j = 0; j < 2 * wk.n_kr; ++j) {
            const float4 a = p[j];
            m_ref = fmaxf(m_ref, a.x);
            su += a.y;
            sq += a.z;
            n += a.w;
          }
          const float mean = su / n;
          const float var = fmaxf(sq / n - mean * mean, 0.f);
          const float sd = sqrtf(var);
          t = cb.all_cand ? -INFINITY : mean + cb.zq * sd;
          if (!cb.all_cand) {
            // share of the row's mass (weights e^s) above t if the scores were
            // N(mean, sd^2): Q((t - mean - sd^2) / sd). Rows where Top-k alone
            // is expected to hold well over p Z skip the second list.
            const float share = 0.5f * erfcf((t - mean - sd * sd) / (sd * 1.41421356f));
            if (!(share >= cb.p_lo)) {
              // expected Top-p length: beyond both lists, the row goes straight
              // back to the full-row selection (no candidates: its count stays 0)
              const float need = static_cast<float>(wk.nkb) * 0.5f * erfcf((sd + cb.zp) * 0.70710678f);
              if (need > static_cast<float>(cb.c_hi + cb.c_lo)) t = INFINITY;
              else tl = fminf(t, mean + cb.zq_lo * sd);
            }
          }
        }
        const float mlog = m_ref * 1.4426950408889634f;
        const RowC rc = row_consts(scale, eq);
        int* cntp = cb.cand_cnt + 2 * (row_ok ? grow : 0);
        uint2* cl = cb.cand + (row_ok ? grow : 0) * (cb.c_hi + cb.c_lo);
        constexpr int XS = 32 * L::EW;                       // stride of a staged column
        float* xst0 = reinterpret_cast<float*>(smem + L::OFF_X) + ew * 32 + lane;
        auto ld_ekq = [&](int kt) -> int {
          const int kcol = kt * kI8TileN + cq * CW + lane;
          return (lane < CW && kcol < wk.nkb) ? __ldg(k_ex + static_cast<long long>(bh) * wk.nkb + kcol) : 0;
        };
        double z = 0.0;
        float mx = -INFINITY;
        int ek_next = kt0 < kt1 ? ld_ekq(kt0) : 0;
        for (int kt = kt0; kt < kt1; ++kt, ++bt) {
          const int ab = bt & 1;
          const int kc0 = kt * kI8TileN + cq * CW;
          const int ek = ek_next;
          if (kt + 1 < kt1) ek_next = ld_ekq(kt + 1);
          // the candidates of two tiles ago, while this tile's MMAs run (their
          // staging buffer is this tile's)
          flush_cands(p2.h, p2.jh, p2.kc0, p2.xb, p2.cl, cb.c_hi, XS);
          flush_cands(p2.l, p2.jl, p2.kc0, p2.xb, p2.cl + cb.c_hi, cb.c_lo, XS);
          ok = __all_sync(0xFFFFFFFFu, mbar_wait(&acc_full[ab], (bt >> 1) & 1, abort_flag));   // warp-uniform
          if (!ok) break;
          tc_fence_after();
          const uint32_t base = lq + ab * kSet;
          uint32_t a2[CW], a3[CW], a4[CW], a5[CW];
          tmem_ld16(base + 0 * kI8TileN, a2);
          tmem_ld16(base + 1 * kI8TileN, a3);
          tmem_ld16(base + 2 * kI8TileN, a4);
          tmem_ld16(base + 3 * kI8TileN, a5);
          if (lane < CW) colf[lane] = pow2f(ek);
          tmem_wait_ld();
          reg_fence16(a2);
          reg_fence16(a3);
          reg_fence16(a4);
          reg_fence16(a5);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[ab]);   // accumulators are in registers: the MMA may go on
          const int nvalid = min(CW, wk.nkb - kc0);
          float* xb = xst0 + ab * CW * XS;
          uint32_t selm = 0u, sell = 0u;      // columns >= t and >= t_lo; size the reservations and the writes
          float m = -INFINITY;
          float w[CW];
#pragma unroll
          for (int i = 0; i < CW; i += 4) {
            const float4 c = *reinterpret_cast<const float4*>(colf + i);
            const float cc[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int ii = i + u;
              const float xv = score_exact(a2[ii], a3[ii], a4[ii], a5[ii], rc) * cc[u];
              w[ii] = cand_weight(xv, mlog);
              selm |= (xv >= t ? 1u : 0u) << ii;
              sell |= (xv >= tl ? 1u : 0u) << ii;
              m = fmaxf(m, xv);
              xb[ii * XS] = xv;
            }
          }
          if (nvalid < CW) {
            // columns past the row end (warp-uniform, the row's last tile
            // only): out of both lists, the normaliser and the max
            const uint32_t vm = nvalid > 0 ? (1u << nvalid) - 1u : 0u;
            selm &= vm;
            sell &= vm;
            m = -INFINITY;
#pragma unroll
            for (int ii = 0; ii < CW; ++ii) {
              if (ii >= nvalid) w[ii] = 0.f;
              else m = fmaxf(m, xb[ii * XS]);
            }
          }
          // pairwise sum of the chunk's weights (fp32, two lanes per add)
          uint64_t q2[CW / 2];
#pragma unroll
          for (int i = 0; i < CW / 2; ++i) q2[i] = f2_make(w[2 * i], w[2 * i + 1]);
#pragma unroll
          for (int h = CW / 4; h > 0; h >>= 1)
#pragma unroll
            for (int i = 0; i < h; ++i) q2[i] = fadd2(q2[i], q2[i + h]);
          float z0, z1;
          f2_split(q2[0], z0, z1);
          const float zt = z0 + z1;
          sell &= ~selm;
          CandPend nw;                            // this tile's (buffer = tile parity, free since p2 is written)
          if ((selm | sell) != 0u) {
            if (selm != 0u) nw.jh = atomicAdd(cntp, __popc(selm));      // read two tiles later
            if (sell != 0u) nw.jl = atomicAdd(cntp + 1, __popc(sell));
            nw.h = selm;
            nw.l = sell;
            nw.kc0 = kc0;
            nw.cl = cl;
            nw.xb = xb;
          }
          p2 = p1;
          p1 = nw;
          z += static_cast<double>(zt);        // fp64 across chunks
          mx = fmaxf(mx, m);
          __syncwarp();
        }
        if (ok && row_ok) {
          ZPart zp;
          zp.z = z;
          zp.mx = mx;
          zp.pad = 0.f;
          cb.st2[grow * (4 * kMaxKr) + kr * 4 + cq] = zp;
          if (kr == 0 && cq == 0) cb.rowinfo[grow] = make_float2(m_ref, t);
        }
      }
    }
    if constexpr (MODE == kScoreCands) {
      constexpr int XS = 32 * L::EW;
      flush_cands(p2.h, p2.jh, p2.kc0, p2.xb, p2.cl, cb.c_hi, XS);
      flush_cands(p2.l, p2.jl, p2.kc0, p2.xb, p2.cl + cb.c_hi, cb.c_lo, XS);
      flush_cands(p1.h, p1.jh, p1.kc0, p1.xb, p1.cl, cb.c_hi, XS);
      flush_cands(p1.l, p1.jl, p1.kc0, p1.xb, p1.cl + cb.c_hi, cb.c_lo, XS);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tm, kAlloc);
  }
}

// ---------------------------------------------------------------- selection
// One warp per query-block row; rows of the grid are strided over the warps.
//
//   keys    monotone uint32 image of the fp32 scores (larger score -> larger key)
//   Top-k   the K_sel-th largest key; ties at the cut are kept in ascending
//           block order (ballot prefix counts)
//   Top-p   only when the Top-k set holds less than p of the mass (Z and every
//           mass in fp64): bitwise search for the largest key v with
//           mass(key >= v) >= p * Z, then the ties at v in block order until
//           the mass is reached
//   output  the union is the longer of the two prefixes of the common order;
//           kept indices are written in ascending order (ballot compaction)
constexpr int kSelWarpsMax = 8;

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

// ---------------------------------------------------------------- selection, candidate path
// Rows of at most 32 * KPL key blocks, with the row's scores in registers
// (element lane + 32 j in x[j]).
// K_sel is a small fraction of the row, so the exact search runs on a short
// candidate list instead of the whole row:
//   1. one pass gives the row max, mean and spread; a value t is then sought
//      with K_sel <= count(s >= t) <= kCandMax, starting from the normal
//      quantile of the row at about twice K_sel (tail quantile by Abramowitz
//      and Stegun 26.2.23) and bracketing from there; usually 1-3 count
//      passes;
//   2. the elements >= t are compacted, in ascending block order, into shared
//      memory, and the K_sel-th largest key is found by a bitwise search over
//      the bits in which the candidates differ;
//   3. the Top-k mass and the kept list come from the candidates alone.
// Rows whose search does not settle (many equal scores), rows whose Top-p set
// is longer than Top-k, and calls that want the u8 mask take full-row passes.
// Weights are e^(s - max) by ex2.approx (relative error ~1e-7, an order of
// magnitude inside the 1e-6 band within which a cumulative sum counts as a
// tie with p); Z and all masses are summed in fp64.
constexpr int kCandMax = 256;                 // candidates of the shared-memory (long row) path
constexpr int kCandPL = kCandMax / 32;
constexpr int kRegCandMax = 128;              // candidates of the register path: the first
constexpr int kRegCandPL = kRegCandMax / 32;  // guess aims near twice K_sel

__device__ __forceinline__ float sel_weight(float x, float mx) {
  return fast_exp2((x - mx) * 1.4426950408889634f);
}

__device__ __forceinline__ float key_value(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// z with P(Z > z) = f for a standard normal Z, 0 < f <= 0.5 (Abramowitz and
// Stegun 26.2.23, absolute error below 4.5e-4).
__device__ __forceinline__ float normal_tail_quantile(float f) {
  const float t = sqrtf(-2.f * logf(f));
  return t - (2.515517f + t * (0.802853f + t * 0.010328f)) /
                 (1.f + t * (1.432788f + t * (0.189269f + t * 0.001308f)));
}

__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

template <int N>
__device__ __forceinline__ int count_ge_f(const float (&x)[N], float t) {
  int n = 0;
#pragma unroll
  for (int j = 0; j < N; ++j) n += x[j] >= t ? 1 : 0;
  return static_cast<int>(__reduce_add_sync(0xFFFFFFFFu, static_cast<unsigned>(n)));
}

template <int N>
__device__ __forceinline__ int count_ge_u(const uint32_t (&k)[N], uint32_t c) {
  int n = 0;
#pragma unroll
  for (int j = 0; j < N; ++j) n += k[j] >= c ? 1 : 0;
  return static_cast<int>(__reduce_add_sync(0xFFFFFFFFu, static_cast<unsigned>(n)));
}

// Keys of x on the fly; elements past the row end never count.
template <int KPL>
__device__ __forceinline__ int count_key_ge(const float (&x)[KPL], int nkb, uint32_t c) {
  const int lane = threadIdx.x & 31;
  int n = 0;
#pragma unroll
  for (int j = 0; j < KPL; ++j) n += (lane + 32 * j < nkb && score_key(x[j]) >= c) ? 1 : 0;
  return static_cast<int>(__reduce_add_sync(0xFFFFFFFFu, static_cast<unsigned>(n)));
}

// Exact K_sel-th largest key of the whole row (fallback of the candidate path).
template <int KPL>
__device__ Cut topk_full(const float (&x)[KPL], int nkb, int k_sel) {
  uint32_t v = 0;
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t c = v | (1u << bit);
    if (count_key_ge(x, nkb, c) >= k_sel) v = c;
  }
  const int above = v == 0xFFFFFFFFu ? 0 : count_key_ge(x, nkb, v + 1u);
  return Cut{v, above, k_sel - above};
}

// Smallest prefix (by key) whose weight reaches target; weights in er[i].
template <int KPL>
__device__ Cut mass_full(const float (&x)[KPL], int nkb, const float* er, double target) {
  const int lane = threadIdx.x & 31;
  uint32_t v = 0;
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t c = v | (1u << bit);
    double w = 0.0;
#pragma unroll
    for (int j = 0; j < KPL; ++j)
      if (lane + 32 * j < nkb && score_key(x[j]) >= c) w += static_cast<double>(er[lane + 32 * j]);
    if (warp_sum_d(w) >= target) v = c;
  }
  int above = 0, nties = 0;
  double w_above = 0.0;
  float e_tie = 0.f;
#pragma unroll
  for (int j = 0; j < KPL; ++j) {
    if (lane + 32 * j >= nkb) continue;
    const uint32_t key = score_key(x[j]);
    if (key > v) {
      ++above;
      w_above += static_cast<double>(er[lane + 32 * j]);
    } else if (key == v) {
      ++nties;
      e_tie = er[lane + 32 * j];
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

// Kept set of a cut over the whole row, in ascending block order.
template <int KPL>
__device__ void output_full(const float (&x)[KPL], int nkb, const Cut& cut, int* __restrict__ out,
                            int* __restrict__ cnt_out, uint8_t* __restrict__ mrow) {
  const int lane = threadIdx.x & 31;
  const uint32_t lt = (1u << lane) - 1u;
  int written = 0, tie_before = 0;
#pragma unroll
  for (int j = 0; j < KPL; ++j) {
    const int i = lane + 32 * j;
    const bool valid = i < nkb;
    const uint32_t key = score_key(x[j]);
    const bool tie = valid && key == cut.key;
    const uint32_t tb = __ballot_sync(0xFFFFFFFFu, tie);
    const bool keep = valid && (key > cut.key || (tie && tie_before + __popc(tb & lt) < cut.ties));
    const uint32_t kb = __ballot_sync(0xFFFFFFFFu, keep);
    if (keep) out[written + __popc(kb & lt)] = i;
    if (mrow && valid) mrow[i] = keep ? 1 : 0;
    written += __popc(kb);
    tie_before += __popc(tb);
  }
  if (lane == 0) *cnt_out = written;
}

// One query-block row per warp. `ckey`/`cidx` hold kRegCandMax candidates and
// `er` 32 * KPL weights, all in this warp's shared memory.
template <int KPL>
__device__ void select_row_fast(const float* __restrict__ srow, int nkb, int k_sel, double topp,
                                int* __restrict__ out, int* __restrict__ cnt_out,
                                uint8_t* __restrict__ mrow, uint32_t* ckey, int* cidx, float* er) {
  const int lane = threadIdx.x & 31;
  const uint32_t lt = (1u << lane) - 1u;
  float x[KPL];
  float mx = -INFINITY, sum = 0.f, sq = 0.f;
#pragma unroll
  for (int j = 0; j < KPL; ++j) {
    const int i = lane + 32 * j;
    x[j] = i < nkb ? srow[i] : -INFINITY;
    if (i < nkb) {
      sum += x[j];
      sq = fmaf(x[j], x[j], sq);
    }
    mx = fmaxf(mx, x[j]);
  }
  mx = warp_max(mx);
  double z0 = 0.0, z1 = 0.0;
#pragma unroll
  for (int j = 0; j < KPL; ++j) {
    const float e = sel_weight(x[j], mx);            // 0 past the row end (x = -inf)
    er[lane + 32 * j] = e;
    if (j & 1) z1 += static_cast<double>(e);
    else z0 += static_cast<double>(e);
  }
  const double z = warp_sum_d(z0 + z1);

  if (topp >= 1.0 || k_sel >= nkb) {
    output_full(x, nkb, Cut{0u, 0, nkb}, out, cnt_out, mrow);   // every finite score's key is > 0
    return;
  }
  const double target = topp * z;

  // ---- 1. a threshold value with K_sel <= count <= kRegCandMax
  bool found = false;
  float t = mx;
  if (k_sel <= kRegCandMax) {
    sum = warp_sum_f(sum);
    sq = warp_sum_f(sq);
    const float mean = sum / nkb;
    const float sd = sqrtf(fmaxf(sq / nkb - mean * mean, 0.f));
    const int want = min(kRegCandMax - 32, max(2 * k_sel, k_sel + 32));
    const float f = fminf(static_cast<float>(want) / nkb, 0.5f);
    t = fminf(mean + normal_tail_quantile(f) * sd, mx);
    const float step = fmaxf(sd, 1e-6f * fmaxf(fabsf(mx), 1.f));
    float tlo = -INFINITY, thi = INFINITY;
    for (int it = 0; it < 12; ++it) {
      const int c = count_ge_f(x, t);
      if (c >= k_sel && c <= kRegCandMax) {
        found = true;
        break;
      }
      if (c < k_sel) thi = t;
      else tlo = t;
      float nt;
      if (tlo > -INFINITY && thi < INFINITY) nt = 0.5f * (tlo + thi);
      else if (thi < INFINITY) nt = thi - step * static_cast<float>(1 << it);
      else nt = fminf(tlo + step * static_cast<float>(1 << it), mx);
      if (nt == t || nt == tlo || nt == thi) break;   // no float left between the bounds
      t = nt;
    }
  }

  Cut cut;
  if (found) {
    // ---- 2. candidates in ascending block order, exact search among them
    int m = 0;
#pragma unroll
    for (int j = 0; j < KPL; ++j) {
      const bool take = x[j] >= t;
      const uint32_t b = __ballot_sync(0xFFFFFFFFu, take);
      if (take) {
        ckey[m + __popc(b & lt)] = score_key(x[j]);
        cidx[m + __popc(b & lt)] = lane + 32 * j;
      }
      m += __popc(b);
    }
    __syncwarp();
    uint32_t ck[kRegCandPL];
    uint32_t kand = 0xFFFFFFFFu, kor = 0u;
#pragma unroll
    for (int q = 0; q < kRegCandPL; ++q) {
      const bool valid = lane + 32 * q < m;
      ck[q] = valid ? ckey[lane + 32 * q] : 0u;
      if (valid) {
        kand &= ck[q];
        kor |= ck[q];
      }
    }
    kand = __reduce_and_sync(0xFFFFFFFFu, kand);
    kor = __reduce_or_sync(0xFFFFFFFFu, kor);
    const uint32_t diff = kand ^ kor;
    const int top = diff ? 31 - __clz(diff) : -1;
    uint32_t v = top >= 0 ? (kand & ~(0xFFFFFFFFu >> (31 - top))) : kand;   // common high bits
    for (int bit = top; bit >= 0; --bit) {
      const uint32_t c = v | (1u << bit);
      if (count_ge_u(ck, c) >= k_sel) v = c;
    }
    const int above = v == 0xFFFFFFFFu ? 0 : count_ge_u(ck, v + 1u);
    cut = Cut{v, above, k_sel - above};
    // ---- 3. Top-k mass over the kept candidates
    double wk = 0.0;
    int tie_before = 0;
#pragma unroll
    for (int q = 0; q < kRegCandPL; ++q) {
      const bool valid = lane + 32 * q < m;
      const bool tie = valid && ck[q] == v;
      const uint32_t tb = __ballot_sync(0xFFFFFFFFu, tie);
      const bool keep = valid && (ck[q] > v || (tie && tie_before + __popc(tb & lt) < cut.ties));
      if (keep) wk += static_cast<double>(sel_weight(key_value(ck[q]), mx));
      tie_before += __popc(tb);
    }
    wk = warp_sum_d(wk);
    if (wk >= target && mrow == nullptr) {
      int written = 0;
      tie_before = 0;
#pragma unroll
      for (int q = 0; q < kRegCandPL; ++q) {
        const bool valid = lane + 32 * q < m;
        const bool tie = valid && ck[q] == v;
        const uint32_t tb = __ballot_sync(0xFFFFFFFFu, tie);
        const bool keep = valid && (ck[q] > v || (tie && tie_before + __popc(tb & lt) < cut.ties));
        const uint32_t kb = __ballot_sync(0xFFFFFFFFu, keep);
        if (keep) out[written + __popc(kb & lt)] = cidx[lane + 32 * q];
        written += __popc(kb);
        tie_before += __popc(tb);
      }
      if (lane == 0) *cnt_out = written;
      __syncwarp();
      return;
    }
    __syncwarp();
    if (wk < target) {
      const Cut cp = mass_full(x, nkb, er, target);
      if (cp.above + cp.ties > k_sel) cut = cp;
    }
  } else {
    cut = topk_full(x, nkb, k_sel);
    // Top-k mass over the whole row
    double wk = 0.0;
    int tie_before = 0;
#pragma unroll
    for (int j = 0; j < KPL; ++j) {
      const bool valid = lane + 32 * j < nkb;
      const uint32_t key = score_key(x[j]);
      const bool tie = valid && key == cut.key;
      const uint32_t tb = __ballot_sync(0xFFFFFFFFu, tie);
      const bool keep = valid && (key > cut.key || (tie && tie_before + __popc(tb & lt) < cut.ties));
      if (keep) wk += static_cast<double>(er[lane + 32 * j]);
      tie_before += __popc(tb);
    }
    wk = warp_sum_d(wk);
    if (wk < target) {
      const Cut cp = mass_full(x, nkb, er, target);
      if (cp.above + cp.ties > k_sel) cut = cp;
    }
  }
  output_full(x, nkb, cut, out, cnt_out, mrow);
}

constexpr int kSelFastWarps = 4;

// With `rows`, the rows are rows[0 .. *n_rows_dev) (rows handed back by the
// candidate selection); otherwise 0 .. n_rows.
template <int KPL>
__global__ void __launch_bounds__(kSelFastWarps * 32, 4) select_fast_kernel(
    const float* __restrict__ s, long long s_ld, int n_rows, int nkb, int k_sel, double topp,
    int* __restrict__ kv_idx, int* __restrict__ kv_cnt, uint8_t* __restrict__ mask,
    const int* __restrict__ rows, const int* __restrict__ n_rows_dev) {
  __shared__ uint32_t ckey_all[kSelFastWarps][kRegCandMax];
  __shared__ int cidx_all[kSelFastWarps][kRegCandMax];
  __shared__ float e_all[kSelFastWarps][32 * KPL];
  grid_dep_wait();
  const int warp = threadIdx.x >> 5;
  const int nr = n_rows_dev ? *n_rows_dev : n_rows;
  for (int ri = blockIdx.x * kSelFastWarps + warp; ri < nr; ri += gridDim.x * kSelFastWarps) {
    const int row = rows ? rows[ri] : ri;
    select_row_fast<KPL>(s + static_cast<long long>(row) * s_ld, nkb, k_sel, topp,
                         kv_idx + static_cast<long long>(row) * nkb, kv_cnt + row,
                         mask ? mask + static_cast<long long>(row) * nkb : nullptr,
                         ckey_all[warp], cidx_all[warp], e_all[warp]);
    __syncwarp();
  }
}

template <int KPL>
static cudaError_t launch_select_fast(const float* s, long long s_ld, int n_rows, int nkb, int k_sel,
                                      double topp, int* kv_idx, int* kv_cnt, uint8_t* mask,
                                      const int* rows, const int* n_rows_dev, int grid_cap, cudaStream_t st) {
  const int want = (n_rows + kSelFastWarps - 1) / kSelFastWarps;
  const int grid = want < grid_cap ? want : grid_cap;
  return launch_pdl(select_fast_kernel<KPL>, dim3(grid), dim3(kSelFastWarps * 32), 0, st, s, s_ld, n_rows, nkb, k_sel,
                    topp, kv_idx, kv_cnt, mask, rows, n_rows_dev);
}

// ---------------------------------------------------------------- selection, long rows
// Rows of more than 32 * 40 key blocks: the same candidate path with the row
// staged once in the warp's shared memory (`xs`) instead of registers; every
// count pass then reads shared memory. The full-row passes for the uncommon
// cases read it too.
__device__ __forceinline__ int smem_count_ge(const float* xs, int n, float t) {
  const int lane = threadIdx.x & 31;
  int c = 0;
#pragma unroll 4
  for (int i = lane; i < n; i += 32) c += xs[i] >= t ? 1 : 0;
  return static_cast<int>(__reduce_add_sync(0xFFFFFFFFu, static_cast<unsigned>(c)));
}

__device__ __forceinline__ int smem_count_key_ge(const float* xs, int n, uint32_t k) {
  const int lane = threadIdx.x & 31;
  int c = 0;
#pragma unroll 4
  for (int i = lane; i < n; i += 32) c += score_key(xs[i]) >= k ? 1 : 0;
  return static_cast<int>(__reduce_add_sync(0xFFFFFFFFu, static_cast<unsigned>(c)));
}

// Weight of the elements kept by `cut` (ties in ascending block order).
__device__ double smem_cut_mass(const float* xs, int n, const Cut& cut, float mx) {
  const int lane = threadIdx.x & 31;
  const uint32_t lt = (1u << lane) - 1u;
  double w = 0.0;
  int tie_before = 0;
  for (int base = 0; base < n; base += 32) {
    const int i = base + lane;
    const float x = i < n ? xs[i] : -INFINITY;
    const uint32_t key = score_key(x);
    const bool tie = i < n && key == cut.key;
    const uint32_t tb = __ballot_sync(0xFFFFFFFFu, tie);
    const bool keep = i < n && (key > cut.key || (tie && tie_before + __popc(tb & lt) < cut.ties));
    if (keep) w += static_cast<double>(sel_weight(x, mx));
    tie_before += __popc(tb);
  }
  return warp_sum_d(w);
}

// Smallest prefix (by key) whose weight reaches target.
__device__ Cut smem_mass(const float* xs, int n, float mx, double target) {
  const int lane = threadIdx.x & 31;
  uint32_t v = 0;
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t c = v | (1u << bit);
    double w = 0.0;
    for (int i = lane; i < n; i += 32) {
      const float x = xs[i];
      if (score_key(x) >= c) w += static_cast<double>(sel_weight(x, mx));
    }
    if (warp_sum_d(w) >= target) v = c;
  }
  int above = 0, nties = 0;
  double w_above = 0.0;
  float e_tie = 0.f;
  for (int i = lane; i < n; i += 32) {
    const float x = xs[i];
    const uint32_t key = score_key(x);
    if (key > v) {
      ++above;
      w_above += static_cast<double>(sel_weight(x, mx));
    } else if (key == v) {
      ++nties;
      e_tie = sel_weight(x, mx);
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

// Kept set of a cut over the whole row, in ascending block order.
__device__ void smem_output(const float* xs, int n, const Cut& cut, int* __restrict__ out,
                            int* __restrict__ cnt_out, uint8_t* __restrict__ mrow) {
  const int lane = threadIdx.x & 31;
  const uint32_t lt = (1u << lane) - 1u;
  int written = 0, tie_before = 0;
  for (int base = 0; base < n; base += 32) {
    const int i = base + lane;
    const bool valid = i < n;
    const uint32_t key = valid ? score_key(xs[i]) : 0u;
    const bool tie = valid && key == cut.key;
    const uint32_t tb = __ballot_sync(0xFFFFFFFFu, tie);
    const bool keep = valid && (key > cut.key || (tie && tie_before + __popc(tb & lt) < cut.ties));
    const uint32_t kb = __ballot_sync(0xFFFFFFFFu, keep);
    if (keep) out[written + __popc(kb & lt)] = i;
    if (mrow && valid) mrow[i] = keep ? 1 : 0;
    written += __popc(kb);
    tie_before += __popc(tb);
  }
  if (lane == 0) *cnt_out = written;
}

__device__ void select_row_long(const float* __restrict__ srow, int nkb, int k_sel, double topp,
                                int* __restrict__ out, int* __restrict__ cnt_out,
                                uint8_t* __restrict__ mrow, float* xs, uint32_t* ckey, int* cidx) {
  const int lane = threadIdx.x & 31;
  const uint32_t lt = (1u << lane) - 1u;
  float mx = -INFINITY, sum = 0.f, sq = 0.f, ns = 0.f;
  for (int i = lane; i < nkb; i += 32) {
    const float v = srow[i];
    xs[i] = v;
    mx = fmaxf(mx, v);
    if (((i >> 5) & 7) == 0) {                 // every eighth column for the mean and spread
      sum += v;
      sq = fmaf(v, v, sq);
      ns += 1.f;
    }
  }
  mx = warp_max(mx);
  __syncwarp();
  double z = 0.0;
  float part = 0.f;
  int np = 0;
  for (int i = lane; i < nkb; i += 32) {
    part += sel_weight(xs[i], mx);             // four weights <= 1 each, exact to 2^-22
    if (++np == 4) {
      z += static_cast<double>(part);
      part = 0.f;
      np = 0;
    }
  }
  z = warp_sum_d(z + static_cast<double>(part));

  if (topp >= 1.0 || k_sel >= nkb) {
    smem_output(xs, nkb, Cut{0u, 0, nkb}, out, cnt_out, mrow);   // every finite score's key is > 0
    return;
  }
  const double target = topp * z;

  // ---- 1. a threshold value with K_sel <= count <= kCandMax
  bool found = false;
  float t = mx;
  if (k_sel <= kCandMax) {
    sum = warp_sum_f(sum);
    sq = warp_sum_f(sq);
    ns = warp_sum_f(ns);
    const float mean = sum / ns;
    const float sd = sqrtf(fmaxf(sq / ns - mean * mean, 0.f));
    const int want = min(kCandMax - 32, max(2 * k_sel, k_sel + 32));
    const float f = fminf(static_cast<float>(want) / nkb, 0.5f);
    t = fminf(mean + normal_tail_quantile(f) * sd, mx);
    const float step = fmaxf(sd, 1e-6f * fmaxf(fabsf(mx), 1.f));
    float tlo = -INFINITY, thi = INFINITY;
    for (int it = 0; it < 12; ++it) {
      const int c = smem_count_ge(xs, nkb, t);
      if (c >= k_sel && c <= kCandMax) {
        found = true;
        break;
      }
      if (c < k_sel) thi = t;
      else tlo = t;
      float nt;
      if (tlo > -INFINITY && thi < INFINITY) nt = 0.5f * (tlo + thi);
      else if (thi < INFINITY) nt = thi - step * static_cast<float>(1 << it);
      else nt = fminf(tlo + step * static_cast<float>(1 << it), mx);
      if (nt == t || nt == tlo || nt == thi) break;   // no float left between the bounds
      t = nt;
    }
  }
  if (!found) {
    uint32_t v = 0;
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t c = v | (1u << bit);
      if (smem_count_key_ge(xs, nkb, c) >= k_sel) v = c;
    }
    const int above = v == 0xFFFFFFFFu ? 0 : smem_count_key_ge(xs, nkb, v + 1u);
    Cut cut{v, above, k_sel - above};
    if (smem_cut_mass(xs, nkb, cut, mx) < target) {
      const Cut cp = smem_mass(xs, nkb, mx, target);
      if (cp.above + cp.ties > k_sel) cut = cp;
    }
    smem_output(xs, nkb, cut, out, cnt_out, mrow);
    return;
  }

  // ---- 2. candidates in ascending block order, exact search among them
  int m = 0;
  for (int base = 0; base < nkb; base += 32) {
    const int i = base + lane;
    const float x = i < nkb ? xs[i] : -INFINITY;
    const bool take = i < nkb && x >= t;
    const uint32_t b = __ballot_sync(0xFFFFFFFFu, take);
    if (take) {
      ckey[m + __popc(b & lt)] = score_key(x);
      cidx[m + __popc(b & lt)] = i;
    }
    m += __popc(b);
  }
  __syncwarp();
  uint32_t ck[kCandPL];
  uint32_t kand = 0xFFFFFFFFu, kor = 0u;
#pragma unroll
  for (int q = 0; q < kCandPL; ++q) {
    const bool valid = lane + 32 * q < m;
    ck[q] = valid ? ckey[lane + 32 * q] : 0u;
    if (valid) {
      kand &= ck[q];
      kor |= ck[q];
    }
  }
  kand = __reduce_and_sync(0xFFFFFFFFu, kand);
  kor = __reduce_or_sync(0xFFFFFFFFu, kor);
  const uint32_t diff = kand ^ kor;
  const int top = diff ? 31 - __clz(diff) : -1;
  uint32_t v = top >= 0 ? (kand & ~(0xFFFFFFFFu >> (31 - top))) : kand;   // common high bits
  for (int bit = top; bit >= 0; --bit) {
    const uint32_t c = v | (1u << bit);
    if (count_ge_u(ck, c) >= k_sel) v = c;
  }
  const int above = v == 0xFFFFFFFFu ? 0 : count_ge_u(ck, v + 1u);
  Cut cut{v, above, k_sel - above};
  // ---- 3. Top-k mass over the kept candidates
  double wk = 0.0;
  int tie_before = 0;
#pragma unroll
  for (int q = 0; q < kCandPL; ++q) {
    const bool valid = lane + 32 * q < m;
    const bool tie = valid && ck[q] == v;
    const uint32_t tb = __ballot_sync(0xFFFFFFFFu, tie);
    const bool keep = valid && (ck[q] > v || (tie && tie_before + __popc(tb & lt) < cut.ties));
    if (keep) wk += static_cast<double>(sel_weight(key_value(ck[q]), mx));
    tie_before += __popc(tb);
  }
  wk = warp_sum_d(wk);
  if (wk >= target && mrow == nullptr) {
    int written = 0;
    tie_before = 0;
#pragma unroll
    for (int q = 0; q < kCandPL; ++q) {
      const bool valid = lane + 32 * q < m;
      const bool tie = valid && ck[q] == v;
      const uint32_t tb = __ballot_sync(0xFFFFFFFFu, tie);
      const bool keep = valid && (ck[q] > v || (tie && tie_before + __popc(tb & lt) < cut.ties));
      const uint32_t kb = __ballot_sync(0xFFFFFFFFu, keep);
      if (keep) out[written + __popc(kb & lt)] = cidx[lane + 32 * q];
      written += __popc(kb);
      tie_before += __popc(tb);
    }
    if (lane == 0) *cnt_out = written;
    return;
  }
  if (wk < target) {
    const Cut cp = smem_mass(xs, nkb, mx, target);
    if (cp.above + cp.ties > k_sel) cut = cp;
  }
  smem_output(xs, nkb, cut, out, cnt_out, mrow);
}

// Per warp: the row (nkb floats), then kCandMax keys and indices.
__global__ void __launch_bounds__(kSelWarpsMax * 32) select_long_kernel(
    const float* __restrict__ s, long long s_ld, int n_rows, int nkb, int k_sel, double topp,
    int* __restrict__ kv_idx, int* __restrict__ kv_cnt, uint8_t* __restrict__ mask, int slice,
    const int* __restrict__ rows, const int* __restrict__ n_rows_dev) {
  extern __shared__ __align__(16) uint8_t sm_long[];
  grid_dep_wait();
  const int warp = threadIdx.x >> 5;
  const int wpc = blockDim.x >> 5;
  float* xs = reinterpret_cast<float*>(sm_long + static_cast<size_t>(warp) * slice);
  uint32_t* ckey = reinterpret_cast<uint32_t*>(xs + nkb);
  int* cidx = reinterpret_cast<int*>(ckey + kCandMax);
  const int nr = n_rows_dev ? *n_rows_dev : n_rows;
  for (int ri = blockIdx.x * wpc + warp; ri < nr; ri += gridDim.x * wpc) {
    const int row = rows ? rows[ri] : ri;
    select_row_long(s + static_cast<long long>(row) * s_ld, nkb, k_sel, topp,
                    kv_idx + static_cast<long long>(row) * nkb, kv_cnt + row,
                    mask ? mask + static_cast<long long>(row) * nkb : nullptr, xs, ckey, cidx);
    __syncwarp();
  }
}

// ---------------------------------------------------------------- selection from candidate lists
// One warp per query-block row, after the kScoreStats and kScoreCands passes.
// The row has two lists: every score >= t (first list), and every score in
// [t_lo, t) (second list), each complete when its count is within its
// capacity.
//   Z       the sum of the row's partial normalisers (fp64, fixed order)
//   Top-k   the K_sel-th largest key; when the first list holds at least
//           K_sel scores it holds every score at or above that key
//           (bitwise search over the bits in which the candidates differ)
//   Top-p   only when the Top-k mass is below p Z: the largest key u whose
//           candidate mass reaches p Z, then the ties at u in block order;
//           the same key as over the whole row as long as the listed
//           candidates' total mass reaches p Z, because every key above the
//           list's threshold is listed
//   output  the union is the longer prefix of the common order; the kept
//           blocks are set as bits in the warp's shared memory (ties at the
//           cut in ascending block order) and written as the ascending list
// Fast path: the first list in registers (up to `cap` entries), when it
// settles both cuts. Wide path: both lists staged in the warp's shared
// memory. A row goes back to the score-matrix path (its query tile rescored
// by kScoreWrite, then the full-row selection) when a list overflowed, when
// even both lists hold less than p Z or fewer than K_sel scores, or when the
// reference max is more than 30 from the exact one (weights relative to
// m_ref could then overflow or lose the row's largest terms).
struct CandSel {
  const ZPart* st2;
  const float2* rowinfo;
  const int* cand_cnt;
  const uint2* cand;
  int c_hi, c_lo, cap, n_parts, nqb, n_qt;
  int* fb_cnt;
  int* fb_rows;
  int* tile_flag;
};
constexpr int kCandSelWarps = 8;

__device__ __forceinline__ void hand_back(const CandSel& cs, int row) {
  if ((threadIdx.x & 31) == 0) {
    const int p = atomicAdd(cs.fb_cnt, 1);
    cs.fb_rows[p] = row;
    cs.tile_flag[(row / cs.nqb) * cs.n_qt + (row % cs.nqb) / kI8TileM] = 1;
  }
}

__device__ __forceinline__ double warp_max_d(double v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmax(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

// Exclusive prefix sum over the lanes.
__device__ __forceinline__ int warp_excl_scan(int v) {
  const int lane = threadIdx.x & 31;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  return x - v;
}

// Ties at the Top-p key u: how many (in block order) reach the target.
__device__ __forceinline__ int topp_ties(double w_above, double e_tie, int above, int nties, double target) {
  int tn = 0;
  double acc = w_above;
  while (acc < target && tn < nties) {
    acc += e_tie;
    ++tn;
  }
  if (acc < target) tn = nties;        // rounding kept the total below the target
  if (above + tn == 0) tn = 1;
  return tn;
}

__device__ __forceinline__ void clear_bits(uint32_t* keep, uint32_t* tieb, int W) {
  const int lane = threadIdx.x & 31;
  for (int i = lane; i < W; i += 32) {
    keep[i] = 0u;
    tieb[i] = 0u;
  }
  __syncwarp();
}

// Marks one candidate: kept above the cut (or at it when every tie is kept),
// otherwise a tie at the cut goes to `tieb`.
__device__ __forceinline__ void mark_bit(uint32_t key, int blk, const Cut& cut, bool all_ties, uint32_t* keep,
                                         uint32_t* tieb) {
  const uint32_t bit = 1u << (blk & 31);
  if (key > cut.key || (key == cut.key && all_ties)) atomicOr(&keep[blk >> 5], bit);
  else if (key == cut.key) atomicOr(&tieb[blk >> 5], bit);
}

// The kept set from the bits: the cut.ties lowest-index ties join unless all
// do, then the ascending list, the optional u8 row and the count.
__device__ void emit_bits(int nkb, const Cut& cut, bool all_ties, int* __restrict__ out, int* __restrict__ cnt_out,
                          uint8_t* __restrict__ mrow, uint32_t* keep, const uint32_t* tieb) {
  const int lane = threadIdx.x & 31;
  __syncwarp();
  const int W = (nkb + 31) >> 5;
  const int wpl = (W + 31) >> 5;                // words per lane, in order
  const int w0 = min(W, lane * wpl), w1 = min(W, w0 + wpl);
  if (!all_ties) {
    int c = 0;
    for (int i = w0; i < w1; ++i) c += __popc(tieb[i]);
    int before = warp_excl_scan(c);
    for (int i = w0; i < w1 && before < cut.ties; ++i) {
      uint32_t b = tieb[i];
      while (b != 0u && before < cut.ties) {
        const uint32_t low = b & (0u - b);
        keep[i] |= low;
        b ^= low;
        ++before;
      }
    }
    __syncwarp();
  }
  int c = 0;
  for (int i = w0; i < w1; ++i) c += __popc(keep[i]);
  int pre = warp_excl_scan(c);                   // kept blocks before this lane's first word
  const int total = __shfl_sync(0xFFFFFFFFu, pre + c, 31);
  // round r: word r of every lane; its nonzero words one at a time, each
  // lane writing its own bit of the word (coalesced, in block order)
  const uint32_t lt = (1u << lane) - 1u;
  for (int r = 0; r < wpl; ++r) {
    const uint32_t word = w0 + r < w1 ? keep[w0 + r] : 0u;
    uint32_t nz = __ballot_sync(0xFFFFFFFFu, word != 0u);
    while (nz != 0u) {
      const int src = __ffs(nz) - 1;
      nz &= nz - 1u;
      const uint32_t wv = __shfl_sync(0xFFFFFFFFu, word, src);
      const int base = __shfl_sync(0xFFFFFFFFu, pre, src);
      if ((wv >> lane) & 1u) out[base + __popc(wv & lt)] = (src * wpl + r) * 32 + lane;
    }
    pre += __popc(word);
  }
  if (mrow)
    for (int i = lane; i < nkb; i += 32) mrow[i] = static_cast<uint8_t>((keep[i >> 5] >> (i & 31)) & 1u);
  if (lane == 0) *cnt_out = total;
}

// Fast path over the first list (cnt <= 32 CPL entries) in registers.
// Returns false, having written nothing, when the Top-p prefix needs more
// than the first list.
template <int CPL>
__device__ bool select_cand_fast(const uint2* cl, int cnt, int nkb, int k_sel, double target, float mlog,
                                 int* __restrict__ out, int* __restrict__ cnt_out, uint8_t* __restrict__ mrow,
                                 uint32_t* keep, uint32_t* tieb) {
  const int lane = threadIdx.x & 31;
  uint32_t ck[CPL];
  int ci[CPL];
  double wd[CPL];
  uint32_t kand = 0xFFFFFFFFu, kor = 0u;
#pragma unroll
  for (int q = 0; q < CPL; ++q) {
    const int sidx = lane + 32 * q;
    ck[q] = 0u;                                 // no finite score has key 0
    ci[q] = 0;
    wd[q] = 0.0;
    if (sidx < cnt) {
      const uint2 e = cl[sidx];
      ck[q] = e.x;
      ci[q] = static_cast<int>(e.y);
      wd[q] = static_cast<double>(cand_weight(key_value(e.x), mlog));
      kand &= e.x;
      kor |= e.x;
    }
  }
  kand = __reduce_and_sync(0xFFFFFFFFu, kand);
  kor = __reduce_or_sync(0xFFFFFFFFu, kor);
  const uint32_t diff = kand ^ kor;
  const int top = diff ? 31 - __clz(diff) : -1;
  const uint32_t pre = top >= 0 ? (kand & ~(0xFFFFFFFFu >> (31 - top))) : kand;   // common high bits
  // ---- Top-k
  uint32_t v = pre;
  for (int bit = top; bit >= 0; --bit) {
    const uint32_t c = v | (1u << bit);
    if (count_ge_u(ck, c) >= k_sel) v = c;
  }
  const int above = v == 0xFFFFFFFFu ? 0 : count_ge_u(ck, v + 1u);
  Cut cut{v, above, k_sel - above};
  double wa = 0.0, wt = 0.0, ev = 0.0;
  int nv = 0;
#pragma unroll
  for (int q = 0; q < CPL; ++q) {
    wt += wd[q];
    if (ck[q] > v) {
      wa += wd[q];
    } else if (ck[q] == v) {
      ev = wd[q];
      ++nv;
    }
  }
  wa = warp_sum_d(wa);
  ev = warp_max_d(ev);                          // every tie has the same weight
  nv = warp_sum_i(nv);
  int n_cut = nv;                               // elements equal to the cut key
  if (wa + static_cast<double>(cut.ties) * ev < target) {
    wt = warp_sum_d(wt);
    if (wt < target) return false;
    // ---- Top-p: the largest key u with mass(key >= u) >= target
    uint32_t u = pre;
    for (int bit = top; bit >= 0; --bit) {
      const uint32_t c = u | (1u << bit);
      double m = 0.0;
#pragma unroll
      for (int q = 0; q < CPL; ++q)
        if (ck[q] >= c) m += wd[q];
      if (warp_sum_d(m) >= target) u = c;
    }
    int pa = 0, nu = 0;
    double wpa = 0.0, eu = 0.0;
#pragma unroll
    for (int q = 0; q < CPL; ++q) {
      if (ck[q] > u) {
        ++pa;
        wpa += wd[q];
      } else if (ck[q] == u) {
        ++nu;
        eu = wd[q];
      }
    }
    pa = warp_sum_i(pa);
    nu = warp_sum_i(nu);
    wpa = warp_sum_d(wpa);
    eu = warp_max_d(eu);
    const int tn = topp_ties(wpa, eu, pa, nu, target);
    if (pa + tn > k_sel) {
      cut = Cut{u, pa, tn};
      n_cut = nu;
    }
  }
  const bool all_ties = cut.ties >= n_cut;
  clear_bits(keep, tieb, (nkb + 31) >> 5);
#pragma unroll
  for (int q = 0; q < CPL; ++q)
    if (ck[q] != 0u) mark_bit(ck[q], ci[q], cut, all_ties, keep, tieb);
  emit_bits(nkb, cut, all_ties, out, cnt_out, mrow, keep, tieb);
  return true;
}

// Wide path: both lists (nh + nl entries), read in place (L1/L2). Returns
// false, having written nothing, when they hold less than the target mass.
__device__ bool select_cand_wide(const uint2* __restrict__ cl, int c_hi, int nh, int nl, int nkb, int k_sel,
                                 double target, float mlog, int* __restrict__ out, int* __restrict__ cnt_out,
                                 uint8_t* __restrict__ mrow, uint32_t* keep, uint32_t* tieb) {
  const int lane = threadIdx.x & 31;
  const int n = nh + nl;
  auto entry = [&](int i) -> uint2 { return __ldg(i < nh ? cl + i : cl + c_hi + (i - nh)); };
  uint32_t kand = 0xFFFFFFFFu, kor = 0u;
  double wt = 0.0;
  for (int i = lane; i < n; i += 32) {
    const uint2 e = entry(i);
    kand &= e.x;
    kor |= e.x;
    wt += static_cast<double>(cand_weight(key_value(e.x), mlog));
  }
  kand = __reduce_and_sync(0xFFFFFFFFu, kand);
  kor = __reduce_or_sync(0xFFFFFFFFu, kor);
  wt = warp_sum_d(wt);
  const uint32_t diff = kand ^ kor;
  const int top = diff ? 31 - __clz(diff) : -1;
  const uint32_t pre = top >= 0 ? (kand & ~(0xFFFFFFFFu >> (31 - top))) : kand;
  auto count_ge = [&](uint32_t c) -> int {
    int k = 0;
    for (int i = lane; i < n; i += 32) k += entry(i).x >= c ? 1 : 0;
    return static_cast<int>(__reduce_add_sync(0xFFFFFFFFu, static_cast<unsigned>(k)));
  };
  // ---- Top-k
  uint32_t v = pre;
  for (int bit = top; bit >= 0; --bit) {
    const uint32_t c = v | (1u << bit);
    if (count_ge(c) >= k_sel) v = c;
  }
  const int above = v == 0xFFFFFFFFu ? 0 : count_ge(v + 1u);
  Cut cut{v, above, k_sel - above};
  double wa = 0.0, ev = 0.0;
  int nv = 0;
  for (int i = lane; i < n; i += 32) {
    const uint32_t key = entry(i).x;
    if (key > v) {
      wa += static_cast<double>(cand_weight(key_value(key), mlog));
    } else if (key == v) {
      ev = static_cast<double>(cand_weight(key_value(key), mlog));
      ++nv;
    }
  }
  wa = warp_sum_d(wa);
  ev = warp_max_d(ev);
  nv = warp_sum_i(nv);
  int n_cut = nv;
  if (wa + static_cast<double>(cut.ties) * ev < target) {
    if (wt < target) return false;
    // ---- Top-p
    uint32_t u = pre;
    for (int bit = top; bit >= 0; --bit) {
      const uint32_t c = u | (1u << bit);
      double m = 0.0;
      for (int i = lane; i < n; i += 32) {
        const uint32_t key = entry(i).x;
        if (key >= c) m += static_cast<double>(cand_weight(key_value(key), mlog));
      }
      if (warp_sum_d(m) >= target) u = c;
    }
    int pa = 0, nu = 0;
    double wpa = 0.0, eu = 0.0;
    for (int i = lane; i < n; i += 32) {
      const uint32_t key = entry(i).x;
      if (key > u) {
        ++pa;
        wpa += static_cast<double>(cand_weight(key_value(key), mlog));
      } else if (key == u) {
        ++nu;
        eu = static_cast<double>(cand_weight(key_value(key), mlog));
      }
    }
    pa = warp_sum_i(pa);
    nu = warp_sum_i(nu);
    wpa = warp_sum_d(wpa);
    eu = warp_max_d(eu);
    const int tn = topp_ties(wpa, eu, pa, nu, target);
    if (pa + tn > k_sel) {
      cut = Cut{u, pa, tn};
      n_cut = nu;
    }
  }
  const bool all_ties = cut.ties >= n_cut;
  clear_bits(keep, tieb, (nkb + 31) >> 5);
  for (int i = lane; i < n; i += 32) {
    const uint2 e = entry(i);
    mark_bit(e.x, static_cast<int>(e.y), cut, all_ties, keep, tieb);
  }
  emit_bits(nkb, cut, all_ties, out, cnt_out, mrow, keep, tieb);
  return true;
}

template <int CPL>
__device__ void select_cand_row(const CandSel& cs, int row, int nkb, int k_sel, double topp,
                                int* __restrict__ out, int* __restrict__ cnt_out, uint8_t* __restrict__ mrow,
                                uint32_t* keep, uint32_t* tieb) {
  const int lane = threadIdx.x & 31;
  if (topp >= 1.0 || k_sel >= nkb) {          // every block (every finite score)
    for (int i = lane; i < nkb; i += 32) {
      out[i] = i;
      if (mrow) mrow[i] = 1;
    }
    if (lane == 0) *cnt_out = nkb;
    return;
  }
  double zp = 0.0;
  float mxp = -INFINITY;
  if (lane < cs.n_parts) {
    const ZPart p = cs.st2[static_cast<long long>(row) * (4 * kMaxKr) + lane];
    zp = p.z;
    mxp = p.mx;
  }
  const double Z = warp_sum_d(zp);
  const float mx = warp_max(mxp);
  const float m_ref = cs.rowinfo[row].x;
  const int2 cnt = *reinterpret_cast<const int2*>(cs.cand_cnt + 2 * static_cast<long long>(row));
  if (!(fabsf(mx - m_ref) <= 30.f && Z > 0.0)) {   // NaN fails too
    hand_back(cs, row);
    return;
  }
  const float mlog = m_ref * 1.4426950408889634f;
  const double target = topp * Z;
  const uint2* cl = cs.cand + static_cast<long long>(row) * (cs.c_hi + cs.c_lo);
  if (cnt.x >= k_sel && cnt.x <= cs.cap &&
      select_cand_fast<CPL>(cl, cnt.x, nkb, k_sel, target, mlog, out, cnt_out, mrow, keep, tieb))
    return;
  if (cnt.x <= cs.c_hi && cnt.y <= cs.c_lo && cnt.x + cnt.y >= k_sel &&
      select_cand_wide(cl, cs.c_hi, cnt.x, cnt.y, nkb, k_sel, target, mlog, out, cnt_out, mrow, keep, tieb))
    return;
  hand_back(cs, row);
}

// Per warp: two bit rows of ceil(nkb / 32) words (kept, ties at the cut).
template <int CPL>
__global__ void __launch_bounds__(kCandSelWarps * 32) select_cand_kernel(
    CandSel cs, int n_rows, int nkb, int k_sel, double topp, int* __restrict__ kv_idx,
    int* __restrict__ kv_cnt, uint8_t* __restrict__ mask) {
  extern __shared__ __align__(16) uint32_t cand_smem[];
  grid_dep_wait();
  grid_dep_trigger();
  const int warp = threadIdx.x >> 5;
  const int W = (nkb + 31) >> 5;
  uint32_t* keep = cand_smem + static_cast<size_t>(warp) * 2 * W;
  uint32_t* tieb = keep + W;
  for (int row = blockIdx.x * kCandSelWarps + warp; row < n_rows; row += gridDim.x * kCandSelWarps) {
    select_cand_row<CPL>(cs, row, nkb, k_sel, topp, kv_idx + static_cast<long long>(row) * nkb, kv_cnt + row,
                         mask ? mask + static_cast<long long>(row) * nkb : nullptr, keep, tieb);
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
                        float* q_pool, float* k_pool, cudaStream_t st, const SliceOut* sl) {
  const SliceOut so = sl ? *sl : SliceOut{nullptr, nullptr, nullptr, nullptr};
  const int nqb = ceil_div(N, bq), nkb = ceil_div(N, bk);
  const long long warps = static_cast<long long>(BH) * (nqb + nkb);
  const long long blocks = (warps * 32 + 255) / 256;
  if (blocks > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  const auto* qq = static_cast<const __nv_bfloat16*>(q);
  const auto* kk = static_cast<const __nv_bfloat16*>(k);
  if (d == 128)
    pool_kernel<128><<<static_cast<unsigned>(blocks), 256, 0, st>>>(qq, kk, BH, N, bq, bk, nqb, nkb, q_pool, k_pool, so);
  else
    pool_kernel<64><<<static_cast<unsigned>(blocks), 256, 0, st>>>(qq, kk, BH, N, bq, bk, nqb, nkb, q_pool, k_pool, so);
  return cudaGetLastError();
}

// Work split of the score kernels: about four items per SM; at most kMaxKr
// key ranges per row where per-row partials are kept (cap_ranges).
struct I8Launch {
  I8Work w;
  int grid;
};

static cudaError_t i8_launch(int BH, int nqb, int nkb, I8Launch* out, bool cap_ranges,
                             int max_tiles_per_item = 0) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  I8Work w;
  w.nqb = nqb;
  w.nkb = nkb;
  w.n_qt = ceil_div(nqb, kI8TileM);
  w.n_kt = ceil_div(nkb, kI8TileN);
  const long long tiles = static_cast<long long>(BH) * w.n_qt * w.n_kt;
  long long per = (tiles + 4LL * sms - 1) / (4LL * sms);
  const long long per_min = cap_ranges ? (w.n_kt + kMaxKr - 1) / kMaxKr : 1;
  per = per < per_min ? per_min : per;
  if (max_tiles_per_item > 0 && per > max_tiles_per_item) per = max_tiles_per_item;
  per = per < 1 ? 1 : (per > w.n_kt ? w.n_kt : per);
  w.kr_tiles = static_cast<int>(per);
  w.n_kr = ceil_div(w.n_kt, w.kr_tiles);
  const long long items = static_cast<long long>(BH) * w.n_qt * w.n_kr;
  if (items > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  w.n_items = static_cast<int>(items);
  out->w = w;
  out->grid = w.n_items < sms ? w.n_items : sms;
  return cudaSuccess;
}

template <int D>
static cudaError_t i8_maps(const SliceOut& sl, int BH, int nqb, int nkb, CUtensorMap* ma, CUtensorMap* mb) {
  constexpr int ROW = 4 * D;
  if (encode_tensor_map_3d_u8(ma, sl.q_sl, ROW, nqb, BH, 128, kI8TileM) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  if (encode_tensor_map_3d_u8(mb, sl.k_sl, ROW, nkb, BH, 128, kI8TileN) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  return cudaSuccess;
}

template <int D, int MODE>
static cudaError_t launch_i8(const CUtensorMap& ma, const CUtensorMap& mb, const SliceOut& sl, const I8Launch& il,
                             double scale, float* s, long long s_ld, const CandBufs& cb, cudaStream_t st) {
  using L = I8Layout<D, MODE>;
  cudaError_t e = cudaFuncSetAttribute(score_i8_kernel<D, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM);
  if (e != cudaSuccess) return e;
  return launch_pdl(score_i8_kernel<D, MODE>, dim3(il.grid), dim3(L::THREADS), L::SMEM, st, ma, mb, sl.q_ex, sl.k_ex,
                    il.w, scale, s, s_ld, cb);
}

cudaError_t launch_scores_i8(const SliceOut& sl, int BH, int nqb, int nkb, int d, double scale,
                             float* s, long long s_ld, cudaStream_t st) {
  I8Launch il;
  cudaError_t e = i8_launch(BH, nqb, nkb, &il, false);
  if (e != cudaSuccess) return e;
  CUtensorMap ma, mb;
  const CandBufs none{};
  if (d == 128) {
    if ((e = i8_maps<128>(sl, BH, nqb, nkb, &ma, &mb)) != cudaSuccess) return e;
    return launch_i8<128, kScoreWrite>(ma, mb, sl, il, scale, s, s_ld, none, st);
  }
  if ((e = i8_maps<64>(sl, BH, nqb, nkb, &ma, &mb)) != cudaSuccess) return e;
  return launch_i8<64, kScoreWrite>(ma, mb, sl, il, scale, s, s_ld, none, st);
}

cudaError_t launch_select(const float* s, long long s_ld, int n_rows, int nkb, int k_sel,
                          double topp, int* kv_idx, int* kv_cnt, uint8_t* mask,
                          cudaStream_t st, const int* rows, const int* n_rows_dev) {
  // with a device-side row count the grid is a fixed size, strided over the rows
  const int cap8 = rows ? 148 * 8 : 65535 * 8;
  // rows of up to 40 blocks per lane: candidate path with the row in registers
  if (nkb <= 32 * 4) return launch_select_fast<4>(s, s_ld, n_rows, nkb, k_sel, topp, kv_idx, kv_cnt, mask, rows, n_rows_dev, cap8, st);
  if (nkb <= 32 * 16) return launch_select_fast<16>(s, s_ld, n_rows, nkb, k_sel, topp, kv_idx, kv_cnt, mask, rows, n_rows_dev, cap8, st);
  if (nkb <= 32 * 40) return launch_select_fast<40>(s, s_ld, n_rows, nkb, k_sel, topp, kv_idx, kv_cnt, mask, rows, n_rows_dev, cap8, st);
  // longer rows: candidate path with the row in shared memory
  const int slice = (nkb * 4 + kCandMax * 8 + 15) / 16 * 16;
  int wpc = (200 * 1024) / slice;
  wpc = wpc < 1 ? 1 : (wpc > 4 ? 4 : wpc);
  const size_t smem = static_cast<size_t>(slice) * wpc;
  cudaError_t e = cudaFuncSetAttribute(select_long_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int want = (n_rows + wpc - 1) / wpc;
  const int cap16 = rows ? 148 * 16 : 65535 * 16;
  const int grid = want < cap16 ? want : cap16;
  return launch_pdl(select_long_kernel, dim3(grid), dim3(wpc * 32), smem, st, s, s_ld, n_rows, nkb, k_sel, topp, kv_idx,
                    kv_cnt, mask, slice, rows, n_rows_dev);
}

// z with P(Z > z) = f for a standard normal Z (bisection on erfc, host fp64).
static double normal_upper_quantile(double f) {
  double lo = -40.0, hi = 40.0;
  for (int i = 0; i < 200; ++i) {
    const double mid = 0.5 * (lo + hi);
    if (0.5 * erfc(mid / sqrt(2.0)) > f) lo = mid;
    else hi = mid;
  }
  return 0.5 * (lo + hi);
}

CandPlan cand_plan(int k_sel, int nkb, long long s_ld) {
  // the lists share the score rows' memory: cand_row_bytes per row
  const long long per_row = cand_row_bytes(s_ld);
  long long store = per_row / 8 / 32 * 32;
  store = store > 2048 ? 2048 : store;
  int lim = 128;
  while (lim < 1024 && 2LL * lim <= store) lim *= 2;
  CandPlan p;
  p.want = k_sel + (k_sel / 2 > 32 ? k_sel / 2 : 32);
  p.cap = 128;
  while (p.cap < lim && p.cap < 1.6 * p.want) p.cap *= 2;
  p.all_cand = nkb <= p.cap ? 1 : 0;
  const long long half = store / 2 / 32 * 32;
  p.c_hi = static_cast<int>(2LL * p.cap < half ? 2LL * p.cap : (half > p.cap ? half : p.cap));
  p.c_lo = static_cast<int>(store - p.c_hi);
  auto quantile = [&](double count) -> float {
    double f = count / nkb;
    f = f < 1e-12 ? 1e-12 : (f > 1.0 - 1e-12 ? 1.0 - 1e-12 : f);
    return static_cast<float>(normal_upper_quantile(f));
  };
  p.zq = p.all_cand ? 0.f : quantile(p.want);
  p.zq_lo = p.all_cand ? 0.f : quantile(p.want + 0.9 * p.c_lo);
  return p;
}

template <int CPL>
static cudaError_t launch_select_cand(const CandSel& cs, int n_rows, int nkb, int k_sel, double topp,
                                      int* kv_idx, int* kv_cnt, uint8_t* mask, cudaStream_t st) {
  const int W = (nkb + 31) >> 5;
  const size_t smem = static_cast<size_t>(kCandSelWarps) * 2 * W * 4;
  cudaError_t e = cudaFuncSetAttribute(select_cand_kernel<CPL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int want = (n_rows + kCandSelWarps - 1) / kCandSelWarps;
  const int grid = want < 148 * 64 ? want : 148 * 64;
  return launch_pdl(select_cand_kernel<CPL>, dim3(grid), dim3(kCandSelWarps * 32), smem, st, cs, n_rows, nkb, k_sel,
                    topp, kv_idx, kv_cnt, mask);
}

// The candidate path of the mask builder: approximate row statistics,
// exact scores reduced to normaliser partials and candidate lists, the
// selection from the lists, and for the rows handed back the score-matrix
// path on their query tiles (two launches that return at once when no row
// was handed back).
template <int D>
static cudaError_t launch_mask_cand_d(const SliceOut& sl, int BH, int nqb, int nkb, double scale, int k_sel,
                                      double topp, float* s, long long s_ld, const CandWs& cw, int* kv_idx,
                                      int* kv_cnt, uint8_t* mask, cudaStream_t st) {
  I8Launch il;
  cudaError_t e = i8_launch(BH, nqb, nkb, &il, true);
  if (e != cudaSuccess) return e;
  CUtensorMap ma, mb;
  if ((e = i8_maps<D>(sl, BH, nqb, nkb, &ma, &mb)) != cudaSuccess) return e;
  const CandPlan plan = cand_plan(k_sel, nkb, s_ld);
  CandBufs cb{};
  cb.st1 = static_cast<float4*>(cw.st1);
  cb.st2 = static_cast<ZPart*>(cw.st2);
  cb.rowinfo = static_cast<float2*>(cw.rowinfo);
  cb.cand_cnt = cw.cand_cnt;
  cb.cand = reinterpret_cast<uint2*>(s);
  cb.c_hi = plan.c_hi;
  cb.c_lo = plan.c_lo;
  cb.zq = plan.zq;
  cb.zq_lo = plan.zq_lo;
  cb.p_lo = static_cast<float>(topp + 0.5 * (1.0 - topp));
  cb.zp = static_cast<float>(normal_upper_quantile(topp <= 1e-12 ? 1e-12 : (topp >= 1.0 - 1e-12 ? 1.0 - 1e-12 : topp)));
  cb.all_cand = plan.all_cand;
  cb.fb_cnt = cw.fb_cnt;
  cb.fb_rows = cw.fb_rows;
  cb.tile_flag = cw.tile_flag;
  cb.n_tile_flags = BH * il.w.n_qt;
  if ((e = launch_i8<D, kScoreStats>(ma, mb, sl, il, scale, nullptr, 0, cb, st)) != cudaSuccess) return e;
  if ((e = launch_i8<D, kScoreCands>(ma, mb, sl, il, scale, nullptr, 0, cb, st)) != cudaSuccess) return e;
  CandSel cs{cb.st2, cb.rowinfo, cb.cand_cnt, cb.cand, plan.c_hi, plan.c_lo, plan.cap, 4 * il.w.n_kr, nqb,
             il.w.n_qt, cb.fb_cnt, cb.fb_rows, cb.tile_flag};
  const int n_rows = BH * nqb;
  switch (plan.cap) {
    case 128: e = launch_select_cand<4>(cs, n_rows, nkb, k_sel, topp, kv_idx, kv_cnt, mask, st); break;
    case 256: e = launch_select_cand<8>(cs, n_rows, nkb, k_sel, topp, kv_idx, kv_cnt, mask, st); break;
    case 512: e = launch_select_cand<16>(cs, n_rows, nkb, k_sel, topp, kv_idx, kv_cnt, mask, st); break;
    default: e = launch_select_cand<32>(cs, n_rows, nkb, k_sel, topp, kv_idx, kv_cnt, mask, st); break;
  }
  if (e != cudaSuccess) return e;
  // rows handed back: their query tiles' score rows (in short key ranges, so
  // that a few flagged tiles spread over many CTAs), then the full-row
  // selection
  CandBufs fb{};
  fb.fb_cnt = cw.fb_cnt;
  fb.tile_flag = cw.tile_flag;
  I8Launch ilw;
  if ((e = i8_launch(BH, nqb, nkb, &ilw, false, 4)) != cudaSuccess) return e;
  if ((e = launch_i8<D, kScoreWrite>(ma, mb, sl, ilw, scale, s, s_ld, fb, st)) != cudaSuccess) return e;
  return launch_select(s, s_ld, n_rows, nkb, k_sel, topp, kv_idx, kv_cnt, mask, st, cw.fb_rows, cw.fb_cnt);
}

cudaError_t launch_mask_cand(const SliceOut& sl, int BH, int nqb, int nkb, int d, double scale, int k_sel,
                             double topp, float* s, long long s_ld, const CandWs& cw, int* kv_idx, int* kv_cnt,
                             uint8_t* mask, cudaStream_t st) {
  return d == 128 ? launch_mask_cand_d<128>(sl, BH, nqb, nkb, scale, k_sel, topp, s, s_ld, cw, kv_idx, kv_cnt, mask, st)
                  : launch_mask_cand_d<64>(sl, BH, nqb, nkb, scale, k_sel, topp, s, s_ld, cw, kv_idx, kv_cnt, mask, st);
}

cudaError_t launch_compact_mask(const uint8_t* mask, int n_rows, int nkb, int* kv_idx,
                                int* kv_cnt, cudaStream_t st) {
  const int grid = (n_rows + kSelWarpsMax - 1) / kSelWarpsMax;
  compact_mask_kernel<<<grid < 65535 * 16 ? grid : 65535 * 16, kSelWarpsMax * 32, 0, st>>>(mask, n_rows, nkb, kv_idx, kv_cnt);
  return cudaGetLastError();
}

}  // namespace sa
