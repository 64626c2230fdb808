// mask_kernels.cu — block pooling, block scores and the hybrid Top-k ∪ Top-p
// selection (pages: "SLA2" 提案手法 ① mean pooling of Q and K;
// "SpargeAttention2" §2(1) hybrid Top-k + Top-p masking per attention row).
//
//   pool_kernel      Q, K [BH, N, d] bf16 -> block means [BH, nb, d] fp32, and
//                    the same means as four signed 7-bit slices per element
//                    with a per-row power-of-two exponent
//   score_i8_kernel  slices -> s[bh, qb, kb] = scale * <Qbar, Kbar> on the
//                    int8 tensor cores (exact s32 slice products, combined in
//                    int64, scaled in fp64, rounded once to fp32)
//   select_*_kernel  one query-block row per warp: the K_sel-th largest score
//                    (Top-k) by a short count search followed by an exact
//                    search among at most 256 candidates, a probability-mass
//                    search for the Top-p cut when Top-k alone does not reach
//                    p, and the ascending compacted index list; the row sits
//                    in registers (up to 1280 key blocks) or shared memory.
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
// are dropped), combined exactly as the int64
//   v = acc2 2^21 + acc3 2^14 + acc4 2^7 + acc5,
// and the score is v * 2^(Eq + Ek - 35) * scale, rounded once in fp64 and
// once to fp32. Its error stays near 1e-7 of the score scale, well inside the
// 1e-6 band within which the mask comparison treats a cut as a tie.
//
// Persistent CTAs over work items (head, 128 query blocks, a range of 64-key
// tiles): warp 0 loads the item's query slices (operand A, M = 128) and
// streams the key-slice tiles (operand B, N = 64) through a 3-stage ring by
// TMA (128-byte swizzled rows, one box per 128-byte column chunk); warp 1
// issues the 10 * d / 32 MMAs of a key tile into one of two TMEM accumulator
// sets; eight epilogue warps (two per TMEM lane quadrant, 32 key columns
// each) combine the levels, transpose each 32 x 32 block through shared
// memory and write score rows with coalesced 128-byte stores.
constexpr int kI8TileM = 128;
constexpr int kI8TileN = 64;
constexpr int kI8BStages = 3;
constexpr int kI8EpiWarps = 8;
constexpr int kI8Threads = 32 * (2 + kI8EpiWarps);

template <int D>
struct I8Layout {
  static constexpr int ROW = 4 * D;                 // bytes per slice row
  static constexpr int NCH = ROW / 128;             // 128-byte column chunks
  static constexpr uint32_t A_CH = kI8TileM * 128;  // bytes of one A chunk
  static constexpr uint32_t B_CH = kI8TileN * 128;
  static constexpr uint32_t A_BYTES = NCH * A_CH;
  static constexpr uint32_t B_BYTES = NCH * B_CH;
  static constexpr uint32_t OFF_A = 0;
  static constexpr uint32_t OFF_B = OFF_A + A_BYTES;
  static constexpr uint32_t OFF_T = OFF_B + kI8BStages * B_BYTES;      // [epi warps][32][33] fp32
  static constexpr uint32_t OFF_BAR = OFF_T + kI8EpiWarps * 32 * 33 * 4;
  static constexpr uint32_t SMEM = OFF_BAR + 128 + 1024;
};

struct I8Work {
  int nqb, nkb, n_qt, n_kt, kr_tiles, n_kr, n_items;
};

template <int D>
__global__ void __launch_bounds__(kI8Threads, 1) score_i8_kernel(const __grid_constant__ CUtensorMap tmA,
                                                                 const __grid_constant__ CUtensorMap tmB,
                                                                 const int* __restrict__ q_ex,
                                                                 const int* __restrict__ k_ex, I8Work wk,
                                                                 double scale, float* __restrict__ s,
                                                                 long long s_ld) {
  using L = I8Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* a_full = bars;                        // item's query slices landed
  uint64_t* a_empty = bars + 1;                   // item's last MMA completed
  uint64_t* b_full = bars + 2;                    // [kI8BStages]
  uint64_t* b_empty = b_full + kI8BStages;        // [kI8BStages]
  uint64_t* acc_full = b_empty + kI8BStages;      // [2]
  uint64_t* acc_empty = acc_full + 2;             // [2] (epilogue warps)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr uint32_t kSet = 4 * kI8TileN;         // columns of one accumulator set (four levels)

  if (threadIdx.x == 0) {
    mbar_init(a_full, 1);
    mbar_init(a_empty, 1);
    for (int i = 0; i < kI8BStages; ++i) {
      mbar_init(&b_full[i], 1);
      mbar_init(&b_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], kI8EpiWarps);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 2 * kSet);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *tmem_slot;

  // work item -> (head, query tile, first and end key tile)
  auto decode = [&](int item, int& bh, int& qt, int& kt0, int& kt1) {
    const int kr = item % wk.n_kr;
    const int rest = item / wk.n_kr;
    qt = rest % wk.n_qt;
    bh = rest / wk.n_qt;
    kt0 = kr * wk.kr_tiles;
    kt1 = min(wk.n_kt, kt0 + wk.kr_tiles);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      int ic = 0, bt = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < wk.n_items; item += gridDim.x, ++ic) {
        int bh, qt, kt0, kt1;
        decode(item, bh, qt, kt0, kt1);
        if (!(ok = mbar_wait(a_empty, (ic & 1) ^ 1, abort_flag))) break;
        mbar_arrive_expect_tx(a_full, L::A_BYTES);
#pragma unroll
        for (int c = 0; c < L::NCH; ++c)
          tma_load_3d(smem + L::OFF_A + c * L::A_CH, &tmA, a_full, c * 128, qt * kI8TileM, bh);
        for (int kt = kt0; kt < kt1; ++kt, ++bt) {
          const int st = bt % kI8BStages;
          if (!(ok = mbar_wait(&b_empty[st], ((bt / kI8BStages) & 1) ^ 1, abort_flag))) break;
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
      int ic = 0, bt = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < wk.n_items; item += gridDim.x, ++ic) {
        int bh, qt, kt0, kt1;
        decode(item, bh, qt, kt0, kt1);
        if (!(ok = mbar_wait(a_full, ic & 1, abort_flag))) break;
        for (int kt = kt0; kt < kt1; ++kt, ++bt) {
          const int st = bt % kI8BStages, ab = bt & 1;
          if (!(ok = mbar_wait(&b_full[st], (bt / kI8BStages) & 1, abort_flag))) break;
          if (!(ok = mbar_wait(&acc_empty[ab], ((bt >> 1) & 1) ^ 1, abort_flag))) break;
          tc_fence_after();
          const uint64_t b0 = b00 + ((st * L::B_BYTES) >> 4);
          const uint32_t acc = tm + ab * kSet;
#pragma unroll
          for (int sa = 1; sa <= 4; ++sa)
#pragma unroll
            for (int tb = 1; sa + tb <= 5; ++tb)
#pragma unroll
              for (int j = 0; j < D / 32; ++j)
                umma_i8_ss(acc + (sa + tb - 2) * kI8TileN, a0 + off(D * (sa - 1) + 32 * j, L::A_CH),
                           b0 + off(D * (tb - 1) + 32 * j, L::B_CH), idesc, (sa == 1 && j == 0) ? 0u : 1u);
          tc_commit(&b_empty[st]);
          tc_commit(&acc_full[ab]);
        }
        if (ok) tc_commit(a_empty);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;                       // 0..7
    const int quad = warp & 3;                     // TMEM lane quadrant
    const int hc = ew >> 2;                        // key columns [32 hc, 32 hc + 32) of the tile
    const uint32_t la = tm + (static_cast<uint32_t>(quad * 32) << 16) + hc * 32;
    float* tbuf = reinterpret_cast<float*>(smem + L::OFF_T) + ew * 32 * 33;
    int bt = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < wk.n_items; item += gridDim.x) {
      int bh, qt, kt0, kt1;
      decode(item, bh, qt, kt0, kt1);
      const int row0 = qt * kI8TileM + quad * 32;  // first query block of this warp's rows
      const int row = row0 + lane;
      const int eq = row < wk.nqb ? __ldg(q_ex + static_cast<long long>(bh) * wk.nqb + row) : 0;
      for (int kt = kt0; kt < kt1; ++kt, ++bt) {
        const int ab = bt & 1;
        const int kcol = kt * kI8TileN + hc * 32 + lane;   // this lane's key in the store phase
        const int ek_l = kcol < wk.nkb ? __ldg(k_ex + static_cast<long long>(bh) * wk.nkb + kcol) : 0;
        if (!(ok = mbar_wait(&acc_full[ab], (bt >> 1) & 1, abort_flag))) break;
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
        // v = hi 2^14 + lo with hi = acc2 2^7 + acc3 and lo = acc4 2^7 + acc5,
        // both exact in int32 (|acc2| <= d 127^2 < 2^22, |acc3| < 2^23, ...);
        // v is then exact in one fp64 fma. The row's factor scale 2^(Eq - 35)
        // rounds once, and 2^Ek is added to the result's exponent, which is
        // exact for the score range.
        const double crow = scale * __longlong_as_double(static_cast<long long>(eq - 35 + 1023) << 52);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int hi = (static_cast<int>(a2[i]) << 7) + static_cast<int>(a3[i]);
          const int lo = (static_cast<int>(a4[i]) << 7) + static_cast<int>(a5[i]);
          const double vd = fma(static_cast<double>(hi), 16384.0, static_cast<double>(lo));
          const double r = vd * crow;
          const int ek = __shfl_sync(0xFFFFFFFFu, ek_l, i);
          const double sc = r == 0.0 ? 0.0
                                     : __hiloint2double(__double2hiint(r) + (ek << 20), __double2loint(r));
          tbuf[lane * 33 + i] = __double2float_rn(sc);
        }
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
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tm, 2 * kSet);
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

template <int KPL>
__global__ void __launch_bounds__(kSelFastWarps * 32, 4) select_fast_kernel(
    const float* __restrict__ s, long long s_ld, int n_rows, int nkb, int k_sel, double topp,
    int* __restrict__ kv_idx, int* __restrict__ kv_cnt, uint8_t* __restrict__ mask) {
  __shared__ uint32_t ckey_all[kSelFastWarps][kRegCandMax];
  __shared__ int cidx_all[kSelFastWarps][kRegCandMax];
  __shared__ float e_all[kSelFastWarps][32 * KPL];
  const int warp = threadIdx.x >> 5;
  for (int row = blockIdx.x * kSelFastWarps + warp; row < n_rows; row += gridDim.x * kSelFastWarps) {
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
                                      cudaStream_t st) {
  const int want = (n_rows + kSelFastWarps - 1) / kSelFastWarps;
  const int grid = want < 65535 * 8 ? want : 65535 * 8;
  select_fast_kernel<KPL><<<grid, kSelFastWarps * 32, 0, st>>>(s, s_ld, n_rows, nkb, k_sel, topp, kv_idx, kv_cnt, mask);
  return cudaGetLastError();
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
    int* __restrict__ kv_idx, int* __restrict__ kv_cnt, uint8_t* __restrict__ mask, int slice) {
  extern __shared__ __align__(16) uint8_t sm_long[];
  const int warp = threadIdx.x >> 5;
  const int wpc = blockDim.x >> 5;
  float* xs = reinterpret_cast<float*>(sm_long + static_cast<size_t>(warp) * slice);
  uint32_t* ckey = reinterpret_cast<uint32_t*>(xs + nkb);
  int* cidx = reinterpret_cast<int*>(ckey + kCandMax);
  for (int row = blockIdx.x * wpc + warp; row < n_rows; row += gridDim.x * wpc) {
    select_row_long(s + static_cast<long long>(row) * s_ld, nkb, k_sel, topp,
                    kv_idx + static_cast<long long>(row) * nkb, kv_cnt + row,
                    mask ? mask + static_cast<long long>(row) * nkb : nullptr, xs, ckey, cidx);
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

template <int D>
static cudaError_t launch_scores_i8_d(const SliceOut& sl, int BH, int nqb, int nkb, double scale,
                                      float* s, long long s_ld, cudaStream_t st) {
  using L = I8Layout<D>;
  CUtensorMap ma, mb;
  if (encode_tensor_map_3d_u8(&ma, sl.q_sl, L::ROW, nqb, BH, 128, kI8TileM) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  if (encode_tensor_map_3d_u8(&mb, sl.k_sl, L::ROW, nkb, BH, 128, kI8TileN) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(score_i8_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  I8Work w;
  w.nqb = nqb;
  w.nkb = nkb;
  w.n_qt = ceil_div(nqb, kI8TileM);
  w.n_kt = ceil_div(nkb, kI8TileN);
  // about four items per SM: key tiles per item from the total tile count
  const long long tiles = static_cast<long long>(BH) * w.n_qt * w.n_kt;
  long long per = (tiles + 4LL * sms - 1) / (4LL * sms);
  per = per < 1 ? 1 : (per > w.n_kt ? w.n_kt : per);
  w.kr_tiles = static_cast<int>(per);
  w.n_kr = ceil_div(w.n_kt, w.kr_tiles);
  const long long items = static_cast<long long>(BH) * w.n_qt * w.n_kr;
  if (items > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  w.n_items = static_cast<int>(items);
  const int grid = w.n_items < sms ? w.n_items : sms;
  score_i8_kernel<D><<<grid, kI8Threads, L::SMEM, st>>>(ma, mb, sl.q_ex, sl.k_ex, w, scale, s, s_ld);
  return cudaGetLastError();
}

cudaError_t launch_scores_i8(const SliceOut& sl, int BH, int nqb, int nkb, int d, double scale,
                             float* s, long long s_ld, cudaStream_t st) {
  return d == 128 ? launch_scores_i8_d<128>(sl, BH, nqb, nkb, scale, s, s_ld, st)
                  : launch_scores_i8_d<64>(sl, BH, nqb, nkb, scale, s, s_ld, st);
}

cudaError_t launch_select(const float* s, long long s_ld, int n_rows, int nkb, int k_sel,
                          double topp, int* kv_idx, int* kv_cnt, uint8_t* mask,
                          cudaStream_t st) {
  // rows of up to 40 blocks per lane: candidate path with the row in registers
  if (nkb <= 32 * 4) return launch_select_fast<4>(s, s_ld, n_rows, nkb, k_sel, topp, kv_idx, kv_cnt, mask, st);
  if (nkb <= 32 * 16) return launch_select_fast<16>(s, s_ld, n_rows, nkb, k_sel, topp, kv_idx, kv_cnt, mask, st);
  if (nkb <= 32 * 40) return launch_select_fast<40>(s, s_ld, n_rows, nkb, k_sel, topp, kv_idx, kv_cnt, mask, st);
  // longer rows: candidate path with the row in shared memory
  const int slice = (nkb * 4 + kCandMax * 8 + 15) / 16 * 16;
  int wpc = (200 * 1024) / slice;
  wpc = wpc < 1 ? 1 : (wpc > 4 ? 4 : wpc);
  const size_t smem = static_cast<size_t>(slice) * wpc;
  cudaError_t e = cudaFuncSetAttribute(select_long_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int want = (n_rows + wpc - 1) / wpc;
  const int grid = want < 65535 * 16 ? want : 65535 * 16;
  select_long_kernel<<<grid, wpc * 32, smem, st>>>(s, s_ld, n_rows, nkb, k_sel, topp, kv_idx, kv_cnt, mask, slice);
  return cudaGetLastError();
}

cudaError_t launch_compact_mask(const uint8_t* mask, int n_rows, int nkb, int* kv_idx,
                                int* kv_cnt, cudaStream_t st) {
  const int grid = (n_rows + kSelWarpsMax - 1) / kSelWarpsMax;
  compact_mask_kernel<<<grid < 65535 * 16 ? grid : 65535 * 16, kSelWarpsMax * 32, 0, st>>>(mask, n_rows, nkb, kv_idx, kv_cnt);
  return cudaGetLastError();
}

}  // namespace sa
