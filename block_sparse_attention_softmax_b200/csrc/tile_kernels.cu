// tile_kernels.cu — tile descriptors and the reference tile heatmap (page:
// "Veda" §2.1, TripPool descriptors and a reference mask that max-pools the full
// attention map over query-key tiles; §2.3, a two-pass heatmap).
//
// trip_pool_kernel  one warp per block of b tokens: per channel the mean, the
//                   maximum and the minimum over the block's valid tokens,
//                   written as [mean | max | min] (fp32).
// heat_kernel       per work item (head, 128-row query tile, from an optional
//                   list of rows) two sweeps over every key tile:
//                     1. S = Q K^T on the tensor core; each softmax thread keeps
//                        an online max and sum of 2^(S * scale * log2 e) over
//                        its 64 columns; the two halves of a row combine once per
//                        item into the row's log-sum-exp;
//                     2. S again; per 64-key block the row's max of
//                        S * scale - LSE (the log of the largest full-attention
//                        probability), reduced over the block's rows with
//                        atomics on the heatmap word of (row, key block).
//                   Roles: warp 0 TMA producer (Q, 3-stage K ring), warp 1
//                   TMEM allocation and the MMA thread, warps 2..9 two per TMEM
//                   lane quadrant, 64 columns each. Every wait is bounded; the
//                   only cross-warp exchange (once per item) meets at an
//                   mbarrier, so a warp that stops never leaves its partner at a
//                   barrier without a bound.
#include "sa_internal.h"

namespace sa {

// ---------------------------------------------------------------- TripPool
template <int D>
__global__ void __launch_bounds__(256) trip_pool_kernel(const __nv_bfloat16* __restrict__ x, int N, int b,
                                                        int n_blocks, long long total, float* __restrict__ out) {
  // 8 warps per CTA, one block of b tokens per warp; lane l holds channels
  // [8 l', 8 l' + 8) of token rows of parity l / (D / 8)
  constexpr int LPR = D / 8;              // lanes per token row (16 B each)
  constexpr int RPI = 32 / LPR;           // token rows per warp iteration
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long gb = static_cast<long long>(blockIdx.x) * 8 + warp;   // (head, block) index
  if (gb >= total) return;
  const long long bh = gb / n_blocks;
  const int blk = static_cast<int>(gb % n_blocks);
  const int t0 = blk * b, t1 = min(N, t0 + b);
  const int c8 = (lane % LPR) * 8;
  const int r0 = lane / LPR;
  float sum[8], mx[8], mn[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    sum[j] = 0.f;
    mx[j] = -INFINITY;
    mn[j] = INFINITY;
  }
  const __nv_bfloat16* base = x + (bh * N) * D;
  for (int t = t0 + r0; t < t1; t += RPI) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(base + static_cast<long long>(t) * D + c8));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float v = __uint_as_float((j & 1) ? (w[j >> 1] & 0xFFFF0000u) : (w[j >> 1] << 16));
      sum[j] += v;
      mx[j] = fmaxf(mx[j], v);
      mn[j] = fminf(mn[j], v);
    }
  }
  // combine the RPI row groups (lanes with the same channels)
#pragma unroll
  for (int off = LPR; off < 32; off <<= 1) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      sum[j] += __shfl_xor_sync(0xFFFFFFFFu, sum[j], off);
      mx[j] = fmaxf(mx[j], __shfl_xor_sync(0xFFFFFFFFu, mx[j], off));
      mn[j] = fminf(mn[j], __shfl_xor_sync(0xFFFFFFFFu, mn[j], off));
    }
  }
  if (r0 == 0) {
    const float inv = 1.f / static_cast<float>(t1 - t0);
    float* o = out + gb * (3 * D);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      o[c8 + j] = sum[j] * inv;
      o[D + c8 + j] = mx[j];
      o[2 * D + c8 + j] = mn[j];
    }
  }
}

cudaError_t launch_trip_pool(const void* x, int BH, int N, int d, int b, float* out, cudaStream_t st) {
  const int n_blocks = (N + b - 1) / b;
  const long long total = static_cast<long long>(BH) * n_blocks;
  const long long grid = (total + 7) / 8;
  if (grid > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  if (d == 128)
    trip_pool_kernel<128><<<static_cast<int>(grid), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(x), N, b, n_blocks, total, out);
  else
    trip_pool_kernel<64><<<static_cast<int>(grid), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(x), N, b, n_blocks, total, out);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- heatmap
namespace heat {

constexpr int kBM = 128;
constexpr int kBN = 128;
constexpr int kKStages = 3;
constexpr int kSBufs = 2;
constexpr int kSoftWarps = 8;
constexpr int kThreads = 32 * (2 + kSoftWarps);

template <int D>
struct Layout {
  static constexpr int NCH = D / 64;
  static constexpr uint32_t Q_BYTES = kBM * D * 2;
  static constexpr uint32_t TILE_BYTES = kBN * D * 2;
  static constexpr uint32_t BLK_BYTES = 64 * D * 2;
  static constexpr uint32_t Q_CHUNK = kBM * 128;
  static constexpr uint32_t KV_CHUNK = kBN * 128;
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = OFF_Q + Q_BYTES;
  static constexpr uint32_t OFF_X = OFF_K + kKStages * TILE_BYTES;   // [2 item parities][2 halves][128 rows] float2
  static constexpr uint32_t OFF_BAR = OFF_X + 2 * 2 * kBM * 8;
  static constexpr uint32_t USED = OFF_BAR + 256;
  static constexpr uint32_t SMEM = USED + 1024;
};

enum {
  B_QFULL = 0,
  B_QEMPTY = 1,
  B_KFULL = 2,                        // [kKStages]
  B_KEMPTY = B_KFULL + kKStages,      // [kKStages]
  B_SFULL = B_KEMPTY + kKStages,      // [kSBufs]
  B_SEMPTY = B_SFULL + kSBufs,        // [kSBufs] every softmax warp has read the buffer
  B_XCH = B_SEMPTY + kSBufs,          // [4 quadrants] both warps posted their half's (max, sum)
  B_DRAIN = B_XCH + 4,
  B_COUNT = B_DRAIN + 1
};

}  // namespace heat

struct HeatArgs {
  const void* q;
  const void* k;
  const int* rows;       // query-block rows (bh * nqb + qb) to evaluate, or null for all
  int n_items;
  int BH, N, bq, nqb, nkb;
  float scale_log2;
  float* heat;           // [BH * nqb, nkb] natural-log heat, rows pre-filled with -inf
  float* lse;            // [BH, N] or null: natural-log LSE of the evaluated rows
};

// Heat words hold floats <= -0; for those the float order is the reverse of
// the signed-int order of their bit patterns (and -inf is the largest int), so
// atomicMin on the bits takes the float maximum.
__device__ __forceinline__ void heat_max(float* w, float v) {
  atomicMin(reinterpret_cast<int*>(w), __float_as_int(fminf(v, -0.f)));
}

template <int D>
__global__ void __launch_bounds__(heat::kThreads, 1)
    heat_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK, HeatArgs a) {
  using namespace heat;
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + L::OFF_Q;
  uint8_t* sK = smem + L::OFF_K;
  float2* xch = reinterpret_cast<float2*>(smem + L::OFF_X);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  static_assert(B_COUNT * 8 + 8 <= 256, "barrier region");
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + B_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = (a.nkb + 1) >> 1;     // key tiles per sweep

  if (threadIdx.x == 0) {
    mbar_init(&bars[B_QFULL], 1);
    mbar_init(&bars[B_QEMPTY], 1);
    for (int i = 0; i < kKStages; ++i) {
      mbar_init(&bars[B_KFULL + i], 1);
      mbar_init(&bars[B_KEMPTY + i], 1);
    }
    for (int i = 0; i < kSBufs; ++i) {
      mbar_init(&bars[B_SFULL + i], 1);
      mbar_init(&bars[B_SEMPTY + i], kSoftWarps);
    }
    for (int i = 0; i < 4; ++i) mbar_init(&bars[B_XCH + i], 2);
    mbar_init(&bars[B_DRAIN], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      int g = 0, ii = 0, q_issued = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < a.n_items; item += gridDim.x, ++ii) {
        const int row = a.rows ? a.rows[item] : item;
        const int bh = row / a.nqb, qb = row % a.nqb;
        if (!(ok = mbar_wait(&bars[B_QEMPTY], (ii & 1) ^ 1, abort_flag))) break;
        mbar_arrive_expect_tx(&bars[B_QFULL], L::Q_BYTES);
#pragma unroll
        for (int c = 0; c < L::NCH; ++c)
          tma_load_3d(sQ + c * L::Q_CHUNK, &tmQ, &bars[B_QFULL], c * 64, qb * a.bq, bh);
        ++q_issued;
        for (int j = 0; ok && j < 2 * T; ++j, ++g) {
          const int t = j % T;
          const int s = g % kKStages;
          const int nblk = min(2, a.nkb - 2 * t);
          if (!(ok = mbar_wait(&bars[B_KEMPTY + s], ((g / kKStages) & 1) ^ 1, abort_flag))) break;
          mbar_arrive_expect_tx(&bars[B_KFULL + s], nblk * L::BLK_BYTES);
          uint8_t* dst = sK + s * L::TILE_BYTES;
#pragma unroll
          for (int c = 0; c < L::NCH; ++c) {
            tma_load_3d(dst + c * L::KV_CHUNK, &tmK, &bars[B_KFULL + s], c * 64, (2 * t) * 64, bh);
            if (nblk > 1) tma_load_3d(dst + c * L::KV_CHUNK + 64 * 128, &tmK, &bars[B_KFULL + s], c * 64, (2 * t + 1) * 64, bh);
          }
        }
      }
      // loads in flight land before the CTA gives up its shared memory
      for (int i = 1; i <= kKStages && i <= g; ++i)
        mbar_drain(&bars[B_KFULL + (g - i) % kKStages], ((g - i) / kKStages) & 1);
      if (q_issued > 0) mbar_drain(&bars[B_QFULL], (q_issued - 1) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA thread
    if (lane == 0) {
      const uint64_t qdesc = sw128_desc(smem_u32(sQ), 16, 1024);
      const uint64_t kdesc0 = sw128_desc(smem_u32(sK), 16, 1024);
      const uint32_t idesc2 = idesc_bf16_f32(kBM, 128, false, false);
      const uint32_t idesc1 = idesc_bf16_f32(kBM, 64, false, false);
      int g = 0, ii = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < a.n_items; item += gridDim.x, ++ii) {
        if (!(ok = mbar_wait(&bars[B_QFULL], ii & 1, abort_flag))) break;
        for (int j = 0; ok && j < 2 * T; ++j, ++g) {
          const int t = j % T;
          const int s = g % kKStages, sb = g % kSBufs;
          if (!(ok = mbar_wait(&bars[B_KFULL + s], (g / kKStages) & 1, abort_flag))) break;
          if (!(ok = mbar_wait(&bars[B_SEMPTY + sb], ((g / kSBufs) & 1) ^ 1, abort_flag))) break;
          tc_fence_after();
          const uint32_t idesc = (a.nkb - 2 * t) >= 2 ? idesc2 : idesc1;
          const uint64_t kd = kdesc0 + ((s * L::TILE_BYTES) >> 4);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            umma_ss(tm + sb * 128, qdesc + ((((kk >> 2) * L::Q_CHUNK) + (kk & 3) * 32u) >> 4),
                    kd + ((((kk >> 2) * L::KV_CHUNK) + (kk & 3) * 32u) >> 4), idesc, kk > 0 ? 1u : 0u);
          tc_commit(&bars[B_SFULL + sb]);
          tc_commit(&bars[B_KEMPTY + s]);
          if (j == 2 * T - 1) tc_commit(&bars[B_QEMPTY]);
        }
      }
      tc_commit(&bars[B_DRAIN]);
      mbar_drain(&bars[B_DRAIN], 0);
    }
  } else {
    // ------------------------------------------------------------ row statistics and tile maxima
    const int sw = warp - 2;
    const int quad = warp & 3;
    const int half = sw >> 2;                 // which 64-key block of each tile
    const int row = quad * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    const float sl2 = a.scale_log2;
    const int tail_valid = a.N - (a.nkb - 1) * 64;
    int g = 0, ii = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < a.n_items; item += gridDim.x, ++ii) {
      const int qrow = a.rows ? a.rows[item] : item;
      const int bh = qrow / a.nqb, qb = qrow % a.nqb;
      const int grow = qb * a.bq + row;
      const bool valid_row = row < a.bq && grow < a.N;
      float m = -INFINITY, l = 0.f;          // this half's running max (log2 units) and sum
      float lse2 = 0.f;
      for (int j = 0; ok && j < 2 * T; ++j, ++g) {
        const int t = j % T;
        const int sb = g % kSBufs;
        if (!(ok = mbar_wait(&bars[B_SFULL + sb], (g / kSBufs) & 1, abort_flag))) break;
        tc_fence_after();
        uint32_t r0[32], r1[32];
        tmem_ld32(tm + lane_addr + sb * 128 + half * 64, r0);
        tmem_ld32(tm + lane_addr + sb * 128 + half * 64 + 32, r1);
        tmem_wait_ld();
        reg_fence(r0);
        reg_fence(r1);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[B_SEMPTY + sb]);
        const int kb = 2 * t + half;
        int valid = kb < a.nkb ? 64 : 0;
        if (kb == a.nkb - 1) valid = tail_valid;
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          if (c < valid) mx = fmaxf(mx, __uint_as_float(r0[c]));
          if (32 + c < valid) mx = fmaxf(mx, __uint_as_float(r1[c]));
        }
        if (j < T) {
          // sweep 1: online log-sum-exp over this half's columns (log2 units)
          if (valid > 0) {
            const float mt = mx * sl2;
            if (mt > m) {
              l *= fast_exp2(m - mt);
              m = mt;
            }
            float acc = 0.f;
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              if (c < valid) acc += fast_exp2(fmaf(__uint_as_float(r0[c]), sl2, -m));
              if (32 + c < valid) acc += fast_exp2(fmaf(__uint_as_float(r1[c]), sl2, -m));
            }
            l += acc;
          }
          if (j == T - 1) {
            // both halves of each row: combine into the row's log-sum-exp
            float2* xp = xch + (ii & 1) * 2 * kBM;
            xp[half * kBM + row] = make_float2(m, l);
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_XCH + quad]);
            if (!(ok = mbar_wait(&bars[B_XCH + quad], ii & 1, abort_flag))) break;
            const float2 o = xp[(half ^ 1) * kBM + row];
            const float mm = fmaxf(m, o.x);
            lse2 = mm + log2f(l * fast_exp2(m - mm) + o.y * fast_exp2(o.x - mm));
            if (a.lse && valid_row && half == 0)
              a.lse[static_cast<long long>(bh) * a.N + grow] = lse2 * 0.69314718055994531f;
          }
        } else if (kb < a.nkb) {
          // sweep 2: the block's largest log probability over its rows
          float v = valid_row ? (mx * sl2 - lse2) * 0.69314718055994531f : -INFINITY;
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, off));
          if (lane == 0 && v > -INFINITY) heat_max(a.heat + static_cast<long long>(qrow) * a.nkb + kb, v);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tm, 256);
  }
}

__global__ void fill_rows_kernel(float* __restrict__ heat, const int* __restrict__ rows, int n_items, int nkb,
                                 float value) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= static_cast<long long>(n_items) * nkb) return;
  const int it = static_cast<int>(i / nkb), kb = static_cast<int>(i % nkb);
  const long long row = rows ? rows[it] : it;
  heat[row * nkb + kb] = value;
}

cudaError_t launch_heat(const void* q, const void* k, int BH, int N, int d, int bq, const int* rows, int n_items,
                        double scale, float* heat, float* lse, cudaStream_t st) {
  const int nqb = (N + bq - 1) / bq, nkb = (N + 63) / 64;
  if (n_items <= 0) return cudaSuccess;
  const long long fills = static_cast<long long>(n_items) * nkb;
  fill_rows_kernel<<<static_cast<int>((fills + 255) / 256), 256, 0, st>>>(heat, rows, n_items, nkb, -INFINITY);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  CUtensorMap mq, mk;
  if (encode_tensor_map_3d_bf16(&mq, q, d, N, BH, 64, heat::kBM) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  if (encode_tensor_map_3d_bf16(&mk, k, d, N, BH, 64, 64) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  HeatArgs a{q, k, rows, n_items, BH, N, bq, nqb, nkb, static_cast<float>(scale * 1.4426950408889634), heat, lse};
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = n_items < sms ? n_items : sms;
  if (d == 128) {
    e = cudaFuncSetAttribute(heat_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, heat::Layout<128>::SMEM);
    if (e != cudaSuccess) return e;
    heat_kernel<128><<<grid, heat::kThreads, heat::Layout<128>::SMEM, st>>>(mq, mk, a);
  } else {
    e = cudaFuncSetAttribute(heat_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, heat::Layout<64>::SMEM);
    if (e != cudaSuccess) return e;
    heat_kernel<64><<<grid, heat::kThreads, heat::Layout<64>::SMEM, st>>>(mq, mk, a);
  }
  return cudaGetLastError();
}

}  // namespace sa
