// bwd_kernels.cu — backward pass of the block-sparse attention (pages:
// "SpargeAttention2" §2(2), the sparse attention is trainable and fine-tuned by
// distillation; "SLA2" 提案手法 ③, the backward pass runs in full precision).
//
// With P the row softmax of S = scale Q K^T over the kept tiles, O = P V, and
// the upstream gradient dO:
//   D_i = sum_c dO_ic O_ic                        (bwd_delta_kernel)
//   dS  = P * (dO V^T - D)                        (elementwise, per tile)
//   dQ  = scale dS K,  dK = scale dS^T Q,  dV = P^T dO
// P is recomputed from the forward's log-sum-exp, so no exchange between warps
// is needed and every sum is owned by one CTA (deterministic, no atomics).
//
// bwd_dq_kernel    per query block (the forward's items and lists): for each
//                  kept tile of two key blocks, S = Q K^T and dP = dO V^T on the
//                  tensor core into TMEM; 8 warps form dS (bf16, written over S);
//                  dQ += dS K accumulates in TMEM. S has two buffers, so S and
//                  dP of the next tile are computed while the warps form dS.
// bwd_dkdv_kernel  per tile of two key blocks: the query blocks that keep
//                  either block (a transposed list with a flag per block, from
//                  col_lists_kernel), for each S^T = K Q^T and dP^T = V dO^T;
//                  8 warps form P^T and dS^T (rows of the block that does not
//                  keep this query block are zero) over the dP^T columns they
//                  came from, so the next block's S^T lands while they work;
//                  dV += P^T dO and dK += dS^T Q accumulate in TMEM.
// Roles in both: warp 0 TMA producer, warp 1 TMEM allocation and the MMA
// thread, then (dK/dV only) a warp staging the query blocks' LSE and D in
// shared memory, and 8 warps, two per TMEM lane quadrant, 64 columns each.
// Every wait is bounded; early exits wait for loads and MMAs in flight.
#include "sa_internal.h"

namespace sa {

// ---------------------------------------------------------------- D = rowsum(dO * O)
template <int D>
__global__ void __launch_bounds__(256) bwd_delta_kernel(const __nv_bfloat16* __restrict__ o,
                                                        const __nv_bfloat16* __restrict__ dout, long long rows,
                                                        float* __restrict__ delta) {
  constexpr int LPR = D / 8, RPW = 32 / LPR;
  const long long warp = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long long r = warp * RPW + lane / LPR;
  float acc = 0.f;
  if (r < rows) {
    const int c8 = (lane % LPR) * 8;
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(o + r * D + c8));
    const uint4 b = __ldg(reinterpret_cast<const uint4*>(dout + r * D + c8));
    const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      acc = fmaf(__uint_as_float(wa[j] << 16), __uint_as_float(wb[j] << 16), acc);
      acc = fmaf(__uint_as_float(wa[j] & 0xFFFF0000u), __uint_as_float(wb[j] & 0xFFFF0000u), acc);
    }
  }
#pragma unroll
  for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, off);
  if (r < rows && lane % LPR == 0) delta[r] = acc;
}

// ---------------------------------------------------------------- transposed lists
// Dense mask from the lists (the mask was cleared first).
__global__ void lists_to_mask_kernel(const int* __restrict__ kv_idx, const int* __restrict__ kv_cnt, long long rows,
                                     int nkb, uint8_t* __restrict__ mask) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= rows * nkb) return;
  const long long r = i / nkb;
  const int j = static_cast<int>(i % nkb);
  const int cnt = min(max(__ldg(kv_cnt + r), 0), nkb);
  if (j >= cnt) return;
  const int kb = __ldg(kv_idx + i);
  if (kb >= 0 && kb < nkb) mask[r * nkb + kb] = 1;
}

// For each tile of two key blocks (2 kt, 2 kt + 1): the query blocks that keep
// either, ascending, as qb | flags << 24 (bit 0: block 2 kt kept, bit 1: 2 kt + 1).
__global__ void col_lists_kernel(const uint8_t* __restrict__ mask, int BH, int nqb, int nkb, int nkt,
                                 int* __restrict__ qt_idx, int* __restrict__ qt_cnt) {
  const long long w = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= static_cast<long long>(BH) * nkt) return;
  const int bh = static_cast<int>(w / nkt), kt = static_cast<int>(w % nkt);
  const int k0 = 2 * kt, k1 = 2 * kt + 1;
  int* out = qt_idx + w * nqb;
  int n = 0;
  for (int base = 0; base < nqb; base += 32) {
    const int qb = base + lane;
    int f = 0;
    if (qb < nqb) {
      const uint8_t* mr = mask + (static_cast<long long>(bh) * nqb + qb) * nkb;
      f = (mr[k0] ? 1 : 0) | ((k1 < nkb && mr[k1]) ? 2 : 0);
    }
    const uint32_t bal = __ballot_sync(0xFFFFFFFFu, f != 0);
    if (f) out[n + __popc(bal & ((1u << lane) - 1u))] = qb | (f << 24);
    n += __popc(bal);
  }
  if (lane == 0) qt_cnt[w] = n;
}

namespace bwd {

constexpr int kBM = 128;
constexpr int kBN = 128;
constexpr int kStages = 2;
constexpr int kCWarps = 8;

template <int D>
struct Sizes {
  static constexpr int NCH = D / 64;
  static constexpr uint32_t ROWS_BYTES = 128 * D * 2;    // 128 rows of Q, dO, K or V
  static constexpr uint32_t BLK_BYTES = 64 * D * 2;
  static constexpr uint32_t CHUNK = 128 * 128;           // bytes per d-chunk of 128 rows
};

}  // namespace bwd

struct BwdArgs {
  const void* q;
  const void* k;
  const void* v;
  const void* dout;
  const float* lse;       // [BH, N] natural log
  const float* delta;     // [BH, N]
  const int* kv_idx;      // dQ: the forward's lists
  const int* kv_cnt;
  const int* qt_idx;      // dK/dV: transposed lists
  const int* qt_cnt;
  float* dq;              // [BH, N, d] fp32
  float* dk;
  float* dv;
  int BH, N, bq, nqb, nkb, nkt;
  float scale, scale_log2;
};

// ---------------------------------------------------------------- dQ
namespace bwd {
template <int D>
struct DQLayout : Sizes<D> {
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_DO = OFF_Q + Sizes<D>::ROWS_BYTES;
  static constexpr uint32_t OFF_K = OFF_DO + Sizes<D>::ROWS_BYTES;
  static constexpr uint32_t OFF_V = OFF_K + kStages * Sizes<D>::ROWS_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_V + kStages * Sizes<D>::ROWS_BYTES;
  static constexpr uint32_t SMEM = OFF_BAR + 256 + 1024;
};
enum {
  DQ_QFULL = 0, DQ_QEMPTY, DQ_KVFULL, DQ_KVEMPTY = DQ_KVFULL + kStages,
  DQ_SFULL = DQ_KVEMPTY + kStages,   // [2] S and dP of the tile in that S buffer landed
  DQ_PFULL = DQ_SFULL + 2,           // [2] dS written over that S buffer
  DQ_DPEMPTY = DQ_PFULL + 2,         // dP read by every compute warp (the next dP may land)
  DQ_OFULL, DQ_OEMPTY, DQ_DRAIN, DQ_COUNT
};
constexpr int kDQThreads = 32 * (2 + kCWarps);
}  // namespace bwd

template <int D>
__global__ void __launch_bounds__(bwd::kDQThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                  const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, BwdArgs a) {
  using namespace bwd;
  using L = DQLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  static_assert(DQ_COUNT * 8 + 8 <= 256, "barrier region");
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + DQ_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = a.BH * a.nqb;
  // two S buffers (dS is written over S), one dP buffer, the dQ accumulator
  constexpr uint32_t TM_S = 0, TM_DP = 256, TM_DQ = 384;

  if (threadIdx.x == 0) {
    mbar_init(&bars[DQ_QFULL], 1);
    mbar_init(&bars[DQ_QEMPTY], 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&bars[DQ_KVFULL + i], 1);
      mbar_init(&bars[DQ_KVEMPTY + i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars[DQ_SFULL + i], 1);
      mbar_init(&bars[DQ_PFULL + i], kCWarps);
    }
    mbar_init(&bars[DQ_DPEMPTY], kCWarps);
    mbar_init(&bars[DQ_OFULL], 1);
    mbar_init(&bars[DQ_OEMPTY], kCWarps);
    mbar_init(&bars[DQ_DRAIN], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *tmem_slot;

  auto item_cnt = [&](int item) { return min(max(__ldg(a.kv_cnt + item), 0), a.nkb); };

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmDO);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int g = 0, ii = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x) {
        const int cnt = item_cnt(item);
        if (cnt == 0) continue;
        const int bh = item / a.nqb, qb = item % a.nqb;
        if (!(ok = mbar_wait(&bars[DQ_QEMPTY], (ii & 1) ^ 1, abort_flag))) break;
        mbar_arrive_expect_tx(&bars[DQ_QFULL], 2 * L::ROWS_BYTES);
#pragma unroll
        for (int c = 0; c < L::NCH; ++c) {
          tma_load_3d(smem + L::OFF_Q + c * L::CHUNK, &tmQ, &bars[DQ_QFULL], c * 64, qb * a.bq, bh);
          tma_load_3d(smem + L::OFF_DO + c * L::CHUNK, &tmDO, &bars[DQ_QFULL], c * 64, qb * a.bq, bh);
        }
        ++ii;
        const int* row = a.kv_idx + static_cast<long long>(item) * a.nkb;
        for (int t = 0; ok && t < (cnt + 1) / 2; ++t, ++g) {
          const int s = g % kStages;
          const int nblk = min(2, cnt - 2 * t);
          const int kb0 = __ldg(row + 2 * t), kb1 = nblk > 1 ? __ldg(row + 2 * t + 1) : 0;
          if (!(ok = mbar_wait(&bars[DQ_KVEMPTY + s], ((g / kStages) & 1) ^ 1, abort_flag))) break;
          mbar_arrive_expect_tx(&bars[DQ_KVFULL + s], 2 * nblk * L::BLK_BYTES);
          uint8_t* dk = smem + L::OFF_K + s * L::ROWS_BYTES;
          uint8_t* dv = smem + L::OFF_V + s * L::ROWS_BYTES;
#pragma unroll
          for (int c = 0; c < L::NCH; ++c) {
            tma_load_3d(dk + c * L::CHUNK, &tmK, &bars[DQ_KVFULL + s], c * 64, kb0 * 64, bh);
            tma_load_3d(dv + c * L::CHUNK, &tmV, &bars[DQ_KVFULL + s], c * 64, kb0 * 64, bh);
            if (nblk > 1) {
              tma_load_3d(dk + c * L::CHUNK + 64 * 128, &tmK, &bars[DQ_KVFULL + s], c * 64, kb1 * 64, bh);
              tma_load_3d(dv + c * L::CHUNK + 64 * 128, &tmV, &bars[DQ_KVFULL + s], c * 64, kb1 * 64, bh);
            }
          }
        }
      }
      for (int i = 1; i <= kStages && i <= g; ++i)
        mbar_drain(&bars[DQ_KVFULL + (g - i) % kStages], ((g - i) / kStages) & 1);
      if (ii > 0) mbar_drain(&bars[DQ_QFULL], (ii - 1) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint64_t qdesc = sw128_desc(smem_u32(smem + L::OFF_Q), 16, 1024);
      const uint64_t dodesc = sw128_desc(smem_u32(smem + L::OFF_DO), 16, 1024);
      const uint64_t kdesc0 = sw128_desc(smem_u32(smem + L::OFF_K), 16, 1024);              // K-major (S = Q K^T)
      const uint64_t vdesc0 = sw128_desc(smem_u32(smem + L::OFF_V), 16, 1024);              // K-major (dP = dO V^T)
      const uint64_t kmn0 = sw128_desc(smem_u32(smem + L::OFF_K), L::CHUNK, 1024);          // MN-major (dQ += dS K)
      const uint32_t id2 = idesc_bf16_f32(kBM, 128, false, false);
      const uint32_t id1 = idesc_bf16_f32(kBM, 64, false, false);
      const uint32_t idq = idesc_bf16_f32(kBM, D, false, true);
      // S and dP of tile t + 1 are issued before the dQ product of tile t, so
      // they run while the compute warps form dS(t); S alternates between two
      // buffers, and dP(t + 1) waits until every compute warp has read dP(t).
      // (tcgen05.mma executes in issue order, so S(t + 2) follows the dQ
      // product that read dS(t) from the same buffer.)
      auto issue_s_dp = [&](int g, int cnt, int t) -> bool {
        const int s = g % kStages, b = g & 1;
        const int nblk = min(2, cnt - 2 * t);
        if (!mbar_wait(&bars[DQ_KVFULL + s], (g / kStages) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t id = nblk == 2 ? id2 : id1;
        const uint64_t kd = kdesc0 + ((s * L::ROWS_BYTES) >> 4), vd = vdesc0 + ((s * L::ROWS_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (((kk >> 2) * L::CHUNK) + (kk & 3) * 32u) >> 4;
          umma_ss(tm + TM_S + b * 128, qdesc + off, kd + off, id, kk > 0 ? 1u : 0u);
        }
        if (g > 0 && !mbar_wait(&bars[DQ_DPEMPTY], (g - 1) & 1, abort_flag)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (((kk >> 2) * L::CHUNK) + (kk & 3) * 32u) >> 4;
          umma_ss(tm + TM_DP, dodesc + off, vd + off, id, kk > 0 ? 1u : 0u);
        }
        tc_commit(&bars[DQ_SFULL + b]);
        return true;
      };
      int g = 0, ii = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x) {
        const int cnt = item_cnt(item);
        if (cnt == 0) continue;
        if (!(ok = mbar_wait(&bars[DQ_QFULL], ii & 1, abort_flag))) break;
        const int T = (cnt + 1) / 2;
        if (!(ok = issue_s_dp(g, cnt, 0))) break;
        for (int t = 0; ok && t < T; ++t, ++g) {
          const int s = g % kStages, b = g & 1;
          const int nblk = min(2, cnt - 2 * t);
          if (t + 1 < T && !(ok = issue_s_dp(g + 1, cnt, t + 1))) break;
          if (!(ok = mbar_wait(&bars[DQ_PFULL + b], (g >> 1) & 1, abort_flag))) break;
          if (t == 0 && !(ok = mbar_wait(&bars[DQ_OEMPTY], (ii & 1) ^ 1, abort_flag))) break;
          tc_fence_after();
          const uint64_t km = kmn0 + ((s * L::ROWS_BYTES) >> 4);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            if (kk < nblk * 4)
              umma_ts(tm + TM_DQ, tm + TM_S + b * 128 + (kk >> 2) * 64 + (kk & 3) * 8, km + ((kk * 2048u) >> 4), idq,
                      (t > 0 || kk > 0) ? 1u : 0u);
          tc_commit(&bars[DQ_KVEMPTY + s]);
          if (t + 1 == T) {
            tc_commit(&bars[DQ_QEMPTY]);
            tc_commit(&bars[DQ_OFULL]);
          }
        }
        ++ii;
      }
      tc_commit(&bars[DQ_DRAIN]);
      mbar_drain(&bars[DQ_DRAIN], 0);
    }
  } else {
    const int cw = warp - 2;
    const int quad = warp & 3, half = cw >> 2;
    const int row = quad * 32 + lane;
    const uint32_t la = static_cast<uint32_t>(quad * 32) << 16;
    const int tail_valid = a.N - (a.nkb - 1) * 64;
    int g = 0, ii = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x) {
      const int bh = item / a.nqb, qb = item % a.nqb;
      const int grow = qb * a.bq + row;
      const bool store = row < a.bq && grow < a.N;
      float* dqrow = a.dq + (static_cast<long long>(bh) * a.N + grow) * D + half * (D / 2);
      const int cnt = item_cnt(item);
      if (cnt == 0) {
        if (store)
          for (int c = 0; c < D / 2; c += 4) *reinterpret_cast<float4*>(dqrow + c) = make_float4(0.f, 0.f, 0.f, 0.f);
        continue;
      }
      const float lse2 = store ? __ldg(a.lse + static_cast<long long>(bh) * a.N + grow) * 1.4426950408889634f : 0.f;
      const float dr = store ? __ldg(a.delta + static_cast<long long>(bh) * a.N + grow) : 0.f;
      bool tail = false;
      if (a.N % 64) tail = __ldg(a.kv_idx + static_cast<long long>(item) * a.nkb + cnt - 1) == a.nkb - 1;
      const int T = (cnt + 1) / 2;
      for (int t = 0; ok && t < T; ++t, ++g) {
        const int b = g & 1;
        if (!(ok = mbar_wait(&bars[DQ_SFULL + b], (g >> 1) & 1, abort_flag))) break;
        tc_fence_after();
        uint32_t s0[32], s1[32], p0[32], p1[32];
        tmem_ld32(tm + la + TM_S + b * 128 + half * 64, s0);
        tmem_ld32(tm + la + TM_S + b * 128 + half * 64 + 32, s1);
        tmem_ld32(tm + la + TM_DP + half * 64, p0);
        tmem_ld32(tm + la + TM_DP + half * 64 + 32, p1);
        tmem_wait_ld();
        reg_fence(s0);
        reg_fence(s1);
        reg_fence(p0);
        reg_fence(p1);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[DQ_DPEMPTY]);   // dP(t) read: the next dP may land
        int valid = 64;
        if (t == T - 1) {
          const int nblk = cnt - 2 * t;
          valid = half < nblk ? 64 : 0;
          if (tail && half == nblk - 1) valid = tail_valid;
        }
        uint32_t ds[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          float e[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int col = 2 * c + u;
            const float sv = __uint_as_float(col < 32 ? s0[col] : s1[col - 32]);
            const float pv = __uint_as_float(col < 32 ? p0[col] : p1[col - 32]);
            // columns past the tile's keys may hold stale values: exact zeros there
            e[u] = col < valid ? fast_exp2(fmaf(sv, a.scale_log2, -lse2)) * (pv - dr) : 0.f;
          }
          ds[c] = pack_bf16x2(e[0], e[1]);
        }
        // dS over the first 32 of this half's own 64 S columns (the other
        // half may not have read its S yet)
        tmem_st32(tm + la + TM_S + b * 128 + half * 64, ds);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[DQ_PFULL + b]);
      }
      if (!ok) break;
      if (!(ok = mbar_wait(&bars[DQ_OFULL], ii & 1, abort_flag))) break;
      tc_fence_after();
      uint32_t o0[32], o1[32];
      tmem_ld32(tm + la + TM_DQ + half * (D / 2), o0);
      if (D == 128) tmem_ld32(tm + la + TM_DQ + half * (D / 2) + 32, o1);
      tmem_wait_ld();
      reg_fence(o0);
      if (D == 128) reg_fence(o1);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[DQ_OEMPTY]);
      ++ii;
      if (store) {
#pragma unroll
        for (int c = 0; c < 32; c += 4)
          *reinterpret_cast<float4*>(dqrow + c) = make_float4(__uint_as_float(o0[c]) * a.scale, __uint_as_float(o0[c + 1]) * a.scale,
                                                              __uint_as_float(o0[c + 2]) * a.scale, __uint_as_float(o0[c + 3]) * a.scale);
        if (D == 128) {
#pragma unroll
          for (int c = 0; c < 32; c += 4)
            *reinterpret_cast<float4*>(dqrow + 32 + c) = make_float4(__uint_as_float(o1[c]) * a.scale, __uint_as_float(o1[c + 1]) * a.scale,
                                                                     __uint_as_float(o1[c + 2]) * a.scale, __uint_as_float(o1[c + 3]) * a.scale);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tm, 512);
  }
}

// ---------------------------------------------------------------- dK, dV
namespace bwd {
template <int D>
struct KVLayout : Sizes<D> {
  static constexpr uint32_t OFF_K = 0;
  static constexpr uint32_t OFF_V = OFF_K + Sizes<D>::ROWS_BYTES;
  static constexpr uint32_t OFF_Q = OFF_V + Sizes<D>::ROWS_BYTES;
  static constexpr uint32_t OFF_DO = OFF_Q + kStages * Sizes<D>::ROWS_BYTES;
  static constexpr uint32_t OFF_ST = OFF_DO + kStages * Sizes<D>::ROWS_BYTES;   // [stage][lse2 | delta][128] float
  static constexpr uint32_t OFF_BAR = OFF_ST + kStages * 2 * 128 * 4;
  static constexpr uint32_t SMEM = OFF_BAR + 256 + 1024;
};
enum {
  KV_KFULL = 0, KV_KEMPTY, KV_QFULL, KV_QEMPTY = KV_QFULL + kStages, KV_STFULL = KV_QEMPTY + kStages,
  KV_STEMPTY = KV_STFULL + kStages, KV_SFULL = KV_STEMPTY + kStages,
  KV_SEMPTY,     // S^T and dP^T read by every compute warp (the next S^T may land)
  KV_PFULL, KV_OFULL, KV_OEMPTY, KV_DRAIN, KV_COUNT
};
constexpr int kKVThreads = 32 * (3 + kCWarps);
}  // namespace bwd

template <int D>
__global__ void __launch_bounds__(bwd::kKVThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, BwdArgs a) {
  using namespace bwd;
  using L = KVLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  static_assert(KV_COUNT * 8 + 8 <= 256, "barrier region");
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + KV_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* stats = reinterpret_cast<float*>(smem + L::OFF_ST);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = a.BH * a.nkt;
  constexpr uint32_t TM_ST = 0, TM_DPT = 128, TM_DV = 256, TM_DK = 384;

  if (threadIdx.x == 0) {
    mbar_init(&bars[KV_KFULL], 1);
    mbar_init(&bars[KV_KEMPTY], 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&bars[KV_QFULL + i], 1);
      mbar_init(&bars[KV_QEMPTY + i], 1);
      mbar_init(&bars[KV_STFULL + i], 1);
      mbar_init(&bars[KV_STEMPTY + i], kCWarps);
    }
    mbar_init(&bars[KV_SFULL], 1);
    mbar_init(&bars[KV_SEMPTY], kCWarps);
    mbar_init(&bars[KV_PFULL], kCWarps);
    mbar_init(&bars[KV_OFULL], 1);
    mbar_init(&bars[KV_OEMPTY], kCWarps);
    mbar_init(&bars[KV_DRAIN], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *tmem_slot;

  auto list_cnt = [&](int item) { return min(max(__ldg(a.qt_cnt + item), 0), a.nqb); };
  auto list_at = [&](int item, int j) { return __ldg(a.qt_idx + static_cast<long long>(item) * a.nqb + j); };

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmDO);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int g = 0, ii = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x) {
        const int cnt = list_cnt(item);
        if (cnt == 0) continue;
        const int bh = item / a.nkt, kt = item % a.nkt;
        const int nblk = min(2, a.nkb - 2 * kt);
        if (!(ok = mbar_wait(&bars[KV_KEMPTY], (ii & 1) ^ 1, abort_flag))) break;
        mbar_arrive_expect_tx(&bars[KV_KFULL], 2 * nblk * L::BLK_BYTES);
#pragma unroll
        for (int c = 0; c < L::NCH; ++c)
          for (int b = 0; b < nblk; ++b) {
            tma_load_3d(smem + L::OFF_K + c * L::CHUNK + b * 64 * 128, &tmK, &bars[KV_KFULL], c * 64, (2 * kt + b) * 64, bh);
            tma_load_3d(smem + L::OFF_V + c * L::CHUNK + b * 64 * 128, &tmV, &bars[KV_KFULL], c * 64, (2 * kt + b) * 64, bh);
          }
        ++ii;
        for (int j = 0; ok && j < cnt; ++j, ++g) {
          const int s = g % kStages;
          const int qb = list_at(item, j) & 0xFFFFFF;
          if (!(ok = mbar_wait(&bars[KV_QEMPTY + s], ((g / kStages) & 1) ^ 1, abort_flag))) break;
          mbar_arrive_expect_tx(&bars[KV_QFULL + s], 2 * L::ROWS_BYTES);
#pragma unroll
          for (int c = 0; c < L::NCH; ++c) {
            tma_load_3d(smem + L::OFF_Q + s * L::ROWS_BYTES + c * L::CHUNK, &tmQ, &bars[KV_QFULL + s], c * 64, qb * a.bq, bh);
            tma_load_3d(smem + L::OFF_DO + s * L::ROWS_BYTES + c * L::CHUNK, &tmDO, &bars[KV_QFULL + s], c * 64, qb * a.bq, bh);
          }
        }
      }
      for (int i = 1; i <= kStages && i <= g; ++i)
        mbar_drain(&bars[KV_QFULL + (g - i) % kStages], ((g - i) / kStages) & 1);
      if (ii > 0) mbar_drain(&bars[KV_KFULL], (ii - 1) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint64_t kdesc = sw128_desc(smem_u32(smem + L::OFF_K), 16, 1024);
      const uint64_t vdesc = sw128_desc(smem_u32(smem + L::OFF_V), 16, 1024);
      const uint64_t qdesc0 = sw128_desc(smem_u32(smem + L::OFF_Q), 16, 1024);          // K-major (S^T = K Q^T)
      const uint64_t dodesc0 = sw128_desc(smem_u32(smem + L::OFF_DO), 16, 1024);        // K-major (dP^T = V dO^T)
      const uint64_t qmn0 = sw128_desc(smem_u32(smem + L::OFF_Q), L::CHUNK, 1024);      // MN-major (dK += dS^T Q)
      const uint64_t domn0 = sw128_desc(smem_u32(smem + L::OFF_DO), L::CHUNK, 1024);    // MN-major (dV += P^T dO)
      const uint32_t id_s = idesc_bf16_f32(kBM, 128, false, false);
      const uint32_t id_acc = idesc_bf16_f32(kBM, D, false, true);
      // P^T and dS^T are written into the dP^T columns, so the S^T buffer is
      // free once the compute warps have read it: S^T of the next query block
      // is computed while they form P^T and dS^T of this one. dP^T of the next
      // block follows the dV and dK products that read this one's P^T and
      // dS^T (tcgen05.mma executes in issue order).
      auto issue_st = [&](int s) {
        const uint64_t qd = qdesc0 + ((s * L::ROWS_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (((kk >> 2) * L::CHUNK) + (kk & 3) * 32u) >> 4;
          umma_ss(tm + TM_ST, kdesc + off, qd + off, id_s, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_dpt = [&](int s) {
        const uint64_t dd = dodesc0 + ((s * L::ROWS_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (((kk >> 2) * L::CHUNK) + (kk & 3) * 32u) >> 4;
          umma_ss(tm + TM_DPT, vdesc + off, dd + off, id_s, kk > 0 ? 1u : 0u);
        }
      };
      int g = 0, ii = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x) {
        const int cnt = list_cnt(item);
        if (cnt == 0) continue;
        if (!(ok = mbar_wait(&bars[KV_KFULL], ii & 1, abort_flag))) break;
        {
          // the item's first query block
          const int s = g % kStages;
          if (!(ok = mbar_wait(&bars[KV_QFULL + s], (g / kStages) & 1, abort_flag))) break;
          if (g > 0 && !(ok = mbar_wait(&bars[KV_SEMPTY], (g - 1) & 1, abort_flag))) break;
          tc_fence_after();
          issue_st(s);
          issue_dpt(s);
          tc_commit(&bars[KV_SFULL]);
        }
        for (int j = 0; ok && j < cnt; ++j, ++g) {
          const int s = g % kStages;
          if (j + 1 < cnt) {
            const int s1 = (g + 1) % kStages;
            if (!(ok = mbar_wait(&bars[KV_QFULL + s1], ((g + 1) / kStages) & 1, abort_flag))) break;
            if (!(ok = mbar_wait(&bars[KV_SEMPTY], g & 1, abort_flag))) break;
            tc_fence_after();
            issue_st(s1);
          }
          if (!(ok = mbar_wait(&bars[KV_PFULL], g & 1, abort_flag))) break;
          if (j == 0 && !(ok = mbar_wait(&bars[KV_OEMPTY], (ii & 1) ^ 1, abort_flag))) break;
          tc_fence_after();
          const uint64_t dmn = domn0 + ((s * L::ROWS_BYTES) >> 4), qmn = qmn0 + ((s * L::ROWS_BYTES) >> 4);
          // K step kk (16 query columns) reads 8 TMEM columns: in each half's
          // 64 dP^T columns, each 32 hold dS^T of 32 query columns in their
          // first 16 and P^T of the same query columns in their second 16
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_ts(tm + TM_DV, tm + TM_DPT + (kk >> 2) * 64 + ((kk & 3) >> 1) * 32 + 16 + (kk & 1) * 8,
                    dmn + ((kk * 2048u) >> 4), id_acc, (j > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_ts(tm + TM_DK, tm + TM_DPT + (kk >> 2) * 64 + ((kk & 3) >> 1) * 32 + (kk & 1) * 8,
                    qmn + ((kk * 2048u) >> 4), id_acc, (j > 0 || kk > 0) ? 1u : 0u);
          tc_commit(&bars[KV_QEMPTY + s]);
          if (j + 1 < cnt) {
            issue_dpt((g + 1) % kStages);
            tc_commit(&bars[KV_SFULL]);
          } else {
            tc_commit(&bars[KV_KEMPTY]);
            tc_commit(&bars[KV_OFULL]);
          }
        }
        ++ii;
      }
      tc_commit(&bars[KV_DRAIN]);
      mbar_drain(&bars[KV_DRAIN], 0);
    }
  } else if (warp == 2) {
    // LSE (log2 units, +inf past the block's valid rows) and D of each query block, in list order
    int g = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x) {
      const int cnt = list_cnt(item);
      const int bh = item / a.nkt;
      for (int j = 0; ok && j < cnt; ++j, ++g) {
        const int s = g % kStages;
        const int qb = list_at(item, j) & 0xFFFFFF;
        if (!(ok = mbar_wait(&bars[KV_STEMPTY + s], ((g / kStages) & 1) ^ 1, abort_flag))) break;
        float* st = stats + s * 256;
        for (int i = lane; i < 128; i += 32) {
          const int qr = qb * a.bq + i;
          const bool v = i < a.bq && qr < a.N;
          const long long off = static_cast<long long>(bh) * a.N + qr;
          st[i] = v ? __ldg(a.lse + off) * 1.4426950408889634f : INFINITY;
          st[128 + i] = v ? __ldg(a.delta + off) : 0.f;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[KV_STFULL + s]);
      }
    }
  } else {
    const int cw = warp - 3;
    const int quad = warp & 3, half = cw >> 2;
    const int row = quad * 32 + lane;                 // key row of the tile
    const uint32_t la = static_cast<uint32_t>(quad * 32) << 16;
    const int blk = row >> 6;                         // which of the tile's two key blocks
    int g = 0, ii = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x) {
      const int bh = item / a.nkt, kt = item % a.nkt;
      const int key = kt * 128 + row;
      const bool store = key < a.N;
      const long long roff = (static_cast<long long>(bh) * a.N + key) * D + half * (D / 2);
      const int cnt = list_cnt(item);
      if (cnt == 0) {
        if (store)
          for (int c = 0; c < D / 2; c += 4) {
            *reinterpret_cast<float4*>(a.dk + roff + c) = make_float4(0.f, 0.f, 0.f, 0.f);
            *reinterpret_cast<float4*>(a.dv + roff + c) = make_float4(0.f, 0.f, 0.f, 0.f);
          }
        continue;
      }
      for (int j = 0; ok && j < cnt; ++j, ++g) {
        const int s = g % kStages;
        const bool keep = (list_at(item, j) >> (24 + blk)) & 1;
        if (!(ok = mbar_wait(&bars[KV_SFULL], g & 1, abort_flag))) break;
        if (!(ok = mbar_wait(&bars[KV_STFULL + s], (g / kStages) & 1, abort_flag))) break;
        tc_fence_after();
        uint32_t s0[32], s1[32], p0[32];
        tmem_ld32(tm + la + TM_ST + half * 64, s0);
        tmem_ld32(tm + la + TM_ST + half * 64 + 32, s1);
        tmem_ld32(tm + la + TM_DPT + half * 64, p0);
        tmem_wait_ld();
        reg_fence(s0);
        reg_fence(s1);
        reg_fence(p0);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[KV_SEMPTY]);   // S^T read: the next S^T may land
        const float* st = stats + s * 256 + half * 64;
        // dS^T and P^T of query columns [32 h2, 32 h2 + 32) of this half go
        // over the 32 dP^T columns those query columns came from (dS^T in the
        // first 16, P^T in the second), so the second 32 dP^T columns are
        // loaded only after the first 32 are done with: fewer live registers.
        // Each half writes only its own 64 columns (the other half may not have
        // read its columns yet; the S^T buffer already holds the next block's S^T).
        auto form = [&](int h2, const uint32_t (&sr)[32], const uint32_t (&pr)[32]) {
          uint32_t pt[16], dst[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            float pp[2], dd[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int col = 32 * h2 + 2 * c + u;
              // rows of a key block that does not keep this query block (or past
              // the last key block, with stale values) contribute exact zeros
              const float p = keep ? fast_exp2(fmaf(__uint_as_float(sr[2 * c + u]), a.scale_log2, -st[col])) : 0.f;
              pp[u] = p;
              dd[u] = keep ? p * (__uint_as_float(pr[2 * c + u]) - st[128 + col]) : 0.f;
            }
            pt[c] = pack_bf16x2(pp[0], pp[1]);
            dst[c] = pack_bf16x2(dd[0], dd[1]);
          }
          tmem_st16(tm + la + TM_DPT + half * 64 + 32 * h2, dst);
          tmem_st16(tm + la + TM_DPT + half * 64 + 32 * h2 + 16, pt);
        };
        form(0, s0, p0);
        {
          uint32_t p1[32];
          tmem_ld32(tm + la + TM_DPT + half * 64 + 32, p1);
          tmem_wait_ld();
          reg_fence(p1);
          form(1, s1, p1);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&bars[KV_PFULL]);
          mbar_arrive(&bars[KV_STEMPTY + s]);
        }
      }
      if (!ok) break;
      if (!(ok = mbar_wait(&bars[KV_OFULL], ii & 1, abort_flag))) break;
      tc_fence_after();
      uint32_t v0[32], v1[32], k0[32], k1[32];
      tmem_ld32(tm + la + TM_DV + half * (D / 2), v0);
      tmem_ld32(tm + la + TM_DK + half * (D / 2), k0);
      if (D == 128) {
        tmem_ld32(tm + la + TM_DV + half * (D / 2) + 32, v1);
        tmem_ld32(tm + la + TM_DK + half * (D / 2) + 32, k1);
      }
      tmem_wait_ld();
      reg_fence(v0);
      reg_fence(k0);
      if (D == 128) {
        reg_fence(v1);
        reg_fence(k1);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[KV_OEMPTY]);
      ++ii;
      if (store) {
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          *reinterpret_cast<float4*>(a.dv + roff + c) = make_float4(__uint_as_float(v0[c]), __uint_as_float(v0[c + 1]),
                                                                    __uint_as_float(v0[c + 2]), __uint_as_float(v0[c + 3]));
          *reinterpret_cast<float4*>(a.dk + roff + c) = make_float4(__uint_as_float(k0[c]) * a.scale, __uint_as_float(k0[c + 1]) * a.scale,
                                                                    __uint_as_float(k0[c + 2]) * a.scale, __uint_as_float(k0[c + 3]) * a.scale);
        }
        if (D == 128) {
#pragma unroll
          for (int c = 0; c < 32; c += 4) {
            *reinterpret_cast<float4*>(a.dv + roff + 32 + c) = make_float4(__uint_as_float(v1[c]), __uint_as_float(v1[c + 1]),
                                                                           __uint_as_float(v1[c + 2]), __uint_as_float(v1[c + 3]));
            *reinterpret_cast<float4*>(a.dk + roff + 32 + c) = make_float4(__uint_as_float(k1[c]) * a.scale, __uint_as_float(k1[c + 1]) * a.scale,
                                                                           __uint_as_float(k1[c + 2]) * a.scale, __uint_as_float(k1[c + 3]) * a.scale);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tm, 512);
  }
}

// Workspace: D [BH, N] fp32, the dense mask, the transposed lists.
size_t bwd_ws_bytes(int BH, int N, int nqb, int nkb) {
  const long long nkt = (nkb + 1) / 2;
  auto up = [](long long x) { return static_cast<size_t>((x + 255) / 256 * 256); };
  return up(static_cast<long long>(BH) * N * 4) + up(static_cast<long long>(BH) * nqb * nkb) +
         up(static_cast<long long>(BH) * nkt * nqb * 4) + up(static_cast<long long>(BH) * nkt * 4);
}

template <int D>
static cudaError_t launch_bwd_d(BwdArgs a, const void* o, char* ws, cudaStream_t st) {
  auto up = [](long long x) { return static_cast<size_t>((x + 255) / 256 * 256); };
  float* delta = reinterpret_cast<float*>(ws);
  uint8_t* mask = reinterpret_cast<uint8_t*>(ws + up(static_cast<long long>(a.BH) * a.N * 4));
  int* qt_idx = reinterpret_cast<int*>(reinterpret_cast<char*>(mask) + up(static_cast<long long>(a.BH) * a.nqb * a.nkb));
  int* qt_cnt = reinterpret_cast<int*>(reinterpret_cast<char*>(qt_idx) + up(static_cast<long long>(a.BH) * a.nkt * a.nqb * 4));
  a.delta = delta;
  a.qt_idx = qt_idx;
  a.qt_cnt = qt_cnt;
  const long long rows = static_cast<long long>(a.BH) * a.N;
  const int rpw = 32 / (D / 8);
  bwd_delta_kernel<D><<<static_cast<int>(((rows + rpw - 1) / rpw * 32 + 255) / 256), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(a.dout), rows, delta);
  cudaError_t e = cudaMemsetAsync(mask, 0, static_cast<size_t>(a.BH) * a.nqb * a.nkb, st);
  if (e != cudaSuccess) return e;
  const long long lrows = static_cast<long long>(a.BH) * a.nqb;
  lists_to_mask_kernel<<<static_cast<int>((lrows * a.nkb + 255) / 256), 256, 0, st>>>(a.kv_idx, a.kv_cnt, lrows, a.nkb, mask);
  const long long warps = static_cast<long long>(a.BH) * a.nkt;
  col_lists_kernel<<<static_cast<int>((warps * 32 + 255) / 256), 256, 0, st>>>(mask, a.BH, a.nqb, a.nkb, a.nkt, qt_idx, qt_cnt);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  CUtensorMap mq, mdo, mk, mv;
  if (encode_tensor_map_3d_bf16(&mq, a.q, D, a.N, a.BH, 64, 128) != CUDA_SUCCESS ||
      encode_tensor_map_3d_bf16(&mdo, a.dout, D, a.N, a.BH, 64, 128) != CUDA_SUCCESS ||
      encode_tensor_map_3d_bf16(&mk, a.k, D, a.N, a.BH, 64, 64) != CUDA_SUCCESS ||
      encode_tensor_map_3d_bf16(&mv, a.v, D, a.N, a.BH, 64, 64) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  using LQ = bwd::DQLayout<D>;
  using LK = bwd::KVLayout<D>;
  if ((e = cudaFuncSetAttribute(bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, LQ::SMEM)) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(bwd_dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, LK::SMEM)) != cudaSuccess) return e;
  const long long nq = lrows, nk = warps;
  bwd_dq_kernel<D><<<static_cast<int>(nq < sms ? nq : sms), bwd::kDQThreads, LQ::SMEM, st>>>(mq, mdo, mk, mv, a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  bwd_dkdv_kernel<D><<<static_cast<int>(nk < sms ? nk : sms), bwd::kKVThreads, LK::SMEM, st>>>(mq, mdo, mk, mv, a);
  return cudaGetLastError();
}

cudaError_t launch_sparse_attn_bwd(const BwdArgs& a, int d, const void* o, void* ws, cudaStream_t st) {
  if (static_cast<long long>(a.BH) * a.nqb > 0x7FFFFFFFLL || static_cast<long long>(a.BH) * a.nkt > 0x7FFFFFFFLL)
    return cudaErrorInvalidValue;
  char* w = static_cast<char*>(ws);
  return d == 128 ? launch_bwd_d<128>(a, o, w, st) : launch_bwd_d<64>(a, o, w, st);
}

}  // namespace sa
