// attn_kernel.cu — block-sparse attention forward for sm_100a
// (page: "SpargeAttention2" §2(3): FlashAttention-based block-sparse kernel that
// skips the masked QK^T and softmax/PV work; Veda §2.3 describes a
// producer/consumer split with TMA fetches of non-contiguous K/V tiles).
//
// One CTA computes one 128-row query tile of one head against the key blocks
// its compacted list keeps. Two 64-key blocks form one 128-key tile.
//
//   warp 0      TMA producer: Q once, then K and V of each kept tile into a
//               2-stage ring (each 64-key block is its own TMA box, so the two
//               blocks of a tile need not be adjacent in memory)
//   warp 1      TMEM allocation and the single MMA-issuing thread:
//                 S_j = Q K_j^T   (tcgen05.mma, A and B from shared memory,
//                                  fp32 accumulator in one of 3 TMEM buffers)
//                 O  += P_j V_j   (tcgen05.mma, A = P_j read from TMEM)
//   warps 2..5  softmax: thread t owns TMEM lane t = query row t. Loads S_j,
//               masks keys past N, keeps the running max m (log2 domain) and
//               sum l, writes P_j = exp2(S_j*scale*log2e - m) as bf16 back into
//               the S buffer, and rescales O in TMEM when m grows by more than
//               2^8 (otherwise the stale max is kept: P stays <= 256).
//               Finally O / l is written as bf16, with the row log-sum-exp.
//
// TMEM columns: S buffers at 0, 128, 256 (fp32, 128 wide); O at 384 (d wide).
#include "sa_internal.h"

namespace sa {

namespace {

constexpr int kBM = 128;    // query rows per tile
constexpr int kBN = 128;    // keys per tile (two 64-key blocks)
constexpr int kStages = 2;  // K/V ring depth
constexpr int kSBufs = 3;   // S/P buffers in TMEM
constexpr int kThreads = 192;

template <int D>
struct Layout {
  static constexpr int NCH = D / 64;                       // 128-byte chunks along d
  static constexpr uint32_t Q_BYTES = kBM * D * 2;
  static constexpr uint32_t TILE_BYTES = kBN * D * 2;       // one K or V tile
  static constexpr uint32_t BLK_BYTES = 64 * D * 2;         // one 64-key block
  static constexpr uint32_t Q_CHUNK = kBM * 128;            // bytes per d-chunk of Q
  static constexpr uint32_t KV_CHUNK = kBN * 128;           // bytes per d-chunk of K/V
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = OFF_Q + Q_BYTES;
  static constexpr uint32_t OFF_V = OFF_K + kStages * TILE_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_V + kStages * TILE_BYTES;
  static constexpr uint32_t USED = OFF_BAR + 256;
  // Ask for enough shared memory that a second CTA never shares the SM (each
  // CTA holds all 512 TMEM columns).
  static constexpr uint32_t SMEM = (USED + 1024 > 120 * 1024) ? USED + 1024 : 120 * 1024;
};

__host__ __device__ constexpr uint32_t tm_s(int b) { return static_cast<uint32_t>(b) * 128u; }
constexpr uint32_t TM_O = 384;
constexpr uint32_t TM_COLS = 512;

// barrier slots
enum {
  B_Q = 0,
  B_KFULL = 1,
  B_KEMPTY = B_KFULL + kStages,
  B_VFULL = B_KEMPTY + kStages,
  B_VEMPTY = B_VFULL + kStages,
  B_SFULL = B_VEMPTY + kStages,
  B_PFULL = B_SFULL + kSBufs,
  B_OREADY = B_PFULL + kSBufs,
  B_COUNT = B_OREADY + kSBufs
};

}  // namespace

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, AttnArgs a) {
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + L::OFF_Q;
  uint8_t* sK = smem + L::OFF_K;
  uint8_t* sV = smem + L::OFF_V;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + B_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int qb = blockIdx.x;
  const int bh = blockIdx.y;
  const int q_row0 = qb * a.bq;

  const int* kv_row = a.dense ? nullptr : a.kv_idx + (static_cast<long long>(bh) * a.nqb + qb) * a.nkb;
  const int cnt = a.dense ? a.nkb : a.kv_cnt[static_cast<long long>(bh) * a.nqb + qb];
  const int T = (cnt + 1) >> 1;

  if (threadIdx.x == 0) {
    mbar_init(&bars[B_Q], 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars[B_KFULL + s], 1);
      mbar_init(&bars[B_KEMPTY + s], 1);
      mbar_init(&bars[B_VFULL + s], 1);
      mbar_init(&bars[B_VEMPTY + s], 1);
    }
    for (int b = 0; b < kSBufs; ++b) {
      mbar_init(&bars[B_SFULL + b], 1);
      mbar_init(&bars[B_PFULL + b], 4);
      mbar_init(&bars[B_OREADY + b], 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *tmem_slot;

  auto block_of = [&](int i) -> int { return a.dense ? i : __ldg(kv_row + i); };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && T > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(&bars[B_Q], L::Q_BYTES);
#pragma unroll
      for (int c = 0; c < L::NCH; ++c) tma_load_3d(sQ + c * L::Q_CHUNK, &tmQ, &bars[B_Q], c * 64, q_row0, bh);
      for (int j = 0; j < T; ++j) {
        const int s = j % kStages;
        const uint32_t ph = (j / kStages) & 1;
        const int nblk = min(2, cnt - 2 * j);
        const int kb0 = block_of(2 * j);
        const int kb1 = nblk > 1 ? block_of(2 * j + 1) : 0;
        if (!mbar_wait(&bars[B_KEMPTY + s], ph ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(&bars[B_KFULL + s], nblk * L::BLK_BYTES);
        uint8_t* kdst = sK + s * L::TILE_BYTES;
#pragma unroll
        for (int c = 0; c < L::NCH; ++c) {
          tma_load_3d(kdst + c * L::KV_CHUNK, &tmK, &bars[B_KFULL + s], c * 64, kb0 * 64, bh);
          if (nblk > 1)
            tma_load_3d(kdst + c * L::KV_CHUNK + 64 * 128, &tmK, &bars[B_KFULL + s], c * 64, kb1 * 64, bh);
        }
        if (!mbar_wait(&bars[B_VEMPTY + s], ph ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(&bars[B_VFULL + s], nblk * L::BLK_BYTES);
        uint8_t* vdst = sV + s * L::TILE_BYTES;
#pragma unroll
        for (int c = 0; c < L::NCH; ++c) {
          tma_load_3d(vdst + c * L::KV_CHUNK, &tmV, &bars[B_VFULL + s], c * 64, kb0 * 64, bh);
          if (nblk > 1)
            tma_load_3d(vdst + c * L::KV_CHUNK + 64 * 128, &tmV, &bars[B_VFULL + s], c * 64, kb1 * 64, bh);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && T > 0) {
      const uint32_t q_base = smem_u32(sQ);
      const uint32_t k_base = smem_u32(sK);
      const uint32_t v_base = smem_u32(sV);
      const uint32_t idesc_pv = idesc_bf16_f32(kBM, D, false, true);
      bool ok = mbar_wait(&bars[B_Q], 0, abort_flag);
      auto issue_qk = [&](int j) -> bool {
        const int s = j % kStages;
        const int b = j % kSBufs;
        const int nblk = min(2, cnt - 2 * j);
        if (!mbar_wait(&bars[B_KFULL + s], (j / kStages) & 1, abort_flag)) return false;
        if (j >= kSBufs && !mbar_wait(&bars[B_OREADY + b], ((j - kSBufs) / kSBufs) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t idesc = idesc_bf16_f32(kBM, nblk * 64, false, false);
        const uint32_t kt = k_base + s * L::TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk & 3) * 32u;  // 16 bf16 = 32 B along K inside a 128-B row
          const uint64_t adesc = sw128_desc(q_base + (kk >> 2) * L::Q_CHUNK + off, 16, 1024);
          const uint64_t bdesc = sw128_desc(kt + (kk >> 2) * L::KV_CHUNK + off, 16, 1024);
          umma_ss(tm + tm_s(b), adesc, bdesc, idesc, kk > 0 ? 1u : 0u);
        }
        tc_commit(&bars[B_SFULL + b]);
        tc_commit(&bars[B_KEMPTY + s]);
        return true;
      };
      if (ok) ok = issue_qk(0);
      for (int j = 0; ok && j < T; ++j) {
        if (j + 1 < T && !issue_qk(j + 1)) break;
        const int s = j % kStages;
        const int b = j % kSBufs;
        const int nblk = min(2, cnt - 2 * j);
        if (!mbar_wait(&bars[B_PFULL + b], (j / kSBufs) & 1, abort_flag)) break;
        if (!mbar_wait(&bars[B_VFULL + s], (j / kStages) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t vt = v_base + s * L::TILE_BYTES;
        for (int kk = 0; kk < nblk * 4; ++kk) {
          const uint64_t bdesc = sw128_desc(vt + kk * 2048u, L::KV_CHUNK, 1024);
          umma_ts(tm + TM_O, tm + tm_s(b) + kk * 8, bdesc, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&bars[B_OREADY + b]);
        tc_commit(&bars[B_VEMPTY + s]);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int quad = warp & 3;                       // TMEM lane quadrant of this warp
    const int row = quad * 32 + lane;                // query row within the tile
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    const float sl2 = a.scale_log2;
    float m = -INFINITY;                             // running max, log2 domain
    float l = 0.f;
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      const int b = j % kSBufs;
      const int nblk = min(2, cnt - 2 * j);
      const int kb0 = block_of(2 * j);
      const int kb1 = nblk > 1 ? block_of(2 * j + 1) : 0;
      const int valid0 = min(64, a.N - kb0 * 64);
      const int valid1 = nblk > 1 ? min(64, a.N - kb1 * 64) : 0;
      if (!mbar_wait(&bars[B_SFULL + b], (j / kSBufs) & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      uint32_t r0[32], r1[32], r2[32], r3[32];
      const uint32_t sa = tm + lane_addr + tm_s(b);
      tmem_ld32(sa + 0, r0);
      tmem_ld32(sa + 32, r1);
      tmem_ld32(sa + 64, r2);
      tmem_ld32(sa + 96, r3);
      tmem_wait_ld();
      reg_fence(r0);
      reg_fence(r1);
      reg_fence(r2);
      reg_fence(r3);
      float x[128];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        x[c] = __uint_as_float(r0[c]);
        x[32 + c] = __uint_as_float(r1[c]);
        x[64 + c] = __uint_as_float(r2[c]);
        x[96 + c] = __uint_as_float(r3[c]);
      }
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        if (c >= valid0) x[c] = -INFINITY;
        if (c >= valid1) x[64 + c] = -INFINITY;
      }
      float mx = x[0];
#pragma unroll
      for (int c = 1; c < 128; ++c) mx = fmaxf(mx, x[c]);
      const float m_tile = mx * sl2;
      float corr = 1.f;
      if (m_tile > m + 8.f) {
        corr = fast_exp2(m - m_tile);   // 0 on the first tile (m = -inf)
        m = m_tile;
        l *= corr;
      }
      float sum = 0.f;
      uint32_t p0[32], p1[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const float e0 = fast_exp2(fmaf(x[2 * c], sl2, -m));
        const float e1 = fast_exp2(fmaf(x[2 * c + 1], sl2, -m));
        const float e2 = fast_exp2(fmaf(x[64 + 2 * c], sl2, -m));
        const float e3 = fast_exp2(fmaf(x[64 + 2 * c + 1], sl2, -m));
        sum += (e0 + e1) + (e2 + e3);
        p0[c] = pack_bf16x2(e0, e1);
        p1[c] = pack_bf16x2(e2, e3);
      }
      l += sum;
      tmem_st32(sa + 0, p0);
      tmem_st32(sa + 32, p1);
      if (j > 0) {
        // O may only be touched once the previous P V product has landed.
        const int pb = (j - 1) % kSBufs;
        if (!mbar_wait(&bars[B_OREADY + pb], ((j - 1) / kSBufs) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        if (__any_sync(0xFFFFFFFFu, corr != 1.f)) {
#pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t o[32];
            tmem_ld32_wait(tm + lane_addr + TM_O + c0, o);
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * corr);
            tmem_st32(tm + lane_addr + TM_O + c0, o);
          }
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[B_PFULL + b]);
    }
    // ------------------------------------------------------------ epilogue
    const int grow = q_row0 + row;
    const bool store = row < a.bq && grow < a.N;
    __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(a.o) + (static_cast<long long>(bh) * a.N + grow) * D;
    if (T > 0 && ok) {
      const int lb = (T - 1) % kSBufs;
      ok = mbar_wait(&bars[B_OREADY + lb], ((T - 1) / kSBufs) & 1, abort_flag);
      tc_fence_after();
    }
    if (T > 0 && ok) {
      const float inv_l = 1.f / l;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t o[32];
        tmem_ld32_wait(tm + lane_addr + TM_O + c0, o);
        if (store) {
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 16; ++c)
            pk[c] = pack_bf16x2(__uint_as_float(o[2 * c]) * inv_l, __uint_as_float(o[2 * c + 1]) * inv_l);
          uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
          for (int c = 0; c < 4; ++c) dst[c] = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        }
      }
      if (store && a.lse) a.lse[static_cast<long long>(bh) * a.N + grow] = (m + log2f(l)) * 0.69314718055994531f;
    } else if (store) {
      uint4* dst = reinterpret_cast<uint4*>(orow);
      for (int c = 0; c < D / 8; ++c) dst[c] = make_uint4(0, 0, 0, 0);
      if (a.lse) a.lse[static_cast<long long>(bh) * a.N + grow] = -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tm, TM_COLS);
  }
}

template <int D>
static cudaError_t launch_d(const AttnArgs& a, cudaStream_t st) {
  using L = Layout<D>;
  CUtensorMap mq, mk, mv;
  if (encode_tensor_map_3d_bf16(&mq, a.q, D, a.N, a.BH, 64, kBM) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  if (encode_tensor_map_3d_bf16(&mk, a.k, D, a.N, a.BH, 64, 64) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  if (encode_tensor_map_3d_bf16(&mv, a.v, D, a.N, a.BH, 64, 64) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(sparse_attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM);
  if (e != cudaSuccess) return e;
  dim3 grid(a.nqb, a.BH);
  sparse_attn_kernel<D><<<grid, kThreads, L::SMEM, st>>>(mq, mk, mv, a);
  return cudaGetLastError();
}

cudaError_t launch_sparse_attn(const AttnArgs& a, cudaStream_t st) {
  if (a.nqb > 0x7FFFFFFF || a.BH > 65535) return cudaErrorInvalidValue;
  return a.d == 128 ? launch_d<128>(a, st) : launch_d<64>(a, st);
}

}  // namespace sa
