// linear_kernels.cu — the parallel linear-attention branch and the alpha blend
// on the sm_100a tensor cores (pages: "SALAD" §2.1, a linear-attention branch
// beside sparse attention over the same Q/K/V; "SLA2" 提案手法 ②,
// O = alpha ⊙ O_s + (1 - alpha) ⊙ O_l).
//
// phi(x) = elu(x) + 1. For each head:
//   state:  S = sum_j phi(k_j) v_j^T  [d, d],  z = sum_j phi(k_j)  [d]
//   output: O_l[i] = phi(q_i)^T S / phi(q_i)^T z
//   blend:  O[i]   = alpha ⊙ O_s[i] + (1 - alpha) ⊙ O_l[i]
//
// linear_state_kernel: persistent, one contiguous range of 128-token tiles per
//   CTA. K and V tiles arrive by TMA; eight warps apply phi to the K tile in
//   shared memory (rounding phi(k) to bf16) and sum z; one thread issues
//   tcgen05.mma D[f, e] += phi(K)^T[f, t] V[t, e] with both operands MN-major,
//   accumulating each head's share in TMEM. Per-(CTA, head) partials are
//   reduced in a fixed order.
// linear_out_kernel: each CTA stages [S | z] of its head in shared memory as a
//   bf16 hi + lo pair (two MMAs recover ~16 mantissa bits), then for each
//   128-token tile: TMA Q, phi in place, D[t, :] = phi(Q)[t, :] [S | z] in TMEM
//   (double buffered), and an epilogue that divides by the z column and blends
//   with O_s.
#include "sa_internal.h"

namespace sa {

namespace lin {

constexpr int kLinTok = 128;       // tokens per tile (K extent of the state MMA)
constexpr int kLinThreads = 192;   // warp 0 TMA, warp 1 MMA, warps 2..5 math
constexpr int kLinStages = 3;

__device__ __forceinline__ float phi_f(float x) { return x > 0.f ? x + 1.f : __expf(x); }

// Persistent geometry of the state kernel: the B*H*ceil(N/128) tiles, head
// after head, are cut into one contiguous range per CTA. A range spans at most
// `heads_per_cta` heads, each of which leaves one partial [S | z] slot.
struct StateGeom {
  int tph;            // tiles per head
  int total;          // tiles over all heads
  int grid;           // CTAs
  int tpc;            // tiles per CTA
  int hpc;            // partial slots per CTA
};

StateGeom state_geom(int BH, int N, int sms) {
  StateGeom g;
  g.tph = ceil_div(N, kLinTok);
  g.total = BH * g.tph;
  int grid = g.total < sms ? g.total : sms;
  g.tpc = ceil_div(g.total, grid);
  g.grid = ceil_div(g.total, g.tpc);
  g.hpc = ceil_div(g.tpc, g.tph) + 1;
  return g;
}

int sm_count() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

template <int D>
struct StateLayout {
  static constexpr uint32_t CHUNK = kLinTok * 128;               // 128 tokens x 64 features
  static constexpr uint32_t K_BYTES = 2 * CHUNK;              // A operand spans M = 128 features
  static constexpr uint32_t V_BYTES = (D / 64) * CHUNK;
  static constexpr uint32_t STAGE = K_BYTES + V_BYTES;
  static constexpr uint32_t OFF_BAR = kLinStages * STAGE;
  static constexpr uint32_t OFF_Z = OFF_BAR + 256;            // [phases][D] fp32 (2048 floats)
  static constexpr uint32_t SMEM = OFF_Z + 2048 * 4 + 1024;
};

template <int D>
struct OutLayout {
  static constexpr int NB = D + 16;                           // MMA N: S columns + z column
  static constexpr int B_CHUNKS = (NB + 63) / 64;
  static constexpr uint32_t B_CHUNK = D * 128;                // D rows (K) x 64 columns
  static constexpr uint32_t B_BYTES = B_CHUNKS * B_CHUNK;     // one of hi / lo
  static constexpr uint32_t Q_CHUNK = kLinTok * 128;
  static constexpr uint32_t Q_BYTES = (D / 64) * Q_CHUNK;
  static constexpr uint32_t OFF_B = 0;
  static constexpr uint32_t OFF_Q = 2 * B_BYTES;
  static constexpr uint32_t OFF_ALPHA = OFF_Q + kLinStages * Q_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_ALPHA + D * 4;
  static constexpr uint32_t SMEM = OFF_BAR + 256 + 1024;
  static constexpr uint32_t ACC_STRIDE = NB <= 128 ? 128 : 256;   // TMEM columns per buffer
  static constexpr uint32_t TM_COLS = 2 * ACC_STRIDE;
};

__device__ __forceinline__ uint8_t* align1k(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

}  // namespace lin

size_t linear_state_ws_bytes(int BH, int N, int d) {
  const lin::StateGeom g = lin::state_geom(BH, N, lin::sm_count());
  return static_cast<size_t>(g.grid) * g.hpc * (static_cast<size_t>(d) * d + d) * sizeof(float);
}

size_t linear_out_ws_bytes(int, int) { return 0; }

// ---------------------------------------------------------------- state
// Persistent: CTA c owns tiles [c*tpc, min(total, (c+1)*tpc)) of the head-major
// tile list. Warp 0 loads K and V tiles (TMA, 3 stages), warps 2..9 apply phi
// to K in shared memory and sum z, warp 1 issues the MMAs into one of two TMEM
// accumulators per head segment; when a segment (the CTA's share of one head)
// ends, the math warps copy its S and z into a partial slot while the next
// segment accumulates into the other buffer.
constexpr int kStateMathWarps = 8;
constexpr int kStateThreads = 64 + 32 * kStateMathWarps;

template <int D>
__global__ void __launch_bounds__(kStateThreads, 1)
    linear_state_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                        int N, lin::StateGeom geo, float* __restrict__ part) {
  using L = lin::StateLayout<D>;
  constexpr int NS = lin::kLinStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = lin::align1k(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* full = bars;                 // [NS] TMA landed
  uint64_t* phi_done = bars + NS;        // [NS] phi applied (math warps)
  uint64_t* empty = bars + 2 * NS;       // [NS] MMA consumed
  uint64_t* acc_full = bars + 3 * NS;    // [2] segment accumulated
  uint64_t* acc_empty = acc_full + 2;    // [2] segment copied out
  uint64_t* zs_full = acc_empty + 2;     // z partials of a segment written (math warps)
  uint64_t* zs_free = zs_full + 1;       // z partials of a segment read (math warps)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(zs_free + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* zs = reinterpret_cast<float*>(smem + L::OFF_Z);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * geo.tpc;
  const int t1 = min(geo.total, t0 + geo.tpc);
  const int n_tiles = max(0, t1 - t0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&phi_done[s], kStateMathWarps);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kStateMathWarps);
    }
    mbar_init(zs_full, kStateMathWarps);
    mbar_init(zs_free, kStateMathWarps);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (D == 64) {
    // the A operand always spans 128 features: zero the upper half once
    for (int s = 0; s < NS; ++s)
      for (int i = threadIdx.x; i < static_cast<int>(L::CHUNK / 16); i += blockDim.x)
        reinterpret_cast<uint4*>(smem + s * L::STAGE + L::CHUNK)[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
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
    if (lane == 0 && n_tiles > 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      for (int i = 0; i < n_tiles; ++i) {
        const int s = i % NS;
        if (!mbar_wait(&empty[s], ((i / NS) & 1) ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(&full[s], (D / 64) * 2 * L::CHUNK);
        uint8_t* st = smem + s * L::STAGE;
        const int t = t0 + i;
        const int row = (t % geo.tph) * lin::kLinTok;
        const int bh = t / geo.tph;
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          tma_load_3d(st + c * L::CHUNK, &tmK, &full[s], c * 64, row, bh);
          tma_load_3d(st + L::K_BYTES + c * L::CHUNK, &tmV, &full[s], c * 64, row, bh);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && n_tiles > 0) {
      const uint32_t idesc = idesc_bf16_f32(128, D, true, true);
      int seg = 0;
      bool first = true;
      for (int i = 0; i < n_tiles; ++i) {
        const int s = i % NS;
        const int t = t0 + i;
        const int ab = seg & 1;
        if (first && seg >= 2 && !mbar_wait(&acc_empty[ab], ((seg >> 1) & 1) ^ 1, abort_flag)) break;
        if (!mbar_wait(&phi_done[s], (i / NS) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t kb = smem_u32(smem + s * L::STAGE);
        const uint32_t vb = kb + L::K_BYTES;
#pragma unroll
        for (int kk = 0; kk < lin::kLinTok / 16; ++kk) {
          const uint64_t a = sw128_desc(kb + kk * 2048u, L::CHUNK, 1024);
          const uint64_t b = sw128_desc(vb + kk * 2048u, L::CHUNK, 1024);
          umma_ss(tm + ab * 128, a, b, idesc, (!first || kk > 0) ? 1u : 0u);
        }
        tc_commit(&empty[s]);
        first = false;
        if (t + 1 == t1 || (t + 1) % geo.tph == 0) {
          tc_commit(&acc_full[ab]);
          ++seg;
          first = true;
        }
      }
    }
  } else {
    // math warps: phi on the K tile, z sums; segment ends copy S and z out
    constexpr int NG = D / 8;                          // 8-feature groups
    constexpr int NP = 32 * kStateMathWarps / NG;      // token phases
    const int mt = threadIdx.x - 64;
    const int gi = mt % NG, phase = mt / NG;
    const int chunk = gi / 8, lu = gi % 8;
    const int pu = lu ^ (phase % 8);     // physical 16-B unit (t % 8 == phase % 8 for every visited token)
    const int quad = warp & 3, half = (warp - 2) >> 2;
    const int frow = quad * 32 + lane;   // TMEM lane = feature row of phi(K)^T
    float z[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) z[e] = 0.f;
    bool ok = true;
    int seg = 0;
    for (int i = 0; i < n_tiles; ++i) {
      const int s = i % NS;
      const int t = t0 + i;
      if (!mbar_wait(&full[s], (i / NS) & 1, abort_flag)) { ok = false; break; }
      uint8_t* kt = smem + s * L::STAGE + chunk * L::CHUNK + pu * 16;
      const int tok0 = (t % geo.tph) * lin::kLinTok;
#pragma unroll 4
      for (int tt = phase; tt < lin::kLinTok; tt += NP) {
        uint4* p = reinterpret_cast<uint4*>(kt + tt * 128);
        uint4 w = *p;
        uint32_t* u = reinterpret_cast<uint32_t*>(&w);
        if (tok0 + tt < N) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float a = lin::phi_f(__uint_as_float(u[e] << 16));
            const float b = lin::phi_f(__uint_as_float(u[e] & 0xFFFF0000u));
            const uint32_t pk = pack_bf16x2(a, b);
            u[e] = pk;
            z[2 * e] += __uint_as_float(pk << 16);
            z[2 * e + 1] += __uint_as_float(pk & 0xFFFF0000u);
          }
        } else {
          w = make_uint4(0, 0, 0, 0);
        }
        *p = w;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&phi_done[s]);
      if (t + 1 == t1 || (t + 1) % geo.tph == 0) {
        // ---- segment end: partial slot (blockIdx.x, seg)
        float* out = part + (static_cast<long long>(blockIdx.x) * geo.hpc + seg) * (D * D + D);
        // z: every warp writes its phases, all read once every warp has written
        if (seg >= 1 && !mbar_wait(zs_free, (seg - 1) & 1, abort_flag)) { ok = false; break; }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          zs[phase * D + gi * 8 + e] = z[e];
          z[e] = 0.f;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(zs_full);
        if (!mbar_wait(zs_full, seg & 1, abort_flag)) { ok = false; break; }
        if (mt < D) {
          float acc = 0.f;
          for (int ph = 0; ph < NP; ++ph) acc += zs[ph * D + mt];
          out[D * D + mt] = acc;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(zs_free);
        const int ab = seg & 1;
        if (!mbar_wait(&acc_full[ab], (seg >> 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        constexpr int HC = D / 2;        // columns per half
#pragma unroll
        for (int c0 = 0; c0 < HC; c0 += 32) {
          uint32_t r[32];
          tmem_ld32_wait(tm + ab * 128 + (static_cast<uint32_t>(quad * 32) << 16) + half * HC + c0, r);
          if (frow < D) {
            float4* dst = reinterpret_cast<float4*>(out + frow * D + half * HC + c0);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              dst[e] = make_float4(__uint_as_float(r[4 * e]), __uint_as_float(r[4 * e + 1]),
                                   __uint_as_float(r[4 * e + 2]), __uint_as_float(r[4 * e + 3]));
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[ab]);
        ++seg;
      }
    }
    (void)ok;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tm, 256);
  }
}

// Head h's partial slots, summed in CTA order.
template <int D>
__global__ void linear_reduce_kernel(const float* __restrict__ part, lin::StateGeom geo,
                                     float* __restrict__ kv_state, float* __restrict__ ksum) {
  const int h = blockIdx.y;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= D * D + D) return;
  const int c_first = (h * geo.tph) / geo.tpc;
  const int c_last = ((h + 1) * geo.tph - 1) / geo.tpc;
  float acc = 0.f;
  for (int c = c_first; c <= c_last; ++c) {
    const int seg = h - (c * geo.tpc) / geo.tph;
    acc += part[(static_cast<long long>(c) * geo.hpc + seg) * (D * D + D) + e];
  }
  if (e < D * D) kv_state[static_cast<long long>(h) * D * D + e] = acc;
  else ksum[static_cast<long long>(h) * D + (e - D * D)] = acc;
}

// ---------------------------------------------------------------- output + blend
template <int D>
__global__ void __launch_bounds__(lin::kLinThreads, 1)
    linear_out_kernel(const __grid_constant__ CUtensorMap tmQ, const float* __restrict__ kv_state,
                      const float* __restrict__ ksum, const uint16_t* __restrict__ o_s,
                      const float* __restrict__ alpha, int H, int N, int tiles_per_cta,
                      uint16_t* __restrict__ o) {
  using L = lin::OutLayout<D>;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = lin::align1k(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* full = bars;                    // [lin::kLinStages]
  uint64_t* phi_done = bars + lin::kLinStages;      // [lin::kLinStages]
  uint64_t* empty = bars + 2 * lin::kLinStages;     // [lin::kLinStages]
  uint64_t* acc_full = bars + 3 * lin::kLinStages;  // [2]
  uint64_t* acc_empty = acc_full + 2;       // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* al = reinterpret_cast<float*>(smem + L::OFF_ALPHA);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int h = bh % H;
  const int tile0 = blockIdx.x * tiles_per_cta;
  const int n_tiles = max(0, min(tiles_per_cta, ceil_div_dev(N, lin::kLinTok) - tile0));

  if (threadIdx.x == 0) {
    for (int s = 0; s < lin::kLinStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&phi_done[s], 4);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  // B operand [S | z] as bf16 hi and lo, MN-major with 128-B swizzle:
  // element (row c, column e) sits in chunk e/64, row c, 16-B unit ((e%64)/8) ^ (c%8).
  {
    const float* Sg = kv_state + static_cast<long long>(bh) * D * D;
    const float* zg = ksum + static_cast<long long>(bh) * D;
    constexpr int UPR = L::B_CHUNKS * 8;    // 16-B units per row (incl. zero padding)
    for (int i = threadIdx.x; i < D * UPR; i += blockDim.x) {
      const int c = i / UPR, u = i % UPR;
      uint32_t hi[4], lo[4];
#pragma unroll
      for (int e2 = 0; e2 < 4; ++e2) {
        float v2[2];
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const int e = u * 8 + e2 * 2 + t;
          v2[t] = e < D ? Sg[c * D + e] : (e == D ? zg[c] : 0.f);
        }
        const __nv_bfloat162 hb = __floats2bfloat162_rn(v2[0], v2[1]);
        const float2 hf = __bfloat1622float2(hb);
        hi[e2] = *reinterpret_cast<const uint32_t*>(&hb);
        lo[e2] = pack_bf16x2(v2[0] - hf.x, v2[1] - hf.y);
      }
      const uint32_t off = (u / 8) * L::B_CHUNK + c * 128 + (((u % 8) ^ (c % 8)) * 16);
      *reinterpret_cast<uint4*>(smem + L::OFF_B + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<uint4*>(smem + L::OFF_B + L::B_BYTES + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
    for (int e = threadIdx.x; e < D; e += blockDim.x) al[e] = alpha ? alpha[static_cast<long long>(h) * D + e] : 0.f;
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *tmem_slot;

  if (warp == 0) {
    if (lane == 0 && n_tiles > 0) {
      tma_prefetch_desc(&tmQ);
      for (int i = 0; i < n_tiles; ++i) {
        const int s = i % lin::kLinStages;
        if (!mbar_wait(&empty[s], ((i / lin::kLinStages) & 1) ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(&full[s], L::Q_BYTES);
        uint8_t* st = smem + L::OFF_Q + s * L::Q_BYTES;
#pragma unroll
        for (int c = 0; c < D / 64; ++c) tma_load_3d(st + c * L::Q_CHUNK, &tmQ, &full[s], c * 64, (tile0 + i) * lin::kLinTok, bh);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && n_tiles > 0) {
      const uint32_t idesc = idesc_bf16_f32(128, L::NB, false, true);
      const uint32_t bhi = smem_u32(smem + L::OFF_B), blo = bhi + L::B_BYTES;
      for (int i = 0; i < n_tiles; ++i) {
        const int s = i % lin::kLinStages, b = i & 1;
        if (!mbar_wait(&phi_done[s], (i / lin::kLinStages) & 1, abort_flag)) break;
        if (!mbar_wait(&acc_empty[b], ((i >> 1) & 1) ^ 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t qb = smem_u32(smem + L::OFF_Q + s * L::Q_BYTES);
        const uint32_t d_tm = tm + b * L::ACC_STRIDE;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t a = sw128_desc(qb + (kk >> 2) * L::Q_CHUNK + (kk & 3) * 32u, 16, 1024);
          umma_ss(d_tm, a, sw128_desc(bhi + kk * 2048u, L::B_CHUNK, 1024), idesc, kk > 0 ? 1u : 0u);
          umma_ss(d_tm, a, sw128_desc(blo + kk * 2048u, L::B_CHUNK, 1024), idesc, 1u);
        }
        tc_commit(&acc_full[b]);
        tc_commit(&empty[s]);
      }
    }
  } else {
    const int mt = threadIdx.x - 64;
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    bool ok = true;
    auto epilogue = [&](int i) {
      const int b = i & 1;
      if (!mbar_wait(&acc_full[b], (i >> 1) & 1, abort_flag)) { ok = false; return; }
      tc_fence_after();
      const int tok = (tile0 + i) * lin::kLinTok + row;
      uint32_t dz[32];
      tmem_ld32_wait(tm + lane_addr + b * L::ACC_STRIDE + D, dz);
      const float inv = 1.f / __uint_as_float(dz[0]);
      const long long base = (static_cast<long long>(bh) * N + tok) * D;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t r[32];
        tmem_ld32_wait(tm + lane_addr + b * L::ACC_STRIDE + c0, r);
        if (tok < N) {
          uint32_t pk[16];
          if (o_s) {
            const uint4* src = reinterpret_cast<const uint4*>(o_s + base + c0);
            uint32_t os[16];
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4) {
              const uint4 w = src[v4];
              os[4 * v4] = w.x; os[4 * v4 + 1] = w.y; os[4 * v4 + 2] = w.z; os[4 * v4 + 3] = w.w;
            }
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float a0 = al[c0 + 2 * e], a1 = al[c0 + 2 * e + 1];
              const float l0 = __uint_as_float(r[2 * e]) * inv, l1 = __uint_as_float(r[2 * e + 1]) * inv;
              const float s0 = __uint_as_float(os[e] << 16), s1 = __uint_as_float(os[e] & 0xFFFF0000u);
              pk[e] = pack_bf16x2(fmaf(a0, s0 - l0, l0), fmaf(a1, s1 - l1, l1));
            }
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e)
              pk[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * inv, __uint_as_float(r[2 * e + 1]) * inv);
          }
          uint4* dst = reinterpret_cast<uint4*>(o + base + c0);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) dst[v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);
    };
    for (int i = 0; i < n_tiles && ok; ++i) {
      const int s = i % lin::kLinStages;
      if (!mbar_wait(&full[s], (i / lin::kLinStages) & 1, abort_flag)) { ok = false; break; }
      // phi in place: elementwise, so the swizzled layout does not matter
      uint4* qt = reinterpret_cast<uint4*>(smem + L::OFF_Q + s * L::Q_BYTES);
#pragma unroll 4
      for (int u = mt; u < static_cast<int>(L::Q_BYTES / 16); u += 128) {
        uint4 w = qt[u];
        uint32_t* x = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
        for (int e = 0; e < 4; ++e)
          x[e] = pack_bf16x2(lin::phi_f(__uint_as_float(x[e] << 16)), lin::phi_f(__uint_as_float(x[e] & 0xFFFF0000u)));
        qt[u] = w;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&phi_done[s]);
      if (i > 0) epilogue(i - 1);
    }
    if (ok && n_tiles > 0) epilogue(n_tiles - 1);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tm, L::TM_COLS);
  }
}

// ---------------------------------------------------------------- launchers
template <int D>
static cudaError_t state_d(const LinearArgs& a, cudaStream_t st) {
  using L = lin::StateLayout<D>;
  const int BH = a.B * a.H;
  const lin::StateGeom geo = lin::state_geom(BH, a.N, lin::sm_count());
  CUtensorMap mk, mv;
  if (encode_tensor_map_3d_bf16(&mk, a.k, D, a.N, BH, 64, lin::kLinTok) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  if (encode_tensor_map_3d_bf16(&mv, a.v, D, a.N, BH, 64, lin::kLinTok) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(linear_state_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM);
  if (e != cudaSuccess) return e;
  float* part = static_cast<float*>(a.ws);
  linear_state_kernel<D><<<geo.grid, kStateThreads, L::SMEM, st>>>(mk, mv, a.N, geo, part);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int n = D * D + D;
  linear_reduce_kernel<D><<<dim3(ceil_div(n, 256), BH), 256, 0, st>>>(part, geo, a.kv_state, a.ksum);
  return cudaGetLastError();
}

cudaError_t launch_linear_state(const LinearArgs& a, cudaStream_t st) {
  return a.d == 128 ? state_d<128>(a, st) : state_d<64>(a, st);
}

template <int D>
static cudaError_t out_d(const LinearArgs& a, cudaStream_t st) {
  using L = lin::OutLayout<D>;
  const int BH = a.B * a.H;
  const int tiles = ceil_div(a.N, lin::kLinTok);
  const int ctas_per_head = max(1, min(tiles, ceil_div(4 * 148, BH)));
  const int tpc = ceil_div(tiles, ctas_per_head);
  CUtensorMap mq;
  if (encode_tensor_map_3d_bf16(&mq, a.q, D, a.N, BH, 64, lin::kLinTok) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(linear_out_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM);
  if (e != cudaSuccess) return e;
  linear_out_kernel<D><<<dim3(ceil_div(tiles, tpc), BH), lin::kLinThreads, L::SMEM, st>>>(
      mq, a.kv_state, a.ksum, static_cast<const uint16_t*>(a.o_s), a.alpha, a.H, a.N, tpc,
      static_cast<uint16_t*>(a.o));
  return cudaGetLastError();
}

cudaError_t launch_linear_out(const LinearArgs& a, cudaStream_t st) {
  return a.d == 128 ? out_d<128>(a, st) : out_d<64>(a, st);
}

}  // namespace sa
