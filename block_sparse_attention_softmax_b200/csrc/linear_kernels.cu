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
// linear_out_kernel: persistent over the same tile list; stages S of the
//   current head in shared memory as a bf16 hi + lo pair (two MMAs recover ~16
//   mantissa bits); per 128-token tile: TMA Q and O_s, phi(Q) in place,
//   D[t, :] = phi(Q)[t, :] S in TMEM (double buffered), and an epilogue that
//   divides by phi(q_t) . z and blends with O_s.
#include "sa_internal.h"

namespace sa {

namespace lin {

constexpr int kLinTok = 128;       // tokens per tile (K extent of the state MMA)
constexpr int kLinThreads = 192;   // warp 0 TMA, warp 1 MMA, warps 2..5 math
constexpr int kLinStages = 3;

// phi(x) = elu(x) + 1, written branch-free: exp(min(x, 0)) + max(x, 0)
// (exactly x + 1 for x > 0, exp(x) otherwise).
__device__ __forceinline__ float phi_f(float x) {
  return fast_exp2(fminf(x, 0.f) * 1.4426950408889634f) + fmaxf(x, 0.f);
}

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
  static constexpr uint32_t OFF_Z = OFF_BAR + 256;            // [phases][D] fp32 (4096 floats)
  static constexpr uint32_t SMEM = OFF_Z + 4096 * 4 + 1024;
};

template <int D>
struct OutLayout {
  static constexpr uint32_t B_CHUNK = D * 128;               // D rows (K) x 64 columns of S
  static constexpr uint32_t B_BYTES = (D / 64) * B_CHUNK;    // one of hi / lo
  static constexpr uint32_t T_CHUNK = kLinTok * 128;         // 128 tokens x 64 features
  static constexpr uint32_t T_BYTES = (D / 64) * T_CHUNK;    // one Q or O_s tile
  static constexpr int NSTG = 2;          // Q and O_s stages with the blend
  static constexpr int NSTG_OL = 4;       // Q stages without it (O_l is staged in the consumed Q stage)
  static constexpr uint32_t OFF_B = 0;
  static constexpr uint32_t OFF_Q = 2 * B_BYTES;
  static constexpr uint32_t OFF_OS = OFF_Q + NSTG * T_BYTES;    // = Q stages 2, 3 without the blend
  static constexpr uint32_t OFF_DEN = OFF_OS + NSTG * T_BYTES;  // [NSTG_OL][4 parts][128 rows] fp32
  static constexpr int ZA_HEADS = 8;                              // z and alpha of up to 8 heads per CTA
  static constexpr uint32_t OFF_ZA = OFF_DEN + NSTG_OL * 4 * 128 * 4;  // [ZA_HEADS][2][D] fp32
  static constexpr uint32_t OFF_BAR = OFF_ZA + ZA_HEADS * 2 * D * 4;
  static constexpr uint32_t SMEM = OFF_BAR + 256 + 1024;
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
constexpr int kStateMathWarps = 16;
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
    constexpr int CG = kStateMathWarps / 4;            // column groups per lane quadrant
    const int quad = warp & 3, cgrp = (warp - 2) >> 2;
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
      const bool full_tile = tok0 + lin::kLinTok <= N;
#pragma unroll
      for (int tt = phase; tt < lin::kLinTok; tt += NP) {
        uint4* p = reinterpret_cast<uint4*>(kt + tt * 128);
        uint4 w = *p;
        uint32_t* u = reinterpret_cast<uint32_t*>(&w);
        if (full_tile || tok0 + tt < N) {
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
          w = make_uint4(0, 0, 0, 0);   // keys past N contribute nothing
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
        constexpr int HC = D / CG;       // columns per column group (32 or 16)
        {
          uint32_t r[32];
          const uint32_t ta = tm + ab * 128 + (static_cast<uint32_t>(quad * 32) << 16) + cgrp * HC;
          if (HC == 32) {
            tmem_ld32_wait(ta, r);
          } else {
            uint32_t r16[16];
            tmem_ld16_wait(ta, r16);
#pragma unroll
            for (int e = 0; e < 16; ++e) r[e] = r16[e];
          }
          if (frow < D) {
            float4* dst = reinterpret_cast<float4*>(out + frow * D + cgrp * HC);
#pragma unroll
            for (int e = 0; e < HC / 4; ++e)
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
// Persistent over the same head-major tile list as the state kernel. Per tile
// of 128 tokens: one warp loads Q by TMA; the math warps apply phi to Q in
// place and, four threads per token, form the denominator phi(q_t) . z; one
// thread issues D[t, :] = phi(Q)[t, :] S_hi + phi(Q)[t, :] S_lo (tcgen05, TMEM
// accumulator, double buffered); the math warps then divide and stage the
// output in shared memory, from where the store warp writes it by TMA.
//   BLEND    2 Q stages (freed by the MMA) and 2 O_s stages: the store warp
//            loads O_s into a stage, the math warps blend alpha O_s + (1 -
//            alpha) O_l over it, and the store warp writes it to O before
//            loading the next O_s into it.
//   !BLEND   O_l only, 4 Q stages: the math warps write O_l over the consumed
//            Q stage (the MMA that read it has completed), and the store warp
//            frees the stage for the next Q once its store has read it. The
//            deeper ring keeps two Q tiles in flight per SM.
// z and alpha of the CTA's heads sit in shared memory. The four warps that
// share TMEM lane quadrant w % 4 split the d columns.
constexpr int kOutMathWarps = 16;
constexpr int kOsWarp = 2 + kOutMathWarps;
constexpr int kOutThreads = 32 * (kOsWarp + 1);

template <int D>
__device__ __forceinline__ void build_head_operand(uint8_t* smem, const float* __restrict__ kv_state,
                                                   int bh, int tid, int nthreads) {
  using L = lin::OutLayout<D>;
  // S as bf16 hi + lo, MN-major with 128-B swizzle: element (row c, column e)
  // sits in chunk e/64, row c, 16-B unit ((e % 64) / 8) ^ (c % 8).
  const float* Sg = kv_state + static_cast<long long>(bh) * D * D;
  constexpr int UPR = D / 8;
  for (int i = tid; i < D * UPR; i += nthreads) {
    const int c = i / UPR, u = i % UPR;
    const float4 a = *reinterpret_cast<const float4*>(Sg + c * D + u * 8);
    const float4 b = *reinterpret_cast<const float4*>(Sg + c * D + u * 8 + 4);
    const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int e2 = 0; e2 < 4; ++e2) {
      const __nv_bfloat162 hb = __floats2bfloat162_rn(v[2 * e2], v[2 * e2 + 1]);
      const float2 hf = __bfloat1622float2(hb);
      hi[e2] = *reinterpret_cast<const uint32_t*>(&hb);
      lo[e2] = pack_bf16x2(v[2 * e2] - hf.x, v[2 * e2 + 1] - hf.y);
    }
    const uint32_t off = (u / 8) * L::B_CHUNK + c * 128 + (((u % 8) ^ (c % 8)) * 16);
    *reinterpret_cast<uint4*>(smem + L::OFF_B + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4*>(smem + L::OFF_B + L::B_BYTES + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
  }
  fence_proxy_async_smem();
}

template <int D, bool BLEND>
__global__ void __launch_bounds__(kOutThreads, 1)
    linear_out_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmOs,
                      const __grid_constant__ CUtensorMap tmO,
                      const float* __restrict__ kv_state, const float* __restrict__ ksum,
                      const float* __restrict__ alpha, int H, int N, lin::StateGeom geo) {
  using L = lin::OutLayout<D>;
  constexpr int NS = BLEND ? L::NSTG : L::NSTG_OL;   // Q stages (and, with the blend, O_s stages)
  constexpr bool blend = BLEND;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = lin::align1k(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* q_full = bars;                  // [NS] Q landed
  uint64_t* q_empty = bars + NS;            // [NS] Q stage free: MMA completed (blend) or O_l store read it
  uint64_t* os_full = bars + 2 * NS;        // [NS] O_s landed (blend only)
  uint64_t* o_ready = bars + 3 * NS;        // [NS] O written into the stage (math warps)
  uint64_t* phi_done = bars + 4 * NS;       // [NS] phi and denominators ready (math warps)
  uint64_t* acc_full = bars + 5 * NS;       // [2]
  uint64_t* acc_empty = acc_full + 2;       // [2] (math warps)
  uint64_t* b_ready = acc_empty + 2;        // operand of a new head built (math warps)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(b_ready + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* den = reinterpret_cast<float*>(smem + L::OFF_DEN);
  float* za = reinterpret_cast<float*>(smem + L::OFF_ZA);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * geo.tpc;
  const int t1 = min(geo.total, t0 + geo.tpc);
  const int n_tiles = max(0, t1 - t0);
  if (n_tiles == 0) return;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
      mbar_init(&os_full[s], 1);
      mbar_init(&o_ready[s], kOutMathWarps);
      mbar_init(&phi_done[s], kOutMathWarps);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kOutMathWarps);
    }
    mbar_init(b_ready, kOutMathWarps);
    *abort_flag = 0;
    fence_barrier_init();
  }
  // the state (and O_s) come from earlier kernels in the stream
  grid_dep_wait();
  grid_dep_trigger();
  build_head_operand<D>(smem, kv_state, t0 / geo.tph, threadIdx.x, blockDim.x);
  // z and alpha of this CTA's heads (from global memory if there are more
  // heads than slots)
  const int h_first = t0 / geo.tph;
  const int n_heads = (t1 - 1) / geo.tph - h_first + 1;
  const bool za_smem = n_heads <= L::ZA_HEADS;
  if (za_smem) {
    for (int i = threadIdx.x; i < n_heads * D; i += blockDim.x) {
      const int hh = i / D, c = i % D;
      za[(hh * 2) * D + c] = ksum[static_cast<long long>(h_first + hh) * D + c];
      za[(hh * 2 + 1) * D + c] = blend ? alpha[static_cast<long long>((h_first + hh) % H) * D + c] : 0.f;
    }
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
    // ------------------------------------------------------------ Q producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      int issued = 0;
      for (int i = 0; i < n_tiles; ++i) {
        const int s = i % NS;
        if (!mbar_wait(&q_empty[s], ((i / NS) & 1) ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(&q_full[s], L::T_BYTES);
        const int t = t0 + i;
        const int row = (t % geo.tph) * lin::kLinTok, bh = t / geo.tph;
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(smem + L::OFF_Q + s * L::T_BYTES + c * L::T_CHUNK, &tmQ, &q_full[s], c * 64, row, bh);
        issued = i + 1;
      }
      // loads still in flight after an early stop land before the CTA gives up its shared memory
      for (int k = 1; k <= NS && k <= issued; ++k) mbar_drain(&q_full[(issued - k) % NS], ((issued - k) / NS) & 1);
    }
  } else if (warp == kOsWarp && !BLEND) {
    // ------------------------------------------------------------ O_l stores from the Q stages
    if (lane == 0) {
      tma_prefetch_desc(&tmO);
      for (int j = 0; j < n_tiles; ++j) {
        const int s = j % NS;
        if (!mbar_wait(&o_ready[s], (j / NS) & 1, abort_flag)) break;
        const int t = t0 + j;
        const int row = (t % geo.tph) * lin::kLinTok, bh = t / geo.tph;
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_store_3d(&tmO, smem + L::OFF_Q + s * L::T_BYTES + c * L::T_CHUNK, c * 64, row, bh);
        bulk_commit();
        // every store but this one has read its stage: hand the previous stage back
        bulk_wait_read<1>();
        if (j > 0) mbar_arrive(&q_empty[(j - 1) % NS]);
      }
      bulk_wait_all();
    }
  } else if (warp == kOsWarp) {
    // ------------------------------------------------------------ O_s loads, O stores
    // Stage s of tile i: once the math warps have written O of tile i - NS
    // into it, store that tile by TMA, wait until the store has read the
    // stage, then load O_s of tile i.
    if (lane == 0) {
      if (blend) tma_prefetch_desc(&tmOs);
      tma_prefetch_desc(&tmO);
      auto store_tile = [&](int j) -> bool {
        const int s = j % NS;
        if (!mbar_wait(&o_ready[s], (j / NS) & 1, abort_flag)) return false;
        const int t = t0 + j;
        const int row = (t % geo.tph) * lin::kLinTok, bh = t / geo.tph;
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_store_3d(&tmO, smem + L::OFF_OS + s * L::T_BYTES + c * L::T_CHUNK, c * 64, row, bh);
        bulk_commit();
        return true;
      };
      bool ok = true;
      for (int i = 0; ok && i < n_tiles; ++i) {
        const int s = i % NS;
        if (i >= NS) {
          if (!(ok = store_tile(i - NS))) break;
          bulk_wait_read_all();
        }
        if (blend) {
          mbar_arrive_expect_tx(&os_full[s], L::T_BYTES);
          const int t = t0 + i;
          const int row = (t % geo.tph) * lin::kLinTok, bh = t / geo.tph;
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(smem + L::OFF_OS + s * L::T_BYTES + c * L::T_CHUNK, &tmOs, &os_full[s], c * 64, row, bh);
        } else {
          mbar_arrive(&os_full[s]);
        }
      }
      for (int j = n_tiles > NS ? n_tiles - NS : 0; ok && j < n_tiles; ++j) ok = store_tile(j);
      bulk_wait_all();
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, D, false, true);
      const uint32_t bhi = smem_u32(smem + L::OFF_B), blo = bhi + L::B_BYTES;
      int changes = 0;
      for (int i = 0; i < n_tiles; ++i) {
        const int s = i % NS, ab = i & 1;
        const int t = t0 + i;
        if (i > 0 && t / geo.tph != (t - 1) / geo.tph) {
          if (!mbar_wait(b_ready, changes & 1, abort_flag)) break;
          ++changes;
        }
        if (!mbar_wait(&phi_done[s], (i / NS) & 1, abort_flag)) break;
        if (!mbar_wait(&acc_empty[ab], ((i >> 1) & 1) ^ 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t qb = smem_u32(smem + L::OFF_Q + s * L::T_BYTES);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t a = sw128_desc(qb + (kk >> 2) * L::T_CHUNK + (kk & 3) * 32u, 16, 1024);
          umma_ss(tm + ab * 128, a, sw128_desc(bhi + kk * 2048u, L::B_CHUNK, 1024), idesc, kk > 0 ? 1u : 0u);
          umma_ss(tm + ab * 128, a, sw128_desc(blo + kk * 2048u, L::B_CHUNK, 1024), idesc, 1u);
        }
        tc_commit(&acc_full[ab]);
        if (BLEND) tc_commit(&q_empty[s]);
      }
    }
  } else {
    // ------------------------------------------------------------ math warps
    const int mt = threadIdx.x - 64;          // 0 .. 511
    const int quad = warp & 3, grp = (warp - 2) >> 2;   // column group 0..3 of this lane quadrant
    const int row = quad * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    constexpr int HC = D / 4;                 // output columns per group
    constexpr int HU = HC / 8;                // 16-B units per group of a row
    // transform mapping: token trow, four threads per token; thread tpart
    // takes units tpart and tpart + 4 of each 64-feature chunk, the even rows
    // of a quarter-warp in one order and the odd rows in the other, so that
    // the quarter-warp's eight 16-byte accesses fall in eight different bank
    // groups of the swizzled rows
    const int trow = mt >> 2, tpart = mt & 3;
    bool ok = true;
    int changes = 0;
    auto epilogue = [&](int j) -> bool {
      const int ab = j & 1, s = j % NS;
      const int t = t0 + j;
      const int bh = t / geo.tph;
      const int tok = (t % geo.tph) * lin::kLinTok + row;
      if (!mbar_wait(&acc_full[ab], (j >> 1) & 1, abort_flag)) return false;
      if (!mbar_wait(&phi_done[s], (j / NS) & 1, abort_flag)) return false;   // denominators visible
      if (BLEND && !mbar_wait(&os_full[s], (j / NS) & 1, abort_flag)) return false;   // O_s in, stage free
      tc_fence_after();
      uint32_t x0[32];
      if (HC == 32) {
        tmem_ld32_wait(tm + ab * 128 + lane_addr + grp * HC, x0);
      } else {
        uint32_t r16[16];
        tmem_ld16_wait(tm + ab * 128 + lane_addr + grp * HC, r16);
#pragma unroll
        for (int e = 0; e < 16; ++e) x0[e] = r16[e];
      }
      const float* dj = den + s * 4 * 128;
      const float inv = 1.f / ((dj[row] + dj[128 + row]) + (dj[256 + row] + dj[384 + row]));
      (void)tok;   // rows past N are clipped by the TMA store
      {
        // the output stage: O_s's (blend) or the consumed Q stage (O_l only)
        uint8_t* osrow = smem + (BLEND ? L::OFF_OS : L::OFF_Q) + s * L::T_BYTES;
        const float* al = za_smem ? za + ((bh - h_first) * 2 + 1) * D : alpha + static_cast<long long>(bh % H) * D;
#pragma unroll
        for (int j2 = 0; j2 < HU; ++j2) {
          const int uu = grp * HU + j2;
          uint4* slot = reinterpret_cast<uint4*>(osrow + (uu >> 3) * L::T_CHUNK + row * 128 + (((uu & 7) ^ (row & 7)) << 4));
          float l[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) l[e] = __uint_as_float(x0[j2 * 8 + e]) * inv;
          uint32_t pk[4];
          if (blend) {
            const uint4 w = *slot;
            const float4 a0 = *reinterpret_cast<const float4*>(al + uu * 8);
            const float4 a1 = *reinterpret_cast<const float4*>(al + uu * 8 + 4);
            const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float s0 = __uint_as_float(wv[e] << 16), s1 = __uint_as_float(wv[e] & 0xFFFF0000u);
              pk[e] = pack_bf16x2(fmaf(av[2 * e], s0 - l[2 * e], l[2 * e]), fmaf(av[2 * e + 1], s1 - l[2 * e + 1], l[2 * e + 1]));
            }
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) pk[e] = pack_bf16x2(l[2 * e], l[2 * e + 1]);
          }
          *slot = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      }
      fence_proxy_async_smem();     // O visible to the TMA store
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&acc_empty[ab]);
        mbar_arrive(&o_ready[s]);
      }
      return true;
    };
    for (int i = 0; ok && i < n_tiles; ++i) {
      const int s = i % NS;
      const int t = t0 + i;
      if (!(ok = mbar_wait(&q_full[s], (i / NS) & 1, abort_flag))) break;
      // the denominator slot of stage s is free once every warp has finished
      // the epilogue of tile i - NS
      if (i >= NS && !(ok = mbar_wait(&o_ready[s], ((i / NS) & 1) ^ 1, abort_flag))) break;
      // phi(Q) in place and the partial denominator of token trow
      {
        const float* zg = za_smem ? za + ((t / geo.tph - h_first) * 2) * D : ksum + static_cast<long long>(t / geo.tph) * D;
        uint8_t* qt = smem + L::OFF_Q + s * L::T_BYTES;
        float dz = 0.f;
#pragma unroll
        for (int j2 = 0; j2 < HU; ++j2) {
          const int uu = (j2 >> 1) * 8 + tpart + 4 * ((j2 & 1) ^ (trow & 1));
          uint4* p = reinterpret_cast<uint4*>(qt + (uu >> 3) * L::T_CHUNK + trow * 128 + (((uu & 7) ^ (trow & 7)) << 4));
          uint4 w = *p;
          uint32_t* x = reinterpret_cast<uint32_t*>(&w);
          const float4 z0 = *reinterpret_cast<const float4*>(zg + uu * 8);
          const float4 z1 = *reinterpret_cast<const float4*>(zg + uu * 8 + 4);
          const float zv[8] = {z0.x, z0.y, z0.z, z0.w, z1.x, z1.y, z1.z, z1.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint32_t pk = pack_bf16x2(lin::phi_f(__uint_as_float(x[e] << 16)), lin::phi_f(__uint_as_float(x[e] & 0xFFFF0000u)));
            x[e] = pk;
            dz = fmaf(__uint_as_float(pk << 16), zv[2 * e], dz);
            dz = fmaf(__uint_as_float(pk & 0xFFFF0000u), zv[2 * e + 1], dz);
          }
          *p = w;
        }
        den[s * 4 * 128 + tpart * 128 + trow] = dz;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&phi_done[s]);
      if (i > 0) {
        if (!(ok = epilogue(i - 1))) break;
        if (t / geo.tph != (t - 1) / geo.tph) {
          // every MMA of the previous head has completed (its last accumulator
          // was just read): rebuild the operand for this head
          build_head_operand<D>(smem, kv_state, t / geo.tph, mt, 32 * kOutMathWarps);
          __syncwarp();
          if (lane == 0) mbar_arrive(b_ready);
          if (!(ok = mbar_wait(b_ready, changes & 1, abort_flag))) break;
          ++changes;
        }
      }
    }
    if (ok) epilogue(n_tiles - 1);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tm, 256);
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
  const lin::StateGeom geo = lin::state_geom(BH, a.N, lin::sm_count());
  CUtensorMap mq, mos, mo;
  if (encode_tensor_map_3d_bf16(&mq, a.q, D, a.N, BH, 64, lin::kLinTok) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  const bool blend = a.o_s != nullptr;
  if (encode_tensor_map_3d_bf16(&mos, blend ? a.o_s : a.q, D, a.N, BH, 64, lin::kLinTok) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (encode_tensor_map_3d_bf16(&mo, a.o, D, a.N, BH, 64, lin::kLinTok) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  auto kern = blend ? linear_out_kernel<D, true> : linear_out_kernel<D, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(geo.grid), dim3(kOutThreads), L::SMEM, st, mq, mos, mo, a.kv_state, a.ksum,
                    blend ? a.alpha : nullptr, a.H, a.N, geo);
}

cudaError_t launch_linear_out(const LinearArgs& a, cudaStream_t st) {
  return a.d == 128 ? out_d<128>(a, st) : out_d<64>(a, st);
}

}  // namespace sa
