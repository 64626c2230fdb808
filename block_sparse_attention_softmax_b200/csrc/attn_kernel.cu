// attn_kernel.cu — block-sparse attention forward for sm_100a
// (page: "SpargeAttention2" §2(3): FlashAttention-based block-sparse kernel that
// skips the masked QK^T and softmax/PV work; Veda §2.3 describes a
// producer/consumer split with TMA fetches of non-contiguous K/V tiles).
//
// Persistent kernel: one CTA per SM walks work items (head, 128-row query
// tile) round-robin in head-major order, so concurrently running CTAs share
// the K/V blocks of one head in L2. Inside an item, two 64-key blocks from the
// item's kept list form one 128-key tile.
//
// The per-tile chain QK(g) -> softmax(g) -> PV(g) is what limits this kernel,
// so the tensor core is kept fed from three S buffers (QK can run up to three
// tiles ahead of PV) and by two MMA-issuing threads: a thread that issues
// tcgen05.mma stalls while the tensor pipe's short queue is full, and its
// mbarrier waits and commits queue behind its own MMAs, so with one thread
// the pipe idles between MMA groups. With one thread for QK and one for PV the
// waits of one overlap the MMAs of the other (measured on B200: dense 1.3B-480p
// attention 1022 -> 1188 TFLOP/s). The QK that overwrites an S buffer waits for
// the P V that read P from it.
//
//   warp 0       TMA producer of Q (two slots, so the next item's Q loads
//                while the current item runs) and K (2-stage ring; a slot is
//                free once the QK that read it has completed, the event that
//                also fills that tile's S buffer)
//   warp 10      TMA producer of V (2-stage ring; a slot is free once the P V
//                that read it has completed); one TMA box per 64-key block,
//                so the two blocks of a tile need not be adjacent. It also
//                runs the O buffer: once per item, after the item's first two
//                V tiles, it stores the previous item's O (staged by the
//                softmax warps) by TMA, waits until the store has read the
//                buffer, and loads this item's O_l into it (with the blend)
//   warp 1       TMEM allocation and the thread issuing
//                  S_g = Q K_g^T  (A = Q, B = K, both from shared memory)
//   warp 11      the thread issuing
//                  O  += P_g V_g  (A = P_g from TMEM, B = V from shared memory)
//   warps 2..9   softmax: TMEM lane quadrant q = warp % 4 holds query rows
//                32q..32q+31; warp w takes lanes 32q..32q+15 and warp w+4
//                lanes 32q+16..32q+31, each with all 128 columns of a tile,
//                through the 16-lane forms of tcgen05.ld/st: four threads of
//                a warp share a row (32 columns each) and combine its max
//                with two shuffles, so no warp ever waits for another inside
//                the softmax. The running max m is kept in the log2 domain and
//                only raised when a tile's max exceeds it by more than 8
//                (P <= 256 otherwise); then O is rescaled in TMEM.
//                P = exp2(S*scale*log2e - m) is written back over the first
//                64 columns of S as packed bf16. At the end of an item the
//                warps sum the row's four shares of l with two shuffles,
//                copy O to registers, release it, and write O / l as bf16 and
//                the row log-sum-exp. O / l is written as bf16 into the O
//                buffer in shared memory (the TMA store's 128-byte swizzled
//                layout, conflict-free for the 16-lane layout), and warp 10
//                stores it while the next item runs: the softmax warps issue
//                no global loads or stores for O. With the linear branch the
//                epilogue blends while O_s is still fp32, O = alpha ⊙ O_s +
//                (1 - alpha) ⊙ O_l (SLA2 提案手法 ②), reading O_l from the same
//                bytes it overwrites: one bf16 rounding of O. A warp whose
//                bounded wait runs out stops; the others learn of it through
//                their own bounded waits (no named barrier is shared).
//
// Low-bit form (F8 = true; SLA2 提案手法 ③, a forward on low-bit queries, keys
// and values): Q, K and V arrive as E4M3 bytes with one fp32 scale per (batch,
// head) each. Both products run as tcgen05.mma kind::f8f6f4 (32 bytes of K per
// instruction, half the instructions of bf16); the softmax folds scale * s_q *
// s_k into its per-item exponent factor, P is written over S as E4M3 (P <= 256
// < 448, so it needs no scale of its own), and the epilogue multiplies by s_v.
// Its softmax keeps the earlier split of each row between two warps with a
// per-tile max exchange (see that branch): four E4M3 keys share a TMEM column,
// and in the 16-lane layout they would lie in two threads.
// Item facts carry the two factors, posted by the K producer with the rest.
//
// TMEM columns: S buffers at 0, 128 and 256 (fp32, 128 wide; P aliases their
// first 64 columns, 32 in the low-bit form), O at 384 (d wide). Shared memory:
// two Q slots, two K and two V stages, and the O buffer (128 rows x d bf16). Every mbarrier wait is bounded (see
// sa_device.cuh), and a CTA that stops early waits (bounded) for the TMA loads
// and MMAs it has issued before it gives up shared and tensor memory.
#include "sa_internal.h"

namespace sa {

namespace attn {

constexpr int kBM = 128;        // query rows per tile
constexpr int kBN = 128;        // keys per tile (two 64-key blocks)
constexpr int kSoftWarps = 8;
constexpr int kQSlots = 2;      // Q of the next item loads while the current one runs
constexpr int kItemRing = 4;    // item facts the K producer posts ahead of the softmax warps
constexpr int kKStages = 2;
constexpr int kVStages = 2;
constexpr int kSBufs = 3;
// Column pairs c (of 32 per thread and tile) with bit (c % 8) set take the
// FMA-pipe exponential instead of MUFU ex2: one pair in four. Measured on B200
// with two MMA issuers, where the softmax sets the pace: fastest of 0, 1, 2, 3
// and 4 pairs in 8 (the polynomial costs 10 issue slots per pair, MUFU costs
// pipe time), both in short runs and under the power cap.
constexpr uint32_t kPolyPairs = 0x88u;
constexpr int kVWarp = 2 + kSoftWarps;               // warp index of the V producer
constexpr int kPVWarp = kVWarp + 1;                  // warp index of the P V issuer
constexpr int kThreads = 32 * (kPVWarp + 1);

constexpr int kRingWords = 8;   // item facts: item, count, tail, then the low-bit factors

template <int D, bool F8 = false>
struct Layout {
  static constexpr int ES = F8 ? 1 : 2;                    // bytes per element of Q, K and V
  static constexpr int NCH = D * ES / 128;                 // 128-byte chunks along d
  static constexpr int CH_ELEMS = 128 / ES;                // elements per chunk
  static constexpr int KSTEP = 32 / ES;                    // K elements per MMA instruction (32 bytes)
  static constexpr uint32_t Q_BYTES = kBM * D * ES;
  static constexpr uint32_t TILE_BYTES = kBN * D * ES;      // one K or V tile
  static constexpr uint32_t BLK_BYTES = 64 * D * ES;        // one 64-key block
  static constexpr uint32_t Q_CHUNK = kBM * 128;            // bytes per d-chunk of Q
  static constexpr uint32_t KV_CHUNK = kBN * 128;           // bytes per d-chunk of K/V
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = OFF_Q + kQSlots * Q_BYTES;
  static constexpr uint32_t OFF_V = OFF_K + kKStages * TILE_BYTES;
  static constexpr uint32_t OB_CHUNK = kBM * 128;            // bytes per 64-column chunk of the O buffer
  static constexpr int NCH_O = D * 2 / 128;                  // 64-column chunks of a bf16 O row
  static constexpr uint32_t OFF_OB = OFF_V + kVStages * TILE_BYTES;
  static constexpr uint32_t OFF_RED = OFF_OB + NCH_O * OB_CHUNK;
  // row max [2][2][128], row sum [2][128], pair flags [4][16] of the E4M3 form's exchange
  static constexpr uint32_t RED_BYTES = F8 ? (2 * 2 + 2) * kBM * 4 + 4 * 16 * 4 : 0;
  static constexpr uint32_t OFF_BAR = OFF_RED + RED_BYTES;
  static constexpr uint32_t OFF_RING = OFF_BAR + 512;    // item ring [kItemRing][kRingWords] int
  static_assert(kItemRing * kRingWords * 4 <= 256, "item ring region");
  static_assert(NCH >= 1, "the low-bit form needs d = 128");
  static constexpr uint32_t USED = OFF_RING + 256;
  // at least 120 KB so that a second CTA never shares the SM (all 512 TMEM columns are held)
  static constexpr uint32_t SMEM = (USED + 1024 > 120 * 1024) ? USED + 1024 : 120 * 1024;
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
};

__host__ __device__ constexpr uint32_t tm_s(int b) { return static_cast<uint32_t>(b) * 128u; }
constexpr uint32_t TM_O = 384;
constexpr uint32_t TM_COLS = 512;

static_assert(kKStages <= kSBufs, "a K slot is freed by the S_FULL commit of the tile kKStages back");

enum {
  B_QFULL = 0,                       // [kQSlots] Q tile landed in shared memory
  B_QEMPTY = B_QFULL + kQSlots,      // [kQSlots] last QK of the item completed
  B_KFULL = B_QEMPTY + kQSlots,      // [kKStages]
  B_VFULL = B_KFULL + kKStages,      // [kVStages]
  B_SFULL = B_VFULL + kVStages,      // [kSBufs]
  B_PFULL = B_SFULL + kSBufs,        // [kSBufs]
  B_PVDONE = B_PFULL + kSBufs,       // [kSBufs] P V of the tile held in that S buffer completed:
                                     // the S buffer and the tile's V slot are free again
  B_OFULL = B_PVDONE + kSBufs,       // last P V of the item completed
  B_OEMPTY = B_OFULL + 1,            // epilogue has copied O out of TMEM
  B_OREADY = B_OEMPTY + 1,           // O buffer free of the previous item's O (its store has read
                                     // it) and, with the blend, holding this item's O_l
  B_OSTAGED = B_OREADY + 1,          // softmax warps have written this item's O into the buffer
  B_IFULL = B_OSTAGED + 1,           // [kItemRing] item facts posted by the K producer
  B_IEMPTY = B_IFULL + kItemRing,    // [kItemRing] item facts read by the softmax warps
  B_DRAIN = B_IEMPTY + kItemRing,    // [2] each MMA thread's last commit (early exit)
  B_COUNT = B_DRAIN + 2
};

// Word a softmax warp of the E4M3 form posts in place of its row max or row
// sum when its wait failed: a NaN whose payload no arithmetic produces.
constexpr uint32_t kStopBits = 0x7FC0DEADu;

// Named barrier of the two softmax warps of one TMEM lane quadrant (E4M3 form);
// shared memory written before it by either warp is visible to both after it.
__device__ __forceinline__ void pair_sync(int bar_id) {
  asm volatile("bar.sync %0, 64;" ::"r"(bar_id) : "memory");
}

// Both warps of a pair post whether their wait succeeded and meet; true only
// if both did. slot[half] is this warp's word, slot[half ^ 1] the partner's.
__device__ __forceinline__ bool pair_agree(int bar_id, volatile int* slot, int half, bool ok) {
  slot[half] = ok ? 1 : 0;
  pair_sync(bar_id);
  return ok && slot[half ^ 1] != 0;
}

// Per-item facts every role derives the same way.
struct Item {
  int bh, qb, cnt, T;
  bool tail;     // the last kept block is the ragged last key block
};

// Kept-block count of list row r, clamped to [0, n_kb] so that a malformed
// count cannot send any role past the end of its row of kv_idx (every role
// reads the count through here, so all of them agree on it).
__device__ __forceinline__ int kept_count(const AttnArgs& a, long long r) {
  return min(max(__ldg(a.kv_cnt + r), 0), a.nkb);
}

__device__ __forceinline__ Item load_item(const AttnArgs& a, int item) {
  Item it;
  it.bh = item / a.nqb;
  it.qb = item % a.nqb;
  const bool ragged = (a.N % 64) != 0;
  if (a.dense) {
    it.cnt = a.nkb;
    it.tail = ragged;
  } else {
    const long long r = static_cast<long long>(it.bh) * a.nqb + it.qb;
    it.cnt = kept_count(a, r);
    it.tail = ragged && it.cnt > 0 && __ldg(a.kv_idx + r * a.nkb + it.cnt - 1) == a.nkb - 1;
  }
  it.T = (it.cnt + 1) >> 1;
  return it;
}

// First item at or after `item` (stepping by `stride`) with at least one tile.
__device__ __forceinline__ int next_nonempty(const AttnArgs& a, int item, int stride, int n_items) {
  for (; item < n_items; item += stride)
    if (load_item(a, item).T > 0) break;
  return item;
}

}  // namespace attn

template <int D, bool F8>
__global__ void __launch_bounds__(attn::kThreads, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV,
                       const __grid_constant__ CUtensorMap tmO,
                       const __grid_constant__ CUtensorMap tmOL, AttnArgs a) {
  using namespace attn;
  using L = Layout<D, F8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + L::OFF_Q;
  uint8_t* sK = smem + L::OFF_K;
  uint8_t* sV = smem + L::OFF_V;
  uint8_t* sOB = smem + L::OFF_OB;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  static_assert(B_COUNT * 8 + 8 <= 512, "barrier region");
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + B_COUNT);
  // [kItemRing][item, cnt, tail, exponent factor, value factor, -, -, -]
  volatile int* item_ring = reinterpret_cast<volatile int*>(smem + L::OFF_RING);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_items = a.BH * a.nqb;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kQSlots; ++i) {
      mbar_init(&bars[B_QFULL + i], 1);
      mbar_init(&bars[B_QEMPTY + i], 1);
    }
    for (int i = 0; i < kItemRing; ++i) {
      mbar_init(&bars[B_IFULL + i], 1);
      mbar_init(&bars[B_IEMPTY + i], kSoftWarps);
    }
    mbar_init(&bars[B_OFULL], 1);
    mbar_init(&bars[B_OEMPTY], kSoftWarps);
    mbar_init(&bars[B_OREADY], 1);
    mbar_init(&bars[B_OSTAGED], kSoftWarps);
    mbar_init(&bars[B_DRAIN + 0], 1);
    mbar_init(&bars[B_DRAIN + 1], 1);
    for (int i = 0; i < kKStages; ++i) mbar_init(&bars[B_KFULL + i], 1);
    for (int i = 0; i < kVStages; ++i) mbar_init(&bars[B_VFULL + i], 1);
    for (int i = 0; i < kSBufs; ++i) {
      mbar_init(&bars[B_SFULL + i], 1);
      mbar_init(&bars[B_PFULL + i], kSoftWarps);
      mbar_init(&bars[B_PVDONE + i], 1);
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
  // the set-up above may overlap the previous kernel in the stream; every
  // input (lists, Q, K, V, O_l) is read after this
  grid_dep_wait();
  grid_dep_trigger();

  if (warp == 0 || warp == kVWarp) {
    // ------------------------------------------------------------ producers
    if (lane == 0) {
      const bool is_k = warp == 0;
      if (is_k) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
      } else {
        tma_prefetch_desc(&tmV);
        tma_prefetch_desc(&tmO);
        if (a.alpha) tma_prefetch_desc(&tmOL);
      }
      const CUtensorMap* map = is_k ? &tmK : &tmV;
      uint8_t* ring = is_k ? sK : sV;
      const int stages = is_k ? kKStages : kVStages;
      const int b_full = is_k ? B_KFULL : B_VFULL;
      int g = 0, qi = 0, q_armed = 0;
      bool ok = true;
      // O buffer turns (V producer): one per item, after the item's first two
      // V tiles (those never wait for the item's own P V). The previous item's
      // O goes out once the softmax warps have staged it; this item's O_l (or,
      // without the blend, the free buffer) is then handed to them.
      int ob_bh = 0, ob_qb = 0, ol_armed = 0;
      auto o_turn = [&](const Item& it) -> bool {
        if (qi > 0) {
          if (!mbar_wait(&bars[B_OSTAGED], (qi - 1) & 1, abort_flag)) return false;
#pragma unroll
          for (int c = 0; c < L::NCH_O; ++c) tma_store_3d(&tmO, sOB + c * L::OB_CHUNK, c * 64, ob_qb * a.bq, ob_bh);
          bulk_commit();
          bulk_wait_read<0>();
        }
        if (a.alpha) {
          mbar_arrive_expect_tx(&bars[B_OREADY], L::NCH_O * a.bq * 128);
#pragma unroll
          for (int c = 0; c < L::NCH_O; ++c)
            tma_load_3d(sOB + c * L::OB_CHUNK, &tmOL, &bars[B_OREADY], c * 64, it.qb * a.bq, it.bh);
          ol_armed = qi + 1;
        } else {
          mbar_arrive(&bars[B_OREADY]);
        }
        ob_bh = it.bh;
        ob_qb = it.qb;
        return true;
      };
      for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x) {
        const Item it = load_item(a, item);
        if (it.T == 0) continue;
        const int* row = a.dense ? nullptr : a.kv_idx + (static_cast<long long>(it.bh) * a.nqb + it.qb) * a.nkb;
        if (is_k) {
          // item facts for the softmax warps (they would otherwise read them
          // from global memory on their critical path)
          const int rs = qi % kItemRing;
          if (!(ok = mbar_wait(&bars[B_IEMPTY + rs], ((qi / kItemRing) & 1) ^ 1, abort_flag))) break;
          item_ring[rs * kRingWords + 0] = item;
          item_ring[rs * kRingWords + 1] = it.cnt;
          item_ring[rs * kRingWords + 2] = it.tail ? 1 : 0;
          if constexpr (F8) {
            // exponent factor scale * log2(e) * s_q * s_k, and s_v
            item_ring[rs * kRingWords + 3] = __float_as_int(a.scale_log2 * __ldg(a.q_scale + it.bh) * __ldg(a.k_scale + it.bh));
            item_ring[rs * kRingWords + 4] = __float_as_int(__ldg(a.v_scale + it.bh));
          }
          mbar_arrive(&bars[B_IFULL + rs]);
          const int qs = qi % kQSlots;
          if (!(ok = mbar_wait(&bars[B_QEMPTY + qs], ((qi / kQSlots) & 1) ^ 1, abort_flag))) break;
          mbar_arrive_expect_tx(&bars[B_QFULL + qs], L::Q_BYTES);
#pragma unroll
          for (int c = 0; c < L::NCH; ++c)
            tma_load_3d(sQ + qs * L::Q_BYTES + c * L::Q_CHUNK, &tmQ, &bars[B_QFULL + qs], c * L::CH_ELEMS, it.qb * a.bq, it.bh);
          q_armed = qi + 1;
        }
        for (int t = 0; t < it.T; ++t, ++g) {
          if (!is_k && t == 2 && !(ok = o_turn(it))) break;
          const int s = g % stages;
          const int nblk = min(2, it.cnt - 2 * t);
          const int kb0 = a.dense ? 2 * t : __ldg(row + 2 * t);
          const int kb1 = nblk > 1 ? (a.dense ? 2 * t + 1 : __ldg(row + 2 * t + 1)) : 0;
          // slot reuse: a K slot is free once the QK that read it completed
          // (S_FULL of the tile kKStages back), a V slot once the P V that read
          // it completed (PV_DONE of the tile kVStages back); both barriers
          // are indexed by S buffer
          if (is_k) {
            if (g >= kKStages) {
              const int gp = g - kKStages;
              if (!(ok = mbar_wait(&bars[B_SFULL + gp % kSBufs], (gp / kSBufs) & 1, abort_flag))) break;
            }
          } else if (g >= kVStages) {
            const int gp = g - kVStages;
            if (!(ok = mbar_wait(&bars[B_PVDONE + gp % kSBufs], (gp / kSBufs) & 1, abort_flag))) break;
          }
          mbar_arrive_expect_tx(&bars[b_full + s], nblk * L::BLK_BYTES);
          uint8_t* dst = ring + s * L::TILE_BYTES;
#pragma unroll
          for (int c = 0; c < L::NCH; ++c) {
            tma_load_3d(dst + c * L::KV_CHUNK, map, &bars[b_full + s], c * L::CH_ELEMS, kb0 * 64, it.bh);
            if (nblk > 1)
              tma_load_3d(dst + c * L::KV_CHUNK + 64 * 128, map, &bars[b_full + s], c * L::CH_ELEMS, kb1 * 64, it.bh);
          }
        }
        if (ok && !is_k && it.T <= 2) ok = o_turn(it);
        ++qi;
      }
      if (is_k && ok) {
        // end of this CTA's items
        const int rs = qi % kItemRing;
        if (mbar_wait(&bars[B_IEMPTY + rs], ((qi / kItemRing) & 1) ^ 1, abort_flag)) {
          item_ring[rs * kRingWords + 0] = n_items;
          mbar_arrive(&bars[B_IFULL + rs]);
        }
      }
      // loads still in flight land before the CTA gives up its shared memory
      // (g tiles and qi Q tiles were issued; a break can leave the last Q
      // unissued, so only the tiles whose barriers were armed are waited for)
      for (int i = 1; i <= stages && i <= g; ++i)
        mbar_drain(&bars[b_full + (g - i) % stages], ((g - i) / stages) & 1);
      if (is_k)
        for (int i = 1; i <= kQSlots && i <= q_armed; ++i)
          mbar_drain(&bars[B_QFULL + (q_armed - i) % kQSlots], ((q_armed - i) / kQSlots) & 1);
      if (!is_k) {
        // the last item's O, then every store complete and the last O_l load landed
        if (ok && qi > 0 && mbar_wait(&bars[B_OSTAGED], (qi - 1) & 1, abort_flag)) {
#pragma unroll
          for (int c = 0; c < L::NCH_O; ++c) tma_store_3d(&tmO, sOB + c * L::OB_CHUNK, c * 64, ob_qb * a.bq, ob_bh);
          bulk_commit();
        }
        bulk_wait_all();
        if (ol_armed > 0) mbar_drain(&bars[B_OREADY], (ol_armed - 1) & 1);
      }
    }
  } else if (warp == 1 || warp == kPVWarp) {
    // ------------------------------------------------------------ MMA issuers
    // Two threads feed the tensor pipe: warp 1 issues S = Q K^T, warp kPVWarp
    // issues O += P V. Each thread stalls while the tensor pipe's queue is
    // full, and its mbarrier waits and commits queue behind its own MMAs; with
    // two issuers the waits of one overlap the MMAs of the other. Since the
    // two streams are not ordered with each other, the QK that overwrites an
    // S buffer first waits for the P V that read P from it (PV_DONE).
    if (lane == 0) {
      const bool is_qk = warp == 1;
      const uint64_t qdesc0 = sw128_desc(smem_u32(sQ), 16, 1024);
      const uint64_t kdesc0 = sw128_desc(smem_u32(sK), 16, 1024);
      const uint64_t vdesc0 = sw128_desc(smem_u32(sV), L::KV_CHUNK, 1024);
      const uint32_t idesc_pv = F8 ? idesc_e4m3_f32(kBM, D, false, true) : idesc_bf16_f32(kBM, D, false, true);
      const uint32_t idesc_qk2 = F8 ? idesc_e4m3_f32(kBM, 128, false, false) : idesc_bf16_f32(kBM, 128, false, false);
      const uint32_t idesc_qk1 = F8 ? idesc_e4m3_f32(kBM, 64, false, false) : idesc_bf16_f32(kBM, 64, false, false);
      const uint32_t o_tm = tm + TM_O;
      struct Ring {
        int slot, n;
        uint32_t phase;
        __device__ void next() {
          if (++slot == n) { slot = 0; phase ^= 1u; }
        }
      };
      Ring kv{0, is_qk ? kKStages : kVStages, 0};   // K ring (QK) or V ring (PV)
      Ring sb{0, kSBufs, 0};
      uint32_t phase1 = 0;   // O_EMPTY phase (PV)
      int g = 0, qi = 0;
      bool ok = true;
      int item = next_nonempty(a, blockIdx.x, gridDim.x, n_items);
      Item it = item < n_items ? load_item(a, item) : Item{};
      while (ok && item < n_items) {
        // facts of the next item, fetched while this one is issued
        const int nitem = next_nonempty(a, item + gridDim.x, gridDim.x, n_items);
        const int ncnt = nitem < n_items ? (a.dense ? a.nkb : kept_count(a, nitem)) : 0;
        for (int t = 0; t < it.T; ++t, ++g) {
          const bool two = it.cnt - 2 * t >= 2;
          if (is_qk) {
            if (g >= kSBufs && !(ok = mbar_wait(&bars[B_PVDONE + sb.slot], sb.phase ^ 1u, abort_flag))) break;
            if (!(ok = mbar_wait(&bars[B_KFULL + kv.slot], kv.phase, abort_flag))) break;
            const int qs = qi % kQSlots;
            if (t == 0 && !(ok = mbar_wait(&bars[B_QFULL + qs], (qi / kQSlots) & 1, abort_flag))) break;
            tc_fence_after();
            const uint32_t idesc = two ? idesc_qk2 : idesc_qk1;
            const uint64_t qd = qdesc0 + ((qs * L::Q_BYTES) >> 4);
            const uint64_t kd = kdesc0 + ((kv.slot * L::TILE_BYTES) >> 4);
            const uint32_t s_tm = tm + tm_s(sb.slot);
#pragma unroll
            for (int kk = 0; kk < D / L::KSTEP; ++kk) {
              const uint64_t ad = qd + ((((kk >> 2) * L::Q_CHUNK) + (kk & 3) * 32u) >> 4);
              const uint64_t bd = kd + ((((kk >> 2) * L::KV_CHUNK) + (kk & 3) * 32u) >> 4);
              if constexpr (F8) umma_f8_ss(s_tm, ad, bd, idesc, kk > 0 ? 1u : 0u);
              else umma_ss(s_tm, ad, bd, idesc, kk > 0 ? 1u : 0u);
            }
            tc_commit(&bars[B_SFULL + sb.slot]);   // S ready, and the K slot free
            if (t + 1 == it.T) tc_commit(&bars[B_QEMPTY + qs]);
          } else {
            if (!(ok = mbar_wait(&bars[B_PFULL + sb.slot], sb.phase, abort_flag))) break;
            if (!(ok = mbar_wait(&bars[B_VFULL + kv.slot], kv.phase, abort_flag))) break;
            if (t == 0) {
              if (!(ok = mbar_wait(&bars[B_OEMPTY], phase1 ^ 1u, abort_flag))) break;
              phase1 ^= 1u;
            }
            tc_fence_after();
            const int nk = (two ? 128 : 64) / L::KSTEP;
            const uint64_t vd = vdesc0 + ((kv.slot * L::TILE_BYTES) >> 4);
            const uint32_t p_tm = tm + tm_s(sb.slot);
#pragma unroll
            for (int kk = 0; kk < 128 / L::KSTEP; ++kk) {
              // K step kk: keys [kk * KSTEP, +KSTEP), 8 TMEM columns of P, KSTEP rows of V
              if (kk >= nk) break;
              const uint64_t bd = vd + ((kk * L::KSTEP * 128u) >> 4);
              if constexpr (F8) umma_f8_ts(o_tm, p_tm + kk * 8, bd, idesc_pv, (t > 0 || kk > 0) ? 1u : 0u);
              else umma_ts(o_tm, p_tm + kk * 8, bd, idesc_pv, (t > 0 || kk > 0) ? 1u : 0u);
            }
            tc_commit(&bars[B_PVDONE + sb.slot]);   // O updated; S buffer and V slot free
            if (t + 1 == it.T) tc_commit(&bars[B_OFULL]);
          }
          kv.next();
          sb.next();
        }
        if (!ok) break;
        item = nitem;
        ++qi;
        if (item < n_items) {
          it.bh = item / a.nqb;
          it.qb = item % a.nqb;
          it.cnt = ncnt;
          it.T = (ncnt + 1) >> 1;
        }
      }
      // every MMA this thread issued has completed before tensor memory is released
      tc_commit(&bars[B_DRAIN + (is_qk ? 0 : 1)]);
      mbar_drain(&bars[B_DRAIN + (is_qk ? 0 : 1)], 0);
    }
  } else {
    if constexpr (F8) {
      // ------------------------------------------------------------ softmax + epilogue (E4M3)
      // The low-bit form keeps the split of each row's 128 columns between the
      // two warps of a lane quadrant (32x32b accesses, 64 columns each), with a
      // per-tile exchange of the row max: its P packs four keys into each TMEM
      // column, which a thread of the 16-lane layout (two keys per column pair)
      // could only do with cross-thread shuffles, and those cost more than the
      // exchange. Every bounded wait of these warps is followed by a barrier of
      // the pair at which each warp also posts whether its wait succeeded: in
      // place of the row max or row sum it posts a NaN with a payload of its own
      // (kStopBits; arithmetic yields the canonical NaN, never this one), or a
      // flag word in the rare rescale path. Each warp stops if either post says
      // so, the same decision in both. A warp whose wait for the next item fails
      // (no barrier follows that wait) posts the stop word in both places its
      // partner reads next and arrives once at the pair barrier before it leaves,
      // so neither waits at a barrier the other has left.
      float* red_max = reinterpret_cast<float*>(smem + L::OFF_RED);   // [2 tile parity][2 halves][128 rows]
      float* red_sum = red_max + 4 * kBM;                              // [2 halves][128 rows]
      // per quadrant: [6,8) rescale (half 0, half 1)
      volatile int* pair_flags = reinterpret_cast<volatile int*>(red_sum + 2 * kBM);
      const int sw = warp - 2;                  // 0..7
      const int quad = warp & 3;                // TMEM lane quadrant
      const int half = sw >> 2;                 // which 64 columns of the tile
      const int row = quad * 32 + lane;         // query row within the tile
      const int pair_bar = 1 + quad;            // named barrier of the two warps of this quadrant
      const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
      const float sl2 = a.scale_log2;
      const int tail_valid = a.N - (a.nkb - 1) * 64;
      int g = 0, qi = 0;
      bool ok = true;

      int prev = blockIdx.x - static_cast<int>(gridDim.x);   // last item handled
      while (ok) {
        // next non-empty item, as posted by the K producer; the items skipped
        // on the way have no kept block
        const int rs = qi % kItemRing;
        if (!mbar_wait(&bars[B_IFULL + rs], (qi / kItemRing) & 1, abort_flag)) {
          // leaving without the partner: post the stop word where it reads next
          // and give it the one arrival its next exchange needs
          red_max[(g & 1) * 2 * kBM + half * kBM + row] = __uint_as_float(kStopBits);
          red_sum[half * kBM + row] = __uint_as_float(kStopBits);
          asm volatile("bar.arrive %0, 64;" ::"r"(pair_bar) : "memory");
          ok = false;
          break;
        }
        const int item = item_ring[rs * kRingWords + 0];
        Item it;
        it.cnt = item_ring[rs * kRingWords + 1];
        it.tail = item_ring[rs * kRingWords + 2] != 0;
        // exponent factor of the scores and factor of the output (the low-bit
        // form's scales folded in)
        const float fexp = F8 ? __int_as_float(item_ring[rs * kRingWords + 3]) : sl2;
        const float fout = F8 ? __int_as_float(item_ring[rs * kRingWords + 4]) : 1.f;
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[B_IEMPTY + rs]);
        for (int z = prev + gridDim.x; z < item; z += gridDim.x) {
          const Item iz = load_item(a, z);
          const int gz = iz.qb * a.bq + row;
          if (row < a.bq && gz < a.N) {
            uint4* dz = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.o) + (static_cast<long long>(iz.bh) * a.N + gz) * D + half * (D / 2));
            for (int c = 0; c < D / 16; ++c) dz[c] = make_uint4(0, 0, 0, 0);
            if (a.lse && half == 0) a.lse[static_cast<long long>(iz.bh) * a.N + gz] = -INFINITY;
          }
        }
        if (item >= n_items) break;
        prev = item;
        it.bh = item / a.nqb;
        it.qb = item % a.nqb;
        it.T = (it.cnt + 1) >> 1;
        const int grow = it.qb * a.bq + row;
        const bool store = row < a.bq && grow < a.N;
        float m = -INFINITY;     // running max (log2 domain), identical in both halves
        float l = 0.f;           // this half's share of the row sum
        for (int t = 0; t < it.T; ++t, ++g) {
          const int b = g % kSBufs;
          // (after a failed wait the loads below read stale tensor memory; the
          // values are dropped when the pair stops at the barrier that follows)
          const bool s_ok = mbar_wait(&bars[B_SFULL + b], (g / kSBufs) & 1, abort_flag);
          float x[64];
          float mx;
          {
            tc_fence_after();
            uint32_t r0[32], r1[32];
            const uint32_t sa = tm + lane_addr + tm_s(b) + half * 64;
            tmem_ld32(sa, r0);
            tmem_ld32(sa + 32, r1);
            tmem_wait_ld();
            reg_fence(r0);
            reg_fence(r1);
  #pragma unroll
            for (int c = 0; c < 32; ++c) {
              x[c] = __uint_as_float(r0[c]);
              x[32 + c] = __uint_as_float(r1[c]);
            }
            if (t == it.T - 1) {
              // last tile: possibly a single block, possibly the ragged last key block
              const int nblk = it.cnt - 2 * t;
              int valid = (half < nblk) ? 64 : 0;
              if (it.tail && half == nblk - 1) valid = tail_valid;
  #pragma unroll
              for (int c = 0; c < 64; ++c)
                if (c >= valid) x[c] = -INFINITY;
            }
            // row max of this half: eight chains of 3-input max
            float mx8[8];
  #pragma unroll
            for (int j = 0; j < 8; ++j) {
              mx8[j] = fmax3(x[j], x[8 + j], x[16 + j]);
              mx8[j] = fmax3(mx8[j], x[24 + j], x[32 + j]);
              mx8[j] = fmax3(mx8[j], x[40 + j], x[48 + j]);
              mx8[j] = fmaxf(mx8[j], x[56 + j]);
            }
            mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
          }
          float* rm = red_max + (g & 1) * 2 * kBM;
          // the low-bit form posts its max in the log2 domain (the factor is the
          // same for both halves; bf16 scales after the exchange)
          const float posted = s_ok ? (F8 ? mx * fexp : mx) : __uint_as_float(kStopBits);
          rm[half * kBM + row] = posted;
          pair_sync(pair_bar);
          const float pmx = rm[(half ^ 1) * kBM + row];
          // Both warps combine the two posted words the same way (fmaxf skips the
          // NaN stop word), so everything up to the end of the tile, branches
          // included, is the same in both; the stop, if any, is taken there.
          const bool stop = !s_ok || __float_as_uint(pmx) == kStopBits;
          mx = fmaxf(posted, pmx);
          const float m_tile = F8 ? mx : mx * sl2;
          float corr = 1.f;
          if (m_tile > m + 8.f) {
            corr = fast_exp2(m - m_tile);   // 0 on the first tile (m = -inf)
            m = m_tile;
            l *= corr;
          }
          // P = 2^(S * scale * log2(e) - m), two columns per packed instruction.
          const uint64_t sl2x2 = f2_make(fexp, fexp);
          const uint64_t negm2 = f2_make(-m, -m);
          uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};   // packed (+0, +0)
          uint32_t p[F8 ? 16 : 32];
  #pragma unroll
          for (int c = 0; c < 32; ++c) {
            const uint64_t a2 = ffma2(f2_make(x[2 * c], x[2 * c + 1]), sl2x2, negm2);
            float e0, e1;
            if ((kPolyPairs >> (c & 7)) & 1) {
              exp2_poly2(a2, e0, e1);
            } else {
              float a0, a1;
              f2_split(a2, a0, a1);
              e0 = fast_exp2(a0);
              e1 = fast_exp2(a1);
            }
            acc[c & 3] = fadd2(acc[c & 3], f2_make(e0, e1));
            if constexpr (F8) {
              // four E4M3 values per column, the lowest key in the lowest byte
              const uint32_t h = pack_e4m3x2(e0, e1);
              p[c >> 1] = (c & 1) ? (p[c >> 1] | (h << 16)) : h;
            } else {
              p[c] = pack_bf16x2(e0, e1);
            }
          }
          {
            float s0, s1;
            f2_split(fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3])), s0, s1);
            l += s0 + s1;
          }
          if constexpr (F8) tmem_st16(tm + lane_addr + tm_s(b) + half * 16, p);
          else tmem_st32(tm + lane_addr + tm_s(b) + half * 32, p);
          if (!stop && t > 0 && __any_sync(0xFFFFFFFFu, corr != 1.f)) {
            // O is complete up to the previous tile once its P V has landed
            const int pb = (g - 1) % kSBufs;
            if (!(ok = pair_agree(pair_bar, pair_flags + quad * 16 + 6, half, mbar_wait(&bars[B_PVDONE + pb], ((g - 1) / kSBufs) & 1, abort_flag)))) break;
            tc_fence_after();
  #pragma unroll 1
            for (int c0 = 0; c0 < D / 2; c0 += 32) {
              uint32_t o[32];
              const uint32_t oa = tm + lane_addr + TM_O + half * (D / 2) + c0;
              tmem_ld32_wait(oa, o);
  #pragma unroll
              for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * corr);
              tmem_st32(oa, o);
            }
          }
          tmem_wait_st();
          if (stop) {   // either warp's wait failed: both stop here
            ok = false;
            break;
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars[B_PFULL + b]);
        }
        if (!ok) break;
        // ---------------------------------------------------------- epilogue
        bool o_ok = mbar_wait(&bars[B_OFULL], qi & 1, abort_flag);
        uint32_t o0[32], o1[32];
        {
          tc_fence_after();
          tmem_ld32(tm + lane_addr + TM_O + half * (D / 2), o0);
          if (D == 128) tmem_ld32(tm + lane_addr + TM_O + half * (D / 2) + 32, o1);
          tmem_wait_ld();
          reg_fence(o0);
          if (D == 128) reg_fence(o1);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars[B_OEMPTY]);   // the next item may overwrite O now
        }
        // the O buffer is free of the previous item's O and, with the blend,
        // holds this item's O_l
        o_ok = o_ok && mbar_wait(&bars[B_OREADY], qi & 1, abort_flag);
        red_sum[half * kBM + row] = o_ok ? l : __uint_as_float(kStopBits);
        pair_sync(pair_bar);
        const float pl = red_sum[(half ^ 1) * kBM + row];
        if (!(ok = o_ok && __float_as_uint(pl) != kStopBits)) break;
        const float lt = l + pl;
        const float inv_l = F8 ? fout / lt : 1.f / lt;
        {
          // this thread's half row is 64-column chunk `half` of row `row` (d =
          // 128): its 16-byte unit c lies at position c ^ (row % 8)
          uint4* ub = reinterpret_cast<uint4*>(sOB + half * L::OB_CHUNK + row * 128);
          const float4* alv = a.alpha ? reinterpret_cast<const float4*>(a.alpha + static_cast<long long>(it.bh % a.H) * D + half * (D / 2)) : nullptr;
  #pragma unroll
          for (int c = 0; c < D / 16; ++c) {
            const uint32_t* oc = (c < 4) ? o0 + 8 * c : o1 + 8 * (c - 4);
            uint4* u = ub + (c ^ (row & 7));
            float r8[8];
  #pragma unroll
            for (int j = 0; j < 8; ++j) r8[j] = __uint_as_float(oc[j]) * inv_l;
            if (a.alpha) {
              // O = alpha ⊙ O_s + (1 - alpha) ⊙ O_l with O_s = o / l not yet rounded
              const uint4 lv = *u;
              const float4 a0 = __ldg(alv + 2 * c), a1 = __ldg(alv + 2 * c + 1);
              const uint32_t lw[4] = {lv.x, lv.y, lv.z, lv.w};
              const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
  #pragma unroll
              for (int j = 0; j < 8; ++j) {
                const float olj = __uint_as_float((j & 1) ? (lw[j >> 1] & 0xFFFF0000u) : (lw[j >> 1] << 16));
                r8[j] = fmaf(av[j], r8[j] - olj, olj);
              }
            }
            *u = make_uint4(pack_bf16x2(r8[0], r8[1]), pack_bf16x2(r8[2], r8[3]),
                            pack_bf16x2(r8[4], r8[5]), pack_bf16x2(r8[6], r8[7]));
          }
        }
        // the TMA store that reads the buffer is issued by the V producer
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[B_OSTAGED]);
        if (store && a.lse && half == 0)
          a.lse[static_cast<long long>(it.bh) * a.N + grow] = (m + log2f(lt)) * 0.69314718055994531f;
        ++qi;
      }
    } else {
      // ------------------------------------------------------------ softmax + epilogue
      // Each warp owns 16 of its quadrant's TMEM lanes (query rows), all 128
      // columns of every tile: thread t holds rows ra and ra + 8 and, of each,
      // the columns 8 k + 2 j4 and 8 k + 2 j4 + 1 (j4 = t % 4, k = 0..15). The
      // four threads of a row combine its max and sum with two shuffles.
      const int sw = warp - 2;                  // 0..7
      const int quad = warp & 3;                // TMEM lane quadrant
      const int half = sw >> 2;                 // which 16 lanes of the quadrant
      const int j4 = lane & 3;
      const int ra = quad * 32 + half * 16 + (lane >> 2);   // rows ra and ra + 8 of the tile
      const uint32_t lane_addr = static_cast<uint32_t>(quad * 32 + half * 16) << 16;
      const int zrow = quad * 32 + lane;        // row and half columns this thread zero-fills
      const float sl2 = a.scale_log2;
      const int tail_valid = a.N - (a.nkb - 1) * 64;
      int g = 0, qi = 0;
      bool ok = true;

      int prev = blockIdx.x - static_cast<int>(gridDim.x);   // last item handled
      while (ok) {
        // next non-empty item, as posted by the K producer; the items skipped
        // on the way have no kept block
        const int rs = qi % kItemRing;
        if (!mbar_wait(&bars[B_IFULL + rs], (qi / kItemRing) & 1, abort_flag)) {
          ok = false;
          break;
        }
        const int item = item_ring[rs * kRingWords + 0];
        Item it;
        it.cnt = item_ring[rs * kRingWords + 1];
        it.tail = item_ring[rs * kRingWords + 2] != 0;
        // exponent factor of the scores and factor of the output (the low-bit
        // form's scales folded in)
        const float fexp = F8 ? __int_as_float(item_ring[rs * kRingWords + 3]) : sl2;
        const float fout = F8 ? __int_as_float(item_ring[rs * kRingWords + 4]) : 1.f;
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[B_IEMPTY + rs]);
        for (int z = prev + gridDim.x; z < item; z += gridDim.x) {
          const Item iz = load_item(a, z);
          const int gz = iz.qb * a.bq + zrow;
          if (zrow < a.bq && gz < a.N) {
            uint4* dz = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.o) + (static_cast<long long>(iz.bh) * a.N + gz) * D + half * (D / 2));
            for (int c = 0; c < D / 16; ++c) dz[c] = make_uint4(0, 0, 0, 0);
            if (a.lse && half == 0) a.lse[static_cast<long long>(iz.bh) * a.N + gz] = -INFINITY;
          }
        }
        if (item >= n_items) break;
        prev = item;
        it.bh = item / a.nqb;
        it.qb = item % a.nqb;
        it.T = (it.cnt + 1) >> 1;
        const int grow_a = it.qb * a.bq + ra;
        const bool store_a = ra < a.bq && grow_a < a.N;
        const bool store_b = ra + 8 < a.bq && grow_a + 8 < a.N;
        float m_a = -INFINITY, m_b = -INFINITY;   // running maxima of the two rows (log2 domain)
        float l_a = 0.f, l_b = 0.f;               // this thread's shares of the row sums
        for (int t = 0; t < it.T; ++t, ++g) {
          const int b = g % kSBufs;
          if (!mbar_wait(&bars[B_SFULL + b], (g / kSBufs) & 1, abort_flag)) {
            ok = false;
            break;
          }
          float xa[32], xb[32];   // [2 k + e]: column 8 k + 2 j4 + e of rows ra, ra + 8
          {
            tc_fence_after();
            uint32_t r0[32], r1[32];
            tmem_ld_16x256b_x8(tm + lane_addr + tm_s(b), r0);
            tmem_ld_16x256b_x8(tm + lane_addr + tm_s(b) + 64, r1);
            tmem_wait_ld();
            reg_fence(r0);
            reg_fence(r1);
  #pragma unroll
            for (int k = 0; k < 8; ++k) {
              xa[2 * k] = __uint_as_float(r0[4 * k]);
              xa[2 * k + 1] = __uint_as_float(r0[4 * k + 1]);
              xb[2 * k] = __uint_as_float(r0[4 * k + 2]);
              xb[2 * k + 1] = __uint_as_float(r0[4 * k + 3]);
              xa[16 + 2 * k] = __uint_as_float(r1[4 * k]);
              xa[16 + 2 * k + 1] = __uint_as_float(r1[4 * k + 1]);
              xb[16 + 2 * k] = __uint_as_float(r1[4 * k + 2]);
              xb[16 + 2 * k + 1] = __uint_as_float(r1[4 * k + 3]);
            }
          }
          if (t == it.T - 1) {
            // last tile: possibly a single block, possibly the ragged last key block
            const int nblk = it.cnt - 2 * t;
            const int limit = (nblk == 2 ? 64 : 0) + (it.tail ? tail_valid : 64);
  #pragma unroll
            for (int i = 0; i < 32; ++i) {
              if (8 * (i >> 1) + 2 * j4 + (i & 1) >= limit) {
                xa[i] = -INFINITY;
                xb[i] = -INFINITY;
              }
            }
          }
          float mx_a, mx_b;
          {
            float ma4[4], mb4[4];
  #pragma unroll
            for (int j = 0; j < 4; ++j) {
              ma4[j] = fmax3(fmax3(xa[j], xa[4 + j], xa[8 + j]), fmax3(xa[12 + j], xa[16 + j], xa[20 + j]), fmaxf(xa[24 + j], xa[28 + j]));
              mb4[j] = fmax3(fmax3(xb[j], xb[4 + j], xb[8 + j]), fmax3(xb[12 + j], xb[16 + j], xb[20 + j]), fmaxf(xb[24 + j], xb[28 + j]));
            }
            mx_a = fmaxf(fmaxf(ma4[0], ma4[1]), fmaxf(ma4[2], ma4[3]));
            mx_b = fmaxf(fmaxf(mb4[0], mb4[1]), fmaxf(mb4[2], mb4[3]));
            mx_a = fmaxf(mx_a, __shfl_xor_sync(0xFFFFFFFFu, mx_a, 1));
            mx_b = fmaxf(mx_b, __shfl_xor_sync(0xFFFFFFFFu, mx_b, 1));
            mx_a = fmaxf(mx_a, __shfl_xor_sync(0xFFFFFFFFu, mx_a, 2));
            mx_b = fmaxf(mx_b, __shfl_xor_sync(0xFFFFFFFFu, mx_b, 2));
          }
          float corr_a = 1.f, corr_b = 1.f;
          {
            const float mt_a = mx_a * fexp, mt_b = mx_b * fexp;
            if (mt_a > m_a + 8.f) {
              corr_a = fast_exp2(m_a - mt_a);   // 0 on the first tile (m = -inf)
              m_a = mt_a;
              l_a *= corr_a;
            }
            if (mt_b > m_b + 8.f) {
              corr_b = fast_exp2(m_b - mt_b);
              m_b = mt_b;
              l_b *= corr_b;
            }
          }
          // P = 2^(S * factor - m), two columns per packed instruction: pairs
          // c < 16 are row ra (columns 8 c + 2 j4, + 1), c >= 16 row ra + 8.
          const uint64_t fx2 = f2_make(fexp, fexp);
          const uint64_t negm_a = f2_make(-m_a, -m_a), negm_b = f2_make(-m_b, -m_b);
          uint64_t acc_a[2] = {0ull, 0ull}, acc_b[2] = {0ull, 0ull};   // packed (+0, +0)
          uint32_t p[32];   // bf16 pairs: [2 k] row ra, [2 k + 1] row ra + 8, column 4 k + j4
  #pragma unroll
          for (int c = 0; c < 32; ++c) {
            const bool rb = c >= 16;
            const int k = c & 15;
            const float* xr = rb ? xb : xa;
            const uint64_t a2 = ffma2(f2_make(xr[2 * k], xr[2 * k + 1]), fx2, rb ? negm_b : negm_a);
            float e0, e1;
            if ((kPolyPairs >> (c & 7)) & 1) {
              exp2_poly2(a2, e0, e1);
            } else {
              float a0, a1;
              f2_split(a2, a0, a1);
              e0 = fast_exp2(a0);
              e1 = fast_exp2(a1);
            }
            if (rb) acc_b[c & 1] = fadd2(acc_b[c & 1], f2_make(e0, e1));
            else acc_a[c & 1] = fadd2(acc_a[c & 1], f2_make(e0, e1));
            p[2 * k + (rb ? 1 : 0)] = pack_bf16x2(e0, e1);
          }
          {
            float s0, s1;
            f2_split(fadd2(acc_a[0], acc_a[1]), s0, s1);
            l_a += s0 + s1;
            f2_split(fadd2(acc_b[0], acc_b[1]), s0, s1);
            l_b += s0 + s1;
          }
          tmem_st_16x128b_x16(tm + lane_addr + tm_s(b), p);
          if (t > 0 && __any_sync(0xFFFFFFFFu, corr_a != 1.f || corr_b != 1.f)) {
            // O is complete up to the previous tile once its P V has landed
            const int pb = (g - 1) % kSBufs;
            if (!mbar_wait(&bars[B_PVDONE + pb], ((g - 1) / kSBufs) & 1, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
  #pragma unroll 1
            for (int c0 = 0; c0 < D; c0 += 64) {
              uint32_t o[32];
              const uint32_t oa = tm + lane_addr + TM_O + c0;
              tmem_ld_16x256b_x8(oa, o);
              tmem_wait_ld();
  #pragma unroll
              for (int k = 0; k < 8; ++k) {
                o[4 * k] = __float_as_uint(__uint_as_float(o[4 * k]) * corr_a);
                o[4 * k + 1] = __float_as_uint(__uint_as_float(o[4 * k + 1]) * corr_a);
                o[4 * k + 2] = __float_as_uint(__uint_as_float(o[4 * k + 2]) * corr_b);
                o[4 * k + 3] = __float_as_uint(__uint_as_float(o[4 * k + 3]) * corr_b);
              }
              tmem_st_16x256b_x8(oa, o);
            }
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars[B_PFULL + b]);
        }
        if (!ok) break;
        // ---------------------------------------------------------- epilogue
        // row sums over the four threads of each row
        l_a += __shfl_xor_sync(0xFFFFFFFFu, l_a, 1);
        l_b += __shfl_xor_sync(0xFFFFFFFFu, l_b, 1);
        l_a += __shfl_xor_sync(0xFFFFFFFFu, l_a, 2);
        l_b += __shfl_xor_sync(0xFFFFFFFFu, l_b, 2);
        const float inv_a = fout / l_a, inv_b = fout / l_b;
        if (!mbar_wait(&bars[B_OFULL], qi & 1, abort_flag)) {
          ok = false;
          break;
        }
        uint32_t o[D / 2];   // [32 h + 4 k + 0..3]: columns 64 h + 8 k + 2 j4 (+1) of rows ra, ra + 8
        {
          tc_fence_after();
          uint32_t r0[32];
          tmem_ld_16x256b_x8(tm + lane_addr + TM_O, r0);
          if constexpr (D == 128) {
            uint32_t r1[32];
            tmem_ld_16x256b_x8(tm + lane_addr + TM_O + 64, r1);
            tmem_wait_ld();
            reg_fence(r0);
            reg_fence(r1);
  #pragma unroll
            for (int i = 0; i < 32; ++i) {
              o[i] = r0[i];
              o[32 + i] = r1[i];
            }
          } else {
            tmem_wait_ld();
            reg_fence(r0);
  #pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = r0[i];
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars[B_OEMPTY]);   // the next item may overwrite O now
        }
        // the O buffer is free of the previous item's O and, with the blend,
        // holds this item's O_l
        if (!mbar_wait(&bars[B_OREADY], qi & 1, abort_flag)) {
          ok = false;
          break;
        }
        {
          // column 8 k + 2 j4 of row r lies in 64-column chunk k / 8, 16-byte
          // unit (k % 8) ^ (r % 8) of the row's 128 bytes; rows ra and ra + 8
          // share r % 8, and the 32 lanes of one k hit 32 distinct banks
          const float* alr = a.alpha ? a.alpha + static_cast<long long>(it.bh % a.H) * D : nullptr;
          uint8_t* rowa = sOB + ra * 128 + 4 * j4;
  #pragma unroll
          for (int k = 0; k < D / 8; ++k) {
            const int col = 8 * k + 2 * j4;
            const int i0 = 32 * (k >> 3) + 4 * (k & 7);
            uint32_t* pa = reinterpret_cast<uint32_t*>(rowa + (k >> 3) * L::OB_CHUNK + (((k & 7) ^ (ra & 7)) << 4));
            uint32_t* pb = pa + 8 * 128 / 4;
            float va0 = __uint_as_float(o[i0]) * inv_a, va1 = __uint_as_float(o[i0 + 1]) * inv_a;
            float vb0 = __uint_as_float(o[i0 + 2]) * inv_b, vb1 = __uint_as_float(o[i0 + 3]) * inv_b;
            if (a.alpha) {
              // O = alpha ⊙ O_s + (1 - alpha) ⊙ O_l with O_s not yet rounded
              const float2 al = __ldg(reinterpret_cast<const float2*>(alr + col));
              const uint32_t wa = *pa, wb = *pb;
              const float la0 = __uint_as_float(wa << 16), la1 = __uint_as_float(wa & 0xFFFF0000u);
              const float lb0 = __uint_as_float(wb << 16), lb1 = __uint_as_float(wb & 0xFFFF0000u);
              va0 = fmaf(al.x, va0 - la0, la0);
              va1 = fmaf(al.y, va1 - la1, la1);
              vb0 = fmaf(al.x, vb0 - lb0, lb0);
              vb1 = fmaf(al.y, vb1 - lb1, lb1);
            }
            *pa = pack_bf16x2(va0, va1);
            *pb = pack_bf16x2(vb0, vb1);
          }
        }
        // the TMA store that reads the buffer is issued by the V producer
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[B_OSTAGED]);
        if (a.lse && j4 == 0) {
          if (store_a) a.lse[static_cast<long long>(it.bh) * a.N + grow_a] = (m_a + log2f(l_a)) * 0.69314718055994531f;
          if (store_b) a.lse[static_cast<long long>(it.bh) * a.N + grow_a + 8] = (m_b + log2f(l_b)) * 0.69314718055994531f;
        }
        ++qi;
      }

    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tm, TM_COLS);
  }
}

template <int D, bool F8>
static cudaError_t launch_d(const AttnArgs& a, cudaStream_t st) {
  using L = attn::Layout<D, F8>;
  CUtensorMap mq, mk, mv, mo, mol;
  auto enc = [&](CUtensorMap* m, const void* base, uint32_t rows) {
    return F8 ? encode_tensor_map_3d_u8(m, base, D, a.N, a.BH, L::CH_ELEMS, rows)
              : encode_tensor_map_3d_bf16(m, base, D, a.N, a.BH, L::CH_ELEMS, rows);
  };
  if (enc(&mq, a.q, attn::kBM) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  if (enc(&mk, a.k, 64) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  if (enc(&mv, a.v, 64) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  // O (stored) and O_l (loaded) in bf16, one box per 64 columns and query block
  if (encode_tensor_map_3d_bf16(&mo, a.o, D, a.N, a.BH, 64, a.bq) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  if (a.alpha) {
    if (encode_tensor_map_3d_bf16(&mol, a.o_l, D, a.N, a.BH, 64, a.bq) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  } else {
    mol = mo;   // not read without the blend
  }
  cudaError_t e = cudaFuncSetAttribute(sparse_attn_kernel<D, F8>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long items = static_cast<long long>(a.BH) * a.nqb;
  const int grid = static_cast<int>(items < sms ? items : sms);
  return launch_pdl(sparse_attn_kernel<D, F8>, dim3(grid), dim3(attn::kThreads), L::SMEM, st, mq, mk, mv, mo, mol, a);
}

cudaError_t launch_sparse_attn(const AttnArgs& a, cudaStream_t st) {
  if (static_cast<long long>(a.BH) * a.nqb > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  if (a.fp8) return a.d == 128 ? launch_d<128, true>(a, st) : cudaErrorInvalidValue;
  return a.d == 128 ? launch_d<128, false>(a, st) : launch_d<64, false>(a, st);
}

}  // namespace sa
