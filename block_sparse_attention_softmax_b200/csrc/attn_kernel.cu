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
// Each CTA keeps two items in flight, in two "lanes". A lane has its own S and
// O accumulators in tensor memory and its own softmax warpgroup, one thread
// per query row over all 128 columns of a tile (no exchange of row maxima
// between warps). One thread issues the MMAs of both lanes in the order
//     ... PV_0(j-1), QK_0(j), PV_1(j-1), QK_1(j), PV_0(j), QK_0(j+1) ...
// so that while one lane's softmax works on its S the tensor core runs the
// other lane's P V and Q K^T: each softmax has about two MMA groups of time.
// P is written as bf16 over the first 64 columns of its lane's S buffer and
// read from there by the P V; the Q K^T that next overwrites that buffer is
// issued by the same thread after that P V, and the tcgen05.mma operations of
// one thread execute in the order issued. A commit after a lane's Q K^T also
// covers the P V issued before it, so when the softmax sees S(j) the lane's O
// already holds tile j-1: the lazy rescale of O needs no extra wait.
//
//   warp 0       scheduler and K producer: hands the CTA's items, in order, to
//                whichever lane finished its previous item (lanes alternate
//                tile by tile), posts each item's facts to that lane's ring,
//                and loads K tiles (one TMA box per 64-key block, so the two
//                blocks of a tile need not be adjacent) into a 2-slot ring in
//                the same alternating order. It also owns the three Q slots:
//                each lane holds the slot of its current item, and the third
//                receives the next non-empty item; when a lane takes that
//                item, the slot of the item it finished is requested for the
//                one after (a slot tied to an item's position in the list
//                could be the slot the other lane still holds).
//   warp 1       TMEM allocation and the MMA-issuing thread
//   warp 2       V producer (2-slot ring, same order as K)
//   warp 3       Q producer: loads each requested Q tile into its slot once
//                the last Q K^T of the slot's previous item has completed, so
//                the next item's Q is resident before a lane takes it
//   warps 4..7   softmax of lane 0, warps 8..11 softmax of lane 1: warp w
//                reads TMEM lane quadrant w % 4 (query rows 32 (w % 4) .. +31
//                of its tile). The running max m is kept in the log2 domain
//                and raised only when a tile's max exceeds it by more than 8
//                (P <= 256 otherwise); then O is rescaled in TMEM. P =
//                exp2(S*scale*log2e - m). At the end of an item the warps copy
//                O to registers, release it, and write O / l as bf16 and the
//                row log-sum-exp; an item with no kept block gets zeros and
//                -inf. With the linear branch, the epilogue blends while O_s
//                is still fp32: O = alpha ⊙ O_s + (1 - alpha) ⊙ O_l (SLA2
//                提案手法 ②), one bf16 rounding of O in all.
//
// TMEM columns: S_0 [0,128), S_1 [128,256) (fp32, 128 wide; P aliases the
// first 64 columns), O_0 at 256, O_1 at 384 (D wide). Every mbarrier wait is
// bounded (sa_device.cuh). A CTA that stops early waits (bounded) for its
// TMA loads and MMAs in flight before it releases shared and tensor memory.
#include "sa_internal.h"

namespace sa {

namespace attn {

constexpr int kBM = 128;        // query rows per tile
constexpr int kBN = 128;        // keys per tile (two 64-key blocks)
constexpr int kLanes = 2;       // items in flight per CTA
constexpr int kQSlots = 3;      // Q slots: both lanes' items plus the next one
constexpr int kQReqRing = 4;    // Q load requests posted ahead of the Q producer
constexpr int kKStages = 2;
constexpr int kVStages = 2;
constexpr int kItemRing = 4;    // item facts per lane posted ahead of its consumers
// Column pairs c (of 64 per thread and tile) with bit (c % 8) set take the
// FMA-pipe exponential instead of MUFU ex2: one pair in four.
constexpr uint32_t kPolyPairs = 0x88u;
constexpr float kRescaleLog2 = 8.f;
constexpr int kKWarp = 0, kMmaWarp = 1, kVWarp = 2, kQWarp = 3, kSoftWarp0 = 4;
constexpr int kLaneWarps = 4;
constexpr int kThreads = 32 * (kSoftWarp0 + kLanes * kLaneWarps);
// consumers of a lane's item ring: V producer, MMA issuer, the lane's softmax warps
constexpr int kRingConsumers = 2 + kLaneWarps;

template <int D>
struct Layout {
  static constexpr int NCH = D / 64;                       // 128-byte chunks along d
  static constexpr uint32_t Q_BYTES = kBM * D * 2;
  static constexpr uint32_t TILE_BYTES = kBN * D * 2;       // one K or V tile
  static constexpr uint32_t BLK_BYTES = 64 * D * 2;         // one 64-key block
  static constexpr uint32_t Q_CHUNK = kBM * 128;            // bytes per d-chunk of Q
  static constexpr uint32_t KV_CHUNK = kBN * 128;           // bytes per d-chunk of K/V
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = OFF_Q + kQSlots * Q_BYTES;
  static constexpr uint32_t OFF_V = OFF_K + kKStages * TILE_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_V + kVStages * TILE_BYTES;
  static constexpr uint32_t OFF_RING = OFF_BAR + 512;      // [kLanes][kItemRing] int4
  static constexpr uint32_t OFF_QREQ = OFF_RING + kLanes * kItemRing * 16;   // [kQReqRing] int2
  static constexpr uint32_t USED = OFF_QREQ + kQReqRing * 8;
  // at least 120 KB so that a second CTA never shares the SM (all 512 TMEM columns are held)
  static constexpr uint32_t SMEM = (USED + 1024 > 120 * 1024) ? USED + 1024 : 120 * 1024;
};
static_assert(Layout<128>::SMEM <= 232448, "shared memory of the d = 128 kernel");

__host__ __device__ constexpr uint32_t tm_s(int l) { return static_cast<uint32_t>(l) * 128u; }
__host__ __device__ constexpr uint32_t tm_o(int l) { return 256u + static_cast<uint32_t>(l) * 128u; }
constexpr uint32_t TM_COLS = 512;

enum {
  B_QFULL = 0,                          // [kQSlots] Q tile landed
  B_QEMPTY = B_QFULL + kQSlots,         // [kQSlots] last Q K^T of the item completed
  B_KFULL = B_QEMPTY + kQSlots,         // [kKStages]
  B_KEMPTY = B_KFULL + kKStages,        // [kKStages] the Q K^T that read the slot completed
  B_VFULL = B_KEMPTY + kKStages,        // [kVStages]
  B_VEMPTY = B_VFULL + kVStages,        // [kVStages] the P V that read the slot completed
  B_SFULL = B_VEMPTY + kVStages,        // [kLanes] S of the lane's tile ready (and O through the tile before)
  B_PFULL = B_SFULL + kLanes,           // [kLanes] P written by the lane's softmax warps
  B_OFULL = B_PFULL + kLanes,           // [kLanes] last P V of the lane's item completed
  B_OEMPTY = B_OFULL + kLanes,          // [kLanes] the lane's epilogue copied O out of TMEM
  B_IFULL = B_OEMPTY + kLanes,          // [kLanes][kItemRing] item facts posted
  B_IEMPTY = B_IFULL + kLanes * kItemRing,  // [kLanes][kItemRing] item facts read by every consumer
  B_RFULL = B_IEMPTY + kLanes * kItemRing,  // [kQReqRing] Q load request posted
  B_REMPTY = B_RFULL + kQReqRing,           // [kQReqRing] Q load request read
  B_DRAIN = B_REMPTY + kQReqRing,           // the MMA thread's last commit (early exit)
  B_COUNT = B_DRAIN + 1
};

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

// Where one lane stands in the schedule. The scheduler and every role that
// follows the alternating tile order keep one per lane and update it the same
// way: a lane that has issued its item's last tile takes a new item at its
// next turn; a lane that met the end marker is out, and the other lane then
// takes every turn.
struct LaneState {
  int item, cnt, T, t, qslot;   // current item, kept blocks, tiles, next tile, Q slot
  int n;                         // ring entries posted (scheduler) or read (consumer)
  bool tail, need, active;
};

__device__ __forceinline__ void lane_init(LaneState& s) {
  s.item = s.cnt = s.T = s.t = s.n = 0;
  s.qslot = -1;
  s.tail = false;
  s.need = s.active = true;
}

// Reads lane l's ring until a non-empty item or the end marker (single-thread
// consumer). Returns false if a wait ran out or another role aborted.
__device__ __forceinline__ bool take_item(uint64_t* bars, const volatile int* ring, int l, LaneState& s,
                                          int n_items, volatile int* abort) {
  while (true) {
    const int slot = s.n % kItemRing;
    if (!mbar_wait(&bars[B_IFULL + l * kItemRing + slot], (s.n / kItemRing) & 1, abort)) return false;
    const volatile int* e = ring + (l * kItemRing + slot) * 4;
    const int item = e[0], cnt = e[1], tail = e[2], qslot = e[3];
    mbar_arrive(&bars[B_IEMPTY + l * kItemRing + slot]);
    ++s.n;
    if (item >= n_items) {
      s.active = false;
      return true;
    }
    if (cnt == 0) continue;     // nothing to load or compute; the lane's softmax writes its zeros
    s.item = item;
    s.cnt = cnt;
    s.T = (cnt + 1) >> 1;
    s.t = 0;
    s.tail = tail != 0;
    s.qslot = qslot;
    s.need = false;
    return true;
  }
}

// Key blocks of tile t of an item: the first, the second (if any) and their count.
__device__ __forceinline__ int tile_blocks(const AttnArgs& a, int item, int cnt, int t, int& kb0, int& kb1) {
  const int nblk = min(2, cnt - 2 * t);
  if (a.dense) {
    kb0 = 2 * t;
    kb1 = 2 * t + 1;
  } else {
    const int* row = a.kv_idx + static_cast<long long>(item) * a.nkb;   // item = bh * nqb + qb
    kb0 = __ldg(row + 2 * t);
    kb1 = nblk > 1 ? __ldg(row + 2 * t + 1) : 0;
  }
  return nblk;
}

}  // namespace attn

template <int D>
__global__ void __launch_bounds__(attn::kThreads, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, AttnArgs a) {
  using namespace attn;
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + L::OFF_Q;
  uint8_t* sK = smem + L::OFF_K;
  uint8_t* sV = smem + L::OFF_V;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  static_assert(B_COUNT * 8 + 8 <= 512, "barrier region");
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + B_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* ring = reinterpret_cast<volatile int*>(smem + L::OFF_RING);   // [lane][slot][item, cnt, tail, Q slot]
  volatile int* qreq = reinterpret_cast<volatile int*>(smem + L::OFF_QREQ);   // [slot][item, Q slot]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_items = a.BH * a.nqb;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kQSlots; ++i) {
      mbar_init(&bars[B_QFULL + i], 1);
      mbar_init(&bars[B_QEMPTY + i], 1);
    }
    for (int i = 0; i < kKStages; ++i) {
      mbar_init(&bars[B_KFULL + i], 1);
      mbar_init(&bars[B_KEMPTY + i], 1);
    }
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(&bars[B_VFULL + i], 1);
      mbar_init(&bars[B_VEMPTY + i], 1);
    }
    for (int l = 0; l < kLanes; ++l) {
      mbar_init(&bars[B_SFULL + l], 1);
      mbar_init(&bars[B_PFULL + l], kLaneWarps);
      mbar_init(&bars[B_OFULL + l], 1);
      mbar_init(&bars[B_OEMPTY + l], kLaneWarps);
      for (int i = 0; i < kItemRing; ++i) {
        mbar_init(&bars[B_IFULL + l * kItemRing + i], 1);
        mbar_init(&bars[B_IEMPTY + l * kItemRing + i], kRingConsumers);
      }
    }
    for (int i = 0; i < kQReqRing; ++i) {
      mbar_init(&bars[B_RFULL + i], 1);
      mbar_init(&bars[B_REMPTY + i], 1);
    }
    mbar_init(&bars[B_DRAIN], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *tmem_slot;

  if (warp == kKWarp) {
    // ------------------------------------------------------------ scheduler + K producer
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      LaneState s0, s1;
      lane_init(s0);
      lane_init(s1);
      int g = 0, nreq = 0;
      uint32_t free_slots = (1u << kQSlots) - 1;
      bool ok = true;
      // first non-empty item at or after `from` in this CTA's list (n_items if none)
      auto find_nonempty = [&](int from) {
        for (int i = from; i < n_items; i += gridDim.x)
          if (load_item(a, i).T > 0) return i;
        return n_items;
      };
      // asks the Q producer to load item's Q into `slot`
      auto request_q = [&](int item, int slot) -> bool {
        const int r = nreq % kQReqRing;
        if (!mbar_wait(&bars[B_REMPTY + r], ((nreq / kQReqRing) & 1) ^ 1, abort_flag)) return false;
        qreq[r * 2 + 0] = item;
        qreq[r * 2 + 1] = slot;
        mbar_arrive(&bars[B_RFULL + r]);
        ++nreq;
        return true;
      };
      // posts one item's facts to lane l's ring
      auto post = [&](int ln, LaneState& c, int item, int cnt, bool tail, int qslot) -> bool {
        const int slot = c.n % kItemRing;
        if (!mbar_wait(&bars[B_IEMPTY + ln * kItemRing + slot], ((c.n / kItemRing) & 1) ^ 1, abort_flag)) return false;
        volatile int* e = ring + (ln * kItemRing + slot) * 4;
        e[0] = item;
        e[1] = cnt;
        e[2] = tail ? 1 : 0;
        e[3] = qslot;
        mbar_arrive(&bars[B_IFULL + ln * kItemRing + slot]);
        ++c.n;
        return true;
      };
      int next = blockIdx.x;               // first item not yet handed to a lane
      int pf = find_nonempty(next);        // the next non-empty item, its Q requested into pf_slot
      int pf_slot = 0;
      if (pf < n_items) free_slots &= ~1u;
      ok = request_q(pf, pf_slot);         // item n_items: no more requests (the Q producer stops)
      // one turn of lane l: a new item if it needs one, then its next K tile
      auto turn = [&](LaneState& c, const int l) -> bool {
        bool ok = true;
        if (c.active && c.need) {
          // the empty items before the next non-empty one go to this lane for their zeros
          for (; ok && next < pf; next += gridDim.x) ok = post(l, c, next, 0, false, -1);
          if (!ok) return false;
          if (pf >= n_items) {
            if (!post(l, c, n_items, 0, false, -1)) return false;
            c.active = false;
          } else {
            const Item it = load_item(a, pf);
            if (!post(l, c, pf, it.cnt, it.tail, pf_slot)) return false;
            if (c.qslot >= 0) free_slots |= 1u << c.qslot;   // reloaded after its last Q K^T
            c.item = pf;
            c.cnt = it.cnt;
            c.T = it.T;
            c.t = 0;
            c.qslot = pf_slot;
            c.need = false;
            next = pf + gridDim.x;
            pf = find_nonempty(next);
            if (pf < n_items) {
              pf_slot = __ffs(free_slots) - 1;
              free_slots &= ~(1u << pf_slot);
            }
            if (!(ok = request_q(pf, pf_slot))) return false;
          }
        }
        if (c.active) {
          const int ks = g % kKStages;
          int kb0, kb1;
          const int nblk = tile_blocks(a, c.item, c.cnt, c.t, kb0, kb1);
          const int bh = c.item / a.nqb;
          if (!mbar_wait(&bars[B_KEMPTY + ks], ((g / kKStages) & 1) ^ 1, abort_flag)) return false;
          mbar_arrive_expect_tx(&bars[B_KFULL + ks], nblk * L::BLK_BYTES);
          uint8_t* dst = sK + ks * L::TILE_BYTES;
#pragma unroll
          for (int ch = 0; ch < L::NCH; ++ch) {
            tma_load_3d(dst + ch * L::KV_CHUNK, &tmK, &bars[B_KFULL + ks], ch * 64, kb0 * 64, bh);
            if (nblk > 1)
              tma_load_3d(dst + ch * L::KV_CHUNK + 64 * 128, &tmK, &bars[B_KFULL + ks], ch * 64, kb1 * 64, bh);
          }
          ++g;
          if (++c.t == c.T) c.need = true;
        }
        return true;
      };
      while (ok && (s0.active || s1.active)) {
        ok = turn(s0, 0);
        if (ok) ok = turn(s1, 1);
      }
      // loads still in flight land before the CTA gives up its shared memory
      for (int i = 1; i <= kKStages && i <= g; ++i)
        mbar_drain(&bars[B_KFULL + (g - i) % kKStages], ((g - i) / kKStages) & 1);
    }
  } else if (warp == kVWarp) {
    // ------------------------------------------------------------ V producer
    if (lane == 0) {
      tma_prefetch_desc(&tmV);
      LaneState s0, s1;
      lane_init(s0);
      lane_init(s1);
      int g = 0;
      bool ok = true;
      auto turn = [&](LaneState& c, const int l) -> bool {
        if (c.active && c.need && !take_item(bars, ring, l, c, n_items, abort_flag)) return false;
        if (c.active) {
          const int vs = g % kVStages;
          int kb0, kb1;
          const int nblk = tile_blocks(a, c.item, c.cnt, c.t, kb0, kb1);
          const int bh = c.item / a.nqb;
          if (!mbar_wait(&bars[B_VEMPTY + vs], ((g / kVStages) & 1) ^ 1, abort_flag)) return false;
          mbar_arrive_expect_tx(&bars[B_VFULL + vs], nblk * L::BLK_BYTES);
          uint8_t* dst = sV + vs * L::TILE_BYTES;
#pragma unroll
          for (int ch = 0; ch < L::NCH; ++ch) {
            tma_load_3d(dst + ch * L::KV_CHUNK, &tmV, &bars[B_VFULL + vs], ch * 64, kb0 * 64, bh);
            if (nblk > 1)
              tma_load_3d(dst + ch * L::KV_CHUNK + 64 * 128, &tmV, &bars[B_VFULL + vs], ch * 64, kb1 * 64, bh);
          }
          ++g;
          if (++c.t == c.T) c.need = true;
        }
        return true;
      };
      while (ok && (s0.active || s1.active)) {
        ok = turn(s0, 0);
        if (ok) ok = turn(s1, 1);
      }
      for (int i = 1; i <= kVStages && i <= g; ++i)
        mbar_drain(&bars[B_VFULL + (g - i) % kVStages], ((g - i) / kVStages) & 1);
    }
  } else if (warp == kQWarp) {
    // ------------------------------------------------------------ Q producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      int loads[kQSlots] = {0, 0, 0};
      bool ok = true;
      for (int r = 0; ok; ++r) {
        // one request per non-empty item of this CTA, in order, then one with item n_items
        const int rs = r % kQReqRing;
        if (!(ok = mbar_wait(&bars[B_RFULL + rs], (r / kQReqRing) & 1, abort_flag))) break;
        const int item = qreq[rs * 2 + 0];
        const int qs = qreq[rs * 2 + 1];
        mbar_arrive(&bars[B_REMPTY + rs]);
        if (item >= n_items) break;
        if (!(ok = mbar_wait(&bars[B_QEMPTY + qs], (loads[qs] & 1) ^ 1, abort_flag))) break;
        const Item it = load_item(a, item);
        mbar_arrive_expect_tx(&bars[B_QFULL + qs], L::Q_BYTES);
#pragma unroll
        for (int ch = 0; ch < L::NCH; ++ch)
          tma_load_3d(sQ + qs * L::Q_BYTES + ch * L::Q_CHUNK, &tmQ, &bars[B_QFULL + qs], ch * 64, it.qb * a.bq, it.bh);
        ++loads[qs];
      }
      for (int qs = 0; qs < kQSlots; ++qs)
        if (loads[qs] > 0) mbar_drain(&bars[B_QFULL + qs], (loads[qs] - 1) & 1);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint64_t qdesc0 = sw128_desc(smem_u32(sQ), 16, 1024);
      const uint64_t kdesc0 = sw128_desc(smem_u32(sK), 16, 1024);
      const uint64_t vdesc0 = sw128_desc(smem_u32(sV), L::KV_CHUNK, 1024);
      const uint32_t idesc_pv = idesc_bf16_f32(kBM, D, false, true);
      const uint32_t idesc_qk2 = idesc_bf16_f32(kBM, 128, false, false);
      const uint32_t idesc_qk1 = idesc_bf16_f32(kBM, 64, false, false);
      // the P V each lane still owes for the last tile whose Q K^T it issued
      struct Pend {
        int g, nblk, lt, oi;
        bool first, last, valid;
      };
      // per lane: the pending P V, tiles issued (S / P phases), items issued (O phases)
      struct LaneMma {
        Pend pend;
        int lt, oi;
      };
      LaneMma m0{}, m1{};
      int quse0 = 0, quse1 = 0, quse2 = 0;   // items that have read each Q slot (Q phases)
      LaneState s0, s1;
      lane_init(s0);
      lane_init(s1);
      int g = 0;
      bool ok = true;
      auto issue_pv = [&](LaneMma& mm, const int ln) -> bool {
        Pend& p = mm.pend;
        if (!mbar_wait(&bars[B_PFULL + ln], p.lt & 1, abort_flag)) return false;
        if (!mbar_wait(&bars[B_VFULL + p.g % kVStages], (p.g / kVStages) & 1, abort_flag)) return false;
        if (p.first && !mbar_wait(&bars[B_OEMPTY + ln], (p.oi & 1) ^ 1, abort_flag)) return false;
        tc_fence_after();
        const uint64_t vd = vdesc0 + (((p.g % kVStages) * L::TILE_BYTES) >> 4);
        const uint32_t p_tm = tm + tm_s(ln);
        const uint32_t o_tm = tm + tm_o(ln);
        const int nk = p.nblk * 4;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          if (kk < nk) umma_ts(o_tm, p_tm + kk * 8, vd + ((kk * 2048u) >> 4), idesc_pv, (p.first && kk == 0) ? 0u : 1u);
        tc_commit(&bars[B_VEMPTY + p.g % kVStages]);   // V slot free once this P V has read it
        if (p.last) tc_commit(&bars[B_OFULL + ln]);
        p.valid = false;
        return true;
      };
      auto turn = [&](LaneState& c, LaneMma& mm, const int l) -> bool {
        if (c.active && c.need) {
          if (!take_item(bars, ring, l, c, n_items, abort_flag)) return false;
          if (!c.active && mm.pend.valid && !issue_pv(mm, l)) return false;
        }
        if (c.active) {
          if (mm.pend.valid && !issue_pv(mm, l)) return false;
          const int ks = g % kKStages;
          const int qs = c.qslot;
          int& quse = qs == 0 ? quse0 : (qs == 1 ? quse1 : quse2);
          if (!mbar_wait(&bars[B_KFULL + ks], (g / kKStages) & 1, abort_flag)) return false;
          if (c.t == 0 && !mbar_wait(&bars[B_QFULL + qs], quse & 1, abort_flag)) return false;
          tc_fence_after();
          const int nblk = min(2, c.cnt - 2 * c.t);
          const uint32_t idesc = nblk == 2 ? idesc_qk2 : idesc_qk1;
          const uint64_t qd = qdesc0 + ((qs * L::Q_BYTES) >> 4);
          const uint64_t kd = kdesc0 + ((ks * L::TILE_BYTES) >> 4);
          const uint32_t s_tm = tm + tm_s(l);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            umma_ss(s_tm, qd + ((((kk >> 2) * L::Q_CHUNK) + (kk & 3) * 32u) >> 4),
                    kd + ((((kk >> 2) * L::KV_CHUNK) + (kk & 3) * 32u) >> 4), idesc, kk > 0 ? 1u : 0u);
          tc_commit(&bars[B_SFULL + l]);      // S ready (and O through the lane's previous tile)
          tc_commit(&bars[B_KEMPTY + ks]);
          mm.pend = Pend{g, nblk, mm.lt, mm.oi, c.t == 0, c.t + 1 == c.T, true};
          if (c.t + 1 == c.T) {
            tc_commit(&bars[B_QEMPTY + qs]);   // the slot may take another item's Q
            ++quse;
            ++mm.oi;
          }
          ++mm.lt;
          ++g;
          if (++c.t == c.T) c.need = true;
        }
        return true;
      };
      while (ok && (s0.active || s1.active)) {
        ok = turn(s0, m0, 0);
        if (ok) ok = turn(s1, m1, 1);
      }
      // every MMA issued has completed before tensor memory is released
      tc_commit(&bars[B_DRAIN]);
      mbar_drain(&bars[B_DRAIN], 0);
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue of one lane
    const int ln = (warp - kSoftWarp0) / kLaneWarps;
    const int quad = warp & 3;                // TMEM lane quadrant
    const int row = quad * 32 + lane;         // query row within the tile
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t s_tm = tm + lane_addr + tm_s(ln);
    const uint32_t o_tm = tm + lane_addr + tm_o(ln);
    const float sl2 = a.scale_log2;
    const int tail_valid = a.N - (a.nkb - 1) * 64;
    int n = 0, lt = 0, oi = 0;
    bool ok = true;
    while (ok) {
      const int slot = n % kItemRing;
      // waits in these warps end the same way on every lane (a timeout on one
      // lane stops the whole warp), so the warp stays converged
      if (!(ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bars[B_IFULL + ln * kItemRing + slot], (n / kItemRing) & 1, abort_flag)))) break;
      const volatile int* e = ring + (ln * kItemRing + slot) * 4;
      const int item = e[0], cnt = e[1];
      const bool tail = e[2] != 0;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[B_IEMPTY + ln * kItemRing + slot]);
      ++n;
      if (item >= n_items) break;
      const int bh = item / a.nqb, qb = item % a.nqb;
      const int grow = qb * a.bq + row;
      const bool store = row < a.bq && grow < a.N;
      const long long orow_off = (static_cast<long long>(bh) * a.N + grow) * D;
      if (cnt == 0) {
        if (store) {
          uint4* dz = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.o) + orow_off);
#pragma unroll
          for (int c = 0; c < D / 8; ++c) dz[c] = make_uint4(0, 0, 0, 0);
          if (a.lse) a.lse[static_cast<long long>(bh) * a.N + grow] = -INFINITY;
        }
        continue;
      }
      const int T = (cnt + 1) >> 1;
      if (a.alpha && store) {
        // the epilogue reads this row of O_l: bring it into L2 while the item runs
        const char* olr = reinterpret_cast<const char*>(static_cast<const __nv_bfloat16*>(a.o_l) + orow_off);
#pragma unroll
        for (int b = 0; b < D * 2; b += 128) asm volatile("prefetch.global.L2 [%0];" ::"l"(olr + b));
      }
      float m = -INFINITY;     // running max, log2 domain
      float lsum = 0.f;        // running row sum
      for (int t = 0; t < T; ++t, ++lt) {
        if (!(ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bars[B_SFULL + ln], lt & 1, abort_flag)))) break;
        tc_fence_after();
        uint32_t r[128];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) tmem_ld32(s_tm + q4 * 32, *reinterpret_cast<uint32_t(*)[32]>(r + 32 * q4));
        tmem_wait_ld();
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) reg_fence(*reinterpret_cast<uint32_t(*)[32]>(r + 32 * q4));
        float x[128];
#pragma unroll
        for (int c = 0; c < 128; ++c) x[c] = __uint_as_float(r[c]);
        if (t == T - 1) {
          // last tile: possibly a single block, possibly the ragged last key block
          const int nblk = cnt - 2 * t;
          const int valid = (nblk - 1) * 64 + (tail ? tail_valid : 64);
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c >= valid) x[c] = -INFINITY;
        }
        // row max: eight chains of 3-input max
        float mx8[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          mx8[j] = x[j];
#pragma unroll
          for (int c = 8; c < 128; c += 16) mx8[j] = fmax3(mx8[j], x[c + j], x[c + 8 + j]);
        }
        const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
        const float m_tile = mx * sl2;
        float corr = 1.f;
        if (m_tile > m + kRescaleLog2) {
          corr = fast_exp2(m - m_tile);   // 0 on the first tile (m = -inf)
          m = m_tile;
          lsum *= corr;
        }
        if (t > 0 && __any_sync(0xFFFFFFFFu, corr != 1.f)) {
          // O holds the lane's tiles up to t-1 (their P V completed before this S)
#pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t o[32];
            tmem_ld32_wait(o_tm + c0, o);
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * corr);
            tmem_st32(o_tm + c0, o);
          }
        }
        // P = 2^(S * scale * log2(e) - m), two columns per packed instruction,
        // written as bf16 over the first 64 columns of S.
        const uint64_t sl2x2 = f2_make(sl2, sl2);
        const uint64_t negm2 = f2_make(-m, -m);
        uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};   // packed (+0, +0)
        auto exp_quarter = [&](const float* xq, int h) {
          uint32_t p[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const uint64_t a2 = ffma2(f2_make(xq[2 * c], xq[2 * c + 1]), sl2x2, negm2);
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
            p[c] = pack_bf16x2(e0, e1);
          }
          tmem_st16(s_tm + h * 16, p);
        };
        exp_quarter(x, 0);
        exp_quarter(x + 32, 1);
        // columns 64..127 again from S (P only covers columns 0..63), so the
        // upper half of the row need not stay in registers through the first half
        {
          uint32_t r2[64];
          tmem_ld32(s_tm + 64, *reinterpret_cast<uint32_t(*)[32]>(r2));
          tmem_ld32(s_tm + 96, *reinterpret_cast<uint32_t(*)[32]>(r2 + 32));
          tmem_wait_ld();
          reg_fence(*reinterpret_cast<uint32_t(*)[32]>(r2));
          reg_fence(*reinterpret_cast<uint32_t(*)[32]>(r2 + 32));
          float y[64];
#pragma unroll
          for (int c = 0; c < 64; ++c) y[c] = __uint_as_float(r2[c]);
          if (t == T - 1) {
            const int nblk = cnt - 2 * t;
            const int valid = (nblk - 1) * 64 + (tail ? tail_valid : 64) - 64;
#pragma unroll
            for (int c = 0; c < 64; ++c)
              if (c >= valid) y[c] = -INFINITY;
          }
          exp_quarter(y, 2);
          exp_quarter(y + 32, 3);
        }
        {
          float s0, s1;
          f2_split(fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3])), s0, s1);
          lsum += s0 + s1;
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[B_PFULL + ln]);
      }
      if (!ok) break;
      // ---------------------------------------------------------- epilogue
      if (!(ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bars[B_OFULL + ln], oi & 1, abort_flag)))) break;
      ++oi;
      tc_fence_after();
      uint32_t o[D];
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) tmem_ld32(o_tm + c0, *reinterpret_cast<uint32_t(*)[32]>(o + c0));
      tmem_wait_ld();
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) reg_fence(*reinterpret_cast<uint32_t(*)[32]>(o + c0));
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[B_OEMPTY + ln]);   // the lane's next item may overwrite O now
      if (store) {
        const float inv_l = 1.f / lsum;
        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.o) + orow_off);
        if (a.alpha) {
          // O = alpha ⊙ O_s + (1 - alpha) ⊙ O_l, O_s = o / l not yet rounded
          const uint4* ol = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.o_l) + orow_off);
          const float4* al = reinterpret_cast<const float4*>(a.alpha + static_cast<long long>(bh % a.H) * D);
#pragma unroll
          for (int c = 0; c < D / 8; ++c) {
            const uint4 lv = __ldg(ol + c);
            const float4 a0 = __ldg(al + 2 * c), a1 = __ldg(al + 2 * c + 1);
            const uint32_t lw[4] = {lv.x, lv.y, lv.z, lv.w};
            const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            float r8[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float olj = __uint_as_float((j & 1) ? (lw[j >> 1] & 0xFFFF0000u) : (lw[j >> 1] << 16));
              r8[j] = fmaf(av[j], __uint_as_float(o[8 * c + j]) * inv_l - olj, olj);
            }
            dst[c] = make_uint4(pack_bf16x2(r8[0], r8[1]), pack_bf16x2(r8[2], r8[3]),
                                pack_bf16x2(r8[4], r8[5]), pack_bf16x2(r8[6], r8[7]));
          }
        } else {
#pragma unroll
          for (int c = 0; c < D / 8; ++c)
            dst[c] = make_uint4(pack_bf16x2(__uint_as_float(o[8 * c + 0]) * inv_l, __uint_as_float(o[8 * c + 1]) * inv_l),
                                pack_bf16x2(__uint_as_float(o[8 * c + 2]) * inv_l, __uint_as_float(o[8 * c + 3]) * inv_l),
                                pack_bf16x2(__uint_as_float(o[8 * c + 4]) * inv_l, __uint_as_float(o[8 * c + 5]) * inv_l),
                                pack_bf16x2(__uint_as_float(o[8 * c + 6]) * inv_l, __uint_as_float(o[8 * c + 7]) * inv_l));
        }
        if (a.lse) a.lse[static_cast<long long>(bh) * a.N + grow] = (m + log2f(lsum)) * 0.69314718055994531f;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tm, TM_COLS);
  }
}

template <int D>
static cudaError_t launch_d(const AttnArgs& a, cudaStream_t st) {
  using L = attn::Layout<D>;
  CUtensorMap mq, mk, mv;
  if (encode_tensor_map_3d_bf16(&mq, a.q, D, a.N, a.BH, 64, attn::kBM) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  if (encode_tensor_map_3d_bf16(&mk, a.k, D, a.N, a.BH, 64, 64) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  if (encode_tensor_map_3d_bf16(&mv, a.v, D, a.N, a.BH, 64, 64) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(sparse_attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long items = static_cast<long long>(a.BH) * a.nqb;
  const int grid = static_cast<int>(items < sms ? items : sms);
  sparse_attn_kernel<D><<<grid, attn::kThreads, L::SMEM, st>>>(mq, mk, mv, a);
  return cudaGetLastError();
}

cudaError_t launch_sparse_attn(const AttnArgs& a, cudaStream_t st) {
  if (static_cast<long long>(a.BH) * a.nqb > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  return a.d == 128 ? launch_d<128>(a, st) : launch_d<64>(a, st);
}

}  // namespace sa
