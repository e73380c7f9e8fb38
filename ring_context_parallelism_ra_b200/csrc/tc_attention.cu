// Tensor-core (tcgen05) attention for bf16 inputs: the fused ring forward and
// the single-block partial.
//
// Method (pages cited by title and section): query partition i stays in place
// while the KV partitions pass in ring order j = i, i-1, ..., i-P+1 (mod P)
// ("AI 推理系列（十一）：Ring Attention 如何让多张 GPU 共同计算一条超长序列",
// "KV 在 Ring 中如何流动"); a KV block wholly in the causal future is skipped
// (same section); each visible block is folded into a running row max, a
// running exponential sum and a rescaled output (same page, "最容易被忽略的细
// 节"), never writing the score matrix to memory.  On one GPU the ring is a
// schedule: the "next KV block" is the next K/V tile, prefetched by TMA into a
// shared-memory ring while the tensor cores work on the current one (the
// overlap of "通信很多，为什么仍然可能划算").
//
// CTA layout (384 threads, one CTA per SM, persistent):
//   warps 0-3  softmax for query tile 0 (row r of the tile = thread r)
//   warps 4-7  softmax for query tile 1
//   warp 8     TMA producer: Q tiles, then K_j, V_j into a slot ring
//   warp 9     tcgen05.mma issuer; owns the tensor-memory allocation
//   warps 10-11 idle
// Warp w runs on sub-partition w % 4, so each sub-partition holds one warp of
// each warpgroup.  The kernel is launched with 168 registers per thread;
// setmaxnreg then moves registers from the third warpgroup to the two softmax
// warpgroups within that launch allocation: 2 x 192 + 120 = 504 = 3 x 168 per
// lane.  (setmaxnreg.inc waits until registers are free, so a split above the
// launch allocation would never proceed; the launcher checks the compiled
// register count against the split before every launch.)
// Work item = 256 query rows (two 128-row tiles) of one (batch, head); items
// come in blocks of KV heads whose K/V fit in L2, heaviest first within a
// block, and the producer of each persistent CTA takes the next one from a
// global counter.
//
// Tensor memory (512 columns x 128 lanes, fp32):
//   [  0,128) S0 = Q0 K^T   (P0 as packed bf16 over its first 64 columns)
//   [128,256) S1 = Q1 K^T   (P1 likewise)
//   [256,256+DV) O0, [384,384+DV) O1   accumulators of P V
// MMA issue order per KV tile j: PV0(j), S0(j+1), PV1(j), S1(j+1), so the
// softmax of one tile overlaps the tensor-core work of the other.  MMAs from
// one thread execute in issue order, so S_a(j+1) overwrites P_a(j) only after
// PV_a(j) has read it, and a completed S_a(j+1) implies PV_a(j) is complete
// (the softmax may then rescale O_a safely before releasing P_a(j+1)).
// Rescaling is skipped unless the row max grows by more than 2^8 (the stale
// max keeps p <= 256; the final division by l makes the result exact).
#include <cuda.h>

#include "block_class.cuh"
#include "common.cuh"
#include "item_queue.cuh"
#include "launch.h"
#include "ptx.cuh"
#include "tmap.h"

namespace ra {

namespace {

constexpr int kBM = 128;          // query rows per tile
constexpr int kBN = 128;          // keys per KV tile
constexpr int kBox = 128 * 64 * 2;  // one TMA box: 128 rows x 64 bf16 = 16 KB
constexpr int kThreads = 384;
constexpr int kRegsLaunch = 168;    // per thread at launch (384 threads, 1 CTA / SM)
constexpr int kRegsSoftmax = 192;   // per thread, softmax warpgroups
constexpr int kRegsOther = 120;     // per thread, producer / MMA warpgroup
static_assert(2 * kRegsSoftmax + kRegsOther <= 3 * kRegsLaunch,
              "register split must fit the launch allocation");
constexpr int kSmemLimit = 232448;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

constexpr int kNT = 16;             // barriers / headers of K and V loads in flight

template <int DQK, int DV>
struct Cfg {
  static constexpr int QBOX = DQK / 64;
  static constexpr int VBOX = DV / 64;
  static constexpr int QTILE = QBOX * kBox;
  // K and V tiles stream through a ring of 16 KB units (one TMA box each): a
  // K tile takes QBOX units (it may wrap around the ring), a V tile VBOX
  // units (kept contiguous: its MMA reads both boxes through one descriptor)
  static constexpr int NUNIT_FIT = (kSmemLimit - 2048 - 2 * QTILE) / kBox;
  static constexpr int NUNIT = NUNIT_FIT > 12 ? 12 : NUNIT_FIT;
  static constexpr int SMEM = 1024 + 2 * QTILE + NUNIT * kBox + 1024;
  // V(j) and K(j+1) are in use together; a V tile may skip up to VBOX - 1
  // units at the end of the ring
  static_assert(NUNIT >= QBOX + 2 * VBOX - 1, "K/V ring too small");
  static_assert(NUNIT <= kNT, "every unit's last load must keep its barrier");
  static_assert(SMEM <= kSmemLimit, "shared memory budget");
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(128, kBN, 0, 0);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, DV, 0, 1);
};

struct TcArgs {
  int B, Hq, Hkv, n_q, n_k, P;
  int q_offset, k_offset, causal;
  int striped;        // 1: row r of partition i is token r * P + i (needs n / P % 256 == 0)
  long long stride;   // position stride (1 contiguous; P striped; any for a strided block)
  float scale_log2;
  void* out;          // [B*Hq, n_q, DV] bf16 or fp32
  float* lse;         // [B*Hq, n_q] or null
  int n_pairs, items;
  int Lq, Lk;         // rows / keys per partition (n_q / P, n_k / P)
  int kv_block;       // (batch, KV head)s per block of items (see item_from_index)
  unsigned int* item_counter;  // items handed out so far (zeroed before the launch)
  DevCtx ctx;
};

// Query rows / ring partition of one work item.
struct Item {
  int bh, b, g;
  int q0[2], qlen[2];
  int i;           // ring partition of the item's first row
  long long qoff;  // query position = qoff + row * stride
};

// Position offset of a partition: contiguous tokens use the call's offsets;
// in the striped split (stride P), tensor row R of partition p (R - p * L its
// index inside the partition) is token (R - p * L) * P + p = R * P + p * (1 -
// L * P).
__device__ __forceinline__ long long pos_stride(const TcArgs& a) { return a.stride; }
__device__ __forceinline__ long long part_offset(const TcArgs& a, int p, int len, int base) {
  return a.striped ? static_cast<long long>(p) * (1 - static_cast<long long>(len) * a.P)
                   : static_cast<long long>(base);
}

// Item `idx` in the order work is handed out (from a global counter, see
// item_queue.cuh): blocks of kv_block (batch, KV head)s whose K and V fit in
// L2 together, every item of a block -- heaviest pairs first, the query heads
// of the block next to each other -- before the next block's, so the CTAs
// that run at the same time stream the same K/V tiles.
__device__ __forceinline__ void item_from_index(const TcArgs& a, long long idx, Item& it) {
  const int G = a.Hq / a.Hkv;
  const int n_kv = a.B * a.Hkv;
  const long long per_kv = static_cast<long long>(a.n_pairs) * G;
  const int blk = static_cast<int>(idx / (per_kv * a.kv_block));
  const int kv0 = blk * a.kv_block;
  const int hb = n_kv - kv0 < a.kv_block ? n_kv - kv0 : a.kv_block;
  const long long in_blk = idx - static_cast<long long>(kv0) * per_kv;
  const int r = static_cast<int>(in_blk / (static_cast<long long>(G) * hb));
  const int within = static_cast<int>(in_blk % (static_cast<long long>(G) * hb));
  const int kvh = kv0 + within / G;
  it.bh = (kvh / a.Hkv) * a.Hq + (kvh % a.Hkv) * G + within % G;
  // heaviest pairs first when causal: work grows with the row's token
  // position, i.e. with the pair index (contiguous) or with the pair index
  // inside its partition (striped, all partitions' pairs of one index together)
  int tp = r;
  if (a.causal) {
    if (a.striped) {
      const int pp = a.n_pairs / a.P;  // pairs per partition (n / P % 256 == 0)
      tp = (r % a.P) * pp + (pp - 1 - r / a.P);
    } else {
      tp = a.n_pairs - 1 - r;
    }
  }
  it.b = it.bh / a.Hq;
  it.g = (it.bh % a.Hq) / (a.Hq / a.Hkv);
  for (int t = 0; t < 2; ++t) {
    it.q0[t] = tp * 2 * kBM + t * kBM;
    const int rem = a.n_q - it.q0[t];
    it.qlen[t] = rem <= 0 ? 0 : (rem < kBM ? rem : kBM);
  }
  const int i = it.q0[0] / a.Lq;
  it.i = i < a.P - 1 ? i : a.P - 1;
  it.qoff = part_offset(a, it.i, a.Lq, a.q_offset);
}

// The KV tiles an item visits, in ring order; every role runs this same walk.
struct TileWalk {
  int s, j, kt, kend;
  long long koff;  // key position = koff + key index * stride, partition j
  __device__ __forceinline__ void start(const TcArgs& a, const Item& it) {
    s = 0;
    j = it.i;
    kt = j * a.Lk;
    kend = kt + a.Lk;
    koff = part_offset(a, j, a.Lk, a.k_offset);
  }
  // Next tile with at least one active query tile: kt0, klen, the partition's
  // key offset and the class per query tile.
  __device__ __forceinline__ bool next(const TcArgs& a, const Item& it, int& kt0, int& klen,
                                       long long& koff_out, int8_t (&cls)[2]) {
    const long long st = pos_stride(a);
    while (true) {
      if (kt >= kend) {
        if (++s >= a.P) return false;
        j = j == 0 ? a.P - 1 : j - 1;
        kt = j * a.Lk;
        kend = kt + a.Lk;
        koff = part_offset(a, j, a.Lk, a.k_offset);
        continue;
      }
      const int len = kend - kt < kBN ? kend - kt : kBN;
      for (int t = 0; t < 2; ++t)
        cls[t] = it.qlen[t] > 0 ? tile_class(it.q0[t], it.qlen[t], kt, len, it.qoff, koff,
                                              a.causal, st)
                                : static_cast<int8_t>(kSkip);
      if (cls[0] == kSkip && cls[1] == kSkip) {
        // key positions only grow inside a partition: with a causal mask
        // nothing later in this partition is visible either
        if (a.causal) kt = kend; else kt += kBN;
        continue;
      }
      kt0 = kt;
      klen = len;
      koff_out = koff;
      kt += kBN;
      return true;
    }
  }
};

// The tiles one query tile visits, in the same ring order as TileWalk but
// only those whose class for this query tile is not SKIP (exactly the tiles
// whose S the MMA thread computes for it).  Used by the softmax warpgroups;
// scalar state only, so nothing of it lands in local memory.
struct RowWalk {
  int s, j, kt, kend, i;
  long long koff, q0, qlen, qoff;
  __device__ __forceinline__ void start(const TcArgs& a, const Item& it, int t) {
    q0 = t ? it.q0[1] : it.q0[0];
    qlen = t ? it.qlen[1] : it.qlen[0];
    qoff = it.qoff;
    i = it.i;
    s = 0;
    j = i;
    kt = j * a.Lk;
    kend = qlen > 0 ? kt + a.Lk : kt;   // a tile without rows visits nothing
    if (qlen <= 0) s = a.P;
    koff = part_offset(a, j, a.Lk, a.k_offset);
  }
  __device__ __forceinline__ bool next(const TcArgs& a, int& kt0, int& klen, long long& koff_out,
                                       int8_t& cls) {
    const long long st = pos_stride(a);
    while (true) {
      if (kt >= kend) {
        if (++s >= a.P) return false;
        j = j == 0 ? a.P - 1 : j - 1;
        kt = j * a.Lk;
        kend = kt + a.Lk;
        koff = part_offset(a, j, a.Lk, a.k_offset);
        continue;
      }
      const int len = kend - kt < kBN ? kend - kt : kBN;
      cls = tile_class(q0, qlen, kt, len, qoff, koff, a.causal, st);
      if (cls == kSkip) {
        // key positions only grow inside a partition
        if (a.causal) kt = kend; else kt += kBN;
        continue;
      }
      kt0 = kt;
      klen = len;
      koff_out = koff;
      kt += kBN;
      return true;
    }
  }
};

// Descriptors of successive K steps differ only in the start-address field
// (bits 0-13, address >> 4), which never carries out for shared memory, so
// they are formed by adding (byte offset >> 4) to the tile's base descriptor.
// First unit of the next K (contiguous = false) or V (contiguous = true) tile
// of `n` units; producer and MMA thread run the same sequence of calls.
template <int NUNIT>
__device__ __forceinline__ int alloc_units(int& pos, int n, bool contiguous) {
  if (contiguous && pos + n > NUNIT) pos = 0;
  const int u0 = pos;
  pos += n;
  if (pos >= NUNIT) pos -= NUNIT;
  return u0;
}

// Header of a K load, written by the producer before the load is armed:
// the two query tiles' classes and whether it is the item's last K/V tile.
__device__ __forceinline__ uint32_t tile_header(const int8_t (&cls)[2], bool last) {
  return static_cast<uint32_t>(static_cast<uint8_t>(cls[0])) |
         (static_cast<uint32_t>(static_cast<uint8_t>(cls[1])) << 8) | (last ? (1u << 16) : 0u);
}

template <int DQK, int DV>
__device__ __forceinline__ void issue_s(uint32_t tmem_d, uint32_t q_base, uint32_t kv_base,
                                        int ku0) {
  using C = Cfg<DQK, DV>;
  const uint64_t da = sdesc_k_sw128(q_base);
  uint64_t db[C::QBOX];
#pragma unroll
  for (int b = 0; b < C::QBOX; ++b) {
    const int u = ku0 + b < C::NUNIT ? ku0 + b : ku0 + b - C::NUNIT;
    db[b] = sdesc_k_sw128(kv_base + u * kBox);
  }
#pragma unroll
  for (int ks = 0; ks < DQK / 16; ++ks) {
    const uint32_t qoff = ((ks >> 2) * kBox + (ks & 3) * 32) >> 4;
    const uint32_t koff = ((ks & 3) * 32) >> 4;
    umma_ss(tmem_d, da + qoff, db[ks >> 2] + koff, C::IDESC_S, ks > 0 ? 1u : 0u);
  }
}

template <int DQK, int DV>
__device__ __forceinline__ void issue_pv(uint32_t tmem_d, uint32_t tmem_p, uint32_t v_base,
                                         bool accumulate) {
  const uint64_t db = sdesc_mn_sw128(v_base, kBox);
#pragma unroll
  for (int ks = 0; ks < kBN / 16; ++ks) {
    umma_ts(tmem_d, tmem_p + ks * 8, db + ((ks * 2048) >> 4), Cfg<DQK, DV>::IDESC_PV,
            (accumulate || ks > 0) ? 1u : 0u);
  }
}

template <int DQK, int DV, bool OUT_F32>
__global__ void __launch_bounds__(kThreads, 1) tc_attention_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_v, TcArgs a) {
  using C = Cfg<DQK, DV>;
  constexpr int NUNIT = C::NUNIT;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = sm;
  uint8_t* sKV = sm + 2 * C::QTILE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sKV + NUNIT * kBox);
  uint64_t* q_full = bars;
  uint64_t* q_empty = bars + 1;
  uint64_t* ld_full = bars + 2;          // [kNT] K / V load L landed
  uint64_t* ld_empty = ld_full + kNT;    // [kNT] load L consumed by the tensor cores
  uint64_t* s_full = ld_empty + kNT;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_full = p_full + 2;
  uint64_t* drain = o_full + 2;
  uint64_t* iq_full = drain + 1;               // [kItemSlots]
  uint64_t* iq_empty = iq_full + kItemSlots;   // [kItemSlots]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(iq_empty + kItemSlots);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* kv_issued = abort_flag + 1;
  volatile int* q_issued = abort_flag + 2;
  volatile uint32_t* item_has_tiles = reinterpret_cast<volatile uint32_t*>(abort_flag + 3);
  volatile uint32_t* hdr = item_has_tiles + 1;  // [kNT] headers of K loads
  int* unit_owner = const_cast<int*>(reinterpret_cast<volatile int*>(hdr + kNT));  // [NUNIT]
  const ItemQueue iq{reinterpret_cast<volatile int*>(unit_owner + NUNIT), iq_full, iq_empty};

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < kNT; ++s) {
      mbar_init(&ld_full[s], 1);
      mbar_init(&ld_empty[s], 1);
    }
    for (int u = 0; u < NUNIT; ++u) unit_owner[u] = -1;
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], kBM);
      mbar_init(&o_full[t], 1);
    }
    mbar_init(drain, 1);
    for (int i = 0; i < kItemSlots; ++i) {
      mbar_init(&iq_full[i], 1);
      mbar_init(&iq_empty[i], 1 + 2 * kBM);  // the MMA thread, the softmax threads
    }
    *abort_flag = 0;
    *kv_issued = 0;
    *q_issued = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp >= 8) regs_dec<kRegsOther>();
  if (warp == 8) {
    // ------------------------------------------------------ TMA producer --
    // Walks each item's tiles one ahead, so that every K load carries the
    // header the MMA thread needs (classes, last tile of the item); a unit
    // is refilled once the load that last used it has been consumed.
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      uint32_t ld = 0, qi = 0;
      int pos = 0;
      Item it;
      bool ok = true;
      // claim `n` units from `u0` for load L: wait until load L - kNT (the
      // previous user of L's barriers and header) has been consumed -- the
      // tensor cores release loads in the order they were issued, so every
      // older load has been too -- and then for each unit's last load where
      // that is more recent.  (A unit the ring skips for a while, e.g. one a
      // contiguous V tile jumps over at the end of the ring, may keep an
      // owner whose barrier has been reused since.)
      auto claim = [&](int u0, int n, uint32_t L) -> bool {
        if (L >= static_cast<uint32_t>(kNT) &&
            !mbar_wait(&ld_empty[L % kNT], ((L - kNT) / kNT) & 1, a.ctx, abort_flag))
          return false;
        int waited = -1;
        for (int b = 0; b < n; ++b) {
          const int u = u0 + b < NUNIT ? u0 + b : u0 + b - NUNIT;
          const int o = unit_owner[u];
          if (o >= 0 && static_cast<uint32_t>(o) + kNT > L && o != waited) {
            if (!mbar_wait(&ld_empty[o % kNT], (static_cast<uint32_t>(o) / kNT) & 1, a.ctx,
                           abort_flag))
              return false;
            waited = o;
          }
          unit_owner[u] = static_cast<int>(L);
        }
        return true;
      };
      for (int round = 0; ok && !*abort_flag; ++round) {
        const int idx = item_publish(iq, a.item_counter, a.items, round, a.ctx, abort_flag);
        if (idx < 0) {
          ok = idx == -1;
          break;
        }
        item_from_index(a, idx, it);
        if (!mbar_wait(q_empty, (qi & 1) ^ 1, a.ctx, abort_flag)) break;
        TileWalk w;
        w.start(a, it);
        int kt, klen, nkt, nklen;
        long long koff, nkoff;
        int8_t cls[2], ncls[2];
        bool have = w.next(a, it, kt, klen, koff, cls);
        *item_has_tiles = have ? 1u : 0u;
        mbar_arrive_expect_tx(q_full, 2 * C::QTILE);
        for (int t = 0; t < 2; ++t)
          for (int bx = 0; bx < C::QBOX; ++bx)
            tma_load_3d(sQ + t * C::QTILE + bx * kBox, &tm_q, q_full, bx * 64, it.q0[t], it.bh);
        *q_issued = static_cast<int>(++qi);
        const int bkv = it.b * a.Hkv + it.g;
        while (have) {
          const bool nhave = w.next(a, it, nkt, nklen, nkoff, ncls);
          // K tile: may wrap around the ring
          uint32_t L = ld;
          int u0 = alloc_units<NUNIT>(pos, C::QBOX, false);
          if (!(ok = claim(u0, C::QBOX, L))) break;
          hdr[L % kNT] = tile_header(cls, !nhave);
          mbar_arrive_expect_tx(&ld_full[L % kNT], C::QBOX * kBox);
          for (int bx = 0; bx < C::QBOX; ++bx) {
            const int u = u0 + bx < NUNIT ? u0 + bx : u0 + bx - NUNIT;
            tma_load_3d(sKV + u * kBox, &tm_k, &ld_full[L % kNT], bx * 64, kt, bkv);
          }
          *kv_issued = static_cast<int>(++ld);
          // V tile: contiguous units
          L = ld;
          u0 = alloc_units<NUNIT>(pos, C::VBOX, true);
          if (!(ok = claim(u0, C::VBOX, L))) break;
          mbar_arrive_expect_tx(&ld_full[L % kNT], C::VBOX * kBox);
          for (int bx = 0; bx < C::VBOX; ++bx)
            tma_load_3d(sKV + (u0 + bx) * kBox, &tm_v, &ld_full[L % kNT], bx * 64, kt, bkv);
          *kv_issued = static_cast<int>(++ld);
          have = nhave;
          kt = nkt;
          klen = nklen;
          koff = nkoff;
          cls[0] = ncls[0];
          cls[1] = ncls[1];
        }
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------- MMA issuer --
    // Follows the producer's loads in order (same unit allocation), reading
    // each K load's header instead of walking the tiles itself: the issuing
    // thread does as little as possible between batches of MMAs, since the
    // tensor pipe idles as soon as its short instruction queue drains.
    if (lane == 0) {
      uint32_t ld = 0, qi = 0, pph[2] = {0, 0};
      int pos = 0;
      const uint32_t q_base[2] = {smem_u32(sQ), smem_u32(sQ + C::QTILE)};
      const uint32_t kv_base = smem_u32(sKV);
      Item it;
      bool ok = true;
      for (int round = 0; ok; ++round) {
        const int idx = item_take(iq, round, a.ctx, abort_flag);
        if (idx < 0) {
          ok = idx == -1;
          break;
        }
        item_from_index(a, idx, it);
        if (!(ok = mbar_wait(q_full, qi & 1, a.ctx, abort_flag))) break;
        ++qi;
        tc_fence_after();
        bool any[2] = {false, false};
        if (*item_has_tiles) {
          uint32_t kL = ld++;
          int ku0 = alloc_units<NUNIT>(pos, C::QBOX, false);
          if (!(ok = mbar_wait(&ld_full[kL % kNT], (kL / kNT) & 1, a.ctx, abort_flag))) break;
          tc_fence_after();
          uint32_t h = hdr[kL % kNT];
          int8_t cls[2] = {static_cast<int8_t>(h & 0xff), static_cast<int8_t>((h >> 8) & 0xff)};
          bool last = (h >> 16) & 1;
          for (int t = 0; t < 2; ++t) {
            if (cls[t] == kSkip) continue;
            issue_s<DQK, DV>(tmem + t * 128, q_base[t], kv_base, ku0);
            umma_commit(&s_full[t]);
          }
          umma_commit(&ld_empty[kL % kNT]);
          while (true) {
            const uint32_t vL = ld++;
            const int vu0 = alloc_units<NUNIT>(pos, C::VBOX, true);
            if (!(ok = mbar_wait(&ld_full[vL % kNT], (vL / kNT) & 1, a.ctx, abort_flag))) break;
            tc_fence_after();
            bool k_ready = false;
            int8_t ncls[2] = {kSkip, kSkip};
            bool nlast = true;
            for (int t = 0; t < 2 && ok; ++t) {
              if (cls[t] != kSkip) {
                if (!(ok = mbar_wait(&p_full[t], pph[t] & 1, a.ctx, abort_flag))) break;
                ++pph[t];
                tc_fence_after();
                issue_pv<DQK, DV>(tmem + 256 + t * 128, tmem + t * 128, kv_base + vu0 * kBox,
                                  any[t]);
                any[t] = true;
              }
              if (!last) {
                if (!k_ready) {
                  kL = ld++;
                  ku0 = alloc_units<NUNIT>(pos, C::QBOX, false);
                  if (!(ok = mbar_wait(&ld_full[kL % kNT], (kL / kNT) & 1, a.ctx, abort_flag)))
                    break;
                  tc_fence_after();
                  h = hdr[kL % kNT];
                  ncls[0] = static_cast<int8_t>(h & 0xff);
                  ncls[1] = static_cast<int8_t>((h >> 8) & 0xff);
                  nlast = (h >> 16) & 1;
                  k_ready = true;
                }
                if (ncls[t] != kSkip) {
                  issue_s<DQK, DV>(tmem + t * 128, q_base[t], kv_base, ku0);
                  umma_commit(&s_full[t]);
                }
              }
            }
            if (!ok) break;
            umma_commit(&ld_empty[vL % kNT]);
            if (last) break;
            umma_commit(&ld_empty[kL % kNT]);
            cls[0] = ncls[0];
            cls[1] = ncls[1];
            last = nlast;
          }
          if (!ok) break;
        }
        for (int t = 0; t < 2; ++t)
          if (any[t]) umma_commit(&o_full[t]);
        umma_commit(q_empty);
      }
      // every MMA issued so far has finished before the allocation goes away
      umma_commit(drain);
      const unsigned long long t0 = globaltimer_ns();
      while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t0 < a.ctx.wait_ns) {
      }
    }
  } else if (warp < 8) {
    // ------------------------------------------------- softmax (2 x WG) --
    regs_inc<kRegsSoftmax>();
    const int t = warp >> 2;            // query tile of this warpgroup
    const int row = threadIdx.x & 127;  // row within the tile = TMEM lane
    const uint32_t lane_base = tmem + ((static_cast<uint32_t>(warp & 3) * 32) << 16);
    const uint32_t s_col = t * 128;
    const uint32_t o_col = 256 + t * 128;
    uint32_t sph = 0, oph = 0;
    Item it;
    bool ok = true;
    for (int round = 0; ok; ++round) {
      const int idx = item_take(iq, round, a.ctx, abort_flag);
      if (idx < 0) {
        ok = idx == -1;
        break;
      }
      item_from_index(a, idx, it);
      float m = -INFINITY, l = 0.f;
      bool any = false;
      const long long st = pos_stride(a);
      RowWalk w;
      w.start(a, it, t);
      int kt, klen;
      long long koff;
      int8_t cls;
      while (w.next(a, kt, klen, koff, cls)) {
        if (!(ok = mbar_wait(&s_full[t], sph & 1, a.ctx, abort_flag))) break;
        ++sph;
        tc_fence_after();
        float s[kBN];
        tmem_ld32f(lane_base + s_col, s);
        tmem_ld32f(lane_base + s_col + 32, s + 32);
        tmem_ld32f(lane_base + s_col + 64, s + 64);
        tmem_ld32f(lane_base + s_col + 96, s + 96);
        tmem_ld_wait();
        reg_fence32(s);
        reg_fence32(s + 32);
        reg_fence32(s + 64);
        reg_fence32(s + 96);
        if (cls == kPartial || klen < kBN) {
          long long lim = klen;
          if (a.causal) {
            const long long vis = visible_keys(w.q0 + row, kt, w.qoff, koff, st);
            lim = vis < lim ? vis : lim;
          }
#pragma unroll
          for (int c = 0; c < kBN; ++c)
            if (c >= lim) s[c] = -INFINITY;
        }
        // row max: eight independent three-input max chains, then a tree
        float mxs[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          float v = fmax3(s[i], s[i + 8], s[i + 16]);
#pragma unroll
          for (int c = 24; c < 120; c += 16) v = fmax3(v, s[c + i], s[c + 8 + i]);
          mxs[i] = fmaxf(v, s[120 + i]);
        }
        const float mx = fmax3(fmax3(mxs[0], mxs[1], mxs[2]), fmax3(mxs[3], mxs[4], mxs[5]),
                               fmaxf(mxs[6], mxs[7]));
        const float m_cand = mx * a.scale_log2;
        const bool grow = m_cand > m + kRescaleThreshold;
        float alpha = 1.f;
        if (grow) {
          alpha = (m == -INFINITY) ? 0.f : fast_exp2(m - m_cand);
          m = m_cand;
        }
        const bool rescale_o = grow && l > 0.f;
        l *= alpha;
        const float neg_m = (m == -INFINITY) ? 0.f : -m;
        // p = 2^(s * scale_log2 - m): packed fp32x2 FMA, exp2, four packed
        // partial sums, bf16 pairs stored into the P columns of tensor memory
        const float2 sc2 = make_float2(a.scale_log2, a.scale_log2);
        const float2 nm2 = make_float2(neg_m, neg_m);
        float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                         make_float2(0.f, 0.f)};
#pragma unroll
        for (int c0 = 0; c0 < kBN; c0 += 32) {
          uint32_t p[16];
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const float2 x = __ffma2_rn(make_float2(s[c0 + c], s[c0 + c + 1]), sc2, nm2);
            const float2 e = make_float2(fast_exp2(x.x), fast_exp2(x.y));
            acc[(c >> 1) & 3] = __fadd2_rn(acc[(c >> 1) & 3], e);
            p[c >> 1] = pack_bf16x2(e.x, e.y);
          }
          tmem_st16(lane_base + s_col + (c0 >> 1), p);
        }
        const float2 acc01 = __fadd2_rn(acc[0], acc[1]);
        const float2 acc23 = __fadd2_rn(acc[2], acc[3]);
        const float rs = (acc01.x + acc01.y) + (acc23.x + acc23.y);
        // O_a holds this item's sum only after its first PV; rescale it when a
        // row of this warp needs it (tcgen05.ld/st are warp-collective).  The
        // previous PV_a is complete: it was issued before S_a of this tile.
        if (__any_sync(0xffffffffu, rescale_o)) {
          const float f = rescale_o ? alpha : 1.f;
#pragma unroll
          for (int c0 = 0; c0 < DV; c0 += 32) {
            float o[32];
            tmem_ld32f(lane_base + o_col + c0, o);
            tmem_ld_wait();
            reg_fence32(o);
            uint32_t ob[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) ob[c] = __float_as_uint(o[c] * f);
            tmem_st32(lane_base + o_col + c0, ob);
          }
        }
        tmem_st_wait();
        l += rs;
        any = true;
        tc_fence_before();
        mbar_arrive(&p_full[t]);
      }
      if (!ok) break;
      // ---- epilogue: O / l and LSE for the rows that exist ----
      const bool valid = row < w.qlen;
      const long long orow = static_cast<long long>(it.bh) * a.n_q + w.q0 + row;
      const float inv = l > 0.f ? 1.f / l : 0.f;
      if (any) {
        if (!(ok = mbar_wait(&o_full[t], oph & 1, a.ctx, abort_flag))) break;
        ++oph;
        tc_fence_after();
      }
#pragma unroll
      for (int c0 = 0; c0 < DV; c0 += 32) {
        float o[32];
        if (any) {
          tmem_ld32f(lane_base + o_col + c0, o);
          tmem_ld_wait();
          reg_fence32(o);
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = 0.f;
        }
        if (valid) {
          if constexpr (OUT_F32) {
            float* dst = static_cast<float*>(a.out) + orow * DV + c0;
#pragma unroll
            for (int c = 0; c < 32; c += 4)
              *reinterpret_cast<float4*>(dst + c) =
                  make_float4(o[c] * inv, o[c + 1] * inv, o[c + 2] * inv, o[c + 3] * inv);
          } else {
            __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.out) + orow * DV + c0;
#pragma unroll
            for (int c = 0; c < 32; c += 8) {
              uint4 v;
              v.x = pack_bf16x2(o[c] * inv, o[c + 1] * inv);
              v.y = pack_bf16x2(o[c + 2] * inv, o[c + 3] * inv);
              v.z = pack_bf16x2(o[c + 4] * inv, o[c + 5] * inv);
              v.w = pack_bf16x2(o[c + 6] * inv, o[c + 7] * inv);
              *reinterpret_cast<uint4*>(dst + c) = v;
            }
          }
        }
      }
      if (valid && a.lse != nullptr)
        a.lse[orow] = l > 0.f ? (m + __log2f(l)) * kLn2 : -INFINITY;
      // the epilogue's TMEM reads are complete (wait::ld) before the next
      // item's first P is released, so the next PV cannot overwrite O early
    }
  }

  // ---------------------------------------------------------- teardown --
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (*abort_flag && threadIdx.x == 0) {
    // let in-flight TMA loads land before shared memory is released (bounded)
    const int n = *kv_issued;
    for (int i = n - kNT < 0 ? 0 : n - kNT; i < n; ++i) {
      const unsigned long long t0 = globaltimer_ns();
      while (!mbar_try_wait(&ld_full[i % kNT], (i / kNT) & 1) &&
             globaltimer_ns() - t0 < a.ctx.wait_ns) {
      }
    }
    const int nq = *q_issued;
    if (nq > 0) {
      const unsigned long long t0 = globaltimer_ns();
      while (!mbar_try_wait(q_full, (nq - 1) & 1) && globaltimer_ns() - t0 < a.ctx.wait_ns) {
      }
    }
  }
  __syncthreads();
  if (warp == 9) tmem_dealloc(tmem, 512);
}

template <int DQK, int DV, bool OUT_F32>
int launch_typed(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                 const TcArgs& args, int grid, cudaStream_t stream) {
  auto kern = tc_attention_kernel<DQK, DV, OUT_F32>;
  constexpr int smem = Cfg<DQK, DV>::SMEM;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return RA_ERR_CUDA;

  kern<<<grid, kThreads, smem, stream>>>(tq, tk, tv, args);
  note_launch();
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

template <bool OUT_F32>
int dispatch(int dqk, int dv, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
             const TcArgs& args, int grid, cudaStream_t st) {
  if (dqk == 128 && dv == 128) return launch_typed<128, 128, OUT_F32>(tq, tk, tv, args, grid, st);
  if (dqk == 192 && dv == 128) return launch_typed<192, 128, OUT_F32>(tq, tk, tv, args, grid, st);
  if (dqk == 64 && dv == 64) return launch_typed<64, 64, OUT_F32>(tq, tk, tv, args, grid, st);
  if (dqk == 64 && dv == 128) return launch_typed<64, 128, OUT_F32>(tq, tk, tv, args, grid, st);
  if (dqk == 128 && dv == 64) return launch_typed<128, 64, OUT_F32>(tq, tk, tv, args, grid, st);
  if (dqk == 192 && dv == 64) return launch_typed<192, 64, OUT_F32>(tq, tk, tv, args, grid, st);
  return RA_ERR_UNSUPPORTED;
}

}  // namespace

int launch_tc_attention(const void* q, const void* k, const void* v, const ra_shape& s, int P,
                        int q_offset, int k_offset, long long stride, int causal,
                        int striped, float scale, void* out, bool out_f32, float* lse,
                        const DeviceInfo& dev, cudaStream_t stream) {
  if (s.dtype != RA_BF16) return RA_ERR_UNSUPPORTED;
  CUtensorMap tq, tk, tv;
  const uint64_t hq = static_cast<uint64_t>(s.B) * s.Hq;
  const uint64_t hkv = static_cast<uint64_t>(s.B) * s.Hkv;
  if (make_tmap_bf16_3d(&tq, q, s.d_qk, s.n_q, hq, s.d_qk * 2ull,
                        static_cast<uint64_t>(s.n_q) * s.d_qk * 2, 64, kBM) != 0 ||
      make_tmap_bf16_3d(&tk, k, s.d_qk, s.n_k, hkv, s.d_qk * 2ull,
                        static_cast<uint64_t>(s.n_k) * s.d_qk * 2, 64, kBN) != 0 ||
      make_tmap_bf16_3d(&tv, v, s.d_v, s.n_k, hkv, s.d_v * 2ull,
                        static_cast<uint64_t>(s.n_k) * s.d_v * 2, 64, kBN) != 0)
    return RA_ERR_CUDA;
  TcArgs a;
  a.B = s.B;
  a.Hq = s.Hq;
  a.Hkv = s.Hkv;
  a.n_q = s.n_q;
  a.n_k = s.n_k;
  a.P = P;
  a.q_offset = q_offset;
  a.k_offset = k_offset;
  a.causal = causal;
  a.striped = striped;
  a.stride = striped ? P : stride;
  a.scale_log2 = scale * kLog2e;
  a.out = out;
  a.lse = lse;
  a.n_pairs = (s.n_q + 2 * kBM - 1) / (2 * kBM);
  a.Lq = s.n_q / P;
  a.Lk = s.n_k / P;
  const long long items = static_cast<long long>(a.n_pairs) * s.B * s.Hq;
  if (items > 0x7fffffffLL) return RA_ERR_UNSUPPORTED;
  a.items = static_cast<int>(items);
  // as many (batch, KV head)s per block of items as fit 48 MB of K and V
  // (well inside the 126 MB L2, which the query tiles stream through too)
  const long long kv_bytes = static_cast<long long>(s.n_k) * (s.d_qk + s.d_v) * 2;
  const long long fit = (48ll << 20) / (kv_bytes > 0 ? kv_bytes : 1);
  const long long n_kv = static_cast<long long>(s.B) * s.Hkv;
  a.kv_block = static_cast<int>(fit < 1 ? 1 : (fit > n_kv ? n_kv : fit));
  a.ctx = dev.ctx;
  const int rc = next_item_counter(dev, stream, &a.item_counter);
  if (rc != RA_OK) return rc;
  const int grid = a.items < dev.num_sms ? a.items : dev.num_sms;
  return out_f32 ? dispatch<true>(s.d_qk, s.d_v, tq, tk, tv, a, grid, stream)
                 : dispatch<false>(s.d_qk, s.d_v, tq, tk, tv, a, grid, stream);
}

}  // namespace ra
