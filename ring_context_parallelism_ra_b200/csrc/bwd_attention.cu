// Backward pass of exact attention on the tensor cores (bf16 inputs) and the
// launcher of the whole backward call (row statistics, the gradient kernel of
// the input dtype, the dQ conversion).  What is computed is stated in bwd.cuh;
// the row kernels are in bwd_rows.cu.
//
// CTA layout of the tensor-core kernel (384 threads, one CTA per SM,
// persistent; work item = one 128-key tile of one (batch, KV head)):
//   warp 0      TMA producer: K, V of the item; then per visit Q, dO (TMA) and
//               the visit's -LSE log2(e) and D vectors (bulk copies), two stages
//   warps 1-3   tcgen05.mma issuers (three, see below); warp 1 owns the
//               tensor-memory allocation
//   warps 4-11  "compute", two warpgroups, query columns 0-63 and 64-127:
//               thread r owns key r of the tile (TMEM lane r) and forms
//               P^T = 2^(scale log2(e) S^T - LSE log2(e)) (into TMEM as bf16)
//               and dS^T = P^T (dP^T - D) (into shared memory as bf16) for
//               its half; between the two it reads the previous visit's dQ
//               (its half of the columns, lane r = query r) out of TMEM and
//               adds it into the fp32 workspace with 16-byte vector
//               reductions; at the end of the item it writes its half of dK, dV
// Registers: launched at 168 per thread; setmaxnreg moves them to 2 x 184
// (compute) + 136 (producer / MMA warpgroup) = 504 = 3 x 168.
//
// Per visit (query tile t of head h against the item's key tile):
//   S^T  = K Q_t^T        M = 128 keys, N = 128 queries   (A, B K-major)
//   dP^T = V dO_t^T       M = 128 keys, N = 128 queries   (A, B K-major)
//   dV  += P^T dO_t       A = P^T in TMEM, B = dO_t MN-major
//   dK  += dS^T Q_t       A = dS^T K-major, B = Q_t MN-major
//   dQ_t = dS K           A = the same dS bytes read MN-major, B = K MN-major
// The dS tile is written once: its rows (keys) of 64 query columns in
// 128-byte-swizzled atoms are at the same time the K-major layout of dS^T and
// the MN-major layout of dS.
//
// Tensor memory (512 columns): S^T [0,128) (P^T packed over its first 64
// columns), dP^T [128,256) (dQ over it once the compute warps have loaded
// dP^T), dV [256,256+DV), dK [256+DV,256+DV+DQK).
// Products per visit v and their issuers: A issues dV(v) then S^T(v+1), B
// issues dK(v), C issues dQ(v) then dP^T(v+1).  MMAs of one thread execute
// in issue order, so S^T(v+1) overwrites P^T(v) only after dV(v) has read
// it; dP^T(v+1) waits until the compute warps have read dQ(v) out; the
// compute warps form P^T(v+1) while the tensor cores run dK(v) and dQ(v).
// Where the products of two issuers meet (the stage of Q / dO, the K / V
// tile, the finished dK / dV) the barrier takes one commit from each.
#include <cuda.h>

#include "block_class.cuh"
#include "bwd.cuh"
#include "bwd_tc.cuh"
#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"
#include "tmap.h"

namespace ra {

namespace {

constexpr int kT = 128;
constexpr int kBox = 128 * 64 * 2;  // TMA box: 128 rows x 64 bf16
constexpr int kThreads = 384;
constexpr int kRegsLaunch = 168;
constexpr int kRegsCompute = 184;
constexpr int kRegsOther = 136;
static_assert(2 * kRegsCompute + kRegsOther <= 3 * kRegsLaunch,
              "register split must fit the launch allocation");
// setmaxnreg.inc may only raise a warpgroup's count and .dec only lower it.
static_assert(kRegsCompute >= kRegsLaunch, "compute warpgroups grow (setmaxnreg.inc)");
static_assert(kRegsOther <= kRegsLaunch, "producer / MMA warpgroup shrinks (setmaxnreg.dec)");
constexpr int kSmemLimit = 232448;

template <int DQK, int DV>
struct BCfg {
  static constexpr int QB = DQK / 64;
  static constexpr int VB = DV / 64;
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = K_OFF + QB * kBox;
  static constexpr int Q_OFF = V_OFF + VB * kBox;      // two stages
  static constexpr int DO_OFF = Q_OFF + 2 * QB * kBox;  // two stages
  static constexpr int DS_OFF = DO_OFF + 2 * VB * kBox;
  static constexpr int VEC_OFF = DS_OFF + 2 * kBox;     // [stage][-LSE log2e | D][128]
  static constexpr int BAR_OFF = VEC_OFF + 2 * 2 * kT * 4;
  static constexpr int USED = BAR_OFF + 256;
  static_assert(USED <= kSmemLimit, "shared memory budget");
  // Room left for aligning the dynamic shared memory base to 1024 bytes.
  static constexpr int SMEM = USED + 1024 <= kSmemLimit ? USED + 1024 : kSmemLimit;
  static constexpr int S_COL = 0;
  static constexpr int DP_COL = 128;
  static constexpr int DV_COL = 256;
  static constexpr int DK_COL = 256 + DV;
  static constexpr int DQ_COL = DP_COL;  // dQ over dP^T once dP^T has been loaded
  static_assert(DQK <= 128 && DV <= 128, "column budget");
  static constexpr uint32_t ID_S = idesc_bf16_f32(128, 128, 0, 0);
  static constexpr uint32_t ID_DV = idesc_bf16_f32(128, DV, 0, 1);
  static constexpr uint32_t ID_DK = idesc_bf16_f32(128, DQK, 0, 1);
  static constexpr uint32_t ID_DQ = idesc_bf16_f32(128, DQK, 1, 1);
};

template <int DQK, int DV>
__global__ void __launch_bounds__(kThreads, 1) bwd_tc_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
    BwdArgs a) {
  using C = BCfg<DQK, DV>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  if (pad > static_cast<uint32_t>(C::SMEM - C::USED)) {  // cannot align the tiles: report
    if (threadIdx.x == 0) atomicExch(a.ctx.status, static_cast<int>(RA_ERR_CUDA));
    return;
  }
  uint8_t* sm = smem_raw + pad;
  uint8_t* sK = sm + C::K_OFF;
  uint8_t* sV = sm + C::V_OFF;
  uint8_t* sQ = sm + C::Q_OFF;
  uint8_t* sdO = sm + C::DO_OFF;
  uint8_t* sdS = sm + C::DS_OFF;
  float* vec = reinterpret_cast<float*>(sm + C::VEC_OFF);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + C::BAR_OFF);
  uint64_t* kv_full = bars + 0;
  uint64_t* kv_empty = bars + 1;
  uint64_t* q_full = bars + 2;   // [2]
  uint64_t* q_empty = bars + 4;  // [2]
  uint64_t* s_full = bars + 6;
  uint64_t* dp_full = bars + 7;
  uint64_t* p_full = bars + 8;
  uint64_t* ds_full = bars + 9;
  uint64_t* dq_full = bars + 10;
  uint64_t* dq_empty = bars + 11;
  uint64_t* acc_full = bars + 12;
  uint64_t* acc_empty = bars + 13;
  uint64_t* drain = bars + 14;
  uint64_t* s_read = bars + 15;  // both compute halves hold their S^T
  uint64_t* dk_done = bars + 16;  // dK(v) has read the dS tile
  const ItemQueue iq{reinterpret_cast<volatile int*>(bars + 17 + 2 * kItemSlots), bars + 17,
                     bars + 17 + kItemSlots};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 17 + 2 * kItemSlots + kItemSlots / 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* kv_issued = abort_flag + 1;
  volatile int* q_issued = abort_flag + 2;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 2);  // issuers A and C
    for (int s = 0; s < 2; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 2);  // issuers A and B
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(p_full, 2 * kT);
    mbar_init(ds_full, 2 * kT);
    mbar_init(dq_full, 1);
    mbar_init(dq_empty, 2 * kT);
    mbar_init(acc_full, 2);  // issuers A (dV) and B (dK)
    mbar_init(acc_empty, 2 * kT);
    mbar_init(drain, 3);
    mbar_init(s_read, 2 * kT);
    mbar_init(dk_done, 1);
    for (int i = 0; i < kItemSlots; ++i) {
      mbar_init(&iq.full[i], 1);
      mbar_init(&iq.empty[i], 3 + 2 * kT);  // the three issuers, the compute threads
    }
    *abort_flag = 0;
    *kv_issued = 0;
    *q_issued = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp < 4) regs_dec<kRegsOther>();

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      prefetch_tmap(&tm_do);
      uint32_t nkv = 0, nq = 0;
      BItem it;
      bool ok = true;
      for (int round = 0; ok && !*abort_flag; ++round) {
        const int idx = item_publish(iq, a.item_counter, a.items, round, a.ctx, abort_flag);
        if (idx < 0) {
          ok = idx == -1;
          break;
        }
        bwd_item_from_index(a, idx, it);
        QWalk w;
        w.start(a, it);
        int qt, h;
        if (!w.next(a, it, qt, h)) continue;
        if (!(ok = mbar_wait(kv_empty, (nkv & 1) ^ 1, a.ctx, abort_flag))) break;
        mbar_arrive_expect_tx(kv_full, (C::QB + C::VB) * kBox);
        for (int bx = 0; bx < C::QB; ++bx)
          tma_load_3d(sK + bx * kBox, &tm_k, kv_full, bx * 64, it.k0, it.bkv);
        for (int bx = 0; bx < C::VB; ++bx)
          tma_load_3d(sV + bx * kBox, &tm_v, kv_full, bx * 64, it.k0, it.bkv);
        *kv_issued = static_cast<int>(++nkv);
        do {
          const int st = nq & 1;
          if (!(ok = mbar_wait(&q_empty[st], ((nq >> 1) & 1) ^ 1, a.ctx, abort_flag))) break;
          const int bh = it.b * a.Hq + h;
          mbar_arrive_expect_tx(&q_full[st], (C::QB + C::VB) * kBox + 2 * kT * 4);
          for (int bx = 0; bx < C::QB; ++bx)
            tma_load_3d(sQ + (st * C::QB + bx) * kBox, &tm_q, &q_full[st], bx * 64, qt * kT, bh);
          for (int bx = 0; bx < C::VB; ++bx)
            tma_load_3d(sdO + (st * C::VB + bx) * kBox, &tm_do, &q_full[st], bx * 64, qt * kT,
                        bh);
          const long long vrow = (static_cast<long long>(bh) * a.ntq_ws + qt) * kT;
          bulk_load(vec + st * 2 * kT, a.ws_nl2 + vrow, kT * 4, &q_full[st]);
          bulk_load(vec + st * 2 * kT + kT, a.ws_d + vrow, kT * 4, &q_full[st]);
          *q_issued = static_cast<int>(++nq);
        } while (w.next(a, it, qt, h));
      }
    }
  } else if (warp <= 3) {
    // ------------------------------------------------------ MMA issuers --
    // One thread issues tcgen05.mma at a limited rate, so three warps issue
    // the visit's five products, each in an order that keeps its own
    // overwrites safe (MMAs of one thread execute in issue order):
    //   A (warp 1): dV(v), then S^T(v+1) over P^T(v), which dV(v) has read
    //   B (warp 2): dK(v)
    //   C (warp 3): dQ(v) over dP^T(v), then dP^T(v+1) once dQ(v) is read out
    // A commit only covers its own thread's MMAs: barriers that speak for
    // products of two issuers take one commit from each.
    if (lane == 0) {
      const uint32_t aK = smem_u32(sK), aV = smem_u32(sV), aQ = smem_u32(sQ);
      const uint32_t adO = smem_u32(sdO), adS = smem_u32(sdS);
      uint32_t nkv = 0, nv = 0, nacc = 0;  // nv: visits so far = query-stage counter
      BItem it;
      bool ok = true;
      for (int round = 0; ok; ++round) {
        const int idx = item_take(iq, round, a.ctx, abort_flag);
        if (idx < 0) {
          ok = idx == -1;
          break;
        }
        bwd_item_from_index(a, idx, it);
        QWalk w;
        w.start(a, it);
        int qt, h;
        if (!w.next(a, it, qt, h)) continue;
        if (warp != 2) {  // A and C read K, V
          if (!(ok = mbar_wait(kv_full, nkv & 1, a.ctx, abort_flag))) break;
          tc_fence_after();
          ++nkv;
        }
        {
          const uint32_t st = nv & 1;
          if (warp == 1) {  // S^T of the item's first visit
            if (!(ok = mbar_wait(&q_full[st], (nv >> 1) & 1, a.ctx, abort_flag))) break;
            tc_fence_after();
            mma_kk<DQK>(tmem + C::S_COL, aK, aQ + st * C::QB * kBox, C::ID_S);
            umma_commit(s_full);
          } else if (warp == 3) {  // its dP^T, over the previous dQ once read out
            if (!(ok = mbar_wait(&q_full[st], (nv >> 1) & 1, a.ctx, abort_flag))) break;
            if (!(ok = mbar_wait(dq_empty, (nv & 1) ^ 1, a.ctx, abort_flag))) break;
            tc_fence_after();
            mma_kk<DV>(tmem + C::DP_COL, aV, adO + st * C::VB * kBox, C::ID_S);
            umma_commit(dp_full);
          }
        }
        bool first = true, has = true;
        while (has) {
          int nqt, nh;
          const bool has_next = w.next(a, it, nqt, nh);
          const uint32_t st = nv & 1, st1 = (nv + 1) & 1;
          if (warp == 1) {
            if (!(ok = mbar_wait(p_full, nv & 1, a.ctx, abort_flag))) break;
            tc_fence_after();
            if (first) {  // the previous item's dK, dV have been read out
              if (!(ok = mbar_wait(acc_empty, (nacc & 1) ^ 1, a.ctx, abort_flag))) break;
              tc_fence_after();
            }
            mma_tm(tmem + C::DV_COL, tmem + C::S_COL, adO + st * C::VB * kBox, C::ID_DV, !first);
            umma_commit(&q_empty[st]);
            if (has_next) {
              if (!(ok = mbar_wait(&q_full[st1], ((nv + 1) >> 1) & 1, a.ctx, abort_flag))) break;
              tc_fence_after();
              mma_kk<DQK>(tmem + C::S_COL, aK, aQ + st1 * C::QB * kBox, C::ID_S);
              umma_commit(s_full);
            } else {
              umma_commit(acc_full);
              umma_commit(kv_empty);
            }
          } else if (warp == 2) {
            if (!(ok = mbar_wait(ds_full, nv & 1, a.ctx, abort_flag))) break;
            tc_fence_after();
            if (first) {
              if (!(ok = mbar_wait(acc_empty, (nacc & 1) ^ 1, a.ctx, abort_flag))) break;
              tc_fence_after();
            }
            mma_km(tmem + C::DK_COL, adS, aQ + st * C::QB * kBox, C::ID_DK, !first);
            umma_commit(&q_empty[st]);
            umma_commit(dk_done);
            if (!has_next) umma_commit(acc_full);
          } else {
            if (!(ok = mbar_wait(ds_full, nv & 1, a.ctx, abort_flag))) break;
            tc_fence_after();
            mma_mm(tmem + C::DQ_COL, adS, aK, C::ID_DQ);  // dP^T(v) was loaded before ds_full
            umma_commit(dq_full);
            if (has_next) {
              if (!(ok = mbar_wait(&q_full[st1], ((nv + 1) >> 1) & 1, a.ctx, abort_flag))) break;
              if (!(ok = mbar_wait(dq_empty, nv & 1, a.ctx, abort_flag))) break;
              tc_fence_after();
              mma_kk<DV>(tmem + C::DP_COL, aV, adO + st1 * C::VB * kBox, C::ID_S);
              umma_commit(dp_full);
            } else {
              umma_commit(kv_empty);
            }
          }
          ++nv;
          first = false;
          qt = nqt;
          h = nh;
          has = has_next;
        }
        if (!ok) break;
        ++nacc;
      }
      // every MMA this thread issued has finished before the allocation goes away
      umma_commit(drain);
      const unsigned long long t0 = globaltimer_ns();
      while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t0 < a.ctx.wait_ns) {
      }
    }
  } else if (warp >= 4) {
    // ------------------- compute: two warpgroups, 64 query columns each --
    regs_inc<kRegsCompute>();
    const int half = (warp >> 2) - 1;  // 0: warps 4-7, 1: warps 8-11
    const int row = threadIdx.x & 127;  // TMEM lane: key (S^T, dP^T, dK, dV), query (dQ)
    const uint32_t lb = tmem + ((static_cast<uint32_t>(warp & 3) * 32) << 16);
    const int qc = half * 64;           // first query column of this warpgroup
    const float2 sc2 = make_float2(a.scale_log2, a.scale_log2);
    uint8_t* ds_row = sdS + half * kBox + row * 128;  // atom `half`: queries qc .. qc+63
    const uint32_t sw = row & 7;
    uint32_t nv = 0, nacc = 0;
    BItem it;
    bool ok = true;
    // dQ of the latest visit, read out of tensor memory (over the dP^T
    // columns) and added into the workspace: this half's DQK / 2 columns,
    // 16-byte vector reductions, a warp covering 512 contiguous bytes
    auto drain_dq = [&](int dq_bh, int dq_qt) -> bool {
      if (!mbar_wait(dq_full, (nv - 1) & 1, a.ctx, abort_flag)) return false;
      tc_fence_after();
      float acc[DQK / 2];
#pragma unroll
      for (int c0 = 0; c0 < DQK / 2; c0 += 32)
        tmem_ld32f(lb + C::DQ_COL + half * (DQK / 2) + c0, acc + c0);
      tmem_ld_wait();
#pragma unroll
      for (int c0 = 0; c0 < DQK / 2; c0 += 32) reg_fence32(acc + c0);
      tc_fence_before();
      mbar_arrive(dq_empty);
      float* dst = a.ws_dq + bwd_dq_index(a, dq_bh, dq_qt * kT + row, half * (DQK / 2), DQK);
#pragma unroll
      for (int c = 0; c < DQK / 2; c += 4)
        atomicAdd(reinterpret_cast<float4*>(dst + (c / 4) * (kT * 4)),
                  make_float4(acc[c], acc[c + 1], acc[c + 2], acc[c + 3]));
      return true;
    };
    for (int round = 0; ok; ++round) {
      const int idx = item_take(iq, round, a.ctx, abort_flag);
      if (idx < 0) {
        ok = idx == -1;
        break;
      }
      bwd_item_from_index(a, idx, it);
      QWalk w;
      w.start(a, it);
      int qt, h;
      int pend_bh = -1, pend_qt = 0;  // visit whose dQ is still in tensor memory
      bool any = false;
      while (w.next(a, it, qt, h)) {
        const int st = nv & 1;
        if (!(ok = mbar_wait(&q_full[st], (nv >> 1) & 1, a.ctx, abort_flag))) break;
        if (!(ok = mbar_wait(s_full, nv & 1, a.ctx, abort_flag))) break;
        tc_fence_after();
        const float* nl = vec + st * 2 * kT + qc;
        const float* dd = vec + st * 2 * kT + kT + qc;
        float p[64];
        tmem_ld32f(lb + C::S_COL + qc, p);
        tmem_ld32f(lb + C::S_COL + qc + 32, p + 32);
        tmem_ld_wait();
        reg_fence32(p);
        reg_fence32(p + 32);
        // P^T (packed, columns [0,64)) overwrites the S^T columns of queries
        // 0-63: both halves must hold their S^T first (a bounded wait)
        mbar_arrive(s_read);
        if (!(ok = mbar_wait(s_read, nv & 1, a.ctx, abort_flag))) break;
        // p = 2^(s scale log2(e) - LSE log2(e)); padding rows carry -inf
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
          const float2 n2 = *reinterpret_cast<const float2*>(nl + c);
          const float2 x = __ffma2_rn(make_float2(p[c], p[c + 1]), sc2, n2);
          p[c] = fast_exp2(x.x);
          p[c + 1] = fast_exp2(x.y);
        }
        if (w.cls == kPartial || it.klen < kT) {
          // key `row` is visible to query column q iff q >= qmin
          long long qmin = 0;
          if (a.causal) qmin = row + it.k0 - w.q0 - floor_div(w.qoff - it.koff, a.stride);
          if (row >= it.klen) qmin = kT;
          qmin -= qc;
          const int qm = qmin < 0 ? 0 : (qmin > 64 ? 64 : static_cast<int>(qmin));
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (c < qm) p[c] = 0.f;
        }
#pragma unroll
        for (int c0 = 0; c0 < 64; c0 += 32) {
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 32; c += 2) pk[c >> 1] = pack_bf16x2(p[c0 + c], p[c0 + c + 1]);
          tmem_st16(lb + C::S_COL + ((qc + c0) >> 1), pk);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(p_full);
        // the previous visit's dQ, while the tensor cores run dV and the next S^T
        if (pend_bh >= 0 && !(ok = drain_dq(pend_bh, pend_qt))) break;
        if (!(ok = mbar_wait(dp_full, nv & 1, a.ctx, abort_flag))) break;
        tc_fence_after();
        // the dS tile is free once dK(v-1) has read it (dQ(v-1) came before dP^T(v))
        if (nv > 0 && !(ok = mbar_wait(dk_done, (nv - 1) & 1, a.ctx, abort_flag))) break;
        // dS^T = P^T (dP^T - D) -> bf16 rows of 64 queries, 128-byte swizzle
        {
          float dp[64];
          tmem_ld32f(lb + C::DP_COL + qc, dp);
          tmem_ld32f(lb + C::DP_COL + qc + 32, dp + 32);
          tmem_ld_wait();
          reg_fence32(dp);
          reg_fence32(dp + 32);
#pragma unroll
          for (int g = 0; g < 8; ++g) {
            uint32_t w4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c = g * 8 + e * 2;
              const float2 d2 = *reinterpret_cast<const float2*>(dd + c);
              w4[e] = pack_bf16x2(p[c] * (dp[c] - d2.x), p[c + 1] * (dp[c + 1] - d2.y));
            }
            *reinterpret_cast<uint4*>(ds_row + ((g ^ sw) << 4)) =
                make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(ds_full);
        pend_bh = it.b * a.Hq + h;
        pend_qt = qt;
        ++nv;
        any = true;
      }
      if (!ok) break;
      if (pend_bh >= 0 && !(ok = drain_dq(pend_bh, pend_qt))) break;
      // ---- dK, dV of the key tile: this half's columns ----
      if (any) {
        if (!(ok = mbar_wait(acc_full, nacc & 1, a.ctx, abort_flag))) break;
        tc_fence_after();
      }
      const bool valid = row < it.klen;
      const long long krow = static_cast<long long>(it.bkv) * a.n_k + it.k0 + row;
      store_key_grad<DV, DV / 2>(lb + C::DV_COL + half * (DV / 2), any, valid, 1.f, a.dv, krow,
                                 half * (DV / 2), a.block_mode);
      store_key_grad<DQK, DQK / 2>(lb + C::DK_COL + half * (DQK / 2), any, valid, a.scale, a.dk,
                                   krow, half * (DQK / 2), a.block_mode);
      if (any) {
        tc_fence_before();
        mbar_arrive(acc_empty);
        ++nacc;
      }
    }
  }

  // ---------------------------------------------------------- teardown --
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (*abort_flag && threadIdx.x == 0) {
    // let in-flight loads land before shared memory is released (bounded)
    const int nk = *kv_issued;
    if (nk > 0) {
      const unsigned long long t0 = globaltimer_ns();
      while (!mbar_try_wait(kv_full, (nk - 1) & 1) && globaltimer_ns() - t0 < a.ctx.wait_ns) {
      }
    }
    const int nq = *q_issued;
    for (int i = nq - 2 < 0 ? 0 : nq - 2; i < nq; ++i) {
      const unsigned long long t0 = globaltimer_ns();
      while (!mbar_try_wait(&q_full[i & 1], (i >> 1) & 1) &&
             globaltimer_ns() - t0 < a.ctx.wait_ns) {
      }
    }
  }
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

template <int DQK, int DV>
int launch_bwd_typed(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                     const CUtensorMap& tdo, const BwdArgs& args, int grid, cudaStream_t stream) {
  auto kern = bwd_tc_kernel<DQK, DV>;
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return RA_ERR_CUDA;
  if (fa.numRegs > kRegsLaunch) return RA_ERR_UNSUPPORTED;  // the register split would not fit
  constexpr int smem = BCfg<DQK, DV>::SMEM;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return RA_ERR_CUDA;
  kern<<<grid, kThreads, smem, stream>>>(tq, tk, tv, tdo, args);
  note_launch();
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

}  // namespace

size_t backward_workspace_bytes(const ra_shape& s) {
  return bwd_layout(s.B, s.Hq, s.n_q, s.d_qk).total;
}

int launch_backward(const void* q, const void* k, const void* v, const void* out,
                    const float* lse, const void* dout, const float* delta, const ra_shape& s,
                    int P, int q_offset, int k_offset, long long stride, int causal, int striped,
                    float scale, void* dq, void* dk, void* dv, bool block_mode, void* workspace,
                    const DeviceInfo& dev, cudaStream_t stream) {
  const BwdLayout L = bwd_layout(s.B, s.Hq, s.n_q, s.d_qk);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* ws_dq = reinterpret_cast<float*>(ws + L.dq_off);
  float* ws_nl2 = reinterpret_cast<float*>(ws + L.nl2_off);
  float* ws_d = reinterpret_cast<float*>(ws + L.d_off);

  int rc = launch_backward_rows(block_mode ? nullptr : out, dout, delta, lse, s, L, ws_nl2, ws_d,
                                ws_dq, reinterpret_cast<unsigned int*>(ws + L.ctr_off), dev,
                                stream);
  if (rc != RA_OK) return rc;

  BwdArgs a{};
  a.B = s.B;
  a.Hq = s.Hq;
  a.Hkv = s.Hkv;
  a.n_q = s.n_q;
  a.n_k = s.n_k;
  a.P = P;
  a.grp = s.Hq / s.Hkv;
  a.q_offset = q_offset;
  a.k_offset = k_offset;
  a.causal = causal;
  a.striped = striped;
  a.stride = striped ? P : stride;
  a.scale = scale;
  a.scale_log2 = scale * kLog2e;
  a.ntq_ws = L.ntq;
  a.ws_dq = ws_dq;
  a.ws_nl2 = ws_nl2;
  a.ws_d = ws_d;
  a.dk = dk;
  a.dv = dv;
  a.block_mode = block_mode ? 1 : 0;
  a.item_counter = reinterpret_cast<unsigned int*>(ws + L.ctr_off);
  a.ctx = dev.ctx;
  // as many (batch, KV head)s per block of items as keep the dQ accumulator
  // of their query heads within 48 MB (well inside the 126 MB L2)
  const long long dq_bytes = static_cast<long long>(s.Hq / s.Hkv) * s.n_q * s.d_qk * 4;
  const long long fit = (48ll << 20) / (dq_bytes > 0 ? dq_bytes : 1);
  const long long nbkv = static_cast<long long>(s.B) * s.Hkv;
  a.kv_block = static_cast<int>(fit < 1 ? 1 : (fit > nbkv ? nbkv : fit));

  if (s.dtype == RA_BF16) {
    a.tq = a.tk = kT;
    a.ntq = L.ntq;
    a.ntk = (s.n_k + kT - 1) / kT;
    const long long items = static_cast<long long>(s.B) * s.Hkv * a.ntk;
    if (items > 0x7fffffffLL) return RA_ERR_UNSUPPORTED;
    a.items = static_cast<int>(items);
    CUtensorMap tq, tk, tv, tdo;
    const uint64_t hq = static_cast<uint64_t>(s.B) * s.Hq;
    const uint64_t hkv = static_cast<uint64_t>(s.B) * s.Hkv;
    if (make_tmap_bf16_3d(&tq, q, s.d_qk, s.n_q, hq, s.d_qk * 2ull,
                          static_cast<uint64_t>(s.n_q) * s.d_qk * 2, 64, kT) != 0 ||
        make_tmap_bf16_3d(&tk, k, s.d_qk, s.n_k, hkv, s.d_qk * 2ull,
                          static_cast<uint64_t>(s.n_k) * s.d_qk * 2, 64, kT) != 0 ||
        make_tmap_bf16_3d(&tv, v, s.d_v, s.n_k, hkv, s.d_v * 2ull,
                          static_cast<uint64_t>(s.n_k) * s.d_v * 2, 64, kT) != 0 ||
        make_tmap_bf16_3d(&tdo, dout, s.d_v, s.n_q, hq, s.d_v * 2ull,
                          static_cast<uint64_t>(s.n_q) * s.d_v * 2, 64, kT) != 0)
      return RA_ERR_CUDA;
    const int grid = a.items < dev.num_sms ? a.items : dev.num_sms;
    if (s.d_qk == 192) rc = launch_bwd_tc192(tq, tk, tv, tdo, a, s.d_v, grid, stream);
    else if (s.d_qk == 128 && s.d_v == 128) rc = launch_bwd_typed<128, 128>(tq, tk, tv, tdo, a, grid, stream);
    else if (s.d_qk == 64 && s.d_v == 64) rc = launch_bwd_typed<64, 64>(tq, tk, tv, tdo, a, grid, stream);
    else if (s.d_qk == 64 && s.d_v == 128) rc = launch_bwd_typed<64, 128>(tq, tk, tv, tdo, a, grid, stream);
    else if (s.d_qk == 128 && s.d_v == 64) rc = launch_bwd_typed<128, 64>(tq, tk, tv, tdo, a, grid, stream);
    else return RA_ERR_UNSUPPORTED;
  } else {
    rc = launch_simt_backward(q, k, v, dout, s, a, dev, stream);
  }
  if (rc != RA_OK) return rc;

  return launch_dq_finalize(ws_dq, dq, s, L, scale, block_mode, stream);
}

}  // namespace ra
