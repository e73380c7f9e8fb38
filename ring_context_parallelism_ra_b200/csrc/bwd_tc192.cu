// Backward pass of exact attention on the tensor cores for the MLA-shaped
// head: bf16, d_qk = 192, d_v in {64, 128}.  It computes the products stated
// in bwd.cuh (the chain rule of page "长上下文的第一性挑战", Eq.
// (lc-ch-attention); the D_qk + D_v head of page "上下文并行 (CP) 收益评估实验
// 设计", Eq. (cpeval-comp)) with the same work items and ring-order walk as
// the d_qk <= 128 kernel in bwd_attention.cu; what differs is how the
// products share tensor memory.
//
// Tensor memory (512 columns) at d_qk = 192: the dK accumulator alone takes
// 192 columns and dV another d_v, so S^T and dP^T cannot both stay resident
// as in the smaller head.  Per visit (query tile t of head h against the
// item's 128 keys) the columns are reused in sequence:
//   [0, 128)    S^T = K Q_t^T, then dP^T = V dO_t^T once both compute
//               warpgroups have loaded S^T, then (with the next range) dQ
//   [128, 192)  P^T as packed bf16, read by dV; then dQ columns 128-191
//   [0, 192)    dQ_t = dS K (queries on the lanes), once dP^T is loaded and
//               dV has read P^T
//   [192, 192 + d_v)              dV accumulator of the item
//   [192 + d_v, 192 + d_v + 192)  dK accumulator of the item
// so the next S^T waits until dQ columns 0-127 have been read out (columns
// 128-191 are read at the next visit, before P^T is written over them, and
// their reductions overlap that visit's dP^T and dV): the products of a visit
// run one after another, S^T -> (P) -> dP^T, dV -> (dS) -> dQ, dK -> (dQ
// read-out), with the exponentials, dS and the dQ reductions on the CUDA
// cores in between.
//
// Shared memory: K (3 atoms) and V of the item, Q in two stages (its last
// reader, dK, comes late in a visit), and one buffer that holds dO of a visit
// until dP^T and dV have read it and then its dS tile (dK reads it K-major as
// dS^T, dQ MN-major as dS), plus the row vectors.
//
// CTA layout (384 threads, one CTA per SM, persistent):
//   warp 0      TMA producer (K, V per item; Q, vectors, dO per visit)
//   warp 1      tcgen05.mma issuer; owns the tensor-memory allocation
//   warps 2-3   idle
//   warps 4-11  two compute warpgroups, query columns 0-63 and 64-127 of
//               S^T / dP^T (thread r = key r), dQ dims 0-63 + 128-159 and
//               64-127 + 160-191 (thread r = query r), dK / dV columns split
//               in halves at the end
// Registers: 2 x 184 (compute) + 136 (warps 0-3) = 504 = 3 x 168 per lane.
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

constexpr int kT = kBwdT;
constexpr int kBox = kBwdBox;
constexpr int kDQK = 192;
constexpr int kThreads = 384;
constexpr int kRegsLaunch = 168;
constexpr int kRegsCompute = 184;
constexpr int kRegsOther = 136;
static_assert(2 * kRegsCompute + kRegsOther <= 3 * kRegsLaunch,
              "register split must fit the launch allocation");
static_assert(kRegsCompute >= kRegsLaunch, "compute warpgroups grow (setmaxnreg.inc)");
static_assert(kRegsOther <= kRegsLaunch, "producer / MMA warpgroup shrinks (setmaxnreg.dec)");
constexpr int kSmemLimit = 232448;

template <int DV>
struct Cfg192 {
  static constexpr int QB = kDQK / 64;
  static constexpr int VB = DV / 64;
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = K_OFF + QB * kBox;
  static constexpr int Q_OFF = V_OFF + VB * kBox;       // two stages
  static constexpr int X_OFF = Q_OFF + 2 * QB * kBox;   // dO of a visit, then its dS
  static constexpr int X_BYTES = 2 * kBox;              // dS: 128 keys x 128 queries >= dO
  static constexpr int VEC_OFF = X_OFF + X_BYTES;       // [stage][-LSE log2e | D][128]
  static constexpr int BAR_OFF = VEC_OFF + 2 * 2 * kT * 4;
  static constexpr int USED = BAR_OFF + 256;
  static_assert(USED <= kSmemLimit, "shared memory budget");
  static constexpr int SMEM = USED + 1024 <= kSmemLimit ? USED + 1024 : kSmemLimit;
  static constexpr int SC = 0;          // S^T, then dP^T
  static constexpr int PT = 128;        // P^T, packed bf16
  static constexpr int DQ = 0;          // dQ over [0, 192)
  static constexpr int DVC = 192;
  static constexpr int DKC = 192 + DV;
  static_assert(DKC + kDQK <= 512, "tensor-memory budget");
  static constexpr uint32_t ID_S = idesc_bf16_f32(128, 128, 0, 0);
  static constexpr uint32_t ID_DV = idesc_bf16_f32(128, DV, 0, 1);
  static constexpr uint32_t ID_DK = idesc_bf16_f32(128, kDQK, 0, 1);
  static constexpr uint32_t ID_DQ = idesc_bf16_f32(128, kDQK, 1, 1);
};

template <int DV>
__global__ void __launch_bounds__(kThreads, 1) bwd_tc192_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
    BwdArgs a) {
  using C = Cfg192<DV>;
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
  uint8_t* sX = sm + C::X_OFF;
  float* vec = reinterpret_cast<float*>(sm + C::VEC_OFF);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + C::BAR_OFF);
  uint64_t* kv_full = bars + 0;
  uint64_t* kv_empty = bars + 1;
  uint64_t* q_full = bars + 2;    // [2] Q and row vectors of a visit
  uint64_t* q_empty = bars + 4;   // [2]
  uint64_t* do_full = bars + 6;   // dO of a visit landed in the X buffer
  uint64_t* x_empty = bars + 7;   // dK and dQ have read the visit's dS
  uint64_t* s_full = bars + 8;
  uint64_t* p_full = bars + 9;    // both halves loaded S^T and stored P^T
  uint64_t* dp_full = bars + 10;  // dP^T and dV done
  uint64_t* ds_full = bars + 11;  // both halves loaded dP^T and wrote dS
  uint64_t* dq_full = bars + 12;
  uint64_t* dq_empty = bars + 13;
  uint64_t* acc_full = bars + 14;
  uint64_t* acc_empty = bars + 15;
  uint64_t* drain = bars + 16;
  const ItemQueue iq{reinterpret_cast<volatile int*>(bars + 17 + 2 * kItemSlots), bars + 17,
                     bars + 17 + kItemSlots};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 17 + 2 * kItemSlots + kItemSlots / 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* kv_issued = abort_flag + 1;
  volatile int* q_issued = abort_flag + 2;
  volatile int* do_issued = abort_flag + 3;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
    }
    mbar_init(do_full, 1);
    mbar_init(x_empty, 1);
    mbar_init(s_full, 1);
    mbar_init(p_full, 2 * kT);
    mbar_init(dp_full, 1);
    mbar_init(ds_full, 2 * kT);
    mbar_init(dq_full, 1);
    mbar_init(dq_empty, 2 * kT);
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 2 * kT);
    mbar_init(drain, 1);
    for (int i = 0; i < kItemSlots; ++i) {
      mbar_init(&iq.full[i], 1);
      mbar_init(&iq.empty[i], 1 + 2 * kT);  // the issuer, the compute threads
    }
    *abort_flag = 0;
    *kv_issued = 0;
    *q_issued = 0;
    *do_issued = 0;
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
          const int bh = it.b * a.Hq + h;
          // Q and the row vectors of this visit (stage st: free once dK of
          // the visit two back has read it)
          if (!(ok = mbar_wait(&q_empty[st], ((nq >> 1) & 1) ^ 1, a.ctx, abort_flag))) break;
          mbar_arrive_expect_tx(&q_full[st], C::QB * kBox + 2 * kT * 4);
          for (int bx = 0; bx < C::QB; ++bx)
            tma_load_3d(sQ + (st * C::QB + bx) * kBox, &tm_q, &q_full[st], bx * 64, qt * kT, bh);
          const long long vrow = (static_cast<long long>(bh) * a.ntq_ws + qt) * kT;
          bulk_load(vec + st * 2 * kT, a.ws_nl2 + vrow, kT * 4, &q_full[st]);
          bulk_load(vec + st * 2 * kT + kT, a.ws_d + vrow, kT * 4, &q_full[st]);
          *q_issued = static_cast<int>(nq + 1);
          // dO of this visit into the X buffer, once the previous visit's
          // dS there has been read by its dK and dQ
          if (!(ok = mbar_wait(x_empty, (nq & 1) ^ 1, a.ctx, abort_flag))) break;
          mbar_arrive_expect_tx(do_full, C::VB * kBox);
          for (int bx = 0; bx < C::VB; ++bx)
            tma_load_3d(sX + bx * kBox, &tm_do, do_full, bx * 64, qt * kT, bh);
          *do_issued = static_cast<int>(++nq);
        } while (w.next(a, it, qt, h));
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      const uint32_t aK = smem_u32(sK), aV = smem_u32(sV), aQ = smem_u32(sQ);
      const uint32_t aX = smem_u32(sX);
      uint32_t nkv = 0, nv = 0, nacc = 0;
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
        if (!(ok = mbar_wait(kv_full, nkv & 1, a.ctx, abort_flag))) break;
        tc_fence_after();
        ++nkv;
        bool first = true, has = true;
        while (has) {
          const uint32_t st = nv & 1;
          const uint32_t aQs = aQ + st * C::QB * kBox;
          // S^T over the columns the previous visit's dQ occupied
          if (!(ok = mbar_wait(&q_full[st], (nv >> 1) & 1, a.ctx, abort_flag))) break;
          if (!(ok = mbar_wait(dq_empty, (nv & 1) ^ 1, a.ctx, abort_flag))) break;
          tc_fence_after();
          mma_kk<kDQK>(tmem + C::SC, aK, aQs, C::ID_S);
          umma_commit(s_full);
          // dP^T over S^T (loaded by both halves), dV from P^T and dO
          if (!(ok = mbar_wait(do_full, nv & 1, a.ctx, abort_flag))) break;
          if (!(ok = mbar_wait(p_full, nv & 1, a.ctx, abort_flag))) break;
          if (first && !(ok = mbar_wait(acc_empty, (nacc & 1) ^ 1, a.ctx, abort_flag))) break;
          tc_fence_after();
          mma_kk<DV>(tmem + C::SC, aV, aX, C::ID_S);
          mma_tm(tmem + C::DVC, tmem + C::PT, aX, C::ID_DV, !first);
          umma_commit(dp_full);
          // dQ over dP^T and P^T (both read), then dK; dS in the X buffer
          if (!(ok = mbar_wait(ds_full, nv & 1, a.ctx, abort_flag))) break;
          tc_fence_after();
          mma_mm(tmem + C::DQ, aX, aK, C::ID_DQ);
          umma_commit(dq_full);
          mma_km(tmem + C::DKC, aX, aQs, C::ID_DK, !first);
          umma_commit(&q_empty[st]);
          umma_commit(x_empty);
          has = w.next(a, it, qt, h);
          if (!has) {
            umma_commit(acc_full);
            umma_commit(kv_empty);
          }
          ++nv;
          first = false;
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
    // ------------------------------------------- compute: two warpgroups --
    regs_inc<kRegsCompute>();
    const int half = (warp >> 2) - 1;   // 0: warps 4-7, 1: warps 8-11
    const int row = threadIdx.x & 127;  // TMEM lane: key (S^T, dP^T, dK, dV), query (dQ)
    const uint32_t lb = tmem + ((static_cast<uint32_t>(warp & 3) * 32) << 16);
    const int qc = half * 64;           // first query column of this warpgroup
    const int dc = half * (kDQK / 2);   // first dK column of this warpgroup
    // dQ columns of this warpgroup: [64 half, +64) inside [0, 128), read as
    // soon as dQ is complete (the next S^T overwrites them), and [128 + 32
    // half, +32) inside the P^T columns, read only at the next visit, just
    // before this warpgroup writes its P^T there; their reductions then run
    // while the tensor cores compute dP^T (off the visit's critical path)
    const int dqa = half * 64;
    const int dqb = 128 + half * 32;
    const float2 sc2 = make_float2(a.scale_log2, a.scale_log2);
    uint8_t* ds_row = sX + half * kBox + row * 128;  // atom `half`: queries qc .. qc+63
    const uint32_t sw = row & 7;
    uint32_t nv = 0, nacc = 0;
    int tail_bh = -1, tail_qt = 0;  // visit whose dQ columns [dqb, dqb + 32) wait in TMEM
    auto tail_dst = [&]() -> float* {
      return a.ws_dq + bwd_dq_index(a, tail_bh, tail_qt * kT + row, dqb, kDQK);
    };
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
      bool any = false;
      while (w.next(a, it, qt, h)) {
        const int st = nv & 1;
        if (!(ok = mbar_wait(&q_full[st], (nv >> 1) & 1, a.ctx, abort_flag))) break;
        if (!(ok = mbar_wait(s_full, nv & 1, a.ctx, abort_flag))) break;
        tc_fence_after();
        const float* nl = vec + st * 2 * kT + qc;
        const float* dd = vec + st * 2 * kT + kT + qc;
        // P^T = 2^(S^T scale log2(e) - LSE log2(e)); padding rows carry -inf
        float p[64];
        tmem_ld32f(lb + C::SC + qc, p);
        tmem_ld32f(lb + C::SC + qc + 32, p + 32);
        tmem_ld_wait();
        reg_fence32(p);
        reg_fence32(p + 32);
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
        // the previous visit's remaining dQ columns leave tensor memory
        // before this warpgroup's P^T is written over them, and are added
        // into the workspace while dP^T and dV run
        uint32_t tail[32];
        if (tail_bh >= 0) {
          tmem_ld32(lb + C::DQ + dqb, tail);
          tmem_ld_wait();
        }
#pragma unroll
        for (int c0 = 0; c0 < 64; c0 += 32) {
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 32; c += 2) pk[c >> 1] = pack_bf16x2(p[c0 + c], p[c0 + c + 1]);
          tmem_st16(lb + C::PT + ((qc + c0) >> 1), pk);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(p_full);
        if (tail_bh >= 0) {
          float* dst = tail_dst();
#pragma unroll
          for (int c = 0; c < 32; c += 4)
            atomicAdd(reinterpret_cast<float4*>(dst + (c / 4) * (kT * 4)),
                      make_float4(__uint_as_float(tail[c]), __uint_as_float(tail[c + 1]),
                                  __uint_as_float(tail[c + 2]), __uint_as_float(tail[c + 3])));
          tail_bh = -1;
        }
        // dS^T = P^T (dP^T - D) -> bf16 rows of 64 queries, 128-byte swizzle,
        // into the X buffer (dO there has been read: dp_full follows dV)
        if (!(ok = mbar_wait(dp_full, nv & 1, a.ctx, abort_flag))) break;
        tc_fence_after();
        {
          float dp[64];
          tmem_ld32f(lb + C::SC + qc, dp);
          tmem_ld32f(lb + C::SC + qc + 32, dp + 32);
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
        // dQ of the visit (query `row`): the 64 columns the next S^T will
        // overwrite now, added into the workspace with 16-byte reductions (a
        // warp: 512 contiguous bytes); the other 32 at the next visit
        if (!(ok = mbar_wait(dq_full, nv & 1, a.ctx, abort_flag))) break;
        tc_fence_after();
        {
          float acc[64];
          tmem_ld32f(lb + C::DQ + dqa, acc);
          tmem_ld32f(lb + C::DQ + dqa + 32, acc + 32);
          tmem_ld_wait();
          reg_fence32(acc);
          reg_fence32(acc + 32);
          tc_fence_before();
          mbar_arrive(dq_empty);
          float* dst = a.ws_dq + bwd_dq_index(a, it.b * a.Hq + h, qt * kT + row, dqa, kDQK);
#pragma unroll
          for (int c = 0; c < 64; c += 4)
            atomicAdd(reinterpret_cast<float4*>(dst + (c / 4) * (kT * 4)),
                      make_float4(acc[c], acc[c + 1], acc[c + 2], acc[c + 3]));
        }
        tail_bh = it.b * a.Hq + h;
        tail_qt = qt;
        ++nv;
        any = true;
      }
      if (!ok) break;
      // ---- dK, dV of the key tile: this half's columns ----
      if (any) {
        if (!(ok = mbar_wait(acc_full, nacc & 1, a.ctx, abort_flag))) break;
        tc_fence_after();
      }
      const bool valid = row < it.klen;
      const long long krow = static_cast<long long>(it.bkv) * a.n_k + it.k0 + row;
      store_key_grad<DV, DV / 2>(lb + C::DVC + half * (DV / 2), any, valid, 1.f, a.dv, krow,
                                 half * (DV / 2), a.block_mode);
      store_key_grad<kDQK, kDQK / 2>(lb + C::DKC + dc, any, valid, a.scale, a.dk, krow, dc,
                                     a.block_mode);
      if (any) {
        tc_fence_before();
        mbar_arrive(acc_empty);
        ++nacc;
      }
    }
    // the last visit's remaining dQ columns (its dq_full was waited above)
    if (ok && tail_bh >= 0) {
      float tail[32];
      tc_fence_after();
      tmem_ld32f(lb + C::DQ + dqb, tail);
      tmem_ld_wait();
      reg_fence32(tail);
      float* dst = tail_dst();
#pragma unroll
      for (int c = 0; c < 32; c += 4)
        atomicAdd(reinterpret_cast<float4*>(dst + (c / 4) * (kT * 4)),
                  make_float4(tail[c], tail[c + 1], tail[c + 2], tail[c + 3]));
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
    const int nd = *do_issued;
    if (nd > 0) {
      const unsigned long long t0 = globaltimer_ns();
      while (!mbar_try_wait(do_full, (nd - 1) & 1) && globaltimer_ns() - t0 < a.ctx.wait_ns) {
      }
    }
  }
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

template <int DV>
int launch_typed(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                 const CUtensorMap& tdo, const BwdArgs& args, int grid, cudaStream_t stream) {
  auto kern = bwd_tc192_kernel<DV>;
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return RA_ERR_CUDA;
  if (fa.numRegs > kRegsLaunch) return RA_ERR_UNSUPPORTED;  // the register split would not fit
  constexpr int smem = Cfg192<DV>::SMEM;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return RA_ERR_CUDA;
  kern<<<grid, kThreads, smem, stream>>>(tq, tk, tv, tdo, args);
  note_launch();
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

}  // namespace

int launch_bwd_tc192(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                     const CUtensorMap& tdo, const BwdArgs& args, int d_v, int grid,
                     cudaStream_t stream) {
  if (d_v == 128) return launch_typed<128>(tq, tk, tv, tdo, args, grid, stream);
  if (d_v == 64) return launch_typed<64>(tq, tk, tv, tdo, args, grid, stream);
  return RA_ERR_UNSUPPORTED;
}

}  // namespace ra
