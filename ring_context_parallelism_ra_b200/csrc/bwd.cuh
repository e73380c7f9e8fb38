// Shared pieces of the backward kernels: arguments, workspace layout, and the
// walk over (key tile, query tile, head) that every role of a kernel repeats.
//
// Gradients of O = softmax(scale * Q K^T + mask) V (page "长上下文的第一性挑战",
// Eq. (lc-ch-attention)) by the chain rule, for a loss that depends on O
// through dO:
//   P = exp(scale * Q K^T - LSE)   (the forward's final LSE, masked pairs 0)
//   dV = P^T dO,  dP = dO V^T,  D = rowsum(dO * O),  dS = P * (dP - D),
//   dQ = scale * dS K,  dK = scale * dS^T Q.
// The ring of page "AI 推理系列（十一）：Ring Attention 如何让多张 GPU 共同计算
// 一条超长序列" ("KV 在 Ring 中如何流动") carries KV_j past every query
// partition; in the backward pass KV_j's gradient accumulators dK_j, dV_j
// travel with it and collect one share per query partition, in ring order
// i = j, j+1, ... (mod P), while dQ_i collects at its partition.  On one GPU a
// work item is one key tile of one (batch, KV head): dK / dV stay on chip for
// the whole walk over the query tiles (ring order, every query head of the
// group), and dQ shares are added into an fp32 workspace.
#pragma once

#include <stdint.h>

#include "block_class.cuh"
#include "common.cuh"

namespace ra {

constexpr int kBwdTile = 128;  // rows of a dQ workspace tile

// Device workspace of a backward call (all fp32):
//   dq   [B*Hq][ntq][d_qk/4][128][4]  dQ accumulator: in each 128-row tile,
//                                 groups of four columns, row by row
//   nl2  [B*Hq][ntq*128]          -LSE * log2(e) (-inf for a row with no key
//                                 and for padding rows)
//   D    [B*Hq][ntq*128]          rowsum(dO * O) (0 for padding rows)
//   ctr  one 32-bit counter: work items handed out so far (zeroed with dQ)
struct BwdLayout {
  int ntq;
  long long rows_pad;
  size_t dq_off, nl2_off, d_off, ctr_off, total;
};

inline size_t bwd_align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

inline BwdLayout bwd_layout(int B, int Hq, int n_q, int d_qk) {
  BwdLayout L;
  L.ntq = (n_q + kBwdTile - 1) / kBwdTile;
  L.rows_pad = static_cast<long long>(B) * Hq * L.ntq * kBwdTile;
  L.dq_off = 0;
  L.nl2_off = bwd_align256(L.dq_off + static_cast<size_t>(L.rows_pad) * d_qk * 4);
  L.d_off = bwd_align256(L.nl2_off + static_cast<size_t>(L.rows_pad) * 4);
  L.ctr_off = bwd_align256(L.d_off + static_cast<size_t>(L.rows_pad) * 4);
  L.total = L.ctr_off + 256;
  return L;
}

struct BwdArgs {
  int B, Hq, Hkv, n_q, n_k, P, grp;
  int q_offset, k_offset, causal;
  int striped;       // fused ring over a striped split (positions r * P + i)
  long long stride;  // position stride inside a partition / block
  float scale, scale_log2;
  int tq, tk;        // query rows per tile, keys per tile
  int ntq, ntk;      // tiles per head (query tiles counted in tq rows)
  int ntq_ws;        // 128-row workspace tiles per head
  int items;         // B * Hkv * ntk
  int kv_block;      // (batch, KV head)s per block of items (see bwd_item_at)
  float* ws_dq;
  const float* ws_nl2;
  const float* ws_d;
  void* dk;          // ring: [B, Hkv, n_k, d_qk] of the input dtype; block: fp32, +=
  void* dv;
  int block_mode;
  unsigned int* item_counter;  // items handed out so far (tensor-core kernels)
  DevCtx ctx;
};

// Position offset of partition p: contiguous tokens use the call's offset; in
// the striped split (stride P) row R of partition p is token (R - p L) P + p.
__device__ __forceinline__ long long bwd_part_offset(const BwdArgs& a, int p, int n, int base) {
  return a.striped ? static_cast<long long>(p) * (1 - static_cast<long long>(n / a.P) * a.P)
                   : static_cast<long long>(base);
}

struct BItem {
  int bkv, b, g, k0, klen, j;
  long long koff;  // key position = koff + key index * stride
};

// Item `idx` in the order work is handed out, heaviest first for a causal
// mask: low key positions are visible to the most queries.  Items come in
// blocks of kv_block (batch, KV head)s whose dQ accumulator fits in L2 (all
// of a block's items before the next block's), so that the CTAs running at
// the same time walk the same query tiles and add their dQ shares into the
// same lines of L2 instead of spreading the reductions over a workspace far
// larger than L2.
__device__ __forceinline__ void bwd_item_from_index(const BwdArgs& a, long long idx, BItem& it) {
  const int nbkv = a.B * a.Hkv;
  const int blk = static_cast<int>(idx / (static_cast<long long>(a.ntk) * a.kv_block));
  const int kv0 = blk * a.kv_block;
  const int hb = nbkv - kv0 < a.kv_block ? nbkv - kv0 : a.kv_block;
  const long long in_blk = idx - static_cast<long long>(kv0) * a.ntk;
  const int r = static_cast<int>(in_blk / hb);
  it.bkv = kv0 + static_cast<int>(in_blk % hb);
  int kt = r;
  if (a.striped) {  // same local tile of every partition together
    const int tpp = a.ntk / a.P;
    kt = (r % a.P) * tpp + r / a.P;
  }
  it.b = it.bkv / a.Hkv;
  it.g = it.bkv % a.Hkv;
  it.k0 = kt * a.tk;
  const int rem = a.n_k - it.k0;
  it.klen = rem < a.tk ? rem : a.tk;
  const int Lk = a.n_k / a.P;
  const int j = it.k0 / Lk;
  it.j = j < a.P - 1 ? j : a.P - 1;
  it.koff = bwd_part_offset(a, it.j, a.n_k, a.k_offset);
}

// Static dealing (one item per CTA and round, snake order over the CTAs),
// for the kernels launched with one CTA per item.
__device__ __forceinline__ bool bwd_item_at(const BwdArgs& a, int round, BItem& it) {
  const int nc = gridDim.x;
  const int c = blockIdx.x;
  const long long idx = static_cast<long long>(round) * nc + ((round & 1) ? (nc - 1 - c) : c);
  if (idx >= a.items) return false;
  bwd_item_from_index(a, idx, it);
  return true;
}

// The (query tile, head) visits of one item: query tiles in ring order from
// the key tile's own partition, fully masked tiles skipped, every query head
// of the KV group per tile.
struct QWalk {
  int m, hi, qt0, qt;
  int8_t cls;
  int q0, qlen;
  long long qoff;
  __device__ __forceinline__ void start(const BwdArgs& a, const BItem& it) {
    const int Lq = a.n_q / a.P;
    m = 0;
    hi = a.grp;
    cls = kSkip;
    qt0 = static_cast<int>((static_cast<long long>(it.j) * Lq) / a.tq);
  }
  __device__ __forceinline__ bool next(const BwdArgs& a, const BItem& it, int& qt_out,
                                       int& h_out) {
    while (hi >= a.grp || cls == kSkip) {
      if (m >= a.ntq) return false;
      qt = qt0 + m;
      if (qt >= a.ntq) qt -= a.ntq;
      ++m;
      q0 = qt * a.tq;
      const int rem = a.n_q - q0;
      qlen = rem < a.tq ? rem : a.tq;
      const int Lq = a.n_q / a.P;
      int i = q0 / Lq;
      i = i < a.P - 1 ? i : a.P - 1;
      qoff = bwd_part_offset(a, i, a.n_q, a.q_offset);
      cls = tile_class(q0, qlen, it.k0, it.klen, qoff, it.koff, a.causal, a.stride);
      hi = 0;
    }
    qt_out = qt;
    h_out = it.g * a.grp + hi;
    ++hi;
    return true;
  }
};

// Index of dQ element (row t, column c) of head bh in the workspace.  A
// 128-row tile is stored as [c / 4][row][c % 4]: four consecutive columns of
// a row are one 16-byte vector and 32 consecutive rows 512 contiguous bytes.
__device__ __forceinline__ long long bwd_dq_index(const BwdArgs& a, int bh, int t, int c, int dqk) {
  return (((static_cast<long long>(bh) * a.ntq_ws + t / kBwdTile) * (dqk / 4) + c / 4) *
              kBwdTile + (t % kBwdTile)) * 4 + (c % 4);
}

}  // namespace ra
