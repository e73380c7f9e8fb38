// Tensor-core pieces shared by the backward kernels (bwd_attention.cu for
// d_qk, d_v in {64, 128}; bwd_tc192.cu for d_qk = 192): the bulk copy of row
// vectors, the tcgen05.mma sequences of the five products and the read-out
// of the dK / dV accumulators.  Operand tiles are 128 rows of 64 bf16 per
// 16 KB atom, 128-byte swizzled, as the TMA writes them.
#pragma once

#include <stdint.h>

#include "common.cuh"
#include "item_queue.cuh"
#include "ptx.cuh"

namespace ra {

constexpr int kBwdBox = 128 * 64 * 2;  // one operand atom: 128 rows x 64 bf16
constexpr int kBwdT = 128;             // keys / queries per tile

// Bulk (non-tensor) copy global -> shared, completion as transaction bytes on
// `bar`.  Both addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(smem_dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (the tensor cores read dS from shared memory).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Descriptors of successive K steps differ only in the start address field.
// K-major operand: a K step of 16 bf16 is 32 bytes inside a 64-wide atom,
// atoms (128 rows each) are kBwdBox apart.  MN-major operand: a K step is 16
// rows of 128 bytes = 2048 bytes.
__device__ __forceinline__ uint32_t kmaj_step(int ks) {
  return static_cast<uint32_t>(((ks >> 2) * kBwdBox + (ks & 3) * 32) >> 4);
}
__device__ __forceinline__ uint32_t mnmaj_step(int ks) {
  return static_cast<uint32_t>((ks * 2048) >> 4);
}

// D[128 x 128] = A B^T, A and B K-major with KD columns (S^T, dP^T).
template <int KD>
__device__ __forceinline__ void mma_kk(uint32_t d, uint32_t a, uint32_t b, uint32_t idesc) {
  const uint64_t da = sdesc_k_sw128(a), db = sdesc_k_sw128(b);
#pragma unroll
  for (int ks = 0; ks < KD / 16; ++ks)
    umma_ss(d, da + kmaj_step(ks), db + kmaj_step(ks), idesc, ks > 0 ? 1u : 0u);
}

// dV (+)= P^T dO: A from tensor memory (128 queries = 64 packed columns).
__device__ __forceinline__ void mma_tm(uint32_t d, uint32_t a_tmem, uint32_t b, uint32_t idesc,
                                       bool acc) {
  const uint64_t db = sdesc_mn_sw128(b, kBwdBox);
#pragma unroll
  for (int ks = 0; ks < kBwdT / 16; ++ks)
    umma_ts(d, a_tmem + ks * 8, db + mnmaj_step(ks), idesc, (acc || ks > 0) ? 1u : 0u);
}

// dK (+)= dS^T Q: A K-major (keys x queries), B MN-major (queries x DQK).
__device__ __forceinline__ void mma_km(uint32_t d, uint32_t a, uint32_t b, uint32_t idesc,
                                       bool acc) {
  const uint64_t da = sdesc_k_sw128(a), db = sdesc_mn_sw128(b, kBwdBox);
#pragma unroll
  for (int ks = 0; ks < kBwdT / 16; ++ks)
    umma_ss(d, da + kmaj_step(ks), db + mnmaj_step(ks), idesc, (acc || ks > 0) ? 1u : 0u);
}

// dQ = dS K: A MN-major (queries along M, keys along K), B MN-major (keys x DQK).
__device__ __forceinline__ void mma_mm(uint32_t d, uint32_t a, uint32_t b, uint32_t idesc) {
  const uint64_t da = sdesc_mn_sw128(a, kBwdBox), db = sdesc_mn_sw128(b, kBwdBox);
#pragma unroll
  for (int ks = 0; ks < kBwdT / 16; ++ks)
    umma_ss(d, da + mnmaj_step(ks), db + mnmaj_step(ks), idesc, ks > 0 ? 1u : 0u);
}

// W columns (from col0) of dK or dV of the item's keys out of tensor memory:
// `mul` times the accumulator, stored (ring: bf16) or added (block: fp32) into
// rows of width D.  Warp-collective.
template <int D, int W>
__device__ __forceinline__ void store_key_grad(uint32_t taddr, bool any, bool valid, float mul,
                                               void* dst, long long krow, int col0,
                                               int block_mode) {
#pragma unroll
  for (int c0 = 0; c0 < W; c0 += 32) {
    float o[32];
    if (any) {
      tmem_ld32f(taddr + c0, o);
      tmem_ld_wait();
      reg_fence32(o);
    } else {
#pragma unroll
      for (int c = 0; c < 32; ++c) o[c] = 0.f;
    }
    if (valid && block_mode) {
      float4* d4 = reinterpret_cast<float4*>(static_cast<float*>(dst) + krow * D + col0 + c0);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        float4 x = d4[c];
        x.x += o[4 * c] * mul;
        x.y += o[4 * c + 1] * mul;
        x.z += o[4 * c + 2] * mul;
        x.w += o[4 * c + 3] * mul;
        d4[c] = x;
      }
    } else if (valid) {
      uint4* d4 =
          reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(dst) + krow * D + col0 + c0);
#pragma unroll
      for (int c = 0; c < 4; ++c)
        d4[c] = make_uint4(pack_bf16x2(o[8 * c] * mul, o[8 * c + 1] * mul),
                           pack_bf16x2(o[8 * c + 2] * mul, o[8 * c + 3] * mul),
                           pack_bf16x2(o[8 * c + 4] * mul, o[8 * c + 5] * mul),
                           pack_bf16x2(o[8 * c + 6] * mul, o[8 * c + 7] * mul));
    }
  }
}


}  // namespace ra
