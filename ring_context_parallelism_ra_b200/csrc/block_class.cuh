// Causal classification of a (query tile, key tile) pair.  One integer rule,
// compiled for host and device, so the host map, the device map and the
// kernels' tile loop agree bit for bit.
//
// Visibility: key at absolute position k_pos is visible to the query at q_pos
// iff k_pos <= q_pos (no query reads a future token; page "AI 推理系列（十一）：
// Ring Attention 如何让多张 GPU 共同计算一条超长序列", section "KV 在 Ring 中如何
// 流动").  Over a tile the visible pairs form a staircase, so only the corner
// pairs decide the class:
//   SKIP    the first key lies after the last query,
//   FULL    the last key lies at or before the first query,
//   PARTIAL otherwise.
#pragma once

#include <stdint.h>

#ifdef __CUDACC__
#define RA_HD __host__ __device__ __forceinline__
#else
#define RA_HD inline
#endif

namespace ra {

enum : int8_t { kSkip = 0, kPartial = 1, kFull = 2 };

// Floor division (rounds toward -inf, also for a negative numerator).
RA_HD long long floor_div(long long a, long long b) {
  const long long q = a / b;
  return (q * b != a && ((a < 0) != (b < 0))) ? q - 1 : q;
}

// q0, q_len: first row and row count of the tile (rows beyond n_q excluded
// by the caller); k0, k_len likewise for keys.  Row t of the tensor sits at
// absolute position q_offset + t * stride, key u at k_offset + u * stride
// (stride 1: contiguous tokens; stride P: a partition of a striped split,
// where token p of the sequence goes to partition p mod P).  Positions grow
// with the index, so the corner pairs still decide the class.
RA_HD int8_t tile_class(long long q0, long long q_len, long long k0, long long k_len,
                        long long q_offset, long long k_offset, int causal,
                        long long stride = 1) {
  if (!causal) return kFull;
  const long long first_q = q_offset + q0 * stride;
  const long long last_q = first_q + (q_len - 1) * stride;
  const long long first_k = k_offset + k0 * stride;
  const long long last_k = first_k + (k_len - 1) * stride;
  if (first_k > last_q) return kSkip;
  if (last_k <= first_q) return kFull;
  return kPartial;
}

// Number of leading keys of a tile (key indices k0, k0 + 1, ...) visible to
// query row t: key u is visible iff k_offset + u * stride <= q_offset + t *
// stride, i.e. u - t <= floor((q_offset - k_offset) / stride).  Not clipped.
RA_HD long long visible_keys(long long t, long long k0, long long q_offset, long long k_offset,
                             long long stride) {
  return floor_div(q_offset - k_offset, stride) + t - k0 + 1;
}

}  // namespace ra
