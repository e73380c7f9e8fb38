// N-way LSE merge of normalised partials (O_p, L_p) over disjoint key sets.
//
//   L* = max_p L_p,  w_p = exp(L_p - L*),  LSE = L* + ln sum_p w_p,
//   O  = sum_p (w_p / sum_q w_q) O_p
//
// This is the closed form of the beta / gamma fold of page "LLM长文本推理Ring
// Attention环形注意力机制实现与优化", section "Ring Attention实现代码与通信重叠",
// applied to P partials at once; partials with L_p = -inf carry no weight.
//
// HBM-bound: each output row reads P * (d_v + 1) floats once.  A row of d_v
// floats is read as d_v / 4 float4 by d_v / 4 lanes (a warp covers one row at
// d_v = 128, two at 64), with streaming loads since nothing is re-read.
#include "common.cuh"
#include "launch.h"

namespace ra {

template <typename OutT>
__device__ __forceinline__ void store4(OutT* dst, float4 v);

template <>
__device__ __forceinline__ void store4<float>(float* dst, float4 v) {
  *reinterpret_cast<float4*>(dst) = v;
}

template <>
__device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16* dst, float4 v) {
  __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y);
  __nv_bfloat162 hi = __floats2bfloat162_rn(v.z, v.w);
  uint2 packed;
  packed.x = *reinterpret_cast<uint32_t*>(&lo);
  packed.y = *reinterpret_cast<uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(dst) = packed;
}

template <typename OutT>
__global__ void __launch_bounds__(256) lse_merge_kernel(const float* __restrict__ o_parts,
                                                        const float* __restrict__ lse_parts,
                                                        int P, long long rows, int d_v,
                                                        OutT* __restrict__ out,
                                                        float* __restrict__ lse_out) {
  const int lanes_per_row = d_v >> 2;            // 32 (d_v = 128) or 16 (d_v = 64)
  const int rows_per_warp = 32 / lanes_per_row;
  const int lane = threadIdx.x & 31;
  const int sub = lane / lanes_per_row;
  const int col = (lane % lanes_per_row) * 4;
  const long long warp = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long n_warps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  const long long part_stride = rows * d_v;

  for (long long r = warp * rows_per_warp + sub; r < rows; r += n_warps * rows_per_warp) {
    float m = -INFINITY;
    for (int p = 0; p < P; ++p) m = fmaxf(m, __ldg(lse_parts + p * rows + r));
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float w_sum = 0.f;
    if (m != -INFINITY) {
      const float* src = o_parts + r * d_v + col;
#pragma unroll 4
      for (int p = 0; p < P; ++p) {
        const float l = __ldg(lse_parts + p * rows + r);
        const float4 o = __ldcs(reinterpret_cast<const float4*>(src + p * part_stride));
        const float w = (l == -INFINITY) ? 0.f : expf(l - m);
        w_sum += w;
        acc.x = fmaf(w, o.x, acc.x);
        acc.y = fmaf(w, o.y, acc.y);
        acc.z = fmaf(w, o.z, acc.z);
        acc.w = fmaf(w, o.w, acc.w);
      }
      const float inv = 1.f / w_sum;
      acc.x *= inv; acc.y *= inv; acc.z *= inv; acc.w *= inv;
    }
    store4<OutT>(out + r * d_v + col, acc);
    if (lse_out != nullptr && col == 0) {
      lse_out[r] = (m == -INFINITY) ? -INFINITY : m + logf(w_sum);
    }
  }
}

// The same merge with at most MAXP partials: every LSE and O load of a row is
// issued before any arithmetic, so a row costs one trip to memory instead of
// two (the LSE maxima first, then the weighted sum).  Each lane covers
// 4 * VEC columns: with many rows VEC = 2 (a warp takes two rows at d_v = 128,
// four at 64), so that each resident warp has twice the bytes in flight and
// the rows need half as many warps; a few rows keep VEC = 1 (shorter per-lane
// latency chain, and the warps are not the limit there).
template <typename OutT, int MAXP, int VEC>
__global__ void __launch_bounds__(256) lse_merge_few_kernel(const float* __restrict__ o_parts,
                                                            const float* __restrict__ lse_parts,
                                                            int P, long long rows, int d_v,
                                                            OutT* __restrict__ out,
                                                            float* __restrict__ lse_out) {
  const int lanes_per_row = d_v / (4 * VEC);
  const int rows_per_warp = 32 / lanes_per_row;
  const int lane = threadIdx.x & 31;
  const int sub = lane / lanes_per_row;
  const int col = (lane % lanes_per_row) * 4 * VEC;
  const long long warp = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long n_warps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  const long long part_stride = rows * d_v;
  for (long long r = warp * rows_per_warp + sub; r < rows; r += n_warps * rows_per_warp) {
    float l[MAXP];
    float4 o[MAXP][VEC];
    const float* src = o_parts + r * d_v + col;
#pragma unroll
    for (int p = 0; p < MAXP; ++p) {
      if (p < P) {
        l[p] = __ldg(lse_parts + p * rows + r);
#pragma unroll
        for (int h = 0; h < VEC; ++h)
          o[p][h] = __ldcs(reinterpret_cast<const float4*>(src + p * part_stride + 4 * h));
      }
    }
    float m = -INFINITY;
#pragma unroll
    for (int p = 0; p < MAXP; ++p)
      if (p < P) m = fmaxf(m, l[p]);
    float4 acc[VEC];
#pragma unroll
    for (int h = 0; h < VEC; ++h) acc[h] = make_float4(0.f, 0.f, 0.f, 0.f);
    float w_sum = 0.f;
    if (m != -INFINITY) {
#pragma unroll
      for (int p = 0; p < MAXP; ++p) {
        if (p < P) {
          const float w = (l[p] == -INFINITY) ? 0.f : expf(l[p] - m);
          w_sum += w;
#pragma unroll
          for (int h = 0; h < VEC; ++h) {
            acc[h].x = fmaf(w, o[p][h].x, acc[h].x);
            acc[h].y = fmaf(w, o[p][h].y, acc[h].y);
            acc[h].z = fmaf(w, o[p][h].z, acc[h].z);
            acc[h].w = fmaf(w, o[p][h].w, acc[h].w);
          }
        }
      }
      const float inv = 1.f / w_sum;
#pragma unroll
      for (int h = 0; h < VEC; ++h) {
        acc[h].x *= inv; acc[h].y *= inv; acc[h].z *= inv; acc[h].w *= inv;
      }
    }
#pragma unroll
    for (int h = 0; h < VEC; ++h) store4<OutT>(out + r * d_v + col + 4 * h, acc[h]);
    if (lse_out != nullptr && col == 0) {
      lse_out[r] = (m == -INFINITY) ? -INFINITY : m + logf(w_sum);
    }
  }
}

// Few rows, many partials (the chunk partials of one decode shard): the
// row-per-warp kernel above would leave the GPU nearly idle and walk P
// partials serially.  Here eight warps share each row group, warp w taking
// partials p = w, w + 8, ...; each warp merges its subset relative to its own
// max, and the eight sub-results are merged the same way through shared memory
// (the merge is associative).
template <typename OutT>
__global__ void __launch_bounds__(256) lse_merge_splitp_kernel(const float* __restrict__ o_parts,
                                                               const float* __restrict__ lse_parts,
                                                               int P, long long rows, int d_v,
                                                               OutT* __restrict__ out,
                                                               float* __restrict__ lse_out) {
  constexpr int kWarps = 8;
  __shared__ float4 s_acc[kWarps][32];
  __shared__ float s_m[kWarps][32];
  __shared__ float s_w[kWarps][32];
  const int lanes_per_row = d_v >> 2;
  const int rows_per_warp = 32 / lanes_per_row;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int sub = lane / lanes_per_row;
  const int col = (lane % lanes_per_row) * 4;
  const long long part_stride = rows * d_v;
  for (long long r0 = static_cast<long long>(blockIdx.x) * rows_per_warp; r0 < rows;
       r0 += static_cast<long long>(gridDim.x) * rows_per_warp) {
    const long long r = r0 + sub;
    float m = -INFINITY, w_sum = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r < rows) {
      for (int p = warp; p < P; p += kWarps) m = fmaxf(m, __ldg(lse_parts + p * rows + r));
      if (m != -INFINITY) {
        const float* src = o_parts + r * d_v + col;
#pragma unroll 4
        for (int p = warp; p < P; p += kWarps) {
          const float l = __ldg(lse_parts + p * rows + r);
          const float4 o = __ldcs(reinterpret_cast<const float4*>(src + p * part_stride));
          const float w = (l == -INFINITY) ? 0.f : expf(l - m);
          w_sum += w;
          acc.x = fmaf(w, o.x, acc.x);
          acc.y = fmaf(w, o.y, acc.y);
          acc.z = fmaf(w, o.z, acc.z);
          acc.w = fmaf(w, o.w, acc.w);
        }
      }
    }
    s_acc[warp][lane] = acc;
    s_m[warp][lane] = m;
    s_w[warp][lane] = w_sum;
    __syncthreads();
    if (warp == 0 && r < rows) {
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) M = fmaxf(M, s_m[w][lane]);
      float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
      float tot = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
          const float mw = s_m[w][lane];
          const float f = (mw == -INFINITY) ? 0.f : expf(mw - M);
          const float4 a = s_acc[w][lane];
          tot = fmaf(f, s_w[w][lane], tot);
          o.x = fmaf(f, a.x, o.x);
          o.y = fmaf(f, a.y, o.y);
          o.z = fmaf(f, a.z, o.z);
          o.w = fmaf(f, a.w, o.w);
        }
        const float inv = 1.f / tot;
        o.x *= inv; o.y *= inv; o.z *= inv; o.w *= inv;
      }
      store4<OutT>(out + r * d_v + col, o);
      if (lse_out != nullptr && col == 0) lse_out[r] = (M == -INFINITY) ? -INFINITY : M + logf(tot);
    }
    __syncthreads();
  }
}

int launch_lse_merge(const float* o_parts, const float* lse_parts, int P, long long rows, int d_v,
                     void* out, ra_dtype out_dtype, float* lse, int num_sms, cudaStream_t stream) {
  const int threads = 256;
  const int rows_per_warp = 32 / (d_v / 4);
  const long long warps_needed = (rows + rows_per_warp - 1) / rows_per_warp;
  if (P >= 8 && warps_needed < static_cast<long long>(num_sms) * 16) {
    // few rows: eight warps per row group, each over a subset of the partials
    const int grid = static_cast<int>(warps_needed);
    if (out_dtype == RA_F32)
      lse_merge_splitp_kernel<float><<<grid, threads, 0, stream>>>(
          o_parts, lse_parts, P, rows, d_v, static_cast<float*>(out), lse);
    else
      lse_merge_splitp_kernel<__nv_bfloat16><<<grid, threads, 0, stream>>>(
          o_parts, lse_parts, P, rows, d_v, static_cast<__nv_bfloat16*>(out), lse);
  } else {
    // P <= 4 with more rows than one row per resident warp covers: two float4
    // per lane, twice the rows per warp
    const bool wide = P <= 4 && warps_needed > static_cast<long long>(num_sms) * 32;
    const int rows_per_cta = (threads / 32) * (wide ? 2 * rows_per_warp : rows_per_warp);
    long long want = (rows + rows_per_cta - 1) / rows_per_cta;
    long long cap = static_cast<long long>(num_sms) * 8;   // 8 resident CTAs / SM
    int grid = static_cast<int>(want < cap ? want : cap);
    if (grid < 1) grid = 1;
    // Up to four partials fit in registers (48 per thread with one float4 a
    // lane, 64 with two); more would cut the resident warps (8 partials: 70
    // registers, 24 warps per SM instead of 64) and lose more than the single
    // round trip gains, so those loop.
    if (P <= 4 && wide && out_dtype == RA_F32) {
      lse_merge_few_kernel<float, 4, 2><<<grid, threads, 0, stream>>>(
          o_parts, lse_parts, P, rows, d_v, static_cast<float*>(out), lse);
    } else if (P <= 4 && wide) {
      lse_merge_few_kernel<__nv_bfloat16, 4, 2><<<grid, threads, 0, stream>>>(
          o_parts, lse_parts, P, rows, d_v, static_cast<__nv_bfloat16*>(out), lse);
    } else if (P <= 4 && out_dtype == RA_F32) {
      lse_merge_few_kernel<float, 4, 1><<<grid, threads, 0, stream>>>(
          o_parts, lse_parts, P, rows, d_v, static_cast<float*>(out), lse);
    } else if (P <= 4) {
      lse_merge_few_kernel<__nv_bfloat16, 4, 1><<<grid, threads, 0, stream>>>(
          o_parts, lse_parts, P, rows, d_v, static_cast<__nv_bfloat16*>(out), lse);
    } else if (out_dtype == RA_F32) {
      lse_merge_kernel<float><<<grid, threads, 0, stream>>>(o_parts, lse_parts, P, rows, d_v,
                                                            static_cast<float*>(out), lse);
    } else {
      lse_merge_kernel<__nv_bfloat16><<<grid, threads, 0, stream>>>(
          o_parts, lse_parts, P, rows, d_v, static_cast<__nv_bfloat16*>(out), lse);
    }
  }
  note_launch();
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

}  // namespace ra
