// Row kernels of the backward pass (HBM-bound): the per-row statistics the
// gradient kernels read (D = rowsum(dO * O), -LSE log2(e)) with the dQ
// accumulator zeroed, and the conversion of the accumulated dQ into its
// output.  The workspace layout is stated in bwd.cuh.
#include "bwd.cuh"
#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace ra {

namespace {

constexpr int kT = kBwdTile;

struct PrepArgs {
  const void* out;     // forward output (D = rowsum(dO * O)), or null
  const void* dout;
  const float* delta;  // caller's D, used when out is null
  const float* lse;    // forward LSE, or null (delta-only mode)
  int n_q, d_v;
  int row_pitch;       // rows per head in the destination arrays
  long long rows;      // B * Hq * row_pitch
  float* nl2;          // [rows] or null
  float* d_ws;         // [rows] or null
  float* dq_ws;        // zeroed when non-null
  long long dq_floats;
  float* delta_out;    // [B * Hq * n_q] or null
  unsigned int* counter;  // backward work-item counter, zeroed when non-null
};

// Eight consecutive elements of a row as fp32 (one 16-byte load for bf16, two
// for fp32).
__device__ __forceinline__ void load8(const __nv_bfloat16* src, float* x) {
  const uint4 u = *reinterpret_cast<const uint4*>(src);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void load8(const float* src, float* x) {
  const float4 a = *reinterpret_cast<const float4*>(src);
  const float4 b = *reinterpret_cast<const float4*>(src + 4);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

// TPR = d_v / 8 threads per destination row, each owning eight consecutive
// elements; the row's dot product closes with shuffles inside the group.
template <typename T, int TPR>
__global__ void __launch_bounds__(256) bwd_prep_kernel(PrepArgs p) {
  const long long nthreads = static_cast<long long>(gridDim.x) * blockDim.x;
  const long long tid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int part = threadIdx.x % TPR;
  const long long rows_span = (p.rows + (nthreads / TPR) - 1) / (nthreads / TPR) * (nthreads / TPR);
  for (long long r = tid / TPR; r < rows_span; r += nthreads / TPR) {
    const bool in = r < p.rows;
    const long long bh = in ? r / p.row_pitch : 0;
    const int t = in ? static_cast<int>(r % p.row_pitch) : p.n_q;
    float dsum = 0.f, nl = -INFINITY;
    if (t < p.n_q) {
      const long long src = bh * p.n_q + t;
      if (p.out != nullptr) {
        float o[8], g[8];
        load8(static_cast<const T*>(p.out) + src * p.d_v + part * 8, o);
        load8(static_cast<const T*>(p.dout) + src * p.d_v + part * 8, g);
#pragma unroll
        for (int i = 0; i < 8; ++i) dsum = fmaf(o[i], g[i], dsum);
      } else if (part == 0) {
        dsum = p.delta[src];
      }
      if (p.lse != nullptr) {
        const float l = p.lse[src];
        nl = (l == -INFINITY) ? -INFINITY : -l * kLog2e;
      }
    }
#pragma unroll
    for (int s = TPR / 2; s > 0; s >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, s, TPR);
    if (in && part == 0) {
      if (p.d_ws) p.d_ws[r] = dsum;
      if (p.nl2) p.nl2[r] = nl;
      if (p.delta_out && t < p.n_q) p.delta_out[bh * p.n_q + t] = dsum;
    }
  }
  if (p.counter != nullptr && tid == 0) *p.counter = 0u;
  if (p.dq_ws != nullptr) {
    float4* z = reinterpret_cast<float4*>(p.dq_ws);
    const long long n4 = p.dq_floats / 4;
    for (long long i = tid; i < n4; i += nthreads) z[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// dQ = scale * workspace (ring: stored in the output dtype) or dQ += scale *
// workspace (block: fp32 accumulator).  One CTA per (head, 128-row tile); 32
// columns at a time pass through shared memory: read as the workspace's
// [column / 4][row][4] float4 vectors, written as eight consecutive columns of
// a row per thread (16 bytes of bf16, 32 of fp32).
template <typename T, bool ACCUM>
__global__ void __launch_bounds__(256) bwd_dq_finalize_kernel(const float* ws, T* dq, float scale,
                                                              int n_q, int d_qk, int ntq) {
  __shared__ float tile[kT][33];
  const long long bh = blockIdx.x / ntq;
  const int qt = blockIdx.x % ntq;
  const float4* src = reinterpret_cast<const float4*>(
      ws + (bh * ntq + qt) * static_cast<long long>(d_qk) * kT);
  const int t0 = qt * kT;
  for (int c0 = 0; c0 < d_qk; c0 += 32) {
    for (int i = threadIdx.x; i < 8 * kT; i += blockDim.x) {
      const int g = i / kT, r = i % kT;
      const float4 x = src[(c0 / 4 + g) * kT + r];
      tile[r][4 * g] = x.x;
      tile[r][4 * g + 1] = x.y;
      tile[r][4 * g + 2] = x.z;
      tile[r][4 * g + 3] = x.w;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < 4 * kT; i += blockDim.x) {
      const int r = i / 4, q8 = (i % 4) * 8;
      if (t0 + r < n_q) {
        float x[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = tile[r][q8 + e] * scale;
        T* d = dq + (bh * n_q + t0 + r) * d_qk + c0 + q8;
        if constexpr (ACCUM) {
          float4* d4 = reinterpret_cast<float4*>(d);
          float4 a = d4[0], b = d4[1];
          a.x += x[0]; a.y += x[1]; a.z += x[2]; a.w += x[3];
          b.x += x[4]; b.y += x[5]; b.z += x[6]; b.w += x[7];
          d4[0] = a;
          d4[1] = b;
        } else if constexpr (sizeof(T) == 4) {
          float4* d4 = reinterpret_cast<float4*>(d);
          d4[0] = make_float4(x[0], x[1], x[2], x[3]);
          d4[1] = make_float4(x[4], x[5], x[6], x[7]);
        } else {
          *reinterpret_cast<uint4*>(d) =
              make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]),
                         pack_bf16x2(x[4], x[5]), pack_bf16x2(x[6], x[7]));
        }
      }
    }
    __syncthreads();
  }
}

int launch_prep(const PrepArgs& p, ra_dtype dt, const DeviceInfo& dev, cudaStream_t st) {
  const int tpr = p.d_v / 8;  // d_v is 64 or 128
  const long long blocks_rows = (p.rows * tpr + 255) / 256;
  long long blocks = blocks_rows < 8LL * dev.num_sms ? blocks_rows : 8LL * dev.num_sms;
  if (blocks < 1) blocks = 1;
  const int b = static_cast<int>(blocks);
  if (dt == RA_BF16) {
    if (tpr == 16) bwd_prep_kernel<__nv_bfloat16, 16><<<b, 256, 0, st>>>(p);
    else bwd_prep_kernel<__nv_bfloat16, 8><<<b, 256, 0, st>>>(p);
  } else {
    if (tpr == 16) bwd_prep_kernel<float, 16><<<b, 256, 0, st>>>(p);
    else bwd_prep_kernel<float, 8><<<b, 256, 0, st>>>(p);
  }
  note_launch();
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

}  // namespace

int launch_backward_delta(const void* out, const void* dout, const ra_shape& s, float* delta,
                          const DeviceInfo& dev, cudaStream_t stream) {
  PrepArgs p{};
  p.out = out;
  p.dout = dout;
  p.n_q = s.n_q;
  p.d_v = s.d_v;
  p.row_pitch = s.n_q;
  p.rows = static_cast<long long>(s.B) * s.Hq * s.n_q;
  p.delta_out = delta;
  return launch_prep(p, s.dtype, dev, stream);
}

int launch_backward_rows(const void* out, const void* dout, const float* delta, const float* lse,
                         const ra_shape& s, const BwdLayout& L, float* nl2, float* d_ws,
                         float* dq_ws, unsigned int* counter, const DeviceInfo& dev,
                         cudaStream_t stream) {
  PrepArgs p{};
  p.counter = counter;
  p.out = out;
  p.dout = dout;
  p.delta = delta;
  p.lse = lse;
  p.n_q = s.n_q;
  p.d_v = s.d_v;
  p.row_pitch = L.ntq * kBwdTile;
  p.rows = L.rows_pad;
  p.nl2 = nl2;
  p.d_ws = d_ws;
  p.dq_ws = dq_ws;
  p.dq_floats = L.rows_pad * s.d_qk;
  return launch_prep(p, s.dtype, dev, stream);
}

int launch_dq_finalize(const float* ws_dq, void* dq, const ra_shape& s, const BwdLayout& L,
                       float scale, bool block_mode, cudaStream_t stream) {
  const long long blocks = static_cast<long long>(s.B) * s.Hq * L.ntq;
  if (blocks > 0x7fffffffLL) return RA_ERR_UNSUPPORTED;
  if (block_mode) {
    bwd_dq_finalize_kernel<float, true><<<static_cast<int>(blocks), 256, 0, stream>>>(
        ws_dq, static_cast<float*>(dq), scale, s.n_q, s.d_qk, L.ntq);
  } else if (s.dtype == RA_BF16) {
    bwd_dq_finalize_kernel<__nv_bfloat16, false><<<static_cast<int>(blocks), 256, 0, stream>>>(
        ws_dq, static_cast<__nv_bfloat16*>(dq), scale, s.n_q, s.d_qk, L.ntq);
  } else {
    bwd_dq_finalize_kernel<float, false><<<static_cast<int>(blocks), 256, 0, stream>>>(
        ws_dq, static_cast<float*>(dq), scale, s.n_q, s.d_qk, L.ntq);
  }
  note_launch();
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

}  // namespace ra
