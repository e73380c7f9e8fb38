// Exact-fp32 backward pass on the FMA pipes (no tensor cores): the same
// gradients and the same walk as the tensor-core kernel (bwd.cuh), with
// 64-key tiles against 64-row query tiles.  It serves fp32 inputs (dK, dV
// stored as fp32, or added into the caller's fp32 accumulators for a block
// share); bf16 inputs run on the tensor cores (bwd_attention.cu,
// bwd_tc192.cu).
//
// One CTA (256 threads) per key tile of one (batch, KV head).  Per visit the
// CTA stages Q_t, dO_t and the rows' -LSE log2(e), D in shared memory, forms
// P and dS for the 64 x 64 pairs (thread (ty, tx) owns queries ty + 16 i and
// keys tx + 16 j), then accumulates dV, dK in registers (thread owns key
// tid / 4, columns tid % 4 + 4 c) and adds dQ_t into the fp32 workspace.
#include "block_class.cuh"
#include "bwd.cuh"
#include "common.cuh"
#include "launch.h"

namespace ra {

namespace {

constexpr int kBT = 64;  // keys per tile and rows per query tile
constexpr int kSimtThreads = 256;

template <int DQK, int DV>
struct SCfg {
  static constexpr int KP = DQK + 1;  // padded row pitch (floats)
  static constexpr int VP = DV + 1;
  static constexpr int SMEM_FLOATS = 2 * kBT * KP + 2 * kBT * VP + 2 * kBT * (kBT + 1) + 2 * kBT;
  static constexpr int SMEM = SMEM_FLOATS * 4;
};

__device__ __forceinline__ float widen(float x) { return x; }

// Store of a finished dK / dV entry: the output for the ring, or added into
// the fp32 accumulator of a block share.
template <typename T>
__device__ __forceinline__ void put(void* base, long long i, float x, int block_mode) {
  static_assert(sizeof(T) == 4, "fp32 inputs only");
  if (block_mode) {
    float* p = static_cast<float*>(base) + i;
    *p += x;
  } else {
    static_cast<float*>(base)[i] = x;
  }
}

template <typename T, int DQK, int DV>
__global__ void __launch_bounds__(kSimtThreads) bwd_simt_kernel(const T* __restrict__ q,
                                                               const T* __restrict__ k,
                                                               const T* __restrict__ v,
                                                               const T* __restrict__ dout,
                                                               BwdArgs a) {
  using C = SCfg<DQK, DV>;
  extern __shared__ float sf[];
  float* sK = sf;
  float* sQ = sK + kBT * C::KP;
  float* sV = sQ + kBT * C::KP;
  float* sdO = sV + kBT * C::VP;
  float* sP = sdO + kBT * C::VP;
  float* sdS = sP + kBT * (kBT + 1);
  float* sNL = sdS + kBT * (kBT + 1);
  float* sD = sNL + kBT;

  BItem it;
  if (!bwd_item_at(a, 0, it)) return;  // grid = items: one item per CTA
  const int tid = threadIdx.x;
  const int ty = tid >> 4, tx = tid & 15;
  const int ku = tid >> 2, kc = tid & 3;

  const T* kb = k + (static_cast<long long>(it.bkv) * a.n_k + it.k0) * DQK;
  const T* vb = v + (static_cast<long long>(it.bkv) * a.n_k + it.k0) * DV;
  for (int i = tid; i < kBT * DQK; i += kSimtThreads) {
    const int r = i / DQK, c = i % DQK;
    sK[r * C::KP + c] = r < it.klen ? widen(kb[i]) : 0.f;
  }
  for (int i = tid; i < kBT * DV; i += kSimtThreads) {
    const int r = i / DV, c = i % DV;
    sV[r * C::VP + c] = r < it.klen ? widen(vb[i]) : 0.f;
  }

  float dk[DQK / 4], dv[DV / 4];
#pragma unroll
  for (int c = 0; c < DQK / 4; ++c) dk[c] = 0.f;
#pragma unroll
  for (int c = 0; c < DV / 4; ++c) dv[c] = 0.f;

  QWalk w;
  w.start(a, it);
  int qt, h;
  while (w.next(a, it, qt, h)) {
    const int bh = it.b * a.Hq + h;
    const int q0 = qt * kBT;
    __syncthreads();  // previous visit done with the staged tiles
    const T* qb = q + (static_cast<long long>(bh) * a.n_q + q0) * DQK;
    const T* gb = dout + (static_cast<long long>(bh) * a.n_q + q0) * DV;
    for (int i = tid; i < kBT * DQK; i += kSimtThreads) {
      const int r = i / DQK, c = i % DQK;
      sQ[r * C::KP + c] = r < w.qlen ? widen(qb[i]) : 0.f;
    }
    for (int i = tid; i < kBT * DV; i += kSimtThreads) {
      const int r = i / DV, c = i % DV;
      sdO[r * C::VP + c] = r < w.qlen ? widen(gb[i]) : 0.f;
    }
    if (tid < kBT) {
      const long long vr = static_cast<long long>(bh) * a.ntq_ws * kBwdTile + q0 + tid;
      sNL[tid] = a.ws_nl2[vr];  // rows past n_q are padding: -inf, D = 0
      sD[tid] = a.ws_d[vr];
    }
    __syncthreads();
    // P and dS for this thread's 4 x 4 pairs
    const long long F = floor_div(w.qoff - it.koff, a.stride);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int qr = ty + 16 * i;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int ur = tx + 16 * j;
        float s = 0.f, dp = 0.f;
#pragma unroll 8
        for (int c = 0; c < DQK; ++c) s = fmaf(sQ[qr * C::KP + c], sK[ur * C::KP + c], s);
#pragma unroll 8
        for (int c = 0; c < DV; ++c) dp = fmaf(sdO[qr * C::VP + c], sV[ur * C::VP + c], dp);
        bool vis = ur < it.klen;
        if (a.causal) vis = vis && (static_cast<long long>(it.k0 + ur) - (q0 + qr) <= F);
        const float pv = vis ? exp2f(fmaf(s, a.scale_log2, sNL[qr])) : 0.f;
        sP[qr * (kBT + 1) + ur] = pv;
        sdS[qr * (kBT + 1) + ur] = pv * (dp - sD[qr]);
      }
    }
    __syncthreads();
    // dV[u] += sum_q P[q][u] dO[q];  dK[u] += sum_q dS[q][u] Q[q]
#pragma unroll 4
    for (int qr = 0; qr < kBT; ++qr) {
      const float pv = sP[qr * (kBT + 1) + ku];
      const float dsv = sdS[qr * (kBT + 1) + ku];
#pragma unroll
      for (int c = 0; c < DV / 4; ++c) dv[c] = fmaf(pv, sdO[qr * C::VP + kc + 4 * c], dv[c]);
#pragma unroll
      for (int c = 0; c < DQK / 4; ++c) dk[c] = fmaf(dsv, sQ[qr * C::KP + kc + 4 * c], dk[c]);
    }
    // dQ[q] = sum_u dS[q][u] K[u], added into the workspace (scaled later)
    {
      const int qr = ku;
      float dq[DQK / 4];
#pragma unroll
      for (int c = 0; c < DQK / 4; ++c) dq[c] = 0.f;
#pragma unroll 4
      for (int ur = 0; ur < kBT; ++ur) {
        const float dsv = sdS[qr * (kBT + 1) + ur];
#pragma unroll
        for (int c = 0; c < DQK / 4; ++c) dq[c] = fmaf(dsv, sK[ur * C::KP + kc + 4 * c], dq[c]);
      }
      if (qr < w.qlen) {
#pragma unroll
        for (int c = 0; c < DQK / 4; ++c)
          atomicAdd(a.ws_dq + bwd_dq_index(a, bh, q0 + qr, kc + 4 * c, DQK), dq[c]);
      }
    }
  }
  if (ku < it.klen) {
    const long long krow = static_cast<long long>(it.bkv) * a.n_k + it.k0 + ku;
#pragma unroll
    for (int c = 0; c < DQK / 4; ++c) put<T>(a.dk, krow * DQK + kc + 4 * c, dk[c] * a.scale, a.block_mode);
#pragma unroll
    for (int c = 0; c < DV / 4; ++c) put<T>(a.dv, krow * DV + kc + 4 * c, dv[c], a.block_mode);
  }
}

template <typename T, int DQK, int DV>
int launch_simt_bwd_typed(const void* q, const void* k, const void* v, const void* dout,
                          const BwdArgs& a, cudaStream_t st) {
  auto kern = bwd_simt_kernel<T, DQK, DV>;
  constexpr int smem = SCfg<DQK, DV>::SMEM;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return RA_ERR_CUDA;
  kern<<<a.items, kSimtThreads, smem, st>>>(static_cast<const T*>(q), static_cast<const T*>(k),
                                            static_cast<const T*>(v), static_cast<const T*>(dout),
                                            a);
  note_launch();
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

}  // namespace

int launch_simt_backward(const void* q, const void* k, const void* v, const void* dout,
                         const ra_shape& s, BwdArgs a, const DeviceInfo& dev,
                         cudaStream_t stream) {
  (void)dev;
  a.tq = a.tk = kBT;
  a.ntq = (s.n_q + kBT - 1) / kBT;
  a.ntk = (s.n_k + kBT - 1) / kBT;
  const long long items = static_cast<long long>(s.B) * s.Hkv * a.ntk;
  if (items > 0x7fffffffLL) return RA_ERR_UNSUPPORTED;
  a.items = static_cast<int>(items);
  if (s.dtype != RA_F32) return RA_ERR_UNSUPPORTED;
  if (s.d_qk == 64 && s.d_v == 64) return launch_simt_bwd_typed<float, 64, 64>(q, k, v, dout, a, stream);
  if (s.d_qk == 128 && s.d_v == 128)
    return launch_simt_bwd_typed<float, 128, 128>(q, k, v, dout, a, stream);
  if (s.d_qk == 64 && s.d_v == 128)
    return launch_simt_bwd_typed<float, 64, 128>(q, k, v, dout, a, stream);
  if (s.d_qk == 128 && s.d_v == 64)
    return launch_simt_bwd_typed<float, 128, 64>(q, k, v, dout, a, stream);
  return RA_ERR_UNSUPPORTED;
}

}  // namespace ra
