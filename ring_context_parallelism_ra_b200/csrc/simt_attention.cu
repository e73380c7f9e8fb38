// Exact-fp32 attention on CUDA cores for fp32 inputs (SIMT FMA, no tensor
// cores: TF32 would not hold fp32 results within 1e-4 of the fp64 definition).
//
// One CTA owns 64 query rows of one (batch, head).  It walks the KV
// partitions in ring order j = i, i-1, ..., i-P+1 (mod P) where i is the
// partition of its first row (page "AI 推理系列（十一）：Ring Attention 如何让多张
// GPU 共同计算一条超长序列", section "KV 在 Ring 中如何流动"), and within a
// partition the 64-key tiles in order.  Tiles whose keys all lie in the causal
// future are skipped; the others are folded into the running row max m, the
// running exponential sum l and the rescaled accumulator o (same page, section
// "最容易被忽略的细节"), in base 2 with log2(e) folded into the scale.
// Four threads share a query row: each scores 16 of the 64 keys and owns a
// quarter of the d_v output columns.
#include "block_class.cuh"
#include "common.cuh"
#include "launch.h"

namespace ra {

namespace {

constexpr int kBM = 64;
constexpr int kBN = 64;
constexpr int kThreads = 256;

template <int DQK, int DV>
constexpr size_t simt_smem_bytes() {
  return sizeof(float) * (kBM * (DQK + 1) + kBN * (DQK + 1) + kBN * DV + kBM * (kBN + 1));
}

template <typename T, typename OutT, int DQK, int DV>
__global__ void __launch_bounds__(kThreads) simt_attention_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, int Hq, int Hkv,
    int n_q, int n_k, int P, int q_offset, int k_offset, long long stride, int causal,
    int striped, float scale_log2, OutT* __restrict__ out, float* __restrict__ lse) {
  constexpr int QS = DQK + 1;
  constexpr int PS = kBN + 1;
  constexpr int CPT = DV / 4;  // output columns per thread
  extern __shared__ float smem[];
  float* Qs = smem;
  float* Ks = Qs + kBM * QS;
  float* Vs = Ks + kBN * QS;
  float* Ps = Vs + kBN * DV;

  const int tid = threadIdx.x;
  const int r = tid >> 2;
  const int c = tid & 3;
  const int row0 = blockIdx.x * kBM;
  const int bh = blockIdx.y;
  const int b = bh / Hq;
  const int h = bh % Hq;
  const int g = h / (Hq / Hkv);
  const int rows_here = min(kBM, n_q - row0);

  const T* qh = q + (static_cast<long long>(bh) * n_q) * DQK;
  const T* kh = k + (static_cast<long long>(b) * Hkv + g) * n_k * DQK;
  const T* vh = v + (static_cast<long long>(b) * Hkv + g) * n_k * DV;

  for (int e = tid; e < kBM * DQK; e += kThreads) {
    const int rr = e / DQK, cc = e % DQK;
    Qs[rr * QS + cc] = (rr < rows_here) ? to_f32(qh[static_cast<long long>(row0 + rr) * DQK + cc]) : 0.f;
  }

  float m = -INFINITY, l = 0.f;
  float o[CPT];
#pragma unroll
  for (int t = 0; t < CPT; ++t) o[t] = 0.f;

  const int part_q = n_q / P;
  const int part_k = n_k / P;
  const int i = min(row0 / part_q, P - 1);
  // positions: row t is token qoff + t * st, key u is token koff + u * st;
  // in the striped split row R of partition p is token R * P + p * (1 - L * P)
  const long long st = striped ? P : stride;
  const long long qoff = striped ? static_cast<long long>(i) * (1 - static_cast<long long>(part_q) * P)
                                 : static_cast<long long>(q_offset);

  for (int s = 0; s < P; ++s) {
    const int j = (i - s + P) % P;
    const int kbeg = j * part_k;
    const int kend = kbeg + part_k;
    const long long koff = striped ? static_cast<long long>(j) * (1 - static_cast<long long>(part_k) * P)
                                   : static_cast<long long>(k_offset);
    for (int kt = kbeg; kt < kend; kt += kBN) {
      const int klen = min(kBN, kend - kt);
      const int8_t cls = tile_class(row0, rows_here, kt, klen, qoff, koff, causal, st);
      if (cls == kSkip) continue;
      __syncthreads();  // previous tile fully consumed (and Q stored, first time)
      for (int e = tid; e < kBN * DQK; e += kThreads) {
        const int rr = e / DQK, cc = e % DQK;
        Ks[rr * QS + cc] = (rr < klen) ? to_f32(kh[static_cast<long long>(kt + rr) * DQK + cc]) : 0.f;
      }
      for (int e = tid; e < kBN * DV; e += kThreads) {
        const int rr = e / DV, cc = e % DV;
        Vs[rr * DV + cc] = (rr < klen) ? to_f32(vh[static_cast<long long>(kt + rr) * DV + cc]) : 0.f;
      }
      __syncthreads();

      const long long lim = (cls == kFull) ? klen : visible_keys(row0 + r, kt, qoff, koff, st);
      float sc[kBN / 4];
      float mx = -INFINITY;
#pragma unroll
      for (int mm = 0; mm < kBN / 4; ++mm) {
        const int jl = c + 4 * mm;
        const float* kr = Ks + jl * QS;
        const float* qr = Qs + r * QS;
        float acc = 0.f;
#pragma unroll 8
        for (int kk = 0; kk < DQK; ++kk) acc = fmaf(qr[kk], kr[kk], acc);
        float sv = acc * scale_log2;
        const bool vis = jl < klen && jl < lim;
        sv = vis ? sv : -INFINITY;
        sc[mm] = sv;
        mx = fmaxf(mx, sv);
      }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float m_new = fmaxf(m, mx);
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = (m == -INFINITY) ? 0.f : exp2f(m - m_use);
      float rs = 0.f;
#pragma unroll
      for (int mm = 0; mm < kBN / 4; ++mm) {
        const float p = exp2f(sc[mm] - m_use);
        rs += p;
        Ps[r * PS + c + 4 * mm] = p;
      }
      rs += __shfl_xor_sync(0xffffffffu, rs, 1);
      rs += __shfl_xor_sync(0xffffffffu, rs, 2);
      l = l * alpha + rs;
#pragma unroll
      for (int t = 0; t < CPT; ++t) o[t] *= alpha;
      __syncwarp();
      for (int jj = 0; jj < klen; ++jj) {
        const float p = Ps[r * PS + jj];
        const float* vr = Vs + jj * DV + c;
#pragma unroll
        for (int t = 0; t < CPT; ++t) o[t] = fmaf(p, vr[4 * t], o[t]);
      }
      m = m_new;
    }
  }

  if (r < rows_here) {
    const long long orow = static_cast<long long>(bh) * n_q + row0 + r;
    const float inv = (l > 0.f) ? 1.f / l : 0.f;
#pragma unroll
    for (int t = 0; t < CPT; ++t) out[orow * DV + c + 4 * t] = from_f32<OutT>(o[t] * inv);
    if (lse != nullptr && c == 0) lse[orow] = (l > 0.f) ? (m + log2f(l)) * kLn2 : -INFINITY;
  }
}

template <typename T, typename OutT, int DQK, int DV>
int launch_typed(const void* q, const void* k, const void* v, const ra_shape& s, int P, int q_offset,
                 int k_offset, long long stride, int causal, int striped, float scale, void* out,
                 float* lse, cudaStream_t stream) {
  auto kern = simt_attention_kernel<T, OutT, DQK, DV>;
  const size_t smem = simt_smem_bytes<DQK, DV>();
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return RA_ERR_CUDA;
  dim3 grid((s.n_q + kBM - 1) / kBM, s.B * s.Hq);
  kern<<<grid, kThreads, smem, stream>>>(static_cast<const T*>(q), static_cast<const T*>(k),
                                         static_cast<const T*>(v), s.Hq, s.Hkv, s.n_q, s.n_k, P,
                                         q_offset, k_offset, stride, causal, striped,
                                         scale * kLog2e, static_cast<OutT*>(out), lse);
  note_launch();
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

template <typename T, typename OutT>
int dispatch_dims(const void* q, const void* k, const void* v, const ra_shape& s, int P, int qo,
                  int ko, long long st, int causal, int striped, float scale, void* out, float* lse,
                  cudaStream_t stm) {
  if (s.d_qk == 64 && s.d_v == 64)
    return launch_typed<T, OutT, 64, 64>(q, k, v, s, P, qo, ko, st, causal, striped, scale, out,
                                         lse, stm);
  if (s.d_qk == 128 && s.d_v == 128)
    return launch_typed<T, OutT, 128, 128>(q, k, v, s, P, qo, ko, st, causal, striped, scale, out,
                                           lse, stm);
  if (s.d_qk == 64 && s.d_v == 128)
    return launch_typed<T, OutT, 64, 128>(q, k, v, s, P, qo, ko, st, causal, striped, scale, out,
                                          lse, stm);
  if (s.d_qk == 128 && s.d_v == 64)
    return launch_typed<T, OutT, 128, 64>(q, k, v, s, P, qo, ko, st, causal, striped, scale, out,
                                          lse, stm);
  return RA_ERR_UNSUPPORTED;
}

}  // namespace

int launch_simt_attention(const void* q, const void* k, const void* v, const ra_shape& s, int P,
                          int q_offset, int k_offset, long long stride, int causal, int striped,
                          float scale, void* out, bool out_f32, float* lse,
                          const DeviceInfo& dev, cudaStream_t stream) {
  (void)dev;
  (void)out_f32;  // fp32 inputs give fp32 outputs
  if (s.dtype != RA_F32) return RA_ERR_UNSUPPORTED;  // bf16 runs on the tensor-core kernel
  return dispatch_dims<float, float>(q, k, v, s, P, q_offset, k_offset, stride, causal, striped,
                                     scale, out, lse, stream);
}

}  // namespace ra
