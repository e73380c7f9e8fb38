// Issue rate of tcgen05.mma (kind::f16, M = 128, K = 16, cta_group::1) from
// one thread, as the attention kernels issue it: batches of 8 instructions
// whose B operand moves to one of 5 shared-memory slots per batch (a K/V
// ring).  One CTA per SM; clock64 around 2048 instructions and the commit
// that tracks them; every wait is bounded.  Prints one JSON object of cycles
// per instruction (nominal: 64 at N = 128, 128 at N = 256).
#include <cstdio>
#include <vector>

#include "ptx.cuh"

using namespace ra;

constexpr int kBatches = 256;
constexpr int kModes = 4;

__device__ __forceinline__ bool elect_lane() {
  uint32_t pred = 0;
  asm volatile("{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\tselp.u32 %0, 1, 0, p;\n\t}"
               : "=r"(pred));
  return pred != 0;
}

// Each form is its own instantiation (MODE), so that the code the compiler
// generates for one does not depend on the others.
template <int MODE>
__global__ void __launch_bounds__(128, 1) probe(long long* out, int* err) {
  constexpr int mode = MODE;
  extern __shared__ uint8_t raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  uint8_t* A = sm;               // 128 rows x 128 bf16: 2 atoms of 16 KB
  uint8_t* B = sm + 32768;       // 3 slots of 256 rows x 128 bf16 (64 KB each)
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + 32768 + 3 * 65536);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < (32768 + 3 * 65536) / 4; i += blockDim.x)
    reinterpret_cast<uint32_t*>(sm)[i] = 0x3c003c00u;
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tslot, 512);
    tmem_relinquish();
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const uint32_t a_base = smem_u32(A), b_base = smem_u32(B);
  constexpr uint32_t id = idesc_bf16_f32(128, mode == 3 ? 256 : 128, 0, 0);
  constexpr bool converged = mode == 1;
  if (warp == 0 && (converged || lane == 0)) {
    const uint64_t da = sdesc_k_sw128(a_base);
    const long long t0 = clock64();
    for (int bt = 0; bt < kBatches; ++bt) {
      const int s = bt % 3;
      const uint64_t db = sdesc_k_sw128(b_base + s * 65536);
      const uint32_t d = tmem + (bt & 1) * 256;
      if constexpr (mode == 2) {  // descriptors formed first, then issued
        uint64_t pa[8], pb[8];
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t off = ((ks >> 2) * 16384 + (ks & 3) * 32) >> 4;
          pa[ks] = da + off;
          pb[ks] = db + (((ks >> 2) * 32768 + (ks & 3) * 32) >> 4);
        }
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) umma_ss(d, pa[ks], pb[ks], id, ks > 0 ? 1u : 0u);
      } else {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t off = ((ks >> 2) * 16384 + (ks & 3) * 32) >> 4;
          const uint32_t offb = ((ks >> 2) * 32768 + (ks & 3) * 32) >> 4;
          if constexpr (converged) {
            if (elect_lane()) umma_ss(d, da + off, db + offb, id, ks > 0 ? 1u : 0u);
            __syncwarp();
          } else {
            umma_ss(d, da + off, db + offb, id, ks > 0 ? 1u : 0u);
          }
        }
      }
    }
    if (!converged || elect_lane()) {
      umma_commit(bar);
      const unsigned long long g0 = globaltimer_ns();
      bool ok = false;
      while (globaltimer_ns() - g0 < 1000000000ull)
        if (mbar_try_wait(bar, 0)) { ok = true; break; }
      if (!ok) atomicExch(err, 1);
      out[blockIdx.x] = clock64() - t0;
    }
    if (converged) __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

template <int MODE>
bool run(int sms, int smem, long long* d_out, int* d_err, double* cyc) {
  cudaFuncSetAttribute(probe<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  for (int rep = 0; rep < 3; ++rep) probe<MODE><<<sms, 128, smem>>>(d_out, d_err);
  if (cudaDeviceSynchronize() != cudaSuccess) return false;
  std::vector<long long> h(sms);
  cudaMemcpy(h.data(), d_out, sms * sizeof(long long), cudaMemcpyDeviceToHost);
  double s = 0;
  for (long long x : h) s += static_cast<double>(x);
  *cyc = s / sms / (kBatches * 8);
  return true;
}

int main() {
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, 0) != cudaSuccess) return 2;
  long long* d_out;
  int* d_err;
  cudaMalloc(&d_out, sms * sizeof(long long));
  cudaMalloc(&d_err, sizeof(int));
  cudaMemset(d_err, 0, sizeof(int));
  const int smem = 1024 + 32768 + 3 * 65536 + 1024;
  if (smem > 232448) return 3;
  double c[kModes];
  if (!run<0>(sms, smem, d_out, d_err, &c[0]) || !run<1>(sms, smem, d_out, d_err, &c[1]) ||
      !run<2>(sms, smem, d_out, d_err, &c[2]) || !run<3>(sms, smem, d_out, d_err, &c[3]))
    return 4;
  int herr = 0;
  cudaMemcpy(&herr, d_err, sizeof(int), cudaMemcpyDeviceToHost);
  printf("{\"lane0_inline\": %.1f, \"converged_elect\": %.1f, \"lane0_formed_first\": %.1f, "
         "\"lane0_inline_n256\": %.1f, \"timeouts\": %d}\n", c[0], c[1], c[2], c[3], herr);
  return herr ? 5 : 0;
}
