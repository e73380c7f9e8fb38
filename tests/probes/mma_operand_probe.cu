// Time per tcgen05.mma (kind::f16, bf16 -> fp32, M = 128, K = 16,
// cta_group::1) by operand form, from one issuing lane: A and B both from
// shared memory with each K-major or MN-major (128-byte swizzle, the layouts
// the attention kernels use), A from tensor memory, and N = 64 against
// N = 128.  One CTA per SM, 2048 instructions in batches of 8 whose B operand
// alternates between two 32 KB slots; clock64 around them and the commit that
// tracks them, the wait bounded.  Prints one JSON object of cycles per
// instruction.
#include <cstdio>
#include <vector>
#include "ptx.cuh"
using namespace ra;
constexpr int kBatches = 256;
__device__ __forceinline__ uint32_t kstep(int ks) { return ((ks >> 2) * 16384 + (ks & 3) * 32) >> 4; }
__device__ __forceinline__ uint32_t mstep(int ks) { return (ks * 2048) >> 4; }
template <int MODE>
__global__ void __launch_bounds__(128, 1) probe(long long* out, int* err) {
  extern __shared__ uint8_t raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  uint8_t* A = sm;            // 32 KB
  uint8_t* B = sm + 32768;    // 2 slots x 32 KB
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + 32768 + 65536);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < (32768 + 65536) / 4; i += blockDim.x)
    reinterpret_cast<uint32_t*>(sm)[i] = 0x3c003c00u;
  if (threadIdx.x == 0) { mbar_init(bar, 1); fence_mbar_init(); }
  if (warp == 0) { tmem_alloc(tslot, 512); tmem_relinquish(); }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const uint32_t a_base = smem_u32(A), b_base = smem_u32(B);
  // forms: 0 A, B K-major; 1 A K-major, B MN-major; 2 both MN-major;
  // 3 A in tensor memory, B MN-major; 4 as 0 at N = 64; 5 A in tensor
  // memory, B K-major.  The A tile of the tensor-memory forms is columns
  // 128..191 (uninitialised: the values do not change the timing).
  constexpr int N = MODE == 4 ? 64 : 128;
  constexpr int amn = MODE == 2 ? 1 : 0;
  constexpr int bmn = (MODE == 1 || MODE == 2 || MODE == 3) ? 1 : 0;
  constexpr uint32_t id = idesc_bf16_f32(128, N, amn, bmn);
  if (warp == 0 && lane == 0) {
    const uint64_t da = amn ? sdesc_mn_sw128(a_base, 16384) : sdesc_k_sw128(a_base);
    const long long t0 = clock64();
    for (int bt = 0; bt < kBatches; ++bt) {
      const uint32_t bb = b_base + (bt & 1) * 32768;
      const uint64_t db = bmn ? sdesc_mn_sw128(bb, 16384) : sdesc_k_sw128(bb);
      const uint32_t d = tmem + 256 + (bt & 1) * 128;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t oa = amn ? mstep(ks) : kstep(ks);
        const uint32_t ob = bmn ? mstep(ks) : kstep(ks);
        if constexpr (MODE == 3 || MODE == 5)
          umma_ts(d, tmem + 128 + ks * 8, db + ob, id, ks > 0 ? 1u : 0u);
        else
          umma_ss(d, da + oa, db + ob, id, ks > 0 ? 1u : 0u);
      }
    }
    umma_commit(bar);
    const unsigned long long g0 = globaltimer_ns();
    bool ok = false;
    while (globaltimer_ns() - g0 < 1000000000ull)
      if (mbar_try_wait(bar, 0)) { ok = true; break; }
    if (!ok) atomicExch(err, 1);
    out[blockIdx.x] = clock64() - t0;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}
template <int MODE>
bool run(int sms, int smem, long long* d_out, double* cyc, int* d_err) {
  cudaFuncSetAttribute(probe<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  for (int rep = 0; rep < 3; ++rep) probe<MODE><<<sms, 128, smem>>>(d_out, d_err);
  if (cudaDeviceSynchronize() != cudaSuccess) return false;
  std::vector<long long> h(sms);
  cudaMemcpy(h.data(), d_out, sms * sizeof(long long), cudaMemcpyDeviceToHost);
  double s = 0;
  for (long long x : h) s += (double)x;
  *cyc = s / sms / (kBatches * 8);
  return true;
}
int main() {
  int sms = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, 0);
  long long* d_out; int* d_err;
  cudaMalloc(&d_out, sms * sizeof(long long));
  cudaMalloc(&d_err, sizeof(int));
  cudaMemset(d_err, 0, sizeof(int));
  const int smem = 1024 + 32768 + 65536 + 1024;
  double c[6];
  if (!run<0>(sms, smem, d_out, &c[0], d_err) || !run<1>(sms, smem, d_out, &c[1], d_err) ||
      !run<2>(sms, smem, d_out, &c[2], d_err) || !run<3>(sms, smem, d_out, &c[3], d_err) ||
      !run<4>(sms, smem, d_out, &c[4], d_err) || !run<5>(sms, smem, d_out, &c[5], d_err)) return 4;
  int herr = 0;
  cudaMemcpy(&herr, d_err, sizeof(int), cudaMemcpyDeviceToHost);
  printf("{\"ss_kk\": %.1f, \"ss_k_mn\": %.1f, \"ss_mn_mn\": %.1f, \"ts_b_mn\": %.1f, \"ss_kk_n64\": %.1f, \"ts_b_k\": %.1f, \"timeouts\": %d}\n", c[0], c[1], c[2], c[3], c[4], c[5], herr);
  return herr ? 5 : 0;
}
