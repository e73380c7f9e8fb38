// C ABI of the library (declared in include/ra.h): argument validation on the
// host, then dispatch to the kernels.  Nothing here allocates device memory;
// the per-device status word is a module global whose address is looked up
// once per device.
#include <atomic>
#include <mutex>

#include "../../include/ra.h"
#include "block_class.cuh"
#include "launch.h"
#include "ptx.cuh"

// One status word per device (module globals are instantiated per device).
__device__ int g_ra_status_word;
// Work-item counters of the forward launches: each launch takes the next slot
// and zeroes it on its stream before the kernel, so launches that run at the
// same time on different streams use different slots as long as fewer than
// kItemCounterSlots are in flight.
__device__ unsigned int g_ra_item_counters[ra::kItemCounterSlots];

namespace ra {

namespace {

std::atomic<unsigned long long> g_launches{0};
std::atomic<unsigned int> g_counter_next{0};
std::atomic<unsigned long long> g_wait_ns{2000000000ull};

constexpr int kMaxDevices = 64;
std::mutex g_dev_mu;
DeviceInfo g_dev[kMaxDevices];
bool g_dev_ready[kMaxDevices] = {};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_common(const ra_shape* s) {
  if (s == nullptr) return RA_ERR_INVALID;
  if (s->B <= 0 || s->Hq <= 0 || s->Hkv <= 0 || s->n_q <= 0 || s->n_k <= 0 || s->d_qk <= 0 ||
      s->d_v <= 0)
    return RA_ERR_INVALID;
  if (s->Hq % s->Hkv != 0) return RA_ERR_INVALID;
  if (s->dtype != RA_F32 && s->dtype != RA_BF16) return RA_ERR_INVALID;
  return RA_OK;
}

int check_attention_dims(const ra_shape* s) {
  if (s->dtype == RA_F32) {
    if ((s->d_qk == 64 || s->d_qk == 128) && (s->d_v == 64 || s->d_v == 128)) return RA_OK;
    return RA_ERR_UNSUPPORTED;
  }
  if ((s->d_qk == 64 || s->d_qk == 128 || s->d_qk == 192) && (s->d_v == 64 || s->d_v == 128))
    return RA_OK;
  return RA_ERR_UNSUPPORTED;
}

int dispatch_attention(const void* q, const void* k, const void* v, const ra_shape& s, int P,
                       int q_offset, int k_offset, long long stride, int causal, int striped,
                       float scale, void* out, bool out_f32, float* lse, cudaStream_t st) {
  DeviceInfo dev;
  int rc = device_info(&dev);
  if (rc != RA_OK) return rc;
  if (s.dtype == RA_BF16)
    return launch_tc_attention(q, k, v, s, P, q_offset, k_offset, stride, causal, striped, scale,
                               out, out_f32, lse, dev, st);
  return launch_simt_attention(q, k, v, s, P, q_offset, k_offset, stride, causal, striped, scale,
                               out, out_f32, lse, dev, st);
}

int check_block_args(const void* q, const void* k, const void* v, const ra_shape* shape,
                     int q_offset, int k_offset, int causal, const float* o_part,
                     const float* lse_part) {
  int rc = check_common(shape);
  if (rc != RA_OK) return rc;
  if (!q || !k || !v || !o_part || !lse_part) return RA_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o_part) || !aligned16(lse_part))
    return RA_ERR_INVALID;
  if ((causal != 0 && causal != 1) || q_offset < 0 || k_offset < 0) return RA_ERR_INVALID;
  return check_attention_dims(shape);
}

int check_ring_args(const void* q, const void* k, const void* v, int P, int causal,
                    const void* out, const float* lse, const ra_shape* shape) {
  int rc = check_common(shape);
  if (rc != RA_OK) return rc;
  if (!q || !k || !v || !out) return RA_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
      (lse && !aligned16(lse)))
    return RA_ERR_INVALID;
  if (P < 1 || shape->n_q != shape->n_k || shape->n_q % P != 0) return RA_ERR_INVALID;
  if (causal != 0 && causal != 1) return RA_ERR_INVALID;
  return check_attention_dims(shape);
}

int check_backward_dims(const ra_shape* s) {
  // d_qk = 192 as the forward supports it: bf16 inputs only
  if (s->d_qk == 192 && s->dtype != RA_BF16) return RA_ERR_UNSUPPORTED;
  if ((s->d_qk == 64 || s->d_qk == 128 || s->d_qk == 192) && (s->d_v == 64 || s->d_v == 128))
    return RA_OK;
  return RA_ERR_UNSUPPORTED;
}

int check_ring_backward_args(const void* q, const void* k, const void* v, const void* out,
                             const float* lse, const void* dout, int P, int causal,
                             const void* dq, const void* dk, const void* dv,
                             const ra_shape* shape, const void* workspace,
                             size_t workspace_bytes) {
  int rc = check_common(shape);
  if (rc != RA_OK) return rc;
  if (!q || !k || !v || !out || !lse || !dout || !dq || !dk || !dv || !workspace)
    return RA_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse) ||
      !aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
      !aligned16(workspace))
    return RA_ERR_INVALID;
  if (P < 1 || shape->n_q != shape->n_k || shape->n_q % P != 0) return RA_ERR_INVALID;
  if (causal != 0 && causal != 1) return RA_ERR_INVALID;
  rc = check_backward_dims(shape);
  if (rc != RA_OK) return rc;
  if (workspace_bytes < backward_workspace_bytes(*shape)) return RA_ERR_INVALID;
  return RA_OK;
}

__global__ void block_class_kernel(int n_q, int n_k, int q_block, int k_block, int q_offset,
                                   int k_offset, int causal, int tq, int tk, int8_t* map) {
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<long long>(tq) * tk) return;
  const int bi = static_cast<int>(idx / tk);
  const int bj = static_cast<int>(idx % tk);
  const long long q0 = static_cast<long long>(bi) * q_block;
  const long long k0 = static_cast<long long>(bj) * k_block;
  const long long ql = (q0 + q_block <= n_q) ? q_block : n_q - q0;
  const long long kl = (k0 + k_block <= n_k) ? k_block : n_k - k0;
  map[idx] = tile_class(q0, ql, k0, kl, q_offset, k_offset, causal);
}

// One warp waits on an mbarrier that nothing arrives on; the bounded wait
// expires, records RA_ERR_TIMEOUT and the kernel returns.
__global__ void wait_timeout_kernel(DevCtx ctx) {
  __shared__ uint64_t bar;
  __shared__ int abort_word;
  volatile int* abort_flag = &abort_word;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, ctx, abort_flag);
}

}  // namespace

void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

int next_item_counter(const DeviceInfo& dev, cudaStream_t stream, unsigned int** out) {
  unsigned int* c = dev.item_counters + (g_counter_next.fetch_add(1) % kItemCounterSlots);
  if (cudaMemsetAsync(c, 0, sizeof(unsigned int), stream) != cudaSuccess) return RA_ERR_CUDA;
  *out = c;
  return RA_OK;
}

int device_info(DeviceInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return RA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_dev_mu);
  if (!g_dev_ready[dev]) {
    DeviceInfo d{};
    d.device = dev;
    if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
            cudaSuccess)
      return RA_ERR_CUDA;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_ra_status_word) != cudaSuccess) return RA_ERR_CUDA;
    d.ctx.status = static_cast<int*>(p);
    if (cudaGetSymbolAddress(&p, g_ra_item_counters) != cudaSuccess) return RA_ERR_CUDA;
    d.item_counters = static_cast<unsigned int*>(p);
    g_dev[dev] = d;
    g_dev_ready[dev] = true;
  }
  *out = g_dev[dev];
  out->ctx.wait_ns = g_wait_ns.load(std::memory_order_relaxed);
  return RA_OK;
}

int launch_block_class(int n_q, int n_k, int q_block, int k_block, int q_offset, int k_offset,
                       int causal, int8_t* map_dev, cudaStream_t stream) {
  const int tq = (n_q + q_block - 1) / q_block;
  const int tk = (n_k + k_block - 1) / k_block;
  const long long n = static_cast<long long>(tq) * tk;
  const int threads = 256;
  const long long blocks = (n + threads - 1) / threads;
  if (blocks > 0x7fffffffLL) return RA_ERR_INVALID;
  block_class_kernel<<<static_cast<int>(blocks), threads, 0, stream>>>(
      n_q, n_k, q_block, k_block, q_offset, k_offset, causal, tq, tk, map_dev);
  note_launch();
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

int launch_wait_timeout_check(const DevCtx& ctx, cudaStream_t stream) {
  wait_timeout_kernel<<<1, 32, 0, stream>>>(ctx);
  note_launch();
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

}  // namespace ra

using namespace ra;

extern "C" {

int ra_block_partial(const void* q, const void* k, const void* v, const ra_shape* shape,
                     int q_offset, int k_offset, int causal, float scale, float* o_part,
                     float* lse_part, void* stream) {
  const int rc = check_block_args(q, k, v, shape, q_offset, k_offset, causal, o_part, lse_part);
  if (rc != RA_OK) return rc;
  return dispatch_attention(q, k, v, *shape, 1, q_offset, k_offset, 1, causal, 0, scale, o_part,
                            true, lse_part, static_cast<cudaStream_t>(stream));
}

int ra_block_partial_strided(const void* q, const void* k, const void* v, const ra_shape* shape,
                             int q_offset, int k_offset, int pos_stride, int causal, float scale,
                             float* o_part, float* lse_part, void* stream) {
  const int rc = check_block_args(q, k, v, shape, q_offset, k_offset, causal, o_part, lse_part);
  if (rc != RA_OK) return rc;
  if (pos_stride < 1) return RA_ERR_INVALID;
  return dispatch_attention(q, k, v, *shape, 1, q_offset, k_offset, pos_stride, causal, 0, scale,
                            o_part, true, lse_part, static_cast<cudaStream_t>(stream));
}

int ra_ring_forward(const void* q, const void* k, const void* v, int P, int causal, float scale,
                    void* out, float* lse, const ra_shape* shape, void* stream) {
  const int rc = check_ring_args(q, k, v, P, causal, out, lse, shape);
  if (rc != RA_OK) return rc;
  return dispatch_attention(q, k, v, *shape, P, 0, 0, 1, causal, 0, scale, out,
                            shape->dtype == RA_F32, lse, static_cast<cudaStream_t>(stream));
}

int ra_ring_forward_striped(const void* q, const void* k, const void* v, int P, int causal,
                            float scale, void* out, float* lse, const ra_shape* shape,
                            void* stream) {
  const int rc = check_ring_args(q, k, v, P, causal, out, lse, shape);
  if (rc != RA_OK) return rc;
  if ((shape->n_q / P) % 256 != 0) return RA_ERR_UNSUPPORTED;
  return dispatch_attention(q, k, v, *shape, P, 0, 0, P, causal, 1, scale, out,
                            shape->dtype == RA_F32, lse, static_cast<cudaStream_t>(stream));
}

int ra_lse_merge(const float* o_parts, const float* lse_parts, int P, const ra_shape* shape,
                 void* out, ra_dtype out_dtype, float* lse, void* stream) {
  if (shape == nullptr || P < 1 || !o_parts || !lse_parts || !out) return RA_ERR_INVALID;
  if (shape->B <= 0 || shape->Hq <= 0 || shape->n_q <= 0) return RA_ERR_INVALID;
  if (shape->d_v != 32 && shape->d_v != 64 && shape->d_v != 128) return RA_ERR_UNSUPPORTED;
  if (out_dtype != RA_F32 && out_dtype != RA_BF16) return RA_ERR_INVALID;
  if (!aligned16(o_parts) || !aligned16(lse_parts) || !aligned16(out) || (lse && !aligned16(lse)))
    return RA_ERR_INVALID;
  DeviceInfo dev;
  int rc = device_info(&dev);
  if (rc != RA_OK) return rc;
  const long long rows = static_cast<long long>(shape->B) * shape->Hq * shape->n_q;
  return launch_lse_merge(o_parts, lse_parts, P, rows, shape->d_v, out, out_dtype, lse,
                          dev.num_sms, static_cast<cudaStream_t>(stream));
}

size_t ra_decode_workspace_bytes(const ra_shape* shape) {
  if (check_common(shape) != RA_OK) return 0;
  return decode_workspace_bytes(*shape);
}

int ra_decode_partial(const void* q, const void* k_shard, const void* v_shard,
                      long long kv_head_stride, const ra_shape* shape, float scale, float* o_part,
                      float* lse_part, void* workspace, size_t workspace_bytes, void* stream) {
  int rc = check_common(shape);
  if (rc != RA_OK) return rc;
  if (!q || !k_shard || !v_shard || !o_part || !lse_part || !workspace) return RA_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k_shard) || !aligned16(v_shard) || !aligned16(o_part) ||
      !aligned16(lse_part) || !aligned16(workspace))
    return RA_ERR_INVALID;
  if (shape->n_q != 1 || kv_head_stride < shape->n_k) return RA_ERR_INVALID;
  if (shape->dtype != RA_BF16 || shape->d_qk != 128 || shape->d_v != 128 ||
      shape->Hq / shape->Hkv > 16)
    return RA_ERR_UNSUPPORTED;
  if (workspace_bytes < decode_workspace_bytes(*shape)) return RA_ERR_INVALID;
  DeviceInfo dev;
  rc = device_info(&dev);
  if (rc != RA_OK) return rc;
  return launch_decode_partial(q, k_shard, v_shard, kv_head_stride, *shape, scale, o_part,
                               lse_part, static_cast<float*>(workspace), dev,
                               static_cast<cudaStream_t>(stream));
}

int ra_decode_partials(const void* q, const void* k, const void* v, int P,
                       const ra_shape* shape, float scale, float* o_parts, float* lse_parts,
                       void* workspace, size_t workspace_bytes, void* stream) {
  int rc = check_common(shape);
  if (rc != RA_OK) return rc;
  if (!q || !k || !v || !o_parts || !lse_parts || !workspace) return RA_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o_parts) ||
      !aligned16(lse_parts) || !aligned16(workspace))
    return RA_ERR_INVALID;
  if (shape->n_q != 1 || P < 1 || shape->n_k % P != 0) return RA_ERR_INVALID;
  if (shape->dtype != RA_BF16 || shape->d_qk != 128 || shape->d_v != 128 ||
      shape->Hq / shape->Hkv > 16 || (P > 1 && (shape->n_k / P) % 2048 != 0))
    return RA_ERR_UNSUPPORTED;
  if (workspace_bytes < decode_workspace_bytes(*shape)) return RA_ERR_INVALID;
  DeviceInfo dev;
  rc = device_info(&dev);
  if (rc != RA_OK) return rc;
  return launch_decode_partial(q, k, v, shape->n_k, *shape, scale, o_parts, lse_parts,
                               static_cast<float*>(workspace), dev,
                               static_cast<cudaStream_t>(stream), P);
}

int ra_decode_partial_noalloc(const void* q, const void* k_shard, const void* v_shard,
                              long long kv_head_stride, const ra_shape* shape, float scale,
                              float* o_part, float* lse_part, void* stream) {
  int rc = check_common(shape);
  if (rc != RA_OK) return rc;
  if (!q || !k_shard || !v_shard || !o_part || !lse_part) return RA_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k_shard) || !aligned16(v_shard) || !aligned16(o_part) ||
      !aligned16(lse_part))
    return RA_ERR_INVALID;
  if (shape->n_q != 1 || kv_head_stride < shape->n_k) return RA_ERR_INVALID;
  if (shape->dtype != RA_BF16 || shape->d_qk != 128 || shape->d_v != 128 ||
      shape->Hq / shape->Hkv > 16)
    return RA_ERR_UNSUPPORTED;
  if (decode_workspace_bytes(*shape) > decode_static_scratch_bytes()) return RA_ERR_UNSUPPORTED;
  DeviceInfo dev;
  rc = device_info(&dev);
  if (rc != RA_OK) return rc;
  return launch_decode_partial_static(q, k_shard, v_shard, kv_head_stride, *shape, scale, o_part,
                                      lse_part, dev, static_cast<cudaStream_t>(stream));
}

int ra_decode_merge(const float* o_parts, const float* lse_parts, int P, const ra_shape* shape,
                    void* out, ra_dtype out_dtype, float* lse, void* stream) {
  if (shape == nullptr || shape->n_q != 1) return RA_ERR_INVALID;
  return ra_lse_merge(o_parts, lse_parts, P, shape, out, out_dtype, lse, stream);
}

int ra_block_class(int n_q, int n_k, int q_block, int k_block, int q_offset, int k_offset,
                   int causal, int8_t* map_host) {
  if (!map_host || n_q <= 0 || n_k <= 0 || q_block <= 0 || k_block <= 0 || q_offset < 0 ||
      k_offset < 0 || (causal != 0 && causal != 1))
    return RA_ERR_INVALID;
  const int tq = (n_q + q_block - 1) / q_block;
  const int tk = (n_k + k_block - 1) / k_block;
  for (int bi = 0; bi < tq; ++bi) {
    const long long q0 = static_cast<long long>(bi) * q_block;
    const long long ql = (q0 + q_block <= n_q) ? q_block : n_q - q0;
    for (int bj = 0; bj < tk; ++bj) {
      const long long k0 = static_cast<long long>(bj) * k_block;
      const long long kl = (k0 + k_block <= n_k) ? k_block : n_k - k0;
      map_host[static_cast<long long>(bi) * tk + bj] =
          tile_class(q0, ql, k0, kl, q_offset, k_offset, causal);
    }
  }
  return RA_OK;
}

int ra_block_class_device(int n_q, int n_k, int q_block, int k_block, int q_offset, int k_offset,
                          int causal, int8_t* map_dev, void* stream) {
  if (!map_dev || n_q <= 0 || n_k <= 0 || q_block <= 0 || k_block <= 0 || q_offset < 0 ||
      k_offset < 0 || (causal != 0 && causal != 1))
    return RA_ERR_INVALID;
  return launch_block_class(n_q, n_k, q_block, k_block, q_offset, k_offset, causal, map_dev,
                            static_cast<cudaStream_t>(stream));
}

size_t ra_backward_workspace_bytes(const ra_shape* shape) {
  if (check_common(shape) != RA_OK) return 0;
  return backward_workspace_bytes(*shape);
}

int ra_backward_delta(const void* out, const void* dout, const ra_shape* shape, float* delta,
                      void* stream) {
  int rc = check_common(shape);
  if (rc != RA_OK) return rc;
  if (!out || !dout || !delta) return RA_ERR_INVALID;
  if (!aligned16(out) || !aligned16(dout) || !aligned16(delta)) return RA_ERR_INVALID;
  if (shape->d_v != 64 && shape->d_v != 128) return RA_ERR_UNSUPPORTED;
  DeviceInfo dev;
  rc = device_info(&dev);
  if (rc != RA_OK) return rc;
  return launch_backward_delta(out, dout, *shape, delta, dev, static_cast<cudaStream_t>(stream));
}

int ra_ring_backward(const void* q, const void* k, const void* v, const void* out,
                     const float* lse, const void* dout, int P, int causal, float scale, void* dq,
                     void* dk, void* dv, const ra_shape* shape, void* workspace,
                     size_t workspace_bytes, void* stream) {
  int rc = check_ring_backward_args(q, k, v, out, lse, dout, P, causal, dq, dk, dv, shape,
                                    workspace, workspace_bytes);
  if (rc != RA_OK) return rc;
  DeviceInfo dev;
  rc = device_info(&dev);
  if (rc != RA_OK) return rc;
  return launch_backward(q, k, v, out, lse, dout, nullptr, *shape, P, 0, 0, 1, causal, 0, scale,
                         dq, dk, dv, false, workspace, dev, static_cast<cudaStream_t>(stream));
}

int ra_ring_backward_striped(const void* q, const void* k, const void* v, const void* out,
                             const float* lse, const void* dout, int P, int causal, float scale,
                             void* dq, void* dk, void* dv, const ra_shape* shape, void* workspace,
                             size_t workspace_bytes, void* stream) {
  int rc = check_ring_backward_args(q, k, v, out, lse, dout, P, causal, dq, dk, dv, shape,
                                    workspace, workspace_bytes);
  if (rc != RA_OK) return rc;
  if ((shape->n_q / P) % 128 != 0) return RA_ERR_UNSUPPORTED;
  DeviceInfo dev;
  rc = device_info(&dev);
  if (rc != RA_OK) return rc;
  return launch_backward(q, k, v, out, lse, dout, nullptr, *shape, P, 0, 0, P, causal, 1, scale,
                         dq, dk, dv, false, workspace, dev, static_cast<cudaStream_t>(stream));
}

int ra_block_backward(const void* q, const void* k, const void* v, const void* dout,
                      const float* lse, const float* delta, const ra_shape* shape, int q_offset,
                      int k_offset, int pos_stride, int causal, float scale, float* dq_acc,
                      float* dk_acc, float* dv_acc, void* workspace, size_t workspace_bytes,
                      void* stream) {
  int rc = check_common(shape);
  if (rc != RA_OK) return rc;
  if (!q || !k || !v || !dout || !lse || !delta || !dq_acc || !dk_acc || !dv_acc || !workspace)
    return RA_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) || !aligned16(lse) ||
      !aligned16(delta) || !aligned16(dq_acc) || !aligned16(dk_acc) || !aligned16(dv_acc) ||
      !aligned16(workspace))
    return RA_ERR_INVALID;
  if ((causal != 0 && causal != 1) || q_offset < 0 || k_offset < 0 || pos_stride < 1)
    return RA_ERR_INVALID;
  rc = check_backward_dims(shape);
  if (rc != RA_OK) return rc;
  if (workspace_bytes < backward_workspace_bytes(*shape)) return RA_ERR_INVALID;
  DeviceInfo dev;
  rc = device_info(&dev);
  if (rc != RA_OK) return rc;
  return launch_backward(q, k, v, nullptr, lse, dout, delta, *shape, 1, q_offset, k_offset,
                         pos_stride, causal, 0, scale, dq_acc, dk_acc, dv_acc, true, workspace,
                         dev, static_cast<cudaStream_t>(stream));
}

int ra_get_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return RA_ERR_CUDA;
  int word = 0;
  if (cudaMemcpyFromSymbol(&word, g_ra_status_word, sizeof(int)) != cudaSuccess)
    return RA_ERR_CUDA;
  if (word != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_ra_status_word, &zero, sizeof(int)) != cudaSuccess)
      return RA_ERR_CUDA;
  }
  return word == 0 ? RA_OK : word;
}

int ra_set_wait_limit_ns(unsigned long long ns) {
  g_wait_ns.store(ns < 1000000ull ? 1000000ull : ns, std::memory_order_relaxed);
  return RA_OK;
}

int ra_check_wait_timeout(unsigned long long limit_ns, void* stream) {
  DeviceInfo dev;
  int rc = device_info(&dev);
  if (rc != RA_OK) return rc;
  dev.ctx.wait_ns = limit_ns < 1000000ull ? 1000000ull : limit_ns;
  return launch_wait_timeout_check(dev.ctx, static_cast<cudaStream_t>(stream));
}

const char* ra_status_string(int status) {
  switch (status) {
    case RA_OK: return "RA_OK";
    case RA_ERR_INVALID: return "RA_ERR_INVALID: invalid argument";
    case RA_ERR_UNSUPPORTED: return "RA_ERR_UNSUPPORTED: shape or dtype not supported";
    case RA_ERR_CUDA: return "RA_ERR_CUDA: CUDA call or kernel launch failed";
    case RA_ERR_TIMEOUT: return "RA_ERR_TIMEOUT: a kernel's bounded wait expired";
    default: return "unknown ra_status";
  }
}

unsigned long long ra_launch_count(void) { return g_launches.load(); }

int ra_shutdown(void) {
  release_host_call_state();
  std::lock_guard<std::mutex> lock(g_dev_mu);
  for (int i = 0; i < kMaxDevices; ++i) g_dev_ready[i] = false;
  return RA_OK;
}

}  // extern "C"
