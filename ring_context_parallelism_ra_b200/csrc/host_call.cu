// ra_ring_forward_host: the fused ring forward on tensors in host memory, one
// call from the host buffers of Q, K, V to the host buffers of O and LSE.
//
// The (batch, KV head) groups are cut into at most kMaxChunks chunks of equal
// size; chunk c's inputs travel host -> device on one copy stream while the
// kernel of chunk c - 1 runs on the caller's stream and chunk c - 2's outputs
// travel device -> host on a second copy stream.  Two buffer sets in the
// caller's device workspace alternate between the chunks.  Every chunk is an
// ordinary ra_ring_forward call on a contiguous run of heads: a group (b, g)
// is query heads g * G .. g * G + G - 1 and KV head g of batch b, and in the
// BHSD layout groups u0 .. u1 - 1 (u = b * Hkv + g) are contiguous in every
// tensor, so a chunk is one pointer offset per tensor.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/ra.h"
#include "launch.h"

namespace ra {

namespace {

constexpr int kMaxChunks = 8;
constexpr long long kMinChunkItems = 1024;  // 256-row work items per chunk
constexpr int kSlots = 2;
constexpr int kMaxHostDevices = 64;

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct HostPlan {
  int per_chunk;  // groups per chunk
  int chunks;
  size_t q_unit, k_unit, v_unit, o_unit, l_unit;  // bytes of one group
  size_t q_off, k_off, v_off, o_off, l_off;       // offsets inside a slot
  size_t slot_bytes;
};

// Chunk size: a divisor of Hkv (chunks inside one batch) or a multiple of Hkv
// dividing B * Hkv (whole batches), so that every chunk is one launch over a
// contiguous run of heads.  The plan takes the most chunks (up to
// kMaxChunks) that still leave every chunk kMinChunkItems work items, and a
// single chunk when no split does.
HostPlan host_plan(const ra_shape& s) {
  HostPlan p{};
  const long long units = static_cast<long long>(s.B) * s.Hkv;
  const int G = s.Hq / s.Hkv;
  const long long items_per_unit = static_cast<long long>(G) * ((s.n_q + 255) / 256);
  long long best = units;  // one chunk
  for (long long c = 1; c <= units; ++c) {
    if (units % c != 0) continue;
    const bool inside = c <= s.Hkv && s.Hkv % c == 0;
    const bool whole = c % s.Hkv == 0;
    if (!inside && !whole) continue;
    const long long n_chunks = units / c;
    if (n_chunks > kMaxChunks || c * items_per_unit < kMinChunkItems) continue;
    best = c;  // ascending c: the first valid one has the most chunks
    break;
  }
  const size_t esz = s.dtype == RA_F32 ? 4 : 2;
  p.per_chunk = static_cast<int>(best);
  p.chunks = static_cast<int>(units / best);
  p.q_unit = static_cast<size_t>(G) * s.n_q * s.d_qk * esz;
  p.k_unit = static_cast<size_t>(s.n_k) * s.d_qk * esz;
  p.v_unit = static_cast<size_t>(s.n_k) * s.d_v * esz;
  p.o_unit = static_cast<size_t>(G) * s.n_q * s.d_v * esz;
  p.l_unit = static_cast<size_t>(G) * s.n_q * 4;
  const size_t c = static_cast<size_t>(best);
  p.q_off = 0;
  p.k_off = align256(p.q_off + c * p.q_unit);
  p.v_off = align256(p.k_off + c * p.k_unit);
  p.o_off = align256(p.v_off + c * p.v_unit);
  p.l_off = align256(p.o_off + c * p.o_unit);
  p.slot_bytes = align256(p.l_off + c * p.l_unit);
  return p;
}

// Copy streams and events of one device, created on first use and kept; the
// mutex serialises the enqueueing of concurrent calls on that device.
struct HostStreams {
  std::mutex mu;
  bool ready = false;
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t start = nullptr;
  cudaEvent_t in_done[kSlots] = {}, comp_done[kSlots] = {}, out_done[kSlots] = {};
};
HostStreams g_hs[kMaxHostDevices];

int host_streams(int dev, HostStreams** out) {
  HostStreams& h = g_hs[dev];
  if (!h.ready) {
    bool ok = cudaStreamCreateWithFlags(&h.in, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&h.out, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&h.start, cudaEventDisableTiming) == cudaSuccess;
    for (int i = 0; ok && i < kSlots; ++i)
      ok = cudaEventCreateWithFlags(&h.in_done[i], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&h.comp_done[i], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&h.out_done[i], cudaEventDisableTiming) == cudaSuccess;
    if (!ok) return RA_ERR_CUDA;
    h.ready = true;
  }
  *out = &h;
  return RA_OK;
}

}  // namespace

void release_host_call_state() {
  for (int d = 0; d < kMaxHostDevices; ++d) {
    HostStreams& h = g_hs[d];
    std::lock_guard<std::mutex> lock(h.mu);
    if (!h.ready) continue;
    int cur = 0;
    cudaGetDevice(&cur);
    cudaSetDevice(d);
    cudaStreamDestroy(h.in);
    cudaStreamDestroy(h.out);
    cudaEventDestroy(h.start);
    for (int i = 0; i < kSlots; ++i) {
      cudaEventDestroy(h.in_done[i]);
      cudaEventDestroy(h.comp_done[i]);
      cudaEventDestroy(h.out_done[i]);
    }
    cudaSetDevice(cur);
    h.ready = false;
  }
}

}  // namespace ra

using namespace ra;

extern "C" {

size_t ra_ring_forward_host_workspace_bytes(const ra_shape* shape) {
  if (shape == nullptr || shape->B <= 0 || shape->Hq <= 0 || shape->Hkv <= 0 ||
      shape->n_q <= 0 || shape->n_k <= 0 || shape->d_qk <= 0 || shape->d_v <= 0 ||
      shape->Hq % shape->Hkv != 0 || (shape->dtype != RA_F32 && shape->dtype != RA_BF16))
    return 0;
  return kSlots * host_plan(*shape).slot_bytes;
}

int ra_ring_forward_host(const void* q, const void* k, const void* v, int P, int causal,
                         float scale, void* out, float* lse, const ra_shape* shape,
                         void* workspace, size_t workspace_bytes, void* stream) {
  if (shape == nullptr || !q || !k || !v || !out || !workspace) return RA_ERR_INVALID;
  const size_t need = ra_ring_forward_host_workspace_bytes(shape);
  if (need == 0) return RA_ERR_INVALID;
  if (workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return RA_ERR_INVALID;
  if (P < 1 || shape->n_q != shape->n_k || shape->n_q % P != 0 || (causal != 0 && causal != 1))
    return RA_ERR_INVALID;
  if (shape->dtype == RA_F32) {
    if (!((shape->d_qk == 64 || shape->d_qk == 128) && (shape->d_v == 64 || shape->d_v == 128)))
      return RA_ERR_UNSUPPORTED;
  } else if (!((shape->d_qk == 64 || shape->d_qk == 128 || shape->d_qk == 192) &&
               (shape->d_v == 64 || shape->d_v == 128))) {
    return RA_ERR_UNSUPPORTED;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxHostDevices) return RA_ERR_CUDA;
  const HostPlan p = host_plan(*shape);
  HostStreams* hs = nullptr;
  std::lock_guard<std::mutex> lock(g_hs[dev].mu);
  int rc = host_streams(dev, &hs);
  if (rc != RA_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const uint8_t* hq = static_cast<const uint8_t*>(q);
  const uint8_t* hk = static_cast<const uint8_t*>(k);
  const uint8_t* hv = static_cast<const uint8_t*>(v);
  uint8_t* ho = static_cast<uint8_t*>(out);
  uint8_t* hl = reinterpret_cast<uint8_t*>(lse);
  const int G = shape->Hq / shape->Hkv;
  const size_t c = static_cast<size_t>(p.per_chunk);
  ra_shape cs = *shape;  // one chunk's shape
  if (p.per_chunk <= shape->Hkv) {
    cs.B = 1;
    cs.Hkv = p.per_chunk;
    cs.Hq = p.per_chunk * G;
  } else {
    cs.B = p.per_chunk / shape->Hkv;
  }
  // everything below is ordered after the work already on the caller's stream
  if (cudaEventRecord(hs->start, st) != cudaSuccess ||
      cudaStreamWaitEvent(hs->in, hs->start, 0) != cudaSuccess ||
      cudaStreamWaitEvent(hs->out, hs->start, 0) != cudaSuccess)
    return RA_ERR_CUDA;
  bool used[kSlots] = {false, false};
  for (int ci = 0; ci < p.chunks; ++ci) {
    const int sl = ci % kSlots;
    uint8_t* base = ws + sl * p.slot_bytes;
    const size_t u0 = static_cast<size_t>(ci) * c;
    // inputs in, once the slot's previous kernel has read them
    if (used[sl] && cudaStreamWaitEvent(hs->in, hs->comp_done[sl], 0) != cudaSuccess)
      return RA_ERR_CUDA;
    if (cudaMemcpyAsync(base + p.q_off, hq + u0 * p.q_unit, c * p.q_unit, cudaMemcpyHostToDevice,
                        hs->in) != cudaSuccess ||
        cudaMemcpyAsync(base + p.k_off, hk + u0 * p.k_unit, c * p.k_unit, cudaMemcpyHostToDevice,
                        hs->in) != cudaSuccess ||
        cudaMemcpyAsync(base + p.v_off, hv + u0 * p.v_unit, c * p.v_unit, cudaMemcpyHostToDevice,
                        hs->in) != cudaSuccess ||
        cudaEventRecord(hs->in_done[sl], hs->in) != cudaSuccess)
      return RA_ERR_CUDA;
    // the kernel, once the inputs are in and the slot's previous outputs out
    if (cudaStreamWaitEvent(st, hs->in_done[sl], 0) != cudaSuccess) return RA_ERR_CUDA;
    if (used[sl] && cudaStreamWaitEvent(st, hs->out_done[sl], 0) != cudaSuccess)
      return RA_ERR_CUDA;
    rc = ra_ring_forward(base + p.q_off, base + p.k_off, base + p.v_off, P, causal, scale,
                         base + p.o_off, hl ? reinterpret_cast<float*>(base + p.l_off) : nullptr,
                         &cs, st);
    if (rc != RA_OK) return rc;
    if (cudaEventRecord(hs->comp_done[sl], st) != cudaSuccess) return RA_ERR_CUDA;
    // outputs back
    if (cudaStreamWaitEvent(hs->out, hs->comp_done[sl], 0) != cudaSuccess ||
        cudaMemcpyAsync(ho + u0 * p.o_unit, base + p.o_off, c * p.o_unit, cudaMemcpyDeviceToHost,
                        hs->out) != cudaSuccess)
      return RA_ERR_CUDA;
    if (hl && cudaMemcpyAsync(hl + u0 * p.l_unit, base + p.l_off, c * p.l_unit,
                              cudaMemcpyDeviceToHost, hs->out) != cudaSuccess)
      return RA_ERR_CUDA;
    if (cudaEventRecord(hs->out_done[sl], hs->out) != cudaSuccess) return RA_ERR_CUDA;
    used[sl] = true;
  }
  // the caller's stream completes only after every output is in host memory
  for (int sl = 0; sl < kSlots; ++sl)
    if (used[sl] && cudaStreamWaitEvent(st, hs->out_done[sl], 0) != cudaSuccess)
      return RA_ERR_CUDA;
  return RA_OK;
}

}  // extern "C"
