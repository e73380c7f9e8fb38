// Host-side launchers of the kernels, called by the C ABI in ra_api.cu after
// argument validation.  Each returns an ra_status.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/ra.h"
#include "common.cuh"

namespace ra {

// Counts kernel launches enqueued by this library (ra_launch_count).
void note_launch();

// Releases the copy streams and events of ra_ring_forward_host (ra_shutdown).
void release_host_call_state();

// Per-device state: SM count, status word address, wait bound, and the
// ring of work-item counters the forward launches take slots of.
constexpr int kItemCounterSlots = 1024;
struct DeviceInfo {
  int device;
  int num_sms;
  int max_smem_optin;
  unsigned int* item_counters;  // [kItemCounterSlots] device memory (module global)
  DevCtx ctx;
};
// The next slot of the device's counter ring, zeroed on `stream`.
int next_item_counter(const DeviceInfo& dev, cudaStream_t stream, unsigned int** out);
int device_info(DeviceInfo* out);

int launch_lse_merge(const float* o_parts, const float* lse_parts, int P, long long rows, int d_v,
                     void* out, ra_dtype out_dtype, float* lse, int num_sms, cudaStream_t stream);

// Attention launchers.  Positions: query row t is token q_offset + t * stride
// and key u is token k_offset + u * stride (block partial: P = 1); with
// striped = 1 (fused ring) row r of partition i is token r * P + i and the
// offsets / stride arguments are ignored.  out_f32 selects fp32 output.
// Exact-fp32 (SIMT) attention for fp32 inputs:
int launch_simt_attention(const void* q, const void* k, const void* v, const ra_shape& s, int P,
                          int q_offset, int k_offset, long long stride, int causal, int striped,
                          float scale, void* out, bool out_f32, float* lse,
                          const DeviceInfo& dev, cudaStream_t stream);

// Tensor-core (tcgen05) attention, bf16 inputs.
int launch_tc_attention(const void* q, const void* k, const void* v, const ra_shape& s, int P,
                        int q_offset, int k_offset, long long stride, int causal, int striped,
                        float scale, void* out, bool out_f32, float* lse, const DeviceInfo& dev,
                        cudaStream_t stream);

// Decode: chunk partials of one shard into the workspace, then the merge.
size_t decode_workspace_bytes(const ra_shape& s);
int launch_decode_partial(const void* q, const void* k, const void* v, long long kv_head_stride,
                          const ra_shape& s, float scale, float* o_part, float* lse_part,
                          float* workspace, const DeviceInfo& dev, cudaStream_t stream, int shards = 1);

// Same without a caller workspace: the chunk partials go to a file-scope
// device array of decode_static_scratch_bytes() bytes.
size_t decode_static_scratch_bytes();
int launch_decode_partial_static(const void* q, const void* k, const void* v,
                                 long long kv_head_stride, const ra_shape& s, float scale,
                                 float* o_part, float* lse_part, const DeviceInfo& dev,
                                 cudaStream_t stream);

// Backward pass (bwd_attention.cu, bwd_simt.cu).  Ring mode (block_mode
// false): dq, dk, dv are outputs of the input dtype and D is computed from
// out / dout.  Block mode: dq, dk, dv are fp32 accumulators (+=) and D comes
// from `delta`.  `workspace` holds at least backward_workspace_bytes(s).
size_t backward_workspace_bytes(const ra_shape& s);
int launch_backward(const void* q, const void* k, const void* v, const void* out,
                    const float* lse, const void* dout, const float* delta, const ra_shape& s,
                    int P, int q_offset, int k_offset, long long stride, int causal, int striped,
                    float scale, void* dq, void* dk, void* dv, bool block_mode, void* workspace,
                    const DeviceInfo& dev, cudaStream_t stream);
int launch_backward_delta(const void* out, const void* dout, const ra_shape& s, float* delta,
                          const DeviceInfo& dev, cudaStream_t stream);
struct BwdArgs;
struct BwdLayout;
// Row statistics, zeroed dQ accumulator and item counter; dQ accumulator ->
// output.
int launch_backward_rows(const void* out, const void* dout, const float* delta, const float* lse,
                         const ra_shape& s, const BwdLayout& L, float* nl2, float* d_ws,
                         float* dq_ws, unsigned int* counter, const DeviceInfo& dev,
                         cudaStream_t stream);
int launch_dq_finalize(const float* ws_dq, void* dq, const ra_shape& s, const BwdLayout& L,
                       float scale, bool block_mode, cudaStream_t stream);
int launch_simt_backward(const void* q, const void* k, const void* v, const void* dout,
                         const ra_shape& s, BwdArgs a, const DeviceInfo& dev,
                         cudaStream_t stream);
// Gradient kernel of bf16 inputs with d_qk = 192 (bwd_tc192.cu); tensor maps
// of q, k, v, dout as launch_backward builds them.
int launch_bwd_tc192(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                     const CUtensorMap& tdo, const BwdArgs& args, int d_v, int grid,
                     cudaStream_t stream);

int launch_block_class(int n_q, int n_k, int q_block, int k_block, int q_offset, int k_offset,
                       int causal, int8_t* map_dev, cudaStream_t stream);

int launch_wait_timeout_check(const DevCtx& ctx, cudaStream_t stream);

}  // namespace ra
