/*
 * ra.h -- C ABI of the Ring Attention hot path on one B200 (sm_100a).
 *
 * What is computed (pages cited by title and section / equation):
 *   O = softmax(scale * Q K^T + mask) V, exactly, per (batch, query head),
 *   page "长上下文的第一性挑战", Eq. (lc-ch-attention).  The sequence is split
 *   into P contiguous partitions; query partition i stays in place while the
 *   KV partitions pass it in ring order (i, i-1, ..., i-P+1 mod P), page
 *   "AI 推理系列（十一）：Ring Attention 如何让多张 GPU 共同计算一条超长序列",
 *   section "KV 在 Ring 中如何流动".  Each (Q_i, KV_j) block is folded into a
 *   running row max / exponential sum / rescaled output, never materialising
 *   the n x n score matrix (same page, section "最容易被忽略的细节"), and blocks
 *   wholly in the causal future are skipped.
 *
 * Conventions shared by every entry point
 *   - Tensors are dense, row-major BHSD in device memory owned by the caller:
 *       q    [B, Hq,  n_q, d_qk]     k [B, Hkv, n_k, d_qk]    v [B, Hkv, n_k, d_v]
 *       out  [B, Hq,  n_q, d_v]      lse [B, Hq, n_q] (fp32, natural log,
 *       scale included).  Grouped-query heads: query head h reads KV head
 *       h / (Hq / Hkv).
 *   - Causal rule: key at absolute position k_offset + u is visible to the
 *     query at q_offset + t iff k_offset + u <= q_offset + t.
 *   - Pointers must be 16-byte aligned.  The library allocates no device
 *     memory per call; what it caches (TMA descriptors, a status word) is
 *     created on first use and released by ra_shutdown().  The persistent
 *     attention kernels take their work items from a counter: the forward
 *     uses one slot of a module-global ring of 1024 counters per call and
 *     zeroes it with a 4-byte cudaMemsetAsync on `stream` before the kernel
 *     (calls running at the same time on different streams get different
 *     slots while fewer than 1024 are in flight); the backward keeps its
 *     counter in the caller's workspace.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Every
 *     compute entry point only enqueues work and returns; it never
 *     synchronises.  Results are ready when the stream reaches them.
 *   - Return value: RA_OK or a negative ra_status.  Argument errors are found
 *     on the host before anything is enqueued.  A device-side bounded wait
 *     that expires cannot be returned by the launching call; it is recorded in
 *     a per-device status word that ra_get_status() reads.
 *   - Thread safety: calls may come from several host threads; the only
 *     shared state (descriptor cache, status word) is guarded internally.
 */
#ifndef RA_H_
#define RA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  RA_OK = 0,
  RA_ERR_INVALID = -1,      /* null / misaligned pointer, inconsistent shape   */
  RA_ERR_UNSUPPORTED = -2,  /* valid request this build does not implement     */
  RA_ERR_CUDA = -3,         /* a CUDA runtime call or kernel launch failed     */
  RA_ERR_TIMEOUT = -4       /* a kernel's bounded wait expired (ra_get_status) */
} ra_status;

typedef enum { RA_F32 = 0, RA_BF16 = 1 } ra_dtype;

typedef struct {
  int B;          /* batch                                                */
  int Hq;         /* query heads                                          */
  int Hkv;        /* KV heads; Hq % Hkv == 0                              */
  int n_q;        /* query tokens per sequence                            */
  int n_k;        /* key / value tokens per sequence (or per shard)       */
  int d_qk;       /* head dim of Q and K                                  */
  int d_v;        /* head dim of V and O                                  */
  ra_dtype dtype; /* element type of q, k, v                              */
} ra_shape;

/*
 * Supported head dims: bf16 d_qk in {64, 128, 192}, d_v in {64, 128} (tensor
 * cores, tcgen05); fp32 d_qk, d_v in {64, 128} (exact fp32 FMA).
 */

/*
 * ra_block_partial -- one (Q range, KV range) block: the block partial of one
 * ring step, page "LLM长文本推理Ring Attention环形注意力机制实现与优化", section
 * "Ring Attention实现代码与通信重叠" (each ring step computes the local
 * attention of Q_i against the KV block that has arrived).
 *   q, k, v     : device, BHSD as above (k, v hold the n_k keys of the block).
 *   q_offset,
 *   k_offset    : absolute position of the first query / key (causal mask).
 *   causal      : 0 or 1.
 *   scale       : multiplies Q K^T (normally 1/sqrt(d_qk)).
 *   o_part      : device fp32 [B, Hq, n_q, d_v], normalised over this block's
 *                 visible keys; a row with no visible key gets 0.
 *   lse_part    : device fp32 [B, Hq, n_q]; -inf for a row with no visible key.
 * Errors: RA_ERR_INVALID (null, misaligned, n <= 0, Hq % Hkv), RA_ERR_UNSUPPORTED
 * (head dims), RA_ERR_CUDA (launch).
 */
int ra_block_partial(const void* q, const void* k, const void* v, const ra_shape* shape,
                     int q_offset, int k_offset, int causal, float scale,
                     float* o_part, float* lse_part, void* stream);

/*
 * ra_block_partial_strided -- ra_block_partial with positions spaced by
 * pos_stride: query row t is token q_offset + t * pos_stride and key u is
 * token k_offset + u * pos_stride.  With the striped split of page
 * "LLM长文本推理Ring Attention环形注意力机制实现与优化", section on tuning
 * (Striped Attention interleaves token positions across devices), partition
 * i holds tokens i, i + P, i + 2P, ...: its block against partition j is this
 * call with q_offset = i, k_offset = j, pos_stride = P.  Every such block is
 * about half visible, which balances causal work across the P devices.
 *   pos_stride  : >= 1 (1 gives ra_block_partial).
 *   Other arguments, outputs and errors as ra_block_partial.
 */
int ra_block_partial_strided(const void* q, const void* k, const void* v, const ra_shape* shape,
                             int q_offset, int k_offset, int pos_stride, int causal, float scale,
                             float* o_part, float* lse_part, void* stream);

/*
 * ra_lse_merge -- N-way merge of normalised partials over disjoint key sets,
 * the closed form of the beta / gamma update of page
 * "LLM长文本推理Ring Attention环形注意力机制实现与优化", section
 * "Ring Attention实现代码与通信重叠":
 *   L* = max_p L_p,  w_p = exp(L_p - L*),  LSE = L* + ln sum w_p,
 *   O = sum_p (w_p / sum w) O_p.   All L_p = -inf gives O = 0, LSE = -inf.
 *   o_parts     : device fp32 [P, B, Hq, n_q, d_v] (P stacked partials).
 *   lse_parts   : device fp32 [P, B, Hq, n_q].
 *   shape       : B, Hq, n_q, d_v are read; dtype, Hkv, n_k, d_qk are ignored.
 *   out         : device [B, Hq, n_q, d_v] of out_dtype (RA_F32 or RA_BF16).
 *   lse         : device fp32 [B, Hq, n_q], or NULL to skip.
 * Errors: RA_ERR_INVALID (P < 1, null, misaligned), RA_ERR_CUDA.
 */
int ra_lse_merge(const float* o_parts, const float* lse_parts, int P, const ra_shape* shape,
                 void* out, ra_dtype out_dtype, float* lse, void* stream);

/*
 * ra_ring_forward -- the fused ring: all P partitions of one sequence in one
 * kernel (split, ring schedule, block partials, fold and final normalisation).
 * Query partition i meets KV partitions in ring order
 * j = i, i-1, ..., i-P+1 (mod P); with causal = 1 the blocks j > i are
 * skipped and the diagonal block is masked.  K/V tiles stream through a
 * shared-memory ring filled by TMA while the previous tile's math runs.
 *   q, k, v     : device BHSD, n_q == n_k == n, n % P == 0.
 *   out         : device [B, Hq, n, d_v], same dtype as q.
 *   lse         : device fp32 [B, Hq, n] (may be NULL).
 * Errors: RA_ERR_INVALID (n_q != n_k, n % P, null, misaligned),
 * RA_ERR_UNSUPPORTED (head dims), RA_ERR_CUDA.
 */
int ra_ring_forward(const void* q, const void* k, const void* v, int P, int causal, float scale,
                    void* out, float* lse, const ra_shape* shape, void* stream);

/*
 * ra_ring_forward_striped -- the fused ring over a striped split (same page
 * and section as ra_block_partial_strided): the tensors hold the P
 * partitions one after another, partition i being tokens i, i + P, i + 2P,
 * ... in order, so tensor row R = i * (n / P) + r is token r * P + i.  Output
 * rows are in the same order.  The causal mask follows the token positions;
 * no partition block is skipped whole (each is half visible), tiles are.
 *   Arguments as ra_ring_forward; additionally (n / P) % 256 == 0, else
 *   RA_ERR_UNSUPPORTED.
 */
int ra_ring_forward_striped(const void* q, const void* k, const void* v, int P, int causal,
                            float scale, void* out, float* lse, const ra_shape* shape,
                            void* stream);

/*
 * ra_ring_forward_host_workspace_bytes -- device bytes ra_ring_forward_host
 * needs for `shape` (two chunk buffer sets).  A pure function of the shape;
 * 0 for an invalid shape.
 */
size_t ra_ring_forward_host_workspace_bytes(const ra_shape* shape);

/*
 * ra_ring_forward_host -- ra_ring_forward (the same fused ring, the same
 * result) on tensors in HOST memory: the inputs are copied in, the ring runs,
 * O and LSE are copied out, all enqueued by this one call.  The (batch, KV
 * head) groups are processed in up to 8 equal chunks of whole groups (a
 * chunk keeps at least 1024 work items of 256 query rows, else the call uses
 * fewer chunks, down to one): chunk c's host-to-device copies run on an
 * internal copy stream while chunk c-1's kernel runs on `stream` and chunk
 * c-2's results return on a second internal copy stream, through two buffer
 * sets that alternate in `workspace`.
 *   q, k, v     : host BHSD as ra_ring_forward (n_q == n_k, n % P == 0).
 *                 Page-locked (pinned) memory lets the copies overlap the
 *                 kernels; pageable memory works, but each copy then holds
 *                 the calling thread until it is done.
 *   out         : host [B, Hq, n, d_v], same dtype as q.
 *   lse         : host fp32 [B, Hq, n], or NULL to skip.
 *   workspace   : device, 256-byte aligned, at least
 *                 ra_ring_forward_host_workspace_bytes(shape) bytes, owned
 *                 by the caller and not used by other work until `stream`
 *                 has passed this call.
 *   stream      : the kernels run on it; the copies start after the work
 *                 already on it, and work enqueued on it later starts only
 *                 after every output byte is in host memory.  The call
 *                 returns after enqueueing: synchronise `stream` before
 *                 reading out / lse or writing q, k, v.
 * The copy streams and their events are created once per device on first
 * use (released by ra_shutdown); concurrent calls on one device are
 * enqueued one after another.  No device memory is allocated.
 * Errors: RA_ERR_INVALID (null, shape, workspace too small or misaligned),
 * RA_ERR_UNSUPPORTED (head dims), RA_ERR_CUDA (a copy, event or launch
 * failed; work enqueued before the failure still runs).
 */
int ra_ring_forward_host(const void* q, const void* k, const void* v, int P, int causal,
                         float scale, void* out, float* lse, const ra_shape* shape,
                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * ra_decode_workspace_bytes -- bytes of device workspace ra_decode_partial
 * needs for `shape` (its split-KV chunk partials).  0 on invalid shape.
 */
size_t ra_decode_workspace_bytes(const ra_shape* shape);

/*
 * ra_decode_partial -- pass-Q decode on one KV shard, page
 * "上下文并行 (CP) 收益评估实验设计", decode section: the query is sent to every
 * shard, each shard computes partial attention over its S/cp tokens, and the
 * partials are reduced (ra_decode_merge).  One query token per sequence sees
 * every token of the shard (no mask).
 *   q           : device bf16 [B, Hq, 1, d_qk].
 *   k_shard,
 *   v_shard     : device bf16; head (b, g) of the shard starts at
 *                 ptr + (b * Hkv + g) * kv_head_stride * d elements and holds
 *                 n_k consecutive tokens (kv_head_stride = n_k for a dense
 *                 shard, = the full cache length for a shard that is a token
 *                 range of a larger [B, Hkv, S, d] cache).
 *   shape       : n_q must be 1; n_k = shard length; d_qk == d_v == 128.
 *   o_part      : device fp32 [B, Hq, d_v] normalised over the shard.
 *   lse_part    : device fp32 [B, Hq].
 *   workspace   : device, >= ra_decode_workspace_bytes(shape), 16-B aligned,
 *                 owned by the caller; contents on entry are ignored.
 * Errors: RA_ERR_INVALID, RA_ERR_UNSUPPORTED (dims, dtype), RA_ERR_CUDA.
 */
int ra_decode_partial(const void* q, const void* k_shard, const void* v_shard,
                      long long kv_head_stride, const ra_shape* shape, float scale,
                      float* o_part, float* lse_part, void* workspace, size_t workspace_bytes,
                      void* stream);

/*
 * ra_decode_partials -- the P shard partials of pass-Q decode (page "上下文并行
 * (CP) 收益评估实验设计", decode section: each chip attends over its S/cp
 * tokens) at once, for a cache that one device holds whole: the same
 * partials as P calls of
 * ra_decode_partial (one per token range of n_k / P tokens), computed by one
 * launch over every chunk of every shard and one merge of each shard's
 * chunks.  With short shards the P separate launches leave SMs idle; this
 * call keeps them busy.  ra_decode_merge then combines the partials.
 *   q           : device bf16 [B, Hq, 1, d_qk].
 *   k, v        : device bf16 [B, Hkv, n_k, d] (the whole cache, dense).
 *   P           : shards; n_k % P == 0, and (n_k / P) % 2048 == 0 when P > 1
 *                 (whole 2048-token chunks per shard), else RA_ERR_UNSUPPORTED.
 *   shape       : n_q must be 1; n_k = the whole cache; d_qk == d_v == 128.
 *   o_parts     : device fp32 [P, B, Hq, d_v], each normalised over its shard.
 *   lse_parts   : device fp32 [P, B, Hq].
 *   workspace   : device, >= ra_decode_workspace_bytes(shape) with n_k the
 *                 whole cache, 16-B aligned, caller-owned.
 * Errors: RA_ERR_INVALID, RA_ERR_UNSUPPORTED (dims, dtype, shard length),
 * RA_ERR_CUDA.
 */
int ra_decode_partials(const void* q, const void* k, const void* v, int P, const ra_shape* shape,
                       float scale, float* o_parts, float* lse_parts, void* workspace,
                       size_t workspace_bytes, void* stream);

/*
 * ra_decode_partial_noalloc -- ra_decode_partial without a caller workspace.
 * The pages have no counterpart of this call; it exists for callers that
 * cannot allocate device memory: a plugin inside a host runtime that owns all
 * device memory and gives its plugins no allocator, or a latency-critical
 * loop that must not call cudaMalloc (which may synchronise the device).
 * The chunk partials live in one file-scope device array of 16 MiB, held on
 * every GPU that loads the library until the process exits.  The call itself
 * allocates nothing and calls no allocating routine.  The CUDA runtime
 * commits the array's device memory when it loads the library's module on a
 * device: at library load under eager module loading, or under lazy loading
 * (the CUDA 12 default) at the first decode call on that device.  That first
 * call can therefore fail with RA_ERR_CUDA when the device is out of memory;
 * make one warm-up call at initialisation, outside any stream capture.
 *   Arguments, layout and results as ra_decode_partial, minus the workspace.
 *   Limit: ceil(n_k / 2048) * B * Hq * (d_v + 1) * 4 + 256 bytes must not
 *   exceed 16 MiB (e.g. a 131072-token shard with B * Hq = 256 needs 8.5 MB);
 *   larger shapes return RA_ERR_UNSUPPORTED before anything is enqueued.
 *   The first call on a device looks up the array's device address (with
 *   that device current) and caches it; make that first call before any
 *   stream capture.  All calls share the array and it keeps the last call's
 *   contents; calls whose kernels overlap on the GPU (e.g. on two unordered
 *   streams) race on it, so order them on one stream.  The cached address
 *   belongs to the device's primary context: do not call the library again
 *   after cudaDeviceReset (or after the primary context was destroyed).
 * Errors: as ra_decode_partial.
 */
int ra_decode_partial_noalloc(const void* q, const void* k_shard, const void* v_shard,
                              long long kv_head_stride, const ra_shape* shape, float scale,
                              float* o_part, float* lse_part, void* stream);

/*
 * ra_decode_merge -- reduce the P shard partials of pass-Q decode;
 * the merge of ra_lse_merge with n_q = 1.
 *   o_parts     : device fp32 [P, B, Hq, d_v];  lse_parts: [P, B, Hq].
 *   out         : device [B, Hq, d_v] of out_dtype;  lse: fp32 [B, Hq] or NULL.
 */
int ra_decode_merge(const float* o_parts, const float* lse_parts, int P, const ra_shape* shape,
                    void* out, ra_dtype out_dtype, float* lse, void* stream);

/*
 * Backward pass.  The pages name it (page "AI 推理系列（十一）：Ring Attention
 * 如何让多张 GPU 共同计算一条超长序列": training keeps what the backward pass
 * needs, and its data dependencies across blocks are a place to look when
 * results go wrong) but give no algorithm; the gradients below are the chain
 * rule of the forward definition (page "长上下文的第一性挑战", Eq.
 * (lc-ch-attention)) for a loss that depends on O through dO:
 *   P = exp(scale Q K^T - LSE) on visible pairs (the forward's final LSE),
 *   dV = P^T dO,  dP = dO V^T,  D = rowsum(dO * O),  dS = P (dP - D),
 *   dQ = scale dS K,  dK = scale dS^T Q,
 * with dK, dV of a KV head summed over the query heads of its group.  In the
 * ring, KV_j travels with its accumulators dK_j, dV_j and collects one share
 * per query partition while dQ_i collects at its partition.
 * Supported head dims: d_qk, d_v in {64, 128} (bf16 on tensor cores, fp32
 * on the CUDA cores); bf16 d_qk = 192 with d_v in {64, 128} (the MLA-shaped
 * head) on tensor cores as well, its products taking turns in tensor memory
 * (the 192-column dK accumulator leaves no room to keep S^T and dP^T apart).
 */

/*
 * ra_backward_workspace_bytes -- device workspace the backward calls need for
 * `shape` (an fp32 dQ accumulator and two row vectors, padded to 128 rows
 * per head, and the counter the tensor-core kernels hand out work items
 * from): about B * Hq * n_q * (d_qk + 2) * 4 bytes.  0 on invalid shape.
 */
size_t ra_backward_workspace_bytes(const ra_shape* shape);

/*
 * ra_backward_delta -- D = rowsum(dO * O) per query row.
 *   out, dout   : device [B, Hq, n_q, d_v] of shape->dtype (O of the forward
 *                 and the gradient arriving at it).
 *   delta       : device fp32 [B, Hq, n_q].
 * Errors: RA_ERR_INVALID, RA_ERR_UNSUPPORTED (d_v other than 64, 128), RA_ERR_CUDA.
 */
int ra_backward_delta(const void* out, const void* dout, const ra_shape* shape, float* delta,
                      void* stream);

/*
 * ra_ring_backward -- gradients of ra_ring_forward for all P partitions of
 * one sequence: dQ, dK, dV of q, k, v.  Each key tile of KV_j meets the query
 * partitions in ring order j, j+1, ... (mod P), fully masked tiles skipped;
 * its dK, dV stay on chip for the whole walk.
 *   q, k, v     : as ra_ring_forward (n_q == n_k == n, n % P == 0).
 *   out, lse    : the forward's outputs for these inputs ([B, Hq, n, d_v] of
 *                 the input dtype; fp32 [B, Hq, n]).
 *   dout        : device [B, Hq, n, d_v], input dtype.
 *   dq, dk, dv  : device outputs of the input dtype, shaped like q, k, v.
 *   workspace   : device, >= ra_backward_workspace_bytes(shape), 16-B
 *                 aligned, owned by the caller; contents on entry ignored.
 * Errors: RA_ERR_INVALID (shapes, null, misaligned, workspace too small),
 * RA_ERR_UNSUPPORTED (head dims), RA_ERR_CUDA.  bf16 runs on the tensor
 * cores; fp32 in exact fp32 arithmetic.
 */
int ra_ring_backward(const void* q, const void* k, const void* v, const void* out,
                     const float* lse, const void* dout, int P, int causal, float scale, void* dq,
                     void* dk, void* dv, const ra_shape* shape, void* workspace,
                     size_t workspace_bytes, void* stream);

/*
 * ra_ring_backward_striped -- the same over the striped split of
 * ra_ring_forward_striped (tensor row R = i * (n / P) + r is token r * P + i;
 * gradients in the same row order).  Needs (n / P) % 128 == 0, else
 * RA_ERR_UNSUPPORTED.
 */
int ra_ring_backward_striped(const void* q, const void* k, const void* v, const void* out,
                             const float* lse, const void* dout, int P, int causal, float scale,
                             void* dq, void* dk, void* dv, const ra_shape* shape, void* workspace,
                             size_t workspace_bytes, void* stream);

/*
 * ra_block_backward -- one (Q range, KV range) block's share of the
 * gradients, added into fp32 accumulators: the step a device of the ring
 * takes when KV_j (with dK_j, dV_j) reaches Q_i.  P is formed against the
 * FINAL row statistics, so shares of different blocks simply add up.
 *   q, k, v, dout : device, shapes as ra_block_partial (dout [B, Hq, n_q, d_v]).
 *   lse           : device fp32 [B, Hq, n_q], the forward's final LSE of
 *                   these rows (over all keys, not just this block).
 *   delta         : device fp32 [B, Hq, n_q], from ra_backward_delta.
 *   q_offset, k_offset, pos_stride, causal : positions as
 *                   ra_block_partial_strided.
 *   dq_acc        : device fp32 [B, Hq, n_q, d_qk], += this block's dQ share.
 *   dk_acc, dv_acc: device fp32 [B, Hkv, n_k, d_qk / d_v], += shares.
 *   workspace     : as ra_ring_backward.
 * Errors: as ra_ring_backward.
 */
int ra_block_backward(const void* q, const void* k, const void* v, const void* dout,
                      const float* lse, const float* delta, const ra_shape* shape, int q_offset,
                      int k_offset, int pos_stride, int causal, float scale, float* dq_acc,
                      float* dk_acc, float* dv_acc, void* workspace, size_t workspace_bytes,
                      void* stream);

/*
 * ra_block_class -- causal class of every (query block, key block) pair,
 * host side: 0 = SKIP (no visible pair), 1 = PARTIAL, 2 = FULL (every pair
 * visible).  Blocks at the ragged end cover only existing rows / keys.  With
 * causal = 0 every block is FULL.  This is the rule the kernels apply to their
 * tiles (page "AI 推理系列（十一）…", section "KV 在 Ring 中如何流动": fully
 * masked blocks may be skipped, the causal semantics must not change).
 *   map_host    : host int8 [ceil(n_q/q_block), ceil(n_k/k_block)], row-major.
 * Errors: RA_ERR_INVALID (null, non-positive sizes).
 */
int ra_block_class(int n_q, int n_k, int q_block, int k_block, int q_offset, int k_offset,
                   int causal, int8_t* map_host);

/*
 * ra_block_class_device -- the same map computed by a kernel with the device
 * copy of the rule the attention kernels use; map_dev is device memory.
 */
int ra_block_class_device(int n_q, int n_k, int q_block, int k_block, int q_offset,
                          int k_offset, int causal, int8_t* map_dev, void* stream);

/*
 * ra_get_status -- synchronise `stream`, then read and clear the current
 * device's status word.  Returns RA_OK, or RA_ERR_TIMEOUT if a kernel's
 * bounded wait expired since the last call (its results are then invalid),
 * or RA_ERR_CUDA if the synchronisation itself failed or a kernel could not
 * align its shared-memory tiles and returned without computing.
 */
int ra_get_status(void* stream);

/*
 * ra_set_wait_limit_ns -- bound, in nanoseconds, on every device-side wait of
 * later launches (default 2e9).  Values below 1e6 are raised to 1e6.
 */
int ra_set_wait_limit_ns(unsigned long long ns);

/*
 * ra_check_wait_timeout -- launch one block whose wait nobody satisfies, so
 * that its bounded wait runs out after `limit_ns`; the kernel records
 * RA_ERR_TIMEOUT in the status word and returns normally.  Used to test the
 * timeout path without faulting or hanging the GPU.
 */
int ra_check_wait_timeout(unsigned long long limit_ns, void* stream);

/* Human-readable name of a status code. */
const char* ra_status_string(int status);

/* Number of kernel launches this library has enqueued since load. */
unsigned long long ra_launch_count(void);

/* Release cached descriptors and the copy streams / events of
 * ra_ring_forward_host.  Safe to call more than once. */
int ra_shutdown(void);

#ifdef __cplusplus
}
#endif

#endif /* RA_H_ */
