// Pass-Q decode on one KV shard (page "上下文并行 (CP) 收益评估实验设计", decode
// section: the query goes to every shard, each shard computes partial attention
// over its tokens, the partials are reduced).  One query token per sequence,
// no mask.
//
// Roofline: one decode step reads the whole cache once (page "长上下文的第一性
// 挑战", table decode-bw), so the kernel is HBM-bound and its job is to keep
// enough bytes in flight.  Arithmetic would still hit the fp32 ALU roof on
// CUDA cores (two FLOPs per byte per query head of the GQA group), so QK^T and
// PV run as bf16 mma.sync with the group's query heads as the M = 16 rows.
//
// Structure: a persistent grid; work unit = (sequence, KV head, 2048-token
// chunk).  Warp 4 is the TMA producer: 64-token K and V tiles (128-byte
// swizzled boxes) go into a 5-stage shared-memory ring guarded by mbarriers.
// Warps 0-3 each take 16 tokens of every stage, fold them into their own
// running max / exp-sum / rescaled output (base 2), and at the end of a
// chunk the four states are merged through shared memory into one normalised
// chunk partial (O_c, LSE_c) in the caller's workspace.  A second kernel (the
// LSE merge) reduces the chunk partials to the shard partial.
#include <cuda.h>

#include <mutex>

#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"
#include "tmap.h"

namespace ra {

namespace {

constexpr int kD = 128;
constexpr int kTok = 64;                       // tokens per stage
constexpr int kStages = 5;
constexpr int kChunk = 2048;                   // tokens per chunk partial
constexpr int kConsumers = 4;                  // warps, 16 tokens each per stage
constexpr int kThreads = (kConsumers + 1) * 32;
constexpr int kBoxBytes = kTok * 64 * 2;       // 64 tokens x 64 dims bf16 = 8 KB
constexpr int kStageBytes = 4 * kBoxBytes;     // K (2 boxes) + V (2 boxes)
constexpr int kCombineBytes = kConsumers * 16 * kD * 4;   // per-warp O, 16 rows
constexpr int kMLBytes = kConsumers * 16 * 2 * 4;
constexpr size_t kSmemBytes = 1024 /*align slack*/ + kStages * kStageBytes + kCombineBytes +
                              kMLBytes + 2 * kStages * 8 + 16;

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Byte offset of the 16-byte chunk holding (row, dims [8*c16, 8*c16+8)) inside
// a 64-dim box written by TMA with the 128-byte swizzle.
__device__ __forceinline__ uint32_t sw128_off(int row, int c16) {
  return static_cast<uint32_t>(row * 128 + ((c16 ^ (row & 7)) << 4));
}

struct DecodeArgs {
  const __nv_bfloat16* q;
  int B, Hq, Hkv, G, n_k;
  int n_chunks;
  int shards;     // the cache is this many equal shards of whole chunks
  float scale_log2;
  // Chunk ch is chunk c = ch % (n_chunks / shards) of shard p = ch / (n_chunks
  // / shards); its partial is row (c * shards + p) * B*Hq + (b*Hq + h), so the
  // chunks of one position c across all shards are consecutive and one LSE
  // merge over the n_chunks / shards positions leaves the shards' partials
  // stacked [shards][B*Hq].  shards = 1: row ch * B*Hq + (b*Hq + h).
  float* ws_o;    // [n_chunks][B*Hq][kD]
  float* ws_lse;  // [n_chunks][B*Hq]
  DevCtx ctx;
};

__global__ void __launch_bounds__(kThreads, 1) decode_chunk_kernel(
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
    DecodeArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* stages = smem;
  float* comb_o = reinterpret_cast<float*>(smem + kStages * kStageBytes);
  float* comb_ml = comb_o + kConsumers * 16 * kD;
  uint64_t* full = reinterpret_cast<uint64_t*>(comb_ml + kConsumers * 16 * 2);
  uint64_t* empty = full + kStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kStages);
  volatile int* issued = abort_flag + 1;   // loads issued by the producer

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumers);
    }
    *abort_flag = 0;
    *issued = 0;
    fence_mbar_init();
  }
  __syncthreads();

  const int units = a.B * a.Hkv * a.n_chunks;

  if (warp == kConsumers) {
    // ------------------------------------------------ TMA producer warp --
    if (lane == 0) {
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      uint32_t it = 0;
      for (int u = blockIdx.x; u < units && !*abort_flag; u += gridDim.x) {
        const int bh = u / a.n_chunks;
        const int ch = u % a.n_chunks;
        const int t_end = min(a.n_k, (ch + 1) * kChunk);
        for (int t0 = ch * kChunk; t0 < t_end; t0 += kTok, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1;
          if (!mbar_wait(&empty[s], ph ^ 1, a.ctx, abort_flag)) break;
          mbar_arrive_expect_tx(&full[s], kStageBytes);
          uint8_t* st = stages + s * kStageBytes;
          tma_load_3d(st, &tm_k, &full[s], 0, t0, bh);
          tma_load_3d(st + kBoxBytes, &tm_k, &full[s], 64, t0, bh);
          tma_load_3d(st + 2 * kBoxBytes, &tm_v, &full[s], 0, t0, bh);
          tma_load_3d(st + 3 * kBoxBytes, &tm_v, &full[s], 64, t0, bh);
          *issued = static_cast<int>(it + 1);
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ consumer warps 0-3 --
    const int grp = lane >> 2;   // row (query head) of the mma fragments
    const int tig = lane & 3;
    uint32_t it = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
      const int bh = u / a.n_chunks;
      const int ch = u % a.n_chunks;
      const int b = bh / a.Hkv;
      const int g = bh % a.Hkv;
      const int t_beg = ch * kChunk;
      const int t_end = min(a.n_k, t_beg + kChunk);

      // Query fragments (A operand, rows = the group's query heads, zero
      // beyond G): a0/a2 rows grp, a1/a3 rows grp + 8; dims 16ks + 2tig (+8).
      uint32_t qa[8][4];
      const __nv_bfloat16* qb = a.q + (static_cast<long long>(b) * a.Hq + g * a.G) * kD;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const int c0 = ks * 16 + 2 * tig;
        qa[ks][0] = grp < a.G ? *reinterpret_cast<const uint32_t*>(qb + grp * kD + c0) : 0u;
        qa[ks][1] = grp + 8 < a.G ? *reinterpret_cast<const uint32_t*>(qb + (grp + 8) * kD + c0) : 0u;
        qa[ks][2] = grp < a.G ? *reinterpret_cast<const uint32_t*>(qb + grp * kD + c0 + 8) : 0u;
        qa[ks][3] = grp + 8 < a.G ? *reinterpret_cast<const uint32_t*>(qb + (grp + 8) * kD + c0 + 8) : 0u;
      }

      float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
      float acc[16][4];
#pragma unroll
      for (int n = 0; n < 16; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;

      for (int t0 = t_beg; t0 < t_end; t0 += kTok, ++it) {
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        if (!mbar_wait(&full[s], ph, a.ctx, abort_flag)) break;
        const uint32_t st = smem_u32(stages + s * kStageBytes);
        const int tw = warp * 16;  // this warp's first token in the stage

        // S = Q K^T for 16 tokens: two n-tiles of 8 tokens.
        float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const int mi = lane >> 3;
          const int row = tw + ((mi >> 1) << 3) + (lane & 7);
          const int dchunk = 2 * ks + (mi & 1);          // 8-dim chunk, 0..15
          const uint32_t addr = st + (dchunk >> 3) * kBoxBytes + sw128_off(row, dchunk & 7);
          uint32_t b0, b1, b2, b3;
          ldsm_x4(addr, b0, b1, b2, b3);
          mma_bf16(sc[0], qa[ks], b0, b1);
          mma_bf16(sc[1], qa[ks], b2, b3);
        }
        // Scale to base 2, mask tokens past the chunk end, online softmax.
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int tok = t0 + tw + nt * 8 + 2 * tig + e;
            const bool ok = tok < t_end;
            sc[nt][e] = ok ? sc[nt][e] * a.scale_log2 : -INFINITY;
            sc[nt][2 + e] = ok ? sc[nt][2 + e] * a.scale_log2 : -INFINITY;
            mx0 = fmaxf(mx0, sc[nt][e]);
            mx1 = fmaxf(mx1, sc[nt][2 + e]);
          }
        }
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
        const float u0 = (n0 == -INFINITY) ? 0.f : n0;
        const float u1 = (n1 == -INFINITY) ? 0.f : n1;
        const float al0 = (m0 == -INFINITY) ? 0.f : exp2f(m0 - u0);
        const float al1 = (m1 == -INFINITY) ? 0.f : exp2f(m1 - u1);
        m0 = n0;
        m1 = n1;
        float p[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          p[nt][0] = exp2f(sc[nt][0] - u0);
          p[nt][1] = exp2f(sc[nt][1] - u0);
          p[nt][2] = exp2f(sc[nt][2] - u1);
          p[nt][3] = exp2f(sc[nt][3] - u1);
        }
        l0 = l0 * al0 + (p[0][0] + p[0][1] + p[1][0] + p[1][1]);
        l1 = l1 * al1 + (p[0][2] + p[0][3] + p[1][2] + p[1][3]);
#pragma unroll
        for (int n = 0; n < 16; ++n) {
          acc[n][0] *= al0; acc[n][1] *= al0;
          acc[n][2] *= al1; acc[n][3] *= al1;
        }
        // P as the A operand (rows = heads, k = the 16 tokens).
        uint32_t pa[4];
        pa[0] = pack_bf16x2(p[0][0], p[0][1]);
        pa[1] = pack_bf16x2(p[0][2], p[0][3]);
        pa[2] = pack_bf16x2(p[1][0], p[1][1]);
        pa[3] = pack_bf16x2(p[1][2], p[1][3]);
        // O += P V: V tile rows are tokens, B fragments via transposed ldmatrix.
        const uint32_t vbase = st + 2 * kBoxBytes;
#pragma unroll
        for (int dn = 0; dn < 16; dn += 2) {
          const int mi = lane >> 3;
          const int row = tw + ((mi & 1) << 3) + (lane & 7);
          const int dchunk = dn + (mi >> 1);
          const uint32_t addr = vbase + (dchunk >> 3) * kBoxBytes + sw128_off(row, dchunk & 7);
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(addr, b0, b1, b2, b3);
          mma_bf16(acc[dn], pa, b0, b1);
          mma_bf16(acc[dn + 1], pa, b2, b3);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }

      // ---- merge the four warps' states into the chunk partial ----------
      l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
      l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
      float* ow = comb_o + warp * 16 * kD;
#pragma unroll
      for (int n = 0; n < 16; ++n) {
        const int c = n * 8 + 2 * tig;
        *reinterpret_cast<float2*>(ow + grp * kD + c) = make_float2(acc[n][0], acc[n][1]);
        *reinterpret_cast<float2*>(ow + (grp + 8) * kD + c) = make_float2(acc[n][2], acc[n][3]);
      }
      if (tig == 0) {
        comb_ml[(warp * 16 + grp) * 2 + 0] = m0;
        comb_ml[(warp * 16 + grp) * 2 + 1] = l0;
        comb_ml[(warp * 16 + grp + 8) * 2 + 0] = m1;
        comb_ml[(warp * 16 + grp + 8) * 2 + 1] = l1;
      }
      named_bar_sync(1, kConsumers * 32);
      {
        const int t = threadIdx.x;        // 0..127
        const int row = t >> 3;           // 16 rows
        const int c0 = (t & 7) * 16;      // 16 columns each
        if (row < a.G) {
          float M = -INFINITY;
#pragma unroll
          for (int w = 0; w < kConsumers; ++w) M = fmaxf(M, comb_ml[(w * 16 + row) * 2]);
          float f[kConsumers];
          float L = 0.f;
#pragma unroll
          for (int w = 0; w < kConsumers; ++w) {
            const float mw = comb_ml[(w * 16 + row) * 2];
            f[w] = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
            L += f[w] * comb_ml[(w * 16 + row) * 2 + 1];
          }
          const float inv = L > 0.f ? 1.f / L : 0.f;
          const int cps = a.n_chunks / a.shards;
          const long long slot = static_cast<long long>(ch % cps) * a.shards + ch / cps;
          const long long orow = slot * a.B * a.Hq + static_cast<long long>(b) * a.Hq +
                                 g * a.G + row;
          float* dst = a.ws_o + orow * kD + c0;
#pragma unroll
          for (int c = 0; c < 16; c += 4) {
            float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int w = 0; w < kConsumers; ++w) {
              const float4 x = *reinterpret_cast<const float4*>(comb_o + (w * 16 + row) * kD + c0 + c);
              o.x = fmaf(f[w], x.x, o.x); o.y = fmaf(f[w], x.y, o.y);
              o.z = fmaf(f[w], x.z, o.z); o.w = fmaf(f[w], x.w, o.w);
            }
            o.x *= inv; o.y *= inv; o.z *= inv; o.w *= inv;
            *reinterpret_cast<float4*>(dst + c) = o;
          }
          if ((t & 7) == 0) a.ws_lse[orow] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
        }
      }
      named_bar_sync(1, kConsumers * 32);
      if (*abort_flag) break;
    }
  }
  __syncthreads();
  // On an aborted run, loads may still be landing in the ring: let the last
  // issued load of every stage complete (bounded) before shared memory goes.
  if (*abort_flag && threadIdx.x == 0) {
    const int n = *issued;
    for (int i = n - kStages < 0 ? 0 : n - kStages; i < n; ++i) {
      const unsigned long long t0 = globaltimer_ns();
      while (!mbar_try_wait(&full[i % kStages], (i / kStages) & 1) &&
             globaltimer_ns() - t0 < a.ctx.wait_ns) {
      }
    }
  }
}

}  // namespace

size_t decode_workspace_bytes(const ra_shape& s) {
  const long long n_chunks = (static_cast<long long>(s.n_k) + kChunk - 1) / kChunk;
  const long long rows = static_cast<long long>(s.B) * s.Hq;
  return static_cast<size_t>(n_chunks * rows * (kD + 1) * sizeof(float)) + 256;
}

int launch_decode_partial(const void* q, const void* k, const void* v, long long kv_head_stride,
                          const ra_shape& s, float scale, float* o_part, float* lse_part,
                          float* workspace, const DeviceInfo& dev, cudaStream_t stream,
                          int shards) {
  if (s.d_qk != kD || s.d_v != kD || s.dtype != RA_BF16 || s.Hq / s.Hkv > 16)
    return RA_ERR_UNSUPPORTED;
  // several shards need whole chunks in every shard
  if (shards < 1 || (shards > 1 && (s.n_k % shards != 0 || (s.n_k / shards) % kChunk != 0)))
    return RA_ERR_UNSUPPORTED;
  CUtensorMap tk, tv;
  const uint64_t heads = static_cast<uint64_t>(s.B) * s.Hkv;
  const uint64_t hstride = static_cast<uint64_t>(kv_head_stride) * kD * 2;
  if (make_tmap_bf16_3d(&tk, k, kD, s.n_k, heads, kD * 2, hstride, 64, kTok) != 0 ||
      make_tmap_bf16_3d(&tv, v, kD, s.n_k, heads, kD * 2, hstride, 64, kTok) != 0)
    return RA_ERR_CUDA;
  DecodeArgs a;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.B = s.B;
  a.Hq = s.Hq;
  a.Hkv = s.Hkv;
  a.G = s.Hq / s.Hkv;
  a.n_k = s.n_k;
  a.n_chunks = (s.n_k + kChunk - 1) / kChunk;
  a.shards = shards;
  a.scale_log2 = scale * kLog2e;
  const long long rows = static_cast<long long>(s.B) * s.Hq;
  a.ws_o = workspace;
  a.ws_lse = workspace + a.n_chunks * rows * kD;
  a.ctx = dev.ctx;
  if (cudaFuncSetAttribute(decode_chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kSmemBytes)) != cudaSuccess)
    return RA_ERR_CUDA;
  const int units = s.B * s.Hkv * a.n_chunks;
  const int grid = units < dev.num_sms ? units : dev.num_sms;
  decode_chunk_kernel<<<grid, kThreads, kSmemBytes, stream>>>(tk, tv, a);
  note_launch();
  if (cudaGetLastError() != cudaSuccess) return RA_ERR_CUDA;
  // o_part / lse_part: [shards][B*Hq](kD): one partial per shard
  return launch_lse_merge(a.ws_o, a.ws_lse, a.n_chunks / shards, rows * shards, kD, o_part,
                          RA_F32, lse_part, dev.num_sms, stream);
}

// ---------------------------------------------------------------------------
// Allocation-free variant.  Some callers cannot allocate device memory: a
// plugin inside a host runtime that owns all device memory and hands its
// plugins no allocator, or a latency-critical loop that must not call
// cudaMalloc (which may synchronise the device and has no latency bound).
// For them the chunk partials live in this file-scope array instead of a
// caller workspace.  Every GPU that loads the library holds the array until
// the process exits.  Calls share it: two calls whose kernels overlap on the
// GPU (different streams, no ordering between them) race on it.  Nothing in
// it needs to start at zero, since the chunk kernel writes every partial that
// the merge then reads; it keeps the last call's contents.
constexpr size_t kStaticScratchBytes = 16u << 20;   // 16 MiB
static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

namespace {

std::mutex g_scratch_mu;
float* g_scratch_ptr[64] = {};

// Device address of the scratch array for the current device.  In host code
// the array's name is only a host-side stand-in, so the address is looked up
// once per device (with that device current) and cached.
int scratch_address(int device, float** out) {
  if (device < 0 || device >= 64) return RA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[device] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr)
      return RA_ERR_CUDA;
    g_scratch_ptr[device] = static_cast<float*>(p);
  }
  *out = g_scratch_ptr[device];
  return RA_OK;
}

}  // namespace

size_t decode_static_scratch_bytes() { return kStaticScratchBytes; }

int launch_decode_partial_static(const void* q, const void* k, const void* v,
                                 long long kv_head_stride, const ra_shape& s, float scale,
                                 float* o_part, float* lse_part, const DeviceInfo& dev,
                                 cudaStream_t stream) {
  if (decode_workspace_bytes(s) > kStaticScratchBytes) return RA_ERR_UNSUPPORTED;
  float* ws = nullptr;
  const int rc = scratch_address(dev.device, &ws);
  if (rc != RA_OK) return rc;
  return launch_decode_partial(q, k, v, kv_head_stride, s, scale, o_part, lse_part, ws, dev,
                               stream);
}

}  // namespace ra
