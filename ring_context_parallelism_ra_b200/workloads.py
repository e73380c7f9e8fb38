"""Seeded synthetic workloads: shapes, sizes and input generators.

This module holds no attention arithmetic.  It is the one piece shared by the
tests, the bench and the oracle side: it draws the inputs, and both the CUDA
path and the fp64 oracle consume the same tensors.

Recipe: every (tensor, batch, head) slice is drawn independently from
``torch.Generator(device).manual_seed(seed)`` as i.i.d. N(0, 1) fp32, where the
seed is a fixed function of (workload seed, tensor, batch, head); Q and K are
then multiplied by the workload's ``qk_mult`` (exact, a power of two) and the
result is rounded to the workload dtype.  Large workloads are drawn directly
on the GPU (torch's own generator; the CPU draws 10^8 values per second at
best) and the oracle receives CPU copies of the slices it checks; small ones
are drawn on the CPU.  The two devices give different (equally valid) values
for the same seed, so one test never mixes them.

The five workloads mirror the shapes the pages discuss: grouped-query heads
with d = 128, 8K to 1M tokens, P = 4..16 partitions, an MLA-like head with
D_qk = 192 and D_v = 128, and a pass-Q decode over a 1M-token cache.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

__all__ = ["Workload", "WORKLOADS", "workload", "draw_slice", "make_qkv", "make_dout",
           "make_workload_inputs", "prefill_flops", "backward_flops", "decode_kv_bytes",
           "striped_order"]

_TENSOR_ID = {"q": 1, "k": 2, "v": 3, "do": 4}


@dataclass(frozen=True)
class Workload:
    key: str
    name: str
    B: int
    Hq: int
    Hkv: int
    n: int               # sequence length (prefill) or cached tokens (decode)
    d_qk: int
    d_v: int
    dtype: str           # "f32" or "bf16"
    P: int               # ring partitions (prefill) or KV shards (decode)
    causal: bool
    decode: bool = False
    qk_mult: float = 1.0
    seed: int = field(default=0)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d_qk)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def n_q(self) -> int:
        return 1 if self.decode else self.n


WORKLOADS = {w.key: w for w in (
    Workload("noncausal_fp32_512", "noncausal_fp32_b1_h1_n512_d64_P4",
             1, 1, 1, 512, 64, 64, "f32", 4, False, seed=1001),
    Workload("causal_mha_8k", "causal_mha_b1_h8_n8192_d128_P4",
             1, 8, 8, 8192, 128, 128, "bf16", 4, True, qk_mult=0.5, seed=1002),
    Workload("causal_gqa_128k", "causal_gqa_b1_h32kv8_n131072_d128_P8",
             1, 32, 8, 131072, 128, 128, "bf16", 8, True, seed=1003),
    Workload("decode_1m", "decode_passq_b4_h64kv8_n1048576_d128_P8",
             4, 64, 8, 1048576, 128, 128, "bf16", 8, False, decode=True, seed=1004),
    Workload("causal_mla_256k", "causal_mla_b1_h16_n262144_dqk192_dv128_P16",
             1, 16, 16, 262144, 192, 128, "bf16", 16, True, seed=1005),
)}


def workload(key: str) -> Workload:
    """The workload registered under `key` (one of ``WORKLOADS``)."""
    return WORKLOADS[key]


def _slice_seed(seed: int, tensor: str, b: int, h: int) -> int:
    return (seed * 16 + _TENSOR_ID[tensor]) * (1 << 20) + b * 4096 + h


def draw_slice(seed: int, tensor: str, b: int, h: int, rows: int, d: int,
               dtype=torch.bfloat16, mult: float = 1.0, device="cpu") -> torch.Tensor:
    """One [rows, d] slice, N(0,1) fp32 * mult, rounded to dtype."""
    g = torch.Generator(device=device).manual_seed(_slice_seed(seed, tensor, b, h))
    x = torch.randn((rows, d), generator=g, dtype=torch.float32, device=device)
    if mult != 1.0:
        x.mul_(mult)
    return x.to(dtype)


def make_dout(B, Hq, n_q, d_v, dtype=torch.bfloat16, seed=0, device="cpu"):
    """Gradient arriving at the output, dO [B, Hq, n_q, d_v]: N(0,1) rounded."""
    g = torch.empty((B, Hq, n_q, d_v), dtype=dtype, device=device)
    for b in range(B):
        for h in range(Hq):
            g[b, h] = draw_slice(seed, "do", b, h, n_q, d_v, dtype, 1.0, device)
    return g


def make_qkv(B, Hq, Hkv, n_q, n_k, d_qk, d_v, dtype=torch.bfloat16, seed=0,
             qk_mult=1.0, device="cpu"):
    """Contiguous BHSD tensors q [B,Hq,n_q,d_qk], k [B,Hkv,n_k,d_qk],
    v [B,Hkv,n_k,d_v] on `device`."""
    q = torch.empty((B, Hq, n_q, d_qk), dtype=dtype, device=device)
    k = torch.empty((B, Hkv, n_k, d_qk), dtype=dtype, device=device)
    v = torch.empty((B, Hkv, n_k, d_v), dtype=dtype, device=device)
    for b in range(B):
        for h in range(Hq):
            q[b, h] = draw_slice(seed, "q", b, h, n_q, d_qk, dtype, qk_mult, device)
        for h in range(Hkv):
            k[b, h] = draw_slice(seed, "k", b, h, n_k, d_qk, dtype, qk_mult, device)
            v[b, h] = draw_slice(seed, "v", b, h, n_k, d_v, dtype, 1.0, device)
    return q, k, v


def make_workload_inputs(wl: Workload, device="cpu"):
    """Tensors of a named workload (q has one row per sequence for decode)."""
    return make_qkv(wl.B, wl.Hq, wl.Hkv, wl.n_q, wl.n, wl.d_qk, wl.d_v,
                    wl.torch_dtype, wl.seed, wl.qk_mult, device=device)


def prefill_flops(wl: Workload) -> float:
    """Algorithmic FLOPs of QK^T and PV over all heads; causal counts half."""
    f = 2.0 * wl.B * wl.Hq * wl.n * wl.n * (wl.d_qk + wl.d_v)
    return f / 2 if wl.causal else f


def backward_flops(wl: Workload) -> float:
    """Algorithmic FLOPs of the backward pass over all heads: the scores
    recomputed, dP = dO V^T, dV = P^T dO, dQ = dS K, dK = dS^T Q; causal
    counts half."""
    f = 2.0 * wl.B * wl.Hq * wl.n * wl.n * (3 * wl.d_qk + 2 * wl.d_v)
    return f / 2 if wl.causal else f


def decode_kv_bytes(wl: Workload) -> int:
    """Bytes of K and V one decode step must read (the whole cache, once)."""
    esz = 4 if wl.dtype == "f32" else 2
    return wl.B * wl.Hkv * wl.n * (wl.d_qk + wl.d_v) * esz


def striped_order(n: int, P: int):
    """Token order of a striped split: partition i holds tokens i, i + P,
    i + 2P, ..., partitions stored one after another, so row i * (n / P) + r
    holds token r * P + i.  Returns that token index for every row (a
    permutation; ``x[:, :, order]`` lays a BHSD tensor out striped and
    ``y[:, :, argsort(order)]`` restores token order)."""
    if n % P:
        raise ValueError("n must be divisible by P")
    L = n // P
    return [r * P + i for i in range(P) for r in range(L)]
