"""FLOP and byte formulas of the pages (algorithmic work per call).

Test infrastructure only (see ``oracle/__init__.py``).  The product's bench
computes the same quantities independently; tests check that the two agree
and that these reproduce the pages' worked numbers.
"""
from __future__ import annotations

__all__ = ["kv_cache_bytes", "decode_latency_lower_bound_s", "prefill_flops",
           "backward_flops", "pass_kv_bytes_per_chip", "mla_ckv_bytes",
           "prefill_compute_time_s", "prefill_time_s", "scaling_efficiency"]


def kv_cache_bytes(L, h_kv, d_h, n, b):
    """Page "长上下文的第一性挑战", Eq. (lc-ch-kv-memory): M_KV = 2 L H_kv d_h n b
    bytes of K plus V for one sequence."""
    return 2 * L * h_kv * d_h * n * b


def decode_latency_lower_bound_s(kv_bytes, hbm_bytes_per_s):
    """Same page, table decode-bw: one decode step reads the whole KV cache
    once, so its attention time is at least bytes / HBM bandwidth."""
    return kv_bytes / hbm_bytes_per_s


def prefill_flops(B, S, d_qk, d_v, heads=1, causal=False):
    """Page "上下文并行 (CP) 收益评估实验设计", Eq. (cpeval-comp) numerator,
    2 B S^2 (D_qk + D_v), the FLOPs of QK^T and PV for one head.  The page's
    formula counts one head and the full square; ``heads`` multiplies it and
    ``causal`` halves it (the causal triangle, 1/2 rather than (n+1)/(2n))."""
    f = 2 * B * S * S * (d_qk + d_v) * heads
    return f // 2 if causal else f


def backward_flops(B, S, d_qk, d_v, heads=1, causal=False):
    """Algorithmic FLOPs of the attention backward pass (the pages give none):
    the five products of its definition, each 2 S^2 times its inner size --
    scores recomputed (D_qk), dP = dO V^T (D_v), dV = P^T dO (D_v),
    dQ = dS K (D_qk), dK = dS^T Q (D_qk).  Causal halves it, as for
    ``prefill_flops``."""
    f = 2 * B * S * S * (3 * d_qk + 2 * d_v) * heads
    return f // 2 if causal else f


def pass_kv_bytes_per_chip(cp, S, c_kv):
    """Same page, prefill section: KV bytes each chip forwards round the ring,
    (cp - 1) / cp * S * c_kv."""
    return (cp - 1) * S * c_kv / cp


def mla_ckv_bytes(kv_lora_rank, rope_dim, bytes_per_value):
    """KV bytes per token per layer of an MLA cache (compressed latent plus the
    decoupled RoPE key), page "上下文并行 (CP) 收益评估实验设计", table of fixed
    parameters (c_kv for DeepSeek-V3 in BF16)."""
    return (kv_lora_rank + rope_dim) * bytes_per_value


def prefill_compute_time_s(B, S, d_qk, d_v, cp, R):
    """Page "上下文并行 (CP) 收益评估实验设计", Eq. (cpeval-comp): each of the cp
    chips computes 2 B S^2 (D_qk + D_v) / cp FLOPs at an effective rate of R
    FLOP/s, so T_comp = 2 B S^2 (D_qk + D_v) / (cp R) (one head, full square,
    as the page writes it)."""
    return 2 * B * S * S * (d_qk + d_v) / (cp * R)


def prefill_time_s(t_comp, t_passkv):
    """Same page, Eq. (cpeval-prefill): with the ring exchange overlapped with
    the block computation the slower of the two is the critical path,
    T_prefill = max(T_comp, T_passkv)."""
    return max(t_comp, t_passkv)


def scaling_efficiency(t_1, t_cp, cp):
    """Same page, terms table ("scaling 效率"): eta(cp) = T(cp = 1) / (cp T(cp)),
    1 for a linear speed-up."""
    return t_1 / (cp * t_cp)
