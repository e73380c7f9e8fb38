"""Plain fp64 definition of (causal, grouped-query) softmax attention.

Test infrastructure only (see ``oracle/__init__.py``).

Definition followed: page "长上下文的第一性挑战", Eq. (lc-ch-attention):
O = softmax(Q K^T / sqrt(d_k)) V with Q, K, V in R^{n x d}.  The scale is an
explicit argument (the pages use 1/sqrt(d_k)).  The causal mask is the rule of
page "AI 推理系列（十一）" section "KV 在 Ring 中如何流动" (a query may not read
a future token): key position <= query position, positions being absolute
token indices ``q_offset + t`` and ``k_offset + u``.  Grouped-query heads
(page "AI 推理系列（十一）", section on GQA) map query head h to KV head
h // (H_q / H_kv).

For each (b, h) and query row t the oracle computes, in fp64,

    s_{t,u} = scale * sum_c q_{t,c} k_{u,c}
    M_t     = max over visible u of s_{t,u}
    LSE_t   = M_t + ln sum_{visible u} exp(s_{t,u} - M_t)
    O_t     = sum_{visible u} exp(s_{t,u} - LSE_t) v_u

A row with no visible key gets O_t = 0 and LSE_t = -inf (the pages are silent
on this case; it only arises for a block with offsets).

Every row sees its whole key range at once: there is no blockwise merge here.
Rows are processed in chunks only to bound memory; each chunk is an
independent set of rows.
"""
from __future__ import annotations

import numpy as np

__all__ = ["attention", "decode_attention", "gqa_group"]


def gqa_group(h_q: int, h_kv: int) -> int:
    """Query heads per KV head; contiguous grouping (h -> h // group)."""
    if h_kv <= 0 or h_q % h_kv != 0:
        raise ValueError(f"H_q={h_q} is not a multiple of H_kv={h_kv}")
    return h_q // h_kv


def _as_f64(x) -> np.ndarray:
    """Exact conversion of float32 / bfloat16-valued arrays to fp64."""
    try:  # torch tensors (bf16 included) without importing torch eagerly
        import torch  # noqa: WPS433

        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def _rows_attention(q_rows, k, v, scale, causal, q_pos, k_pos):
    """Attention for a set of query rows against one head's full key range.

    q_rows [r, dqk], k [n_k, dqk], v [n_k, dv], q_pos [r], k_pos [n_k] (int64
    absolute positions).  Returns (O [r, dv], LSE [r]) in fp64.
    """
    s = (q_rows @ k.T) * scale  # [r, n_k]
    if causal:
        visible = k_pos[None, :] <= q_pos[:, None]
        s = np.where(visible, s, -np.inf)
    m = s.max(axis=1) if s.shape[1] > 0 else np.full(s.shape[0], -np.inf)
    empty = ~np.isfinite(m)
    m_safe = np.where(empty, 0.0, m)
    e = np.exp(s - m_safe[:, None])  # exp(-inf) = 0 for masked keys
    z = e.sum(axis=1)
    with np.errstate(divide="ignore"):
        lse = np.where(empty, -np.inf, m_safe + np.log(np.where(empty, 1.0, z)))
    o = (e @ v) / np.where(empty, 1.0, z)[:, None]
    o[empty] = 0.0
    return o, lse


def attention(q, k, v, scale: float, causal: bool, q_offset: int = 0,
              k_offset: int = 0, rows=None, heads=None, row_chunk: int = 512,
              q_positions=None, k_positions=None):
    """fp64 attention over BHSD tensors.

    q [B, H_q, n_q, dqk], k [B, H_kv, n_k, dqk], v [B, H_kv, n_k, dv] (numpy
    or torch, any float dtype; converted exactly to fp64 per head).
    ``rows``: optional 1-D array of query row indices (default: all rows).
    ``heads``: optional list of query heads (default: all).
    ``q_positions`` / ``k_positions``: optional absolute token positions of
    every query row / key (default q_offset + t, k_offset + u); the causal
    rule compares these.
    Returns (O [B, len(heads), len(rows), dv], LSE [B, len(heads), len(rows)]).
    """
    B, h_q, n_q, dqk = q.shape
    _, h_kv, n_k, dqk2 = k.shape
    dv = v.shape[-1]
    if dqk2 != dqk or v.shape[:3] != k.shape[:3]:
        raise ValueError("inconsistent q/k/v shapes")
    grp = gqa_group(h_q, h_kv)
    rows = np.arange(n_q) if rows is None else np.asarray(rows, dtype=np.int64)
    heads = list(range(h_q)) if heads is None else list(heads)
    out = np.zeros((B, len(heads), len(rows), dv))
    lse = np.zeros((B, len(heads), len(rows)))
    k_pos = (k_offset + np.arange(n_k, dtype=np.int64) if k_positions is None
             else np.asarray(k_positions, dtype=np.int64))
    q_pos_all = (q_offset + np.arange(n_q, dtype=np.int64) if q_positions is None
                 else np.asarray(q_positions, dtype=np.int64))
    for b in range(B):
        cached_g, kk, vv = None, None, None
        for hi, h in enumerate(heads):
            g = h // grp
            if g != cached_g:
                kk, vv, cached_g = _as_f64(k[b, g]), _as_f64(v[b, g]), g
            qh = q[b, h]
            for c0 in range(0, len(rows), row_chunk):
                r = rows[c0:c0 + row_chunk]
                q_rows = _as_f64(qh[r])
                o_c, l_c = _rows_attention(q_rows, kk, vv, scale, causal,
                                           q_pos_all[r], k_pos)
                out[b, hi, c0:c0 + len(r)] = o_c
                lse[b, hi, c0:c0 + len(r)] = l_c
    return out, lse


def decode_attention(q, k, v, scale: float):
    """Single-token decode (pass-Q): the one query token of each sequence sees
    every cached token (no causal mask).  q [B, H_q, 1, d], k/v [B, H_kv, S, d].

    Same definition as ``attention`` with n_q = 1 and causal = False; page
    "长上下文的第一性挑战", section on the KV cache as the decode bottleneck,
    where each decode step reads the whole cache once.
    """
    return attention(q, k, v, scale, causal=False)
