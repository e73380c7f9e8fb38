"""The pages' blockwise ring algorithm, step by step, in fp64.

Test infrastructure only (see ``oracle/__init__.py``).  These routines exist to
pin ``oracle.attention`` (the plain definition) against the method's own
invariants: for any number of partitions P and any order of the KV blocks the
blockwise result must equal full attention, and P = 1 must reduce to plain
attention.

Steps followed:

* Partition: the sequence is split into P equal contiguous ranges; page
  "LLM长文本推理Ring Attention环形注意力机制实现与优化", opening section (uniform
  split into P parts, device i holds Q_i, K_i, V_i), and page
  "AI 推理系列（十一）" (128K tokens -> 4 x 32K contiguous).
* Ring order: Q_i stays in place; at step s it meets KV_{(i - s) mod P}
  (device i receives from device i - 1 and sends to i + 1); page
  "AI 推理系列（十一）", section "KV 在 Ring 中如何流动".
* Causal skip: a block whose keys all lie in the future of all its queries
  contributes nothing and is skipped; page "AI 推理系列（十一）", same section,
  and page "LLM长文本推理…", section on tuning (causal sparsity).
* Fold, normalised form: page "LLM长文本推理…", section "Ring Attention实现代码与
  通信重叠": each block yields a row max, the exponentials relative to it and
  their sum; the running (out, lse) is updated with weights beta for the old
  output and gamma for the block's normalised output, both derived from the
  new log-sum-exp.
* Fold, online-softmax form: page "AI 推理系列（十一）", section "最容易被忽略的
  细节": keep the running row max, the running exponential sum and an
  unnormalised output; when the max grows, rescale the old accumulator to the
  new max before adding the block's contribution; normalise at the end.
"""
from __future__ import annotations

import numpy as np

from .attention import _as_f64, gqa_group

__all__ = ["partition_bounds", "ring_order", "block_scores", "striped_positions",
           "ring_attention_normalised", "ring_attention_online", "striped_block_visible"]


def partition_bounds(n: int, P: int):
    """Contiguous equal split of n tokens into P partitions: [(start, stop)]."""
    if P <= 0 or n % P != 0:
        raise ValueError(f"n={n} is not divisible into P={P} equal partitions")
    size = n // P
    return [(i * size, (i + 1) * size) for i in range(P)]


def ring_order(P: int, i: int):
    """KV partitions met by query partition i, in step order s = 0..P-1."""
    return [(i - s) % P for s in range(P)]


def striped_positions(n: int, P: int, i: int):
    """Token positions held by partition i of a striped split (page
    "LLM长文本推理…", tuning section: Striped Attention hands sequence positions
    to the devices interleaved): i, i + P, i + 2P, ..."""
    if P <= 0 or n % P != 0:
        raise ValueError(f"n={n} is not divisible into P={P} equal partitions")
    return np.arange(i, n, P, dtype=np.int64)


def striped_block_visible(n: int, P: int, i: int, j: int) -> int:
    """Number of visible (query, key) pairs in block (Q_i, KV_j) of a striped
    split, counted from the explicit positions."""
    qp, kp = striped_positions(n, P, i), striped_positions(n, P, j)
    return int((kp[None, :] <= qp[:, None]).sum())


def block_scores(q_blk, k_blk, scale, causal, q_pos, k_pos):
    """Scaled scores of one (Q_i, KV_j) block with the causal mask applied."""
    s = (q_blk @ k_blk.T) * scale
    if causal:
        s = np.where(k_pos[None, :] <= q_pos[:, None], s, -np.inf)
    return s


def _fold_normalised(out, lse, s, v_blk):
    """One step of the beta / gamma update on rows that see >= 1 key here."""
    max_val = s.max(axis=1)
    live = np.isfinite(max_val)
    if not live.any():
        return out, lse
    s, max_val, vb = s[live], max_val[live], v_blk
    w = np.exp(s - max_val[:, None])
    w_sum = w.sum(axis=1)
    blk_out = (w / w_sum[:, None]) @ vb          # block-normalised output
    old = lse[live]
    old_safe = np.where(np.isfinite(old), old, max_val)
    # new_lse = log(exp(old) + w_sum * exp(max_val)), computed relative to max_val
    new_lse = max_val + np.log(np.exp(old - max_val) * np.isfinite(old) + w_sum)
    beta = np.where(np.isfinite(old), np.exp(old_safe - new_lse), 0.0)
    gamma = w_sum * np.exp(max_val - new_lse)
    out = out.copy()
    lse = lse.copy()
    out[live] = beta[:, None] * out[live] + gamma[:, None] * blk_out
    lse[live] = new_lse
    return out, lse


def _fold_online(m, l, acc, s, v_blk):
    """One step of the running-max / exp-sum / rescaled-accumulator update."""
    blk_max = s.max(axis=1)
    m_new = np.maximum(m, blk_max)
    live = np.isfinite(m_new)
    m_ref = np.where(live, m_new, 0.0)
    alpha = np.where(np.isfinite(m), np.exp(m - m_ref), 0.0)
    p = np.exp(s - m_ref[:, None])
    l = alpha * l + p.sum(axis=1)
    acc = alpha[:, None] * acc + p @ v_blk
    return m_new, l, acc


def _ring_attention(q, k, v, P, scale, causal, order, form):
    B, h_q, n, dqk = q.shape
    _, h_kv, n_k, _ = k.shape
    dv = v.shape[-1]
    if n_k != n:
        raise ValueError("the ring splits one sequence: n_q must equal n_k")
    grp = gqa_group(h_q, h_kv)
    parts = partition_bounds(n, P)
    out = np.zeros((B, h_q, n, dv))
    lse = np.zeros((B, h_q, n))
    for b in range(B):
        for h in range(h_q):
            g = h // grp
            qh, kh, vh = _as_f64(q[b, h]), _as_f64(k[b, g]), _as_f64(v[b, g])
            for i, (q0, q1) in enumerate(parts):
                q_pos = np.arange(q0, q1)
                steps = ring_order(P, i) if order is None else order(i)
                r = q1 - q0
                if form == "normalised":
                    o_i, l_i = np.zeros((r, dv)), np.full(r, -np.inf)
                else:
                    m_i, s_i, a_i = np.full(r, -np.inf), np.zeros(r), np.zeros((r, dv))
                for j in steps:
                    k0, k1 = parts[j]
                    if causal and k0 > q1 - 1:
                        continue  # the whole block lies in the future: skip
                    s = block_scores(qh[q0:q1], kh[k0:k1], scale, causal,
                                     q_pos, np.arange(k0, k1))
                    if form == "normalised":
                        o_i, l_i = _fold_normalised(o_i, l_i, s, vh[k0:k1])
                    else:
                        m_i, s_i, a_i = _fold_online(m_i, s_i, a_i, s, vh[k0:k1])
                if form != "normalised":
                    empty = s_i == 0.0
                    with np.errstate(divide="ignore", invalid="ignore"):
                        o_i = np.where(empty[:, None], 0.0, a_i / np.where(empty, 1.0, s_i)[:, None])
                        l_i = np.where(empty, -np.inf, m_i + np.log(np.where(empty, 1.0, s_i)))
                out[b, h, q0:q1] = o_i
                lse[b, h, q0:q1] = l_i
    return out, lse


def ring_attention_normalised(q, k, v, P, scale, causal, order=None):
    """Blockwise ring attention with the beta / gamma fold of normalised block
    outputs.  ``order(i)`` may override the ring order (any permutation of
    range(P)); the result must not depend on it beyond rounding."""
    return _ring_attention(q, k, v, P, scale, causal, order, "normalised")


def ring_attention_online(q, k, v, P, scale, causal, order=None):
    """Blockwise ring attention with the running-max / exp-sum fold and a final
    normalisation (the form the GPU kernels use on chip)."""
    return _ring_attention(q, k, v, P, scale, causal, order, "online")
