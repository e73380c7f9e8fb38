"""Causal classification of (query tile, key tile) blocks from the mask.

Test infrastructure only (see ``oracle/__init__.py``).

A block is SKIP (0) when none of its (query, key) pairs is visible, FULL (2)
when all are, PARTIAL (1) otherwise.  Visibility is the causal rule of page
"AI 推理系列（十一）：Ring Attention 如何让多张 GPU 共同计算一条超长序列", section
"KV 在 Ring 中如何流动" (no query reads a future token), on absolute positions
q_offset + t and k_offset + u.  Without the causal mask every block is FULL.
Blocks at the ragged end cover only the rows / keys that exist.

The classification is derived from the mask itself: per query row, the number
of visible keys of the block, clip(q_pos - k_start + 1, 0, k_len); the block is
FULL if every row sees all k_len keys and SKIP if every row sees none.
``block_class_bruteforce`` builds the boolean mask explicitly.
"""
from __future__ import annotations

import numpy as np

SKIP, PARTIAL, FULL = 0, 1, 2

__all__ = ["SKIP", "PARTIAL", "FULL", "block_class", "block_class_bruteforce",
           "partition_class"]


def block_class(n_q, n_k, q_block, k_block, q_offset=0, k_offset=0, causal=True):
    """int8 map [ceil(n_q/q_block), ceil(n_k/k_block)] of SKIP/PARTIAL/FULL."""
    tq = -(-n_q // q_block)
    tk = -(-n_k // k_block)
    out = np.full((tq, tk), FULL, dtype=np.int8)
    if not causal:
        return out
    q_pos = q_offset + np.arange(n_q, dtype=np.int64)
    for bj in range(tk):
        k_start = bj * k_block
        k_len = min(k_block, n_k - k_start)
        # visible keys of this block for every query row
        vis = np.clip(q_pos - (k_offset + k_start) + 1, 0, k_len)
        for bi in range(tq):
            r = vis[bi * q_block:(bi + 1) * q_block]
            if (r == k_len).all():
                out[bi, bj] = FULL
            elif (r == 0).all():
                out[bi, bj] = SKIP
            else:
                out[bi, bj] = PARTIAL
    return out


def block_class_bruteforce(n_q, n_k, q_block, k_block, q_offset=0, k_offset=0,
                           causal=True):
    """Same map from the explicit n_q x n_k boolean mask (small sizes only)."""
    if causal:
        mask = ((k_offset + np.arange(n_k))[None, :]
                <= (q_offset + np.arange(n_q))[:, None])
    else:
        mask = np.ones((n_q, n_k), dtype=bool)
    tq = -(-n_q // q_block)
    tk = -(-n_k // k_block)
    out = np.empty((tq, tk), dtype=np.int8)
    for bi in range(tq):
        for bj in range(tk):
            blk = mask[bi * q_block:(bi + 1) * q_block, bj * k_block:(bj + 1) * k_block]
            out[bi, bj] = FULL if blk.all() else (SKIP if not blk.any() else PARTIAL)
    return out


def partition_class(n, P, causal=True):
    """[P, P] class of (Q_i, KV_j) partition blocks for the contiguous split."""
    if n % P:
        raise ValueError("n must be divisible by P")
    return block_class(n, n, n // P, n // P, 0, 0, causal)
