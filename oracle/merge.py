"""N-way merge of normalised attention partials (O_p, LSE_p), fp64.

Test infrastructure only (see ``oracle/__init__.py``).

Each partial is attention of the same query rows over a disjoint key subset:
O_p is normalised over its own keys and LSE_p is the natural-log sum of its
exponentiated scores.  The merge is the closed form of the beta / gamma fold
of page "LLM长文本推理Ring Attention环形注意力机制实现与优化", section
"Ring Attention实现代码与通信重叠", applied to all P partials at once, and the
reduction step of pass-Q decode of page "上下文并行 (CP) 收益评估实验设计",
section on decode (query sent to every shard, partial attention, then reduced):

    L*  = max_p LSE_p
    w_p = exp(LSE_p - L*)
    LSE = L* + ln sum_p w_p
    O   = sum_p (w_p / sum_q w_q) O_p

Partials with LSE_p = -inf (no visible key) carry zero weight; if every
partial of a row is -inf the row's result is O = 0, LSE = -inf.
"""
from __future__ import annotations

import numpy as np

__all__ = ["lse_merge"]


def lse_merge(o_parts, lse_parts):
    """o_parts [P, ..., dv], lse_parts [P, ...] -> (O [..., dv], LSE [...])."""
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    l_star = lse_parts.max(axis=0)
    empty = ~np.isfinite(l_star)
    l_ref = np.where(empty, 0.0, l_star)
    w = np.exp(lse_parts - l_ref[None])          # exp(-inf) = 0
    w_sum = w.sum(axis=0)
    safe = np.where(empty, 1.0, w_sum)
    o = (w[..., None] * o_parts).sum(axis=0) / safe[..., None]
    o[empty] = 0.0
    with np.errstate(divide="ignore"):
        lse = np.where(empty, -np.inf, l_ref + np.log(safe))
    return o, lse
