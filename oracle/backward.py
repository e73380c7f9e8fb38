"""fp64 gradients of (causal, grouped-query) softmax attention.

Test infrastructure only (see ``oracle/__init__.py``).

The pages name the backward pass without giving an algorithm: page
"AI 推理系列（十一）：Ring Attention 如何让多张 GPU 共同计算一条超长序列",
opening section (training keeps the information the backward pass needs, and
it grows with the sequence) and section on verification (a wrong result is to
be looked for in the causal mask, the block edges, the softmax carried across
blocks and the data dependencies of the backward pass).  What the gradient is
follows from the forward definition of page "长上下文的第一性挑战", Eq.
(lc-ch-attention), by the chain rule; this module writes it out.

For one (b, query head h) with KV head g = h // (H_q / H_kv), a loss that
depends on the output O through dO = dLoss/dO, and the row statistics of the
forward pass (P_{t,u} = exp(s_{t,u} - LSE_t) on visible pairs, 0 elsewhere):

    dV_u  += sum_t P_{t,u} dO_t
    dP_{t,u} = dO_t . v_u
    D_t    = sum_u P_{t,u} dP_{t,u}  ( = dO_t . O_t )
    dS_{t,u} = P_{t,u} (dP_{t,u} - D_t)
    dQ_t   = scale * sum_u dS_{t,u} k_u
    dK_u  += scale * sum_t dS_{t,u} q_t

The "+=" sums over the query heads of one KV group.  A row with no visible
key has P = 0 and contributes nothing.  Only dO enters; the loss is taken not
to depend on LSE (the forward's second output), the plainest reading of a
training step that consumes O.

``attention_backward`` is that definition with each row seeing its whole key
range at once.  ``ring_attention_backward`` takes the ring's blocks one at a
time (Q_i, dO_i and the forward's final LSE_i and D_i stay put; KV_j and its
gradient accumulators dK_j, dV_j travel), so that the tests can pin the
definition against the blockwise form for any P and block order.
"""
from __future__ import annotations

import numpy as np

from .attention import _as_f64, attention, gqa_group
from .blockwise import partition_bounds, ring_order

__all__ = ["attention_backward", "attention_backward_sampled", "ring_attention_backward",
           "block_backward_share", "row_delta"]


def _positions(n, offset, positions):
    if positions is None:
        return offset + np.arange(n, dtype=np.int64)
    return np.asarray(positions, dtype=np.int64)


def _probs(q_rows, k, scale, causal, q_pos, k_pos):
    """Softmax probabilities of a set of rows over one head's keys (fp64)."""
    s = (q_rows @ k.T) * scale
    if causal:
        s = np.where(k_pos[None, :] <= q_pos[:, None], s, -np.inf)
    m = s.max(axis=1) if s.shape[1] else np.full(s.shape[0], -np.inf)
    empty = ~np.isfinite(m)
    e = np.exp(s - np.where(empty, 0.0, m)[:, None])
    z = e.sum(axis=1)
    p = e / np.where(empty, 1.0, z)[:, None]
    p[empty] = 0.0
    return p


def attention_backward(q, k, v, do, scale: float, causal: bool, q_offset: int = 0,
                       k_offset: int = 0, q_positions=None, k_positions=None,
                       row_chunk: int = 512):
    """Gradients (dQ, dK, dV) in fp64 for BHSD inputs.

    q [B, H_q, n_q, dqk], k [B, H_kv, n_k, dqk], v [B, H_kv, n_k, dv],
    do [B, H_q, n_q, dv]; positions as in ``oracle.attention.attention``.
    Returns dq [B, H_q, n_q, dqk], dk [B, H_kv, n_k, dqk], dv [B, H_kv, n_k, dv].
    """
    B, h_q, n_q, dqk = q.shape
    _, h_kv, n_k, _ = k.shape
    dvd = v.shape[-1]
    grp = gqa_group(h_q, h_kv)
    q_pos = _positions(n_q, q_offset, q_positions)
    k_pos = _positions(n_k, k_offset, k_positions)
    dq = np.zeros((B, h_q, n_q, dqk))
    dk = np.zeros((B, h_kv, n_k, dqk))
    dv = np.zeros((B, h_kv, n_k, dvd))
    for b in range(B):
        for h in range(h_q):
            g = h // grp
            kk, vv = _as_f64(k[b, g]), _as_f64(v[b, g])
            qh, doh = _as_f64(q[b, h]), _as_f64(do[b, h])
            for c0 in range(0, n_q, row_chunk):
                r = slice(c0, min(n_q, c0 + row_chunk))
                p = _probs(qh[r], kk, scale, causal, q_pos[r], k_pos)
                o = p @ vv
                dp = doh[r] @ vv.T
                d_row = (doh[r] * o).sum(axis=1)
                ds = p * (dp - d_row[:, None])
                dv[b, g] += p.T @ doh[r]
                dq[b, h, r] = scale * (ds @ kk)
                dk[b, g] += scale * (ds.T @ qh[r])
    return dq, dk, dv


def attention_backward_sampled(q, k, v, do, scale: float, causal: bool, rows, keys,
                               heads=None, kv_heads=None, row_chunk: int = 2048):
    """The same gradients at a sample: dQ at query ``rows`` of query ``heads``,
    dK and dV at ``keys`` of ``kv_heads`` (positions 0..n-1, n_q == n_k).

    dQ_t needs only row t; dK_u, dV_u need column u of every row that sees
    key u (every row, or with a causal mask the rows t >= u), i.e. those
    rows' LSE and D, which come from ``oracle.attention.attention`` over just
    those rows.  Returns dq [B, len(heads), len(rows), dqk],
    dk [B, len(kv_heads), len(keys), dqk], dv [B, len(kv_heads), len(keys), dv].
    """
    B, h_q, n, dqk = q.shape
    h_kv = k.shape[1]
    dvd = v.shape[-1]
    grp = gqa_group(h_q, h_kv)
    rows = np.asarray(rows, dtype=np.int64)
    keys = np.asarray(keys, dtype=np.int64)
    heads = list(range(h_q)) if heads is None else list(heads)
    kv_heads = list(range(h_kv)) if kv_heads is None else list(kv_heads)
    pos = np.arange(n, dtype=np.int64)
    dq = np.zeros((B, len(heads), len(rows), dqk))
    dk = np.zeros((B, len(kv_heads), len(keys), dqk))
    dv = np.zeros((B, len(kv_heads), len(keys), dvd))
    need_heads = sorted(set(heads) | {g * grp + r for g in kv_heads for r in range(grp)})
    # rows whose statistics are needed: the sampled rows, plus every row that
    # can see a sampled key
    tail = np.arange(int(keys.min()) if (causal and len(keys)) else 0, n, dtype=np.int64)
    need_rows = np.union1d(rows, tail if len(keys) else np.zeros(0, np.int64))
    for b in range(B):
        stats = {}
        for h in need_heads:
            o, lse_r = attention(q[b:b + 1], k[b:b + 1], v[b:b + 1], scale, causal,
                                 heads=[h], rows=need_rows, row_chunk=row_chunk)
            lse = np.full(n, np.nan)
            dlt = np.full(n, np.nan)
            lse[need_rows] = lse_r[0, 0]
            dlt[need_rows] = (o[0, 0] * _as_f64(do[b, h][need_rows])).sum(axis=1)
            stats[h] = (lse, dlt)
        for hi, h in enumerate(heads):
            g = h // grp
            kk, vv = _as_f64(k[b, g]), _as_f64(v[b, g])
            qr, dor = _as_f64(q[b, h][rows]), _as_f64(do[b, h][rows])
            lse, dlt = stats[h][0][rows], stats[h][1][rows]
            s = (qr @ kk.T) * scale
            if causal:
                s = np.where(pos[None, :] <= rows[:, None], s, -np.inf)
            live = np.isfinite(lse)
            p = np.zeros_like(s)
            p[live] = np.exp(s[live] - lse[live, None])
            ds = p * (dor @ vv.T - dlt[:, None])
            dq[b, hi] = scale * (ds @ kk)
        for gi, g in enumerate(kv_heads):
            kc, vc = _as_f64(k[b, g][keys]), _as_f64(v[b, g][keys])
            for r in range(grp):
                h = g * grp + r
                qa, doa = _as_f64(q[b, h][tail]), _as_f64(do[b, h][tail])
                lse, dlt = stats[h][0][tail], stats[h][1][tail]
                st = (qa @ kc.T) * scale                      # [len(tail), len(keys)]
                if causal:
                    st = np.where(keys[None, :] <= tail[:, None], st, -np.inf)
                live = np.isfinite(lse)
                p = np.zeros_like(st)
                p[live] = np.exp(st[live] - lse[live, None])
                ds = p * (doa @ vc.T - dlt[:, None])
                dk[b, gi] += scale * (ds.T @ qa)
                dv[b, gi] += p.T @ doa
    return dq, dk, dv


def block_backward_share(q, k, v, do, lse, delta, scale: float, causal: bool, q_positions,
                         k_positions):
    """One block's share of the gradients (dQ, dK, dV) in fp64, formed against
    the query rows' final LSE and D = rowsum(dO * O) (passed in), for query
    rows at ``q_positions`` and keys at ``k_positions``: what a device of the
    ring adds when KV_j reaches Q_i.  Shapes as ``attention_backward``; lse,
    delta [B, H_q, n_q]."""
    B, h_q, n_q, dqk = q.shape
    h_kv = k.shape[1]
    grp = gqa_group(h_q, h_kv)
    qp = np.asarray(q_positions, dtype=np.int64)
    kp = np.asarray(k_positions, dtype=np.int64)
    lse, delta = _as_f64(lse), _as_f64(delta)
    dq = np.zeros((B, h_q, n_q, dqk))
    dk = np.zeros(k.shape[:3] + (dqk,))
    dv = np.zeros(v.shape)
    for b in range(B):
        for h in range(h_q):
            g = h // grp
            qh, doh = _as_f64(q[b, h]), _as_f64(do[b, h])
            kk, vv = _as_f64(k[b, g]), _as_f64(v[b, g])
            s = (qh @ kk.T) * scale
            if causal:
                s = np.where(kp[None, :] <= qp[:, None], s, -np.inf)
            live = np.isfinite(lse[b, h])
            p = np.zeros_like(s)
            p[live] = np.exp(s[live] - lse[b, h][live, None])
            ds = p * (doh @ vv.T - delta[b, h][:, None])
            dq[b, h] += scale * (ds @ kk)
            dk[b, g] += scale * (ds.T @ qh)
            dv[b, g] += p.T @ doh
    return dq, dk, dv


def row_delta(o, do):
    """D_t = dO_t . O_t per row, fp64 ([..., n, dv] -> [..., n])."""
    return (_as_f64(do) * _as_f64(o)).sum(axis=-1)


def ring_attention_backward(q, k, v, do, scale: float, causal: bool, P: int,
                            order=None, q_positions=None, k_positions=None):
    """Blockwise gradients over a P-way split, block by block in ring order.

    The forward's final (O, LSE) come from ``oracle.attention.attention``;
    D = rowsum(dO * O).  For query partition i and ring step s the block
    (Q_i, KV_j), j = (i - s) mod P, adds its share to dQ_i, dK_j and dV_j,
    with P_{t,u} = exp(s_{t,u} - LSE_t) taken against the FINAL LSE, so each
    block's share is final and the blocks may come in any order.
    ``order``: optional callable (P, i) -> list of j (default: ring order).
    ``q_positions`` / ``k_positions``: absolute positions of all n tokens
    (default 0..n-1), e.g. a striped layout.
    """
    B, h_q, n, dqk = q.shape
    h_kv = k.shape[1]
    dvd = v.shape[-1]
    grp = gqa_group(h_q, h_kv)
    order = order or ring_order
    pos_q = _positions(n, 0, q_positions)
    pos_k = _positions(n, 0, k_positions)
    o, lse = attention(q, k, v, scale, causal, q_positions=pos_q, k_positions=pos_k)
    dlt = row_delta(o, do)
    bounds = partition_bounds(n, P)
    dq = np.zeros((B, h_q, n, dqk))
    dk = np.zeros((B, h_kv, n, dqk))
    dv = np.zeros((B, h_kv, n, dvd))
    for b in range(B):
        for h in range(h_q):
            g = h // grp
            qh, doh = _as_f64(q[b, h]), _as_f64(do[b, h])
            kk, vv = _as_f64(k[b, g]), _as_f64(v[b, g])
            for i, (q0, q1) in enumerate(bounds):
                lse_i = lse[b, h, q0:q1]
                live = np.isfinite(lse_i)
                for j in order(P, i):
                    k0, k1 = bounds[j]
                    s = (qh[q0:q1] @ kk[k0:k1].T) * scale
                    if causal:
                        vis = pos_k[None, k0:k1] <= pos_q[q0:q1, None]
                        if not vis.any():
                            continue           # fully masked block: skipped
                        s = np.where(vis, s, -np.inf)
                    p = np.zeros_like(s)
                    p[live] = np.exp(s[live] - lse_i[live, None])
                    dp = doh[q0:q1] @ vv[k0:k1].T
                    ds = p * (dp - dlt[b, h, q0:q1, None])
                    dq[b, h, q0:q1] += scale * (ds @ kk[k0:k1])
                    dk[b, g, k0:k1] += scale * (ds.T @ qh[q0:q1])
                    dv[b, g, k0:k1] += p.T @ doh[q0:q1]
    return dq, dk, dv
