"""Pins of the backward oracle (CPU only).

``oracle.backward`` writes out the chain rule of the attention definition.
Nothing here re-types that formula: the gradients are checked against central
finite differences of the forward oracle, against reverse-mode automatic
differentiation of a forward written independently below with torch ops, and
against identities that hold for any input (the softmax gradient sums to zero
over a row, the probabilities of a row sum to one, the causal dependence
pattern), and the blockwise ring form against the whole-row form for any P
and block order.
"""
import math

import numpy as np
import pytest
import torch

from oracle.attention import attention
from oracle.backward import (attention_backward, attention_backward_sampled,
                             ring_attention_backward, row_delta)
from oracle.blockwise import striped_positions
from oracle.costs import backward_flops, prefill_flops


def _inputs(seed, B=1, hq=2, hkv=1, nq=6, nk=6, d=3, dv=4):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((B, hq, nq, d)), rng.standard_normal((B, hkv, nk, d)),
            rng.standard_normal((B, hkv, nk, dv)), rng.standard_normal((B, hq, nq, dv)))


def _loss(q, k, v, g, scale, causal, **kw):
    o, _ = attention(q, k, v, scale, causal, **kw)
    return float((o * g).sum())


def _fd_grad(x, f, h=1e-6):
    """Central differences of a scalar f with respect to every entry of x."""
    gr = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        idx = it.multi_index
        x0 = x[idx]
        x[idx] = x0 + h
        fp = f()
        x[idx] = x0 - h
        fm = f()
        x[idx] = x0
        gr[idx] = (fp - fm) / (2 * h)
    return gr


FD_CASES = [
    # (hq, hkv, nq, nk, causal, q_offset, k_offset)
    (1, 1, 5, 5, False, 0, 0),
    (2, 1, 6, 6, True, 0, 0),
    (4, 2, 5, 7, True, 3, 0),      # block below the diagonal, GQA
    (2, 2, 6, 4, True, 0, 2),      # rows 0 and 1 see no key at all
]


@pytest.mark.parametrize("case", FD_CASES)
def test_gradients_match_finite_differences(case):
    hq, hkv, nq, nk, causal, qo, ko = case
    q, k, v, g = _inputs(hash(case) % 1000, hq=hq, hkv=hkv, nq=nq, nk=nk)
    scale = 0.7
    kw = dict(q_offset=qo, k_offset=ko)
    dq, dk, dv = attention_backward(q, k, v, g, scale, causal, **kw)
    f = lambda: _loss(q, k, v, g, scale, causal, **kw)  # noqa: E731
    for got, x in ((dq, q), (dk, k), (dv, v)):
        want = _fd_grad(x, f)
        assert np.abs(got - want).max() <= 1e-7 * max(1.0, np.abs(want).max())


def _torch_attention(q, k, v, scale, causal, q_pos, k_pos):
    """Forward written with torch ops for autograd: masked scores, softmax
    with -inf masking, product with V.  Rows with no visible key are not
    produced by the inputs used below."""
    grp = q.shape[1] // k.shape[1]
    k = k.repeat_interleave(grp, dim=1)
    v = v.repeat_interleave(grp, dim=1)
    s = torch.einsum("bhtc,bhuc->bhtu", q, k) * scale
    if causal:
        s = s.masked_fill(k_pos[None, :] > q_pos[:, None], float("-inf"))
    return torch.einsum("bhtu,bhuc->bhtc", torch.softmax(s, dim=-1), v)


@pytest.mark.parametrize("causal", [False, True])
def test_gradients_match_reverse_mode_autodiff(causal):
    q, k, v, g = _inputs(5, B=2, hq=4, hkv=2, nq=40, nk=40, d=8, dv=6)
    scale = 1 / math.sqrt(8)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    pos = torch.arange(40)
    o = _torch_attention(tq, tk, tv, scale, causal, pos, pos)
    (o * torch.tensor(g)).sum().backward()
    dq, dk, dv = attention_backward(q, k, v, g, scale, causal, row_chunk=16)
    for got, t in ((dq, tq), (dk, tk), (dv, tv)):
        assert np.abs(got - t.grad.numpy()).max() <= 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_softmax_gradient_sums_to_zero_over_keys(causal):
    # sum_u dS_{t,u} = D_t - D_t = 0 for every row, so sum_u dK_u = 0.
    q, k, v, g = _inputs(8, hq=4, hkv=2, nq=30, nk=30, d=5, dv=3)
    _, dk, _ = attention_backward(q, k, v, g, 0.4, causal)
    assert np.abs(dk.sum(axis=2)).max() <= 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_dv_column_sum_is_dout_sum(causal):
    # sum_u P_{t,u} = 1 on every row with a visible key, so
    # sum_u dV_u = sum over the group's heads and live rows of dO_t.
    q, k, v, g = _inputs(9, hq=4, hkv=2, nq=12, nk=9, d=5, dv=3)
    _, dk, dv = attention_backward(q, k, v, g, 0.4, causal, q_offset=0, k_offset=3)
    live = np.arange(12) >= 3 if causal else np.ones(12, bool)
    want = g[:, :, live].reshape(1, 2, 2, -1, 3).sum(axis=(2, 3))
    assert np.abs(dv.sum(axis=2) - want).max() <= 1e-12


def test_row_with_a_single_visible_key_has_zero_dq():
    # Causal row 0 sees only key 0: P_00 = 1, D_0 = dP_00, so dS_00 = 0.
    q, k, v, g = _inputs(10, nq=5, nk=5)
    dq, _, _ = attention_backward(q, k, v, g, 0.9, True)
    assert np.abs(dq[:, :, 0]).max() <= 1e-12
    assert np.abs(dq[:, :, 1:]).max() > 1e-3


def test_fully_masked_rows_contribute_nothing():
    q, k, v, g = _inputs(11, nq=6, nk=4)
    dq, dk, dv = attention_backward(q, k, v, g, 0.5, True, q_offset=0, k_offset=2)
    assert np.abs(dq[:, :, :2]).max() == 0.0
    g2 = g.copy()
    g2[:, :, :2] += 100.0        # the dead rows' dO must not matter
    _, dk2, dv2 = attention_backward(q, k, v, g2, 0.5, True, q_offset=0, k_offset=2)
    assert np.abs(dk2 - dk).max() == 0.0 and np.abs(dv2 - dv).max() == 0.0


def test_causal_dependence_pattern():
    # dK_u, dV_u see only rows t >= u; dQ_t sees only keys u <= t.
    q, k, v, g = _inputs(12, nq=10, nk=10, d=4, dv=4)
    dq, dk, dv = attention_backward(q, k, v, g, 0.6, True)
    g2 = g.copy()
    g2[:, :, :4] = 7.0
    _, dk2, dv2 = attention_backward(q, k, v, g2, 0.6, True)
    assert np.array_equal(dk2[:, :, 4:], dk[:, :, 4:])
    assert np.array_equal(dv2[:, :, 4:], dv[:, :, 4:])
    k2, v2 = k.copy(), v.copy()
    k2[:, :, 6:] = -3.0
    v2[:, :, 6:] = 5.0
    dq2, _, _ = attention_backward(q, k2, v2, g, 0.6, True)
    assert np.array_equal(dq2[:, :, :6], dq[:, :, :6])


def test_row_delta_equals_probability_weighted_dp():
    # D_t = dO_t . O_t equals sum_u P_{t,u} (dO_t . v_u) because O_t = sum_u P v_u.
    q, k, v, g = _inputs(13, nq=7, nk=7)
    o, lse = attention(q, k, v, 0.8, True)
    s = np.einsum("bhtc,bhuc->bhtu", q, np.repeat(k, 2, axis=1)) * 0.8
    s = np.where(np.tril(np.ones((7, 7), bool)), s, -np.inf)
    p = np.exp(s - lse[..., None])
    dp = np.einsum("bhtc,bhuc->bhtu", g, np.repeat(v, 2, axis=1))
    assert np.abs(row_delta(o, g) - (p * dp).sum(-1)).max() <= 1e-12


@pytest.mark.parametrize("P", [1, 2, 3, 4, 6])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_backward_equals_whole_rows_any_order(P, causal):
    q, k, v, g = _inputs(20 + P, B=2, hq=4, hkv=2, nq=24, nk=24, d=6, dv=5)
    want = attention_backward(q, k, v, g, 0.45, causal)
    rng = np.random.default_rng(P)
    perm = {i: list(rng.permutation(P)) for i in range(P)}
    for order in (None, lambda P_, i: perm[i]):
        got = ring_attention_backward(q, k, v, g, 0.45, causal, P, order=order)
        for a, b in zip(got, want):
            assert np.abs(a - b).max() <= 1e-12


def test_ring_backward_striped_positions():
    # Striped split: partition i holds positions i, i+P, ...; the ring over the
    # permuted tensors equals the whole-row gradients permuted the same way.
    n, P = 24, 4
    q, k, v, g = _inputs(31, hq=2, hkv=1, nq=n, nk=n, d=4, dv=4)
    order = np.concatenate([striped_positions(n, P, i) for i in range(P)])
    want = attention_backward(q, k, v, g, 0.5, True)
    got = ring_attention_backward(q[:, :, order], k[:, :, order], v[:, :, order],
                                  g[:, :, order], 0.5, True, P,
                                  q_positions=order, k_positions=order)
    for a, b in zip(got, want):
        assert np.abs(a - b[:, :, order]).max() <= 1e-12


def test_backward_flops_closed_form():
    # Five products of size S x S x d: 10 S^2 d per head when D_qk = D_v = d,
    # i.e. 2.5 times the forward's two products.
    assert backward_flops(1, 8192, 128, 128, heads=8, causal=True) == \
        5 * prefill_flops(1, 8192, 128, 128, heads=8, causal=True) // 2
    assert backward_flops(2, 100, 64, 32, heads=3) == 2 * 2 * 100 * 100 * (3 * 64 + 2 * 32) * 3


@pytest.mark.parametrize("causal", [False, True])
def test_sampled_gradients_equal_whole_backward(causal):
    q, k, v, g = _inputs(40, B=2, hq=4, hkv=2, nq=37, nk=37, d=6, dv=5)
    dq, dk, dv = attention_backward(q, k, v, g, 0.4, causal)
    rows, keys = [0, 5, 36, 17], [36, 0, 9]
    sq, sk, sv = attention_backward_sampled(q, k, v, g, 0.4, causal, rows, keys,
                                            heads=[3, 0], kv_heads=[1])
    assert np.abs(sq - dq[:, [3, 0]][:, :, rows]).max() <= 1e-12
    assert np.abs(sk - dk[:, [1]][:, :, keys]).max() <= 1e-12
    assert np.abs(sv - dv[:, [1]][:, :, keys]).max() <= 1e-12


def test_sampled_gradients_of_late_keys_use_only_later_rows():
    # With a causal mask, dK_u and dV_u of late keys need only rows t >= u;
    # the restricted computation must equal the whole backward.
    q, k, v, g = _inputs(41, B=1, hq=4, hkv=2, nq=50, nk=50, d=6, dv=5)
    dq, dk, dv = attention_backward(q, k, v, g, 0.4, True)
    rows, keys = [3, 44], [49, 40, 45]
    sq, sk, sv = attention_backward_sampled(q, k, v, g, 0.4, True, rows, keys)
    assert np.abs(sq - dq[:, :, rows]).max() <= 1e-12
    assert np.abs(sk - dk[:, :, keys]).max() <= 1e-12
    assert np.abs(sv - dv[:, :, keys]).max() <= 1e-12


@pytest.mark.parametrize("striped", [False, True])
def test_block_shares_sum_to_the_whole_gradient(striped):
    # Shares of every (Q_i, KV_j) block against the final LSE and D add up to
    # the whole-row gradients (contiguous and striped positions).
    from oracle.backward import block_backward_share
    n, P = 24, 3
    L = n // P
    q, k, v, g = _inputs(51, B=1, hq=4, hkv=2, nq=n, nk=n, d=5, dv=4)
    o, lse = attention(q, k, v, 0.5, True)
    dlt = row_delta(o, g)
    want = attention_backward(q, k, v, g, 0.5, True)
    pos = lambda r: (np.arange(r, n, P) if striped else np.arange(r * L, (r + 1) * L))  # noqa: E731
    dq = np.zeros(q.shape)
    dk = np.zeros(k.shape)
    dv = np.zeros(v.shape)
    for i in range(P):
        for j in range(P):
            qi, kj = pos(i), pos(j)
            a, b, c = block_backward_share(q[:, :, qi], k[:, :, kj], v[:, :, kj], g[:, :, qi],
                                           lse[:, :, qi], dlt[:, :, qi], 0.5, True, qi, kj)
            dq[:, :, qi] += a
            dk[:, :, kj] += b
            dv[:, :, kj] += c
    for x, y in zip((dq, dk, dv), want):
        assert np.abs(x - y).max() <= 1e-12
