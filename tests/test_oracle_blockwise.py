"""Pins of the oracle against the method's invariants (CPU only).

The pages' blockwise ring algorithm, written out step by step in
``oracle.blockwise``, must equal the plain definition in ``oracle.attention``
for any number of partitions and any block order (exact in real arithmetic);
P = 1 must reduce to plain attention; and the schedule must match the pages'
4-GPU worked example.
"""
import json
import math
import os

import numpy as np
import pytest

from oracle.attention import attention
from oracle.blockwise import (partition_bounds, ring_attention_normalised,
                              ring_attention_online, ring_order)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _inputs(seed, B=1, hq=2, hkv=1, n=24, d=8, dv=8):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((B, hq, n, d)), rng.standard_normal((B, hkv, n, d)),
            rng.standard_normal((B, hkv, n, dv)))


@pytest.mark.parametrize("form", [ring_attention_normalised, ring_attention_online])
@pytest.mark.parametrize("causal", [False, True])
def test_single_partition_is_plain_attention(form, causal):
    q, k, v = _inputs(10, n=20)
    O, L = attention(q, k, v, 0.35, causal)
    Ob, Lb = form(q, k, v, 1, 0.35, causal)
    assert np.abs(O - Ob).max() <= 1e-12
    assert np.abs(L - Lb).max() <= 1e-12


@pytest.mark.parametrize("form", [ring_attention_normalised, ring_attention_online])
@pytest.mark.parametrize("P", [2, 3, 4, 8])
@pytest.mark.parametrize("causal", [False, True])
def test_any_partition_count_equals_full(form, P, causal):
    q, k, v = _inputs(20 + P, B=2, hq=4, hkv=2, n=48, d=8, dv=5)
    O, L = attention(q, k, v, 1 / math.sqrt(8), causal)
    Ob, Lb = form(q, k, v, P, 1 / math.sqrt(8), causal)
    assert np.abs(O - Ob).max() <= 1e-12
    assert np.abs(L - Lb).max() <= 1e-12


@pytest.mark.parametrize("form", [ring_attention_normalised, ring_attention_online])
@pytest.mark.parametrize("causal", [False, True])
def test_block_order_does_not_matter(form, causal):
    q, k, v = _inputs(30, hq=2, hkv=2, n=40, d=6, dv=6)
    P = 8
    rng = np.random.default_rng(31)
    perms = [list(rng.permutation(P)) for _ in range(P)]
    O, L = attention(q, k, v, 0.5, causal)
    Ob, Lb = form(q, k, v, P, 0.5, causal, order=lambda i: perms[i])
    assert np.abs(O - Ob).max() <= 1e-12
    assert np.abs(L - Lb).max() <= 1e-12


def test_large_score_spread_stays_exact():
    # scores spanning hundreds of nats exercise the rescale path of both folds
    q, k, v = _inputs(40, n=32, d=4, dv=3)
    q *= 12.0
    O, L = attention(q, k, v, 1.0, True)
    for form in (ring_attention_normalised, ring_attention_online):
        Ob, Lb = form(q, k, v, 4, 1.0, True)
        assert np.abs(O - Ob).max() <= 1e-11
        assert np.abs(L - Lb).max() <= 1e-10 * max(1.0, np.abs(L).max())


def test_schedule_matches_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "ring_schedule.json")))
    P = g["P"]
    assert [ring_order(P, i)[0] for i in range(P)] == g["step0"]
    assert ring_order(P, 0)[1] == g["step1_gpu0"]
    assert ring_order(P, 1)[1] == g["step1_gpu1"]
    for i in range(P):  # every query partition meets every KV partition once
        assert sorted(ring_order(P, i)) == list(range(P))
    ex = g["partition_example"]
    bounds = partition_bounds(ex["n"], ex["P"])
    assert all(b - a == ex["tokens_per_gpu"] for a, b in bounds)
    assert all(bounds[i][1] == bounds[i + 1][0] for i in range(len(bounds) - 1))
    assert bounds[0][0] == 0 and bounds[-1][1] == ex["n"]


def test_ring_order_is_receive_from_previous():
    # the KV block device i holds at step s+1 is the one device i-1 held at step s
    for P in (2, 3, 5, 8, 16):
        for s in range(P - 1):
            for i in range(P):
                assert ring_order(P, i)[s + 1] == ring_order(P, (i - 1) % P)[s]


def test_uneven_split_rejected():
    with pytest.raises(ValueError):
        partition_bounds(10, 4)


# ---------------------------------------------------------- striped split --

def _brute_positions(q, k, v, scale, qp, kp):
    import math as m
    nq, d = q.shape
    nk = k.shape[0]
    O = np.zeros((nq, v.shape[1]))
    L = np.zeros(nq)
    for t in range(nq):
        vis = [u for u in range(nk) if kp[u] <= qp[t]]
        if not vis:
            L[t] = -np.inf
            continue
        s = {u: scale * m.fsum(q[t, c] * k[u, c] for c in range(d)) for u in vis}
        mx = max(s.values())
        lse = mx + m.log(m.fsum(m.exp(s[u] - mx) for u in vis))
        L[t] = lse
        for c in range(v.shape[1]):
            O[t, c] = m.fsum(m.exp(s[u] - lse) * v[u, c] for u in vis)
    return O, L


def test_explicit_positions_match_brute_force():
    from oracle.blockwise import striped_positions
    rng = np.random.default_rng(60)
    n, P = 12, 3
    q = rng.standard_normal((1, 1, 4, 5))
    k = rng.standard_normal((1, 1, 4, 5))
    v = rng.standard_normal((1, 1, 4, 3))
    for i in range(P):
        for j in range(P):
            qp, kp = striped_positions(n, P, i), striped_positions(n, P, j)
            O, L = attention(q, k, v, 0.6, True, q_positions=qp, k_positions=kp)
            Ob, Lb = _brute_positions(q[0, 0], k[0, 0], v[0, 0], 0.6, qp, kp)
            fin = np.isfinite(Lb)
            assert np.array_equal(np.isfinite(L[0, 0]), fin)
            assert np.abs(O[0, 0] - Ob).max() <= 1e-12
            assert np.abs(L[0, 0][fin] - Lb[fin]).max() <= 1e-12


def test_striped_layout_is_a_permutation_of_full_attention():
    from ring_context_parallelism_ra_b200.workloads import striped_order
    rng = np.random.default_rng(61)
    n, P = 24, 4
    q = rng.standard_normal((1, 2, n, 6))
    k = rng.standard_normal((1, 1, n, 6))
    v = rng.standard_normal((1, 1, n, 4))
    order = np.array(striped_order(n, P))
    assert sorted(order.tolist()) == list(range(n))
    assert order[1] == P and order[n // P] == 1          # row r of partition i is r*P + i
    O, L = attention(q, k, v, 0.4, True)
    Os, Ls = attention(q[:, :, order], k[:, :, order], v[:, :, order], 0.4, True,
                       q_positions=order, k_positions=order)
    assert np.abs(Os - O[:, :, order]).max() <= 1e-12
    assert np.abs(Ls - L[:, :, order]).max() <= 1e-12


def test_striped_blocks_are_balanced():
    # contiguous split: block (i, j) has L^2, L(L+1)/2 or 0 visible pairs;
    # striped split: L(L+1)/2 for j <= i and L(L-1)/2 for j > i (every block
    # about half full, the page's reason for striping)
    from oracle.blockwise import striped_block_visible
    for n, P in [(16, 4), (48, 3), (64, 8)]:
        L = n // P
        for i in range(P):
            for j in range(P):
                want = L * (L + 1) // 2 if j <= i else L * (L - 1) // 2
                assert striped_block_visible(n, P, i, j) == want
        total = sum(striped_block_visible(n, P, i, j) for i in range(P) for j in range(P))
        assert total == n * (n + 1) // 2
