"""Pins of the fp64 oracle's attention definition (CPU only).

Each test fixes the oracle against something other than itself: brute force
with pure-Python loops, closed forms, and exact invariants of softmax
attention.
"""
import math

import numpy as np
import pytest

from oracle.attention import attention, decode_attention

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _brute(q, k, v, scale, causal, q_off=0, k_off=0):
    """Pure-Python loops with math.fsum; GQA by h // (Hq // Hkv)."""
    B, hq, nq, d = q.shape
    _, hkv, nk, _ = k.shape
    dv = v.shape[-1]
    grp = hq // hkv
    O = np.zeros((B, hq, nq, dv))
    L = np.zeros((B, hq, nq))
    for b in range(B):
        for h in range(hq):
            g = h // grp
            for t in range(nq):
                vis = [u for u in range(nk) if (not causal) or (k_off + u <= q_off + t)]
                if not vis:
                    L[b, h, t] = -math.inf
                    continue
                s = {u: scale * math.fsum(float(q[b, h, t, c]) * float(k[b, g, u, c]) for c in range(d))
                     for u in vis}
                m = max(s.values())
                z = math.fsum(math.exp(s[u] - m) for u in vis)
                lse = m + math.log(z)
                L[b, h, t] = lse
                for c in range(dv):
                    O[b, h, t, c] = math.fsum(math.exp(s[u] - lse) * float(v[b, g, u, c]) for u in vis)
    return O, L


CASES = [
    # B, hq, hkv, nq, nk, dqk, dv, causal, q_off, k_off
    (1, 1, 1, 7, 7, 3, 2, True, 0, 0),
    (1, 1, 1, 9, 9, 4, 4, False, 0, 0),
    (2, 4, 2, 6, 6, 5, 3, True, 0, 0),
    (1, 6, 2, 5, 11, 4, 2, True, 10, 3),
    (1, 2, 1, 8, 5, 3, 3, True, 2, 6),    # some rows see no key
    (1, 2, 2, 16, 16, 6, 4, True, 0, 0),
    (1, 3, 1, 4, 13, 2, 5, False, 0, 0),
]


@pytest.mark.parametrize("case", CASES)
def test_matches_brute_force(case):
    B, hq, hkv, nq, nk, d, dv, causal, qo, ko = case
    rng = np.random.default_rng(hash(case) % 2**32)
    q = rng.standard_normal((B, hq, nq, d))
    k = rng.standard_normal((B, hkv, nk, d))
    v = rng.standard_normal((B, hkv, nk, dv))
    scale = 1.0 / math.sqrt(d)
    O, L = attention(q, k, v, scale, causal, qo, ko, row_chunk=3)
    Ob, Lb = _brute(q, k, v, scale, causal, qo, ko)
    assert np.array_equal(np.isinf(L), np.isinf(Lb))
    fin = np.isfinite(Lb)
    assert np.max(np.abs(L[fin] - Lb[fin])) <= 1e-12
    assert np.max(np.abs(O - Ob)) <= 1e-12
    assert np.all(O[~fin] == 0.0)


def test_two_key_hand_example():
    # q = e1, keys e1 and e2, values e1 and e2, scale 1:
    # scores (1, 0) -> weights e/(1+e), 1/(1+e); LSE = ln(1+e).
    q = np.array([[[[1.0, 0.0]]]])
    k = np.array([[[[1.0, 0.0], [0.0, 1.0]]]])
    v = np.array([[[[1.0, 0.0], [0.0, 1.0]]]])
    O, L = attention(q, k, v, 1.0, False)
    e = math.e
    assert O[0, 0, 0, 0] == pytest.approx(e / (1 + e), abs=1e-15)
    assert O[0, 0, 0, 1] == pytest.approx(1 / (1 + e), abs=1e-15)
    assert L[0, 0, 0] == pytest.approx(math.log(1 + e), abs=1e-15)


@pytest.mark.parametrize("causal", [False, True])
def test_zero_query_gives_uniform_weights(causal):
    rng = np.random.default_rng(1)
    n, d = 40, 8
    q = np.zeros((1, 2, n, d))
    k = rng.standard_normal((1, 1, n, d))
    v = rng.standard_normal((1, 1, n, 3))
    O, L = attention(q, k, v, 0.7, causal)
    for t in range(n):
        cnt = t + 1 if causal else n
        np.testing.assert_allclose(O[0, :, t], np.broadcast_to(v[0, 0, :cnt].mean(0), (2, 3)), atol=1e-13)
        np.testing.assert_allclose(L[0, :, t], math.log(cnt), atol=1e-13)


def test_dominant_key_selects_its_value():
    rng = np.random.default_rng(2)
    n, d = 30, 16
    q = rng.standard_normal((1, 1, n, d))
    k = rng.standard_normal((1, 1, n, d)) * 0.01
    v = rng.standard_normal((1, 1, n, 4))
    t, u = 20, 7
    k[0, 0, u] = 400.0 * q[0, 0, t] / np.linalg.norm(q[0, 0, t])
    O, _ = attention(q, k, v, 1.0, True)
    np.testing.assert_allclose(O[0, 0, t], v[0, 0, u], atol=1e-9)


def test_weights_sum_to_one_and_affine_values():
    rng = np.random.default_rng(3)
    q = rng.standard_normal((1, 4, 33, 8))
    k = rng.standard_normal((1, 2, 33, 8))
    v = rng.standard_normal((1, 2, 33, 5))
    O, L = attention(q, k, v, 0.4, True)
    # sum_u exp(s - LSE) = 1 on every row
    for h in range(4):
        s = 0.4 * q[0, h] @ k[0, h // 2].T
        s[np.triu_indices(33, 1)] = -np.inf
        np.testing.assert_allclose(np.exp(s - L[0, h][:, None]).sum(1), 1.0, atol=1e-13)
    # values enter affinely: v -> a v + c gives O -> a O + c
    O2, L2 = attention(q, k, 3.0 * v - 1.25, 0.4, True)
    np.testing.assert_allclose(O2, 3.0 * O - 1.25, atol=1e-12)
    np.testing.assert_array_equal(L2, L)


def test_noncausal_key_permutation_invariance():
    rng = np.random.default_rng(4)
    q = rng.standard_normal((1, 2, 10, 6))
    k = rng.standard_normal((1, 1, 25, 6))
    v = rng.standard_normal((1, 1, 25, 3))
    perm = rng.permutation(25)
    O, L = attention(q, k, v, 0.5, False)
    Op, Lp = attention(q, k[:, :, perm], v[:, :, perm], 0.5, False)
    np.testing.assert_allclose(Op, O, atol=1e-13)
    np.testing.assert_allclose(Lp, L, atol=1e-13)


def test_causal_output_ignores_future_tokens():
    rng = np.random.default_rng(5)
    n = 48
    q = rng.standard_normal((1, 2, n, 8))
    k = rng.standard_normal((1, 2, n, 8))
    v = rng.standard_normal((1, 2, n, 8))
    O, L = attention(q, k, v, 0.3, True)
    t = 19
    k2, v2 = k.copy(), v.copy()
    k2[:, :, t + 1:] = rng.standard_normal(k2[:, :, t + 1:].shape) * 5
    v2[:, :, t + 1:] = rng.standard_normal(v2[:, :, t + 1:].shape) * 5
    O2, L2 = attention(q, k2, v2, 0.3, True)
    np.testing.assert_array_equal(O2[:, :, :t + 1], O[:, :, :t + 1])
    np.testing.assert_array_equal(L2[:, :, :t + 1], L[:, :, :t + 1])
    assert np.abs(O2[:, :, t + 1:] - O[:, :, t + 1:]).max() > 1e-3


def test_gqa_equals_expanded_mha():
    rng = np.random.default_rng(6)
    q = rng.standard_normal((2, 8, 12, 4))
    k = rng.standard_normal((2, 2, 12, 4))
    v = rng.standard_normal((2, 2, 12, 4))
    O, L = attention(q, k, v, 0.5, True)
    Oe, Le = attention(q, np.repeat(k, 4, axis=1), np.repeat(v, 4, axis=1), 0.5, True)
    np.testing.assert_array_equal(O, Oe)
    np.testing.assert_array_equal(L, Le)


def test_row_subset_and_head_subset_match_full():
    rng = np.random.default_rng(7)
    q = rng.standard_normal((1, 4, 50, 4))
    k = rng.standard_normal((1, 2, 50, 4))
    v = rng.standard_normal((1, 2, 50, 3))
    O, L = attention(q, k, v, 0.5, True)
    rows = np.array([0, 1, 17, 49])
    Os, Ls = attention(q, k, v, 0.5, True, rows=rows, heads=[3, 1])
    # BLAS may round differently for a different row count: 1e-14
    np.testing.assert_allclose(Os, O[:, [3, 1]][:, :, rows], rtol=0, atol=1e-14)
    np.testing.assert_allclose(Ls, L[:, [3, 1]][:, :, rows], rtol=0, atol=1e-14)


def test_decode_is_noncausal_single_row():
    rng = np.random.default_rng(8)
    q = rng.standard_normal((3, 8, 1, 16))
    k = rng.standard_normal((3, 2, 70, 16))
    v = rng.standard_normal((3, 2, 70, 16))
    O, L = decode_attention(q, k, v, 0.25)
    Ob, Lb = _brute(q, k, v, 0.25, False)
    assert np.abs(O - Ob).max() <= 1e-12 and np.abs(L - Lb).max() <= 1e-12
