"""Randomised properties of the oracle (CPU only, hypothesis).

Shapes, offsets, head groupings and partition counts are drawn at random;
each property is a fact of the mathematics, independent of the oracle's code:
agreement with the pure-Python brute force, independence of the merge from
the order and grouping of its partials, equality of the blockwise ring with
the full-row definition, and the tile classification against the explicit
boolean mask.
"""
import numpy as np
import pytest
from hypothesis import given, settings
from hypothesis import strategies as st

from oracle.attention import attention
from oracle.block_class import block_class, block_class_bruteforce
from oracle.blockwise import ring_attention_normalised, ring_attention_online
from oracle.merge import lse_merge
from tests.test_oracle_attention import _brute

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")

SETTINGS = settings(max_examples=40, deadline=None, derandomize=True)


@SETTINGS
@given(B=st.integers(1, 2), hkv=st.integers(1, 2), grp=st.integers(1, 3), nq=st.integers(1, 7),
       nk=st.integers(1, 7), d=st.integers(1, 4), dv=st.integers(1, 3), causal=st.booleans(),
       qo=st.integers(0, 6), ko=st.integers(0, 6), seed=st.integers(0, 2**31 - 1))
def test_attention_equals_brute_force(B, hkv, grp, nq, nk, d, dv, causal, qo, ko, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, hkv * grp, nq, d))
    k = rng.standard_normal((B, hkv, nk, d))
    v = rng.standard_normal((B, hkv, nk, dv))
    o, lse = attention(q, k, v, 0.7, causal, q_offset=qo, k_offset=ko)
    wo, wl = _brute(q, k, v, 0.7, causal, qo, ko)
    assert np.allclose(o, wo, atol=1e-12, rtol=0)
    fin = np.isfinite(wl)
    assert (np.isfinite(lse) == fin).all()
    assert np.allclose(lse[fin], wl[fin], atol=1e-12, rtol=0)


@SETTINGS
@given(n=st.integers(2, 16), cuts=st.lists(st.integers(1, 15), min_size=1, max_size=4, unique=True),
       seed=st.integers(0, 2**31 - 1), causal=st.booleans())
def test_merge_of_any_key_split_in_any_order_is_full_attention(n, cuts, seed, causal):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((1, 2, n, 3)) * 2
    k = rng.standard_normal((1, 2, n, 3)) * 2
    v = rng.standard_normal((1, 2, n, 2))
    edges = sorted({0, n} | {c for c in cuts if c < n})
    parts = [attention(q, k[:, :, a:b], v[:, :, a:b], 0.8, causal, k_offset=a)
             for a, b in zip(edges[:-1], edges[1:])]
    perm = rng.permutation(len(parts))
    o, lse = lse_merge(np.stack([parts[i][0] for i in perm]), np.stack([parts[i][1] for i in perm]))
    want_o, want_l = attention(q, k, v, 0.8, causal)
    assert np.abs(o - want_o).max() <= 1e-12
    fin = np.isfinite(want_l)
    assert np.abs(lse[fin] - want_l[fin]).max() <= 1e-12 and (lse[~fin] == -np.inf).all()


@SETTINGS
@given(P=st.integers(1, 6), L=st.integers(1, 4), grp=st.integers(1, 2), causal=st.booleans(),
       seed=st.integers(0, 2**31 - 1), online=st.booleans())
def test_ring_equals_definition_for_any_partition_count(P, L, grp, causal, seed, online):
    rng = np.random.default_rng(seed)
    n = P * L
    q = rng.standard_normal((1, 2 * grp, n, 3)) * 1.5
    k = rng.standard_normal((1, 2, n, 3)) * 1.5
    v = rng.standard_normal((1, 2, n, 2))
    ring = ring_attention_online if online else ring_attention_normalised
    order = [list(rng.permutation(P)) for _ in range(P)]
    o, lse = ring(q, k, v, P, 0.6, causal, order=lambda i: order[i])
    want_o, want_l = attention(q, k, v, 0.6, causal)
    assert np.abs(o - want_o).max() <= 1e-12 and np.abs(lse - want_l).max() <= 1e-12


@SETTINGS
@given(nq=st.integers(1, 40), nk=st.integers(1, 40), bq=st.integers(1, 9), bk=st.integers(1, 9),
       qo=st.integers(0, 30), ko=st.integers(0, 30), causal=st.booleans())
def test_tile_class_equals_mask(nq, nk, bq, bk, qo, ko, causal):
    assert np.array_equal(block_class(nq, nk, bq, bk, qo, ko, causal),
                          block_class_bruteforce(nq, nk, bq, bk, qo, ko, causal))


@SETTINGS
@given(P=st.integers(1, 5), L=st.integers(1, 4), grp=st.integers(1, 2), causal=st.booleans(),
       seed=st.integers(0, 2**31 - 1))
def test_ring_backward_equals_whole_rows(P, L, grp, causal, seed):
    from oracle.backward import attention_backward, ring_attention_backward
    rng = np.random.default_rng(seed)
    n = P * L
    q = rng.standard_normal((1, 2 * grp, n, 3))
    k = rng.standard_normal((1, 2, n, 3))
    v = rng.standard_normal((1, 2, n, 2))
    g = rng.standard_normal((1, 2 * grp, n, 2))
    order = [list(rng.permutation(P)) for _ in range(P)]
    got = ring_attention_backward(q, k, v, g, 0.5, causal, P, order=lambda P_, i: order[i])
    for a, b in zip(got, attention_backward(q, k, v, g, 0.5, causal)):
        assert np.abs(a - b).max() <= 1e-12


@SETTINGS
@given(nq=st.integers(2, 6), nk=st.integers(2, 6), grp=st.integers(1, 2), causal=st.booleans(),
       qo=st.integers(0, 4), seed=st.integers(0, 2**31 - 1))
def test_backward_equals_autodiff(nq, nk, grp, causal, qo, seed):
    import torch

    from oracle.backward import attention_backward
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((1, 2 * grp, nq, 3))
    k = rng.standard_normal((1, 2, nk, 3))
    v = rng.standard_normal((1, 2, nk, 2))
    g = rng.standard_normal((1, 2 * grp, nq, 2))
    qpos, kpos = qo + np.arange(nq), np.arange(nk)
    if causal and (kpos[0] > qpos).any():
        return            # rows that see no key have no softmax to differentiate
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    kk = tk.repeat_interleave(grp, dim=1)
    vv = tv.repeat_interleave(grp, dim=1)
    s = torch.einsum("bhtc,bhuc->bhtu", tq, kk) * 0.9
    if causal:
        s = s.masked_fill(torch.tensor(kpos[None, :] > qpos[:, None]), float("-inf"))
    o = torch.einsum("bhtu,bhuc->bhtc", torch.softmax(s, dim=-1), vv)
    (o * torch.tensor(g)).sum().backward()
    got = attention_backward(q, k, v, g, 0.9, causal, q_offset=qo)
    for a, t in zip(got, (tq, tk, tv)):
        assert np.abs(a - t.grad.numpy()).max() <= 1e-12
