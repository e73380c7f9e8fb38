"""Pins of the oracle's merge, block classification and cost formulas (CPU)."""
import json
import math
import os

import numpy as np
import pytest

from oracle.attention import attention
from oracle.block_class import (FULL, PARTIAL, SKIP, block_class,
                                block_class_bruteforce, partition_class)
from oracle.costs import (decode_latency_lower_bound_s, kv_cache_bytes, prefill_compute_time_s,
                          prefill_time_s, scaling_efficiency,
                          mla_ckv_bytes, pass_kv_bytes_per_chip, prefill_flops)
from oracle.merge import lse_merge

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- merge ----

@pytest.mark.parametrize("causal", [False, True])
def test_merge_of_key_range_partials_is_full_attention(causal):
    rng = np.random.default_rng(50)
    n, d = 60, 8
    q = rng.standard_normal((1, 4, n, d))
    k = rng.standard_normal((1, 2, n, d))
    v = rng.standard_normal((1, 2, n, 6))
    cuts = [0, 7, 20, 21, 45, 60]
    parts = [attention(q, k[:, :, a:b], v[:, :, a:b], 0.3, causal, 0, a)
             for a, b in zip(cuts[:-1], cuts[1:])]
    O, L = lse_merge([p[0] for p in parts], [p[1] for p in parts])
    Of, Lf = attention(q, k, v, 0.3, causal)
    assert np.abs(O - Of).max() <= 1e-12
    assert np.abs(L - Lf).max() <= 1e-12


def test_merge_is_order_free_and_associative():
    rng = np.random.default_rng(51)
    P = 5
    o = rng.standard_normal((P, 3, 7, 4))
    l = rng.standard_normal((P, 3, 7)) * 4
    O, L = lse_merge(o, l)
    perm = rng.permutation(P)
    Op, Lp = lse_merge(o[perm], l[perm])
    assert np.abs(O - Op).max() <= 1e-13 and np.abs(L - Lp).max() <= 1e-13
    Oa, La = lse_merge(o[:2], l[:2])
    Ob, Lb = lse_merge(o[2:], l[2:])
    O2, L2 = lse_merge([Oa, Ob], [La, Lb])
    assert np.abs(O - O2).max() <= 1e-13 and np.abs(L - L2).max() <= 1e-13


def test_merge_empty_partials():
    o = np.ones((3, 2, 4))
    l = np.full((3, 2), -np.inf)
    l[1, 0] = 0.5
    O, L = lse_merge(o * np.arange(3)[:, None, None], l)
    assert np.all(O[1] == 0.0) and L[1] == -np.inf       # every partial empty
    np.testing.assert_array_equal(O[0], np.ones(4))      # only partial 1 counts
    assert L[0] == 0.5


def test_merge_two_equal_lse_halves_weights():
    o = np.array([[[2.0, 0.0]], [[0.0, 4.0]]])
    l = np.array([[1.0], [1.0]])
    O, L = lse_merge(o, l)
    np.testing.assert_allclose(O[0], [1.0, 2.0], atol=1e-15)
    assert L[0] == pytest.approx(1.0 + math.log(2.0), abs=1e-15)


# --------------------------------------------------------- classification --

@pytest.mark.parametrize("nq,nk", [(1, 1), (7, 7), (16, 16), (33, 17), (64, 64), (100, 130)])
@pytest.mark.parametrize("bq,bk", [(1, 1), (4, 4), (8, 16), (16, 8), (32, 32)])
def test_class_matches_bruteforce_mask(nq, nk, bq, bk):
    for qo, ko in [(0, 0), (5, 0), (0, 9), (31, 17), (100, 3)]:
        for causal in (True, False):
            a = block_class(nq, nk, bq, bk, qo, ko, causal)
            b = block_class_bruteforce(nq, nk, bq, bk, qo, ko, causal)
            np.testing.assert_array_equal(a, b)


def test_class_exhaustive_small():
    for n in range(1, 40, 3):
        for bq in (1, 2, 3, 8, 16):
            for bk in (1, 4, 5, 16):
                for off in (-3, 0, 2):
                    a = block_class(n, n, bq, bk, max(off, 0), max(-off, 0), True)
                    b = block_class_bruteforce(n, n, bq, bk, max(off, 0), max(-off, 0), True)
                    np.testing.assert_array_equal(a, b)


@pytest.mark.parametrize("n,P,counts", [
    (131072, 8, (28, 8, 28)),     # (SKIP, PARTIAL, FULL): strict lower triangle FULL
    (262144, 16, (120, 16, 120)),
    (8192, 4, (6, 4, 6)),
])
def test_partition_class_counts(n, P, counts):
    m = partition_class(n, P, True)
    assert ((m == SKIP).sum(), (m == PARTIAL).sum(), (m == FULL).sum()) == counts
    assert all(m[i, i] == PARTIAL for i in range(P))
    assert all(m[i, j] == (FULL if j < i else SKIP) for i in range(P) for j in range(P) if i != j)
    assert (partition_class(n, P, False) == FULL).all()


# ---------------------------------------------------------------- costs ----

def test_kv_cache_table():
    g = json.load(open(os.path.join(GOLDEN, "kv_cache_sizes.json")))
    for row in g["rows"]:
        b = kv_cache_bytes(g["L"], g["h_kv"], g["d_h"], row["n"], g["b"])
        assert b / 2**30 == row["gib"]


def test_decode_latency_table():
    g = json.load(open(os.path.join(GOLDEN, "decode_latency.json")))
    for row in g["rows"]:
        t = decode_latency_lower_bound_s(row["kv_gib"] * 1e9, g["hbm_bytes_per_s"])
        assert abs(t * 1e3 - row["ms"]) / row["ms"] <= 0.10
    # the per-card KV at 32K and 128K is the 70B total divided by TP = 4
    kv = json.load(open(os.path.join(GOLDEN, "kv_cache_sizes.json")))
    tot = {r["n"]: r["gib"] for r in kv["rows"]}
    for row in g["rows"][:2]:
        assert tot[row["n"]] / 4 == row["kv_gib"]


def test_mla_ckv():
    g = json.load(open(os.path.join(GOLDEN, "mla_ckv.json")))
    assert mla_ckv_bytes(g["kv_lora_rank"], 64, g["bytes_per_value"]) == g["c_kv_bytes_per_token_per_layer"]


def test_prefill_flops_counts_pairs():
    # 2 FLOP per multiply-add, one QK^T dot of length d_qk and one PV row of
    # length d_v per visible (query, key) pair: count the pairs by brute force
    for n, dqk, dv, H in [(16, 8, 4, 2), (64, 192, 128, 3)]:
        pairs = sum(1 for t in range(n) for u in range(n))
        assert prefill_flops(1, n, dqk, dv, H, causal=False) == 2 * pairs * (dqk + dv) * H
        causal_pairs = sum(1 for t in range(n) for u in range(t + 1))
        f = prefill_flops(1, n, dqk, dv, H, causal=True)
        assert f == (n * n) * (dqk + dv) * H            # the 1/2 convention
        assert abs(f - 2 * causal_pairs * (dqk + dv) * H) / f == pytest.approx(1 / n)


def test_pass_kv_bytes():
    assert pass_kv_bytes_per_chip(1, 1000, 1152) == 0
    assert pass_kv_bytes_per_chip(8, 1 << 20, 1152) == 7 * (1 << 20) * 1152 / 8


def test_prefill_compute_time_is_the_pair_count_split_over_chips():
    # T_comp * cp * R is the non-causal FLOP count, itself pinned by counting
    # (query, key) pairs above; the time falls as 1 / cp
    for B, S, dqk, dv in [(1, 64, 192, 128), (2, 1 << 17, 128, 128)]:
        for cp in (1, 2, 8):
            t = prefill_compute_time_s(B, S, dqk, dv, cp, 1e15)
            assert t * cp * 1e15 == pytest.approx(prefill_flops(B, S, dqk, dv, 1, causal=False))
        assert prefill_compute_time_s(B, S, dqk, dv, 1, 1e15) == pytest.approx(
            4 * prefill_compute_time_s(B, S, dqk, dv, 4, 1e15))


def test_scaling_efficiency_hidden_and_exposed_regimes():
    # the page's model: T(cp) = max(T_comp(cp), pass-KV bytes / bandwidth).
    # While the exchange hides under the computation the speed-up is cp
    # (eta = 1); once it is exposed the speed-up is below cp and falls as the
    # link gets slower (the page's validation criteria).
    B, S, dqk, dv, R, c_kv = 1, 1 << 17, 192, 128, 1e15, 576
    t1 = prefill_time_s(prefill_compute_time_s(B, S, dqk, dv, 1, R),
                        pass_kv_bytes_per_chip(1, S, c_kv) / 1e9)
    for cp in (2, 4, 8, 16):
        t_comp = prefill_compute_time_s(B, S, dqk, dv, cp, R)
        prev = None
        for bw in (1e12, 1e9, 1e6, 1e5, 1e4, 1e3):
            t_kv = pass_kv_bytes_per_chip(cp, S, c_kv) / bw
            t = prefill_time_s(t_comp, t_kv)
            eta = scaling_efficiency(t1, t, cp)
            speedup = t1 / t
            if t_kv <= t_comp:
                assert eta == pytest.approx(1.0) and speedup == pytest.approx(cp)
            else:
                assert speedup < cp and eta < 1
                assert prev is None or speedup < prev
                prev = speedup
        assert prev is not None             # the sweep reached the exposed regime
    assert scaling_efficiency(3.0, 3.0, 1) == 1.0
