"""Planted mistakes in the oracle (CPU only).

Each case loads a copy of one oracle module with one plausible mistake
written into its source (a dropped term, a wrong sign, an off-by-one mask, a
wrong head map, a swapped operand), runs that module's pins against the
copy, and requires at least one pin to fail.  The same pins hold for the
unmodified oracle (the ``test_oracle_*`` files); this file shows that they
would notice such a mistake.

A mutation that cannot change any result (an equivalent rewrite) is not
listed: clearing rows whose weights are already zero, or transposing a
product twice, leaves every output as it was.
"""
import math
import os
import types

import numpy as np
import pytest
import torch

from tests.test_oracle_attention import CASES, _brute
from tests.test_oracle_backward import FD_CASES, _fd_grad, _inputs, _torch_attention

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _mutant(module, old, new):
    """oracle/<module>.py with `old` replaced by `new` (every occurrence),
    loaded as a module of the oracle package (its relative imports resolve to
    the unmodified modules)."""
    path = os.path.join(ROOT, "oracle", module + ".py")
    src = open(path).read()
    assert old in src, f"mutation site not found in oracle/{module}.py: {old!r}"
    mod = types.ModuleType(f"oracle._mutant_{module}")
    mod.__package__ = "oracle"
    exec(compile(src.replace(old, new), path, "exec"), mod.__dict__)  # noqa: S102
    return mod


def _holds(check, *args):
    """True when the pin holds for the function under test; an exception
    (a shape error from a wrong operand, say) counts as a failed pin."""
    try:
        check(*args)
        return True
    except Exception:  # noqa: BLE001
        return False


# ------------------------------------------------------------ attention --

def _pin_brute_force(att):
    for case in CASES:
        B, hq, hkv, nq, nk, d, dv, causal, qo, ko = case
        rng = np.random.default_rng(abs(hash(case)) % 2**32)
        q = rng.standard_normal((B, hq, nq, d))
        k = rng.standard_normal((B, hkv, nk, d))
        v = rng.standard_normal((B, hkv, nk, dv))
        o, lse = att(q, k, v, 0.6, causal, q_offset=qo, k_offset=ko)
        wo, wl = _brute(q, k, v, 0.6, causal, qo, ko)
        assert np.allclose(o, wo, atol=1e-12, rtol=0)
        fin = np.isfinite(wl)
        assert (np.isfinite(lse) == fin).all()
        assert np.allclose(lse[fin], wl[fin], atol=1e-12, rtol=0)


def _pin_zero_query(att):
    rng = np.random.default_rng(3)
    n = 9
    q = np.zeros((1, 1, n, 4))
    k = rng.standard_normal((1, 1, n, 4))
    v = rng.standard_normal((1, 1, n, 3))
    o, lse = att(q, k, v, 0.8, True)
    for t in range(n):
        assert abs(lse[0, 0, t] - math.log(t + 1)) <= 1e-12
        assert np.abs(o[0, 0, t] - v[0, 0, :t + 1].mean(axis=0)).max() <= 1e-12


def _pin_causal_independence(att):
    rng = np.random.default_rng(4)
    q, k, v = (rng.standard_normal((1, 2, 10, 3)) for _ in range(3))
    o1, _ = att(q, k, v, 0.5, True)
    k2, v2 = k.copy(), v.copy()
    k2[:, :, 6:] += 5.0
    v2[:, :, 6:] -= 3.0
    o2, _ = att(q, k2, v2, 0.5, True)
    assert np.array_equal(o1[:, :, :6], o2[:, :, :6])


ATTENTION_PINS = [_pin_brute_force, _pin_zero_query, _pin_causal_independence]

ATTENTION_MUTANTS = {
    "scale dropped": ("(q_rows @ k.T) * scale", "(q_rows @ k.T)"),
    "mask off by one": ("k_pos[None, :] <= q_pos[:, None]", "k_pos[None, :] < q_pos[:, None]"),
    "mask reversed": ("k_pos[None, :] <= q_pos[:, None]", "q_pos[:, None] <= k_pos[None, :]"),
    "interleaved GQA map": ("g = h // grp", "g = h % h_kv"),
    "LSE in base 2": ("m_safe + np.log(", "m_safe + np.log2("),
    "max added, not subtracted": ("np.exp(s - m_safe[:, None])", "np.exp(s + m_safe[:, None])"),
    "normalisation dropped": ("o = (e @ v) / np.where(empty, 1.0, z)[:, None]", "o = (e @ v)"),
    "query offset taken from keys": ("q_offset + np.arange(n_q", "k_offset + np.arange(n_q"),
}


def test_attention_pins_hold_for_the_oracle():
    from oracle.attention import attention
    assert all(_holds(p, attention) for p in ATTENTION_PINS)


@pytest.mark.parametrize("name", sorted(ATTENTION_MUTANTS))
def test_attention_pins_catch_planted_mistake(name):
    old, new = ATTENTION_MUTANTS[name]
    att = _mutant("attention", old, new).attention
    assert not all(_holds(p, att) for p in ATTENTION_PINS), name


# ---------------------------------------------------------------- merge --

def _pin_merge_equals_full(merge):
    from oracle.attention import attention
    rng = np.random.default_rng(5)
    q = rng.standard_normal((1, 2, 7, 4))
    k = rng.standard_normal((1, 2, 12, 4))
    v = rng.standard_normal((1, 2, 12, 3))
    want_o, want_l = attention(q, k, v, 0.7, False)
    parts = [attention(q, k[:, :, a:b], v[:, :, a:b], 0.7, False) for a, b in ((0, 3), (3, 8), (8, 12))]
    o, lse = merge(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
    assert np.abs(o - want_o).max() <= 1e-12 and np.abs(lse - want_l).max() <= 1e-12


def _pin_merge_empty(merge):
    o, lse = merge(np.ones((2, 3, 4)), np.full((2, 3), -np.inf))
    assert (o == 0).all() and (lse == -np.inf).all()
    o1 = np.arange(4.0)
    for parts, lses in (([o1, 7 * np.ones(4)], [0.3, -np.inf]),
                        ([7 * np.ones(4), o1], [-np.inf, 0.3])):   # empty partial first
        o, lse = merge(np.stack(parts), np.array(lses))
        assert np.array_equal(o, o1) and lse == 0.3


def _pin_merge_equal_halves(merge):
    a, b = np.array([1.0, -2.0]), np.array([3.0, 4.0])
    o, lse = merge(np.stack([a, b]), np.array([1.5, 1.5]))
    assert np.abs(o - (a + b) / 2).max() <= 1e-15 and abs(lse - (1.5 + math.log(2))) <= 1e-15


MERGE_PINS = [_pin_merge_equals_full, _pin_merge_empty, _pin_merge_equal_halves]

MERGE_MUTANTS = {
    "weight exponent negated": ("w = np.exp(lse_parts - l_ref[None])", "w = np.exp(l_ref[None] - lse_parts)"),
    "LSE without the sum": ("l_ref + np.log(safe)", "l_ref"),
    "normalisation dropped": ("/ safe[..., None]", ""),
    "first partial as the reference": ("l_star = lse_parts.max(axis=0)", "l_star = lse_parts[0]"),
}


def test_merge_pins_hold_for_the_oracle():
    from oracle.merge import lse_merge
    assert all(_holds(p, lse_merge) for p in MERGE_PINS)


@pytest.mark.parametrize("name", sorted(MERGE_MUTANTS))
def test_merge_pins_catch_planted_mistake(name):
    old, new = MERGE_MUTANTS[name]
    merge = _mutant("merge", old, new).lse_merge
    assert not all(_holds(p, merge) for p in MERGE_PINS), name


# ------------------------------------------------------------- backward --

def _pin_finite_differences(bwd):
    from oracle.attention import attention
    for case in FD_CASES:
        hq, hkv, nq, nk, causal, qo, ko = case
        q, k, v, g = _inputs(abs(hash(case)) % 1000, hq=hq, hkv=hkv, nq=nq, nk=nk)
        kw = dict(q_offset=qo, k_offset=ko)
        dq, dk, dv = bwd(q, k, v, g, 0.7, causal, **kw)

        def f():
            return float((attention(q, k, v, 0.7, causal, **kw)[0] * g).sum())
        for got, x in ((dq, q), (dk, k), (dv, v)):
            want = _fd_grad(x, f)
            assert np.abs(got - want).max() <= 1e-7 * max(1.0, np.abs(want).max())


def _pin_autodiff(bwd):
    q, k, v, g = _inputs(5, B=1, hq=4, hkv=2, nq=12, nk=12, d=5, dv=3)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    pos = torch.arange(12)
    (_torch_attention(tq, tk, tv, 0.45, True, pos, pos) * torch.tensor(g)).sum().backward()
    dq, dk, dv = bwd(q, k, v, g, 0.45, True, row_chunk=5)
    for got, t in ((dq, tq), (dk, tk), (dv, tv)):
        assert np.abs(got - t.grad.numpy()).max() <= 1e-12


def _pin_identities(bwd):
    q, k, v, g = _inputs(8, hq=4, hkv=2, nq=10, nk=10, d=5, dv=3)
    _, dk, dv = bwd(q, k, v, g, 0.4, True)
    assert np.abs(dk.sum(axis=2)).max() <= 1e-12
    want = g.reshape(1, 2, 2, 10, 3).sum(axis=(2, 3))
    assert np.abs(dv.sum(axis=2) - want).max() <= 1e-12


BACKWARD_PINS = [_pin_finite_differences, _pin_autodiff, _pin_identities]

BACKWARD_MUTANTS = {
    "row term D dropped": ("ds = p * (dp - d_row[:, None])", "ds = p * dp"),
    "scale dropped from dQ": ("dq[b, h, r] = scale * (ds @ kk)", "dq[b, h, r] = ds @ kk"),
    "dK from P instead of dS": ("dk[b, g] += scale * (ds.T @ qh[r])", "dk[b, g] += scale * (p.T @ qh[r])"),
    "dV overwritten across a group": ("dv[b, g] += p.T @ doh[r]", "dv[b, g] = p.T @ doh[r]"),
    "D summed over the wrong axis": ("d_row = (doh[r] * o).sum(axis=1)", "d_row = (doh[r] * o).sum(axis=0)"),
    "dS sign flipped": ("ds = p * (dp - d_row[:, None])", "ds = p * (d_row[:, None] - dp)"),
}


def test_backward_pins_hold_for_the_oracle():
    from oracle.backward import attention_backward
    assert all(_holds(p, attention_backward) for p in BACKWARD_PINS)


@pytest.mark.parametrize("name", sorted(BACKWARD_MUTANTS))
def test_backward_pins_catch_planted_mistake(name):
    old, new = BACKWARD_MUTANTS[name]
    bwd = _mutant("backward", old, new).attention_backward
    assert not all(_holds(p, bwd) for p in BACKWARD_PINS), name


# ------------------------------------------------------------ blockwise --

def _pin_ring_equals_definition(mod):
    from oracle.attention import attention
    rng = np.random.default_rng(6)
    q = rng.standard_normal((1, 4, 24, 5)) * 2.0     # wide score spread: maxima move
    k = rng.standard_normal((1, 2, 24, 5)) * 2.0
    v = rng.standard_normal((1, 2, 24, 3))
    for causal in (True, False):
        want_o, want_l = attention(q, k, v, 0.6, causal)
        for P in (1, 2, 3, 4, 8):
            for ring in (mod.ring_attention_normalised, mod.ring_attention_online):
                o, lse = ring(q, k, v, P, 0.6, causal)
                assert np.abs(o - want_o).max() <= 1e-12
                assert np.abs(lse - want_l).max() <= 1e-12


def _pin_ring_any_block_order(mod):
    from oracle.attention import attention
    rng = np.random.default_rng(7)
    q, k, v = (rng.standard_normal((1, 1, 20, 4)) for _ in range(3))
    want_o, _ = attention(q, k, v, 0.5, True)
    perms = [list(rng.permutation(4)) for _ in range(4)]
    for ring in (mod.ring_attention_normalised, mod.ring_attention_online):
        o, _ = ring(q, k, v, 4, 0.5, True, order=lambda i: perms[i])
        assert np.abs(o - want_o).max() <= 1e-12


BLOCKWISE_PINS = [_pin_ring_equals_definition, _pin_ring_any_block_order]

BLOCKWISE_MUTANTS = {
    "beta exponent negated": ("np.exp(old_safe - new_lse)", "np.exp(new_lse - old_safe)"),
    "gamma without the block sum": ("gamma = w_sum * np.exp(max_val - new_lse)",
                                    "gamma = np.exp(max_val - new_lse)"),
    "running sum not rescaled": ("l = alpha * l + p.sum(axis=1)", "l = l + p.sum(axis=1)"),
    "accumulator not rescaled": ("acc = alpha[:, None] * acc + p @ v_blk", "acc = acc + p @ v_blk"),
    "diagonal block skipped": ("if causal and k0 > q1 - 1:", "if causal and k0 >= q0:"),
    "interleaved GQA map": ("g = h // grp", "g = h % h_kv"),
}


def test_blockwise_pins_hold_for_the_oracle():
    import oracle.blockwise as mod
    assert all(_holds(p, mod) for p in BLOCKWISE_PINS)


@pytest.mark.parametrize("name", sorted(BLOCKWISE_MUTANTS))
def test_blockwise_pins_catch_planted_mistake(name):
    old, new = BLOCKWISE_MUTANTS[name]
    mod = _mutant("blockwise", old, new)
    assert not all(_holds(p, mod) for p in BLOCKWISE_PINS), name


# ----------------------------------------------- blockwise backward forms --

def _pin_ring_backward_equals_whole(mod):
    from oracle.backward import attention_backward     # the unmodified oracle
    rng = np.random.default_rng(12)
    q = rng.standard_normal((1, 4, 12, 3))
    k = rng.standard_normal((1, 2, 12, 3))
    v = rng.standard_normal((1, 2, 12, 2))
    g = rng.standard_normal((1, 4, 12, 2))
    for causal in (True, False):
        want = attention_backward(q, k, v, g, 0.6, causal)
        for P in (1, 2, 3, 4):
            got = mod.ring_attention_backward(q, k, v, g, 0.6, causal, P)
            for a, b in zip(got, want):
                assert np.abs(a - b).max() <= 1e-12


def _pin_block_shares_sum_to_whole(mod):
    from oracle.attention import attention
    from oracle.backward import attention_backward, row_delta
    rng = np.random.default_rng(13)
    n, P = 12, 3
    q = rng.standard_normal((1, 2, n, 3))
    k = rng.standard_normal((1, 1, n, 3))
    v = rng.standard_normal((1, 1, n, 2))
    g = rng.standard_normal((1, 2, n, 2))
    o, lse = attention(q, k, v, 0.5, True)
    d = row_delta(o, g)
    dq, dk, dv = np.zeros(q.shape), np.zeros(k.shape), np.zeros(v.shape)
    L = n // P
    pos = np.arange(n)
    for i in range(P):
        r = slice(i * L, (i + 1) * L)
        for j in range(P):
            c = slice(j * L, (j + 1) * L)
            a, b, e = mod.block_backward_share(q[:, :, r], k[:, :, c], v[:, :, c], g[:, :, r],
                                               lse[:, :, r], d[:, :, r], 0.5, True, pos[r], pos[c])
            dq[:, :, r] += a
            dk[:, :, c] += b
            dv[:, :, c] += e
    for x, w in zip((dq, dk, dv), attention_backward(q, k, v, g, 0.5, True)):
        assert np.abs(x - w).max() <= 1e-12


BLOCK_BACKWARD_PINS = [_pin_ring_backward_equals_whole, _pin_block_shares_sum_to_whole]

BLOCK_BACKWARD_MUTANTS = {
    "dK share delivered to the query partition": (
        "dk[b, g, k0:k1] += scale * (ds.T @ qh[q0:q1])", "dk[b, g, q0:q1] += scale * (ds.T @ qh[q0:q1])"),
    "block-local softmax instead of the final LSE": (
        "p[live] = np.exp(s[live] - lse_i[live, None])",
        "p[live] = np.exp(s[live] - s[live].max(axis=1, keepdims=True))"),
    "diagonal blocks skipped": ("if not vis.any():", "if not vis.all():"),
    "D of the key rows": ("ds = p * (dp - dlt[b, h, q0:q1, None])", "ds = p * (dp - dlt[b, h, k0:k1, None])"),
    "block share without D": ("ds = p * (doh @ vv.T - delta[b, h][:, None])", "ds = p * (doh @ vv.T)"),
    "block share mask off by one": ("s = np.where(kp[None, :] <= qp[:, None], s, -np.inf)",
                                    "s = np.where(kp[None, :] < qp[:, None], s, -np.inf)"),
}


def test_block_backward_pins_hold_for_the_oracle():
    import oracle.backward as mod
    assert all(_holds(p, mod) for p in BLOCK_BACKWARD_PINS)


@pytest.mark.parametrize("name", sorted(BLOCK_BACKWARD_MUTANTS))
def test_block_backward_pins_catch_planted_mistake(name):
    old, new = BLOCK_BACKWARD_MUTANTS[name]
    mod = _mutant("backward", old, new)
    assert not all(_holds(p, mod) for p in BLOCK_BACKWARD_PINS), name


# ------------------------------------------------- classification, costs --

def _pin_class_matches_mask(mod):
    from oracle.block_class import block_class_bruteforce   # the unmodified rule
    for n, bq, bk in ((37, 8, 5), (64, 16, 16), (20, 3, 4)):
        for qo, ko in ((0, 0), (5, 0), (0, 9)):
            for causal in (True, False):
                a = mod.block_class(n, n, bq, bk, qo, ko, causal)
                b = block_class_bruteforce(n, n, bq, bk, qo, ko, causal)
                assert np.array_equal(a, b)


def _pin_partition_counts(mod):
    m = mod.partition_class(8192, 4)
    assert [(m == c).sum() for c in (0, 1, 2)] == [6, 4, 6]


CLASS_PINS = [_pin_class_matches_mask, _pin_partition_counts]

CLASS_MUTANTS = {
    "visible count off by one": ("vis = np.clip(q_pos - (k_offset + k_start) + 1, 0, k_len)",
                                 "vis = np.clip(q_pos - (k_offset + k_start), 0, k_len)"),
    "FULL when any row sees the whole tile": ("if (r == k_len).all():", "if (r == k_len).any():"),
    "query positions from the key offset": ("q_pos = q_offset + np.arange", "q_pos = k_offset + np.arange"),
}


def test_class_pins_hold_for_the_oracle():
    import oracle.block_class as mod
    assert all(_holds(p, mod) for p in CLASS_PINS)


@pytest.mark.parametrize("name", sorted(CLASS_MUTANTS))
def test_class_pins_catch_planted_mistake(name):
    old, new = CLASS_MUTANTS[name]
    assert not all(_holds(p, _mutant("block_class", old, new)) for p in CLASS_PINS), name


def _pin_flops_count_pairs(mod):
    for n, dqk, dv, H in ((16, 8, 4, 2), (12, 192, 128, 3)):
        pairs = n * n
        assert mod.prefill_flops(1, n, dqk, dv, H, causal=False) == 2 * pairs * (dqk + dv) * H
        assert mod.prefill_flops(1, n, dqk, dv, H, causal=True) == pairs * (dqk + dv) * H


def _pin_kv_table_and_ring_bytes(mod):
    import json
    g = json.load(open(os.path.join(ROOT, "tests", "golden", "kv_cache_sizes.json")))
    for row in g["rows"]:
        assert mod.kv_cache_bytes(g["L"], g["h_kv"], g["d_h"], row["n"], g["b"]) / 2**30 == row["gib"]
    assert mod.pass_kv_bytes_per_chip(1, 1000, 1152) == 0          # one chip sends nothing


COST_PINS = [_pin_flops_count_pairs, _pin_kv_table_and_ring_bytes]

COST_MUTANTS = {
    "heads not counted": ("f = 2 * B * S * S * (d_qk + d_v) * heads", "f = 2 * B * S * S * (d_qk + d_v)"),
    "causal not halved": ("return f // 2 if causal else f\n\n\ndef backward_flops",
                          "return f\n\n\ndef backward_flops"),
    "K or V missing from the cache": ("return 2 * L * h_kv * d_h * n * b", "return L * h_kv * d_h * n * b"),
    "ring bytes without the (cp - 1) / cp factor": ("return (cp - 1) * S * c_kv / cp", "return S * c_kv / cp"),
}


def test_cost_pins_hold_for_the_oracle():
    import oracle.costs as mod
    assert all(_holds(p, mod) for p in COST_PINS)


@pytest.mark.parametrize("name", sorted(COST_MUTANTS))
def test_cost_pins_catch_planted_mistake(name):
    old, new = COST_MUTANTS[name]
    assert not all(_holds(p, _mutant("costs", old, new)) for p in COST_PINS), name
