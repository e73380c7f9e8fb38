"""GPU parity of the backward pass (dQ, dK, dV) against the fp64 oracle on the
same seeded inputs: the fused ring backward (contiguous and striped), the
per-block shares that a device of the ring adds up, D = rowsum(dO * O), the
causal dependence pattern, and a sampled check at the 8K MHA workload size.
The forward's own outputs (O, LSE) feed the backward, as in training."""
import math
import zlib

import numpy as np
import pytest
import torch

from oracle.attention import attention as oracle_attention
from oracle.backward import attention_backward, attention_backward_sampled, row_delta
from ring_context_parallelism_ra_b200 import ra
from ring_context_parallelism_ra_b200.workloads import (make_dout, make_qkv, striped_order,
                                                        workload)
from tests.parity_util import check_grad, sum_identity_bar, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"
BF, F32 = torch.bfloat16, torch.float32


def _seed(case):
    return zlib.crc32(repr(case).encode()) % 100000


@pytest.fixture(autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    ra.lib()
    yield
    assert ra.get_status() == ra.RA_OK
    torch.cuda.synchronize()


def _kind(dt):
    return "f32" if dt == F32 else "bf16"


RING_CASES = [
    # B, Hq, Hkv, n, dqk, dv, P, causal, dtype
    (1, 2, 1, 320, 128, 128, 2, True, BF),    # ragged last tile (160-token partitions)
    (1, 4, 2, 512, 128, 128, 4, True, BF),    # grouped-query heads
    (2, 2, 2, 384, 128, 128, 3, False, BF),   # non-causal, batch 2
    (1, 2, 1, 256, 64, 64, 2, True, BF),
    (1, 2, 1, 300, 64, 128, 3, True, BF),
    (1, 2, 2, 256, 128, 64, 1, True, BF),
    (1, 1, 1, 512, 64, 64, 4, False, F32),    # shape of the fp32 correctness workload
    (1, 2, 1, 320, 128, 128, 2, True, F32),
    (1, 4, 2, 200, 64, 128, 4, True, F32),
    (1, 2, 2, 96, 128, 128, 8, True, BF),     # 12-token partitions
    (1, 2, 1, 16, 128, 128, 16, True, BF),    # one token per partition
    (1, 1, 1, 1, 128, 128, 1, True, BF),      # a single token: every gradient is 0 but dV
    (1, 4, 2, 320, 192, 128, 2, True, BF),    # MLA-shaped head (its own tensor-core kernel)
    (1, 2, 2, 200, 192, 64, 4, False, BF),
    (1, 8, 1, 257, 192, 128, 1, True, BF),    # d_qk 192: GQA 8:1, ragged tail
    (2, 2, 2, 96, 192, 128, 8, True, BF),     # d_qk 192: 12-token partitions, batch 2
    (1, 1, 1, 1, 192, 128, 1, True, BF),      # d_qk 192: a single token
    (1, 2, 1, 640, 192, 64, 5, True, BF),     # d_qk 192, d_v 64, several key tiles
]


@pytest.mark.parametrize("case", RING_CASES)
def test_ring_backward_matches_oracle(case):
    B, Hq, Hkv, n, dqk, dv, P, causal, dt = case
    seed = _seed(case)
    q, k, v = make_qkv(B, Hq, Hkv, n, n, dqk, dv, dt, seed=seed)
    g = make_dout(B, Hq, n, dv, dt, seed=seed)
    qd, kd, vd, gd = (x.to(DEV) for x in (q, k, v, g))
    scale = 1.0 / math.sqrt(dqk)
    out, lse = ra.ring_forward(qd, kd, vd, P, causal, scale)
    dq, dk, dvv = ra.ring_backward(qd, kd, vd, out, lse, gd, P, causal, scale)
    assert dq.dtype == dt and dk.shape == k.shape and dvv.shape == v.shape
    want = attention_backward(q, k, v, g, scale, causal)
    kind = _kind(dt)
    check_grad(dq, want[0], kind, "dQ")
    check_grad(dk, want[1], kind, "dK")
    check_grad(dvv, want[2], kind, "dV")


@pytest.mark.parametrize("dt", [BF, F32])
def test_backward_delta_matches_oracle(dt):
    B, Hq, n, dv = 2, 3, 333, 128
    q, k, v = make_qkv(B, Hq, Hq, n, n, 128, dv, dt, seed=5)
    g = make_dout(B, Hq, n, dv, dt, seed=5)
    out, _ = ra.ring_forward(q.to(DEV), k.to(DEV), v.to(DEV), 1, True)
    d = ra.backward_delta(out, g.to(DEV))
    want = row_delta(to64(out), g)          # D of the output actually produced
    err = np.abs(to64(d) - want)
    assert err.max() <= 1e-4 * max(1.0, np.abs(want).max())


@pytest.mark.parametrize("dt,d,dvd", [(BF, 128, 128), (F32, 128, 128), (BF, 192, 128)])
def test_block_backward_shares_sum_to_the_gradient(dt, d, dvd):
    # Device i of a P-way ring holds Q_i, dO_i and the final LSE_i, D_i; each
    # KV_j that passes adds its share to dQ_i and to the travelling dK_j, dV_j.
    # Every block is called, the fully masked ones included.
    B, Hq, Hkv, n, P = 1, 4, 2, 512, 4
    L = n // P
    q, k, v = make_qkv(B, Hq, Hkv, n, n, d, dvd, dt, seed=11)
    g = make_dout(B, Hq, n, dvd, dt, seed=11)
    qd, kd, vd, gd = (x.to(DEV) for x in (q, k, v, g))
    out, lse = ra.ring_forward(qd, kd, vd, P, True)
    delta = ra.backward_delta(out, gd)
    part = lambda x, i: x[:, :, i * L:(i + 1) * L].contiguous()  # noqa: E731
    dq = [torch.zeros((B, Hq, L, d), device=DEV) for _ in range(P)]
    dk = [torch.zeros((B, Hkv, L, d), device=DEV) for _ in range(P)]
    dv = [torch.zeros((B, Hkv, L, dvd), device=DEV) for _ in range(P)]
    for i in range(P):
        for s in range(P):
            j = (i - s) % P
            ra.block_backward(part(qd, i), part(kd, j), part(vd, j), part(gd, i), part(lse, i),
                              part(delta, i), q_offset=i * L, k_offset=j * L, causal=True,
                              dq_acc=dq[i], dk_acc=dk[j], dv_acc=dv[j])
    want = attention_backward(q, k, v, g, 1 / math.sqrt(d), True)
    kind = _kind(dt)
    check_grad(torch.cat(dq, 2), want[0], kind, "dQ")
    check_grad(torch.cat(dk, 2), want[1], kind, "dK")
    check_grad(torch.cat(dv, 2), want[2], kind, "dV")


@pytest.mark.parametrize("d", [128, 192])
def test_block_backward_strided_and_ragged(d):
    # One strided block (query partition 2, key partition 1 of a 4-way striped
    # split) with a ragged key count, against the oracle with explicit positions.
    dt, P = BF, 4
    B, Hq, Hkv, nq, nk = 1, 2, 1, 200, 150
    q, k, v = make_qkv(B, Hq, Hkv, nq, nk, d, 128, dt, seed=21)
    g = make_dout(B, Hq, nq, 128, dt, seed=21)
    qp = 2 + P * np.arange(nq)
    kp = 1 + P * np.arange(nk)
    scale = 1 / math.sqrt(d)
    o, l = oracle_attention(q, k, v, scale, True, q_positions=qp, k_positions=kp)
    lse = torch.tensor(l, dtype=torch.float32, device=DEV)
    delta = torch.tensor(row_delta(o, g), dtype=torch.float32, device=DEV)
    dq, dk, dv = ra.block_backward(q.to(DEV), k.to(DEV), v.to(DEV), g.to(DEV), lse, delta,
                                   q_offset=2, k_offset=1, pos_stride=P, causal=True)
    want = attention_backward(q, k, v, g, scale, True, q_positions=qp, k_positions=kp)
    check_grad(dq, want[0], "bf16", "dQ")
    check_grad(dk, want[1], "bf16", "dK")
    check_grad(dv, want[2], "bf16", "dV")


@pytest.mark.parametrize("dt,n,P,d", [(BF, 1024, 4, 128), (F32, 1024, 4, 128), (BF, 768, 3, 192)])
def test_striped_ring_backward_matches_oracle(dt, n, P, d):
    B, Hq, Hkv, dvd = 1, 2, 1, 128
    q, k, v = make_qkv(B, Hq, Hkv, n, n, d, dvd, dt, seed=31)
    g = make_dout(B, Hq, n, dvd, dt, seed=31)
    order = torch.tensor(striped_order(n, P))
    inv = torch.argsort(order)
    qs, ks, vs, gs = (x[:, :, order].contiguous().to(DEV) for x in (q, k, v, g))
    out, lse = ra.ring_forward_striped(qs, ks, vs, P, True)
    dq, dk, dv = ra.ring_backward_striped(qs, ks, vs, out, lse, gs, P, True)
    want = attention_backward(q, k, v, g, 1 / math.sqrt(d), True)
    idx = inv.to(DEV)
    kind = _kind(dt)
    check_grad(dq[:, :, idx], want[0], kind, "dQ")
    check_grad(dk[:, :, idx], want[1], kind, "dK")
    check_grad(dv[:, :, idx], want[2], kind, "dV")


def test_backward_causal_dependence():
    # dK_u, dV_u depend on rows t >= u only; dQ_t on keys u <= t only.
    B, Hq, Hkv, n, d, P = 1, 2, 1, 512, 128, 4
    q, k, v = make_qkv(B, Hq, Hkv, n, n, d, d, BF, seed=41)
    g = make_dout(B, Hq, n, d, BF, seed=41)
    qd, kd, vd, gd = (x.to(DEV) for x in (q, k, v, g))
    out, lse = ra.ring_forward(qd, kd, vd, P, True)
    dq, dk, dv = ra.ring_backward(qd, kd, vd, out, lse, gd, P, True)
    g2 = gd.clone()
    g2[:, :, :200] = 3.0
    _, dk2, dv2 = ra.ring_backward(qd, kd, vd, out, lse, g2, P, True)
    assert torch.equal(dk2[:, :, 200:], dk[:, :, 200:])   # one CTA, fixed order per key tile
    assert torch.equal(dv2[:, :, 200:], dv[:, :, 200:])
    k2, v2 = kd.clone(), vd.clone()
    k2[:, :, 300:] = -2.0
    v2[:, :, 300:] = 5.0
    out2, lse2 = ra.ring_forward(qd, k2, v2, P, True)
    dq2, _, _ = ra.ring_backward(qd, k2, v2, out2, lse2, gd, P, True)
    # dQ sums key tiles with float atomics in arbitrary order, so the fp32 sum
    # may differ in its last bits and the bf16 result by one bf16 step
    a, b = to64(dq2[:, :, :300]), to64(dq[:, :, :300])
    assert (np.abs(a - b) <= 2 ** -7 * np.abs(b) + 1e-6).all()


def test_backward_rejects_what_it_does_not_support():
    q = torch.zeros((1, 1, 256, 96), device=DEV, dtype=BF)
    v = torch.zeros((1, 1, 256, 128), device=DEV, dtype=BF)
    out = torch.zeros((1, 1, 256, 128), device=DEV, dtype=BF)
    lse = torch.zeros((1, 1, 256), device=DEV)
    with pytest.raises(ra.RAError) as e:
        ra.ring_backward(q, q, v, out, lse, out, 2, True)
    assert e.value.status == ra.RA_ERR_UNSUPPORTED


def test_backward_sampled_at_8k_mha_workload():
    # The 8K causal MHA workload (8 heads, d 128, P 4, Q and K scaled by 0.5),
    # the configuration the bench times: exact gradients on sampled rows / keys
    # of every head, plus identities over all keys.
    wl = workload("causal_mha_8k")
    q, k, v = make_qkv(wl.B, wl.Hq, wl.Hkv, wl.n, wl.n, wl.d_qk, wl.d_v, BF, seed=wl.seed,
                       qk_mult=wl.qk_mult, device=DEV)
    g = make_dout(wl.B, wl.Hq, wl.n, wl.d_v, BF, seed=wl.seed, device=DEV)
    out, lse = ra.ring_forward(q, k, v, wl.P, True)
    dq, dk, dv = ra.ring_backward(q, k, v, out, lse, g, wl.P, True)
    assert torch.isfinite(dq.float()).all() and torch.isfinite(dk.float()).all()
    rng = np.random.default_rng(7)
    L = wl.n // wl.P
    edges = sorted({0, 1, wl.n - 1, *[i * L for i in range(wl.P)],
                    *[i * L - 1 for i in range(1, wl.P)], 127, 128, 255})
    sample = np.unique(np.concatenate([edges, rng.choice(wl.n, 120, replace=False)]))
    qc, kc, vc, gc = (x.cpu() for x in (q, k, v, g))
    scale = 1 / math.sqrt(wl.d_qk)
    wq, wk, wv = attention_backward_sampled(qc, kc, vc, gc, scale, True, sample, sample)
    check_grad(dq[:, :, sample], wq, "bf16", "dQ sampled rows")
    check_grad(dk[:, :, sample], wk, "bf16", "dK sampled keys")
    check_grad(dv[:, :, sample], wv, "bf16", "dV sampled keys")
    # identities over every key (per column): sum_u dK_u = 0 and
    # sum_u dV_u = sum_t dO_t.  The longest dK / dV accumulator (the first
    # key tile) takes G * n / 16 steps in tensor memory.
    dk64, dv64 = to64(dk), to64(dv)
    steps = (wl.Hq // wl.Hkv) * wl.n // 16
    assert (np.abs(dk64.sum(axis=2)) <= sum_identity_bar(dk64, steps, 2)).all()
    want_sv = to64(g).reshape(wl.B, wl.Hkv, -1, wl.n, wl.d_v).sum(axis=(2, 3))
    assert (np.abs(dv64.sum(axis=2) - want_sv) <= sum_identity_bar(dv64, steps, 2)).all()


@pytest.mark.parametrize("dt", [BF, F32])
def test_block_backward_rows_without_keys_and_noncausal(dt):
    # Keys placed after every query of the first rows: those rows see no key
    # (LSE -inf) and get no gradient; a non-causal block with a ragged tail.
    B, Hq, Hkv, nq, nk, d = 1, 8, 1, 200, 130, 64
    q, k, v = make_qkv(B, Hq, Hkv, nq, nk, d, d, dt, seed=81)
    g = make_dout(B, Hq, nq, d, dt, seed=81)
    scale = 1 / math.sqrt(d)
    for causal, ko in ((True, 60), (False, 0)):
        o, l = oracle_attention(q, k, v, scale, causal, q_offset=0, k_offset=ko)
        lse = torch.tensor(l, dtype=torch.float32, device=DEV)
        delta = torch.tensor(row_delta(o, g), dtype=torch.float32, device=DEV)
        dq, dk, dv = ra.block_backward(q.to(DEV), k.to(DEV), v.to(DEV), g.to(DEV), lse, delta,
                                       q_offset=0, k_offset=ko, causal=causal)
        want = attention_backward(q, k, v, g, scale, causal, q_offset=0, k_offset=ko)
        kind = _kind(dt)
        check_grad(dq, want[0], kind, "dQ")
        check_grad(dk, want[1], kind, "dK")
        check_grad(dv, want[2], kind, "dV")
        if causal:
            assert (dq[:, :, :ko] == 0).all()   # rows 0..59 see no key


def test_ring_backward_gqa_8_to_1_ragged():
    B, Hq, Hkv, n, d, P = 1, 8, 1, 700, 128, 7
    q, k, v = make_qkv(B, Hq, Hkv, n, n, d, d, BF, seed=91)
    g = make_dout(B, Hq, n, d, BF, seed=91)
    qd, kd, vd, gd = (x.to(DEV) for x in (q, k, v, g))
    out, lse = ra.ring_forward(qd, kd, vd, P, True)
    dq, dk, dv = ra.ring_backward(qd, kd, vd, out, lse, gd, P, True)
    want = attention_backward(q, k, v, g, 1 / math.sqrt(d), True)
    check_grad(dq, want[0], "bf16", "dQ")
    check_grad(dk, want[1], "bf16", "dK")
    check_grad(dv, want[2], "bf16", "dV")
