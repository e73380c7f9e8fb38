"""GPU parity at the full workload sizes, in the launch configuration the bench
times.  The oracle checks sampled outputs one by one (rows are independent,
so each sampled row is an exact check); every other output is checked for
finiteness.  Inputs are drawn on the GPU (see workloads.py) and the oracle
receives CPU copies of the slices it needs."""
import numpy as np
import pytest
import torch

from oracle.attention import attention as oracle_attention
from ring_context_parallelism_ra_b200 import ra
from ring_context_parallelism_ra_b200.workloads import make_workload_inputs, workload
from tests.parity_util import check_lse, check_out

pytestmark = pytest.mark.gpu


def sample_rows(n, P, tile=128, n_uniform=64, seed=0):
    """Rows 0, 1, n-1; first/last row of every partition; first/last row of
    the first and last four 128-row tiles of partitions 0 and P-1; plus
    seeded uniform rows."""
    L = n // P
    rows = {0, 1, n - 1}
    for i in range(P):
        rows |= {i * L, i * L + L - 1}
    for i in (0, P - 1):
        nt = L // tile
        for t in list(range(min(4, nt))) + list(range(max(0, nt - 4), nt)):
            rows |= {i * L + t * tile, i * L + t * tile + tile - 1}
    rng = np.random.default_rng(seed)
    rows |= set(rng.integers(0, n, n_uniform).tolist())
    return np.array(sorted(rows), dtype=np.int64)


def _check_prefill(key, heads, row_seed):
    wl = workload(key)
    torch.cuda.empty_cache()
    q, k, v = make_workload_inputs(wl, device="cuda")
    out, lse = ra.ring_forward(q, k, v, wl.P, wl.causal, wl.scale)
    assert ra.get_status() == ra.RA_OK
    assert torch.isfinite(out).all().item()
    assert torch.isfinite(lse).all().item()
    rows = sample_rows(wl.n, wl.P, seed=row_seed)
    G = wl.Hq // wl.Hkv
    q_s = q[:, heads].cpu()
    k_s = torch.stack([k[:, h // G] for h in heads], dim=1).cpu()
    v_s = torch.stack([v[:, h // G] for h in heads], dim=1).cpu()
    want_o, want_l = oracle_attention(q_s, k_s, v_s, wl.scale, wl.causal, rows=rows)
    idx = torch.as_tensor(rows, device="cuda")
    got_o = out[:, heads][:, :, idx]
    got_l = lse[:, heads][:, :, idx]
    check_out(got_o, want_o, wl.dtype)
    check_lse(got_l, want_l)
    del q, k, v, out, lse
    torch.cuda.empty_cache()


def test_causal_gqa_128k_full_size():
    _check_prefill("causal_gqa_128k", heads=[0, 3, 4, 31], row_seed=3)


def test_causal_mla_256k_full_size():
    _check_prefill("causal_mla_256k", heads=[0, 15], row_seed=5)


def test_decode_pass_q_1m_full_size():
    wl = workload("decode_1m")
    torch.cuda.empty_cache()
    q, k, v = make_workload_inputs(wl, device="cuda")
    out, lse = ra.decode_pass_q(q, k, v, wl.P, wl.scale)
    assert ra.get_status() == ra.RA_OK
    assert torch.isfinite(out).all().item() and torch.isfinite(lse).all().item()
    G = wl.Hq // wl.Hkv
    for b, g in [(0, 0), (3, 7), (1, 4)]:
        heads = list(range(g * G, (g + 1) * G))
        q_s = q[b:b + 1, heads].cpu()
        k_s = k[b:b + 1, g:g + 1].cpu()
        v_s = v[b:b + 1, g:g + 1].cpu()
        want_o, want_l = oracle_attention(q_s, k_s, v_s, wl.scale, False)
        check_out(out[b:b + 1, heads], want_o[:, :, 0], wl.dtype, f"O b={b} g={g}")
        check_lse(lse[b:b + 1, heads], want_l[:, :, 0], f"LSE b={b} g={g}")
    del q, k, v
    torch.cuda.empty_cache()


def _check_backward(key, row_seed):
    """The ring backward on a full-size workload in the bench's configuration:
    exact gradients on sampled query rows (dQ) and on the last 256 keys (dK,
    dV; a causal key u needs only rows t >= u), for the query heads of the
    first and the last KV head; identities over every key of every head:
    sum_u dK_u = 0 and sum_u dV_u = sum_t dO_t (per column)."""
    from oracle.backward import attention_backward_sampled
    from ring_context_parallelism_ra_b200.workloads import make_dout
    from tests.parity_util import check_grad, sum_identity_bar
    wl = workload(key)
    torch.cuda.empty_cache()
    q, k, v = make_workload_inputs(wl, device="cuda")
    g = make_dout(wl.B, wl.Hq, wl.n, wl.d_v, wl.torch_dtype, seed=wl.seed, device="cuda")
    out, lse = ra.ring_forward(q, k, v, wl.P, wl.causal, wl.scale)
    dq, dk, dv = ra.ring_backward(q, k, v, out, lse, g, wl.P, wl.causal, wl.scale)
    assert ra.get_status() == ra.RA_OK
    for t in (dq, dk, dv):
        assert torch.isfinite(t).all().item()
    G = wl.Hq // wl.Hkv
    rows = sample_rows(wl.n, wl.P, n_uniform=24, seed=row_seed)
    keys = np.arange(wl.n - 256, wl.n)
    for grp in (0, wl.Hkv - 1):
        heads = list(range(grp * G, (grp + 1) * G))
        if G == 1:
            heads = [grp]
        q_s, g_s = q[:, heads].cpu(), g[:, heads].cpu()
        k_s, v_s = k[:, grp:grp + 1].cpu(), v[:, grp:grp + 1].cpu()
        wq, wk, wv = attention_backward_sampled(q_s, k_s, v_s, g_s, wl.scale, True, rows, keys)
        ri = torch.as_tensor(rows, device="cuda")
        ki = torch.as_tensor(keys, device="cuda")
        check_grad(dq[:, heads][:, :, ri], wq, "bf16", "dQ sampled rows")
        check_grad(dk[:, grp:grp + 1][:, :, ki], wk, "bf16", "dK last keys")
        check_grad(dv[:, grp:grp + 1][:, :, ki], wv, "bf16", "dV last keys")
    # the longest dK / dV accumulator (the first key tile of a KV head) takes
    # G * n / 16 round-toward-zero steps in tensor memory
    steps = G * wl.n // 16
    dk64 = dk.double()
    dv64 = dv.double()
    assert (dk64.sum(dim=2).abs().cpu().numpy() <= sum_identity_bar(dk64, steps, 2)).all()
    want_sv = g.double().reshape(wl.B, wl.Hkv, G, wl.n, wl.d_v).sum(dim=(2, 3))
    assert ((dv64.sum(dim=2) - want_sv).abs().cpu().numpy() <= sum_identity_bar(dv64, steps, 2)).all()
    del q, k, v, g, out, lse, dq, dk, dv, dk64, dv64
    torch.cuda.empty_cache()


def test_backward_causal_gqa_128k_full_size():
    _check_backward("causal_gqa_128k", 33)


def test_backward_causal_mla_256k_full_size():
    # the MLA-shaped head (d_qk 192, d_v 128) on its tensor-core kernel
    _check_backward("causal_mla_256k", 35)
