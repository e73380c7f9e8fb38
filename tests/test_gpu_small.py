"""GPU parity at sizes the oracle finishes in seconds: every entry point of the
C ABI against the fp64 oracle, element by element, on seeded inputs that span
several tiles and a ragged tail, plus the method's edge cases."""
import math
import zlib

import numpy as np
import pytest
import torch

from oracle.attention import attention as oracle_attention
from oracle.block_class import block_class as oracle_block_class
from oracle.merge import lse_merge as oracle_merge
from ring_context_parallelism_ra_b200 import ra
from ring_context_parallelism_ra_b200.workloads import make_qkv, workload, make_workload_inputs
from tests.parity_util import check_lse, check_out


def _seed(case):
    return zlib.crc32(repr(case).encode()) % 100000

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    ra.lib()
    yield
    assert ra.get_status() == ra.RA_OK
    torch.cuda.synchronize()


# ---------------------------------------------------------------- merge ----

@pytest.mark.parametrize("P,dv,out_dtype", [(1, 128, torch.float32), (2, 64, torch.bfloat16),
                                            (5, 128, torch.bfloat16), (16, 128, torch.float32),
                                            (3, 32, torch.float32)])
def test_lse_merge_matches_oracle(P, dv, out_dtype):
    g = torch.Generator().manual_seed(100 + P)
    B, H, n = 2, 3, 77
    o = torch.randn((P, B, H, n, dv), generator=g)
    l = torch.randn((P, B, H, n), generator=g) * 3
    l[0, 0, 0, :5] = -math.inf                 # one empty partial on some rows
    l[:, 1, 2, 7] = -math.inf                  # a row with every partial empty
    out, lse = ra.lse_merge(o.to(DEV), l.to(DEV), out_dtype)
    want_o, want_l = oracle_merge(o.numpy(), l.numpy())
    check_out(out, want_o, "f32" if out_dtype == torch.float32 else "bf16")
    check_lse(lse, want_l)
    assert (out[1, 2, 7] == 0).all() and lse[1, 2, 7].item() == -math.inf


@pytest.mark.parametrize("P,B,H,n,dv", [(8, 1, 8, 4096, 128),    # many rows: one warp per row
                                        (4, 1, 8, 2048, 128),    # P <= 4: all loads issued at once
                                        (24, 1, 2, 2048, 128),   # P > 16, many rows: looped row kernel
                                        (12, 1, 3, 37, 64),      # few rows, odd count: split-P
                                        (64, 4, 64, 1, 128),     # decode chunk partials
                                        (9, 2, 2, 5, 32)])
def test_lse_merge_both_kernels(P, B, H, n, dv):
    g = torch.Generator().manual_seed(P * 1000 + n)
    o = torch.randn((P, B, H, n, dv), generator=g)
    l = torch.randn((P, B, H, n), generator=g) * 4
    l[P - 1, 0, 0, 0] = -math.inf
    l[:, B - 1, H - 1, n - 1] = -math.inf
    for out_dtype in (torch.float32, torch.bfloat16):
        out, lse = ra.lse_merge(o.to(DEV), l.to(DEV), out_dtype)
        want_o, want_l = oracle_merge(o.numpy(), l.numpy())
        check_out(out, want_o, "f32" if out_dtype == torch.float32 else "bf16")
        check_lse(lse, want_l)


def test_decode_merge_matches_oracle():
    g = torch.Generator().manual_seed(7)
    P, B, H, d = 8, 4, 64, 128
    o = torch.randn((P, B, H, d), generator=g)
    l = torch.randn((P, B, H), generator=g) * 2 + 9
    out, lse = ra.decode_merge(o.to(DEV), l.to(DEV), torch.bfloat16)
    want_o, want_l = oracle_merge(o.numpy(), l.numpy())
    check_out(out, want_o, "bf16")
    check_lse(lse, want_l)


# ------------------------------------------------------- classification ----

@pytest.mark.parametrize("nq,nk,bq,bk,qo,ko", [(131072, 131072, 16384, 16384, 0, 0),
                                               (1000, 1300, 128, 128, 0, 0),
                                               (777, 555, 128, 64, 300, 17),
                                               (4096, 4096, 128, 128, 0, 4096)])
def test_device_block_class_bit_exact(nq, nk, bq, bk, qo, ko):
    for causal in (0, 1):
        dev = ra.block_class_device(nq, nk, bq, bk, qo, ko, causal).cpu().numpy()
        host = ra.block_class(nq, nk, bq, bk, qo, ko, causal)
        want = oracle_block_class(nq, nk, bq, bk, qo, ko, bool(causal))
        np.testing.assert_array_equal(dev, want)
        np.testing.assert_array_equal(host, want)


# ------------------------------------------------------------ attention ----

RING_CASES = [
    # B, Hq, Hkv, n, dqk, dv, P, causal, dtype
    (1, 1, 1, 512, 64, 64, 4, False, torch.float32),
    (1, 2, 1, 384, 128, 128, 3, True, torch.float32),
    (2, 2, 2, 200, 64, 128, 2, True, torch.float32),
    (1, 4, 2, 1024, 128, 128, 4, True, torch.bfloat16),
    (1, 2, 2, 864, 128, 128, 4, True, torch.bfloat16),      # 216-token partitions: ragged tiles
    (2, 4, 1, 640, 128, 128, 5, False, torch.bfloat16),
    (1, 2, 1, 520, 64, 64, 2, True, torch.bfloat16),
    (1, 2, 2, 768, 192, 128, 3, True, torch.bfloat16),      # MLA-shaped head
    (1, 8, 2, 257, 128, 128, 1, True, torch.bfloat16),      # P = 1, ragged tail
    (1, 1, 1, 1, 128, 128, 1, True, torch.bfloat16),        # a single token
    (1, 2, 1, 300, 64, 128, 3, True, torch.bfloat16),       # the other head-dim pairs
    (1, 2, 2, 256, 128, 64, 2, True, torch.bfloat16),
    (1, 2, 1, 384, 192, 64, 4, True, torch.bfloat16),
    (1, 2, 2, 96, 128, 128, 8, True, torch.bfloat16),       # 12-token partitions
    (1, 2, 1, 16, 128, 128, 16, True, torch.bfloat16),      # one token per partition
    (1, 1, 1, 8, 64, 64, 8, True, torch.float32),
]


@pytest.mark.parametrize("case", RING_CASES)
def test_ring_forward_matches_oracle(case):
    B, Hq, Hkv, n, dqk, dv, P, causal, dt = case
    q, k, v = make_qkv(B, Hq, Hkv, n, n, dqk, dv, dt, seed=_seed(case))
    scale = 1.0 / math.sqrt(dqk)
    out, lse = ra.ring_forward(q.to(DEV), k.to(DEV), v.to(DEV), P, causal, scale)
    want_o, want_l = oracle_attention(q, k, v, scale, causal)
    check_out(out, want_o, "f32" if dt == torch.float32 else "bf16")
    check_lse(lse, want_l)


BLOCK_CASES = [
    # B, Hq, Hkv, nq, nk, dqk, dv, q_off, k_off, causal, dtype
    (1, 2, 1, 300, 200, 128, 128, 200, 0, True, torch.bfloat16),
    (1, 2, 2, 256, 256, 128, 128, 256, 256, True, torch.bfloat16),   # diagonal block
    (1, 2, 1, 130, 260, 64, 64, 0, 0, False, torch.bfloat16),
    (1, 1, 1, 200, 300, 128, 128, 100, 150, True, torch.bfloat16),   # rows with no key
    (1, 2, 1, 192, 192, 192, 128, 192, 0, True, torch.bfloat16),
    (1, 1, 1, 100, 70, 128, 128, 40, 60, True, torch.float32),
    (2, 2, 1, 64, 64, 64, 64, 0, 64, True, torch.float32),           # fully masked block
]


@pytest.mark.parametrize("case", BLOCK_CASES)
def test_block_partial_matches_oracle(case):
    B, Hq, Hkv, nq, nk, dqk, dv, qo, ko, causal, dt = case
    q, k, v = make_qkv(B, Hq, Hkv, nq, nk, dqk, dv, dt, seed=_seed(case) + 7)
    scale = 1.0 / math.sqrt(dqk)
    o, l = ra.block_partial(q.to(DEV), k.to(DEV), v.to(DEV), qo, ko, causal, scale)
    want_o, want_l = oracle_attention(q, k, v, scale, causal, qo, ko)
    check_out(o, want_o, "f32" if dt == torch.float32 else "bf16")
    check_lse(l, want_l)


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float32])
def test_block_partials_merged_in_ring_order_equal_fused_ring(dt):
    """The unfused ring (one block partial per ring step, then the LSE merge)
    and the fused kernel both reproduce full attention."""
    B, Hq, Hkv, n, d, P = 1, 4, 2, 1024, 128, 4
    q, k, v = make_qkv(B, Hq, Hkv, n, n, d, d, dt, seed=42)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    L = n // P
    o_fused, l_fused = ra.ring_forward(qd, kd, vd, P, True)
    want_o, want_l = oracle_attention(q, k, v, 1 / math.sqrt(d), True)
    kind = "f32" if dt == torch.float32 else "bf16"
    outs, lses = [], []
    for i in range(P):
        o_parts = torch.empty((P, B, Hq, L, d), device=DEV)
        l_parts = torch.empty((P, B, Hq, L), device=DEV)
        for s in range(P):
            j = (i - s) % P
            ra.block_partial(qd[:, :, i * L:(i + 1) * L].contiguous(),
                             kd[:, :, j * L:(j + 1) * L].contiguous(),
                             vd[:, :, j * L:(j + 1) * L].contiguous(),
                             i * L, j * L, True, None, o_parts[s], l_parts[s])
        o_i, l_i = ra.lse_merge(o_parts, l_parts, dt)
        outs.append(o_i)
        lses.append(l_i)
    o_unfused = torch.cat(outs, dim=2)
    l_unfused = torch.cat(lses, dim=2)
    check_out(o_unfused, want_o, kind, "unfused O")
    check_lse(l_unfused, want_l, "unfused LSE")
    check_out(o_fused, want_o, kind, "fused O")
    check_lse(l_fused, want_l, "fused LSE")


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float32])
def test_causal_output_ignores_future_tokens(dt):
    B, H, n, d = 1, 2, 512, 128 if dt == torch.bfloat16 else 64
    q, k, v = make_qkv(B, H, H, n, n, d, d, dt, seed=5)
    t = 300
    k2, v2 = k.clone(), v.clone()
    g = torch.Generator().manual_seed(9)
    k2[:, :, t + 1:] = (torch.randn(k2[:, :, t + 1:].shape, generator=g) * 3).to(dt)
    v2[:, :, t + 1:] = (torch.randn(v2[:, :, t + 1:].shape, generator=g) * 3).to(dt)
    o1, l1 = ra.ring_forward(q.to(DEV), k.to(DEV), v.to(DEV), 4, True)
    o2, l2 = ra.ring_forward(q.to(DEV), k2.to(DEV), v2.to(DEV), 4, True)
    assert torch.equal(o1[:, :, :t + 1], o2[:, :, :t + 1])
    assert torch.equal(l1[:, :, :t + 1], l2[:, :, :t + 1])


def test_noncausal_fp32_512_full():
    wl = workload("noncausal_fp32_512")
    q, k, v = make_workload_inputs(wl)
    out, lse = ra.ring_forward(q.to(DEV), k.to(DEV), v.to(DEV), wl.P, wl.causal, wl.scale)
    want_o, want_l = oracle_attention(q, k, v, wl.scale, wl.causal)
    check_out(out, want_o, "f32")
    check_lse(lse, want_l)


def test_causal_mha_8k_full_bf16():
    wl = workload("causal_mha_8k")
    q, k, v = make_workload_inputs(wl)
    out, lse = ra.ring_forward(q.to(DEV), k.to(DEV), v.to(DEV), wl.P, wl.causal, wl.scale)
    want_o, want_l = oracle_attention(q, k, v, wl.scale, wl.causal)
    check_out(out, want_o, "bf16")
    check_lse(lse, want_l)


# --------------------------------------------------------------- decode ----

DECODE_CASES = [
    # B, Hq, Hkv, S, P
    (1, 8, 1, 4096, 1),
    (2, 16, 2, 10000, 4),       # 2500-token shards: a ragged chunk tail
    (3, 4, 4, 777, 3),          # G = 1
    (1, 32, 2, 6144, 2),        # G = 16
    (1, 8, 8, 64, 1),
]


@pytest.mark.parametrize("case", DECODE_CASES)
def test_decode_pass_q_matches_oracle(case):
    B, Hq, Hkv, S, P = case
    q, k, v = make_qkv(B, Hq, Hkv, 1, S, 128, 128, torch.bfloat16, seed=_seed(case))
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    scale = 1 / math.sqrt(128)
    L = S // P
    parts = [ra.decode_partial(qd, kd, vd, p * L, L, scale) for p in range(P)]
    for p, (o_p, l_p) in enumerate(parts):
        wo, wl_ = oracle_attention(q, k[:, :, p * L:(p + 1) * L], v[:, :, p * L:(p + 1) * L],
                                   scale, False)
        check_out(o_p, wo[:, :, 0], "bf16", f"shard {p} O")
        check_lse(l_p, wl_[:, :, 0], f"shard {p} LSE")
    out, lse = ra.decode_pass_q(qd, kd, vd, P, scale)
    want_o, want_l = oracle_attention(q, k, v, scale, False)
    check_out(out, want_o[:, :, 0], "bf16")
    check_lse(lse, want_l[:, :, 0])


@pytest.mark.parametrize("B,Hq,Hkv,S,P", [(2, 16, 2, 16384, 4), (1, 8, 1, 8192, 2),
                                         (4, 64, 8, 32768, 8), (1, 8, 2, 6144, 3)])
def test_decode_partials_one_launch_match_per_shard_oracle(B, Hq, Hkv, S, P):
    # every shard's partial from one launch, then the shard merge
    q, k, v = make_qkv(B, Hq, Hkv, 1, S, 128, 128, torch.bfloat16, seed=S + P)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    scale = 1 / math.sqrt(128)
    L = S // P
    o_parts, l_parts = ra.decode_partials(qd, kd, vd, P, scale)
    for p in range(P):
        wo, wl_ = oracle_attention(q, k[:, :, p * L:(p + 1) * L], v[:, :, p * L:(p + 1) * L],
                                   scale, False)
        check_out(o_parts[p], wo[:, :, 0], "bf16", f"shard {p} O")
        check_lse(l_parts[p], wl_[:, :, 0], f"shard {p} LSE")
    out, lse = ra.decode_pass_q(qd, kd, vd, P, scale)
    want_o, want_l = oracle_attention(q, k, v, scale, False)
    check_out(out, want_o[:, :, 0], "bf16")
    check_lse(lse, want_l[:, :, 0])


# ------------------------------------------------------------- failure ----

def test_bounded_wait_reports_timeout_and_context_survives():
    ra.check_wait_timeout(20_000_000)            # 20 ms
    assert ra.get_status() == ra.RA_ERR_TIMEOUT
    assert ra.get_status() == ra.RA_OK           # the word was cleared
    q, k, v = make_qkv(1, 1, 1, 128, 128, 64, 64, torch.float32, seed=1)
    out, lse = ra.ring_forward(q.to(DEV), k.to(DEV), v.to(DEV), 1, True)
    want_o, want_l = oracle_attention(q, k, v, 1 / 8, True)
    check_out(out, want_o, "f32")


def test_library_rejects_host_pointer_shapes():
    q = torch.zeros((1, 2, 128, 128), device=DEV, dtype=torch.bfloat16)
    k = torch.zeros((1, 3, 128, 128), device=DEV, dtype=torch.bfloat16)
    with pytest.raises(ra.RAError) as e:
        ra.ring_forward(q, k, k, 1, True)
    assert e.value.status == ra.RA_ERR_INVALID


def test_host_pipeline_equals_direct_calls():
    # The overlapped host pipeline returns, for every batch, exactly what a
    # direct ring_forward on the same inputs returns (same kernel).
    from ring_context_parallelism_ra_b200.host_pipeline import RingForwardPipeline
    shape = (1, 4, 2, 640, 640, 128, 128)
    batches = [make_qkv(*shape, torch.bfloat16, seed=300 + i) for i in range(5)]
    pipe = RingForwardPipeline(batches[0][0].shape, batches[0][1].shape, batches[0][2].shape,
                               torch.bfloat16, 4, True)
    pinned = [tuple(x.pin_memory() for x in b) for b in batches]
    for i, (q, k, v) in enumerate(pinned):
        slot = pipe.submit(q, k, v)
        if i >= 1:  # results of the previous batch while this one is in flight
            o_prev, l_prev = pipe.wait((slot - 1) % pipe.depth)
            want_o, want_l = ra.ring_forward(*(x.to(DEV) for x in batches[i - 1]), 4, True)
            assert torch.equal(o_prev, want_o.cpu()) and torch.equal(l_prev, want_l.cpu())
    o_last, l_last = pipe.wait((len(batches) - 1) % pipe.depth)
    want_o, want_l = ra.ring_forward(*(x.to(DEV) for x in batches[-1]), 4, True)
    assert torch.equal(o_last, want_o.cpu()) and torch.equal(l_last, want_l.cpu())


def test_pass_q_decode_graph_replays_match_oracle():
    # one captured decode step replayed for two different query tokens
    from ring_context_parallelism_ra_b200.host_pipeline import PassQDecodeGraph
    B, Hq, Hkv, S, d, P = 2, 16, 2, 8192, 128, 4
    _, k, v = make_qkv(B, Hq, Hkv, 1, S, d, d, torch.bfloat16, seed=81)
    graph = PassQDecodeGraph(k.to(DEV), v.to(DEV), P, Hq)
    for seed in (82, 83):
        q, _, _ = make_qkv(B, Hq, Hkv, 1, 1, d, d, torch.bfloat16, seed=seed)
        graph.q.copy_(q.to(DEV))
        out, lse = graph.replay()
        torch.cuda.synchronize()
        want_o, want_l = oracle_attention(q, k, v, 1.0 / math.sqrt(d), False)
        check_out(out, want_o[:, :, 0], "bf16")
        check_lse(lse, want_l[:, :, 0])
