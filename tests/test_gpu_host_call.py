"""GPU tests of ra_ring_forward_host: the fused ring from host buffers to host
buffers.  Each chunk is an ordinary ring launch over whole (batch, KV head)
groups, so the result must equal ra_ring_forward on device copies bit for
bit; a small case is also checked against the fp64 oracle."""
import ctypes
import zlib

import numpy as np
import pytest
import torch

from oracle.attention import attention as oracle_attention
from ring_context_parallelism_ra_b200 import ra
from ring_context_parallelism_ra_b200.workloads import make_qkv
from tests.parity_util import check_lse, check_out

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    ra.lib()
    yield
    assert ra.get_status() == ra.RA_OK
    torch.cuda.synchronize()


def _host_inputs(B, Hq, Hkv, n, dqk, dv, dtype, seed, pinned=True):
    q, k, v = (t.cpu() for t in make_qkv(B, Hq, Hkv, n, n, dqk, dv, dtype, seed, device="cuda"))
    if pinned:
        q, k, v = q.pin_memory(), k.pin_memory(), v.pin_memory()
    return q, k, v


# (B, Hq, Hkv, n, d_qk, d_v, P, causal, dtype): one chunk; chunks inside a
# batch; chunks of whole batches; MLA-shaped head
CASES = [
    (1, 4, 2, 640, 128, 128, 5, True, torch.bfloat16),
    (2, 8, 2, 65536, 128, 128, 8, True, torch.bfloat16),      # 4 chunks of one group
    (8, 2, 2, 32768, 64, 64, 4, True, torch.bfloat16),        # 2 chunks of 4 whole batches
    (1, 4, 4, 65536, 192, 128, 16, True, torch.bfloat16),     # 4 chunks, d_qk = 192
    (1, 2, 1, 1024, 128, 64, 4, False, torch.bfloat16),
    (1, 2, 2, 512, 64, 64, 4, True, torch.float32),
]


@pytest.mark.parametrize("case", CASES)
def test_host_call_equals_device_ring_forward(case):
    B, Hq, Hkv, n, dqk, dv, P, causal, dtype = case
    q, k, v = _host_inputs(B, Hq, Hkv, n, dqk, dv, dtype, seed=zlib.crc32(repr(case).encode()) % 9973)
    out_h, lse_h = ra.ring_forward_host(q, k, v, P, causal)
    out_d, lse_d = ra.ring_forward(q.cuda(), k.cuda(), v.cuda(), P, causal)
    torch.cuda.synchronize()
    assert torch.equal(out_h, out_d.cpu())
    assert torch.equal(lse_h, lse_d.cpu())


def test_host_call_matches_oracle_and_skips_lse():
    B, Hq, Hkv, n, d, P = 1, 4, 2, 768, 128, 3
    q, k, v = _host_inputs(B, Hq, Hkv, n, d, d, torch.bfloat16, seed=71)
    out, lse = ra.ring_forward_host(q, k, v, P, True)
    want_o, want_l = oracle_attention(q, k, v, d ** -0.5, True)
    check_out(out, want_o, "bf16")
    check_lse(lse, want_l)
    # without LSE: the same O, nothing written to a LSE buffer
    L = ra.lib()
    s = ra._shape(q, k, v)
    ws = torch.empty(ra.ring_forward_host_workspace_bytes(q, k, v), dtype=torch.uint8,
                     device="cuda")
    out2 = torch.full_like(out, 7.0).pin_memory()
    st = torch.cuda.current_stream()
    rc = L.ra_ring_forward_host(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                                ctypes.c_void_p(v.data_ptr()), P, 1, float(d ** -0.5),
                                ctypes.c_void_p(out2.data_ptr()), None, ctypes.byref(s),
                                ctypes.c_void_p(ws.data_ptr()), ctypes.c_size_t(ws.numel()),
                                ctypes.c_void_p(st.cuda_stream))
    assert rc == ra.RA_OK
    st.synchronize()
    assert torch.equal(out2, out)


def test_host_call_from_pageable_memory_and_back_to_back():
    # pageable inputs (copies hold the calling thread) give the same result;
    # two calls in a row through one workspace do not see each other
    case = (1, 8, 2, 32768, 128, 128, 4, True)
    B, Hq, Hkv, n, dqk, dv, P, causal = case
    q1, k1, v1 = _host_inputs(B, Hq, Hkv, n, dqk, dv, torch.bfloat16, seed=5, pinned=False)
    q2, k2, v2 = _host_inputs(B, Hq, Hkv, n, dqk, dv, torch.bfloat16, seed=6, pinned=True)
    ws = torch.empty(ra.ring_forward_host_workspace_bytes(q1, k1, v1), dtype=torch.uint8,
                     device="cuda")
    o1, l1 = ra.ring_forward_host(q1, k1, v1, P, causal, workspace=ws, synchronize=False)
    o2, l2 = ra.ring_forward_host(q2, k2, v2, P, causal, workspace=ws, synchronize=False)
    torch.cuda.current_stream().synchronize()
    for (q, k, v), o, l in (((q1, k1, v1), o1, l1), ((q2, k2, v2), o2, l2)):
        od, ld = ra.ring_forward(q.cuda(), k.cuda(), v.cuda(), P, causal)
        assert torch.equal(o, od.cpu())
        assert torch.equal(l, ld.cpu())
    assert not torch.equal(o1, o2)
    assert np.isfinite(l1.numpy()).all()
