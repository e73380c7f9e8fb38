"""CPU tests of the C ABI: the library loads, exports every symbol the header
declares, and its host-side logic (argument validation, block classification)
behaves, without launching anything on a GPU."""
import ctypes
import os
import re
import subprocess
import sys

import numpy as np
import pytest
import torch

from oracle.block_class import block_class as oracle_block_class
from oracle.block_class import partition_class
from ring_context_parallelism_ra_b200 import ra

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_symbols():
    text = open(os.path.join(ROOT, "include", "ra.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ra_[a-z_0-9]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    L = ra.lib()
    syms = _header_symbols()
    assert syms, "no declarations found in include/ra.h"
    for name in syms:
        assert hasattr(L, name), f"libra.so does not export {name}"
    assert sorted(ra.EXPORTED) == syms


def test_status_strings():
    for code in (0, -1, -2, -3, -4):
        assert ra.status_string(code).startswith("RA_")
    assert "unknown" in ra.status_string(7)


@pytest.mark.parametrize("nq,nk,bq,bk", [(1, 1, 1, 1), (300, 300, 128, 128), (257, 511, 64, 128),
                                         (1000, 200, 128, 64), (4096, 4096, 128, 128)])
def test_host_block_class_matches_oracle(nq, nk, bq, bk):
    for qo, ko in [(0, 0), (100, 0), (0, 77), (300, 299)]:
        for causal in (0, 1):
            got = ra.block_class(nq, nk, bq, bk, qo, ko, causal)
            want = oracle_block_class(nq, nk, bq, bk, qo, ko, bool(causal))
            np.testing.assert_array_equal(got, want)


def test_host_partition_map_for_ring_configs():
    for n, P in [(8192, 4), (131072, 8), (262144, 16)]:
        got = ra.block_class(n, n, n // P, n // P, 0, 0, 1)
        np.testing.assert_array_equal(got, partition_class(n, P, True))


def _shape(**kw):
    d = dict(B=1, Hq=2, Hkv=1, n_q=128, n_k=128, d_qk=128, d_v=128, dtype=ra.RA_BF16)
    d.update(kw)
    return ra.Shape(**d)


def test_validation_rejects_bad_arguments_before_launch():
    L = ra.lib()
    p = ctypes.c_void_p(256)   # aligned dummy; never dereferenced on these paths
    nul = ctypes.c_void_p(0)
    mis = ctypes.c_void_p(258)
    INV, UNS = ra.RA_ERR_INVALID, ra.RA_ERR_UNSUPPORTED
    s = _shape()
    assert L.ra_ring_forward(nul, p, p, 1, 1, 1.0, p, p, ctypes.byref(s), nul) == INV
    assert L.ra_ring_forward(p, p, p, 0, 1, 1.0, p, p, ctypes.byref(s), nul) == INV
    assert L.ra_ring_forward(p, p, p, 3, 1, 1.0, p, p, ctypes.byref(s), nul) == INV   # 128 % 3
    assert L.ra_ring_forward(mis, p, p, 1, 1, 1.0, p, p, ctypes.byref(s), nul) == INV
    s2 = _shape(n_k=64)
    assert L.ra_ring_forward(p, p, p, 1, 1, 1.0, p, p, ctypes.byref(s2), nul) == INV  # n_q != n_k
    s3 = _shape(Hq=3, Hkv=2)
    assert L.ra_block_partial(p, p, p, ctypes.byref(s3), 0, 0, 1, 1.0, p, p, nul) == INV
    s4 = _shape(d_qk=96)
    assert L.ra_block_partial(p, p, p, ctypes.byref(s4), 0, 0, 1, 1.0, p, p, nul) == UNS
    s5 = _shape(dtype=ra.RA_F32, d_qk=192)
    assert L.ra_block_partial(p, p, p, ctypes.byref(s5), 0, 0, 1, 1.0, p, p, nul) == UNS
    assert L.ra_block_partial(p, p, p, ctypes.byref(s), -1, 0, 1, 1.0, p, p, nul) == INV
    assert L.ra_block_partial(p, p, p, ctypes.byref(s), 0, 0, 2, 1.0, p, p, nul) == INV
    assert L.ra_block_partial(p, p, p, None, 0, 0, 1, 1.0, p, p, nul) == INV
    assert L.ra_lse_merge(p, p, 0, ctypes.byref(s), p, 0, p, nul) == INV
    s6 = _shape(d_v=96)
    assert L.ra_lse_merge(p, p, 2, ctypes.byref(s6), p, 0, p, nul) == UNS
    sd = _shape(n_q=1, Hq=8, Hkv=1, n_k=4096)
    assert L.ra_decode_partial(p, p, p, 4096, ctypes.byref(sd), 1.0, p, p, p, 0, nul) == INV  # ws
    assert L.ra_decode_partial(p, p, p, 100, ctypes.byref(sd), 1.0, p, p, p, 1 << 30, nul) == INV
    sd2 = _shape(n_q=2, Hq=8, Hkv=1, n_k=4096)
    assert L.ra_decode_partial(p, p, p, 4096, ctypes.byref(sd2), 1.0, p, p, p, 1 << 30, nul) == INV
    sd3 = _shape(n_q=1, Hq=8, Hkv=1, n_k=4096, d_qk=64, d_v=64)
    assert L.ra_decode_partial(p, p, p, 4096, ctypes.byref(sd3), 1.0, p, p, p, 1 << 30, nul) == UNS
    assert L.ra_decode_merge(p, p, 2, ctypes.byref(_shape(n_q=4)), p, 0, p, nul) == INV
    # shards in one launch need whole 2048-token chunks per shard
    sp = _shape(n_q=1, Hq=8, Hkv=1, n_k=6000)
    assert L.ra_decode_partials(p, p, p, 3, ctypes.byref(sp), 1.0, p, p, p, 1 << 30, nul) == UNS
    assert L.ra_decode_partials(p, p, p, 7, ctypes.byref(sp), 1.0, p, p, p, 1 << 30, nul) == INV
    sp2 = _shape(n_q=1, Hq=8, Hkv=1, n_k=8192)
    assert L.ra_decode_partials(p, p, p, 4, ctypes.byref(sp2), 1.0, p, p, p, 16, nul) == INV  # ws
    # empty inputs are rejected, not launched: no sequence, no batch, no heads
    s0 = _shape(n_q=0, n_k=0)
    assert L.ra_ring_forward(p, p, p, 1, 1, 1.0, p, p, ctypes.byref(s0), nul) == INV
    assert L.ra_block_partial(p, p, p, ctypes.byref(_shape(n_k=0)), 0, 0, 1, 1.0, p, p, nul) == INV
    assert L.ra_block_partial(p, p, p, ctypes.byref(_shape(B=0)), 0, 0, 1, 1.0, p, p, nul) == INV
    assert L.ra_lse_merge(p, p, 2, ctypes.byref(_shape(Hq=0, Hkv=0)), p, 0, p, nul) == INV
    assert L.ra_decode_partial(p, p, p, 0, ctypes.byref(_shape(n_q=1, Hq=8, Hkv=1, n_k=0)), 1.0,
                               p, p, p, 1 << 30, nul) == INV
    out = np.empty(4, dtype=np.int8)
    assert L.ra_block_class(0, 4, 1, 1, 0, 0, 1, out.ctypes.data_as(ctypes.c_void_p)) == INV
    assert L.ra_block_class(4, 4, 0, 1, 0, 0, 1, out.ctypes.data_as(ctypes.c_void_p)) == INV
    assert L.ra_block_class(4, 4, 1, 1, 0, 0, 1, None) == INV


def test_decode_workspace_size_is_chunk_partials():
    # (chunks of 2048 tokens) x rows x (d + 1) floats, plus slack
    n = ra.decode_workspace_bytes(4, 64, 8, 131072)
    assert n >= 64 * 4 * 64 * 129 * 4
    assert n < 64 * 4 * 64 * 129 * 4 + 4096


def test_backward_validation_rejects_bad_arguments_before_launch():
    L = ra.lib()
    p = ctypes.c_void_p(256)
    nul = ctypes.c_void_p(0)
    mis = ctypes.c_void_p(264)
    INV, UNS = ra.RA_ERR_INVALID, ra.RA_ERR_UNSUPPORTED
    s = _shape()
    ws = L.ra_backward_workspace_bytes(ctypes.byref(s))
    big = ctypes.c_size_t(ws)

    def ring(fn, shape, P=1, causal=1, q=p, wsb=big):
        return fn(q, p, p, p, p, p, P, causal, 1.0, p, p, p, ctypes.byref(shape), p, wsb, nul)

    for fn in (L.ra_ring_backward, L.ra_ring_backward_striped):
        assert ring(fn, s, q=nul) == INV
        assert ring(fn, s, q=mis) == INV
        assert ring(fn, s, P=0) == INV
        assert ring(fn, s, P=3) == INV                       # 128 % 3
        assert ring(fn, s, causal=2) == INV
        assert ring(fn, _shape(n_k=64)) == INV               # n_q != n_k
        assert ring(fn, _shape(d_qk=96)) == UNS              # head dims outside {64, 128, 192}
        assert ring(fn, _shape(dtype=ra.RA_F32, d_qk=192)) == UNS   # as the forward: bf16 only
        assert ring(fn, _shape(dtype=ra.RA_F32, d_v=32)) == UNS
        assert ring(fn, s, wsb=ctypes.c_size_t(ws - 1)) == INV
    # striped needs whole 128-row tiles per partition
    s_odd = _shape(n_q=384, n_k=384)
    ws_odd = ctypes.c_size_t(L.ra_backward_workspace_bytes(ctypes.byref(s_odd)))
    assert ring(L.ra_ring_backward_striped, s_odd, P=2, wsb=ws_odd) == UNS   # 192-row partitions

    def blk(shape, qo=0, ko=0, st=1, causal=1, lse=p, wsb=big):
        return L.ra_block_backward(p, p, p, p, lse, p, ctypes.byref(shape), qo, ko, st, causal,
                                   1.0, p, p, p, p, wsb, nul)

    assert blk(s, lse=nul) == INV
    assert blk(s, qo=-1) == INV
    assert blk(s, st=0) == INV
    assert blk(s, causal=3) == INV
    assert blk(_shape(Hq=3, Hkv=2)) == INV
    assert blk(_shape(d_qk=96)) == UNS
    assert blk(s, wsb=ctypes.c_size_t(0)) == INV
    assert L.ra_backward_delta(nul, p, ctypes.byref(s), p, nul) == INV
    assert L.ra_backward_delta(p, p, None, p, nul) == INV
    assert L.ra_backward_delta(p, p, ctypes.byref(_shape(d_v=32)), p, nul) == UNS


def test_backward_workspace_size():
    # fp32 dQ accumulator plus two row vectors, rows padded to 128 per head
    for B, H, n, d in [(1, 8, 8192, 128), (2, 3, 1000, 64)]:
        s = _shape(B=B, Hq=H, Hkv=1, n_q=n, n_k=n, d_qk=d, d_v=d)
        rows = B * H * ((n + 127) // 128) * 128
        got = ra.lib().ra_backward_workspace_bytes(ctypes.byref(s))
        assert rows * (d + 2) * 4 <= got < rows * (d + 2) * 4 + 1024


def test_no_cpu_fallback_cpu_tensors_are_rejected():
    # the binding only marshals device pointers: CPU tensors are an error,
    # never a silent host computation
    q = torch.zeros((1, 1, 128, 64), dtype=torch.bfloat16)
    with pytest.raises(TypeError, match="CUDA tensor"):
        ra.ring_forward(q, q, q, 1, True)
    with pytest.raises(TypeError, match="CUDA tensor"):
        ra.lse_merge(torch.zeros((2, 1, 1, 4, 64)), torch.zeros((2, 1, 1, 4)), torch.float32)


def test_missing_library_fails_loudly(tmp_path):
    # with the compiled library absent the package raises on first use
    code = (
        "import sys; sys.path.insert(0, %r)\n"
        "from ring_context_parallelism_ra_b200 import ra\n"
        "ra.library_path = lambda: %r\n"
        "try:\n"
        "    ra.lib()\n"
        "except RuntimeError as e:\n"
        "    print('raised:', e)\n"
        "    sys.exit(0)\n"
        "sys.exit(3)\n" % (ROOT, str(tmp_path / "libra.so")))
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "is missing" in r.stdout


def test_decode_graph_rejects_uneven_shards_before_any_gpu_work():
    from ring_context_parallelism_ra_b200.host_pipeline import PassQDecodeGraph
    k = torch.zeros((1, 1, 1000, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="equal shards"):
        PassQDecodeGraph(k, k, 3, 8)


def _host_slot_bytes(B, Hq, Hkv, n, dqk, dv, esz, per_chunk):
    """One chunk buffer set as ra.h describes it: Q, K, V, O, LSE of
    `per_chunk` (batch, KV head) groups, each buffer 256-byte aligned."""
    G = Hq // Hkv
    al = lambda x: (x + 255) // 256 * 256  # noqa: E731
    parts = [G * n * dqk * esz, n * dqk * esz, n * dv * esz, G * n * dv * esz, G * n * 4]
    return sum(al(per_chunk * b) for b in parts)


@pytest.mark.parametrize("dims,per_chunk", [
    ((1, 16, 16, 262144, 192, 128), 2),   # 1024 items per group: 8 chunks of 2 groups
    ((1, 32, 8, 131072, 128, 128), 1),    # 2048 items per group: 8 chunks of 1
    ((1, 8, 8, 8192, 128, 128), 8),       # 32 items per group: one chunk
    ((8, 2, 2, 32768, 128, 128), 8),      # 128 per group: chunks of 4 whole batches
    ((2, 8, 2, 65536, 128, 128), 1),      # 1024 per group: 4 chunks (within a batch)
    ((3, 1, 1, 1000, 64, 64), 3),         # nothing splits: one chunk
])
def test_host_call_workspace_follows_the_chunk_rule(dims, per_chunk):
    B, Hq, Hkv, n, dqk, dv = dims
    s = _shape(B=B, Hq=Hq, Hkv=Hkv, n_q=n, n_k=n, d_qk=dqk, d_v=dv)
    want = 2 * _host_slot_bytes(B, Hq, Hkv, n, dqk, dv, 2, per_chunk)
    assert ra.lib().ra_ring_forward_host_workspace_bytes(ctypes.byref(s)) == want
    s32 = _shape(B=B, Hq=Hq, Hkv=Hkv, n_q=n, n_k=n, d_qk=dqk, d_v=dv, dtype=ra.RA_F32)
    want32 = 2 * _host_slot_bytes(B, Hq, Hkv, n, dqk, dv, 4, per_chunk)
    assert ra.lib().ra_ring_forward_host_workspace_bytes(ctypes.byref(s32)) == want32


def test_host_call_rejects_bad_arguments_before_any_gpu_work():
    L = ra.lib()
    p = ctypes.c_void_p(256)   # never dereferenced on these paths
    nul = ctypes.c_void_p(0)
    INV, UNS = ra.RA_ERR_INVALID, ra.RA_ERR_UNSUPPORTED
    s = _shape()
    ws = L.ra_ring_forward_host_workspace_bytes(ctypes.byref(s))
    assert ws > 0
    big = ctypes.c_size_t(ws)

    def call(shape=s, P=1, causal=1, q=p, w=p, wsb=big):
        return L.ra_ring_forward_host(q, p, p, P, causal, 1.0, p, p, ctypes.byref(shape), w,
                                      wsb, nul)

    assert call(q=nul) == INV
    assert call(w=nul) == INV
    assert call(w=ctypes.c_void_p(256 + 16)) == INV          # workspace not 256-byte aligned
    assert call(wsb=ctypes.c_size_t(ws - 1)) == INV          # workspace too small
    assert call(P=0) == INV
    assert call(P=3) == INV                                  # 128 % 3
    assert call(causal=2) == INV
    assert call(shape=_shape(n_k=64)) == INV                 # n_q != n_k
    assert call(shape=_shape(Hq=3, Hkv=2)) == INV
    assert call(shape=_shape(n_q=0, n_k=0)) == INV
    wide = _shape(d_qk=96)
    assert call(shape=wide, wsb=ctypes.c_size_t(1 << 40)) == UNS
    assert L.ra_ring_forward_host_workspace_bytes(None) == 0
    assert L.ra_ring_forward_host_workspace_bytes(ctypes.byref(_shape(Hq=3, Hkv=2))) == 0
