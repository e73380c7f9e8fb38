"""GPU tests of ra_decode_partial_noalloc, the decode entry point for callers
that cannot allocate device memory: a plugin whose host runtime owns every
device allocation and gives its plugins no allocator, or a latency-critical
loop that must not call cudaMalloc (it may synchronise the device and has no
latency bound).  The call keeps its chunk partials in the library's static
device array instead of a caller workspace.

Each call is checked twice over: against the fp64 oracle on the same shard,
at the bf16 / LSE bars every decode parity test uses, and against
ra_decode_partial (the workspace entry point) on the same inputs.  Every
shape is called twice in a row, and the shapes run one after another, so a
call that read the previous call's leftovers in the shared array would fail.

This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes on its own in a fresh process.
"""
import math

import pytest
import torch

from oracle.attention import attention as oracle_attention
from ring_context_parallelism_ra_b200 import ra
from tests.parity_util import check_lse, check_out

pytestmark = pytest.mark.gpu

D = 128
SCALE = 1 / math.sqrt(D)
# bytes of chunk partials one call needs: ceil(n_k / 2048) chunks x B*Hq rows
# x (d_v + 1) fp32, plus 256 bytes of alignment slack; the array holds 16 MiB
LIMIT_BYTES = 16 << 20


def _need_bytes(B, Hq, n_k):
    return -(-n_k // 2048) * B * Hq * (D + 1) * 4 + 256


def _draw(B, Hq, Hkv, S, seed):
    """Seeded i.i.d. N(0, 1) bf16 query, K and V cache on the GPU (one
    generator for the whole tensor: some shapes here have 32K query rows)."""
    g = torch.Generator(device="cuda").manual_seed(seed)
    q = torch.randn((B, Hq, 1, D), device="cuda", generator=g).to(torch.bfloat16)
    k = torch.randn((B, Hkv, S, D), device="cuda", generator=g).to(torch.bfloat16)
    v = torch.randn((B, Hkv, S, D), device="cuda", generator=g).to(torch.bfloat16)
    return q, k, v


# B, Hq, Hkv, cache tokens, shard start, shard length, seed
CASES = [
    (2, 16, 2, 10000, 2500, 2500, 11),      # ragged shard inside a longer cache
    (4, 64, 8, 131072, 0, 131072, 12),      # one shard of the 1M-token pass-Q workload
    (2032, 16, 1, 1, 0, 1, 13),             # one token per shard; the largest row count that fits
]


def test_shapes_sit_where_intended_against_the_limit():
    assert _need_bytes(2032, 16, 1) <= LIMIT_BYTES < _need_bytes(2033, 16, 1)
    assert _need_bytes(4, 64, 131072) <= LIMIT_BYTES


def test_noalloc_decode_matches_oracle_and_workspace_decode_twice():
    assert torch.cuda.is_available(), "GPU test needs a CUDA device"
    for B, Hq, Hkv, S, start, count, seed in CASES:
        q, k, v = _draw(B, Hq, Hkv, S, seed)
        qc, kc, vc = q.cpu(), k[:, :, start:start + count].cpu(), v[:, :, start:start + count].cpu()
        want_o, want_l = oracle_attention(qc, kc, vc, SCALE, False)
        ws_o, ws_l = ra.decode_partial(q, k, v, start, count, SCALE)
        o_part = torch.empty((B, Hq, D), device="cuda", dtype=torch.float32)
        lse_part = torch.empty((B, Hq), device="cuda", dtype=torch.float32)
        for call in range(2):
            o_part.fill_(float("nan"))
            lse_part.fill_(float("nan"))
            got_o, got_l = ra.decode_partial_noalloc(q, k, v, start, count, SCALE, o_part, lse_part)
            assert ra.get_status() == ra.RA_OK
            what = f"B={B} Hq={Hq} shard {count} call {call}"
            check_out(got_o, want_o[:, :, 0], "bf16", f"{what}: O vs oracle")
            check_lse(got_l, want_l[:, :, 0], f"{what}: LSE vs oracle")
            check_out(got_o, ws_o, "bf16", f"{what}: O vs ra_decode_partial")
            check_lse(got_l, ws_l, f"{what}: LSE vs ra_decode_partial")


def test_noalloc_decode_rejects_shapes_beyond_its_scratch():
    assert torch.cuda.is_available(), "GPU test needs a CUDA device"
    B, Hq, Hkv, S = 2033, 16, 1, 1          # 32528 rows x 516 B > 16 MiB
    q, k, v = _draw(B, Hq, Hkv, S, 14)
    o_part = torch.full((B, Hq, D), 7.0, device="cuda", dtype=torch.float32)
    lse_part = torch.full((B, Hq), 7.0, device="cuda", dtype=torch.float32)
    with pytest.raises(ra.RAError) as e:
        ra.decode_partial_noalloc(q, k, v, 0, S, SCALE, o_part, lse_part)
    assert e.value.status == ra.RA_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    # rejected before anything was enqueued: the outputs are untouched
    assert bool((o_part == 7.0).all()) and bool((lse_part == 7.0).all())
    assert ra.get_status() == ra.RA_OK
