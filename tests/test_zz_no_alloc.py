"""GPU test of ra_decode_partial_noalloc, the decode entry point for callers
that cannot allocate device memory (a plugin whose host runtime owns all
device memory and offers no allocator, or a latency-critical loop that must
not call cudaMalloc).  It keeps its chunk partials in the library's static
device array instead of a caller workspace; its results must match
ra_decode_partial's, call after call.

This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes on its own in a fresh process.
"""
import math

import pytest
import torch

from ring_context_parallelism_ra_b200 import ra
from ring_context_parallelism_ra_b200.workloads import make_qkv
from tests.parity_util import check_lse, check_out

pytestmark = pytest.mark.gpu


def test_noalloc_decode_matches_workspace_decode_twice():
    assert torch.cuda.is_available(), "GPU test needs a CUDA device"
    dev = "cuda"
    scale = 1 / math.sqrt(128)
    # two different problems, one after the other: the shared static array
    # keeps the first call's contents, which must not leak into the second
    cases = [(2, 16, 2, 10000, 2500, 2500, 11), (4, 64, 8, 131072, 0, 131072, 12)]
    for B, Hq, Hkv, S, start, count, seed in cases:
        q, k, v = make_qkv(B, Hq, Hkv, 1, S, 128, 128, torch.bfloat16, seed=seed, device=dev)
        want_o, want_l = ra.decode_partial(q, k, v, start, count, scale)
        o_part = torch.empty((B, Hq, 128), device=dev, dtype=torch.float32)
        lse_part = torch.empty((B, Hq), device=dev, dtype=torch.float32)
        for _ in range(2):
            o_part.fill_(float("nan"))
            lse_part.fill_(float("nan"))
            got_o, got_l = ra.decode_partial_noalloc(q, k, v, start, count, scale, o_part, lse_part)
            assert ra.get_status() == ra.RA_OK
            check_out(got_o, want_o, "bf16", "noalloc O")
            check_lse(got_l, want_l, "noalloc LSE")


def test_noalloc_decode_rejects_shapes_beyond_its_scratch():
    q = torch.zeros((4, 64, 1, 128), device="cuda", dtype=torch.bfloat16)
    k = torch.empty((4, 8, 1 << 19, 128), device="cuda", dtype=torch.bfloat16)
    with pytest.raises(ra.RAError) as e:
        ra.decode_partial_noalloc(q, k, k)         # 256 chunks x 256 rows: 34 MB > 16 MiB
    assert e.value.status == ra.RA_ERR_UNSUPPORTED
