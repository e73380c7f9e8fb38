"""GPU parity of the striped split (token p in partition p mod P): the fused
striped ring and the strided block partials, against the fp64 oracle on the
same seeded inputs."""
import math
import zlib

import numpy as np
import pytest
import torch

from oracle.attention import attention as oracle_attention
from ring_context_parallelism_ra_b200 import ra
from ring_context_parallelism_ra_b200.workloads import make_qkv, striped_order
from tests.parity_util import check_lse, check_out

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _seed(case):
    return zlib.crc32(repr(case).encode()) % 100000


@pytest.fixture(autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    yield
    assert ra.get_status() == ra.RA_OK


CASES = [
    # B, Hq, Hkv, n, dqk, dv, P, dtype
    (1, 4, 2, 1024, 128, 128, 4, torch.bfloat16),
    (1, 2, 2, 2048, 128, 128, 8, torch.bfloat16),
    (2, 2, 1, 768, 192, 128, 3, torch.bfloat16),
    (1, 2, 1, 512, 64, 64, 2, torch.bfloat16),
    (1, 2, 1, 512, 128, 128, 2, torch.float32),
    (1, 1, 1, 1024, 64, 64, 4, torch.float32),
]


@pytest.mark.parametrize("case", CASES)
def test_striped_ring_matches_oracle(case):
    B, Hq, Hkv, n, dqk, dv, P, dt = case
    q, k, v = make_qkv(B, Hq, Hkv, n, n, dqk, dv, dt, seed=_seed(case))
    order = torch.tensor(striped_order(n, P))
    scale = 1.0 / math.sqrt(dqk)
    out, lse = ra.ring_forward_striped(q[:, :, order].contiguous().to(DEV),
                                       k[:, :, order].contiguous().to(DEV),
                                       v[:, :, order].contiguous().to(DEV), P, True, scale)
    inv = torch.argsort(order)
    want_o, want_l = oracle_attention(q, k, v, scale, True)
    kind = "f32" if dt == torch.float32 else "bf16"
    check_out(out[:, :, inv.to(DEV)], want_o, kind)
    check_lse(lse[:, :, inv.to(DEV)], want_l)


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float32])
def test_striped_block_partials_merge_to_the_striped_ring(dt):
    B, Hq, Hkv, n, d, P = 1, 2, 1, 1024, 128, 4
    L = n // P
    q, k, v = make_qkv(B, Hq, Hkv, n, n, d, d, dt, seed=77)
    order = striped_order(n, P)
    qs = q[:, :, order].contiguous().to(DEV)
    ks = k[:, :, order].contiguous().to(DEV)
    vs = v[:, :, order].contiguous().to(DEV)
    kind = "f32" if dt == torch.float32 else "bf16"
    ring_o, ring_l = ra.ring_forward_striped(qs, ks, vs, P, True)
    for i in range(P):
        o_parts = torch.empty((P, B, Hq, L, d), device=DEV)
        l_parts = torch.empty((P, B, Hq, L), device=DEV)
        qp = np.arange(i, n, P)
        for s in range(P):
            j = (i - s) % P
            kp = np.arange(j, n, P)
            qi = qs[:, :, i * L:(i + 1) * L].contiguous()
            kj = ks[:, :, j * L:(j + 1) * L].contiguous()
            vj = vs[:, :, j * L:(j + 1) * L].contiguous()
            ra.block_partial_strided(qi, kj, vj, i, j, P, True, None, o_parts[s], l_parts[s])
            want_o, want_l = oracle_attention(qi.cpu(), kj.cpu(), vj.cpu(), 1 / math.sqrt(d), True,
                                              q_positions=qp, k_positions=kp)
            check_out(o_parts[s], want_o, kind, f"block ({i},{j}) O")
            check_lse(l_parts[s], want_l, f"block ({i},{j}) LSE")
        o_i, l_i = ra.lse_merge(o_parts, l_parts, dt)
        check_out(o_i, ring_o[:, :, i * L:(i + 1) * L].float().cpu().numpy(), kind, "merged vs ring")
        check_lse(l_i, ring_l[:, :, i * L:(i + 1) * L].cpu().numpy(), "merged vs ring LSE")


def test_striped_requires_whole_tile_pairs_per_partition():
    q = torch.zeros((1, 1, 1000, 128), device=DEV, dtype=torch.bfloat16)
    with pytest.raises(ra.RAError) as e:
        ra.ring_forward_striped(q, q, q, 4, True)     # 250-token partitions
    assert e.value.status == ra.RA_ERR_UNSUPPORTED
