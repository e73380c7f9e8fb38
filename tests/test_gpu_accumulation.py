"""GPU test of a property of the hardware that the bars of the long-sum
identity checks rest on: the tensor cores accumulate in fp32 with each step
rounded toward zero, so a long accumulation in tensor memory shrinks
systematically, by up to about 2^-24 of the running sum per K = 16 step.

The probe sums go through the library's own entry points with inputs whose
exact result is a plain sum of positive numbers:
  forward  -- ra_block_partial with q = 0: every score is 0, every weight
              p = 1, so O * n_k = sum_u v_u (one fp32 accumulator per column,
              n_k / 16 steps; l = n_k is exact, and so is dividing by it);
  backward -- ra_block_backward with q = 0 and LSE = ln(n_k): every P is
              2^-7 exactly, so dV_u = 2^-7 sum_t dO_t over n_q / 16 steps.
Rounding to nearest would leave a relative error of order 1e-7 of either
sign; rounding toward zero leaves every column short, by a fraction that
grows with the number of steps.
"""
import math

import numpy as np
import pytest
import torch

from ring_context_parallelism_ra_b200 import ra
from tests.parity_util import ACCUM_SHRINK_PER_STEP

pytestmark = pytest.mark.gpu

N = 131072
STEPS = N // 16


def _check_shrink(got, exact):
    rel = (got - exact) / exact
    # every column short, by more than rounding to nearest could explain and
    # by no more than the per-step allowance the identity bars use
    assert (rel < 0).all(), rel
    assert -STEPS * ACCUM_SHRINK_PER_STEP <= rel.mean() <= -0.1 * STEPS * ACCUM_SHRINK_PER_STEP, \
        rel.mean()


def test_forward_accumulation_rounds_toward_zero():
    assert torch.cuda.is_available(), "GPU test needs a CUDA device"
    g = torch.Generator(device="cuda").manual_seed(5)
    q = torch.zeros((1, 1, 256, 128), device="cuda", dtype=torch.bfloat16)
    k = torch.randn((1, 1, N, 128), device="cuda", generator=g).to(torch.bfloat16)
    v = torch.rand((1, 1, N, 128), device="cuda", generator=g).to(torch.bfloat16)
    o, lse = ra.block_partial(q, k, v, 0, 0, False, 1 / math.sqrt(128))
    assert ra.get_status() == ra.RA_OK
    assert np.allclose(lse.cpu().numpy(), math.log(N), atol=1e-6)
    got = o[0, 0].double().cpu().numpy() * N          # [256 rows, 128 columns]
    assert (got == got[0]).all()                      # every row sums the same keys
    exact = v[0, 0].double().cpu().numpy().sum(axis=0)
    _check_shrink(got[0], exact)


def test_backward_accumulation_rounds_toward_zero():
    assert torch.cuda.is_available(), "GPU test needs a CUDA device"
    g = torch.Generator(device="cuda").manual_seed(6)
    n_k = 128
    q = torch.zeros((1, 1, N, 128), device="cuda", dtype=torch.bfloat16)
    k = torch.randn((1, 1, n_k, 128), device="cuda", generator=g).to(torch.bfloat16)
    v = torch.randn((1, 1, n_k, 128), device="cuda", generator=g).to(torch.bfloat16)
    dout = torch.rand((1, 1, N, 128), device="cuda", generator=g).to(torch.bfloat16)
    lse = torch.full((1, 1, N), math.log(n_k), device="cuda")
    delta = torch.zeros((1, 1, N), device="cuda")
    _, _, dv = ra.block_backward(q, k, v, dout, lse, delta, 0, 0, 1, False, 1 / math.sqrt(128))
    assert ra.get_status() == ra.RA_OK
    got = dv[0, 0].double().cpu().numpy() * n_k       # [keys, columns]
    assert (got == got[0]).all()                      # every key sums the same rows
    exact = dout[0, 0].double().cpu().numpy().sum(axis=0)
    _check_shrink(got[0], exact)
