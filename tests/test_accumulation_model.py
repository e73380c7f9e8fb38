"""CPU check of the rounding model behind the long-sum bars
(tests/parity_util.py: ACCUM_SHRINK_PER_STEP).  A chain of fp32
accumulation steps, each adding the exact sum of 16 products, is emulated
with numpy twice: rounding each step to nearest, and rounding it toward zero
(what the tensor cores do; tests/test_gpu_accumulation.py measures it on the
GPU).  On a long positive sum rounding to nearest leaves no systematic error,
while rounding toward zero leaves the result short by a fraction that grows
in proportion to the number of steps and stays below 2^-24 per step."""
import numpy as np

from tests.parity_util import ACCUM_SHRINK_PER_STEP


def _toward_zero(x64):
    x32 = x64.astype(np.float32)
    over = np.abs(x32.astype(np.float64)) > np.abs(x64)
    x32[over] = np.nextafter(x32[over], np.float32(0))
    return x32


def _chain(terms, toward_zero):
    acc = np.zeros(terms.shape[1], np.float32)
    for i in range(0, terms.shape[0], 16):
        s = acc.astype(np.float64) + terms[i:i + 16].sum(axis=0)
        acc = _toward_zero(s) if toward_zero else s.astype(np.float32)
    return acc.astype(np.float64)


def test_toward_zero_chain_shrinks_in_proportion_to_its_steps():
    rng = np.random.default_rng(3)
    for n in (8192, 32768):
        terms = rng.random((n, 64)).astype(np.float32).astype(np.float64)
        exact = terms.sum(axis=0)
        steps = n // 16
        rel_rn = (_chain(terms, False) - exact) / exact
        rel_rz = (_chain(terms, True) - exact) / exact
        assert np.abs(rel_rn.mean()) < 1e-6
        assert (rel_rz < 0).all()
        assert -steps * ACCUM_SHRINK_PER_STEP <= rel_rz.mean() <= -0.1 * steps * ACCUM_SHRINK_PER_STEP
