"""Tolerances and comparison helpers for GPU-vs-oracle parity tests.

Bars (stated for the method's outputs): bf16 inputs with fp32 accumulation
give O within max-abs 2e-2 and mean-abs 2e-3 of the fp64 definition; fp32
inputs give O within 1e-4; the log-sum-exp within 1e-3.

Gradients (backward pass) take the same bars in units of their own size
when that exceeds 1: O is a convex combination of the values (|O| is at most
max |v|, about 4 for N(0,1) inputs), a gradient is not.  Every rounding in
the bf16 backward (P and dS to bf16 before their products, the forward's O
in bf16 inside D = rowsum(dO * O), the bf16 results) is relative, so its
error scales with the gradient: max-abs err <= 2e-2 * max(1, max |ref|) and
mean-abs err <= 2e-3 * max(1, mean |ref|); fp32: 1e-4 * max(1, max |ref|).
"""
import numpy as np
import torch

# The tensor cores' fp32 accumulation rounds each step toward zero
# (tests/test_gpu_accumulation.py measures it), so an accumulator that takes
# `steps` K = 16 steps shrinks by up to about steps x 2^-24 of its size: a
# long positive sum loses on average half an ulp per step, and an ulp is at
# most 2^-23 of the running sum.
ACCUM_SHRINK_PER_STEP = 2.0 ** -24

BF16_MAX_ABS = 2e-2
BF16_MEAN_ABS = 2e-3
F32_MAX_ABS = 1e-4
LSE_MAX_ABS = 1e-3


def to64(x):
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def check_out(got, want, dtype, what="O"):
    """Element-wise comparison of an output against the oracle."""
    g, w = to64(got), to64(want)
    assert g.shape == w.shape, (g.shape, w.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite values"
    err = np.abs(g - w)
    mx, mean = float(err.max()), float(err.mean())
    if dtype in ("f32", torch.float32):
        assert mx <= F32_MAX_ABS, f"{what}: max abs {mx:.3g} > {F32_MAX_ABS}"
    else:
        assert mx <= BF16_MAX_ABS, f"{what}: max abs {mx:.3g} > {BF16_MAX_ABS}"
        assert mean <= BF16_MEAN_ABS, f"{what}: mean abs {mean:.3g} > {BF16_MEAN_ABS}"
    return mx, mean


def check_lse(got, want, what="LSE"):
    g, w = to64(got), to64(want)
    assert g.shape == w.shape, (g.shape, w.shape)
    inf_g, inf_w = np.isneginf(g), np.isneginf(w)
    assert np.array_equal(inf_g, inf_w), f"{what}: -inf pattern differs"
    fin = ~inf_w
    assert np.isfinite(g[fin]).all(), f"{what}: non-finite values"
    mx = float(np.abs(g[fin] - w[fin]).max()) if fin.any() else 0.0
    assert mx <= LSE_MAX_ABS, f"{what}: max abs {mx:.3g} > {LSE_MAX_ABS}"
    return mx


def check_grad(got, want, dtype, what="grad"):
    """Element-wise comparison of a gradient against the oracle, with the bars
    scaled by the reference's magnitude when it exceeds 1."""
    g, w = to64(got), to64(want)
    assert g.shape == w.shape, (g.shape, w.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite values"
    err = np.abs(g - w)
    mx, mean = float(err.max()), float(err.mean())
    s_max = max(1.0, float(np.abs(w).max()))
    s_mean = max(1.0, float(np.abs(w).mean()))
    if dtype in ("f32", torch.float32):
        assert mx <= F32_MAX_ABS * s_max, f"{what}: max abs {mx:.3g} > {F32_MAX_ABS} x {s_max:.3g}"
    else:
        assert mx <= BF16_MAX_ABS * s_max, f"{what}: max abs {mx:.3g} > {BF16_MAX_ABS} x {s_max:.3g}"
        assert mean <= BF16_MEAN_ABS * s_mean, \
            f"{what}: mean abs {mean:.3g} > {BF16_MEAN_ABS} x {s_mean:.3g}"
    return mx, mean


def sum_identity_bar(x, steps, axis):
    """Bar on |sum of n entries - its exact value| for entries each computed by
    the bf16 kernels: the systematic shrinkage of the tensor cores'
    round-toward-zero accumulation (``steps`` K-steps of the longest
    accumulator, ACCUM_SHRINK_PER_STEP each, relative to the entries' sizes)
    plus random rounding, which adds up like a random walk (root sum of
    squares at the bf16 max-abs bar)."""
    if isinstance(x, torch.Tensor):   # reduce where the tensor lives, then fetch
        x = x.double()
        bar = (steps * ACCUM_SHRINK_PER_STEP * x.abs().sum(dim=axis)
               + BF16_MAX_ABS * (x * x).sum(dim=axis).sqrt())
        return to64(bar)
    x = to64(x)
    return (steps * ACCUM_SHRINK_PER_STEP * np.abs(x).sum(axis=axis)
            + BF16_MAX_ABS * np.sqrt((x ** 2).sum(axis=axis)))
