"""The FMA-pipe exponential of the attention kernels, pinned on the CPU.

The kernels compute part of their exponentials 2^x without the MUFU unit:
x = n + f with n = round(x) (by the float-rounding constant 1.5 * 2^23), a
cubic in f on [-1/2, 1/2], and n added to the exponent field.  This test reads
the cubic's coefficients from the CUDA source, evaluates the same fp32 steps
in numpy (IEEE single rounding for every add, one rounding per fused
multiply-add) and checks the stated relative error bound, 8e-5, against fp64
2^x over the whole range the kernels use, [-125, 126], and the clamp below it.
The GPU check of the device function itself is tests/test_gpu_exp2.py.
"""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "evoformer_pair_bias_b200", "csrc", "sm100.cuh")
BOUND = 8e-5


def coefficients():
    text = open(SRC).read()
    c = [float(re.search(rf"kExp2C{k}\s*=\s*([0-9.eE+-]+)f", text).group(1)) for k in range(4)]
    rnd = float(re.search(r"kExp2Round\s*=\s*([0-9.eE+-]+)f", text).group(1))
    return np.float32(c), np.float32(rnd)


def fma32(a, b, c):
    """One fp32 rounding of a*b + c (the product is exact in fp64)."""
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_fma_emulated(x):
    c, rnd = coefficients()
    x = np.asarray(x, np.float32)
    xc = np.maximum(x, np.float32(-125.0))
    r = (xc + rnd).astype(np.float32)
    n = (r - rnd).astype(np.float32)
    f = fma32(n, np.float32(-1.0), xc)
    p = fma32(np.full_like(f, c[3]), f, np.full_like(f, c[2]))
    p = fma32(p, f, np.full_like(f, c[1]))
    p = fma32(p, f, np.full_like(f, c[0]))
    bits = p.view(np.uint32).astype(np.uint64) + (r.view(np.uint32).astype(np.uint64) << np.uint64(23))
    return (bits & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)


def sweep():
    fine = np.linspace(-125.0, 126.0, 2_000_001, dtype=np.float64).astype(np.float32)
    ints = np.arange(-125, 127, dtype=np.float32)
    halves = ints[:-1] + np.float32(0.5)
    near = np.concatenate([np.nextafter(halves, np.float32(-np.inf)), np.nextafter(halves, np.float32(np.inf))])
    return np.concatenate([fine, ints, halves, near]).astype(np.float32)


def test_relative_error_bound_over_the_whole_range():
    x = sweep()
    got = exp2_fma_emulated(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got - want) / want
    assert np.all(np.isfinite(got)) and np.all(got > 0)
    assert rel.max() < BOUND, (rel.max(), x[rel.argmax()])
    # and not loose by orders of magnitude: the cubic is a real fit, close to its bound
    assert rel.max() > BOUND / 10


def test_integer_arguments_are_close_to_exact_powers():
    x = np.arange(-125, 127, dtype=np.float32)
    got = exp2_fma_emulated(x).astype(np.float64)
    assert np.all(np.abs(got / np.exp2(x.astype(np.float64)) - 1) < 1e-4)


def test_arguments_below_the_range_clamp_to_two_to_the_minus_125():
    x = np.array([-125.0, -126.0, -200.0, -1e9, -np.inf], np.float32)
    got = exp2_fma_emulated(x).astype(np.float64)
    assert np.all(np.abs(got / 2.0 ** -125 - 1) < BOUND)


def test_a_wrong_coefficient_breaks_the_bound():
    """Planted mistake on the CPU: the bound is tight enough to catch a perturbed cubic."""
    c, _ = coefficients()
    x = sweep()[::7].astype(np.float64)
    n = np.round(x)
    f = x - n
    for k, delta in ((0, 2e-4), (1, 5e-4), (3, 5e-3)):
        cc = c.astype(np.float64).copy()
        cc[k] += delta
        p = ((cc[3] * f + cc[2]) * f + cc[1]) * f + cc[0]
        rel = np.abs(p * np.exp2(n) / np.exp2(x) - 1)
        assert rel.max() > BOUND, k
