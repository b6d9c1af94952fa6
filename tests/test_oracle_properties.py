"""Property-based pins of the oracle's contractions over random small shapes.

Fixed-shape pins can miss an indexing mistake that only shows for some
shapes (a transposed operand when two sizes happen to coincide, a stride
that is right only for square inputs).  These draw the sizes and values:
the triangular multiplicative update against numpy einsum in both edge
directions ("Evoformer: the memory wall ZeRO cannot move", section "The three
operations"), and the outer product mean against einsum with unequal
channel counts and column subsets, plus its invariance to the order of the
sequences (same page, section "Two properties the tests assert").
"""
import numpy as np
from hypothesis import given, settings, strategies as st

import oracle

SETTINGS = dict(max_examples=25, deadline=None)


@settings(**SETTINGS)
@given(B=st.integers(1, 2), N=st.integers(1, 9), C=st.integers(1, 4), seed=st.integers(0, 2**31 - 1),
       incoming=st.booleans())
def test_tri_mul_matches_einsum_for_any_shape(B, N, C, seed, incoming):
    r = np.random.default_rng(seed)
    a, b = r.standard_normal((B, N, N, C)), r.standard_normal((B, N, N, C))
    ref = np.einsum("bkic,bkjc->bijc" if incoming else "bikc,bjkc->bijc", a, b)
    np.testing.assert_allclose(oracle.tri_mul(a, b, incoming), ref, rtol=1e-12, atol=1e-12)


@settings(**SETTINGS)
@given(B=st.integers(1, 2), S=st.integers(1, 7), N=st.integers(1, 8), Ca=st.integers(1, 5),
       Cb=st.integers(1, 5), seed=st.integers(0, 2**31 - 1))
def test_outer_product_mean_matches_einsum_for_any_shape(B, S, N, Ca, Cb, seed):
    r = np.random.default_rng(seed)
    a, b = r.standard_normal((B, S, N, Ca)), r.standard_normal((B, S, N, Cb))
    ref = np.einsum("bsic,bsjd->bijcd", a, b) / S
    np.testing.assert_allclose(oracle.outer_product_mean(a, b), ref, rtol=1e-12, atol=1e-12)
    # a subset of columns i is the matching block
    idx = np.arange(0, N, 2)
    np.testing.assert_array_equal(oracle.outer_product_mean(np.ascontiguousarray(a[:, :, idx]), b),
                                  oracle.outer_product_mean(a, b)[:, idx])


@settings(**SETTINGS)
@given(S=st.integers(2, 8), N=st.integers(1, 6), seed=st.integers(0, 2**31 - 1))
def test_outer_product_mean_ignores_sequence_order(S, N, seed):
    r = np.random.default_rng(seed)
    a, b = r.standard_normal((1, S, N, 3)), r.standard_normal((1, S, N, 2))
    perm = r.permutation(S)
    np.testing.assert_allclose(oracle.outer_product_mean(a[:, perm], b[:, perm]), oracle.outer_product_mean(a, b),
                               rtol=0, atol=1e-12)
