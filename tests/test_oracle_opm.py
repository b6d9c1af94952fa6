"""Pins of the oracle's outer product mean.

The outer product of MSA columns i and j averaged over the sequences
("Evoformer: the memory wall ZeRO cannot move", section "The three
operations"): out[i, j, c1, c2] = (1/S) sum_s a[s, i, c1] b[s, j, c2].  The
oracle is pinned against numpy einsum, the single-sequence closed form (a
plain outer product), a hand-computed case, the symmetry for a = b, the
residue-permutation equivariance and the invariance to the order of the
sequences that the same page asserts (section "Two properties the tests
assert"), and two planted mistakes that must fail the pins.
"""
import numpy as np
import pytest

import oracle


def rnd(B, S, N, Ca, Cb, seed):
    r = np.random.default_rng(seed)
    return r.standard_normal((B, S, N, Ca)), r.standard_normal((B, S, N, Cb))


def rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


@pytest.mark.parametrize("B,S,N,Ca,Cb", [(1, 3, 4, 2, 3), (2, 7, 9, 4, 4), (1, 16, 12, 8, 5)])
def test_matches_einsum(B, S, N, Ca, Cb):
    a, b = rnd(B, S, N, Ca, Cb, S + N)
    ref = np.einsum("bsic,bsjd->bijcd", a, b) / S
    assert rel(oracle.outer_product_mean(a, b), ref) < 1e-13


def test_single_sequence_is_the_outer_product():
    a, b = rnd(1, 1, 5, 3, 4, 1)
    out = oracle.outer_product_mean(a, b)
    for i in range(5):
        for j in range(5):
            assert np.allclose(out[0, i, j], np.outer(a[0, 0, i], b[0, 0, j]), rtol=0, atol=1e-15)


def test_hand_computed_two_sequences():
    # S = 2, N = 1, one channel each: out = (a0 b0 + a1 b1) / 2
    a = np.array([1.0, 3.0]).reshape(1, 2, 1, 1)
    b = np.array([2.0, 5.0]).reshape(1, 2, 1, 1)
    assert oracle.outer_product_mean(a, b)[0, 0, 0, 0, 0] == (1 * 2 + 3 * 5) / 2


def test_equal_operands_give_the_transposed_pair():
    a, _ = rnd(1, 6, 7, 4, 4, 2)
    out = oracle.outer_product_mean(a, a)
    assert np.allclose(out, out.transpose(0, 2, 1, 4, 3), rtol=0, atol=1e-13)


def test_residue_permutation_equivariance():
    a, b = rnd(1, 5, 8, 3, 2, 3)
    perm = np.random.default_rng(4).permutation(8)
    out = oracle.outer_product_mean(a[:, :, perm], b[:, :, perm])
    assert np.allclose(out, oracle.outer_product_mean(a, b)[:, perm][:, :, perm], rtol=0, atol=1e-13)


def test_sequence_order_does_not_matter():
    a, b = rnd(1, 9, 6, 3, 3, 5)
    perm = np.random.default_rng(6).permutation(9)
    assert np.allclose(oracle.outer_product_mean(a[:, perm], b[:, perm]), oracle.outer_product_mean(a, b),
                       rtol=0, atol=1e-13)


def test_constant_sequences_average_to_themselves():
    # every sequence the same: the mean is that sequence's outer product
    a1, b1 = rnd(1, 1, 4, 2, 2, 7)
    a, b = np.repeat(a1, 5, axis=1), np.repeat(b1, 5, axis=1)
    assert np.allclose(oracle.outer_product_mean(a, b), oracle.outer_product_mean(a1, b1), rtol=0, atol=1e-13)


def test_column_subset_is_the_matching_block():
    # evaluating a subset of columns i gives exactly those rows of the full result
    a, b = rnd(2, 7, 10, 3, 4, 9)
    full = oracle.outer_product_mean(a, b)
    idx = [1, 4, 9]
    assert np.array_equal(oracle.outer_product_mean(np.ascontiguousarray(a[:, :, idx]), b), full[:, idx])


@pytest.mark.parametrize("mutant", oracle.OPM_MUTANTS)
def test_planted_mistakes_fail_the_pins(mutant):
    assert oracle.mutant_id(mutant) == mutant
    a, b = rnd(1, 6, 5, 3, 3, 8)
    ref = np.einsum("bsic,bsjd->bijcd", a, b) / 6
    assert rel(oracle.outer_product_mean(a, b, mutant=mutant), ref) > 0.1
