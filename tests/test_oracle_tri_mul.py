"""Pins of the oracle's triangular multiplicative update (its contraction).

Edge (i, j) is updated from every third residue k, channel by channel:
z[i, j] = sum_k a[i, k] * b[j, k] for outgoing edges, sum_k a[k, i] * b[k, j]
for incoming ones ("Evoformer: the memory wall ZeRO cannot move", section
"The three operations").  The oracle is pinned against an independent
library routine (numpy einsum), a hand-computed example, closed forms,
symmetry, the residue-permutation equivariance the same page asserts
(section "Two properties the tests assert"), and the page's own broken
counterexample (the third index dropped), which must fail the pins.
"""
import numpy as np
import pytest

import oracle


def rnd(B, N, C, seed):
    r = np.random.default_rng(seed)
    return r.standard_normal((B, N, N, C)), r.standard_normal((B, N, N, C))


def rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


@pytest.mark.parametrize("B,N,C", [(1, 5, 3), (2, 17, 8), (1, 40, 16)])
def test_matches_einsum(B, N, C):
    a, b = rnd(B, N, C, N * C)
    assert rel(oracle.tri_mul(a, b), np.einsum("bikc,bjkc->bijc", a, b)) < 1e-13
    assert rel(oracle.tri_mul(a, b, incoming=True), np.einsum("bkic,bkjc->bijc", a, b)) < 1e-13


def test_hand_computed_two_residues():
    a = np.array([[1.0, 2.0], [3.0, 4.0]]).reshape(1, 2, 2, 1)
    b = np.array([[5.0, 6.0], [7.0, 8.0]]).reshape(1, 2, 2, 1)
    # outgoing: z_ij = sum_k a_ik b_jk = (a b^T)_ij
    assert np.array_equal(oracle.tri_mul(a, b)[0, :, :, 0], [[17.0, 23.0], [39.0, 53.0]])
    # incoming: z_ij = sum_k a_ki b_kj = (a^T b)_ij
    assert np.array_equal(oracle.tri_mul(a, b, incoming=True)[0, :, :, 0], [[26.0, 30.0], [38.0, 44.0]])


def test_ones_give_row_sums():
    # a = 1: every edge (i, j) sees the sum over k of b[j, k] (outgoing) / b[k, j] (incoming)
    _, b = rnd(1, 9, 4, 3)
    a = np.ones_like(b)
    z = oracle.tri_mul(a, b)
    for i in range(9):
        assert np.allclose(z[0, i], b[0].sum(axis=1), rtol=0, atol=1e-13)
    zi = oracle.tri_mul(a, b, incoming=True)
    for i in range(9):
        assert np.allclose(zi[0, i], b[0].sum(axis=0), rtol=0, atol=1e-13)


def test_equal_operands_give_a_symmetric_update():
    a, _ = rnd(1, 12, 5, 4)
    z = oracle.tri_mul(a, a)
    assert np.allclose(z, z.transpose(0, 2, 1, 3), rtol=0, atol=1e-13)


def test_incoming_is_outgoing_on_the_transposed_pair():
    a, b = rnd(2, 11, 3, 5)
    t = lambda x: np.ascontiguousarray(x.transpose(0, 2, 1, 3))
    assert np.allclose(oracle.tri_mul(a, b, incoming=True), oracle.tri_mul(t(a), t(b)), rtol=0, atol=1e-13)


def test_residue_permutation_equivariance():
    # relabelling the residues relabels the update on both axes
    a, b = rnd(1, 14, 6, 6)
    perm = np.random.default_rng(7).permutation(14)
    p = lambda x: x[:, perm][:, :, perm]
    for inc in (False, True):
        assert np.allclose(oracle.tri_mul(p(a), p(b), incoming=inc), p(oracle.tri_mul(a, b, incoming=inc)),
                           rtol=0, atol=1e-12)


def test_channels_are_independent():
    a, b = rnd(1, 8, 6, 8)
    z = oracle.tri_mul(a, b)
    for c in range(6):
        assert np.array_equal(z[..., c:c + 1], oracle.tri_mul(a[..., c:c + 1], b[..., c:c + 1]))


@pytest.mark.parametrize("mutant", oracle.TRI_MUL_MUTANTS)
def test_planted_mistakes_fail_the_pins(mutant):
    assert oracle.mutant_id(mutant) == mutant
    a, b = rnd(1, 10, 4, 9)
    ref = np.einsum("bikc,bjkc->bijc", a, b)
    assert rel(oracle.tri_mul(a, b, mutant=mutant), ref) > 0.1
