"""Pins of the oracle's rank-ordered fp32 sum of d_pair_bias partials.

When the rows s of one problem are split over GPUs, each GPU's backward
returns the sum of dS over its own rows, and d_pair_bias is the sum of those
partials: the pair bias is one additive term broadcast over the rows
(MegaFold summary, section "EvoFlash-3D"), and a sequence-parallel group
partitions the pair tensor's rows (same page, section "EvoSP-3D").  The
exchange adds the partials left to right in fp32.  The pins: worked IEEE
binary32 cases where the order decides the result, exact integer sums, the
recursive-summation error bound against an fp64 sum, the split of a small
problem's rows by row_range whose partials (from the oracle's backward) add
up to the unsplit d_pair_bias, and two planted mistakes that must fail.
"""
import numpy as np
import pytest

import oracle
from evoformer_pair_bias_b200.row_shards import row_range
from evoformer_pair_bias_b200.workloads import Workload, make_inputs


def col(*xs):
    return np.array(xs, np.float64).reshape(len(xs), 1)


def test_order_decides_and_is_left_to_right():
    # binary32 has a 24-bit significand: 1e8 + 1 rounds back to 1e8, so
    # ((1 + 1e8) - 1e8) = 0 while ((-1e8 + 1e8) + 1) = 1
    assert oracle.ordered_sum_f32(col(1.0, 1e8, -1e8))[0] == 0.0
    assert oracle.ordered_sum_f32(col(-1e8, 1e8, 1.0))[0] == 1.0
    # 2^24 + 1 is a tie between 2^24 and 2^24 + 2 and rounds to the even 2^24, twice
    assert oracle.ordered_sum_f32(col(2.0 ** 24, 1.0, 1.0))[0] == 2.0 ** 24
    assert oracle.ordered_sum_f32(col(1.0, 1.0, 2.0 ** 24))[0] == 2.0 ** 24 + 2


@pytest.mark.parametrize("count", [1, 2, 5, 64])
def test_small_integers_add_exactly(count):
    r = np.random.default_rng(count)
    parts = r.integers(-1000, 1000, size=(count, 37))
    got = oracle.ordered_sum_f32(parts.astype(np.float64))
    assert np.array_equal(got.astype(np.int64), parts.sum(axis=0))


def test_single_partial_is_returned_unchanged():
    x = np.random.default_rng(2).standard_normal((1, 3, 4)).astype(np.float32)
    assert np.array_equal(oracle.ordered_sum_f32(x), x[0])


def test_within_the_recursive_summation_bound():
    # |fl(sum) - sum| <= (count - 1) u sum|p| + O(u^2), u = 2^-24 (recursive summation)
    r = np.random.default_rng(3)
    parts = (r.standard_normal((9, 500)) * 10.0 ** r.integers(-3, 4, size=(9, 1))).astype(np.float32)
    exact = parts.astype(np.float64).sum(axis=0)
    bound = 8 * 2.0 ** -24 * np.abs(parts.astype(np.float64)).sum(axis=0) * (1 + 1e-6)
    assert np.all(np.abs(oracle.ordered_sum_f32(parts) - exact) <= bound)


@pytest.mark.parametrize("S,world", [(7, 2), (7, 3), (2, 3)])
def test_row_blocks_partials_add_up_to_the_full_gradient(S, world):
    w = Workload("split", 1, S, 16, 2, 8, "f32", "msa_row", 1.0, "frac:0.2", 31 + S)
    x = {k: (None if v is None else v.double().numpy()) for k, v in make_inputs(w, device="cpu").items()}
    full = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["mask_bias"], x["pair_bias"], x["dout"],
                           want=("d_pair_bias",))["d_pair_bias"]
    parts = []
    for rank in range(world):
        s0, s1 = row_range(S, world, rank)
        if s1 == s0:                                   # an empty block adds the empty sum
            parts.append(np.zeros_like(full))
            continue
        sl = {k: (v if v is None or k == "pair_bias" else v[:, s0:s1]) for k, v in x.items()}
        parts.append(oracle.backward(sl["q"], sl["k"], sl["v"], sl["g"], sl["mask_bias"], sl["pair_bias"],
                                     sl["dout"], want=("d_pair_bias",))["d_pair_bias"])
    got = oracle.ordered_sum_f32(np.stack(parts))
    assert np.allclose(got, full, rtol=0, atol=world * 2.0 ** -23 * np.abs(np.stack(parts)).sum(axis=0).max())
    assert np.allclose(sum(parts), full, rtol=0, atol=1e-12)


@pytest.mark.parametrize("S,world", [(0, 1), (1, 4), (5, 5), (7, 3), (100, 8), (9, 1)])
def test_row_range_covers_every_row_once(S, world):
    blocks = [row_range(S, world, r) for r in range(world)]
    assert blocks[0][0] == 0 and blocks[-1][1] == S
    assert all(blocks[r][1] == blocks[r + 1][0] for r in range(world - 1))
    sizes = [s1 - s0 for s0, s1 in blocks]
    assert max(sizes) - min(sizes) <= 1 and sizes == sorted(sizes, reverse=True)
    with pytest.raises(ValueError):
        row_range(S, world, world)


@pytest.mark.parametrize("mutant", oracle.PARTIALS_MUTANTS)
def test_planted_mistakes_fail_the_pins(mutant):
    assert oracle.mutant_id(mutant) == mutant
    p = col(1.0, 1e8, -1e8)
    r = np.random.default_rng(4).integers(-9, 9, size=(4, 11)).astype(np.float64)
    wrong_order = oracle.ordered_sum_f32(p, mutant=mutant)[0] != 0.0
    wrong_sum = not np.array_equal(oracle.ordered_sum_f32(r, mutant=mutant), r.sum(axis=0))
    assert wrong_order or wrong_sum
