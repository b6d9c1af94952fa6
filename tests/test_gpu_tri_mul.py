"""GPU parity of the triangular multiplicative update contraction against the fp64 oracle.

z[b, c, i, j] = sum_k a[b, c, i, k] b[b, c, j, k] (outgoing edges) or
sum_k a[b, c, k, i] b[b, c, k, j] (incoming), "Evoformer: the memory wall ZeRO
cannot move", section "The three operations".  The kernel reads channel-first
[B, C, N, N] bf16; the oracle gets the same rounded values in its [B, N, N, C]
layout.  Tolerance (tri_mul_bound in the parity helpers, from the
arithmetic): per element 2^-8 |z| + 2^-12 sum_k |a| |b|, and rel-L2 <= 5e-3.
Covers both edge directions, one and several (up to eight or more) tiles per
CTA, ragged edges in i, j and k, the full-size workload, and the degenerate
sizes.
"""
import numpy as np
import pytest
import torch

import oracle
from _parity import TOL, metrics, tri_mul_bound
from evoformer_pair_bias_b200 import attention as A
from evoformer_pair_bias_b200.workloads import TRI_MUL_WORKLOADS, TriMulWorkload, make_tri_mul_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from evoformer_pair_bias_b200 import build
    build.build()
    A.load_library()


def to_oracle(t):                      # [B, C, N, N] -> fp64 [B, N, N, C]
    return t.detach().to("cpu", torch.float64).permute(0, 2, 3, 1).contiguous().numpy()


def check(w, incoming):
    d = make_tri_mul_inputs(w, device="cuda")
    z = A.tri_mul(d["a"], d["b"], incoming=incoming)
    torch.cuda.synchronize()
    a, b = to_oracle(d["a"]), to_oracle(d["b"])
    ref = oracle.tri_mul(a, b, incoming)
    got = to_oracle(z)
    m = metrics(got, ref)
    assert m["finite"], m
    assert m["rel_l2"] <= TOL["bf16"]["rel_l2"], (w.name, incoming, m)
    excess = np.abs(got - ref) - tri_mul_bound(a, b, incoming, ref)
    assert excess.max() <= 0, (w.name, incoming, m, float(excess.max()))
    assert A.device_status(clear=True) == 0
    return m


@pytest.mark.parametrize("incoming", [False, True])
@pytest.mark.parametrize("N,C,B", [(40, 3, 2), (128, 2, 1), (200, 4, 1), (264, 2, 1), (512, 1, 1)])
def test_contraction_matches_the_oracle(N, C, B, incoming):
    check(TriMulWorkload("case", B, N, C, 9000 + N + C), incoming)


@pytest.mark.parametrize("incoming", [False, True])
@pytest.mark.parametrize("N,C", [(128, 300), (128, 400), (136, 160), (192, 300), (256, 160),
                                 (128, 1200), (136, 700)])
def test_several_tiles_per_cta(N, C, incoming):
    # enough channels for two or more tiles per SM, so that CTAs run several tiles through
    # the double-buffered accumulators.  With N not a multiple of 256 some 64-column groups
    # lie wholly past N and store nothing, between groups that do.  The last two cases give
    # every CTA eight or more tiles
    check(TriMulWorkload("many", 1, N, C, 9100 + N + C), incoming)


@pytest.mark.parametrize("incoming", [False, True])
def test_full_size_workload(incoming):
    check(TRI_MUL_WORKLOADS["tri_mul_256"], incoming)


def test_degenerate_sizes_are_no_ops_or_errors():
    lib = A.load_library()
    x = torch.zeros((1, 1, 16, 16), dtype=torch.bfloat16, device="cuda")
    assert lib.evo_tri_mul(0, 1, 16, A._ptr(x), A._ptr(x), 0, A._ptr(x), A._stream(x.device)) == 0
    assert lib.evo_tri_mul(1, 1, 0, A._ptr(x), A._ptr(x), 0, A._ptr(x), A._stream(x.device)) == 0
    y = torch.zeros((1, 1, 12, 12), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(A.EvoError) as e:
        A.tri_mul(y, y)
    assert e.value.code == 2                               # N not a multiple of 8


def test_single_residue_block_is_exact_for_small_integers():
    # small integers are exact in bf16 and their sums of products exact in fp32
    g = torch.Generator("cpu").manual_seed(5)
    a = torch.randint(-3, 4, (1, 2, 8, 8), generator=g).to(torch.bfloat16).cuda()
    b = torch.randint(-3, 4, (1, 2, 8, 8), generator=g).to(torch.bfloat16).cuda()
    for inc in (False, True):
        z = A.tri_mul(a, b, incoming=inc)
        ref = oracle.tri_mul(to_oracle(a), to_oracle(b), inc)
        assert np.array_equal(to_oracle(z), ref)
