"""GPU parity of the outer product mean against the fp64 oracle.

out[b, i, c1, j, c2] = (1/S) sum_s a[b, s, i, c1] b[b, s, j, c2] ("Evoformer:
the memory wall ZeRO cannot move", section "The three operations": the outer
product of MSA columns i and j averaged over the sequences).  The kernel writes
[B, N, Ca, N, Cb]; the comparison takes its pair view [B, N, N, Ca, Cb].
Tolerance (opm_bound in the parity helpers, from the arithmetic): per element
2^-8 |out| + 2^-12 mean_s |a| |b|, and rel-L2 <= 5e-3.  Covers ragged row,
column and sequence counts (M = N Ca, Nc = N Cb not multiples of the tile, S
not a multiple of 64), one sequence, unequal channel counts, several tiles per
CTA, the full-size workload on sampled columns i, and the degenerate sizes.
"""
import numpy as np
import pytest
import torch

import oracle
from _parity import TOL, metrics, opm_bound
from evoformer_pair_bias_b200 import attention as A
from evoformer_pair_bias_b200.workloads import OPM_WORKLOADS, make_opm_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from evoformer_pair_bias_b200 import build
    build.build()
    A.load_library()


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def check(a, b, rows=None):
    out = A.outer_product_mean(a, b)
    torch.cuda.synchronize()
    got = f64(A.opm_pair_view(out))
    af, bf = f64(a), f64(b)
    if rows is not None:                       # sampled columns i (full-size cases)
        af, got = np.ascontiguousarray(af[:, :, rows]), got[:, rows]
    ref = oracle.outer_product_mean(af, bf)
    m = metrics(got, ref)
    assert m["finite"], m
    assert m["rel_l2"] <= TOL["bf16"]["rel_l2"], m
    excess = np.abs(got - ref) - opm_bound(af, bf, ref)
    assert excess.max() <= 0, (m, float(excess.max()))
    assert A.device_status(clear=True) == 0
    return m


def rnd(B, S, N, Ca, Cb, seed):
    g = torch.Generator("cpu").manual_seed(seed)
    a = torch.randn((B, S, N, Ca), generator=g).to(torch.bfloat16).cuda()
    b = torch.randn((B, S, N, Cb), generator=g).to(torch.bfloat16).cuda()
    return a, b


@pytest.mark.parametrize("B,S,N,Ca,Cb", [(2, 5, 12, 8, 8), (1, 1, 40, 8, 8), (2, 33, 20, 8, 16),
                                        (1, 200, 24, 16, 8), (1, 128, 64, 32, 32), (3, 70, 36, 32, 32)])
def test_matches_the_oracle(B, S, N, Ca, Cb):
    check(*rnd(B, S, N, Ca, Cb, 31 * S + N))


def test_full_size_workload_on_sampled_columns():
    w = OPM_WORKLOADS["opm_256"]
    d = make_opm_inputs(w, device="cuda")
    rows = np.random.default_rng(0).choice(w.N, 12, replace=False)
    rows.sort()
    check(d["a"], d["b"], rows=rows)


def test_degenerate_sizes():
    lib = A.load_library()
    x = torch.zeros((1, 2, 8, 8), dtype=torch.bfloat16, device="cuda")
    s = A._stream(x.device)
    assert lib.evo_outer_product_mean(0, 2, 8, 8, 8, A._ptr(x), A._ptr(x), A._ptr(x), s) == 0    # B = 0
    assert lib.evo_outer_product_mean(1, 0, 8, 8, 8, A._ptr(x), A._ptr(x), A._ptr(x), s) == 1    # no mean
    y = torch.zeros((1, 2, 3, 5), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(A.EvoError) as e:
        A.outer_product_mean(y, y)                     # N * C = 15, not a multiple of 8
    assert e.value.code == 2
