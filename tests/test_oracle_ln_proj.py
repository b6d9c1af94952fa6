"""Pins of the oracle's fused pre-attention projection (LayerNorm + linear).

The operation is the pair EvoFusion computes without writing the normalised
tensor to memory (MegaFold summary, section "EvoFusion : Pile d'Operateurs
Fusionnes"): y = LayerNorm(x) @ w + bias over the rows of the MSA or pair
representation.  The oracle is pinned against an independent library
routine (torch fp64 layer_norm and matmul), closed forms, invariances and a
hand-computed example; planted mistakes must fail by orders of magnitude.
"""
import numpy as np
import pytest
import torch

import oracle

RTOL = 1e-12


def rel(a, b):
    return float(np.linalg.norm(np.asarray(a) - np.asarray(b)) / max(np.linalg.norm(np.asarray(b)), 1e-300))


def torch_ref(x, ln_w, ln_b, eps, w, bias):
    xt = torch.tensor(x, dtype=torch.float64)
    n = torch.nn.functional.layer_norm(xt, (x.shape[-1],),
                                       None if ln_w is None else torch.tensor(ln_w, dtype=torch.float64),
                                       None if ln_b is None else torch.tensor(ln_b, dtype=torch.float64), eps)
    y = n @ torch.tensor(w, dtype=torch.float64)
    if bias is not None:
        y = y + torch.tensor(bias, dtype=torch.float64)
    return y.numpy()


def case(rows, c_in, n_out, seed):
    r = np.random.default_rng(seed)
    return (r.standard_normal((rows, c_in)) * 1.7 + 0.3, 1 + 0.1 * r.standard_normal(c_in),
            0.1 * r.standard_normal(c_in), r.standard_normal((c_in, n_out)) / np.sqrt(c_in),
            r.standard_normal(n_out))


@pytest.mark.parametrize("rows,c_in,n_out", [(7, 16, 8), (33, 128, 4), (64, 256, 1024)])
def test_matches_torch_layer_norm_and_matmul(rows, c_in, n_out):
    x, lw, lb, w, b = case(rows, c_in, n_out, seed=rows + c_in)
    assert rel(oracle.ln_linear(x, lw, lb, 1e-5, w, b), torch_ref(x, lw, lb, 1e-5, w, b)) < RTOL


def test_identity_weight_gives_unit_normalised_rows():
    x, _, _, _, _ = case(20, 32, 32, seed=3)
    eps = 1e-5
    y = oracle.ln_linear(x, None, None, eps, np.eye(32))
    var = x.var(axis=1)
    assert np.abs(y.mean(axis=1)).max() < 1e-13
    assert np.abs((y ** 2).mean(axis=1) - var / (var + eps)).max() < 1e-13


def test_constant_rows_give_the_projected_shift():
    c_in, n_out = 24, 6
    _, lw, lb, w, b = case(1, c_in, n_out, seed=5)
    x = np.full((3, c_in), 2.5)
    y = oracle.ln_linear(x, lw, lb, 1e-5, w, b)
    assert np.abs(y - (lb @ w + b)[None, :]).max() < 1e-13


def test_row_shift_and_scale_invariance():
    x, lw, lb, w, b = case(9, 40, 12, seed=7)
    y = oracle.ln_linear(x, lw, lb, 0.0, w, b)
    assert rel(oracle.ln_linear(x + 3.25, lw, lb, 0.0, w, b), y) < 1e-13
    assert rel(oracle.ln_linear(x * 4.0, lw, lb, 0.0, w, b), y) < 1e-13


def test_hand_computed_two_channel_row():
    # x = [1, 3]: mean 2, variance 1, so with eps = 0 the normalised row is [-1, 1]
    w = np.array([[2.0, -1.0, 0.5], [5.0, 4.0, -3.0]])
    y = oracle.ln_linear(np.array([[1.0, 3.0]]), None, None, 0.0, w, np.array([0.25, 0.0, 1.0]))
    assert np.allclose(y, [[5.0 - 2.0 + 0.25, 4.0 + 1.0, -3.0 - 0.5 + 1.0]], rtol=0, atol=1e-15)


@pytest.mark.parametrize("mutant", oracle.LN_LINEAR_MUTANTS)
def test_planted_mistakes_fail_the_pins(mutant):
    assert oracle.mutant_id(mutant) == mutant
    x, lw, lb, w, b = case(17, 64, 48, seed=11)
    ref = torch_ref(x, lw, lb, 1e-5, w, b)
    assert rel(oracle.ln_linear(x, lw, lb, 1e-5, w, b, mutant=mutant), ref) > 1e-3
    assert rel(oracle.ln_linear(x, lw, lb, 1e-5, w, b), ref) < RTOL


def test_projection_bound_covers_a_bf16_emulation_and_is_tight():
    # the GPU tolerance (projection_bound) against a CPU emulation of the
    # tensor-core path's two roundings: LN(x) to bf16 before the product, y to
    # bf16 after it; every element inside the bound, and the bound not vacuous
    from _parity import projection_bound
    r = np.random.default_rng(11)
    rows, c_in, n_out = 4096, 256, 256
    x = torch.tensor(r.standard_normal((rows, c_in))).to(torch.bfloat16).double().numpy()
    w = torch.tensor(r.standard_normal((c_in, n_out)) / 16).to(torch.bfloat16).double().numpy()
    lw, lb, b = 1 + 0.1 * r.standard_normal(c_in), 0.1 * r.standard_normal(c_in), r.standard_normal(n_out)
    ref = oracle.ln_linear(x, lw, lb, 1e-5, w, b)
    ln = torch.nn.functional.layer_norm(torch.tensor(x, dtype=torch.float32), (c_in,),
                                        torch.tensor(lw, dtype=torch.float32), torch.tensor(lb, dtype=torch.float32),
                                        1e-5)
    y = (ln.to(torch.bfloat16).float() @ torch.tensor(w, dtype=torch.float32) + torch.tensor(b, dtype=torch.float32))
    emu = y.to(torch.bfloat16).double().numpy()
    bound = projection_bound(x, lw, lb, 1e-5, w, ref)
    err = np.abs(emu - ref)
    assert np.all(err <= bound)
    assert err.max() > 0.1 * bound.max()                  # the emulation comes within 10x of the bound
    assert not np.all(np.abs(ref + 0.05 - emu) <= bound)  # a 0.05 shift of y is caught
