"""Pins for the fp64 CPU oracle (no GPU).

The oracle is only trusted once it agrees with things other than itself:

* a library special case: with the gate saturated (g = 40 gives sigmoid(g) == 1
  exactly in fp64) the op is ``torch.nn.functional.scaled_dot_product_attention``
  with a float attention mask ``mask_bias + pair_bias``; autograd of that call
  gives dq, dk, dv and d_pair_bias (the sum over the broadcast row axis s);
* closed forms: the gate, dg, a single key, q = 0 (mean of v over unmasked keys),
  v = 1 (softmax rows sum to one);
* invariants: masked keys contribute exactly zero, shift invariance of a bias
  row, lse bounds, residue-permutation equivariance (the property test of
  "Evoformer: the memory wall ZeRO cannot move", section "Two properties the
  tests assert"), row-permutation equivariance, sum rules of the backward;
* central finite differences in fp64 for every gradient;
* planted mistakes (the page's "counterexample that makes the check mean
  something", same section): each mutant build of the oracle must fail the
  pins by orders of magnitude.
"""
import numpy as np
import pytest
import torch

import oracle

RTOL = 1e-12


def rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.linalg.norm(b.ravel())
    return float(np.linalg.norm((a - b).ravel()) / (den if den > 0 else 1.0))


def make(B, S, N, H, C, seed, masked=(), bias=True, gsat=False, Nq=None):
    rng = np.random.default_rng(seed)
    Nq = N if Nq is None else Nq
    q = rng.standard_normal((B, S, Nq, H, C))
    k = rng.standard_normal((B, S, N, H, C))
    v = rng.standard_normal((B, S, N, H, C))
    g = np.full((B, S, Nq, H, C), 40.0) if gsat else rng.standard_normal((B, S, Nq, H, C))
    pb = rng.standard_normal((B, 1, H, Nq, N)) if bias else None
    m = None
    if masked is not None and len(masked):
        m = np.zeros((B, S, 1, 1, N))
        m[..., list(masked)] = -1e9
    dout = rng.standard_normal((B, S, Nq, H, C))
    return dict(q=q, k=k, v=v, g=g, mask_bias=m, pair_bias=pb, dout=dout)


def sdpa_reference(t):
    """Ungated attention via torch SDPA (fp64, CPU) + autograd; returns (out, grads)."""
    B, S, N, H, C = t["q"].shape
    Nk = t["k"].shape[2]
    q = torch.tensor(t["q"], requires_grad=True)
    k = torch.tensor(t["k"], requires_grad=True)
    v = torch.tensor(t["v"], requires_grad=True)
    pb = None if t["pair_bias"] is None else torch.tensor(t["pair_bias"], requires_grad=True)
    to_bh = lambda x: x.permute(0, 1, 3, 2, 4).reshape(B * S, H, x.shape[2], C)  # noqa: E731
    mask = torch.zeros((B, S, H, N, Nk), dtype=torch.float64)
    if t["mask_bias"] is not None:
        mask = mask + torch.tensor(t["mask_bias"]).reshape(B, S, 1, 1, Nk)
    if pb is not None:
        mask = mask + pb.expand(B, S, H, N, Nk)
    o = torch.nn.functional.scaled_dot_product_attention(
        to_bh(q), to_bh(k), to_bh(v), attn_mask=mask.reshape(B * S, H, N, Nk))
    o = o.reshape(B, S, H, N, C).permute(0, 1, 3, 2, 4)
    o.backward(torch.tensor(t["dout"]))
    grads = dict(dq=q.grad.numpy(), dk=k.grad.numpy(), dv=v.grad.numpy())
    if pb is not None:
        grads["d_pair_bias"] = pb.grad.numpy()
    return o.detach().numpy(), grads


SHAPES = [  # (B, S, N, H, C, masked residues)
    (1, 4, 32, 4, 8, range(28, 32)),
    (1, 3, 17, 2, 32, (0, 5)),
    (2, 2, 9, 3, 16, ()),
    (1, 2, 40, 1, 4, (39,)),
]


@pytest.mark.parametrize("B,S,N,H,C,masked", SHAPES)
def test_matches_sdpa_and_autograd(B, S, N, H, C, masked):
    t = make(B, S, N, H, C, seed=1 + N, masked=masked, gsat=True)
    out, lse = oracle.forward(t["q"], t["k"], t["v"], t["g"], t["mask_bias"], t["pair_bias"])
    ref, grads = sdpa_reference(t)
    assert rel(out, ref) < RTOL
    got = oracle.backward(t["q"], t["k"], t["v"], t["g"], t["mask_bias"], t["pair_bias"], t["dout"])
    for name, val in grads.items():
        assert rel(got[name], val) < 1e-11, name


def test_zero_bias_no_mask_is_plain_multihead_attention():
    t = make(1, 3, 24, 2, 16, seed=7, masked=(), bias=False, gsat=True)
    out, _ = oracle.forward(t["q"], t["k"], t["v"], t["g"], None, None)
    ref, grads = sdpa_reference(t)
    assert rel(out, ref) < RTOL
    got = oracle.backward(t["q"], t["k"], t["v"], t["g"], None, None, t["dout"],
                          want=("dq", "dk", "dv"))
    for name in ("dq", "dk", "dv"):
        assert rel(got[name], grads[name]) < 1e-11


def test_gate_and_dg_closed_form():
    t = make(1, 2, 20, 2, 8, seed=11, masked=(3,))
    sat = dict(t, g=np.full_like(t["g"], 40.0))
    A, lse_a = oracle.forward(sat["q"], sat["k"], sat["v"], sat["g"], t["mask_bias"], t["pair_bias"])
    out, lse = oracle.forward(t["q"], t["k"], t["v"], t["g"], t["mask_bias"], t["pair_bias"])
    sig = 1.0 / (1.0 + np.exp(-t["g"]))
    assert rel(out, sig * A) < RTOL
    assert np.array_equal(lse, lse_a)
    dg = oracle.backward(t["q"], t["k"], t["v"], t["g"], t["mask_bias"], t["pair_bias"],
                         t["dout"], want=("dg",))["dg"]
    assert rel(dg, t["dout"] * A * sig * (1 - sig)) < RTOL


def test_rows_sum_to_one():
    t = make(1, 2, 33, 3, 8, seed=5, masked=(1, 2, 30))
    v1 = np.ones_like(t["v"])
    out, _ = oracle.forward(t["q"], t["k"], v1, t["g"], t["mask_bias"], t["pair_bias"])
    sig = 1.0 / (1.0 + np.exp(-t["g"]))
    assert np.max(np.abs(out / sig - 1.0)) < 1e-13


def test_masked_keys_contribute_exactly_zero():
    masked = (0, 7, 8, 19)
    t = make(1, 3, 20, 2, 8, seed=9, masked=masked)
    base_o, base_l = oracle.forward(t["q"], t["k"], t["v"], t["g"], t["mask_bias"], t["pair_bias"])
    base_g = oracle.backward(t["q"], t["k"], t["v"], t["g"], t["mask_bias"], t["pair_bias"], t["dout"])
    k2, v2 = t["k"].copy(), t["v"].copy()
    rng = np.random.default_rng(3)
    for j in masked:
        k2[:, :, j] += 5 * rng.standard_normal(k2[:, :, j].shape)
        v2[:, :, j] += 5 * rng.standard_normal(v2[:, :, j].shape)
    o, l = oracle.forward(t["q"], k2, v2, t["g"], t["mask_bias"], t["pair_bias"])
    assert np.array_equal(o, base_o) and np.array_equal(l, base_l)
    gr = oracle.backward(t["q"], k2, v2, t["g"], t["mask_bias"], t["pair_bias"], t["dout"])
    for name in ("dq", "dg"):
        assert np.array_equal(gr[name], base_g[name])
    for j in masked:
        assert np.all(gr["dk"][:, :, j] == 0) and np.all(gr["dv"][:, :, j] == 0)
        assert np.all(gr["d_pair_bias"][..., j] == 0)


def test_q_zero_gives_mean_of_unmasked_v():
    masked = (2, 4, 11)
    t = make(1, 2, 13, 2, 8, seed=13, masked=masked, bias=False, gsat=True)
    q0 = np.zeros_like(t["q"])
    out, lse = oracle.forward(q0, t["k"], t["v"], t["g"], t["mask_bias"], None)
    keep = [j for j in range(13) if j not in masked]
    mean_v = t["v"][:, :, keep].mean(axis=2, keepdims=True)
    assert rel(out, np.broadcast_to(mean_v, out.shape)) < RTOL
    assert np.max(np.abs(lse - np.log(len(keep)))) < 1e-13


def test_single_key():
    t = make(2, 3, 1, 2, 8, seed=17, masked=(), gsat=False)
    m = np.full((2, 3, 1, 1, 1), 0.25)
    out, lse = oracle.forward(t["q"], t["k"], t["v"], t["g"], m, t["pair_bias"])
    sig = 1.0 / (1.0 + np.exp(-t["g"]))
    assert rel(out, sig * t["v"]) < RTOL
    dot = np.einsum("bsihc,bsjhc->bshij", t["q"], t["k"])[..., 0, 0] / np.sqrt(8)
    expect = dot + 0.25 + t["pair_bias"][:, 0, :, 0, 0][:, None, :]
    assert np.max(np.abs(lse[..., 0] - expect)) < 1e-13


def test_bias_row_shift_invariance():
    t = make(1, 2, 15, 3, 8, seed=19, masked=(14,))
    shift = np.random.default_rng(0).standard_normal((1, 1, 3, 15, 1)) * 3
    o1, l1 = oracle.forward(t["q"], t["k"], t["v"], t["g"], t["mask_bias"], t["pair_bias"])
    o2, l2 = oracle.forward(t["q"], t["k"], t["v"], t["g"], t["mask_bias"], t["pair_bias"] + shift)
    assert rel(o2, o1) < RTOL
    assert np.max(np.abs(l2 - l1 - shift[:, 0, :, :, 0][:, None])) < 1e-12


def test_lse_bounds():
    t = make(1, 3, 21, 2, 16, seed=23, masked=(0, 20))
    _, lse = oracle.forward(t["q"], t["k"], t["v"], t["g"], t["mask_bias"], t["pair_bias"])
    x = (np.einsum("bsihc,bsjhc->bshij", t["q"], t["k"]) / 4.0
         + t["mask_bias"].reshape(1, 3, 1, 1, 21) + t["pair_bias"][:, 0][:, None])
    mx = x.max(axis=-1)
    assert np.all(lse >= mx - 1e-12) and np.all(lse <= mx + np.log(21) + 1e-12)


def test_residue_permutation_equivariance():
    N = 18
    t = make(1, 2, N, 2, 8, seed=29, masked=(3, 10))
    perm = np.random.default_rng(1).permutation(N)
    P = lambda x: x[:, :, perm]  # noqa: E731
    tp = dict(q=P(t["q"]), k=P(t["k"]), v=P(t["v"]), g=P(t["g"]), dout=P(t["dout"]),
              mask_bias=t["mask_bias"][..., perm],
              pair_bias=t["pair_bias"][..., perm, :][..., perm])
    o, l = oracle.forward(t["q"], t["k"], t["v"], t["g"], t["mask_bias"], t["pair_bias"])
    op, lp = oracle.forward(tp["q"], tp["k"], tp["v"], tp["g"], tp["mask_bias"], tp["pair_bias"])
    assert rel(op, P(o)) < RTOL and rel(lp, l[..., perm]) < RTOL
    g = oracle.backward(t["q"], t["k"], t["v"], t["g"], t["mask_bias"], t["pair_bias"], t["dout"])
    gp = oracle.backward(tp["q"], tp["k"], tp["v"], tp["g"], tp["mask_bias"], tp["pair_bias"], tp["dout"])
    for name in ("dq", "dk", "dv", "dg"):
        assert rel(gp[name], P(g[name])) < 1e-11, name
    assert rel(gp["d_pair_bias"], g["d_pair_bias"][..., perm, :][..., perm]) < 1e-11


def test_row_permutation_equivariance_and_bias_grad_invariance():
    S = 5
    t = make(1, S, 12, 2, 8, seed=31, masked=(4,))
    t["mask_bias"][0, 2, 0, 0, 7] = -1e9          # rows carry different masks
    perm = np.random.default_rng(2).permutation(S)
    P = lambda x: x[:, perm]  # noqa: E731
    tp = {n: (P(x) if n != "pair_bias" else x) for n, x in t.items()}
    o, l = oracle.forward(t["q"], t["k"], t["v"], t["g"], t["mask_bias"], t["pair_bias"])
    op, lp = oracle.forward(tp["q"], tp["k"], tp["v"], tp["g"], tp["mask_bias"], tp["pair_bias"])
    assert rel(op, P(o)) < RTOL and rel(lp, P(l)) < RTOL
    g = oracle.backward(*(t[n] for n in ("q", "k", "v", "g", "mask_bias", "pair_bias", "dout")))
    gp = oracle.backward(*(tp[n] for n in ("q", "k", "v", "g", "mask_bias", "pair_bias", "dout")))
    for name in ("dq", "dk", "dv", "dg"):
        assert rel(gp[name], P(g[name])) < 1e-11
    assert rel(gp["d_pair_bias"], g["d_pair_bias"]) < 1e-12


def test_backward_sum_rules():
    t = make(1, 3, 16, 2, 8, seed=37, masked=(5,))
    g = oracle.backward(*(t[n] for n in ("q", "k", "v", "g", "mask_bias", "pair_bias", "dout")))
    scale = np.max(np.abs(g["d_pair_bias"]))
    assert np.max(np.abs(g["d_pair_bias"].sum(axis=-1))) < 1e-12 * max(1.0, scale) * 16
    assert np.max(np.abs(g["dk"].sum(axis=2))) < 1e-11
    sig = 1.0 / (1.0 + np.exp(-t["g"]))
    dA = t["dout"] * sig
    assert np.max(np.abs(g["dv"].sum(axis=2) - dA.sum(axis=2))) < 1e-11


def _fd_check(t, eps=1e-6, mutant=0):
    """Max relative error between oracle gradients and central differences of sum(out * dout)."""
    names = ("q", "k", "v", "g", "pair_bias")
    gmap = {"q": "dq", "k": "dk", "v": "dv", "g": "dg", "pair_bias": "d_pair_bias"}
    got = oracle.backward(*(t[n] for n in ("q", "k", "v", "g", "mask_bias", "pair_bias", "dout")),
                          mutant=mutant)

    def loss(tt):
        o, _ = oracle.forward(tt["q"], tt["k"], tt["v"], tt["g"], tt["mask_bias"], tt["pair_bias"],
                              mutant=mutant)
        return float(np.sum(o * tt["dout"]))

    worst = 0.0
    for n in names:
        x = t[n]
        fd = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            tp = {kk: (vv.copy() if kk == n else vv) for kk, vv in t.items()}
            tm = {kk: (vv.copy() if kk == n else vv) for kk, vv in t.items()}
            tp[n][idx] += eps
            tm[n][idx] -= eps
            fd[idx] = (loss(tp) - loss(tm)) / (2 * eps)
        worst = max(worst, rel(got[gmap[n]], fd))
    return worst


@pytest.mark.parametrize("B,S,N,H,C,masked", [(1, 2, 5, 2, 4, (4,)), (2, 3, 7, 1, 3, ()),
                                              (1, 1, 8, 2, 4, (0, 1))])
def test_finite_differences(B, S, N, H, C, masked):
    t = make(B, S, N, H, C, seed=41 + N, masked=masked)
    assert _fd_check(t) < 1e-6


def test_query_subset_equals_full_rows():
    """Evaluating the definition at a subset of query rows (Nq < Nk) reproduces those rows."""
    t = make(1, 3, 19, 2, 8, seed=43, masked=(2, 18))
    rows = [0, 5, 18]
    full_o, full_l = oracle.forward(t["q"], t["k"], t["v"], t["g"], t["mask_bias"], t["pair_bias"])
    full_g = oracle.backward(*(t[n] for n in ("q", "k", "v", "g", "mask_bias", "pair_bias", "dout")))
    sub = dict(t, q=t["q"][:, :, rows], g=t["g"][:, :, rows], dout=t["dout"][:, :, rows],
               pair_bias=t["pair_bias"][..., rows, :])
    o, l = oracle.forward(sub["q"], sub["k"], sub["v"], sub["g"], sub["mask_bias"], sub["pair_bias"])
    assert np.array_equal(o, full_o[:, :, rows]) and np.array_equal(l, full_l[..., rows])
    gs = oracle.backward(*(sub[n] for n in ("q", "k", "v", "g", "mask_bias", "pair_bias", "dout")),
                         want=("dq", "dg", "d_pair_bias"))
    assert np.array_equal(gs["dq"], full_g["dq"][:, :, rows])
    assert np.array_equal(gs["dg"], full_g["dg"][:, :, rows])
    assert np.array_equal(gs["d_pair_bias"], full_g["d_pair_bias"][..., rows, :])


@pytest.mark.parametrize("mutant", oracle.ATTENTION_MUTANTS)
def test_planted_mistakes_fail_the_pins(mutant):
    """Each planted mistake must be caught, by a margin of many orders of magnitude."""
    assert oracle.mutant_id(mutant) == mutant
    t = make(1, 3, 17, 2, 32, seed=47, masked=(0, 5))
    t_sat = dict(t, g=np.full_like(t["g"], 40.0))
    ref, grads = sdpa_reference(t_sat)
    out, _ = oracle.forward(t["q"], t["k"], t["v"], t["g"], t["mask_bias"], t["pair_bias"],
                            mutant=mutant)
    sig = 1.0 / (1.0 + np.exp(-t["g"]))
    err_fwd = rel(out, sig * ref)
    got = oracle.backward(*(t_sat[n] for n in ("q", "k", "v", "g", "mask_bias", "pair_bias", "dout")),
                          mutant=mutant)
    err_bwd = max(rel(got[n], grads[n]) for n in grads)
    assert max(err_fwd, err_bwd) > 1e-3, (mutant, err_fwd, err_bwd)
    # and the unmutated build passes the same check
    assert rel(oracle.forward(t["q"], t["k"], t["v"], t["g"], t["mask_bias"], t["pair_bias"])[0],
               sig * ref) < RTOL
