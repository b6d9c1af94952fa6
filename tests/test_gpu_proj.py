"""GPU parity of the fused pre-attention projection against the fp64 oracle.

y = LayerNorm(x) @ w + bias (MegaFold summary, section "EvoFusion"): bf16
inputs and outputs, fp32 statistics and accumulation, compared element by
element with the oracle evaluated on the same bf16-rounded inputs.

Tolerance, from the arithmetic (projection_bound in the parity helpers): the
path rounds LN(x) to bf16 before the product and y to bf16 on the store, so
each element must lie within 2^-8 * (|y_ref| + (|LN(x)| @ |w|)_n), and the
tensor's rel-L2 within 5e-3 as for the attention.  The attention's fixed
max-abs 2e-2 does not carry over: y reaches |y| ~ 6 over 3e7 samples, where
half a bf16 ulp alone is 1.6e-2.  The pair-bias path (fp32 operands, one
output rounding) and the attention fed by the projection keep the
attention's tolerances.  Covers both column-tile widths
(n_out a multiple of 256, and of 128 only), every supported c_in, ragged
row counts, the pair-bias projection, and q, k, v, g used by the attention
directly as strided views of the projection's output.
"""
import numpy as np
import pytest
import torch

import oracle
from _parity import TOL, metrics, projection_bound
from evoformer_pair_bias_b200 import attention as A
from evoformer_pair_bias_b200.workloads import PROJ_WORKLOADS, ProjWorkload, make_proj_inputs

pytestmark = pytest.mark.gpu
EPS = 1e-5


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def check(got, ref, name):
    m = metrics(f64(got), ref)
    tol = TOL["bf16"]
    assert m["finite"], (name, m)
    assert m["rel_l2"] <= tol["rel_l2"] and m["max_abs"] <= tol["max_abs"], (name, m)
    return m


def check_projection(got, d, ln_w, ln_b, w, bias, name):
    """Element-wise bound of two bf16 roundings (module docstring) plus rel-L2."""
    x, w = f64(d), f64(w)
    ln_w, ln_b = (None if t is None else f64(t) for t in (ln_w, ln_b))
    ref = oracle.ln_linear(x, ln_w, ln_b, EPS, w, None if bias is None else f64(bias))
    bound = projection_bound(x, ln_w, ln_b, EPS, w, ref)
    g = f64(got)
    m = metrics(g, ref)
    assert m["finite"], (name, m)
    assert m["rel_l2"] <= TOL["bf16"]["rel_l2"], (name, m)
    excess = np.abs(g - ref) - bound
    assert excess.max() <= 0, (name, m, float(excess.max()), np.unravel_index(excess.argmax(), excess.shape))
    return m


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from evoformer_pair_bias_b200 import build
    build.build()
    A.load_library()


@pytest.mark.parametrize("name", ["msa_proj_256", "pair_proj_256", "tiny_proj"])
def test_ln_linear_matches_the_oracle(name):
    w = PROJ_WORKLOADS[name]
    d = make_proj_inputs(w, device="cuda")
    y = A.ln_linear(d["x"], d["ln_w"], d["ln_b"], EPS, d["w"], d["bias"])
    torch.cuda.synchronize()
    check_projection(y, d["x"], d["ln_w"], d["ln_b"], d["w"], d["bias"], name)
    assert A.device_status(clear=True) == 0


@pytest.mark.parametrize("rows,c_in,n_out", [(1, 64, 128), (130, 128, 384), (257, 192, 256), (127, 256, 640),
                                            (296 * 128 + 40, 64, 128), (296 * 128 + 50, 256, 384),
                                            (74 * 128 * 3 + 70, 128, 512)])
def test_ln_linear_shapes_and_ragged_rows(rows, c_in, n_out):
    # the last three cases give CTAs three row blocks with a ragged last one (some epilogue
    # warps have no rows to store right after storing a full block): w resident in one
    # column group, w streamed from L2 (c_in = 256), and two column groups (c_in = 128)
    w = ProjWorkload("shape", 1, 1, rows, c_in, 1, 32, 7000 + rows + c_in)
    d = make_proj_inputs(w, n_out=n_out, device="cuda")
    y = A.ln_linear(d["x"], d["ln_w"], d["ln_b"], EPS, d["w"], d["bias"])
    check_projection(y, d["x"], d["ln_w"], d["ln_b"], d["w"], d["bias"], (rows, c_in, n_out))


def test_ln_linear_defaults_and_row_pitch():
    # no LayerNorm affine, no bias, output written with a wider row pitch
    w = ProjWorkload("pitch", 1, 2, 64, 128, 1, 32, 7100)
    d = make_proj_inputs(w, n_out=256, device="cuda")
    big = torch.full((2 * 64, 384), 7.0, dtype=torch.bfloat16, device="cuda")
    lib = A.load_library()
    x = d["x"].reshape(-1, 128).contiguous()
    rc = lib.evo_ln_linear(x.shape[0], 128, 256, A._ptr(x), None, None, EPS, A._ptr(d["w"]), None, A._ptr(big),
                           384, A._stream(x.device))
    assert rc == 0
    check_projection(big[:, :256], x, None, None, d["w"], None, "pitch")
    assert torch.all(big[:, 256:] == 7.0)                 # columns beyond n_out untouched


def test_pair_bias_projection_matches_the_oracle():
    w = PROJ_WORKLOADS["pair_proj_256"]
    H = w.H
    g = torch.Generator("cpu").manual_seed(w.seed + 1)
    z = torch.randn((w.B, w.N, w.N, w.c_in), generator=g).to(torch.bfloat16).cuda()
    wb = (torch.randn((w.c_in, H), generator=g) / w.c_in ** 0.5).to(torch.bfloat16).cuda()
    ln_w = (1 + 0.1 * torch.randn(w.c_in, generator=g)).cuda()
    ln_b = (0.1 * torch.randn(w.c_in, generator=g)).cuda()
    bias = torch.randn(H, generator=g).cuda()
    pb = A.ln_pair_bias(z, ln_w, ln_b, EPS, wb, bias)
    y = oracle.ln_linear(f64(z), f64(ln_w), f64(ln_b), EPS, f64(wb), f64(bias))     # [B, N, N, H]
    check(pb, np.transpose(y, (0, 3, 1, 2))[:, None], "pair_bias")


def test_projected_qkvg_feed_the_attention_as_strided_views():
    # q, k, v, g straight out of the projection (row stride 4*H*C), pair bias from
    # the pair projection: the attention reads them through strides, no copy
    w = PROJ_WORKLOADS["tiny_proj"]
    B, S, N, H, C = w.B, 4, 64, 2, 32
    pw = ProjWorkload("feed", B, S, N, 64, H, C, 7200)
    d = make_proj_inputs(pw, device="cuda")
    y = A.ln_linear(d["x"], d["ln_w"], d["ln_b"], EPS, d["w"], d["bias"])
    q, k, v, g = A.qkvg_views(y, H)
    assert q.stride() == (S * N * 4 * H * C, N * 4 * H * C, 4 * H * C, C, 1)
    gen = torch.Generator("cpu").manual_seed(7201)
    z = torch.randn((B, N, N, 64), generator=gen).to(torch.bfloat16).cuda()
    wb = (torch.randn((64, H), generator=gen) / 8).to(torch.bfloat16).cuda()
    pb = A.ln_pair_bias(z, None, None, EPS, wb)
    out, lse = A.evo_attn_fwd(q, k, v, g, None, pb)
    ref_out, ref_lse = oracle.forward(f64(q), f64(k), f64(v), f64(g), None, f64(pb))
    check(out, ref_out, "out")
    m = metrics(f64(lse), ref_lse)
    assert m["max_abs"] <= TOL["bf16"]["max_abs"], m


def test_unsupported_projection_shapes_raise():
    x = torch.zeros((4, 96), dtype=torch.bfloat16, device="cuda")
    wt = torch.zeros((96, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(A.EvoError) as e:
        A.ln_linear(x, None, None, EPS, wt)
    assert e.value.code == 2                               # c_in not a multiple of 64


@pytest.mark.parametrize("c_z,H,N,B", [(8, 1, 24, 2), (40, 2, 17, 1), (136, 3, 33, 1), (264, 6, 20, 1),
                                       (520, 13, 12, 1), (1024, 16, 9, 2)])
def test_pair_bias_projection_shapes(c_z, H, N, B):
    # every lane layout (2..32 lanes per row, 1..4 chunks per lane) and head-group count
    g = torch.Generator("cpu").manual_seed(c_z * 31 + H)
    z = torch.randn((B, N, N, c_z), generator=g).to(torch.bfloat16).cuda()
    wb = (torch.randn((c_z, H), generator=g) / c_z ** 0.5).to(torch.bfloat16).cuda()
    ln_w = (1 + 0.1 * torch.randn(c_z, generator=g)).cuda()
    ln_b = (0.1 * torch.randn(c_z, generator=g)).cuda()
    bias = torch.randn(H, generator=g).cuda()
    pb = A.ln_pair_bias(z, ln_w, ln_b, EPS, wb, bias)
    y = oracle.ln_linear(f64(z), f64(ln_w), f64(ln_b), EPS, f64(wb), f64(bias))
    check(pb, np.transpose(y, (0, 3, 1, 2))[:, None], ("pair_bias", c_z, H))
