"""evo_attn_bwd_noalloc: the backward pass for callers that cannot allocate.

Some callers cannot call cudaMalloc at all (a plug-in inside a framework that
owns every byte of device memory, a service whose footprint is fixed at start)
and have no buffer to lend as workspace.  evo_attn_bwd_noalloc runs the same
backward kernels on the library's own fixed scratch area instead.  This test
calls it through the C-ABI twice in a row and checks each result against the
regular evo_attn_bwd (caller-provided workspace), within the bf16 tolerances
the parity tests use.  It lives in its own file, collected last, and passes
both alone in a fresh process and after the other GPU tests.
"""
import pytest
import torch

from _parity import TOL, metrics
from evoformer_pair_bias_b200 import attention as A
from evoformer_pair_bias_b200.workloads import Workload, make_inputs

pytestmark = pytest.mark.gpu


def test_noalloc_backward_matches_the_workspace_backward_twice():
    from evoformer_pair_bias_b200 import build
    build.build()
    A.load_library()
    w = Workload("noalloc", 1, 32, 256, 4, 32, "bf16", "msa_row", 1.0, "frac:0.1", 31337)
    d = {k: (None if v is None else v.cuda()) for k, v in make_inputs(w).items()}
    assert A.workspace_bytes(d["q"]) <= A.NOALLOC_WORKSPACE_BYTES
    out, lse = A.evo_attn_fwd(d["q"], d["k"], d["v"], d["g"], d["mask_bias"], d["pair_bias"])
    ref = A.evo_attn_bwd(d["q"], d["k"], d["v"], d["g"], d["mask_bias"], d["pair_bias"], out, lse, d["dout"])
    torch.cuda.synchronize()
    tol = TOL["bf16"]
    for call in range(2):
        got = A.evo_attn_bwd_noalloc(d["q"], d["k"], d["v"], d["g"], d["mask_bias"], d["pair_bias"],
                                     out, lse, d["dout"])
        torch.cuda.synchronize()
        for name in ("dq", "dk", "dv", "dg", "d_pair_bias"):
            m = metrics(got[name].double().cpu().numpy(), ref[name].double().cpu().numpy())
            assert m["finite"], (call, name)
            assert m["rel_l2"] <= tol["rel_l2"] and m["max_abs"] <= tol["max_abs"], (call, name, m)
        # everything but dq (fp32 atomics across key tiles) is bitwise reproducible
        for name in ("dk", "dv", "dg", "d_pair_bias"):
            assert torch.equal(got[name], ref[name]), (call, name)
    assert A.device_status(clear=True) == 0


def test_noalloc_backward_rejects_shapes_beyond_its_scratch():
    A.load_library()
    w = Workload("noalloc_big", 1, 128, 256, 8, 32, "bf16", "msa_row", 1.0, "none", 7)
    d = {k: (None if v is None else v.cuda()) for k, v in make_inputs(w).items()}
    assert A.workspace_bytes(d["q"]) > A.NOALLOC_WORKSPACE_BYTES
    out, lse = A.evo_attn_fwd(d["q"], d["k"], d["v"], d["g"], None, d["pair_bias"])
    with pytest.raises(A.EvoError) as e:
        A.evo_attn_bwd_noalloc(d["q"], d["k"], d["v"], d["g"], None, d["pair_bias"], out, lse, d["dout"])
    assert e.value.code == 3                        # EVO_ERR_WORKSPACE_TOO_SMALL, nothing enqueued
    assert A.device_status(clear=True) == 0
