"""A bounded in-kernel wait that runs out is reported, and the context survives.

Nothing is broken on purpose: only the limit of the forward kernel's waits
changes (evo_attn_set_wait_limit_ns).  With a limit of 0 every wait that is
not satisfied at once gives up; the kernel drains its own copies and MMAs
(those drains keep the 2 s default) and returns, and evo_attn_device_status
reports EVO_ERR_DEVICE_TIMEOUT.  With the default limit restored the next
call is correct again, on the same context.
"""
import pytest
import torch

from _parity import compare_all, gpu_fwd_bwd, oracle_fwd_bwd, to_gpu, workload_inputs
from evoformer_pair_bias_b200 import attention as A
from evoformer_pair_bias_b200.workloads import Workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from evoformer_pair_bias_b200 import build
    build.build()
    A.load_library()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    assert A.device_status(clear=True) == 0
    yield
    A.set_wait_limit_ns(A.DEFAULT_WAIT_LIMIT_NS)
    A.device_status(clear=True)


def test_zero_wait_limit_times_out_and_the_context_stays_usable():
    w = Workload("timeout", 1, 4, 384, 2, 32, "bf16", "msa_row", 1.0, "frac:0.1", 31)
    inp = workload_inputs(w)
    d = to_gpu(inp)
    prev = A.set_wait_limit_ns(0)
    try:
        assert prev == A.DEFAULT_WAIT_LIMIT_NS
        A.evo_attn_fwd(d["q"], d["k"], d["v"], d["g"], d["mask_bias"], d["pair_bias"])
        assert A.device_status(clear=True) == 5           # EVO_ERR_DEVICE_TIMEOUT
    finally:
        assert A.set_wait_limit_ns(prev) == 0
    assert A.device_status(clear=True) == 0              # cleared, and nothing new
    gpu = gpu_fwd_bwd(d)
    assert A.device_status(clear=True) == 0
    compare_all(w.name, gpu, oracle_fwd_bwd(inp), "bf16")
