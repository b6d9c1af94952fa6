"""The kernels' FMA-pipe exponential on the GPU, through evo_exp2_fma.

The same device function the attention kernels use for part of their
exponentials, evaluated on a sweep of [-125, 126] (and the clamp below it),
against fp64 2^x at its stated relative error bound, 8e-5, and bit for bit
against the CPU emulation of its fp32 steps (tests/test_exp2_poly.py).
"""
import numpy as np
import pytest
import torch

from evoformer_pair_bias_b200 import attention as A
from test_exp2_poly import BOUND, exp2_fma_emulated, sweep

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from evoformer_pair_bias_b200 import build
    build.build()
    A.load_library()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    yield


def test_device_exp2_within_bound_and_equal_to_its_emulation():
    x = sweep()
    xs = np.concatenate([x, np.array([-126.0, -300.0, -np.inf], np.float32)])
    for n in (xs.size, xs.size - 1):                  # even and odd counts (the last value alone)
        got = A.exp2_fma(torch.from_numpy(xs[:n]).cuda()).cpu().numpy()
        want = np.exp2(np.maximum(xs[:n], -125.0).astype(np.float64))
        rel = np.abs(got.astype(np.float64) - want) / want
        assert rel.max() < BOUND, (rel.max(), xs[rel.argmax()])
        emu = exp2_fma_emulated(xs[:n])
        assert np.array_equal(got.view(np.uint32), emu.view(np.uint32))


def test_empty_and_invalid_calls():
    lib = A.load_library()
    assert lib.evo_exp2_fma(None, None, 0, None) == 0
    assert lib.evo_exp2_fma(None, None, -1, None) == 1
    assert lib.evo_exp2_fma(None, None, 4, None) == 1
