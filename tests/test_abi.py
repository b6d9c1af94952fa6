"""The C-ABI library builds, loads and exports every symbol include/evo_attn.h
declares; host-side argument checks answer without touching a GPU."""
import ctypes
import os
import re

import pytest

from evoformer_pair_bias_b200 import attention as A
from evoformer_pair_bias_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "evo_attn.h")


def header_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(evo_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return A.load_library()


def test_header_declares_the_binding_exports():
    assert header_functions() == sorted(A.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in header_functions():
        assert hasattr(lib, name), name
    out = os.popen(f"nm -D --defined-only {A.LIB_PATH}").read()
    for name in header_functions():
        assert re.search(rf"\bT {name}\b", out), name


def test_status_strings_and_version(lib):
    for code, name in A.STATUS.items():
        assert lib.evo_status_string(code).decode() == name
    assert lib.evo_attn_version() >= 10000


def test_workspace_query_is_pure_and_linear(lib):
    def ws(Bb, S, N, H, C, dt):
        return lib.evo_attn_bwd_workspace_bytes(ctypes.byref(A.Shape(Bb, S, N, H, C)), dt)
    assert ws(1, 128, 256, 8, 32, 0) == ws(1, 128, 256, 8, 32, 0)
    assert ws(1, 4, 32, 4, 8, 1) > 0
    assert lib.evo_attn_bwd_workspace_bytes(None, 0) == 0
    assert ws(1, 4, 32, 4, 0, 0) == 0            # C = 0 is invalid
    # no cubic term: for S = N rows the workspace grows like N^2 * (per-row + pair) terms
    big, small = ws(1, 1536, 1536, 4, 32, 0), ws(1, 768, 768, 4, 32, 0)
    assert big < 4.5 * small


def test_host_argument_errors_need_no_gpu(lib):
    st = A.Strides(0, 0, 0, 0)
    sh = A.Shape(1, 2, 8, 1, 32)
    nul = None
    rc = lib.evo_attn_fwd(None, 0, nul, nul, nul, nul, ctypes.byref(st), nul, nul, nul, nul, ctypes.byref(st), nul,
                          nul)
    assert rc == 1
    rc = lib.evo_attn_fwd(ctypes.byref(sh), 7, nul, nul, nul, nul, ctypes.byref(st), nul, nul, nul, nul,
                          ctypes.byref(st), nul, nul)
    assert rc == 1                                # unknown dtype
    rc = lib.evo_attn_fwd(ctypes.byref(sh), 0, nul, nul, nul, nul, ctypes.byref(st), nul, nul, nul, nul,
                          ctypes.byref(st), nul, nul)
    assert rc == 1                                # null tensors
    empty = A.Shape(1, 0, 8, 1, 32)
    rc = lib.evo_attn_fwd(ctypes.byref(empty), 0, nul, nul, nul, nul, ctypes.byref(st), nul, nul, nul, nul,
                          ctypes.byref(st), nul, nul)
    assert rc == 0                                # empty call: nothing to do
    neg = A.Shape(1, -1, 8, 1, 32)
    rc = lib.evo_attn_fwd(ctypes.byref(neg), 0, nul, nul, nul, nul, ctypes.byref(st), nul, nul, nul, nul,
                          ctypes.byref(st), nul, nul)
    assert rc == 1


def test_timing_hooks_answer_without_a_gpu(lib):
    m = re.search(r"#define EVO_TIMING_PHASES (\d+)", open(HEADER).read())
    assert m and int(m.group(1)) == len(A.PHASES)
    assert lib.evo_attn_timing_collect(None) == 1
    A.timing_enable(True)
    A.timing_enable(False)
    assert A.timing_collect() == {p: (0, 0.0) for p in A.PHASES}   # nothing recorded, nothing waited on


def test_projection_host_checks_need_no_gpu(lib):
    nul, fake = None, ctypes.c_void_p(1 << 20)            # never dereferenced: the checks fail first
    assert lib.evo_ln_linear(0, 256, 1024, nul, nul, nul, 1e-5, nul, nul, nul, 1024, nul) == 0   # empty
    assert lib.evo_ln_linear(-1, 256, 1024, nul, nul, nul, 1e-5, nul, nul, nul, 1024, nul) == 1
    assert lib.evo_ln_linear(8, 256, 1024, nul, nul, nul, 1e-5, nul, nul, nul, 1024, nul) == 1   # null x
    assert lib.evo_ln_linear(8, 256, 1024, fake, nul, nul, 1e-5, fake, nul, fake, 512, nul) == 1  # ldy < n_out
    assert lib.evo_ln_linear(8, 48, 1024, fake, nul, nul, 1e-5, fake, nul, fake, 1024, nul) == 2  # c_in % 64
    assert lib.evo_ln_linear(8, 320, 1024, fake, nul, nul, 1e-5, fake, nul, fake, 1024, nul) == 2  # c_in > 256
    assert lib.evo_ln_linear(8, 256, 192, fake, nul, nul, 1e-5, fake, nul, fake, 192, nul) == 2   # n_out % 128
    odd = ctypes.c_void_p((1 << 20) + 4)                  # 4-byte but not 16-byte aligned
    assert lib.evo_ln_linear(8, 256, 1024, fake, nul, nul, 1e-5, fake, odd, fake, 1024, nul) == 2  # bias
    assert lib.evo_tri_mul(1, 2, 12, fake, fake, 0, fake, nul) == 2                                # N % 8
    assert lib.evo_tri_mul(1, 2, 16, fake, odd, 0, fake, nul) == 2                                 # alignment
    assert lib.evo_tri_mul(1, 0, 16, nul, nul, 0, nul, nul) == 0                                   # empty
    assert lib.evo_tri_mul(-1, 2, 16, fake, fake, 0, fake, nul) == 1
    assert lib.evo_outer_product_mean(0, 4, 8, 8, 8, nul, nul, nul, nul) == 0           # B = 0: no-op
    assert lib.evo_outer_product_mean(1, 0, 8, 8, 8, fake, fake, fake, nul) == 1        # S = 0: no mean
    assert lib.evo_outer_product_mean(1, 4, 3, 5, 5, fake, fake, fake, nul) == 2        # N*C % 8
    assert lib.evo_outer_product_mean(1, 4, 8, 8, 8, fake, odd, fake, nul) == 2        # alignment
    assert lib.evo_outer_product_mean(1, 4, 8, 0, 8, fake, fake, fake, nul) == 1        # no channels
    assert lib.evo_ln_pair_bias(1, 16, 128, 17, fake, nul, nul, 1e-5, fake, nul, fake, nul) == 2  # H > 16
    assert lib.evo_ln_pair_bias(1, 16, 12, 4, fake, nul, nul, 1e-5, fake, nul, fake, nul) == 2    # c_z % 8
    assert lib.evo_ln_pair_bias(1, 0, 128, 4, nul, nul, nul, 1e-5, nul, nul, nul, nul) == 0       # empty


def test_sum_partials_host_checks_need_no_gpu(lib):
    fake, odd, nul = 1 << 20, (1 << 20) + 2, None          # never dereferenced: the checks fail first
    arr = lambda *ps: (ctypes.c_void_p * len(ps))(*ps)    # noqa: E731
    out = ctypes.c_void_p(fake)
    assert lib.evo_sum_partials(2, arr(fake, fake), 0, out, nul) == 0              # n = 0: no-op
    assert lib.evo_sum_partials(0, arr(fake), 8, out, nul) == 1                    # no partials
    assert lib.evo_sum_partials(2, None, 8, out, nul) == 1                         # null array
    assert lib.evo_sum_partials(2, arr(fake, 0), 8, out, nul) == 1                 # null partial
    assert lib.evo_sum_partials(1, arr(fake), -1, out, nul) == 1                   # negative size
    assert lib.evo_sum_partials(1, arr(fake), 8, None, nul) == 1                   # null out
    assert lib.evo_sum_partials(2, arr(fake, odd), 8, out, nul) == 2               # not 4-byte aligned
    assert lib.evo_sum_partials(1, arr(fake), 8, ctypes.c_void_p(odd), nul) == 2
    assert lib.evo_sum_partials(A.MAX_PARTIALS + 1, arr(*[fake] * (A.MAX_PARTIALS + 1)), 8, out, nul) == 2
    assert lib.evo_sum_partials(A.MAX_PARTIALS, arr(*[fake] * A.MAX_PARTIALS), 0, out, nul) == 0
    assert "EVO_MAX_PARTIALS %d" % A.MAX_PARTIALS in open(HEADER).read().replace("  ", " ")


def test_product_path_never_touches_the_oracle():
    """The package must not import, load or mention the CPU oracle."""
    pkg = os.path.join(ROOT, "evoformer_pair_bias_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "evo_ref" not in text and "libevo_ref" not in text, f


def test_binding_refuses_strided_or_mistyped_biases_before_any_call(lib):
    """A strided mask slice (rows s0:s1 of a B = 2 mask), an fp32 pair bias with bf16 q and a
    non-contiguous lse are refused by the binding in the forward and in both backward entry
    points, before the library sees a pointer it would read as a dense array of the wrong values."""
    import torch
    B, S, N, H, C = 2, 6, 16, 2, 32
    q = torch.zeros(B, S, N, H, C, dtype=torch.bfloat16)
    full_mask = torch.zeros(B, 2 * S, 1, 1, N, dtype=torch.bfloat16)
    strided_mask = full_mask[:, 2:2 + S]               # rows of a larger mask: a strided view when B > 1
    assert not strided_mask.is_contiguous()
    pb = torch.zeros(B, 1, H, N, N, dtype=torch.bfloat16)
    lse = torch.zeros(B, S, H, N, dtype=torch.float32)
    calls = (A.evo_attn_bwd, A.evo_attn_bwd_noalloc)
    for bwd in calls:
        with pytest.raises(ValueError, match="mask_bias must be contiguous"):
            bwd(q, q, q, q, strided_mask, pb, q, lse, q)
        with pytest.raises(ValueError, match="pair_bias must be of q's dtype"):
            bwd(q, q, q, q, None, pb.float(), q, lse, q)
        with pytest.raises(ValueError, match="pair_bias must have shape"):
            bwd(q, q, q, q, None, pb[:, :, :1], q, lse, q)
        with pytest.raises(ValueError, match="lse must be"):
            bwd(q, q, q, q, None, pb, q, lse.transpose(2, 3).contiguous().transpose(2, 3), q)
    with pytest.raises(ValueError, match="mask_bias must be contiguous"):
        A.evo_attn_fwd(q, q, q, q, strided_mask, pb)
    with pytest.raises(ValueError, match="lse must be"):
        A.evo_attn_fwd(q, q, q, q, None, pb, lse=lse[:, :1])
