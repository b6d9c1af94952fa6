"""GPU parity of the row-split backward's exchange step against the oracle.

evo_sum_partials adds fp32 partials left to right; it must equal the
oracle's rank-ordered fp32 sum bit for bit, on the 16-byte path, the scalar
path (pointers 4-byte aligned only) and in place.  The row split itself runs
here on one GPU as one rank after another (independent launches, nothing
waits on another rank): each block of rows from row_range goes through
evo_attn_fwd / evo_attn_bwd, and the blocks' d_pair_bias partials are added
by evo_sum_partials.  Every per-row output must match the oracle's rows, and
the summed d_pair_bias the oracle's full gradient, with the attention's own
tolerances: the row split only regroups the sum over s (the pair bias is one
term broadcast over the rows, MegaFold summary, section "EvoFlash-3D"; the
rows split over a sequence-parallel group, same page, section "EvoSP-3D").
"""
import zlib

import numpy as np
import pytest
import torch

import oracle
from _parity import assert_close, f64, gpu_fwd_bwd, oracle_fwd_bwd, to_gpu, workload_inputs
from evoformer_pair_bias_b200 import attention as A
from evoformer_pair_bias_b200 import row_shards
from evoformer_pair_bias_b200.workloads import Workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from evoformer_pair_bias_b200 import build
    build.build()
    A.load_library()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    yield
    assert A.device_status(clear=True) == 0, "a kernel reported a timed-out wait"


def mixed_partials(count, n, off, seed):
    """count partials of n fp32 values with magnitudes 1e-2 .. 1e3 (so the order of the
    additions shows in the last bits), each starting `off` elements into its own
    16-byte aligned slot: off = 0 takes the 16-byte loads (and a scalar tail when
    n % 4 != 0), any other off the scalar path."""
    g = torch.Generator("cpu").manual_seed(seed)
    slot = (n + 8 + 3) // 4 * 4
    host = torch.randn(count * slot, generator=g)
    for r in range(count):
        host[r * slot:(r + 1) * slot] *= 10.0 ** (r % 6 - 2)
    buf = host.cuda()
    return [buf[r * slot + off:r * slot + off + n] for r in range(count)]


@pytest.mark.parametrize("count,n,off", [(1, 1000, 0), (2, 4099, 0), (3, 12345, 1), (8, 3 * 65536 + 3, 0),
                                         (5, 70001, 2), (64, 777, 0), (64, 513, 3)])
def test_sum_partials_is_the_rank_ordered_fp32_sum(count, n, off):
    parts = mixed_partials(count, n, off, count * 1000 + n)
    got = A.sum_partials(parts)
    torch.cuda.synchronize()
    want = oracle.ordered_sum_f32(np.stack([p.cpu().numpy() for p in parts]))
    assert np.array_equal(got.cpu().numpy(), want)


def test_sum_partials_in_place_and_from_a_gathered_buffer():
    parts = mixed_partials(4, 8192, 0, 11)
    want = oracle.ordered_sum_f32(np.stack([p.cpu().numpy() for p in parts]))
    gathered = torch.stack(parts)                          # [world, n], as an all-gather returns it
    assert np.array_equal(A.sum_partials(gathered).cpu().numpy(), want)
    A.sum_partials(parts, out=parts[0])                    # into the first partial
    torch.cuda.synchronize()
    assert np.array_equal(parts[0].cpu().numpy(), want)
    empty = torch.empty(0, device="cuda")
    assert A.sum_partials([empty, empty]).numel() == 0


SPLITS = [
    # name, B, S, N, H, C, dtype, layout, mask, ranks
    ("msa_200_3", 1, 7, 200, 2, 32, "bf16", "msa_row", "frac:0.1", 3),
    ("b2_64_2", 2, 5, 64, 3, 32, "bf16", "msa_row", "tail:5", 2),
    ("tri_end_136_4", 1, 136, 136, 2, 32, "bf16", "tri_end", "frac:0.05", 4),
    ("empty_block", 1, 2, 64, 1, 32, "bf16", "msa_row", "none", 3),
    ("f32_45_2", 1, 4, 45, 3, 16, "f32", "msa_row", "frac:0.1", 2),
]


@pytest.mark.parametrize("spec", SPLITS, ids=[s[0] for s in SPLITS])
def test_row_split_backward_matches_the_oracle(spec):
    name, B, S, N, H, C, dt, layout, mask, world = spec
    w = Workload(name, B, S, N, H, C, dt, layout, 1.0, mask, seed=zlib.crc32(name.encode()) % 100000 + 3)
    inp = workload_inputs(w)
    ref = oracle_fwd_bwd(inp)
    d = to_gpu(inp)
    parts = []
    for rank in range(world):
        s0, s1 = row_shards.row_range(S, world, rank)
        blk = {k: (v if v is None or k == "pair_bias" else v[:, s0:s1]) for k, v in d.items()}
        if blk["mask_bias"] is not None:
            blk["mask_bias"] = blk["mask_bias"].contiguous()
        got = gpu_fwd_bwd(blk)
        if s1 > s0:
            for n in ("out", "lse", "dq", "dk", "dv", "dg"):
                assert_close(f"{name}/rank{rank}", n, f64(got[n]), ref[n][:, s0:s1], dt)
        else:
            assert torch.count_nonzero(got["d_pair_bias"]) == 0          # no rows: the empty sum
        parts.append(got["d_pair_bias"])
    total = A.sum_partials(parts)
    torch.cuda.synchronize()
    assert_close(name, "d_pair_bias", f64(total), ref["d_pair_bias"], dt)
    host = np.stack([p.cpu().numpy() for p in parts])
    assert np.array_equal(total.cpu().numpy(), oracle.ordered_sum_f32(host))   # the exchange adds exactly so
    assert torch.equal(A.sum_partials(parts), total)                             # and the same bits every time


def test_one_rank_needs_no_exchange():
    w = Workload("one_rank", 1, 3, 64, 2, 32, "bf16", "msa_row", 1.0, "none", 5)
    d = to_gpu(workload_inputs(w))
    out, lse = row_shards.attn_fwd(d["q"], d["k"], d["v"], d["g"], None, d["pair_bias"])
    n0 = A.launch_count()
    grads = row_shards.attn_bwd(d["q"], d["k"], d["v"], d["g"], None, d["pair_bias"], out, lse, d["dout"])
    n1 = A.launch_count()
    plain = A.evo_attn_bwd(d["q"], d["k"], d["v"], d["g"], None, d["pair_bias"], out, lse, d["dout"])
    n2 = A.launch_count()
    torch.cuda.synchronize()
    assert torch.equal(grads["d_pair_bias"], plain["d_pair_bias"])
    assert n1 - n0 == n2 - n1                              # no collective and no sum: the plain backward
    grads2, pending = row_shards.attn_bwd(d["q"], d["k"], d["v"], d["g"], None, d["pair_bias"], out, lse,
                                          d["dout"], async_op=True)
    assert pending.wait() is grads2["d_pair_bias"]
    torch.cuda.synchronize()
    assert torch.equal(grads2["d_pair_bias"], plain["d_pair_bias"])


class _DoneWork:
    """Stands in for a finished all-gather handle: wait() has nothing left to wait for."""

    def __init__(self):
        self.waited = 0

    def wait(self):
        self.waited += 1


def test_pending_wait_sums_gathered_parts_in_place():
    """PendingPairBiasGrad.wait() with a work handle: the branch a world > 1 backward takes.

    The gathered buffer holds the per-block partials of a row split (run block
    after block on this GPU); wait() must add them in rank order into the
    tensor that held this rank's partial and return that very tensor, bit-equal
    to the oracle's rank-ordered fp32 sum.
    """
    w = Workload("pending", 1, 7, 136, 2, 32, "bf16", "msa_row", 1.0, "frac:0.1", 17)
    d = to_gpu(workload_inputs(w))
    world = 3
    parts = []
    for rank in range(world):
        s0, s1 = row_shards.row_range(w.S, world, rank)
        blk = {k: (v if v is None or k == "pair_bias" else v[:, s0:s1].contiguous()) for k, v in d.items()}
        parts.append(gpu_fwd_bwd(blk)["d_pair_bias"])
    gathered = torch.stack(parts)                      # what the all-gather leaves in its buffer
    mine = parts[1].clone()                            # this rank's partial, to be overwritten by the sum
    work = _DoneWork()
    pending = row_shards.PendingPairBiasGrad(gathered, work, mine)
    got = pending.wait()
    torch.cuda.synchronize()
    assert got is mine and work.waited == 1
    assert np.array_equal(got.cpu().numpy(), oracle.ordered_sum_f32(gathered.cpu().numpy()))
    assert pending.wait() is mine and work.waited == 1  # a second wait() does nothing more


def test_pair_shards_on_one_gpu_match_the_oracle():
    """The pair-sharded triangle attentions (pair_shards) with a single rank, on the GPU kernels:
    around the starting node in place, around the ending node through the transposed view of the
    (here whole) column block, forward and backward; each output against the oracle run on the
    pair (ending node: on the explicitly transposed pair)."""
    from evoformer_pair_bias_b200 import pair_shards
    N = 136
    w = Workload("pair_gpu", 1, N, N, 2, 32, "bf16", "tri_start", 1.0, "frac:0.1", 4711)
    inp = workload_inputs(w)
    d = to_gpu(inp)
    x = {k: f64(v) for k, v in inp.items()}
    T = lambda a: np.ascontiguousarray(np.swapaxes(a, 1, 2))            # noqa: E731
    # starting node: rows s = i, keys j
    out_s, lse_s = pair_shards.tri_start_fwd(d["q"], d["k"], d["v"], d["g"], d["mask_bias"], d["pair_bias"])
    g_s = pair_shards.tri_start_bwd(d["q"], d["k"], d["v"], d["g"], d["mask_bias"], d["pair_bias"], out_s, lse_s,
                                    d["dout"])
    torch.cuda.synchronize()
    ref_out, _ = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["mask_bias"], x["pair_bias"])
    ref = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["mask_bias"], x["pair_bias"], x["dout"])
    assert_close("pair_gpu/start", "out", f64(out_s), ref_out, "bf16")
    for n in ("dq", "dk", "dv", "dg", "d_pair_bias"):
        assert_close("pair_gpu/start", n, f64(g_s[n]), ref[n], "bf16")
    # ending node: rows s = j, keys i, on the row-sharded (here whole) pair
    out_e, lse_e, saved = pair_shards.tri_end_fwd(d["q"], d["k"], d["v"], d["g"], d["mask_bias"], d["pair_bias"], N)
    g_e = pair_shards.tri_end_bwd(saved, d["mask_bias"], d["pair_bias"], lse_e, d["dout"], N)
    torch.cuda.synchronize()
    xt = {n: T(x[n]) for n in ("q", "k", "v", "g", "dout")}
    ref_out_e, _ = oracle.forward(xt["q"], xt["k"], xt["v"], xt["g"], x["mask_bias"], x["pair_bias"])
    ref_e = oracle.backward(xt["q"], xt["k"], xt["v"], xt["g"], x["mask_bias"], x["pair_bias"], xt["dout"])
    assert_close("pair_gpu/end", "out", f64(out_e), T(ref_out_e), "bf16")
    for n in ("dq", "dk", "dv", "dg"):
        assert_close("pair_gpu/end", n, f64(g_e[n]), T(ref_e[n]), "bf16")
    assert_close("pair_gpu/end", "d_pair_bias", f64(g_e["d_pair_bias"]), ref_e["d_pair_bias"], "bf16")
