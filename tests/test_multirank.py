"""The multi-process path of bench.py on CPU: world_size 2 over gloo.

Rows s are independent problems, so N GPUs run N replicas with no collective
on the data path; the only cross-rank step is the max over ranks of the
device timings, and the job's value counts the work of every rank.  These
tests run that step over a real 2-rank gloo process group, and the reference
arm under torchrun, where rank 0 alone prints the line.  They also run the
exchange of a backward whose rows are split over ranks (row_shards): the
partial d_pair_bias of each rank's rows all-gathered in rank order.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        got = bench.max_over_ranks([rank + 1.0, 10.0 - rank, 3.0], world, "cpu")
        value = bench.job_throughput(1e12, 10, world, got[0])
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"max": got, "value": value}, f)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value_with_two_gloo_ranks(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    for rank in range(world):
        r = json.load(open(tmp_path / f"rank{rank}.json"))
        assert r["max"] == [2.0, 10.0, 3.0]                  # every rank sees the slowest rank's times
        assert r["value"] == pytest.approx(1e12 * 10 * world / 2e-3 / 1e12)   # all ranks' work / max time


def _shard_main(rank, world, port, out_dir, S):
    """One rank of a row-split backward: the oracle's partial over this rank's rows
    stands in for evo_attn_bwd's, and the exchange runs through row_shards over gloo."""
    import datetime

    import numpy as np
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle
    from evoformer_pair_bias_b200 import row_shards
    from evoformer_pair_bias_b200.workloads import Workload, make_inputs
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = Workload("split", 1, S, 16, 2, 8, "f32", "msa_row", 1.0, "frac:0.2", 77)
        x = {k: (None if v is None else v.double().numpy()) for k, v in make_inputs(w, device="cpu").items()}
        s0, s1 = row_shards.row_range(S, world, rank)
        if s1 > s0:
            sl = {k: (v if v is None or k == "pair_bias" else v[:, s0:s1]) for k, v in x.items()}
            part = oracle.backward(sl["q"], sl["k"], sl["v"], sl["g"], sl["mask_bias"], sl["pair_bias"],
                                   sl["dout"], want=("d_pair_bias",))["d_pair_bias"]
        else:
            part = np.zeros((1, 1, 2, 16, 16))
        part = torch.from_numpy(part.astype(np.float32))
        gathered = row_shards.gather_partials(part)
        started, work = row_shards.start_gather(part)       # the asynchronous form, same collective
        work.wait()
        assert torch.equal(started, gathered)
        np.save(os.path.join(out_dir, f"part{rank}.npy"), part.numpy())
        np.save(os.path.join(out_dir, f"gathered{rank}.npy"), gathered.numpy())
        np.save(os.path.join(out_dir, f"sum{rank}.npy"), oracle.ordered_sum_f32(gathered.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("S", [7, 1])
def test_row_split_exchange_gathers_in_rank_order_with_two_gloo_ranks(tmp_path, S):
    import numpy as np

    import oracle
    from evoformer_pair_bias_b200.workloads import Workload, make_inputs
    world = 2
    mp.start_processes(_shard_main, args=(world, _free_port(), str(tmp_path), S), nprocs=world, join=True,
                       start_method="spawn")
    parts = [np.load(tmp_path / f"part{r}.npy") for r in range(world)]
    sums = [np.load(tmp_path / f"sum{r}.npy") for r in range(world)]
    for r in range(world):
        g = np.load(tmp_path / f"gathered{r}.npy")
        assert g.shape == (world,) + parts[0].shape
        assert all(np.array_equal(g[i], parts[i]) for i in range(world))    # rank i's partial at index i
    assert np.array_equal(sums[0], sums[1])                                 # every rank holds the same bits
    w = Workload("split", 1, S, 16, 2, 8, "f32", "msa_row", 1.0, "frac:0.2", 77)
    x = {k: (None if v is None else v.double().numpy()) for k, v in make_inputs(w, device="cpu").items()}
    full = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["mask_bias"], x["pair_bias"], x["dout"],
                           want=("d_pair_bias",))["d_pair_bias"]
    assert np.allclose(sums[0], full, rtol=1e-5, atol=1e-6)


def _bench_split_main(rank, world, port, out_dir, S):
    """One rank of bench.py's row-split pass (bench.row_block + bench.split_pass over
    row_shards), with the oracle standing in for the CUDA library on CPU."""
    import datetime

    import numpy as np
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    import oracle
    from evoformer_pair_bias_b200 import row_shards
    from evoformer_pair_bias_b200.workloads import Workload, make_inputs
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    f64 = lambda t: None if t is None else t.double().numpy()         # noqa: E731
    f32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float32))  # noqa: E731

    def cpu_fwd(q, k, v, g, m, pb, out=None, lse=None):
        o, l_ = oracle.forward(f64(q), f64(k), f64(v), f64(g), f64(m), f64(pb))
        return f32(o), f32(l_)

    def cpu_bwd(q, k, v, g, m, pb, out, lse, dout, grads=None, workspace=None):
        if q.shape[1] == 0:
            return {"d_pair_bias": torch.zeros(pb.shape[0], 1, pb.shape[2], pb.shape[3], pb.shape[4])}
        r = oracle.backward(f64(q), f64(k), f64(v), f64(g), f64(m), f64(pb), f64(dout))
        return {n: f32(a) for n, a in r.items()}

    def cpu_sum(parts, out):
        out.copy_(f32(oracle.ordered_sum_f32(parts.numpy())))
        return out

    try:
        w = Workload("split", 1, S, 16, 2, 8, "f32", "msa_row", 1.0, "frac:0.2", 77)
        inp = make_inputs(w, device="cpu")
        s0, s1 = row_shards.row_range(S, world, rank)
        blk = bench.row_block(inp, s0, s1)
        assert all(v is None or v.is_contiguous() for v in blk.values())
        assert blk["pair_bias"] is inp["pair_bias"]                        # the bias is shared, not split
        mine = cpu_bwd(*[blk[n] for n in ("q", "k", "v", "g", "mask_bias", "pair_bias")], None, None,
                       blk["dout"])["d_pair_bias"]
        out, lse, grads = bench.split_pass(blk, None, fwd=cpu_fwd, backward=cpu_bwd, summer=cpu_sum)
        np.save(os.path.join(out_dir, f"bpart{rank}.npy"), mine.numpy())
        np.save(os.path.join(out_dir, f"bsum{rank}.npy"), grads["d_pair_bias"].numpy())
        if s1 > s0:
            np.save(os.path.join(out_dir, f"bout{rank}.npy"), out.numpy())
            np.save(os.path.join(out_dir, f"bdq{rank}.npy"), grads["dq"].numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("S", [7, 1])
def test_bench_row_split_pass_with_two_gloo_ranks(tmp_path, S):
    """bench.py's multi-GPU pass (row blocks, forward, backward, d_pair_bias exchange in rank
    order) on two CPU ranks: both ranks end with the same bits, the rank-ordered fp32 sum of the
    blocks' partials, which matches the unsplit gradient; each rank's rows match the oracle's."""
    import numpy as np

    import oracle
    from evoformer_pair_bias_b200 import row_shards
    from evoformer_pair_bias_b200.workloads import Workload, make_inputs
    world = 2
    mp.start_processes(_bench_split_main, args=(world, _free_port(), str(tmp_path), S), nprocs=world, join=True,
                       start_method="spawn")
    parts = np.stack([np.load(tmp_path / f"bpart{r}.npy") for r in range(world)])
    sums = [np.load(tmp_path / f"bsum{r}.npy") for r in range(world)]
    assert np.array_equal(sums[0], sums[1])
    assert np.array_equal(sums[0], oracle.ordered_sum_f32(parts))
    w = Workload("split", 1, S, 16, 2, 8, "f32", "msa_row", 1.0, "frac:0.2", 77)
    x = {k: (None if v is None else v.double().numpy()) for k, v in make_inputs(w, device="cpu").items()}
    full = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["mask_bias"], x["pair_bias"], x["dout"])
    assert np.allclose(sums[0], full["d_pair_bias"], rtol=1e-5, atol=1e-6)
    fo, _ = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["mask_bias"], x["pair_bias"])
    for r in range(world):
        s0, s1 = row_shards.row_range(S, world, r)
        if s1 > s0:
            assert np.allclose(np.load(tmp_path / f"bout{r}.npy"), fo[:, s0:s1], rtol=1e-5, atol=1e-6)
            assert np.allclose(np.load(tmp_path / f"bdq{r}.npy"), full["dq"][:, s0:s1], rtol=1e-5, atol=1e-6)


def _pair_main(rank, world, port, out_dir, N):
    """One rank of a row-sharded pair representation: triangle attention around the starting
    node in place, around the ending node through the all_to_all rotation, both backwards with
    the rank-ordered d_pair_bias exchange; the oracle stands in for the CUDA library."""
    import datetime

    import numpy as np
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle
    from evoformer_pair_bias_b200 import pair_shards
    from evoformer_pair_bias_b200.workloads import Workload, make_inputs
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    f64 = lambda t: None if t is None else t.double().numpy()               # noqa: E731
    f32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float32))  # noqa: E731

    def cpu_fwd(q, k, v, g, m, pb, out=None, lse=None):
        o, l_ = oracle.forward(f64(q), f64(k), f64(v), f64(g), f64(m), f64(pb))
        return f32(o), f32(l_)

    def cpu_bwd(q, k, v, g, m, pb, out, lse, dout, grads=None, workspace=None):
        r = oracle.backward(f64(q), f64(k), f64(v), f64(g), f64(m), f64(pb), f64(dout))
        return {n: f32(a) for n, a in r.items()}

    def cpu_sum(parts, out):
        out.copy_(f32(oracle.ordered_sum_f32(parts.numpy())))
        return out

    try:
        w = Workload("pair", 1, N, N, 2, 8, "f32", "tri_start", 1.0, "frac:0.2", 91)
        full = make_inputs(w, device="cpu")                     # [B, i, j, H, C] pair layout, rows s = i
        i0, i1 = pair_shards.row_range(N, world, rank)
        rows = {n: full[n][:, i0:i1].contiguous() for n in ("q", "k", "v", "g", "dout")}
        bias = pair_shards.gather_bias_rows(full["pair_bias"][:, :, :, i0:i1], N)
        assert torch.equal(bias, full["pair_bias"])
        mask_rows = full["mask_bias"][:, i0:i1].contiguous()
        # around the starting node: the row shard in place
        o_s, l_s = pair_shards.tri_start_fwd(rows["q"], rows["k"], rows["v"], rows["g"], mask_rows, bias,
                                             fwd=cpu_fwd)
        g_s = pair_shards.tri_start_bwd(rows["q"], rows["k"], rows["v"], rows["g"], mask_rows, bias, o_s, l_s,
                                        rows["dout"], bwd=cpu_bwd, summer=cpu_sum)
        # around the ending node: rows s = j after the rotation; the mask over keys i of rows j
        o_e, l_e, saved = pair_shards.tri_end_fwd(rows["q"], rows["k"], rows["v"], rows["g"], mask_rows, bias, N,
                                                  fwd=cpu_fwd)
        g_e = pair_shards.tri_end_bwd(saved, mask_rows, bias, l_e, rows["dout"], N, bwd=cpu_bwd, summer=cpu_sum)
        for name, t in (("o_s", o_s), ("o_e", o_e), ("dpb_s", g_s["d_pair_bias"]), ("dpb_e", g_e["d_pair_bias"]),
                        ("dq_e", g_e["dq"]), ("dk_e", g_e["dk"]), ("dv_e", g_e["dv"]), ("dg_e", g_e["dg"]),
                        ("dq_s", g_s["dq"])):
            np.save(os.path.join(out_dir, f"{name}{rank}.npy"), t.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("N", [13, 8])
def test_pair_shards_triangle_attentions_with_two_gloo_ranks(tmp_path, N):
    """A pair representation split by rows over two CPU ranks: the starting-node attention runs
    in place, the ending-node one through rows_to_cols / cols_to_rows (all_to_all).  Every rank's
    rows of every output match the oracle on the whole pair; d_pair_bias is the same bits on both
    ranks and matches the oracle's full gradient."""
    import numpy as np

    import oracle
    from evoformer_pair_bias_b200 import pair_shards
    from evoformer_pair_bias_b200.workloads import Workload, make_inputs
    world = 2
    mp.start_processes(_pair_main, args=(world, _free_port(), str(tmp_path), N), nprocs=world, join=True,
                       start_method="spawn")
    w = Workload("pair", 1, N, N, 2, 8, "f32", "tri_start", 1.0, "frac:0.2", 91)
    x = {k: (None if v is None else v.double().numpy()) for k, v in make_inputs(w, device="cpu").items()}
    T = lambda a: np.ascontiguousarray(np.swapaxes(a, 1, 2))            # noqa: E731  pair transpose i <-> j
    ref_s_out, _ = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["mask_bias"], x["pair_bias"])
    ref_s = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["mask_bias"], x["pair_bias"], x["dout"])
    # ending node: the same op on the transposed pair (rows s = j), mask rows indexed by j
    xt = {n: T(x[n]) for n in ("q", "k", "v", "g", "dout")}
    ref_e_out, _ = oracle.forward(xt["q"], xt["k"], xt["v"], xt["g"], x["mask_bias"], x["pair_bias"])
    ref_e = oracle.backward(xt["q"], xt["k"], xt["v"], xt["g"], x["mask_bias"], x["pair_bias"], xt["dout"])
    close = lambda a, b: np.allclose(a, b, rtol=1e-5, atol=1e-6)       # noqa: E731
    for r in range(world):
        i0, i1 = pair_shards.row_range(N, world, r)
        ld = lambda n: np.load(tmp_path / f"{n}{r}.npy")                  # noqa: E731
        assert close(ld("o_s"), ref_s_out[:, i0:i1])
        assert close(ld("dq_s"), ref_s["dq"][:, i0:i1])
        assert close(ld("o_e"), T(ref_e_out)[:, i0:i1])
        for n in ("dq", "dk", "dv", "dg"):
            assert close(ld(f"{n}_e"), T(ref_e[n])[:, i0:i1]), n
        assert close(ld("dpb_s"), ref_s["d_pair_bias"]) and close(ld("dpb_e"), ref_e["d_pair_bias"])
    for n in ("dpb_s", "dpb_e"):
        assert np.array_equal(np.load(tmp_path / f"{n}0.npy"), np.load(tmp_path / f"{n}1.npy"))


def test_rotation_between_row_and_column_shards_is_a_transpose_of_blocks(tmp_path):
    """rows_to_cols then cols_to_rows is the identity, and rows_to_cols gives every rank all rows of
    its own columns (checked against slicing the whole tensor), for uneven blocks (N = 7, 3 ranks)."""
    mp.start_processes(_rotation_main, args=(3, _free_port(), str(tmp_path)), nprocs=3, join=True,
                       start_method="spawn")
    for r in range(3):
        assert (tmp_path / f"rot_ok{r}").exists()


def _rotation_main(rank, world, port, out_dir):
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from evoformer_pair_bias_b200 import pair_shards
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        N = 7
        full = torch.arange(2 * N * N * 3, dtype=torch.float32).view(2, N, N, 3)
        i0, i1 = pair_shards.row_range(N, world, rank)
        cols = pair_shards.rows_to_cols(full[:, i0:i1].contiguous(), N)
        assert torch.equal(cols, full[:, :, i0:i1])
        back = pair_shards.cols_to_rows(cols, N)
        assert torch.equal(back, full[:, i0:i1])
        open(os.path.join(out_dir, f"rot_ok{rank}"), "w").close()
    finally:
        dist.destroy_process_group()


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([1.5, 2.5], 1, "cpu") == [1.5, 2.5]
    assert bench.job_throughput(2e12, 4, 1, 1000.0) == pytest.approx(8.0)   # 8 TFLOP in 1 s


def test_reference_arm_under_torchrun_prints_one_line_from_rank_zero():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "3", "--workload", "tiny_f32"]
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, res.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["steps"] == 1
    assert line["cpu_baseline"]["kind"] == "oracle" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0
