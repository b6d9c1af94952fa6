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
