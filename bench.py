"""Benchmark: Evoformer pair-bias attention forward + backward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = R forward and backward passes (every kernel of the path) over one
batch of the workload's synthetic inputs, which are resident in HBM when the
timed region starts; R (``passes_per_step`` in the JSON line, usually 1) is
the smallest count that makes the K timed steps last at least 0.5 s, so that
the clock samples see the GPU under load.  The default workload is the long
triangle attention (N_res = 1536).  The L2 cache (126 MB) is flushed before
every pass by writing a 256 MB buffer outside the per-pass CUDA-event
brackets.  The
metric is achieved TFLOP/s (FlashAttention flop convention: 4*L*C forward,
10*L*C backward, L = B*S*H*N^2 logits) and its fraction of the measured bf16
dense tensor peak.

Multi-GPU (attention workloads): one problem, its rows s split over the N
ranks (strong scaling).  The forward needs no communication; the backward's
one exchange, the all-gather of the fp32 d_pair_bias partials over NCCL and
their rank-ordered sum, is inside the timed region and reported on its own
next to its NVLink floor.  The reported time is the max over ranks and
``value`` counts the whole problem once.  The other workloads (projection,
triangular update, outer product mean) run independent replicas (weak
scaling).

``--impl reference`` times the fp64 CPU oracle (the correctness reference)
on a bounded sample of the same workload, on this host's cores.

``--workload msa_proj_256 | pair_proj_256`` benchmarks the fused pre-attention
projection instead (MegaFold summary, section "EvoFusion"): one step is
y = LayerNorm(x) @ [w_q | w_k | w_v | w_g] + bias over every row of the MSA
(or pair) representation, and for the pair representation also the
pair-bias projection LayerNorm(z) @ w_b + b_b.  Metric: TFLOP/s of the
projection GEMMs (2 * rows * c_in * n_out), with the same timing rules.

``--workload tri_mul_256 | tri_mul_384 | tri_mul_768`` benchmarks the
contraction of the triangular multiplicative update ("Evoformer: the memory
wall ZeRO cannot move", section "The three operations"): one step is the
outgoing-edge update z[b,c,i,j] = sum_k a[b,c,i,k] b[b,c,j,k] over every channel,
then the incoming-edge one; metric TFLOP/s (2 * B * C * N^3 per direction).

``--workload opm_256 | opm_384`` benchmarks the outer product mean (same
section): one step is out[b,i,c1,j,c2] = (1/S) sum_s a[b,s,i,c1] b[b,s,j,c2];
metric TFLOP/s (2 * B * S * (N C)^2).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from evoformer_pair_bias_b200 import attention as A  # noqa: E402
from evoformer_pair_bias_b200.workloads import (WORKLOADS, DEFAULT_BENCH, PROJ_WORKLOADS, logical_view,  # noqa: E402
                                                make_inputs, make_pair_bias_params, make_proj_inputs,
                                                TRI_MUL_WORKLOADS, make_tri_mul_inputs, OPM_WORKLOADS,
                                                make_opm_inputs)

METRIC = "Evoformer pair-bias attention fwd+bwd TFLOP/s and % of B200 bf16 tensor peak"
PROJ_METRIC = "fused LayerNorm + linear pre-attention projection TFLOP/s"
TRI_METRIC = "triangular multiplicative update contraction TFLOP/s"
OPM_METRIC = "outer product mean TFLOP/s"
PROJ_EPS = 1e-5
NOMINAL_BF16_TFLOPS = 2250.0


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(bf16=float(p["bf16_tflops"]), bf16_sustained=float(p["bf16_tflops_sustained"]),
                    hbm=float(p["hbm_gbs"]), source="measured")
    except Exception:
        return dict(bf16=1590.0, bf16_sustained=1400.0, hbm=6650.0, source="fallback")


class ClockSampler:
    """SM clocks, power and clock-event (throttle) reasons sampled during the timed region.

    Polls NVML (the library nvidia-smi reads) every 5 ms from a thread, plus one
    sample on entry and one on exit, so that even a timed region of a few
    milliseconds is covered.  Falls back to ``nvidia-smi -lms 200`` if NVML
    cannot be loaded.
    """

    # NVML clocks-event reason bits
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}
    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str, period_s: float = 0.005):
        self.uuid, self.period = uuid, period_s
        self.samples = []          # (sm_mhz, max_mhz, power_w, reason bits)
        self.smi_lines = []
        self.nvml = None
        self.proc = None
        self.stop = threading.Event()

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        for i in range(pynvml.nvmlDeviceGetCount()):
            h = pynvml.nvmlDeviceGetHandleByIndex(i)
            u = pynvml.nvmlDeviceGetUUID(h)
            u = u.decode() if isinstance(u, bytes) else u
            if not self.uuid or u == self.uuid:
                return pynvml, h
        raise RuntimeError("GPU not found through NVML")

    def _sample(self):
        nv, h = self.nvml
        try:
            rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
        except AttributeError:
            rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(h)
        self.samples.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM),
                             nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM),
                             nv.nvmlDeviceGetPowerUsage(h) / 1000.0, int(rs)))

    def _poll(self):
        while not self.stop.wait(self.period):
            try:
                self._sample()
            except Exception:
                return

    def _read_smi(self):
        for line in self.proc.stdout:
            self.smi_lines.append(line.strip())

    def __enter__(self):
        try:
            self.nvml = self._nvml_handle()
            self._sample()
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
            return self
        except Exception:
            self.nvml = None
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read_smi, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.nvml is not None:
            self.stop.set()
            self.thread.join(timeout=2)
            try:
                self._sample()
            except Exception:
                pass
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if self.nvml is not None and self.samples:
            reasons = set()
            for *_, bits in self.samples:
                reasons.update(n for b, n in self.REASONS.items() if bits & b)
            return {"sm_mhz": statistics.median(x[0] for x in self.samples), "sm_max_mhz": self.samples[-1][1],
                    "power_w_max": max(x[2] for x in self.samples), "reasons": sorted(reasons),
                    "samples": len(self.samples), "source": "NVML, 5 ms"}
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.smi_lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9 or (self.uuid and self.uuid not in parts[0]):
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm), "source": "nvidia-smi, 200 ms"}


def gpu_uuid(dev) -> str:
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return ""


def flops(w):
    return w.fwd_flops, w.bwd_flops


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) per launch of a
# kernel on a workload, from one ncu capture of the command named in the
# profiles/ summary, together with the SHA-256 of the kernel's source file at
# that time.  Reported only while the source is unchanged.
TRAFFIC = {
    # DRAM bytes (read + write) per launch from one ncu pass over the full workload, with the
    # sha256 of the kernel's source when they were taken (a changed source reports null)
    ("bwd_main", "tri_long_1536"): (6792.4e6, "bwd_sm100.cuh",
                                    "1a57e2faf557fd3e48ec3573e4ab4c4cb412c524263084820ac37c4ec8877bad"),
    ("fwd_main", "tri_long_1536"): (7386.8e6, "fwd_sm100.cuh",
                                    "544d01e7d70e54ae914c1911ddec10d569d264f81c909a0aa34a17a5a74827e5"),
    ("bwd_dbias", "tri_long_1536"): (12003.6e6, "dbias_sm100.cuh",
                                     "da55b81462a57b720508e9c6dc5514fa6746503d42e82561eba31d04d4341b06"),
    ("fwd_main", "msa_row_384"): (1179.5e6, "fwd_sm100.cuh",
                                  "544d01e7d70e54ae914c1911ddec10d569d264f81c909a0aa34a17a5a74827e5"),
    ("bwd_main", "msa_row_384"): (1086.2e6, "bwd_sm100.cuh",
                                  "1a57e2faf557fd3e48ec3573e4ab4c4cb412c524263084820ac37c4ec8877bad"),
    ("bwd_dbias", "msa_row_384"): (518.9e6, "dbias_sm100.cuh",
                                   "da55b81462a57b720508e9c6dc5514fa6746503d42e82561eba31d04d4341b06"),
    # one pass after three warm-up steps; output bytes still held in the 126 MB L2 when the
    # captured launch ends are written back later and are not in the count
    ("qkvg", "msa_proj_256"): (24.35e6, "proj_sm100.cuh",
                               "6c2182c8d5b44ebf32b4e064911b57597fedb307f26dceeddf97abe34433cbdf"),
    ("qkvg", "pair_proj_256"): (22.02e6, "proj_sm100.cuh",
                                "6c2182c8d5b44ebf32b4e064911b57597fedb307f26dceeddf97abe34433cbdf"),
    ("pair_bias", "pair_proj_256"): (16.80e6, "proj_sm100.cuh",
                                     "6c2182c8d5b44ebf32b4e064911b57597fedb307f26dceeddf97abe34433cbdf"),
    ("tri_mul", "tri_mul_256"): (33.59e6, "trimul_sm100.cuh",
                                 "be2f55f772d42b87dee464a884fd73b2a16746a963bbc5a26cc0ac4a1ef7507a"),
    ("opm", "opm_256"): (77.79e6, "trimul_sm100.cuh",
                         "be2f55f772d42b87dee464a884fd73b2a16746a963bbc5a26cc0ac4a1ef7507a"),
}


def _source_sha(name: str) -> str:
    import hashlib
    with open(os.path.join(ROOT, "evoformer_pair_bias_b200", "csrc", name), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


def algorithmic(w, phase: str):
    """(FLOPs, bytes) one launch of the main kernel must do: each input read once, each output written once."""
    e = 2 if w.dtype == "bf16" else 4
    rows = w.B * w.S * w.N * w.H                 # (b, s, i, h) rows of C elements
    pair = w.B * w.H * w.N * w.N                 # pair_bias / d_pair_bias elements
    mask = w.B * w.S * w.N if w.mask != "none" else 0
    stats = w.B * w.S * w.H * w.N * 4            # one fp32 per (b, s, h, i)
    ff, bf = flops(w)
    if phase == "fwd_main":                      # q, k, v, g, mask, bias -> out, lse
        return ff, rows * w.C * e * 5 + (mask + pair) * e + stats
    if phase == "bwd_dbias":                     # q, k, v, gated dout, lse, D, mask, bias -> d_pair_bias
        # its own work: S and dP recomputed (two of the five backward products), 4*C per logit
        return 4 * w.logits * w.C, rows * w.C * e * 4 + (mask + pair) * e + 2 * stats + pair * 4
    # q, k, v, gated dout, lse, D, mask, bias -> dq, dk, dv (all five products, 10*C per logit)
    return bf, rows * w.C * e * 7 + (mask + pair) * e + 2 * stats


def roofline(w, kt, pk, timed_s: float):
    """Roofline entry for the main kernel that took the most device time in the timed region."""
    phase = max(("fwd_main", "bwd_main", "bwd_dbias"), key=lambda p: kt[p][1])
    n, ms = kt[phase]
    if n == 0:
        return None
    sec = ms * 1e-3 / n
    fl, by = algorithmic(w, phase)
    sustained = timed_s > 1.0                    # a long timed region runs under the power cap
    tflops_peak = pk["bf16_sustained"] if sustained else pk["bf16"]
    t_tensor, t_hbm = fl / (tflops_peak * 1e12), by / (pk["hbm"] * 1e9)
    traffic = None
    tr = TRAFFIC.get((phase, w.name))
    if tr is not None and tr[2] is not None and _source_sha(tr[1]) == tr[2]:
        traffic = tr[0]
    kernel = {"fwd_main": "fwd::fwd_bf16_kernel", "bwd_main": "bwd::bwd_main_kernel",
              "bwd_dbias": "dbias::dbias_kernel"}[phase]
    if w.dtype != "bf16":
        kernel = {"fwd_main": "simt::fwd_kernel", "bwd_main": "simt backward", "bwd_dbias": "simt backward"}[phase]
    common = {"kernel": kernel, "launches": n, "us_per_launch": sec * 1e6, "flops_per_launch": fl,
              "algorithmic_bytes_per_launch": by, "traffic": traffic,
              "tensor_floor_us": t_tensor * 1e6, "hbm_floor_us": t_hbm * 1e6}
    if t_tensor >= t_hbm:
        a = fl / sec / 1e12
        return {"bound": "tensor", "achieved": a, "peak": tflops_peak, "unit": "TFLOP/s",
                "frac": a / tflops_peak,
                "peak_source": f"{pk['source']} bf16 {'sustained' if sustained else 'burst'}", **common}
    a = by / sec / 1e9
    return {"bound": "hbm", "achieved": a, "peak": pk["hbm"], "unit": "GB/s", "frac": a / pk["hbm"],
            "peak_source": f"{pk['source']} HBM copy", "tensor_frac": fl / sec / 1e12 / tflops_peak, **common}


def cpu_oracle_sample(w, target_s: float = 12.0, max_rows=None):
    """Time the fp64 oracle (fwd + bwd) on the first r rows s of the workload, r (and a repeat
    count) sized for about target_s seconds of CPU work."""
    import oracle
    oracle.build()
    inp = make_inputs(w, device="cpu")

    def rows(r):
        return {k: (None if v is None else (v[:, :r] if k in ("q", "k", "v", "g", "dout", "mask_bias") else v)
                    ).double().numpy() if v is not None else None for k, v in inp.items()}

    def run(x):
        t0 = time.perf_counter()
        oracle.forward(x["q"], x["k"], x["v"], x["g"], x["mask_bias"], x["pair_bias"])
        oracle.backward(x["q"], x["k"], x["v"], x["g"], x["mask_bias"], x["pair_bias"], x["dout"])
        return time.perf_counter() - t0

    t1 = run(rows(1))
    r = max(1, min(w.S, int(target_s / max(t1, 1e-3))))
    if max_rows:
        r = min(r, max_rows)
    x = rows(r)
    t, reps = 0.0, 0
    while reps == 0 or t < 0.7 * target_s:
        t += run(x)
        reps += 1
    L = w.B * r * w.H * w.N * w.N * reps
    fl = 14 * L * w.C
    return dict(value=fl / t / 1e12, unit="TFLOP/s", cores=oracle_threads(), kind="oracle",
                sample=f"{r} of {w.S} rows s (all {w.H} heads, N={w.N}) x{reps}, fwd+bwd, fp64, {t:.2f} s",
                seconds=t)


def oracle_threads() -> int:
    """Threads the OpenMP oracle runs with on this host."""
    v = os.environ.get("OMP_NUM_THREADS")
    if v and v.isdigit():
        return int(v)
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count()


def max_over_ranks(vals, world: int, device) -> list:
    """Element-wise maximum of per-rank timings (device time: the slowest rank decides)."""
    if world <= 1:
        return [float(v) for v in vals]
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_throughput(flops_per_step: float, steps: int, world: int, max_ms: float) -> float:
    """Whole-job TFLOP/s: the work of every rank over the slowest rank's time."""
    return flops_per_step * steps * world / (max_ms * 1e-3) / 1e12


def run_e2e(K: int, h2d, compute, d2h, world: int, dev, barrier) -> float:
    """End-to-end device milliseconds for K steps, copies overlapped across steps.

    Step j uses buffer set j % 2.  Its inputs are copied host -> device on one
    stream, its compute runs on a second, and its results are copied
    device -> host on a third, so one step's copies overlap its neighbours'
    compute (PCIe is full duplex).  Events order each step's three parts and
    keep a buffer set from being refilled before the step that used it two
    steps earlier is done with it.  Every step's copies are inside the timed
    region.  h2d(b), compute(b) and d2h(b) enqueue on the current stream.
    Returns the max over ranks.
    """
    st = [torch.cuda.Stream(device=dev) for _ in range(3)]
    ev = {(k, b): torch.cuda.Event() for k in ("in", "cmp", "out") for b in (0, 1)}

    def step(j):
        b = j % 2
        with torch.cuda.stream(st[0]):
            if j >= 2:
                st[0].wait_event(ev[("cmp", b)])       # the compute that read these inputs is done
            h2d(b)
            ev[("in", b)].record(st[0])
        with torch.cuda.stream(st[1]):
            st[1].wait_event(ev[("in", b)])
            if j >= 2:
                st[1].wait_event(ev[("out", b)])       # the copy-out of these results is done
            compute(b)
            ev[("cmp", b)].record(st[1])
        with torch.cuda.stream(st[2]):
            st[2].wait_event(ev[("cmp", b)])
            d2h(b)
            ev[("out", b)].record(st[2])

    for j in range(2):
        step(j)
    torch.cuda.synchronize()
    barrier()
    cur = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(cur)
    for x in st:
        x.wait_event(e0)
    for j in range(K):
        step(j)
    for x in st:
        cur.wait_stream(x)
    e1.record(cur)
    torch.cuda.synchronize()
    return max_over_ranks([e0.elapsed_time(e1)], world, dev)[0]


MIN_TIMED_S = 0.5


# ---------------------------------------------------------------------------
# Several GPUs: the rows s of one problem split over the ranks (row_shards).


def row_block(inp: dict, s0: int, s1: int) -> dict:
    """Rows [s0, s1) of one problem: the per-row tensors and the mask sliced (contiguous
    copies, so a transposed-pair layout becomes a plain block), the pair bias whole."""
    return {k: (v if v is None or k == "pair_bias" else v[:, s0:s1].contiguous()) for k, v in inp.items()}


def split_pass(blk: dict, group=None, fwd=None, bwd=None, **bwd_kw):
    """One forward + backward pass of this rank's row block, with d_pair_bias summed over
    every rank of ``group`` (rank order).  fwd / bwd default to row_shards.attn_fwd /
    attn_bwd; returns (out, lse, grads)."""
    from evoformer_pair_bias_b200 import row_shards
    fwd = fwd or row_shards.attn_fwd
    bwd = bwd or row_shards.attn_bwd
    out, lse = fwd(blk["q"], blk["k"], blk["v"], blk["g"], blk["mask_bias"], blk["pair_bias"])
    grads = bwd(blk["q"], blk["k"], blk["v"], blk["g"], blk["mask_bias"], blk["pair_bias"], out, lse, blk["dout"],
                group=group, **bwd_kw)
    return out, lse, grads


def run_row_split(args, w, rank, world, local):
    """--gpus N > 1: one problem, its rows split over the N ranks (strong scaling).

    Each rank runs the forward and backward of its own block of rows; the one
    exchange is the all-gather of the fp32 d_pair_bias partials (NCCL) and
    their rank-ordered sum (evo_sum_partials), inside the timed region.  The
    pass's time is the slowest rank's; ``value`` counts the whole problem once.
    """
    import datetime

    import torch.distributed as dist
    from evoformer_pair_bias_b200 import row_shards
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    try:
        A.load_library()
        s0, s1 = row_shards.row_range(w.S, world, rank)
        inp = make_inputs(w, device="cpu")
        host = row_block(inp, s0, s1)
        blk = {k: (None if v is None else v.to(dev)) for k, v in host.items()}
        bw = w.with_(S=s1 - s0, layout="msa_row" if w.layout == "tri_end" else w.layout)
        q = blk["q"]
        out = A.empty_like_rows(q)
        lse = torch.empty((w.B, s1 - s0, w.H, w.N), dtype=torch.float32, device=dev)
        grads = {n: A.empty_like_rows(q) for n in ("dq", "dk", "dv", "dg")}
        grads["d_pair_bias"] = torch.empty((w.B, 1, w.H, w.N, w.N), dtype=torch.float32, device=dev)
        ws = torch.empty(max(A.workspace_bytes(q), 1), dtype=torch.uint8, device=dev)
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        out_lo = A.empty_like_rows(q) if w.dtype == "bf16" else None

        def fwd_bwd(evs=None):
            if evs:
                evs[0].record()
            row_shards.attn_fwd(q, blk["k"], blk["v"], blk["g"], blk["mask_bias"], blk["pair_bias"], out=out,
                                lse=lse, out_lo=out_lo)
            if evs:
                evs[1].record()
            _, pending = row_shards.attn_bwd(q, blk["k"], blk["v"], blk["g"], blk["mask_bias"], blk["pair_bias"],
                                             out, lse, blk["dout"], grads=grads, workspace=ws, async_op=True,
                                             out_lo=out_lo)
            if evs:
                evs[2].record()
            pending.wait()
            if evs:
                evs[3].record()

        A.timing_enable(True)
        wev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        for i in range(args.warmup):
            flush.zero_()
            fwd_bwd(wev if i == args.warmup - 1 else None)
        torch.cuda.synchronize()
        A.timing_collect()
        if A.device_status(clear=True) != 0:
            raise RuntimeError("a kernel reported a timed-out wait during warm-up")
        K = args.steps
        R = passes_per_step(wev[0].elapsed_time(wev[3]), K, world, dev)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K * R)]
        with ClockSampler(gpu_uuid(dev)) as clk:
            dist.barrier()
            torch.cuda.synchronize()
            n0 = A.launch_count()
            for i in range(K * R):
                flush.zero_()
                fwd_bwd(ev[i])
            torch.cuda.synchronize()
            dist.barrier()
            launches = A.launch_count() - n0
        kt = A.timing_collect()
        A.timing_enable(False)
        f_ms = sum(e[0].elapsed_time(e[1]) for e in ev)
        b_ms = sum(e[1].elapsed_time(e[2]) for e in ev)
        x_ms = sum(e[2].elapsed_time(e[3]) for e in ev)
        tot = sum(e[0].elapsed_time(e[3]) for e in ev)
        tot, f_ms, b_ms, x_ms = max_over_ranks([tot, f_ms, b_ms, x_ms], world, dev)
        if A.device_status(clear=True) != 0:
            raise RuntimeError("a kernel reported a timed-out wait during the timed region")
        ff, bf = flops(w)
        value = (ff + bf) * K * R / (tot * 1e-3) / 1e12

        # end to end: each rank copies its block in from pinned host memory and its results out
        e2e = None
        if not args.no_e2e:
            hin = {k: (None if v is None else v.pin_memory()) for k, v in host.items()}
            h2d = sum(v.numel() * v.element_size() for v in hin.values() if v is not None)
            slots = []
            for _ in range(2):
                sl = {"in": {k: (None if v is None else torch.empty_like(v, device=dev)) for k, v in hin.items()}}
                sl["host"] = {"out": torch.empty(out.shape, dtype=out.dtype).pin_memory(),
                              "lse": torch.empty(lse.shape, dtype=lse.dtype).pin_memory()}
                for n_, g_ in grads.items():
                    sl["host"][n_] = torch.empty(g_.shape, dtype=g_.dtype).pin_memory()
                slots.append(sl)
            d2h = sum(v.numel() * v.element_size() for v in slots[0]["host"].values())
            res = [{}, {}]

            def e2e_h2d(b):
                for k_, v_ in hin.items():
                    if v_ is not None:
                        slots[b]["in"][k_].copy_(v_, non_blocking=True)

            def e2e_compute(b):
                o, l_, g_ = split_pass(slots[b]["in"], workspace=ws)
                res[b] = dict(g_, out=o, lse=l_)

            def e2e_d2h(b):
                for n_, t_ in slots[b]["host"].items():
                    t_.copy_(res[b][n_], non_blocking=True)

            et = run_e2e(K, e2e_h2d, e2e_compute, e2e_d2h, world, dev, dist.barrier)
            e2e = {"value": (ff + bf) * K / (et * 1e-3) / 1e12, "unit": "TFLOP/s",
                   "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": et / K,
                   "note": "per rank: its row block in, its results and the summed d_pair_bias out"}
        if rank == 0:
            pk = peaks()
            pair = w.B * w.H * w.N * w.N
            link_gbs = 770.0
            line = {
                "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
                "warmup": args.warmup, "ms_per_step": tot / K, "ms_per_pass": tot / (K * R),
                "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": w.dtype,
                "data": "synthetic",
                "config": {"workload": w.name, "B": w.B, "N_seq": w.S, "N_res": w.N, "H": w.H, "c": w.C,
                           "layout": w.layout, "mask": w.mask, "passes_per_step": R,
                           "l2": "flushed (256 MB write) before every pass, outside the timed brackets",
                           "parallelism": f"rows s split over {world} ranks ({s1 - s0} on rank 0); d_pair_bias "
                                          "partials all-gathered with NCCL and summed in rank order"},
                "fwd": {"us_per_call": 1e3 * f_ms / (K * R)},
                "bwd": {"us_per_call": 1e3 * b_ms / (K * R)},
                "exchange": {"us_per_pass": 1e3 * x_ms / (K * R), "bytes_in_per_rank": (world - 1) * pair * 4,
                             "nvlink_floor_us": (world - 1) * pair * 4 / (link_gbs * 1e9) * 1e6,
                             "link_gbs": link_gbs, "what": "all-gather wait + evo_sum_partials, after the "
                                                           "backward kernels"},
                "roofline": roofline(bw, kt, pk, timed_s=tot * 1e-3),
                "kernels": {p_: {"launches": kt[p_][0], "us_per_launch": 1e3 * kt[p_][1] / max(kt[p_][0], 1)}
                            for p_ in A.PHASES if kt[p_][0]},
                "cpu_baseline": None,
                "e2e": e2e,
                "gpu_launches": launches,
                "clocks": clk.summary(),
            }
            print(json.dumps(line), flush=True)
    finally:
        dist.destroy_process_group()
    return 0


def passes_per_step(pass_ms: float, steps: int, world: int, device) -> int:
    """Forward + backward passes per timed step so that `steps` steps take >= MIN_TIMED_S.

    From one warm-up pass's device time (the slowest rank's, so every rank
    agrees); at least 1.
    """
    pass_ms = max_over_ranks([pass_ms], world, device)[0]
    need = MIN_TIMED_S * 1e3 / max(pass_ms * max(steps, 1), 1e-6)
    return max(1, int(np.ceil(need)))


def run_reference(args, w, rank, world):
    if rank != 0:
        return 0
    steps, warm = args.steps, args.warmup
    info = cpu_oracle_sample(w, target_s=max(0.5, 60.0 / max(1, steps + warm)), max_rows=None)
    rows = int(info["sample"].split()[0])
    import oracle
    inp = make_inputs(w, device="cpu")
    x = {k: (None if v is None else (v[:, :rows] if k in ("q", "k", "v", "g", "dout", "mask_bias") else v)
             ).double().numpy() if v is not None else None for k, v in inp.items()}
    times = []
    for i in range(warm + steps):
        t0 = time.perf_counter()
        oracle.forward(x["q"], x["k"], x["v"], x["g"], x["mask_bias"], x["pair_bias"])
        oracle.backward(x["q"], x["k"], x["v"], x["g"], x["mask_bias"], x["pair_bias"], x["dout"])
        if i >= warm:
            times.append(time.perf_counter() - t0)
    t = sum(times)
    fl = 14 * w.B * rows * w.H * w.N * w.N * w.C * steps
    val = fl / t / 1e12
    line = {"metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": steps,
            "warmup": warm, "ms_per_step": 1e3 * t / steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": w.name, "B": w.B, "N_seq": w.S, "N_res": w.N, "H": w.H, "c": w.C,
                       "sample_rows": rows, "l2": "n/a (CPU)"},
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": oracle_threads(), "kind": "oracle",
                             "sample": f"{rows} of {w.S} rows s per step, fwd+bwd, fp64"},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# Fused pre-attention projection (LayerNorm + linear)


def proj_parts(pw):
    """The projections one step runs: the q, k, v, g projection, plus the pair bias for the pair representation."""
    return ("qkvg", "pair_bias") if pw.name.startswith("pair") else ("qkvg",)


def proj_algorithmic(pw, part: str):
    """(FLOPs, bytes) of one launch: x read once, w and the LayerNorm/bias vectors read once, y written once."""
    n_out = pw.n_out if part == "qkvg" else pw.H
    fl = 2 * pw.rows * pw.c_in * n_out
    by = pw.rows * pw.c_in * 2 + pw.c_in * n_out * 2 + (2 * pw.c_in + n_out) * 4 + pw.rows * n_out * 2
    return fl, by


def proj_roofline(pw, part, us, pk, timed_s):
    fl, by = proj_algorithmic(pw, part)
    sec = us * 1e-6
    sustained = timed_s > 1.0
    tflops_peak = pk["bf16_sustained"] if sustained else pk["bf16"]
    t_tensor, t_hbm = fl / (tflops_peak * 1e12), by / (pk["hbm"] * 1e9)
    tr = TRAFFIC.get((part, pw.name))
    traffic = tr[0] if tr is not None and _source_sha(tr[1]) == tr[2] else None
    kernel = {"qkvg": "proj::ln_linear_kernel", "pair_bias": "proj::pair_bias_kernel"}[part]
    common = {"kernel": kernel, "us_per_launch": us, "flops_per_launch": fl, "algorithmic_bytes_per_launch": by,
              "traffic": traffic, "tensor_floor_us": t_tensor * 1e6, "hbm_floor_us": t_hbm * 1e6}
    if t_tensor >= t_hbm:
        a = fl / sec / 1e12
        return {"bound": "tensor", "achieved": a, "peak": tflops_peak, "unit": "TFLOP/s", "frac": a / tflops_peak,
                "peak_source": f"{pk['source']} bf16 {'sustained' if sustained else 'burst'}", **common}
    a = by / sec / 1e9
    return {"bound": "hbm", "achieved": a, "peak": pk["hbm"], "unit": "GB/s", "frac": a / pk["hbm"],
            "peak_source": f"{pk['source']} HBM copy", "tensor_frac": fl / sec / 1e12 / tflops_peak, **common}


def proj_oracle_sample(pw, target_s: float = 12.0):
    """Time the fp64 oracle projection on the first r rows of the workload, sized for about target_s."""
    import oracle
    oracle.build()
    d = make_proj_inputs(pw)
    pb = make_pair_bias_params(pw) if "pair_bias" in proj_parts(pw) else None
    x_all = d["x"].reshape(-1, pw.c_in)
    f = {k: d[k].double().numpy() for k in ("w", "ln_w", "ln_b", "bias")}
    fb = None if pb is None else {k: v.double().numpy() for k, v in pb.items()}

    def run(r):
        x = x_all[:r].double().numpy()
        t0 = time.perf_counter()
        oracle.ln_linear(x, f["ln_w"], f["ln_b"], PROJ_EPS, f["w"], f["bias"])
        if fb is not None:
            oracle.ln_linear(x, fb["ln_w"], fb["ln_b"], PROJ_EPS, fb["w"], fb["bias"])
        return time.perf_counter() - t0

    t1 = run(64) / 64
    r = max(64, min(pw.rows, int(target_s / max(t1, 1e-9))))
    t, reps = 0.0, 0
    while reps == 0 or t < 0.7 * target_s:
        t += run(r)
        reps += 1
    fl = sum(proj_algorithmic(pw, p)[0] for p in proj_parts(pw)) * r / pw.rows * reps
    return dict(value=fl / t / 1e12, unit="TFLOP/s", cores=oracle_threads(), kind="oracle",
                sample=f"{r} of {pw.rows} rows x{reps}, {'+'.join(proj_parts(pw))}, fp64, {t:.2f} s",
                seconds=t, rows=r)


def run_projection(args, pw, rank, world, local):
    parts = proj_parts(pw)
    fl_step = sum(proj_algorithmic(pw, p)[0] for p in parts)
    base_cfg = {"workload": pw.name, "B": pw.B, "rows_per_batch": pw.S, "N_res": pw.N, "c_in": pw.c_in,
                "H": pw.H, "c": pw.C, "n_out": pw.n_out, "projections": list(parts), "eps": PROJ_EPS}
    if args.impl == "reference":
        if rank != 0:
            return 0
        steps, warm = args.steps, args.warmup
        info = proj_oracle_sample(pw, target_s=max(0.5, 60.0 / max(1, steps + warm)))
        r = info["rows"]
        import oracle
        d = make_proj_inputs(pw)
        x = d["x"].reshape(-1, pw.c_in)[:r].double().numpy()
        f = {k: d[k].double().numpy() for k in ("w", "ln_w", "ln_b", "bias")}
        fb = ({k: v.double().numpy() for k, v in make_pair_bias_params(pw).items()}
              if "pair_bias" in parts else None)
        times = []
        for i in range(warm + steps):
            t0 = time.perf_counter()
            oracle.ln_linear(x, f["ln_w"], f["ln_b"], PROJ_EPS, f["w"], f["bias"])
            if fb is not None:
                oracle.ln_linear(x, fb["ln_w"], fb["ln_b"], PROJ_EPS, fb["w"], fb["bias"])
            if i >= warm:
                times.append(time.perf_counter() - t0)
        t = sum(times)
        val = fl_step * r / pw.rows * steps / t / 1e12
        line = {"metric": PROJ_METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": steps,
                "warmup": warm, "ms_per_step": 1e3 * t / steps, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
                "config": {**base_cfg, "sample_rows": r, "l2": "n/a (CPU)"},
                "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": oracle_threads(), "kind": "oracle",
                                 "sample": f"{r} of {pw.rows} rows per step, fp64"},
                "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0

    if world > 1:
        return run_row_split(args, w, rank, world, local)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    A.load_library()
    hin = make_proj_inputs(pw)
    d = {k: v.to(dev) for k, v in hin.items()}
    pbp = {k: v.to(dev) for k, v in make_pair_bias_params(pw).items()} if "pair_bias" in parts else None
    y = torch.empty(pw.B, pw.S, pw.N, pw.n_out, dtype=torch.bfloat16, device=dev)
    pb = torch.empty(pw.B, 1, pw.H, pw.N, pw.N, dtype=torch.bfloat16, device=dev) if pbp else None
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def step(x):
        A.ln_linear(x, d["ln_w"], d["ln_b"], PROJ_EPS, d["w"], d["bias"], y=y)
        if pbp is not None:
            A.ln_pair_bias(x, pbp["ln_w"], pbp["ln_b"], PROJ_EPS, pbp["w"], pbp["bias"], out=pb)

    A.timing_enable(True)
    for _ in range(args.warmup):
        flush.zero_()
        step(d["x"])
    torch.cuda.synchronize()
    A.timing_collect()
    if A.device_status(clear=True) != 0:
        raise RuntimeError("a kernel reported an error during warm-up")
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    with ClockSampler(gpu_uuid(dev)) as clk:
        barrier()
        torch.cuda.synchronize()
        n0 = A.launch_count()
        for i in range(K):
            flush.zero_()
            ev[i][0].record()
            step(d["x"])
            ev[i][1].record()
        torch.cuda.synchronize()
        barrier()
        launches = A.launch_count() - n0
    kt = A.timing_collect()
    A.timing_enable(False)
    tot = max_over_ranks([sum(e0.elapsed_time(e1) for e0, e1 in ev)], world, dev)[0]
    if A.device_status(clear=True) != 0:
        raise RuntimeError("a kernel reported an error during the timed region")
    value = job_throughput(fl_step, K, world, tot)
    pk = peaks()
    phase = {"qkvg": "proj", "pair_bias": "pair_bias"}
    us = {p: 1e3 * kt[phase[p]][1] / max(kt[phase[p]][0], 1) for p in parts}

    # the same step replayed from a CUDA graph: no host launch overhead between the kernels
    graph_ms = None
    try:
        s_cap = torch.cuda.Stream()
        s_cap.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s_cap):
            step(d["x"])
        torch.cuda.current_stream().wait_stream(s_cap)
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            step(d["x"])
        gev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
        for i in range(K):
            flush.zero_()
            gev[i][0].record()
            gr.replay()
            gev[i][1].record()
        torch.cuda.synchronize()
        graph_ms = max_over_ranks([sum(a.elapsed_time(b) for a, b in gev)], world, dev)[0] / K
        del gr
    except Exception as exc:  # reported, never required
        graph_ms = repr(exc)

    e2e = None
    if not args.no_e2e:
        hx = hin["x"].pin_memory()
        slots = []
        for _ in range(2):
            sl = {"x": torch.empty_like(hx, device=dev), "y": torch.empty_like(y),
                  "pb": torch.empty_like(pb) if pb is not None else None,
                  "hy": torch.empty(y.shape, dtype=y.dtype).pin_memory(),
                  "hpb": torch.empty(pb.shape, dtype=pb.dtype).pin_memory() if pb is not None else None}
            slots.append(sl)

        def e2e_h2d(b):
            slots[b]["x"].copy_(hx, non_blocking=True)

        def e2e_compute(b):
            sl = slots[b]
            A.ln_linear(sl["x"], d["ln_w"], d["ln_b"], PROJ_EPS, d["w"], d["bias"], y=sl["y"])
            if pbp is not None:
                A.ln_pair_bias(sl["x"], pbp["ln_w"], pbp["ln_b"], PROJ_EPS, pbp["w"], pbp["bias"], out=sl["pb"])

        def e2e_d2h(b):
            sl = slots[b]
            sl["hy"].copy_(sl["y"], non_blocking=True)
            if sl["hpb"] is not None:
                sl["hpb"].copy_(sl["pb"], non_blocking=True)

        et = run_e2e(K, e2e_h2d, e2e_compute, e2e_d2h, world, dev, barrier)
        hy, hpb = slots[0]["hy"], slots[0]["hpb"]
        e2e = {"value": job_throughput(fl_step, K, world, et), "unit": "TFLOP/s",
               "h2d_bytes_per_step": hx.numel() * hx.element_size(),
               "d2h_bytes_per_step": hy.numel() * hy.element_size() + (0 if hpb is None else
                                                                       hpb.numel() * hpb.element_size()),
               "ms_per_step": et / K,
               "pipelining": "step j+1's input in and step j-1's results out overlap step j's compute"}

    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        try:
            cpu = proj_oracle_sample(pw)
            cpu.pop("seconds", None)
            cpu.pop("rows", None)
        except Exception as exc:  # the baseline is reported, never required
            cpu = {"error": repr(exc)}

    if rank == 0:
        top = max(parts, key=lambda p: us[p])
        line = {
            "metric": PROJ_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": tot / K, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {**base_cfg, "l2": "flushed (256 MB write) before every step",
                       "parallelism": f"replicas x{world}, rows independent, no collective"},
            "roofline": proj_roofline(pw, top, us[top], pk, timed_s=tot * 1e-3),
            "kernels": {p: {"launches": kt[phase[p]][0], "us_per_launch": us[p],
                            "roofline": proj_roofline(pw, p, us[p], pk, timed_s=tot * 1e-3)} for p in parts},
            "graph_ms_per_step": graph_ms,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches,
            "clocks": clk.summary(),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


# ---------------------------------------------------------------------------
# Triangular multiplicative update (its contraction)


def tri_algorithmic(tw):
    """(FLOPs, bytes) of one launch (one direction): a and b read once, z written once (bf16)."""
    return tw.flops, 3 * tw.B * tw.C * tw.N * tw.N * 2


def tri_oracle_sample(tw, target_s: float = 12.0):
    """Time the fp64 oracle (both directions) on the first r channels of the workload."""
    import oracle
    oracle.build()
    d = make_tri_mul_inputs(tw)
    a_all = d["a"].double().permute(0, 2, 3, 1)
    b_all = d["b"].double().permute(0, 2, 3, 1)

    def run(r):
        a = a_all[:1, :, :, :r].contiguous().numpy()
        b = b_all[:1, :, :, :r].contiguous().numpy()
        t0 = time.perf_counter()
        oracle.tri_mul(a, b, False)
        oracle.tri_mul(a, b, True)
        return time.perf_counter() - t0

    t1 = run(1)
    r = max(1, min(tw.C, int(target_s / max(t1, 1e-6) / 2)))
    t, reps = 0.0, 0
    while reps == 0 or t < 0.7 * target_s:
        t += run(r)
        reps += 1
    fl = 2 * 2 * r * tw.N ** 3 * reps
    return dict(value=fl / t / 1e12, unit="TFLOP/s", cores=oracle_threads(), kind="oracle",
                sample=f"{r} of {tw.B * tw.C} channel matrices x{reps}, both directions, fp64, {t:.2f} s",
                seconds=t, channels=r)


def run_tri_mul(args, tw, rank, world, local):
    fl_launch, by_launch = tri_algorithmic(tw)
    fl_step = 2 * fl_launch
    cfg = {"workload": tw.name, "B": tw.B, "N_res": tw.N, "C": tw.C, "layout": "channel-first [B, C, N, N]",
           "directions": ["outgoing", "incoming"]}
    if args.impl == "reference":
        if rank != 0:
            return 0
        steps, warm = args.steps, args.warmup
        info = tri_oracle_sample(tw, target_s=max(0.5, 60.0 / max(1, steps + warm)))
        r = info["channels"]
        import oracle
        d = make_tri_mul_inputs(tw)
        a = d["a"].double().permute(0, 2, 3, 1)[:1, :, :, :r].contiguous().numpy()
        b = d["b"].double().permute(0, 2, 3, 1)[:1, :, :, :r].contiguous().numpy()
        times = []
        for i in range(warm + steps):
            t0 = time.perf_counter()
            oracle.tri_mul(a, b, False)
            oracle.tri_mul(a, b, True)
            if i >= warm:
                times.append(time.perf_counter() - t0)
        t = sum(times)
        val = 2 * 2 * r * tw.N ** 3 * steps / t / 1e12
        line = {"metric": TRI_METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": steps,
                "warmup": warm, "ms_per_step": 1e3 * t / steps, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
                "config": {**cfg, "sample_channels": r, "l2": "n/a (CPU)"},
                "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": oracle_threads(), "kind": "oracle",
                                 "sample": f"{r} of {tw.B * tw.C} channel matrices per step, fp64"},
                "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0

    import datetime
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    A.load_library()
    hin = make_tri_mul_inputs(tw)
    d = {k: v.to(dev) for k, v in hin.items()}
    z_out = torch.empty_like(d["a"])
    z_in = torch.empty_like(d["a"])
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def step(a, b):
        A.tri_mul(a, b, False, z=z_out)
        A.tri_mul(a, b, True, z=z_in)

    A.timing_enable(True)
    for _ in range(args.warmup):
        flush.zero_()
        step(d["a"], d["b"])
    torch.cuda.synchronize()
    A.timing_collect()
    if A.device_status(clear=True) != 0:
        raise RuntimeError("a kernel reported an error during warm-up")
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    with ClockSampler(gpu_uuid(dev)) as clk:
        barrier()
        torch.cuda.synchronize()
        n0 = A.launch_count()
        for i in range(K):
            flush.zero_()
            ev[i][0].record()
            step(d["a"], d["b"])
            ev[i][1].record()
        torch.cuda.synchronize()
        barrier()
        launches = A.launch_count() - n0
    kt = A.timing_collect()
    A.timing_enable(False)
    tot = max_over_ranks([sum(e0.elapsed_time(e1) for e0, e1 in ev)], world, dev)[0]
    if A.device_status(clear=True) != 0:
        raise RuntimeError("a kernel reported an error during the timed region")
    value = job_throughput(fl_step, K, world, tot)
    pk = peaks()
    n_l, ms_l = kt["tri_mul"]
    us = 1e3 * ms_l / max(n_l, 1)
    sec = us * 1e-6
    sustained = tot * 1e-3 > 1.0
    tflops_peak = pk["bf16_sustained"] if sustained else pk["bf16"]
    t_tensor, t_hbm = fl_launch / (tflops_peak * 1e12), by_launch / (pk["hbm"] * 1e9)
    tr = TRAFFIC.get(("tri_mul", tw.name))
    common = {"kernel": "trimul::tri_mul_kernel", "launches": n_l, "us_per_launch": us, "flops_per_launch": fl_launch,
              "algorithmic_bytes_per_launch": by_launch,
              "traffic": tr[0] if tr is not None and _source_sha(tr[1]) == tr[2] else None,
              "tensor_floor_us": t_tensor * 1e6, "hbm_floor_us": t_hbm * 1e6}
    if t_tensor >= t_hbm:
        a_ = fl_launch / sec / 1e12
        roof = {"bound": "tensor", "achieved": a_, "peak": tflops_peak, "unit": "TFLOP/s", "frac": a_ / tflops_peak,
                "peak_source": f"{pk['source']} bf16 {'sustained' if sustained else 'burst'}", **common}
    else:
        a_ = by_launch / sec / 1e9
        roof = {"bound": "hbm", "achieved": a_, "peak": pk["hbm"], "unit": "GB/s", "frac": a_ / pk["hbm"],
                "peak_source": f"{pk['source']} HBM copy", "tensor_frac": fl_launch / sec / 1e12 / tflops_peak,
                **common}

    e2e = None
    if not args.no_e2e:
        ha, hb = hin["a"].pin_memory(), hin["b"].pin_memory()
        slots = [{"a": torch.empty_like(ha, device=dev), "b": torch.empty_like(hb, device=dev),
                  "zo": torch.empty_like(z_out), "zi": torch.empty_like(z_in),
                  "hzo": torch.empty(z_out.shape, dtype=z_out.dtype).pin_memory(),
                  "hzi": torch.empty(z_in.shape, dtype=z_in.dtype).pin_memory()} for _ in range(2)]

        def e2e_h2d(b):
            slots[b]["a"].copy_(ha, non_blocking=True)
            slots[b]["b"].copy_(hb, non_blocking=True)

        def e2e_compute(b):
            sl = slots[b]
            A.tri_mul(sl["a"], sl["b"], False, z=sl["zo"])
            A.tri_mul(sl["a"], sl["b"], True, z=sl["zi"])

        def e2e_d2h(b):
            sl = slots[b]
            sl["hzo"].copy_(sl["zo"], non_blocking=True)
            sl["hzi"].copy_(sl["zi"], non_blocking=True)

        et = run_e2e(K, e2e_h2d, e2e_compute, e2e_d2h, world, dev, barrier)
        e2e = {"value": job_throughput(fl_step, K, world, et), "unit": "TFLOP/s",
               "h2d_bytes_per_step": 2 * ha.numel() * ha.element_size(),
               "d2h_bytes_per_step": 2 * z_out.numel() * z_out.element_size(), "ms_per_step": et / K,
               "pipelining": "step j+1's inputs in and step j-1's results out overlap step j's compute"}

    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        try:
            cpu = tri_oracle_sample(tw)
            cpu.pop("seconds", None)
            cpu.pop("channels", None)
        except Exception as exc:  # the baseline is reported, never required
            cpu = {"error": repr(exc)}

    if rank == 0:
        line = {
            "metric": TRI_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": tot / K, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {**cfg, "l2": "flushed (256 MB write) before every step",
                       "parallelism": f"replicas x{world}, channels independent, no collective"},
            "roofline": roof,
            "kernels": {"tri_mul": {"launches": n_l, "us_per_launch": us}},
            "frac_measured_peak": value / world / pk["bf16"],
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches,
            "clocks": clk.summary(),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


# ---------------------------------------------------------------------------
# Outer product mean


def opm_oracle_sample(ow, target_s: float = 12.0):
    """Time the fp64 oracle on the first r columns i of the workload (all j), sized for about target_s."""
    import oracle
    oracle.build()
    d = make_opm_inputs(ow)
    a_all, b = d["a"].double().numpy(), d["b"].double().numpy()

    def run(r):
        a = np.ascontiguousarray(a_all[:, :, :r])
        t0 = time.perf_counter()
        oracle.outer_product_mean(a, b)
        return time.perf_counter() - t0

    t1 = run(1)
    r = max(1, min(ow.N, int(target_s / max(t1, 1e-6) / 2)))
    t, reps = 0.0, 0
    while reps == 0 or t < 0.7 * target_s:
        t += run(r)
        reps += 1
    fl = ow.flops * r / ow.N * reps
    return dict(value=fl / t / 1e12, unit="TFLOP/s", cores=oracle_threads(), kind="oracle",
                sample=f"{r} of {ow.N} columns i (all j) x{reps}, fp64, {t:.2f} s", seconds=t, rows=r)


def run_opm(args, ow, rank, world, local):
    fl = ow.flops
    by = 2 * ow.B * ow.S * ow.N * ow.C * 2 + ow.B * (ow.N * ow.C) ** 2 * 2
    cfg = {"workload": ow.name, "B": ow.B, "N_seq": ow.S, "N_res": ow.N, "C": ow.C,
           "output": "bf16 [B, N, C, N, C]"}
    if args.impl == "reference":
        if rank != 0:
            return 0
        steps, warm = args.steps, args.warmup
        info = opm_oracle_sample(ow, target_s=max(0.5, 60.0 / max(1, steps + warm)))
        r = info["rows"]
        import oracle
        d = make_opm_inputs(ow)
        a = np.ascontiguousarray(d["a"].double().numpy()[:, :, :r])
        b = d["b"].double().numpy()
        times = []
        for i in range(warm + steps):
            t0 = time.perf_counter()
            oracle.outer_product_mean(a, b)
            if i >= warm:
                times.append(time.perf_counter() - t0)
        t = sum(times)
        val = fl * r / ow.N * steps / t / 1e12
        line = {"metric": OPM_METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": steps,
                "warmup": warm, "ms_per_step": 1e3 * t / steps, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
                "config": {**cfg, "sample_columns": r, "l2": "n/a (CPU)"},
                "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": oracle_threads(), "kind": "oracle",
                                 "sample": f"{r} of {ow.N} columns i per step, fp64"},
                "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0

    import datetime
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    A.load_library()
    hin = make_opm_inputs(ow)
    d = {k: v.to(dev) for k, v in hin.items()}
    out = torch.empty((ow.B, ow.N, ow.C, ow.N, ow.C), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    A.timing_enable(True)
    for _ in range(args.warmup):
        flush.zero_()
        A.outer_product_mean(d["a"], d["b"], out=out)
    torch.cuda.synchronize()
    A.timing_collect()
    if A.device_status(clear=True) != 0:
        raise RuntimeError("a kernel reported an error during warm-up")
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    with ClockSampler(gpu_uuid(dev)) as clk:
        barrier()
        torch.cuda.synchronize()
        n0 = A.launch_count()
        for i in range(K):
            flush.zero_()
            ev[i][0].record()
            A.outer_product_mean(d["a"], d["b"], out=out)
            ev[i][1].record()
        torch.cuda.synchronize()
        barrier()
        launches = A.launch_count() - n0
    kt = A.timing_collect()
    A.timing_enable(False)
    tot = max_over_ranks([sum(e0.elapsed_time(e1) for e0, e1 in ev)], world, dev)[0]
    if A.device_status(clear=True) != 0:
        raise RuntimeError("a kernel reported an error during the timed region")
    value = job_throughput(fl, K, world, tot)
    pk = peaks()
    n_l, ms_l = kt["opm"]
    us = 1e3 * ms_l / max(n_l, 1)
    sec = us * 1e-6
    sustained = tot * 1e-3 > 1.0
    tflops_peak = pk["bf16_sustained"] if sustained else pk["bf16"]
    t_tensor, t_hbm = fl / (tflops_peak * 1e12), by / (pk["hbm"] * 1e9)
    tr = TRAFFIC.get(("opm", ow.name))
    common = {"kernel": "trimul::tri_mul_kernel (MN-major, scale 1/S)", "launches": n_l, "us_per_launch": us,
              "flops_per_launch": fl, "algorithmic_bytes_per_launch": by,
              "traffic": tr[0] if tr is not None and _source_sha(tr[1]) == tr[2] else None,
              "tensor_floor_us": t_tensor * 1e6, "hbm_floor_us": t_hbm * 1e6}
    if t_tensor >= t_hbm:
        a_ = fl / sec / 1e12
        roof = {"bound": "tensor", "achieved": a_, "peak": tflops_peak, "unit": "TFLOP/s", "frac": a_ / tflops_peak,
                "peak_source": f"{pk['source']} bf16 {'sustained' if sustained else 'burst'}", **common}
    else:
        a_ = by / sec / 1e9
        roof = {"bound": "hbm", "achieved": a_, "peak": pk["hbm"], "unit": "GB/s", "frac": a_ / pk["hbm"],
                "peak_source": f"{pk['source']} HBM copy", "tensor_frac": fl / sec / 1e12 / tflops_peak, **common}

    e2e = None
    if not args.no_e2e:
        ha, hb = hin["a"].pin_memory(), hin["b"].pin_memory()
        slots = [{"a": torch.empty_like(ha, device=dev), "b": torch.empty_like(hb, device=dev),
                  "o": torch.empty_like(out), "ho": torch.empty(out.shape, dtype=out.dtype).pin_memory()}
                 for _ in range(2)]

        def e2e_h2d(b):
            slots[b]["a"].copy_(ha, non_blocking=True)
            slots[b]["b"].copy_(hb, non_blocking=True)

        def e2e_compute(b):
            A.outer_product_mean(slots[b]["a"], slots[b]["b"], out=slots[b]["o"])

        def e2e_d2h(b):
            slots[b]["ho"].copy_(slots[b]["o"], non_blocking=True)

        et = run_e2e(K, e2e_h2d, e2e_compute, e2e_d2h, world, dev, barrier)
        e2e = {"value": job_throughput(fl, K, world, et), "unit": "TFLOP/s",
               "h2d_bytes_per_step": 2 * ha.numel() * ha.element_size(),
               "d2h_bytes_per_step": out.numel() * out.element_size(), "ms_per_step": et / K,
               "pipelining": "step j+1's inputs in and step j-1's results out overlap step j's compute"}

    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        try:
            cpu = opm_oracle_sample(ow)
            cpu.pop("seconds", None)
            cpu.pop("rows", None)
        except Exception as exc:  # the baseline is reported, never required
            cpu = {"error": repr(exc)}

    if rank == 0:
        line = {
            "metric": OPM_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": tot / K, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {**cfg, "l2": "flushed (256 MB write) before every step",
                       "parallelism": f"replicas x{world}, batches independent, no collective"},
            "roofline": roof,
            "kernels": {"opm": {"launches": n_l, "us_per_launch": us}},
            "frac_measured_peak": value / world / pk["bf16"],
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches,
            "clocks": clk.summary(),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_BENCH, choices=sorted(WORKLOADS) + sorted(PROJ_WORKLOADS) + sorted(TRI_MUL_WORKLOADS) + sorted(OPM_WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.workload in PROJ_WORKLOADS:
        return run_projection(args, PROJ_WORKLOADS[args.workload], rank, world, local)
    if args.workload in TRI_MUL_WORKLOADS:
        return run_tri_mul(args, TRI_MUL_WORKLOADS[args.workload], rank, world, local)
    if args.workload in OPM_WORKLOADS:
        return run_opm(args, OPM_WORKLOADS[args.workload], rank, world, local)
    w = WORKLOADS[args.workload]

    if args.impl == "reference":
        return run_reference(args, w, rank, world)

    import datetime
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    A.load_library()
    inp = make_inputs(w, device="cpu")
    d = {k: (None if v is None else v.to(dev)) for k, v in inp.items()}
    out = A.empty_like_rows(d["q"])
    lse = torch.empty((w.B, w.S, w.H, w.N), dtype=torch.float32, device=dev)
    dout = d["dout"] if d["dout"].stride() == out.stride() else A.empty_like_rows(out).copy_(d["dout"])
    grads = {n: A.empty_like_rows(d["q"]) for n in ("dq", "dk", "dv", "dg")}
    grads["d_pair_bias"] = torch.empty((w.B, 1, w.H, w.N, w.N), dtype=torch.float32, device=dev)
    ws = torch.empty(max(A.workspace_bytes(d["q"]), 1), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    # bf16: the forward also writes out's rounding residual, which the backward uses for D_i
    out_lo = A.empty_like_rows(d["q"]) if w.dtype == "bf16" else None

    def fwd():
        A.evo_attn_fwd(d["q"], d["k"], d["v"], d["g"], d["mask_bias"], d["pair_bias"], out=out, lse=lse,
                       out_lo=out_lo)

    def bwd():
        A.evo_attn_bwd(d["q"], d["k"], d["v"], d["g"], d["mask_bias"], d["pair_bias"], out, lse, dout,
                       grads=grads, workspace=ws, out_lo=out_lo)

    def step():
        fwd()
        bwd()

    A.timing_enable(True)
    wev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    for i in range(args.warmup):
        flush.zero_()
        if i == args.warmup - 1:
            wev[0].record()
        step()
    wev[1].record()
    torch.cuda.synchronize()
    A.timing_collect()
    if A.device_status(clear=True) != 0:
        raise RuntimeError("a kernel reported a timed-out wait during warm-up")

    K = args.steps
    # Passes per step: enough forward + backward passes that the K timed steps
    # span at least MIN_TIMED_S of device time (so that the clock samples see
    # the GPU under load), the same number on every rank.
    R = passes_per_step(wev[0].elapsed_time(wev[1]), K, world, dev)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K * R)]
    with ClockSampler(gpu_uuid(dev)) as clk:
        barrier()
        torch.cuda.synchronize()
        n0 = A.launch_count()
        for i in range(K * R):
            flush.zero_()
            ev[i][0].record()
            fwd()
            ev[i][1].record()
            bwd()
            ev[i][2].record()
        torch.cuda.synchronize()
        barrier()
        launches = A.launch_count() - n0
    kt = A.timing_collect()
    A.timing_enable(False)
    fwd_ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(K * R)]
    bwd_ms = [ev[i][1].elapsed_time(ev[i][2]) for i in range(K * R)]
    tot_ms = sum(fwd_ms) + sum(bwd_ms)
    tot_ms, fsum, bsum = max_over_ranks([tot_ms, sum(fwd_ms), sum(bwd_ms)], world, dev)
    if A.device_status(clear=True) != 0:
        raise RuntimeError("a kernel reported a timed-out wait during the timed region")

    ff, bf = flops(w)
    pk = peaks()
    value = job_throughput(R * (ff + bf), K, world, tot_ms)
    fwd_tf = ff * K * R / (fsum * 1e-3) / 1e12
    bwd_tf = bf * K * R / (bsum * 1e-3) / 1e12

    # end to end: pinned host inputs -> device, fwd + bwd through the public API, results -> pinned host
    e2e = None
    if not args.no_e2e:
        def storage(name, v):  # the underlying (contiguous) buffer of a logical view
            if w.layout == "tri_end" and name in ("q", "k", "v", "g", "dout"):
                return v.permute(0, 2, 1, 3, 4)
            return v
        hin = {k: (None if v is None else storage(k, v).contiguous().pin_memory()) for k, v in inp.items()}
        h2d = sum(v.numel() * v.element_size() for v in hin.values() if v is not None)
        slots = []
        for _ in range(2):           # device inputs, outputs and pinned host results per buffer set
            sl = {"in": {k: (None if v is None else torch.empty_like(v, device=dev)) for k, v in hin.items()},
                  "out": A.empty_like_rows(d["q"]),
                  "out_lo": A.empty_like_rows(d["q"]) if w.dtype == "bf16" else None,
                  "lse": torch.empty((w.B, w.S, w.H, w.N), dtype=torch.float32, device=dev),
                  "dout": A.empty_like_rows(d["q"]),
                  "grads": {n: A.empty_like_rows(d["q"]) for n in ("dq", "dk", "dv", "dg")}}
            sl["grads"]["d_pair_bias"] = torch.empty((w.B, 1, w.H, w.N, w.N), dtype=torch.float32, device=dev)
            sl["host"] = {"out": torch.empty(out.shape, dtype=out.dtype).pin_memory(),
                          "lse": torch.empty(lse.shape, dtype=lse.dtype).pin_memory()}
            for n, g in sl["grads"].items():
                sl["host"][n] = torch.empty(g.shape, dtype=g.dtype).pin_memory()
            slots.append(sl)
        d2h = sum(v.numel() * v.element_size() for v in slots[0]["host"].values())

        def e2e_h2d(b):
            for k, v in hin.items():
                if v is not None:
                    slots[b]["in"][k].copy_(v, non_blocking=True)

        def e2e_compute(b):
            sl = slots[b]
            di = sl["in"]
            q, k_, v_, g_, do = (logical_view(w, di[n]) for n in ("q", "k", "v", "g", "dout"))
            r = A.evo_attn_fwd(q, k_, v_, g_, di["mask_bias"], di["pair_bias"], out=sl["out"], lse=sl["lse"],
                               out_lo=sl["out_lo"])
            o, l_ = r[0], r[1]
            do = do if do.stride() == o.stride() else sl["dout"].copy_(do)
            A.evo_attn_bwd(q, k_, v_, g_, di["mask_bias"], di["pair_bias"], o, l_, do, grads=sl["grads"],
                           workspace=ws, out_lo=sl["out_lo"])

        def e2e_d2h(b):
            sl = slots[b]
            sl["host"]["out"].copy_(sl["out"], non_blocking=True)
            sl["host"]["lse"].copy_(sl["lse"], non_blocking=True)
            for n, g in sl["grads"].items():
                sl["host"][n].copy_(g, non_blocking=True)

        et = run_e2e(K, e2e_h2d, e2e_compute, e2e_d2h, world, dev, barrier)
        e2e = {"value": job_throughput(ff + bf, K, world, et), "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": et / K,
               "pipelining": "step j+1's inputs in and step j-1's results out overlap step j's compute "
                             "(three streams, two buffer sets)"}

    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        try:
            cpu = cpu_oracle_sample(w)
            cpu.pop("seconds", None)
        except Exception as exc:  # the baseline is reported, never required
            cpu = {"error": repr(exc)}

    if rank == 0:
        fwd_us = 1e3 * fsum / (K * R)
        roof = roofline(w, kt, pk, timed_s=tot_ms * 1e-3)
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": tot_ms / K, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "N_seq": w.S, "N_res": w.N, "H": w.H, "c": w.C,
                       "layout": w.layout, "mask": w.mask, "passes_per_step": R,
                       "l2": "flushed (256 MB write) before every forward + backward pass, outside the timed "
                             "brackets" + ("; inputs also larger than L2" if 5 * w.B * w.S * w.N * w.H
                                                                            * w.C * 2 > (126 << 20) else ""),
                       "parallelism": "one GPU (with --gpus N the rows are split over N ranks)"},
            "ms_per_pass": tot_ms / (K * R),
            "fwd": {"tflops": fwd_tf, "us_per_call": fwd_us, "frac_measured_peak": fwd_tf / pk["bf16"],
                    "frac_nominal_peak": fwd_tf / NOMINAL_BF16_TFLOPS},
            "bwd": {"tflops": bwd_tf, "us_per_call": 1e3 * bsum / (K * R),
                    "frac_measured_peak": bwd_tf / pk["bf16"],
                    "frac_nominal_peak": bwd_tf / NOMINAL_BF16_TFLOPS},
            "frac_measured_peak": value / world / pk["bf16"],
            "roofline": roof,
            "kernels": {p: {"launches": kt[p][0], "us_per_launch": 1e3 * kt[p][1] / max(kt[p][0], 1)}
                        for p in A.PHASES if kt[p][0]},
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches,
            "clocks": clk.summary(),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
