#!/usr/bin/env python3
"""Throughput of the selective scan (S6) on B200: one JSON line on stdout.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mss|reference]

A step is one pass of the whole hot path over one batch of the
Mamba-1.4B-shaped layer workload (batch 4, d_inner 4096, N 16, L 4096, bf16
inputs, fp32 state and arithmetic): the forward scan over the full sequences
(load, step size, discretisation, scan, gated read-out, final state) followed
by one decode token for the same channels, continuing from the final state.
Inputs are synthetic and seeded (selective_state_space_mss_b200.inputs).

`value` is whole-job channel-tokens per second with inputs resident in HBM.
With N > 1 (torchrun, one process per GPU, NCCL) every rank runs its own
replica of the workload -- the channels are independent, so the path shards
with no data-path collective -- and the time is the max over ranks.

`--impl reference` times the fp64 CPU oracle on a bounded sample of the same
workload (rank 0 only) and prints the same line with "impl": "reference".
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from selective_state_space_mss_b200 import inputs as gen  # noqa: E402

METRIC = "selective-scan fwd: achieved HBM GB/s (% of B200 peak) and channel-tokens/s"
UNIT = "channel-tokens/s"
WORKLOAD = gen.BENCH_WORKLOAD
FALLBACK_HBM_GBS = 6650.0
# the files the timed forward kernel (and its launch) is built from: the
# recorded DRAM traffic is reported only while they are unchanged
KERNEL_SOURCES = ["selective_state_space_mss_b200/csrc/" + f for f in (
    "scan_seq.cuh", "scan_seq4.cuh", "tma.cuh", "mss_device.cuh", "mss_params.h", "host_common.h", "forward.cuh",
    "fwd_bf16_n16.cu")]


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# ---------------------------------------------------------------------------
# Algorithmic bytes: every element read or written once.

def fwd_bytes(batch, dim, N, L, esz=2, z=True):
    seq = batch * dim * L * esz
    return (seq * (3 if z else 2)            # u, delta, z read
            + seq                             # y written
            + 2 * batch * N * L * esz         # B, C read once per (batch, token)
            + dim * N * 4 + 2 * dim * 4       # A, D, bias
            + batch * dim * N * 4)            # last_state written


def decode_bytes(batch, dim, N, esz=2, z=True):
    return (2 * batch * dim * N * 4           # state read + written
            + batch * dim * esz * (4 if z else 3)  # u, delta, z read, y written
            + 2 * batch * N * esz + dim * N * 4 + 2 * dim * 4)


def fwd_alu_ops(batch, dim, N, L):
    """Algorithmic fp32 lane operations of one forward launch: per token and
    state the definition's four (transition via the S4D-Real identity, input
    term, update, read-out), per token ten more (bias add, softplus, Delta*u,
    Delta*A_0, skip, read-out sum, gate)."""
    return batch * dim * L * (4 * N + 10)


def bwd_alu_ops(batch, dim, N, L, checkpoint_pass=True):
    """Algorithmic fp32 lane operations of one backward call (Euler rule): per
    token and state, three to form the state again (transition, input term,
    update) and nine for the reverse step (g = gh + dr C, gh' = g Abar,
    q = gh' h_prev, dA += Delta q, the sums of q A and g B, the dB and dC terms,
    the read-out C h for dz); three more per token and state when the call
    also runs its checkpoint pass (the forward fold); per token twenty (the
    step, its slope, the gate and its slope, the per-token gradients)."""
    return batch * dim * L * ((15 if checkpoint_pass else 12) * N + 20)


# B200: 148 SMs x 128 fp32 lanes per SM and clock, at the maximum SM clock.
SMS, FP32_LANES_PER_SM = 148, 128


def alu_peak_ops(sm_max_mhz):
    return SMS * FP32_LANES_PER_SM * sm_max_mhz * 1e6


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured", float(d.get("sm_max_mhz", 1965.0))
    except Exception:
        return FALLBACK_HBM_GBS, "fallback", 1965.0


def measured_bf16_tflops():
    """The pool's measured dense bf16 GEMM rate (burst), TFLOP/s, or the
    fallback figure."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


def kernel_source_hash():
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(os.path.basename(rel).encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def recorded_traffic():
    """DRAM bytes per launch of the forward kernel from the committed ncu
    summary, if it was taken on the kernel as it is now; else None."""
    p = os.path.join(ROOT, "profiles", "scan_fwd_dram_traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        if d.get("kernel_source_sha") == kernel_source_hash() and d.get("workload") == WORKLOAD:
            return float(d["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


# ---------------------------------------------------------------------------
# Clocks during the timed region (nvidia-smi sampled every 200 ms).

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
        return False

    def summary(self):
        rows = []
        for line in (self.out or "").splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), max=float(parts[2]), power=float(parts[3]),
                                 hw=parts[5], hw_thermal=parts[6], sw_thermal=parts[7],
                                 power_cap=parts[8]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        reasons = []
        for key, name in [("hw", "hw_slowdown"), ("hw_thermal", "hw_thermal_slowdown"),
                          ("sw_thermal", "sw_thermal_slowdown"), ("power_cap", "sw_power_cap")]:
            if any(r[key].lower().startswith("active") for r in rows):
                reasons.append(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in rows),
                "sm_max_mhz": max(r["max"] for r in rows),
                "power_w_max": max(r["power"] for r in rows),
                "reasons": reasons, "samples": len(rows)}


def nvml_device_id(dev, local_rank):
    """The CUDA device's UUID in NVML's form ("GPU-..."), so that NVML reads
    the same physical GPU whatever the enumeration order; else its index."""
    try:
        import torch

        u = str(torch.cuda.get_device_properties(dev).uuid)
        if u:
            return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        pass
    return physical_gpu_index(local_rank)


class NvmlSampler:
    """SM clock, power and clock-event reasons read through NVML every ~2 ms
    by a host thread while the timed region runs (the host waits in
    synchronize while the GPU works, so the samples fall under load).  Only
    reads; any NVML failure leaves it with no samples."""

    REASONS = (("sw_power_cap", 0x4), ("hw_slowdown", 0x8), ("sw_thermal_slowdown", 0x20),
               ("hw_thermal_slowdown", 0x40))

    def __init__(self, gpu_index, period_s=0.002):
        self.gpu = str(gpu_index)
        self.period = period_s
        self.rows = []
        self.max_mhz = None
        self._thread = None
        self._nvml = None
        self._t0 = self._t1 = None
        self._first = 0
        self.stopped_early = False

    def mark(self):
        """Start of the window the summary covers (the samples before it, taken
        while the sampler started up and the warm-up ran, are left out)."""
        self._first = len(self.rows)
        self._t0 = time.perf_counter()

    def __enter__(self):
        import threading

        try:
            import pynvml

            pynvml.nvmlInit()
            self._nvml = pynvml
            h = (pynvml.nvmlDeviceGetHandleByUUID(self.gpu) if self.gpu.startswith("GPU-")
                 else pynvml.nvmlDeviceGetHandleByIndex(int(self.gpu)))
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            reasons = (getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None)
                       or pynvml.nvmlDeviceGetCurrentClocksThrottleReasons)
        except Exception:
            return self
        self._stop = threading.Event()

        def run():
            while not self._stop.is_set():
                try:
                    self.rows.append((float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)),
                                      int(reasons(h)), pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0))
                except Exception:
                    self.stopped_early = True
                    return
                time.sleep(self.period)

        self._t0 = time.perf_counter()
        self._thread = threading.Thread(target=run, daemon=True)
        self._thread.start()
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=5)
            self._t1 = time.perf_counter()
        if self._nvml is not None:
            try:
                self._nvml.nvmlShutdown()
            except Exception:
                pass
            self._nvml = None
        return False

    def summary(self):
        rows = self.rows[self._first:]
        if not rows:
            return None
        mask = 0
        for _, r, _ in rows:
            mask |= r
        # samples one thread can take in the window (each read also takes time,
        # so the count comes in below this); far fewer means it stopped early
        expected = None if self._t1 is None else int((self._t1 - self._t0) / self.period)
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": self.max_mhz,
                "power_w_max": max(r[2] for r in rows),
                "reasons": [name for name, bit in self.REASONS if mask & bit], "samples": len(rows),
                "samples_at_most": expected, "sampler_stopped_early": self.stopped_early,
                "source": "NVML every 2 ms during the timed region"}


# ---------------------------------------------------------------------------
# Multi-rank plumbing: every rank runs its own replica of the workload (the
# channels are independent, so there is no data-path collective); the only
# collectives are barriers and the max-over-ranks of the measured time.

def rank_seed(base_seed, rank):
    """Seed of rank `rank`'s replica (distinct inputs per rank)."""
    return base_seed + 100 * rank


def max_over_ranks(ms, world, device):
    """The slowest rank's time (collective: every rank must call it)."""
    if world <= 1:
        return float(ms)
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank, world, steps, ms_max):
    """Units of all ranks per second over the slowest rank's time."""
    return world * units_per_rank * steps / (ms_max * 1e-3)


def physical_gpu_index(local_rank):
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if local_rank < len(ids):
            return ids[local_rank]
    return str(local_rank)


# ---------------------------------------------------------------------------
# The CPU oracle, timed (cpu_baseline and the reference arm).

def oracle_sample_rate(inp, rows, nthreads):
    """Run the oracle on the first `rows` channels of every batch row;
    returns (channel-tokens, seconds)."""
    import oracle

    L = inp["seqlen"]
    t0 = time.perf_counter()
    oracle.scan_fwd(inp["u"].values[:, :rows], inp["delta"].values[:, :rows], inp["A"][:rows],
                    inp["B"].values, inp["C"].values, D=inp["D"][:rows],
                    z=inp["z"].values[:, :rows], delta_bias=inp["delta_bias"][:rows],
                    nthreads=nthreads)
    return inp["batch"] * rows * L, time.perf_counter() - t0


def calibrate_rows(inp, nthreads, target_s):
    """Channels per batch row for one oracle pass of about target_s seconds
    (at most the whole workload)."""
    rows = min(inp["dim"], max(nthreads, 16))
    _, sec = oracle_sample_rate(inp, rows, nthreads)
    per_row = sec / rows
    return int(min(inp["dim"], max(nthreads, target_s / max(per_row, 1e-9))))


def cpu_model():
    """The host CPU's model name (Linux), for the baseline's record."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(inp, target_s=10.0):
    """The oracle on the host cores over the same workload, repeated until
    about target_s seconds of work."""
    import oracle

    nthreads = oracle.default_threads()
    rows = calibrate_rows(inp, nthreads, target_s)
    total_ct, total_s, passes = 0, 0.0, 0
    while total_s < target_s or passes == 0:
        ct, sec = oracle_sample_rate(inp, rows, nthreads)
        total_ct, total_s, passes = total_ct + ct, total_s + sec, passes + 1
    # the same oracle on one thread, over a few channels per batch row (about 2 s)
    rows1 = max(1, min(inp["dim"], calibrate_rows(inp, 1, 1.0) // 2))
    ct1, s1, passes1 = 0, 0.0, 0
    while s1 < 2.0 or passes1 == 0:
        ct, sec = oracle_sample_rate(inp, rows1, 1)
        ct1, s1, passes1 = ct1 + ct, s1 + sec, passes1 + 1
    return {"value": total_ct / total_s, "unit": UNIT, "cores": nthreads, "kind": "oracle", "cpu": cpu_model(),
            "sample": f"{passes} pass(es) of {inp['batch']}x{rows} channels x {inp['seqlen']} tokens "
                      f"of {WORKLOAD} (fp64, {nthreads} threads, {total_s:.1f} s)",
            "single_thread": {"value": ct1 / s1, "unit": UNIT,
                              "sample": f"{passes1} pass(es) of {inp['batch']}x{rows1} channels x "
                                        f"{inp['seqlen']} tokens (fp64, 1 thread, {s1:.1f} s)"}}


def run_reference(args, rank):
    if rank != 0:
        return 0
    import oracle

    inp = gen.workload_inputs(WORKLOAD)
    nthreads = oracle.default_threads()
    # each step: one oracle pass over as much of the workload as fits ~8 s
    rows = calibrate_rows(inp, nthreads, target_s=min(8.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample_rate(inp, rows, nthreads)
    times = []
    for _ in range(args.steps):
        _, sec = oracle_sample_rate(inp, rows, nthreads)
        times.append(sec)
    total = sum(times)
    ct_step = inp["batch"] * rows * inp["seqlen"]
    value = ct_step * args.steps / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "sample_channels_per_batch_row": rows, "seqlen": inp["seqlen"]},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": nthreads, "kind": "oracle",
                         "sample": f"{inp['batch']}x{rows} channels x {inp['seqlen']} tokens per step, fp64"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# The CUDA path.

def kernel_only(args, mss, d, y, state, w, dev, to_dev, rank):
    """warmup + steps launches of one kernel on its workload, nothing timed
    and no JSON line: the command that profiler captures run."""
    import torch

    n = args.warmup + args.steps
    if args.kernel == "forward":
        for _ in range(n):
            mss.scan_fwd(**d, y=y, last_state=state)
        what = f"{w.batch}x{w.dim}x{w.dstate}x{w.seqlen}"
    elif args.kernel == "backward":
        dy_h, dlast_h = gen.upstream_gradients(w.batch, w.dim, w.dstate, w.seqlen, w.dtype, rank_seed(w.seed, rank))
        dy_d, dlast_d = to_dev(dy_h), torch.from_numpy(dlast_h).to(dev)
        ws = torch.empty(mss.bwd_workspace_size(w.batch, w.dim, w.dstate, w.seqlen), dtype=torch.uint8, device=dev)
        for _ in range(n):
            mss.scan_bwd(**d, dy=dy_d, dlast=dlast_d, workspace=ws)
        what = f"{w.batch}x{w.dim}x{w.dstate}x{w.seqlen}"
    elif args.kernel == "decode":
        dw = gen.WORKLOADS[gen.DECODE_WORKLOAD]
        A5, D5, b5 = (torch.from_numpy(x).to(dev) for x in gen.channel_params(dw.dim, dw.dstate, dw.d_skip, dw.seed))
        st5 = torch.zeros(dw.batch, dw.dim, dw.dstate, device=dev)
        steps5 = [{k: to_dev(v) for k, v in gen.decode_step_inputs(dw.batch, dw.dim, dw.dstate, dw.dtype,
                                                                  dw.seed, t).items()} for t in range(4)]
        y5 = torch.empty(dw.batch, dw.dim, dtype=torch.bfloat16, device=dev)
        for t in range(n):
            mss.state_update(st5, A=A5, D=D5, delta_bias=b5, y=y5, **steps5[t % 4])
        what = f"{dw.batch}x{dw.dim}x{dw.dstate}"
    else:
        ss = dict(gen.SSD_SHAPES[gen.SSD_WORKLOAD])
        if args.seqlen:
            ss["seqlen"] = args.seqlen
        sin = gen.ssd_inputs(**ss)
        sd = dict(x=to_dev(sin["x"]), dt=to_dev(sin["dt"]), A=torch.from_numpy(sin["A"]).to(dev),
                  B=to_dev(sin["B"]), C=to_dev(sin["C"]), D=torch.from_numpy(sin["D"]).to(dev),
                  z=to_dev(sin["z"]), dt_bias=torch.from_numpy(sin["dt_bias"]).to(dev))
        for _ in range(n):
            mss.ssd_fwd(**sd)
        what = "x".join(str(ss[k]) for k in ("batch", "seqlen", "nheads", "headdim", "dstate"))
    torch.cuda.synchronize(dev)
    assert mss.get_device_error() == 0
    log(f"kernel-only: {n} {args.kernel} launches on {what}")
    return 0


def forward_record(w, ms_avg, ms_list, launches, segments=None, note=None):
    """Throughput of one forward workload: CUDA-event time per call, channel-
    tokens/s, algorithmic HBM GB/s and its fraction of the peak, and the
    fraction of the fp32 lane-operation peak."""
    peak, peak_kind, sm_max_mhz = measured_peaks()
    esz = 2 if w.dtype == "bf16" else 4
    nbytes = fwd_bytes(w.batch, w.dim, w.dstate, w.seqlen, esz=esz)
    ops = fwd_alu_ops(w.batch, w.dim, w.dstate, w.seqlen)
    ct = w.batch * w.dim * w.seqlen
    rec = {"batch": w.batch, "d_inner": w.dim, "dstate": w.dstate, "seqlen": w.seqlen, "io_dtype": w.dtype,
           "ms_avg": ms_avg, "ms_p10_p50_p90": [float(np.percentile(ms_list, q)) for q in (10, 50, 90)],
           "launches_per_call": launches,
           "channel_tokens_per_s": ct / (ms_avg * 1e-3),
           "algorithmic_bytes": nbytes, "achieved_gbs": nbytes / (ms_avg * 1e-3) / 1e9,
           "hbm_frac": nbytes / (ms_avg * 1e-3) / 1e9 / peak, "hbm_peak_kind": peak_kind,
           "alu_frac": ops / (ms_avg * 1e-3) / alu_peak_ops(sm_max_mhz)}
    if segments is not None:
        rec["sequence_segments"] = segments
    if note:
        rec["note"] = note
    return rec


def time_workload(mss, name, args, dev, stream, rank):
    """One forward workload timed alone: warm-up, then `steps` calls with CUDA
    events around each (the call's launches: the fold pass and the full pass
    where the sequence is split)."""
    import torch

    w = gen.WORKLOADS[name]
    inp = gen.scan_inputs(w.batch, w.dim, w.dstate, w.seqlen, w.dtype, rank_seed(w.seed, rank), w.d_skip)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32

    def to_dev(t):
        if w.dtype == "f32":
            return torch.from_numpy(np.ascontiguousarray(t.stored)).to(dev)
        return torch.from_numpy(np.ascontiguousarray(t.stored).view(np.int16)).view(torch.bfloat16).to(dev)

    d = dict(u=to_dev(inp["u"]), delta=to_dev(inp["delta"]), z=to_dev(inp["z"]), B=to_dev(inp["B"]),
             C=to_dev(inp["C"]), A=torch.from_numpy(inp["A"]).to(dev), D=torch.from_numpy(inp["D"]).to(dev),
             delta_bias=torch.from_numpy(inp["delta_bias"]).to(dev))
    del inp
    y = torch.empty_like(d["u"])
    last = torch.empty(w.batch, w.dim, w.dstate, dtype=torch.float32, device=dev)
    nbytes = mss.workspace_size(w.batch, w.dim, w.dstate, w.seqlen, tdt, device=dev)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev) if nbytes > 0 else None
    evs = []
    for i in range(args.warmup + args.steps):
        a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a_.record(stream)
        mss.scan_fwd(**d, y=y, last_state=last, workspace=ws)
        b_.record(stream)
        if i >= args.warmup:
            evs.append((a_, b_))
    torch.cuda.synchronize(dev)
    ms_list = [a_.elapsed_time(b_) for a_, b_ in evs]
    segs = None
    if nbytes > 0:
        # the split's aggregates take (segments - 1) * 2 * rows * N fp32 values
        segs = 1 + nbytes // (2 * w.batch * w.dim * w.dstate * 4)
    note = "launch-bound parity workload; its throughput says little" if w.seqlen * w.dim * w.batch < 1e6 else None
    return forward_record(w, sum(ms_list) / len(ms_list), ms_list, launches=2 if segs else 1, segments=segs,
                          note=note)


def run_mss(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import selective_state_space_mss_b200 as mss
    from selective_state_space_mss_b200 import build as mss_build

    if not os.path.exists(mss.library_path()):
        mss_build.build()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)

    w = gen.WORKLOADS[WORKLOAD]
    if args.seqlen:
        import dataclasses

        w = dataclasses.replace(w, seqlen=args.seqlen)
    inp = gen.scan_inputs(w.batch, w.dim, w.dstate, w.seqlen, w.dtype, rank_seed(w.seed, rank), w.d_skip)
    nxt = gen.decode_step_inputs(w.batch, w.dim, w.dstate, w.dtype, rank_seed(w.seed, rank), 0)

    def to_dev(t):
        return torch.from_numpy(np.ascontiguousarray(t.stored).view(np.int16)).view(torch.bfloat16).to(dev)

    d = dict(u=to_dev(inp["u"]), delta=to_dev(inp["delta"]), z=to_dev(inp["z"]),
             B=to_dev(inp["B"]), C=to_dev(inp["C"]), A=torch.from_numpy(inp["A"]).to(dev),
             D=torch.from_numpy(inp["D"]).to(dev), delta_bias=torch.from_numpy(inp["delta_bias"]).to(dev))
    s1 = {k: to_dev(nxt[k]) for k in ("u", "delta", "z", "B", "C")}
    y = torch.empty_like(d["u"])
    state = torch.empty(w.batch, w.dim, w.dstate, dtype=torch.float32, device=dev)
    y1 = torch.empty_like(s1["u"])

    def step(flags=0, ev=None):
        if ev is not None:
            ev[0].record(stream)
        mss.scan_fwd(**d, y=y, last_state=state, flags=flags)
        if ev is not None:
            ev[1].record(stream)
        mss.state_update(state, A=d["A"], D=d["D"], delta_bias=d["delta_bias"], y=y1,
                         flags=flags & mss.FLAG_ZOH_INPUT, **s1)

    launches_per_step = 2
    ct_per_step = w.batch * w.dim * w.seqlen + w.batch * w.dim
    bytes_fwd = fwd_bytes(w.batch, w.dim, w.dstate, w.seqlen)
    bytes_step = bytes_fwd + decode_bytes(w.batch, w.dim, w.dstate)

    def timed(flags, k, warm, with_clocks=False):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(k)]
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        sampler = ClockSampler(physical_gpu_index(local_rank))
        nvml = NvmlSampler(nvml_device_id(dev, local_rank))
        if with_clocks:
            # the samplers start (and nvidia-smi gets its first reading) before
            # the warm-up, so that the GPU does not idle between the warm-up
            # and the timed steps
            sampler.__enter__()
            nvml.__enter__()
            time.sleep(0.3)
        for _ in range(warm):
            step(flags)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        if with_clocks:
            nvml.mark()
        start.record(stream)
        for i in range(k):
            step(flags, evs[i])
        end.record(stream)
        torch.cuda.synchronize(dev)
        if with_clocks:
            nvml.__exit__(None, None, None)
            sampler.__exit__(None, None, None)
        if world > 1:
            dist.barrier()
        ms = max_over_ranks(start.elapsed_time(end), world, dev)
        fwd_ms = [a.elapsed_time(b) for a, b in evs]
        clocks = None
        if with_clocks:
            clocks = nvml.summary()
            smi = sampler.summary()
            if clocks is None:
                clocks = smi
            else:
                clocks["nvidia_smi"] = smi
        return ms, fwd_ms, clocks

    assert mss.get_device_error() == 0
    if args.kernel_only:
        return kernel_only(args, mss, d, y, state, w, dev, to_dev, rank)
    ms, fwd_ms, clocks = timed(0, args.steps, args.warmup, with_clocks=True)
    assert mss.get_device_error() == 0

    # the same step in a loop of at least 1.5 s with the clocks sampled
    # throughout, so that the clock record of the step is long enough to read
    reps = max(args.steps, int(math.ceil(1.5 / max(ms / args.steps * 1e-3, 1e-6))))
    ms_loop, _, clocks_loop = timed(0, reps, args.warmup, with_clocks=True)
    loop_step_ms = ms_loop / reps
    clock_loop = {"steps": reps, "seconds": ms_loop * 1e-3, "ms_per_step": loop_step_ms,
                  "clocks": clocks_loop,
                  "ms_x_median_sm_mhz": (loop_step_ms * clocks_loop["sm_mhz"]
                                         if clocks_loop and clocks_loop.get("sm_mhz") else None)}
    assert mss.get_device_error() == 0
    ms_gen, fwd_ms_gen, _ = timed(mss.FLAG_GENERAL_A, args.steps, args.warmup)
    ms_zoh, fwd_ms_zoh, _ = timed(mss.FLAG_ZOH_INPUT, args.steps, args.warmup)

    # the forward pass with the causal convolution (width 4) in front: u is
    # read as the convolution's input x
    cw, cb = (torch.from_numpy(v).to(dev) for v in gen.conv_params(w.dim, 4, rank_seed(w.seed, rank)))
    cs_in = torch.zeros(w.batch, w.dim, 3, dtype=torch.bfloat16, device=dev)
    cs_out = torch.empty_like(cs_in)
    conv_ms = []
    for i in range(args.warmup + args.steps):
        a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a_.record(stream)
        mss.scan_fwd_conv(d["u"], cw, d["delta"], d["A"], d["B"], d["C"], conv_b=cb, conv_state=cs_in,
                          D=d["D"], z=d["z"], delta_bias=d["delta_bias"], y=y, last_state=state,
                          conv_state_out=cs_out)
        b_.record(stream)
        if i >= args.warmup:
            conv_ms.append((a_, b_))
    torch.cuda.synchronize(dev)
    conv_ms = [a_.elapsed_time(b_) for a_, b_ in conv_ms]
    assert mss.get_device_error() == 0

    # the other forward workloads, each in the launch configuration the
    # library picks (sequence split with its workspace where it applies)
    workloads = {WORKLOAD: forward_record(w, sum(fwd_ms) / len(fwd_ms), fwd_ms, launches=1)}
    for name in ("mamba130m-layer-bf16-b8-d1536-n16-l2048", "long-seq-bf16-b1-d2048-n16-l131072",
                 "s6-fwd-fp32-b1-d16-n4-l256"):
        workloads[name] = time_workload(mss, name, args, dev, stream, rank)
        assert mss.get_device_error() == 0

    # the structured-state-space-duality (Mamba-2) layer: its own workloads,
    # each on the tcgen05 kernel and, for comparison, the warp-level one
    def time_ssd(name):
        ss = gen.SSD_SHAPES[name]
        sin = gen.ssd_inputs(**ss)
        sd = dict(x=to_dev(sin["x"]), dt=to_dev(sin["dt"]), A=torch.from_numpy(sin["A"]).to(dev),
                  B=to_dev(sin["B"]), C=to_dev(sin["C"]), D=torch.from_numpy(sin["D"]).to(dev),
                  z=to_dev(sin["z"]), dt_bias=torch.from_numpy(sin["dt_bias"]).to(dev))
        ssd_y = torch.empty_like(sd["x"])
        ssd_last = torch.empty(ss["batch"], ss["nheads"], ss["dstate"], ss["headdim"], device=dev)

        def one(flags):
            ev = []
            for i in range(args.warmup + args.steps):
                a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a_.record(stream)
                mss.ssd_fwd(**sd, y=ssd_y, last_state=ssd_last, flags=flags)
                b_.record(stream)
                if i >= args.warmup:
                    ev.append((a_, b_))
            torch.cuda.synchronize(dev)
            assert mss.get_device_error() == 0
            return sum(a_.elapsed_time(b_) for a_, b_ in ev) / len(ev)

        ms_tc = one(0)  # the tcgen05 kernel
        ms_warp = one(mss.SSD_FLAG_WARP_MMA)  # the warp-level (mma.sync) kernel
        # algorithmic bytes: x, z read and y written (bf16), dt read, B and C
        # read once per (batch, token, group), A, D, dt_bias, and last_state
        # written; matrix-form flops per (token, head) of chunks of 128
        # tokens: C B^T and M X within the chunk, C S and the state product
        # B^T X across chunks
        nbytes = (3 * ss["batch"] * ss["seqlen"] * ss["nheads"] * ss["headdim"] * 2
                  + ss["batch"] * ss["seqlen"] * ss["nheads"] * 2
                  + 2 * ss["batch"] * ss["seqlen"] * ss["ngroups"] * ss["dstate"] * 2
                  + 3 * ss["nheads"] * 4 + ss["batch"] * ss["nheads"] * ss["dstate"] * ss["headdim"] * 4)
        flops = ss["batch"] * ss["seqlen"] * ss["nheads"] * (
            2 * 128 * ss["dstate"] + 2 * 128 * ss["headdim"] + 2 * ss["dstate"] * ss["headdim"] * 2)
        return ss, ms_tc, ms_warp, nbytes, flops

    ss, ssd_ms, ssd_ms_warp, ssd_bytes, ssd_flops = time_ssd(gen.SSD_WORKLOAD)
    ss2, ssd2_ms, ssd2_ms_warp, ssd2_bytes, ssd2_flops = time_ssd(gen.SSD_WORKLOAD_2)

    # the backward pass (gradients of every input, states recomputed from
    # checkpoints) on the same workload
    dy_h, dlast_h = gen.upstream_gradients(w.batch, w.dim, w.dstate, w.seqlen, w.dtype, rank_seed(w.seed, rank))
    dy_d, dlast_d = to_dev(dy_h), torch.from_numpy(dlast_h).to(dev)
    ws_b = torch.empty(mss.bwd_workspace_size(w.batch, w.dim, w.dstate, w.seqlen), dtype=torch.uint8, device=dev)
    bwd_ev = []
    for i in range(args.warmup + args.steps):
        a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a_.record(stream)
        mss.scan_bwd(**d, dy=dy_d, dlast=dlast_d, workspace=ws_b)
        b_.record(stream)
        if i >= args.warmup:
            bwd_ev.append((a_, b_))
    torch.cuda.synchronize(dev)
    bwd_ms = [a_.elapsed_time(b_) for a_, b_ in bwd_ev]

    # a training step: the forward pass that stores the states, then the
    # backward pass from them (no checkpoint pass)
    y_t = torch.empty_like(y)
    st_t = torch.empty_like(state)
    tr_ev = []
    for i in range(args.warmup + args.steps):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        e[0].record(stream)
        mss.scan_fwd_save(**d, y=y_t, last_state=st_t, states=ws_b)
        e[1].record(stream)
        mss.scan_bwd(**d, dy=dy_d, dlast=dlast_d, saved_states=ws_b)
        e[2].record(stream)
        if i >= args.warmup:
            tr_ev.append(e)
    torch.cuda.synchronize(dev)
    fwd_save_ms = [e[0].elapsed_time(e[1]) for e in tr_ev]
    bwd_saved_ms = [e[1].elapsed_time(e[2]) for e in tr_ev]
    assert mss.get_device_error() == 0
    assert mss.get_device_error() == 0

    # end to end through the public calls with host buffers, every step: the
    # forward pass over pinned host inputs and outputs (mss_scan_fwd_host:
    # the library copies pieces in, runs them and copies y and last_state out,
    # overlapping the two directions), then the decode token from that state
    # (state and token inputs copied in, y and the new state copied out)
    host = {k: v.cpu().pin_memory() for k, v in d.items()}
    host1 = {k: v.cpu().pin_memory() for k, v in s1.items()}
    y_host = torch.empty(y.shape, dtype=y.dtype, pin_memory=True)
    st_host = torch.empty(state.shape, dtype=state.dtype, pin_memory=True)
    st1_host = torch.empty(state.shape, dtype=state.dtype, pin_memory=True)
    y1_host = torch.empty(y1.shape, dtype=y1.dtype, pin_memory=True)
    ws_host = torch.empty(int(mss.load_library().mss_scan_fwd_host_workspace_size(
        w.batch, w.dim, w.dstate, w.seqlen, mss.DTYPE_BF16, 1, 1, 1, 0, 1)), dtype=torch.uint8, device=dev)
    h2d = (sum(v.numel() * v.element_size() for v in list(host.values()) + list(host1.values()))
           + st_host.numel() * 4)
    d2h = y_host.numel() * 2 + st_host.numel() * 4 + y1_host.numel() * 2 + st1_host.numel() * 4

    def e2e_step():
        mss.scan_fwd_host(**host, y=y_host, last_state=st_host, workspace=ws_host, device=dev)
        state.copy_(st_host, non_blocking=True)
        for k_, v in host1.items():
            s1[k_].copy_(v, non_blocking=True)
        mss.state_update(state, A=d["A"], D=d["D"], delta_bias=d["delta_bias"], y=y1, **s1)
        y1_host.copy_(y1, non_blocking=True)
        st1_host.copy_(state, non_blocking=True)

    for _ in range(max(1, args.warmup)):
        e2e_step()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    assert mss.get_device_error() == 0

    # decode workload (256 x 5120 x 16 state): per-token time with L2 flushed
    # before every timed token, since the 84 MB state would otherwise stay in L2
    dw = gen.WORKLOADS[gen.DECODE_WORKLOAD]
    A5, D5, b5 = (torch.from_numpy(x).to(dev) for x in gen.channel_params(dw.dim, dw.dstate, dw.d_skip, dw.seed))
    st5 = torch.zeros(dw.batch, dw.dim, dw.dstate, device=dev)
    steps5 = [{k: to_dev(v) for k, v in gen.decode_step_inputs(dw.batch, dw.dim, dw.dstate, dw.dtype,
                                                              dw.seed, t).items()} for t in range(4)]
    y5 = torch.empty(dw.batch, dw.dim, dtype=torch.bfloat16, device=dev)
    # L2 flush before each timed token: write a 512 MB buffer (more than L2),
    # then read another 256 MB one, so that the flush's own dirty lines are
    # written back before the token starts rather than during it
    flush = torch.empty(512 * 2 ** 20, dtype=torch.uint8, device=dev)
    clean = torch.ones(256 * 2 ** 20, dtype=torch.uint8, device=dev)
    dec_ms = []
    for t in range(args.warmup + 20):
        flush.fill_(t & 0xff)
        clean.sum(dtype=torch.int64)
        a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a_.record(stream)
        mss.state_update(st5, A=A5, D=D5, delta_bias=b5, y=y5, **steps5[t % 4])
        b_.record(stream)
        torch.cuda.synchronize(dev)
        if t >= args.warmup:
            dec_ms.append(a_.elapsed_time(b_))
    dec_med = statistics.median(dec_ms)
    dec_bytes = decode_bytes(dw.batch, dw.dim, dw.dstate)
    # the same tokens back to back from a CUDA graph (16 tokens per replay, no
    # flush: the state stays partly in L2 between tokens, as when serving)
    graph_tokens = 16
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        for t in range(graph_tokens):  # the first calls run outside the capture
            mss.state_update(st5, A=A5, D=D5, delta_bias=b5, y=y5, **steps5[t % 4])
    stream.wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        for t in range(graph_tokens):
            mss.state_update(st5, A=A5, D=D5, delta_bias=b5, y=y5, **steps5[t % 4])
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize(dev)
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g0.record(stream)
    for _ in range(10):
        graph.replay()
    g1.record(stream)
    torch.cuda.synchronize(dev)
    dec_graph_ms = g0.elapsed_time(g1) / (10 * graph_tokens)
    del graph
    assert mss.get_device_error() == 0

    peak, peak_kind, sm_max_mhz = measured_peaks()
    alu_ops = fwd_alu_ops(w.batch, w.dim, w.dstate, w.seqlen)
    alu_peak = alu_peak_ops(sm_max_mhz)
    fwd_avg = sum(fwd_ms) / len(fwd_ms)
    fwd_avg_gen = sum(fwd_ms_gen) / len(fwd_ms_gen)
    fwd_avg_zoh = sum(fwd_ms_zoh) / len(fwd_ms_zoh)
    fwd_avg_conv = sum(conv_ms) / len(conv_ms)
    bwd_avg = sum(bwd_ms) / len(bwd_ms)
    # backward traffic: u, delta read by the checkpoint pass; u, delta, z, dy
    # read and du, ddelta, dz written by the backward kernel (bf16); B, C read
    # by both passes, dB, dC written (fp32); checkpoints (one fp32 state per
    # 8-token group) written and read
    n_ck = (w.seqlen + 7) // 8
    bytes_bwd = (w.batch * w.dim * w.seqlen * 2 * (2 + 4 + 3) + 2 * w.batch * w.dstate * w.seqlen * (2 + 2 + 4)
                 + 2 * w.batch * w.dim * n_ck * w.dstate * 4)
    bytes_conv = bytes_fwd + 2 * w.batch * w.dim * 3 * 2 + w.dim * 5 * 4  # + conv states and taps
    achieved = bytes_fwd / (fwd_avg * 1e-3) / 1e9
    achieved_gen = bytes_fwd / (fwd_avg_gen * 1e-3) / 1e9
    value = whole_job_rate(ct_per_step, world, args.steps, ms)
    # what the fp32, multi-function and shuffle units deliver per SM and clock
    # (outside every timed region)
    pipe_rates = mss.probe_pipe_rates()
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic: seeded N(0,1) u/z/B/C, delta_raw 0.1*N(0,1), log-uniform steps "
                "[1e-3,1e-1], A=-(n+1), D~N(1,0.1); bf16 storage",
        "config": {"workload": WORKLOAD, "batch": w.batch, "d_inner": w.dim, "dstate": w.dstate,
                   "seqlen": w.seqlen, "io_dtype": "bf16",
                   "step": "forward scan over all tokens + one decode token (all hot-path rows)",
                   "l2": f"inputs larger than L2: {bytes_step / 1e6:.0f} MB of algorithmic traffic per step",
                   "parallelism": f"replicas x{world} (channels shard with no collective)"},
        "achieved_hbm_gbs": world * bytes_step * args.steps / (ms * 1e-3) / 1e9,
        "roofline": {"bound": "alu", "achieved": alu_ops / (fwd_avg * 1e-3) / 1e12,
                     "peak": alu_peak / 1e12, "unit": "Tops/s (fp32 lane ops)",
                     "frac": alu_ops / (fwd_avg * 1e-3) / alu_peak, "traffic": recorded_traffic(),
                     "kernel": "scan_fwd_seq (forward scan)",
                     "peak_kind": f"derived: {SMS} SMs x {FP32_LANES_PER_SM} fp32 lanes x {sm_max_mhz:.0f} MHz",
                     "probe_per_sm_per_clk": pipe_rates,
                     "peak_probe_ffma2": pipe_rates["ffma2"] * SMS * sm_max_mhz * 1e6 / 1e12,
                     "algorithmic_ops_per_launch": alu_ops, "algorithmic_bytes_per_launch": bytes_fwd,
                     "launch_ms_avg": fwd_avg,
                     "launch_ms_p10_p50_p90": [float(np.percentile(fwd_ms, q)) for q in (10, 50, 90)],
                     "state_updates_per_s": w.batch * w.dim * w.seqlen * w.dstate / (fwd_avg * 1e-3)},
        "roofline_hbm": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": recorded_traffic(),
                         "peak_kind": peak_kind, "algorithmic_bytes_per_launch": bytes_fwd},
        "general_A_path": {"fwd_ms_avg": fwd_avg_gen, "achieved_gbs": achieved_gen,
                           "frac": achieved_gen / peak,
                           "channel_tokens_per_s": w.batch * w.dim * w.seqlen / (fwd_avg_gen * 1e-3)},
        "conv_path": {"fwd_ms_avg": fwd_avg_conv, "conv_width": 4,
                      "achieved_gbs": bytes_conv / (fwd_avg_conv * 1e-3) / 1e9,
                      "frac": bytes_conv / (fwd_avg_conv * 1e-3) / 1e9 / peak,
                      "channel_tokens_per_s": w.batch * w.dim * w.seqlen / (fwd_avg_conv * 1e-3)},
        "backward": {"ms_avg": bwd_avg, "channel_tokens_per_s": w.batch * w.dim * w.seqlen / (bwd_avg * 1e-3),
                     "achieved_gbs": bytes_bwd / (bwd_avg * 1e-3) / 1e9,
                     "frac": bytes_bwd / (bwd_avg * 1e-3) / 1e9 / peak,
                     "alu_ops": bwd_alu_ops(w.batch, w.dim, w.dstate, w.seqlen),
                     "alu_frac": bwd_alu_ops(w.batch, w.dim, w.dstate, w.seqlen) / (bwd_avg * 1e-3) / alu_peak,
                     "note": "gradients of u, delta, A, B, C, D, z, bias, starting state; checkpoint pass included"},
        "training_step": {"fwd_save_ms_avg": sum(fwd_save_ms) / len(fwd_save_ms),
                          "bwd_saved_ms_avg": sum(bwd_saved_ms) / len(bwd_saved_ms),
                          "step_ms": sum(fwd_save_ms) / len(fwd_save_ms) + sum(bwd_saved_ms) / len(bwd_saved_ms),
                          "recompute_step_ms": fwd_avg + bwd_avg,
                          "bwd_saved_alu_frac": bwd_alu_ops(w.batch, w.dim, w.dstate, w.seqlen, False)
                          / (sum(bwd_saved_ms) / len(bwd_saved_ms) * 1e-3) / alu_peak,
                          "states_bytes": int(ws_b.numel()),
                          "note": "mss_scan_fwd_save (the forward pass also storing the state at every 8-token "
                                  "group) then mss_scan_bwd with MSS_FLAG_SAVED_STATES; recompute_step_ms: "
                                  "mss_scan_fwd_ex2 then mss_scan_bwd with its checkpoint pass"},
        "ssd_path": {"workload": gen.SSD_WORKLOAD, "ms_avg": ssd_ms,
                     "channel_tokens_per_s": ss["batch"] * ss["seqlen"] * ss["nheads"] * ss["headdim"] / (ssd_ms * 1e-3),
                     # the binding roof at the measured peaks: HBM (its bytes take longer
                     # than its matrix-form flops at the bf16 GEMM rate)
                     "roofline": {"bound": "hbm", "achieved": ssd_bytes / (ssd_ms * 1e-3) / 1e9, "peak": peak,
                                  "unit": "GB/s", "frac": ssd_bytes / (ssd_ms * 1e-3) / 1e9 / peak,
                                  "peak_kind": peak_kind, "algorithmic_bytes_per_launch": ssd_bytes,
                                  "time_at_peak_us": 1e6 * ssd_bytes / (peak * 1e9)},
                     "roofline_tensor": {"bound": "tensor", "achieved": ssd_flops / (ssd_ms * 1e-3) / 1e12,
                                         "peak": measured_bf16_tflops()[0], "unit": "TFLOP/s",
                                         "frac": ssd_flops / (ssd_ms * 1e-3) / 1e12 / measured_bf16_tflops()[0],
                                         "peak_kind": measured_bf16_tflops()[1],
                                         "time_at_peak_us": ssd_flops / (measured_bf16_tflops()[0] * 1e6),
                                         "note": "tcgen05.mma bf16 products, fp32 accumulators in TMEM, "
                                                 "chunks of 128 tokens"},
                     "warp_mma_kernel": {"ms_avg": ssd_ms_warp,
                                         "achieved_gbs": ssd_bytes / (ssd_ms_warp * 1e-3) / 1e9,
                                         "note": "the warp-level mma.sync kernel (chunks of 64), "
                                                 "MSS_SSD_FLAG_WARP_MMA"},
                     "second_workload": {
                         "workload": gen.SSD_WORKLOAD_2, "ms_avg": ssd2_ms, "warp_mma_ms_avg": ssd2_ms_warp,
                         "channel_tokens_per_s": ss2["batch"] * ss2["seqlen"] * ss2["nheads"] * ss2["headdim"]
                         / (ssd2_ms * 1e-3),
                         "hbm_frac": ssd2_bytes / (ssd2_ms * 1e-3) / 1e9 / peak,
                         "tensor_frac": ssd2_flops / (ssd2_ms * 1e-3) / 1e12 / measured_bf16_tflops()[0],
                         "algorithmic_bytes_per_launch": ssd2_bytes,
                         "note": "160 (batch, head) pairs: a wave of 148 on the tcgen05 kernel, the 12 past it "
                                 "on the chunk-parallel passes (the library's workspace)"}},
        "zoh_input_path": {"fwd_ms_avg": fwd_avg_zoh,
                           "achieved_gbs": bytes_fwd / (fwd_avg_zoh * 1e-3) / 1e9,
                           "frac": bytes_fwd / (fwd_avg_zoh * 1e-3) / 1e9 / peak,
                           "channel_tokens_per_s": w.batch * w.dim * w.seqlen / (fwd_avg_zoh * 1e-3)},
        "decode": {"workload": gen.DECODE_WORKLOAD, "ms_per_token_median": dec_med,
                   "achieved_gbs": dec_bytes / (dec_med * 1e-3) / 1e9,
                   "frac": dec_bytes / (dec_med * 1e-3) / 1e9 / peak,
                   "l2": "flushed before each token (512 MB written, then 256 MB of another buffer read)",
                   "graph_ms_per_token": dec_graph_ms,
                   "graph_note": f"{graph_tokens} tokens per CUDA graph replay, back to back, no flush"},
        "e2e": {"value": whole_job_rate(ct_per_step, world, args.steps, e2e_ms), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "clock_loop": clock_loop,
        "workloads": workloads,
        "kernel_source_sha": kernel_source_hash(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(inp)
    elif rank == 0:
        line["cpu_baseline"] = None
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def pipe_rates_only(args):
    """Print one JSON line: the pipe rates (operations per SM and clock) of
    `args.steps` calls of mss_probe_pipe_rates, each key's median and range."""
    import torch

    import selective_state_space_mss_b200 as mss

    torch.cuda.set_device(0)
    runs = [mss.probe_pipe_rates() for _ in range(max(1, args.steps))]
    out = {}
    for k in mss.PIPE_RATE_NAMES:
        v = sorted(r[k] for r in runs)
        out[k] = {"median": v[len(v) // 2], "min": v[0], "max": v[-1]}
    print(json.dumps({"pipe_rates_per_sm_per_clk": out, "calls": len(runs),
                      "device": torch.cuda.get_device_name(0),
                      "sms": torch.cuda.get_device_properties(0).multi_processor_count}), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["mss", "reference"], default="mss")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kernel-only", action="store_true",
                    help="only launch one kernel (warmup + steps times); for profiler captures")
    ap.add_argument("--kernel", choices=["forward", "backward", "decode", "ssd"], default="forward",
                    help="which kernel --kernel-only launches")
    ap.add_argument("--pipe-rates", action="store_true",
                    help="only measure the fp32 fma, packed fma, ex2 and shuffle rates per SM and clock")
    ap.add_argument("--seqlen", type=int, default=0,
                    help="override the workload's sequence length (the SSD workload's with --kernel ssd)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank)
    if args.pipe_rates:
        return pipe_rates_only(args)

    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist

        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        return run_mss(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
