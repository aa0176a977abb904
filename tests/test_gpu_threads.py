"""Calls from several host threads at once.

include/mss.h promises that calls from several host threads are safe; the
library's only host state is created per device on first use (a driver
entry point, occupancy figures, the host-buffer call's streams).  A fresh
process computes the oracle's results first, then loads the library and
releases eight threads together, each making its first calls on its own
stream: the forward pass with its sequence split, the four-lane forward
kernel (bf16 and fp32), the host-buffer forward pass, a decode step, the
backward pass and the SSD layer.  Every thread's outputs must match the
oracle, and the device error word must stay clear.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r"""
import sys, threading
import numpy as np, torch
sys.path.insert(0, ".")
import oracle
import selective_state_space_mss_b200 as mss
from selective_state_space_mss_b200 import inputs as gen
from tests.helpers import assert_close, device_inputs, to_numpy, to_torch

dev = torch.device("cuda", 0)
torch.cuda.set_device(dev)
jobs = []


def fwd_job(seed, batch, dim, L, dtype, workspace):
    inp = gen.scan_inputs(batch, dim, 16, L, dtype, seed=seed, d_skip="normal")
    y_ref, s_ref = oracle.scan_fwd(inp["u"].values, inp["delta"].values, inp["A"], inp["B"].values,
                                   inp["C"].values, D=inp["D"], z=inp["z"].values, delta_bias=inp["delta_bias"])

    def run(stream):
        d = device_inputs(inp, dev)
        y, s = mss.scan_fwd(**d, workspace=workspace, stream=stream)
        stream.synchronize()
        assert_close(to_numpy(y), y_ref, dtype, f"forward {seed} y")
        assert_close(to_numpy(s), s_ref, dtype, f"forward {seed} last_state")
    return run


def host_job(seed):
    inp = gen.scan_inputs(2, 96, 16, 1024, "bf16", seed=seed, d_skip="normal")
    y_ref, s_ref = oracle.scan_fwd(inp["u"].values, inp["delta"].values, inp["A"], inp["B"].values,
                                   inp["C"].values, D=inp["D"], z=inp["z"].values, delta_bias=inp["delta_bias"])

    def run(stream):
        cpu = torch.device("cpu")
        h = {k: to_torch(inp[k], cpu).pin_memory() for k in ("u", "delta", "z", "B", "C")}
        y, s = mss.scan_fwd_host(A=torch.from_numpy(inp["A"]), D=torch.from_numpy(inp["D"]),
                                 delta_bias=torch.from_numpy(inp["delta_bias"]), device=dev, stream=stream, **h)
        stream.synchronize()
        assert_close(to_numpy(y), y_ref, "bf16", "host y")
        assert_close(to_numpy(s), s_ref, "bf16", "host last_state")
    return run


def decode_job(seed):
    batch, dim, N = 3, 256, 16
    A, D, bias = gen.channel_params(dim, N, "normal", seed)
    h0 = gen.initial_state(batch, dim, N, seed + 1, "normal")
    st = gen.decode_step_inputs(batch, dim, N, "bf16", seed + 2, 0)
    y_ref, s_ref = oracle.state_update(h0.astype(np.float64), st["u"].values, st["delta"].values, A, st["B"].values,
                                       st["C"].values, D=D, z=st["z"].values, delta_bias=bias)

    def run(stream):
        state = torch.from_numpy(h0.copy()).to(dev)
        y = mss.state_update(state, *(to_torch(st[k], dev) for k in ("u", "delta")), torch.from_numpy(A).to(dev),
                             to_torch(st["B"], dev), to_torch(st["C"], dev), D=torch.from_numpy(D).to(dev),
                             z=to_torch(st["z"], dev), delta_bias=torch.from_numpy(bias).to(dev), stream=stream)
        stream.synchronize()
        assert_close(to_numpy(y), y_ref, "bf16", "decode y")
        assert_close(to_numpy(state), s_ref, "bf16", "decode state")
    return run


def bwd_job(seed):
    inp = gen.scan_inputs(2, 32, 16, 512, "bf16", seed=seed, d_skip="normal")
    dy, dl = gen.upstream_gradients(2, 32, 16, 512, "bf16", seed + 1)
    ref = oracle.scan_bwd(inp["u"].values, inp["delta"].values, inp["A"], inp["B"].values, inp["C"].values,
                          dy.values, D=inp["D"], z=inp["z"].values, delta_bias=inp["delta_bias"],
                          dlast=dl.astype(np.float64))

    def run(stream):
        d = device_inputs(inp, dev)
        g = mss.scan_bwd(**d, dy=to_torch(dy, dev), dlast=torch.from_numpy(dl).to(dev), stream=stream)
        stream.synchronize()
        for k in ("du", "ddelta", "dz", "dA", "dB", "dC", "dD", "dbias"):
            assert_close(to_numpy(g[k]), ref[k], "bf16", f"backward {k}")
    return run


def ssd_job(seed):
    inp = gen.ssd_inputs(2, 256, 4, 64, 1, 128, seed=seed)
    y_ref, s_ref = oracle.ssd_fwd(inp["x"].values, inp["dt"].values, inp["A"], inp["B"].values, inp["C"].values,
                                  D=inp["D"], z=inp["z"].values, dt_bias=inp["dt_bias"])

    def run(stream):
        y, s = mss.ssd_fwd(to_torch(inp["x"], dev), to_torch(inp["dt"], dev), torch.from_numpy(inp["A"]).to(dev),
                           to_torch(inp["B"], dev), to_torch(inp["C"], dev), D=torch.from_numpy(inp["D"]).to(dev),
                           z=to_torch(inp["z"], dev), dt_bias=torch.from_numpy(inp["dt_bias"]).to(dev),
                           workspace=None, stream=stream)
        stream.synchronize()
        assert_close(to_numpy(y), y_ref, "bf16", "ssd y")
        assert_close(to_numpy(s), s_ref, "bf16", "ssd last_state")
    return run


jobs = [fwd_job(901, 2, 64, 1024, "bf16", "auto"), fwd_job(902, 1, 48, 2048, "bf16", "auto"),
        fwd_job(903, 2, 40, 1024, "bf16", None), fwd_job(904, 2, 40, 512, "f32", None),
        host_job(905), decode_job(906), bwd_job(907), ssd_job(908)]
gate = threading.Barrier(len(jobs))
errors = []


def worker(job):
    try:
        stream = torch.cuda.Stream(device=dev)
        gate.wait(timeout=60)
        with torch.cuda.stream(stream):
            for _ in range(3):
                job(stream)
    except BaseException as e:  # reported by the main thread
        errors.append(repr(e))


threads = [threading.Thread(target=worker, args=(j,)) for j in jobs]
for t in threads:
    t.start()
for t in threads:
    t.join(timeout=300)
assert not any(t.is_alive() for t in threads), "a thread did not finish"
assert not errors, errors
assert mss.get_device_error() == 0
print("threads ok")
"""


def test_first_calls_from_eight_threads():
    r = subprocess.run([sys.executable, "-c", SCRIPT], cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0 and "threads ok" in r.stdout, (r.stdout[-3000:], r.stderr[-3000:])
