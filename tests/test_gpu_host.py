"""GPU tests of the forward pass over host buffers (mss_scan_fwd_host).

The call stages pieces of the channels through a device workspace and runs
the forward pass on each piece.  A piece may take the four-lane kernel where
the whole call takes the pair kernel (small grids of bf16 channels); the two
sum in the same order and agree bit for bit wherever they take the same
transition path, which these inputs' A rows (uniform within each group of 16
channels) guarantee.  So the outputs must equal, bit for bit, those of the
device call on the same inputs, and the oracle within the tolerances of
tests/helpers.py.  The cases cover all rows in one piece,
whole batch rows grouped into more pieces than workspace slots (slot
reuse), several pieces per batch row with a ragged last piece, the optional
inputs, an empty sequence, pageable host memory and chaining.
"""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_mss_b200 as mss
from selective_state_space_mss_b200 import inputs as gen

from tests.helpers import assert_close, device_inputs, to_numpy, to_torch

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)
CPU = torch.device("cpu")


def _host_inputs(inp, pin=True, with_z=True, with_D=True, with_bias=True):
    h = device_inputs(inp, CPU, with_z=with_z, with_D=with_D, with_bias=with_bias)
    if pin:
        h = {k: (v.pin_memory() if v is not None else None) for k, v in h.items()}
    return h


def _device_twin(h):
    return {k: (v.to(DEV) if v is not None else None) for k, v in h.items()}


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("batch", [1, 5])
def test_host_call_matches_oracle_and_device_call(dtype, batch):
    # L = 300: a ragged tail; the rows are small, so one piece holds them all
    inp = gen.scan_inputs(batch, 40, 16, 300, dtype, seed=800 + batch, d_skip="normal")
    h = _host_inputs(inp)
    h0 = torch.randn(batch, 40, 16, generator=torch.Generator().manual_seed(801)).pin_memory()
    y, last = mss.scan_fwd_host(**h, initial_state=h0)
    torch.cuda.synchronize()
    assert mss.get_device_error() == 0
    y_ref, last_ref = oracle.scan_fwd(inp["u"].values, inp["delta"].values, inp["A"], inp["B"].values,
                                      inp["C"].values, D=inp["D"], z=inp["z"].values,
                                      delta_bias=inp["delta_bias"], initial_state=h0.numpy().astype(np.float64))
    assert_close(to_numpy(y), y_ref, dtype, "y")
    assert_close(to_numpy(last), last_ref, dtype, "last_state")
    yd, lastd = mss.scan_fwd(**_device_twin(h), initial_state=h0.to(DEV), workspace=None,
                             flags=mss.FLAG_NO_SPLIT)
    torch.cuda.synchronize()
    assert torch.equal(y, yd.cpu()) and torch.equal(last, lastd.cpu())


def test_host_call_pieces_within_a_batch_row():
    """Rows of 4144 channels x 4096 bf16 tokens (about 100 MB of inputs) are
    cut in two pieces of 2080 and 2064 channels; batch 2 makes four pieces."""
    batch, dim, N, L = 2, 4144, 16, 4096
    inp = gen.scan_inputs(batch, dim, N, L, "bf16", seed=810, d_skip="normal")
    h = _host_inputs(inp)
    y, last = mss.scan_fwd_host(**h)
    yd, lastd = mss.scan_fwd(**_device_twin(h), workspace=None, flags=mss.FLAG_NO_SPLIT)
    torch.cuda.synchronize()
    assert mss.get_device_error() == 0
    assert torch.equal(y, yd.cpu()) and torch.equal(last, lastd.cpu())
    # and a sampled channel on each side of the piece boundary against the oracle
    for b, d in ((0, 2079), (1, 2080), (1, dim - 1)):
        y_ref, last_ref = oracle.scan_fwd(inp["u"].values[b:b + 1, d:d + 1], inp["delta"].values[b:b + 1, d:d + 1],
                                          inp["A"][d:d + 1], inp["B"].values[b:b + 1], inp["C"].values[b:b + 1],
                                          D=inp["D"][d:d + 1], z=inp["z"].values[b:b + 1, d:d + 1],
                                          delta_bias=inp["delta_bias"][d:d + 1])
        assert_close(to_numpy(y[b:b + 1, d:d + 1]), y_ref, "bf16", f"y of ({b}, {d})")
        assert_close(to_numpy(last[b:b + 1, d:d + 1]), last_ref, "bf16", f"state of ({b}, {d})")


def test_host_call_groups_whole_batch_rows():
    """Rows of 2048 channels x 2048 bf16 tokens (about 25 MB of inputs): two
    whole batch rows to a piece, nine rows in five pieces (the last one row),
    so the three workspace slots are reused."""
    batch, dim, N, L = 9, 2048, 16, 2048
    inp = gen.scan_inputs(batch, dim, N, L, "bf16", seed=815, d_skip="normal")
    h = _host_inputs(inp)
    y, last = mss.scan_fwd_host(**h)
    yd, lastd = mss.scan_fwd(**_device_twin(h), workspace=None, flags=mss.FLAG_NO_SPLIT)
    torch.cuda.synchronize()
    assert mss.get_device_error() == 0
    assert torch.equal(y, yd.cpu()) and torch.equal(last, lastd.cpu())
    for b, d in ((1, 0), (2, 2047), (8, 1000)):
        y_ref, last_ref = oracle.scan_fwd(inp["u"].values[b:b + 1, d:d + 1], inp["delta"].values[b:b + 1, d:d + 1],
                                          inp["A"][d:d + 1], inp["B"].values[b:b + 1], inp["C"].values[b:b + 1],
                                          D=inp["D"][d:d + 1], z=inp["z"].values[b:b + 1, d:d + 1],
                                          delta_bias=inp["delta_bias"][d:d + 1])
        assert_close(to_numpy(y[b:b + 1, d:d + 1]), y_ref, "bf16", f"y of ({b}, {d})")
        assert_close(to_numpy(last[b:b + 1, d:d + 1]), last_ref, "bf16", f"state of ({b}, {d})")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_host_call_without_optional_inputs_and_with_zoh(dtype):
    inp = gen.scan_inputs(4, 32, 8, 256, dtype, seed=820, d_skip="normal")
    h = _host_inputs(inp, with_z=False, with_D=False, with_bias=False)
    y, last = mss.scan_fwd_host(**h, want_last_state=False, flags=mss.FLAG_ZOH_INPUT)
    torch.cuda.synchronize()
    assert last is None
    y_ref, _ = oracle.scan_fwd(inp["u"].values, inp["delta"].values, inp["A"], inp["B"].values, inp["C"].values,
                               zoh_input=True)
    assert_close(to_numpy(y), y_ref, dtype, "y")


def test_host_call_pageable_memory_and_empty_sequence():
    inp = gen.scan_inputs(3, 24, 16, 128, "bf16", seed=830, d_skip="normal")
    h = _host_inputs(inp, pin=False)
    y, last = mss.scan_fwd_host(**h, y=torch.empty(3, 24, 128, dtype=torch.bfloat16),
                                last_state=torch.empty(3, 24, 16))
    yd, lastd = mss.scan_fwd(**_device_twin(h), workspace=None, flags=mss.FLAG_NO_SPLIT)
    torch.cuda.synchronize()
    assert torch.equal(y, yd.cpu()) and torch.equal(last, lastd.cpu())
    # no tokens: the final state is the starting state
    empty = {k: (v[..., :0].contiguous() if k in ("u", "delta", "z", "B", "C") else v) for k, v in h.items()}
    h0 = torch.randn(3, 24, 16)
    _, last0 = mss.scan_fwd_host(**empty, initial_state=h0)
    torch.cuda.synchronize()
    assert torch.equal(last0, h0)


def test_host_call_chains_with_the_next_call():
    """Work queued on the stream after the call sees its outputs: a second
    call reads the first one's last_state as its starting state."""
    inp = gen.scan_inputs(2, 32, 16, 512, "f32", seed=840, d_skip="normal")
    h = _host_inputs(inp)
    part = lambda t0, t1: {k: (v[..., t0:t1].contiguous().pin_memory() if k in ("u", "delta", "z", "B", "C") else v)
                           for k, v in h.items()}
    y_all, last_all = mss.scan_fwd_host(**h)
    y0, last0 = mss.scan_fwd_host(**part(0, 200))
    y1, last1 = mss.scan_fwd_host(**part(200, 512), initial_state=last0)
    torch.cuda.synchronize()
    assert_close(to_numpy(torch.cat([y0, y1], dim=2)), to_numpy(y_all).astype(np.float64), "f32", "chained y")
    assert_close(to_numpy(last1), to_numpy(last_all).astype(np.float64), "f32", "chained state")
