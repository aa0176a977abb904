"""GPU parity of the single-token decode update, called through the C ABI.

The generation-time view of the same recurrence ("Exercises -- State-space
models (Mamba, S4)": one token at a time, constant-size state).  Checked
against the fp64 oracle step by step, against the forward pass, and on the
full decode workload (256 x 5120 x 16 state, 1024 tokens) with y compared on
every channel after every step.
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


def _step_dev(s):
    return {k: to_torch(s[k], DEV) for k in ("u", "delta", "z", "B", "C")}


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N", [1, 2, 4, 8, 16])
@pytest.mark.parametrize("init", ["zero", "normal"])
def test_decode_steps_match_oracle(N, dtype, init):
    batch, dim, steps = 3, 37, 40
    A, D, bias = gen.channel_params(dim, N, "normal", 77)
    h0 = gen.initial_state(batch, dim, N, 78, init)
    state = torch.from_numpy(h0.copy()).to(DEV)
    ref_state = h0.astype(np.float64)
    Ad, Dd, bd = (torch.from_numpy(x).to(DEV) for x in (A, D, bias))
    for t in range(steps):
        s = gen.decode_step_inputs(batch, dim, N, dtype, 79, t)
        y = mss.state_update(state, A=Ad, D=Dd, delta_bias=bd, **_step_dev(s))
        y_ref, ref_state = oracle.state_update(ref_state, s["u"].values, s["delta"].values, A,
                                               s["B"].values, s["C"].values, D=D, z=s["z"].values,
                                               delta_bias=bias)
        torch.cuda.synchronize()
        assert_close(to_numpy(y), y_ref, dtype, f"step {t} y")
    assert_close(to_numpy(state), ref_state, dtype, "final state")
    assert mss.get_device_error() == 0


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_decode_equals_forward_and_chains(dtype):
    """L decode steps reproduce the forward pass; forward(L0) + decode steps
    reproduce forward(L)."""
    batch, dim, N, L, L0 = 2, 64, 16, 96, 64
    inp = gen.scan_inputs(batch, dim, N, L, dtype, seed=81, d_skip="normal")
    d = device_inputs(inp, DEV)
    y_full, last_full = mss.scan_fwd(**d)
    pre = {k: (d[k][..., :L0].contiguous() if k in ("u", "delta", "z", "B", "C") else d[k]) for k in d}
    _, state = mss.scan_fwd(**pre)
    for t in range(L0, L):
        step = {k: d[k][..., t].contiguous() for k in ("u", "delta", "z", "B", "C")}
        y = mss.state_update(state, A=d["A"], D=d["D"], delta_bias=d["delta_bias"], **step)
        assert_close(to_numpy(y), to_numpy(y_full[..., t]).astype(np.float64), dtype, f"token {t}")
    assert_close(to_numpy(state), to_numpy(last_full).astype(np.float64), dtype, "state")
    state0 = torch.zeros(batch, dim, N, device=DEV)
    for t in range(L):
        step = {k: d[k][..., t].contiguous() for k in ("u", "delta", "z", "B", "C")}
        y = mss.state_update(state0, A=d["A"], D=d["D"], delta_bias=d["delta_bias"], **step)
        assert_close(to_numpy(y), to_numpy(y_full[..., t]).astype(np.float64), dtype, f"token {t}")


def test_decode_workload_every_step_all_channels():
    """The decode workload at full size (256 x 5120 x 16 state, 1024 tokens):
    the oracle advances the whole fp64 state alongside, and y and the state
    are compared over every channel after every token."""
    w = gen.WORKLOADS[gen.DECODE_WORKLOAD]
    batch, dim, N = w.batch, w.dim, w.dstate
    A, D, bias = gen.channel_params(dim, N, w.d_skip, w.seed)
    state = torch.zeros(batch, dim, N, device=DEV)
    Ad, Dd, bd = (torch.from_numpy(x).to(DEV) for x in (A, D, bias))
    ref_state = np.zeros((batch, dim, N))
    for t in range(w.decode_steps):
        s = gen.decode_step_inputs(batch, dim, N, w.dtype, w.seed, t)
        y = mss.state_update(state, A=Ad, D=Dd, delta_bias=bd, **_step_dev(s))
        y_ref, ref_state = oracle.state_update(ref_state, s["u"].values, s["delta"].values, A, s["B"].values,
                                               s["C"].values, D=D, z=s["z"].values, delta_bias=bias)
        assert_close(to_numpy(y), y_ref, w.dtype, f"step {t} y")
        if t in (0, w.decode_steps // 2 - 1, w.decode_steps - 1):
            assert_close(to_numpy(state), ref_state, w.dtype, f"step {t} state")
    assert mss.get_device_error() == 0


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N", [4, 8, 16])
@pytest.mark.parametrize("zoh", [False, True])
@pytest.mark.parametrize("gate", [True, False])
def test_decode_staged_path_matches_oracle(dtype, N, zoh, gate):
    """Shapes whose channel count is a whole number of 8 KB state tiles
    (2048/N channels) take the bulk-staged decode kernel; several batch rows
    per channel block, several channel blocks, and more steps than stages."""
    batch, dim, steps = 5, 2 * 2048 // N, 6
    A, D, bias = gen.channel_params(dim, N, "normal", 90 + N)
    h0 = gen.initial_state(batch, dim, N, 91, "normal")
    state = torch.from_numpy(h0.copy()).to(DEV)
    ref_state = h0.astype(np.float64)
    Ad, Dd, bd = (torch.from_numpy(x).to(DEV) for x in (A, D, bias))
    flags = mss.FLAG_ZOH_INPUT if zoh else 0
    for t in range(steps):
        s = gen.decode_step_inputs(batch, dim, N, dtype, 92, t)
        dev = _step_dev(s)
        if not gate:
            dev["z"] = None
        y = mss.state_update(state, A=Ad, D=Dd, delta_bias=bd, flags=flags, **dev)
        y_ref, ref_state = oracle.state_update(ref_state, s["u"].values, s["delta"].values, A,
                                               s["B"].values, s["C"].values, D=D,
                                               z=s["z"].values if gate else None,
                                               delta_bias=bias, zoh_input=zoh)
        torch.cuda.synchronize()
        assert_close(to_numpy(y), y_ref, dtype, f"step {t} y")
    assert_close(to_numpy(state), ref_state, dtype, "final state")
    assert mss.get_device_error() == 0
