"""GPU parity of the zero-order-hold input rule (MSS_FLAG_ZOH_INPUT).

The input matrix Bbar = (exp(Delta A) - 1)/A * B of the exact discretisation
("Mamba" paper review, section "SSM"; "Paper: Mamba", Objectives) against the
fp64 oracle run with zoh_input=True, on every kernel that takes the flag: the
throughput kernel on its fast transition (A[d,n] = (n+1) A[d,0]) and on its
general path, the one-thread-per-channel kernel, the sequence split, and the
decode update.  Tolerances are those of tests/helpers.py.
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
ZOH = mss.FLAG_ZOH_INPUT


def _oracle(inp, h0=None, A=None):
    return oracle.scan_fwd(inp["u"].values, inp["delta"].values, inp["A"] if A is None else A,
                           inp["B"].values, inp["C"].values, D=inp["D"], z=inp["z"].values,
                           delta_bias=inp["delta_bias"], initial_state=h0, zoh_input=True)


PATHS = {"fast": ZOH, "general": ZOH | mss.FLAG_GENERAL_A, "simple": ZOH | mss.FLAG_SIMPLE}


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N", [4, 8, 16])
@pytest.mark.parametrize("path", sorted(PATHS))
def test_zoh_forward_matches_oracle(dtype, N, path):
    # L = 1000: several chunks and a ragged last group
    batch, dim, L = 2, 40, 1000
    inp = gen.scan_inputs(batch, dim, N, L, dtype, seed=300 + N, d_skip="normal")
    d = device_inputs(inp, DEV)
    y, last = mss.scan_fwd(**d, flags=PATHS[path], workspace=None)
    torch.cuda.synchronize()
    assert mss.get_device_error() == 0
    y_ref, last_ref = _oracle(inp)
    assert_close(to_numpy(y), y_ref, dtype, f"zoh {path} y")
    assert_close(to_numpy(last), last_ref, dtype, f"zoh {path} last_state")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_zoh_differs_from_euler(dtype):
    """The flag changes the result by more than the tolerance (it is not ignored)."""
    inp = gen.scan_inputs(1, 32, 16, 512, dtype, seed=310, d_skip="normal")
    d = device_inputs(inp, DEV)
    _, last_e = mss.scan_fwd(**d)
    _, last_z = mss.scan_fwd(**d, flags=ZOH)
    torch.cuda.synchronize()
    ref_z = _oracle(inp)[1]
    ref_e = oracle.scan_fwd(inp["u"].values, inp["delta"].values, inp["A"], inp["B"].values,
                            inp["C"].values, D=inp["D"], z=inp["z"].values,
                            delta_bias=inp["delta_bias"])[1]
    assert np.max(np.abs(ref_z - ref_e)) > 10 * (1e-4 if dtype == "f32" else 2e-2) * np.sqrt(np.mean(ref_z ** 2))
    assert_close(to_numpy(last_z), ref_z, dtype, "zoh last_state")
    assert_close(to_numpy(last_e), ref_e, dtype, "euler last_state")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_zoh_zero_and_positive_A(dtype):
    """A = 0 (weight Delta, the limit of (e^x - 1)/A) on one channel's whole row
    -- still the fast transition, (n+1)*0 = 0 -- and mixed zero and positive
    entries on the general path."""
    batch, dim, N, L = 1, 32, 16, 256
    inp = gen.scan_inputs(batch, dim, N, L, dtype, seed=320, d_skip="normal")
    A = inp["A"].copy()
    A[:16] = 0.0                      # first CTA: all zero, fast transition
    A[16:, 3] = 0.0                   # second CTA: general path
    A[16:, 5] = 0.05
    d = device_inputs(inp, DEV)
    d["A"] = torch.from_numpy(A).to(DEV)
    for flags in (ZOH, ZOH | mss.FLAG_SIMPLE):
        y, last = mss.scan_fwd(**d, flags=flags, workspace=None)
        torch.cuda.synchronize()
        y_ref, last_ref = _oracle(inp, A=A)
        assert_close(to_numpy(y), y_ref, dtype, f"zoh A=0 y flags={flags}")
        assert_close(to_numpy(last), last_ref, dtype, f"zoh A=0 last_state flags={flags}")


@pytest.mark.parametrize("shape", [(1, 16, 16, 4096, "bf16"), (2, 40, 8, 4096 + 448, "bf16"),
                                   (1, 16, 16, 2048, "f32")], ids=lambda s: "x".join(map(str, s)))
def test_zoh_sequence_split(shape):
    batch, dim, N, L, dtype = shape
    assert mss.workspace_size(batch, dim, N, L, torch.bfloat16 if dtype == "bf16" else torch.float32,
                              flags=ZOH) > 0
    inp = gen.scan_inputs(batch, dim, N, L, dtype, seed=330 + L, d_skip="normal")
    d = device_inputs(inp, DEV)
    h0 = np.random.default_rng(331).standard_normal((batch, dim, N)).astype(np.float32)
    y, last = mss.scan_fwd(**d, initial_state=torch.from_numpy(h0).to(DEV), flags=ZOH)
    torch.cuda.synchronize()
    assert mss.get_device_error() == 0
    y_ref, last_ref = _oracle(inp, h0=h0.astype(np.float64))
    assert_close(to_numpy(y), y_ref, dtype, f"{shape} zoh split y")
    assert_close(to_numpy(last), last_ref, dtype, f"{shape} zoh split last_state")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N", [1, 4, 16])
def test_zoh_decode_matches_oracle(dtype, N):
    batch, dim, steps = 3, 37, 12
    A, D, bias = gen.channel_params(dim, N, "normal", 340)
    h0 = gen.initial_state(batch, dim, N, 341, "normal")
    state = torch.from_numpy(h0.copy()).to(DEV)
    ref_state = h0.astype(np.float64)
    Ad, Dd, bd = (torch.from_numpy(x).to(DEV) for x in (A, D, bias))
    for t in range(steps):
        s = gen.decode_step_inputs(batch, dim, N, dtype, 342, t)
        dev = {k: to_torch(s[k], DEV) for k in ("u", "delta", "z", "B", "C")}
        y = mss.state_update(state, A=Ad, D=Dd, delta_bias=bd, flags=ZOH, **dev)
        y_ref, ref_state = oracle.state_update(ref_state, s["u"].values, s["delta"].values, A,
                                               s["B"].values, s["C"].values, D=D, z=s["z"].values,
                                               delta_bias=bias, zoh_input=True)
        torch.cuda.synchronize()
        assert_close(to_numpy(y), y_ref, dtype, f"zoh decode step {t} y")
    assert_close(to_numpy(state), ref_state, dtype, "zoh decode final state")
    assert mss.get_device_error() == 0


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_zoh_forward_then_decode(dtype):
    """Decode tokens continuing a zero-order-hold forward pass give the
    oracle's longer zero-order-hold forward pass."""
    batch, dim, N, L0, extra = 2, 24, 16, 256, 6
    inp = gen.scan_inputs(batch, dim, N, L0 + extra, dtype, seed=350, d_skip="normal")
    d = device_inputs(inp, DEV)
    pre = {k: (v[..., :L0].contiguous() if k in ("u", "delta", "z", "B", "C") else v) for k, v in d.items()}
    _, state = mss.scan_fwd(**pre, flags=ZOH)
    y_ref, last_ref = _oracle(inp)
    for t in range(L0, L0 + extra):
        step = {k: d[k][..., t].contiguous() for k in ("u", "delta", "z", "B", "C")}
        y = mss.state_update(state, A=d["A"], D=d["D"], delta_bias=d["delta_bias"], flags=ZOH, **step)
        torch.cuda.synchronize()
        assert_close(to_numpy(y), y_ref[..., t], dtype, f"decode token {t}")
    assert_close(to_numpy(state), last_ref, dtype, "state after decode")
