"""GPU parity: the CUDA path, called through the C ABI, against the fp64 oracle.

Every input is generated on the host by the seeded generator; the same values
go to the GPU (as fp32 or bf16 bytes) and, widened exactly, to the oracle.
Tolerances are in tests/helpers.py.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import selective_state_space_mss_b200 as mss
from selective_state_space_mss_b200 import inputs as gen
from tests.helpers import assert_close, device_inputs, to_numpy

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)
PATHS = {"default": 0, "general-A": mss.FLAG_GENERAL_A, "simple": mss.FLAG_SIMPLE}


def run_fwd(inp, flags=0, softplus=True, with_z=True, with_D=True, with_bias=True):
    d = device_inputs(inp, DEV, with_z, with_D, with_bias)
    y, last = mss.scan_fwd(**d, softplus=softplus, flags=flags)
    torch.cuda.synchronize()
    assert mss.get_device_error() == 0
    return to_numpy(y), to_numpy(last)


def oracle_fwd(inp, softplus=True, with_z=True, with_D=True, with_bias=True):
    return oracle.scan_fwd(inp["u"].values, inp["delta"].values, inp["A"], inp["B"].values,
                           inp["C"].values, D=inp["D"] if with_D else None,
                           z=inp["z"].values if with_z else None,
                           delta_bias=inp["delta_bias"] if with_bias else None,
                           softplus_flag=softplus)


# ---------------------------------------------------------------------------
# The workloads, every element compared with the oracle

@pytest.mark.parametrize("path", sorted(PATHS))
@pytest.mark.parametrize("name", ["s6-fwd-fp32-b1-d16-n4-l256", "mamba130m-layer-bf16-b8-d1536-n16-l2048"])
def test_workload_full(name, path):
    inp = gen.workload_inputs(name)
    y, last = run_fwd(inp, PATHS[path])
    y_ref, last_ref = oracle_fwd(inp)
    dt = gen.WORKLOADS[name].dtype
    assert_close(y, y_ref, dt, f"{name}/{path} y")
    assert_close(last, last_ref, dt, f"{name}/{path} last_state")


@pytest.mark.parametrize("path", ["default", "general-A"])
@pytest.mark.parametrize("name", ["mamba1.4b-layer-bf16-b4-d4096-n16-l4096", "long-seq-bf16-b1-d2048-n16-l131072"])
def test_workload_full_size(name, path):
    """The two large workloads at full size, in the launch configuration the
    bench times (sequence split with the library's workspace where it
    applies), compared element by element with the oracle over every
    channel and token."""
    w = gen.WORKLOADS[name]
    inp = gen.workload_inputs(name)
    y, last = run_fwd(inp, PATHS[path])
    y_ref, last_ref = oracle_fwd(inp)
    assert_close(y, y_ref, w.dtype, f"{name}/{path} y")
    assert_close(last, last_ref, w.dtype, f"{name}/{path} last_state")


# ---------------------------------------------------------------------------
# Edge shapes: ragged tails, every N, small and odd sizes, optional inputs off

EDGE = [
    (1, 1, 1, 1), (1, 1, 16, 1), (1, 3, 2, 7), (2, 5, 4, 33), (1, 33, 8, 255),
    (3, 40, 16, 257), (2, 64, 16, 1000), (1, 130, 16, 4097), (2, 17, 16, 2049), (1, 8, 16, 8),
]


@pytest.mark.parametrize("path", sorted(PATHS))
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", EDGE, ids=lambda s: "x".join(map(str, s)))
def test_edge_shapes(shape, dtype, path):
    batch, dim, N, L = shape
    inp = gen.scan_inputs(batch, dim, N, L, dtype, seed=7 + L + dim, d_skip="normal")
    y, last = run_fwd(inp, PATHS[path])
    y_ref, last_ref = oracle_fwd(inp)
    assert_close(y, y_ref, dtype, f"{shape}/{dtype}/{path} y")
    assert_close(last, last_ref, dtype, f"{shape}/{dtype}/{path} last_state")


@pytest.mark.parametrize("path", sorted(PATHS))
@pytest.mark.parametrize("opts", [dict(with_z=False), dict(with_D=False), dict(with_bias=False),
                                  dict(softplus=False), dict(with_z=False, with_D=False, with_bias=False)],
                         ids=["no-z", "no-D", "no-bias", "no-softplus", "bare"])
def test_optional_inputs(opts, path):
    inp = gen.scan_inputs(2, 48, 16, 300, "bf16", seed=5, d_skip="normal")
    if opts.get("softplus") is False:
        # keep the step positive without softplus
        inp["delta"].values[:] = np.abs(inp["delta"].values) + np.float32(0.01)
        inp["delta"].stored[:] = gen.to_bf16_bits(inp["delta"].values)
        inp["delta"].values[:] = gen.bf16_bits_to_f32(inp["delta"].stored)
        inp["delta_bias"][:] = 0.0
    y, last = run_fwd(inp, PATHS[path], **opts)
    y_ref, last_ref = oracle_fwd(inp, **opts)
    assert_close(y, y_ref, "bf16", f"{opts}/{path} y")
    assert_close(last, last_ref, "bf16", f"{opts}/{path} last_state")


def test_unaligned_rows_take_the_scalar_path():
    # L = 13: bf16 rows start at odd multiples of 2 bytes, so they are not
    # 16-byte aligned; the call must still be right
    inp = gen.scan_inputs(2, 9, 16, 13, "bf16", seed=12, d_skip="normal")
    y, last = run_fwd(inp)
    y_ref, last_ref = oracle_fwd(inp)
    assert_close(y, y_ref, "bf16", "y")
    assert_close(last, last_ref, "bf16", "last_state")
    # a base pointer offset by one element
    d = device_inputs(inp, DEV)
    big = torch.empty(d["u"].numel() + 1, dtype=torch.bfloat16, device=DEV)
    big[1:] = d["u"].reshape(-1)
    d["u"] = big[1:].view(d["u"].shape)
    y2, _ = mss.scan_fwd(**d)
    torch.cuda.synchronize()
    assert np.array_equal(to_numpy(y2), y)


def test_zero_length_and_empty():
    inp = gen.scan_inputs(2, 4, 16, 0, "bf16", seed=1)
    d = device_inputs(inp, DEV)
    last = torch.full((2, 4, 16), 7.0, device=DEV)
    y, last = mss.scan_fwd(**d, last_state=last)
    torch.cuda.synchronize()
    assert y.shape == (2, 4, 0) and torch.all(last == 0)
    inp = gen.scan_inputs(0, 4, 16, 10, "bf16", seed=1)
    y, last = mss.scan_fwd(**device_inputs(inp, DEV))
    assert y.shape == (0, 4, 10)


# ---------------------------------------------------------------------------
# Values the pages print, through the GPU entry point
# ("Exercises -- State-space models (Mamba, S4)")

def _impulse(A_vals, B_vals, C_vals, step, L, dtype=torch.float32):
    N = len(A_vals)
    u = torch.zeros(1, 1, L, device=DEV, dtype=dtype)
    u[0, 0, 0] = 1
    return dict(u=u, delta=torch.full((1, 1, L), step, device=DEV, dtype=dtype),
                A=torch.tensor([A_vals], device=DEV, dtype=torch.float32),
                B=torch.tensor(B_vals, device=DEV, dtype=dtype).view(1, N, 1).repeat(1, 1, L),
                C=torch.tensor(C_vals, device=DEV, dtype=dtype).view(1, N, 1).repeat(1, 1, L))


@pytest.mark.parametrize("path", sorted(PATHS))
def test_worked_example_impulse_response(path):
    # Abar = diag(0.8, 0.4), Bbar = (0.5, 1), C = (2, -1), impulse -> y = (0, 0.4, 0.48)
    d = _impulse([math.log(0.8), math.log(0.4)], [0.5, 1.0], [2.0, -1.0], 1.0, 3)
    y, last = mss.scan_fwd(**d, softplus=False, flags=PATHS[path])
    torch.cuda.synchronize()
    np.testing.assert_allclose(to_numpy(y)[0, 0], [0.0, 0.4, 0.48], atol=2e-6)
    np.testing.assert_allclose(to_numpy(last)[0, 0], [0.32, 0.16], atol=2e-6)


@pytest.mark.parametrize("path", sorted(PATHS))
def test_printed_softplus_and_abar_values(path):
    cases = [(-1.0, 3.0, 3.0486, 0.0474), (-1.0, -3.0, 0.04859, 0.9526),
             (-0.02, 3.0, 3.0486, 0.9408), (-0.02, -3.0, 0.04859, 0.99903)]
    for A, raw, step_printed, abar_printed in cases:
        d = _impulse([A], [1.0], [1.0], raw, 2)
        y, _ = mss.scan_fwd(**d, softplus=True, flags=PATHS[path])
        torch.cuda.synchronize()
        y = to_numpy(y)[0, 0].astype(np.float64)
        step_digits = len(str(step_printed).split(".")[1])
        abar_digits = len(str(abar_printed).split(".")[1])
        assert abs(y[0] - step_printed) <= 0.5 * 10 ** -step_digits + 1e-6
        assert abs(y[1] / y[0] - abar_printed) <= 0.5 * 10 ** -abar_digits + 1e-5


# ---------------------------------------------------------------------------
# Exact properties of the GPU output

@pytest.mark.parametrize("path", sorted(PATHS))
def test_causality_bitwise(path):
    inp = gen.scan_inputs(2, 40, 16, 700, "bf16", seed=21, d_skip="normal")
    d = device_inputs(inp, DEV)
    y0, _ = mss.scan_fwd(**d, flags=PATHS[path])
    t0 = 411
    d["u"][:, :, t0] += 1.0
    d["B"][:, :, t0] *= -2.0
    y1, _ = mss.scan_fwd(**d, flags=PATHS[path])
    torch.cuda.synchronize()
    assert torch.equal(y0[..., :t0], y1[..., :t0])
    assert not torch.equal(y0[..., t0:], y1[..., t0:])


@pytest.mark.parametrize("path", sorted(PATHS))
def test_zero_step_keeps_state_bitwise(path):
    inp = gen.scan_inputs(1, 32, 16, 64, "f32", seed=22, d_skip="normal")
    d = device_inputs(inp, DEV, with_bias=False)
    d["delta"] = d["delta"].abs() + 0.01
    d["delta"][..., 40] = 0.0
    _, before = mss.scan_fwd(**{**d, **{k: d[k][..., :40].contiguous() for k in ("u", "delta", "z", "B", "C")}},
                             softplus=False, flags=PATHS[path])
    _, after = mss.scan_fwd(**{**d, **{k: d[k][..., :41].contiguous() for k in ("u", "delta", "z", "B", "C")}},
                            softplus=False, flags=PATHS[path])
    torch.cuda.synchronize()
    assert torch.equal(before, after)


def test_paths_agree_with_each_other():
    inp = gen.workload_inputs("mamba130m-layer-bf16-b8-d1536-n16-l2048")
    y0, l0 = run_fwd(inp, 0)
    y1, l1 = run_fwd(inp, mss.FLAG_SIMPLE)
    assert_close(y0, y1.astype(np.float64), "bf16", "default vs simple y")
    assert_close(l0, l1.astype(np.float64), "bf16", "default vs simple last_state")


def test_repeated_calls_are_deterministic():
    inp = gen.scan_inputs(2, 256, 16, 1500, "bf16", seed=30, d_skip="normal")
    d = device_inputs(inp, DEV)
    ya, la = mss.scan_fwd(**d)
    yb, lb = mss.scan_fwd(**d)
    torch.cuda.synchronize()
    assert torch.equal(ya, yb) and torch.equal(la, lb)


# ---------------------------------------------------------------------------
# Starting state and the sequence split

def _inputs_dev_and_oracle(batch, dim, N, L, dtype, seed):
    inp = gen.scan_inputs(batch, dim, N, L, dtype, seed=seed, d_skip="normal")
    return inp, device_inputs(inp, DEV)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_initial_state_matches_oracle_and_chains(dtype):
    batch, dim, N, L = 2, 48, 16, 512
    inp, d = _inputs_dev_and_oracle(batch, dim, N, L, dtype, 41)
    h0 = np.random.default_rng(42).standard_normal((batch, dim, N)).astype(np.float32)
    y, last = mss.scan_fwd(**d, initial_state=torch.from_numpy(h0).to(DEV))
    y_ref, last_ref = oracle.scan_fwd(inp["u"].values, inp["delta"].values, inp["A"], inp["B"].values,
                                      inp["C"].values, D=inp["D"], z=inp["z"].values,
                                      delta_bias=inp["delta_bias"], initial_state=h0.astype(np.float64))
    assert_close(to_numpy(y), y_ref, dtype, "y from a starting state")
    assert_close(to_numpy(last), last_ref, dtype, "last_state from a starting state")
    # two calls chained through last_state equal one call
    L0 = 192
    part = lambda t0, t1: {k: (v[..., t0:t1].contiguous() if k in ("u", "delta", "z", "B", "C") else v)
                           for k, v in d.items()}
    y_all, last_all = mss.scan_fwd(**d)
    y0, last0 = mss.scan_fwd(**part(0, L0))
    y1, last1 = mss.scan_fwd(**part(L0, L), initial_state=last0)
    torch.cuda.synchronize()
    assert_close(to_numpy(torch.cat([y0, y1], dim=2)), to_numpy(y_all).astype(np.float64), dtype, "chained y")
    assert_close(to_numpy(last1), to_numpy(last_all).astype(np.float64), dtype, "chained last_state")


SPLIT_SHAPES = [(1, 16, 16, 4096, "bf16"), (2, 40, 16, 4096 + 448, "bf16"), (1, 32, 8, 8192, "bf16"),
                (1, 16, 4, 2048, "bf16"), (1, 16, 16, 2048, "f32"), (3, 16, 16, 1024 + 8, "bf16")]


@pytest.mark.parametrize("shape", SPLIT_SHAPES, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("with_h0", [False, True])
def test_sequence_split_matches_oracle(shape, with_h0):
    batch, dim, N, L, dtype = shape
    assert mss.workspace_size(batch, dim, N, L, torch.bfloat16 if dtype == "bf16" else torch.float32) > 0
    inp, d = _inputs_dev_and_oracle(batch, dim, N, L, dtype, 50 + L + N)
    h0 = np.random.default_rng(51).standard_normal((batch, dim, N)).astype(np.float32) if with_h0 else None
    h0d = torch.from_numpy(h0).to(DEV) if with_h0 else None
    y, last = mss.scan_fwd(**d, initial_state=h0d)                      # split (auto workspace)
    y_ns, last_ns = mss.scan_fwd(**d, initial_state=h0d, workspace=None)  # not split
    torch.cuda.synchronize()
    assert mss.get_device_error() == 0
    y_ref, last_ref = oracle.scan_fwd(inp["u"].values, inp["delta"].values, inp["A"], inp["B"].values,
                                      inp["C"].values, D=inp["D"], z=inp["z"].values,
                                      delta_bias=inp["delta_bias"],
                                      initial_state=None if h0 is None else h0.astype(np.float64))
    assert_close(to_numpy(y), y_ref, dtype, f"{shape} split y")
    assert_close(to_numpy(last), last_ref, dtype, f"{shape} split last_state")
    assert_close(to_numpy(y_ns), y_ref, dtype, f"{shape} unsplit y")
    # outside the split's first segment only rounding differs from the unsplit pass
    assert_close(to_numpy(y), to_numpy(y_ns).astype(np.float64), dtype, f"{shape} split vs unsplit")


def test_zero_length_copies_initial_state():
    inp, d = _inputs_dev_and_oracle(2, 4, 16, 0, "bf16", 3)
    h0 = torch.randn(2, 4, 16, device=DEV)
    _, last = mss.scan_fwd(**d, initial_state=h0)
    torch.cuda.synchronize()
    assert torch.equal(last, h0)
