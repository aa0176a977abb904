"""GPU parity of the four-lane forward kernel (scan_seq4.cuh: N = 8 and 16,
one pass over the sequence, Euler input rule; fp32 io on any grid, bf16 io
on grids of at most 384 units of 16 channels) against the fp64 oracle, and
against the two-lane kernel (FLAG_PAIR_LANES).

The two kernels add up the read-out in the same order (each lane's pairs
through one chain of packed fused multiply-adds, then the two halves, then
the lanes of the channel), so their outputs agree bit for bit; the oracle
comparison uses the bound of tests/helpers.py for the io type.  With bf16 io
both kernels take the fast transition (Abar_n = r^(n+1)) per warp when every
channel of the warp has A[d,n] = (n+1) A[d,0]; the four-lane kernel's warps
hold 8 channels, the pair kernel's 16, so where a row of 16 channels mixes
the two kinds they take different paths and only the oracle comparison
applies.  A profiler trace shows which kernel a call launched.
"""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_mss_b200 as mss
from selective_state_space_mss_b200 import inputs as gen
from tests.helpers import assert_close, device_inputs, to_numpy
from tests.test_gpu_failure import Canary

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _run(inp, gate, softplus, h0, flags):
    d = device_inputs(inp, DEV, with_z=gate, with_bias=inp["delta_bias"] is not None)
    return mss.scan_fwd(**d, softplus=softplus, initial_state=h0, workspace=None, flags=flags)


@pytest.mark.parametrize("dim", [16, 40, 17], ids=["one-cta", "ragged-cta", "odd"])
@pytest.mark.parametrize("a_init", ["s4d-real", "mixed"])
@pytest.mark.parametrize("softplus", [True, False], ids=["softplus", "raw-delta"])
@pytest.mark.parametrize("gate", [True, False], ids=["gate", "no-gate"])
@pytest.mark.parametrize("N", [8, 16])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_four_lane_matches_oracle_and_pair_kernel(dtype, N, gate, softplus, a_init, dim):
    # 1000 tokens: 31 chunks of 32 fp32 tokens (15 of 64 bf16 tokens) and a
    # ragged last one
    batch, L = 2, 1000
    inp = gen.scan_inputs(batch, dim, N, L, dtype, seed=800 + N + dim, d_skip="normal", a_init=a_init)
    if not softplus:
        # step sizes that stay positive without softplus (no bias)
        inp["delta"] = gen._store((np.abs(inp["delta"].values) * 0.1 + 0.01).astype(np.float32), dtype)
        inp["delta_bias"] = None
    h0 = np.random.default_rng(801).standard_normal((batch, dim, N)).astype(np.float32)
    h0_d = torch.from_numpy(h0).to(DEV)
    y4, s4 = _run(inp, gate, softplus, h0_d, 0)
    yp, sp = _run(inp, gate, softplus, h0_d, mss.FLAG_PAIR_LANES)
    torch.cuda.synchronize()
    assert mss.get_device_error() == 0
    assert torch.equal(y4, yp) and torch.equal(s4, sp)
    y_ref, s_ref = oracle.scan_fwd(inp["u"].values, inp["delta"].values, inp["A"], inp["B"].values, inp["C"].values,
                                   D=inp["D"], z=inp["z"].values if gate else None, delta_bias=inp["delta_bias"],
                                   softplus_flag=softplus, initial_state=h0.astype(np.float64))
    assert_close(to_numpy(y4), y_ref, dtype, "y")
    assert_close(to_numpy(s4), s_ref, dtype, "last_state")


def test_four_lane_bf16_fast_transition_per_eight_channels():
    # channels 0-7 of each 16 take A = -(n+1) (S4D-Real), 8-15 per-state
    # random A: the four-lane kernel's first warp of each CTA takes the fast
    # transition and its second the general one, the pair kernel's warp the
    # general one throughout; both against the oracle
    batch, dim, N, L = 2, 48, 16, 512
    inp = gen.scan_inputs(batch, dim, N, L, "bf16", seed=805, d_skip="normal")
    rnd = gen.a_matrix(dim, N, "random", 806)
    for d in range(dim):
        if d % 16 >= 8:
            inp["A"][d] = rnd[d]
    y_ref, s_ref = oracle.scan_fwd(inp["u"].values, inp["delta"].values, inp["A"], inp["B"].values, inp["C"].values,
                                   D=inp["D"], z=inp["z"].values, delta_bias=inp["delta_bias"])
    for flags in (0, mss.FLAG_PAIR_LANES):
        y, s = mss.scan_fwd(**device_inputs(inp, DEV), workspace=None, flags=flags)
        assert mss.get_device_error() == 0
        assert_close(to_numpy(y), y_ref, "bf16", f"y flags={flags}")
        assert_close(to_numpy(s), s_ref, "bf16", f"last_state flags={flags}")


SHAPES = [(1, 17, 16, 4), (2, 33, 8, 68), (1, 16, 16, 4096), (3, 9, 16, 36)]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_four_lane_outputs_stay_in_bounds(shape, dtype):
    batch, dim, N, L = shape
    inp = gen.scan_inputs(batch, dim, N, L, dtype, seed=810 + L, d_skip="normal")
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    y, last = Canary((batch, dim, L), tdt), Canary((batch, dim, N), torch.float32)
    mss.scan_fwd(**device_inputs(inp, DEV), y=y.t, last_state=last.t, workspace=None)
    assert mss.get_device_error() == 0
    assert y.intact() and last.intact()
    y_ref, last_ref = oracle.scan_fwd(inp["u"].values, inp["delta"].values, inp["A"], inp["B"].values,
                                      inp["C"].values, D=inp["D"], z=inp["z"].values, delta_bias=inp["delta_bias"])
    assert_close(to_numpy(y.t), y_ref, dtype, "y")
    assert_close(to_numpy(last.t), last_ref, dtype, "last_state")


def _kernels_launched(fn):
    from torch.profiler import ProfilerActivity, profile
    with profile(activities=[ProfilerActivity.CUDA], acc_events=True) as prof:
        fn()
        torch.cuda.synchronize()
    return [e.name for e in prof.events() if e.device_type.name == "CUDA"]


@pytest.mark.parametrize("dtype,batch,dim,flags,expect", [
    ("f32", 2, 32, 0, "scan_fwd_seq4_kernel"),
    ("f32", 2, 32, mss.FLAG_PAIR_LANES, "scan_fwd_seq_kernel"),
    ("bf16", 2, 32, 0, "scan_fwd_seq4_kernel"),
    ("bf16", 2, 32, mss.FLAG_PAIR_LANES, "scan_fwd_seq_kernel"),
    ("bf16", 4, 1536, 0, "scan_fwd_seq4_kernel"),   # 384 units of 16 channels
    ("bf16", 4, 1552, 0, "scan_fwd_seq_kernel"),    # 388 units
], ids=["f32-default", "f32-pair-flag", "bf16-small-grid", "bf16-pair-flag", "bf16-384-units",
        "bf16-388-units"])
def test_kernel_choice(dtype, batch, dim, flags, expect):
    inp = gen.scan_inputs(batch, dim, 16, 256, dtype, seed=820)
    d = device_inputs(inp, DEV)
    mss.scan_fwd(**d, workspace=None, flags=flags)  # loads the library outside the trace
    try:
        names = _kernels_launched(lambda: mss.scan_fwd(**d, workspace=None, flags=flags))
    except Exception as e:  # a box without a working CUDA profiler
        pytest.skip(f"profiler unavailable: {e}")
    ours = [n for n in names if "scan_fwd" in n]
    assert len(ours) == 1, names
    assert expect + "<" in ours[0], ours
