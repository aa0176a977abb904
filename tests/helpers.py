"""Shared test helpers: device upload of generated inputs and the parity
tolerances.

Tolerances, written out:
* fp32 inputs: |y_gpu - y_ref| <= 1e-4 * (1 + |y_ref|) elementwise.
* bf16 inputs: |y_gpu - y_ref| <= 2e-2 * max(|y_ref|, rms(y_ref)) elementwise,
  with the oracle run on the same bf16-rounded values widened exactly to fp64
  (rms over all compared elements).
The same rules apply to last_state and to the decode state and outputs.
"""
import numpy as np
import torch

from selective_state_space_mss_b200 import inputs as gen

FP32_TOL = 1e-4
BF16_TOL = 2e-2


def to_torch(t: "gen.Tensor", device):
    if t.dtype == "f32":
        return torch.from_numpy(np.ascontiguousarray(t.stored)).to(device)
    return torch.from_numpy(np.ascontiguousarray(t.stored).view(np.int16)).view(torch.bfloat16).to(device)


def device_inputs(inp: dict, device, with_z=True, with_D=True, with_bias=True):
    return dict(
        u=to_torch(inp["u"], device), delta=to_torch(inp["delta"], device),
        A=torch.from_numpy(inp["A"]).to(device),
        B=to_torch(inp["B"], device), C=to_torch(inp["C"], device),
        D=torch.from_numpy(inp["D"]).to(device) if with_D else None,
        z=to_torch(inp["z"], device) if with_z else None,
        delta_bias=torch.from_numpy(inp["delta_bias"]).to(device) if with_bias else None,
    )


def oracle_inputs(inp: dict, rows=None, with_z=True, with_D=True, with_bias=True):
    """fp32 values for the oracle; `rows` = list of (b, d) to keep (each as its
    own batch row of one channel), or None for everything."""
    if rows is None:
        return dict(u=inp["u"].values, delta=inp["delta"].values, A=inp["A"],
                    B=inp["B"].values, C=inp["C"].values,
                    D=inp["D"] if with_D else None,
                    z=inp["z"].values if with_z else None,
                    delta_bias=inp["delta_bias"] if with_bias else None)
    raise NotImplementedError


def assert_close(got, ref, dtype, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    if got.size == 0:
        return
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    err = np.abs(got - ref)
    if dtype == "f32":
        bound = FP32_TOL * (1.0 + np.abs(ref))
    else:
        rms = np.sqrt(np.mean(ref * ref))
        bound = BF16_TOL * np.maximum(np.abs(ref), rms)
    bad = err > bound
    if np.any(bad):
        i = np.unravel_index(np.argmax(err / np.maximum(bound, 1e-300)), err.shape)
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {err.size} elements out of tolerance; worst at {i}: "
            f"got {got[i]!r}, ref {ref[i]!r}, bound {bound[i]!r}")


def to_numpy(t):
    return t.detach().float().cpu().numpy()
