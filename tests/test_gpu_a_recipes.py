"""GPU parity with A other than the workloads' S4D-Real rows, through every
kernel family, against the fp64 oracle.

A is diagonal and real, one single-input single-output system per channel
("Mamba" paper review, section "SSM"), so nothing ties one channel's A to
another's.  The recipes of the input generator:

* scaled: A[d, n] = -(n + 1) * s_d -- still exactly geometric per channel, so
  the kernels keep their fast transition, but every channel differs (a read
  of another channel's row shows);
* random: per channel and state, log-uniform on [0.1, 20] (negated) -- the
  general transition, no structure to lean on;
* mixed: channels cycle through S4D-Real, random and scaled rows, so every
  group of channels a warp serves mixes rows that pass and fail the fast
  path's test (the warp must take the general path for all of them).

Each runs through the forward kernels (default, general-A, scalar, sequence
split, causal convolution in front), both decode kernels and the backward
pass, under the Euler and the zero-order-hold input rules.  Tolerances are
those of tests/helpers.py.
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
RECIPES = ["scaled", "random", "mixed"]
PATHS = {"default": 0, "general-A": mss.FLAG_GENERAL_A, "simple": mss.FLAG_SIMPLE}


def _flags(path, zoh):
    return PATHS[path] | (mss.FLAG_ZOH_INPUT if zoh else 0)


def _oracle_fwd(inp, zoh, initial_state=None):
    return oracle.scan_fwd(inp["u"].values, inp["delta"].values, inp["A"], inp["B"].values, inp["C"].values,
                           D=inp["D"], z=inp["z"].values, delta_bias=inp["delta_bias"], zoh_input=zoh,
                           initial_state=initial_state)


@pytest.mark.parametrize("zoh", [False, True], ids=["euler", "zoh"])
@pytest.mark.parametrize("path", sorted(PATHS))
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N", [4, 16])
@pytest.mark.parametrize("recipe", RECIPES)
def test_forward(recipe, N, dtype, path, zoh):
    # 80 channels: several warps of channels and a ragged last one; L = 1000: a ragged last chunk
    inp = gen.scan_inputs(2, 80, N, 1000, dtype, seed=600 + N, d_skip="normal", a_init=recipe)
    d = device_inputs(inp, DEV)
    y, last = mss.scan_fwd(**d, flags=_flags(path, zoh), workspace=None)
    torch.cuda.synchronize()
    assert mss.get_device_error() == 0
    y_ref, last_ref = _oracle_fwd(inp, zoh)
    assert_close(to_numpy(y), y_ref, dtype, f"{recipe}/{path} y")
    assert_close(to_numpy(last), last_ref, dtype, f"{recipe}/{path} last_state")


@pytest.mark.parametrize("zoh", [False, True], ids=["euler", "zoh"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("recipe", RECIPES)
def test_forward_split(recipe, dtype, zoh):
    batch, dim, N, L = 1, 48, 16, 4096
    assert mss.workspace_size(batch, dim, N, L, torch.bfloat16 if dtype == "bf16" else torch.float32) > 0
    inp = gen.scan_inputs(batch, dim, N, L, dtype, seed=610, d_skip="normal", a_init=recipe)
    h0 = np.random.default_rng(611).standard_normal((batch, dim, N)).astype(np.float32)
    d = device_inputs(inp, DEV)
    y, last = mss.scan_fwd(**d, initial_state=torch.from_numpy(h0).to(DEV),
                           flags=mss.FLAG_ZOH_INPUT if zoh else 0)
    torch.cuda.synchronize()
    assert mss.get_device_error() == 0
    y_ref, last_ref = _oracle_fwd(inp, zoh, initial_state=h0.astype(np.float64))
    assert_close(to_numpy(y), y_ref, dtype, f"{recipe} split y")
    assert_close(to_numpy(last), last_ref, dtype, f"{recipe} split last_state")


@pytest.mark.parametrize("zoh", [False, True], ids=["euler", "zoh"])
@pytest.mark.parametrize("path", sorted(PATHS))
@pytest.mark.parametrize("recipe", RECIPES)
def test_forward_with_conv(recipe, path, zoh):
    dtype, batch, dim, N, L, K = "bf16", 2, 40, 16, 1000, 4
    inp = gen.scan_inputs(batch, dim, N, L, dtype, seed=620, d_skip="normal", a_init=recipe)
    w, b = gen.conv_params(dim, K, 621)
    cs = gen.conv_state(batch, dim, K, dtype, 622)
    d = device_inputs(inp, DEV)
    d["x"] = d.pop("u")
    y, last, cso = mss.scan_fwd_conv(**d, conv_w=torch.from_numpy(w).to(DEV), conv_b=torch.from_numpy(b).to(DEV),
                                     conv_state=to_torch(cs, DEV), flags=_flags(path, zoh), workspace=None)
    torch.cuda.synchronize()
    assert mss.get_device_error() == 0
    y_ref, last_ref, cs_ref = oracle.scan_fwd_conv(
        inp["u"].values, w, inp["delta"].values, inp["A"], inp["B"].values, inp["C"].values, conv_b=b,
        conv_state=cs.values, D=inp["D"], z=inp["z"].values, delta_bias=inp["delta_bias"], zoh_input=zoh)
    assert_close(to_numpy(y), y_ref, dtype, f"{recipe}/{path} conv y")
    assert_close(to_numpy(last), last_ref, dtype, f"{recipe}/{path} conv last_state")
    assert np.array_equal(to_numpy(cso).astype(np.float64), cs_ref)


@pytest.mark.parametrize("zoh", [False, True], ids=["euler", "zoh"])
@pytest.mark.parametrize("dim_kind", ["tiles", "ragged"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("recipe", RECIPES)
def test_decode(recipe, dtype, dim_kind, zoh):
    """Both decode kernels: whole 8 KB state tiles (bulk-staged) and a channel
    count that is not (per-thread)."""
    batch, N, steps = 3, 16, 6
    dim = 2 * 2048 // N if dim_kind == "tiles" else 37
    A, D, bias = gen.channel_params(dim, N, "normal", 630, a_init=recipe)
    h0 = gen.initial_state(batch, dim, N, 631, "normal")
    state = torch.from_numpy(h0.copy()).to(DEV)
    ref_state = h0.astype(np.float64)
    Ad, Dd, bd = (torch.from_numpy(x).to(DEV) for x in (A, D, bias))
    flags = mss.FLAG_ZOH_INPUT if zoh else 0
    for t in range(steps):
        s = gen.decode_step_inputs(batch, dim, N, dtype, 632, t)
        y = mss.state_update(state, A=Ad, D=Dd, delta_bias=bd, flags=flags,
                             **{k: to_torch(s[k], DEV) for k in ("u", "delta", "z", "B", "C")})
        y_ref, ref_state = oracle.state_update(ref_state, s["u"].values, s["delta"].values, A, s["B"].values,
                                               s["C"].values, D=D, z=s["z"].values, delta_bias=bias,
                                               zoh_input=zoh)
        torch.cuda.synchronize()
        assert_close(to_numpy(y), y_ref, dtype, f"{recipe} step {t} y")
    assert_close(to_numpy(state), ref_state, dtype, f"{recipe} final state")
    assert mss.get_device_error() == 0


BWD_PATHS = {"default": 0, "general-A": mss.FLAG_GENERAL_A, "simple": mss.FLAG_SIMPLE}


@pytest.mark.parametrize("zoh", [False, True], ids=["euler", "zoh"])
@pytest.mark.parametrize("path", sorted(BWD_PATHS))
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("recipe", RECIPES)
def test_backward(recipe, dtype, path, zoh):
    batch, dim, N, L = 2, 40, 16, 1000
    inp = gen.scan_inputs(batch, dim, N, L, dtype, seed=640, d_skip="normal", a_init=recipe)
    if dtype == "f32":
        # fp32 holds the 1e-4 bound where a state's memory 1/(Delta |A|) stays
        # well below 1e-4 / 2^-24 (about 1700 tokens): the rounding of
        # Abar = exp(Delta A) near 1 is carried over that many tokens, and the
        # summed dA adds up the error of every token (Delta >= 1e-3 here, so
        # |A| >= 1 keeps the memory under 1000 tokens).  The full range of the
        # recipe (|A| down to 0.1) runs in bf16 with its 2e-2 bound.
        inp["A"] = np.minimum(inp["A"], np.float32(-1.0))
    d = device_inputs(inp, DEV)
    dy, dl = gen.upstream_gradients(batch, dim, N, L, dtype, 641)
    h0 = np.random.default_rng(642).standard_normal((batch, dim, N)).astype(np.float32)
    flags = BWD_PATHS[path] | (mss.FLAG_ZOH_INPUT if zoh else 0)
    g = mss.scan_bwd(**d, dy=to_torch(dy, DEV), dlast=torch.from_numpy(dl).to(DEV),
                     initial_state=torch.from_numpy(h0).to(DEV), flags=flags)
    torch.cuda.synchronize()
    assert mss.get_device_error() == 0
    ref = oracle.scan_bwd(inp["u"].values, inp["delta"].values, inp["A"], inp["B"].values, inp["C"].values,
                          dy.values, D=inp["D"], z=inp["z"].values, delta_bias=inp["delta_bias"],
                          initial_state=h0.astype(np.float64), dlast=dl.astype(np.float64), zoh_input=zoh)
    for k in ("du", "ddelta", "dz", "dA", "dB", "dC", "dD", "dbias", "dinit"):
        assert_close(to_numpy(g[k]), ref[k], dtype, f"{recipe}/{path} {k}")
