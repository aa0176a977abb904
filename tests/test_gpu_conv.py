"""GPU parity of the causal convolution in front of the scan
(mss_scan_fwd_conv, mss_state_update_conv).

u = silu(conv_b + causal depthwise convolution of x), the convolution and
non-linearity between the input projection and the SSM bank ("Mamba" paper
review, section "SSM", block description; "NN Lab -- Mamba": the fused
kernel includes the causal 1D convolution).  Every kernel path is compared
with the fp64 oracle (scan_fwd_conv, state_update_conv) on the same seeded
inputs; the conv state, a copy of inputs, must match exactly.  Tolerances are
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

PATHS = {"fast": 0, "general": mss.FLAG_GENERAL_A, "simple": mss.FLAG_SIMPLE}


def _case(batch, dim, N, L, K, dtype, seed, with_state=True):
    inp = gen.scan_inputs(batch, dim, N, L, dtype, seed=seed, d_skip="normal")
    w, b = gen.conv_params(dim, K, seed + 1)
    cs = gen.conv_state(batch, dim, K, dtype, seed + 2) if with_state else None
    d = device_inputs(inp, DEV)
    d["x"] = d.pop("u")
    dev = dict(d, conv_w=torch.from_numpy(w).to(DEV), conv_b=torch.from_numpy(b).to(DEV),
               conv_state=to_torch(cs, DEV) if cs is not None else None)
    return inp, w, b, cs, dev


def _oracle(inp, w, b, cs, h0=None, zoh=False):
    return oracle.scan_fwd_conv(inp["u"].values, w, inp["delta"].values, inp["A"], inp["B"].values,
                                inp["C"].values, conv_b=b, conv_state=None if cs is None else cs.values,
                                D=inp["D"], z=inp["z"].values, delta_bias=inp["delta_bias"],
                                initial_state=h0, zoh_input=zoh)


def _check_all(y, last, cso, ref, dtype, what):
    y_ref, last_ref, cs_ref = ref
    torch.cuda.synchronize()
    assert mss.get_device_error() == 0
    assert_close(to_numpy(y), y_ref, dtype, f"{what} y")
    assert_close(to_numpy(last), last_ref, dtype, f"{what} last_state")
    if cso is not None:
        assert np.array_equal(to_numpy(cso).astype(np.float64), cs_ref), f"{what} conv state"


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N", [4, 16])
@pytest.mark.parametrize("K", [2, 4])
@pytest.mark.parametrize("path", sorted(PATHS))
def test_conv_forward_matches_oracle(dtype, N, K, path):
    # L = 1000: several chunks and a ragged last chunk; a starting conv state
    inp, w, b, cs, dev = _case(2, 40, N, 1000, K, dtype, 400 + N + K)
    y, last, cso = mss.scan_fwd_conv(**dev, flags=PATHS[path], workspace=None)
    _check_all(y, last, cso, _oracle(inp, w, b, cs), dtype, f"conv {path}")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("K", [1, 3])
def test_conv_widths_and_no_state(dtype, K):
    """Odd widths, no starting conv state, no conv bias, no gate, zero-order hold."""
    inp, w, _, _, dev = _case(2, 48, 16, 512, K, dtype, 410 + K, with_state=False)
    dev["conv_b"] = None
    dev["z"] = None
    for flags in (mss.FLAG_ZOH_INPUT, mss.FLAG_ZOH_INPUT | mss.FLAG_SIMPLE):
        y, last, cso = mss.scan_fwd_conv(**dev, flags=flags)
        ref = oracle.scan_fwd_conv(inp["u"].values, w, inp["delta"].values, inp["A"], inp["B"].values,
                                   inp["C"].values, D=inp["D"], delta_bias=inp["delta_bias"], zoh_input=True)
        _check_all(y, last, cso, ref, dtype, f"K={K} flags={flags}")


@pytest.mark.parametrize("shape", [(1, 16, 16, 4096, "bf16"), (2, 40, 8, 4096 + 448, "bf16"),
                                   (1, 16, 16, 2048, "f32")], ids=lambda s: "x".join(map(str, s)))
def test_conv_sequence_split(shape):
    """Split sequences: later segments take their first window from x itself."""
    batch, dim, N, L, dtype = shape
    assert mss.workspace_size(batch, dim, N, L, torch.bfloat16 if dtype == "bf16" else torch.float32) > 0
    inp, w, b, cs, dev = _case(batch, dim, N, L, 4, dtype, 420 + L)
    h0 = np.random.default_rng(421).standard_normal((batch, dim, N)).astype(np.float32)
    y, last, cso = mss.scan_fwd_conv(**dev, initial_state=torch.from_numpy(h0).to(DEV))
    _check_all(y, last, cso, _oracle(inp, w, b, cs, h0=h0.astype(np.float64)), dtype, f"{shape} split")
    y2, last2, _ = mss.scan_fwd_conv(**dev, initial_state=torch.from_numpy(h0).to(DEV), workspace=None)
    torch.cuda.synchronize()
    assert_close(to_numpy(y2), to_numpy(y).astype(np.float64), dtype, "unsplit = split")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_conv_forward_chains_through_both_states(dtype):
    """Two calls chained through last_state and conv_state_out equal one call."""
    inp, w, b, cs, dev = _case(2, 32, 16, 512, 4, dtype, 430)
    y_all, last_all, cs_all = mss.scan_fwd_conv(**dev)
    L0 = 192
    part = lambda t0, t1: {k: (v[..., t0:t1].contiguous() if k in ("x", "delta", "z", "B", "C") else v)
                           for k, v in dev.items()}
    y0, last0, cs0 = mss.scan_fwd_conv(**part(0, L0))
    y1, last1, cs1 = mss.scan_fwd_conv(**dict(part(L0, 512), conv_state=cs0), initial_state=last0)
    torch.cuda.synchronize()
    assert_close(to_numpy(torch.cat([y0, y1], dim=2)), to_numpy(y_all).astype(np.float64), dtype, "chained y")
    assert_close(to_numpy(last1), to_numpy(last_all).astype(np.float64), dtype, "chained last_state")
    assert torch.equal(cs1, cs_all)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_conv_short_and_empty_sequences(dtype):
    """Fewer tokens than the window (the old conv state shifts through), and
    no tokens at all (the conv state is passed on unchanged)."""
    for L in (1, 2):
        inp, w, b, cs, dev = _case(2, 8, 4, L, 4, dtype, 440 + L)
        y, last, cso = mss.scan_fwd_conv(**dev)
        _check_all(y, last, cso, _oracle(inp, w, b, cs), dtype, f"L={L}")
    inp, w, b, cs, dev = _case(2, 8, 4, 1, 4, dtype, 445)
    empty = {k: (v[..., :0].contiguous() if k in ("x", "delta", "z", "B", "C") else v) for k, v in dev.items()}
    _, last, cso = mss.scan_fwd_conv(**empty)
    torch.cuda.synchronize()
    assert torch.equal(cso, dev["conv_state"])
    assert torch.count_nonzero(last) == 0


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N", [4, 16])
@pytest.mark.parametrize("K", [1, 2, 4])
@pytest.mark.parametrize("dim_kind", ["tiles", "ragged"])
def test_conv_decode_matches_oracle(dtype, N, K, dim_kind):
    """Both decode kernels: whole 8 KB state tiles (bulk-staged) and a
    channel count that is not (per-thread)."""
    batch, steps = 3, 6
    dim = 2 * 2048 // N if dim_kind == "tiles" else 37
    A, D, bias = gen.channel_params(dim, N, "normal", 450 + N)
    w, b = gen.conv_params(dim, K, 451)
    h0 = gen.initial_state(batch, dim, N, 452, "normal")
    cs0 = gen.conv_state(batch, dim, K, dtype, 453)
    state = torch.from_numpy(h0.copy()).to(DEV)
    cstate = to_torch(cs0, DEV) if K > 1 else None
    ref_state, ref_cs = h0.astype(np.float64), cs0.values.astype(np.float64)
    Ad, Dd, bd, wd, bbd = (torch.from_numpy(v).to(DEV) for v in (A, D, bias, w, b))
    for t in range(steps):
        s = gen.decode_step_inputs(batch, dim, N, dtype, 454, t)
        dev = {k: to_torch(s[k], DEV) for k in ("u", "delta", "z", "B", "C")}
        dev["x"] = dev.pop("u")
        y = mss.state_update_conv(state, cstate, conv_w=wd, conv_b=bbd, A=Ad, D=Dd, delta_bias=bd, **dev)
        y_ref, ref_state, ref_cs = oracle.state_update_conv(ref_state, ref_cs, s["u"].values, w, s["delta"].values,
                                                            A, s["B"].values, s["C"].values, conv_b=b, D=D,
                                                            z=s["z"].values, delta_bias=bias)
        torch.cuda.synchronize()
        assert_close(to_numpy(y), y_ref, dtype, f"step {t} y")
        if K > 1:
            assert np.array_equal(to_numpy(cstate).astype(np.float64), ref_cs), f"step {t} conv state"
    assert_close(to_numpy(state), ref_state, dtype, "final state")
    assert mss.get_device_error() == 0


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_conv_forward_then_decode(dtype):
    """Decode tokens continuing a forward pass through both of its states
    give the oracle's longer forward pass."""
    batch, dim, N, L0, extra = 2, 64, 16, 256, 5
    inp, w, b, cs, dev = _case(batch, dim, N, L0 + extra, 4, dtype, 460)
    pre = {k: (v[..., :L0].contiguous() if k in ("x", "delta", "z", "B", "C") else v) for k, v in dev.items()}
    _, state, cstate = mss.scan_fwd_conv(**pre)
    y_ref, last_ref, cs_ref = _oracle(inp, w, b, cs)
    for t in range(L0, L0 + extra):
        step = {k: dev[k][..., t].contiguous() for k in ("x", "delta", "z", "B", "C")}
        y = mss.state_update_conv(state, cstate, conv_w=dev["conv_w"], conv_b=dev["conv_b"], A=dev["A"],
                                  D=dev["D"], delta_bias=dev["delta_bias"], **step)
        torch.cuda.synchronize()
        assert_close(to_numpy(y), y_ref[..., t], dtype, f"decode token {t}")
    assert_close(to_numpy(state), last_ref, dtype, "state after decode")
    assert np.array_equal(to_numpy(cstate).astype(np.float64), cs_ref)
