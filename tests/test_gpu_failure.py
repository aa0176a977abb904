"""Failure paths and out-of-bounds stores, tested without faulting the GPU.

Bounded waits: every wait of the tiled kernels on a staging barrier gives up
after a time limit, sets the library's device error word and lets the CTA
return.  MSS_FLAG_SELFTEST_TIMEOUT makes the forward kernel wait, with a 1 ms
limit, on a barrier that no copy will complete, before it has issued any copy
(nothing is in flight when it gives up).  The error must reach the host once
through mss_get_device_error, the outputs must stay untouched, and the next
call must be clean and right.

Canaries: every output is placed inside a larger buffer filled with a
sentinel bit pattern; after ragged shapes (a sequence of 1, 63, 65 or 4097
tokens, 17 or 33 channels) the margins before and after the output must be
bit-identical, so no kernel stores past the end of a row or a tensor on its
masked tail.
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
PAD = 64  # elements of margin on each side: keeps 16-byte alignment for every dtype here


# ---------------------------------------------------------------------------
# Bounded waits

@pytest.mark.parametrize("lanes", [0, mss.FLAG_PAIR_LANES], ids=["four-lane", "pair"])
def test_bounded_wait_gives_up_and_the_next_call_is_clean(lanes):
    # 8 units of 16 bf16 channels: the four-lane kernel unless the flag asks
    # for the pair kernel
    assert mss.get_device_error() == 0
    inp = gen.scan_inputs(2, 64, 16, 512, "bf16", seed=700, d_skip="normal")
    d = device_inputs(inp, DEV)
    y = torch.full((2, 64, 512), 3.0, dtype=torch.bfloat16, device=DEV)
    last = torch.full((2, 64, 16), 5.0, device=DEV)
    mss.scan_fwd(**d, y=y, last_state=last, flags=mss.FLAG_SELFTEST_TIMEOUT | lanes)
    assert mss.get_device_error() == mss.ERR_DEVICE_TIMEOUT
    assert mss.get_device_error() == 0  # reported once, then cleared
    assert torch.all(y == 3.0) and torch.all(last == 5.0)  # nothing was written
    # the context is usable and the same call without the flag is right
    y2, last2 = mss.scan_fwd(**d, flags=lanes)
    assert mss.get_device_error() == 0
    y_ref, last_ref = oracle.scan_fwd(inp["u"].values, inp["delta"].values, inp["A"], inp["B"].values,
                                      inp["C"].values, D=inp["D"], z=inp["z"].values, delta_bias=inp["delta_bias"])
    assert_close(to_numpy(y2), y_ref, "bf16", "y after the timeout")
    assert_close(to_numpy(last2), last_ref, "bf16", "last_state after the timeout")


def test_bounded_wait_self_test_needs_the_tiled_kernel():
    # L = 13 bf16: rows are not 16-byte aligned, so the scalar kernel would
    # run; it has no staging waits, so the flag is refused before any launch
    inp = gen.scan_inputs(1, 8, 16, 13, "bf16", seed=701)
    with pytest.raises(mss.MssError) as e:
        mss.scan_fwd(**device_inputs(inp, DEV), flags=mss.FLAG_SELFTEST_TIMEOUT)
    assert e.value.code == mss.ERR_FLAGS
    assert mss.get_device_error() == 0


# ---------------------------------------------------------------------------
# Canaries

def _sentinel(dtype):
    # a NaN bit pattern no kernel produces from finite inputs
    return {torch.bfloat16: -0x5a5b, torch.float32: -0x5a5b5a5b}[dtype]


class Canary:
    """An output of `shape` inside a buffer with PAD sentinel elements on each side."""

    def __init__(self, shape, dtype):
        n = int(np.prod(shape))
        ity = torch.int16 if dtype == torch.bfloat16 else torch.int32
        self.raw = torch.full((n + 2 * PAD,), _sentinel(dtype), dtype=ity, device=DEV)
        self.n = n
        self.t = self.raw[PAD:PAD + n].view(dtype).view(shape)

    def intact(self):
        torch.cuda.synchronize()
        s = _sentinel(self.t.dtype)
        return bool(torch.all(self.raw[:PAD] == s)) and bool(torch.all(self.raw[PAD + self.n:] == s))


SHAPES = [(1, 17, 16, 1), (2, 17, 16, 63), (2, 33, 16, 65), (1, 33, 16, 4097), (2, 17, 8, 4097),
          (1, 33, 4, 64)]
FWD_PATHS = {"default": 0, "general-A": mss.FLAG_GENERAL_A, "simple": mss.FLAG_SIMPLE}


@pytest.mark.parametrize("path", sorted(FWD_PATHS))
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_forward_outputs_stay_in_bounds(shape, dtype, path):
    batch, dim, N, L = shape
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    inp = gen.scan_inputs(batch, dim, N, L, dtype, seed=710 + L, d_skip="normal")
    y, last = Canary((batch, dim, L), tdt), Canary((batch, dim, N), torch.float32)
    mss.scan_fwd(**device_inputs(inp, DEV), y=y.t, last_state=last.t, flags=FWD_PATHS[path])
    assert mss.get_device_error() == 0
    assert y.intact() and last.intact()
    y_ref, last_ref = oracle.scan_fwd(inp["u"].values, inp["delta"].values, inp["A"], inp["B"].values,
                                      inp["C"].values, D=inp["D"], z=inp["z"].values, delta_bias=inp["delta_bias"])
    assert_close(to_numpy(y.t), y_ref, dtype, "y")
    assert_close(to_numpy(last.t), last_ref, dtype, "last_state")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_split_forward_outputs_stay_in_bounds(dtype):
    batch, dim, N, L = 1, 33, 16, 4096 + 64
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    assert mss.workspace_size(batch, dim, N, L, tdt) > 0
    inp = gen.scan_inputs(batch, dim, N, L, dtype, seed=720, d_skip="normal")
    y, last = Canary((batch, dim, L), tdt), Canary((batch, dim, N), torch.float32)
    ws = Canary((mss.workspace_size(batch, dim, N, L, tdt) // 4,), torch.float32)
    mss.scan_fwd(**device_inputs(inp, DEV), y=y.t, last_state=last.t, workspace=ws.t.view(torch.uint8))
    assert mss.get_device_error() == 0
    assert y.intact() and last.intact() and ws.intact()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dim", [17, 33, 128, 256])
def test_decode_outputs_stay_in_bounds(dtype, dim):
    # 128 and 256 channels at N = 16 take the staged kernel, 17 and 33 the per-thread one
    batch, N = 3, 16
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    A, D, bias = gen.channel_params(dim, N, "normal", 730)
    h0 = gen.initial_state(batch, dim, N, 731, "normal")
    state, y = Canary((batch, dim, N), torch.float32), Canary((batch, dim), tdt)
    state.t.copy_(torch.from_numpy(h0))
    ref_state = h0.astype(np.float64)
    for t in range(3):
        s = gen.decode_step_inputs(batch, dim, N, dtype, 732, t)
        mss.state_update(state.t, A=torch.from_numpy(A).to(DEV), D=torch.from_numpy(D).to(DEV),
                         delta_bias=torch.from_numpy(bias).to(DEV), y=y.t,
                         **{k: to_torch(s[k], DEV) for k in ("u", "delta", "z", "B", "C")})
        y_ref, ref_state = oracle.state_update(ref_state, s["u"].values, s["delta"].values, A, s["B"].values,
                                               s["C"].values, D=D, z=s["z"].values, delta_bias=bias)
        assert y.intact() and state.intact()
        assert_close(to_numpy(y.t), y_ref, dtype, f"step {t} y")
    assert_close(to_numpy(state.t), ref_state, dtype, "state")


@pytest.mark.parametrize("shape", [(2, 17, 16, 63), (1, 33, 16, 4097), (2, 33, 4, 65)],
                         ids=lambda s: "x".join(map(str, s)))
def test_conv_forward_outputs_stay_in_bounds(shape):
    batch, dim, N, L = shape
    K = 4
    inp = gen.scan_inputs(batch, dim, N, L, "bf16", seed=740 + L, d_skip="normal")
    w, b = gen.conv_params(dim, K, 741)
    d = device_inputs(inp, DEV)
    d["x"] = d.pop("u")
    y, last = Canary((batch, dim, L), torch.bfloat16), Canary((batch, dim, N), torch.float32)
    cso = Canary((batch, dim, K - 1), torch.bfloat16)
    mss.scan_fwd_conv(**d, conv_w=torch.from_numpy(w).to(DEV), conv_b=torch.from_numpy(b).to(DEV),
                      y=y.t, last_state=last.t, conv_state_out=cso.t)
    assert mss.get_device_error() == 0
    assert y.intact() and last.intact() and cso.intact()
    y_ref, last_ref, cs_ref = oracle.scan_fwd_conv(inp["u"].values, w, inp["delta"].values, inp["A"],
                                                   inp["B"].values, inp["C"].values, conv_b=b, D=inp["D"],
                                                   z=inp["z"].values, delta_bias=inp["delta_bias"])
    assert_close(to_numpy(y.t), y_ref, "bf16", "conv y")
    assert np.array_equal(to_numpy(cso.t).astype(np.float64), cs_ref)


@pytest.mark.parametrize("flags", [0, mss.FLAG_SIMPLE], ids=["tiled", "simple"])
@pytest.mark.parametrize("shape", [(2, 17, 16, 63), (1, 33, 16, 4097), (2, 33, 8, 65)],
                         ids=lambda s: "x".join(map(str, s)))
def test_backward_outputs_stay_in_bounds(shape, flags):
    batch, dim, N, L = shape
    dtype, tdt = "bf16", torch.bfloat16
    inp = gen.scan_inputs(batch, dim, N, L, dtype, seed=750 + L, d_skip="normal")
    dy, dl = gen.upstream_gradients(batch, dim, N, L, dtype, 751)
    shapes = dict(du=((batch, dim, L), tdt), ddelta=((batch, dim, L), tdt), dz=((batch, dim, L), tdt),
                  dA=((dim, N), torch.float32), dB=((batch, N, L), torch.float32),
                  dC=((batch, N, L), torch.float32), dD=((dim,), torch.float32),
                  dbias=((dim,), torch.float32), dinit=((batch, dim, N), torch.float32))
    outs = {k: Canary(s, t) for k, (s, t) in shapes.items()}
    g = mss.scan_bwd(**device_inputs(inp, DEV), dy=to_torch(dy, DEV), dlast=torch.from_numpy(dl).to(DEV),
                     flags=flags, out={k: c.t for k, c in outs.items()})
    assert mss.get_device_error() == 0
    for k, c in outs.items():
        assert c.intact(), f"{k}: a store landed outside the tensor"
    ref = oracle.scan_bwd(inp["u"].values, inp["delta"].values, inp["A"], inp["B"].values, inp["C"].values,
                          dy.values, D=inp["D"], z=inp["z"].values, delta_bias=inp["delta_bias"],
                          dlast=dl.astype(np.float64))
    for k in shapes:
        assert_close(to_numpy(g[k]), ref[k], dtype, f"backward {k}")


@pytest.mark.parametrize("seqlen", [1, 63, 65, 200])
@pytest.mark.parametrize("chunked", [False, True], ids=["in-order", "chunk-parallel"])
def test_ssd_outputs_stay_in_bounds(seqlen, chunked):
    batch, H, P, G, N = 2, 3, 64, 1, 64
    si = gen.ssd_inputs(batch, seqlen, H, P, G, N, seed=760 + seqlen)
    d = {k: to_torch(si[k], DEV) for k in ("x", "dt", "B", "C", "z")}
    y, last = Canary((batch, seqlen, H, P), torch.bfloat16), Canary((batch, H, N, P), torch.float32)
    mss.ssd_fwd(A=torch.from_numpy(si["A"]).to(DEV), D=torch.from_numpy(si["D"]).to(DEV),
                dt_bias=torch.from_numpy(si["dt_bias"]).to(DEV), y=y.t, last_state=last.t,
                workspace="auto" if chunked else None, **d)
    assert mss.get_device_error() == 0
    assert y.intact() and last.intact()
    y_ref, last_ref = oracle.ssd_fwd(si["x"].values, si["dt"].values, si["A"], si["B"].values, si["C"].values,
                                     D=si["D"], z=si["z"].values, dt_bias=si["dt_bias"])
    assert_close(to_numpy(y.t), y_ref, "bf16", "SSD y")
    assert_close(to_numpy(last.t), last_ref, "bf16", "SSD last_state")
