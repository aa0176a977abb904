"""GPU parity of the backward pass (mss_scan_bwd) against the fp64 oracle's
backward (itself pinned to finite differences and automatic
differentiation of the forward definition).

Every kernel path (the throughput kernel on its fast and general
transitions, the scalar kernel), both input rules, fp32 and bf16, N = 4, 8,
16, with and without the optional inputs.  The per-token gradients follow the
io type's tolerance of tests/helpers.py; the summed ones (dA, dB, dC, dD,
dbias) and dinit are fp32 but computed from the same inputs, so the same rule
of the io type applies to them.
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
KEYS = ("du", "ddelta", "dz", "dA", "dB", "dC", "dD", "dbias", "dinit")


def _run(batch, dim, N, L, dtype, seed, flags=0, gate=True, with_D=True, with_bias=True, h0=True, dlast=True):
    inp = gen.scan_inputs(batch, dim, N, L, dtype, seed=seed, d_skip="normal")
    d = device_inputs(inp, DEV, with_z=gate, with_D=with_D, with_bias=with_bias)
    dy, dl = gen.upstream_gradients(batch, dim, N, L, dtype, seed + 1)
    h = np.random.default_rng(seed + 2).standard_normal((batch, dim, N)).astype(np.float32) if h0 else None
    g = mss.scan_bwd(**d, dy=to_torch(dy, DEV), dlast=torch.from_numpy(dl).to(DEV) if dlast else None,
                     initial_state=torch.from_numpy(h).to(DEV) if h0 else None, flags=flags)
    torch.cuda.synchronize()
    assert mss.get_device_error() == 0
    ref = oracle.scan_bwd(inp["u"].values, inp["delta"].values, inp["A"], inp["B"].values, inp["C"].values,
                          dy.values, D=inp["D"] if with_D else None, z=inp["z"].values if gate else None,
                          delta_bias=inp["delta_bias"] if with_bias else None,
                          initial_state=None if h is None else h.astype(np.float64),
                          dlast=dl.astype(np.float64) if dlast else None,
                          zoh_input=bool(flags & mss.FLAG_ZOH_INPUT))
    return g, ref


def _compare(g, ref, dtype, what, keys=KEYS):
    for k in keys:
        if ref.get(k) is None or g.get(k) is None:
            continue
        assert_close(to_numpy(g[k]), ref[k], dtype, f"{what} {k}")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N", [4, 8, 16])
@pytest.mark.parametrize("path", sorted(PATHS))
@pytest.mark.parametrize("zoh", [False, True])
def test_bwd_matches_oracle(dtype, N, path, zoh):
    # L = 1000: several chunks, a partial last chunk
    flags = PATHS[path] | (mss.FLAG_ZOH_INPUT if zoh else 0)
    g, ref = _run(2, 40, N, 1000, dtype, 500 + N, flags=flags)
    _compare(g, ref, dtype, f"{path} zoh={zoh}")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_bwd_without_optional_inputs(dtype):
    g, ref = _run(2, 32, 16, 512, dtype, 520, gate=False, with_D=False, with_bias=False, h0=False, dlast=False)
    assert g["dz"] is None
    _compare(g, ref, dtype, "bare")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_bwd_without_softplus(dtype):
    inp = gen.scan_inputs(2, 32, 16, 256, dtype, seed=530, d_skip="normal")
    # step sizes that stay positive without softplus
    dl = np.abs(inp["delta"].values) * 0.1 + 0.01
    inp["delta"] = gen._store(dl.astype(np.float32), dtype)
    d = device_inputs(inp, DEV, with_bias=False)
    dy, dlast = gen.upstream_gradients(2, 32, 16, 256, dtype, 531)
    g = mss.scan_bwd(**d, dy=to_torch(dy, DEV), dlast=torch.from_numpy(dlast).to(DEV), softplus=False)
    ref = oracle.scan_bwd(inp["u"].values, inp["delta"].values, inp["A"], inp["B"].values, inp["C"].values,
                          dy.values, D=inp["D"], z=inp["z"].values, softplus_flag=False,
                          dlast=dlast.astype(np.float64))
    torch.cuda.synchronize()
    _compare(g, ref, dtype, "no softplus")


@pytest.mark.parametrize("L", [1, 7, 96])
def test_bwd_short_and_unaligned_sequences(L):
    """Rows that are not 16-byte multiples take the scalar backward."""
    g, ref = _run(2, 24, 16, L, "f32" if L != 96 else "bf16", 540 + L)
    _compare(g, ref, "f32" if L != 96 else "bf16", f"L={L}")


def test_bwd_layer_sized():
    """A Mamba-130M-shaped slice (2 x 256 channels x 2048 tokens, bf16):
    every gradient against the oracle."""
    g, ref = _run(2, 256, 16, 2048, "bf16", 550)
    _compare(g, ref, "bf16", "layer slice")


def test_bwd_zero_length():
    d = device_inputs(gen.scan_inputs(2, 8, 4, 1, "f32", seed=560), DEV)
    empty = {k: (v[..., :0].contiguous() if k in ("u", "delta", "z", "B", "C") else v) for k, v in d.items()}
    dl = torch.randn(2, 8, 4, device=DEV)
    g = mss.scan_bwd(**empty, dy=torch.empty(2, 8, 0, device=DEV), dlast=dl)
    torch.cuda.synchronize()
    assert torch.equal(g["dinit"], dl)
    assert torch.count_nonzero(g["dA"]) == 0 and torch.count_nonzero(g["dD"]) == 0


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N", [4, 8, 16])
@pytest.mark.parametrize("zoh", [False, True], ids=["euler", "zoh"])
@pytest.mark.parametrize("split", [False, True], ids=["one-pass", "split"])
def test_saved_states_training_step(dtype, N, zoh, split):
    """scan_fwd_save + scan_bwd(saved_states=...): y and last_state bit for bit
    those of scan_fwd, every gradient within the oracle's bound; without a
    sequence split the stored states are the checkpoint pass's, so the
    per-token gradients and dinit also equal those of scan_bwd bit for bit."""
    # few channels: with a workspace the forward pass takes its two-pass
    # sequence split, without one it runs in one pass
    batch, dim, L = (1, 48, 4096) if split else (2, 40, 1000)
    flags = mss.FLAG_ZOH_INPUT if zoh else 0
    io = torch.bfloat16 if dtype == "bf16" else torch.float32
    ws = "auto" if split else None
    assert mss.workspace_size(batch, dim, N, L, io) > 0
    inp = gen.scan_inputs(batch, dim, N, L, dtype, seed=700 + N, d_skip="normal")
    d = device_inputs(inp, DEV)
    dy, dl = gen.upstream_gradients(batch, dim, N, L, dtype, 701)
    h0 = np.random.default_rng(702).standard_normal((batch, dim, N)).astype(np.float32)
    h0_d, dy_d, dl_d = torch.from_numpy(h0).to(DEV), to_torch(dy, DEV), torch.from_numpy(dl).to(DEV)
    y_s, last_s, states = mss.scan_fwd_save(**d, initial_state=h0_d, flags=flags, workspace=ws)
    y, last = mss.scan_fwd(**d, initial_state=h0_d, flags=flags, workspace=ws)
    g_s = mss.scan_bwd(**d, dy=dy_d, dlast=dl_d, initial_state=h0_d, flags=flags, saved_states=states)
    g = mss.scan_bwd(**d, dy=dy_d, dlast=dl_d, initial_state=h0_d, flags=flags)
    torch.cuda.synchronize()
    assert mss.get_device_error() == 0
    assert states.numel() == mss.bwd_workspace_size(batch, dim, N, L, io, flags)
    assert torch.equal(y_s, y) and torch.equal(last_s, last)
    ref = oracle.scan_bwd(inp["u"].values, inp["delta"].values, inp["A"], inp["B"].values, inp["C"].values,
                          dy.values, D=inp["D"], z=inp["z"].values, delta_bias=inp["delta_bias"],
                          initial_state=h0.astype(np.float64), dlast=dl.astype(np.float64), zoh_input=zoh)
    _compare(g_s, ref, dtype, f"saved N={N}")
    if not split:
        for k in ("du", "ddelta", "dz", "dinit"):
            assert torch.equal(g_s[k], g[k]), k


def test_saved_states_refused_off_the_tiled_path():
    inp = gen.scan_inputs(2, 40, 2, 64, "bf16", seed=710)
    d = device_inputs(inp, DEV)
    with pytest.raises(mss.MssError) as e:
        mss.scan_fwd_save(**d)
    assert e.value.code == mss.ERR_PATH
    inp = gen.scan_inputs(2, 40, 16, 64, "bf16", seed=711)
    d = device_inputs(inp, DEV)
    with pytest.raises(mss.MssError) as e:
        mss.scan_fwd_save(**d, flags=mss.FLAG_SIMPLE)
    assert e.value.code == mss.ERR_PATH
