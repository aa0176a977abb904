"""A seeded random sweep of the forward pass (on device buffers, on host
buffers, and with the causal convolution in front), the backward pass, the
decode step (plain and with the convolution) and the
structured-state-space-duality (Mamba-2) forward pass against the fp64
oracle.

Each case draws its sizes (odd channel counts; sequence lengths that are
multiples of the 16-byte row unit, which the tiled kernels take, or ragged,
which the scalar kernels take), dstate, io type, flags (zero-order-hold
input, general A, scalar kernel, pair kernel, no split), optional inputs
(gate, skip, bias, softplus), A recipe, starting state and workspace, so
that combinations the fixed parametrizations do not list still meet the
oracle.  The draws are fixed by the case index; the tolerances are those of
tests/helpers.py.
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
N_FWD, N_BWD, N_CONV, N_DEC, N_SSD, N_HOST, N_DEC_CONV = 320, 96, 64, 64, 64, 24, 32
KEYS = ("du", "ddelta", "dz", "dA", "dB", "dC", "dD", "dbias", "dinit")


def _draw(i, max_len):
    rng = np.random.default_rng([2026, 12, i])
    c = {}
    c["dtype"] = str(rng.choice(["f32", "bf16"]))
    c["N"] = int(rng.choice([1, 2, 4, 8, 16]))
    c["batch"] = int(rng.integers(1, 4))
    c["dim"] = int(rng.integers(1, 72))
    unit = 8 if c["dtype"] == "bf16" else 4  # tokens per 16 bytes of a row
    if rng.random() < 0.6:
        c["L"] = int(rng.integers(1, max_len // unit + 1)) * unit
    else:
        c["L"] = int(rng.integers(1, max_len + 1))
    flags = 0
    if rng.random() < 0.3:
        flags |= mss.FLAG_ZOH_INPUT
    if rng.random() < 0.25:
        flags |= mss.FLAG_GENERAL_A
    if rng.random() < 0.1:
        flags |= mss.FLAG_SIMPLE
    if rng.random() < 0.2:
        flags |= mss.FLAG_NO_SPLIT
    c["flags"] = flags
    c["pair"] = bool(rng.random() < 0.2)
    c["gate"] = bool(rng.random() < 0.8)
    c["softplus"] = bool(rng.random() < 0.85)
    c["with_D"] = bool(rng.random() < 0.8)
    c["with_bias"] = bool(rng.random() < 0.8) and c["softplus"]
    c["a_init"] = str(rng.choice(list(gen.A_RECIPES)))
    c["h0"] = bool(rng.random() < 0.5)
    c["workspace"] = bool(rng.random() < 0.7)
    c["seed"] = 3000 + i
    return c


def _inputs(c):
    inp = gen.scan_inputs(c["batch"], c["dim"], c["N"], c["L"], c["dtype"], seed=c["seed"], d_skip="normal",
                          a_init=c["a_init"])
    if not c["softplus"]:
        # step sizes that stay positive without softplus
        inp["delta"] = gen._store((np.abs(inp["delta"].values) * 0.1 + 0.01).astype(np.float32), c["dtype"])
    h0 = None
    if c["h0"]:
        h0 = np.random.default_rng(c["seed"] + 1).standard_normal((c["batch"], c["dim"], c["N"])).astype(np.float32)
    return inp, h0


def _id(i, max_len):
    c = _draw(i, max_len)
    return f"{i}-{c['dtype']}-b{c['batch']}d{c['dim']}n{c['N']}l{c['L']}-f{c['flags']:x}"


@pytest.mark.parametrize("i", range(N_FWD), ids=lambda i: _id(i, 720))
def test_forward_random_case(i):
    c = _draw(i, 720)
    inp, h0 = _inputs(c)
    d = device_inputs(inp, DEV, with_z=c["gate"], with_D=c["with_D"], with_bias=c["with_bias"])
    flags = c["flags"] | (mss.FLAG_PAIR_LANES if c["pair"] else 0)
    y, last = mss.scan_fwd(**d, softplus=c["softplus"],
                           initial_state=None if h0 is None else torch.from_numpy(h0).to(DEV),
                           workspace="auto" if c["workspace"] else None, flags=flags)
    torch.cuda.synchronize()
    assert mss.get_device_error() == 0
    y_ref, last_ref = oracle.scan_fwd(inp["u"].values, inp["delta"].values, inp["A"], inp["B"].values,
                                      inp["C"].values, D=inp["D"] if c["with_D"] else None,
                                      z=inp["z"].values if c["gate"] else None,
                                      delta_bias=inp["delta_bias"] if c["with_bias"] else None,
                                      softplus_flag=c["softplus"],
                                      initial_state=None if h0 is None else h0.astype(np.float64),
                                      zoh_input=bool(c["flags"] & mss.FLAG_ZOH_INPUT))
    assert_close(to_numpy(y), y_ref, c["dtype"], f"case {i} y")
    assert_close(to_numpy(last), last_ref, c["dtype"], f"case {i} last_state")


@pytest.mark.parametrize("i", range(N_BWD), ids=lambda i: _id(1000 + i, 400))
def test_backward_random_case(i):
    c = _draw(1000 + i, 400)
    flags = c["flags"] & (mss.FLAG_ZOH_INPUT | mss.FLAG_GENERAL_A | mss.FLAG_SIMPLE)
    inp, h0 = _inputs(c)
    d = device_inputs(inp, DEV, with_z=c["gate"], with_D=c["with_D"], with_bias=c["with_bias"])
    dy, dl = gen.upstream_gradients(c["batch"], c["dim"], c["N"], c["L"], c["dtype"], c["seed"] + 2)
    h0_d = None if h0 is None else torch.from_numpy(h0).to(DEV)
    g = mss.scan_bwd(**d, dy=to_torch(dy, DEV), dlast=torch.from_numpy(dl).to(DEV), softplus=c["softplus"],
                     initial_state=h0_d, flags=flags)
    torch.cuda.synchronize()
    assert mss.get_device_error() == 0
    ref = oracle.scan_bwd(inp["u"].values, inp["delta"].values, inp["A"], inp["B"].values, inp["C"].values,
                          dy.values, D=inp["D"] if c["with_D"] else None,
                          z=inp["z"].values if c["gate"] else None,
                          delta_bias=inp["delta_bias"] if c["with_bias"] else None,
                          softplus_flag=c["softplus"],
                          initial_state=None if h0 is None else h0.astype(np.float64),
                          dlast=dl.astype(np.float64), zoh_input=bool(flags & mss.FLAG_ZOH_INPUT))
    for k in KEYS:
        if ref.get(k) is None or g.get(k) is None:
            continue
        assert_close(to_numpy(g[k]), ref[k], c["dtype"], f"case {i} {k}")
    # the training-step form (states stored by the forward pass) where the
    # tiled kernels take the call
    try:
        _, _, states = mss.scan_fwd_save(**d, softplus=c["softplus"], initial_state=h0_d, flags=flags)
    except mss.MssError as e:
        assert e.code == mss.ERR_PATH
        return
    g2 = mss.scan_bwd(**d, dy=to_torch(dy, DEV), dlast=torch.from_numpy(dl).to(DEV), softplus=c["softplus"],
                      initial_state=h0_d, flags=flags, saved_states=states)
    torch.cuda.synchronize()
    assert mss.get_device_error() == 0
    for k in KEYS:
        if ref.get(k) is None or g2.get(k) is None:
            continue
        assert_close(to_numpy(g2[k]), ref[k], c["dtype"], f"case {i} saved-states {k}")


@pytest.mark.parametrize("i", range(N_CONV), ids=lambda i: _id(2000 + i, 600))
def test_conv_forward_random_case(i):
    c = _draw(2000 + i, 600)
    rng = np.random.default_rng([2026, 13, i])
    K = int(rng.integers(1, 5))
    flags = c["flags"] & (mss.FLAG_ZOH_INPUT | mss.FLAG_GENERAL_A | mss.FLAG_SIMPLE | mss.FLAG_NO_SPLIT)
    inp, h0 = _inputs(c)
    cw, cb = gen.conv_params(c["dim"], K, c["seed"] + 3)
    cs = gen.conv_state(c["batch"], c["dim"], K, c["dtype"], c["seed"] + 4) if (K > 1 and rng.random() < 0.6) \
        else None
    d = device_inputs(inp, DEV, with_z=c["gate"], with_D=c["with_D"], with_bias=c["with_bias"])
    y, last, cs_out = mss.scan_fwd_conv(d["u"], torch.from_numpy(cw).to(DEV), d["delta"], d["A"], d["B"], d["C"],
                                        conv_b=torch.from_numpy(cb).to(DEV),
                                        conv_state=None if cs is None else to_torch(cs, DEV), D=d["D"], z=d["z"],
                                        delta_bias=d["delta_bias"], softplus=c["softplus"],
                                        initial_state=None if h0 is None else torch.from_numpy(h0).to(DEV),
                                        workspace="auto" if c["workspace"] else None, flags=flags)
    torch.cuda.synchronize()
    assert mss.get_device_error() == 0
    y_ref, last_ref, cs_ref = oracle.scan_fwd_conv(
        inp["u"].values, cw, inp["delta"].values, inp["A"], inp["B"].values, inp["C"].values, conv_b=cb,
        conv_state=None if cs is None else cs.values, D=inp["D"] if c["with_D"] else None,
        z=inp["z"].values if c["gate"] else None, delta_bias=inp["delta_bias"] if c["with_bias"] else None,
        softplus_flag=c["softplus"], initial_state=None if h0 is None else h0.astype(np.float64),
        zoh_input=bool(flags & mss.FLAG_ZOH_INPUT))
    assert_close(to_numpy(y), y_ref, c["dtype"], f"case {i} K={K} y")
    assert_close(to_numpy(last), last_ref, c["dtype"], f"case {i} K={K} last_state")
    if K > 1:
        assert_close(to_numpy(cs_out), cs_ref, c["dtype"], f"case {i} K={K} conv_state")


@pytest.mark.parametrize("i", range(N_DEC))
def test_decode_random_case(i):
    rng = np.random.default_rng([2026, 14, i])
    dtype = str(rng.choice(["f32", "bf16"]))
    N = int(rng.choice([1, 2, 4, 8, 16]))
    batch = int(rng.integers(1, 5))
    # half the cases on whole tiles of the staged kernel (2048 / N channels)
    dim = int(rng.integers(1, 4)) * (2048 // N) if rng.random() < 0.5 else int(rng.integers(1, 300))
    zoh = bool(rng.random() < 0.3)
    gate, softplus = bool(rng.random() < 0.8), bool(rng.random() < 0.85)
    with_D, with_bias = bool(rng.random() < 0.8), bool(rng.random() < 0.8) and softplus
    seed = 4000 + i
    A = gen.a_matrix(dim, N, str(rng.choice(list(gen.A_RECIPES))), seed)
    _, D, bias = gen.channel_params(dim, N, "normal", seed)
    h0 = gen.initial_state(batch, dim, N, seed + 1, "normal")
    state = torch.from_numpy(h0.copy()).to(DEV)
    ref_state = h0.astype(np.float64)
    Ad, Dd, bd = (torch.from_numpy(x).to(DEV) for x in (A, D, bias))
    for t in range(4):
        s = gen.decode_step_inputs(batch, dim, N, dtype, seed + 2, t)
        if not softplus:
            s["delta"] = gen._store((np.abs(s["delta"].values) * 0.1 + 0.01).astype(np.float32), dtype)
        y = mss.state_update(state, to_torch(s["u"], DEV), to_torch(s["delta"], DEV), Ad, to_torch(s["B"], DEV),
                             to_torch(s["C"], DEV), D=Dd if with_D else None,
                             z=to_torch(s["z"], DEV) if gate else None, delta_bias=bd if with_bias else None,
                             softplus=softplus, flags=mss.FLAG_ZOH_INPUT if zoh else 0)
        y_ref, ref_state = oracle.state_update(ref_state, s["u"].values, s["delta"].values, A, s["B"].values,
                                               s["C"].values, D=D if with_D else None,
                                               z=s["z"].values if gate else None,
                                               delta_bias=bias if with_bias else None, softplus_flag=softplus,
                                               zoh_input=zoh)
        torch.cuda.synchronize()
        assert_close(to_numpy(y), y_ref, dtype, f"case {i} step {t} y")
    assert_close(to_numpy(state), ref_state, dtype, f"case {i} state")
    assert mss.get_device_error() == 0


@pytest.mark.parametrize("i", range(N_SSD))
def test_ssd_random_case(i):
    rng = np.random.default_rng([2026, 15, i])
    batch = int(rng.integers(1, 3))
    L = int(rng.integers(1, 5)) * 128 if rng.random() < 0.4 else int(rng.integers(1, 600))
    G = int(rng.choice([1, 2]))
    H = G * int(rng.integers(1, 4))
    N = int(rng.choice([64, 128]))
    flags = mss.SSD_FLAG_WARP_MMA if rng.random() < 0.3 else 0
    gate, with_D, with_bias = (bool(rng.random() < 0.8) for _ in range(3))
    workspace = "auto" if rng.random() < 0.5 else None
    inp = gen.ssd_inputs(batch, L, H, 64, G, N, seed=5000 + i)
    h0 = (np.random.default_rng(5100 + i).standard_normal((batch, H, N, 64)).astype(np.float32) * 0.1
          if rng.random() < 0.5 else None)
    y, last = mss.ssd_fwd(to_torch(inp["x"], DEV), to_torch(inp["dt"], DEV), torch.from_numpy(inp["A"]).to(DEV),
                          to_torch(inp["B"], DEV), to_torch(inp["C"], DEV),
                          D=torch.from_numpy(inp["D"]).to(DEV) if with_D else None,
                          z=to_torch(inp["z"], DEV) if gate else None,
                          dt_bias=torch.from_numpy(inp["dt_bias"]).to(DEV) if with_bias else None,
                          initial_state=None if h0 is None else torch.from_numpy(h0).to(DEV),
                          workspace=workspace, flags=flags)
    torch.cuda.synchronize()
    assert mss.get_device_error() == 0
    y_ref, last_ref = oracle.ssd_fwd(inp["x"].values, inp["dt"].values, inp["A"], inp["B"].values, inp["C"].values,
                                     D=inp["D"] if with_D else None, z=inp["z"].values if gate else None,
                                     dt_bias=inp["dt_bias"] if with_bias else None,
                                     initial_state=None if h0 is None else h0.astype(np.float64))
    what = f"case {i} b{batch} L{L} H{H} G{G} N{N} flags {flags}"
    # The products run on bf16 operands (the masked scores, the w-scaled x,
    # the state read by the next chunk), so an output's rounding error scales
    # with the sum of the absolute values of its products, not with the
    # output, which can cancel: without the skip term and with small steps
    # y is a small difference of larger terms.  That sum is the same pass
    # with every input in absolute value (the decays are positive) and the
    # gate's magnitude applied afterwards.
    y_abs, last_abs = oracle.ssd_fwd(np.abs(inp["x"].values), inp["dt"].values, inp["A"], np.abs(inp["B"].values),
                                     np.abs(inp["C"].values), D=np.abs(inp["D"]) if with_D else None,
                                     dt_bias=inp["dt_bias"] if with_bias else None,
                                     initial_state=None if h0 is None else np.abs(h0).astype(np.float64))
    if gate:
        zz = inp["z"].values.astype(np.float64)
        y_abs = y_abs * np.abs(zz / (1.0 + np.exp(-zz)))
    _assert_within_products(to_numpy(y), y_ref, y_abs, what + " y")
    _assert_within_products(to_numpy(last), last_ref, last_abs, what + " last_state")


@pytest.mark.parametrize("i", range(N_HOST), ids=lambda i: _id(3000 + i, 600))
def test_host_forward_random_case(i):
    c = _draw(3000 + i, 600)
    flags = c["flags"] & (mss.FLAG_ZOH_INPUT | mss.FLAG_GENERAL_A | mss.FLAG_SIMPLE | mss.FLAG_NO_SPLIT)
    inp, h0 = _inputs(c)
    cpu = torch.device("cpu")
    pin = c["workspace"]  # pinned or pageable host memory

    def host(t):
        t = to_torch(t, cpu) if not isinstance(t, np.ndarray) else torch.from_numpy(t)
        return t.pin_memory() if pin else t

    y, last = mss.scan_fwd_host(host(inp["u"]), host(inp["delta"]), host(inp["A"]), host(inp["B"]), host(inp["C"]),
                                D=host(inp["D"]) if c["with_D"] else None,
                                z=host(inp["z"]) if c["gate"] else None,
                                delta_bias=host(inp["delta_bias"]) if c["with_bias"] else None,
                                softplus=c["softplus"], initial_state=None if h0 is None else host(h0),
                                flags=flags, device=DEV)
    torch.cuda.synchronize()
    assert mss.get_device_error() == 0
    y_ref, last_ref = oracle.scan_fwd(inp["u"].values, inp["delta"].values, inp["A"], inp["B"].values,
                                      inp["C"].values, D=inp["D"] if c["with_D"] else None,
                                      z=inp["z"].values if c["gate"] else None,
                                      delta_bias=inp["delta_bias"] if c["with_bias"] else None,
                                      softplus_flag=c["softplus"],
                                      initial_state=None if h0 is None else h0.astype(np.float64),
                                      zoh_input=bool(flags & mss.FLAG_ZOH_INPUT))
    assert_close(to_numpy(y), y_ref, c["dtype"], f"case {i} y")
    assert_close(to_numpy(last), last_ref, c["dtype"], f"case {i} last_state")


@pytest.mark.parametrize("i", range(N_DEC_CONV))
def test_decode_conv_random_case(i):
    rng = np.random.default_rng([2026, 16, i])
    dtype = str(rng.choice(["f32", "bf16"]))
    N = int(rng.choice([1, 2, 4, 8, 16]))
    batch = int(rng.integers(1, 4))
    dim = int(rng.integers(1, 3)) * (2048 // N) if rng.random() < 0.5 else int(rng.integers(1, 200))
    K = int(rng.integers(1, 5))
    zoh = bool(rng.random() < 0.3)
    gate, with_D = bool(rng.random() < 0.8), bool(rng.random() < 0.8)
    seed = 6000 + i
    A, D, bias = gen.channel_params(dim, N, "normal", seed, str(rng.choice(list(gen.A_RECIPES))))
    cw, cb = gen.conv_params(dim, K, seed + 1)
    h0 = gen.initial_state(batch, dim, N, seed + 2, "normal")
    state = torch.from_numpy(h0.copy()).to(DEV)
    ref_state = h0.astype(np.float64)
    cs_ref = np.zeros((batch, dim, 0))
    cs = None
    if K > 1:
        cs0 = gen.conv_state(batch, dim, K, dtype, seed + 3)
        cs = to_torch(cs0, DEV).clone()
        cs_ref = cs0.values.astype(np.float64).copy()
    Ad, Dd, bd, cwd, cbd = (torch.from_numpy(x).to(DEV) for x in (A, D, bias, cw, cb))
    for t in range(3):
        s = gen.decode_step_inputs(batch, dim, N, dtype, seed + 4, t)
        y = mss.state_update_conv(state, cs, to_torch(s["u"], DEV), cwd, to_torch(s["delta"], DEV), Ad,
                                  to_torch(s["B"], DEV), to_torch(s["C"], DEV), conv_b=cbd,
                                  D=Dd if with_D else None, z=to_torch(s["z"], DEV) if gate else None,
                                  delta_bias=bd, flags=mss.FLAG_ZOH_INPUT if zoh else 0)
        y_ref, ref_state, cs_ref = oracle.state_update_conv(
            ref_state, cs_ref, s["u"].values, cw, s["delta"].values, A, s["B"].values, s["C"].values, conv_b=cb,
            D=D if with_D else None, z=s["z"].values if gate else None, delta_bias=bias, zoh_input=zoh)
        torch.cuda.synchronize()
        assert_close(to_numpy(y), y_ref, dtype, f"case {i} K={K} step {t} y")
    assert_close(to_numpy(state), ref_state, dtype, f"case {i} K={K} state")
    if K > 1:
        assert_close(to_numpy(cs), cs_ref, dtype, f"case {i} K={K} conv_state")
    assert mss.get_device_error() == 0


def _assert_within_products(got, ref, scale, what):
    """|got - ref| <= 2^-7 (sum of |products|) + 2^-8 |ref|: a few bf16
    operand roundings (2^-9 each) of every product, plus the bf16 output."""
    got, ref, scale = (np.asarray(a, dtype=np.float64) for a in (got, ref, scale))
    assert got.shape == ref.shape
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    bound = 2.0 ** -7 * scale + 2.0 ** -8 * np.abs(ref)
    bad = np.abs(got - ref) > bound
    if np.any(bad):
        k = np.unravel_index(np.argmax(np.abs(got - ref) / np.maximum(bound, 1e-300)), got.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} of {got.size} elements out of bound; worst at {k}: "
                             f"got {got[k]!r}, ref {ref[k]!r}, bound {bound[k]!r}")
