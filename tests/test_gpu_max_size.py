"""The largest tensors: more than 2^31 elements in u, delta, z and y
(1 x 16400 channels x 131072 tokens, 4.3 GB per bf16 tensor), so that every
element offset past 2^31 must be formed in 64 bits.  The forward pass and
the backward pass run over the whole tensors; the channels the oracle checks
are the last ones of the tensor (the largest offsets), one in the middle and
the first, read back from the device with their inputs.  The backward pass's
per-channel gradients (du, ddelta, dz, dA, dD, dbias) are checked; dB and dC
sum over every channel, which the sampled oracle cannot.  The decode step
runs on a state of 2^31 elements and the SSD layer on x, z and y of 2^31
elements each, checked on sampled rows and heads in the same way."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_mss_b200 as mss
from selective_state_space_mss_b200 import inputs as gen
from tests.helpers import assert_close, to_numpy

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)
BATCH, DIM, N, L = 1, 16400, 16, 131072
SAMPLE = (0, DIM // 2, DIM - 17, DIM - 2, DIM - 1)


@pytest.fixture(scope="module")
def big():
    assert BATCH * DIM * L > 2 ** 31
    torch.cuda.empty_cache()  # blocks other tests left in torch's cache
    free, _ = torch.cuda.mem_get_info(DEV)
    if free < 60 * 2 ** 30:
        pytest.skip(f"needs about 60 GB of free device memory, {free / 2**30:.0f} GB free")
    d = gen.device_scan_inputs(BATCH, DIM, N, L, seed=1101, device=DEV)
    yield d
    del d
    torch.cuda.empty_cache()


def _host(t, ch):
    return t[:, ch:ch + 1].float().cpu().numpy()


def test_forward_beyond_2_to_31_elements(big):
    y, last = mss.scan_fwd(**big)
    torch.cuda.synchronize()
    assert mss.get_device_error() == 0
    B, C = big["B"].float().cpu().numpy(), big["C"].float().cpu().numpy()
    A, D, bias = (big[k].cpu().numpy() for k in ("A", "D", "delta_bias"))
    for ch in SAMPLE:
        y_ref, s_ref = oracle.scan_fwd(_host(big["u"], ch), _host(big["delta"], ch), A[ch:ch + 1], B, C,
                                       D=D[ch:ch + 1], z=_host(big["z"], ch), delta_bias=bias[ch:ch + 1])
        assert_close(to_numpy(y[:, ch:ch + 1]), y_ref, "bf16", f"channel {ch} y")
        assert_close(to_numpy(last[:, ch:ch + 1]), s_ref, "bf16", f"channel {ch} last_state")
    del y, last


def test_backward_beyond_2_to_31_elements(big):
    g = torch.Generator(device=DEV)
    g.manual_seed(1102)
    dy = torch.randn(BATCH, DIM, L, generator=g, device=DEV).to(torch.bfloat16)
    g_out = mss.scan_bwd(**big, dy=dy)
    torch.cuda.synchronize()
    assert mss.get_device_error() == 0
    B, C = big["B"].float().cpu().numpy(), big["C"].float().cpu().numpy()
    A, D, bias = (big[k].cpu().numpy() for k in ("A", "D", "delta_bias"))
    for ch in SAMPLE:
        ref = oracle.scan_bwd(_host(big["u"], ch), _host(big["delta"], ch), A[ch:ch + 1], B, C, _host(dy, ch),
                              D=D[ch:ch + 1], z=_host(big["z"], ch), delta_bias=bias[ch:ch + 1])
        for k in ("du", "ddelta", "dz"):
            assert_close(to_numpy(g_out[k][:, ch:ch + 1]), ref[k], "bf16", f"channel {ch} {k}")
        for k in ("dA", "dD", "dbias"):
            assert_close(to_numpy(g_out[k][ch:ch + 1]), ref[k], "bf16", f"channel {ch} {k}")
    del g_out, dy


def test_decode_state_beyond_2_to_31_elements():
    # state [4096, 32768, 16] fp32: 2^31 elements (8.6 GB), one token
    batch, dim, n = 4096, 32768, 16
    torch.cuda.empty_cache()  # blocks other tests left in torch's cache
    free, _ = torch.cuda.mem_get_info(DEV)
    if free < 24 * 2 ** 30:
        pytest.skip(f"needs about 24 GB of free device memory, {free / 2**30:.0f} GB free")
    g = torch.Generator(device=DEV)
    g.manual_seed(1103)
    state = torch.randn(batch, dim, n, generator=g, device=DEV)
    assert state.numel() >= 2 ** 31
    step = {k: torch.randn(batch, dim, generator=g, device=DEV).to(torch.bfloat16) for k in ("u", "z")}
    step["delta"] = (0.1 * torch.randn(batch, dim, generator=g, device=DEV)).to(torch.bfloat16)
    B = torch.randn(batch, n, generator=g, device=DEV).to(torch.bfloat16)
    C = torch.randn(batch, n, generator=g, device=DEV).to(torch.bfloat16)
    A, D, bias = gen.channel_params(dim, n, "normal", 1104)
    rows = ((0, 0), (batch // 2, dim // 3), (batch - 1, dim - 1), (batch - 1, dim - 129))
    before = {r: state[r[0], r[1]].double().cpu().numpy() for r in rows}
    y = mss.state_update(state, step["u"], step["delta"], torch.from_numpy(A).to(DEV), B, C,
                         D=torch.from_numpy(D).to(DEV), z=step["z"], delta_bias=torch.from_numpy(bias).to(DEV))
    torch.cuda.synchronize()
    assert mss.get_device_error() == 0
    for (b, d) in rows:
        one = lambda t: t[b:b + 1, d:d + 1].float().cpu().numpy()
        y_ref, s_ref = oracle.state_update(before[(b, d)].reshape(1, 1, n).copy(), one(step["u"]), one(step["delta"]),
                                           A[d:d + 1], B[b:b + 1].float().cpu().numpy(),
                                           C[b:b + 1].float().cpu().numpy(), D=D[d:d + 1], z=one(step["z"]),
                                           delta_bias=bias[d:d + 1])
        assert_close(to_numpy(y[b:b + 1, d:d + 1]), y_ref, "bf16", f"row {b},{d} y")
        assert_close(to_numpy(state[b:b + 1, d:d + 1]), s_ref, "bf16", f"row {b},{d} state")
    del state, step, y


def test_ssd_beyond_2_to_31_elements():
    # x, z, y [1, 131072, 256, 64] bf16: 2^31 elements each
    batch, L, H, P, G, NS = 1, 131072, 256, 64, 1, 128
    torch.cuda.empty_cache()  # blocks other tests left in torch's cache
    free, _ = torch.cuda.mem_get_info(DEV)
    if free < 40 * 2 ** 30:
        pytest.skip(f"needs about 40 GB of free device memory, {free / 2**30:.0f} GB free")
    g = torch.Generator(device=DEV)
    g.manual_seed(1105)
    x = torch.randn(batch, L, H, P, generator=g, device=DEV).to(torch.bfloat16)
    z = torch.randn(batch, L, H, P, generator=g, device=DEV).to(torch.bfloat16)
    assert x.numel() >= 2 ** 31
    dt = (0.1 * torch.randn(batch, L, H, generator=g, device=DEV)).to(torch.bfloat16)
    B = (torch.randn(batch, L, G, NS, generator=g, device=DEV) / NS ** 0.5).to(torch.bfloat16)
    C = (torch.randn(batch, L, G, NS, generator=g, device=DEV) / NS ** 0.5).to(torch.bfloat16)
    rng = np.random.default_rng(1106)
    A = -np.exp(rng.uniform(0.0, np.log(16.0), H)).astype(np.float32)
    D = (1.0 + 0.1 * rng.standard_normal(H)).astype(np.float32)
    steps = np.exp(rng.uniform(np.log(1e-3), np.log(1e-1), H))
    bias = np.log(np.expm1(steps)).astype(np.float32)
    y, last = mss.ssd_fwd(x, dt, torch.from_numpy(A).to(DEV), B, C, D=torch.from_numpy(D).to(DEV), z=z,
                          dt_bias=torch.from_numpy(bias).to(DEV))
    torch.cuda.synchronize()
    assert mss.get_device_error() == 0
    Bh, Ch = B.float().cpu().numpy(), C.float().cpu().numpy()
    for h in (0, H - 1):
        xh = x[:, :, h:h + 1].float().cpu().numpy()
        zh = z[:, :, h:h + 1].float().cpu().numpy()
        dth = dt[:, :, h:h + 1].float().cpu().numpy()
        y_ref, s_ref = oracle.ssd_fwd(xh, dth, A[h:h + 1], Bh, Ch, D=D[h:h + 1], z=zh, dt_bias=bias[h:h + 1])
        assert_close(to_numpy(y[:, :, h:h + 1]), y_ref, "bf16", f"head {h} y")
        assert_close(to_numpy(last[:, h:h + 1]), s_ref, "bf16", f"head {h} last_state")
    del x, z, y
