"""The library captures into CUDA graphs: no allocation, no host
synchronisation and no stream other than the caller's on the forward,
decode and backward paths.  A captured forward + decode token (and a
captured backward) replayed from the graph gives the eager results."""
import numpy as np
import pytest
import torch

import selective_state_space_mss_b200 as mss
from selective_state_space_mss_b200 import inputs as gen

from tests.helpers import device_inputs, to_torch

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _capture(fn, stream):
    stream.wait_stream(torch.cuda.current_stream(DEV))
    with torch.cuda.stream(stream):
        fn()  # the first call (lazy device queries) outside the capture
    torch.cuda.current_stream(DEV).wait_stream(stream)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    return g


@pytest.mark.parametrize("shape", [(2, 64, 16, 512), (1, 16, 16, 4096)], ids=["plain", "split"])
def test_forward_and_decode_replay_from_a_graph(shape):
    batch, dim, N, L = shape
    inp = gen.scan_inputs(batch, dim, N, L, "bf16", seed=600, d_skip="normal")
    d = device_inputs(inp, DEV)
    step = {k: to_torch(v, DEV) for k, v in gen.decode_step_inputs(batch, dim, N, "bf16", 601, 0).items()}
    ws = torch.empty(mss.workspace_size(batch, dim, N, L), dtype=torch.uint8, device=DEV)
    y, last, y1 = torch.empty_like(d["u"]), torch.empty(batch, dim, N, device=DEV), torch.empty_like(step["u"])

    def run():
        mss.scan_fwd(**d, y=y, last_state=last, workspace=ws if ws.numel() else None)
        mss.state_update(last, A=d["A"], D=d["D"], delta_bias=d["delta_bias"], y=y1, **step)

    run()
    torch.cuda.synchronize()
    y_e, last_e, y1_e = y.clone(), last.clone(), y1.clone()
    g = _capture(run, torch.cuda.Stream(DEV))
    for _ in range(3):
        y.zero_(); last.zero_(); y1.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(y, y_e) and torch.equal(last, last_e) and torch.equal(y1, y1_e)
    assert mss.get_device_error() == 0


def test_backward_replays_from_a_graph():
    batch, dim, N, L = 2, 64, 16, 512
    inp = gen.scan_inputs(batch, dim, N, L, "bf16", seed=610, d_skip="normal")
    d = device_inputs(inp, DEV)
    dy, _ = gen.upstream_gradients(batch, dim, N, L, "bf16", 611)
    dy = to_torch(dy, DEV)
    ws = torch.empty(mss.bwd_workspace_size(batch, dim, N, L), dtype=torch.uint8, device=DEV)
    out = {}

    def run():
        out.update(mss.scan_bwd(**d, dy=dy, workspace=ws))

    run()
    torch.cuda.synchronize()
    ref = {k: v.clone() for k, v in out.items() if v is not None}
    g = _capture(run, torch.cuda.Stream(DEV))
    g.replay()
    torch.cuda.synchronize()
    for k, v in ref.items():
        # per-token gradients are exact; the atomic sums agree to rounding
        if k in ("du", "ddelta", "dz", "dinit"):
            assert torch.equal(out[k], v), k
        else:
            np.testing.assert_allclose(out[k].cpu().numpy(), v.cpu().numpy(), rtol=1e-5, atol=1e-5, err_msg=k)
    assert mss.get_device_error() == 0
