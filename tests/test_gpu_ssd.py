"""GPU parity of the structured-state-space-duality (Mamba-2) forward pass
(mss_ssd_fwd) against the fp64 oracle (oracle.ssd_fwd, pinned to the Mamba-1
oracle, the semiseparable matrix and the chunked algorithm).  bf16 io, so the
bf16 tolerance of tests/helpers.py applies; the tensor-core operands (masked
scores, the carried state) round to bf16 inside the kernel as well."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_mss_b200 as mss
from selective_state_space_mss_b200 import inputs as gen

from tests.helpers import assert_close, to_numpy, to_torch

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _dev(inp, gate=True, with_D=True, with_bias=True):
    return dict(x=to_torch(inp["x"], DEV), dt=to_torch(inp["dt"], DEV), A=torch.from_numpy(inp["A"]).to(DEV),
                B=to_torch(inp["B"], DEV), C=to_torch(inp["C"], DEV),
                D=torch.from_numpy(inp["D"]).to(DEV) if with_D else None,
                z=to_torch(inp["z"], DEV) if gate else None,
                dt_bias=torch.from_numpy(inp["dt_bias"]).to(DEV) if with_bias else None)


def _ref(inp, gate=True, with_D=True, with_bias=True, h0=None):
    return oracle.ssd_fwd(inp["x"].values, inp["dt"].values, inp["A"], inp["B"].values, inp["C"].values,
                          D=inp["D"] if with_D else None, z=inp["z"].values if gate else None,
                          dt_bias=inp["dt_bias"] if with_bias else None, initial_state=h0)


# the tcgen05 kernel (N = 128; N = 64 runs the warp-level kernels either way)
# and the warp-level (mma.sync) kernels
KERNELS = {"tcgen05": 0, "warp": mss.SSD_FLAG_WARP_MMA}


@pytest.mark.parametrize("kernel", sorted(KERNELS))
@pytest.mark.parametrize("N", [64, 128])
@pytest.mark.parametrize("L", [64, 200, 512])
@pytest.mark.parametrize("G", [1, 2])
@pytest.mark.parametrize("chunks", ["parallel", "in-order"])
def test_ssd_matches_oracle(N, L, G, chunks, kernel):
    """Whole chunks, a ragged last chunk, one or two groups of heads; the
    chunk-parallel passes (with a workspace) and the in-order kernels."""
    inp = gen.ssd_inputs(2, L, 4, 64, G, N, seed=700 + L + N + G)
    y, last = mss.ssd_fwd(**_dev(inp), workspace="auto" if chunks == "parallel" else None, flags=KERNELS[kernel])
    torch.cuda.synchronize()
    assert mss.get_device_error() == 0
    y_ref, last_ref = _ref(inp)
    assert_close(to_numpy(y), y_ref, "bf16", f"N={N} L={L} G={G} y")
    assert_close(to_numpy(last), last_ref, "bf16", f"N={N} L={L} G={G} last_state")


@pytest.mark.parametrize("kernel", sorted(KERNELS))
def test_ssd_starting_state_and_chaining(kernel):
    f = KERNELS[kernel]
    inp = gen.ssd_inputs(2, 320, 4, 64, 1, 128, seed=720)
    h0 = np.random.default_rng(721).standard_normal((2, 4, 128, 64)).astype(np.float32) * 0.1
    d = _dev(inp)
    y_ref, last_ref = _ref(inp, h0=h0.astype(np.float64))
    for ws in ("auto", None):
        y, last = mss.ssd_fwd(**d, initial_state=torch.from_numpy(h0).to(DEV), workspace=ws, flags=f)
        torch.cuda.synchronize()
        assert_close(to_numpy(y), y_ref, "bf16", f"y from a starting state (workspace {ws})")
        assert_close(to_numpy(last), last_ref, "bf16", f"last_state from a starting state (workspace {ws})")
    # two calls chained through last_state equal one call
    part = lambda t0, t1: {k: (v[:, t0:t1].contiguous() if k in ("x", "dt", "B", "C", "z") else v)
                           for k, v in d.items()}
    y0, last0 = mss.ssd_fwd(**part(0, 128), flags=f)
    y1, last1 = mss.ssd_fwd(**part(128, 320), initial_state=last0, flags=f)
    y_all, last_all = mss.ssd_fwd(**d, flags=f)
    torch.cuda.synchronize()
    assert_close(to_numpy(torch.cat([y0, y1], dim=1)), to_numpy(y_all).astype(np.float64), "bf16", "chained y")
    assert_close(to_numpy(last1), to_numpy(last_all).astype(np.float64), "bf16", "chained state")


def test_ssd_workspace_only_when_it_pays():
    """Few (batch, head) pairs take the chunk-parallel passes, many the
    in-order kernel: up to about 115 pairs on 148 SMs for the warp-level
    in-order kernel, up to about 28 for the tcgen05 one (N = 128, one CTA
    per SM).  Each gives the oracle's result."""
    lib = mss.load_library()
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    w = mss.SSD_FLAG_WARP_MMA
    assert lib.mss_ssd_fwd_workspace_size_ex(1, 4096, 4, 64, 1, 128, w) > 0
    assert lib.mss_ssd_fwd_workspace_size_ex(4, 4096, sms, 64, 1, 128, w) == 0
    assert lib.mss_ssd_fwd_workspace_size(1, 4096, 4, 64, 1, 128) > 0
    assert lib.mss_ssd_fwd_workspace_size(1, 4096, 64, 64, 1, 128) == 0
    assert lib.mss_ssd_fwd_workspace_size(1, 4096, 64, 64, 1, 64) > 0
    assert lib.mss_ssd_fwd_workspace_size(1, 4096, 4, 64, 1, 64) > 0
    inp = gen.ssd_inputs(1, 1024, 2, 64, 1, 128, seed=735)
    y_ref, last_ref = _ref(inp)
    for f in (0, w):
        for ws in ("auto", None):
            y, last = mss.ssd_fwd(**_dev(inp), flags=f, workspace=ws)
            torch.cuda.synchronize()
            assert_close(to_numpy(y), y_ref, "bf16", f"few heads y (flags {f}, workspace {ws})")
            assert_close(to_numpy(last), last_ref, "bf16", f"few heads last_state (flags {f}, workspace {ws})")


@pytest.mark.parametrize("N", [64, 128])
def test_ssd_without_optional_inputs(N):
    inp = gen.ssd_inputs(1, 256, 2, 64, 1, N, seed=730)
    y, last = mss.ssd_fwd(**_dev(inp, gate=False, with_D=False, with_bias=False))
    torch.cuda.synchronize()
    y_ref, last_ref = _ref(inp, gate=False, with_D=False, with_bias=False)
    assert_close(to_numpy(y), y_ref, "bf16", "bare y")
    assert_close(to_numpy(last), last_ref, "bf16", "bare last_state")


@pytest.mark.parametrize("kernel", sorted(KERNELS))
@pytest.mark.parametrize("batch", [4, 1])
def test_ssd_workload_sampled_heads(batch, kernel):
    """The bench workload (4 x 4096 tokens, 64 heads of 64, N = 128) and one
    sequence of it, on each kernel (the warp-level kernels take the
    chunk-parallel passes for the single sequence): y and the final state of
    sampled (batch, head) pairs against the oracle."""
    f = KERNELS[kernel]
    s = dict(gen.SSD_SHAPES[gen.SSD_WORKLOAD], batch=batch)
    ws = mss.load_library().mss_ssd_fwd_workspace_size_ex(batch, s["seqlen"], s["nheads"], s["headdim"],
                                                           s["ngroups"], s["dstate"], f)
    assert (ws > 0) == (batch == 1 and f != 0)
    inp = gen.ssd_inputs(**s)
    y, last = mss.ssd_fwd(**_dev(inp), flags=f)
    torch.cuda.synchronize()
    assert mss.get_device_error() == 0
    yn, ln = to_numpy(y), to_numpy(last)
    rng = np.random.default_rng(740)
    for _ in range(6):
        b, h = int(rng.integers(s["batch"])), int(rng.integers(s["nheads"]))
        sub = {k: (v.values[b:b + 1, :, h:h + 1] if k in ("x", "z", "dt") else v)
               for k, v in inp.items() if k in ("x", "z", "dt")}
        y_ref, last_ref = oracle.ssd_fwd(sub["x"], sub["dt"], inp["A"][h:h + 1], inp["B"].values[b:b + 1],
                                         inp["C"].values[b:b + 1], D=inp["D"][h:h + 1], z=sub["z"],
                                         dt_bias=inp["dt_bias"][h:h + 1])
        assert_close(yn[b:b + 1, :, h:h + 1], y_ref, "bf16", f"y of (b={b}, h={h})")
        assert_close(ln[b:b + 1, h:h + 1], last_ref, "bf16", f"state of (b={b}, h={h})")


@pytest.mark.parametrize("kernel", sorted(KERNELS))
@pytest.mark.parametrize("N", [64, 128])
@pytest.mark.parametrize("L", [1, 63, 65, 127, 129])
@pytest.mark.parametrize("chunks", ["parallel", "in-order"])
def test_ssd_short_and_ragged_sequences(L, chunks, N, kernel):
    """One token, one token short of a chunk, one token past it (chunks of 64
    and of 128 tokens); every head its own group (G = H)."""
    inp = gen.ssd_inputs(1, L, 4, 64, 4, N, seed=750 + L)
    y, last = mss.ssd_fwd(**_dev(inp), workspace="auto" if chunks == "parallel" else None, flags=KERNELS[kernel])
    torch.cuda.synchronize()
    assert mss.get_device_error() == 0
    y_ref, last_ref = _ref(inp)
    assert_close(to_numpy(y), y_ref, "bf16", f"L={L} y")
    assert_close(to_numpy(last), last_ref, "bf16", f"L={L} last_state")


def test_ssd_empty_sequence_passes_the_state_on():
    inp = gen.ssd_inputs(2, 1, 4, 64, 1, 128, seed=760)
    d = {k: (v[:, :0].contiguous() if k in ("x", "dt", "B", "C", "z") else v) for k, v in _dev(inp).items()}
    h0 = torch.randn(2, 4, 128, 64, device=DEV)
    _, last = mss.ssd_fwd(**d, initial_state=h0)
    _, last0 = mss.ssd_fwd(**d)
    torch.cuda.synchronize()
    assert torch.equal(last, h0)
    assert torch.count_nonzero(last0) == 0


@pytest.mark.parametrize("kernel", sorted(KERNELS))
def test_ssd_second_workload_sampled_heads(kernel):
    """The second bench workload (2 x 4096 tokens, 80 heads of 64, N = 128) on
    each kernel: y and the final state of sampled (batch, head) pairs against
    the oracle."""
    s = dict(gen.SSD_SHAPES[gen.SSD_WORKLOAD_2])
    inp = gen.ssd_inputs(**s)
    y, last = mss.ssd_fwd(**_dev(inp), flags=KERNELS[kernel])
    torch.cuda.synchronize()
    assert mss.get_device_error() == 0
    yn, ln = to_numpy(y), to_numpy(last)
    rng = np.random.default_rng(741)
    for _ in range(4):
        b, h = int(rng.integers(s["batch"])), int(rng.integers(s["nheads"]))
        sub = {k: inp[k].values[b:b + 1, :, h:h + 1] for k in ("x", "z", "dt")}
        y_ref, last_ref = oracle.ssd_fwd(sub["x"], sub["dt"], inp["A"][h:h + 1], inp["B"].values[b:b + 1],
                                         inp["C"].values[b:b + 1], D=inp["D"][h:h + 1], z=sub["z"],
                                         dt_bias=inp["dt_bias"][h:h + 1])
        assert_close(yn[b:b + 1, :, h:h + 1], y_ref, "bf16", f"y of (b={b}, h={h})")
        assert_close(ln[b:b + 1, h:h + 1], last_ref, "bf16", f"state of (b={b}, h={h})")


@pytest.mark.parametrize("extra", [0, 5, 30], ids=["whole-waves", "short-tail", "long-tail"])
def test_ssd_tail_past_the_last_wave(extra):
    """N = 128 with a workspace: (batch, head) pairs past the tcgen05
    kernel's last full wave of CTAs (one per SM) go to the chunk-parallel
    passes when they are few; whole waves, or a long tail, stay on the
    tcgen05 kernel.  Each against the oracle, with a starting state."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    H = sms + extra
    lib = mss.load_library()
    ws = lib.mss_ssd_fwd_workspace_size(1, 256, H, 64, 1, 128)
    if extra == 5:
        # the chunk states of the 5 tail pairs only
        assert ws == lib.mss_ssd_fwd_workspace_size_ex(1, 256, 5, 64, 1, 128, mss.SSD_FLAG_WARP_MMA) > 0
    else:
        assert ws == 0
    inp = gen.ssd_inputs(1, 256, H, 64, 1, 128, seed=740 + extra)
    h0 = np.random.default_rng(741).standard_normal((1, H, 128, 64)).astype(np.float32) * 0.1
    y, last = mss.ssd_fwd(**_dev(inp), initial_state=torch.from_numpy(h0).to(DEV), workspace="auto")
    torch.cuda.synchronize()
    assert mss.get_device_error() == 0
    y_ref, last_ref = _ref(inp, h0=h0.astype(np.float64))
    assert_close(to_numpy(y), y_ref, "bf16", f"{extra} past the wave: y")
    assert_close(to_numpy(last), last_ref, "bf16", f"{extra} past the wave: last_state")
