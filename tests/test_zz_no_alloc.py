"""mss_scan_fwd_noalloc, the forward pass for callers that cannot allocate.

Callers without a device allocator of their own -- a C program that is only
handed its buffers, a plug-in inside a framework that owns all device memory,
a serving loop that must not allocate after start-up -- cannot pass the usual
workspace for a long-sequence split.  This entry point takes its split
scratch from a fixed array in the library image instead.  The test calls it
through the C ABI twice in a row, on different inputs that both take the
split (so stale contents left by the first call would show), and checks each
result against the workspace entry point within the bf16 parity tolerance.
It sits in a file of its own that pytest collects last.
"""
import ctypes

import pytest
import torch

import selective_state_space_mss_b200 as mss
from selective_state_space_mss_b200 import inputs as gen
from tests.helpers import assert_close, device_inputs, to_numpy

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _lib():
    lib = mss.load_library()
    vp, i64, i, u32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_uint
    lib.mss_scan_fwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, vp, vp, vp,
                                         i64, i64, i64, i64, i, u32, vp]
    lib.mss_scan_fwd_noalloc.restype = i
    lib.mss_scan_fwd_noalloc_scratch_bytes.argtypes = []
    lib.mss_scan_fwd_noalloc_scratch_bytes.restype = i64
    return lib


def _call_noalloc(lib, d, y, last, h0=None, flags=0):
    ptr = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    batch, dim, L = d["u"].shape
    N = d["A"].shape[1]
    dtype = 1 if d["u"].dtype == torch.bfloat16 else 0
    return lib.mss_scan_fwd_noalloc(
        ptr(d["u"]), ptr(d["delta"]), ptr(d["A"]), ptr(d["B"]), ptr(d["C"]), ptr(d["D"]), ptr(d["z"]),
        ptr(d["delta_bias"]), 1, ptr(h0), ptr(y), ptr(last), batch, dim, N, L, dtype, flags,
        ctypes.c_void_p(torch.cuda.current_stream(DEV).cuda_stream))


def test_noalloc_matches_the_workspace_path_on_two_calls_in_a_row():
    lib = _lib()
    limit = lib.mss_scan_fwd_noalloc_scratch_bytes()
    cases = [(1, 32, 16, 8192, 61, None), (2, 16, 16, 4096 + 64, 62, 63)]
    for batch, dim, N, L, seed, h0_seed in cases:
        need = mss.workspace_size(batch, dim, N, L, torch.bfloat16, device=DEV)
        assert 0 < need <= limit  # the split is taken and fits the fixed scratch
        inp = gen.scan_inputs(batch, dim, N, L, "bf16", seed=seed, d_skip="normal")
        d = device_inputs(inp, DEV)
        h0 = None
        if h0_seed is not None:
            h0 = torch.randn(batch, dim, N, generator=torch.Generator().manual_seed(h0_seed)).to(DEV)
        y_ref, last_ref = mss.scan_fwd(**d, initial_state=h0)  # workspace from PyTorch
        y = torch.empty_like(y_ref)
        last = torch.empty_like(last_ref)
        assert _call_noalloc(lib, d, y, last, h0) == 0
        torch.cuda.synchronize()
        assert mss.get_device_error() == 0
        assert_close(to_numpy(y), to_numpy(y_ref).astype("float64"), "bf16", f"{(batch, dim, N, L)} y")
        assert_close(to_numpy(last), to_numpy(last_ref).astype("float64"), "bf16",
                     f"{(batch, dim, N, L)} last_state")


def test_noalloc_without_a_split_and_in_fp32():
    """Calls that need no scratch (no split asked for; enough channels to
    fill the GPU: the array is not touched) and an fp32 call that does, each
    against the workspace entry point; the fp32 one also against the fp64
    oracle."""
    import oracle

    lib = _lib()
    cases = [("bf16", (1, 32, 16, 8192), mss.FLAG_NO_SPLIT, 0),
             ("bf16", (8, 2048, 16, 256), 0, 0),   # enough channels to fill the GPU: no split
             ("f32", (1, 16, 16, 4096), 0, 1)]
    for dtype, (batch, dim, N, L), flags, splits in cases:
        tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
        need = mss.workspace_size(batch, dim, N, L, tdt, flags=flags, device=DEV)
        assert (need > 0) == bool(splits)
        inp = gen.scan_inputs(batch, dim, N, L, dtype, seed=70 + L, d_skip="normal")
        d = device_inputs(inp, DEV)
        y_ref, last_ref = mss.scan_fwd(**d, flags=flags)
        y, last = torch.empty_like(y_ref), torch.empty_like(last_ref)
        assert _call_noalloc(lib, d, y, last, flags=flags) == 0
        torch.cuda.synchronize()
        assert mss.get_device_error() == 0
        what = f"{dtype} {(batch, dim, N, L)} flags={flags}"
        assert_close(to_numpy(y), to_numpy(y_ref).astype("float64"), dtype, f"{what} y")
        assert_close(to_numpy(last), to_numpy(last_ref).astype("float64"), dtype, f"{what} last_state")
        if dtype == "f32":
            yo, lo = oracle.scan_fwd(inp["u"].values, inp["delta"].values, inp["A"], inp["B"].values,
                                     inp["C"].values, D=inp["D"], z=inp["z"].values, delta_bias=inp["delta_bias"])
            assert_close(to_numpy(y), yo, dtype, f"{what} y vs oracle")
            assert_close(to_numpy(last), lo, dtype, f"{what} last_state vs oracle")
