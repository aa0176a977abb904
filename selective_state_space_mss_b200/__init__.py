"""B200-native selective scan (S6): thin Python binding over libmss.so.

Argument marshalling only.  Every step of the forward pass and of the decode
update runs in the CUDA kernels of libmss.so; PyTorch supplies device memory
and streams.  There is no fallback: if the library is missing or a tensor is
not on a CUDA device, the call raises.

    y, last_state = scan_fwd(u, delta, A, B, C, D=D, z=z, delta_bias=bias)
    y = state_update(state, u, delta, A, B, C, D=D, z=z, delta_bias=bias)

Layouts (C-contiguous): u, delta, z, y [batch, dim, L]; B, C [batch, N, L];
A [dim, N] float32; D, delta_bias [dim] float32; last_state [batch, dim, N]
float32.  Decode: state [batch, dim, N] float32 (updated in place); u, delta,
z, y [batch, dim]; B, C [batch, N].  u, delta, z, B, C share one dtype,
float32 or bfloat16, which is also the dtype of y.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

__all__ = ["scan_fwd", "scan_fwd_host", "scan_fwd_conv", "scan_bwd", "ssd_fwd", "bwd_workspace_size", "state_update", "state_update_conv",
           "get_device_error", "probe_pipe_rates",
           "library_path", "workspace_size",
           "FLAG_GENERAL_A", "FLAG_SIMPLE", "FLAG_NO_SPLIT", "FLAG_ZOH_INPUT", "FLAG_SELFTEST_TIMEOUT",
           "ERR_DEVICE_TIMEOUT", "ERR_FLAGS", "SSD_FLAG_WARP_MMA", "MssError", "load_library"]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libmss.so")

DTYPE_F32 = 0
DTYPE_BF16 = 1
FLAG_GENERAL_A = 0x1
FLAG_SIMPLE = 0x2
FLAG_NO_SPLIT = 0x4
FLAG_ZOH_INPUT = 0x8  # zero-order-hold input matrix (e^{Delta A} - 1)/A * B instead of Delta * B
FLAG_SELFTEST_TIMEOUT = 0x10  # the tiled kernel's bounded wait gives up on purpose (failure-path tests)
FLAG_SAVED_STATES = 0x20  # scan_bwd: the workspace holds the states scan_fwd_save stored
FLAG_PAIR_LANES = 0x40  # forward: the two-lanes-per-channel kernel where the four-lane one would run (fp32 io; bf16 io on grids of at most 384 units of 16 channels)
ERR_PATH = -12
ERR_FLAGS = -8
SSD_FLAG_WARP_MMA = 0x1  # ssd_fwd: the warp-level (mma.sync) kernels instead of the tcgen05 one
ERR_DEVICE_TIMEOUT = -7

_lib = None
_lock = threading.Lock()


class MssError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what} failed: {_strerror(code)} (code {code})")


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load libmss.so (built in-tree by __graft_entry__.build() or
    ``python -m selective_state_space_mss_b200.build``)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH):
                raise RuntimeError(
                    f"{_LIB_PATH} is not built; run `python -m selective_state_space_mss_b200.build`")
            lib = ctypes.CDLL(_LIB_PATH)
            vp, fp, i64, i, u32 = (ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                   ctypes.c_int, ctypes.c_uint)
            lib.mss_scan_fwd_ex.argtypes = [vp, vp, fp, vp, vp, fp, vp, fp, i, vp, fp,
                                            i64, i64, i64, i64, i, u32, vp]
            lib.mss_scan_fwd_ex.restype = i
            lib.mss_scan_fwd.argtypes = [vp, vp, fp, vp, vp, fp, vp, fp, i, vp, fp,
                                         i64, i64, i64, i64, i, vp]
            lib.mss_scan_fwd.restype = i
            lib.mss_scan_fwd_ex2.argtypes = [vp, vp, fp, vp, vp, fp, vp, fp, i, fp, vp, fp,
                                             i64, i64, i64, i64, i, u32, vp, i64, vp]
            lib.mss_scan_fwd_ex2.restype = i
            lib.mss_scan_fwd_save.argtypes = [vp, vp, fp, vp, vp, fp, vp, fp, i, fp, vp, fp,
                                              i64, i64, i64, i64, i, u32, vp, i64, vp, i64, vp]
            lib.mss_scan_fwd_save.restype = i
            lib.mss_scan_fwd_workspace_size.argtypes = [i64, i64, i64, i64, i, u32]
            lib.mss_scan_fwd_workspace_size.restype = i64
            lib.mss_state_update.argtypes = [fp, vp, vp, fp, vp, vp, fp, vp, fp, i, vp,
                                             i64, i64, i64, i, vp]
            lib.mss_state_update.restype = i
            lib.mss_state_update_ex.argtypes = [fp, vp, vp, fp, vp, vp, fp, vp, fp, i, vp,
                                                i64, i64, i64, i, u32, vp]
            lib.mss_state_update_ex.restype = i
            lib.mss_scan_bwd.argtypes = [vp, vp, fp, vp, vp, fp, vp, fp, i, fp, vp, fp,
                                         vp, vp, vp, fp, fp, fp, fp, fp, fp, i64, i64, i64, i64, i, u32, vp, i64, vp]
            lib.mss_scan_bwd.restype = i
            lib.mss_scan_bwd_workspace_size.argtypes = [i64, i64, i64, i64, i, u32]
            lib.mss_scan_bwd_workspace_size.restype = i64
            lib.mss_ssd_fwd.argtypes = [vp, vp, fp, vp, vp, fp, vp, fp, i, fp, vp, fp,
                                        i64, i64, i64, i64, i64, i64, i, vp]
            lib.mss_ssd_fwd.restype = i
            lib.mss_ssd_fwd_ex.argtypes = [vp, vp, fp, vp, vp, fp, vp, fp, i, fp, vp, fp,
                                           i64, i64, i64, i64, i64, i64, i, vp, i64, vp]
            lib.mss_ssd_fwd_ex.restype = i
            lib.mss_ssd_fwd_workspace_size.argtypes = [i64, i64, i64, i64, i64, i64]
            lib.mss_ssd_fwd_workspace_size.restype = i64
            lib.mss_ssd_fwd_ex2.argtypes = [vp, vp, fp, vp, vp, fp, vp, fp, i, fp, vp, fp,
                                            i64, i64, i64, i64, i64, i64, i, u32, vp, i64, vp]
            lib.mss_ssd_fwd_ex2.restype = i
            lib.mss_ssd_fwd_workspace_size_ex.argtypes = [i64, i64, i64, i64, i64, i64, u32]
            lib.mss_ssd_fwd_workspace_size_ex.restype = i64
            lib.mss_scan_fwd_conv.argtypes = [vp, fp, fp, i, vp, vp, vp, fp, vp, vp, fp, vp, fp, i, fp, vp, fp,
                                              i64, i64, i64, i64, i, u32, vp, i64, vp]
            lib.mss_scan_fwd_conv.restype = i
            lib.mss_state_update_conv.argtypes = [fp, vp, vp, fp, fp, i, vp, fp, vp, vp, fp, vp, fp, i, vp,
                                                  i64, i64, i64, i, u32, vp]
            lib.mss_state_update_conv.restype = i
            lib.mss_scan_fwd_host.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, vp, vp, vp,
                                              i64, i64, i64, i64, i, u32, vp, i64, vp]
            lib.mss_scan_fwd_host.restype = i
            lib.mss_scan_fwd_host_workspace_size.argtypes = [i64, i64, i64, i64, i, i, i, i, i, i]
            lib.mss_scan_fwd_host_workspace_size.restype = i64
            lib.mss_get_device_error.argtypes = [vp]
            lib.mss_get_device_error.restype = i
            lib.mss_strerror.argtypes = [i]
            lib.mss_strerror.restype = ctypes.c_char_p
            lib.mss_version.argtypes = []
            lib.mss_version.restype = i
            lib.mss_probe_pipe_rates.argtypes = [ctypes.POINTER(ctypes.c_double), i, vp]
            lib.mss_probe_pipe_rates.restype = i
            _lib = lib
    return _lib


def _strerror(code: int) -> str:
    return load_library().mss_strerror(int(code)).decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check(t, name, shape, dtype, device, optional=False):
    if t is None:
        if optional:
            return
        raise ValueError(f"{name} is required")
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _io_dtype(t):
    if t.dtype == torch.float32:
        return DTYPE_F32
    if t.dtype == torch.bfloat16:
        return DTYPE_BF16
    raise TypeError(f"unsupported dtype {t.dtype}: use torch.float32 or torch.bfloat16")


def _stream_handle(stream, device):
    s = torch.cuda.current_stream(device) if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def workspace_size(batch, dim, dstate, seqlen, dtype=torch.bfloat16, flags=0, device=None) -> int:
    """Bytes of workspace the forward pass would use to split the sequence
    on `device` (0: no split)."""
    code = DTYPE_BF16 if dtype == torch.bfloat16 else DTYPE_F32
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        n = int(load_library().mss_scan_fwd_workspace_size(batch, dim, dstate, seqlen, code, int(flags)))
    if n < 0:
        raise MssError(n, "mss_scan_fwd_workspace_size")
    return n


def scan_fwd(u, delta, A, B, C, D=None, z=None, delta_bias=None, softplus=True,
             y=None, last_state=None, want_last_state=True, initial_state=None,
             workspace="auto", flags=0, stream=None):
    """Selective-scan forward pass (mss_scan_fwd_ex2).  Returns (y, last_state);
    last_state is None when want_last_state is False and none was given.

    initial_state: [batch, dim, N] float32 state before the first token (None:
    zero).  flags: FLAG_* bits; FLAG_ZOH_INPUT selects the zero-order-hold
    input matrix.  workspace: "auto" (the size the library asks for, allocated from
    PyTorch's caching allocator), None (no sequence split), or a uint8 CUDA
    tensor the call may use."""
    y, last_state, _ = _scan_fwd(u, delta, A, B, C, D, z, delta_bias, softplus, y, last_state, want_last_state,
                                 initial_state, workspace, flags, stream, None)
    return y, last_state


def scan_fwd_save(u, delta, A, B, C, D=None, z=None, delta_bias=None, softplus=True,
                  y=None, last_state=None, want_last_state=True, initial_state=None,
                  workspace="auto", states="auto", flags=0, stream=None):
    """The forward pass of a training step (mss_scan_fwd_save): scan_fwd that
    also stores the states scan_bwd needs.  Returns (y, last_state, states);
    pass `states` to scan_bwd(saved_states=...) with the same inputs and flags.
    states: "auto" (allocated here) or a uint8 CUDA tensor of at least
    bwd_workspace_size(...) bytes.  Raises MssError(ERR_PATH) for calls the
    tiled kernels do not take (then use scan_fwd and scan_bwd without it)."""
    return _scan_fwd(u, delta, A, B, C, D, z, delta_bias, softplus, y, last_state, want_last_state,
                     initial_state, workspace, flags, stream, states)


def _scan_fwd(u, delta, A, B, C, D, z, delta_bias, softplus, y, last_state, want_last_state, initial_state,
              workspace, flags, stream, states):
    if not isinstance(u, torch.Tensor) or u.device.type != "cuda":
        raise ValueError("u must be a CUDA tensor (there is no CPU path)")
    if u.dim() != 3:
        raise ValueError("u must be [batch, dim, L]")
    batch, dim, L = u.shape
    dev, dt = u.device, u.dtype
    code = _io_dtype(u)
    if A.dim() != 2:
        raise ValueError("A must be [dim, N]")
    N = A.shape[1]
    _check(u, "u", (batch, dim, L), dt, dev)
    _check(delta, "delta", (batch, dim, L), dt, dev)
    _check(A, "A", (dim, N), torch.float32, dev)
    _check(B, "B", (batch, N, L), dt, dev)
    _check(C, "C", (batch, N, L), dt, dev)
    _check(D, "D", (dim,), torch.float32, dev, optional=True)
    _check(z, "z", (batch, dim, L), dt, dev, optional=True)
    _check(delta_bias, "delta_bias", (dim,), torch.float32, dev, optional=True)
    _check(initial_state, "initial_state", (batch, dim, N), torch.float32, dev, optional=True)
    if y is None:
        y = torch.empty((batch, dim, L), dtype=dt, device=dev)
    _check(y, "y", (batch, dim, L), dt, dev)
    if last_state is None and want_last_state:
        last_state = torch.empty((batch, dim, N), dtype=torch.float32, device=dev)
    _check(last_state, "last_state", (batch, dim, N), torch.float32, dev, optional=True)
    if isinstance(workspace, str):
        if workspace != "auto":
            raise ValueError("workspace must be 'auto', None or a uint8 CUDA tensor")
        nbytes = workspace_size(batch, dim, N, L, dt, flags, dev)
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev) if nbytes > 0 else None
    if workspace is not None:
        _check(workspace, "workspace", (workspace.numel(),), torch.uint8, dev)
    if states is None:
        rc = load_library().mss_scan_fwd_ex2(
            _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias),
            int(bool(softplus)), _ptr(initial_state), _ptr(y), _ptr(last_state), batch, dim, N, L, code,
            int(flags), _ptr(workspace), 0 if workspace is None else workspace.numel(),
            _stream_handle(stream, dev))
        if rc != 0:
            raise MssError(rc, "mss_scan_fwd")
        return y, last_state, None
    if isinstance(states, str):
        if states != "auto":
            raise ValueError("states must be 'auto' or a uint8 CUDA tensor")
        states = torch.empty(max(bwd_workspace_size(batch, dim, N, L, dt, flags), 16), dtype=torch.uint8,
                             device=dev)
    _check(states, "states", (states.numel(),), torch.uint8, dev)
    rc = load_library().mss_scan_fwd_save(
        _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias),
        int(bool(softplus)), _ptr(initial_state), _ptr(y), _ptr(last_state), batch, dim, N, L, code,
        int(flags), _ptr(workspace), 0 if workspace is None else workspace.numel(), _ptr(states),
        states.numel(), _stream_handle(stream, dev))
    if rc != 0:
        raise MssError(rc, "mss_scan_fwd_save")
    return y, last_state, states


def scan_fwd_host(u, delta, A, B, C, D=None, z=None, delta_bias=None, softplus=True,
                  y=None, last_state=None, want_last_state=True, initial_state=None,
                  workspace="auto", flags=0, device=None, stream=None):
    """The forward pass over CPU tensors (mss_scan_fwd_host): the library
    copies the inputs to `device` piece by piece through a device workspace,
    runs the kernels and copies y and last_state back, overlapping the copies
    of different pieces with each other and with the kernels.  Inputs and
    outputs are CPU tensors in the layouts of scan_fwd.  Pinned memory is
    needed for the overlap, and outputs created here are pinned.  The call is
    asynchronous on `stream` (default: the current stream of `device`), so
    the outputs are complete only after that stream has been synchronised.
    Returns (y, last_state)."""
    if not isinstance(u, torch.Tensor) or u.device.type != "cpu":
        raise ValueError("u must be a CPU tensor (scan_fwd takes CUDA tensors)")
    if u.dim() != 3 or A.dim() != 2:
        raise ValueError("u must be [batch, dim, L] and A [dim, N]")
    batch, dim, L = u.shape
    N = A.shape[1]
    cpu, dt = torch.device("cpu"), u.dtype
    code = _io_dtype(u)
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    for t, name, shape, typ, opt in ((u, "u", (batch, dim, L), dt, False), (delta, "delta", (batch, dim, L), dt, False),
                                     (A, "A", (dim, N), torch.float32, False), (B, "B", (batch, N, L), dt, False),
                                     (C, "C", (batch, N, L), dt, False), (D, "D", (dim,), torch.float32, True),
                                     (z, "z", (batch, dim, L), dt, True),
                                     (delta_bias, "delta_bias", (dim,), torch.float32, True),
                                     (initial_state, "initial_state", (batch, dim, N), torch.float32, True)):
        _check(t, name, shape, typ, cpu, optional=opt)
    if y is None:
        y = torch.empty((batch, dim, L), dtype=dt, pin_memory=True)
    _check(y, "y", (batch, dim, L), dt, cpu)
    if last_state is None and want_last_state:
        last_state = torch.empty((batch, dim, N), dtype=torch.float32, pin_memory=True)
    _check(last_state, "last_state", (batch, dim, N), torch.float32, cpu, optional=True)
    lib = load_library()
    with torch.cuda.device(dev):
        if isinstance(workspace, str):
            if workspace != "auto":
                raise ValueError("workspace must be 'auto' or a uint8 CUDA tensor")
            nbytes = int(lib.mss_scan_fwd_host_workspace_size(
                batch, dim, N, L, code, int(z is not None), int(D is not None), int(delta_bias is not None),
                int(initial_state is not None), int(last_state is not None)))
            if nbytes < 0:
                raise MssError(nbytes, "mss_scan_fwd_host_workspace_size")
            workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=dev)
        _check(workspace, "workspace", (workspace.numel(),), torch.uint8, dev)
        rc = lib.mss_scan_fwd_host(
            _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias),
            int(bool(softplus)), _ptr(initial_state), _ptr(y), _ptr(last_state), batch, dim, N, L, code,
            int(flags), _ptr(workspace), workspace.numel(), _stream_handle(stream, dev))
    if rc != 0:
        raise MssError(rc, "mss_scan_fwd_host")
    return y, last_state


def scan_fwd_conv(x, conv_w, delta, A, B, C, conv_b=None, conv_state=None, D=None, z=None,
                  delta_bias=None, softplus=True, y=None, last_state=None, want_last_state=True,
                  conv_state_out=None, want_conv_state=True, initial_state=None, workspace="auto",
                  flags=0, stream=None):
    """Forward pass with the causal convolution and SiLU in front
    (mss_scan_fwd_conv): u = silu(conv_b + causal conv of x with conv_w).
    Returns (y, last_state, conv_state_out); each state is None when not
    wanted and not given.

    x: [batch, dim, L]; conv_w: [dim, K] float32 (K = 1..4); conv_b: [dim]
    float32; conv_state: [batch, dim, K-1] in x's dtype (None: zeros).  Other
    arguments as scan_fwd."""
    if not isinstance(x, torch.Tensor) or x.device.type != "cuda":
        raise ValueError("x must be a CUDA tensor (there is no CPU path)")
    if x.dim() != 3:
        raise ValueError("x must be [batch, dim, L]")
    batch, dim, L = x.shape
    dev, dt = x.device, x.dtype
    code = _io_dtype(x)
    if A.dim() != 2 or conv_w.dim() != 2:
        raise ValueError("A must be [dim, N] and conv_w [dim, K]")
    N, K = A.shape[1], conv_w.shape[1]
    _check(x, "x", (batch, dim, L), dt, dev)
    _check(conv_w, "conv_w", (dim, K), torch.float32, dev)
    _check(conv_b, "conv_b", (dim,), torch.float32, dev, optional=True)
    _check(conv_state, "conv_state", (batch, dim, K - 1), dt, dev, optional=True)
    _check(delta, "delta", (batch, dim, L), dt, dev)
    _check(A, "A", (dim, N), torch.float32, dev)
    _check(B, "B", (batch, N, L), dt, dev)
    _check(C, "C", (batch, N, L), dt, dev)
    _check(D, "D", (dim,), torch.float32, dev, optional=True)
    _check(z, "z", (batch, dim, L), dt, dev, optional=True)
    _check(delta_bias, "delta_bias", (dim,), torch.float32, dev, optional=True)
    _check(initial_state, "initial_state", (batch, dim, N), torch.float32, dev, optional=True)
    if y is None:
        y = torch.empty((batch, dim, L), dtype=dt, device=dev)
    _check(y, "y", (batch, dim, L), dt, dev)
    if last_state is None and want_last_state:
        last_state = torch.empty((batch, dim, N), dtype=torch.float32, device=dev)
    _check(last_state, "last_state", (batch, dim, N), torch.float32, dev, optional=True)
    if conv_state_out is None and want_conv_state:
        conv_state_out = torch.empty((batch, dim, K - 1), dtype=dt, device=dev)
    _check(conv_state_out, "conv_state_out", (batch, dim, K - 1), dt, dev, optional=True)
    if isinstance(workspace, str):
        if workspace != "auto":
            raise ValueError("workspace must be 'auto', None or a uint8 CUDA tensor")
        nbytes = workspace_size(batch, dim, N, L, dt, flags, dev)
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev) if nbytes > 0 else None
    if workspace is not None:
        _check(workspace, "workspace", (workspace.numel(),), torch.uint8, dev)
    rc = load_library().mss_scan_fwd_conv(
        _ptr(x), _ptr(conv_w), _ptr(conv_b), int(K), _ptr(conv_state), _ptr(conv_state_out),
        _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias), int(bool(softplus)),
        _ptr(initial_state), _ptr(y), _ptr(last_state), batch, dim, N, L, code, int(flags),
        _ptr(workspace), 0 if workspace is None else workspace.numel(), _stream_handle(stream, dev))
    if rc != 0:
        raise MssError(rc, "mss_scan_fwd_conv")
    return y, last_state, conv_state_out


def ssd_fwd(x, dt, A, B, C, D=None, z=None, dt_bias=None, softplus=True, initial_state=None, y=None,
            last_state=None, want_last_state=True, workspace="auto", flags=0, stream=None):
    """Structured-state-space-duality forward pass (mss_ssd_fwd_ex2).  x, z:
    [batch, L, H, P] bf16; dt: [batch, L, H] bf16; A, D, dt_bias: [H]
    float32; B, C: [batch, L, G, N] bf16; initial_state: [batch, H, N, P]
    float32.  workspace: "auto" (what mss_ssd_fwd_workspace_size_ex asks for,
    from PyTorch's allocator: every chunk in parallel where that beats one CTA
    per head -- for N = 128 also only the few pairs past the tcgen05 kernel's
    last full wave -- else nothing), None (one CTA per head walks its chunks)
    or a uint8 CUDA tensor.  flags: 0 (the tcgen05 kernel for N = 128, unless a
    workspace is given and the chunk-parallel passes are faster for so few
    (batch, head) pairs) or SSD_FLAG_WARP_MMA (the warp-level kernels).
    Returns (y, last_state)."""
    if not isinstance(x, torch.Tensor) or x.device.type != "cuda":
        raise ValueError("x must be a CUDA tensor (there is no CPU path)")
    if x.dim() != 4 or B.dim() != 4:
        raise ValueError("x must be [batch, L, H, P] and B [batch, L, G, N]")
    batch, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    dev, dt_ = x.device, x.dtype
    code = _io_dtype(x)
    for t, name, shape, typ, opt in ((x, "x", (batch, L, H, P), dt_, False), (dt, "dt", (batch, L, H), dt_, False),
                                     (A, "A", (H,), torch.float32, False), (B, "B", (batch, L, G, N), dt_, False),
                                     (C, "C", (batch, L, G, N), dt_, False), (D, "D", (H,), torch.float32, True),
                                     (z, "z", (batch, L, H, P), dt_, True),
                                     (dt_bias, "dt_bias", (H,), torch.float32, True),
                                     (initial_state, "initial_state", (batch, H, N, P), torch.float32, True)):
        _check(t, name, shape, typ, dev, optional=opt)
    if y is None:
        y = torch.empty((batch, L, H, P), dtype=dt_, device=dev)
    _check(y, "y", (batch, L, H, P), dt_, dev)
    if last_state is None and want_last_state:
        last_state = torch.empty((batch, H, N, P), dtype=torch.float32, device=dev)
    _check(last_state, "last_state", (batch, H, N, P), torch.float32, dev, optional=True)
    if isinstance(workspace, str):
        if workspace != "auto":
            raise ValueError("workspace must be 'auto', None or a uint8 CUDA tensor")
        nbytes = int(load_library().mss_ssd_fwd_workspace_size_ex(batch, L, H, P, G, N, int(flags)))
        if nbytes < 0:
            raise MssError(nbytes, "mss_ssd_fwd_workspace_size_ex")
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev) if nbytes > 0 else None
    if workspace is not None:
        _check(workspace, "workspace", (workspace.numel(),), torch.uint8, dev)
    rc = load_library().mss_ssd_fwd_ex2(
        _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(dt_bias), int(bool(softplus)),
        _ptr(initial_state), _ptr(y), _ptr(last_state), batch, L, H, P, G, N, code, int(flags), _ptr(workspace),
        0 if workspace is None else workspace.numel(), _stream_handle(stream, dev))
    if rc != 0:
        raise MssError(rc, "mss_ssd_fwd")
    return y, last_state


def bwd_workspace_size(batch, dim, dstate, seqlen, dtype=torch.bfloat16, flags=0) -> int:
    """Bytes of workspace scan_bwd needs (16-byte aligned tensors)."""
    code = DTYPE_BF16 if dtype == torch.bfloat16 else DTYPE_F32
    n = int(load_library().mss_scan_bwd_workspace_size(batch, dim, dstate, seqlen, code, int(flags)))
    if n < 0:
        raise MssError(n, "mss_scan_bwd_workspace_size")
    return n


def scan_bwd(u, delta, A, B, C, dy, D=None, z=None, delta_bias=None, softplus=True, initial_state=None,
             dlast=None, flags=0, workspace="auto", want_dinit=True, out=None, stream=None, saved_states=None):
    """Backward pass of scan_fwd (mss_scan_bwd).  dy: [batch, dim, L] (the io
    dtype), dlast: [batch, dim, N] float32 or None.  Returns a dict with du,
    ddelta, dz (None without z) in the io dtype, dA [dim, N], dB, dC
    [batch, N, L], dD, dbias [dim] and dinit [batch, dim, N] in float32.
    out: optional dict of caller-owned output tensors under those names (the
    rest are allocated).  saved_states: the states scan_fwd_save returned for
    these inputs and flags; the call then skips its checkpoint pass (the
    tensor is its workspace)."""
    if saved_states is not None:
        flags = int(flags) | FLAG_SAVED_STATES
        workspace = saved_states
    if not isinstance(u, torch.Tensor) or u.device.type != "cuda":
        raise ValueError("u must be a CUDA tensor (there is no CPU path)")
    batch, dim, L = u.shape
    dev, dt = u.device, u.dtype
    code = _io_dtype(u)
    N = A.shape[1]
    for t, name, shape, typ, opt in ((u, "u", (batch, dim, L), dt, False), (delta, "delta", (batch, dim, L), dt, False),
                                     (A, "A", (dim, N), torch.float32, False), (B, "B", (batch, N, L), dt, False),
                                     (C, "C", (batch, N, L), dt, False), (dy, "dy", (batch, dim, L), dt, False),
                                     (D, "D", (dim,), torch.float32, True), (z, "z", (batch, dim, L), dt, True),
                                     (delta_bias, "delta_bias", (dim,), torch.float32, True),
                                     (initial_state, "initial_state", (batch, dim, N), torch.float32, True),
                                     (dlast, "dlast", (batch, dim, N), torch.float32, True)):
        _check(t, name, shape, typ, dev, optional=opt)
    f32 = dict(dtype=torch.float32, device=dev)
    ret = dict(du=torch.empty((batch, dim, L), dtype=dt, device=dev),
               ddelta=torch.empty((batch, dim, L), dtype=dt, device=dev),
               dz=torch.empty((batch, dim, L), dtype=dt, device=dev) if z is not None else None,
               dA=torch.empty((dim, N), **f32), dB=torch.empty((batch, N, L), **f32),
               dC=torch.empty((batch, N, L), **f32), dD=torch.empty((dim,), **f32),
               dbias=torch.empty((dim,), **f32),
               dinit=torch.empty((batch, dim, N), **f32) if want_dinit else None)
    for k, t in (out or {}).items():
        if k not in ret or ret[k] is None:
            raise ValueError(f"out[{k!r}]: no such output here")
        _check(t, k, tuple(ret[k].shape), ret[k].dtype, dev)
        ret[k] = t
    if isinstance(workspace, str):
        if workspace != "auto":
            raise ValueError("workspace must be 'auto', None or a uint8 CUDA tensor")
        nbytes = bwd_workspace_size(batch, dim, N, L, dt, flags)
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev) if nbytes > 0 else None
    if workspace is not None:
        _check(workspace, "workspace", (workspace.numel(),), torch.uint8, dev)
    rc = load_library().mss_scan_bwd(
        _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias), int(bool(softplus)),
        _ptr(initial_state), _ptr(dy), _ptr(dlast), _ptr(ret["du"]), _ptr(ret["ddelta"]), _ptr(ret["dz"]),
        _ptr(ret["dA"]), _ptr(ret["dB"]), _ptr(ret["dC"]), _ptr(ret["dD"]), _ptr(ret["dbias"]), _ptr(ret["dinit"]),
        batch, dim, N, L, code, int(flags), _ptr(workspace), 0 if workspace is None else workspace.numel(),
        _stream_handle(stream, dev))
    if rc != 0:
        raise MssError(rc, "mss_scan_bwd")
    return ret


def state_update_conv(state, conv_state, x, conv_w, delta, A, B, C, conv_b=None, D=None, z=None,
                      delta_bias=None, softplus=True, y=None, flags=0, stream=None):
    """One decode token with the causal convolution in front
    (mss_state_update_conv); `state` and `conv_state` ([batch, dim, K-1] in
    x's dtype, None when K = 1) are updated in place.  Returns y [batch, dim]."""
    if not isinstance(state, torch.Tensor) or state.device.type != "cuda":
        raise ValueError("state must be a CUDA tensor (there is no CPU path)")
    if state.dim() != 3:
        raise ValueError("state must be [batch, dim, N]")
    batch, dim, N = state.shape
    dev, dt = state.device, x.dtype
    code = _io_dtype(x)
    if conv_w.dim() != 2:
        raise ValueError("conv_w must be [dim, K]")
    K = conv_w.shape[1]
    _check(state, "state", (batch, dim, N), torch.float32, dev)
    _check(conv_state, "conv_state", (batch, dim, K - 1), dt, dev, optional=K == 1)
    _check(x, "x", (batch, dim), dt, dev)
    _check(conv_w, "conv_w", (dim, K), torch.float32, dev)
    _check(conv_b, "conv_b", (dim,), torch.float32, dev, optional=True)
    _check(delta, "delta", (batch, dim), dt, dev)
    _check(A, "A", (dim, N), torch.float32, dev)
    _check(B, "B", (batch, N), dt, dev)
    _check(C, "C", (batch, N), dt, dev)
    _check(D, "D", (dim,), torch.float32, dev, optional=True)
    _check(z, "z", (batch, dim), dt, dev, optional=True)
    _check(delta_bias, "delta_bias", (dim,), torch.float32, dev, optional=True)
    if y is None:
        y = torch.empty((batch, dim), dtype=dt, device=dev)
    _check(y, "y", (batch, dim), dt, dev)
    rc = load_library().mss_state_update_conv(
        _ptr(state), _ptr(conv_state), _ptr(x), _ptr(conv_w), _ptr(conv_b), int(K), _ptr(delta), _ptr(A),
        _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias), int(bool(softplus)), _ptr(y), batch, dim, N,
        code, int(flags), _stream_handle(stream, dev))
    if rc != 0:
        raise MssError(rc, "mss_state_update_conv")
    return y


def state_update(state, u, delta, A, B, C, D=None, z=None, delta_bias=None, softplus=True,
                 y=None, flags=0, stream=None):
    """One decode token (mss_state_update_ex); `state` is updated in place.
    Returns y [batch, dim].  flags: 0 or FLAG_ZOH_INPUT."""
    if not isinstance(state, torch.Tensor) or state.device.type != "cuda":
        raise ValueError("state must be a CUDA tensor (there is no CPU path)")
    if state.dim() != 3:
        raise ValueError("state must be [batch, dim, N]")
    batch, dim, N = state.shape
    dev, dt = state.device, u.dtype
    code = _io_dtype(u)
    _check(state, "state", (batch, dim, N), torch.float32, dev)
    _check(u, "u", (batch, dim), dt, dev)
    _check(delta, "delta", (batch, dim), dt, dev)
    _check(A, "A", (dim, N), torch.float32, dev)
    _check(B, "B", (batch, N), dt, dev)
    _check(C, "C", (batch, N), dt, dev)
    _check(D, "D", (dim,), torch.float32, dev, optional=True)
    _check(z, "z", (batch, dim), dt, dev, optional=True)
    _check(delta_bias, "delta_bias", (dim,), torch.float32, dev, optional=True)
    if y is None:
        y = torch.empty((batch, dim), dtype=dt, device=dev)
    _check(y, "y", (batch, dim), dt, dev)
    rc = load_library().mss_state_update_ex(
        _ptr(state), _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
        _ptr(delta_bias), int(bool(softplus)), _ptr(y), batch, dim, N, code, int(flags),
        _stream_handle(stream, dev))
    if rc != 0:
        raise MssError(rc, "mss_state_update")
    return y


PIPE_RATE_NAMES = ("ffma", "ffma2", "mufu_ex2", "shfl")


def probe_pipe_rates(stream=None, device=None) -> dict:
    """Measured throughput of the fp32 fma pipe (scalar and packed, lane
    operations), the multi-function unit (ex2 results) and warp shuffles
    (results), per SM and SM clock cycle, on the current device
    (mss_probe_pipe_rates)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    out = (ctypes.c_double * len(PIPE_RATE_NAMES))()
    rc = load_library().mss_probe_pipe_rates(out, len(PIPE_RATE_NAMES), _stream_handle(stream, dev))
    if rc != 0:
        raise MssError(rc, "mss_probe_pipe_rates")
    return {k: float(v) for k, v in zip(PIPE_RATE_NAMES, out)}


def get_device_error(stream=None, device=None) -> int:
    """Synchronise the stream and return (and clear) the library's device
    error status: 0, or a negative mss_status code."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    return int(load_library().mss_get_device_error(_stream_handle(stream, dev)))
