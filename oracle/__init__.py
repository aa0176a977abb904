"""fp64 CPU oracle for the selective scan (S6): Python side.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference leg of ``bench.py`` may import this package.  The
product path (the ``selective_state_space_mss_b200`` package and its CUDA
library) never imports it, and it never imports the product path: the two
share no code.  The only module both sides use is the seeded input generator,
which holds none of the method's arithmetic.

``mss_oracle.c`` holds the definition of the forward pass and of the decode
step (citations are in its header); this module builds it with gcc, loads it
with ctypes and converts numpy arrays.  ``scans.py`` holds the alternative
scan orders and matrix views used to pin the sequential definition.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mss_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``mss_oracle.c`` into ``liboracle.so`` next to it (gcc, -O2).

    Plain C99 with libm and pthreads; no fast-math, so every operation is an
    IEEE fp64 operation in program order.
    """
    if force or not os.path.exists(_LIB_PATH) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    ):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-std=c99", "-O2", "-fno-fast-math", "-ffp-contract=off",
             "-Wall", "-Wextra", "-fPIC", "-shared", "-o", tmp, _SRC,
             "-lm", "-lpthread"]
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            # MSS_ORACLE_LIB points the pins at another build of this same
            # source (the mutation test plants mistakes in copies of it).
            path = os.environ.get("MSS_ORACLE_LIB") or build()
            lib = ctypes.CDLL(path)
            f, d, i64, i = (ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_double),
                            ctypes.c_int64, ctypes.c_int)
            lib.mss_oracle_scan_fwd.argtypes = [f, f, f, f, f, f, f, f, i, i, d, d, d,
                                                i64, i64, i64, i64, i]
            lib.mss_oracle_scan_fwd.restype = i
            lib.mss_oracle_state_update.argtypes = [d, f, f, f, f, f, f, f, f, i, i, d,
                                                    i64, i64, i64, i]
            lib.mss_oracle_state_update.restype = i
            lib.mss_oracle_scan_fwd_conv.argtypes = [f, f, f, i, d, d, f, f, f, f, f, f, f, i, i, d, d, d,
                                                     i64, i64, i64, i64, i]
            lib.mss_oracle_scan_fwd_conv.restype = i
            lib.mss_oracle_causal_conv.argtypes = [f, f, f, i, d, d, d, i64, i64, i64]
            lib.mss_oracle_causal_conv.restype = i
            lib.mss_oracle_state_update_conv.argtypes = [d, d, f, f, f, i, f, f, f, f, f, f, f, i, i, d,
                                                         i64, i64, i64, i]
            lib.mss_oracle_state_update_conv.restype = i
            lib.mss_oracle_scan_bwd.argtypes = [f, f, f, f, f, f, f, f, i, i, d, f, d,
                                                d, d, d, d, d, d, d, d, d, i64, i64, i64, i64, i]
            lib.mss_oracle_scan_bwd.restype = i
            lib.mss_oracle_ssd_fwd.argtypes = [f, f, f, f, f, f, f, f, i, d, d, d, i64, i64, i64, i64, i64, i64, i]
            lib.mss_oracle_ssd_fwd.restype = i
            lib.mss_oracle_recurrence.argtypes = [d, d, d, i64, i64, d, d]
            lib.mss_oracle_recurrence.restype = i
            lib.mss_oracle_softplus.argtypes = [ctypes.c_double]
            lib.mss_oracle_softplus.restype = ctypes.c_double
            lib.mss_oracle_silu.argtypes = [ctypes.c_double]
            lib.mss_oracle_silu.restype = ctypes.c_double
            _lib = lib
    return _lib


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def _f32(x, shape=None, name="array"):
    if x is None:
        return None, None
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    if shape is not None and a.shape != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {a.shape}")
    return a, a.ctypes.data_as(ctypes.POINTER(ctypes.c_float))


def _dptr(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def softplus(s: float) -> float:
    """ln(1 + e^s) in fp64."""
    return _load().mss_oracle_softplus(float(s))


def silu(z: float) -> float:
    """z / (1 + e^-z) in fp64."""
    return _load().mss_oracle_silu(float(z))


def scan_fwd(u, delta, A, B, C, D=None, z=None, delta_bias=None, softplus_flag=True,
             initial_state=None, zoh_input=False, nthreads=None):
    """Selective-scan forward pass in fp64.

    u, delta, z: [batch, dim, L]; A: [dim, N]; B, C: [batch, N, L];
    D, delta_bias: [dim]; initial_state: [batch, dim, N] (the state before
    the first token; None for zero); zoh_input: exact zero-order-hold input
    matrix (e^{Delta A} - 1)/A * B instead of the Euler Delta * B.  Values are taken as fp32 (bf16 inputs
    must already be widened, which is exact); initial_state as fp64.
    Returns (y [batch, dim, L] fp64, last_state [batch, dim, N] fp64).
    """
    u_a, u_p = _f32(u, name="u")
    if u_a.ndim != 3:
        raise ValueError("u must be [batch, dim, L]")
    batch, dim, L = u_a.shape
    A_a, A_p = _f32(A, name="A")
    if A_a.ndim != 2 or A_a.shape[0] != dim:
        raise ValueError("A must be [dim, N]")
    N = A_a.shape[1]
    d_a, d_p = _f32(delta, (batch, dim, L), "delta")
    B_a, B_p = _f32(B, (batch, N, L), "B")
    C_a, C_p = _f32(C, (batch, N, L), "C")
    D_a, D_p = _f32(D, (dim,), "D")
    z_a, z_p = _f32(z, (batch, dim, L), "z")
    b_a, b_p = _f32(delta_bias, (dim,), "delta_bias")
    h0 = None
    if initial_state is not None:
        h0 = np.ascontiguousarray(np.asarray(initial_state, dtype=np.float64))
        if h0.shape != (batch, dim, N):
            raise ValueError(f"initial_state: expected shape {(batch, dim, N)}, got {h0.shape}")
    y = np.empty((batch, dim, L), dtype=np.float64)
    last = np.empty((batch, dim, N), dtype=np.float64)
    rc = _load().mss_oracle_scan_fwd(
        u_p, d_p, A_p, B_p, C_p, D_p, z_p, b_p, int(bool(softplus_flag)), int(bool(zoh_input)),
        _dptr(h0) if h0 is not None else None, _dptr(y), _dptr(last), batch, dim, N, L,
        default_threads() if nthreads is None else int(nthreads))
    if rc != 0:
        raise RuntimeError(f"mss_oracle_scan_fwd failed with code {rc}")
    del u_a, d_a, B_a, C_a, D_a, z_a, b_a, A_a  # keep buffers alive until here
    return y, last


def _f64_opt(x, shape, name):
    if x is None:
        return None
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    if a.shape != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {a.shape}")
    return a


def causal_conv(x, conv_w, conv_b=None, conv_state=None):
    """Causal depthwise convolution, pre-activation, in fp64.

    x: [batch, dim, L]; conv_w: [dim, K] (tap k multiplies x_{t-(K-1)+k});
    conv_b: [dim]; conv_state: [batch, dim, K-1] values before the first
    token (None: zeros).  Returns (xc [batch, dim, L], conv_state_out
    [batch, dim, K-1])."""
    x_a, x_p = _f32(x, name="x")
    batch, dim, L = x_a.shape
    w_a, w_p = _f32(conv_w, name="conv_w")
    K = w_a.shape[1]
    cb_a, cb_p = _f32(conv_b, (dim,), "conv_b")
    cs = _f64_opt(conv_state, (batch, dim, K - 1), "conv_state")
    xc = np.empty((batch, dim, L), dtype=np.float64)
    cs_out = np.empty((batch, dim, K - 1), dtype=np.float64)
    rc = _load().mss_oracle_causal_conv(x_p, w_p, cb_p, K, None if cs is None else _dptr(cs), _dptr(xc),
                                        _dptr(cs_out), batch, dim, L)
    if rc != 0:
        raise RuntimeError(f"mss_oracle_causal_conv failed with code {rc}")
    del x_a, w_a, cb_a
    return xc, cs_out


def scan_fwd_conv(x, conv_w, delta, A, B, C, conv_b=None, conv_state=None, D=None, z=None,
                  delta_bias=None, softplus_flag=True, initial_state=None, zoh_input=False,
                  nthreads=None):
    """Forward pass with the causal convolution and SiLU in front, in fp64:
    u = silu(causal_conv(x)).  Arguments as scan_fwd and causal_conv.
    Returns (y, last_state, conv_state_out)."""
    x_a, x_p = _f32(x, name="x")
    if x_a.ndim != 3:
        raise ValueError("x must be [batch, dim, L]")
    batch, dim, L = x_a.shape
    w_a, w_p = _f32(conv_w, name="conv_w")
    if w_a.ndim != 2 or w_a.shape[0] != dim:
        raise ValueError("conv_w must be [dim, K]")
    K = w_a.shape[1]
    A_a, A_p = _f32(A, name="A")
    N = A_a.shape[1]
    cb_a, cb_p = _f32(conv_b, (dim,), "conv_b")
    cs = _f64_opt(conv_state, (batch, dim, K - 1), "conv_state")
    d_a, d_p = _f32(delta, (batch, dim, L), "delta")
    B_a, B_p = _f32(B, (batch, N, L), "B")
    C_a, C_p = _f32(C, (batch, N, L), "C")
    D_a, D_p = _f32(D, (dim,), "D")
    z_a, z_p = _f32(z, (batch, dim, L), "z")
    b_a, b_p = _f32(delta_bias, (dim,), "delta_bias")
    h0 = _f64_opt(initial_state, (batch, dim, N), "initial_state")
    y = np.empty((batch, dim, L), dtype=np.float64)
    last = np.empty((batch, dim, N), dtype=np.float64)
    cs_out = np.empty((batch, dim, K - 1), dtype=np.float64)
    rc = _load().mss_oracle_scan_fwd_conv(
        x_p, w_p, cb_p, K, None if cs is None else _dptr(cs), _dptr(cs_out),
        d_p, A_p, B_p, C_p, D_p, z_p, b_p, int(bool(softplus_flag)), int(bool(zoh_input)),
        None if h0 is None else _dptr(h0), _dptr(y), _dptr(last), batch, dim, N, L,
        default_threads() if nthreads is None else int(nthreads))
    if rc != 0:
        raise RuntimeError(f"mss_oracle_scan_fwd_conv failed with code {rc}")
    del x_a, w_a, cb_a, d_a, B_a, C_a, D_a, z_a, b_a, A_a
    return y, last, cs_out


def state_update_conv(state, conv_state, x, conv_w, delta, A, B, C, conv_b=None, D=None, z=None,
                      delta_bias=None, softplus_flag=True, zoh_input=False, nthreads=None):
    """One decode step with the causal convolution in front, in fp64.

    state: [batch, dim, N] and conv_state: [batch, dim, K-1], both fp64 and
    updated in place; x: [batch, dim]; other arguments as state_update.
    Returns (y, state, conv_state)."""
    for name, a in (("state", state), ("conv_state", conv_state)):
        if not (isinstance(a, np.ndarray) and a.dtype == np.float64 and a.flags.c_contiguous):
            raise ValueError(f"{name} must be a C-contiguous float64 numpy array")
    batch, dim, N = state.shape
    w_a, w_p = _f32(conv_w, name="conv_w")
    K = w_a.shape[1]
    if conv_state.shape != (batch, dim, K - 1):
        raise ValueError("conv_state must be [batch, dim, K-1]")
    x_a, x_p = _f32(x, (batch, dim), "x")
    cb_a, cb_p = _f32(conv_b, (dim,), "conv_b")
    d_a, d_p = _f32(delta, (batch, dim), "delta")
    A_a, A_p = _f32(A, (dim, N), "A")
    B_a, B_p = _f32(B, (batch, N), "B")
    C_a, C_p = _f32(C, (batch, N), "C")
    D_a, D_p = _f32(D, (dim,), "D")
    z_a, z_p = _f32(z, (batch, dim), "z")
    b_a, b_p = _f32(delta_bias, (dim,), "delta_bias")
    y = np.empty((batch, dim), dtype=np.float64)
    rc = _load().mss_oracle_state_update_conv(
        _dptr(state), _dptr(conv_state), x_p, w_p, cb_p, K, d_p, A_p, B_p, C_p, D_p, z_p, b_p,
        int(bool(softplus_flag)), int(bool(zoh_input)), _dptr(y), batch, dim, N,
        default_threads() if nthreads is None else int(nthreads))
    if rc != 0:
        raise RuntimeError(f"mss_oracle_state_update_conv failed with code {rc}")
    del x_a, w_a, cb_a, d_a, A_a, B_a, C_a, D_a, z_a, b_a
    return y, state, conv_state


def scan_bwd(u, delta, A, B, C, dy, D=None, z=None, delta_bias=None, softplus_flag=True,
             initial_state=None, dlast=None, zoh_input=False, nthreads=None):
    """Backward pass of scan_fwd in fp64 (reverse mode).

    dy: [batch, dim, L] gradient with respect to y; dlast: [batch, dim, N]
    gradient with respect to last_state (None: 0).  Returns a dict with du,
    ddelta (with respect to delta_raw), dz (None without z), dA [dim, N],
    dB, dC [batch, N, L], dD, dbias [dim] and dinit [batch, dim, N]
    (with respect to initial_state)."""
    u_a, u_p = _f32(u, name="u")
    batch, dim, L = u_a.shape
    A_a, A_p = _f32(A, name="A")
    N = A_a.shape[1]
    d_a, d_p = _f32(delta, (batch, dim, L), "delta")
    B_a, B_p = _f32(B, (batch, N, L), "B")
    C_a, C_p = _f32(C, (batch, N, L), "C")
    D_a, D_p = _f32(D, (dim,), "D")
    z_a, z_p = _f32(z, (batch, dim, L), "z")
    b_a, b_p = _f32(delta_bias, (dim,), "delta_bias")
    g_a, g_p = _f32(dy, (batch, dim, L), "dy")
    h0 = _f64_opt(initial_state, (batch, dim, N), "initial_state")
    dl = _f64_opt(dlast, (batch, dim, N), "dlast")
    out = {k: np.zeros(shape, dtype=np.float64) for k, shape in
           (("du", (batch, dim, L)), ("ddelta", (batch, dim, L)), ("dz", (batch, dim, L)), ("dA", (dim, N)),
            ("dB", (batch, N, L)), ("dC", (batch, N, L)), ("dD", (dim,)), ("dbias", (dim,)),
            ("dinit", (batch, dim, N)))}
    rc = _load().mss_oracle_scan_bwd(
        u_p, d_p, A_p, B_p, C_p, D_p, z_p, b_p, int(bool(softplus_flag)), int(bool(zoh_input)),
        None if h0 is None else _dptr(h0), g_p, None if dl is None else _dptr(dl),
        _dptr(out["du"]), _dptr(out["ddelta"]), _dptr(out["dz"]) if z is not None else None, _dptr(out["dA"]),
        _dptr(out["dB"]), _dptr(out["dC"]), _dptr(out["dD"]), _dptr(out["dbias"]), _dptr(out["dinit"]),
        batch, dim, N, L, default_threads() if nthreads is None else int(nthreads))
    if rc != 0:
        raise RuntimeError(f"mss_oracle_scan_bwd failed with code {rc}")
    if z is None:
        out["dz"] = None
    del u_a, d_a, B_a, C_a, D_a, z_a, b_a, g_a, A_a
    return out


def state_update(state, u, delta, A, B, C, D=None, z=None, delta_bias=None,
                 softplus_flag=True, zoh_input=False, nthreads=None):
    """One decode step in fp64.

    state: [batch, dim, N] (fp64, updated in place and returned);
    u, delta, z: [batch, dim]; A: [dim, N]; B, C: [batch, N]; D, delta_bias: [dim].
    Returns (y [batch, dim] fp64, state).
    """
    if not (isinstance(state, np.ndarray) and state.dtype == np.float64
            and state.flags.c_contiguous):
        raise ValueError("state must be a C-contiguous float64 numpy array")
    batch, dim, N = state.shape
    u_a, u_p = _f32(u, (batch, dim), "u")
    d_a, d_p = _f32(delta, (batch, dim), "delta")
    A_a, A_p = _f32(A, (dim, N), "A")
    B_a, B_p = _f32(B, (batch, N), "B")
    C_a, C_p = _f32(C, (batch, N), "C")
    D_a, D_p = _f32(D, (dim,), "D")
    z_a, z_p = _f32(z, (batch, dim), "z")
    b_a, b_p = _f32(delta_bias, (dim,), "delta_bias")
    y = np.empty((batch, dim), dtype=np.float64)
    rc = _load().mss_oracle_state_update(
        _dptr(state), u_p, d_p, A_p, B_p, C_p, D_p, z_p, b_p, int(bool(softplus_flag)),
        int(bool(zoh_input)), _dptr(y), batch, dim, N,
        default_threads() if nthreads is None else int(nthreads))
    if rc != 0:
        raise RuntimeError(f"mss_oracle_state_update failed with code {rc}")
    del u_a, d_a, A_a, B_a, C_a, D_a, z_a, b_a
    return y, state


def ssd_fwd(x, dt, A, B, C, D=None, z=None, dt_bias=None, softplus_flag=True, initial_state=None,
            nthreads=None):
    """Structured state space duality (Mamba-2) forward pass in fp64: A is a
    scalar per head.  x, z: [batch, L, H, P]; dt: [batch, L, H]; A, D,
    dt_bias: [H]; B, C: [batch, L, G, N] (head h reads group h // (H // G));
    initial_state: [batch, H, N, P].  Returns (y [batch, L, H, P],
    last_state [batch, H, N, P])."""
    x_a, x_p = _f32(x, name="x")
    if x_a.ndim != 4:
        raise ValueError("x must be [batch, L, H, P]")
    batch, L, H, P = x_a.shape
    B_a, B_p = _f32(B, name="B")
    if B_a.ndim != 4 or B_a.shape[:2] != (batch, L):
        raise ValueError("B must be [batch, L, G, N]")
    G, N = B_a.shape[2], B_a.shape[3]
    dt_a, dt_p = _f32(dt, (batch, L, H), "dt")
    A_a, A_p = _f32(A, (H,), "A")
    C_a, C_p = _f32(C, (batch, L, G, N), "C")
    D_a, D_p = _f32(D, (H,), "D")
    z_a, z_p = _f32(z, (batch, L, H, P), "z")
    b_a, b_p = _f32(dt_bias, (H,), "dt_bias")
    h0 = _f64_opt(initial_state, (batch, H, N, P), "initial_state")
    y = np.empty((batch, L, H, P), dtype=np.float64)
    last = np.empty((batch, H, N, P), dtype=np.float64)
    rc = _load().mss_oracle_ssd_fwd(x_p, dt_p, A_p, B_p, C_p, D_p, z_p, b_p, int(bool(softplus_flag)),
                                    None if h0 is None else _dptr(h0), _dptr(y), _dptr(last),
                                    batch, L, H, P, G, N, default_threads() if nthreads is None else int(nthreads))
    if rc != 0:
        raise RuntimeError(f"mss_oracle_ssd_fwd failed with code {rc}")
    del x_a, dt_a, A_a, B_a, C_a, D_a, z_a, b_a
    return y, last


def recurrence(abar, bbar_x, c):
    """Discrete recurrence with given coefficients (rows are tokens).

    abar, bbar_x, c: [L, N] fp64.  Returns (h [L, N], y [L]) with h starting at 0.
    """
    abar = np.ascontiguousarray(abar, dtype=np.float64)
    bbar_x = np.ascontiguousarray(bbar_x, dtype=np.float64)
    c = np.ascontiguousarray(c, dtype=np.float64)
    L, N = abar.shape
    if bbar_x.shape != (L, N) or c.shape != (L, N):
        raise ValueError("abar, bbar_x, c must share the shape [L, N]")
    h = np.empty((L, N), dtype=np.float64)
    y = np.empty((L,), dtype=np.float64)
    rc = _load().mss_oracle_recurrence(_dptr(abar), _dptr(bbar_x), _dptr(c), L, N,
                                       _dptr(h), _dptr(y))
    if rc != 0:
        raise RuntimeError(f"mss_oracle_recurrence failed with code {rc}")
    return h, y
