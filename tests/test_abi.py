"""The C ABI: the library loads and exports what include/mss.h declares, and
argument errors are reported before any launch (so these run without a GPU:
every call below fails a host-side check and touches no device)."""
import ctypes
import os
import re

import pytest
import torch

import selective_state_space_mss_b200 as mss
from selective_state_space_mss_b200 import build as mss_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mss.h")


@pytest.fixture(scope="module")
def lib():
    mss_build.build()
    return mss.load_library()


def _header():
    with open(HEADER) as f:
        return f.read()


def _declared_functions():
    return re.findall(r"^MSS_API\s+[\w\s\*]+?\b(mss_\w+)\s*\(", _header(), flags=re.M)


def _enum(name):
    body = re.search(r"enum %s \{(.*?)\};" % name, _header(), flags=re.S).group(1)
    return {k: int(v) for k, v in re.findall(r"(MSS_\w+)\s*=\s*(-?\d+)", body)}


def test_exports_every_declared_symbol(lib):
    declared = _declared_functions()
    assert set(declared) >= {"mss_scan_fwd", "mss_scan_fwd_ex", "mss_state_update",
                             "mss_get_device_error", "mss_strerror", "mss_version"}
    for name in declared:
        assert hasattr(lib, name), f"{name} declared in mss.h but not exported"


def test_exports_nothing_else(lib):
    out = os.popen(f"nm -D --defined-only {mss.library_path()}").read()
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    assert exported == set(_declared_functions())


def test_version_and_strerror(lib):
    ver = int(re.search(r"#define MSS_VERSION (\d+)", _header()).group(1))
    assert lib.mss_version() == ver
    codes = _enum("mss_status")
    texts = {lib.mss_strerror(c).decode() for c in codes.values()}
    assert len(texts) == len(codes) and all(texts)
    assert lib.mss_strerror(12345).decode() == "unknown status code"


P = 0x10000  # a fake, 256-byte aligned address: never dereferenced below


def _fwd(lib, **kw):
    a = dict(u=P, delta=P + 0x1000000, A=P + 0x2000000, B=P + 0x3000000, C=P + 0x4000000,
             D=None, z=None, bias=None, softplus=1, y=P + 0x5000000, last=None,
             batch=2, dim=8, N=16, L=32, dtype=1, flags=0)
    a.update(kw)
    v = lambda x: ctypes.c_void_p(x) if x is not None else None
    return lib.mss_scan_fwd_ex(v(a["u"]), v(a["delta"]), v(a["A"]), v(a["B"]), v(a["C"]),
                               v(a["D"]), v(a["z"]), v(a["bias"]), a["softplus"], v(a["y"]),
                               v(a["last"]), a["batch"], a["dim"], a["N"], a["L"], a["dtype"],
                               a["flags"], None)


def test_forward_argument_errors(lib):
    codes = _enum("mss_status")
    assert _fwd(lib, dtype=7) == codes["MSS_ERR_DTYPE"]
    assert _fwd(lib, flags=0x100) == codes["MSS_ERR_FLAGS"]
    assert _fwd(lib, batch=-1) == codes["MSS_ERR_SHAPE"]
    assert _fwd(lib, L=-5) == codes["MSS_ERR_SHAPE"]
    assert _fwd(lib, batch=2 ** 40, dim=2 ** 30) == codes["MSS_ERR_SHAPE"]
    for n in (0, 3, 32, -16):
        assert _fwd(lib, N=n) == codes["MSS_ERR_UNSUPPORTED_N"]
    for k in ("u", "delta", "A", "B", "C", "y"):
        assert _fwd(lib, **{k: None}) == codes["MSS_ERR_NULL"], k
    assert _fwd(lib, u=P + 1) == codes["MSS_ERR_ALIGN"]
    assert _fwd(lib, A=P + 2) == codes["MSS_ERR_ALIGN"]
    assert _fwd(lib, dtype=0, z=P + 0x6000002) == codes["MSS_ERR_ALIGN"]
    assert _fwd(lib, y=P + 64) == codes["MSS_ERR_ALIAS"]          # y inside u
    assert _fwd(lib, last=P + 0x3000000) == codes["MSS_ERR_ALIAS"]  # last_state on B
    # nothing to do: accepted without a launch
    assert _fwd(lib, batch=0) == 0 and _fwd(lib, dim=0, u=None) == 0


def test_decode_argument_errors(lib):
    codes = _enum("mss_status")
    v = ctypes.c_void_p

    def step(**kw):
        a = dict(state=P, u=P + 0x1000000, delta=P + 0x2000000, A=P + 0x3000000,
                 B=P + 0x4000000, C=P + 0x5000000, y=P + 0x6000000, batch=4, dim=8, N=16, dtype=1)
        a.update(kw)
        w = lambda x: v(x) if x is not None else None
        return lib.mss_state_update(w(a["state"]), w(a["u"]), w(a["delta"]), w(a["A"]), w(a["B"]),
                                    w(a["C"]), None, None, None, 1, w(a["y"]), a["batch"],
                                    a["dim"], a["N"], a["dtype"], None)

    assert step(dtype=2) == codes["MSS_ERR_DTYPE"]
    assert step(N=5) == codes["MSS_ERR_UNSUPPORTED_N"]
    assert step(dim=-1) == codes["MSS_ERR_SHAPE"]
    assert step(state=None) == codes["MSS_ERR_NULL"]
    assert step(state=P + 2) == codes["MSS_ERR_ALIGN"]
    assert step(y=P + 8) == codes["MSS_ERR_ALIAS"]  # y on the state
    assert step(batch=0) == 0

    def step_ex(flags, **kw):
        a = dict(state=P, u=P + 0x1000000, delta=P + 0x2000000, A=P + 0x3000000,
                 B=P + 0x4000000, C=P + 0x5000000, y=P + 0x6000000, batch=4, dim=8, N=16, dtype=1)
        a.update(kw)
        w = lambda x: v(x) if x is not None else None
        return lib.mss_state_update_ex(w(a["state"]), w(a["u"]), w(a["delta"]), w(a["A"]), w(a["B"]),
                                       w(a["C"]), None, None, None, 1, w(a["y"]), a["batch"],
                                       a["dim"], a["N"], a["dtype"], ctypes.c_uint(flags), None)

    flag_zoh = int(re.search(r"#define MSS_FLAG_ZOH_INPUT (0x[0-9a-f]+)u", _header()).group(1), 16)
    assert step_ex(0x1) == codes["MSS_ERR_FLAGS"]        # only the input-rule flag applies to decode
    assert step_ex(flag_zoh, N=5) == codes["MSS_ERR_UNSUPPORTED_N"]
    assert step_ex(flag_zoh, state=None) == codes["MSS_ERR_NULL"]
    assert step_ex(flag_zoh, batch=0) == 0


def test_binding_refuses_cpu_tensors():
    import torch

    x = torch.zeros(1, 2, 3)
    with pytest.raises(ValueError, match="CUDA"):
        mss.scan_fwd(x, x, torch.zeros(2, 4), x, x)


def test_ex2_and_workspace_argument_errors(lib):
    codes = _enum("mss_status")
    v = ctypes.c_void_p

    def ex2(**kw):
        a = dict(u=P, delta=P + 0x1000000, A=P + 0x2000000, B=P + 0x3000000, C=P + 0x4000000,
                 h0=None, y=P + 0x5000000, last=None, ws=None, wsb=0, batch=2, dim=8, N=16, L=32,
                 dtype=1, flags=0)
        a.update(kw)
        w = lambda x: v(x) if x is not None else None
        return lib.mss_scan_fwd_ex2(w(a["u"]), w(a["delta"]), w(a["A"]), w(a["B"]), w(a["C"]), None, None,
                                    None, 1, w(a["h0"]), w(a["y"]), w(a["last"]), a["batch"], a["dim"],
                                    a["N"], a["L"], a["dtype"], a["flags"], w(a["ws"]), a["wsb"], None)

    assert ex2(flags=0x80) == codes["MSS_ERR_FLAGS"]
    assert ex2(wsb=-1) == codes["MSS_ERR_SHAPE"]
    assert ex2(h0=P + 0x6000002) == codes["MSS_ERR_ALIGN"]
    assert ex2(ws=P + 0x6000001, wsb=64) == codes["MSS_ERR_ALIGN"]
    assert ex2(h0=P + 0x7000000, last=P + 0x7000000) == codes["MSS_ERR_ALIAS"]   # h0 on last_state
    assert ex2(ws=P + 0x5000000, wsb=256) == codes["MSS_ERR_ALIAS"]              # workspace on y
    assert ex2(ws=P + 0x2000000, wsb=256) == codes["MSS_ERR_ALIAS"]              # workspace on A
    assert ex2(batch=0) == 0
    assert ex2(flags=0x8, batch=0) == 0      # zero-order-hold input rule: a known flag


def test_workspace_size_queries(lib):
    codes = _enum("mss_status")
    lib.mss_scan_fwd_workspace_size.restype = ctypes.c_int64
    q = lambda *a: lib.mss_scan_fwd_workspace_size(*a)
    assert q(1, 16, 16, 4096, 7, 0) == codes["MSS_ERR_DTYPE"]
    assert q(1, 16, 3, 4096, 1, 0) == codes["MSS_ERR_UNSUPPORTED_N"]
    assert q(-1, 16, 16, 4096, 1, 0) == codes["MSS_ERR_SHAPE"]
    assert q(1, 16, 16, 4096, 1, 0x80) == codes["MSS_ERR_FLAGS"]
    assert q(1, 16, 16, 4096, 1, 0x8) >= 0
    # no split: scalar kernel, split disabled, nothing to do, rows not 16-byte multiples
    assert q(1, 16, 16, 4096, 1, 0x2) == 0
    assert q(1, 16, 16, 4096, 1, 0x4) == 0
    assert q(1, 16, 16, 0, 1, 0) == 0
    assert q(1, 16, 16, 4097, 1, 0) == 0
    assert q(1, 16, 2, 4096, 1, 0) == 0


def test_conv_argument_errors(lib):
    codes = _enum("mss_status")
    v = ctypes.c_void_p
    lib.mss_scan_fwd_conv.restype = ctypes.c_int
    lib.mss_state_update_conv.restype = ctypes.c_int

    def fwd(**kw):
        a = dict(x=P, w=P + 0x1000000, b=None, K=4, csi=None, cso=P + 0x2000000, delta=P + 0x3000000,
                 A=P + 0x4000000, B=P + 0x5000000, C=P + 0x6000000, y=P + 0x7000000, batch=2, dim=8, N=16,
                 L=32, dtype=1)
        a.update(kw)
        w = lambda x: v(x) if x is not None else None
        return lib.mss_scan_fwd_conv(w(a["x"]), w(a["w"]), w(a["b"]), a["K"], w(a["csi"]), w(a["cso"]),
                                     w(a["delta"]), w(a["A"]), w(a["B"]), w(a["C"]), None, None, None, 1, None,
                                     w(a["y"]), None, ctypes.c_int64(a["batch"]), ctypes.c_int64(a["dim"]),
                                     ctypes.c_int64(a["N"]), ctypes.c_int64(a["L"]), a["dtype"], ctypes.c_uint(0),
                                     None, ctypes.c_int64(0), None)

    assert fwd(K=0) == codes["MSS_ERR_SHAPE"]
    assert fwd(K=5) == codes["MSS_ERR_SHAPE"]
    assert fwd(w=None) == codes["MSS_ERR_NULL"]
    assert fwd(cso=P + 0x2000001) == codes["MSS_ERR_ALIGN"]          # bf16 conv state: 2-byte elements
    assert fwd(w=P + 0x1000002) == codes["MSS_ERR_ALIGN"]            # fp32 taps
    assert fwd(cso=P + 0x7000000) == codes["MSS_ERR_ALIAS"]          # conv state out on y
    assert fwd(cso=P + 0x1000000) == codes["MSS_ERR_ALIAS"]          # conv state out on the taps
    assert fwd(batch=0) == 0

    def step(**kw):
        a = dict(state=P, cs=P + 0x1000000, x=P + 0x2000000, w=P + 0x3000000, K=4, delta=P + 0x4000000,
                 A=P + 0x5000000, B=P + 0x6000000, C=P + 0x7000000, y=P + 0x8000000, batch=4, dim=8, N=16,
                 dtype=1, flags=0)
        a.update(kw)
        w = lambda x: v(x) if x is not None else None
        return lib.mss_state_update_conv(w(a["state"]), w(a["cs"]), w(a["x"]), w(a["w"]), None, a["K"],
                                         w(a["delta"]), w(a["A"]), w(a["B"]), w(a["C"]), None, None, None, 1,
                                         w(a["y"]), ctypes.c_int64(a["batch"]), ctypes.c_int64(a["dim"]),
                                         ctypes.c_int64(a["N"]), a["dtype"], ctypes.c_uint(a["flags"]), None)

    assert step(K=0) == codes["MSS_ERR_SHAPE"]
    assert step(K=5) == codes["MSS_ERR_SHAPE"]
    assert step(cs=None) == codes["MSS_ERR_NULL"]
    assert step(w=None) == codes["MSS_ERR_NULL"]
    assert step(cs=P + 0x1000001) == codes["MSS_ERR_ALIGN"]
    assert step(cs=P + 0x40) == codes["MSS_ERR_ALIAS"]               # conv state on the state
    assert step(cs=P + 0x2000000) == codes["MSS_ERR_ALIAS"]          # conv state on x
    assert step(flags=0x1) == codes["MSS_ERR_FLAGS"]
    assert step(batch=0) == 0


def test_bwd_argument_errors(lib):
    codes = _enum("mss_status")
    v = ctypes.c_void_p
    lib.mss_scan_bwd.restype = ctypes.c_int
    lib.mss_scan_bwd_workspace_size.restype = ctypes.c_int64

    def bwd(**kw):
        a = dict(u=P, delta=P + 0x1000000, A=P + 0x2000000, B=P + 0x3000000, C=P + 0x4000000, z=None,
                 dy=P + 0x5000000, du=P + 0x6000000, ddelta=P + 0x7000000, dz=None, dA=P + 0x8000000,
                 dB=P + 0x9000000, dC=P + 0xa000000, ws=P + 0xb000000, wsb=1 << 20, batch=2, dim=8, N=16, L=32,
                 dtype=1, flags=0)
        a.update(kw)
        w = lambda x: v(x) if x is not None else None
        return lib.mss_scan_bwd(w(a["u"]), w(a["delta"]), w(a["A"]), w(a["B"]), w(a["C"]), None, w(a["z"]), None, 1,
                                None, w(a["dy"]), None, w(a["du"]), w(a["ddelta"]), w(a["dz"]), w(a["dA"]),
                                w(a["dB"]), w(a["dC"]), None, None, None, ctypes.c_int64(a["batch"]),
                                ctypes.c_int64(a["dim"]), ctypes.c_int64(a["N"]), ctypes.c_int64(a["L"]), a["dtype"],
                                ctypes.c_uint(a["flags"]), w(a["ws"]), ctypes.c_int64(a["wsb"]), None)

    assert bwd(dtype=3) == codes["MSS_ERR_DTYPE"]
    assert bwd(flags=0x4) == codes["MSS_ERR_FLAGS"]      # no sequence split in the backward pass
    assert bwd(N=3) == codes["MSS_ERR_UNSUPPORTED_N"]
    assert bwd(L=-1) == codes["MSS_ERR_SHAPE"]
    assert bwd(dy=None) == codes["MSS_ERR_NULL"]
    assert bwd(z=P + 0xc000000) == codes["MSS_ERR_NULL"]  # z given without dz
    assert bwd(dB=P + 0x9000002) == codes["MSS_ERR_ALIGN"]
    assert bwd(du=P + 0x5000000) == codes["MSS_ERR_ALIAS"]   # du on dy
    assert bwd(dC=P + 0x9000000) == codes["MSS_ERR_ALIAS"]   # dC on dB
    assert bwd(ws=P + 0x8000000) == codes["MSS_ERR_ALIAS"]   # workspace on dA
    assert bwd(batch=0) == 0
    q = lambda *a: lib.mss_scan_bwd_workspace_size(*a)
    assert q(1, 16, 16, 4096, 1, 0) == 16 * 512 * 16 * 4           # one state per 8-token group
    assert q(1, 16, 16, 4096, 1, 0x2) == 16 * 256 * 16 * 4         # scalar path: one per 16 tokens
    assert q(1, 16, 16, 4097, 1, 0) == 16 * 257 * 16 * 4           # odd rows take the scalar path
    assert q(1, 16, 16, 0, 1, 0) == 0
    assert q(1, 16, 3, 64, 1, 0) == codes["MSS_ERR_UNSUPPORTED_N"]
    # more batch rows than the tiled kernels' grid takes: the scalar path's size
    assert q(70000, 16, 16, 64, 1, 0) == 70000 * 16 * 4 * 16 * 4
    assert q(65535, 16, 16, 64, 1, 0) == 65535 * 16 * 8 * 16 * 4
    assert q(1, 16, 16, 4096, 0, 0) == 16 * 1024 * 16 * 4          # fp32: one per 4-token group


def test_saved_states_argument_errors(lib):
    """mss_scan_fwd_save and MSS_FLAG_SAVED_STATES: the checks that need no
    device (sizes, alignment, overlap, the tiled-path test)."""
    codes = _enum("mss_status")
    flag = int(re.search(r"#define MSS_FLAG_SAVED_STATES (0x[0-9a-f]+)u", _header()).group(1), 16)
    v = ctypes.c_void_p
    lib.mss_scan_fwd_save.restype = ctypes.c_int
    lib.mss_scan_bwd.restype = ctypes.c_int
    lib.mss_scan_bwd_workspace_size.restype = ctypes.c_int64
    need = lib.mss_scan_bwd_workspace_size(ctypes.c_int64(2), ctypes.c_int64(8), ctypes.c_int64(16),
                                           ctypes.c_int64(32), 1, ctypes.c_uint(0))
    assert need == 2 * 8 * 4 * 16 * 4  # one state per 8-token group
    assert lib.mss_scan_bwd_workspace_size(ctypes.c_int64(2), ctypes.c_int64(8), ctypes.c_int64(16),
                                           ctypes.c_int64(32), 1, ctypes.c_uint(flag)) == need

    def save(**kw):
        a = dict(u=P, delta=P + 0x1000000, B=P + 0x3000000, C=P + 0x4000000, y=P + 0x5000000,
                 st=P + 0x6000000, stb=need, batch=2, dim=8, N=16, L=32, dtype=1, flags=0)
        a.update(kw)
        w = lambda x: v(x) if x is not None else None
        return lib.mss_scan_fwd_save(w(a["u"]), w(a["delta"]), v(P + 0x2000000), w(a["B"]), w(a["C"]), None, None,
                                     None, 1, None, w(a["y"]), None, ctypes.c_int64(a["batch"]),
                                     ctypes.c_int64(a["dim"]), ctypes.c_int64(a["N"]), ctypes.c_int64(a["L"]),
                                     a["dtype"], ctypes.c_uint(a["flags"]), None, ctypes.c_int64(0), w(a["st"]),
                                     ctypes.c_int64(a["stb"]), None)

    assert save(st=None) == codes["MSS_ERR_WORKSPACE"]
    assert save(stb=need - 1) == codes["MSS_ERR_WORKSPACE"]
    assert save(stb=-1) == codes["MSS_ERR_SHAPE"]
    assert save(st=P + 0x6000008) == codes["MSS_ERR_ALIGN"]          # states need 16-byte alignment
    assert save(st=P + 0x5000000) == codes["MSS_ERR_ALIAS"]          # states on y
    assert save(st=P + 0x1000000) == codes["MSS_ERR_ALIAS"]          # states on delta
    assert save(flags=0x2, stb=1 << 20) == codes["MSS_ERR_PATH"]     # the scalar kernel stores none
    assert save(N=2, stb=1 << 20) == codes["MSS_ERR_PATH"]
    assert save(u=P + 2) == codes["MSS_ERR_PATH"]                   # rows not 16-byte aligned
    assert save(L=33, stb=1 << 20) == codes["MSS_ERR_PATH"]          # odd rows
    assert save(flags=0x80) == codes["MSS_ERR_FLAGS"]
    assert save(batch=0) == 0
    assert save(L=0, st=None, stb=0) == 0

    def bwd(**kw):
        a = dict(du=P + 0x6000000, dB=P + 0x9000000, N=16, L=32, flags=flag)
        a.update(kw)
        return lib.mss_scan_bwd(v(P), v(P + 0x1000000), v(P + 0x2000000), v(P + 0x3000000), v(P + 0x4000000), None,
                                None, None, 1, None, v(P + 0x5000000), None, v(a["du"]), v(P + 0x7000000), None,
                                v(P + 0x8000000), v(a["dB"]), v(P + 0xa000000), None, None, None, ctypes.c_int64(2),
                                ctypes.c_int64(8), ctypes.c_int64(a["N"]), ctypes.c_int64(a["L"]), 1,
                                ctypes.c_uint(a["flags"]), v(P + 0xb000000), ctypes.c_int64(1 << 20), None)

    assert bwd(flags=flag | 0x2) == codes["MSS_ERR_PATH"]
    assert bwd(N=2) == codes["MSS_ERR_PATH"]
    assert bwd(du=P + 0x6000002) == codes["MSS_ERR_PATH"]   # a gradient row not 16-byte aligned
    assert bwd(dB=P + 0x9000004) == codes["MSS_ERR_PATH"]
    assert bwd(flags=0x40) == codes["MSS_ERR_FLAGS"]
    assert "tiled" in lib.mss_strerror(codes["MSS_ERR_PATH"]).decode()


def test_ssd_argument_errors(lib):
    codes = _enum("mss_status")
    v = ctypes.c_void_p
    lib.mss_ssd_fwd.restype = ctypes.c_int

    def ssd(**kw):
        a = dict(x=P, dt=P + 0x1000000, A=P + 0x2000000, B=P + 0x3000000, C=P + 0x4000000, y=P + 0x5000000,
                 last=None, batch=2, L=64, H=4, Pd=64, G=1, N=128, dtype=1)
        a.update(kw)
        w = lambda x: v(x) if x is not None else None
        return lib.mss_ssd_fwd(w(a["x"]), w(a["dt"]), w(a["A"]), w(a["B"]), w(a["C"]), None, None, None, 1, None,
                               w(a["y"]), w(a["last"]), ctypes.c_int64(a["batch"]), ctypes.c_int64(a["L"]),
                               ctypes.c_int64(a["H"]), ctypes.c_int64(a["Pd"]), ctypes.c_int64(a["G"]),
                               ctypes.c_int64(a["N"]), a["dtype"], None)

    assert ssd(dtype=0) == codes["MSS_ERR_DTYPE"]          # the tensor-core path takes bf16
    assert ssd(Pd=32) == codes["MSS_ERR_SHAPE"]
    assert ssd(N=96) == codes["MSS_ERR_SHAPE"]
    assert ssd(H=3, G=2) == codes["MSS_ERR_SHAPE"]
    assert ssd(x=None) == codes["MSS_ERR_NULL"]
    assert ssd(B=P + 0x3000008) == codes["MSS_ERR_ALIGN"]
    assert ssd(y=P) == codes["MSS_ERR_ALIAS"]
    assert ssd(batch=0) == 0


def test_ssd_workspace_queries(lib):
    codes = _enum("mss_status")
    lib.mss_ssd_fwd_workspace_size.restype = ctypes.c_int64
    lib.mss_ssd_fwd_workspace_size_ex.restype = ctypes.c_int64
    q = lambda *a: lib.mss_ssd_fwd_workspace_size(*[ctypes.c_int64(x) for x in a])
    qx = lambda *a, flags=0: lib.mss_ssd_fwd_workspace_size_ex(*[ctypes.c_int64(x) for x in a], ctypes.c_uint(flags))
    warp = 0x1  # MSS_SSD_FLAG_WARP_MMA
    chunked = 2 * 4 * 2 * (128 * 64 * 6 + 4)  # per chunk of 64 tokens: fp32 chunk state, its bf16 copy, decay
    # 8 (batch, head) pairs take the warp-level chunk-parallel passes on a
    # device; without a device the in-order kernel, which takes no workspace
    ws = q(2, 128, 4, 64, 1, 64)
    assert ws == (2 * 4 * 2 * (64 * 64 * 6 + 4) if torch.cuda.is_available() else 0)
    assert qx(2, 128, 4, 64, 1, 128, flags=warp) == (chunked if torch.cuda.is_available() else 0)
    # dstate 128 runs the tcgen05 kernel in order: no workspace
    assert q(2, 128, 4, 64, 1, 128) == 0 and qx(2, 128, 4, 64, 1, 128) == 0
    assert q(2, 0, 4, 64, 1, 128) == 0
    assert q(2, 128, 4, 32, 1, 128) == codes["MSS_ERR_SHAPE"]
    assert q(2, 128, 3, 64, 2, 128) == codes["MSS_ERR_SHAPE"]
    assert qx(2, 128, 4, 64, 1, 128, flags=0x2) == codes["MSS_ERR_FLAGS"]
    if ws == 0 and torch.cuda.is_available():
        return  # the call below would launch on the made-up pointers
    lib.mss_ssd_fwd_ex.restype = ctypes.c_int
    v = ctypes.c_void_p
    rc = lib.mss_ssd_fwd_ex(v(P), v(P + 0x1000000), v(P + 0x2000000), v(P + 0x3000000), v(P + 0x4000000), None,
                            None, None, 1, None, v(P + 0x5000000), None, ctypes.c_int64(2), ctypes.c_int64(128),
                            ctypes.c_int64(4), ctypes.c_int64(64), ctypes.c_int64(1), ctypes.c_int64(64), 1,
                            v(P + 0x6000000), ctypes.c_int64(100), None)
    # too small (checked before any launch), or no device to launch on
    assert rc == (codes["MSS_ERR_WORKSPACE"] if ws else codes["MSS_ERR_CUDA"])


def test_ssd_ex2_flag_errors(lib):
    codes = _enum("mss_status")
    lib.mss_ssd_fwd_ex2.restype = ctypes.c_int
    v = ctypes.c_void_p

    def call(flags, dtype=1):
        return lib.mss_ssd_fwd_ex2(v(P), v(P + 0x1000000), v(P + 0x2000000), v(P + 0x3000000), v(P + 0x4000000),
                                   None, None, None, 1, None, v(P + 0x5000000), None, ctypes.c_int64(2),
                                   ctypes.c_int64(128), ctypes.c_int64(4), ctypes.c_int64(64), ctypes.c_int64(1),
                                   ctypes.c_int64(128), dtype, ctypes.c_uint(flags), None, ctypes.c_int64(0), None)

    assert call(0x2) == codes["MSS_ERR_FLAGS"]          # unknown bit, refused before anything else
    assert call(0x1, dtype=0) == codes["MSS_ERR_DTYPE"]  # bf16 io only, on either kernel


def test_host_call_argument_errors(lib):
    """mss_scan_fwd_host: every error below is found before anything is
    queued (the pointers are made up and never dereferenced)."""
    codes = _enum("mss_status")
    v = ctypes.c_void_p
    lib.mss_scan_fwd_host_workspace_size.restype = ctypes.c_int64
    need = lib.mss_scan_fwd_host_workspace_size(ctypes.c_int64(2), ctypes.c_int64(8), ctypes.c_int64(16),
                                                ctypes.c_int64(32), 1, 0, 0, 0, 0, 0)
    # A, B, C once; both batch rows fit one piece, so one slot of u, delta,
    # y for 2 x 8 channels x 32 tokens of bf16
    assert need == 512 + 2 * 2048 + 3 * 1024

    def host(**kw):
        a = dict(u=P, delta=P + 0x1000000, A=P + 0x2000000, B=P + 0x3000000, C=P + 0x4000000,
                 y=P + 0x5000000, last=None, ws=P + 0x6000000, wsb=need, batch=2, dim=8, N=16, L=32,
                 dtype=1, flags=0)
        a.update(kw)
        w = lambda x: v(x) if x is not None else None
        return lib.mss_scan_fwd_host(w(a["u"]), w(a["delta"]), w(a["A"]), w(a["B"]), w(a["C"]), None, None,
                                     None, 1, None, w(a["y"]), w(a["last"]), ctypes.c_int64(a["batch"]),
                                     ctypes.c_int64(a["dim"]), ctypes.c_int64(a["N"]), ctypes.c_int64(a["L"]),
                                     a["dtype"], a["flags"], w(a["ws"]), ctypes.c_int64(a["wsb"]), None)

    assert host(dtype=5) == codes["MSS_ERR_DTYPE"]
    assert host(flags=0x40) == codes["MSS_ERR_FLAGS"]
    assert host(batch=-1) == codes["MSS_ERR_SHAPE"]
    assert host(N=3) == codes["MSS_ERR_UNSUPPORTED_N"]
    assert host(u=None) == codes["MSS_ERR_NULL"]
    assert host(ws=None) == codes["MSS_ERR_NULL"]
    assert host(u=P + 1) == codes["MSS_ERR_ALIGN"]
    assert host(ws=P + 0x6000010) == codes["MSS_ERR_ALIGN"]        # 16 but not 256-byte aligned
    assert host(y=P + 0x1000000) == codes["MSS_ERR_ALIAS"]         # y on delta
    assert host(last=P + 0x5000000) == codes["MSS_ERR_ALIAS"]      # last_state on y
    assert host(wsb=need - 1) == codes["MSS_ERR_WORKSPACE"]
    assert host(batch=0) == 0
    q = lambda *a: lib.mss_scan_fwd_host_workspace_size(*[ctypes.c_int64(x) for x in a[:4]], *a[4:])
    assert q(0, 8, 16, 32, 1, 1, 1, 1, 1, 1) == 0
    assert q(2, 8, 16, 32, 9, 0, 0, 0, 0, 0) == codes["MSS_ERR_DTYPE"]
    assert q(2, 8, 5, 32, 1, 0, 0, 0, 0, 0) == codes["MSS_ERR_UNSUPPORTED_N"]
    # every optional input adds its own buffer: z one more [16 x 32] slot
    # tensor, D and bias [dim] floats, the two states [16 x 16] floats
    assert q(2, 8, 16, 32, 1, 1, 1, 1, 1, 1) == need + 1024 + 2 * 256 + 2 * 1024
    # rows beyond 64 MB of inputs are cut: 4144 channels x 4096 bf16 tokens with
    # z is about 100 MB a row, so two pieces of 2080 channels, three slots
    big = q(2, 4144, 16, 4096, 1, 1, 0, 0, 0, 0)
    params = 4144 * 16 * 4 + 2 * (2 * 16 * 4096 * 2)
    assert big == params + 3 * 4 * (2080 * 4096 * 2)


def test_plain_c_client_compiles_links_and_runs(lib):
    """include/mss.h is a C header and libmss.so a C library: a C99 program
    (tests/c_client.c) compiles against the header, links the library and
    makes the calls that need no GPU."""
    import shutil
    import subprocess

    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    out_dir = os.path.join(ROOT, "selective_state_space_mss_b200", "_build")
    os.makedirs(out_dir, exist_ok=True)
    exe = os.path.join(out_dir, "c_client")
    lib_dir = os.path.dirname(mss.library_path())
    build = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                            os.path.join(ROOT, "tests", "c_client.c"), "-o", exe, mss.library_path(),
                            "-Wl,-rpath," + lib_dir], capture_output=True, text=True)
    assert build.returncode == 0, build.stderr
    run = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0 and run.stdout.strip() == "ok", run.stdout + run.stderr


def test_probe_argument_errors(lib):
    codes = _enum("mss_status")
    buf = (ctypes.c_double * 4)()
    assert lib.mss_probe_pipe_rates(None, 4, None) == codes["MSS_ERR_NULL"]
    assert lib.mss_probe_pipe_rates(buf, -1, None) == codes["MSS_ERR_SHAPE"]
