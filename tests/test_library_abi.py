"""The C-ABI library loads, exports every symbol include/sscan.h declares, and
rejects bad arguments on the host before touching a device.  CPU only: no call
here reaches a kernel launch or a CUDA runtime call."""
import ctypes
import os
import re

import pytest

from selective_state_space_33_b200 import binding as sb
from selective_state_space_33_b200 import build as lib_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    lib_build.build()
    return sb.load_library()


def _declared_symbols():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"SSCAN_API\s+[\w\s\*]*?\b(sscan_\w+)\s*\(", text)
    return names


def test_every_declared_symbol_is_exported(lib):
    names = _declared_symbols()
    assert {"sscan_fwd", "sscan_last_state", "sscan_bwd", "sscan_workspace_size"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n
        assert ctypes.cast(getattr(lib, n), ctypes.c_void_p).value


def test_version_and_status_strings(lib):
    assert lib.sscan_version() >= 100
    assert lib.sscan_status_string(0) == b"SSCAN_OK"
    assert lib.sscan_status_string(3) == b"SSCAN_ERR_WORKSPACE"
    assert lib.sscan_status_string(99) == b"SSCAN_ERR_UNKNOWN"


def _p(batch=2, L=64, D=32, N=16, io=0, flags=1):
    return sb.Problem(batch, L, D, N, io, flags)


def _fwd(lib, p, **ptrs):
    names = ["u", "delta_raw", "delta_bias", "A", "B", "C", "D_skip", "z", "h0", "out", "h_last"]
    fake = ctypes.c_void_p(0x10000)  # never dereferenced: every case below fails validation first
    args = [ptrs.get(n, fake) for n in names]
    return lib.sscan_fwd(ctypes.byref(p), *args, ptrs.get("ws", None), ptrs.get("ws_bytes", 0), None)


def test_fwd_rejects_bad_arguments(lib):
    assert lib.sscan_fwd(None, *([None] * 11), None, 0, None) == 1
    assert _fwd(lib, _p(batch=-1)) == 1
    assert _fwd(lib, _p(N=0)) == 1
    assert _fwd(lib, _p(N=17)) == 2
    assert b"dstate" in lib.sscan_last_error()
    assert _fwd(lib, _p(io=7)) == 1
    assert _fwd(lib, _p(flags=6)) == 1
    assert b"0x4" in lib.sscan_last_error()
    # SSCAN_DELTA_SOFTPLUS | SSCAN_INPUT_SILU is a valid flag set: validation goes on to
    # the pointers
    assert _fwd(lib, _p(flags=3), u=None) == 1
    assert b"required" in lib.sscan_last_error()
    assert _fwd(lib, _p(), u=None) == 1
    assert _fwd(lib, _p(), out=None, h_last=None) == 1
    assert b"both NULL" in lib.sscan_last_error()
    assert _fwd(lib, _p(), C=None) == 1


def test_workspace_is_required_when_planned(lib):
    # few rows and a long sequence: the forward pass splits L and needs a workspace
    p = _p(batch=1, L=1 << 20, D=1536, N=16, io=1)
    need = lib.sscan_workspace_size(ctypes.byref(p), 0)
    assert need > 0 and need % 256 == 0
    assert _fwd(lib, p, ws=None, ws_bytes=0) == 3
    assert _fwd(lib, p, ws=ctypes.c_void_p(0x10000), ws_bytes=need - 1) == 3
    assert lib.sscan_workspace_size(ctypes.byref(p), 1) == need
    # many rows: no split, no workspace
    assert lib.sscan_workspace_size(ctypes.byref(_p(batch=8, L=2048, D=5120)), 0) == 0
    # backward always keeps checkpoints
    assert lib.sscan_workspace_size(ctypes.byref(_p(batch=8, L=2048, D=1536)), 2) > 0
    assert lib.sscan_workspace_size(ctypes.byref(_p(N=0)), 0) == 0
    assert lib.sscan_workspace_size(ctypes.byref(_p()), 9) == 0


def test_backward_workspaces_hold_their_documented_contents(lib):
    """Host-side sizing only (no device work): the complex backward's workspace is the
    fp32 dB, dC accumulators (2 x batch L N) plus the complex state before every 8th step
    (batch x ceil(L/8) x D x N x 2 floats), rounded up to 256 bytes; the real backward's
    holds at least the accumulators and the fp32 checkpoints (batch x ceil(L/8) x D x N);
    empty problems need none."""
    for batch, L, D, N in ((8, 2048, 1536, 16), (2, 777, 40, 8), (1, 9, 5, 1)):
        p = _p(batch=batch, L=L, D=D, N=N, io=1)
        nck = -(-L // 8)
        floats = 2 * batch * L * N + batch * nck * D * N * 2
        assert lib.sscan_workspace_size(ctypes.byref(p), 4) == -(-floats * 4 // 256) * 256
        need = lib.sscan_workspace_size(ctypes.byref(p), 2)
        assert need >= (2 * batch * L * N + batch * nck * D * N) * 4 and need % 256 == 0
    for batch, L, D in ((0, 10, 4), (2, 0, 4), (2, 10, 0)):
        assert lib.sscan_workspace_size(ctypes.byref(_p(batch=batch, L=L, D=D, N=4)), 4) == 0


def test_last_state_and_bwd_reject_bad_arguments(lib):
    p = _p()
    fake = ctypes.c_void_p(0x10000)
    assert lib.sscan_last_state(ctypes.byref(p), fake, fake, None, fake, fake, None, None, None, 0, None) == 1
    # dz without z
    args = [fake] * 19
    args[7] = None   # z
    args[17] = fake  # dz
    assert lib.sscan_bwd(ctypes.byref(p), *args, None, 0, None) == 1
    assert b"dz" in lib.sscan_last_error()
    # dD without D_skip
    args = [fake] * 19
    args[6] = None   # D_skip
    assert lib.sscan_bwd(ctypes.byref(p), *args, None, 0, None) == 1


def test_binding_refuses_cpu_tensors(lib):
    import torch
    u = torch.zeros(1, 4, 4)
    with pytest.raises(ValueError):
        sb.sscan_fwd(u, u, torch.zeros(4, 4), torch.zeros(1, 4, 4), torch.zeros(1, 4, 4))


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(sb.SscanError):
        sb.load_library(str(tmp_path / "nope.so"))


def test_step_requires_single_token(lib):
    fake = ctypes.c_void_p(0x10000)
    p = _p(L=2)
    assert lib.sscan_step(ctypes.byref(p), *([fake] * 10), None) == 1
    assert b"seqlen" in lib.sscan_last_error()
    p = _p(L=1)
    args = [fake] * 10
    args[8] = None  # state
    assert lib.sscan_step(ctypes.byref(p), *args, None) == 1


def test_debug_build_exports_the_same_interface(lib):
    """The debug build (index checks compiled in, reported through the device status
    word) exports the same symbols and says which build it is; the release build
    compiles the checks out."""
    path = lib_build.build(debug=True)
    dbg = sb.load_library(path)
    for n in _declared_symbols():
        assert hasattr(dbg, n), n
    dbg.sscan_debug_bounds.restype = ctypes.c_int
    lib.sscan_debug_bounds.restype = ctypes.c_int
    assert dbg.sscan_debug_bounds() == 1
    assert lib.sscan_debug_bounds() == 0
