"""The debug build (libsscan_debug.so: every computed index into a workspace, parameter
or state array checked, a bad one reported through bit 3 of the device status word
and its access skipped) on the paths whose workspace layouts are most involved: the
sequence split of the tiled and the general forward kernels, and the segmented
reverse sweep of the tiled and the general backward kernels.  Each must match the
oracle with the status word clear."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from selective_state_space_33_b200 import binding as sb
from selective_state_space_33_b200 import build as lib_build
from selective_state_space_33_b200 import workloads as W

from .helpers import TOL, normwise, to_f64, to_torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dbg():
    lib = sb.load_library(lib_build.build(debug=True))
    lib.sscan_debug_bounds.restype = ctypes.c_int
    assert lib.sscan_debug_bounds() == 1
    return lib


def _status(lib):
    flags = ctypes.c_uint(0)
    rc = lib.sscan_device_status(1, ctypes.byref(flags))
    return rc, flags.value


def _offset(t):
    buf = torch.empty(t.numel() + 1, dtype=t.dtype, device=t.device)
    v = buf[1:].view(t.shape)
    v.copy_(t)
    return v


@pytest.mark.parametrize("general", [False, True])
def test_forward_with_sequence_split(cuda_device, dbg, monkeypatch, general):
    monkeypatch.setattr(sb, "_lib", dbg)
    _status(dbg)
    x = W.small_case(1, 20000, 64, 16, io="f32", seed=301)
    t = to_torch(x, cuda_device)
    if general:
        for k in ("u", "delta_raw", "z"):
            t[k] = _offset(t[k])
    h0 = np.random.default_rng(301).standard_normal((1, 64, 16)).astype(np.float32)
    out, hl = sb.sscan_fwd(t["u"], t["delta_raw"], t["A"], t["B"], t["C"], t["delta_bias"], t["D_skip"], t["z"],
                           torch.from_numpy(h0).to(cuda_device), return_last_state=True)
    assert dbg.sscan_last_launch_count() >= 3   # chunk pass, carry, output pass
    torch.cuda.synchronize()
    assert _status(dbg) == (0, 0)
    ref, ref_h = oracle.fwd(x["u"], x["delta_raw"], x["A"], x["B"], x["C"], delta_bias=x["delta_bias"],
                            D_skip=x["D_skip"], z=x["z"], h0=h0.astype(np.float64))
    assert normwise(to_f64(out), ref) <= TOL["f32"]
    assert normwise(to_f64(hl), ref_h) <= TOL["f32"]


@pytest.mark.parametrize("general", [False, True])
def test_backward_with_segments(cuda_device, dbg, monkeypatch, general):
    monkeypatch.setattr(sb, "_lib", dbg)
    _status(dbg)
    x = W.small_case(1, 1000, 64, 16, io="bf16", seed=302, backward=True)
    t = to_torch(x, cuda_device)
    if general:
        for k in ("u", "delta_raw", "z", "dout"):
            t[k] = _offset(t[k])
    h0 = np.random.default_rng(302).standard_normal((1, 64, 16)).astype(np.float32) * 0.3
    g = sb.sscan_bwd(t["u"], t["delta_raw"], t["A"], t["B"], t["C"], t["dout"], t["delta_bias"], t["D_skip"],
                     t["z"], torch.from_numpy(h0).to(cuda_device))
    torch.cuda.synchronize()
    assert _status(dbg) == (0, 0)
    ref = oracle.bwd(x["u"], x["delta_raw"], x["A"], x["B"], x["C"], x["dout"], delta_bias=x["delta_bias"],
                     D_skip=x["D_skip"], z=x["z"], h0=h0.astype(np.float64))
    errs = {k: normwise(to_f64(g[k]), ref[k]) for k in ref}
    assert all(e <= TOL["bf16"] for e in errs.values()), errs
