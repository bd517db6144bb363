"""sscan_fwd_noalloc: the forward scan for callers that cannot allocate device memory.

Some callers may not call cudaMalloc at all -- a plugin running inside a host
framework that owns the whole device memory pool, or latency-critical code that
cannot take cudaMalloc's implicit device synchronisation.  For them the library
keeps its scratch in a fixed device array of its own, so the call needs no
workspace argument.  These tests call that entry point through the C ABI on long
sequences with few channels (the case that does need scratch: per-chunk states for
the cross-chunk carry), once through the TMA-tiled kernels and once, with inputs
that start off a 16-byte boundary, through the general row kernels.  Each case runs
twice in a row with different inputs, so stale scratch contents from the first call
cannot leak into the second.  Both entry points run the same kernels on the same
plan, so their results must be identical bit for bit; the oracle checks both.  The
file is named to run last.
"""
import ctypes

import numpy as np
import pytest

import oracle
from selective_state_space_33_b200 import binding as sb
from selective_state_space_33_b200 import workloads as W

from .helpers import TOL, normwise, to_f64, to_torch


def _lib():
    lib = sb.load_library()
    vp = ctypes.c_void_p
    lib.sscan_fwd_noalloc.argtypes = [ctypes.POINTER(sb.Problem)] + [vp] * 11 + [vp]
    lib.sscan_fwd_noalloc.restype = ctypes.c_int
    return lib


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def test_noalloc_rejects_problems_beyond_its_scratch():
    """Host-side size check.  Unaligned tensors go down the general path, whose plan
    for a million steps over 1536 channels needs more than the fixed 4 MiB scratch,
    so the call must refuse before launching anything."""
    lib = _lib()
    big = sb.make_problem(1, 1 << 20, 1536, 16, sb.SSCAN_F32)
    odd = ctypes.c_void_p(0x10004)   # 4-byte aligned only; never dereferenced
    fake = ctypes.c_void_p(0x10000)
    args = [odd, odd, fake, fake, fake, fake, fake, odd, None, odd, fake]
    rc = lib.sscan_fwd_noalloc(ctypes.byref(big), *args, None)
    assert rc == 3  # SSCAN_ERR_WORKSPACE
    assert b"static scratch" in lib.sscan_last_error()


def _offset_copy(t):
    """The same values one element past a 16-byte boundary (general row kernels)."""
    import torch
    buf = torch.empty(t.numel() + 1, dtype=t.dtype, device=t.device)
    v = buf[1:].view(t.shape)
    v.copy_(t)
    return v


@pytest.mark.gpu
@pytest.mark.parametrize("path,shape", [("tiled", (1, 1 << 15, 64, 16)), ("rows", (1, 1 << 15, 8, 16))])
def test_noalloc_matches_sscan_fwd_twice(cuda_device, path, shape):
    import torch
    lib = _lib()
    batch, L, D, N = shape
    prob = sb.make_problem(batch, L, D, N, sb.SSCAN_F32)
    assert sb.sscan_workspace_size(prob, sb.SSCAN_OP_FWD) > 0  # this case uses scratch
    for seed in (901, 902):
        x = W.small_case(batch, L, D, N, io="f32", seed=seed)
        t = to_torch(x, cuda_device)
        if path == "rows":
            for k in ("u", "delta_raw", "z"):
                t[k] = _offset_copy(t[k])
        h0_np = np.random.default_rng(seed).standard_normal((batch, D, N)).astype(np.float32)
        h0 = torch.from_numpy(h0_np).to(cuda_device)
        ref_out, ref_h = sb.sscan_fwd(t["u"], t["delta_raw"], t["A"], t["B"], t["C"], t["delta_bias"],
                                      t["D_skip"], t["z"], h0, return_last_state=True)
        assert sb.load_library().sscan_last_launch_count() >= 3  # chunk pass, carry, output pass
        out = torch.full_like(ref_out, float("nan"))
        h_last = torch.full_like(ref_h, float("nan"))
        stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        rc = lib.sscan_fwd_noalloc(ctypes.byref(prob), _p(t["u"]), _p(t["delta_raw"]), _p(t["delta_bias"]),
                                   _p(t["A"]), _p(t["B"]), _p(t["C"]), _p(t["D_skip"]), _p(t["z"]), _p(h0),
                                   _p(out), _p(h_last), stream)
        assert rc == 0, lib.sscan_last_error()
        torch.cuda.synchronize()
        assert torch.equal(out, ref_out)
        assert torch.equal(h_last, ref_h)
        ref, ref_hl = oracle.fwd(x["u"], x["delta_raw"], x["A"], x["B"], x["C"], delta_bias=x["delta_bias"],
                                 D_skip=x["D_skip"], z=x["z"], h0=h0_np.astype(np.float64))
        assert normwise(to_f64(out), ref) <= TOL["f32"]
        assert normwise(to_f64(h_last), ref_hl) <= TOL["f32"]
