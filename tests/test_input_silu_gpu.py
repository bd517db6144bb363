"""The input-branch activation (SSCAN_INPUT_SILU: the scan's input is x = SiLU(u),
Fig. 3 caption of the technical summary page) through every path of the library,
against the fp64 oracle run with the same flag.  Tolerances as everywhere: normwise
1e-4 for fp32 I/O, 2e-2 for bf16 I/O."""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_33_b200 import binding as sb
from selective_state_space_33_b200 import workloads as W

from .helpers import TOL, normwise, to_f64, to_torch

pytestmark = pytest.mark.gpu


def _offset(t):
    """Same values one element past a 16-byte boundary: the general row kernels."""
    buf = torch.empty(t.numel() + 1, dtype=t.dtype, device=t.device)
    v = buf[1:].view(t.shape)
    v.copy_(t)
    return v


def _fwd_case(x, io, dev, general=False, h0=None):
    t = to_torch(x, dev)
    if general:
        for k in ("u", "delta_raw", "z"):
            t[k] = _offset(t[k])
    h0_t = None if h0 is None else torch.from_numpy(h0.astype(np.float32)).to(dev)
    out, hl = sb.sscan_fwd(t["u"], t["delta_raw"], t["A"], t["B"], t["C"], t["delta_bias"], t["D_skip"], t["z"],
                           h0_t, input_silu=True, return_last_state=True)
    torch.cuda.synchronize()
    ref, ref_h = oracle.fwd(x["u"], x["delta_raw"], x["A"], x["B"], x["C"], delta_bias=x["delta_bias"],
                            D_skip=x["D_skip"], z=x["z"], input_silu=True,
                            h0=None if h0 is None else h0.astype(np.float32).astype(np.float64))
    assert normwise(to_f64(out), ref) <= TOL[io]
    assert normwise(to_f64(hl), ref_h) <= TOL[io]
    # the flag is applied (the plain scan differs)
    plain, _ = oracle.fwd(x["u"], x["delta_raw"], x["A"], x["B"], x["C"], delta_bias=x["delta_bias"],
                          D_skip=x["D_skip"], z=x["z"])
    assert normwise(plain, ref) > 10 * TOL[io]


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [(2, 100, 64, 16), (1, 70, 37, 16), (2, 50, 40, 4), (1, 33, 24, 8)])
def test_forward_tiled_and_general(cuda_device, io, shape):
    x = W.small_case(*shape, io=io, seed=sum(shape) + 200)
    h0 = np.random.default_rng(2).standard_normal((shape[0], shape[2], shape[3])) * 0.5
    _fwd_case(x, io, cuda_device, h0=h0)
    _fwd_case(x, io, cuda_device, general=True, h0=h0)


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_forward_sequence_split(cuda_device, io):
    """Few channels and a long sequence: the chunk pass, the carry and the output pass
    all see the activated input."""
    x = W.small_case(1, 20000, 64, 16, io=io, seed=201)
    _fwd_case(x, io, cuda_device)
    _fwd_case(x, io, cuda_device, general=True)


def test_last_state_and_summary(cuda_device):
    x = W.small_case(2, 3000, 32, 16, io="f32", seed=202)
    t = to_torch(x, cuda_device)
    hl = sb.sscan_last_state(t["u"], t["delta_raw"], t["A"], t["B"], t["delta_bias"], input_silu=True)
    P, H = sb.sscan_chunk_summary(t["u"], t["delta_raw"], t["A"], t["B"], t["delta_bias"], input_silu=True)
    torch.cuda.synchronize()
    _, ref_h = oracle.fwd(x["u"], x["delta_raw"], x["A"], x["B"], x["C"], delta_bias=x["delta_bias"],
                          input_silu=True, want_out=False)
    assert normwise(to_f64(hl), ref_h) <= TOL["f32"]
    assert normwise(to_f64(H), ref_h) <= TOL["f32"]


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_generation_step(cuda_device, io):
    batch, D, N = 8, 512, 16
    x = W.small_case(batch, 1, D, N, io=io, seed=203)
    h0 = np.random.default_rng(203).standard_normal((batch, D, N)).astype(np.float32)
    t = to_torch(x, cuda_device)
    state = torch.from_numpy(h0).to(cuda_device)
    out = sb.sscan_step(t["u"][:, 0].contiguous(), t["delta_raw"][:, 0].contiguous(), t["A"],
                        t["B"][:, 0].contiguous(), t["C"][:, 0].contiguous(), state, t["delta_bias"], t["D_skip"],
                        t["z"][:, 0].contiguous(), input_silu=True)
    torch.cuda.synchronize()
    ref, ref_h = oracle.fwd(x["u"], x["delta_raw"], x["A"], x["B"], x["C"], delta_bias=x["delta_bias"],
                            D_skip=x["D_skip"], z=x["z"], h0=h0.astype(np.float64), input_silu=True)
    assert normwise(to_f64(out), ref[:, 0]) <= TOL[io]
    assert normwise(to_f64(state), ref_h) <= 1e-5


def _bwd_case(x, io, dev, general=False, h0=None):
    t = to_torch(x, dev)
    if general:
        for k in ("u", "delta_raw", "z", "dout"):
            t[k] = _offset(t[k])
    h0_t = None if h0 is None else torch.from_numpy(h0.astype(np.float32)).to(dev)
    g = sb.sscan_bwd(t["u"], t["delta_raw"], t["A"], t["B"], t["C"], t["dout"], t["delta_bias"], t["D_skip"],
                     t["z"], h0_t, input_silu=True)
    torch.cuda.synchronize()
    ref = oracle.bwd(x["u"], x["delta_raw"], x["A"], x["B"], x["C"], x["dout"], delta_bias=x["delta_bias"],
                     D_skip=x["D_skip"], z=x["z"], input_silu=True,
                     h0=None if h0 is None else h0.astype(np.float32).astype(np.float64))
    errs = {k: normwise(to_f64(g[k]), ref[k]) for k in ref}
    assert all(e <= TOL[io] for e in errs.values()), errs


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [(2, 100, 64, 16), (1, 1000, 64, 16), (2, 77, 40, 8), (1, 50, 24, 4)])
def test_backward_tiled_and_general(cuda_device, io, shape):
    """(1, 1000, 64, 16) splits the reverse sweep into sequence segments."""
    x = W.small_case(*shape, io=io, seed=sum(shape) + 210, backward=True)
    h0 = np.random.default_rng(4).standard_normal((shape[0], shape[2], shape[3])) * 0.3
    _bwd_case(x, io, cuda_device, h0=h0)
    _bwd_case(x, io, cuda_device, general=True, h0=h0)


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_complex_forward_and_backward(cuda_device, io):
    x = W.small_case(2, 90, 40, 16, io=io, seed=220, complex_a=True, backward=True)
    t = to_torch(x, cuda_device)
    A_t = torch.from_numpy(np.ascontiguousarray(x["A"].astype(np.complex64))).to(cuda_device)
    out = sb.sscan_fwd_complex(t["u"], t["delta_raw"], A_t, t["B"], t["C"], t["delta_bias"], t["D_skip"], t["z"],
                               input_silu=True)
    g = sb.sscan_bwd_complex(t["u"], t["delta_raw"], A_t, t["B"], t["C"], t["dout"], t["delta_bias"], t["D_skip"],
                             t["z"], input_silu=True)
    torch.cuda.synchronize()
    Ac = x["A"].astype(np.complex128)
    ref, _ = oracle.fwd_complex(x["u"], x["delta_raw"], Ac, x["B"], x["C"], delta_bias=x["delta_bias"],
                                D_skip=x["D_skip"], z=x["z"], input_silu=True)
    assert normwise(to_f64(out), ref) <= TOL[io]
    gref = oracle.bwd_complex(x["u"], x["delta_raw"], Ac, x["B"], x["C"], x["dout"], delta_bias=x["delta_bias"],
                              D_skip=x["D_skip"], z=x["z"], input_silu=True)
    for k in ("du", "ddelta_raw", "dB", "dC", "dz", "dD", "ddelta_bias"):
        assert normwise(to_f64(g[k]), gref[k]) <= TOL[io], k
    dA = g["dA"].detach().cpu().numpy().astype(np.complex128)
    assert np.max(np.abs(dA - gref["dA"])) / np.max(np.abs(gref["dA"])) <= TOL[io]
