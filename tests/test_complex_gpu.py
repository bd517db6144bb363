"""sscan_fwd_complex (complex diagonal A, the -1/2 + n i initialisation of the A-init
ablation table) against the fp64 oracle's complex scan, on the GPU."""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_33_b200 import binding as sb
from selective_state_space_33_b200 import workloads as W

from .helpers import TOL, normwise, to_f64, to_torch

pytestmark = pytest.mark.gpu


def _run(x, io, dev, h0=None, A=None):
    t = to_torch(x, dev)
    A_np = x["A"] if A is None else A
    A_t = torch.from_numpy(np.ascontiguousarray(A_np.astype(np.complex64))).to(dev)
    h0_t = None if h0 is None else torch.from_numpy(h0.astype(np.complex64)).to(dev)
    out, h_last = sb.sscan_fwd_complex(t["u"], t["delta_raw"], A_t, t["B"], t["C"], t["delta_bias"], t["D_skip"],
                                       t.get("z"), h0_t, return_last_state=True)
    torch.cuda.synchronize()
    ref, ref_h = oracle.fwd_complex(x["u"], x["delta_raw"], A_np.astype(np.complex64).astype(np.complex128),
                                    x["B"], x["C"], delta_bias=x["delta_bias"], D_skip=x["D_skip"], z=x.get("z"),
                                    h0=None if h0 is None else h0.astype(np.complex64).astype(np.complex128))
    e_out = normwise(to_f64(out), ref)
    hl = h_last.detach().cpu().numpy().astype(np.complex128)
    e_h = float(np.max(np.abs(hl - ref_h)) / max(np.max(np.abs(ref_h)), 1e-300))
    return e_out, e_h


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [(2, 100, 37, 16), (1, 257, 8, 4), (3, 33, 5, 1), (2, 64, 40, 7),
                                   (1, 40, 130, 16), (2, 50, 136, 2)])
def test_complex_shapes_and_tails(cuda_device, io, shape):
    x = W.small_case(*shape, io=io, seed=sum(shape) + 5, complex_a=True)
    h0 = np.random.default_rng(3).standard_normal((shape[0], shape[2], shape[3], 2)) @ np.array([1.0, 1j]) * 0.5
    e_out, e_h = _run(x, io, cuda_device, h0=h0)
    assert e_out <= TOL[io], e_out
    assert e_h <= 1e-4, e_h


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_complex_large_grid_geometry(cuda_device, io):
    """Enough (batch, channel-block) CTAs that the kernel keeps four complex states per
    lane (small grids take two): both geometries must match the oracle."""
    x = W.small_case(20, 40, 1024, 16, io=io, seed=74, complex_a=True)
    e_out, e_h = _run(x, io, cuda_device)
    assert e_out <= TOL[io], e_out
    assert e_h <= 1e-4, e_h


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_complex_general_A_values(cuda_device, io):
    """Random complex A with large angles, a zero and tiny entries: the channel block holding
    the small ones takes the series form, the others the fast form."""
    x = W.small_case(2, 80, 64, 16, io=io, seed=71, complex_a=True)
    rng = np.random.default_rng(71)
    A = (-np.exp(rng.uniform(-3, 2, size=(64, 16))) + 1j * rng.uniform(-40, 40, size=(64, 16)))
    A[0, 0] = 0.0
    A[1, 3] = 1e-5 - 2e-5j
    A[40, 2] = -3e-2 + 1e-2j  # small delta*a, but the block takes the fast form
    e_out, e_h = _run(x, io, cuda_device, A=A)
    assert e_out <= TOL[io], e_out
    assert e_h <= 1e-4, e_h


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_complex_large_angles(cuda_device, io):
    """Im(a) up to 2000, so delta Im(a) reaches ~200 rad: the angle reduction takes multiples
    of 2 pi up to ~30 turns before the MUFU sine and cosine (the turn count is rounded on the
    FMA pipe), forward and backward."""
    x = W.small_case(2, 70, 32, 16, io=io, seed=77, complex_a=True)
    rng = np.random.default_rng(77)
    A = (-np.exp(rng.uniform(-3, 1, size=(32, 16))) + 1j * rng.uniform(-2000, 2000, size=(32, 16)))
    e_out, e_h = _run(x, io, cuda_device, A=A)
    assert e_out <= TOL[io], e_out
    assert e_h <= 1e-4, e_h
    # The gradients that sum a Abar h over states (d delta, d bias, dh0, dA) are ill-conditioned
    # at such angles: a relative change of A of 2^-23 (its fp32 rounding) already moves the
    # oracle's own values by ~1e-3.  Their bound is ten times that measured spread.
    xb = W.small_case(2, 70, 32, 16, io=io, seed=77, backward=True, complex_a=True)
    A64 = A.astype(np.complex64).astype(np.complex128)

    def orc(Av):
        return oracle.bwd_complex(xb["u"], xb["delta_raw"], Av, xb["B"], xb["C"], xb["dout"],
                                  delta_bias=xb["delta_bias"], D_skip=xb["D_skip"], z=xb.get("z"))

    ref = orc(A64)
    pert = orc(A64 * (1 + 2.0 ** -23 * np.random.default_rng(78).standard_normal(A64.shape)))
    spread = {k: float(np.max(np.abs(pert[k] - ref[k])) / max(np.max(np.abs(ref[k])), 1e-300)) for k in ref}
    _check_complex_bwd(xb, io, cuda_device, A=A, tol={k: 10 * v for k, v in spread.items()})


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_complex_tma_and_plain_load_paths_agree(cuda_device, io):
    """16-byte aligned rows travel through the TMA ring; a copy starting one element
    past the boundary takes the plain-load path.  Both match the oracle and each other,
    for the forward and for the backward (whose checkpoint pass is the same kernel)."""
    x = W.small_case(2, 150, 64, 16, io=io, seed=75, complex_a=True, backward=True)
    t = to_torch(x, cuda_device)
    A_t = torch.from_numpy(np.ascontiguousarray(x["A"].astype(np.complex64))).to(cuda_device)

    def shifted(v):
        buf = torch.empty(v.numel() + 1, dtype=v.dtype, device=v.device)
        w = buf[1:].view(v.shape)
        w.copy_(v)
        return w

    m = dict(t)
    for k in ("u", "delta_raw", "z", "dout"):
        m[k] = shifted(t[k])
    outs, grads = [], []
    for tt in (t, m):
        outs.append(sb.sscan_fwd_complex(tt["u"], tt["delta_raw"], A_t, tt["B"], tt["C"], tt["delta_bias"],
                                         tt["D_skip"], tt["z"]))
        grads.append(sb.sscan_bwd_complex(tt["u"], tt["delta_raw"], A_t, tt["B"], tt["C"], tt["dout"],
                                          tt["delta_bias"], tt["D_skip"], tt["z"]))
    torch.cuda.synchronize()
    ref, _ = oracle.fwd_complex(x["u"], x["delta_raw"], x["A"].astype(np.complex128), x["B"], x["C"],
                                delta_bias=x["delta_bias"], D_skip=x["D_skip"], z=x["z"])
    for o in outs:
        assert normwise(to_f64(o), ref) <= TOL[io]
    assert normwise(to_f64(outs[0]), to_f64(outs[1])) <= (1e-6 if io == "f32" else 1e-2)
    for k in ("du", "ddelta_raw", "dB", "dC"):
        assert normwise(to_f64(grads[0][k]), to_f64(grads[1][k])) <= (1e-5 if io == "f32" else 2e-2), k
    assert sb.device_status(clear=True) == 0


def test_complex_with_zero_imaginary_part_matches_the_real_kernel(cuda_device):
    x = W.small_case(2, 300, 64, 16, io="f32", seed=72)
    t = to_torch(x, cuda_device)
    real_out = sb.sscan_fwd(t["u"], t["delta_raw"], t["A"], t["B"], t["C"], t["delta_bias"], t["D_skip"], t["z"])
    A_c = torch.complex(t["A"], torch.zeros_like(t["A"]))
    cplx_out = sb.sscan_fwd_complex(t["u"], t["delta_raw"], A_c, t["B"], t["C"], t["delta_bias"], t["D_skip"],
                                    t["z"])
    torch.cuda.synchronize()
    assert normwise(to_f64(cplx_out), to_f64(real_out)) <= 1e-5


def test_complex130m_sampled(cuda_device):
    """The benchmark's workload (batch 8, L 2048, D 1536, N 16) in one launch; the first
    batch element is checked against the oracle."""
    w = W.WORKLOADS["complex130m"]
    x = W.make_inputs(w)
    t = to_torch(x, cuda_device)
    out, h_last = sb.sscan_fwd_complex(t["u"], t["delta_raw"], t["A"], t["B"], t["C"], t["delta_bias"],
                                       t["D_skip"], t["z"], return_last_state=True)
    torch.cuda.synchronize()
    one = {k: (v[:1] if k in ("u", "delta_raw", "z", "B", "C") else v) for k, v in x.items()}
    ref, ref_h = oracle.fwd_complex(one["u"], one["delta_raw"], x["A"].astype(np.complex128), one["B"], one["C"],
                                    delta_bias=x["delta_bias"], D_skip=x["D_skip"], z=one["z"])
    assert normwise(to_f64(out[:1]), ref) <= TOL["bf16"]
    hl = h_last[:1].cpu().numpy().astype(np.complex128)
    assert np.max(np.abs(hl - ref_h)) / np.max(np.abs(ref_h)) <= 1e-4


def test_complex_empty_inputs(cuda_device):
    """No steps: the final state is h0 and every gradient but the pass-through ones is
    zero; no batch or no channels: nothing to compute, parameter gradients zero, and with
    no channels dB and dC are zero sums.  The caching allocator is first filled with NaN
    blocks so that outputs the library leaves unwritten show."""
    for shape in ((2, 0, 5, 4), (0, 10, 4, 4), (2, 10, 0, 4)):
        batch, L, D, N = shape
        x = W.small_case(*shape, io="f32", seed=6, backward=True, complex_a=True)
        t = to_torch(x, cuda_device)
        A_t = torch.from_numpy(np.ascontiguousarray(x["A"].astype(np.complex64))).to(cuda_device)
        h0 = torch.randn(batch, D, N, dtype=torch.complex64, device=cuda_device)
        out, hl = sb.sscan_fwd_complex(t["u"], t["delta_raw"], A_t, t["B"], t["C"], t["delta_bias"], t["D_skip"],
                                       t["z"], h0, return_last_state=True)
        torch.cuda.synchronize()
        assert out.numel() == batch * L * D
        if L == 0:
            assert torch.equal(hl, h0)
        filler = [torch.full((1 << 16,), float("nan"), device=cuda_device) for _ in range(8)]
        del filler
        g = sb.sscan_bwd_complex(t["u"], t["delta_raw"], A_t, t["B"], t["C"], t["dout"], t["delta_bias"],
                                 t["D_skip"], t["z"], h0)
        torch.cuda.synchronize()
        for k, v in g.items():
            assert torch.all(v == 0), (shape, k)


def test_complex_rejects_bad_A(cuda_device):
    x = W.small_case(1, 16, 8, 4, io="f32", seed=73, complex_a=True)
    t = to_torch(x, cuda_device)
    with pytest.raises((TypeError, ValueError)):
        sb.sscan_fwd_complex(t["u"], t["delta_raw"], torch.zeros(8, 4, device=cuda_device), t["B"], t["C"])
    with pytest.raises((TypeError, ValueError)):
        sb.sscan_fwd_complex(t["u"], t["delta_raw"], torch.zeros(8, 5, dtype=torch.complex64, device=cuda_device),
                             t["B"], t["C"])


# ---------------------------------------------------------------- backward
def _check_complex_bwd(x, io, dev, A=None, h0=None, tol=None):
    t = to_torch(x, dev)
    A_np = (x["A"] if A is None else A).astype(np.complex64)
    A_t = torch.from_numpy(np.ascontiguousarray(A_np)).to(dev)
    h0_t = None if h0 is None else torch.from_numpy(h0.astype(np.complex64)).to(dev)
    g = sb.sscan_bwd_complex(t["u"], t["delta_raw"], A_t, t["B"], t["C"], t["dout"], t["delta_bias"], t["D_skip"],
                             t.get("z"), h0_t)
    torch.cuda.synchronize()
    ref = oracle.bwd_complex(x["u"], x["delta_raw"], A_np.astype(np.complex128), x["B"], x["C"], x["dout"],
                             delta_bias=x["delta_bias"], D_skip=x["D_skip"], z=x.get("z"),
                             h0=None if h0 is None else h0.astype(np.complex64).astype(np.complex128))
    errs = {}
    for k, r in ref.items():
        got = g[k].detach().cpu()
        got = got.numpy().astype(np.complex128) if got.is_complex() else to_f64(g[k])
        errs[k] = float(np.max(np.abs(got - r)) / max(np.max(np.abs(r)), 1e-300))
    bad = {k: e for k, e in errs.items() if not e <= max(TOL[io], (tol or {}).get(k, 0.0))}
    assert not bad, errs
    return errs


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [(2, 100, 37, 16), (1, 70, 8, 4), (3, 33, 5, 1), (2, 64, 40, 7), (1, 45, 130, 16),
                                   (2, 50, 136, 2)])
def test_complex_backward_small(cuda_device, io, shape):
    x = W.small_case(*shape, io=io, seed=sum(shape) + 9, backward=True, complex_a=True)
    h0 = np.random.default_rng(4).standard_normal((shape[0], shape[2], shape[3], 2)) @ np.array([1.0, 1j]) * 0.5
    _check_complex_bwd(x, io, cuda_device, h0=h0)


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_complex_backward_general_A_values(cuda_device, io):
    x = W.small_case(2, 60, 32, 16, io=io, seed=75, backward=True, complex_a=True)
    rng = np.random.default_rng(75)
    A = (-np.exp(rng.uniform(-3, 2, size=(32, 16))) + 1j * rng.uniform(-40, 40, size=(32, 16)))
    A[0, 0] = 0.0
    A[1, 3] = 1e-5 - 2e-5j
    A[5, 2] = -3e-2 + 1e-2j
    _check_complex_bwd(x, io, cuda_device, A=A)


def test_complex_backward_long_sequence(cuda_device):
    """L 2048 at the layer's state size (batch 1, D 256, N 16, bf16): 256 checkpoint tiles."""
    x = W.small_case(1, 2048, 256, 16, io="bf16", seed=76, backward=True, complex_a=True)
    _check_complex_bwd(x, "bf16", cuda_device)
