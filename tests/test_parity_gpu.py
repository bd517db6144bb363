"""GPU parity: the CUDA library (through its C ABI) against the fp64 CPU oracle on
the same seeded inputs.  Tolerance (normwise, per tensor): max|gpu - ref| / max|ref|
<= 1e-4 for fp32 I/O and <= 2e-2 for bf16 I/O.  The pointwise relative error over
the elements with |ref| >= 1e-3 max|ref| is reported beside it (and bounded where
a test says so)."""
import math

import numpy as np
import pytest
import torch

import oracle
from selective_state_space_33_b200 import binding as sb
from selective_state_space_33_b200 import workloads as W

from .helpers import TOL, normwise, pointwise, to_f64, to_torch

pytestmark = pytest.mark.gpu


def _oracle_fwd(x, rows=None, **kw):
    return oracle.fwd(x["u"], x["delta_raw"], x["A"], x["B"], x["C"], delta_bias=x.get("delta_bias"),
                      D_skip=x.get("D_skip"), z=x.get("z"), rows=rows, **kw)


def _gpu_fwd(t, **kw):
    return sb.sscan_fwd(t["u"], t["delta_raw"], t["A"], t["B"], t["C"], t.get("delta_bias"),
                        t.get("D_skip"), t.get("z"), t.get("h0"), **kw)


def _check_full(x, io, dev, h0=None, **kw):
    t = to_torch(x, dev)
    if h0 is not None:
        t["h0"] = torch.from_numpy(h0.astype(np.float32)).to(dev)
    out, hl = _gpu_fwd(t, return_last_state=True, **kw)
    torch.cuda.synchronize()
    ref, ref_h = oracle.fwd(x["u"], x["delta_raw"], x["A"], x["B"], x["C"], delta_bias=x.get("delta_bias"),
                            D_skip=x.get("D_skip"), z=x.get("z"),
                            h0=None if h0 is None else h0.astype(np.float32).astype(np.float64), **kw)
    e_out, e_h = normwise(to_f64(out), ref), normwise(to_f64(hl), ref_h)
    assert e_out <= TOL[io], e_out
    assert e_h <= TOL[io], e_h
    return e_out, e_h


# ---------------------------------------------------------------- configs at full size
def test_tiny_fp32(cuda_device):
    x = W.make_inputs(W.WORKLOADS["tiny"])
    _check_full(x, "f32", cuda_device)


def test_mamba130m_bf16_full(cuda_device):
    x = W.make_inputs(W.WORKLOADS["mamba130m"])
    _check_full(x, "bf16", cuda_device)


def _block_rows(w, per_block, seed, dc=32):
    """(batch, channel) rows covering every block of ``dc`` consecutive channels (the
    tiled kernel's CTA width at N = 16): ``per_block`` random channels of each block,
    each in a random batch, plus the first and last channel of the first and last
    batch."""
    rng = np.random.default_rng(seed)
    rows = []
    for c0 in range(0, w.dim, dc):
        width = min(dc, w.dim - c0)
        ch = c0 + rng.choice(width, size=min(per_block, width), replace=False)
        rows.extend(rng.integers(0, w.batch, size=ch.size) * w.dim + ch)
    rows.extend([0, w.dim - 1, (w.batch - 1) * w.dim, w.batch * w.dim - 1])
    return np.unique(np.asarray(rows, np.int64))


def _report(name, **errs):
    print(f"[parity] {name}: " + ", ".join(f"{k}={v:.3e}" for k, v in errs.items()))


# Pointwise bounds (|ref| >= 1e-3 max|ref|).  fp32 arithmetic leaves a normwise error
# near 1e-6, which an element at 1e-3 of the maximum sees as up to ~1e-3 relative;
# bf16 I/O adds the output's own rounding (2^-9 relative).  Measured on B200: fp32
# out 2.3e-4, bf16 out 4.0e-3, final states up to 3.2e-3.
POINTWISE = {"f32": 1e-3, "bf16": 2e-2, "state": 1e-2}


def _check_whole(w, dev):
    """Every output element and every final state of a full-size workload against the
    oracle (about a second of oracle time per pass on a 16-core host)."""
    x = W.make_inputs(w)
    t = to_torch(x, dev)
    out, hl = _gpu_fwd(t, return_last_state=True)
    torch.cuda.synchronize()
    del t
    got, got_h = to_f64(out), to_f64(hl)
    del out, hl
    ref, ref_h = _oracle_fwd(x)
    e_out, e_h = normwise(got, ref), normwise(got_h, ref_h)
    p_out, p_h = pointwise(got, ref), pointwise(got_h, ref_h)
    _report(w.name, out_normwise=e_out, out_pointwise=p_out, h_normwise=e_h, h_pointwise=p_h)
    assert np.isfinite(got).all()
    assert e_out <= TOL[w.io], e_out
    assert e_h <= TOL[w.io], e_h
    assert p_out <= POINTWISE[w.io], p_out
    assert p_h <= POINTWISE["state"], p_h
    return p_out, p_h


def test_mamba2p8b_bf16_whole(cuda_device):
    _check_whole(W.WORKLOADS["mamba2.8b"], cuda_device)


def test_mamba2p8b_fp32_whole(cuda_device):
    _check_whole(W.WORKLOADS["mamba2.8b-f32"], cuda_device)


def test_million_length_sampled(cuda_device):
    """L = 2^20 over 1536 channels: the sequence is split into chunks joined by the
    cross-chunk carry.  Three rows of every 32-channel block (144 rows, about 150 M
    elements of oracle work) and their final states."""
    w = W.WORKLOADS["million"]
    x = W.make_inputs(w)
    t = to_torch(x, cuda_device)
    out, hl = _gpu_fwd(t, return_last_state=True)
    torch.cuda.synchronize()
    rows = _block_rows(w, 3, w.seed)
    assert rows.size >= 144
    b, d = rows // w.dim, rows % w.dim
    got = to_f64(out[b, :, d])                     # (rows, L)
    got_h = to_f64(hl.reshape(-1, w.dstate)[rows])
    del out, t
    ref, ref_h = _oracle_fwd(x, rows=rows)
    e_out, e_h = normwise(got, ref), normwise(got_h, ref_h)
    p_out, p_h = pointwise(got, ref), pointwise(got_h, ref_h)
    _report(w.name, rows=rows.size, out_normwise=e_out, out_pointwise=p_out, h_normwise=e_h, h_pointwise=p_h)
    assert e_out <= TOL[w.io], e_out
    assert e_h <= TOL[w.io], e_h
    assert p_out <= POINTWISE[w.io], p_out
    assert p_h <= POINTWISE["state"], p_h
    assert np.isfinite(got).all()


@pytest.mark.parametrize("variant", ["skip_gate", "bare"])
@pytest.mark.parametrize("shape", [(1, 65536, 64, 16), (4, 2047, 96, 16)])
def test_fp32_small_delta_long_sequence(cuda_device, variant, shape):
    """fp32 I/O with delta log-uniform in [1e-4, 1e-2] and A = -(n+1), the million-step
    workload's regime, where |delta A| reaches 1e-4 and a step's increment
    (Abar - 1)(h - v) is a small difference: held to the fp32 tolerance.  The long
    case (2^16 steps, 64 channels) runs through the sequence split and carry, the
    other through one pass per row.  'bare' drops the skip term and the gate, so the
    output is the readout C.h alone and no larger term hides an error in the state."""
    batch, L, D, N = shape
    x = W.small_case(batch, L, D, N, io="f32", seed=L + D, dt_min=1e-4, dt_max=1e-2, dskip="ones")
    if variant == "bare":
        del x["z"], x["D_skip"]
    t = to_torch(x, cuda_device)
    out, hl = _gpu_fwd(t, return_last_state=True)
    torch.cuda.synchronize()
    ref, ref_h = _oracle_fwd(x)
    got, got_h = to_f64(out), to_f64(hl)
    e_out, e_h = normwise(got, ref), normwise(got_h, ref_h)
    p_out, p_h = pointwise(got, ref), pointwise(got_h, ref_h)
    _report(f"small-delta {shape} {variant}", out_normwise=e_out, out_pointwise=p_out, h_normwise=e_h,
            h_pointwise=p_h)
    assert e_out <= TOL["f32"], e_out
    assert e_h <= TOL["f32"], e_h
    assert p_h <= POINTWISE["state"], p_h
    if variant == "skip_gate":
        assert p_out <= POINTWISE["f32"], p_out


# ---------------------------------------------------------------- tails, options, N
@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [(2, 100, 37, 16), (1, 257, 8, 4), (3, 33, 5, 1), (2, 64, 40, 7),
                                   (1, 1, 3, 16), (2, 1030, 24, 8)])
def test_shapes_and_tails(cuda_device, io, shape):
    batch, L, D, N = shape
    x = W.small_case(batch, L, D, N, io=io, seed=sum(shape))
    _check_full(x, io, cuda_device)


@pytest.mark.parametrize("variant", ["no_gate", "no_skip", "no_bias", "no_softplus", "h0", "bare"])
def test_optional_inputs(cuda_device, variant):
    x = W.small_case(2, 96, 19, 16, io="f32", seed=31)
    kw, h0 = {}, None
    if variant in ("no_gate", "bare"):
        del x["z"]
    if variant in ("no_skip", "bare"):
        del x["D_skip"]
    if variant in ("no_bias", "bare"):
        del x["delta_bias"]
    if variant == "no_softplus":
        # delta = delta_raw directly, so keep it positive and drop the (negative) bias
        x["delta_raw"] = np.abs(x["delta_raw"]) * 0.05
        del x["delta_bias"]
        kw["delta_softplus"] = False
    if variant == "h0":
        h0 = np.random.default_rng(3).standard_normal((2, 19, 16))
    _check_full(x, "f32", cuda_device, h0=h0, **kw)


def test_general_A_values(cuda_device):
    """A with zeros (the delta B limit), tiny and large magnitudes, and positive entries."""
    x = W.small_case(2, 80, 12, 16, io="f32", seed=41)
    rng = np.random.default_rng(41)
    A = -np.exp(rng.uniform(-6, 3, size=(12, 16))).astype(np.float32)
    A[0, :4] = 0.0
    A[1, 5] = 0.25
    A[2, 7] = -1e-7
    x["A"] = A
    _check_full(x, "f32", cuda_device)


# ---------------------------------------------------------------- pins through the ABI
def test_hand_case_through_abi(cuda_device):
    ln2 = math.log(2.0)
    t = {"u": torch.tensor([1.0, 2, 3, 4]).reshape(1, 4, 1), "delta_raw": torch.tensor([1.0, 2, 1, 0]).reshape(1, 4, 1),
         "A": torch.tensor([[-ln2]]), "B": torch.full((1, 4, 1), ln2), "C": torch.tensor([1.0, 1, 2, 1]).reshape(1, 4, 1)}
    t = {k: v.float().to(cuda_device) for k, v in t.items()}
    out, hl = _gpu_fwd(t, delta_softplus=False, return_last_state=True)
    np.testing.assert_allclose(to_f64(out).ravel(), [0.5, 1.625, 4.625, 2.3125], rtol=1e-5)
    np.testing.assert_allclose(to_f64(hl).ravel(), [2.3125], rtol=1e-5)


@pytest.mark.parametrize("k", [1, 255, 256, 257, 700])
def test_split_with_carry_on_gpu(cuda_device, k):
    x = W.small_case(2, 1024, 24, 16, io="f32", seed=51)
    t = to_torch(x, cuda_device)
    full, hl = _gpu_fwd(t, return_last_state=True)
    cut = lambda v, s: v[:, s].contiguous()
    s1, s2 = slice(0, k), slice(k, None)
    a = {n: (cut(v, s1) if n in ("u", "delta_raw", "z", "B", "C") else v) for n, v in t.items()}
    o1, h1 = _gpu_fwd(a, return_last_state=True)
    b = {n: (cut(v, s2) if n in ("u", "delta_raw", "z", "B", "C") else v) for n, v in t.items()}
    b["h0"] = h1
    o2, h2 = _gpu_fwd(b, return_last_state=True)
    assert normwise(to_f64(torch.cat([o1, o2], 1)), to_f64(full)) <= 1e-5
    assert normwise(to_f64(h2), to_f64(hl)) <= 1e-5


def test_last_state_matches_oracle(cuda_device):
    for w in (W.small_case(2, 3000, 16, 16, io="bf16", seed=61),
              W.small_case(1, 5000, 4, 8, io="f32", seed=62)):
        t = to_torch(w, cuda_device)
        hl = sb.sscan_last_state(t["u"], t["delta_raw"], t["A"], t["B"], t["delta_bias"])
        torch.cuda.synchronize()
        _, ref_h = oracle.fwd(w["u"], w["delta_raw"], w["A"], w["B"], w["C"], delta_bias=w["delta_bias"],
                              want_out=False)
        io = "bf16" if w["u"].dtype == np.uint16 else "f32"
        assert normwise(to_f64(hl), ref_h) <= TOL[io]


def test_delta_to_zero_on_gpu(cuda_device):
    x = W.small_case(2, 50, 9, 16, io="f32", seed=71)
    x["delta_raw"] = np.full_like(x["delta_raw"], -40.0)
    h0 = np.random.default_rng(71).standard_normal((2, 9, 16))
    _check_full(x, "f32", cuda_device, h0=h0)


# ---------------------------------------------------------------- edge cases
def test_empty_sequence_returns_h0(cuda_device):
    t = to_torch(W.small_case(2, 0, 5, 4, io="f32", seed=1), cuda_device)
    h0 = torch.randn(2, 5, 4, device=cuda_device)
    out, hl = sb.sscan_fwd(t["u"], t["delta_raw"], t["A"], t["B"], t["C"], h0=h0, return_last_state=True)
    torch.cuda.synchronize()
    assert out.numel() == 0 and torch.equal(hl, h0)
    hl = sb.sscan_last_state(t["u"], t["delta_raw"], t["A"], t["B"])
    torch.cuda.synchronize()
    assert torch.count_nonzero(hl) == 0


def test_empty_batch_and_channels(cuda_device):
    for shape in ((0, 10, 4, 4), (2, 10, 0, 4)):
        t = to_torch(W.small_case(*shape, io="f32", seed=2), cuda_device)
        out = sb.sscan_fwd(t["u"], t["delta_raw"], t["A"], t["B"], t["C"])
        torch.cuda.synchronize()
        assert out.numel() == 0


def test_backward_empty_inputs(cuda_device):
    """No steps, no batch or no channels: every gradient is a sum over nothing, so the
    library writes zeros (the outputs start as NaN to show anything left unwritten)."""
    for shape in ((2, 0, 5, 4), (0, 10, 4, 4), (2, 10, 0, 4)):
        batch, L, D, N = shape
        t = to_torch(W.small_case(*shape, io="f32", seed=5, backward=True), cuda_device)
        h0 = torch.randn(batch, D, N, device=cuda_device)
        nan = lambda *size: torch.full(size, float("nan"), device=cuda_device)
        grads = {"du": nan(*t["u"].shape), "ddelta_raw": nan(*t["u"].shape), "dz": nan(*t["u"].shape),
                 "dA": nan(D, N), "dB": nan(*t["B"].shape), "dC": nan(*t["C"].shape), "ddelta_bias": nan(D),
                 "dD": nan(D), "dh0": nan(batch, D, N)}
        g = sb.sscan_bwd(t["u"], t["delta_raw"], t["A"], t["B"], t["C"], t["dout"], t["delta_bias"], t["D_skip"],
                         t["z"], h0, grads=grads)
        torch.cuda.synchronize()
        for k, v in g.items():
            assert torch.all(v == 0), (shape, k)


def test_errors_through_binding(cuda_device):
    t = to_torch(W.small_case(1, 16, 4, 4, io="f32", seed=3), cuda_device)
    with pytest.raises(sb.SscanError) as e:
        sb.sscan_fwd(t["u"], t["delta_raw"], torch.zeros(4, 17, device=cuda_device),
                     torch.zeros(1, 16, 17, device=cuda_device), torch.zeros(1, 16, 17, device=cuda_device))
    assert e.value.name == "SSCAN_ERR_UNSUPPORTED"
    big = to_torch(W.small_case(1, 4096, 8, 4, io="f32", seed=4), cuda_device)
    prob = sb.make_problem(1, 4096, 8, 4, sb.SSCAN_F32)
    need = sb.sscan_workspace_size(prob, sb.SSCAN_OP_FWD)
    assert need > 0
    with pytest.raises(sb.SscanError) as e:
        sb.sscan_fwd(big["u"], big["delta_raw"], big["A"], big["B"], big["C"],
                     workspace=torch.empty(need // 2, dtype=torch.uint8, device=cuda_device))
    assert e.value.name == "SSCAN_ERR_WORKSPACE"


# ---------------------------------------------------------------- backward
def _check_bwd(x, io, dev, h0=None):
    t = to_torch(x, dev)
    if h0 is not None:
        t["h0"] = torch.from_numpy(h0.astype(np.float32)).to(dev)
    g = sb.sscan_bwd(t["u"], t["delta_raw"], t["A"], t["B"], t["C"], t["dout"], t.get("delta_bias"),
                     t.get("D_skip"), t.get("z"), t.get("h0"))
    torch.cuda.synchronize()
    ref = oracle.bwd(x["u"], x["delta_raw"], x["A"], x["B"], x["C"], x["dout"], delta_bias=x.get("delta_bias"),
                     D_skip=x.get("D_skip"), z=x.get("z"),
                     h0=None if h0 is None else h0.astype(np.float32).astype(np.float64))
    errs = {k: normwise(to_f64(g[k]), ref[k]) for k in ref}
    bad = {k: e for k, e in errs.items() if not e <= TOL[io]}
    assert not bad, errs
    return errs


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [(1, 64, 4, 4), (2, 100, 37, 16), (1, 33, 5, 1), (2, 70, 9, 7),
                                   (2, 100, 64, 16), (1, 37, 32, 8), (3, 50, 24, 4), (1, 300, 96, 16),
                                   (1, 1000, 64, 16), (2, 777, 40, 8), (1, 1100, 8, 4)])
def test_backward_small(cuda_device, io, shape):
    """Includes shapes whose reverse sweep the library splits into sequence segments
    (L >= 256 with few channel blocks), with a ragged last segment."""
    x = W.small_case(*shape, io=io, seed=sum(shape) + 1, backward=True)
    h0 = np.random.default_rng(5).standard_normal((shape[0], shape[2], shape[3])) * 0.3
    _check_bwd(x, io, cuda_device, h0=h0)


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_backward_general_A_values(cuda_device, io):
    """A with zeros (the delta B limit), tiny and large magnitudes: the channel block
    holding them recomputes states with phi1's series, the other block with the
    forward kernel's form; both must match the oracle."""
    x = W.small_case(2, 90, 64, 16, io=io, seed=43, backward=True)
    rng = np.random.default_rng(43)
    A = -np.exp(rng.uniform(-6, 3, size=(64, 16))).astype(np.float32)
    A[0, :4] = 0.0
    A[2, 7] = -1e-7
    A[5, 3] = -3e-4
    x["A"] = A
    _check_bwd(x, io, cuda_device)


def test_backward_mamba130m_full(cuda_device):
    x = W.make_inputs(W.WORKLOADS["bwd130m"])
    _check_bwd(x, "bf16", cuda_device)


# ---------------------------------------------------------------- both kernel paths
def _misaligned_copy(t):
    """Same values, contiguous, but starting one element past a 16-byte boundary, which
    sends the call down the general row kernels instead of the TMA-tiled kernel."""
    buf = torch.empty(t.numel() + 1, dtype=t.dtype, device=t.device)
    v = buf[1:].view(t.shape)
    v.copy_(t)
    return v


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_general_path_matches_tiled_path(cuda_device, io):
    x = W.small_case(2, 300, 64, 16, io=io, seed=81)
    t = to_torch(x, cuda_device)
    fast, hf = _gpu_fwd(t, return_last_state=True)
    m = dict(t)
    for k in ("u", "delta_raw", "z"):
        m[k] = _misaligned_copy(t[k])
    slow, hs = _gpu_fwd(m, return_last_state=True)
    torch.cuda.synchronize()
    ref, ref_h = _oracle_fwd(x)
    for got, gh in ((fast, hf), (slow, hs)):
        assert normwise(to_f64(got), ref) <= TOL[io]
        assert normwise(to_f64(gh), ref_h) <= TOL[io]
    assert normwise(to_f64(fast), to_f64(slow)) <= (1e-5 if io == "f32" else 1e-2)


def test_device_status_is_clear(cuda_device):
    import ctypes
    lib = sb.load_library()
    lib.sscan_device_status.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_uint)]
    lib.sscan_device_status.restype = ctypes.c_int
    x = W.small_case(2, 100, 64, 16, io="bf16", seed=82)
    t = to_torch(x, cuda_device)
    _gpu_fwd(t)
    flags = ctypes.c_uint(123)
    assert lib.sscan_device_status(1, ctypes.byref(flags)) == 0
    assert flags.value == 0


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_backward_general_path_matches_tiled_path(cuda_device, io):
    """Misaligned copies of the inputs send the call down the general row kernel; both
    paths must agree with the oracle and with each other."""
    x = W.small_case(2, 120, 64, 16, io=io, seed=91, backward=True)
    t = to_torch(x, cuda_device)
    args = lambda tt: (tt["u"], tt["delta_raw"], tt["A"], tt["B"], tt["C"], tt["dout"], tt["delta_bias"],
                       tt["D_skip"], tt["z"])
    fast = sb.sscan_bwd(*args(t))
    m = dict(t)
    for k in ("u", "delta_raw", "z", "dout"):
        m[k] = _misaligned_copy(t[k])
    slow = sb.sscan_bwd(*args(m))
    torch.cuda.synchronize()
    ref = oracle.bwd(x["u"], x["delta_raw"], x["A"], x["B"], x["C"], x["dout"], delta_bias=x["delta_bias"],
                     D_skip=x["D_skip"], z=x["z"])
    for k in ref:
        assert normwise(to_f64(fast[k]), ref[k]) <= TOL[io], k
        assert normwise(to_f64(slow[k]), ref[k]) <= TOL[io], k
