"""Thin Python binding of libsscan (include/sscan.h): argument marshalling only.

Each function takes CUDA ``torch.Tensor``s, checks their dtypes, shapes and
contiguity, allocates any output or workspace the caller did not pass (PyTorch
is the allocator), and calls the C function of the same name on the current
CUDA stream.  All arithmetic runs in the library's kernels; there is no CPU or
PyTorch fallback, and a missing library is an error.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsscan.so")

SSCAN_F32, SSCAN_BF16 = 0, 1
SSCAN_DELTA_SOFTPLUS = 1
SSCAN_INPUT_SILU = 2
SSCAN_OP_FWD, SSCAN_OP_LAST_STATE, SSCAN_OP_BWD, SSCAN_OP_SUMMARY, SSCAN_OP_BWD_COMPLEX = 0, 1, 2, 3, 4
SSCAN_ERR_TIMEOUT = 5

_IO_CODES = {torch.float32: SSCAN_F32, torch.bfloat16: SSCAN_BF16}
_lib = None


class SscanError(RuntimeError):
    """A libsscan call returned a non-zero sscan_status."""

    def __init__(self, status: int, name: str, detail: str):
        super().__init__(f"{name}: {detail}" if detail else name)
        self.status = status
        self.name = name


class Problem(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64), ("dim", ctypes.c_int64),
                ("dstate", ctypes.c_int64), ("io_dtype", ctypes.c_int32), ("flags", ctypes.c_uint32)]


def load_library(path: str | None = None) -> ctypes.CDLL:
    """Load libsscan.so (built in-tree by ``selective_state_space_33_b200/build.py``)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise SscanError(-1, "SSCAN_LIBRARY_MISSING",
                         f"{p} not found; build it with python selective_state_space_33_b200/build.py")
    lib = ctypes.CDLL(p)
    vp, sz, pp = ctypes.c_void_p, ctypes.c_size_t, ctypes.POINTER(Problem)
    lib.sscan_workspace_size.argtypes = [pp, ctypes.c_int]
    lib.sscan_workspace_size.restype = sz
    lib.sscan_fwd.argtypes = [pp] + [vp] * 12 + [sz, vp]
    lib.sscan_fwd_complex.argtypes = [pp] + [vp] * 12
    lib.sscan_fwd_complex.restype = ctypes.c_int
    lib.sscan_bwd_complex.argtypes = [pp] + [vp] * 20 + [sz, vp]
    lib.sscan_bwd_complex.restype = ctypes.c_int
    lib.sscan_fwd.restype = ctypes.c_int
    lib.sscan_last_state.argtypes = [pp] + [vp] * 8 + [sz, vp]
    lib.sscan_last_state.restype = ctypes.c_int
    lib.sscan_bwd.argtypes = [pp] + [vp] * 20 + [sz, vp]
    lib.sscan_bwd.restype = ctypes.c_int
    lib.sscan_chunk_summary.argtypes = [pp] + [vp] * 8 + [sz, vp]
    lib.sscan_chunk_summary.restype = ctypes.c_int
    lib.sscan_carry.argtypes = [pp, ctypes.c_int64] + [vp] * 5 + [vp]
    lib.sscan_carry.restype = ctypes.c_int
    lib.sscan_step.argtypes = [pp] + [vp] * 10 + [vp]
    lib.sscan_step.restype = ctypes.c_int
    lib.sscan_status_string.argtypes = [ctypes.c_int]
    lib.sscan_status_string.restype = ctypes.c_char_p
    lib.sscan_last_error.argtypes = []
    lib.sscan_last_error.restype = ctypes.c_char_p
    lib.sscan_version.argtypes = []
    lib.sscan_version.restype = ctypes.c_int
    lib.sscan_device_status.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_uint)]
    lib.sscan_device_status.restype = ctypes.c_int
    lib.sscan_probe_wait_timeout.argtypes = [ctypes.c_uint, vp]
    lib.sscan_probe_wait_timeout.restype = ctypes.c_int
    if path is None:
        _lib = lib
    return lib


def _check(status: int):
    if status != 0:
        lib = load_library()
        raise SscanError(status, lib.sscan_status_string(status).decode(), lib.sscan_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def make_problem(batch, seqlen, dim, dstate, io_dtype, delta_softplus=True, input_silu=False) -> Problem:
    """input_silu: the scan's input is SiLU(u) (the block's input-branch activation)."""
    return Problem(int(batch), int(seqlen), int(dim), int(dstate), int(io_dtype),
                   (SSCAN_DELTA_SOFTPLUS if delta_softplus else 0) | (SSCAN_INPUT_SILU if input_silu else 0))


def _io_problem(u, B, delta_softplus, input_silu=False):
    if u.dim() != 3 or B.dim() != 3:
        raise ValueError("u must be (batch, L, D) and B (batch, L, N)")
    if u.dtype not in _IO_CODES:
        raise TypeError(f"I/O tensors must be float32 or bfloat16, got {u.dtype}")
    batch, L, D = u.shape
    if B.shape[0] != batch or B.shape[1] != L:
        raise ValueError(f"B has shape {tuple(B.shape)}, expected ({batch}, {L}, N)")
    return make_problem(batch, L, D, B.shape[2], _IO_CODES[u.dtype], delta_softplus, input_silu)


def _expect(t, name, shape, dtype, device):
    if t is None:
        return
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


def sscan_workspace_size(problem: Problem, op: int) -> int:
    return int(load_library().sscan_workspace_size(ctypes.byref(problem), int(op)))


def _workspace(problem, op, workspace, device):
    need = sscan_workspace_size(problem, op)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=device)
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    return workspace, nbytes


def _check_inputs(prob, u, delta_raw, A, B, C, delta_bias, D_skip, z, h0):
    dev, io = u.device, u.dtype
    if dev.type != "cuda":
        raise ValueError("libsscan works on CUDA tensors only")
    bld, bln = (prob.batch, prob.seqlen, prob.dim), (prob.batch, prob.seqlen, prob.dstate)
    _expect(u, "u", bld, io, dev)
    _expect(delta_raw, "delta_raw", bld, io, dev)
    _expect(B, "B", bln, io, dev)
    _expect(C, "C", bln, io, dev)
    _expect(z, "z", bld, io, dev)
    _expect(A, "A", (prob.dim, prob.dstate), torch.float32, dev)
    _expect(delta_bias, "delta_bias", (prob.dim,), torch.float32, dev)
    _expect(D_skip, "D_skip", (prob.dim,), torch.float32, dev)
    _expect(h0, "h0", (prob.batch, prob.dim, prob.dstate), torch.float32, dev)


def sscan_fwd(u, delta_raw, A, B, C, delta_bias=None, D_skip=None, z=None, h0=None, *,
              delta_softplus=True, input_silu=False, out=None, h_last=None, return_last_state=False,
              workspace=None, stream=None):
    """Forward selective scan.  Returns ``out`` or ``(out, h_last)``."""
    prob = _io_problem(u, B, delta_softplus, input_silu)
    _check_inputs(prob, u, delta_raw, A, B, C, delta_bias, D_skip, z, h0)
    if out is None:
        out = torch.empty_like(u)
    _expect(out, "out", u.shape, u.dtype, u.device)
    if return_last_state and h_last is None:
        h_last = torch.empty((prob.batch, prob.dim, prob.dstate), dtype=torch.float32, device=u.device)
    _expect(h_last, "h_last", (prob.batch, prob.dim, prob.dstate), torch.float32, u.device)
    ws, nbytes = _workspace(prob, SSCAN_OP_FWD, workspace, u.device)
    _check(load_library().sscan_fwd(ctypes.byref(prob), _ptr(u), _ptr(delta_raw), _ptr(delta_bias),
                                    _ptr(A), _ptr(B), _ptr(C), _ptr(D_skip), _ptr(z), _ptr(h0),
                                    _ptr(out), _ptr(h_last), _ptr(ws), nbytes, _stream(stream)))
    return (out, h_last) if (return_last_state or h_last is not None) else out


def _as_pairs(t, name, shape, dev):
    """complex64 (...) -> float32 (..., 2) view of (re, im) pairs; float32 (..., 2) as is."""
    if t is None:
        return None
    if t.is_complex():
        if t.dtype != torch.complex64:
            raise ValueError(f"{name}: complex64 expected, got {t.dtype}")
        t = torch.view_as_real(t)
    _expect(t, name, tuple(shape) + (2,), torch.float32, dev)
    return t


def sscan_fwd_complex(u, delta_raw, A, B, C, delta_bias=None, D_skip=None, z=None, h0=None, *,
                      delta_softplus=True, input_silu=False, out=None, return_last_state=False, stream=None):
    """Forward scan with a complex diagonal A: (D, N) complex64 or (D, N, 2) float32
    (re, im) pairs; h0 likewise (batch, D, N).  B, C real.  Returns ``out`` or
    ``(out, h_last)`` with h_last (batch, D, N) complex64."""
    prob = _io_problem(u, B, delta_softplus, input_silu)
    dev = u.device
    _check_inputs(prob, u, delta_raw, None, B, C, delta_bias, D_skip, z, None)
    A2 = _as_pairs(A, "A", (prob.dim, prob.dstate), dev)
    h02 = _as_pairs(h0, "h0", (prob.batch, prob.dim, prob.dstate), dev)
    if out is None:
        out = torch.empty_like(u)
    _expect(out, "out", u.shape, u.dtype, dev)
    h_last = (torch.empty((prob.batch, prob.dim, prob.dstate, 2), dtype=torch.float32, device=dev)
              if return_last_state else None)
    _check(load_library().sscan_fwd_complex(ctypes.byref(prob), _ptr(u), _ptr(delta_raw), _ptr(delta_bias),
                                            _ptr(A2), _ptr(B), _ptr(C), _ptr(D_skip), _ptr(z), _ptr(h02),
                                            _ptr(out), _ptr(h_last), _stream(stream)))
    return (out, torch.view_as_complex(h_last)) if return_last_state else out


def sscan_bwd_complex(u, delta_raw, A, B, C, dout, delta_bias=None, D_skip=None, z=None, h0=None, *,
                      delta_softplus=True, input_silu=False, want_dh0=True, workspace=None, stream=None):
    """Gradients of sum(out * dout) for the complex-A scan.  Returns a dict keyed du,
    ddelta_raw, dA (D, N) complex64, dB, dC and, when the matching input is given,
    ddelta_bias, dD, dz; dh0 (batch, D, N) complex64 when ``want_dh0``."""
    prob = _io_problem(u, B, delta_softplus, input_silu)
    dev = u.device
    _check_inputs(prob, u, delta_raw, None, B, C, delta_bias, D_skip, z, None)
    _expect(dout, "dout", u.shape, u.dtype, dev)
    A2 = _as_pairs(A, "A", (prob.dim, prob.dstate), dev)
    h02 = _as_pairs(h0, "h0", (prob.batch, prob.dim, prob.dstate), dev)
    f32 = dict(dtype=torch.float32, device=dev)
    g = {"du": torch.empty_like(u), "ddelta_raw": torch.empty_like(u),
         "dA": torch.empty((prob.dim, prob.dstate, 2), **f32), "dB": torch.empty_like(B), "dC": torch.empty_like(C)}
    if delta_bias is not None:
        g["ddelta_bias"] = torch.empty((prob.dim,), **f32)
    if D_skip is not None:
        g["dD"] = torch.empty((prob.dim,), **f32)
    if z is not None:
        g["dz"] = torch.empty_like(z)
    if want_dh0:
        g["dh0"] = torch.empty((prob.batch, prob.dim, prob.dstate, 2), **f32)
    ws, nbytes = _workspace(prob, SSCAN_OP_BWD_COMPLEX, workspace, dev)
    _check(load_library().sscan_bwd_complex(
        ctypes.byref(prob), _ptr(u), _ptr(delta_raw), _ptr(delta_bias), _ptr(A2), _ptr(B), _ptr(C), _ptr(D_skip),
        _ptr(z), _ptr(h02), _ptr(dout), _ptr(g["du"]), _ptr(g["ddelta_raw"]), _ptr(g.get("ddelta_bias")),
        _ptr(g["dA"]), _ptr(g["dB"]), _ptr(g["dC"]), _ptr(g.get("dD")), _ptr(g.get("dz")), _ptr(g.get("dh0")),
        _ptr(ws), nbytes, _stream(stream)))
    g["dA"] = torch.view_as_complex(g["dA"])
    if want_dh0:
        g["dh0"] = torch.view_as_complex(g["dh0"])
    return g


def sscan_last_state(u, delta_raw, A, B, delta_bias=None, h0=None, *, delta_softplus=True, input_silu=False,
                     h_last=None, workspace=None, stream=None):
    """Final state h_{L-1} (batch, D, N) only."""
    prob = _io_problem(u, B, delta_softplus, input_silu)
    _check_inputs(prob, u, delta_raw, A, B, None, delta_bias, None, None, h0)
    if h_last is None:
        h_last = torch.empty((prob.batch, prob.dim, prob.dstate), dtype=torch.float32, device=u.device)
    _expect(h_last, "h_last", (prob.batch, prob.dim, prob.dstate), torch.float32, u.device)
    ws, nbytes = _workspace(prob, SSCAN_OP_LAST_STATE, workspace, u.device)
    _check(load_library().sscan_last_state(ctypes.byref(prob), _ptr(u), _ptr(delta_raw), _ptr(delta_bias),
                                           _ptr(A), _ptr(B), _ptr(h0), _ptr(h_last), _ptr(ws), nbytes,
                                           _stream(stream)))
    return h_last


def sscan_bwd(u, delta_raw, A, B, C, dout, delta_bias=None, D_skip=None, z=None, h0=None, *,
              delta_softplus=True, input_silu=False, want_dh0=True, grads=None, workspace=None, stream=None):
    """Gradients of sum(out * dout).  Returns a dict keyed du, ddelta_raw, dA, dB, dC and,
    when the matching input is given, ddelta_bias, dD, dz; dh0 when ``want_dh0``.
    ``grads`` may supply preallocated outputs under the same keys."""
    prob = _io_problem(u, B, delta_softplus, input_silu)
    _check_inputs(prob, u, delta_raw, A, B, C, delta_bias, D_skip, z, h0)
    _expect(dout, "dout", u.shape, u.dtype, u.device)
    f32 = dict(dtype=torch.float32, device=u.device)
    pre = grads or {}
    g = {"du": pre.get("du", None), "ddelta_raw": pre.get("ddelta_raw", None), "dA": pre.get("dA", None),
         "dB": pre.get("dB", None), "dC": pre.get("dC", None)}
    g["du"] = g["du"] if g["du"] is not None else torch.empty_like(u)
    g["ddelta_raw"] = g["ddelta_raw"] if g["ddelta_raw"] is not None else torch.empty_like(u)
    g["dA"] = g["dA"] if g["dA"] is not None else torch.empty((prob.dim, prob.dstate), **f32)
    g["dB"] = g["dB"] if g["dB"] is not None else torch.empty_like(B)
    g["dC"] = g["dC"] if g["dC"] is not None else torch.empty_like(C)
    g["ddelta_bias"] = (pre.get("ddelta_bias") if pre.get("ddelta_bias") is not None
                        else torch.empty(prob.dim, **f32)) if delta_bias is not None else None
    g["dD"] = (pre.get("dD") if pre.get("dD") is not None else torch.empty(prob.dim, **f32)) \
        if D_skip is not None else None
    g["dz"] = (pre.get("dz") if pre.get("dz") is not None else torch.empty_like(u)) if z is not None else None
    g["dh0"] = (pre.get("dh0") if pre.get("dh0") is not None
                else torch.empty((prob.batch, prob.dim, prob.dstate), **f32)) if want_dh0 else None
    for k, ref in (("du", u), ("ddelta_raw", u), ("dB", B), ("dC", C), ("dz", u)):
        if g[k] is not None:
            _expect(g[k], k, ref.shape, ref.dtype, u.device)
    _expect(g["dA"], "dA", (prob.dim, prob.dstate), torch.float32, u.device)
    _expect(g["ddelta_bias"], "ddelta_bias", (prob.dim,), torch.float32, u.device)
    _expect(g["dD"], "dD", (prob.dim,), torch.float32, u.device)
    _expect(g["dh0"], "dh0", (prob.batch, prob.dim, prob.dstate), torch.float32, u.device)
    ws, nbytes = _workspace(prob, SSCAN_OP_BWD, workspace, u.device)
    _check(load_library().sscan_bwd(ctypes.byref(prob), _ptr(u), _ptr(delta_raw), _ptr(delta_bias), _ptr(A),
                                    _ptr(B), _ptr(C), _ptr(D_skip), _ptr(z), _ptr(h0), _ptr(dout),
                                    _ptr(g["du"]), _ptr(g["ddelta_raw"]), _ptr(g["ddelta_bias"]),
                                    _ptr(g["dA"]), _ptr(g["dB"]), _ptr(g["dC"]), _ptr(g["dD"]),
                                    _ptr(g["dz"]), _ptr(g["dh0"]), _ptr(ws), nbytes, _stream(stream)))
    return {k: v for k, v in g.items() if v is not None}


def sscan_step(u, delta_raw, A, B, C, state, delta_bias=None, D_skip=None, z=None, *, delta_softplus=True, input_silu=False,
               out=None, stream=None):
    """One generation step: u, delta_raw, z (batch, D); B, C (batch, N); state (batch, D, N)
    fp32 updated in place.  Returns out (batch, D)."""
    if u.dim() != 2 or B.dim() != 2:
        raise ValueError("u must be (batch, D) and B (batch, N)")
    if u.dtype not in _IO_CODES:
        raise TypeError(f"I/O tensors must be float32 or bfloat16, got {u.dtype}")
    batch, D = u.shape
    N = B.shape[1]
    prob = make_problem(batch, 1, D, N, _IO_CODES[u.dtype], delta_softplus, input_silu)
    dev, io = u.device, u.dtype
    if dev.type != "cuda":
        raise ValueError("libsscan works on CUDA tensors only")
    for t, name, shape in ((delta_raw, "delta_raw", (batch, D)), (z, "z", (batch, D)), (B, "B", (batch, N)),
                           (C, "C", (batch, N))):
        _expect(t, name, shape, io, dev)
    _expect(A, "A", (D, N), torch.float32, dev)
    _expect(delta_bias, "delta_bias", (D,), torch.float32, dev)
    _expect(D_skip, "D_skip", (D,), torch.float32, dev)
    _expect(state, "state", (batch, D, N), torch.float32, dev)
    if out is None:
        out = torch.empty_like(u)
    _expect(out, "out", (batch, D), io, dev)
    _check(load_library().sscan_step(ctypes.byref(prob), _ptr(u), _ptr(delta_raw), _ptr(delta_bias), _ptr(A),
                                     _ptr(B), _ptr(C), _ptr(D_skip), _ptr(z), _ptr(state), _ptr(out),
                                     _stream(stream)))
    return out


def sscan_chunk_summary(u, delta_raw, A, B, delta_bias=None, *, delta_softplus=True, input_silu=False, workspace=None,
                        stream=None):
    """(P, H), each (batch, D, N) fp32: the stretch u[:, 0:L] acts on its initial state as
    h -> P h + H (P = exp(A * sum of delta), H = final state from zero)."""
    prob = _io_problem(u, B, delta_softplus, input_silu)
    _check_inputs(prob, u, delta_raw, A, B, None, delta_bias, None, None, None)
    f32 = dict(dtype=torch.float32, device=u.device)
    P = torch.empty((prob.batch, prob.dim, prob.dstate), **f32)
    H = torch.empty((prob.batch, prob.dim, prob.dstate), **f32)
    ws, nbytes = _workspace(prob, SSCAN_OP_SUMMARY, workspace, u.device)
    _check(load_library().sscan_chunk_summary(ctypes.byref(prob), _ptr(u), _ptr(delta_raw), _ptr(delta_bias),
                                              _ptr(A), _ptr(B), _ptr(P), _ptr(H), _ptr(ws), nbytes,
                                              _stream(stream)))
    return P, H


def sscan_carry(P, H, h0=None, *, stream=None):
    """Compose K stretch summaries P, H (K, batch, D, N) in order from h0 (batch, D, N):
    returns (carry_in (K, batch, D, N), h_final (batch, D, N))."""
    if P.dim() != 4 or P.shape != H.shape:
        raise ValueError("P and H must both be (K, batch, D, N)")
    K, batch, D, N = P.shape
    dev = P.device
    _expect(P, "P", P.shape, torch.float32, dev)
    _expect(H, "H", P.shape, torch.float32, dev)
    _expect(h0, "h0", (batch, D, N), torch.float32, dev)
    prob = make_problem(batch, 0, D, N, SSCAN_F32)
    carry = torch.empty_like(P)
    h_final = torch.empty((batch, D, N), dtype=torch.float32, device=dev)
    _check(load_library().sscan_carry(ctypes.byref(prob), int(K), _ptr(P), _ptr(H), _ptr(h0), _ptr(carry),
                                      _ptr(h_final), _stream(stream)))
    return carry, h_final


def device_status(clear: bool = False) -> int:
    """Error bits the library's kernels raised on the current device since the last
    clear (0: none; bit 0 forward, bit 1 backward: a bounded wait for a tile copy gave
    up; bit 2: the wait-timeout probe).  Synchronous."""
    lib = load_library()
    flags = ctypes.c_uint(0)
    st = lib.sscan_device_status(int(clear), ctypes.byref(flags))
    if st not in (0, SSCAN_ERR_TIMEOUT):
        _check(st)
    return flags.value


def probe_wait_timeout(polls: int = 4096, *, stream=None):
    """Enqueue the bounded-wait self-test: one thread waits on a barrier nothing
    arrives on, gives up after ``polls`` polls and raises bit 2 of the device status."""
    _check(load_library().sscan_probe_wait_timeout(polls, _stream(stream)))
