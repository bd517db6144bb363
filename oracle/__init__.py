"""fp64 CPU oracle for the selective scan (Mamba S6) -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may
import this package.  It shares no code with the CUDA library: the arithmetic lives in
``sscan_oracle.c`` (plain C, IEEE double, one loop per (batch, channel) row), and this
module only marshals numpy arrays into it.

Arrays follow the layouts of the scan problem: u, delta_raw, z, dout are
(batch, L, D); B, C are (batch, L, N); A is (D, N); delta_bias, D_skip are (D,);
h0 is (batch, D, N).  The element type of u, delta_raw, z, B, C, dout is float64,
float32, or uint16 holding bfloat16 bit patterns; all are widened exactly.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_F32, _BF16, _F64 = 0, 1, 2
_lib = None


class _Problem(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64),
                ("dim", ctypes.c_int64), ("dstate", ctypes.c_int64),
                ("io_dtype", ctypes.c_int32), ("delta_softplus", ctypes.c_int32),
                ("input_silu", ctypes.c_int32)]


def _load():
    global _lib
    if _lib is None:
        # SSCAN_ORACLE_LIB lets the mutation test point the pins at a deliberately
        # broken build of the same source; normal use builds and loads our own.
        path = os.environ.get("SSCAN_ORACLE_LIB") or _build.build()
        lib = ctypes.CDLL(path)
        vp = ctypes.c_void_p
        lib.orc_fwd.argtypes = [ctypes.POINTER(_Problem)] + [vp] * 10 + [ctypes.c_int64, vp, vp]
        lib.orc_fwd.restype = ctypes.c_int
        lib.orc_bwd.argtypes = [ctypes.POINTER(_Problem)] + [vp] * 19
        lib.orc_bwd.restype = ctypes.c_int
        lib.orc_fwd_complex.argtypes = [ctypes.POINTER(_Problem)] + [vp] * 11
        lib.orc_fwd_complex.restype = ctypes.c_int
        lib.orc_bwd_complex.argtypes = [ctypes.POINTER(_Problem)] + [vp] * 19
        lib.orc_bwd_complex.restype = ctypes.c_int
        lib.orc_set_threads.argtypes = [ctypes.c_int]
        lib.orc_set_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def set_threads(n: int = 0) -> int:
    """Set the OpenMP thread count (0 keeps the default); returns the count in use."""
    return _load().orc_set_threads(int(n))


def _code(a):
    code = {np.dtype(np.float32): _F32, np.dtype(np.uint16): _BF16,
            np.dtype(np.float64): _F64}.get(a.dtype)
    if code is None:
        raise TypeError(f"oracle inputs must be float64, float32 or uint16 (bf16 bits), got {a.dtype}")
    return code


def _widen(a):
    """Exact float64 copy of a float32 / float64 / bf16-bit-pattern array."""
    if a.dtype == np.uint16:
        a = (a.astype(np.uint32) << np.uint32(16)).view(np.float32)
    return a.astype(np.float64)


def _ios(*arrs):
    """Give the (non-None) I/O arrays one element type: their own if they agree,
    else float64 (every supported type widens to it exactly)."""
    arrs = [None if a is None else np.ascontiguousarray(a) for a in arrs]
    codes = {_code(a) for a in arrs if a is not None}
    if len(codes) > 1:
        arrs = [None if a is None else _widen(a) for a in arrs]
        codes = {_F64}
    return arrs, codes.pop()


def _f64(arr):
    return None if arr is None else np.ascontiguousarray(arr, dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def fwd(u, delta_raw, A, B, C, *, delta_bias=None, D_skip=None, z=None, h0=None,
        delta_softplus=True, rows=None, want_out=True, input_silu=False):
    """Forward scan in fp64.  Returns (out, h_last).

    rows=None: out (batch, L, D), h_last (batch, D, N).
    rows=[b*D+d, ...]: out (len(rows), L), h_last (len(rows), N) for those rows only.
    want_out=False computes only h_last (the last-state operation).
    input_silu=True feeds x = SiLU(u) to the scan instead of u (the input-branch
    activation of the Mamba block, Fig. 3 caption).
    """
    (u, delta_raw, B, C, z), code = _ios(u, delta_raw, B, C, z)
    batch, L, D = u.shape
    N = B.shape[-1]
    assert delta_raw.shape == u.shape and B.shape == (batch, L, N) and C.shape == (batch, L, N)
    A = _f64(A)
    assert A.shape == (D, N)
    delta_bias, D_skip, h0 = _f64(delta_bias), _f64(D_skip), _f64(h0)
    if rows is not None:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        nr = rows.shape[0]
        out = np.empty((nr, L), np.float64) if want_out else None
        h_last = np.empty((nr, N), np.float64)
    else:
        nr = 0
        out = np.empty((batch, L, D), np.float64) if want_out else None
        h_last = np.empty((batch, D, N), np.float64)
    prob = _Problem(batch, L, D, N, code, 1 if delta_softplus else 0, 1 if input_silu else 0)
    rc = _load().orc_fwd(ctypes.byref(prob), _ptr(u), _ptr(delta_raw), _ptr(delta_bias), _ptr(A),
                         _ptr(B), _ptr(C), _ptr(D_skip), _ptr(z), _ptr(h0), _ptr(rows), nr,
                         _ptr(out), _ptr(h_last))
    if rc != 0:
        raise ValueError("orc_fwd rejected its arguments")
    return out, h_last


def bwd(u, delta_raw, A, B, C, dout, *, delta_bias=None, D_skip=None, z=None, h0=None,
        delta_softplus=True, input_silu=False):
    """Reverse-mode gradients of sum(out * dout) in fp64.

    Returns a dict with du, ddelta_raw (batch, L, D); dA (D, N); dB, dC (batch, L, N);
    and, when the matching input is given, ddelta_bias (D,), dD (D,), dz (batch, L, D);
    dh0 (batch, D, N) always.
    """
    (u, delta_raw, B, C, dout, z), code = _ios(u, delta_raw, B, C, dout, z)
    batch, L, D = u.shape
    N = B.shape[-1]
    A = _f64(A)
    delta_bias, D_skip, h0 = _f64(delta_bias), _f64(D_skip), _f64(h0)
    g = {"du": np.empty((batch, L, D)), "ddelta_raw": np.empty((batch, L, D)),
         "dA": np.empty((D, N)), "dB": np.empty((batch, L, N)), "dC": np.empty((batch, L, N)),
         "dh0": np.empty((batch, D, N))}
    g["ddelta_bias"] = np.empty(D) if delta_bias is not None else None
    g["dD"] = np.empty(D) if D_skip is not None else None
    g["dz"] = np.empty((batch, L, D)) if z is not None else None
    prob = _Problem(batch, L, D, N, code, 1 if delta_softplus else 0, 1 if input_silu else 0)
    rc = _load().orc_bwd(ctypes.byref(prob), _ptr(u), _ptr(delta_raw), _ptr(delta_bias), _ptr(A),
                         _ptr(B), _ptr(C), _ptr(D_skip), _ptr(z), _ptr(h0), _ptr(dout),
                         _ptr(g["du"]), _ptr(g["ddelta_raw"]), _ptr(g["ddelta_bias"]),
                         _ptr(g["dA"]), _ptr(g["dB"]), _ptr(g["dC"]), _ptr(g["dD"]),
                         _ptr(g["dz"]), _ptr(g["dh0"]))
    if rc != 0:
        raise ValueError("orc_bwd rejected its arguments")
    return {k: v for k, v in g.items() if v is not None}


def _interleave(c, shape):
    """complex (…) or real (…, 2) -> contiguous float64 (…, 2) pairs (re, im)."""
    if c is None:
        return None
    c = np.asarray(c)
    if np.iscomplexobj(c):
        c = np.stack([c.real, c.imag], axis=-1)
    c = np.ascontiguousarray(c, dtype=np.float64)
    assert c.shape == tuple(shape) + (2,), (c.shape, shape)
    return c


def fwd_complex(u, delta_raw, A, B, C, *, delta_bias=None, D_skip=None, z=None, h0=None,
                delta_softplus=True, want_out=True, input_silu=False):
    """Forward scan with a complex diagonal A in fp64.  A: (D, N) complex (or (D, N, 2)
    real pairs); h0: (batch, D, N) complex or None.  B, C real (batch, L, N).
    Returns (out (batch, L, D) real, h_last (batch, D, N) complex128)."""
    (u, delta_raw, B, C, z), code = _ios(u, delta_raw, B, C, z)
    batch, L, D = u.shape
    N = B.shape[-1]
    A2 = _interleave(A, (D, N))
    h02 = _interleave(h0, (batch, D, N))
    delta_bias, D_skip = _f64(delta_bias), _f64(D_skip)
    out = np.empty((batch, L, D), np.float64) if want_out else None
    h_last = np.empty((batch, D, N, 2), np.float64)
    prob = _Problem(batch, L, D, N, code, 1 if delta_softplus else 0, 1 if input_silu else 0)
    rc = _load().orc_fwd_complex(ctypes.byref(prob), _ptr(u), _ptr(delta_raw), _ptr(delta_bias), _ptr(A2),
                                 _ptr(B), _ptr(C), _ptr(D_skip), _ptr(z), _ptr(h02), _ptr(out), _ptr(h_last))
    if rc != 0:
        raise ValueError("orc_fwd_complex rejected its arguments")
    return out, h_last[..., 0] + 1j * h_last[..., 1]


def bwd_complex(u, delta_raw, A, B, C, dout, *, delta_bias=None, D_skip=None, z=None, h0=None,
                delta_softplus=True, input_silu=False):
    """Reverse-mode gradients of sum(out * dout) for the complex-A scan, fp64.
    dA (D, N) and dh0 (batch, D, N) are complex128 (dL/dRe + i dL/dIm); the rest real,
    keyed as in ``bwd``."""
    (u, delta_raw, B, C, dout, z), code = _ios(u, delta_raw, B, C, dout, z)
    batch, L, D = u.shape
    N = B.shape[-1]
    A2 = _interleave(A, (D, N))
    h02 = _interleave(h0, (batch, D, N))
    delta_bias, D_skip = _f64(delta_bias), _f64(D_skip)
    g = {"du": np.empty((batch, L, D)), "ddelta_raw": np.empty((batch, L, D)),
         "dA": np.empty((D, N, 2)), "dB": np.empty((batch, L, N)), "dC": np.empty((batch, L, N)),
         "dh0": np.empty((batch, D, N, 2))}
    g["ddelta_bias"] = np.empty(D) if delta_bias is not None else None
    g["dD"] = np.empty(D) if D_skip is not None else None
    g["dz"] = np.empty((batch, L, D)) if z is not None else None
    prob = _Problem(batch, L, D, N, code, 1 if delta_softplus else 0, 1 if input_silu else 0)
    rc = _load().orc_bwd_complex(ctypes.byref(prob), _ptr(u), _ptr(delta_raw), _ptr(delta_bias), _ptr(A2),
                                 _ptr(B), _ptr(C), _ptr(D_skip), _ptr(z), _ptr(h02), _ptr(dout),
                                 _ptr(g["du"]), _ptr(g["ddelta_raw"]), _ptr(g["ddelta_bias"]),
                                 _ptr(g["dA"]), _ptr(g["dB"]), _ptr(g["dC"]), _ptr(g["dD"]),
                                 _ptr(g["dz"]), _ptr(g["dh0"]))
    if rc != 0:
        raise ValueError("orc_bwd_complex rejected its arguments")
    g["dA"] = g["dA"][..., 0] + 1j * g["dA"][..., 1]
    g["dh0"] = g["dh0"][..., 0] + 1j * g["dh0"][..., 1]
    return {k: v for k, v in g.items() if v is not None}


__all__ = ["fwd", "bwd", "fwd_complex", "bwd_complex", "set_threads"]
