"""Pins for the oracle's complex-A forward scan (the complex initialisation
A_n = -1/2 + n i of the A-init ablation table, sec. 6.5 of the Mamba technical
summary page), each against something other than the oracle itself: the real
oracle in the Im(A) = 0 special case, a brute-force convolution with complex powers
(eq. 4), a numerical integration of the continuous system (eq. 1, which pins the
discretisation eq. 2), the continuous step response, exact splitting with a carried
state, linearity and causality; and for its backward, central finite differences of
every input (real and imaginary parts of A and h0 separately), the real backward in
the Im(A) = 0 case, and the adjoint identity.  CPU only.
"""
import numpy as np
import pytest

import oracle
from selective_state_space_33_b200 import workloads as W


def _complex_A(D, N, seed):
    rng = np.random.default_rng(seed)
    re = -np.exp(rng.uniform(-3, 1, size=(D, N)))
    im = rng.uniform(-6, 6, size=(D, N))
    return re + 1j * im


def test_zero_imaginary_part_is_the_real_scan():
    x = W.small_case(2, 50, 6, 5, io="f32", seed=61)
    A = x["A"].astype(np.float64)
    A[1, 2] = 0.0  # the A = 0 limit too
    kw = dict(delta_bias=x["delta_bias"], D_skip=x["D_skip"], z=x["z"])
    h0 = np.random.default_rng(1).standard_normal((2, 6, 5))
    out_r, h_r = oracle.fwd(x["u"], x["delta_raw"], A, x["B"], x["C"], h0=h0, **kw)
    out_c, h_c = oracle.fwd_complex(x["u"], x["delta_raw"], A + 0j, x["B"], x["C"], h0=h0 + 0j, **kw)
    np.testing.assert_allclose(out_c, out_r, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(h_c.real, h_r, rtol=1e-12, atol=1e-13)
    assert np.all(h_c.imag == 0.0)


@pytest.mark.parametrize("N", [1, 4])
def test_lti_equals_convolution_with_complex_powers(N):
    """Delta, B, C constant in t, no skip, no gate: y_t = sum_k Re(sum_n C_n Abar_n^(t-k)
    Bbar_n) x_k (eq. 4), with the kernel formed from complex powers, not the recurrence."""
    batch, L, D = 1, 24, 3
    rng = np.random.default_rng(7 + N)
    A = _complex_A(D, N, 70 + N)
    u = rng.standard_normal((batch, L, D))
    dr = np.repeat(rng.uniform(-4, -1, size=(batch, 1, D)), L, axis=1)
    B = np.repeat(rng.standard_normal((batch, 1, N)), L, axis=1)
    C = np.repeat(rng.standard_normal((batch, 1, N)), L, axis=1)
    out, _ = oracle.fwd_complex(u, dr, A, B, C)
    delta = np.log1p(np.exp(dr[0, 0]))  # softplus, per channel
    for d in range(D):
        ab = np.exp(delta[d] * A[d])
        bb = (ab - 1.0) / A[d] * B[0, 0]
        K = np.array([np.real(np.sum(C[0, 0] * ab ** k * bb)) for k in range(L)])
        ref = np.array([np.sum(K[:t + 1][::-1] * u[0, :t + 1, d]) for t in range(L)])
        np.testing.assert_allclose(out[0, :, d], ref, rtol=1e-10, atol=1e-12)


def test_zoh_matches_the_continuous_system():
    """With x held constant over each step of length delta, the discrete state equals
    the solution of h' = a h + B x integrated numerically (RK4, fine steps): eq. (1)
    -> eq. (2) exactly, for complex a."""
    batch, L, D, N = 1, 6, 2, 3
    rng = np.random.default_rng(11)
    A = _complex_A(D, N, 12)
    u = rng.standard_normal((batch, L, D))
    dr = rng.uniform(-2.5, 0.5, size=(batch, L, D))
    B = rng.standard_normal((batch, L, N))
    C = rng.standard_normal((batch, L, N))
    h0 = rng.standard_normal((batch, D, N)) + 1j * rng.standard_normal((batch, D, N))
    out, h_last = oracle.fwd_complex(u, dr, A, B, C, h0=h0)
    delta = np.log1p(np.exp(dr))
    for d in range(D):
        h = h0[0, d].copy()
        for t in range(L):
            f = lambda hh: A[d] * hh + B[0, t] * u[0, t, d]
            steps = 400
            dt = delta[0, t, d] / steps
            for _ in range(steps):
                k1 = f(h)
                k2 = f(h + 0.5 * dt * k1)
                k3 = f(h + 0.5 * dt * k2)
                k4 = f(h + dt * k3)
                h = h + dt / 6.0 * (k1 + 2 * k2 + 2 * k3 + k4)
            np.testing.assert_allclose(out[0, t, d], np.real(np.sum(C[0, t] * h)), rtol=1e-8, atol=1e-10)
        np.testing.assert_allclose(h_last[0, d], h, rtol=1e-8, atol=1e-10)


def test_step_response_closed_form():
    """N = 1, x = 1, constant delta and B, h0 = 0: h_t = B/(-a) (1 - e^(a delta (t+1)))."""
    L = 30
    a = -0.5 + 3.0j
    dr = np.full((1, L, 1), -1.2)
    delta = np.log1p(np.exp(-1.2))
    u = np.ones((1, L, 1))
    B = np.full((1, L, 1), 0.7)
    C = np.full((1, L, 1), 1.3)
    out, h_last = oracle.fwd_complex(u, dr, np.array([[a]]), B, C)
    t = np.arange(1, L + 1)
    h = 0.7 / (-a) * (1.0 - np.exp(a * delta * t))
    np.testing.assert_allclose(out[0, :, 0], 1.3 * h.real, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(h_last[0, 0, 0], h[-1], rtol=1e-12)


@pytest.mark.parametrize("k", [1, 17, 39])
def test_split_with_carry_is_exact(k):
    x = W.small_case(2, 40, 4, 3, io="f32", seed=13)
    A = _complex_A(4, 3, 14)
    kw = dict(delta_bias=x["delta_bias"], D_skip=x["D_skip"])
    full, hf = oracle.fwd_complex(x["u"], x["delta_raw"], A, x["B"], x["C"], z=x["z"], **kw)
    cut = lambda a, s: np.ascontiguousarray(a[:, s])
    o1, h1 = oracle.fwd_complex(cut(x["u"], slice(0, k)), cut(x["delta_raw"], slice(0, k)), A,
                                cut(x["B"], slice(0, k)), cut(x["C"], slice(0, k)), z=cut(x["z"], slice(0, k)), **kw)
    o2, h2 = oracle.fwd_complex(cut(x["u"], slice(k, None)), cut(x["delta_raw"], slice(k, None)), A,
                                cut(x["B"], slice(k, None)), cut(x["C"], slice(k, None)),
                                z=cut(x["z"], slice(k, None)), h0=h1, **kw)
    assert np.array_equal(np.concatenate([o1, o2], axis=1), full)
    assert np.array_equal(h2, hf)


def test_linearity_and_causality():
    rng = np.random.default_rng(15)
    x = W.small_case(1, 30, 3, 4, io="f32", seed=15)
    A = _complex_A(3, 4, 16)
    u1 = x["u"].astype(np.float64)
    u2 = rng.standard_normal(u1.shape)
    c = lambda: rng.standard_normal((1, 3, 4)) + 1j * rng.standard_normal((1, 3, 4))
    g1, g2 = c(), c()
    f = lambda uu, hh: oracle.fwd_complex(uu, x["delta_raw"], A, x["B"], x["C"], D_skip=x["D_skip"], h0=hh)
    o1, l1 = f(u1, g1)
    o2, l2 = f(u2, g2)
    o3, l3 = f(2.0 * u1 - 3.0 * u2, 2.0 * g1 - 3.0 * g2)
    np.testing.assert_allclose(o3, 2.0 * o1 - 3.0 * o2, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(l3, 2.0 * l1 - 3.0 * l2, rtol=1e-11, atol=1e-11)
    up = u1.copy()
    up[:, 20, :] += 4.0
    op, _ = f(up, g1)
    assert np.array_equal(op[:, :20], o1[:, :20]) and not np.allclose(op[:, 20:], o1[:, 20:])


# ---------------------------------------------------------------- backward
def _bwd_case(seed):
    """Small case with every optional input, complex A and h0, in float64."""
    x = W.small_case(1, 24, 3, 3, io="f32", seed=seed, backward=True, complex_a=True)
    rng = np.random.default_rng(200 + seed)
    p = {k: x[k].astype(np.float64) for k in ("u", "delta_raw", "z", "B", "C", "delta_bias", "D_skip")}
    p["A"] = _complex_A(3, 3, 300 + seed)
    p["h0"] = (rng.standard_normal((1, 3, 3)) + 1j * rng.standard_normal((1, 3, 3))) * 0.5
    dout = rng.standard_normal((1, 24, 3))
    return p, dout


def _closs(p, dout):
    out, _ = oracle.fwd_complex(p["u"], p["delta_raw"], p["A"], p["B"], p["C"], delta_bias=p["delta_bias"],
                                D_skip=p["D_skip"], z=p["z"], h0=p["h0"])
    return float(np.sum(out * dout))


def _cgrads(p, dout):
    return oracle.bwd_complex(p["u"], p["delta_raw"], p["A"], p["B"], p["C"], dout, delta_bias=p["delta_bias"],
                              D_skip=p["D_skip"], z=p["z"], h0=p["h0"])


def test_complex_backward_matches_central_differences():
    p, dout = _bwd_case(0)
    g = _cgrads(p, dout)
    names = {"u": "du", "delta_raw": "ddelta_raw", "z": "dz", "B": "dB", "C": "dC", "delta_bias": "ddelta_bias",
             "D_skip": "dD", "A": "dA", "h0": "dh0"}
    for pn, gn in names.items():
        arr = p[pn]
        parts = [(1.0, np.real)] + ([(1j, np.imag)] if np.iscomplexobj(arr) else [])
        for unit, take in parts:
            fd = np.empty(arr.shape)
            for idx in np.ndindex(arr.shape):
                v = arr[idx]
                step = 1e-6 * max(1.0, abs(v))
                arr[idx] = v + unit * step
                lp = _closs(p, dout)
                arr[idx] = v - unit * step
                lm = _closs(p, dout)
                arr[idx] = v
                fd[idx] = (lp - lm) / (2 * step)
            ref = take(g[gn]) if np.iscomplexobj(g[gn]) else g[gn]
            err = np.max(np.abs(fd - ref)) / max(np.max(np.abs(ref)), 1e-300)
            assert err < 1e-6, (pn, take.__name__, err)


def test_complex_backward_with_zero_imaginary_part_is_the_real_backward():
    x = W.small_case(2, 30, 4, 3, io="f32", seed=31, backward=True)
    A = x["A"].astype(np.float64)
    A[1, 1] = 0.0
    h0 = np.random.default_rng(32).standard_normal((2, 4, 3))
    kw = dict(delta_bias=x["delta_bias"], D_skip=x["D_skip"], z=x["z"])
    gr = oracle.bwd(x["u"], x["delta_raw"], A, x["B"], x["C"], x["dout"], h0=h0, **kw)
    gc = oracle.bwd_complex(x["u"], x["delta_raw"], A + 0j, x["B"], x["C"], x["dout"], h0=h0 + 0j, **kw)
    for k in gr:
        got = gc[k].real if np.iscomplexobj(gc[k]) else gc[k]
        np.testing.assert_allclose(got, gr[k], rtol=1e-9, atol=1e-11, err_msg=k)


def test_complex_backward_adjoint_identity():
    p, dout = _bwd_case(1)
    g = _cgrads(p, dout)
    rng = np.random.default_rng(9)
    names = {"u": "du", "delta_raw": "ddelta_raw", "z": "dz", "B": "dB", "C": "dC", "delta_bias": "ddelta_bias",
             "D_skip": "dD", "A": "dA", "h0": "dh0"}
    v = {k: (rng.standard_normal(p[k].shape) + (1j * rng.standard_normal(p[k].shape) if np.iscomplexobj(p[k])
                                                else 0.0)) for k in names}
    eps = 1e-6
    plus = {k: p[k] + eps * v[k] for k in p}
    minus = {k: p[k] - eps * v[k] for k in p}
    jvp = (_closs(plus, dout) - _closs(minus, dout)) / (2 * eps)
    # for complex parameters, <grad, v> pairs the real parts and the imaginary parts
    vjp = sum(float(np.sum(np.real(g[gn]) * np.real(v[pn]) + np.imag(g[gn]) * np.imag(v[pn])))
              for pn, gn in names.items())
    assert abs(jvp - vjp) <= 1e-7 * max(1.0, abs(vjp))


@pytest.mark.parametrize("delta,a", [(1e-3, -0.5 + 0.3j), (2e-4, -0.5 + 2.0j), (0.05, -0.01 + 0.01j),
                                     (0.7, -0.5 + 4.0j), (1e-6, -3.0 + 1.0j)])
def test_complex_single_step_gradient_against_mpmath(delta, a):
    """L = 1, N = 1, h0 = 0, no skip, no gate, softplus off: the A-gradient of one step is
    dout C B x delta^2 conj(psi(delta a)) with psi(q) = (q e^q - (e^q - 1)) / q^2, here
    evaluated in 50-digit arithmetic (mpmath), small q included."""
    import mpmath
    mpmath.mp.dps = 50
    q = mpmath.mpc(delta) * mpmath.mpc(a.real, a.imag)
    psi = (q * mpmath.exp(q) - mpmath.expm1(q)) / (q * q)
    B, C, x, go = 0.7, -1.3, 0.9, 1.1
    g = oracle.bwd_complex(np.full((1, 1, 1), x), np.full((1, 1, 1), delta), np.array([[a]]),
                           np.full((1, 1, 1), B), np.full((1, 1, 1), C), np.full((1, 1, 1), go),
                           delta_softplus=False)
    ref = go * C * B * x * delta * delta * complex(mpmath.conj(psi))
    assert abs(g["dA"][0, 0] - ref) <= 1e-12 * abs(ref)
