"""Pins for the fp64 CPU oracle against facts the paper and mathematics fix.

None of these re-types the oracle's own loop: each checks it against an
independent statement of the same result (a hand-worked case, the convolution
form of eq. (4), numerical integration of the continuous ODE of eq. (1), a closed
form, library routines, finite differences).  CPU only.
"""
import math
import os

import numpy as np
import pytest

import oracle
from selective_state_space_33_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
LN2 = math.log(2.0)


def _read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, *v = line.split()
            vals[k] = np.array([float(s) for s in v])
    return vals


def _hand_inputs(g, delta, Bv, Dskip=None):
    L = len(g["x"])
    u = g["x"].reshape(1, L, 1)
    dr = np.asarray(delta, np.float64).reshape(1, L, 1)
    A = g["A"].reshape(1, 1)
    B = np.full((1, L, 1), Bv)
    C = g["C"].reshape(1, L, 1)
    return dict(u=u, delta_raw=dr, A=A, B=B, C=C, D_skip=Dskip, delta_softplus=False)


# ---------------------------------------------------------------- hand-worked case (P4)
def test_hand_case_forward():
    g = _read_golden("hand_n1_l4.txt")
    kw = _hand_inputs(g, g["delta"], g["B"][0])
    out, h_last = oracle.fwd(**kw)
    np.testing.assert_allclose(out.ravel(), g["y"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(h_last.ravel(), g["h_last"], rtol=0, atol=1e-14)
    kw["D_skip"] = np.ones(1)
    out, _ = oracle.fwd(**kw)
    np.testing.assert_allclose(out.ravel(), g["y_dskip1"], rtol=0, atol=1e-14)
    kw = _hand_inputs(g, np.ones(4), g["const_B"][0])
    kw["C"] = np.ones((1, 4, 1))
    out, _ = oracle.fwd(**kw)
    np.testing.assert_allclose(out.ravel(), g["const_y"], rtol=0, atol=1e-14)


def test_hand_case_backward():
    g = _read_golden("hand_n1_l4.txt")
    kw = _hand_inputs(g, g["delta"], g["B"][0])
    dout = np.zeros((1, 4, 1))
    dout[0, 3, 0] = 1.0
    gr = oracle.bwd(kw["u"], kw["delta_raw"], kw["A"], kw["B"], kw["C"], dout, delta_softplus=False)
    np.testing.assert_allclose(gr["du"].ravel(), g["du"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(gr["dC"].ravel(), g["dC"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(gr["ddelta_raw"][0, 3, 0], g["ddelta_4"][0], rtol=1e-14)


# ---------------------------------------------------------------- LTI == convolution (P1, eq. 4)
@pytest.mark.parametrize("N", [1, 3, 16])
def test_lti_equals_convolution(N):
    """With delta, B, C constant in time the recurrence equals y = x * Kbar with
    Kbar_k = sum_n C_n Abar_n^k Bbar_n (eq. 4a/4b), evaluated here by brute force."""
    rng = np.random.default_rng(10 + N)
    batch, L, D = 2, 40, 3
    delta = np.exp(rng.uniform(math.log(0.01), math.log(0.5), size=(batch, D)))
    A = -np.exp(rng.uniform(-1, 1.5, size=(D, N)))
    Bc = rng.standard_normal((batch, N))
    Cc = rng.standard_normal((batch, N))
    u = rng.standard_normal((batch, L, D))
    dr = np.broadcast_to(delta[:, None, :], (batch, L, D)).copy()
    B = np.broadcast_to(Bc[:, None, :], (batch, L, N)).copy()
    C = np.broadcast_to(Cc[:, None, :], (batch, L, N)).copy()
    out, _ = oracle.fwd(u, dr, A, B, C, delta_softplus=False)
    for b in range(batch):
        for d in range(D):
            Abar = np.exp(delta[b, d] * A[d])
            Bbar = np.expm1(delta[b, d] * A[d]) / A[d] * Bc[b]
            K = np.array([np.sum(Cc[b] * Abar ** k * Bbar) for k in range(L)])
            y = np.convolve(u[b, :, d], K)[:L]
            np.testing.assert_allclose(out[b, :, d], y, rtol=1e-11, atol=1e-13)


# ---------------------------------------------------------------- ZOH exactness (P6, eqs. 1 -> 2)
def _rk4_step(h, A, drive, dt, m):
    """Integrate h' = A h + drive over time dt with m classical RK4 substeps."""
    k = dt / m
    for _ in range(m):
        k1 = A * h + drive
        k2 = A * (h + 0.5 * k * k1) + drive
        k3 = A * (h + 0.5 * k * k2) + drive
        k4 = A * (h + k * k3) + drive
        h = h + (k / 6.0) * (k1 + 2 * k2 + 2 * k3 + k4)
    return h


def test_zoh_matches_continuous_ode():
    """For input held constant over each step of length delta_t, eq. (2)+(3) must equal
    the continuous system h' = A h + B x (eq. 1a) integrated numerically, including the
    A = 0 limit (Bbar = delta B) and a positive A."""
    rng = np.random.default_rng(7)
    batch, L, D, N = 2, 12, 3, 4
    A = -np.exp(rng.uniform(-1.0, 1.5, size=(D, N)))
    A[0, 1] = 0.0
    A[2, 3] = 0.3
    u = rng.standard_normal((batch, L, D))
    dr = rng.uniform(0.05, 0.8, size=(batch, L, D))
    B = rng.standard_normal((batch, L, N))
    C = rng.standard_normal((batch, L, N))
    h0 = rng.standard_normal((batch, D, N))
    out, h_last = oracle.fwd(u, dr, A, B, C, h0=h0, delta_softplus=False)
    for b in range(batch):
        for d in range(D):
            h = h0[b, d].copy()
            for t in range(L):
                h = _rk4_step(h, A[d], B[b, t] * u[b, t, d], dr[b, t, d], 400)
                np.testing.assert_allclose(out[b, t, d], np.dot(C[b, t], h), rtol=1e-9, atol=1e-11)
            np.testing.assert_allclose(h_last[b, d], h, rtol=1e-9, atol=1e-11)


# ---------------------------------------------------------------- geometric closed form (P5)
def test_step_response_closed_form():
    """x = 1, N = 1, LTI, A < 0: h_t = (B / -A)(1 - exp(A delta t)), the continuous step
    response at time t*delta."""
    L, dlt, a, bv = 300, 0.037, -1.7, 0.9
    u = np.ones((1, L, 1))
    dr = np.full((1, L, 1), dlt)
    out, h_last = oracle.fwd(u, dr, np.array([[a]]), np.full((1, L, 1), bv), np.ones((1, L, 1)),
                             delta_softplus=False)
    t = np.arange(1, L + 1)
    np.testing.assert_allclose(out.ravel(), bv / -a * -np.expm1(a * dlt * t), rtol=1e-12)


# ---------------------------------------------------------------- delta -> 0 (P2, sec. 3.3)
def test_delta_to_zero_ignores_input_and_holds_state():
    rng = np.random.default_rng(3)
    batch, L, D, N = 2, 17, 5, 4
    x = W.small_case(batch, L, D, N, io="f32", seed=3)
    dr = np.full((batch, L, D), -40.0)
    h0 = rng.standard_normal((batch, D, N))
    out, h_last = oracle.fwd(x["u"], dr, x["A"], x["B"], x["C"], D_skip=x["D_skip"], z=x["z"],
                             h0=h0, delta_softplus=True)
    # delta = softplus(-40) ~ 4e-18: the state is held, so y_t = C_t . h0 + D x_t
    u, z = x["u"].astype(np.float64), x["z"].astype(np.float64)
    Cm = x["C"].astype(np.float64)
    gate = z / (1.0 + np.exp(-z))
    ref = (np.einsum("bln,bdn->bld", Cm, h0) + x["D_skip"].astype(np.float64) * u) * gate
    np.testing.assert_allclose(out, ref, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(h_last, h0, rtol=1e-14)


# ---------------------------------------------------------------- split with carry (P3)
@pytest.mark.parametrize("k", [1, 31, 32, 33, 63])
def test_split_with_carry_is_exact(k):
    x = W.small_case(2, 64, 3, 4, io="f32", seed=5)
    full, hl = oracle.fwd(x["u"], x["delta_raw"], x["A"], x["B"], x["C"], delta_bias=x["delta_bias"],
                          D_skip=x["D_skip"], z=x["z"])
    cut = lambda a, s: np.ascontiguousarray(a[:, s])
    s1, s2 = slice(0, k), slice(k, 64)
    o1, h1 = oracle.fwd(cut(x["u"], s1), cut(x["delta_raw"], s1), x["A"], cut(x["B"], s1),
                        cut(x["C"], s1), delta_bias=x["delta_bias"], D_skip=x["D_skip"],
                        z=cut(x["z"], s1))
    o2, h2 = oracle.fwd(cut(x["u"], s2), cut(x["delta_raw"], s2), x["A"], cut(x["B"], s2),
                        cut(x["C"], s2), delta_bias=x["delta_bias"], D_skip=x["D_skip"],
                        z=cut(x["z"], s2), h0=h1)
    assert np.array_equal(np.concatenate([o1, o2], axis=1), full)
    assert np.array_equal(h2, hl)


# ---------------------------------------------------------------- softplus / gate / readout pins
def test_softplus_against_library():
    """One step with N = 1, A = -a, B = C = x = 1, h0 = 0 gives y = (1 - e^{-a delta}) / a,
    so delta can be read back and compared with numpy's logaddexp(0, r) = softplus(r)."""
    r = np.array([-30.0, -9.0, -2.0, 0.0, math.log(math.e - 1.0), 1.5, 20.0, 40.0])
    a = 1e-3
    n = r.size
    out, _ = oracle.fwd(np.ones((1, 1, n)), r.reshape(1, 1, n), np.full((n, 1), -a),
                        np.ones((1, 1, 1)), np.ones((1, 1, 1)), delta_softplus=True)
    delta = -np.log1p(-a * out.ravel()) / a
    np.testing.assert_allclose(delta, np.logaddexp(0.0, r), rtol=1e-9)
    assert abs(delta[3] - LN2) < 1e-12 and abs(delta[4] - 1.0) < 1e-12


def test_gate_against_library():
    """With B = 0 the state stays zero and out = D x SiLU(z) (Fig. 3: SiLU gate)."""
    from scipy.special import expit
    x = W.small_case(2, 9, 6, 3, io="f32", seed=11)
    out, _ = oracle.fwd(x["u"], x["delta_raw"], x["A"], np.zeros_like(x["B"]), x["C"],
                        delta_bias=x["delta_bias"], D_skip=x["D_skip"], z=x["z"])
    z = x["z"].astype(np.float64)
    np.testing.assert_allclose(out, x["D_skip"] * x["u"].astype(np.float64) * z * expit(z),
                               rtol=1e-14, atol=1e-300)


def test_bf16_inputs_widen_exactly():
    x = W.small_case(1, 20, 8, 4, io="bf16", seed=12)
    o16, _ = oracle.fwd(x["u"], x["delta_raw"], x["A"], x["B"], x["C"], delta_bias=x["delta_bias"],
                        D_skip=x["D_skip"], z=x["z"])
    f = {k: W.bf16_bits_to_f32(x[k]) for k in ("u", "delta_raw", "B", "C", "z")}
    o32, _ = oracle.fwd(f["u"], f["delta_raw"], x["A"], f["B"], f["C"], delta_bias=x["delta_bias"],
                        D_skip=x["D_skip"], z=f["z"])
    assert np.array_equal(o16, o32)


# ---------------------------------------------------------------- structural invariants (P7)
def test_linearity_causality_and_independence():
    rng = np.random.default_rng(21)
    x = W.small_case(2, 30, 5, 4, io="f32", seed=21)
    args = (x["delta_raw"], x["A"], x["B"], x["C"])
    kw = dict(delta_bias=x["delta_bias"], D_skip=x["D_skip"])
    u1 = x["u"].astype(np.float64)
    u2 = rng.standard_normal(u1.shape)
    h1, h2 = rng.standard_normal((2, 5, 4)), rng.standard_normal((2, 5, 4))
    f = lambda uu, hh: oracle.fwd(uu, args[0].astype(np.float64), args[1], args[2].astype(np.float64),
                                  args[3].astype(np.float64), h0=hh, **kw)
    o1, l1 = f(u1, h1)
    o2, l2 = f(u2, h2)
    o3, l3 = f(2.0 * u1 - 3.0 * u2, 2.0 * h1 - 3.0 * h2)
    np.testing.assert_allclose(o3, 2.0 * o1 - 3.0 * o2, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(l3, 2.0 * l1 - 3.0 * l2, rtol=1e-12, atol=1e-12)
    # causality: perturbing x at t' leaves y_{t<t'} unchanged
    up = u1.copy()
    up[:, 17, :] += 5.0
    op, _ = f(up, h1)
    assert np.array_equal(op[:, :17], o1[:, :17]) and not np.allclose(op[:, 17:], o1[:, 17:])
    # channel permutation equivariance (B, C shared across channels)
    perm = np.array([3, 0, 4, 1, 2])
    o_full, _ = oracle.fwd(x["u"], x["delta_raw"], x["A"], x["B"], x["C"], z=x["z"], **kw)
    kwp = dict(delta_bias=x["delta_bias"][perm], D_skip=x["D_skip"][perm])
    o_perm, _ = oracle.fwd(x["u"][:, :, perm], x["delta_raw"][:, :, perm], x["A"][perm], x["B"], x["C"],
                           z=x["z"][:, :, perm], **kwp)
    assert np.array_equal(o_perm, o_full[:, :, perm])
    # row subset equals the full computation
    rows = np.array([0, 7, 9])
    o_rows, _ = oracle.fwd(x["u"], x["delta_raw"], x["A"], x["B"], x["C"], z=x["z"], rows=rows, **kw)
    for i, r in enumerate(rows):
        assert np.array_equal(o_rows[i], o_full[r // 5, :, r % 5])


# ---------------------------------------------------------------- backward: finite differences
def _fd_case(seed=0):
    """Config-0 shape (batch 1, L 64, D 4, N 4) in float64 with every optional input."""
    w = W.WORKLOADS["tiny"]
    x = W.make_inputs(w.with_(seed=seed))
    rng = np.random.default_rng(100 + seed)
    p = {k: x[k].astype(np.float64) for k in ("u", "delta_raw", "z", "B", "C", "A", "delta_bias", "D_skip")}
    p["h0"] = rng.standard_normal((w.batch, w.dim, w.dstate)) * 0.5
    dout = rng.standard_normal((w.batch, w.seqlen, w.dim))
    return p, dout


def _loss(p, dout):
    out, _ = oracle.fwd(p["u"], p["delta_raw"], p["A"], p["B"], p["C"], delta_bias=p["delta_bias"],
                        D_skip=p["D_skip"], z=p["z"], h0=p["h0"])
    return float(np.sum(out * dout))


def test_backward_matches_central_differences():
    p, dout = _fd_case()
    g = oracle.bwd(p["u"], p["delta_raw"], p["A"], p["B"], p["C"], dout, delta_bias=p["delta_bias"],
                   D_skip=p["D_skip"], z=p["z"], h0=p["h0"])
    names = {"u": "du", "delta_raw": "ddelta_raw", "z": "dz", "B": "dB", "C": "dC", "A": "dA",
             "delta_bias": "ddelta_bias", "D_skip": "dD", "h0": "dh0"}
    for pn, gn in names.items():
        fd = np.empty_like(p[pn])
        flat = p[pn].reshape(-1)
        for i in range(flat.size):
            v = flat[i]
            step = 1e-6 * max(1.0, abs(v))
            flat[i] = v + step
            lp = _loss(p, dout)
            flat[i] = v - step
            lm = _loss(p, dout)
            flat[i] = v
            fd.reshape(-1)[i] = (lp - lm) / (2 * step)
        err = np.max(np.abs(fd - g[gn])) / max(np.max(np.abs(g[gn])), 1e-300)
        assert err < 1e-6, (pn, err)


def test_backward_adjoint_identity():
    """<dout, J v> = <J^T dout, v> for a random joint direction v over every input."""
    p, dout = _fd_case(seed=1)
    rng = np.random.default_rng(5)
    g = oracle.bwd(p["u"], p["delta_raw"], p["A"], p["B"], p["C"], dout, delta_bias=p["delta_bias"],
                   D_skip=p["D_skip"], z=p["z"], h0=p["h0"])
    names = {"u": "du", "delta_raw": "ddelta_raw", "z": "dz", "B": "dB", "C": "dC", "A": "dA",
             "delta_bias": "ddelta_bias", "D_skip": "dD", "h0": "dh0"}
    v = {k: rng.standard_normal(p[k].shape) for k in names}
    eps = 1e-6
    plus = {k: p[k] + eps * v[k] for k in p}
    minus = {k: p[k] - eps * v[k] for k in p}
    jvp = (_loss(plus, dout) - _loss(minus, dout)) / (2 * eps)
    vjp = sum(float(np.sum(g[gn] * v[pn])) for pn, gn in names.items())
    assert abs(jvp - vjp) <= 1e-7 * max(1.0, abs(vjp))


def test_backward_skip_gradient_closed_form():
    """dD_d = sum_{b,t} dout * SiLU(z) * x (out is linear in D_skip)."""
    p, dout = _fd_case(seed=2)
    g = oracle.bwd(p["u"], p["delta_raw"], p["A"], p["B"], p["C"], dout, delta_bias=p["delta_bias"],
                   D_skip=p["D_skip"], z=p["z"], h0=p["h0"])
    from scipy.special import expit
    s = p["z"] * expit(p["z"])
    np.testing.assert_allclose(g["dD"], np.sum(dout * s * p["u"], axis=(0, 1)), rtol=1e-12)


def test_backward_gate_gradient_closed_form():
    """dz = dout * y * sigma(z) * (1 + z (1 - sigma(z))), y the ungated output (the
    derivative of SiLU(z) = z sigma(z); the gate of Fig. 3)."""
    p, dout = _fd_case(seed=3)
    g = oracle.bwd(p["u"], p["delta_raw"], p["A"], p["B"], p["C"], dout, delta_bias=p["delta_bias"],
                   D_skip=p["D_skip"], z=p["z"], h0=p["h0"])
    y, _ = oracle.fwd(p["u"], p["delta_raw"], p["A"], p["B"], p["C"], delta_bias=p["delta_bias"],
                      D_skip=p["D_skip"], h0=p["h0"])
    from scipy.special import expit
    sg = expit(p["z"])
    np.testing.assert_allclose(g["dz"], dout * y * sg * (1.0 + p["z"] * (1.0 - sg)), rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- one step, high precision
def _dec_expm1_over(q_str, a_str, digits=60):
    """expm1(q)/a and the A-derivative delta^2 (q e^q - expm1(q))/q^2 in 60-digit decimals."""
    import decimal
    ctx = decimal.Context(prec=digits)
    q, a = decimal.Decimal(q_str), decimal.Decimal(a_str)
    em1 = ctx.exp(q) - 1
    return em1, q * ctx.exp(q) - em1


@pytest.mark.parametrize("delta,a", [(1e-3, -0.5), (2e-4, -0.5), (1e-3, -2.0), (0.3, -1.0),
                                     (0.7, -4.0), (1e-6, -3.0), (0.05, 0.2)])
def test_single_step_against_decimal_arithmetic(delta, a):
    """One step from h0 = 0 with x = B = C = 1: y = Bbar = expm1(delta a)/a (eq. 2), and
    d y / d A = (q e^q - expm1(q)) / a^2 with q = delta a; both evaluated to 60 digits."""
    import decimal
    dd, ad = decimal.Decimal(repr(delta)), decimal.Decimal(repr(a))
    em1, num = _dec_expm1_over(str(dd * ad), str(ad))
    y_ref = float(em1 / ad)
    dA_ref = float(num / (ad * ad))
    one = np.ones((1, 1, 1))
    out, _ = oracle.fwd(one, np.full((1, 1, 1), delta), np.array([[a]]), one, one, delta_softplus=False)
    g = oracle.bwd(one, np.full((1, 1, 1), delta), np.array([[a]]), one, one, one, delta_softplus=False)
    assert abs(out.item() - y_ref) <= 4e-16 * abs(y_ref)
    assert abs(g["dA"].item() - dA_ref) <= 1e-12 * abs(dA_ref), (g["dA"].item(), dA_ref)


# ---------------------------------------------------------------- input-branch activation (Fig. 3)
def test_input_silu_equals_scan_of_activated_input():
    """With the input-branch activation the scan's input is x = SiLU(u) (Fig. 3
    caption: the block's first gate becomes an activation, sigma = SiLU).  Forming
    u * expit(u) with scipy and scanning it without the flag must give the same
    outputs and final states, in the state update and the skip term alike."""
    from scipy.special import expit
    x = W.small_case(2, 40, 6, 5, io="f32", seed=31)
    u = x["u"].astype(np.float64)
    h0 = np.random.default_rng(31).standard_normal((2, 6, 5))
    kw = dict(delta_bias=x["delta_bias"], D_skip=x["D_skip"], z=x["z"], h0=h0)
    o1, l1 = oracle.fwd(u, x["delta_raw"], x["A"], x["B"], x["C"], input_silu=True, **kw)
    o2, l2 = oracle.fwd(u * expit(u), x["delta_raw"].astype(np.float64), x["A"], x["B"].astype(np.float64),
                        x["C"].astype(np.float64), **kw)
    np.testing.assert_allclose(o1, o2, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(l1, l2, rtol=1e-13, atol=1e-15)
    # the flag changes the result (it is not ignored)
    o3, _ = oracle.fwd(u, x["delta_raw"], x["A"], x["B"], x["C"], **kw)
    assert np.max(np.abs(o3 - o1)) > 1e-3


def test_input_silu_complex_equals_scan_of_activated_input():
    from scipy.special import expit
    x = W.small_case(1, 30, 4, 3, io="f32", seed=32, complex_a=True)
    u = x["u"].astype(np.float64)
    kw = dict(delta_bias=x["delta_bias"], D_skip=x["D_skip"], z=x["z"])
    o1, l1 = oracle.fwd_complex(u, x["delta_raw"], x["A"], x["B"], x["C"], input_silu=True, **kw)
    o2, l2 = oracle.fwd_complex(u * expit(u), x["delta_raw"].astype(np.float64), x["A"],
                                x["B"].astype(np.float64), x["C"].astype(np.float64), **kw)
    np.testing.assert_allclose(o1, o2, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(l1, l2, rtol=1e-13, atol=1e-15)


def _loss_silu(p, dout, complex_a=False):
    f = oracle.fwd_complex if complex_a else oracle.fwd
    out, _ = f(p["u"], p["delta_raw"], p["A"], p["B"], p["C"], delta_bias=p["delta_bias"], D_skip=p["D_skip"],
               z=p["z"], h0=p.get("h0"), input_silu=True)
    return float(np.sum(out * dout))


def _central(p, name, dout, **kw):
    fd = np.empty_like(p[name])
    flat = p[name].reshape(-1)
    for i in range(flat.size):
        v = flat[i]
        step = 1e-6 * max(1.0, abs(v))
        flat[i] = v + step
        lp = _loss_silu(p, dout, **kw)
        flat[i] = v - step
        lm = _loss_silu(p, dout, **kw)
        flat[i] = v
        fd.reshape(-1)[i] = (lp - lm) / (2 * step)
    return fd


def test_input_silu_backward_matches_central_differences():
    """Every gradient of the scan with the input activation, against central
    differences of the forward oracle at the config-0 shape."""
    p, dout = _fd_case(seed=3)
    g = oracle.bwd(p["u"], p["delta_raw"], p["A"], p["B"], p["C"], dout, delta_bias=p["delta_bias"],
                   D_skip=p["D_skip"], z=p["z"], h0=p["h0"], input_silu=True)
    names = {"u": "du", "delta_raw": "ddelta_raw", "z": "dz", "B": "dB", "C": "dC", "A": "dA",
             "delta_bias": "ddelta_bias", "D_skip": "dD", "h0": "dh0"}
    for pn, gn in names.items():
        fd = _central(p, pn, dout)
        err = np.max(np.abs(fd - g[gn])) / max(np.max(np.abs(g[gn])), 1e-300)
        assert err < 1e-6, (pn, err)


def test_input_silu_complex_backward_matches_central_differences():
    w = W.WORKLOADS["tiny"]
    x = W.make_inputs(w.with_(seed=4, complex_a=True))
    p = {k: x[k].astype(np.float64) for k in ("u", "delta_raw", "z", "B", "C", "delta_bias", "D_skip")}
    p["A"] = x["A"]
    dout = np.random.default_rng(44).standard_normal((w.batch, w.seqlen, w.dim))
    g = oracle.bwd_complex(p["u"], p["delta_raw"], p["A"], p["B"], p["C"], dout, delta_bias=p["delta_bias"],
                           D_skip=p["D_skip"], z=p["z"], input_silu=True)
    for pn, gn in {"u": "du", "delta_raw": "ddelta_raw", "B": "dB"}.items():
        fd = _central(p, pn, dout, complex_a=True)
        err = np.max(np.abs(fd - g[gn])) / max(np.max(np.abs(g[gn])), 1e-300)
        assert err < 1e-6, (pn, err)
