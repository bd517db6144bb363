"""The oracle's pins must be strong enough to catch plausible mistakes.

Each case plants one mistake in a temporary copy of the oracle's C source (a dropped
term, a wrong sign, a wrong index, a swapped order), builds it, and runs the pin
suite against that build in a subprocess: the suite must fail.  CPU only.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "sscan_oracle.c")

MUTANTS = {
    "euler_bbar": ("const double bbar = bbar_coef(delta, a) * ld(B, dt, s + n);",
                   "const double bbar = delta * ld(B, dt, s + n);"),
    "no_skip": ("if (D_skip) y += D_skip[d] * x;", ";"),
    "sigmoid_gate": ("if (z) y *= silu(ld(z, dt, e));", "if (z) y *= sigmoid(ld(z, dt, e));"),
    "readout_before_update": (
        "h[n] = abar * h[n] + bbar * x;                         /* eq. (3a) */\n"
        "                if (out) y += ld(C, dt, s + n) * h[n];                 /* eq. (3b) */",
        "if (out) y += ld(C, dt, s + n) * h[n];\n"
        "                h[n] = abar * h[n] + bbar * x;"),
    "A_transposed": ("const double a = A[d * N + n];\n                const double abar = exp(delta * a);",
                     "const double a = A[n * D + d];\n                const double abar = exp(delta * a);"),
    "softplus_no_max": ("return (r > 0.0 ? r : 0.0) + log1p(exp(-fabs(r)));", "return log1p(exp(-fabs(r)));"),
    "bias_ignored": ("ld(delta_raw, dt, e) + (delta_bias ? delta_bias[d] : 0.0);", "ld(delta_raw, dt, e);"),
    "h0_ignored": ("for (int64_t n = 0; n < N; ++n) h[n] = h0 ? h0[row * N + n] : 0.0;",
                   "for (int64_t n = 0; n < N; ++n) h[n] = 0.0;"),
    "B_wrong_index": ("const double bbar = bbar_coef(delta, a) * ld(B, dt, s + n);",
                      "const double bbar = bbar_coef(delta, a) * ld(B, dt, s + (n + d) % N);"),
    "bwd_psi_sign": ("+ dbeta * delta * delta * psi(q);", "- dbeta * delta * delta * psi(q);"),
    "bwd_dB_no_beta": ("dB[s + n] += l * beta * x;", "dB[s + n] += l * x;"),
    "bwd_lam_no_decay": ("lam[n] = abar * l;", "lam[n] = l;"),
    "bwd_dz_formula": ("(1.0 + zz * (1.0 - sg))", "(1.0 + (1.0 - sg))"),
    "bwd_no_softplus_chain": ("ddelta * sigmoid(r) : ddelta;", "ddelta : ddelta;"),
    "psi_series_term": ("q * (1.0 / 8.0 + q * (1.0 / 30.0", "q * (1.0 / 6.0 + q * (1.0 / 30.0"),
    "complex_rotation_sign": ("const double abr = ex * cos(qi), abi = ex * sin(qi);",
                              "const double abr = ex * cos(qi), abi = -ex * sin(qi);"),
    "complex_readout_imag": ("if (out) y += ld(C, dt, s + n) * hr[n];", "if (out) y += ld(C, dt, s + n) * hi[n];"),
    "complex_division_sign": ("ci = (em1i * ar - em1r * ai) / den;", "ci = (em1i * ar + em1r * ai) / den;"),
    "complex_state_mix": ("const double ni = abr * hi[n] + abi * hr[n] + ci * bx;",
                          "const double ni = abr * hi[n] - abi * hr[n] + ci * bx;"),
    "complex_half_angle": ("- 2.0 * sh * sh, em1i", "- sh * sh, em1i"),
    "complex_bwd_no_conj": ("lam[n] = conj(abar) * l;", "lam[n] = abar * l;"),
    "complex_bwd_dA_imag_sign": ("dA[(d * N + n) * 2 + 1] -= cimag(g);", "dA[(d * N + n) * 2 + 1] += cimag(g);"),
    "complex_bwd_psi_term": ("q * (1.0 / 8.0 + q * (1.0 / 30.0 + q * (1.0 / 144.0))));\n    return (q * cexp(q)",
                             "q * (1.0 / 6.0 + q * (1.0 / 30.0 + q * (1.0 / 144.0))));\n    return (q * cexp(q)"),
    "input_silu_skip_raw": ("if (D_skip) y += D_skip[d] * x;", "if (D_skip) y += D_skip[d] * ld(u, dt, e);"),
    "input_silu_no_chain": ("du[e] = dx * scan_input_grad(p, ld(u, dt, e));", "du[e] = dx;"),
    "complex_bwd_ddelta_drop": ("ddelta += creal(conj(l) * (a * abar * hp + abar * Bn * x));",
                                "ddelta += creal(conj(l) * (abar * Bn * x));"),
}
PIN_FILES = ["test_oracle_pins.py", "test_oracle_complex_pins.py"]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor not found: {name}"
    mutated = tmp_path / "mutant.c"
    mutated.write_text(src.replace(old, new, 1))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp", str(mutated),
                    "-o", str(lib), "-lm"], check=True)
    env = dict(os.environ, SSCAN_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider"]
                       + [os.path.join(ROOT, "tests", f) for f in PIN_FILES],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"pins did not catch mutant {name}:\n{r.stdout[-2000:]}"
