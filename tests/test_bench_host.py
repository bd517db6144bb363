"""Host-side arithmetic of bench.py (no device work): the algorithmic units behind the
roofline fractions, the whole-job aggregate, the source hashing that keys the
recorded DRAM traffic, and the CPU-baseline sampler's passes."""
import importlib.util
import os

import pytest

from selective_state_space_33_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_forward_units_at_the_2p8b_layer_shape(bench):
    # batch 8, L 2048, D 5120, N 16, bf16: u, delta_raw, z in and out back (4 x 2 bytes per
    # element), B and C (2 x 2 bytes per (b, t, n)), A (D x N) and bias, D_skip fp32 once;
    # exponentials: N for Abar plus softplus and the SiLU gate per element
    u = bench.roofline_units(W.WORKLOADS["mamba2.8b"])
    E = 8 * 2048 * 5120
    assert u["elements"] == E
    assert u["bytes"] == 8 * E + 4 * 8 * 2048 * 16 + (5120 * 16 + 2 * 5120) * 4 == 672505856
    assert u["exps"] == 18 * E == 1509949440


def test_other_workload_units(bench):
    bwd = bench.roofline_units(W.WORKLOADS["bwd130m"])
    E = 8 * 2048 * 1536
    assert bwd["exps"] == 19 * E and bwd["bytes"] == 14 * E + 8 * 8 * 2048 * 16 + 2 * (1536 * 16 + 2 * 1536) * 4
    cx = bench.roofline_units(W.WORKLOADS["complex130m"])
    assert cx["exps"] == (3 * 16 + 2) * E
    cxb = bench.roofline_units(W.WORKLOADS["complexbwd130m"])
    assert cxb["exps"] == (6 * 16 + 4) * E
    dec = W.WORKLOADS["decode2.8b"]
    ud = bench.roofline_units(dec)
    # the fp32 state read and written dominates a generation step
    assert ud["bytes"] > 2 * dec.batch * dec.dim * dec.dstate * 4


def test_aggregate_is_whole_job_throughput(bench):
    # 4 ranks x 10 steps x 1e6 elements in 2 s (the slowest rank's time)
    assert bench.aggregate(10 ** 6, 10, 4, 2.0) == pytest.approx(4 * 10 * 1e6 / 2.0 / 1e9)


def test_code_only_ignores_comments_and_blank_lines(bench):
    a = "int x = 1;  // one\n\n// a comment line\nint y = 2;\n"
    b = "int x = 1;\nint y = 2;   \n"
    assert bench.code_only(a) == bench.code_only(b) == "int x = 1;\nint y = 2;"
    # a // inside a string literal is code
    assert bench.code_only('const char* s = "a//b";') == 'const char* s = "a//b";'
    assert bench.code_only("int x = 1;") != bench.code_only("int x = 2;")


def test_cpu_sampler_repeats_a_quick_workload(bench):
    w = W.Workload("tiny", 1, 64, 8, 4, "f32", 1e-3, 1e-1, "ones", 5)
    x = W.make_inputs(w)
    rate, threads, rows, secs, passes = bench.cpu_oracle_rate(x, w, 0.2, with_passes=True)
    assert rows == w.batch * w.dim and passes > 1 and rate > 0 and threads >= 1
    assert secs > 0.05


def _parity_case(complex_a):
    import dataclasses
    base = W.WORKLOADS["complex130m" if complex_a else "mamba130m"]
    return dataclasses.replace(base, batch=2, seqlen=40, dim=72, io="f32")


@pytest.mark.parametrize("complex_a", [False, True])
def test_parity_helpers_reproduce_the_oracle_and_catch_a_bad_row(bench, complex_a):
    # The bench's parity record compares the timed output with the oracle on a row sample
    # covering every 32-channel block.  Given the oracle's own full output (as fp32), both
    # helpers report errors at fp32 rounding; a mistake planted in one sampled row (one
    # channel of one batch row, the whole sequence) must fail the tolerance.
    import numpy as np
    import torch

    import oracle
    w = _parity_case(complex_a)
    x = W.make_inputs(w)
    kw = dict(delta_bias=x["delta_bias"], D_skip=x["D_skip"], z=x.get("z"))
    if complex_a:
        ref, _ = oracle.fwd_complex(x["u"], x["delta_raw"], x["A"], x["B"], x["C"], **kw)
        check = bench.complex_oracle_parity
    else:
        ref, _ = oracle.fwd(x["u"], x["delta_raw"], x["A"], x["B"], x["C"], **kw)
        check = bench.oracle_parity
    out = torch.from_numpy(ref.astype(np.float32))
    good = check(x, w, out)
    assert good["ok"] and good["normwise"] < 1e-6, good
    rows = bench.block_rows(w, 2, 77)
    assert np.unique(rows % w.dim // 32).size == (w.dim + 31) // 32  # every channel block sampled
    r = int(rows[len(rows) // 2])
    bad_out = out.clone()
    bad_out[r // w.dim, :, r % w.dim] += 0.01 * float(np.abs(ref).max())
    bad = check(x, w, bad_out)
    assert not bad["ok"] and bad["normwise"] > 1e-4, bad
