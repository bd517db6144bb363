"""sscan_step (one generation step) against the fp64 oracle: a single step is the
forward scan with L = 1 and h0 = the carried state; repeated steps must match
one forward pass over the same tokens."""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_33_b200 import binding as sb
from selective_state_space_33_b200 import workloads as W

from .helpers import TOL, normwise, to_f64, to_torch

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [(4, 257, 16), (3, 64, 8), (2, 33, 5), (5, 40, 1), (64, 5120, 16), (3, 50, 4),
                                   (2, 1000, 16), (1, 7, 12)])
def test_single_step_matches_oracle(cuda_device, io, shape):
    batch, D, N = shape
    x = W.small_case(batch, 1, D, N, io=io, seed=batch * D + N)
    h0 = np.random.default_rng(N).standard_normal((batch, D, N)).astype(np.float32)
    t = to_torch(x, cuda_device)
    state = torch.from_numpy(h0).to(cuda_device)
    out = sb.sscan_step(t["u"][:, 0].contiguous(), t["delta_raw"][:, 0].contiguous(), t["A"],
                        t["B"][:, 0].contiguous(), t["C"][:, 0].contiguous(), state, t["delta_bias"],
                        t["D_skip"], t["z"][:, 0].contiguous())
    torch.cuda.synchronize()
    ref, ref_h = oracle.fwd(x["u"], x["delta_raw"], x["A"], x["B"], x["C"], delta_bias=x["delta_bias"],
                            D_skip=x["D_skip"], z=x["z"], h0=h0.astype(np.float64))
    assert normwise(to_f64(out), ref[:, 0]) <= TOL[io]
    assert normwise(to_f64(state), ref_h) <= 1e-5   # the state stays fp32


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_repeated_steps_match_forward(cuda_device, io):
    batch, L, D, N = 2, 64, 96, 16
    x = W.small_case(batch, L, D, N, io=io, seed=7)
    t = to_torch(x, cuda_device)
    full, hl = sb.sscan_fwd(t["u"], t["delta_raw"], t["A"], t["B"], t["C"], t["delta_bias"], t["D_skip"], t["z"],
                            return_last_state=True)
    state = torch.zeros(batch, D, N, device=cuda_device)
    outs = []
    for s in range(L):
        outs.append(sb.sscan_step(t["u"][:, s].contiguous(), t["delta_raw"][:, s].contiguous(), t["A"],
                                  t["B"][:, s].contiguous(), t["C"][:, s].contiguous(), state, t["delta_bias"],
                                  t["D_skip"], t["z"][:, s].contiguous()))
    torch.cuda.synchronize()
    steps = torch.stack(outs, 1)
    assert normwise(to_f64(steps), to_f64(full)) <= (1e-5 if io == "f32" else 1e-2)
    assert normwise(to_f64(state), to_f64(hl)) <= 1e-5


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_unaligned_state_takes_general_kernel(cuda_device, io):
    """A state buffer off a 16-byte boundary sends N = 16 down the one-thread-per-row
    kernel instead of the 4-states-per-lane one; both must match the oracle."""
    batch, D, N = 3, 200, 16
    x = W.small_case(batch, 1, D, N, io=io, seed=11)
    h0 = np.random.default_rng(12).standard_normal((batch, D, N)).astype(np.float32)
    t = to_torch(x, cuda_device)
    buf = torch.empty(batch * D * N + 1, device=cuda_device)
    state = buf[1:].view(batch, D, N)
    state.copy_(torch.from_numpy(h0).to(cuda_device))
    out = sb.sscan_step(t["u"][:, 0].contiguous(), t["delta_raw"][:, 0].contiguous(), t["A"],
                        t["B"][:, 0].contiguous(), t["C"][:, 0].contiguous(), state, t["delta_bias"],
                        t["D_skip"], t["z"][:, 0].contiguous())
    torch.cuda.synchronize()
    ref, ref_h = oracle.fwd(x["u"], x["delta_raw"], x["A"], x["B"], x["C"], delta_bias=x["delta_bias"],
                            D_skip=x["D_skip"], z=x["z"], h0=h0.astype(np.float64))
    assert normwise(to_f64(out), ref[:, 0]) <= TOL[io]
    assert normwise(to_f64(state), ref_h) <= 1e-5


def test_step_with_no_batch_or_channels(cuda_device):
    """batch 0 or D 0: nothing to do, an empty output and no error."""
    for batch, D, N in ((0, 64, 16), (3, 0, 16)):
        x = W.small_case(batch, 1, D, N, io="f32", seed=9)
        t = to_torch(x, cuda_device)
        state = torch.zeros(batch, D, N, device=cuda_device)
        out = sb.sscan_step(t["u"][:, 0].contiguous(), t["delta_raw"][:, 0].contiguous(), t["A"],
                            t["B"][:, 0].contiguous(), t["C"][:, 0].contiguous(), state, t["delta_bias"],
                            t["D_skip"], t["z"][:, 0].contiguous())
        torch.cuda.synchronize()
        assert out.numel() == 0
