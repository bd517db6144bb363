"""Failure reporting without a fault: every wait in the library's kernels is
bounded, and a wait that runs out sets a device status bit that the host reads.
The probe waits on a shared-memory barrier that nothing arrives on (a flag that
nothing sets), so its wait runs out on purpose; the context must stay usable."""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_33_b200 import binding as sb
from selective_state_space_33_b200 import workloads as W

from .helpers import TOL, normwise, to_f64, to_torch

@pytest.mark.gpu
def test_bounded_wait_reports_timeout_and_context_survives(cuda_device):
    sb.device_status(clear=True)
    assert sb.device_status() == 0
    sb.probe_wait_timeout(4096)
    flags = sb.device_status(clear=True)
    assert flags & 4, flags
    assert sb.device_status() == 0
    # the context is still usable: a forward call right after matches the oracle
    x = W.small_case(2, 100, 64, 16, io="f32", seed=123)
    t = to_torch(x, cuda_device)
    out = sb.sscan_fwd(t["u"], t["delta_raw"], t["A"], t["B"], t["C"], t["delta_bias"], t["D_skip"], t["z"])
    torch.cuda.synchronize()
    ref, _ = oracle.fwd(x["u"], x["delta_raw"], x["A"], x["B"], x["C"], delta_bias=x["delta_bias"],
                        D_skip=x["D_skip"], z=x["z"])
    assert normwise(to_f64(out), ref) <= TOL["f32"]
    assert sb.device_status() == 0


def test_probe_rejects_bad_poll_counts():
    """Checked on the host before any launch (no GPU needed)."""
    lib = sb.load_library()
    for polls in (0, (1 << 20) + 1):
        assert lib.sscan_probe_wait_timeout(polls, None) == 1  # SSCAN_ERR_INVALID_ARG
