"""The forward kernels choose their tile length from the grid size (64-step tiles when the
whole grid fits the GPU at once with them, else 32).  The tile length only moves the
barriers and copies between tiles, not the arithmetic of any element, so a batch row must
come out bit-identical from a grid large enough for 32-step tiles and from a grid of that
row alone (64-step tiles)."""
import numpy as np
import pytest
import torch

from selective_state_space_33_b200 import binding as sb
from selective_state_space_33_b200 import workloads as W

from .helpers import to_torch

pytestmark = pytest.mark.gpu


def _slice_batch(t: dict, b: int) -> dict:
    out = {}
    for k, v in t.items():
        if torch.is_tensor(v) and v.dim() == 3:
            out[k] = v[b:b + 1].contiguous()
        else:
            out[k] = v
    return out


@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_real_forward_same_result_for_either_tile_length(cuda_device, io):
    # batch 8, D 5120: 1280 CTAs -> 32-step tiles; one batch row alone: 160 CTAs -> 64-step tiles
    x = W.small_case(8, 300, 5120, 16, io=io, seed=91)
    t = to_torch(x, cuda_device)
    big, _ = sb.sscan_fwd(t["u"], t["delta_raw"], t["A"], t["B"], t["C"], t["delta_bias"], t["D_skip"], t["z"],
                          return_last_state=True)
    for b in (0, 5):
        s = _slice_batch(t, b)
        one, _ = sb.sscan_fwd(s["u"], s["delta_raw"], s["A"], s["B"], s["C"], s["delta_bias"], s["D_skip"], s["z"],
                              return_last_state=True)
        torch.cuda.synchronize()
        assert torch.equal(big[b:b + 1], one), (io, b)


def test_complex_forward_same_result_for_either_tile_length(cuda_device):
    # batch 12, D 1536, N 16: 1152 CTAs of 2 complex states per lane -> 32-step tiles; one
    # batch row alone -> 64-step tiles (the same lane geometry: the 4-state one would take
    # over only from 592 four-state CTAs, i.e. batch 13)
    x = W.small_case(12, 200, 1536, 16, io="bf16", seed=93, complex_a=True)
    t = to_torch(x, cuda_device)
    A = torch.from_numpy(np.ascontiguousarray(x["A"].astype(np.complex64))).to(cuda_device)
    big = sb.sscan_fwd_complex(t["u"], t["delta_raw"], A, t["B"], t["C"], t["delta_bias"], t["D_skip"], t.get("z"))
    s = _slice_batch(t, 3)
    one = sb.sscan_fwd_complex(s["u"], s["delta_raw"], A, s["B"], s["C"], s["delta_bias"], s["D_skip"], s.get("z"))
    torch.cuda.synchronize()
    assert torch.equal(big[3:4], one)
