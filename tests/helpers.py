"""Shared test helpers: moving seeded numpy inputs to torch and the error measures."""
import numpy as np
import torch

from selective_state_space_33_b200.workloads import to_device


def to_torch(x: dict, device) -> dict:
    """numpy inputs from workloads.make_inputs -> torch tensors (uint16 -> bfloat16 bits)."""
    return to_device(x, device)


def to_f64(t) -> np.ndarray:
    return t.detach().to(torch.float64).cpu().numpy()


def normwise(got, ref) -> float:
    """max |got - ref| / max |ref| (the tolerance form used for every tensor)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    denom = np.max(np.abs(ref)) if ref.size else 0.0
    if ref.size == 0:
        return 0.0
    err = np.max(np.abs(got - ref))
    return float(err / denom) if denom > 0 else float(err)


def pointwise(got, ref, floor: float = 1e-3) -> float:
    """max |got - ref| / |ref| over the elements with |ref| >= floor * max |ref|.

    Reported beside the normwise error: outputs gated by SiLU(z) with z near 0, or
    whose readout and skip term nearly cancel, sit close to zero, where a relative
    error says little; the floor leaves those out."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    if ref.size == 0:
        return 0.0
    a = np.abs(ref)
    keep = a >= floor * a.max()
    if not keep.any():
        return 0.0
    return float(np.max(np.abs(got[keep] - ref[keep]) / a[keep]))


TOL = {"f32": 1e-4, "bf16": 2e-2}
