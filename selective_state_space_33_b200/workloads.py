"""Seeded synthetic inputs for the selective scan, shaped like the Mamba layers the
paper evaluates (Mamba-130M and Mamba-2.8B inner widths, a million-step sequence).

This module holds no arithmetic of the scan itself: it only draws random numbers
and lays them out.  The CUDA library's tests and benchmark, and the CPU oracle's
tests, take their inputs from here so that both sides see identical values.

Recipe (numpy ``default_rng(seed)``, draws in this order, each tensor in fixed
chunks of ``_CHUNK`` elements so the stream does not depend on memory limits):
  u, delta_raw, z ~ N(0, 1), shape (batch, L, D)
  B, C            ~ N(0, 1), shape (batch, L, N), shared by all D channels
  log_dt          ~ U[ln dt_min, ln dt_max], shape (D,)
  D_skip          = 1, or ~ N(0, 1) when the workload says so, shape (D,)
  dout            ~ N(0, 1), shape (batch, L, D), only for backward workloads
  A[d, n]         = -(n + 1)                      (S4D-real initialisation), or,
                    for complex-A workloads, -1/2 + n i (complex64)
  delta_bias[d]   = log(expm1(dt_d)), the value whose softplus is dt_d, so that
                    softplus(delta_raw + bias) centres log-uniformly in
                    [dt_min, dt_max] before the N(0,1) draw spreads it.
Values are drawn in float32; bf16 workloads round them once to bfloat16
(round-to-nearest-even) and carry them as uint16 bit patterns.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

_CHUNK = 1 << 24


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    seqlen: int
    dim: int
    dstate: int
    io: str                      # "f32" or "bf16"
    dt_min: float
    dt_max: float
    dskip: str                   # "ones" or "normal"
    seed: int
    backward: bool = False
    decode: bool = False         # one-token generation steps (seqlen 1, carried state)
    gate: bool = True
    complex_a: bool = False      # A_n = -1/2 + n i (complex diagonal A)
    description: str = ""

    @property
    def elements(self) -> int:
        return self.batch * self.seqlen * self.dim

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 64, 4, 4, "f32", 1e-3, 1e-1, "ones", 0,
                     description="tiny fp32 scan, batch 1, L 64, D 4, N 4"),
    "mamba130m": Workload("mamba130m", 8, 2048, 1536, 16, "bf16", 1e-3, 1e-1, "ones", 1,
                          description="Mamba-130M-shaped layer, bf16 I/O"),
    "mamba2.8b": Workload("mamba2.8b", 8, 2048, 5120, 16, "bf16", 1e-3, 1e-1, "normal", 2,
                          description="Mamba-2.8B-shaped layer, bf16 I/O"),
    "mamba2.8b-f32": Workload("mamba2.8b-f32", 8, 2048, 5120, 16, "f32", 1e-3, 1e-1, "normal", 2,
                              description="Mamba-2.8B-shaped layer, fp32 I/O"),
    "million": Workload("million", 1, 1 << 20, 1536, 16, "bf16", 1e-4, 1e-2, "ones", 3,
                        description="million-step sequence, D 1536, bf16 I/O"),
    "bwd130m": Workload("bwd130m", 8, 2048, 1536, 16, "bf16", 1e-3, 1e-1, "ones", 4,
                        backward=True, description="backward at the Mamba-130M layer shape"),
    "decode2.8b": Workload("decode2.8b", 64, 1, 5120, 16, "bf16", 1e-3, 1e-1, "normal", 5,
                           decode=True, description="one generation step, 64 sequences, Mamba-2.8B layer width"),
    "complex130m": Workload("complex130m", 8, 2048, 1536, 16, "bf16", 1e-3, 1e-1, "ones", 6, complex_a=True,
                            description="complex A = -1/2 + n i at the Mamba-130M layer shape, bf16 I/O"),
    "complexbwd130m": Workload("complexbwd130m", 8, 2048, 1536, 16, "bf16", 1e-3, 1e-1, "ones", 7,
                               backward=True, complex_a=True,
                               description="backward with complex A = -1/2 + n i at the Mamba-130M layer shape"),
}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even); return the uint16 bit patterns."""
    bits = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = bits + (np.uint32(0x7FFF) + ((bits >> np.uint32(16)) & np.uint32(1)))
    return (rounded >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns (uint16) to float32 exactly."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal(rng: np.random.Generator, shape, io: str) -> np.ndarray:
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16 if io == "bf16" else np.float32)
    for s in range(0, n, _CHUNK):
        e = min(n, s + _CHUNK)
        v = rng.standard_normal(e - s, dtype=np.float32)
        out[s:e] = f32_to_bf16_bits(v) if io == "bf16" else v
    return out.reshape(shape)


def make_inputs(w: Workload) -> dict:
    """Draw one workload's inputs.  I/O tensors are float32 or uint16 (bf16 bits);
    A, delta_bias and D_skip are float32."""
    if w.io not in ("f32", "bf16"):
        raise ValueError(w.io)
    rng = np.random.default_rng(w.seed)
    big = (w.batch, w.seqlen, w.dim)
    small = (w.batch, w.seqlen, w.dstate)
    x = {}
    x["u"] = _normal(rng, big, w.io)
    x["delta_raw"] = _normal(rng, big, w.io)
    x["z"] = _normal(rng, big, w.io)
    x["B"] = _normal(rng, small, w.io)
    x["C"] = _normal(rng, small, w.io)
    log_dt = rng.uniform(math.log(w.dt_min), math.log(w.dt_max), size=w.dim)
    if w.dskip == "normal":
        x["D_skip"] = rng.standard_normal(w.dim, dtype=np.float32)
    else:
        x["D_skip"] = np.ones(w.dim, dtype=np.float32)
    if w.backward:
        x["dout"] = _normal(rng, big, w.io)
    dt = np.exp(log_dt)
    x["delta_bias"] = np.log(np.expm1(dt)).astype(np.float32)
    if w.complex_a:
        x["A"] = np.ascontiguousarray(np.broadcast_to(
            (-0.5 + 1j * np.arange(w.dstate)).astype(np.complex64), (w.dim, w.dstate)))
    else:
        x["A"] = np.ascontiguousarray(
            np.broadcast_to(-(np.arange(w.dstate, dtype=np.float32) + 1.0), (w.dim, w.dstate)))
    if w.decode:
        x["state"] = rng.standard_normal((w.batch, w.dim, w.dstate), dtype=np.float32)
    if not w.gate:
        del x["z"]
    return x


def small_case(batch: int, seqlen: int, dim: int, dstate: int, io: str = "f32", seed: int = 0,
               dt_min: float = 1e-3, dt_max: float = 1e-1, dskip: str = "normal",
               backward: bool = False, complex_a: bool = False) -> dict:
    """Inputs of any shape drawn with the same recipe (for tails and edge cases)."""
    return make_inputs(Workload("custom", batch, seqlen, dim, dstate, io, dt_min, dt_max,
                                dskip, seed, backward=backward, complex_a=complex_a))


def to_device(x: dict, device) -> dict:
    """Copy drawn inputs to torch tensors on ``device`` (uint16 arrays become bfloat16
    tensors with the same bits)."""
    import torch
    out = {}
    for k, v in x.items():
        t = torch.from_numpy(np.ascontiguousarray(v))
        if v.dtype == np.uint16:
            t = t.view(torch.bfloat16)
        out[k] = t.to(device)
    return out
