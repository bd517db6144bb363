"""Sequence-parallel selective scan: one long sequence split in time across ranks.

The recurrence h_t = Abar_t h_{t-1} + Bbar_t x_t is affine in the state, so a
stretch of steps acts on its initial state as h -> P h + H (P = product of its
Abar, H = its end state from zero).  Each rank summarises its own stretch
(``sscan_chunk_summary``), the ranks exchange the (P, H) pairs with one
all-gather, every rank composes the summaries of the stretches before it
(``sscan_carry``), and then scans its stretch from that carried state
(``sscan_fwd``) -- the result equals one unsplit scan.  The only data crossing
ranks is 2 x (batch, D, N) fp32 per rank; all arithmetic runs in the library's
kernels.

Ranks must hold consecutive stretches in rank order (rank 0 holds the first steps).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import binding as sb


class CudaOps:
    """The three library calls the driver needs (swappable for testing the exchange)."""

    def summary(self, u, delta_raw, A, B, delta_bias, delta_softplus):
        return sb.sscan_chunk_summary(u, delta_raw, A, B, delta_bias, delta_softplus=delta_softplus)

    def carry(self, P, H, h0):
        return sb.sscan_carry(P, H, h0)

    def fwd(self, u, delta_raw, A, B, C, delta_bias, D_skip, z, h0, delta_softplus):
        return sb.sscan_fwd(u, delta_raw, A, B, C, delta_bias, D_skip, z, h0, delta_softplus=delta_softplus)


def sequence_parallel_fwd(u, delta_raw, A, B, C, delta_bias=None, D_skip=None, z=None, h0=None, *,
                          group=None, delta_softplus=True, ops=None):
    """Forward scan of this rank's stretch (batch, L_r, D) of a sequence split across the
    ranks of ``group``.  ``h0`` is the initial state of the whole sequence (used on every
    rank; NULL = zero).  Returns (out of this stretch, final state of the whole sequence)."""
    ops = ops or CudaOps()
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    P, H = ops.summary(u, delta_raw, A, B, delta_bias, delta_softplus)
    Ps = [torch.empty_like(P) for _ in range(world)]
    Hs = [torch.empty_like(H) for _ in range(world)]
    dist.all_gather(Ps, P.contiguous(), group=group)
    dist.all_gather(Hs, H.contiguous(), group=group)
    carry, h_final = ops.carry(torch.stack(Ps), torch.stack(Hs), h0)
    out = ops.fwd(u, delta_raw, A, B, C, delta_bias, D_skip, z, carry[rank].contiguous(), delta_softplus)
    return out, h_final
