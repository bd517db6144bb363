"""Sequence-split scan: stretch summaries, their composition, and the rank-level
driver.  GPU tests run the library calls with the stretches emulated in one process
(the exchange is host-side, nothing waits on another rank); the CPU test runs the
driver's exchange across two gloo ranks with the fp64 oracle standing in for the
library calls."""
import os
import socket
import sys

import numpy as np
import pytest
import torch

import oracle
from selective_state_space_33_b200 import binding as sb
from selective_state_space_33_b200 import workloads as W

from .helpers import TOL, normwise, to_f64, to_torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _cut(t, s):
    return {k: (v[:, s].contiguous() if k in ("u", "delta_raw", "z", "B", "C") else v) for k, v in t.items()}


@pytest.mark.gpu
@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("cuts", [(512,), (100, 700, 1500), (1,), (2047,)])
def test_split_sequence_matches_unsplit(cuda_device, io, cuts):
    batch, L, D, N = 2, 2048, 64, 16
    x = W.small_case(batch, L, D, N, io=io, seed=sum(cuts))
    t = to_torch(x, cuda_device)
    h0 = torch.randn(batch, D, N, device=cuda_device)
    full, hl = sb.sscan_fwd(t["u"], t["delta_raw"], t["A"], t["B"], t["C"], t["delta_bias"], t["D_skip"], t["z"],
                            h0, return_last_state=True)
    bounds = [0, *cuts, L]
    parts = [_cut(t, slice(a, b)) for a, b in zip(bounds[:-1], bounds[1:])]
    sums = [sb.sscan_chunk_summary(p["u"], p["delta_raw"], p["A"], p["B"], p["delta_bias"]) for p in parts]
    carry, h_final = sb.sscan_carry(torch.stack([s[0] for s in sums]), torch.stack([s[1] for s in sums]), h0)
    outs = [sb.sscan_fwd(p["u"], p["delta_raw"], p["A"], p["B"], p["C"], p["delta_bias"], p["D_skip"], p["z"],
                         carry[k].contiguous()) for k, p in enumerate(parts)]
    torch.cuda.synchronize()
    got = torch.cat(outs, 1)
    tol = 1e-5 if io == "f32" else 1e-2
    assert normwise(to_f64(got), to_f64(full)) <= tol
    assert normwise(to_f64(h_final), to_f64(hl)) <= 1e-5
    ref, ref_h = oracle.fwd(x["u"], x["delta_raw"], x["A"], x["B"], x["C"], delta_bias=x["delta_bias"],
                            D_skip=x["D_skip"], z=x["z"], h0=h0.cpu().double().numpy())
    assert normwise(to_f64(got), ref) <= TOL[io]
    assert normwise(to_f64(h_final), ref_h) <= TOL[io]


@pytest.mark.gpu
def test_summary_of_empty_stretch_is_identity(cuda_device):
    t = to_torch(W.small_case(2, 0, 8, 4, io="f32", seed=1), cuda_device)
    P, H = sb.sscan_chunk_summary(t["u"], t["delta_raw"], t["A"], t["B"], t["delta_bias"])
    torch.cuda.synchronize()
    assert torch.all(P == 1) and torch.all(H == 0)


# ---------------------------------------------------------------- driver over gloo ranks (CPU)
class _OracleOps:
    """The driver's three calls done by the fp64 oracle on CPU tensors: the summary from
    last-state runs (H from zero; P from the same stretch with x = 0 and h0 = 1), the carry
    by composing the maps in order, the stretch by a forward run from the carry."""

    def summary(self, u, delta_raw, A, B, delta_bias, delta_softplus):
        a = dict(delta_bias=delta_bias.numpy(), delta_softplus=delta_softplus, want_out=False)
        C = np.zeros(B.shape)
        _, H = oracle.fwd(u.numpy(), delta_raw.numpy(), A.numpy(), B.numpy(), C, **a)
        one = np.ones((u.shape[0], u.shape[2], B.shape[2]))
        _, P = oracle.fwd(np.zeros(u.shape), delta_raw.numpy(), A.numpy(), B.numpy(), C, h0=one, **a)
        return torch.from_numpy(P), torch.from_numpy(H)

    def carry(self, P, H, h0):
        h = torch.zeros_like(P[0]) if h0 is None else h0.double()
        ins = []
        for k in range(P.shape[0]):
            ins.append(h)
            h = P[k] * h + H[k]
        return torch.stack(ins), h

    def fwd(self, u, delta_raw, A, B, C, delta_bias, D_skip, z, h0, delta_softplus):
        out, _ = oracle.fwd(u.numpy(), delta_raw.numpy(), A.numpy(), B.numpy(), C.numpy(),
                            delta_bias=delta_bias.numpy(), D_skip=D_skip.numpy(), z=z.numpy(),
                            h0=h0.numpy(), delta_softplus=delta_softplus)
        return torch.from_numpy(out)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    from selective_state_space_33_b200.sequence_parallel import sequence_parallel_fwd
    from tests.test_sequence_parallel import _OracleOps
    dist.init_process_group("gloo", rank=rank, world_size=world)
    x = W.small_case(1, 96, 5, 4, io="f32", seed=77)
    bounds = [0, 30, 61, 96][: world + 1] if world == 3 else [0, 40, 96]
    s = slice(bounds[rank], bounds[rank + 1])
    f = {k: torch.from_numpy(np.ascontiguousarray(x[k][:, s] if k in ("u", "delta_raw", "z", "B", "C")
                                                  else x[k]).astype(np.float64)) for k in x}
    h0 = torch.from_numpy(np.random.default_rng(3).standard_normal((1, 5, 4)))
    out, hf = sequence_parallel_fwd(f["u"], f["delta_raw"], f["A"], f["B"], f["C"], f["delta_bias"],
                                    f["D_skip"], f["z"], h0, ops=_OracleOps())
    q.put((rank, out.numpy(), hf.numpy()))
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_driver_exchange_over_gloo(world):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in ps:
        p.start()
    res = dict((r, (o, h)) for r, o, h in (q.get(timeout=300) for _ in ps))
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    x = W.small_case(1, 96, 5, 4, io="f32", seed=77)
    h0 = np.random.default_rng(3).standard_normal((1, 5, 4))
    ref, ref_h = oracle.fwd(x["u"], x["delta_raw"], x["A"], x["B"], x["C"], delta_bias=x["delta_bias"],
                            D_skip=x["D_skip"], z=x["z"], h0=h0)
    got = np.concatenate([res[r][0] for r in range(world)], axis=1)
    np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-12)
    for r in range(world):
        np.testing.assert_allclose(res[r][1], ref_h, rtol=1e-10, atol=1e-12)
