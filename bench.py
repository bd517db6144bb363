#!/usr/bin/env python
"""Selective-scan forward benchmark on B200: Gelem/s (elements = batch*L*D) and the
achieved fraction of the HBM / MUFU roofline at the Mamba-2.8B layer shape
(batch 8, L 2048, D 5120, N 16, bf16 I/O, fp32 state), on seeded synthetic inputs.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One process per GPU (torchrun for N > 1).  Each rank runs its own replica of the
workload (the scan has no cross-rank step), so per-GPU work is fixed: weak scaling.
Rank 0 prints one JSON line.  ``--impl reference`` times the fp64 CPU oracle on the
host cores instead (the reference arm: a plain sequential scan, never tuned).
"""
from __future__ import annotations

import argparse
import ctypes
import json
import math
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from selective_state_space_33_b200 import workloads as W  # noqa: E402

METRIC = "selective-scan fwd Gelem/s (B·L·D) & % of HBM/MUFU roofline at 2.8B-layer shape"
METRIC_FWD = "selective-scan fwd Gelem/s (B·L·D)"
METRIC_BWD = "selective-scan bwd Gelem/s (B·L·D), states recomputed on chip"
METRIC_STEP = "selective-scan generation step Gelem/s (batch·D per token), state read and written in HBM"
METRIC_COMPLEX = "selective-scan fwd with complex diagonal A, Gelem/s (B·L·D)"
METRIC_COMPLEX_BWD = "selective-scan bwd with complex diagonal A, Gelem/s (B·L·D), states recomputed on chip"
UNIT = "Gelem/s"
DEFAULT_WORKLOAD = "mamba2.8b"
SM_COUNT = 148
MUFU_PER_SM_CLK = 16          # ex2 results per SM per clock (4 per sub-partition)
HBM_FALLBACK_GBS = 6650.0     # used only when MEASURED_PEAKS.json is absent
HBM_NOMINAL_GBS = 7700.0      # B200 HBM3e nominal (HGX figure), for context


# ----------------------------------------------------------------------------- ranks
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(backend: str):
    import datetime

    import torch.distributed as dist
    world, rank, _ = dist_env()
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def reduce_max(value: float, device=None) -> float:
    """Max of a scalar over all ranks (the step time every rank waits for)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(elements_per_rank_step: int, steps: int, world: int, max_seconds: float) -> float:
    """Whole-job throughput in Gelem/s: every rank's elements over the slowest rank's time."""
    return elements_per_rank_step * steps * world / max_seconds / 1e9


# ----------------------------------------------------------------------------- model
def roofline_units(w: W.Workload) -> dict:
    """Algorithmic bytes and exponentials of one forward pass.

    bytes: read u, delta_raw, z and write out (4 * E * s), read B and C
    (2 * batch * L * N * s), read A, bias, D_skip once (fp32); the (batch, L, D, N)
    state is never moved (the method keeps it on chip).
    exps: N per element for Abar = exp(delta A), plus one for softplus and one for
    the SiLU gate (Bbar reuses Abar's exponential)."""
    s = 2 if w.io == "bf16" else 4
    E = w.batch * w.seqlen * w.dim
    BLN = w.batch * w.seqlen * w.dstate
    if w.complex_a and w.backward:
        # complex backward: read u, delta_raw, z, dout, B, C; write du, ddelta_raw, dz and
        # dB, dC; the checkpoint pass and the reverse kernel each take 2^x, cos and sin
        # per state (the recomputation and the reverse step): 2 x 3 N + 4 MUFU operations.
        bytes_ = 7 * E * s + 4 * BLN * s + 2 * (2 * w.dim * w.dstate + 2 * w.dim) * 4
        return {"elements": E, "bytes": bytes_, "exps": E * (6 * w.dstate + 4)}
    if w.complex_a:
        # complex A: the same bytes (A is (D, N, 2) fp32); per state the MUFU computes
        # 2^(delta Re a), cos and sin of delta Im a: 3 N + 2 MUFU operations per element.
        bytes_ = 4 * E * s + 2 * BLN * s + (2 * w.dim * w.dstate + 2 * w.dim) * 4
        return {"elements": E, "bytes": bytes_, "exps": E * (3 * w.dstate + 2)}
    if w.decode:
        # one token: read and write the fp32 state (the dominant term), read u, delta_raw,
        # z and write out (batch, D), read B, C (batch, N) and the parameters.
        bytes_ = 2 * w.batch * w.dim * w.dstate * 4 + 4 * E * s + 2 * BLN * s + (w.dim * w.dstate + 2 * w.dim) * 4
        return {"elements": E, "bytes": bytes_, "exps": E * (w.dstate + 2)}
    if w.backward:
        # read u, delta_raw, z, dout, write du, ddelta_raw, dz; read B, C, write dB, dC;
        # A, bias, D_skip in and their gradients out.  Exponentials: Abar once per state
        # (recomputed on chip), softplus, the gate's sigmoid, softplus' derivative.
        bytes_ = 7 * E * s + 4 * BLN * s + 2 * (w.dim * w.dstate + 2 * w.dim) * 4
        return {"elements": E, "bytes": bytes_, "exps": E * (w.dstate + 3)}
    bytes_ = 4 * E * s + 2 * BLN * s + (w.dim * w.dstate + 2 * w.dim) * 4
    return {"elements": E, "bytes": bytes_, "exps": E * (w.dstate + 2)}


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of each
# workload's dominant kernel, read from one ncu capture of that workload (summaries
# under profiles/).  A figure holds only for the kernel source it was taken on: it is
# keyed by the SHA-256 of those source files (with comments and blank lines removed,
# so that only code counts) and reported as null once the code changes.
NCU_TRAFFIC = {
    "mamba2.8b": {"kernel": "fwd_tiled_kernel", "bytes": 506067200 + 151426048,
        "sources": ('sscan_tiled.cu', 'sscan_act.cuh', 'sscan_tma.cuh', 'sscan_math.cuh', 'sscan_check.cuh', 'sscan_plan.h'), "sha256": "519275463ead877d",
        "profile": "profiles/fwd_tiled_kernel_mamba2.8b_bf16.md"},
    "bwd130m": {"kernel": "bwd_tiled_kernel", "bytes": 410449408 + 133641984,
        "sources": ('sscan_bwd_tiled.cu', 'sscan_tma.cuh', 'sscan_math.cuh', 'sscan_check.cuh'), "sha256": "5a0552a6bbd9fdb2",
        "profile": "profiles/bwd_tiled_kernel_bwd130m_bf16.md"},
    "decode2.8b": {"kernel": "step_quad_kernel", "bytes": 23317760 + 0,
        "sources": ('sscan_step.cu', 'sscan_math.cuh'), "sha256": "c1a451e4bc5a2b5e",
        "profile": "profiles/step_quad_kernel_decode2.8b_bf16.md"},
    "complex130m": {"kernel": "fwd_complex_kernel", "bytes": 152524288 + 34057216,
        "sources": ('sscan_complex.cu', 'sscan_act.cuh', 'sscan_complex_math.cuh', 'sscan_math.cuh', 'sscan_tma.cuh', 'sscan_plan.h'), "sha256": "ba36ed06671d95dd",
        "profile": "profiles/fwd_complex_kernel_complex130m_bf16.md"},
    "complexbwd130m": {"kernel": "bwd_complex_kernel", "bytes": 614995968 + 141339136,
        "sources": ('sscan_complex_bwd.cu', 'sscan_complex_math.cuh', 'sscan_math.cuh'), "sha256": "4e5bc25eb2db58a4",
        "profile": "profiles/bwd_complex_kernel_complexbwd130m_bf16.md"},
}


def ncu_traffic(workload: str):
    """The recorded per-launch DRAM traffic of the workload's dominant kernel, or None
    when none was recorded or the kernel's sources changed since the capture."""
    import hashlib
    rec = NCU_TRAFFIC.get(workload)
    if rec is None:
        return None
    h = hashlib.sha256()
    for name in rec["sources"]:
        path = os.path.join(ROOT, "selective_state_space_33_b200", "csrc", name)
        if not os.path.exists(path):
            return None
        with open(path) as f:
            h.update(code_only(f.read()).encode())
    return rec["bytes"] if h.hexdigest()[:16] == rec["sha256"] else None


def code_only(src: str) -> str:
    """C++/CUDA source without // comments, trailing spaces and blank lines."""
    lines = []
    for line in src.splitlines():
        cut = line.find("//")
        if cut >= 0 and line.count('"', 0, cut) % 2 == 0:
            line = line[:cut]
        line = line.rstrip()
        if line:
            lines.append(line)
    return "\n".join(lines)


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f)
    return {}


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples this GPU's SM clock and clock-event (throttle) reasons through NVML
    every 10 ms on a host thread; read-only.  ``mark()`` brackets the timed region
    so the summary uses the samples taken during it (plus a short busy tail when
    the region is shorter than a few sample periods)."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, uuid: str, period_s: float = 0.01):
        self.uuid, self.period = uuid, period_s
        self.samples = []          # (host time, sm MHz, max MHz, reasons mask)
        self.marks = []
        self._stop = None
        self._thread = None
        self.error = None

    def start(self):
        import threading
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = nv.nvmlDeviceGetHandleByUUID(self.uuid) if self.uuid else nv.nvmlDeviceGetHandleByIndex(0)
            getr = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons
        except Exception as e:  # NVML missing: report no clocks rather than guess
            self.error = f"nvml unavailable: {e}"
            return
        self._stop = threading.Event()

        def loop():
            while not self._stop.is_set():
                try:
                    sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                    mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
                    rs = getr(h)
                    self.samples.append((time.perf_counter(), sm, mx, rs))
                except Exception as e:
                    self.error = str(e)
                self._stop.wait(self.period)

        self._thread = threading.Thread(target=loop, daemon=True)
        self._thread.start()

    def mark(self):
        self.marks.append(time.perf_counter())

    def stop(self) -> dict:
        if self._thread is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [self.error or "no samples"]}
        self._stop.set()
        self._thread.join(timeout=2)
        t0, t1 = (self.marks[0], self.marks[-1]) if len(self.marks) >= 2 else (0.0, float("inf"))
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        if len(inside) < 5:  # short region: add the busy tail that follows it
            inside = [s for s in self.samples if s[0] >= t0]
        mask = 0
        for s in inside:
            mask |= int(s[3])
        reasons = sorted(name for bit, name in self.REASONS.items() if mask & bit)
        return {"sm_mhz": statistics.median([s[1] for s in inside]) if inside else None,
                "sm_max_mhz": max(s[2] for s in inside) if inside else None,
                "reasons": reasons, "samples": len(inside)}


# ----------------------------------------------------------------------------- CPU arms
def cpu_oracle_rate(x: dict, w: W.Workload, target_s: float, seed: int = 0, with_passes: bool = False):
    """Time the fp64 oracle on a random sample of (batch, channel) rows, each the full
    sequence; the sample is sized for about ``target_s`` seconds, and when even every
    row takes well under that, the whole workload is run several times (passes).
    Returns (Gelem/s, threads, rows, seconds), plus the pass count if ``with_passes``."""
    import oracle
    threads = oracle.set_threads(0)
    rng = np.random.default_rng(seed)
    total_rows = w.batch * w.dim

    def run(k):
        rows = np.sort(rng.choice(total_rows, size=k, replace=False))
        t0 = time.perf_counter()
        oracle.fwd(x["u"], x["delta_raw"], x["A"], x["B"], x["C"], delta_bias=x["delta_bias"],
                   D_skip=x["D_skip"], z=x.get("z"), rows=rows)
        return time.perf_counter() - t0

    k0 = min(total_rows, 8 * threads)
    dt0 = run(k0)
    k = int(min(total_rows, max(k0, k0 * target_s / max(dt0, 1e-6))))
    dt = run(k)
    if dt < target_s / 3 and k < total_rows:  # the small first sample mis-sized it: once more
        k = int(min(total_rows, max(k, k * target_s / max(dt, 1e-6))))
        dt = run(k)
    passes = 1
    if k == total_rows and dt < target_s / 2:  # the whole workload is quick: repeat it
        passes = int(math.ceil(target_s / max(dt, 1e-6)))
        dt = sum(run(k) for _ in range(passes))
    rate = passes * k * w.seqlen / dt / 1e9
    return (rate, threads, k, dt, passes) if with_passes else (rate, threads, k, dt)


def cpu_oracle_rate_1thread(x: dict, w: W.Workload, target_s: float = 2.0, seed: int = 1):
    """The same oracle on one host thread, for scale (Gelem/s, rows, seconds, passes)."""
    import oracle
    threads = oracle.set_threads(0)
    oracle.set_threads(1)
    try:
        rate, _, rows, secs, passes = cpu_oracle_rate(x, w, target_s, seed, with_passes=True)
    finally:
        oracle.set_threads(threads)
    return rate, rows, secs, passes


def block_rows(w: W.Workload, per_block: int, seed: int, dc: int = 32) -> np.ndarray:
    """(batch, channel) rows covering every block of ``dc`` consecutive channels (the
    tiled kernel's CTA width at N = 16): ``per_block`` random channels of each block,
    each in a random batch."""
    rng = np.random.default_rng(seed)
    rows = []
    for c0 in range(0, w.dim, dc):
        width = min(dc, w.dim - c0)
        ch = c0 + rng.choice(width, size=min(per_block, width), replace=False)
        rows.extend(rng.integers(0, w.batch, size=ch.size) * w.dim + ch)
    return np.unique(np.asarray(rows, np.int64))


def error_measures(got: np.ndarray, ref: np.ndarray, floor: float = 1e-3) -> dict:
    """Normwise max|got - ref| / max|ref|, and the pointwise max |got - ref| / |ref| over
    the elements with |ref| >= floor * max|ref|."""
    a = np.abs(ref)
    mx = float(a.max()) if a.size else 0.0
    err = np.abs(got - ref)
    keep = a >= floor * mx
    return {"normwise": float(err.max() / mx) if mx > 0 else float(err.max(initial=0.0)),
            "pointwise": float((err[keep] / a[keep]).max()) if keep.any() else 0.0}


def oracle_parity(x: dict, w: W.Workload, out, per_block: int = 2, seed: int = 77) -> dict:
    """The timed run's own output against the fp64 oracle on a row sample that covers
    every channel block (``per_block`` rows per 32-channel block, each a whole
    sequence)."""
    import oracle
    import torch
    rows = block_rows(w, per_block, seed)
    b = torch.as_tensor(rows // w.dim, device=out.device)
    d = torch.as_tensor(rows % w.dim, device=out.device)
    got = out[b, :, d].double().cpu().numpy()
    ref, _ = oracle.fwd(x["u"], x["delta_raw"], x["A"], x["B"], x["C"], delta_bias=x["delta_bias"],
                        D_skip=x["D_skip"], z=x.get("z"), rows=rows)
    tol = 2e-2 if w.io == "bf16" else 1e-4
    m = error_measures(got, ref)
    return {**m, "tolerance_normwise": tol, "ok": bool(m["normwise"] <= tol),
            "sample": f"{rows.size} rows ({per_block} per 32-channel block, every block) x L={w.seqlen}"}


def complex_oracle_parity(x: dict, w: W.Workload, out, per_block: int = 2, seed: int = 77) -> dict:
    """oracle_parity for the complex-A forward: the sampled rows' channels of each batch
    form a sub-problem of the fp64 complex oracle (channels are independent)."""
    import oracle
    import torch
    rows = block_rows(w, per_block, seed)
    got, ref = [], []
    for b in np.unique(rows // w.dim):
        ds = np.sort(rows[rows // w.dim == b] % w.dim)

        def sub(a):
            return None if a is None else np.ascontiguousarray(a[b:b + 1][:, :, ds])
        r, _ = oracle.fwd_complex(sub(x["u"]), sub(x["delta_raw"]), x["A"][ds], x["B"][b:b + 1], x["C"][b:b + 1],
                                  delta_bias=x["delta_bias"][ds], D_skip=x["D_skip"][ds], z=sub(x.get("z")))
        ref.append(r[0].T)
        got.append(out[int(b), :, torch.as_tensor(ds, device=out.device)].double().cpu().numpy().T)
    got, ref = np.concatenate(got), np.concatenate(ref)
    tol = 2e-2 if w.io == "bf16" else 1e-4
    m = error_measures(got, ref)
    return {**m, "tolerance_normwise": tol, "ok": bool(m["normwise"] <= tol),
            "sample": f"{rows.size} rows ({per_block} per 32-channel block, every block) x L={w.seqlen}"}


def reference_arm(args, w: W.Workload):
    """The oracle as it stands, timed on the host cores: K timed steps (after W
    warm-up steps), each a bounded random sample of the workload's rows."""
    world, rank, _ = dist_env()
    if rank != 0:
        return
    import oracle
    x = W.make_inputs(w)
    threads = oracle.set_threads(0)
    total_rows = w.batch * w.dim
    rng = np.random.default_rng(1234)
    rate0, _, _, _ = cpu_oracle_rate(x, w, 2.0)
    per_step_rows = int(min(total_rows, max(threads, rate0 * 1e9 * 2.0 / w.seqlen)))  # ~2 s per step

    def step():
        rows = np.sort(rng.choice(total_rows, size=per_step_rows, replace=False))
        oracle.fwd(x["u"], x["delta_raw"], x["A"], x["B"], x["C"], delta_bias=x["delta_bias"],
                   D_skip=x["D_skip"], z=x.get("z"), rows=rows)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = per_step_rows * w.seqlen * args.steps / dt / 1e9
    sample = f"{per_step_rows} random rows x L={w.seqlen} per step ({per_step_rows * w.seqlen} elements)"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def workload_config(w: W.Workload, world: int, l2: str = "inputs larger than L2 (no flush needed)") -> dict:
    return {"workload": f"{w.name}: {w.description}", "batch": w.batch, "seq_len": w.seqlen,
            "d_inner": w.dim, "d_state": w.dstate, "io_dtype": w.io, "state_dtype": "f32",
            "global_batch": w.batch * world, "parallelism": f"replicas x{world}", "l2": l2}


# ----------------------------------------------------------------------------- GPU arm
def ex2_probe(torch, lib, device, repeats=5):
    """Measured MUFU ex2 rate (exps/s) of the whole GPU."""
    blocks, threads, iters = SM_COUNT * 8, 256, 4096
    sink = torch.empty(blocks * threads, dtype=torch.float32, device=device)
    st = torch.cuda.current_stream()
    lib.sscan_probe_ex2.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]
    lib.sscan_probe_ex2.restype = ctypes.c_int
    best = None
    for _ in range(repeats):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        rc = lib.sscan_probe_ex2(ctypes.c_void_p(sink.data_ptr()), iters, blocks, threads,
                                 ctypes.c_void_p(st.cuda_stream))
        b.record(st)
        if rc != 0:
            return None
        b.synchronize()
        ms = a.elapsed_time(b)
        best = ms if best is None else min(best, ms)
    return blocks * threads * 8 * iters / (best * 1e-3)


def gpu_arm(args, w: W.Workload):
    import torch

    from selective_state_space_33_b200 import binding as sb
    world, rank = init_dist("nccl" if int(os.environ.get("WORLD_SIZE", "1")) > 1 else "gloo")
    _, _, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    lib = sb.load_library()

    x = W.make_inputs(w.with_(seed=w.seed + rank)) if world > 1 else W.make_inputs(w)
    t = W.to_device(x, dev)
    out = torch.empty_like(t["u"])
    prob = sb.make_problem(w.batch, w.seqlen, w.dim, w.dstate, sb.SSCAN_BF16 if w.io == "bf16" else sb.SSCAN_F32)
    op = (sb.SSCAN_OP_BWD_COMPLEX if w.backward and w.complex_a else sb.SSCAN_OP_BWD if w.backward
          else sb.SSCAN_OP_FWD)
    ws_bytes = sb.sscan_workspace_size(prob, op)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    st = torch.cuda.current_stream()
    grads = None
    if w.backward and not w.complex_a:
        grads = sb.sscan_bwd(t["u"], t["delta_raw"], t["A"], t["B"], t["C"], t["dout"], t["delta_bias"],
                             t["D_skip"], t.get("z"), workspace=ws)

    l2_note = "inputs larger than L2 (no flush needed)"
    if w.decode:
        # One step's tensors (about 45 MB at the 2.8B width) fit in the 126 MB L2, so
        # consecutive steps rotate over enough independent sets (state, activations,
        # parameters: like the layers of a model) that together exceed L2 three times;
        # each step then reads its state from HBM, not from the last step's L2 lines.
        sq0 = {k: (v[:, 0].contiguous() if k in ("u", "delta_raw", "z", "B", "C") else v)
               for k, v in t.items() if torch.is_tensor(v)}
        set_bytes = sum(v.numel() * v.element_size() for v in sq0.values()) + sq0["u"].numel() * sq0["u"].element_size()
        l2_bytes = int(getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 126 << 20))
        nsets = max(1, -(-3 * l2_bytes // set_bytes))
        sets = [sq0] + [{k: v.clone() for k, v in sq0.items()} for _ in range(nsets - 1)]
        outs = [torch.empty_like(sq0["u"]) for _ in range(nsets)]
        l2_note = (f"{nsets} rotating sets of {set_bytes / 1e6:.1f} MB, one per step "
                   f"({nsets * set_bytes / 1e6:.0f} MB > {l2_bytes / 1e6:.0f} MB L2)")
    nstep = [0]

    def step(stream=st):
        if w.complex_a and w.backward:
            sb.sscan_bwd_complex(t["u"], t["delta_raw"], t["A"], t["B"], t["C"], t["dout"], t["delta_bias"],
                                 t["D_skip"], t.get("z"), workspace=ws, stream=stream)
        elif w.complex_a:
            sb.sscan_fwd_complex(t["u"], t["delta_raw"], t["A"], t["B"], t["C"], t["delta_bias"], t["D_skip"],
                                 t.get("z"), out=out, stream=stream)
        elif w.decode:
            i = nstep[0] % nsets
            nstep[0] += 1
            sq = sets[i]
            sb.sscan_step(sq["u"], sq["delta_raw"], sq["A"], sq["B"], sq["C"], sq["state"], sq["delta_bias"],
                          sq["D_skip"], sq.get("z"), out=outs[i], stream=stream)
        elif w.backward:
            sb.sscan_bwd(t["u"], t["delta_raw"], t["A"], t["B"], t["C"], t["dout"], t["delta_bias"], t["D_skip"],
                         t.get("z"), grads=grads, workspace=ws, stream=stream)
        else:
            sb.sscan_fwd(t["u"], t["delta_raw"], t["A"], t["B"], t["C"], t["delta_bias"], t["D_skip"], t.get("z"),
                         out=out, workspace=ws, stream=stream)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    lib.sscan_last_launch_count.restype = ctypes.c_int
    launches_per_step = int(lib.sscan_last_launch_count())  # kernels one step enqueues

    uuid = ""
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    clocks = ClockSampler(uuid)
    clocks.start()
    time.sleep(0.05)
    graph = None
    if w.decode:
        # A generation step is a few microseconds of device work, less than the host
        # takes to marshal one call, so the K steps are captured once into a CUDA graph
        # and replayed as one launch: the timed region is K back-to-back state updates
        # (the state advancing in place), as a graph-captured decode loop runs them.
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            cs = torch.cuda.current_stream()
            for _ in range(args.steps):
                step(cs)
        for _ in range(max(args.warmup, 3)):
            graph.replay()
        torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    clocks.mark()
    if graph is not None:
        starts[0].record(st)
        graph.replay()
        ends[-1].record(st)
    else:
        for i in range(args.steps):
            starts[i].record(st)
            step()
            ends[i].record(st)
    torch.cuda.synchronize()
    clocks.mark()
    barrier()
    if not args.profile_run:
        # a short busy tail so that a brief timed region still has clock samples under load
        tail = min(2000, max(1, int(0.3 / max(starts[0].elapsed_time(ends[-1]) * 1e-3 / args.steps, 1e-5))))
        for _ in range(tail):
            step()
        torch.cuda.synchronize()
    clk = clocks.stop()
    total_s = starts[0].elapsed_time(ends[-1]) * 1e-3
    if graph is not None:
        per_launch_ms = [total_s * 1e3 / args.steps]
    else:
        per_launch_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    max_s = reduce_max(total_s, dev if world > 1 else None)
    units = roofline_units(w)
    value = aggregate(units["elements"], args.steps, world, max_s)

    if args.profile_run:
        if rank == 0:
            print(json.dumps({"profile_run": True, "workload": w.name, "value": value, "unit": UNIT,
                              "per_launch_ms": statistics.mean(per_launch_ms)}), flush=True)
        return
    if w.backward or w.decode or w.complex_a:
        e2e_value, h2d, d2h = None, 0, 0
    else:
        e2e_value, h2d, d2h = e2e_leg(args, t, out, ws, st, units, world, dev)
    if rank != 0:
        return
    secondary, others = None, None
    if world == 1 and args.workload == DEFAULT_WORKLOAD and not args.no_secondary:
        del t
        secondary = fp32_record(args, lib, dev)
        others = [other_record(args, W.WORKLOADS[name])
                  for name in ("mamba130m", "bwd130m", "complex130m", "complexbwd130m", "million")]
    finish(args, w, x, lib, dev, torch, units, value, max_s, per_launch_ms, clk, e2e_value, h2d, d2h,
           launches_per_step, world, l2_note, out=out if not (w.backward or w.decode or w.complex_a) else None,
           secondary=secondary, others=others)


def other_record(args, w: W.Workload) -> dict:
    """A further workload timed the same way after the headline (K steps after the
    warm-up, CUDA events per step): its Gelem/s, per-launch time and MUFU roofline
    fraction; for a forward workload also the output's error against the oracle on a
    row sample covering every channel block."""
    import torch

    from selective_state_space_33_b200 import binding as sb
    x = W.make_inputs(w)
    dev = torch.device("cuda", torch.cuda.current_device())
    t = W.to_device(x, dev)
    st = torch.cuda.current_stream()
    prob = sb.make_problem(w.batch, w.seqlen, w.dim, w.dstate, sb.SSCAN_BF16 if w.io == "bf16" else sb.SSCAN_F32)
    op = sb.SSCAN_OP_BWD if w.backward else sb.SSCAN_OP_FWD
    ws = torch.empty(max(sb.sscan_workspace_size(prob, op), 256), dtype=torch.uint8, device=dev)
    out = torch.empty_like(t["u"])
    grads = None
    if w.backward and not w.complex_a:
        grads = sb.sscan_bwd(t["u"], t["delta_raw"], t["A"], t["B"], t["C"], t["dout"], t["delta_bias"],
                             t["D_skip"], t["z"], workspace=ws)
    elif w.backward:
        cws = torch.empty(max(sb.sscan_workspace_size(prob, sb.SSCAN_OP_BWD_COMPLEX), 256), dtype=torch.uint8,
                          device=dev)

    def step():
        if w.backward and w.complex_a:
            sb.sscan_bwd_complex(t["u"], t["delta_raw"], t["A"], t["B"], t["C"], t["dout"], t["delta_bias"],
                                 t["D_skip"], t.get("z"), workspace=cws, stream=st)
        elif w.backward:
            sb.sscan_bwd(t["u"], t["delta_raw"], t["A"], t["B"], t["C"], t["dout"], t["delta_bias"], t["D_skip"],
                         t["z"], grads=grads, workspace=ws, stream=st)
        elif w.complex_a:
            sb.sscan_fwd_complex(t["u"], t["delta_raw"], t["A"], t["B"], t["C"], t["delta_bias"], t["D_skip"],
                                 t.get("z"), out=out, stream=st)
        else:
            sb.sscan_fwd(t["u"], t["delta_raw"], t["A"], t["B"], t["C"], t["delta_bias"], t["D_skip"], t["z"],
                         out=out, workspace=ws, stream=st)

    steps = min(args.steps, 10) if w.seqlen > 65536 else args.steps  # the million-step pass is ~20 ms
    for _ in range(max(args.warmup, 3)):
        step()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda.synchronize()
    for a, b in ev:
        a.record(st)
        step()
        b.record(st)
    torch.cuda.synchronize()
    per_launch = statistics.mean(a.elapsed_time(b) for a, b in ev) * 1e-3
    total = ev[0][0].elapsed_time(ev[-1][1]) * 1e-3
    units = roofline_units(w)
    mufu = SM_COUNT * MUFU_PER_SM_CLK * float(measured_peaks().get("sm_max_mhz", 1965.0)) * 1e6
    rec = {"workload": f"{w.name}: {w.description}", "io_dtype": w.io,
           "metric": ((METRIC_COMPLEX_BWD if w.complex_a else METRIC_BWD) if w.backward
                      else (METRIC_COMPLEX if w.complex_a else METRIC_FWD)),
           "value": aggregate(units["elements"], steps, 1, total), "unit": UNIT, "steps": steps,
           "ms_per_step": total / steps * 1e3,
           "roofline": {"bound": "alu", "pipe": "MUFU (ex2, sin, cos)" if w.complex_a else "MUFU ex2",
                        "achieved": units["exps"] / per_launch / 1e9,
                        "peak": mufu / 1e9, "unit": "Gexp/s", "frac": units["exps"] / per_launch / mufu,
                        "per_launch_ms": per_launch * 1e3, "alg_exps_per_launch": units["exps"],
                        "alg_bytes_per_launch": units["bytes"]}}
    if not w.backward and not args.no_cpu_baseline:
        if w.complex_a:
            rec["parity"] = complex_oracle_parity(x, w, out)
        else:
            # the million-step rows are 2^20 long: one row per channel block
            rec["parity"] = oracle_parity(x, w, out, per_block=1 if w.seqlen > 65536 else 2)
    del t, out, x
    torch.cuda.empty_cache()
    return rec


def fp32_record(args, lib, dev) -> dict:
    """The same layer with fp32 I/O (the headline shape's second precision): K timed
    forward passes after the warm-up, their per-launch time, Gelem/s, roofline fraction
    and the output's error against the oracle on a row sample covering every channel
    block.  Runs after the bf16 measurement, once its tensors are released."""
    import torch

    from selective_state_space_33_b200 import binding as sb
    w = W.WORKLOADS["mamba2.8b-f32"]
    x = W.make_inputs(w)
    t = W.to_device(x, dev)
    out = torch.empty_like(t["u"])
    prob = sb.make_problem(w.batch, w.seqlen, w.dim, w.dstate, sb.SSCAN_F32)
    ws = torch.empty(max(sb.sscan_workspace_size(prob, sb.SSCAN_OP_FWD), 256), dtype=torch.uint8, device=dev)
    st = torch.cuda.current_stream()

    def step():
        sb.sscan_fwd(t["u"], t["delta_raw"], t["A"], t["B"], t["C"], t["delta_bias"], t["D_skip"], t["z"],
                     out=out, workspace=ws, stream=st)

    for _ in range(max(args.warmup, 3)):
        step()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    torch.cuda.synchronize()
    for a, b in ev:
        a.record(st)
        step()
        b.record(st)
    torch.cuda.synchronize()
    per_launch = statistics.mean(a.elapsed_time(b) for a, b in ev) * 1e-3
    total = ev[0][0].elapsed_time(ev[-1][1]) * 1e-3
    units = roofline_units(w)
    peaks = measured_peaks()
    hbm_peak = float(peaks.get("hbm_gbs", HBM_FALLBACK_GBS))
    mufu = SM_COUNT * MUFU_PER_SM_CLK * float(peaks.get("sm_max_mhz", 1965.0)) * 1e6
    rec = {"workload": f"{w.name}: {w.description}", "io_dtype": "f32",
           "value": aggregate(units["elements"], args.steps, 1, total), "unit": UNIT,
           "ms_per_step": total / args.steps * 1e3, "steps": args.steps,
           "roofline": {"bound": "alu", "pipe": "MUFU ex2", "achieved": units["exps"] / per_launch / 1e9,
                        "peak": mufu / 1e9, "unit": "Gexp/s", "frac": units["exps"] / per_launch / mufu,
                        "per_launch_ms": per_launch * 1e3, "alg_exps_per_launch": units["exps"],
                        "hbm": {"achieved": units["bytes"] / per_launch / 1e9, "peak": hbm_peak, "unit": "GB/s",
                                "frac": units["bytes"] / per_launch / 1e9 / hbm_peak,
                                "alg_bytes_per_launch": units["bytes"]}}}
    if not args.no_cpu_baseline:
        rec["parity"] = oracle_parity(x, w, out)
    return rec


def e2e_leg(args, t, out, ws, st, units, world, dev):
    """End to end through the C ABI from pinned host buffers: every step copies its
    inputs host -> device, runs the scan and copies its output back.  Steps are
    pipelined as a serving loop would run them: two device buffer sets, the
    host -> device copies on one stream, the scans on another, the device -> host
    copies on a third (the link carries both directions at once), ordered by events
    so that step i's copy-in overlaps step i-1's scan and step i-2's copy-out.  The
    timed region runs from before the first copy-in to after the last copy-out."""
    import torch

    from selective_state_space_33_b200 import binding as sb
    host = {k: v.cpu().pin_memory() for k, v in t.items()}
    dev_in = [{k: torch.empty_like(v) for k, v in t.items()} for _ in range(2)]
    outs = [out, torch.empty_like(out)]
    host_out = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    wss = [ws, torch.empty_like(ws)]
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = host_out[0].numel() * host_out[0].element_size()
    s_in, s_run, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    copied, scanned, returned = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    used = [False, False]

    def e2e_step(i):
        k = i % 2
        if used[k]:
            s_in.wait_event(scanned[k])   # the scan two steps back has read dev_in[k]
        for name in host:
            with torch.cuda.stream(s_in):
                dev_in[k][name].copy_(host[name], non_blocking=True)
        copied[k].record(s_in)
        s_run.wait_event(copied[k])
        if used[k]:
            s_run.wait_event(returned[k])  # outs[k] has been copied out
        d = dev_in[k]
        sb.sscan_fwd(d["u"], d["delta_raw"], d["A"], d["B"], d["C"], d["delta_bias"], d["D_skip"], d.get("z"),
                     out=outs[k], workspace=wss[k], stream=s_run)
        scanned[k].record(s_run)
        s_out.wait_event(scanned[k])
        with torch.cuda.stream(s_out):
            host_out[k].copy_(outs[k], non_blocking=True)
        returned[k].record(s_out)
        used[k] = True

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier()
    ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ea.record(st)
    s_in.wait_stream(st)
    for i in range(args.steps):
        e2e_step(i)
    st.wait_stream(s_out)
    eb.record(st)
    torch.cuda.synchronize()
    e2e_s = reduce_max(ea.elapsed_time(eb) * 1e-3, dev if world > 1 else None)
    return aggregate(units["elements"], args.steps, world, e2e_s), h2d, d2h


def finish(args, w, x, lib, dev, torch, units, value, max_s, per_launch_ms, clk, e2e_value, h2d, d2h,
           launches_per_step, world, l2_note, out=None, secondary=None, others=None):
    peaks = measured_peaks()
    hbm_peak = float(peaks.get("hbm_gbs", HBM_FALLBACK_GBS))
    hbm_src = "measured" if "hbm_gbs" in peaks else "fallback"
    sm_max = float(peaks.get("sm_max_mhz", 1965.0))
    mufu_nominal = SM_COUNT * MUFU_PER_SM_CLK * sm_max * 1e6
    # the same unit count at the SM clock sampled during the timed region
    mufu_at_clock = SM_COUNT * MUFU_PER_SM_CLK * float(clk["sm_mhz"]) * 1e6 if clk.get("sm_mhz") else None
    mufu_probe = ex2_probe(torch, lib, dev)
    launch_s = statistics.mean(per_launch_ms) * 1e-3
    exps_rate = units["exps"] / launch_s
    gbs = units["bytes"] / launch_s / 1e9
    t_roof = max(units["bytes"] / (hbm_peak * 1e9), units["exps"] / mufu_nominal)
    cpu = None
    if world == 1 and not args.no_cpu_baseline and not w.backward and not w.decode and not w.complex_a:
        rate, cores, rows, secs, passes = cpu_oracle_rate(x, w, args.cpu_seconds, with_passes=True)
        rate1, rows1, secs1, passes1 = cpu_oracle_rate_1thread(x, w)
        what = (f"{passes} passes over all {rows} rows" if passes > 1 else
                f"{rows} random rows of {w.batch * w.dim}")
        cpu = {"value": rate, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"{what} x L={w.seqlen} ({passes * rows * w.seqlen} elements, {secs:.1f} s)",
               "single_thread": {"value": rate1, "unit": UNIT,
                                 "sample": f"{rows1} random rows x L={w.seqlen}"
                                           + (f", {passes1} passes" if passes1 > 1 else "")
                                           + f", {secs1:.1f} s on 1 thread"}}
        if out is not None:
            cpu["parity"] = oracle_parity(x, w, out)
    line = {
        "metric": (METRIC_COMPLEX_BWD if w.backward and w.complex_a else METRIC_BWD if w.backward
                   else METRIC_STEP if w.decode else METRIC_COMPLEX if w.complex_a else METRIC), "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": max_s / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": workload_config(w, world, l2_note),
        "clocks": {"sm_mhz": clk["sm_mhz"], "sm_max_mhz": clk["sm_max_mhz"], "reasons": clk["reasons"]},
        "e2e": None if e2e_value is None else {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                                               "d2h_bytes_per_step": d2h},
        "gpu_launches": launches_per_step * args.steps,
        "roofline": hbm_roofline(units, launch_s, hbm_peak, hbm_src, ncu_traffic(args.workload)) if w.decode else {
            "bound": "alu", "pipe": "MUFU (ex2, sin, cos)" if w.complex_a else "MUFU ex2",
            "achieved": exps_rate / 1e9, "peak": mufu_nominal / 1e9,
            "unit": "Gexp/s", "frac": exps_rate / mufu_nominal, "traffic": ncu_traffic(args.workload),
            "peak_source": f"derived: {SM_COUNT} SMs x {MUFU_PER_SM_CLK} ex2/clk x {sm_max:.0f} MHz",
            "peak_probe_gexps": None if mufu_probe is None else mufu_probe / 1e9,
            "frac_of_probe": None if mufu_probe is None else exps_rate / mufu_probe,
            "peak_at_sampled_clock_gexps": mufu_at_clock / 1e9 if mufu_at_clock else None,
            "frac_at_sampled_clock": exps_rate / mufu_at_clock if mufu_at_clock else None,
            "hbm": {"achieved": gbs, "peak": hbm_peak, "unit": "GB/s", "frac": gbs / hbm_peak,
                    "source": hbm_src, "nominal": HBM_NOMINAL_GBS, "frac_nominal": gbs / HBM_NOMINAL_GBS},
            "roofline_frac": t_roof / launch_s,
            "per_launch_ms": launch_s * 1e3,
            "alg_bytes_per_launch": units["bytes"], "alg_exps_per_launch": units["exps"],
        },
        "cpu_baseline": cpu,
    }
    if cpu is not None and "parity" in cpu:
        line["parity"] = cpu["parity"]
    if secondary is not None:
        line["secondary"] = secondary
    if others:
        line["others"] = others
    print(json.dumps(line), flush=True)


def hbm_roofline(units, launch_s, hbm_peak, hbm_src, traffic=None):
    gbs = units["bytes"] / launch_s / 1e9
    return {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s", "frac": gbs / hbm_peak,
            "traffic": traffic, "source": hbm_src, "per_launch_ms": launch_s * 1e3,
            "alg_bytes_per_launch": units["bytes"]}


def launch_ranks(n: int, argv: list):
    """Run this script as ``n`` ranks on one node (one process per GPU) through
    torch.distributed.run on the loopback address; replaces the current process."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__)] + argv
    sys.stdout.flush()
    os.execv(sys.executable, cmd)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(W.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the records that follow the default (bf16) workload: fp32 I/O, the "
                         "Mamba-130M-shaped forward and backward")
    ap.add_argument("--profile-run", action="store_true",
                    help="timed steps only (no clock tail, end-to-end leg, probe or CPU baseline): "
                         "the command line used under ncu")
    args = ap.parse_args(argv)
    world_env = os.environ.get("WORLD_SIZE")
    if world_env is None and args.gpus > 1:
        launch_ranks(args.gpus, sys.argv[1:] if argv is None else list(argv))
    if world_env is not None and int(world_env) != args.gpus:
        sys.exit(f"bench.py: --gpus {args.gpus} but the launcher started WORLD_SIZE={world_env} ranks")
    w = W.WORKLOADS[args.workload]
    if args.impl == "reference":
        reference_arm(args, w)
    else:
        gpu_arm(args, w)
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
