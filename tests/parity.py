"""Helpers shared by the GPU parity tests: run the CUDA path and the oracle on the
same seeded inputs and measure the normwise error max|gpu - ref| / max|ref|."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import selective_state_space_22_b200 as ssd
from selective_state_space_22_b200 import inputs

TOL_F32 = 1e-4   # float32 inputs (real and complex)
TOL_BF16 = 2e-2  # bf16 inputs, float32 state


def rel_err(got, ref) -> float:
    got = np.asarray(got, dtype=np.complex128 if np.iscomplexobj(got) else np.float64)
    ref = np.asarray(ref, dtype=np.complex128 if np.iscomplexobj(ref) else np.float64)
    den = float(np.max(np.abs(ref))) if ref.size else 0.0
    num = float(np.max(np.abs(got - ref))) if ref.size else 0.0
    return num / den if den > 0 else num


def to_dev(inp: dict, dev="cuda") -> dict:
    return {k: (None if v is None else v.to(dev)) for k, v in inp.items()}


def gpu_scan(inp: dict, chunk: int, complex_: bool):
    d = to_dev(inp)
    fn = ssd.ssd_scan_fwd_complex if complex_ else ssd.ssd_scan_fwd
    y, fs = fn(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["init_state"], chunk_size=chunk)
    ssd.ssd_get_device_status()
    return y.float().cpu(), fs.cpu()


def oracle_scan(inp: dict, heads=None, batches=None):
    """Oracle on the whole problem, or on the given (batch, head) sub-problems.

    Slicing heads is exact when every head has its own group or all share one.
    Returns y [b', T, h', P] and final state [b', h', P, N] for the selection.
    """
    w = inputs.widen_all(inp)
    H = w["x"].shape[2]
    G = w["B"].shape[2]
    if heads is None and batches is None:
        return oracle.scan(w["x"], w["dt"], w["A"], w["B"], w["C"], w["D"], w["init_state"])
    assert G == 1 or G == H
    hs = list(range(H)) if heads is None else list(heads)
    bs = list(range(w["x"].shape[0])) if batches is None else list(batches)
    c = np.ascontiguousarray
    sel = lambda a, ax_b, ax_h: c(np.take(np.take(a, bs, axis=ax_b), hs, axis=ax_h))
    x = sel(w["x"], 0, 2)
    dt = sel(w["dt"], 0, 2)
    A = c(w["A"][hs])
    D = None if w["D"] is None else c(w["D"][hs])
    if G == 1:
        B, C = c(w["B"][bs]), c(w["C"][bs])
    else:
        B, C = sel(w["B"], 0, 2), sel(w["C"], 0, 2)
    h0 = None if w["init_state"] is None else sel(w["init_state"], 0, 1)
    return oracle.scan(x, dt, A, B, C, D, h0)


def pick(t: torch.Tensor, batches, heads, ax_b, ax_h) -> np.ndarray:
    a = t.numpy()
    return np.take(np.take(a, list(batches), axis=ax_b), list(heads), axis=ax_h)


def elem_rel_err(got, ref, floor: float = 1e-3) -> float:
    """Per-element relative error, max_i |got_i - ref_i| / max(|ref_i|, floor * max|ref|).

    Reported for information beside the normwise error (which the tests assert):
    it shows a small-magnitude region of the output that is far off."""
    got = np.asarray(got, dtype=np.complex128 if np.iscomplexobj(got) else np.float64)
    ref = np.asarray(ref, dtype=np.complex128 if np.iscomplexobj(ref) else np.float64)
    if ref.size == 0:
        return 0.0
    scale = float(np.max(np.abs(ref)))
    if scale == 0.0:
        return float(np.max(np.abs(got)))
    return float(np.max(np.abs(got - ref) / np.maximum(np.abs(ref), floor * scale)))


# ------------------------------------------------------------ oracle pools
# The oracle is slow (sequential fp64); big parity cases run it on independent
# sub-problems in a process pool.  The pool is started with "spawn", so it does
# not inherit the parent's CUDA context.

def _scan_unit(args):
    return oracle.scan(*args)


def _bwd_unit(args):
    return oracle.scan_bwd(*args)


def oracle_pool_map(fn, jobs, procs=None):
    import multiprocessing as mp
    import os

    if not jobs:
        return []
    n = procs or max(1, min(len(jobs), len(os.sched_getaffinity(0))))
    if n == 1:
        return [fn(j) for j in jobs]
    with mp.get_context("spawn").Pool(n) as pool:
        return pool.map(fn, jobs, chunksize=1)


def oracle_scan_units(w: dict, units):
    """The oracle on (batch, head) sequences in a process pool; w holds the widened
    inputs of the whole problem (B, C with one group, or one group per head).
    Returns [(y [T, P], final [P, N]) per unit]."""
    c = np.ascontiguousarray
    G = w["B"].shape[2]
    jobs = []
    for b, h in units:
        g = 0 if G == 1 else h
        jobs.append((c(w["x"][b:b + 1, :, h:h + 1]), c(w["dt"][b:b + 1, :, h:h + 1]), c(w["A"][h:h + 1]),
                     c(w["B"][b:b + 1, :, g:g + 1]), c(w["C"][b:b + 1, :, g:g + 1]),
                     None if w["D"] is None else c(w["D"][h:h + 1]),
                     None if w["init_state"] is None else c(w["init_state"][b:b + 1, h:h + 1])))
    out = oracle_pool_map(_scan_unit, jobs)
    return [(y[0, :, 0], fs[0, 0]) for y, fs in out]
