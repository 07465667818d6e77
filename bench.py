#!/usr/bin/env python
"""Throughput of the chunked SSD scan on B200, one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

A step is one ``ssd_scan_fwd`` call over one batch of the workload, i.e. the
whole scan (cumulative decay, segsum decay, diagonal block, chunk states,
inter-chunk state passing, off-diagonal output, D skip).  The default workload
is the Mamba-2 BitMamba-1B layer shape (batch 2, T 2048, 64 heads, head dim 64,
d_state 128, one group, chunk 256, bf16 x/B/C/y, float32 dt/A/D/state).

Timing: inputs are resident in HBM; the K timed steps are bracketed by a
barrier and a device synchronize; each step is timed with CUDA events on the
launching stream and L2 is flushed (a 512 MiB write) between steps, outside the
event pairs; the reported time is the max over ranks.  Under torchrun every
rank scans its own copy of the workload (independent sequences: weak scaling,
no collective on the data path).

``--workload decode-bitmamba1b-256seq`` times the one-step decode update
instead: a step is one ``ssd_state_update`` call that advances 256 sequences by
one token each (the float32 state, 537 MB, is streamed through HBM every step,
so L2 holds nothing from one step to the next).

``--workload mamba2-bitmamba1b-layer-bwd-f32`` times the backward instead: a
step is one ``ssd_scan_bwd`` call (all seven gradients of the float32 scan at
the layer shape, given seeded dy and dfinal), timed and flushed as above;
``--workload mamba3lite-complex-bwd-f32`` does the same for the complex scan
(``ssd_scan_bwd_complex``) at the Mamba-3-Lite layer shape.

``--impl reference`` times the fp64 CPU oracle (the program the GPU results are
checked against) on the host cores instead, each step a bounded sample of the
same workload; under torchrun only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "SSD scan tokens/s at Mamba-2 1B layer shape; % of roofline (TC or HBM)"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
L2_FLUSH_BYTES = 512 << 20


# ----------------------------------------------------------------- ranks
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def dist_init(backend: str):
    import torch.distributed as dist

    rank, world, _ = dist_env()
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=300))
    return rank, world


def dist_barrier():
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def dist_max(value: float, device=None) -> float:
    """Max of a host float over all ranks (identity on one rank)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------- algorithmic work
def algorithmic_bytes(shape) -> int:
    """Each input read once and each output written once; chunk states count zero."""
    io = 4 if (shape.io_dtype == "f32" or shape.complex) else 2
    bc = 8 if shape.complex else io
    st = 8 if shape.complex else 4
    b, T, H, P, G, N = shape.batch, shape.seqlen, shape.nheads, shape.headdim, shape.ngroups, shape.dstate
    n = 2 * b * T * H * P * io            # x in, y out
    n += b * T * H * 4                     # dt
    n += 2 * b * T * G * N * bc            # B, C
    n += H * (8 if shape.complex else 4) + H * 4  # A, D
    n += b * H * P * N * st                # final state out
    if shape.init_state:
        n += b * H * P * N * st
    return n


def algorithmic_flops(shape, chunk=None) -> int:
    """2 flops per MAC; causal half of each intra-chunk product; exps not counted.
    ``chunk`` is the chunk length the kernel evaluates (default: the shape's)."""
    b, T, H, P, G, N = (shape.batch, shape.seqlen, shape.nheads, shape.headdim, shape.ngroups,
                        shape.dstate)
    Q = chunk or shape.chunk
    total = 0
    for c0 in range(0, T, Q):
        q = min(Q, T - c0)
        tri = q * (q + 1) // 2
        per_head = 2 * tri * P + 2 * q * N * P + 2 * q * N * P   # diag, chunk state, off-diagonal
        per_group = 2 * tri * N                                  # C B^T
        if shape.complex:
            # Re(M) x is real; the chunk state is a complex MAC (8 flops); the
            # off-diagonal readout keeps only the real part (4 flops per MAC)
            per_head = 2 * tri * P + 8 * q * N * P + 4 * q * N * P
            per_group = 8 * tri * N
        total += b * (H * per_head + G * per_group)
    return total


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return dict(FALLBACK_PEAKS, bf16_tflops_sustained=1400.0, source="fallback")


def kernel_source_sha(path: str) -> str:
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def lookup_traffic(kernel: str, source: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it is for this source."""
    try:
        with open(TRAFFIC_FILE) as f:
            table = json.load(f)
    except Exception:
        return None
    sha = kernel_source_sha(source)
    for row in table.get("entries", []):
        if row.get("kernel") == kernel and row.get("workload") == workload and row.get("source_sha") == sha:
            return row.get("dram_bytes_per_launch")
    return None


# ------------------------------------------------------------ configs
# Both arms (ours and the oracle) print the same config dict for a workload.
def scan_config(shape, world: int) -> dict:
    return {"workload": shape.name, "batch": shape.batch, "seqlen": shape.seqlen,
            "nheads": shape.nheads, "headdim": shape.headdim, "ngroups": shape.ngroups,
            "dstate": shape.dstate, "chunk": shape.chunk, "complex": shape.complex,
            "io_dtype": "f32" if shape.complex else shape.io_dtype,
            "state_dtype": "c64" if shape.complex else "f32", "init_state": shape.init_state,
            "l2": "flushed between timed steps (512 MiB write)",
            "parallelism": f"replicas x{world}" if world > 1 else "1 GPU"}


def decode_config(shape, world: int) -> dict:
    return {"workload": shape.name, "batch": shape.batch, "nheads": shape.nheads,
            "headdim": shape.headdim, "ngroups": shape.ngroups, "dstate": shape.dstate,
            "io_dtype": shape.io_dtype, "state_dtype": "f32",
            "l2": "state (537 MB) larger than L2, streamed every step",
            "parallelism": f"replicas x{world}" if world > 1 else "1 GPU"}


def bwd_config(shape, world: int) -> dict:
    return {"workload": shape.name, "batch": shape.batch, "seqlen": shape.seqlen, "nheads": shape.nheads,
            "headdim": shape.headdim, "ngroups": shape.ngroups, "dstate": shape.dstate,
            "chunk": shape.chunk, "io_dtype": "f32", "complex": shape.complex,
            "l2": "flushed between timed steps (512 MiB write)",
            "parallelism": f"replicas x{world}" if world > 1 else "1 GPU"}


MIN_TIMED_S = 0.12  # default step count: at least this much timed device work


def pick_steps(args, warm_ms: list) -> int:
    """--steps when given, else enough steps for MIN_TIMED_S of timed device time."""
    if args.steps is not None:
        return args.steps
    t = max(statistics.median(warm_ms), 1e-3)
    return int(min(20000, max(100, -(-MIN_TIMED_S * 1e3 // t))))


def e2e_overlapped(hin: dict, dsets: list, run, douts: list, hout: list, k: int):
    """End-to-end time of k steps through the public API with host buffers.

    The device buffer sets (len(dsets), two or more) are used in turn.  Step i
    copies its inputs host -> device on one stream, runs on a second and copies
    its outputs device -> host on a third, so that step i's results travel back
    while later steps' inputs come in and run.  Events order each buffer's
    reuse.  Returns seconds from the first input copy to the last output copy
    (device events)."""
    import torch

    n = len(dsets)
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    in_done, cmp_done, out_done = [ev() for _ in range(n)], [ev() for _ in range(n)], [ev() for _ in range(n)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record(s_in)
    for i in range(k):
        j = i % n
        with torch.cuda.stream(s_in):
            if i >= n:
                s_in.wait_event(cmp_done[j])     # step i-n has read this set's inputs
            for name, v in hin.items():
                dsets[j][name].copy_(v, non_blocking=True)
            in_done[j].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(in_done[j])
            if i >= n:
                s_cmp.wait_event(out_done[j])    # step i-n's outputs have left this set
            run(j)
            cmp_done[j].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(cmp_done[j])
            for name, v in hout[j].items():
                v.copy_(douts[j][name], non_blocking=True)
            out_done[j].record(s_out)
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_cmp)
    end.record(s_out)
    torch.cuda.synchronize()
    return start.elapsed_time(end) / 1e3


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """Polls NVML for the SM clock and the clock-event reasons in a thread."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.samples = []
        self.period = period_s
        self._stop = threading.Event()
        self.ok = False
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as exc:  # no NVML: report clocks as unavailable
            self.err = repr(exc)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                try:
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except Exception:
                    rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def stop(self):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self, t0: float, t1: float):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": "NVML unavailable"}
        win = [s for s in self.samples if t0 <= s[0] <= t1]
        if not win:  # a very short region: take the samples nearest to it
            win = sorted(self.samples, key=lambda s: min(abs(s[0] - t0), abs(s[0] - t1)))[:3]
        reasons = set()
        for _, _, rs in win:
            for bit, name in self.REASONS.items():
                if rs & bit and name != "gpu_idle":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s[1] for s in win) if win else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons), "samples": len(win)}


# ------------------------------------------------------------ CPU oracle
def oracle_threads():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def run_oracle_units(w: dict, units, threads: int) -> float:
    """Oracle over the given (batch, head) sequences, one per thread; seconds."""
    import numpy as np

    import oracle

    lib = oracle.load()
    G = w["B"].shape[2]
    c = np.ascontiguousarray

    def one(unit):
        b, h = unit
        g = 0 if G == 1 else h
        oracle.scan(c(w["x"][b:b + 1, :, h:h + 1]), c(w["dt"][b:b + 1, :, h:h + 1]), c(w["A"][h:h + 1]),
                    c(w["B"][b:b + 1, :, g:g + 1]), c(w["C"][b:b + 1, :, g:g + 1]),
                    None if w["D"] is None else c(w["D"][h:h + 1]),
                    None if w["init_state"] is None else c(w["init_state"][b:b + 1, h:h + 1]), lib=lib)

    t0 = time.perf_counter()
    with cf.ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(one, units))
    return time.perf_counter() - t0


def cpu_baseline(shape, max_updates: float = 4e9):
    """The oracle as it stands, timed on this host's cores on a bounded sample:
    the first (batch, head) sequences of the workload, up to ~max_updates state
    element updates (the whole workload when it fits)."""
    from selective_state_space_22_b200 import inputs

    threads = oracle_threads()
    w = inputs.widen_all(inputs.scan_inputs(shape))
    total = shape.batch * shape.nheads
    per_unit = shape.seqlen * shape.headdim * shape.dstate
    n = max(1, min(total, int(max_updates // per_unit)))
    units = [(i // shape.nheads, i % shape.nheads) for i in range(n)]
    secs = run_oracle_units(w, units, threads)
    tokens = shape.seqlen * n / shape.nheads
    return {"value": tokens / secs, "unit": "tokens/s", "cores": min(threads, n), "kind": "oracle",
            "sample": f"{n} of {total} (batch, head) sequences of {shape.name} (T={shape.seqlen}); "
                      f"fp64 sequential recurrence, one sequence per thread; tokens/s counts "
                      f"sequences/nheads x T",
            "seconds": secs}


# ---------------------------------------------------------------- decode
DECODE_POOL = 8  # distinct per-step inputs resident on the device, used in turn


def decode_bytes(shape) -> int:
    """Per step: the state read and written once, x in, y out, dt, B, C, A, D."""
    io = 4 if shape.io_dtype == "f32" else 2
    b, H, P, G, N = shape.batch, shape.nheads, shape.headdim, shape.ngroups, shape.dstate
    return 2 * b * H * P * N * 4 + 2 * b * H * P * io + b * H * 4 + 2 * b * G * N * io + 2 * H * 4


def decode_cpu_baseline(shape, seqs: int = 16, steps: int = 8):
    """The oracle's one-step update on the first ``seqs`` sequences, one
    sequence per thread, ``steps`` steps; tokens/s = sequences x steps / s."""
    import numpy as np

    import oracle
    from selective_state_space_22_b200 import inputs

    threads = oracle_threads()
    lib = oracle.load()
    gen, const = inputs.decode_setup(shape)
    st = inputs.widen(const["state"][:seqs])
    A, D = inputs.widen(const["A"]), inputs.widen(const["D"])
    step_inp = [inputs.widen_all(inputs.decode_step_inputs(gen, shape)) for _ in range(steps)]
    c = np.ascontiguousarray
    states = [c(st[i:i + 1]) for i in range(seqs)]

    def one(i, w):
        _, states[i] = oracle.state_update(states[i], c(w["x"][i:i + 1]), c(w["dt"][i:i + 1]), A,
                                           c(w["B"][i:i + 1]), c(w["C"][i:i + 1]), D, lib=lib)

    t0 = time.perf_counter()
    with cf.ThreadPoolExecutor(max_workers=threads) as ex:
        for w in step_inp:
            list(ex.map(lambda i: one(i, w), range(seqs)))
    secs = time.perf_counter() - t0
    return {"value": seqs * steps / secs, "unit": "tokens/s", "cores": min(threads, seqs), "kind": "oracle",
            "sample": f"{seqs} of {shape.batch} sequences x {steps} decode steps of {shape.name}; fp64 "
                      f"one-step update, one sequence per thread",
            "seconds": secs}


def bench_decode(args, shape):
    import torch

    import selective_state_space_22_b200 as ssd
    from selective_state_space_22_b200 import inputs

    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device for --impl ours")
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist_init("nccl")
    ssd.load_library()

    gen, const = inputs.decode_setup(shape)
    state = const["state"].to(dev)
    A, D = const["A"].to(dev), const["D"].to(dev)
    pool_host = [inputs.decode_step_inputs(gen, shape) for _ in range(DECODE_POOL)]
    pool = [{k: v.to(dev) for k, v in p.items()} for p in pool_host]
    y = torch.empty_like(pool[0]["x"])

    def step(i):
        p = pool[i % DECODE_POOL]
        ssd.ssd_state_update(state, p["x"], p["dt"], A, p["B"], p["C"], D, y=y)

    stream = torch.cuda.current_stream()
    sampler = ClockSampler(local).start()
    warm_ms = []
    for i in range(max(args.warmup, 3)):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        step(i)
        b.record(stream)
        torch.cuda.synchronize()
        warm_ms.append(a.elapsed_time(b))
    ssd.ssd_get_device_status()
    steps = int(dist_max(float(pick_steps(args, warm_ms)), dev))
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    dist_barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    torch.cuda._sleep(20_000_000)  # let the host queue run ahead of the device
    for i in range(steps):
        starts[i].record(stream)
        step(i)
        ends[i].record(stream)
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    dist_barrier()
    sampler.stop()
    ssd.ssd_get_device_status()
    per_step_ms = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    total_s = dist_max(sum(per_step_ms) / 1e3, dev)
    value = shape.batch * world * steps / total_s
    peaks = load_peaks()
    abytes = decode_bytes(shape)
    t_launch = statistics.median(per_step_ms) / 1e3
    kernel = "update_real_vec" if shape.dstate % 128 == 0 else "update_generic"
    src = os.path.join(ROOT, "selective_state_space_22_b200", "csrc", "decode.cu")
    roofline = {"bound": "hbm", "achieved": abytes / t_launch / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": abytes / t_launch / 1e9 / peaks["hbm_gbs"],
                "traffic": lookup_traffic(kernel, src, shape.name), "kernel": kernel,
                "algorithmic_bytes_per_launch": abytes,
                "peak_source": f"{peaks['source']} (MEASURED_PEAKS.json burst)"
                if peaks["source"] == "measured" else "fallback (6.65 TB/s, 1.59 PFLOP/s)",
                "roofline_time_us": 1e6 * abytes / (peaks["hbm_gbs"] * 1e9), "kernel_time_us": 1e6 * t_launch}

    e2e = None
    if not args.no_e2e:
        # per step: that step's x, dt, B, C in from pinned host memory, y back out
        # (the state stays resident: decoding updates it in place on the device)
        hin = {k: v.pin_memory() for k, v in pool_host[0].items()}
        dsets = [{k: torch.empty_like(v) for k, v in pool[0].items()} for _ in range(2)]
        douts = [{"y": torch.empty_like(y)} for _ in range(2)]
        hout = [{"y": torch.empty(y.shape, dtype=y.dtype).pin_memory()} for _ in range(2)]
        h2d = sum(v.numel() * v.element_size() for v in hin.values())
        d2h = hout[0]["y"].numel() * hout[0]["y"].element_size()
        k_e2e = max(4, min(steps, 64))

        def run(j):
            p = dsets[j]
            ssd.ssd_state_update(state, p["x"], p["dt"], A, p["B"], p["C"], D, y=douts[j]["y"])

        e2e_overlapped(hin, dsets, run, douts, hout, 2)
        dist_barrier()
        e2e_s = dist_max(e2e_overlapped(hin, dsets, run, douts, hout, k_e2e), dev)
        dist_barrier()
        e2e = {"value": shape.batch * world * k_e2e / e2e_s, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "steps": k_e2e, "ms_per_step": 1e3 * e2e_s / k_e2e,
               "how": "two device buffer sets; H2D, compute and D2H on three streams, overlapped"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = decode_cpu_baseline(shape)
        cpu.pop("seconds", None)
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": steps,
        "warmup": max(args.warmup, 3), "ms_per_step": 1e3 * total_s / steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic", "impl": "ours",
        "config": decode_config(shape, world),
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "clocks": sampler.summary(t0, t1),
        "gpu_launches": steps,
        "step_ms_p10_p50_p90": [statistics.quantiles(per_step_ms, n=10)[0], statistics.median(per_step_ms),
                                statistics.quantiles(per_step_ms, n=10)[-1]],
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    import torch.distributed as dist

    if dist.is_initialized():
        dist.destroy_process_group()
    return 0


def bench_reference_decode(args, shape):
    rank, world = dist_init("gloo")
    if rank != 0:
        return 0
    for _ in range(args.warmup):
        decode_cpu_baseline(shape, seqs=1, steps=1)
    steps = args.steps if args.steps is not None else 3
    res = [decode_cpu_baseline(shape) for _ in range(steps)]
    secs = sum(r["seconds"] for r in res)
    tokens = sum(r["value"] * r["seconds"] for r in res)
    value = tokens / secs
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * secs / steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": decode_config(shape, world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": res[0]["cores"], "kind": "oracle",
                         "sample": "per step " + res[0]["sample"]},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ arms
def bench_reference(args, shape):
    rank, world = dist_init("gloo")
    if rank != 0:
        return 0
    from selective_state_space_22_b200 import inputs

    threads = oracle_threads()
    inp = inputs.scan_inputs(shape)
    w = inputs.widen_all(inp)
    n_heads = min(shape.nheads, max(threads, 1))
    heads = list(range(n_heads))
    units = [(0, h) for h in heads]
    for _ in range(args.warmup):
        run_oracle_units(w, units[:1], 1)
    steps = args.steps if args.steps is not None else 3
    times = [run_oracle_units(w, units, threads) for _ in range(steps)]
    secs = sum(times)
    tokens = shape.seqlen * n_heads / shape.nheads * steps
    value = tokens / secs
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * secs / steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "impl": "reference",
        "config": scan_config(shape, world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": min(threads, n_heads),
                         "kind": "oracle",
                         "sample": f"per step {n_heads} of {shape.nheads} heads of batch 0 "
                                   f"(T={shape.seqlen}), one sequence per thread"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def bench_ours(args, shape):
    import torch

    import selective_state_space_22_b200 as ssd
    from selective_state_space_22_b200 import inputs

    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device for --impl ours")
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist_init("nccl")
    ssd.load_library()

    # inputs resident in HBM
    inp = inputs.scan_inputs(shape)
    d = {k: (None if v is None else v.to(dev)) for k, v in inp.items()}
    cplx = shape.complex
    io = ssd.SSD_F32 if (cplx or shape.io_dtype == "f32") else ssd.SSD_BF16
    y = torch.empty_like(d["x"])
    fs = torch.empty((shape.batch, shape.nheads, shape.headdim, shape.dstate),
                     dtype=torch.complex64 if cplx else torch.float32, device=dev)
    nbytes = ssd.ssd_scan_workspace_size(shape.batch, shape.seqlen, shape.nheads, shape.headdim,
                                         shape.ngroups, shape.dstate, shape.chunk, cplx, io)
    ws = torch.zeros(max(nbytes, 16), dtype=torch.uint8, device=dev)
    fn = ssd.ssd_scan_fwd_complex if cplx else ssd.ssd_scan_fwd
    launches = ssd.ssd_scan_kernel_launches(shape.batch, shape.seqlen, shape.nheads, shape.headdim,
                                            shape.ngroups, shape.dstate, shape.chunk, cplx, io)
    tc_path = (not cplx and io == ssd.SSD_BF16 and shape.headdim == 64 and shape.dstate == 128
               and shape.seqlen >= 128)  # the tcgen05 kernel (1 launch; 3 for batch 1 cut in two)
    cplx_tc = cplx and shape.headdim == 64 and shape.dstate == 64  # the tcgen05 complex kernels
    kernel_chunk = 128 if (tc_path or cplx_tc) else shape.chunk  # the tensor-core kernels tile 128 tokens

    def step(dd=d, yy=y, ff=fs, w=ws):
        fn(dd["x"], dd["dt"], dd["A"], dd["B"], dd["C"], dd["D"], dd["init_state"], chunk_size=shape.chunk,
           y=yy, final_state=ff, workspace=w)

    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    sampler = ClockSampler(local).start()

    warm_ms = []
    for _ in range(max(args.warmup, 3)):
        flush.fill_(1)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        step()
        b.record(stream)
        torch.cuda.synchronize()
        warm_ms.append(a.elapsed_time(b))
    ssd.ssd_get_device_status()
    steps = int(dist_max(float(pick_steps(args, warm_ms)), dev))  # every rank the same K

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    dist_barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    torch.cuda._sleep(20_000_000)  # let the host queue run ahead of the device
    for i in range(steps):
        flush.fill_(i & 0xFF)
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    dist_barrier()
    sampler.stop()
    ssd.ssd_get_device_status()
    per_step_ms = [s_.elapsed_time(e_) for s_, e_ in zip(starts, ends)]
    local_s = sum(per_step_ms) / 1e3
    total_s = dist_max(local_s, dev)
    tokens = shape.tokens * world * steps
    value = tokens / total_s
    ms_per_step = 1e3 * total_s / steps

    # roofline of the dominant kernel (the whole call when it is one launch)
    peaks = load_peaks()
    abytes = algorithmic_bytes(shape)
    aflops = algorithmic_flops(shape, kernel_chunk)
    t_launch = statistics.median(per_step_ms) / 1e3 if launches == 1 else sum(per_step_ms) / len(per_step_ms) / 1e3
    hbm_t = abytes / (peaks["hbm_gbs"] * 1e9)
    tc_t = aflops / (peaks["bf16_tflops"] * 1e12)
    bound = "hbm" if hbm_t >= tc_t else "tensor"
    if bound == "hbm":
        achieved, peak, unit = abytes / t_launch / 1e9, peaks["hbm_gbs"], "GB/s"
    else:
        achieved, peak, unit = aflops / t_launch / 1e12, peaks["bf16_tflops"], "TFLOP/s"
    if tc_path:
        kernel, src_name = "ssd_scan_tc_kernel", "scan_tc.cu"
    elif cplx_tc:
        kernel, src_name = ("state_kernel+cplx_state_pass+scan_kernel (3 launches, tcgen05, timed as one call)",
                            "scan_complex_tc.cuh")
    elif cplx:
        kernel, src_name = "cplx_chunk_state+cplx_state_pass+cplx_chunk_scan (3 kernels)", "scan_complex.cu"
    else:
        kernel, src_name = "chunk_state+state_pass+chunk_scan (3 kernels)", "scan_generic.cu"
    src = os.path.join(ROOT, "selective_state_space_22_b200", "csrc", src_name)
    traffic = lookup_traffic(kernel, src, shape.name)
    roofline = {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
                "frac": achieved / peak, "traffic": traffic, "kernel": kernel,
                "kernel_chunk": kernel_chunk, "launches_per_call": launches,
                "algorithmic_bytes_per_launch": abytes, "algorithmic_flops_per_launch": aflops,
                "peak_source": f"{peaks['source']} (MEASURED_PEAKS.json burst)"
                if peaks["source"] == "measured" else "fallback (6.65 TB/s, 1.59 PFLOP/s)",
                "roofline_time_us": 1e6 * max(hbm_t, tc_t), "kernel_time_us": 1e6 * t_launch,
                "frac_of_roofline_time": max(hbm_t, tc_t) / t_launch}

    # end to end through the public API: pinned host inputs in, results back out
    e2e = None
    if not args.no_e2e:
        hin = {k: v.pin_memory() for k, v in inp.items() if v is not None}
        # two buffer sets (three measured slower: 0.94 against 0.87 ms per step)
        dsets = [{k: d[k] for k in hin}, {k: torch.empty_like(d[k]) for k in hin}]
        douts = [{"y": y, "final_state": fs}, {"y": torch.empty_like(y), "final_state": torch.empty_like(fs)}]
        hout = [{k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in o.items()} for o in douts]
        h2d = sum(v.numel() * v.element_size() for v in hin.values())
        d2h = sum(v.numel() * v.element_size() for v in hout[0].values())
        k_e2e = max(4, min(steps, 40))
        full = lambda j: dict(dsets[j], **{k: None for k in d if k not in hin})

        def run(j):
            step(full(j), douts[j]["y"], douts[j]["final_state"])

        e2e_overlapped(hin, dsets, run, douts, hout, 2)  # warm-up
        dist_barrier()
        e2e_s = dist_max(e2e_overlapped(hin, dsets, run, douts, hout, k_e2e), dev)
        dist_barrier()
        e2e = {"value": shape.tokens * world * k_e2e / e2e_s, "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": k_e2e,
               "ms_per_step": 1e3 * e2e_s / k_e2e,
               "how": "two device buffer sets; H2D, compute and D2H on three streams, overlapped"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(shape)
        cpu.pop("seconds", None)

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": steps,
        "warmup": max(args.warmup, 3), "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if tc_path else "f32",
        "data": "synthetic",
        "impl": "ours",
        "config": scan_config(shape, world),
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "clocks": sampler.summary(t0, t1),
        "gpu_launches": launches * steps,
        "step_ms_p10_p50_p90": [statistics.quantiles(per_step_ms, n=10)[0] if len(per_step_ms) > 1 else per_step_ms[0],
                                statistics.median(per_step_ms),
                                statistics.quantiles(per_step_ms, n=10)[-1] if len(per_step_ms) > 1 else per_step_ms[0]],
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    import torch.distributed as dist

    if dist.is_initialized():
        dist.destroy_process_group()
    return 0


# ------------------------------------------------- packed projection input
def packed_bytes(shape) -> dict:
    """Per call.  fused: the projection output read once (bf16), y written, the
    final state written.  unpacked: the block's separate unpacking pass (read the
    projection, write x float32, B and C complex64, dt float32) and then the scan
    reading those.  The difference is what reading the slices in place saves."""
    b, T, H, P, N = shape.batch, shape.seqlen, shape.nheads, shape.headdim, shape.dstate
    tok = b * T
    W = H * (P + 4 * N + 1)
    proj = tok * W * 2
    out = tok * H * P * 4 + b * H * P * N * 8
    unpacked = tok * (H * P * 4 + 2 * H * N * 8 + H * 4)
    return {"fused": proj + out + 8 * H, "unpack_then_scan": proj + 2 * unpacked + out + 8 * H}


def bench_packed(args, shape):
    import torch

    import selective_state_space_22_b200 as ssd
    from selective_state_space_22_b200 import inputs

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist_init("nccl")
    ssd.load_library()
    inp = inputs.packed_inputs(shape, "bf16")
    d = {k: (None if v is None else v.to(dev)) for k, v in inp.items()}
    H, P, N = shape.nheads, shape.headdim, shape.dstate
    y = torch.empty((shape.batch, shape.seqlen, H, P), dtype=torch.float32, device=dev)
    fs = torch.empty((shape.batch, H, P, N), dtype=torch.complex64, device=dev)
    ws = torch.zeros(max(16, ssd.ssd_scan_workspace_size(shape.batch, shape.seqlen, H, P, H, N, shape.chunk, True,
                                                         ssd.SSD_F32)), dtype=torch.uint8, device=dev)

    def step():
        ssd.ssd_scan_fwd_complex_packed(d["proj"], d["A"], d["D"], None, nheads=H, headdim=P, dstate=N,
                                        dt_bias=d["dt_bias"], chunk_size=shape.chunk, y=y, final_state=fs,
                                        workspace=ws)

    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    sampler = ClockSampler(local).start()
    warm_ms = []
    for _ in range(max(args.warmup, 3)):
        flush.fill_(1)
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        step()
        b_.record(stream)
        torch.cuda.synchronize()
        warm_ms.append(a.elapsed_time(b_))
    ssd.ssd_get_device_status()
    steps = int(dist_max(float(pick_steps(args, warm_ms)), dev))
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    dist_barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    torch.cuda._sleep(20_000_000)
    for i in range(steps):
        flush.fill_(i & 0xFF)
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    dist_barrier()
    sampler.stop()
    ssd.ssd_get_device_status()
    per_step_ms = [a.elapsed_time(b_) for a, b_ in zip(starts, ends)]
    total_s = dist_max(sum(per_step_ms) / 1e3, dev)
    t_call = statistics.median(per_step_ms) / 1e3
    peaks = load_peaks()
    by = packed_bytes(shape)
    line = {
        "metric": METRIC, "value": shape.tokens * world * steps / total_s, "unit": "tokens/s", "n_gpus": world,
        "steps": steps, "warmup": max(args.warmup, 3), "ms_per_step": 1e3 * total_s / steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "impl": "ours", "config": dict(scan_config(shape, world), io_dtype="bf16 projection"),
        "roofline": {"bound": "hbm", "achieved": by["fused"] / t_call / 1e9, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": by["fused"] / t_call / 1e9 / peaks["hbm_gbs"], "traffic": None,
                     "kernel": "complex scan from the packed projection (3 launches, timed as one call)",
                     "algorithmic_bytes_per_launch": by["fused"],
                     "bytes_unpack_then_scan": by["unpack_then_scan"],
                     "bytes_saved": by["unpack_then_scan"] - by["fused"], "kernel_time_us": 1e6 * t_call},
        "cpu_baseline": None, "e2e": None, "clocks": sampler.summary(t0, t1), "gpu_launches": 3 * steps,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    import torch.distributed as dist

    if dist.is_initialized():
        dist.destroy_process_group()
    return 0


# ------------------------------------------------------------- variants
SFU_EXP_PER_CLK_SM = 16  # exponentials per clock per SM (4 per sub-partition)


def bench_variant(args, name):
    """The conv1d prologue or the Mamba-1 selective scan, one call per step."""
    import torch

    import selective_state_space_22_b200 as ssd
    from selective_state_space_22_b200 import inputs

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist_init("nccl")
    ssd.load_library()
    peaks = load_peaks()
    if name == inputs.MAMBA2_CONV.name:
        sh = inputs.MAMBA2_CONV
        inp = inputs.conv_inputs(sh)
        d = {k: (None if v is None else v.to(dev)) for k, v in inp.items()}
        Ct = sh.x_channels + 2 * sh.bc_channels
        out = (torch.empty((sh.batch, sh.seqlen, sh.x_channels), dtype=d["xbc"].dtype, device=dev),
               torch.empty((sh.batch, sh.seqlen, sh.bc_channels), dtype=d["xbc"].dtype, device=dev),
               torch.empty((sh.batch, sh.seqlen, sh.bc_channels), dtype=d["xbc"].dtype, device=dev))
        step = lambda: ssd.ssd_conv1d_xbc(d["xbc"], d["weight"], d["bias"], None, x_channels=sh.x_channels,
                                          bc_channels=sh.bc_channels, silu=sh.silu, out=out)
        tokens = sh.batch * sh.seqlen
        esz = 2 if sh.io_dtype == "bf16" else 4
        abytes = 2 * sh.batch * sh.seqlen * Ct * esz + Ct * (sh.width + 1) * 4
        kernel, bound, alu_peak = "conv1d_xbc_tile_kernel", "hbm", None
    else:
        sh = inputs.MAMBA1_50M
        inp = inputs.selective_inputs(sh)
        d = {k: (None if v is None else v.to(dev)) for k, v in inp.items()}
        y = torch.empty_like(d["x"])
        fs = torch.empty((sh.batch, sh.channels, sh.dstate), dtype=torch.float32, device=dev)
        step = lambda: ssd.ssd_selective_scan(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["init_state"],
                                              y=y, final_state=fs)
        tokens = sh.tokens
        esz = 2 if sh.io_dtype == "bf16" else 4
        abytes = (sh.tokens * sh.channels * (2 * esz + 4) + 2 * sh.tokens * sh.ngroups * sh.dstate * esz
                  + sh.batch * sh.channels * sh.dstate * 4 + sh.channels * (sh.dstate + 1) * 4)
        exps = sh.tokens * sh.channels * sh.dstate
        kernel = "selective_scan_tile_kernel"
        alu_peak = 148 * SFU_EXP_PER_CLK_SM * 1.965e9  # exponentials per second at the max SM clock
        bound = "alu" if exps / alu_peak > abytes / (peaks["hbm_gbs"] * 1e9) else "hbm"
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    sampler = ClockSampler(local).start()
    warm_ms = []
    for _ in range(max(args.warmup, 3)):
        flush.fill_(1)
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        step()
        b_.record(stream)
        torch.cuda.synchronize()
        warm_ms.append(a.elapsed_time(b_))
    ssd.ssd_get_device_status()
    steps = int(dist_max(float(pick_steps(args, warm_ms)), dev))
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    dist_barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    torch.cuda._sleep(20_000_000)
    for i in range(steps):
        flush.fill_(i & 0xFF)
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    dist_barrier()
    sampler.stop()
    ssd.ssd_get_device_status()
    per_step_ms = [a.elapsed_time(b_) for a, b_ in zip(starts, ends)]
    total_s = dist_max(sum(per_step_ms) / 1e3, dev)
    t_call = statistics.median(per_step_ms) / 1e3
    if bound == "alu":
        roof = {"bound": "alu", "achieved": exps / t_call / 1e12, "peak": alu_peak / 1e12, "unit": "Texp/s",
                "frac": exps / t_call / alu_peak,
                "peak_source": "derived: 148 SMs x 16 exponentials per clock x 1965 MHz",
                "hbm_frac": abytes / t_call / 1e9 / peaks["hbm_gbs"]}
    else:
        roof = {"bound": "hbm", "achieved": abytes / t_call / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": abytes / t_call / 1e9 / peaks["hbm_gbs"]}
    roof.update({"traffic": lookup_traffic(kernel, os.path.join(ROOT, "selective_state_space_22_b200", "csrc",
                                                                "variants.cu"), sh.name),
                 "kernel": kernel, "algorithmic_bytes_per_launch": abytes, "kernel_time_us": 1e6 * t_call})
    line = {
        "metric": METRIC, "value": tokens * world * steps / total_s, "unit": "tokens/s", "n_gpus": world,
        "steps": steps, "warmup": max(args.warmup, 3), "ms_per_step": 1e3 * total_s / steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "impl": "ours", "config": dict(dataclasses_asdict(sh), parallelism="1 GPU" if world == 1 else f"replicas x{world}"),
        "roofline": roof, "cpu_baseline": None, "e2e": None, "clocks": sampler.summary(t0, t1), "gpu_launches": steps,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    import torch.distributed as dist

    if dist.is_initialized():
        dist.destroy_process_group()
    return 0


def dataclasses_asdict(obj):
    import dataclasses

    dd = dataclasses.asdict(obj)
    dd["workload"] = dd.pop("name")
    return dd


# ------------------------------------------------------- sequence split
def bench_seqpar(args, shape):
    """One sequence of shape.seqlen tokens cut into consecutive slices, one per
    rank: state-only scan of each slice, all-gather of the slice end states and
    log-decays over NCCL, fold, full scan of each slice from its entering state
    (selective_state_space_22_b200.seqpar).  Strong scaling: the whole job is one
    sequence whatever the number of GPUs; value = its tokens / max over ranks."""
    import torch

    import selective_state_space_22_b200 as ssd
    from selective_state_space_22_b200 import inputs
    from selective_state_space_22_b200.seqpar import scan_fwd_sequence_parallel

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist_init("nccl")
    ssd.load_library()
    inp = inputs.scan_inputs(shape)
    t0, t1 = shape.seqlen * rank // world, shape.seqlen * (rank + 1) // world
    sl = lambda t: None if t is None else t[:, t0:t1].contiguous().to(dev)
    d = {k: sl(inp[k]) for k in ("x", "dt", "B", "C")}
    d.update(A=inp["A"].to(dev), D=inp["D"].to(dev),
             init_state=inp["init_state"].to(dev) if (rank == 0 and inp["init_state"] is not None) else None)

    def step():
        return scan_fwd_sequence_parallel(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["init_state"],
                                          chunk_size=shape.chunk)

    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    sampler = ClockSampler(local).start()
    warm_ms = []
    for _ in range(max(args.warmup, 3)):
        flush.fill_(1)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        step()
        b.record(stream)
        torch.cuda.synchronize()
        warm_ms.append(a.elapsed_time(b))
    ssd.ssd_get_device_status()
    steps = int(dist_max(float(pick_steps(args, warm_ms)), dev))
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    dist_barrier()
    torch.cuda.synchronize()
    t_0 = time.perf_counter()
    for i in range(steps):
        flush.fill_(i & 0xFF)
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize()
    t_1 = time.perf_counter()
    dist_barrier()
    sampler.stop()
    ssd.ssd_get_device_status()
    per_step_ms = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    total_s = dist_max(sum(per_step_ms) / 1e3, dev)
    value = shape.tokens * steps / total_s
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": steps,
        "warmup": max(args.warmup, 3), "ms_per_step": 1e3 * total_s / steps, "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "impl": "ours",
        "config": dict(scan_config(shape, world), parallelism=f"sequence split x{world}"),
        "roofline": None, "cpu_baseline": None, "e2e": None, "clocks": sampler.summary(t_0, t_1),
        "gpu_launches": None,
        "note": "per step per rank: state-only scan of its slice, NCCL all-gather of (end state, log-decay), "
                "fold, full scan of the slice",
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    import torch.distributed as dist

    if dist.is_initialized():
        dist.destroy_process_group()
    return 0


# --------------------------------------------------------------- backward
BWD_METRIC = {False: "SSD scan backward tokens/s at Mamba-2 1B layer shape (float32); % of HBM roofline",
              True: "SSD complex scan backward tokens/s at Mamba-3-Lite layer shape (float32); % of HBM roofline"}


def bwd_bytes(shape) -> int:
    """Per call: x and dy read, dx written; dt read, ddt written; B and C read, dB
    and dC written; init_state and dfinal read, dinit written; A and D read, dA
    and dD written.  Float32, with the complex tensors (A, B, C, states and their
    gradients) at 8 bytes an element for a complex workload."""
    b, T, H, P, G, N = shape.batch, shape.seqlen, shape.nheads, shape.headdim, shape.ngroups, shape.dstate
    tok = b * T
    z = 8 if shape.complex else 4
    return 4 * (3 * tok * H * P + 2 * tok * H + 2 * H) + z * (4 * tok * G * N + 3 * b * H * P * N + 2 * H)


def bwd_cpu_units(shape, units, threads):
    """The oracle's gradient over the given (batch, head) sequences, one per
    thread; returns seconds."""
    import numpy as np
    import torch

    import oracle
    from selective_state_space_22_b200 import inputs

    lib = oracle.load()
    w = inputs.widen_all(inputs.scan_inputs(shape))
    up = {k: (v.to(torch.complex128) if v.is_complex() else v.double()).numpy()
          for k, v in inputs.bwd_upstream(shape).items()}
    c = np.ascontiguousarray

    def one(unit):
        b, h = unit
        g = 0 if shape.ngroups == 1 else h * shape.ngroups // shape.nheads
        oracle.scan_bwd(c(w["x"][b:b + 1, :, h:h + 1]), c(w["dt"][b:b + 1, :, h:h + 1]), c(w["A"][h:h + 1]),
                        c(w["B"][b:b + 1, :, g:g + 1]), c(w["C"][b:b + 1, :, g:g + 1]),
                        None if w["D"] is None else c(w["D"][h:h + 1]),
                        None if w["init_state"] is None else c(w["init_state"][b:b + 1, h:h + 1]),
                        c(up["dy"][b:b + 1, :, h:h + 1]), c(up["dfinal"][b:b + 1, h:h + 1]), lib=lib)

    t0 = time.perf_counter()
    with cf.ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(one, units))
    return time.perf_counter() - t0


def bwd_cpu_baseline(shape, max_units: int = 16):
    threads = oracle_threads()
    total = shape.batch * shape.nheads
    n = max(1, min(total, max_units, threads))
    units = [(i // shape.nheads, i % shape.nheads) for i in range(n)]
    secs = bwd_cpu_units(shape, units, threads)
    return {"value": shape.seqlen * n / shape.nheads / secs, "unit": "tokens/s", "cores": min(threads, n),
            "kind": "oracle",
            "sample": f"{n} of {total} (batch, head) sequences of {shape.name} (T={shape.seqlen}); fp64 "
                      f"sequential adjoint, one sequence per thread; tokens/s counts sequences/nheads x T",
            "seconds": secs}


def bench_bwd(args, shape):
    import torch

    import selective_state_space_22_b200 as ssd
    from selective_state_space_22_b200 import inputs

    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device for --impl ours")
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist_init("nccl")
    ssd.load_library()

    inp = inputs.scan_inputs(shape)
    up = inputs.bwd_upstream(shape)
    d = {k: (None if v is None else v.to(dev)) for k, v in inp.items()}
    u = {k: v.to(dev) for k, v in up.items()}
    size_fn = ssd.ssd_scan_bwd_complex_workspace_size if shape.complex else ssd.ssd_scan_bwd_workspace_size
    nbytes = size_fn(shape.batch, shape.seqlen, shape.nheads, shape.headdim, shape.ngroups, shape.dstate)
    ws = torch.zeros(max(nbytes, 16), dtype=torch.uint8, device=dev)
    out = {}

    fn = ssd.ssd_scan_bwd_complex if shape.complex else ssd.ssd_scan_bwd

    def step():
        out.update(fn(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["init_state"],
                      u["dy"], u["dfinal"], workspace=ws))

    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    sampler = ClockSampler(local).start()
    warm_ms = []
    for _ in range(max(args.warmup, 3)):
        flush.fill_(1)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        step()
        b.record(stream)
        torch.cuda.synchronize()
        warm_ms.append(a.elapsed_time(b))
    ssd.ssd_get_device_status()
    steps = int(dist_max(float(pick_steps(args, warm_ms)), dev))
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    dist_barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    torch.cuda._sleep(20_000_000)  # let the host queue run ahead of the device
    for i in range(steps):
        flush.fill_(i & 0xFF)
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    dist_barrier()
    sampler.stop()
    ssd.ssd_get_device_status()
    per_step_ms = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    total_s = dist_max(sum(per_step_ms) / 1e3, dev)
    value = shape.tokens * world * steps / total_s
    peaks = load_peaks()
    abytes = bwd_bytes(shape)
    t_call = statistics.median(per_step_ms) / 1e3
    roofline = {"bound": "hbm", "achieved": abytes / t_call / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": abytes / t_call / 1e9 / peaks["hbm_gbs"], "traffic": None,
                "kernel": ("ssd_scan_bwd_complex" if shape.complex else "ssd_scan_bwd")
                + (" (7 launches, two of them tcgen05, timed as one call)" if shape.complex
                   or shape.nheads // shape.ngroups < 2 else " (8 launches, two of them tcgen05, timed as one call)"),
                "algorithmic_bytes_per_launch": abytes,
                "peak_source": f"{peaks['source']} (MEASURED_PEAKS.json burst)"
                if peaks["source"] == "measured" else "fallback (6.65 TB/s, 1.59 PFLOP/s)",
                "roofline_time_us": 1e6 * abytes / (peaks["hbm_gbs"] * 1e9), "kernel_time_us": 1e6 * t_call}

    e2e = None
    if not args.no_e2e:
        hin = {k: v.pin_memory() for k, v in list(inp.items()) + list(up.items()) if v is not None}
        dsets = [{k: (d[k] if k in d else u[k]) for k in hin}, {}]
        dsets[1] = {k: torch.empty_like(v) for k, v in dsets[0].items()}
        step()
        torch.cuda.synchronize()
        douts = [{k: v for k, v in out.items() if v is not None}, {}]
        douts[1] = {k: torch.empty_like(v) for k, v in douts[0].items()}
        hout = [{k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in o.items()} for o in douts]
        h2d = sum(v.numel() * v.element_size() for v in hin.values())
        d2h = sum(v.numel() * v.element_size() for v in hout[0].values())
        k_e2e = max(4, min(steps, 20))
        size_ws = ws.numel()
        ws2 = [ws, torch.zeros(size_ws, dtype=torch.uint8, device=dev)]

        def run(j):
            q = dsets[j]
            fn(q["x"], q["dt"], q["A"], q["B"], q["C"], q.get("D"), q.get("init_state"), q["dy"], q["dfinal"],
               out=dict(douts[j]), workspace=ws2[j])

        e2e_overlapped(hin, dsets, run, douts, hout, 2)
        dist_barrier()
        e2e_s = dist_max(e2e_overlapped(hin, dsets, run, douts, hout, k_e2e), dev)
        dist_barrier()
        e2e = {"value": shape.tokens * world * k_e2e / e2e_s, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "steps": k_e2e, "ms_per_step": 1e3 * e2e_s / k_e2e,
               "how": "two device buffer sets; H2D, compute and D2H on three streams, overlapped"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = bwd_cpu_baseline(shape)
        cpu.pop("seconds", None)
    line = {
        "metric": BWD_METRIC[shape.complex],
        "value": value, "unit": "tokens/s", "n_gpus": world, "steps": steps,
        "warmup": max(args.warmup, 3), "ms_per_step": 1e3 * total_s / steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic", "impl": "ours",
        "config": bwd_config(shape, world),
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "clocks": sampler.summary(t0, t1),
        # seven phases, and an eighth (C B^T once per group) when heads share a group
        "gpu_launches": (7 + (0 if shape.complex or shape.nheads // shape.ngroups < 2 else 1)) * steps,
        "step_ms_p10_p50_p90": [statistics.quantiles(per_step_ms, n=10)[0], statistics.median(per_step_ms),
                                statistics.quantiles(per_step_ms, n=10)[-1]],
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    import torch.distributed as dist

    if dist.is_initialized():
        dist.destroy_process_group()
    return 0


def bench_reference_bwd(args, shape):
    """The oracle's gradient on the host cores, a bounded sample per step."""
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    threads = oracle_threads()
    n = max(1, min(shape.batch * shape.nheads, 16, threads))
    units = [(i // shape.nheads, i % shape.nheads) for i in range(n)]
    steps = args.steps if args.steps is not None else 3
    secs = [bwd_cpu_units(shape, units, threads) for _ in range(steps)]
    tokens = shape.seqlen * n / shape.nheads
    value = tokens * steps / sum(secs)
    cpu = {"value": value, "unit": "tokens/s", "cores": min(threads, n), "kind": "oracle",
           "sample": f"{n} of {shape.batch * shape.nheads} (batch, head) sequences per step of {shape.name}"}
    line = {"metric": BWD_METRIC[shape.complex],
            "value": value, "unit": "tokens/s", "n_gpus": world, "steps": steps,
            "warmup": max(args.warmup, 3), "ms_per_step": 1e3 * sum(secs) / steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": bwd_config(shape, world),
            "cpu_baseline": cpu,
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: enough for ~0.12 s of timed device work, >= 100)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="mamba2-bitmamba1b-layer-bf16")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args(argv)
    from selective_state_space_22_b200 import inputs

    if args.workload in inputs.BWD_WORKLOADS:
        shape = inputs.BWD_WORKLOADS[args.workload]
        return bench_reference_bwd(args, shape) if args.impl == "reference" else bench_bwd(args, shape)
    if args.workload == inputs.DECODE.name:
        shape = inputs.DECODE
        return bench_reference_decode(args, shape) if args.impl == "reference" else bench_decode(args, shape)
    if args.workload in (inputs.MAMBA2_CONV.name, inputs.MAMBA1_50M.name):
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the variant workloads are timed against their "
                              "roofline only; their oracle is used for parity"}))
            return 0
        return bench_variant(args, args.workload)
    if args.workload == inputs.MAMBA3_PACKED.name:
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the packed-input workload has no separate "
                              "reference arm: the oracle of the complex workload covers the same scan"}))
            return 0
        return bench_packed(args, inputs.MAMBA3_PACKED)
    shape = inputs.WORKLOADS[args.workload]
    if args.impl == "reference":
        return bench_reference(args, shape)
    if shape is inputs.LONG and dist_env()[1] > 1:
        return bench_seqpar(args, shape)  # one long sequence split across the GPUs
    return bench_ours(args, shape)


if __name__ == "__main__":
    sys.exit(main())
