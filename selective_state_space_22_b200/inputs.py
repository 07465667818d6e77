"""Seeded synthetic inputs for the scan and the decode step.

This module is the only thing the CUDA path and the oracle share.  It draws
random tensors on the CPU with a seeded ``torch.Generator`` and casts them to
the dtypes each workload uses; it holds none of the scan's arithmetic.

Recipes (the workloads are Mamba-2 / Mamba-3-Lite layer shapes; none of the
pages publishes data for the scan, so every input is synthetic):

* x, B, C ~ N(0, 1) (complex B, C: real and imaginary parts each N(0, 1/2),
  so E|B|^2 = 1);
* dt = clamp(softplus(z + dt_bias_h), 1e-3, 0.1), z ~ N(0, 1), with
  dt_bias_h = log(expm1(dt0_h)) and dt0_h log-uniform in [1e-3, 0.1]: dt is
  what the caller hands the scan after softplus and dt_bias;
* real A_h = -exp(A_log_h), A_log_h = log U[1, 16], so A_h in [-16, -1];
  complex A_h = -U[0.5, 2] + i U[-pi, pi];
* D_h ~ N(0, 1); the initial state is zero unless asked for, then N(0, 1)
  (complex: N(0, 1/2) per part).

Draw order from one generator: x, z, dt0, A, B, C, D, init.  The seed of the
k-th named workload is 20261202 + k.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

SEED_BASE = 20261202


@dataclass(frozen=True)
class ScanShape:
    name: str
    batch: int
    seqlen: int
    nheads: int
    headdim: int
    ngroups: int
    dstate: int
    chunk: int
    io_dtype: str          # "f32" or "bf16" for x, B, C, y (complex: always f32)
    complex: bool = False
    init_state: bool = False
    seed: int = SEED_BASE

    @property
    def tokens(self) -> int:
        return self.batch * self.seqlen


@dataclass(frozen=True)
class DecodeShape:
    name: str
    batch: int
    nheads: int
    headdim: int
    ngroups: int
    dstate: int
    steps: int
    io_dtype: str = "bf16"
    seed: int = SEED_BASE + 4


# The five named workloads: tiny real, Mamba-2 BitMamba-1B layer, Mamba-3-Lite
# complex layer, long-sequence real, and decode at the BitMamba-1B shape.
TINY = ScanShape("tiny-real-f32", 1, 256, 2, 16, 1, 8, 64, "f32", seed=SEED_BASE + 0)
MAMBA2_1B = ScanShape("mamba2-bitmamba1b-layer-bf16", 2, 2048, 64, 64, 1, 128, 256, "bf16",
                      seed=SEED_BASE + 1)
MAMBA3_COMPLEX = ScanShape("mamba3lite-complex-f32", 4, 2048, 16, 64, 16, 64, 256, "f32",
                           complex=True, seed=SEED_BASE + 2)
LONG = ScanShape("mamba2-long-65536-bf16", 1, 65536, 64, 64, 1, 128, 256, "bf16",
                 init_state=True, seed=SEED_BASE + 3)
DECODE = DecodeShape("decode-bitmamba1b-256seq", 256, 64, 64, 1, 128, 1024)

WORKLOADS = {w.name: w for w in (TINY, MAMBA2_1B, MAMBA3_COMPLEX, LONG)}

# Gradients through the scan at the Mamba-2 layer shape, float32 (the backward
# takes float32 tensors); dy and dfinal from bwd_upstream.
BWD = ScanShape("mamba2-bitmamba1b-layer-bwd-f32", 2, 2048, 64, 64, 1, 128, 64, "f32",
                init_state=True, seed=SEED_BASE + 5)


# The same at the Mamba-3-Lite complex layer shape (32-token chunks).
BWD_COMPLEX = ScanShape("mamba3lite-complex-bwd-f32", 4, 2048, 16, 64, 16, 64, 32, "f32",
                        complex=True, init_state=True, seed=SEED_BASE + 6)
BWD_WORKLOADS = {w.name: w for w in (BWD, BWD_COMPLEX)}


def bwd_upstream(shape: ScanShape) -> dict:
    """The gradients arriving at y and final_state: dy [b,T,H,P] float32 N(0,1)
    and dfinal [b,H,P,N] (float32 N(0,1), or complex64 with re/im N(0,1/2) for a
    complex workload), seeded from the workload's seed."""
    gen = torch.Generator().manual_seed(shape.seed + 1000)
    b, T, H, P, N = shape.batch, shape.seqlen, shape.nheads, shape.headdim, shape.dstate
    dy = torch.randn((b, T, H, P), generator=gen)
    if shape.complex:
        re = torch.randn((b, H, P, N), generator=gen) * 0.5 ** 0.5
        im = torch.randn((b, H, P, N), generator=gen) * 0.5 ** 0.5
        return {"dy": dy, "dfinal": torch.complex(re, im)}
    return {"dy": dy, "dfinal": torch.randn((b, H, P, N), generator=gen)}


def _tdtype(name: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def _dt_draw(gen, shape, nheads):
    z = torch.randn(shape, generator=gen, dtype=torch.float32)
    lo, hi = math.log(1e-3), math.log(0.1)
    dt0 = torch.exp(torch.rand(nheads, generator=gen, dtype=torch.float32) * (hi - lo) + lo)
    dt_bias = torch.log(torch.expm1(dt0))
    return torch.nn.functional.softplus(z + dt_bias).clamp(1e-3, 0.1).contiguous()


def _real_A(gen, nheads):
    a_log = torch.log(torch.rand(nheads, generator=gen, dtype=torch.float32) * 15.0 + 1.0)
    return (-torch.exp(a_log)).contiguous()


def _complex_A(gen, nheads):
    re = -(torch.rand(nheads, generator=gen, dtype=torch.float32) * 1.5 + 0.5)
    im = (torch.rand(nheads, generator=gen, dtype=torch.float32) * 2.0 - 1.0) * math.pi
    return torch.complex(re, im).contiguous()


def _cnormal(gen, shape):
    s = 1.0 / math.sqrt(2.0)
    re = torch.randn(shape, generator=gen, dtype=torch.float32) * s
    im = torch.randn(shape, generator=gen, dtype=torch.float32) * s
    return torch.complex(re, im).contiguous()


def scan_inputs(shape: ScanShape, seqlen: int | None = None, batch: int | None = None) -> dict:
    """CPU tensors for one scan call, in the dtypes the library takes.

    ``seqlen``/``batch`` override the shape's sizes (the draw order is kept, so
    a shorter override is not a prefix of the longer one).
    """
    b = shape.batch if batch is None else batch
    T = shape.seqlen if seqlen is None else seqlen
    H, P, G, N = shape.nheads, shape.headdim, shape.ngroups, shape.dstate
    gen = torch.Generator().manual_seed(shape.seed)
    io = torch.float32 if shape.complex else _tdtype(shape.io_dtype)
    x = torch.randn((b, T, H, P), generator=gen, dtype=torch.float32).to(io).contiguous()
    dt = _dt_draw(gen, (b, T, H), H)
    if shape.complex:
        A = _complex_A(gen, H)
        B = _cnormal(gen, (b, T, G, N))
        C = _cnormal(gen, (b, T, G, N))
    else:
        A = _real_A(gen, H)
        B = torch.randn((b, T, G, N), generator=gen, dtype=torch.float32).to(io).contiguous()
        C = torch.randn((b, T, G, N), generator=gen, dtype=torch.float32).to(io).contiguous()
    D = torch.randn(H, generator=gen, dtype=torch.float32)
    init = None
    if shape.init_state:
        if shape.complex:
            init = _cnormal(gen, (b, H, P, N))
        else:
            init = torch.randn((b, H, P, N), generator=gen, dtype=torch.float32)
    return {"x": x, "dt": dt, "A": A, "B": B, "C": C, "D": D, "init_state": init}


def packed_inputs(shape: ScanShape, proj_dtype: str = "f32") -> dict:
    """Inputs of the packed complex scan: the projection output proj
    [b, T, H (P + 4N + 1)] in head-major slices x | Re B | Im B | Re C | Im C | dt
    ("Block Anatomy, Numerical Stability & Scaling", Block Anatomy 4.1-4.2), and
    dt_bias, A, D and the initial state.  x ~ N(0, 1); the B and C slices
    N(0, 1/2) (so E|B|^2 = 1); the dt slice N(0, 1) before the bias;
    dt_bias_h = log(expm1(dt0_h)) with dt0_h log-uniform in [1e-3, 0.1] (the
    scan applies softplus(dt + dt_bias) itself).  One group per head."""
    b, T, H, P, N = shape.batch, shape.seqlen, shape.nheads, shape.headdim, shape.dstate
    gen = torch.Generator().manual_seed(shape.seed)
    s = 1.0 / math.sqrt(2.0)
    x = torch.randn((b, T, H * P), generator=gen)
    bc = torch.randn((b, T, 4 * H * N), generator=gen) * s
    z = torch.randn((b, T, H), generator=gen)
    lo, hi = math.log(1e-3), math.log(0.1)
    dt0 = torch.exp(torch.rand(H, generator=gen) * (hi - lo) + lo)
    dt_bias = torch.log(torch.expm1(dt0))
    A = _complex_A(gen, H)
    D = torch.randn(H, generator=gen)
    init = _cnormal(gen, (b, H, P, N)) if shape.init_state else None
    proj = torch.cat([x, bc, z], dim=-1).to(_tdtype(proj_dtype)).contiguous()
    return {"proj": proj, "dt_bias": dt_bias.contiguous(), "A": A, "D": D, "init_state": init}


def unpack_projection(proj: torch.Tensor, nheads: int, headdim: int, dstate: int) -> dict:
    """The slices of a packed projection output as separate CPU tensors (x
    [b,T,H,P], B and C complex [b,T,H,N], raw dt [b,T,H]), widened exactly to
    float64 / complex128: how the block unpacks them before a scan that takes
    separate tensors.  Slicing only, no scan arithmetic."""
    b, T, _ = proj.shape
    H, P, N = nheads, headdim, dstate
    p = proj.to(torch.float64)
    o = [0, H * P, H * P + H * N, H * P + 2 * H * N, H * P + 3 * H * N, H * P + 4 * H * N]
    x = p[..., o[0]:o[1]].reshape(b, T, H, P)
    B = torch.complex(p[..., o[1]:o[2]], p[..., o[2]:o[3]]).reshape(b, T, H, N)
    C = torch.complex(p[..., o[3]:o[4]], p[..., o[4]:o[5]]).reshape(b, T, H, N)
    dt_raw = p[..., o[5]:]
    return {"x": x.contiguous(), "B": B.contiguous(), "C": C.contiguous(), "dt_raw": dt_raw.contiguous()}


# The Mamba-3-Lite layer fed from its packed projection output, bf16 (the
# projection's dtype under the block's bf16 autocast).
MAMBA3_PACKED = ScanShape("mamba3lite-complex-packed-bf16", 4, 2048, 16, 64, 16, 64, 256, "bf16", complex=True,
                          seed=SEED_BASE + 7)


@dataclass(frozen=True)
class ConvShape:
    """The causal conv1d prologue over packed x | B | C channels."""
    name: str
    batch: int
    seqlen: int
    x_channels: int
    bc_channels: int
    width: int
    io_dtype: str
    silu: bool = True
    init: bool = False
    seed: int = SEED_BASE + 8


@dataclass(frozen=True)
class SelectiveShape:
    """The Mamba-1 selective scan (per-state A)."""
    name: str
    batch: int
    seqlen: int
    channels: int
    ngroups: int
    dstate: int
    io_dtype: str
    init_state: bool = False
    seed: int = SEED_BASE + 9

    @property
    def tokens(self) -> int:
        return self.batch * self.seqlen


# The BitMamba-1B layer's prologue: x (64 heads x 64) and B, C (one group x 128)
# channels, kernel 4, SiLU.
MAMBA2_CONV = ConvShape("mamba2-conv1d-bitmamba1b-bf16", 2, 2048, 4096, 128, 4, "bf16")
# A Mamba-1 layer at the "Mamba-50M" card's batch (64) and context (512); the
# card gives no widths, so d_inner 1024 and d_state 16 (the Mamba-1 default).
MAMBA1_50M = SelectiveShape("mamba1-50m-layer-bf16", 64, 512, 1024, 1, 16, "bf16")


def conv_inputs(shape: ConvShape) -> dict:
    """xbc [b,T,Cx+2Cb] ~ N(0,1), weight [C,K] ~ N(0, 1/K), bias [C] ~ N(0, 0.1^2),
    conv_init [b,C,K-1] ~ N(0,1) when asked for."""
    gen = torch.Generator().manual_seed(shape.seed)
    Ct = shape.x_channels + 2 * shape.bc_channels
    io = _tdtype(shape.io_dtype)
    xbc = torch.randn((shape.batch, shape.seqlen, Ct), generator=gen).to(io).contiguous()
    w = (torch.randn((Ct, shape.width), generator=gen) / math.sqrt(shape.width)).contiguous()
    bias = (torch.randn(Ct, generator=gen) * 0.1).contiguous()
    init = None
    if shape.init:
        init = torch.randn((shape.batch, Ct, shape.width - 1), generator=gen).to(io).contiguous()
    return {"xbc": xbc, "weight": w, "bias": bias, "conv_init": init}


def selective_inputs(shape: SelectiveShape) -> dict:
    """x, B, C ~ N(0,1) (io dtype); dt as for the scans (c12 recipe, per channel);
    A[d,n] = -U[1,16] per state; D ~ N(0,1); init N(0,1) when asked for."""
    gen = torch.Generator().manual_seed(shape.seed)
    b, T, Dc, G, N = shape.batch, shape.seqlen, shape.channels, shape.ngroups, shape.dstate
    io = _tdtype(shape.io_dtype)
    x = torch.randn((b, T, Dc), generator=gen).to(io).contiguous()
    dt = _dt_draw(gen, (b, T, Dc), Dc)
    A = (-(torch.rand((Dc, N), generator=gen) * 15.0 + 1.0)).contiguous()
    B = torch.randn((b, T, G, N), generator=gen).to(io).contiguous()
    C = torch.randn((b, T, G, N), generator=gen).to(io).contiguous()
    D = torch.randn(Dc, generator=gen)
    init = torch.randn((b, Dc, N), generator=gen) if shape.init_state else None
    return {"x": x, "dt": dt, "A": A, "B": B, "C": C, "D": D, "init_state": init}


def decode_step_inputs(gen: torch.Generator, shape: DecodeShape) -> dict:
    """Per-step decode inputs x [b,H,P], dt [b,H], B, C [b,G,N] (io dtype)."""
    b, H, P, G, N = shape.batch, shape.nheads, shape.headdim, shape.ngroups, shape.dstate
    io = _tdtype(shape.io_dtype)
    x = torch.randn((b, H, P), generator=gen, dtype=torch.float32).to(io).contiguous()
    dt = _dt_draw(gen, (b, H), H)
    B = torch.randn((b, G, N), generator=gen, dtype=torch.float32).to(io).contiguous()
    C = torch.randn((b, G, N), generator=gen, dtype=torch.float32).to(io).contiguous()
    return {"x": x, "dt": dt, "B": B, "C": C}


def decode_setup(shape: DecodeShape) -> tuple[torch.Generator, dict]:
    """Generator positioned after the per-call constants, plus A, D and the state."""
    gen = torch.Generator().manual_seed(shape.seed)
    H, P, N = shape.nheads, shape.headdim, shape.dstate
    A = _real_A(gen, H)
    D = torch.randn(H, generator=gen, dtype=torch.float32)
    state = torch.randn((shape.batch, H, P, N), generator=gen, dtype=torch.float32)
    return gen, {"A": A, "D": D, "state": state}


def widen(t) -> np.ndarray | None:
    """Exact fp64 (complex128) numpy copy of a CPU tensor, for the oracle."""
    if t is None:
        return None
    if t.is_complex():
        return np.ascontiguousarray(t.to(torch.complex128).numpy())
    return np.ascontiguousarray(t.to(torch.float64).numpy())


def widen_all(inp: dict) -> dict:
    return {k: widen(v) for k, v in inp.items()}
