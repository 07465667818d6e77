"""The backward kernels' arithmetic, run on the CPU, against the fp64 adjoint.

`bwd_emul.cpp` runs the very phase functions the CUDA backward kernels call
(csrc/scan_bwd_body.cuh), block by block and thread by thread with a barrier
between phases, and with shared memory poisoned with NaN before every block.
This checks the kernels' indexing, masking of ragged chunks and arithmetic on a
machine without a GPU; launch configuration is left to the GPU tests.
Tolerance: float32 arithmetic against the fp64 oracle, 1e-4 normwise.
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest

import oracle
import pins

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "..", "selective_state_space_22_b200", "csrc")
F = ctypes.POINTER(ctypes.c_float)
TOL = 1e-4


@pytest.fixture(scope="module")
def emul(tmp_path_factory):
    out = str(tmp_path_factory.mktemp("bwd") / "libbwd_emul.so")
    subprocess.check_call(["g++", "-std=c++17", "-O2", "-fPIC", "-shared", "-I", CSRC, "-o", out,
                           os.path.join(HERE, "bwd_emul.cpp")])
    lib = ctypes.CDLL(out)
    lib.emulate_scan_bwd.argtypes = [F] * 16 + [ctypes.c_int] * 6
    lib.emulate_scan_bwd.restype = ctypes.c_int
    return lib


def _f32(a):
    return None if a is None else np.ascontiguousarray(a, np.float32)


def _p(a):
    return None if a is None else a.ctypes.data_as(F)


def run(emul, b, T, H, P, G, N, init=True, use_D=True, use_dfinal=True, seed=0, a_range=(1.0, 16.0)):
    rng = np.random.default_rng(seed)
    p = pins.rand_problem(rng, b, T, H, P, G, N, init=init, a_range=a_range)
    if not use_D:
        p["D"] = None
    # float32 values, widened exactly for the oracle
    p = {k: (None if v is None else _f32(v).astype(np.float64)) for k, v in p.items()}
    dy = _f32(rng.standard_normal((b, T, H, P))).astype(np.float64)
    dfinal = _f32(rng.standard_normal((b, H, P, N))).astype(np.float64) if use_dfinal else None
    ref = oracle.scan_bwd(p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"], p["init_state"], dy, dfinal)
    out = dict(dx=np.zeros((b, T, H, P), np.float32), ddt=np.zeros((b, T, H), np.float32),
               dA=np.zeros(H, np.float32), dB=np.zeros((b, T, G, N), np.float32),
               dC=np.zeros((b, T, G, N), np.float32), dD=np.zeros(H, np.float32),
               dinit=np.zeros((b, H, P, N), np.float32))
    args = [_f32(p["x"]), _f32(p["dt"]), _f32(p["A"]), _f32(p["B"]), _f32(p["C"]), _f32(p["D"]),
            _f32(p["init_state"]), _f32(dy), _f32(dfinal)]
    names = ("dx", "ddt", "dA", "dB", "dC", "dD", "dinit")
    rc = emul.emulate_scan_bwd(*[_p(a) for a in args], *[_p(out[k]) for k in names], b, T, H, P, G, N)
    assert rc == 0
    return {k: pins.rel_err(out[k], ref[k]) for k in names}


@pytest.mark.parametrize("T", [1, 63, 64, 65, 130, 200])
def test_ragged_and_multi_chunk(emul, T):
    errs = run(emul, 2, T, 4, 8, 2, 16, init=(T % 2 == 0), seed=T)
    assert max(errs.values()) <= TOL, errs


def test_mamba2_head_shape(emul):
    """Head dim 64 and d_state 128, the largest the kernels take, one group."""
    errs = run(emul, 1, 96, 2, 64, 1, 128, seed=3)
    assert max(errs.values()) <= TOL, errs


@pytest.mark.parametrize("G", [1, 3, 6])
def test_groups(emul, G):
    errs = run(emul, 1, 70, 6, 4, G, 8, seed=10 + G)
    assert max(errs.values()) <= TOL, errs


def test_optional_inputs_absent(emul):
    errs = run(emul, 2, 100, 2, 4, 1, 8, init=False, use_D=False, use_dfinal=False, seed=21)
    assert max(errs.values()) <= TOL, errs


def test_empty_sequence(emul):
    """T = 0: dinit = dfinal, dA = dD = 0."""
    errs = run(emul, 2, 0, 3, 4, 1, 8, seed=22)
    assert max(errs.values()) <= TOL, errs


def test_steep_decay(emul):
    """A in [-100, -40]: per-step decays far below one; nothing may overflow."""
    errs = run(emul, 1, 150, 2, 4, 1, 8, seed=23, a_range=(40.0, 100.0))
    assert max(errs.values()) <= TOL, errs
