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
    for name in ("emulate_scan_bwd_real", "emulate_scan_bwd_complex"):
        getattr(lib, name).argtypes = [F] * 16 + [ctypes.c_int] * 6
        getattr(lib, name).restype = ctypes.c_int
    return lib


def _f32(a):
    return None if a is None else np.ascontiguousarray(a, np.float32)


def _p(a):
    return None if a is None else a.ctypes.data_as(F)


def _c64(a):
    """complex128 -> interleaved float32 pairs (complex64 memory)."""
    return None if a is None else np.ascontiguousarray(a, np.complex64).view(np.float32)


def run(emul, b, T, H, P, G, N, init=True, use_D=True, use_dfinal=True, seed=0, a_range=(1.0, 16.0),
        cplx=False):
    rng = np.random.default_rng(seed)
    p = pins.rand_problem(rng, b, T, H, P, G, N, cplx=cplx, init=init, a_range=a_range)
    if not use_D:
        p["D"] = None
    # float32 / complex64 values, widened exactly for the oracle
    narrow = lambda v: v.astype(np.complex64 if np.iscomplexobj(v) else np.float32)
    p = {k: (None if v is None else np.ascontiguousarray(narrow(v).astype(
        np.complex128 if np.iscomplexobj(v) else np.float64))) for k, v in p.items()}
    dy = _f32(rng.standard_normal((b, T, H, P))).astype(np.float64)
    shp = (b, H, P, N)
    dfinal = None
    if use_dfinal:
        dfinal = rng.standard_normal(shp) + (1j * rng.standard_normal(shp) if cplx else 0)
        dfinal = np.ascontiguousarray(narrow(dfinal).astype(np.complex128 if cplx else np.float64))
    ref = oracle.scan_bwd(p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"], p["init_state"], dy, dfinal)
    sdt = np.complex64 if cplx else np.float32
    out = dict(dx=np.zeros((b, T, H, P), np.float32), ddt=np.zeros((b, T, H), np.float32),
               dA=np.zeros(H, sdt), dB=np.zeros((b, T, G, N), sdt), dC=np.zeros((b, T, G, N), sdt),
               dD=np.zeros(H, np.float32), dinit=np.zeros((b, H, P, N), sdt))
    st = _c64 if cplx else _f32
    args = [_f32(p["x"]), _f32(p["dt"]), st(p["A"]), st(p["B"]), st(p["C"]), _f32(p["D"]),
            st(p["init_state"]), _f32(dy), st(dfinal)]
    names = ("dx", "ddt", "dA", "dB", "dC", "dD", "dinit")
    fn = emul.emulate_scan_bwd_complex if cplx else emul.emulate_scan_bwd_real
    outp = [(out[k].view(np.float32) if out[k].dtype == np.complex64 else out[k]) for k in names]
    rc = fn(*[_p(a) for a in args], *[_p(o) for o in outp], b, T, H, P, G, N)
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


# ------------------------------------------------------------------ complex
@pytest.mark.parametrize("T", [1, 31, 32, 33, 100])
def test_complex_ragged_and_multi_chunk(emul, T):
    errs = run(emul, 2, T, 4, 8, 2, 16, init=(T % 2 == 1), seed=40 + T, cplx=True)
    assert max(errs.values()) <= TOL, errs


def test_complex_mamba3lite_head_shape(emul):
    """Head dim 64 and complex d_state 64 (the Mamba-3-Lite head), one group per head."""
    errs = run(emul, 1, 70, 2, 64, 2, 64, seed=50, cplx=True)
    assert max(errs.values()) <= TOL, errs


def test_complex_optional_inputs_absent_and_empty(emul):
    errs = run(emul, 2, 50, 2, 4, 1, 8, init=False, use_D=False, use_dfinal=False, seed=51, cplx=True)
    assert max(errs.values()) <= TOL, errs
    errs = run(emul, 2, 0, 3, 4, 1, 8, seed=52, cplx=True)
    assert max(errs.values()) <= TOL, errs


def _run_custom(emul, p, dy, dfinal, cplx=False):
    """Run the phases on a given float32/complex64-exact problem and return the errors."""
    ref = oracle.scan_bwd(p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"], p["init_state"], dy, dfinal)
    b, T, H, P = p["x"].shape
    G, N = p["B"].shape[2], p["B"].shape[3]
    sdt = np.complex64 if cplx else np.float32
    out = dict(dx=np.zeros((b, T, H, P), np.float32), ddt=np.zeros((b, T, H), np.float32),
               dA=np.zeros(H, sdt), dB=np.zeros((b, T, G, N), sdt), dC=np.zeros((b, T, G, N), sdt),
               dD=np.zeros(H, np.float32), dinit=np.zeros((b, H, P, N), sdt))
    st = _c64 if cplx else _f32
    args = [_f32(p["x"]), _f32(p["dt"]), st(p["A"]), st(p["B"]), st(p["C"]), _f32(p["D"]),
            st(p["init_state"]), _f32(dy), st(dfinal)]
    names = ("dx", "ddt", "dA", "dB", "dC", "dD", "dinit")
    fn = emul.emulate_scan_bwd_complex if cplx else emul.emulate_scan_bwd_real
    outp = [(out[k].view(np.float32) if out[k].dtype == np.complex64 else out[k]) for k in names]
    assert fn(*[_p(a) for a in args], *[_p(o) for o in outp], b, T, H, P, G, N) == 0
    return {k: pins.rel_err(out[k], ref[k]) for k in names}


def _exact(p):
    narrow = lambda v: v.astype(np.complex64 if np.iscomplexobj(v) else np.float32)
    return {k: (None if v is None else np.ascontiguousarray(narrow(v).astype(
        np.complex128 if np.iscomplexobj(v) else np.float64))) for k, v in p.items()}


@pytest.mark.parametrize("cplx", [False, True])
def test_zero_dt_tokens_inside_the_sequence(emul, cplx):
    """dt = 0 on some valid tokens: no decay and no input there, but D x still
    reaches y, so dx keeps its D dy part."""
    rng = np.random.default_rng(60)
    p = pins.rand_problem(rng, 1, 90, 2, 4, 1, 8, cplx=cplx, init=True)
    p["dt"][0, ::7, :] = 0.0
    p = _exact(p)
    dy = rng.standard_normal((1, 90, 2, 4)).astype(np.float32).astype(np.float64)
    dfinal = rng.standard_normal((1, 2, 4, 8)) + (1j * rng.standard_normal((1, 2, 4, 8)) if cplx else 0)
    dfinal = _exact({"d": dfinal})["d"]
    errs = _run_custom(emul, p, dy, dfinal, cplx)
    assert max(errs.values()) <= TOL, errs


@pytest.mark.parametrize("cplx", [False, True])
def test_no_decay(emul, cplx):
    """A = 0 (real part 0 for complex: a pure rotation): the state never decays."""
    rng = np.random.default_rng(61)
    p = pins.rand_problem(rng, 1, 80, 2, 4, 1, 8, cplx=cplx, init=True)
    p["A"] = (1j * p["A"].imag) if cplx else np.zeros_like(p["A"])
    p = _exact(p)
    dy = rng.standard_normal((1, 80, 2, 4)).astype(np.float32).astype(np.float64)
    errs = _run_custom(emul, p, dy, None, cplx)
    assert max(errs.values()) <= TOL, errs
