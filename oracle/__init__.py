"""ctypes wrapper around the fp64 sequential oracle (``ssd_oracle.c``).

TEST INFRASTRUCTURE ONLY.  This package may be imported by ``tests/``, by the
package's ``smoke()`` check and by the CPU-baseline leg of ``bench.py``, and by
nothing else.  It shares no code with the CUDA library: both sides only see the
same seeded inputs.

All arrays are numpy, C-contiguous; real data is float64 and complex data is
complex128 (interleaved re/im doubles, the layout the C file reads).  Inputs
that were bf16 on the GPU side are passed here widened to float64 exactly.

Reference: "Mamba-3-Lite" README (the recurrence section) and "Block Anatomy,
Numerical Stability & Scaling" (Numerical Stability, section 4); the C file
header lists the readings taken.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssd_oracle.c")
_LIB = os.path.join(_HERE, "libssd_oracle.so")
_lock = threading.Lock()
_lib = None

_D = ctypes.POINTER(ctypes.c_double)
_L = ctypes.c_long


def build(force: bool = False, src: str = _SRC, out: str = _LIB) -> str:
    """Compile the oracle with gcc (-O2, no fast-math: fp64 semantics kept)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-std=c99", "-O2", "-fPIC", "-shared",
                               "-fno-fast-math", "-o", tmp, src, "-lm"])
        os.replace(tmp, out)
    return out


def load(path: str | None = None):
    """Load (building first if needed) and declare the oracle's entry points."""
    global _lib
    if path is None:
        with _lock:
            if _lib is None:
                _lib = _declare(ctypes.CDLL(build()))
            return _lib
    return _declare(ctypes.CDLL(path))


def _declare(lib):
    scan_args = [_D, _D, _D, _D, _D, _D, _D, _D, _D, _L, _L, _L, _L, _L, _L]
    upd_args = [_D, _D, _D, _D, _D, _D, _D, _D, _L, _L, _L, _L, _L]
    for name in ("oracle_scan_real", "oracle_scan_complex"):
        getattr(lib, name).argtypes = scan_args
        getattr(lib, name).restype = ctypes.c_int
    for name in ("oracle_state_update_real", "oracle_state_update_complex"):
        getattr(lib, name).argtypes = upd_args
        getattr(lib, name).restype = ctypes.c_int
    lib.oracle_causal_conv1d.argtypes = [_D, _D, _D, _D, ctypes.c_int, _D, _L, _L, _L, _L]
    lib.oracle_causal_conv1d.restype = ctypes.c_int
    lib.oracle_selective_scan.argtypes = [_D] * 9 + [_L] * 5
    lib.oracle_selective_scan.restype = ctypes.c_int
    bwd_args = [_D] * 16 + [_L] * 6
    for name in ("oracle_scan_bwd_real", "oracle_scan_bwd_complex"):
        getattr(lib, name).argtypes = bwd_args
        getattr(lib, name).restype = ctypes.c_int
    return lib


def _ptr(a, dtype):
    if a is None:
        return None
    assert a.dtype == dtype and a.flags["C_CONTIGUOUS"], (a.dtype, a.flags)
    return a.ctypes.data_as(_D)


def scan(x, dt, A, B, C, D=None, init_state=None, ngroups=None, lib=None):
    """Run the sequential scan.  Complex variant when A is complex.

    x [b,T,H,P] float64, dt [b,T,H] float64, A [H] (float64 or complex128),
    B, C [b,T,G,N] (float64 or complex128), D [H] float64 or None,
    init_state [b,H,P,N] (float64 or complex128) or None.
    Returns (y [b,T,H,P] float64, final_state [b,H,P,N]).
    """
    lib = lib or load()
    cplx = np.iscomplexobj(A)
    sdt = np.complex128 if cplx else np.float64
    b, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    y = np.zeros((b, T, H, P), np.float64)
    fs = np.zeros((b, H, P, N), sdt)
    fn = lib.oracle_scan_complex if cplx else lib.oracle_scan_real
    rc = fn(_ptr(x, np.float64), _ptr(dt, np.float64), _ptr(A, sdt), _ptr(B, sdt),
            _ptr(C, sdt), _ptr(D, np.float64), _ptr(init_state, sdt),
            _ptr(y, np.float64), _ptr(fs, sdt), b, T, H, P, G, N)
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return y, fs


def state_update(state, x, dt, A, B, C, D=None, lib=None):
    """One decoding step.  Returns (y [b,H,P], new state); the input is not modified.

    state [b,H,P,N], x [b,H,P], dt [b,H], A [H], B, C [b,G,N], D [H] or None.
    """
    lib = lib or load()
    cplx = np.iscomplexobj(A)
    sdt = np.complex128 if cplx else np.float64
    st = np.array(state, dtype=sdt, copy=True, order="C")
    b, H, P, N = st.shape
    G = B.shape[1]
    y = np.zeros((b, H, P), np.float64)
    fn = lib.oracle_state_update_complex if cplx else lib.oracle_state_update_real
    rc = fn(_ptr(st, sdt), _ptr(x, np.float64), _ptr(dt, np.float64), _ptr(A, sdt),
            _ptr(B, sdt), _ptr(C, sdt), _ptr(D, np.float64), _ptr(y, np.float64),
            b, H, P, G, N)
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return y, st


def scan_bwd(x, dt, A, B, C, D, init_state, dy, dfinal=None, lib=None):
    """Gradients of L = sum <dy, y> + Re <dfinal, final_state> through the scan.

    Same inputs as ``scan``; dy [b,T,H,P] float64, dfinal [b,H,P,N] (state
    dtype) or None.  Returns a dict with dx, ddt, dA, dB, dC, dD and dinit,
    shaped like x, dt, A, B, C, D [H] and the state.  For complex tensors the
    gradient of z = u + iv is dL/du + i dL/dv.
    """
    lib = lib or load()
    cplx = np.iscomplexobj(A)
    sdt = np.complex128 if cplx else np.float64
    b, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    out = dict(dx=np.zeros_like(x), ddt=np.zeros_like(dt), dA=np.zeros(H, sdt),
               dB=np.zeros((b, T, G, N), sdt), dC=np.zeros((b, T, G, N), sdt),
               dD=np.zeros(H, np.float64), dinit=np.zeros((b, H, P, N), sdt))
    fn = lib.oracle_scan_bwd_complex if cplx else lib.oracle_scan_bwd_real
    rc = fn(_ptr(x, np.float64), _ptr(dt, np.float64), _ptr(A, sdt), _ptr(B, sdt),
            _ptr(C, sdt), _ptr(D, np.float64), _ptr(init_state, sdt), _ptr(dy, np.float64),
            _ptr(dfinal, sdt), _ptr(out["dx"], np.float64), _ptr(out["ddt"], np.float64),
            _ptr(out["dA"], sdt), _ptr(out["dB"], sdt), _ptr(out["dC"], sdt),
            _ptr(out["dD"], np.float64), _ptr(out["dinit"], sdt), b, T, H, P, G, N)
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return out


def causal_conv1d(x, w, bias=None, init=None, silu=False, lib=None):
    """Causal depthwise convolution, x [b,T,C] float64, w [C,K], bias [C],
    init [b,C,K-1] (the inputs before t = 0) or None.  Returns out [b,T,C]."""
    lib = lib or load()
    b, T, Cn = x.shape
    K = w.shape[1]
    out = np.zeros((b, T, Cn), np.float64)
    rc = lib.oracle_causal_conv1d(_ptr(x, np.float64), _ptr(w, np.float64), _ptr(bias, np.float64),
                                  _ptr(init, np.float64), int(bool(silu)), _ptr(out, np.float64), b, T, Cn, K)
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return out


def selective_scan(x, dt, A, B, C, D=None, init_state=None, lib=None):
    """Mamba-1 selective scan with a per-state A: x, dt [b,T,Dc], A [Dc,N],
    B, C [b,T,G,N], D [Dc], init_state [b,Dc,N].  Returns (y [b,T,Dc],
    final_state [b,Dc,N])."""
    lib = lib or load()
    b, T, Dc = x.shape
    G, N = B.shape[2], B.shape[3]
    y = np.zeros((b, T, Dc), np.float64)
    fs = np.zeros((b, Dc, N), np.float64)
    rc = lib.oracle_selective_scan(_ptr(x, np.float64), _ptr(dt, np.float64), _ptr(A, np.float64),
                                   _ptr(B, np.float64), _ptr(C, np.float64), _ptr(D, np.float64),
                                   _ptr(init_state, np.float64), _ptr(y, np.float64), _ptr(fs, np.float64),
                                   b, T, Dc, G, N)
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return y, fs
