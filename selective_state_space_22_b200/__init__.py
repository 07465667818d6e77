"""B200-native chunked selective state-space (SSD) scan.

All arithmetic runs in ``libssd.so`` (hand-written CUDA for sm_100a behind the
C ABI of ``include/ssd.h``).  The functions here have the C entry points'
names and only marshal arguments: they check that the torch tensors are CUDA,
contiguous and of the right dtype, pass their device pointers and the current
stream, and raise :class:`SSDError` on a non-OK status.  There is no fallback:
if the library is missing, every call raises.

    y, h_T = ssd_scan_fwd(x, dt, A, B, C, D, init_state, chunk_size=256)
    y, h_T = ssd_scan_fwd_complex(x, dt, A, B, C, D, init_state)
    y = ssd_state_update(state, x, dt, A, B, C, D)          # state updated in place
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

__all__ = ["SSDError", "ssd_scan_fwd", "ssd_scan_fwd_complex", "ssd_state_update",
           "ssd_state_update_complex", "ssd_scan_workspace_size", "ssd_scan_kernel_launches", "ssd_get_device_status",
           "ssd_scan_fwd_noalloc", "ssd_last_error", "ssd_version", "load_library", "LIB_PATH",
           "SSD_WORKSPACE_INVALID", "ssd_scan_bwd", "ssd_scan_bwd_workspace_size",
           "ssd_scan_bwd_complex", "ssd_scan_bwd_complex_workspace_size"]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libssd.so")

SSD_OK, SSD_ERR_INVALID_ARG, SSD_ERR_UNSUPPORTED, SSD_ERR_CUDA, SSD_ERR_TIMEOUT, SSD_ERR_WORKSPACE = range(6)
SSD_F32, SSD_BF16 = 0, 1
_STATUS = {0: "SSD_OK", 1: "SSD_ERR_INVALID_ARG", 2: "SSD_ERR_UNSUPPORTED", 3: "SSD_ERR_CUDA",
           4: "SSD_ERR_TIMEOUT", 5: "SSD_ERR_WORKSPACE"}


class SSDError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{_STATUS.get(status, status)}: {message}")
        self.status = status


_lib = None
_lock = threading.Lock()
_VP, _FP, _I, _SZ = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t


def load_library(path: str | None = None):
    """Load libssd.so and declare its C signatures (raises if it is not built)."""
    global _lib
    with _lock:
        if _lib is not None and path is None:
            return _lib
        p = path or LIB_PATH
        if not os.path.exists(p):
            raise RuntimeError(f"{p} is missing: build it with "
                               "`python -m selective_state_space_22_b200.build`")
        lib = ctypes.CDLL(p)
        lib.ssd_scan_workspace_size.argtypes = [_I] * 8 + [_I]
        lib.ssd_scan_workspace_size.restype = _SZ
        lib.ssd_scan_kernel_launches.argtypes = [_I] * 9
        lib.ssd_scan_kernel_launches.restype = _I
        lib.ssd_scan_fwd.argtypes = [_VP] * 9 + [_I] * 8 + [_VP, _SZ, _VP]
        lib.ssd_scan_fwd.restype = _I
        lib.ssd_scan_fwd_complex.argtypes = [_VP] * 9 + [_I] * 7 + [_VP, _SZ, _VP]
        lib.ssd_scan_fwd_complex.restype = _I
        lib.ssd_state_update.argtypes = [_VP] * 8 + [_I] * 6 + [_VP]
        lib.ssd_state_update.restype = _I
        lib.ssd_state_update_complex.argtypes = [_VP] * 8 + [_I] * 5 + [_VP]
        lib.ssd_state_update_complex.restype = _I
        lib.ssd_scan_fwd_noalloc.argtypes = [_VP] * 9 + [_I] * 8 + [_VP]
        lib.ssd_scan_fwd_noalloc.restype = _I
        lib.ssd_scan_bwd_workspace_size.argtypes = [_I] * 6
        lib.ssd_scan_bwd_workspace_size.restype = _SZ
        lib.ssd_scan_bwd.argtypes = [_VP] * 16 + [_I] * 6 + [_VP, _SZ, _VP]
        lib.ssd_scan_bwd.restype = _I
        lib.ssd_scan_bwd_complex_workspace_size.argtypes = [_I] * 6
        lib.ssd_scan_bwd_complex_workspace_size.restype = _SZ
        lib.ssd_scan_bwd_complex.argtypes = [_VP] * 16 + [_I] * 6 + [_VP, _SZ, _VP]
        lib.ssd_scan_bwd_complex.restype = _I
        lib.ssd_debug_inject_stall.argtypes = [_I, ctypes.c_ulonglong]
        lib.ssd_debug_inject_stall.restype = _I
        lib.ssd_get_device_status.argtypes = [_VP]
        lib.ssd_get_device_status.restype = _I
        lib.ssd_last_error.argtypes = []
        lib.ssd_last_error.restype = ctypes.c_char_p
        lib.ssd_version.argtypes = []
        lib.ssd_version.restype = ctypes.c_char_p
        if path is None:
            _lib = lib
        return lib


def ssd_last_error() -> str:
    return load_library().ssd_last_error().decode()


def ssd_version() -> str:
    return load_library().ssd_version().decode()


def _check(status: int):
    if status != SSD_OK:
        raise SSDError(status, ssd_last_error())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, name, dtype, device, shape=None, allow_none=False):
    if t is None:
        if allow_none:
            return
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


_ws_cache: dict = {}


def _workspace(device, nbytes: int):
    """A cached per-device workspace of at least nbytes (no initialisation needed)."""
    if nbytes == 0:
        return None
    key = device.index
    buf = _ws_cache.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.zeros(max(nbytes, 1 << 20), dtype=torch.uint8, device=device)
        _ws_cache[key] = buf
    return buf


SSD_WORKSPACE_INVALID = (1 << 64) - 1  # (size_t)-1: sizes that no scan accepts


def ssd_scan_workspace_size(batch, seqlen, nheads, headdim, ngroups, dstate, chunk_size,
                            is_complex=False, io_dtype=SSD_BF16) -> int:
    """Workspace bytes the scan needs (0: none); SSD_WORKSPACE_INVALID for invalid sizes."""
    return int(load_library().ssd_scan_workspace_size(batch, seqlen, nheads, headdim, ngroups,
                                                      dstate, chunk_size, int(bool(is_complex)),
                                                      io_dtype))


def ssd_scan_kernel_launches(batch, seqlen, nheads, headdim, ngroups, dstate, chunk_size,
                             is_complex=False, io_dtype=SSD_BF16) -> int:
    return int(load_library().ssd_scan_kernel_launches(batch, seqlen, nheads, headdim, ngroups,
                                                       dstate, chunk_size, int(bool(is_complex)),
                                                       io_dtype))


def ssd_scan_fwd(x, dt, A, B, C, D=None, init_state=None, *, chunk_size=256, y=None,
                 final_state=None, return_final_state=True, workspace=None, stream=None):
    """Real chunked scan.  Returns (y, final_state or None).

    x [b,T,H,P] and B, C [b,T,G,N] bf16 or float32 (same dtype); dt [b,T,H], A [H],
    D [H], init_state [b,H,P,N] float32.  ``workspace`` is an optional
    uint8 CUDA tensor (a cached one is used otherwise).
    """
    lib = load_library()
    dev = x.device
    b, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    io = {torch.bfloat16: SSD_BF16, torch.float32: SSD_F32}.get(x.dtype)
    if io is None:
        raise ValueError("x must be bfloat16 or float32")
    _need(x, "x", x.dtype, dev)
    _need(dt, "dt", torch.float32, dev, (b, T, H))
    _need(A, "A", torch.float32, dev, (H,))
    _need(B, "B", x.dtype, dev, (b, T, G, N))
    _need(C, "C", x.dtype, dev, (b, T, G, N))
    _need(D, "D", torch.float32, dev, (H,), allow_none=True)
    _need(init_state, "init_state", torch.float32, dev, (b, H, P, N), allow_none=True)
    if y is None:
        y = torch.empty_like(x)
    _need(y, "y", x.dtype, dev, x.shape)
    if final_state is None and return_final_state:
        final_state = torch.empty((b, H, P, N), dtype=torch.float32, device=dev)
    _need(final_state, "final_state", torch.float32, dev, (b, H, P, N), allow_none=True)
    nbytes = ssd_scan_workspace_size(b, T, H, P, G, N, chunk_size, False, io)
    ws = workspace if workspace is not None else _workspace(dev, nbytes)
    with torch.cuda.device(dev):
        st = lib.ssd_scan_fwd(_ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(init_state),
                              _ptr(final_state), _ptr(y), io, b, T, H, P, G, N, chunk_size,
                              _ptr(ws), 0 if ws is None else ws.numel(), _stream_handle(stream))
    _check(st)
    return y, final_state


def ssd_scan_fwd_noalloc(x, dt, A, B, C, D=None, init_state=None, *, chunk_size=256, y=None,
                         final_state=None, return_final_state=True, stream=None):
    """Real scan with the library's fixed scratch array instead of a workspace
    (float32 CUDA-core kernels; sizes whose scratch exceeds the array raise).
    Same tensors and return value as ssd_scan_fwd."""
    lib = load_library()
    dev = x.device
    b, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    io = {torch.bfloat16: SSD_BF16, torch.float32: SSD_F32}.get(x.dtype)
    if io is None:
        raise ValueError("x must be bfloat16 or float32")
    _need(x, "x", x.dtype, dev)
    _need(dt, "dt", torch.float32, dev, (b, T, H))
    _need(A, "A", torch.float32, dev, (H,))
    _need(B, "B", x.dtype, dev, (b, T, G, N))
    _need(C, "C", x.dtype, dev, (b, T, G, N))
    _need(D, "D", torch.float32, dev, (H,), allow_none=True)
    _need(init_state, "init_state", torch.float32, dev, (b, H, P, N), allow_none=True)
    if y is None:
        y = torch.empty_like(x)
    _need(y, "y", x.dtype, dev, x.shape)
    if final_state is None and return_final_state:
        final_state = torch.empty((b, H, P, N), dtype=torch.float32, device=dev)
    _need(final_state, "final_state", torch.float32, dev, (b, H, P, N), allow_none=True)
    with torch.cuda.device(dev):
        st = lib.ssd_scan_fwd_noalloc(_ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(init_state),
                                      _ptr(final_state), _ptr(y), io, b, T, H, P, G, N, chunk_size,
                                      _stream_handle(stream))
    _check(st)
    return y, final_state


def ssd_scan_fwd_complex(x, dt, A, B, C, D=None, init_state=None, *, chunk_size=256, y=None,
                         final_state=None, return_final_state=True, workspace=None, stream=None):
    """Complex chunked scan.  Returns (y, final_state or None).

    x [b,T,H,P] float32, dt [b,T,H] float32, A [H] complex64, B, C [b,T,G,N]
    complex64, D [H] float32, init_state [b,H,P,N] complex64.
    """
    lib = load_library()
    dev = x.device
    b, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    _need(x, "x", torch.float32, dev)
    _need(dt, "dt", torch.float32, dev, (b, T, H))
    _need(A, "A", torch.complex64, dev, (H,))
    _need(B, "B", torch.complex64, dev, (b, T, G, N))
    _need(C, "C", torch.complex64, dev, (b, T, G, N))
    _need(D, "D", torch.float32, dev, (H,), allow_none=True)
    _need(init_state, "init_state", torch.complex64, dev, (b, H, P, N), allow_none=True)
    if y is None:
        y = torch.empty_like(x)
    _need(y, "y", torch.float32, dev, x.shape)
    if final_state is None and return_final_state:
        final_state = torch.empty((b, H, P, N), dtype=torch.complex64, device=dev)
    _need(final_state, "final_state", torch.complex64, dev, (b, H, P, N), allow_none=True)
    nbytes = ssd_scan_workspace_size(b, T, H, P, G, N, chunk_size, True, SSD_F32)
    ws = workspace if workspace is not None else _workspace(dev, nbytes)
    with torch.cuda.device(dev):
        st = lib.ssd_scan_fwd_complex(_ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                      _ptr(init_state), _ptr(final_state), _ptr(y), b, T, H, P, G, N,
                                      chunk_size, _ptr(ws), 0 if ws is None else ws.numel(),
                                      _stream_handle(stream))
    _check(st)
    return y, final_state


def ssd_state_update(state, x, dt, A, B, C, D=None, *, y=None, stream=None):
    """One decoding step; ``state`` [b,H,P,N] float32 is updated in place.  Returns y."""
    lib = load_library()
    dev = state.device
    b, H, P, N = state.shape
    G = B.shape[1]
    io = {torch.bfloat16: SSD_BF16, torch.float32: SSD_F32}.get(x.dtype)
    if io is None:
        raise ValueError("x must be bfloat16 or float32")
    _need(state, "state", torch.float32, dev)
    _need(x, "x", x.dtype, dev, (b, H, P))
    _need(dt, "dt", torch.float32, dev, (b, H))
    _need(A, "A", torch.float32, dev, (H,))
    _need(B, "B", x.dtype, dev, (b, G, N))
    _need(C, "C", x.dtype, dev, (b, G, N))
    _need(D, "D", torch.float32, dev, (H,), allow_none=True)
    if y is None:
        y = torch.empty_like(x)
    _need(y, "y", x.dtype, dev, (b, H, P))
    with torch.cuda.device(dev):
        st = lib.ssd_state_update(_ptr(state), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                  _ptr(y), io, b, H, P, G, N, _stream_handle(stream))
    _check(st)
    return y


def ssd_state_update_complex(state, x, dt, A, B, C, D=None, *, y=None, stream=None):
    """Complex decoding step; ``state`` [b,H,P,N] complex64 is updated in place."""
    lib = load_library()
    dev = state.device
    b, H, P, N = state.shape
    G = B.shape[1]
    _need(state, "state", torch.complex64, dev)
    _need(x, "x", torch.float32, dev, (b, H, P))
    _need(dt, "dt", torch.float32, dev, (b, H))
    _need(A, "A", torch.complex64, dev, (H,))
    _need(B, "B", torch.complex64, dev, (b, G, N))
    _need(C, "C", torch.complex64, dev, (b, G, N))
    _need(D, "D", torch.float32, dev, (H,), allow_none=True)
    if y is None:
        y = torch.empty_like(x)
    _need(y, "y", torch.float32, dev, (b, H, P))
    with torch.cuda.device(dev):
        st = lib.ssd_state_update_complex(_ptr(state), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C),
                                          _ptr(D), _ptr(y), b, H, P, G, N, _stream_handle(stream))
    _check(st)
    return y


def ssd_scan_bwd_workspace_size(batch, seqlen, nheads, headdim, ngroups, dstate) -> int:
    n = load_library().ssd_scan_bwd_workspace_size(batch, seqlen, nheads, headdim, ngroups, dstate)
    if n == SSD_WORKSPACE_INVALID:
        raise SSDError(1, "invalid sizes for the backward scan")
    return n


def _bwd_outputs(out, like, dev):
    """The gradient tensors: ``out`` (a dict of preallocated tensors, checked)
    or fresh ones shaped like the inputs."""
    if out is None:
        return {k: (None if v is None else torch.empty(v[0], dtype=v[1], device=dev)) for k, v in like.items()}
    for k, v in like.items():
        if v is None:
            out.setdefault(k, None)
            continue
        _need(out.get(k), k, v[1], dev, v[0])
    return out


def ssd_scan_bwd(x, dt, A, B, C, D, init_state, dy, dfinal=None, *, out=None, workspace=None, stream=None):
    """Gradients of L = sum <dy, y> + <dfinal, final_state> through the real
    float32 scan.  Returns a dict with dx, ddt, dA, dB, dC, dD and dinit (dD is
    None when D is None); ``out`` may pass that dict preallocated."""
    lib = load_library()
    dev = x.device
    b, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    f = torch.float32
    _need(x, "x", f, dev)
    _need(dt, "dt", f, dev, (b, T, H))
    _need(A, "A", f, dev, (H,))
    _need(B, "B", f, dev, (b, T, G, N))
    _need(C, "C", f, dev, (b, T, G, N))
    _need(D, "D", f, dev, (H,), allow_none=True)
    _need(init_state, "init_state", f, dev, (b, H, P, N), allow_none=True)
    _need(dy, "dy", f, dev, (b, T, H, P))
    _need(dfinal, "dfinal", f, dev, (b, H, P, N), allow_none=True)
    out = _bwd_outputs(out, dict(dx=(x.shape, f), ddt=(dt.shape, f), dA=(A.shape, f), dB=(B.shape, f),
                                 dC=(C.shape, f), dD=None if D is None else (D.shape, f),
                                 dinit=((b, H, P, N), f)), dev)
    nbytes = ssd_scan_bwd_workspace_size(b, T, H, P, G, N)
    ws = workspace if workspace is not None else _workspace(dev, nbytes)
    with torch.cuda.device(dev):
        st = lib.ssd_scan_bwd(_ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(init_state),
                              _ptr(dy), _ptr(dfinal), _ptr(out["dx"]), _ptr(out["ddt"]), _ptr(out["dA"]),
                              _ptr(out["dB"]), _ptr(out["dC"]), _ptr(out["dD"]), _ptr(out["dinit"]),
                              b, T, H, P, G, N, _ptr(ws), 0 if ws is None else ws.numel(),
                              _stream_handle(stream))
    _check(st)
    return out


def ssd_scan_bwd_complex_workspace_size(batch, seqlen, nheads, headdim, ngroups, dstate) -> int:
    n = load_library().ssd_scan_bwd_complex_workspace_size(batch, seqlen, nheads, headdim, ngroups, dstate)
    if n == SSD_WORKSPACE_INVALID:
        raise SSDError(1, "invalid sizes for the complex backward scan")
    return n


def ssd_scan_bwd_complex(x, dt, A, B, C, D, init_state, dy, dfinal=None, *, out=None, workspace=None,
                         stream=None):
    """Gradients of L = sum <dy, y> + Re <dfinal, final_state> through the complex
    scan.  A, B, C, init_state, dfinal complex64; x, dt, D, dy float32.  Returns
    a dict with dx, ddt (float32), dA, dB, dC, dinit (complex64) and dD (float32,
    None when D is None)."""
    lib = load_library()
    dev = x.device
    b, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    f, c = torch.float32, torch.complex64
    _need(x, "x", f, dev)
    _need(dt, "dt", f, dev, (b, T, H))
    _need(A, "A", c, dev, (H,))
    _need(B, "B", c, dev, (b, T, G, N))
    _need(C, "C", c, dev, (b, T, G, N))
    _need(D, "D", f, dev, (H,), allow_none=True)
    _need(init_state, "init_state", c, dev, (b, H, P, N), allow_none=True)
    _need(dy, "dy", f, dev, (b, T, H, P))
    _need(dfinal, "dfinal", c, dev, (b, H, P, N), allow_none=True)
    out = _bwd_outputs(out, dict(dx=(x.shape, f), ddt=(dt.shape, f), dA=(A.shape, c), dB=(B.shape, c),
                                 dC=(C.shape, c), dD=None if D is None else (D.shape, f),
                                 dinit=((b, H, P, N), c)), dev)
    ws = workspace if workspace is not None else _workspace(dev, ssd_scan_bwd_complex_workspace_size(b, T, H, P, G, N))
    with torch.cuda.device(dev):
        st = lib.ssd_scan_bwd_complex(_ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(init_state),
                                      _ptr(dy), _ptr(dfinal), _ptr(out["dx"]), _ptr(out["ddt"]), _ptr(out["dA"]),
                                      _ptr(out["dB"]), _ptr(out["dC"]), _ptr(out["dD"]), _ptr(out["dinit"]),
                                      b, T, H, P, G, N, _ptr(ws), 0 if ws is None else ws.numel(),
                                      _stream_handle(stream))
    _check(st)
    return out


def ssd_get_device_status(stream=None) -> None:
    """Wait for the stream and raise SSDError if a kernel flagged a device-side error."""
    _check(load_library().ssd_get_device_status(_stream_handle(stream)))
