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
           "ssd_scan_bwd_complex", "ssd_scan_bwd_complex_workspace_size", "ssd_scan_final_state",
           "ssd_fold_states", "ssd_scan_fwd_complex_packed", "ssd_conv1d_xbc", "ssd_selective_scan"]

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
        lib.ssd_conv1d_xbc.argtypes = [_VP] * 8 + [_I] * 7 + [_VP]
        lib.ssd_conv1d_xbc.restype = _I
        lib.ssd_selective_scan.argtypes = [_VP] * 9 + [_I] * 6 + [_VP]
        lib.ssd_selective_scan.restype = _I
        lib.ssd_scan_fwd_complex_packed.argtypes = [_VP, _I] + [_VP] * 6 + [_I] * 6 + [_VP, _SZ, _VP]
        lib.ssd_scan_fwd_complex_packed.restype = _I
        lib.ssd_scan_final_state.argtypes = [_VP] * 7 + [_I] * 8 + [_VP, _SZ, _VP]
        lib.ssd_scan_final_state.restype = _I
        lib.ssd_fold_states.argtypes = [_VP, _VP, _I, _VP, _I, _I, _I, _I, _VP]
        lib.ssd_fold_states.restype = _I
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


def ssd_conv1d_xbc(xbc, weight, bias=None, conv_init=None, *, x_channels, bc_channels, silu=True,
                   out=None, conv_final=None, stream=None):
    """Causal depthwise conv over packed x|B|C channels, split into the scan's
    inputs.  xbc [b,T,Cx+2Cb] bf16/float32, weight [Cx+2Cb, K] float32, bias
    [Cx+2Cb] float32, conv_init [b, Cx+2Cb, K-1].  Returns (x [b,T,Cx],
    B [b,T,Cb], C [b,T,Cb]) (``out`` may pass them preallocated)."""
    lib = load_library()
    dev = xbc.device
    b, T, Ct = xbc.shape
    if Ct != x_channels + 2 * bc_channels:
        raise ValueError("xbc width must be x_channels + 2 bc_channels")
    io = {torch.bfloat16: SSD_BF16, torch.float32: SSD_F32}.get(xbc.dtype)
    if io is None:
        raise ValueError("xbc must be bfloat16 or float32")
    K = weight.shape[1]
    _need(xbc, "xbc", xbc.dtype, dev)
    _need(weight, "weight", torch.float32, dev, (Ct, K))
    _need(bias, "bias", torch.float32, dev, (Ct,), allow_none=True)
    _need(conv_init, "conv_init", xbc.dtype, dev, (b, Ct, K - 1), allow_none=True)
    _need(conv_final, "conv_final", xbc.dtype, dev, (b, Ct, K - 1), allow_none=True)
    if out is None:
        out = (torch.empty((b, T, x_channels), dtype=xbc.dtype, device=dev),
               torch.empty((b, T, bc_channels), dtype=xbc.dtype, device=dev),
               torch.empty((b, T, bc_channels), dtype=xbc.dtype, device=dev))
    xo, bo, co = out
    with torch.cuda.device(dev):
        st = lib.ssd_conv1d_xbc(_ptr(xbc), _ptr(weight), _ptr(bias), _ptr(conv_init), _ptr(xo), _ptr(bo), _ptr(co),
                                _ptr(conv_final), io, b, T, x_channels, bc_channels, K, int(bool(silu)),
                                _stream_handle(stream))
    _check(st)
    return xo, bo, co


def ssd_selective_scan(x, dt, A, B, C, D=None, init_state=None, *, y=None, final_state=None,
                       return_final_state=True, stream=None):
    """Mamba-1 selective scan (per-state A).  x [b,T,Dc] bf16/float32, dt [b,T,Dc]
    float32, A [Dc,N] float32, B, C [b,T,G,N] (dtype of x), D [Dc], init_state
    [b,Dc,N] float32.  Returns (y [b,T,Dc], final_state or None)."""
    lib = load_library()
    dev = x.device
    b, T, Dc = x.shape
    G, N = B.shape[2], B.shape[3]
    io = {torch.bfloat16: SSD_BF16, torch.float32: SSD_F32}.get(x.dtype)
    if io is None:
        raise ValueError("x must be bfloat16 or float32")
    _need(x, "x", x.dtype, dev)
    _need(dt, "dt", torch.float32, dev, (b, T, Dc))
    _need(A, "A", torch.float32, dev, (Dc, N))
    _need(B, "B", x.dtype, dev, (b, T, G, N))
    _need(C, "C", x.dtype, dev, (b, T, G, N))
    _need(D, "D", torch.float32, dev, (Dc,), allow_none=True)
    _need(init_state, "init_state", torch.float32, dev, (b, Dc, N), allow_none=True)
    if y is None:
        y = torch.empty_like(x)
    if final_state is None and return_final_state:
        final_state = torch.empty((b, Dc, N), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        st = lib.ssd_selective_scan(_ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(init_state),
                                    _ptr(final_state), _ptr(y), io, b, T, Dc, G, N, _stream_handle(stream))
    _check(st)
    return y, final_state


def ssd_scan_fwd_complex_packed(proj, A, D=None, init_state=None, *, nheads, headdim, dstate, dt_bias=None,
                                chunk_size=256, y=None, final_state=None, return_final_state=True, workspace=None,
                                stream=None):
    """The complex scan reading the packed projection output in place.

    proj [b, T, H (headdim + 4 dstate + 1)] float32 or bf16, head-major slices
    x | Re B | Im B | Re C | Im C | dt; dt = softplus(dt + dt_bias) inside the scan.
    A [H] complex64, D [H] float32, dt_bias [H] float32, init_state [b,H,P,N]
    complex64.  Returns (y [b,T,H,P] float32, final_state or None)."""
    lib = load_library()
    dev = proj.device
    b, T, W = proj.shape
    H, P, N = nheads, headdim, dstate
    if W != H * (P + 4 * N + 1):
        raise ValueError(f"proj width {W} != nheads (headdim + 4 dstate + 1) = {H * (P + 4 * N + 1)}")
    io = {torch.bfloat16: SSD_BF16, torch.float32: SSD_F32}.get(proj.dtype)
    if io is None:
        raise ValueError("proj must be bfloat16 or float32")
    _need(proj, "proj", proj.dtype, dev)
    _need(A, "A", torch.complex64, dev, (H,))
    _need(D, "D", torch.float32, dev, (H,), allow_none=True)
    _need(dt_bias, "dt_bias", torch.float32, dev, (H,), allow_none=True)
    _need(init_state, "init_state", torch.complex64, dev, (b, H, P, N), allow_none=True)
    if y is None:
        y = torch.empty((b, T, H, P), dtype=torch.float32, device=dev)
    _need(y, "y", torch.float32, dev, (b, T, H, P))
    if final_state is None and return_final_state:
        final_state = torch.empty((b, H, P, N), dtype=torch.complex64, device=dev)
    _need(final_state, "final_state", torch.complex64, dev, (b, H, P, N), allow_none=True)
    nbytes = ssd_scan_workspace_size(b, T, H, P, H, N, chunk_size, True, SSD_F32)
    ws = workspace if workspace is not None else _workspace(dev, nbytes)
    with torch.cuda.device(dev):
        st = lib.ssd_scan_fwd_complex_packed(_ptr(proj), io, _ptr(dt_bias), _ptr(A), _ptr(D), _ptr(init_state),
                                             _ptr(final_state), _ptr(y), b, T, H, P, N, chunk_size, _ptr(ws),
                                             0 if ws is None else ws.numel(), _stream_handle(stream))
    _check(st)
    return y, final_state


def ssd_scan_final_state(x, dt, A, B, init_state=None, *, chunk_size=256, final_state=None,
                         total_log_decay=None, workspace=None, stream=None):
    """Final state and total log-decay of a (slice of a) sequence, without its
    outputs: the state-only scan.  Returns (final_state [b,H,P,N] float32,
    total_log_decay [b,H] float32 = A * sum of dt)."""
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
    _need(init_state, "init_state", torch.float32, dev, (b, H, P, N), allow_none=True)
    if final_state is None:
        final_state = torch.empty((b, H, P, N), dtype=torch.float32, device=dev)
    _need(final_state, "final_state", torch.float32, dev, (b, H, P, N))
    if total_log_decay is None:
        total_log_decay = torch.empty((b, H), dtype=torch.float32, device=dev)
    _need(total_log_decay, "total_log_decay", torch.float32, dev, (b, H))
    nbytes = ssd_scan_workspace_size(b, T, H, P, G, N, chunk_size, False, io)
    ws = workspace if workspace is not None else _workspace(dev, nbytes)
    with torch.cuda.device(dev):
        st = lib.ssd_scan_final_state(_ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(init_state), _ptr(final_state),
                                      _ptr(total_log_decay), io, b, T, H, P, G, N, chunk_size, _ptr(ws),
                                      0 if ws is None else ws.numel(), _stream_handle(stream))
    _check(st)
    return final_state, total_log_decay


def ssd_fold_states(states, log_decay, *, out=None, stream=None):
    """The state entering the slice after the given ones: h_0 = states[0],
    h_j = exp(log_decay[j]) h_{j-1} + states[j]; returns h_{n-1}.
    states [n, b, H, P, N] float32, log_decay [n, b, H] float32."""
    lib = load_library()
    dev = states.device
    n, b, H, P, N = states.shape
    _need(states, "states", torch.float32, dev)
    _need(log_decay, "log_decay", torch.float32, dev, (n, b, H))
    if out is None:
        out = torch.empty((b, H, P, N), dtype=torch.float32, device=dev)
    _need(out, "out", torch.float32, dev, (b, H, P, N))
    with torch.cuda.device(dev):
        st = lib.ssd_fold_states(_ptr(states), _ptr(log_decay), n, _ptr(out), b, H, P, N, _stream_handle(stream))
    _check(st)
    return out


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
