"""ssd_scan_fwd_noalloc: the scan for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc or pass a workspace (a plugin inside an
application that owns all device memory; a path that cannot afford an
allocation).  This entry point keeps its scratch in a fixed array inside the
library instead.  The test calls it through the C ABI twice in a row and checks
both results against the fp64 oracle, within the tolerances the other parity
tests use.  The two calls differ: the first is the larger problem (more chunks
and sequences) with one seed, the second a smaller one with another seed and
another initial state, so a kernel that read scratch left over from the first
call instead of writing it would give a wrong second result.  It also checks
that sizes beyond the array are refused before anything runs.
"""
import ctypes

import numpy as np
import pytest
import torch

import selective_state_space_22_b200 as ssd
from selective_state_space_22_b200 import inputs
from parity import TOL_BF16, TOL_F32, oracle_scan, rel_err, to_dev

pytestmark = pytest.mark.gpu

_VP, _I = ctypes.c_void_p, ctypes.c_int


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = ssd.load_library()
    lib.ssd_scan_fwd_noalloc.argtypes = [_VP] * 9 + [_I] * 8 + [_VP]
    lib.ssd_scan_fwd_noalloc.restype = _I
    return lib


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def noalloc_scan(lib, d, shape):
    b, T, H, P = d["x"].shape
    G, N = d["B"].shape[2], d["B"].shape[3]
    y = torch.empty_like(d["x"])
    fs = torch.empty((b, H, P, N), dtype=torch.float32, device=d["x"].device)
    io = ssd.SSD_BF16 if d["x"].dtype == torch.bfloat16 else ssd.SSD_F32
    st = lib.ssd_scan_fwd_noalloc(_p(d["x"]), _p(d["dt"]), _p(d["A"]), _p(d["B"]), _p(d["C"]), _p(d["D"]),
                                  _p(d["init_state"]), _p(fs), _p(y), io, b, T, H, P, G, N, shape.chunk,
                                  ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == ssd.SSD_OK, ssd.ssd_last_error()
    ssd.ssd_get_device_status()
    return y.float().cpu(), fs.cpu()


@pytest.mark.parametrize("io,tol", [("f32", TOL_F32), ("bf16", TOL_BF16)])
def test_noalloc_two_calls_match_the_oracle(lib, io, tol):
    big = inputs.ScanShape("noalloc-big", 3, 700, 4, 64, 2, 128, 128, io, init_state=True, seed=91)
    small = inputs.ScanShape("noalloc-small", 2, 300, 4, 64, 1, 128, 128, io, init_state=True, seed=93)
    for shape in (big, small):
        inp = inputs.scan_inputs(shape)
        y, fs = noalloc_scan(lib, to_dev(inp), shape)
        y_ref, fs_ref = oracle_scan(inp)
        assert rel_err(y.numpy(), y_ref) <= tol, shape.name
        assert rel_err(fs.numpy(), fs_ref) <= tol, shape.name


def test_noalloc_rejects_sizes_beyond_its_scratch(lib):
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the size check fails first
    st = lib.ssd_scan_fwd_noalloc(fake, fake, fake, fake, fake, None, None, None, fake, ssd.SSD_BF16,
                                  2, 65536, 64, 64, 1, 128, 256, None)
    assert st == ssd.SSD_ERR_WORKSPACE
    assert "scratch" in ssd.ssd_last_error()


def test_noalloc_python_binding_matches_the_oracle():
    """The Python wrapper of the same name marshals the same call."""
    shape = inputs.ScanShape("noalloc-py", 1, 200, 2, 64, 1, 128, 64, "f32", init_state=True, seed=92)
    inp = inputs.scan_inputs(shape)
    d = to_dev(inp)
    y, fs = ssd.ssd_scan_fwd_noalloc(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["init_state"],
                                     chunk_size=shape.chunk)
    ssd.ssd_get_device_status()
    y_ref, fs_ref = oracle_scan(inp)
    assert rel_err(y.cpu().numpy(), y_ref) <= TOL_F32
    assert rel_err(fs.cpu().numpy(), fs_ref) <= TOL_F32
