"""The failure path of the tensor-core kernel, and canary guard bands (needs a B200).

* A bounded wait that runs out: a test hook makes the kernel's load producer
  issue nothing, so every other role waits for data that never comes.  The
  waits give up after a shortened bound (10 ms), the kernel leaves at once,
  ssd_get_device_status reports SSD_ERR_TIMEOUT, and the next normal call on
  the same context matches the oracle.  Nothing faults: the failure is a flag
  that nothing sets.
* Guard bands: y and the final state are views inside larger buffers filled
  with a sentinel byte pattern; after scans with ragged sequence lengths (rows
  past the end of the sequence are skipped, not written) the bands are
  byte-identical, on the tensor-core path and on the CUDA-core path.
"""
import ctypes
import time

import numpy as np
import pytest
import torch

import selective_state_space_22_b200 as ssd
from selective_state_space_22_b200 import inputs
from parity import TOL_BF16, TOL_F32, oracle_scan, rel_err, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = ssd.load_library()
    lib.ssd_debug_inject_stall.argtypes = [ctypes.c_int, ctypes.c_ulonglong]
    lib.ssd_debug_inject_stall.restype = ctypes.c_int
    return lib


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def test_timeout_is_reported_quickly_and_the_next_call_is_correct(lib):
    shape = inputs.ScanShape("stall", 2, 2048, 8, 64, 1, 128, 128, "bf16", init_state=True, seed=31)
    inp = inputs.scan_inputs(shape)
    d = to_dev(inp)
    ssd.ssd_scan_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["init_state"], chunk_size=128)
    assert lib.ssd_get_device_status(_stream()) == ssd.SSD_OK
    assert ssd.ssd_scan_kernel_launches(2, 2048, 8, 64, 1, 128, 128) == 1  # the tensor-core kernel
    try:
        assert lib.ssd_debug_inject_stall(1, 10_000_000) == ssd.SSD_OK
        t0 = time.perf_counter()
        ssd.ssd_scan_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["init_state"], chunk_size=128)
        st = lib.ssd_get_device_status(_stream())
        elapsed = time.perf_counter() - t0
    finally:
        lib.ssd_debug_inject_stall(0, 0)
    assert st == ssd.SSD_ERR_TIMEOUT, (st, ssd.ssd_last_error())
    assert elapsed < 1.0, elapsed
    # the error was read and cleared; the context is usable and the next call correct
    assert lib.ssd_get_device_status(_stream()) == ssd.SSD_OK
    y, fs = ssd.ssd_scan_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["init_state"],
                             chunk_size=128)
    assert lib.ssd_get_device_status(_stream()) == ssd.SSD_OK
    y_ref, fs_ref = oracle_scan(inp, heads=[0, 5], batches=[1])
    got_y = y.float().cpu().numpy()[[1]][:, :, [0, 5]]
    got_fs = fs.cpu().numpy()[[1]][:, [0, 5]]
    assert rel_err(got_y, y_ref) <= TOL_BF16
    assert rel_err(got_fs, fs_ref) <= TOL_BF16


def test_timeout_in_the_state_only_form(lib):
    """The state-only form (no y) runs its own kernel instance, in which the math
    warpgroup waits for each tile's slot and X before building W.  With the
    producer withheld, those waits run out too: SSD_ERR_TIMEOUT within a
    second, and the next state-only call matches the oracle's final state."""
    shape = inputs.ScanShape("stall-so", 1, 2048, 8, 64, 1, 128, 128, "bf16", init_state=True, seed=32)
    inp = inputs.scan_inputs(shape)
    d = to_dev(inp)
    ssd.ssd_scan_final_state(d["x"], d["dt"], d["A"], d["B"], d["init_state"], chunk_size=128)
    assert lib.ssd_get_device_status(_stream()) == ssd.SSD_OK
    try:
        assert lib.ssd_debug_inject_stall(1, 10_000_000) == ssd.SSD_OK
        t0 = time.perf_counter()
        ssd.ssd_scan_final_state(d["x"], d["dt"], d["A"], d["B"], d["init_state"], chunk_size=128)
        st = lib.ssd_get_device_status(_stream())
        elapsed = time.perf_counter() - t0
    finally:
        lib.ssd_debug_inject_stall(0, 0)
    assert st == ssd.SSD_ERR_TIMEOUT, (st, ssd.ssd_last_error())
    assert elapsed < 1.0, elapsed
    assert lib.ssd_get_device_status(_stream()) == ssd.SSD_OK
    fs, _ = ssd.ssd_scan_final_state(d["x"], d["dt"], d["A"], d["B"], d["init_state"], chunk_size=128)
    assert lib.ssd_get_device_status(_stream()) == ssd.SSD_OK
    _, fs_ref = oracle_scan(inp, heads=[0, 7], batches=[0])
    assert rel_err(fs.cpu().numpy()[[0]][:, [0, 7]], fs_ref) <= TOL_BF16


SENTINEL = 0x5A


def _guarded(shape, dtype, pad_bytes=4096):
    """A tensor of `shape` inside a byte buffer with pad_bytes of sentinel on each side."""
    n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
    buf = torch.full((n + 2 * pad_bytes,), SENTINEL, dtype=torch.uint8, device="cuda")
    view = buf[pad_bytes:pad_bytes + n].view(dtype).view(shape)
    return buf, view


@pytest.mark.parametrize("io", ["bf16", "f32"])
@pytest.mark.parametrize("T", [129, 255, 2565])
def test_outputs_stay_inside_their_buffers(io, T):
    shape = inputs.ScanShape("guard", 1, T, 4, 64, 1, 128, 128, io, init_state=True, seed=T)
    inp = inputs.scan_inputs(shape)
    d = to_dev(inp)
    ybuf, y = _guarded(tuple(d["x"].shape), d["x"].dtype)
    fbuf, fs = _guarded((1, 4, 64, 128), torch.float32)
    ssd.ssd_scan_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["init_state"], chunk_size=128,
                     y=y, final_state=fs)
    ssd.ssd_get_device_status()
    for buf in (ybuf, fbuf):
        b = buf.cpu().numpy()
        assert (b[:4096] == SENTINEL).all() and (b[-4096:] == SENTINEL).all()
    y_ref, fs_ref = oracle_scan(inp)
    tol = TOL_BF16 if io == "bf16" else TOL_F32
    assert rel_err(y.float().cpu().numpy(), y_ref) <= tol
    assert rel_err(fs.cpu().numpy(), fs_ref) <= tol
