"""CUDA path vs the fp64 oracle on identical seeded inputs (needs a B200).

Small problems are compared element by element in full; they span several
chunks and end in a ragged partial chunk.  The full-size workloads (the
BitMamba-1B layer shape, the Mamba-3-Lite complex layer, the 65536-token
sequence) run exactly as the benchmark launches them and are compared on
sampled (batch, head) sequences, which the oracle computes one by one.
Tolerances: max|gpu - ref| / max|ref| <= 1e-4 for float32 inputs and <= 2e-2
for bf16 inputs (float32 state), for y and for the final state.
"""
import dataclasses

import numpy as np
import pytest
import torch

import selective_state_space_22_b200 as ssd
from selective_state_space_22_b200 import inputs
from parity import TOL_BF16, TOL_F32, elem_rel_err, gpu_scan, oracle_scan, pick, rel_err, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ssd.load_library()


def small(name, b, T, H, P, G, N, chunk, io, cplx=False, init=False, seed=11):
    return inputs.ScanShape(name, b, T, H, P, G, N, chunk, io, complex=cplx, init_state=init, seed=seed)


def check_full(shape, tol):
    inp = inputs.scan_inputs(shape)
    y, fs = gpu_scan(inp, shape.chunk, shape.complex)
    y_ref, fs_ref = oracle_scan(inp)
    ey, ef = rel_err(y.numpy(), y_ref), rel_err(fs.numpy(), fs_ref)
    # for information: the per-element relative error (floor 1e-3 max|ref|)
    print(f"{shape.name} T={shape.seqlen}: normwise y {ey:.2e} final {ef:.2e}; per element "
          f"y {elem_rel_err(y.numpy(), y_ref):.2e} final {elem_rel_err(fs.numpy(), fs_ref):.2e}")
    assert ey <= tol and ef <= tol, (shape.name, ey, ef)
    return ey, ef


# ------------------------------------------------------------------ small, full
def test_tiny_real_f32_workload():
    check_full(inputs.TINY, TOL_F32)


@pytest.mark.parametrize("T", [1, 63, 64, 65, 200, 517])
@pytest.mark.parametrize("chunk", [64, 128, 256])
def test_real_f32_ragged(T, chunk):
    check_full(small("rf32", 2, T, 4, 16, 2, 8, chunk, "f32", init=(T % 2 == 1)), TOL_F32)


@pytest.mark.parametrize("P,N,G", [(64, 128, 1), (32, 64, 2), (64, 64, 4), (48, 40, 1)])
def test_real_f32_shapes(P, N, G):
    check_full(small("rf32s", 1, 333, 4, P, G, N, 128, "f32", init=True), TOL_F32)


@pytest.mark.parametrize("T,chunk", [(1, 256), (255, 256), (256, 256), (600, 256), (777, 128),
                                     (300, 64)])
@pytest.mark.parametrize("init", [False, True])
def test_real_bf16(T, chunk, init):
    check_full(small("rbf16", 2, T, 4, 64, 1, 128, chunk, "bf16", init=init), TOL_BF16)


@pytest.mark.parametrize("P,N,G", [(64, 64, 2), (32, 128, 1), (16, 8, 1)])
def test_real_bf16_other_shapes(P, N, G):
    check_full(small("rbf16s", 1, 400, 4, P, G, N, 256, "bf16", init=True), TOL_BF16)


@pytest.mark.parametrize("T,chunk", [(1, 256), (300, 256), (256, 64), (517, 128)])
@pytest.mark.parametrize("G", [1, 4])
def test_complex(T, chunk, G):
    check_full(small("cplx", 2, T, 4, 64, G, 64, chunk, "f32", cplx=True, init=(T % 2 == 1)), TOL_F32)


def test_complex_small_dims():
    check_full(small("cplx2", 1, 129, 2, 16, 2, 8, 64, "f32", cplx=True, init=True), TOL_F32)


@pytest.mark.parametrize("P,N,G", [(64, 96, 1), (100, 128, 2), (32, 200, 4)])
def test_complex_wide_state_and_head_dim(P, N, G):
    """2N > 128 takes the K-sliced chunk scan and several chunk-state tiles;
    P > 64 several head-dim tiles."""
    check_full(small("cplx3", 2, 333, 4, P, G, N, 128, "f32", cplx=True, init=True), TOL_F32)


# ------------------------------------------------------------------- edge cases
def test_empty_sequence_copies_initial_state():
    shape = small("empty", 2, 0, 4, 64, 1, 128, 256, "bf16", init=True)
    inp = inputs.scan_inputs(shape)
    y, fs = gpu_scan(inp, 256, False)
    assert y.numel() == 0
    assert torch.equal(fs, inp["init_state"])
    shape = dataclasses.replace(shape, init_state=False)
    y, fs = gpu_scan(inputs.scan_inputs(shape), 256, False)
    assert float(fs.abs().max()) == 0.0


def test_final_state_aliases_initial_state():
    shape = small("alias", 1, 300, 4, 64, 1, 128, 128, "bf16", init=True)
    inp = inputs.scan_inputs(shape)
    y_ref, fs_ref = oracle_scan(inp)
    d = to_dev(inp)
    h = d["init_state"].clone()
    y, fs = ssd.ssd_scan_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], h, final_state=h,
                             chunk_size=128)
    ssd.ssd_get_device_status()
    assert rel_err(y.float().cpu().numpy(), y_ref) <= TOL_BF16
    assert rel_err(h.cpu().numpy(), fs_ref) <= TOL_BF16


def test_no_D_no_final_state():
    shape = small("noD", 1, 130, 2, 64, 1, 128, 64, "bf16")
    inp = inputs.scan_inputs(shape)
    inp["D"] = None
    d = to_dev(inp)
    y, fs = ssd.ssd_scan_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], None, None,
                             return_final_state=False, chunk_size=64)
    assert fs is None
    y_ref, _ = oracle_scan(inp)
    assert rel_err(y.float().cpu().numpy(), y_ref) <= TOL_BF16


@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_repeated_calls_are_bitwise_equal(io):
    """Neither kernel family has a data-dependent summation order (no atomics, no
    inter-block races), so repeated calls give identical bits."""
    shape = small("rep", 2, 700, 4, 64, 1, 128, 256, io, init=True)
    inp = inputs.scan_inputs(shape)
    y0, f0 = gpu_scan(inp, 256, False)
    for _ in range(3):
        y1, f1 = gpu_scan(inp, 256, False)
        assert torch.equal(y1, y0)
        assert torch.equal(f1, f0)


def _tc(shape):
    """The shapes the tensor-core kernel takes (bf16, head dim 64, d_state 128, at
    least one 128-token chunk): one launch, or three with batch 1 when each
    sequence is cut in two."""
    n = ssd.ssd_scan_kernel_launches(shape.batch, shape.seqlen, shape.nheads, shape.headdim,
                                     shape.ngroups, shape.dstate, shape.chunk, False, ssd.SSD_BF16)
    return (shape.headdim == 64 and shape.dstate == 128 and shape.seqlen >= 128
            and (n == 1 or (n == 3 and shape.batch == 1)))


@pytest.mark.parametrize("T", [128, 129, 256, 1000, 128 * 20 + 5])
@pytest.mark.parametrize("H,G", [(1, 1), (4, 2), (6, 6)])
def test_tcgen05_path(T, H, G):
    """The tensor-core kernel: one chunk, ragged tails, more chunks than ring slots
    (slot reuse), several groups."""
    shape = small("tc", 2, T, H, 64, G, 128, 256, "bf16", init=(H != 1), seed=T + H)
    assert _tc(shape), "expected the tcgen05 kernel for this shape"
    check_full(shape, TOL_BF16)


@pytest.mark.parametrize("T,H", [(300, 64), (128 * 9 + 17, 50), (256, 74)])
def test_batch1_cut_in_two(T, H):
    """Batch 1 with fewer sequences than SMs: the first part of each sequence on the
    caller's stream, the state-only prefix and the rest on a second stream (three
    launches); ragged tails, a nonzero initial state."""
    shape = small("b1split", 1, T, H, 64, 1, 128, 256, "bf16", init=True, seed=T + H)
    assert ssd.ssd_scan_kernel_launches(1, T, H, 64, 1, 128, 256, False, ssd.SSD_BF16) == 3
    check_full(shape, TOL_BF16)


def test_batch1_cut_in_two_final_state_aliases_initial_state():
    """The second stream writes the final state while the first may still read the
    initial one: with the two aliased, both halves start from a copy."""
    shape = small("b1alias", 1, 700, 64, 64, 1, 128, 128, "bf16", init=True, seed=5)
    inp = inputs.scan_inputs(shape)
    y_ref, fs_ref = oracle_scan(inp)
    d = to_dev(inp)
    h = d["init_state"].clone()
    y, fs = ssd.ssd_scan_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], h, final_state=h, chunk_size=128)
    ssd.ssd_get_device_status()
    assert rel_err(y.float().cpu().numpy(), y_ref) <= TOL_BF16
    assert rel_err(h.cpu().numpy(), fs_ref) <= TOL_BF16


@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_steep_decay(io):
    """A in [-100, -40] with dt up to 0.1: a 32-token block can span well over 80 of
    log-decay, so the kernels take their per-element decay path (the factored
    form's factors would leave the float range).  Nothing may overflow."""
    shape = small("steep", 2, 700, 4, 64, 1, 128, 256, io, init=True, seed=99)
    inp = inputs.scan_inputs(shape)
    inp["A"] = -torch.linspace(40.0, 100.0, shape.nheads)
    inp["dt"] = (inp["dt"] * 4.0).clamp(max=0.1).contiguous()
    if io == "bf16":
        assert _tc(shape)
    y, fs = gpu_scan(inp, shape.chunk, False)
    assert torch.isfinite(y).all() and torch.isfinite(fs).all()
    y_ref, fs_ref = oracle_scan(inp)
    tol = TOL_BF16 if io == "bf16" else TOL_F32
    ey, ef = rel_err(y.numpy(), y_ref), rel_err(fs.numpy(), fs_ref)
    assert ey <= tol and ef <= tol, (ey, ef)


def test_steep_decay_complex():
    """Complex A with real part in [-100, -40]: decays that underflow within a
    chunk must come out as zeros, never as inf or NaN."""
    shape = small("steepc", 2, 500, 4, 64, 4, 64, 256, "f32", cplx=True, init=True, seed=98)
    inp = inputs.scan_inputs(shape)
    inp["A"] = torch.complex(-torch.linspace(40.0, 100.0, shape.nheads), inp["A"].imag).contiguous()
    inp["dt"] = (inp["dt"] * 4.0).clamp(max=0.1).contiguous()
    y, fs = gpu_scan(inp, shape.chunk, True)
    assert torch.isfinite(y).all() and torch.isfinite(torch.view_as_real(fs)).all()
    y_ref, fs_ref = oracle_scan(inp)
    ey, ef = rel_err(y.numpy(), y_ref), rel_err(fs.numpy(), fs_ref)
    assert ey <= TOL_F32 and ef <= TOL_F32, (ey, ef)


# --------------------------------------------------------- full-size, sampled
def _sampled(shape, samples, tol):
    inp = inputs.scan_inputs(shape)
    y, fs = gpu_scan(inp, shape.chunk, shape.complex)
    worst = [0.0, 0.0, 0.0]
    for b, h in samples:
        y_ref, fs_ref = oracle_scan(inp, heads=[h], batches=[b])
        yg = pick(y, [b], [h], 0, 2)
        ey = rel_err(yg, y_ref)
        ef = rel_err(pick(fs, [b], [h], 0, 1), fs_ref)
        worst = [max(worst[0], ey), max(worst[1], ef), max(worst[2], elem_rel_err(yg, y_ref))]
        assert ey <= tol and ef <= tol, (shape.name, b, h, ey, ef)
    print(f"{shape.name} sampled (batch, head) {samples}: normwise y {worst[0]:.2e} final {worst[1]:.2e}; "
          f"per element y {worst[2]:.2e}")
    assert torch.isfinite(y).all()


def test_mamba2_1b_layer_sampled():
    assert _tc(inputs.MAMBA2_1B)
    _sampled(inputs.MAMBA2_1B, [(0, 0), (0, 37), (1, 5), (1, 63)], TOL_BF16)


def test_mamba3_complex_layer_sampled():
    _sampled(inputs.MAMBA3_COMPLEX, [(0, 0), (1, 7), (2, 11), (3, 15)], TOL_F32)


def test_long_sequence_sampled():
    assert _tc(inputs.LONG)
    _sampled(inputs.LONG, [(0, 3), (0, 60)], TOL_BF16)
