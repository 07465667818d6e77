"""The variants against the oracle (needs a B200): the causal conv1d prologue
(ssd_conv1d_xbc) and the Mamba-1 selective scan with a per-state A
(ssd_selective_scan).  Element by element over every output."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import selective_state_space_22_b200 as ssd
from selective_state_space_22_b200 import inputs
from parity import TOL_BF16, TOL_F32, elem_rel_err, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ssd.load_library()


def conv_case(shape):
    inp = inputs.conv_inputs(shape)
    d = {k: (None if v is None else v.cuda()) for k, v in inp.items()}
    Ct = shape.x_channels + 2 * shape.bc_channels
    fin = torch.empty((shape.batch, Ct, shape.width - 1), dtype=d["xbc"].dtype, device="cuda") \
        if shape.width > 1 else None
    xo, bo, co = ssd.ssd_conv1d_xbc(d["xbc"], d["weight"], d["bias"], d["conv_init"], x_channels=shape.x_channels,
                                    bc_channels=shape.bc_channels, silu=shape.silu, conv_final=fin)
    ssd.ssd_get_device_status()
    w = inputs.widen_all(inp)
    ref = oracle.causal_conv1d(w["xbc"], w["weight"], w["bias"], w["conv_init"], silu=shape.silu)
    got = np.concatenate([t.float().cpu().numpy() for t in (xo, bo, co)], axis=-1)
    tol = TOL_F32 if shape.io_dtype == "f32" else TOL_BF16
    assert rel_err(got, ref) <= tol, rel_err(got, ref)
    if fin is not None:  # the last K-1 inputs (from conv_init where the sequence is shorter)
        full = np.concatenate([np.transpose(w["conv_init"], (0, 2, 1)) if w["conv_init"] is not None
                               else np.zeros((shape.batch, shape.width - 1, Ct)), w["xbc"]], axis=1)
        want = np.transpose(full[:, -(shape.width - 1):], (0, 2, 1))
        assert np.array_equal(fin.float().cpu().numpy(), want)


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("T,Cx,Cb,K,silu,init", [(1, 64, 16, 4, True, True), (5, 100, 8, 4, False, True),
                                                 (33, 128, 16, 3, True, False), (100, 40, 0, 2, True, True),
                                                 (257, 256, 64, 4, True, False), (2, 64, 16, 1, False, False)])
def test_conv1d(io, T, Cx, Cb, K, silu, init):
    conv_case(inputs.ConvShape("conv", 2, T, Cx, Cb, K, io, silu=silu, init=init, seed=T + K))


def test_conv1d_bitmamba_prologue():
    """The BitMamba-1B layer's prologue (4096 x channels, 128 + 128 B/C channels,
    kernel 4, SiLU), every output."""
    conv_case(inputs.MAMBA2_CONV)


def sel_case(shape, sample=None):
    inp = inputs.selective_inputs(shape)
    d = {k: (None if v is None else v.cuda()) for k, v in inp.items()}
    y, fs = ssd.ssd_selective_scan(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["init_state"])
    ssd.ssd_get_device_status()
    w = inputs.widen_all(inp)
    y, fs = y.float().cpu().numpy(), fs.cpu().numpy()
    if sample is not None:  # channels of one group only (B and C whole)
        c = np.ascontiguousarray
        bs, ds = sample
        sel = lambda a: c(a[bs][:, :, ds])
        y_ref, fs_ref = oracle.selective_scan(sel(w["x"]), sel(w["dt"]), c(w["A"][ds]), c(w["B"][bs]),
                                              c(w["C"][bs]), c(w["D"][ds]),
                                              None if w["init_state"] is None else c(w["init_state"][bs][:, ds]))
        y, fs = y[bs][:, :, ds], fs[bs][:, ds]
    else:
        y_ref, fs_ref = oracle.selective_scan(w["x"], w["dt"], w["A"], w["B"], w["C"], w["D"], w["init_state"])
    tol = TOL_F32 if shape.io_dtype == "f32" else TOL_BF16
    ey, ef = rel_err(y, y_ref), rel_err(fs, fs_ref)
    print(f"{shape.name}: y {ey:.2e} (per element {elem_rel_err(y, y_ref):.2e}) final {ef:.2e}")
    assert ey <= tol and ef <= tol, (ey, ef)


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("T,Dc,G,N,init", [(1, 64, 1, 16, True), (17, 100, 2, 8, False), (300, 256, 1, 16, True),
                                           (130, 96, 3, 32, True), (64, 33, 1, 4, False),
                                           (150, 128, 2, 32, True), (45, 128, 1, 8, False)])
def test_selective_scan(io, T, Dc, G, N, init):
    """Both kernels: 64-channel groups take the double-buffered tile kernel (runs
    of 32 tokens, 16 for float32 with 32 states; N = 8 reads B and C per element),
    the others the per-lane kernel; ragged last runs, one token."""
    sel_case(inputs.SelectiveShape("sel", 2, T, Dc, G, N, io, init_state=init, seed=T + N))


def test_selective_scan_empty_sequence():
    shape = inputs.SelectiveShape("sel0", 2, 0, 64, 1, 16, "f32", init_state=True)
    inp = inputs.selective_inputs(shape)
    d = {k: (None if v is None else v.cuda()) for k, v in inp.items()}
    _, fs = ssd.ssd_selective_scan(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["init_state"])
    assert torch.equal(fs.cpu(), inp["init_state"])


def test_selective_scan_mamba1_50m_layer_sampled():
    """The Mamba-1 layer workload (batch 64, T 512, 1024 channels, 16 states):
    sampled sequences and channels against the oracle."""
    sel_case(inputs.MAMBA1_50M, sample=([0, 37, 63], [0, 1, 511, 1000, 1023]))
