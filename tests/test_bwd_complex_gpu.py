"""The complex backward scan on the GPU against the fp64 complex adjoint (needs a B200).

Same checks as the real backward's GPU test, for the Mamba-3-Lite variant:
every gradient element by element, tolerance 1e-4 normwise.
"""
import numpy as np
import pytest
import torch

import oracle
import pins
import selective_state_space_22_b200 as ssd

pytestmark = pytest.mark.gpu
TOL = 1e-4
NAMES = ("dx", "ddt", "dA", "dB", "dC", "dD", "dinit")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ssd.load_library()


def problem(b, T, H, P, G, N, init=True, use_D=True, use_dfinal=True, seed=0):
    rng = np.random.default_rng(seed)
    p = pins.rand_problem(rng, b, T, H, P, G, N, cplx=True, init=init)
    if not use_D:
        p["D"] = None
    narrow = {True: np.complex64, False: np.float32}
    wide = {True: np.complex128, False: np.float64}
    p = {k: (None if v is None else v.astype(narrow[np.iscomplexobj(v)]).astype(wide[np.iscomplexobj(v)]))
         for k, v in p.items()}
    dy = rng.standard_normal((b, T, H, P)).astype(np.float32).astype(np.float64)
    dfinal = None
    if use_dfinal:
        shp = (b, H, P, N)
        dfinal = (rng.standard_normal(shp) + 1j * rng.standard_normal(shp)).astype(np.complex64).astype(np.complex128)
    return p, dy, dfinal


def to_dev(a):
    if a is None:
        return None
    dt = np.complex64 if np.iscomplexobj(a) else np.float32
    return torch.from_numpy(np.ascontiguousarray(a, dt)).cuda()


def check(b, T, H, P, G, N, **kw):
    p, dy, dfinal = problem(b, T, H, P, G, N, **kw)
    out = ssd.ssd_scan_bwd_complex(to_dev(p["x"]), to_dev(p["dt"]), to_dev(p["A"]), to_dev(p["B"]),
                                   to_dev(p["C"]), to_dev(p["D"]), to_dev(p["init_state"]), to_dev(dy),
                                   to_dev(dfinal))
    ssd.ssd_get_device_status()
    got = {k: (None if v is None else v.cpu().numpy()) for k, v in out.items()}
    ref = oracle.scan_bwd(p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"], p["init_state"], dy, dfinal)
    errs = {k: pins.rel_err(got[k], ref[k]) for k in NAMES if got[k] is not None}
    assert max(errs.values()) <= TOL, errs
    return got


@pytest.mark.parametrize("T", [1, 32, 33, 100])
def test_complex_ragged_and_multi_chunk(T):
    check(2, T, 4, 8, 2, 16, init=(T % 2 == 1), seed=T)


def test_complex_mamba3lite_head_shape():
    check(1, 96, 4, 64, 4, 64, seed=3)


@pytest.mark.parametrize("T", [1, 33, 70])
def test_complex_tensor_core_phases_ragged(T):
    """Head dim 64 and 64 complex states take the tcgen05 chunk-state and readout
    kernels: ragged last chunks, one token, optional inputs absent."""
    check(2, T, 4, 64, 4, 64, init=(T != 33), seed=40 + T)
    got = check(1, T, 2, 64, 1, 64, init=False, use_D=False, use_dfinal=False, seed=50 + T)
    assert got["dD"] is None


def test_complex_optional_inputs_absent_and_empty():
    got = check(2, 50, 2, 4, 1, 8, init=False, use_D=False, use_dfinal=False, seed=4)
    assert got["dD"] is None
    check(2, 0, 3, 4, 1, 8, seed=5)
