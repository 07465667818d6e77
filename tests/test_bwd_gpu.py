"""The backward scan on the GPU against the fp64 adjoint (needs a B200).

Gradients of L = sum <dy, y> + <dfinal, final_state> through the real float32
scan, compared element by element over every output; tolerance 1e-4 normwise
(float32 arithmetic against fp64).
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
    p = pins.rand_problem(rng, b, T, H, P, G, N, init=init)
    if not use_D:
        p["D"] = None
    p = {k: (None if v is None else v.astype(np.float32).astype(np.float64)) for k, v in p.items()}
    dy = rng.standard_normal((b, T, H, P)).astype(np.float32).astype(np.float64)
    dfinal = rng.standard_normal((b, H, P, N)).astype(np.float32).astype(np.float64) if use_dfinal else None
    return p, dy, dfinal


def gpu_bwd(p, dy, dfinal):
    d = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()
    out = ssd.ssd_scan_bwd(d(p["x"]), d(p["dt"]), d(p["A"]), d(p["B"]), d(p["C"]), d(p["D"]),
                           d(p["init_state"]), d(dy), d(dfinal))
    ssd.ssd_get_device_status()
    return {k: (None if v is None else v.cpu().numpy()) for k, v in out.items()}


def check(b, T, H, P, G, N, **kw):
    p, dy, dfinal = problem(b, T, H, P, G, N, **kw)
    got = gpu_bwd(p, dy, dfinal)
    ref = oracle.scan_bwd(p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"], p["init_state"], dy, dfinal)
    errs = {k: pins.rel_err(got[k], ref[k]) for k in NAMES if got[k] is not None}
    assert max(errs.values()) <= TOL, errs
    return got


@pytest.mark.parametrize("T", [1, 64, 65, 200])
def test_ragged_and_multi_chunk(T):
    check(2, T, 4, 8, 2, 16, init=(T % 2 == 1), seed=T)


def test_mamba2_head_shape():
    check(1, 256, 8, 64, 2, 128, seed=3)


@pytest.mark.parametrize("T", [1, 65, 200])
def test_tensor_core_phases_ragged(T):
    """Head dim 64 and d_state 128 take the tcgen05 chunk-state and readout
    kernels (and, with heads sharing a group, the per-group C B^T): ragged last
    chunks, one token, optional inputs absent."""
    check(2, T, 4, 64, 2, 128, init=(T != 65), seed=40 + T)
    got = check(1, T, 2, 64, 1, 128, init=False, use_D=False, use_dfinal=False, seed=50 + T)
    assert got["dD"] is None


def test_tensor_core_phases_bitwise_repeatable():
    p, dy, dfinal = problem(1, 150, 4, 64, 1, 128, seed=8)
    first = gpu_bwd(p, dy, dfinal)
    again = gpu_bwd(p, dy, dfinal)
    for k in NAMES:
        assert np.array_equal(first[k], again[k]), k


def test_optional_inputs_absent():
    got = check(2, 100, 2, 4, 1, 8, init=False, use_D=False, use_dfinal=False, seed=4)
    assert got["dD"] is None


def test_empty_sequence():
    check(2, 0, 3, 4, 1, 8, seed=5)


def test_repeated_calls_are_bitwise_equal():
    p, dy, dfinal = problem(2, 300, 4, 16, 2, 32, seed=6)
    first = gpu_bwd(p, dy, dfinal)
    for _ in range(2):
        again = gpu_bwd(p, dy, dfinal)
        for k in NAMES:
            assert np.array_equal(first[k], again[k]), k
