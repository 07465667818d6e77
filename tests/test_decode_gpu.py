"""The one-step decode update vs the oracle (needs a B200)."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_22_b200 as ssd
from selective_state_space_22_b200 import inputs
from parity import TOL_BF16, TOL_F32, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def run_steps(shape, steps, sample=None, cplx=False):
    gen, const = inputs.decode_setup(shape)
    A, D, state = const["A"], const["D"], const["state"]
    if cplx:
        g2 = torch.Generator().manual_seed(shape.seed + 100)
        A = torch.complex(-(torch.rand(shape.nheads, generator=g2) * 1.5 + 0.5),
                          (torch.rand(shape.nheads, generator=g2) * 2 - 1) * 3.14159)
        state = torch.complex(state, torch.randn(state.shape, generator=g2))
    st_gpu = state.cuda()
    st_ref = inputs.widen(state)
    bs = range(shape.batch) if sample is None else [s[0] for s in sample]
    worst = 0.0
    for _ in range(steps):
        s = inputs.decode_step_inputs(gen, shape)
        if cplx:
            s["B"] = torch.complex(s["B"].float(), s["C"].float().flip(-1))
            s["C"] = torch.complex(s["C"].float(), s["B"].real.flip(-1))
            s["x"] = s["x"].float()
        d = {k: v.cuda() for k, v in s.items()}
        fn = ssd.ssd_state_update_complex if cplx else ssd.ssd_state_update
        y = fn(st_gpu, d["x"], d["dt"], A.cuda(), d["B"], d["C"], D.cuda())
        w = inputs.widen_all(s)
        y_ref, st_ref = oracle.state_update(st_ref, w["x"], w["dt"], inputs.widen(A), w["B"], w["C"],
                                            inputs.widen(D))
        worst = max(worst, rel_err(y.float().cpu().numpy(), y_ref))
    worst = max(worst, rel_err(st_gpu.cpu().numpy(), st_ref))
    return worst


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("N", [128, 256, 40])
def test_decode_real_small(io, N):
    shape = inputs.DecodeShape("dec", 3, 4, 64, 2, N, 5, io_dtype=io, seed=77)
    err = run_steps(shape, 5)
    assert err <= (TOL_F32 if io == "f32" else TOL_BF16), err


def test_decode_complex_small():
    shape = inputs.DecodeShape("decc", 2, 4, 16, 4, 64, 4, io_dtype="f32", seed=78)
    assert run_steps(shape, 4, cplx=True) <= TOL_F32


def test_decode_bitmamba_shape_steps():
    """The full decode shape (256 sequences, H64 P64 N128), several steps, all of it."""
    shape = inputs.DECODE
    err = run_steps(shape, 4)
    assert err <= TOL_BF16, err
