"""The one-step decode update vs the oracle (needs a B200)."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_22_b200 as ssd
from selective_state_space_22_b200 import inputs
from parity import TOL_BF16, TOL_F32, elem_rel_err, oracle_pool_map, _scan_unit, rel_err

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


def test_decode_bitmamba_1024_steps_sampled():
    """The decode workload as stated: 256 sequences at the BitMamba-1B head shape
    (64 heads, head dim 64, d_state 128, bf16 x/B/C/y, float32 state) advanced by
    1024 consecutive in-place calls.  y of every step and the state after the
    last one are compared with the oracle on 8 sampled sequences (all 64 heads
    each).  The oracle's decode step applied 1024 times equals its scan over the
    same 1024 tokens (a pin of the oracle), so each sampled sequence is one
    oracle scan, run in a process pool."""
    shape = inputs.DECODE
    assert shape.steps == 1024
    samples = [0, 37, 74, 111, 148, 185, 222, 255]
    gen, const = inputs.decode_setup(shape)
    A, D = const["A"].cuda(), const["D"].cuda()
    st_gpu = const["state"].cuda()
    keep = {k: [] for k in ("x", "dt", "B", "C")}
    ys = []
    idx = torch.tensor(samples)
    for _ in range(shape.steps):
        s = inputs.decode_step_inputs(gen, shape)
        d = {k: v.cuda() for k, v in s.items()}
        y = ssd.ssd_state_update(st_gpu, d["x"], d["dt"], A, d["B"], d["C"], D)
        ys.append(y.index_select(0, idx.cuda()).float().cpu())
        for k in keep:
            keep[k].append(s[k].index_select(0, idx))
    ssd.ssd_get_device_status()
    st_got = st_gpu.index_select(0, idx.cuda()).cpu().numpy()
    y_got = torch.stack(ys, 1).numpy()                      # [8, 1024, H, P]
    seq = {k: torch.stack(v, 1) for k, v in keep.items()}   # [8, 1024, ...]
    c = np.ascontiguousarray
    jobs = []
    for i, sidx in enumerate(samples):
        jobs.append((c(inputs.widen(seq["x"][i:i + 1])), c(inputs.widen(seq["dt"][i:i + 1])),
                     inputs.widen(const["A"]), c(inputs.widen(seq["B"][i:i + 1])),
                     c(inputs.widen(seq["C"][i:i + 1])), inputs.widen(const["D"]),
                     c(inputs.widen(const["state"][sidx:sidx + 1]))))
    ref = oracle_pool_map(_scan_unit, jobs)
    y_ref = np.concatenate([r[0] for r in ref])
    st_ref = np.concatenate([r[1] for r in ref])
    ey, es = rel_err(y_got, y_ref), rel_err(st_got, st_ref)
    print(f"decode 1024 steps, 8 sequences: y {ey:.2e} (per element {elem_rel_err(y_got, y_ref):.2e}), "
          f"state {es:.2e} (per element {elem_rel_err(st_got, st_ref):.2e})")
    assert ey <= TOL_BF16, ey
    assert es <= TOL_F32, es
