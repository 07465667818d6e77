"""Both backward scans at the shapes bench.py times them, against the fp64 adjoint.

The real one at the Mamba-2 BitMamba-1B layer shape (batch 2, T 2048, 64 heads,
head dim 64, d_state 128, one group: 32 chunks of 64 tokens, dB and dC summed
over all 64 heads), the complex one at the Mamba-3-Lite layer shape (batch 4,
T 2048, 16 heads, head dim 64, d_state 64 complex, one group per head), on the
seeded inputs and upstream gradients of those bench workloads.

The oracle's adjoint runs on every (batch, head) sequence in a process pool; the
per-sequence gradients of the shared tensors (dB, dC over the heads of a group;
dA, dD over batch) are summed with numpy.  Every element of all seven gradients
is compared, normwise 1e-4 per gradient (float32 against fp64).
"""
import numpy as np
import pytest
import torch

import selective_state_space_22_b200 as ssd
from selective_state_space_22_b200 import inputs
from parity import TOL_F32, _bwd_unit, elem_rel_err, oracle_pool_map, rel_err

pytestmark = pytest.mark.gpu
NAMES = ("dx", "ddt", "dA", "dB", "dC", "dD", "dinit")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ssd.load_library()


def oracle_bwd_units(w, dy, dfinal):
    b, T, H, P = w["x"].shape
    G = w["B"].shape[2]
    cplx = np.iscomplexobj(w["A"])
    c = np.ascontiguousarray
    units = [(bi, h) for bi in range(b) for h in range(H)]
    jobs = []
    for bi, h in units:
        g = h // (H // G)
        jobs.append((c(w["x"][bi:bi + 1, :, h:h + 1]), c(w["dt"][bi:bi + 1, :, h:h + 1]), c(w["A"][h:h + 1]),
                     c(w["B"][bi:bi + 1, :, g:g + 1]), c(w["C"][bi:bi + 1, :, g:g + 1]),
                     c(w["D"][h:h + 1]), c(w["init_state"][bi:bi + 1, h:h + 1]),
                     c(dy[bi:bi + 1, :, h:h + 1]), c(dfinal[bi:bi + 1, h:h + 1])))
    outs = oracle_pool_map(_bwd_unit, jobs)
    sdt = np.complex128 if cplx else np.float64
    ref = dict(dx=np.zeros_like(w["x"]), ddt=np.zeros_like(w["dt"]), dA=np.zeros(H, sdt),
               dB=np.zeros(w["B"].shape, sdt), dC=np.zeros(w["C"].shape, sdt), dD=np.zeros(H),
               dinit=np.zeros(w["init_state"].shape, sdt))
    for (bi, h), o in zip(units, outs):
        g = h // (H // G)
        ref["dx"][bi, :, h] = o["dx"][0, :, 0]
        ref["ddt"][bi, :, h] = o["ddt"][0, :, 0]
        ref["dinit"][bi, h] = o["dinit"][0, 0]
        ref["dA"][h] += o["dA"][0]
        ref["dD"][h] += o["dD"][0]
        ref["dB"][bi, :, g] += o["dB"][0, :, 0]
        ref["dC"][bi, :, g] += o["dC"][0, :, 0]
    return ref


def run(shape):
    inp = inputs.scan_inputs(shape)
    up = inputs.bwd_upstream(shape)
    d = {k: (None if v is None else v.cuda()) for k, v in inp.items()}
    fn = ssd.ssd_scan_bwd_complex if shape.complex else ssd.ssd_scan_bwd
    got = fn(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["init_state"], up["dy"].cuda(),
             up["dfinal"].cuda())
    ssd.ssd_get_device_status()
    got = {k: v.cpu().numpy() for k, v in got.items()}
    ref = oracle_bwd_units(inputs.widen_all(inp), inputs.widen(up["dy"]), inputs.widen(up["dfinal"]))
    errs = {k: rel_err(got[k], ref[k]) for k in NAMES}
    info = {k: elem_rel_err(got[k], ref[k]) for k in NAMES}
    print(shape.name, "normwise", {k: f"{v:.1e}" for k, v in errs.items()},
          "per element", {k: f"{v:.1e}" for k, v in info.items()})
    assert max(errs.values()) <= TOL_F32, errs


def test_bwd_at_mamba2_layer_shape():
    assert (inputs.BWD.batch, inputs.BWD.seqlen, inputs.BWD.nheads, inputs.BWD.ngroups) == (2, 2048, 64, 1)
    run(inputs.BWD)


def test_bwd_complex_at_mamba3lite_layer_shape():
    s = inputs.BWD_COMPLEX
    assert (s.batch, s.seqlen, s.nheads, s.ngroups, s.dstate) == (4, 2048, 16, 16, 64)
    run(s)
