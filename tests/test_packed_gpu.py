"""The complex scan fed from the packed projection output (needs a B200).

ssd_scan_fwd_complex_packed reads x, B, C and dt straight from the
[b, T, H (P + 4N + 1)] projection output ("Block Anatomy, Numerical Stability &
Scaling", Block Anatomy 4.1-4.3) and applies softplus(dt + dt_bias) itself.
Its result is compared with the oracle fed the unpacked slices (widened
exactly; dt = log(1 + exp(dt_raw + dt_bias)) in float64), and with the library's
own scan given the unpacked tensors.
"""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_22_b200 as ssd
from selective_state_space_22_b200 import inputs
from parity import TOL_F32, elem_rel_err, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ssd.load_library()


def reference(inp, H, P, N):
    u = inputs.unpack_projection(inp["proj"], H, P, N)
    dt = np.log1p(np.exp(u["dt_raw"].numpy() + inputs.widen(inp["dt_bias"])[None, None, :]))
    c = np.ascontiguousarray
    return oracle.scan(c(u["x"].numpy()), c(dt), inputs.widen(inp["A"]), c(u["B"].numpy()), c(u["C"].numpy()),
                       inputs.widen(inp["D"]), inputs.widen(inp["init_state"])), u, dt


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T,P,N", [(300, 64, 64), (129, 64, 64), (200, 32, 16)])
def test_packed_matches_the_oracle(dtype, T, P, N):
    shape = inputs.ScanShape("packed", 2, T, 3, P, 3, N, 128, dtype, complex=True, init_state=True, seed=T + P)
    inp = inputs.packed_inputs(shape, dtype)
    d = {k: (None if v is None else v.cuda()) for k, v in inp.items()}
    y, fs = ssd.ssd_scan_fwd_complex_packed(d["proj"], d["A"], d["D"], d["init_state"], nheads=3, headdim=P,
                                            dstate=N, dt_bias=d["dt_bias"], chunk_size=128)
    ssd.ssd_get_device_status()
    (y_ref, fs_ref), u, dt = reference(inp, 3, P, N)
    ey, ef = rel_err(y.cpu().numpy(), y_ref), rel_err(fs.cpu().numpy(), fs_ref)
    print(f"packed {dtype} T={T} P={P} N={N}: y {ey:.2e} (per element {elem_rel_err(y.cpu().numpy(), y_ref):.2e}), "
          f"final {ef:.2e}")
    assert ey <= TOL_F32 and ef <= TOL_F32, (ey, ef)
    # the same values unpacked, through the scan that takes separate tensors
    f = lambda t: t.to(torch.float32).cuda()
    y2, fs2 = ssd.ssd_scan_fwd_complex(f(u["x"]), torch.from_numpy(dt).float().cuda(), d["A"],
                                       u["B"].to(torch.complex64).cuda(), u["C"].to(torch.complex64).cuda(), d["D"],
                                       d["init_state"], chunk_size=128)
    assert rel_err(y.cpu().numpy(), y2.cpu().numpy()) <= TOL_F32


def test_packed_layer_shape_sampled():
    """The Mamba-3-Lite layer (batch 4, T 2048, 16 heads, head dim 64, 64 complex
    states) from a bf16 projection: sampled heads against the oracle."""
    shape = inputs.MAMBA3_PACKED
    inp = inputs.packed_inputs(shape, "bf16")
    d = {k: (None if v is None else v.cuda()) for k, v in inp.items()}
    H, P, N = shape.nheads, shape.headdim, shape.dstate
    y, fs = ssd.ssd_scan_fwd_complex_packed(d["proj"], d["A"], d["D"], None, nheads=H, headdim=P, dstate=N,
                                            dt_bias=d["dt_bias"], chunk_size=shape.chunk)
    ssd.ssd_get_device_status()
    u = inputs.unpack_projection(inp["proj"], H, P, N)
    dt = np.log1p(np.exp(u["dt_raw"].numpy() + inputs.widen(inp["dt_bias"])[None, None, :]))
    c = np.ascontiguousarray
    for b, h in [(0, 0), (3, 15), (1, 7)]:
        y_ref, fs_ref = oracle.scan(c(u["x"].numpy()[b:b + 1, :, h:h + 1]), c(dt[b:b + 1, :, h:h + 1]),
                                    inputs.widen(inp["A"])[h:h + 1], c(u["B"].numpy()[b:b + 1, :, h:h + 1]),
                                    c(u["C"].numpy()[b:b + 1, :, h:h + 1]), inputs.widen(inp["D"])[h:h + 1], None)
        assert rel_err(y.cpu().numpy()[b:b + 1, :, h:h + 1], y_ref) <= TOL_F32
        assert rel_err(fs.cpu().numpy()[b:b + 1, h:h + 1], fs_ref) <= TOL_F32
