"""The seeded workload generators follow their stated recipes."""
import math

import torch

from selective_state_space_22_b200 import inputs


def test_real_recipe_ranges_and_determinism():
    a = inputs.scan_inputs(inputs.MAMBA2_1B, seqlen=128)
    b = inputs.scan_inputs(inputs.MAMBA2_1B, seqlen=128)
    for k in ("x", "dt", "A", "B", "C", "D"):
        assert torch.equal(a[k], b[k])
    assert a["x"].dtype == torch.bfloat16 and a["B"].dtype == torch.bfloat16
    assert a["dt"].dtype == torch.float32 and a["A"].dtype == torch.float32
    assert float(a["dt"].min()) >= 1e-3 - 1e-7 and float(a["dt"].max()) <= 0.1 + 1e-7
    assert float(a["A"].max()) <= -1.0 + 1e-6 and float(a["A"].min()) >= -16.0 - 1e-5
    assert a["init_state"] is None
    assert tuple(a["x"].shape) == (2, 128, 64, 64) and tuple(a["B"].shape) == (2, 128, 1, 128)


def test_complex_recipe():
    c = inputs.scan_inputs(inputs.MAMBA3_COMPLEX, seqlen=256)
    assert c["B"].dtype == torch.complex64 and c["x"].dtype == torch.float32
    assert float(c["A"].real.max()) <= -0.5 and float(c["A"].real.min()) >= -2.0
    assert float(c["A"].imag.abs().max()) <= math.pi + 1e-6
    var = float(c["B"].real.var())
    assert abs(var - 0.5) < 0.02, var


def test_long_has_init_state():
    d = inputs.scan_inputs(inputs.LONG, seqlen=64)
    assert d["init_state"] is not None and d["init_state"].dtype == torch.float32


def test_widen_is_exact():
    a = inputs.scan_inputs(inputs.MAMBA2_1B, seqlen=16)
    w = inputs.widen(a["x"])
    assert w.dtype.name == "float64"
    assert torch.equal(torch.from_numpy(w).to(torch.bfloat16), a["x"])
