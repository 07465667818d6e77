"""The oracle on two problems worked out by hand (tests/golden/hand_worked.json)."""
import json
import os

import numpy as np

import oracle

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")))
TOL = 1e-12


def _arr(v, shape, cplx=False):
    a = np.asarray(v, np.float64)
    if cplx:
        a = a.reshape(-1, 2)
        a = a[:, 0] + 1j * a[:, 1]
    return np.ascontiguousarray(a.reshape(shape))


def test_hand_worked_real():
    g = GOLD["real"]
    d = g["dims"]
    b, T, H, P, G, N = (d[k] for k in ("batch", "seqlen", "nheads", "headdim", "ngroups", "dstate"))
    args = dict(x=_arr(g["x"], (b, T, H, P)), dt=_arr(g["dt"], (b, T, H)), A=_arr(g["A"], (H,)),
                B=_arr(g["B"], (b, T, G, N)), C=_arr(g["C"], (b, T, G, N)), D=_arr(g["D"], (H,)),
                init_state=_arr(g["init_state"], (b, H, P, N)))
    y, fs = oracle.scan(**args)
    assert np.max(np.abs(y - _arr(g["y"], (b, T, H, P)))) < TOL
    assert np.max(np.abs(fs - _arr(g["final_state"], (b, H, P, N)))) < TOL
    # the same two steps through the decode entry point
    st = args["init_state"]
    for t in range(T):
        yt, st = oracle.state_update(st, np.ascontiguousarray(args["x"][:, t]),
                                     np.ascontiguousarray(args["dt"][:, t]), args["A"],
                                     np.ascontiguousarray(args["B"][:, t]),
                                     np.ascontiguousarray(args["C"][:, t]), args["D"])
        assert np.max(np.abs(yt - _arr(g["y"], (b, T, H, P))[:, t])) < TOL
    assert np.max(np.abs(st - _arr(g["final_state"], (b, H, P, N)))) < TOL


def test_hand_worked_complex():
    g = GOLD["complex"]
    d = g["dims"]
    b, T, H, P, G, N = (d[k] for k in ("batch", "seqlen", "nheads", "headdim", "ngroups", "dstate"))
    args = dict(x=_arr(g["x"], (b, T, H, P)), dt=_arr(g["dt"], (b, T, H)),
                A=_arr(g["A"], (H,), True), B=_arr(g["B"], (b, T, G, N), True),
                C=_arr(g["C"], (b, T, G, N), True), D=_arr(g["D"], (H,)),
                init_state=_arr(g["init_state"], (b, H, P, N), True))
    y, fs = oracle.scan(**args)
    assert np.max(np.abs(y - _arr(g["y"], (b, T, H, P)))) < TOL
    assert np.max(np.abs(fs - _arr(g["final_state"], (b, H, P, N), True))) < TOL
