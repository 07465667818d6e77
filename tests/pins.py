"""Checks that pin the fp64 oracle to something other than itself.

Each pin takes a loaded oracle library handle (so the same checks can be run
against deliberately broken copies of the oracle) and returns the largest
normwise error it saw.  The independent formulations here are:

* the materialised quadratic (semiseparable-matrix) form of the scan, by brute
  force over all (t, s) pairs for T <= 8;
* the chunkwise algorithm as the Mamba-3-Lite pages lay it out ("Block
  Anatomy, Numerical Stability & Scaling", Numerical Stability section 4):
  inclusive within-chunk cumulative log-decay, intra-chunk decay
  L[l, s] = exp(A_cs[l] - A_cs[s]) for l >= s, end-of-chunk states, and the
  strict-lower-triangular inter-chunk propagation exp(CD[z-1] - CD[c]) with
  exp(CD[z-1]) for the initial state;
* closed forms (zero input gives pure decay; A = 0 gives a prefix sum);
* the complex state written as a real 2-vector under a 2x2 decay-rotation;
* invariants: linearity, state continuation, decode steps equal the scan,
  the contraction bound, complex with zero imaginary parts equal to real.
"""
from __future__ import annotations

import math

import numpy as np

import oracle


def rel_err(got, ref) -> float:
    got = np.asarray(got)
    ref = np.asarray(ref)
    den = float(np.max(np.abs(ref))) if ref.size else 0.0
    num = float(np.max(np.abs(got - ref))) if ref.size else 0.0
    return num / den if den > 0 else num


def rand_problem(rng, b, T, H, P, G, N, cplx=False, init=True, dt_hi=0.1, a_range=(1.0, 16.0)):
    x = rng.standard_normal((b, T, H, P))
    dt = np.exp(rng.uniform(math.log(1e-3), math.log(dt_hi), (b, T, H)))
    if cplx:
        A = -rng.uniform(0.5, 2.0, H) + 1j * rng.uniform(-math.pi, math.pi, H)
        B = (rng.standard_normal((b, T, G, N)) + 1j * rng.standard_normal((b, T, G, N))) / math.sqrt(2)
        C = (rng.standard_normal((b, T, G, N)) + 1j * rng.standard_normal((b, T, G, N))) / math.sqrt(2)
        h0 = (rng.standard_normal((b, H, P, N)) + 1j * rng.standard_normal((b, H, P, N))) if init else None
    else:
        A = -rng.uniform(*a_range, H)
        B = rng.standard_normal((b, T, G, N))
        C = rng.standard_normal((b, T, G, N))
        h0 = rng.standard_normal((b, H, P, N)) if init else None
    D = rng.standard_normal(H)
    c = lambda a: None if a is None else np.ascontiguousarray(a)
    return dict(x=c(x), dt=c(dt), A=c(A), B=c(B), C=c(C), D=c(D), init_state=c(h0))


def run(lib, p, **over):
    q = dict(p)
    q.update(over)
    return oracle.scan(q["x"], q["dt"], q["A"], q["B"], q["C"], q["D"], q["init_state"], lib=lib)


# ---------------------------------------------------------------- brute force
def brute_force(p):
    """Quadratic form: y_t = sum_{s<=t} (C_t . B_s) e^{A sum_{s<u<=t} dt_u} dt_s x_s
    + e^{A sum_{u<=t} dt_u} (h0 C_t) + D x_t, and the matching final state."""
    x, dt, A, B, C, D, h0 = (p[k] for k in ("x", "dt", "A", "B", "C", "D", "init_state"))
    b, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    cplx = np.iscomplexobj(A)
    y = np.zeros((b, T, H, P))
    fs = np.zeros((b, H, P, N), complex if cplx else float)
    for bi in range(b):
        for h in range(H):
            g = h // (H // G)
            for t in range(T):
                acc = np.zeros(P, complex)
                for s in range(t + 1):
                    decay = np.exp(A[h] * dt[bi, s + 1:t + 1, h].sum())
                    cb = np.sum(C[bi, t, g, :] * B[bi, s, g, :])
                    acc += cb * decay * dt[bi, s, h] * x[bi, s, h, :]
                if h0 is not None:
                    acc += np.exp(A[h] * dt[bi, :t + 1, h].sum()) * (h0[bi, h] @ C[bi, t, g, :])
                y[bi, t, h, :] = acc.real + (D[h] * x[bi, t, h, :] if D is not None else 0.0)
            st = np.zeros((P, N), complex)
            for s in range(T):
                decay = np.exp(A[h] * dt[bi, s + 1:T, h].sum())
                st += decay * dt[bi, s, h] * np.outer(x[bi, s, h, :], B[bi, s, g, :])
            if h0 is not None:
                st += np.exp(A[h] * dt[bi, :, h].sum()) * h0[bi, h]
            fs[bi, h] = st if cplx else st.real
    return y, fs


def pin_brute_force(lib, cplx=False, seed=1):
    err = 0.0
    rng = np.random.default_rng(seed)
    for (b, T, H, P, G, N) in [(1, 1, 1, 1, 1, 1), (2, 5, 4, 3, 2, 5), (1, 8, 2, 2, 1, 3),
                               (1, 8, 4, 2, 4, 2)]:
        for init in (False, True):
            p = rand_problem(rng, b, T, H, P, G, N, cplx=cplx, init=init, dt_hi=0.5)
            y, fs = run(lib, p)
            y_ref, fs_ref = brute_force(p)
            err = max(err, rel_err(y, y_ref), rel_err(fs, fs_ref))
    return err


# ---------------------------------------------------- the pages' chunkwise form
def chunkwise(p, Q):
    """Chunked SSD in the pages' decay_chunk form, fp64/complex128, per (b, h)."""
    x, dt, A, B, C, D, h0 = (p[k] for k in ("x", "dt", "A", "B", "C", "D", "init_state"))
    b, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    cplx = np.iscomplexobj(A)
    nc = max(1, -(-T // Q))
    Tp = nc * Q
    y = np.zeros((b, T, H, P))
    fs = np.zeros((b, H, P, N), complex if cplx else float)
    for bi in range(b):
        for h in range(H):
            g = h // (H // G)
            # pad to whole chunks with dt = 0 and x = 0 (decay 1, nothing injected)
            xp = np.zeros((Tp, P)); xp[:T] = x[bi, :, h]
            dtp = np.zeros(Tp); dtp[:T] = dt[bi, :, h]
            Bp = np.zeros((Tp, N), complex); Bp[:T] = B[bi, :, g]
            Cp = np.zeros((Tp, N), complex); Cp[:T] = C[bi, :, g]
            xc, dtc = xp.reshape(nc, Q, P), dtp.reshape(nc, Q)
            Bc, Cc = Bp.reshape(nc, Q, N), Cp.reshape(nc, Q, N)
            A_cs = np.cumsum(dtc * A[h], axis=1)                      # inclusive, per chunk
            seg = A_cs[:, :, None] - A_cs[:, None, :]                 # [c, l, s]
            mask = np.tril(np.ones((Q, Q), bool))
            L = np.where(mask, np.exp(np.where(mask, seg, 0.0)), 0.0)
            G_ls = np.einsum("cln,csn->cls", Cc, Bc)
            Y_diag = np.einsum("cls,cs,csp->clp", G_ls * L, dtc, xc)
            decay_states = np.exp(A_cs[:, -1:] - A_cs)                # [c, s]
            S = np.einsum("cs,cs,csp,csn->cpn", decay_states, dtc, xc, Bc)
            Lam = A_cs[:, -1]
            CD = np.cumsum(Lam)
            h_in = np.zeros((nc + 1, P, N), complex)
            for z in range(nc + 1):
                cdz = CD[z - 1] if z > 0 else 0.0
                for c in range(z):                                  # strict tril: c < z
                    h_in[z] += np.exp(cdz - CD[c]) * S[c]
                if h0 is not None:
                    h_in[z] += np.exp(cdz) * h0[bi, h]
            Y_off = np.einsum("cl,cln,cpn->clp", np.exp(A_cs), Cc, h_in[:nc])
            yy = (Y_diag + Y_off).reshape(Tp, P)[:T].real
            y[bi, :, h] = yy + (D[h] * x[bi, :, h] if D is not None else 0.0)
            fs[bi, h] = h_in[nc] if cplx else h_in[nc].real
    return y, fs


def pin_chunkwise(lib, cplx=False, seed=2):
    err = 0.0
    rng = np.random.default_rng(seed)
    T = 67
    p = rand_problem(rng, 2, T, 4, 3, 2, 4, cplx=cplx, init=True)
    y, fs = run(lib, p)
    for Q in (1, 2, 3, 4, 16, 64, T, 100):
        y_ref, fs_ref = chunkwise(p, Q)
        err = max(err, rel_err(y, y_ref), rel_err(fs, fs_ref))
    return err


# ------------------------------------------------------------------ closed forms
def pin_zero_input(lib, cplx=False, seed=3):
    """x = 0: the state only decays, S_t = e^{A sum_{u<=t} dt_u} h0, y_t = Re(S_t C_t)."""
    rng = np.random.default_rng(seed)
    p = rand_problem(rng, 1, 12, 2, 3, 1, 4, cplx=cplx, init=True)
    p["x"] = np.zeros_like(p["x"])
    y, fs = run(lib, p)
    cum = np.cumsum(p["dt"], axis=1)                                # [b, T, H]
    err = 0.0
    for h in range(2):
        for t in range(12):
            St = np.exp(p["A"][h] * cum[0, t, h]) * p["init_state"][0, h]
            err = max(err, rel_err(y[0, t, h], (St @ p["C"][0, t, 0]).real))
        ref_fs = np.exp(p["A"][h] * cum[0, -1, h]) * p["init_state"][0, h]
        err = max(err, rel_err(fs[0, h], ref_fs))
    return err


def pin_prefix_sum(lib, cplx=False, seed=4):
    """A = 0: no decay, S_t = h0 + sum_{s<=t} dt_s x_s B_s^T (a running sum)."""
    rng = np.random.default_rng(seed)
    p = rand_problem(rng, 1, 10, 2, 2, 2, 3, cplx=cplx, init=True)
    p["A"] = np.zeros_like(p["A"])
    y, fs = run(lib, p)
    err = 0.0
    for h in range(2):
        S = p["init_state"][0, h].astype(complex)
        for t in range(10):
            S = S + p["dt"][0, t, h] * np.outer(p["x"][0, t, h], p["B"][0, t, h])
            ref = (S @ p["C"][0, t, h]).real + p["D"][h] * p["x"][0, t, h]
            err = max(err, rel_err(y[0, t, h], ref))
        err = max(err, rel_err(fs[0, h], S if cplx else S.real))
    return err


# ------------------------------------------------------------------ invariants
def pin_linearity(lib, cplx=False, seed=5):
    rng = np.random.default_rng(seed)
    p = rand_problem(rng, 1, 20, 2, 3, 1, 4, cplx=cplx, init=False)
    p["D"] = None
    x1 = p["x"]
    x2 = np.ascontiguousarray(rng.standard_normal(x1.shape))
    y1, f1 = run(lib, p, x=x1)
    y2, f2 = run(lib, p, x=x2)
    y3, f3 = run(lib, p, x=np.ascontiguousarray(2.5 * x1 - 0.75 * x2))
    err = max(rel_err(y3, 2.5 * y1 - 0.75 * y2), rel_err(f3, 2.5 * f1 - 0.75 * f2))
    # linear in the initial state at zero input
    q = rand_problem(rng, 1, 20, 2, 3, 1, 4, cplx=cplx, init=True)
    q["x"] = np.zeros_like(q["x"])
    ha = q["init_state"]
    hb = np.ascontiguousarray(rng.standard_normal(ha.shape) * (1 + 0j if cplx else 1))
    ya, fa = run(lib, q, init_state=ha)
    yb, fb = run(lib, q, init_state=hb)
    yc, fc = run(lib, q, init_state=np.ascontiguousarray(ha - 3.0 * hb))
    return max(err, rel_err(yc, ya - 3.0 * yb), rel_err(fc, fa - 3.0 * fb))


def pin_continuation(lib, cplx=False, seed=6):
    """scan(T1 + T2) equals scan(T2) started from the final state of scan(T1)."""
    rng = np.random.default_rng(seed)
    p = rand_problem(rng, 2, 30, 4, 3, 2, 5, cplx=cplx, init=True)
    y, fs = run(lib, p)
    T1 = 13
    first = {k: (np.ascontiguousarray(v[:, :T1]) if k in ("x", "dt", "B", "C") else v)
             for k, v in p.items()}
    second = {k: (np.ascontiguousarray(v[:, T1:]) if k in ("x", "dt", "B", "C") else v)
              for k, v in p.items()}
    y1, f1 = run(lib, first)
    y2, f2 = run(lib, second, init_state=f1)
    return max(rel_err(np.concatenate([y1, y2], axis=1), y), rel_err(f2, fs))


def pin_decode_equals_scan(lib, cplx=False, seed=7):
    rng = np.random.default_rng(seed)
    p = rand_problem(rng, 2, 9, 4, 3, 2, 5, cplx=cplx, init=True)
    y, fs = run(lib, p)
    st = p["init_state"]
    err = 0.0
    for t in range(9):
        yt, st = oracle.state_update(st, np.ascontiguousarray(p["x"][:, t]),
                                     np.ascontiguousarray(p["dt"][:, t]), p["A"],
                                     np.ascontiguousarray(p["B"][:, t]),
                                     np.ascontiguousarray(p["C"][:, t]), p["D"], lib=lib)
        err = max(err, rel_err(yt, y[:, t]))
    return max(err, rel_err(st, fs))


def pin_contraction(lib, cplx=False, seed=8):
    """With Re A <= 0 the state norm is bounded by |h0| + sum of injections."""
    rng = np.random.default_rng(seed)
    p = rand_problem(rng, 1, 40, 1, 2, 1, 3, cplx=cplx, init=True)
    _, fs = run(lib, p)
    bound = np.linalg.norm(p["init_state"][0, 0])
    for t in range(40):
        bound += np.linalg.norm(p["dt"][0, t, 0] * np.outer(p["x"][0, t, 0], p["B"][0, t, 0]))
    return 0.0 if np.linalg.norm(fs[0, 0]) <= bound * (1 + 1e-12) else 1.0


def pin_complex_zero_imag_is_real(lib, seed=9):
    rng = np.random.default_rng(seed)
    p = rand_problem(rng, 2, 15, 4, 3, 2, 5, cplx=False, init=True)
    yr, fr = run(lib, p)
    q = {k: (None if v is None else v) for k, v in p.items()}
    for k in ("A", "B", "C", "init_state"):
        q[k] = np.ascontiguousarray(p[k].astype(np.complex128))
    yc, fc = run(lib, q)
    return max(rel_err(yc, yr), rel_err(fc.real, fr), float(np.max(np.abs(fc.imag))))


def pin_complex_is_rotation_block(lib, seed=10):
    """One complex state component u + iv evolves as a real 2-vector under
    e^{dt a}[[cos dt w, -sin dt w], [sin dt w, cos dt w]] with input dt x (B_r, B_i)
    and readout C_r u - C_i v (the Mamba-3-Lite decay-plus-rotation picture)."""
    rng = np.random.default_rng(seed)
    p = rand_problem(rng, 1, 25, 2, 2, 1, 3, cplx=True, init=True)
    y, fs = run(lib, p)
    err = 0.0
    for h in range(2):
        a, w = p["A"][h].real, p["A"][h].imag
        u = p["init_state"][0, h].real.copy()
        v = p["init_state"][0, h].imag.copy()
        for t in range(25):
            d = p["dt"][0, t, h]
            r = math.exp(d * a)
            cs, sn = math.cos(d * w), math.sin(d * w)
            u, v = r * (cs * u - sn * v), r * (sn * u + cs * v)
            xb = d * p["x"][0, t, h][:, None]
            u = u + xb * p["B"][0, t, 0].real[None, :]
            v = v + xb * p["B"][0, t, 0].imag[None, :]
            ref = u @ p["C"][0, t, 0].real - v @ p["C"][0, t, 0].imag + p["D"][h] * p["x"][0, t, h]
            err = max(err, rel_err(y[0, t, h], ref))
        err = max(err, rel_err(fs[0, h], u + 1j * v))
    return err


def _loss(lib, p, dy, dfinal):
    y, fs = run(lib, p)
    return float(np.sum(y * dy)) + float(np.real(np.sum(np.conj(dfinal) * fs)))


def _dot(g, v) -> float:
    """<g, v> over the real parameters: sum Re(conj(g) v)."""
    return float(np.real(np.sum(np.conj(g) * v)))


def pin_gradient_finite_difference(lib, cplx=False, seed=11):
    """The adjoint (oracle scan_bwd) against central differences of the forward
    oracle, one random direction per input.  The scan is affine in x, B, C, D and
    h0 along any one of them, so there the difference quotient is exact up to
    rounding; dt and A enter through exp, so theirs is Richardson-extrapolated
    (error O(eps^4)).  dt moves by a relative step so it stays positive.  The
    error is taken relative to |g| |v|, the bound on the directional derivative,
    so a direction along which the loss barely moves is not a false alarm."""
    rng = np.random.default_rng(seed)
    err = 0.0
    for (b, T, H, P, G, N) in [(2, 7, 4, 3, 2, 5), (1, 13, 2, 2, 1, 3), (1, 4, 1, 2, 1, 2)]:
        p = rand_problem(rng, b, T, H, P, G, N, cplx=cplx, init=True, a_range=(0.5, 4.0))
        dy = rng.standard_normal((b, T, H, P))
        shp = (b, H, P, N)
        dfin = rng.standard_normal(shp) + (1j * rng.standard_normal(shp) if cplx else 0)
        dfin = np.ascontiguousarray(dfin)
        g = oracle.scan_bwd(p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"], p["init_state"], dy, dfin,
                            lib=lib)
        for name, gname, exact in [("x", "dx", True), ("B", "dB", True), ("C", "dC", True), ("D", "dD", True),
                                   ("init_state", "dinit", True), ("dt", "ddt", False), ("A", "dA", False)]:
            base = p[name]
            v = rng.standard_normal(base.shape)
            if np.iscomplexobj(base):
                v = v + 1j * rng.standard_normal(base.shape)
            if name == "dt":
                v = base * rng.uniform(-1.0, 1.0, base.shape)

            def diff(eps):
                up = _loss(lib, dict(p, **{name: np.ascontiguousarray(base + eps * v)}), dy, dfin)
                dn = _loss(lib, dict(p, **{name: np.ascontiguousarray(base - eps * v)}), dy, dfin)
                return (up - dn) / (2 * eps)

            if exact:
                fd = diff(1e-2)
            else:
                eps = 1e-2
                fd = (4 * diff(eps / 2) - diff(eps)) / 3
            an = _dot(g[gname], v)
            # relative to |g| |v|, the largest the directional derivative can be
            scale = float(np.linalg.norm(g[gname]) * np.linalg.norm(v))
            err = max(err, abs(fd - an) / max(scale, 1e-300))
    return err


def pin_gradient_empty_and_dfinal(lib, cplx=False, seed=12):
    """T = 0: every gradient is zero except dinit = dfinal.  And with dy = 0 and
    a single step, dinit = conj(exp(dt A)) dfinal exactly (the state only decays)."""
    rng = np.random.default_rng(seed)
    p = rand_problem(rng, 1, 0, 2, 2, 1, 3, cplx=cplx, init=True)
    shp = (1, 2, 2, 3)
    dfin = np.ascontiguousarray(rng.standard_normal(shp) + (1j * rng.standard_normal(shp) if cplx else 0))
    g = oracle.scan_bwd(p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"], p["init_state"],
                        np.zeros((1, 0, 2, 2)), dfin, lib=lib)
    err = rel_err(g["dinit"], dfin) + float(np.max(np.abs(g["dA"]))) + float(np.max(np.abs(g["dD"])))
    p = rand_problem(rng, 1, 1, 2, 2, 1, 3, cplx=cplx, init=True)
    g = oracle.scan_bwd(p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"], p["init_state"],
                        np.zeros((1, 1, 2, 2)), dfin, lib=lib)
    a = np.exp(p["dt"][0, 0, :] * p["A"])  # per head
    return err + rel_err(g["dinit"], np.conj(a)[None, :, None, None] * dfin)


def chunked_gradients(p, dy, dfinal, Q):
    """The gradient of L = sum <dy, y> + Re <dfinal, final> evaluated chunk by
    chunk, the way a chunked kernel does it (written independently of the
    sequential adjoint).  Per (batch, head) and chunk, with acs the inclusive
    within-chunk cumulative sum of dt A, Lam = acs[-1], Lm[l, s] = exp(acs[l] -
    acs[s]) for l >= s, Gm = C B^T, w_s = exp(Lam - acs[s]) dt_s and Gh the
    gradient of the chunk's final state:
      dX  = Re(Mc^T dY) + D dY + Re(conj(w) (conj(B) Gh^T)),  Mc = Gm o Lm o dt
      dC  = conj((Lm o dt o dY X^T) B + e^{acs} (dY h_in))
      dB  = conj((Lm o dt o dY X^T)^T C) + conj(w) (X Gh)
      dh_in = conj(e^{Lam}) Gh + (conj(e^{acs}) dY)^T conj(C)   (Gh of the chunk before)
    and the decay gradient through acs: with E = Gm o Lm o dt o (dY X^T),
    dacs = conj(rowsum E - colsum E) + conj(e^{acs} dY.(h_in C)) and, from the
    final state, conj(H0 + sum K) at the last token and -conj(K_s) at each s;
    d alpha is the reverse cumulative sum of dacs, ddt += Re(conj(d alpha) A),
    dA += sum dt d alpha."""
    x, dt, A, B, C, D, h0 = p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"], p["init_state"]
    b, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    cplx = np.iscomplexobj(A)
    sdt = np.complex128 if cplx else np.float64
    re = (lambda z: np.real(z)) if cplx else (lambda z: z)
    Dv = np.zeros(H) if D is None else D
    out = dict(dx=np.zeros_like(x), ddt=np.zeros_like(dt), dA=np.zeros(H, sdt), dB=np.zeros((b, T, G, N), sdt),
               dC=np.zeros((b, T, G, N), sdt), dD=np.zeros(H), dinit=np.zeros((b, H, P, N), sdt))
    hpg = H // G
    for bi in range(b):
        for h in range(H):
            g = h // hpg
            chunks = [(c0, min(c0 + Q, T)) for c0 in range(0, T, Q)]
            # forward over chunks: the state entering each chunk
            hin = []
            hs = np.zeros((P, N), sdt) if h0 is None else h0[bi, h].astype(sdt)
            for c0, c1 in chunks:
                hin.append(hs)
                d = dt[bi, c0:c1, h]
                acs = np.cumsum(d * A[h])
                w = np.exp(acs[-1] - acs) * d
                hs = np.exp(acs[-1]) * hs + (w[:, None] * x[bi, c0:c1, h]).T @ B[bi, c0:c1, g]
            Gh = np.zeros((P, N), sdt) if dfinal is None else dfinal[bi, h].astype(sdt)
            for ci in range(len(chunks) - 1, -1, -1):
                c0, c1 = chunks[ci]
                d = dt[bi, c0:c1, h]
                X, dY = x[bi, c0:c1, h], dy[bi, c0:c1, h]
                Bc, Cc, hi = B[bi, c0:c1, g], C[bi, c0:c1, g], hin[ci]
                acs = np.cumsum(d * A[h])
                lam = acs[-1]
                Lm = np.tril(np.exp(acs[:, None] - acs[None, :]))
                Gm = Cc @ Bc.T
                w = np.exp(lam - acs) * d
                XdY = dY @ X.T  # [l, s] = dy_l . x_s
                Mc = Gm * Lm * d[None, :]
                out["dx"][bi, c0:c1, h] = re(Mc.T @ dY) + Dv[h] * dY + re(np.conj(w)[:, None] * (np.conj(Bc) @ Gh.T))
                out["dD"][h] += float(np.sum(dY * X))
                K = Lm * d[None, :] * XdY
                eacs = np.exp(acs)
                out["dC"][bi, c0:c1, g] += np.conj(K @ Bc + eacs[:, None] * (dY @ hi))
                out["dB"][bi, c0:c1, g] += np.conj(K.T @ Cc) + np.conj(w)[:, None] * (X @ Gh)
                # dt where it multiplies directly (not through the decay)
                ddt_dir = re(np.sum(Gm * Lm * XdY, axis=0)) + re(np.exp(lam - acs) * np.einsum(
                    "sp,pn,sn->s", X, np.conj(Gh), Bc))
                # decay: gradient with respect to acs, then alpha = dt A
                E = Gm * Lm * d[None, :] * XdY
                F = eacs * np.einsum("lp,pn,ln->l", dY, hi, Cc)
                Ks = w * np.einsum("sp,pn,sn->s", X, np.conj(Gh), Bc)
                H0 = np.exp(lam) * np.sum(np.conj(Gh) * hi)
                dacs = np.conj(E.sum(axis=1) - E.sum(axis=0)) + np.conj(F) - np.conj(Ks)
                dacs[-1] += np.conj(H0 + Ks.sum())
                dalpha = np.cumsum(dacs[::-1])[::-1]
                out["ddt"][bi, c0:c1, h] = ddt_dir + re(np.conj(dalpha) * A[h])
                out["dA"][h] += np.sum(d * dalpha)
                Gh = np.conj(np.exp(lam)) * Gh + (np.conj(eacs)[:, None] * dY).T @ np.conj(Cc)
            out["dinit"][bi, h] = Gh
    return out


def pin_gradient_chunkwise(lib, cplx=False, seed=13):
    """The sequential adjoint equals the chunked gradient above for several chunk
    sizes (1, ragged, one chunk, larger than T)."""
    rng = np.random.default_rng(seed)
    err = 0.0
    for (b, T, H, P, G, N, Qs) in [(2, 23, 4, 3, 2, 5, (1, 4, 7, 23, 40)), (1, 9, 2, 2, 1, 3, (2, 9))]:
        p = rand_problem(rng, b, T, H, P, G, N, cplx=cplx, init=True)
        dy = rng.standard_normal((b, T, H, P))
        shp = (b, H, P, N)
        dfin = np.ascontiguousarray(rng.standard_normal(shp) + (1j * rng.standard_normal(shp) if cplx else 0))
        ref = oracle.scan_bwd(p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"], p["init_state"], dy, dfin, lib=lib)
        for Q in Qs:
            got = chunked_gradients(p, dy, dfin, Q)
            for k in ref:
                err = max(err, rel_err(got[k], ref[k]))
    return err


# ----------------------------------------------------------- the variants
def pin_conv1d_library(lib, seed=20):
    """The causal depthwise convolution equals numpy's full convolution of each
    channel with its reversed kernel, cut to the first T outputs (a library
    routine), plus the bias; SiLU equals torch's; the identity kernel returns
    the input and the one-step shift kernel the input delayed by one token."""
    import torch

    rng = np.random.default_rng(seed)
    err = 0.0
    b, T, Cn, K = 2, 11, 5, 4
    x = rng.standard_normal((b, T, Cn))
    w = rng.standard_normal((Cn, K))
    bias = rng.standard_normal(Cn)
    ref = np.zeros_like(x)
    for bi in range(b):
        for c in range(Cn):
            ref[bi, :, c] = np.convolve(x[bi, :, c], w[c, ::-1])[:T] + bias[c]
    err = max(err, rel_err(oracle.causal_conv1d(x, w, bias, lib=lib), ref))
    silu = torch.nn.functional.silu(torch.from_numpy(ref)).numpy()
    err = max(err, rel_err(oracle.causal_conv1d(x, w, bias, silu=True, lib=lib), silu))
    eye = np.zeros((Cn, K))
    eye[:, K - 1] = 1.0
    err = max(err, rel_err(oracle.causal_conv1d(x, eye, lib=lib), x))
    shift = np.zeros((Cn, K))
    shift[:, K - 2] = 1.0
    delayed = np.concatenate([np.zeros((b, 1, Cn)), x[:, :-1]], axis=1)
    err = max(err, rel_err(oracle.causal_conv1d(x, shift, lib=lib), delayed))
    return err


def pin_conv1d_continuation(lib, seed=21):
    """A sequence convolved in two parts, the second given the last K-1 inputs of
    the first as its initial window, equals the whole sequence convolved."""
    rng = np.random.default_rng(seed)
    b, T1, T2, Cn, K = 2, 7, 6, 3, 4
    x = rng.standard_normal((b, T1 + T2, Cn))
    w = rng.standard_normal((Cn, K))
    whole = oracle.causal_conv1d(x, w, lib=lib)
    init = np.ascontiguousarray(np.transpose(x[:, T1 - (K - 1):T1], (0, 2, 1)))
    part = oracle.causal_conv1d(np.ascontiguousarray(x[:, T1:]), w, init=init, lib=lib)
    return rel_err(part, whole[:, T1:])


def _selective_problem(rng, b, T, Dc, G, N, init=True):
    return dict(x=rng.standard_normal((b, T, Dc)), dt=rng.uniform(1e-3, 0.1, (b, T, Dc)),
                A=-rng.uniform(1.0, 16.0, (Dc, N)), B=rng.standard_normal((b, T, G, N)),
                C=rng.standard_normal((b, T, G, N)), D=rng.standard_normal(Dc),
                init_state=rng.standard_normal((b, Dc, N)) if init else None)


def pin_selective_scalar_A_is_ssd(lib, seed=22):
    """With the same A for every state of a channel, the Mamba-1 scan is the
    scalar-A scan with one head per channel and head dim 1 (the pinned SSD
    oracle)."""
    rng = np.random.default_rng(seed)
    b, T, Dc, G, N = 2, 13, 6, 2, 5
    p = _selective_problem(rng, b, T, Dc, G, N)
    a = -rng.uniform(1.0, 16.0, Dc)
    A = np.ascontiguousarray(np.repeat(a[:, None], N, axis=1))
    y, fs = oracle.selective_scan(p["x"], p["dt"], A, p["B"], p["C"], p["D"], p["init_state"], lib=lib)
    c = np.ascontiguousarray
    y_ref, fs_ref = oracle.scan(c(p["x"][..., None]), p["dt"], a, p["B"], p["C"], p["D"],
                                c(p["init_state"][:, :, None, :]), lib=lib)
    return max(rel_err(y, y_ref[..., 0]), rel_err(fs, fs_ref[:, :, 0, :]))


def pin_selective_brute_force(lib, seed=23):
    """Short sequences against the explicit sum over source tokens, each state
    with its own decay: y_t = sum_n C_t[n] (sum_{s<=t} exp(A[n] sum_{s<u<=t} dt_u)
    dt_s B_s[n] x_s + exp(A[n] sum_{u<=t} dt_u) h0[n]) + D x_t; and with x = 0
    the pure decay of h0."""
    rng = np.random.default_rng(seed)
    b, T, Dc, G, N = 1, 6, 4, 2, 3
    p = _selective_problem(rng, b, T, Dc, G, N)
    y, fs = oracle.selective_scan(p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"], p["init_state"], lib=lib)
    ref = np.zeros_like(y)
    for d in range(Dc):
        g = d // (Dc // G)
        for t in range(T):
            tot = 0.0
            for n in range(N):
                s_sum = 0.0
                for s in range(t + 1):
                    decay = np.exp(p["A"][d, n] * p["dt"][0, s + 1:t + 1, d].sum())
                    s_sum += decay * p["dt"][0, s, d] * p["B"][0, s, g, n] * p["x"][0, s, d]
                s_sum += np.exp(p["A"][d, n] * p["dt"][0, :t + 1, d].sum()) * p["init_state"][0, d, n]
                tot += p["C"][0, t, g, n] * s_sum
            ref[0, t, d] = tot + p["D"][d] * p["x"][0, t, d]
    err = rel_err(y, ref)
    z = dict(p, x=np.zeros_like(p["x"]))
    _, fs0 = oracle.selective_scan(z["x"], z["dt"], z["A"], z["B"], z["C"], z["D"], z["init_state"], lib=lib)
    closed = np.exp(p["A"][None] * p["dt"].sum(axis=1)[:, :, None]) * p["init_state"]
    return max(err, rel_err(fs0, closed))


VARIANT_PINS = [pin_conv1d_library, pin_conv1d_continuation, pin_selective_scalar_A_is_ssd,
                pin_selective_brute_force]


REAL_PINS = [pin_brute_force, pin_chunkwise, pin_zero_input, pin_prefix_sum, pin_linearity,
             pin_continuation, pin_decode_equals_scan, pin_contraction,
             pin_gradient_finite_difference, pin_gradient_empty_and_dfinal, pin_gradient_chunkwise]
COMPLEX_ONLY_PINS = [pin_complex_zero_imag_is_real, pin_complex_is_rotation_block]


def all_pins():
    """(name, callable(lib) -> error) for every pin, real and complex."""
    out = []
    for f in REAL_PINS:
        out.append((f.__name__ + "[real]", lambda lib, f=f: f(lib, cplx=False)))
        out.append((f.__name__ + "[complex]", lambda lib, f=f: f(lib, cplx=True)))
    for f in COMPLEX_ONLY_PINS + VARIANT_PINS:
        out.append((f.__name__, f))
    return out


PIN_TOL = 1e-9
