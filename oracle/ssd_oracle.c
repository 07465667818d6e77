/*
 * ssd_oracle.c -- the sequential fp64 oracle for the selective state-space scan.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call
 * this file: only the tests, the package's smoke() check and the CPU-baseline
 * leg of the benchmark use it.  It shares no code, header, table or helper with
 * the CUDA library; the two meet only through the seeded inputs.
 *
 * What it computes is the plain definition of the method, step by step in time,
 * with no chunking, blocking, fusion or reordering:
 *
 *   h_t = exp(dt_t * A_h) * h_{t-1} + dt_t * x_t B_t^T        (state, P x N per head)
 *   y_t = Re( h_t C_t ) + D_h * x_t                           (readout, P per head)
 *
 * Sources (page title, section):
 *  - "Mamba-3-Lite" README, the section on the classical Mamba-2 recurrence and
 *    its complex promotion: h_t = exp(A dt) h_{t-1} + B x_t, y_t = C h_t, and the
 *    complex form with A = A_real + i A_imag, B and C complex.
 *  - "Block Anatomy, Numerical Stability & Scaling", Numerical Stability section 4
 *    (the decay bound): the per-step transition is exp(dt * A) with dt already
 *    passed through softplus; section 6 of Block Anatomy (code walkthrough): the
 *    state starts at zero for every call and only the real part of the output
 *    leaves the scan.
 *  - "BitMamba 1B" (Portuguese edition, "Contexto"): the Mamba-2 layer shape,
 *    64 heads and d_state 128, one real A per head (A_log parameterisation).
 *
 * Readings taken where the pages are silent or garbled (each is listed in the
 * design notes):
 *  - the input is injected as dt_t * B_t x_t^T (the simplified Euler form of
 *    Mamba-2); the README line writes B x_t without dt;
 *  - dt arrives after softplus + dt_bias, so no softplus is applied here;
 *  - the complex readout is Re(sum_n C_n h_n) with no conjugate;
 *  - D * x is added when D is given (NULL means no skip term);
 *  - head h reads group h / (H / G) (contiguous heads share B and C);
 *  - the readout uses the state after the update at the same step.
 *
 * Layouts (all row-major, contiguous, fp64):
 *   x [b][t][h][p], dt [b][t][h], A [h] (complex: [h][2] = re, im),
 *   B, C [b][t][g][n] (complex: [b][t][g][n][2]), D [h],
 *   state [b][h][p][n] (complex: [b][h][p][n][2]), y [b][t][h][p].
 *
 * Every entry point returns 0 on success and -1 on an argument error.
 *
 * The gradient entry points (oracle_scan_bwd_*) at the end of the file are the
 * plain adjoint of the same recurrence; their pins are central finite
 * differences of the forward entry points.
 */
#include <complex.h>
#include <math.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>

#define IDX2(i, j, nj) ((size_t)(i) * (size_t)(nj) + (size_t)(j))

static int bad_dims(long batch, long seqlen, long nheads, long headdim,
                    long ngroups, long dstate) {
    if (batch < 0 || seqlen < 0 || nheads <= 0 || headdim <= 0 ||
        ngroups <= 0 || dstate <= 0)
        return 1;
    if (nheads % ngroups != 0) return 1;
    return 0;
}

/* Real variant: one real A per head (Mamba-2 layout). */
int oracle_scan_real(const double *x, const double *dt, const double *A,
                     const double *B, const double *C, const double *D,
                     const double *init_state, double *y, double *final_state,
                     long batch, long seqlen, long nheads, long headdim,
                     long ngroups, long dstate) {
    if (bad_dims(batch, seqlen, nheads, headdim, ngroups, dstate)) return -1;
    const long heads_per_group = nheads / ngroups;
    double *S = (double *)malloc(sizeof(double) * (size_t)headdim * (size_t)dstate);
    if (!S) return -1;

    for (long b = 0; b < batch; ++b) {
        for (long h = 0; h < nheads; ++h) {
            const long g = h / heads_per_group;
            /* initial state: the caller's, else zero */
            for (long p = 0; p < headdim; ++p)
                for (long n = 0; n < dstate; ++n) {
                    size_t si = ((size_t)(b * nheads + h) * headdim + p) * dstate + n;
                    S[IDX2(p, n, dstate)] = init_state ? init_state[si] : 0.0;
                }
            for (long t = 0; t < seqlen; ++t) {
                const double d = dt[((size_t)b * seqlen + t) * nheads + h];
                const double a = exp(d * A[h]); /* one step of decay */
                const double *xt = x + (((size_t)b * seqlen + t) * nheads + h) * headdim;
                const double *Bt = B + (((size_t)b * seqlen + t) * ngroups + g) * dstate;
                const double *Ct = C + (((size_t)b * seqlen + t) * ngroups + g) * dstate;
                double *yt = y + (((size_t)b * seqlen + t) * nheads + h) * headdim;
                for (long p = 0; p < headdim; ++p) {
                    double acc = 0.0;
                    for (long n = 0; n < dstate; ++n) {
                        double s = a * S[IDX2(p, n, dstate)] + d * xt[p] * Bt[n];
                        S[IDX2(p, n, dstate)] = s;
                        acc += Ct[n] * s;
                    }
                    yt[p] = acc + (D ? D[h] * xt[p] : 0.0);
                }
            }
            if (final_state)
                for (long p = 0; p < headdim; ++p)
                    for (long n = 0; n < dstate; ++n)
                        final_state[((size_t)(b * nheads + h) * headdim + p) * dstate + n] =
                            S[IDX2(p, n, dstate)];
        }
    }
    free(S);
    return 0;
}

/* Complex variant: one complex A per head, complex B/C/state, real x and y. */
int oracle_scan_complex(const double *x, const double *dt, const double *A,
                        const double *B, const double *C, const double *D,
                        const double *init_state, double *y, double *final_state,
                        long batch, long seqlen, long nheads, long headdim,
                        long ngroups, long dstate) {
    if (bad_dims(batch, seqlen, nheads, headdim, ngroups, dstate)) return -1;
    const long heads_per_group = nheads / ngroups;
    const double complex *Ac = (const double complex *)A;
    const double complex *Bc = (const double complex *)B;
    const double complex *Cc = (const double complex *)C;
    const double complex *H0 = (const double complex *)init_state;
    double complex *HF = (double complex *)final_state;
    double complex *S = (double complex *)malloc(sizeof(double complex) *
                                                 (size_t)headdim * (size_t)dstate);
    if (!S) return -1;

    for (long b = 0; b < batch; ++b) {
        for (long h = 0; h < nheads; ++h) {
            const long g = h / heads_per_group;
            for (long p = 0; p < headdim; ++p)
                for (long n = 0; n < dstate; ++n) {
                    size_t si = ((size_t)(b * nheads + h) * headdim + p) * dstate + n;
                    S[IDX2(p, n, dstate)] = H0 ? H0[si] : 0.0;
                }
            for (long t = 0; t < seqlen; ++t) {
                const double d = dt[((size_t)b * seqlen + t) * nheads + h];
                /* exp((A_re + i A_im) dt) = e^{A_re dt} (cos(A_im dt) + i sin(A_im dt)) */
                const double complex a = cexp(d * Ac[h]);
                const double *xt = x + (((size_t)b * seqlen + t) * nheads + h) * headdim;
                const double complex *Bt = Bc + (((size_t)b * seqlen + t) * ngroups + g) * dstate;
                const double complex *Ct = Cc + (((size_t)b * seqlen + t) * ngroups + g) * dstate;
                double *yt = y + (((size_t)b * seqlen + t) * nheads + h) * headdim;
                for (long p = 0; p < headdim; ++p) {
                    double complex acc = 0.0;
                    for (long n = 0; n < dstate; ++n) {
                        double complex s = a * S[IDX2(p, n, dstate)] + (d * xt[p]) * Bt[n];
                        S[IDX2(p, n, dstate)] = s;
                        acc += Ct[n] * s;
                    }
                    yt[p] = creal(acc) + (D ? D[h] * xt[p] : 0.0);
                }
            }
            if (HF)
                for (long p = 0; p < headdim; ++p)
                    for (long n = 0; n < dstate; ++n)
                        HF[((size_t)(b * nheads + h) * headdim + p) * dstate + n] =
                            S[IDX2(p, n, dstate)];
        }
    }
    free(S);
    return 0;
}

/*
 * One decoding step, in place on the state: the body of the time loop above,
 * applied once.  x [b][h][p], dt [b][h], B, C [b][g][n], state [b][h][p][n],
 * y [b][h][p].
 */
int oracle_state_update_real(double *state, const double *x, const double *dt,
                             const double *A, const double *B, const double *C,
                             const double *D, double *y, long batch, long nheads,
                             long headdim, long ngroups, long dstate) {
    if (bad_dims(batch, 1, nheads, headdim, ngroups, dstate)) return -1;
    const long heads_per_group = nheads / ngroups;
    for (long b = 0; b < batch; ++b)
        for (long h = 0; h < nheads; ++h) {
            const long g = h / heads_per_group;
            const double d = dt[(size_t)b * nheads + h];
            const double a = exp(d * A[h]);
            const double *xb = x + ((size_t)b * nheads + h) * headdim;
            const double *Bb = B + ((size_t)b * ngroups + g) * dstate;
            const double *Cb = C + ((size_t)b * ngroups + g) * dstate;
            for (long p = 0; p < headdim; ++p) {
                double *Sp = state + (((size_t)b * nheads + h) * headdim + p) * dstate;
                double acc = 0.0;
                for (long n = 0; n < dstate; ++n) {
                    Sp[n] = a * Sp[n] + d * xb[p] * Bb[n];
                    acc += Cb[n] * Sp[n];
                }
                y[((size_t)b * nheads + h) * headdim + p] = acc + (D ? D[h] * xb[p] : 0.0);
            }
        }
    return 0;
}

int oracle_state_update_complex(double *state, const double *x, const double *dt,
                                const double *A, const double *B, const double *C,
                                const double *D, double *y, long batch, long nheads,
                                long headdim, long ngroups, long dstate) {
    if (bad_dims(batch, 1, nheads, headdim, ngroups, dstate)) return -1;
    const long heads_per_group = nheads / ngroups;
    double complex *St = (double complex *)state;
    const double complex *Ac = (const double complex *)A;
    const double complex *Bc = (const double complex *)B;
    const double complex *Cc = (const double complex *)C;
    for (long b = 0; b < batch; ++b)
        for (long h = 0; h < nheads; ++h) {
            const long g = h / heads_per_group;
            const double d = dt[(size_t)b * nheads + h];
            const double complex a = cexp(d * Ac[h]);
            const double *xb = x + ((size_t)b * nheads + h) * headdim;
            const double complex *Bb = Bc + ((size_t)b * ngroups + g) * dstate;
            const double complex *Cb = Cc + ((size_t)b * ngroups + g) * dstate;
            for (long p = 0; p < headdim; ++p) {
                double complex *Sp = St + (((size_t)b * nheads + h) * headdim + p) * dstate;
                double complex acc = 0.0;
                for (long n = 0; n < dstate; ++n) {
                    Sp[n] = a * Sp[n] + (d * xb[p]) * Bb[n];
                    acc += Cb[n] * Sp[n];
                }
                y[((size_t)b * nheads + h) * headdim + p] = creal(acc) + (D ? D[h] * xb[p] : 0.0);
            }
        }
    return 0;
}

/*
 * Gradients of the scan (reverse-mode, by the adjoint of the same sequential
 * recurrence, step by step backwards in time).  The pages train through the
 * scan: "Block Anatomy, Numerical Stability & Scaling", Numerical Stability
 * section 5.3 (the backward differentiates the products of exp factors), and
 * the "Mamba-3-Lite" README's test list (an autograd gradcheck of the kernel's
 * backward).  They print no backward formula; this is the chain rule through
 * the recurrence at the top of this file.  The loss is taken as
 *
 *   L = sum_t <dy_t, y_t> + Re <dfinal, h_{T-1}>
 *
 * so dy [b][t][h][p] and dfinal [b][h][p][n] (nullable: zero) are the upstream
 * gradients.  Outputs: dx [b][t][h][p], ddt [b][t][h], dA [h], dB and dC
 * [b][t][g][n] (summed over the heads of a group), dD [h] (nullable), dinit
 * [b][h][p][n] (nullable).  For complex tensors the gradient of z = u + iv is
 * dL/du + i dL/dv.
 *
 * With G_t the gradient of the state h_t, the backward step is
 *   G_t  = dfinal (t = T-1, before the readout term) ;
 *   G_t += conj(C_t) dy_t                                  (readout at step t)
 *   dC_t += sum_p dy_t[p] conj(h_t[p])
 *   r_p   = sum_n Re(conj(B_t[n]) G_t[p][n])               (grad of dt_t x_t[p])
 *   dx_t  = dt_t r + D dy_t ;  dB_t += dt_t sum_p x_t[p] G_t[p]
 *   g_a   = sum conj(h_{t-1}) G_t                          (grad of a_t = exp(dt_t A))
 *   ddt_t = sum_p x_t[p] r_p + Re(g_a conj(A a_t)) ;  dA += dt_t conj(a_t) g_a
 *   G_{t-1} = conj(a_t) G_t ;  dinit = G_{-1}
 * which is the chain rule through h_t = a_t h_{t-1} + dt_t x_t B_t^T and
 * y_t = Re(h_t C_t) + D x_t.  The forward states are kept (T+1 of them per
 * (batch, head)), so this is for the small problems the tests use.
 */
int oracle_scan_bwd_real(const double *x, const double *dt, const double *A,
                         const double *B, const double *C, const double *D,
                         const double *init_state, const double *dy, const double *dfinal,
                         double *dx, double *ddt, double *dA, double *dB, double *dC,
                         double *dD, double *dinit, long batch, long seqlen, long nheads,
                         long headdim, long ngroups, long dstate) {
    if (bad_dims(batch, seqlen, nheads, headdim, ngroups, dstate)) return -1;
    const long hpg = nheads / ngroups;
    const size_t PN = (size_t)headdim * (size_t)dstate;
    double *hist = (double *)malloc(sizeof(double) * PN * (size_t)(seqlen + 1));
    double *Gs = (double *)malloc(sizeof(double) * PN);
    if (!hist || !Gs) {
        free(hist); free(Gs);
        return -1;
    }
    memset(dA, 0, sizeof(double) * (size_t)nheads);
    if (dD) memset(dD, 0, sizeof(double) * (size_t)nheads);
    memset(dB, 0, sizeof(double) * (size_t)batch * seqlen * ngroups * dstate);
    memset(dC, 0, sizeof(double) * (size_t)batch * seqlen * ngroups * dstate);

    for (long b = 0; b < batch; ++b) {
        for (long h = 0; h < nheads; ++h) {
            const long g = h / hpg;
            const size_t so = (size_t)(b * nheads + h) * PN;
            /* forward again, keeping every state: hist[t+1] = h_t, hist[0] = h_{-1} */
            for (size_t i = 0; i < PN; ++i) hist[i] = init_state ? init_state[so + i] : 0.0;
            for (long t = 0; t < seqlen; ++t) {
                const double d = dt[((size_t)b * seqlen + t) * nheads + h];
                const double a = exp(d * A[h]);
                const double *xt = x + (((size_t)b * seqlen + t) * nheads + h) * headdim;
                const double *Bt = B + (((size_t)b * seqlen + t) * ngroups + g) * dstate;
                const double *prev = hist + (size_t)t * PN;
                double *cur = hist + (size_t)(t + 1) * PN;
                for (long p = 0; p < headdim; ++p)
                    for (long n = 0; n < dstate; ++n)
                        cur[IDX2(p, n, dstate)] = a * prev[IDX2(p, n, dstate)] + d * xt[p] * Bt[n];
            }
            /* backward */
            for (size_t i = 0; i < PN; ++i) Gs[i] = dfinal ? dfinal[so + i] : 0.0;
            for (long t = seqlen - 1; t >= 0; --t) {
                const size_t tb = (size_t)b * seqlen + t;
                const double d = dt[tb * nheads + h];
                const double a = exp(d * A[h]);
                const double *xt = x + (tb * nheads + h) * headdim;
                const double *dyt = dy + (tb * nheads + h) * headdim;
                const double *Bt = B + (tb * ngroups + g) * dstate;
                const double *Ct = C + (tb * ngroups + g) * dstate;
                double *dBt = dB + (tb * ngroups + g) * dstate;
                double *dCt = dC + (tb * ngroups + g) * dstate;
                double *dxt = dx + (tb * nheads + h) * headdim;
                const double *ht = hist + (size_t)(t + 1) * PN, *hp = hist + (size_t)t * PN;
                for (long p = 0; p < headdim; ++p)
                    for (long n = 0; n < dstate; ++n) {
                        Gs[IDX2(p, n, dstate)] += Ct[n] * dyt[p]; /* readout of h_t */
                        dCt[n] += dyt[p] * ht[IDX2(p, n, dstate)];
                    }
                double ga = 0.0, ddt_in = 0.0;
                for (long p = 0; p < headdim; ++p) {
                    double rp = 0.0;
                    for (long n = 0; n < dstate; ++n) {
                        rp += Bt[n] * Gs[IDX2(p, n, dstate)];
                        dBt[n] += d * xt[p] * Gs[IDX2(p, n, dstate)];
                        ga += hp[IDX2(p, n, dstate)] * Gs[IDX2(p, n, dstate)];
                    }
                    dxt[p] = d * rp + (D ? D[h] * dyt[p] : 0.0);
                    ddt_in += xt[p] * rp;
                    if (dD) dD[h] += dyt[p] * xt[p];
                }
                ddt[tb * nheads + h] = ddt_in + ga * A[h] * a; /* d a_t / d dt_t = A a_t */
                dA[h] += ga * d * a;                          /* d a_t / d A = dt_t a_t */
                for (size_t i = 0; i < PN; ++i) Gs[i] *= a;    /* gradient of h_{t-1} */
            }
            if (dinit)
                for (size_t i = 0; i < PN; ++i) dinit[so + i] = Gs[i];
        }
    }
    free(hist); free(Gs);
    return 0;
}

int oracle_scan_bwd_complex(const double *x, const double *dt, const double *A,
                            const double *B, const double *C, const double *D,
                            const double *init_state, const double *dy, const double *dfinal,
                            double *dx, double *ddt, double *dA, double *dB, double *dC,
                            double *dD, double *dinit, long batch, long seqlen, long nheads,
                            long headdim, long ngroups, long dstate) {
    if (bad_dims(batch, seqlen, nheads, headdim, ngroups, dstate)) return -1;
    const long hpg = nheads / ngroups;
    const size_t PN = (size_t)headdim * (size_t)dstate;
    const double complex *Ac = (const double complex *)A;
    const double complex *Bc = (const double complex *)B;
    const double complex *Cc = (const double complex *)C;
    const double complex *H0 = (const double complex *)init_state;
    const double complex *GF = (const double complex *)dfinal;
    double complex *dAc = (double complex *)dA;
    double complex *dBc = (double complex *)dB;
    double complex *dCc = (double complex *)dC;
    double complex *dH0 = (double complex *)dinit;
    double complex *hist = (double complex *)malloc(sizeof(double complex) * PN * (size_t)(seqlen + 1));
    double complex *Gs = (double complex *)malloc(sizeof(double complex) * PN);
    if (!hist || !Gs) {
        free(hist); free(Gs);
        return -1;
    }
    memset(dA, 0, sizeof(double complex) * (size_t)nheads);
    if (dD) memset(dD, 0, sizeof(double) * (size_t)nheads);
    memset(dB, 0, sizeof(double complex) * (size_t)batch * seqlen * ngroups * dstate);
    memset(dC, 0, sizeof(double complex) * (size_t)batch * seqlen * ngroups * dstate);

    for (long b = 0; b < batch; ++b) {
        for (long h = 0; h < nheads; ++h) {
            const long g = h / hpg;
            const size_t so = (size_t)(b * nheads + h) * PN;
            for (size_t i = 0; i < PN; ++i) hist[i] = H0 ? H0[so + i] : 0.0;
            for (long t = 0; t < seqlen; ++t) {
                const double d = dt[((size_t)b * seqlen + t) * nheads + h];
                const double complex a = cexp(d * Ac[h]); /* a_t, as in the forward scan */
                const double *xt = x + (((size_t)b * seqlen + t) * nheads + h) * headdim;
                const double complex *Bt = Bc + (((size_t)b * seqlen + t) * ngroups + g) * dstate;
                const double complex *prev = hist + (size_t)t * PN;
                double complex *cur = hist + (size_t)(t + 1) * PN;
                for (long p = 0; p < headdim; ++p)
                    for (long n = 0; n < dstate; ++n)
                        cur[IDX2(p, n, dstate)] = a * prev[IDX2(p, n, dstate)] + (d * xt[p]) * Bt[n];
            }
            for (size_t i = 0; i < PN; ++i) Gs[i] = GF ? GF[so + i] : 0.0;
            for (long t = seqlen - 1; t >= 0; --t) {
                const size_t tb = (size_t)b * seqlen + t;
                const double d = dt[tb * nheads + h];
                const double complex a = cexp(d * Ac[h]); /* a_t again, going backwards */
                const double *xt = x + (tb * nheads + h) * headdim;
                const double *dyt = dy + (tb * nheads + h) * headdim;
                const double complex *Bt = Bc + (tb * ngroups + g) * dstate;
                const double complex *Ct = Cc + (tb * ngroups + g) * dstate;
                double complex *dBt = dBc + (tb * ngroups + g) * dstate;
                double complex *dCt = dCc + (tb * ngroups + g) * dstate;
                double *dxt = dx + (tb * nheads + h) * headdim;
                const double complex *ht = hist + (size_t)(t + 1) * PN, *hp = hist + (size_t)t * PN;
                for (long p = 0; p < headdim; ++p)
                    for (long n = 0; n < dstate; ++n) {
                        Gs[IDX2(p, n, dstate)] += conj(Ct[n]) * dyt[p]; /* readout Re(C h) */
                        dCt[n] += dyt[p] * conj(ht[IDX2(p, n, dstate)]);
                    }
                double complex ga = 0.0;
                double ddt_in = 0.0;
                for (long p = 0; p < headdim; ++p) {
                    double rp = 0.0;
                    for (long n = 0; n < dstate; ++n) {
                        rp += creal(conj(Bt[n]) * Gs[IDX2(p, n, dstate)]);
                        dBt[n] += (d * xt[p]) * Gs[IDX2(p, n, dstate)];
                        ga += conj(hp[IDX2(p, n, dstate)]) * Gs[IDX2(p, n, dstate)];
                    }
                    dxt[p] = d * rp + (D ? D[h] * dyt[p] : 0.0);
                    ddt_in += xt[p] * rp;
                    if (dD) dD[h] += dyt[p] * xt[p];
                }
                ddt[tb * nheads + h] = ddt_in + creal(ga * conj(Ac[h] * a));
                dAc[h] += d * conj(a) * ga;
                for (size_t i = 0; i < PN; ++i) Gs[i] *= conj(a);
            }
            if (dH0)
                for (size_t i = 0; i < PN; ++i) dH0[so + i] = Gs[i];
        }
    }
    free(hist); free(Gs);
    return 0;
}

/* ------------------------------------------------------------------------
 * Variants named on the pages beside the Mamba-2 / Mamba-3-Lite scan.
 *
 * Causal depthwise convolution ("Block Anatomy, Numerical Stability &
 * Scaling", Block Anatomy section 5.1): Mamba-1 and Mamba-2 convolve each
 * channel of the projected input over the current and the K-1 previous
 * positions (K = 4) before the scan.  out[t][c] = bias[c] + sum_k w[c][k] *
 * in[t - (K-1) + k][c]; inputs before t = 0 come from init (the previous K-1
 * inputs of a continued sequence, [b][c][K-1]) or are zero.  With silu != 0 the
 * result goes through v / (1 + exp(-v)) (the Mamba-2 activation; the pages
 * name the convolution only, so the activation is the caller's choice).
 *
 * Layouts: in, out [b][t][c]; w [c][K]; bias [c]; init [b][c][K-1].
 */
int oracle_causal_conv1d(const double *in, const double *w, const double *bias,
                         const double *init, int silu, double *out, long batch,
                         long seqlen, long channels, long width) {
    if (batch < 0 || seqlen < 0 || channels <= 0 || width <= 0) return -1;
    for (long b = 0; b < batch; ++b)
        for (long t = 0; t < seqlen; ++t)
            for (long c = 0; c < channels; ++c) {
                double v = bias ? bias[c] : 0.0;
                for (long k = 0; k < width; ++k) {
                    const long s = t - (width - 1) + k;
                    double u = 0.0;
                    if (s >= 0)
                        u = in[(b * seqlen + s) * channels + c];
                    else if (init)  /* s = -1 is init[..][K-2], s = -(K-1) is init[..][0] */
                        u = init[(b * channels + c) * (width - 1) + (width - 1) + s];
                    v += w[c * width + k] * u;
                }
                if (silu) v = v / (1.0 + exp(-v));
                out[(b * seqlen + t) * channels + c] = v;
            }
    return 0;
}

/*
 * Mamba-1 selective scan: a per-state decay ("Block Anatomy, Numerical
 * Stability & Scaling", Block Anatomy section 4.4: A of shape (H, N), one decay
 * rate per state component; the "Mamba-50M" card: a Mamba (selective SSM)
 * model).  Each channel d has its own step dt and N states:
 *
 *   h_t[n] = exp(dt_t[d] A[d][n]) h_{t-1}[n] + dt_t[d] B_t[n] x_t[d]
 *   y_t[d] = sum_n C_t[n] h_t[n] + D[d] x_t[d]
 *
 * Channel d reads group d / (channels / ngroups) of B and C.
 * Layouts: x, dt, y [b][t][d]; A [d][n]; B, C [b][t][g][n]; D [d];
 * state [b][d][n].
 */
int oracle_selective_scan(const double *x, const double *dt, const double *A,
                          const double *B, const double *C, const double *D,
                          const double *init_state, double *y, double *final_state,
                          long batch, long seqlen, long channels, long ngroups,
                          long dstate) {
    if (batch < 0 || seqlen < 0 || channels <= 0 || ngroups <= 0 || dstate <= 0 ||
        channels % ngroups != 0)
        return -1;
    double *h = (double *)malloc((size_t)dstate * sizeof(double));
    if (!h) return -1;
    for (long b = 0; b < batch; ++b)
        for (long d = 0; d < channels; ++d) {
            const long g = d / (channels / ngroups);
            for (long n = 0; n < dstate; ++n)
                h[n] = init_state ? init_state[(b * channels + d) * dstate + n] : 0.0;
            for (long t = 0; t < seqlen; ++t) {
                const size_t bt = (size_t)(b * seqlen + t);
                const double u = x[bt * channels + d], step = dt[bt * channels + d];
                double acc = 0.0;
                for (long n = 0; n < dstate; ++n) {
                    const size_t bc = (bt * ngroups + g) * dstate + n;
                    h[n] = exp(step * A[d * dstate + n]) * h[n] + step * B[bc] * u;
                    acc += C[bc] * h[n];
                }
                y[bt * channels + d] = acc + (D ? D[d] * u : 0.0);
            }
            if (final_state)
                for (long n = 0; n < dstate; ++n) final_state[(b * channels + d) * dstate + n] = h[n];
        }
    free(h);
    return 0;
}
