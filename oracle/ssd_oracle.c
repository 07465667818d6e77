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
