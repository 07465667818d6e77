// scan_bwd_body.cuh -- the phases of the chunked backward scan (real A, fp32).
//
// Gradients of L = sum_t <dy_t, y_t> + <dfinal, h_final> through the scan
//   h_t = exp(dt_t A) h_{t-1} + dt_t x_t B_t^T ,   y_t = h_t C_t + D x_t .
// The pages train through the scan ("Block Anatomy, Numerical Stability &
// Scaling", Numerical Stability section 5.3: the backward differentiates the
// products of the exp factors L, decay_chunk and exp(A_cumsum)); they print no
// backward formula, so this is the chain rule through the chunked form.  Per
// (batch, head) and 64-token chunk, with acs the inclusive within-chunk
// cumulative sum of dt A, lam = acs[last], L[l][s] = exp(acs[l] - acs[s]) for
// l >= s, w_s = exp(lam - acs[s]) dt_s, h_in the state entering the chunk and
// Gh the gradient of the state leaving it:
//   Gh(previous chunk) = exp(lam) Gh + sum_l exp(acs[l]) dy_l C_l^T
//   dx_s = sum_l (C_l.B_s) L[l][s] dt_s dy_l + D dy_s + w_s Gh B_s
//   dB_s = sum_l K[l][s] C_l + w_s Gh^T x_s ,  K[l][s] = L[l][s] dt_s (dy_l . x_s)
//   dC_l = sum_s K[l][s] B_s + exp(acs[l]) h_in^T dy_l
// and the decay gradient through acs: with E[l][s] = (C_l.B_s) K[l][s],
//   dacs[t] = sum_s E[t][s] - sum_l E[l][t] + exp(acs[t]) dy_t.(h_in C_t)
//             - w_t x_t.(Gh B_t)   (+ exp(lam) <Gh, h_in> + sum_s w_s x_s.(Gh B_s) at the last token)
//   dalpha = reverse cumulative sum of dacs;  ddt += A dalpha;  dA += sum dt dalpha.
// Rows past the end of the sequence are zero (dt = 0: decay 1, no input).
//
// Every phase is a __host__ __device__ function of (block, thread): the CUDA
// kernels run them separated by __syncthreads(), and a CPU harness in the tests
// runs the same functions thread by thread between the same barriers.
#pragma once

#include <math.h>
#include <stddef.h>

#ifndef __CUDACC__
#define __host__
#define __device__
#endif

namespace ssd {
namespace bwd {

constexpr int QB = 64;       // tokens per chunk
constexpr int NT = 256;      // threads per block
constexpr int P_MAX = 64;    // head dim
constexpr int N_MAX = 128;   // state dim
// Shared-memory row strides, one float longer than a row, so that lanes walking
// down a column hit 32 different banks.
constexpr int PS = P_MAX + 1, NS = N_MAX + 1, QS = QB + 1;

struct BwdArgs {
    const float *x, *dt, *A, *B, *C, *D, *init, *dy, *dfinal;
    float *dx, *ddt, *dA, *dB, *dC, *dD, *dinit;
    int batch, seqlen, nheads, headdim, ngroups, dstate, nchunks;
    // workspace
    float *acs;   // [b][h][nchunks * QB]
    float *lam;   // [b][h][nchunks]
    float *st;    // [b][h][nchunks][P*N]: chunk states, then the readout terms R
    float *hin;   // [b][h][nchunks][P*N]
    float *gh;    // [b][h][nchunks][P*N]
    float *dBh;   // [b][T][h][N]: dB of each head
    float *dCh;   // [b][T][h][N]
    float *dAp;   // [b][h][nchunks]
    float *dDp;   // [b][h][nchunks]
};

// Workspace floats for one call (each region padded to 4 floats).
__host__ __device__ inline size_t ws_floats(int batch, int seqlen, int nheads, int headdim, int dstate,
                                            int nchunks) {
    auto r4 = [](size_t v) { return (v + 3) / 4 * 4; };
    const size_t bh = (size_t)batch * nheads, pn = (size_t)headdim * dstate;
    return r4(bh * nchunks * QB) + r4(bh * nchunks) + 3 * r4(bh * nchunks * pn) +
           2 * r4((size_t)batch * seqlen * nheads * dstate) + 2 * r4(bh * nchunks);
}

__host__ __device__ inline void carve(BwdArgs &a, float *ws) {
    auto r4 = [](size_t v) { return (v + 3) / 4 * 4; };
    const size_t bh = (size_t)a.batch * a.nheads, pn = (size_t)a.headdim * a.dstate;
    float *p = ws;
    a.acs = p; p += r4(bh * a.nchunks * QB);
    a.lam = p; p += r4(bh * a.nchunks);
    a.st = p; p += r4(bh * a.nchunks * pn);
    a.hin = p; p += r4(bh * a.nchunks * pn);
    a.gh = p; p += r4(bh * a.nchunks * pn);
    a.dBh = p; p += r4((size_t)a.batch * a.seqlen * a.nheads * a.dstate);
    a.dCh = p; p += r4((size_t)a.batch * a.seqlen * a.nheads * a.dstate);
    a.dAp = p; p += r4(bh * a.nchunks);
    a.dDp = p;
}

// ------------------------------------------------------------- indexing
__host__ __device__ inline size_t ix_x(const BwdArgs &a, int b, int t, int h, int p) {
    return (((size_t)b * a.seqlen + t) * a.nheads + h) * a.headdim + p;
}
__host__ __device__ inline size_t ix_dt(const BwdArgs &a, int b, int t, int h) {
    return ((size_t)b * a.seqlen + t) * a.nheads + h;
}
__host__ __device__ inline size_t ix_bc(const BwdArgs &a, int b, int t, int g, int n) {
    return (((size_t)b * a.seqlen + t) * a.ngroups + g) * a.dstate + n;
}
__host__ __device__ inline size_t ix_bh(const BwdArgs &a, int b, int h) { return (size_t)b * a.nheads + h; }
__host__ __device__ inline size_t ix_pn(const BwdArgs &a, int b, int h, int c) {
    return (ix_bh(a, b, h) * a.nchunks + c) * ((size_t)a.headdim * a.dstate);
}
__host__ __device__ inline int group_of(const BwdArgs &a, int h) { return h / (a.nheads / a.ngroups); }

// ------------------------------------------------ shared-memory layout
// One layout serves every chunk kernel (fixed row strides PS, NS, QS).
struct Smem {
    float *d, *acs, *e, *w;           // [QB]
    float *X, *dY;                    // [QB][PS]
    float *Bs, *Cs;                   // [QB][NS]
    float *Hin, *Gh;                  // [P_MAX][NS]
    float *GL, *XY, *K;               // [QB][QS]
    float *rowE, *colG, *F, *Ksr;     // [QB]
    float *red;                       // [2 * QB]
    float *misc;                      // [4]: lam, ...
};
constexpr size_t SMEM_FLOATS = 4 * QB + 2 * QB * PS + 2 * QB * NS + 2 * P_MAX * NS + 3 * QB * QS +
                               4 * QB + 2 * QB + 4;
__host__ __device__ inline Smem smem_map(float *s) {
    Smem m;
    m.d = s; s += QB;
    m.acs = s; s += QB;
    m.e = s; s += QB;
    m.w = s; s += QB;
    m.X = s; s += QB * PS;
    m.dY = s; s += QB * PS;
    m.Bs = s; s += QB * NS;
    m.Cs = s; s += QB * NS;
    m.Hin = s; s += P_MAX * NS;
    m.Gh = s; s += P_MAX * NS;
    m.GL = s; s += QB * QS;
    m.XY = s; s += QB * QS;
    m.K = s; s += QB * QS;
    m.rowE = s; s += QB;
    m.colG = s; s += QB;
    m.F = s; s += QB;
    m.Ksr = s; s += QB;
    m.red = s; s += 2 * QB;
    m.misc = s;
    return m;
}

// ------------------------------------------------ shared loading phases
// dt of the chunk (0 past the end), and x or dy [QB][P], B or C [QB][N].
__host__ __device__ inline void load_dt(const BwdArgs &a, int c, int h, int b, int tid, const Smem &m) {
    for (int i = tid; i < QB; i += NT) {
        const int t = c * QB + i;
        m.d[i] = t < a.seqlen ? a.dt[ix_dt(a, b, t, h)] : 0.f;
    }
}
__host__ __device__ inline void load_rows_p(const BwdArgs &a, const float *src, int c, int h, int b, int tid,
                                            float *dst) {
    for (int i = tid; i < QB * a.headdim; i += NT) {
        const int s = i / a.headdim, p = i % a.headdim, t = c * QB + s;
        dst[s * PS + p] = t < a.seqlen ? src[ix_x(a, b, t, h, p)] : 0.f;
    }
}
__host__ __device__ inline void load_rows_n(const BwdArgs &a, const float *src, int c, int g, int b, int tid,
                                            float *dst) {
    for (int i = tid; i < QB * a.dstate; i += NT) {
        const int s = i / a.dstate, n = i % a.dstate, t = c * QB + s;
        dst[s * NS + n] = t < a.seqlen ? src[ix_bc(a, b, t, g, n)] : 0.f;
    }
}
__host__ __device__ inline void load_pn(const BwdArgs &a, const float *src, int tid, float *dst) {
    for (int i = tid; i < a.headdim * a.dstate; i += NT) {
        const int p = i / a.dstate, n = i % a.dstate;
        dst[p * NS + n] = src[i];
    }
}

// ---------------------------------------------- 1: chunk states (forward)
__host__ __device__ inline void k1_load(const BwdArgs &a, int c, int h, int b, int tid, const Smem &m) {
    load_dt(a, c, h, b, tid, m);
    load_rows_p(a, a.x, c, h, b, tid, m.X);
    load_rows_n(a, a.B, c, group_of(a, h), b, tid, m.Bs);
}
// Thread 0: the inclusive cumulative decay, lam and w.
__host__ __device__ inline void k1_cumsum(const BwdArgs &a, int c, int h, int b, int tid, const Smem &m) {
    if (tid != 0) return;
    const float Ah = a.A[h];
    float v = 0.f;
    float *acs_g = a.acs + (ix_bh(a, b, h) * a.nchunks + c) * QB;
    for (int i = 0; i < QB; ++i) {
        v += m.d[i] * Ah;
        m.acs[i] = v;
        acs_g[i] = v;
    }
    m.misc[0] = v;
    a.lam[ix_bh(a, b, h) * a.nchunks + c] = v;
    for (int i = 0; i < QB; ++i) m.w[i] = expf(v - m.acs[i]) * m.d[i];
}
// S[p][n] = sum_s w_s x_s[p] B_s[n]
__host__ __device__ inline void k1_state(const BwdArgs &a, int c, int h, int b, int tid, const Smem &m) {
    float *S = a.st + ix_pn(a, b, h, c);
    for (int i = tid; i < a.headdim * a.dstate; i += NT) {
        const int p = i / a.dstate, n = i % a.dstate;
        float acc = 0.f;
        for (int s = 0; s < QB; ++s) acc += m.w[s] * m.X[s * PS + p] * m.Bs[s * NS + n];
        S[i] = acc;
    }
}

// ------------------------------------- 2: state entering each chunk (forward)
__host__ __device__ inline void k2_pass(const BwdArgs &a, int h, int b, int tid) {
    const size_t pn = (size_t)a.headdim * a.dstate;
    for (size_t i = tid; i < pn; i += NT) {
        float hv = a.init ? a.init[ix_bh(a, b, h) * pn + i] : 0.f;
        for (int c = 0; c < a.nchunks; ++c) {
            const size_t o = ix_pn(a, b, h, c) + i;
            a.hin[o] = hv;
            hv = expf(a.lam[ix_bh(a, b, h) * a.nchunks + c]) * hv + a.st[o];
        }
    }
}

// ------------------------------- 3: readout terms R = sum_l e^{acs[l]} dy_l C_l^T
__host__ __device__ inline void k3_load(const BwdArgs &a, int c, int h, int b, int tid, const Smem &m) {
    const float *acs_g = a.acs + (ix_bh(a, b, h) * a.nchunks + c) * QB;
    for (int i = tid; i < QB; i += NT) m.e[i] = expf(acs_g[i]);
    load_rows_p(a, a.dy, c, h, b, tid, m.dY);
    load_rows_n(a, a.C, c, group_of(a, h), b, tid, m.Cs);
}
__host__ __device__ inline void k3_r(const BwdArgs &a, int c, int h, int b, int tid, const Smem &m) {
    float *R = a.st + ix_pn(a, b, h, c);  // the chunk states were consumed by pass 2
    for (int i = tid; i < a.headdim * a.dstate; i += NT) {
        const int p = i / a.dstate, n = i % a.dstate;
        float acc = 0.f;
        for (int l = 0; l < QB; ++l) acc += m.e[l] * m.dY[l * PS + p] * m.Cs[l * NS + n];
        R[i] = acc;
    }
}

// --------------------- 4: gradient of the state leaving each chunk (backward)
__host__ __device__ inline void k4_pass(const BwdArgs &a, int h, int b, int tid) {
    const size_t pn = (size_t)a.headdim * a.dstate;
    for (size_t i = tid; i < pn; i += NT) {
        float gv = a.dfinal ? a.dfinal[ix_bh(a, b, h) * pn + i] : 0.f;
        for (int c = a.nchunks - 1; c >= 0; --c) {
            const size_t o = ix_pn(a, b, h, c) + i;
            a.gh[o] = gv;
            gv = expf(a.lam[ix_bh(a, b, h) * a.nchunks + c]) * gv + a.st[o];
        }
        if (a.dinit) a.dinit[ix_bh(a, b, h) * pn + i] = gv;
    }
}

// ------------------------------------------------ 5: gradients of one chunk
__host__ __device__ inline void k5_load(const BwdArgs &a, int c, int h, int b, int tid, const Smem &m) {
    const int g = group_of(a, h);
    load_dt(a, c, h, b, tid, m);
    const float *acs_g = a.acs + (ix_bh(a, b, h) * a.nchunks + c) * QB;
    const float lam = a.lam[ix_bh(a, b, h) * a.nchunks + c];
    for (int i = tid; i < QB; i += NT) {
        const int t = c * QB + i;
        const float d = t < a.seqlen ? a.dt[ix_dt(a, b, t, h)] : 0.f;
        m.acs[i] = acs_g[i];
        m.e[i] = expf(acs_g[i]);
        m.w[i] = expf(lam - acs_g[i]) * d;
    }
    if (tid == 0) m.misc[0] = lam;
    load_rows_p(a, a.x, c, h, b, tid, m.X);
    load_rows_p(a, a.dy, c, h, b, tid, m.dY);
    load_rows_n(a, a.B, c, g, b, tid, m.Bs);
    load_rows_n(a, a.C, c, g, b, tid, m.Cs);
    load_pn(a, a.hin + ix_pn(a, b, h, c), tid, m.Hin);
    load_pn(a, a.gh + ix_pn(a, b, h, c), tid, m.Gh);
}
// GL = (C B^T) o L (causal), XY = dy x^T, K = L o dt_s o XY.
__host__ __device__ inline void k5_mats(const BwdArgs &a, int tid, const Smem &m) {
    for (int i = tid; i < QB * QB; i += NT) {
        const int l = i / QB, s = i % QB;
        float gm = 0.f, xy = 0.f;
        for (int n = 0; n < a.dstate; ++n) gm += m.Cs[l * NS + n] * m.Bs[s * NS + n];
        for (int p = 0; p < a.headdim; ++p) xy += m.dY[l * PS + p] * m.X[s * PS + p];
        m.XY[l * QS + s] = xy;
        if (l >= s) {
            const float L = expf(m.acs[l] - m.acs[s]);
            m.GL[l * QS + s] = gm * L;
            m.K[l * QS + s] = L * m.d[s] * xy;
        } else {
            m.GL[l * QS + s] = 0.f;
            m.K[l * QS + s] = 0.f;
        }
    }
}
// Per token: the row sums of E, the column sums of GL o XY, and the two
// state-coupling dot products; the last 64 threads reduce <Gh, h_in> and dy.x.
__host__ __device__ inline void k5_tokens(const BwdArgs &a, int tid, const Smem &m) {
    if (tid < QB) {
        const int t = tid;
        float re = 0.f, cg = 0.f;
        for (int s = 0; s < QB; ++s) re += m.GL[t * QS + s] * m.XY[t * QS + s] * m.d[s];
        for (int l = 0; l < QB; ++l) cg += m.GL[l * QS + t] * m.XY[l * QS + t];
        m.rowE[t] = re;
        m.colG[t] = cg;
    } else if (tid < 2 * QB) {  // F[t] = e^{acs[t]} dy_t . (h_in C_t)
        const int t = tid - QB;
        float acc = 0.f;
        for (int p = 0; p < a.headdim; ++p) {
            float hc = 0.f;
            for (int n = 0; n < a.dstate; ++n) hc += m.Hin[p * NS + n] * m.Cs[t * NS + n];
            acc += m.dY[t * PS + p] * hc;
        }
        m.F[t] = m.e[t] * acc;
    } else if (tid < 3 * QB) {  // Ksr[t] = x_t . (Gh B_t)
        const int t = tid - 2 * QB;
        float acc = 0.f;
        for (int p = 0; p < a.headdim; ++p) {
            float gb = 0.f;
            for (int n = 0; n < a.dstate; ++n) gb += m.Gh[p * NS + n] * m.Bs[t * NS + n];
            acc += m.X[t * PS + p] * gb;
        }
        m.Ksr[t] = acc;
    } else if (tid < 4 * QB) {
        const int r = tid - 3 * QB;
        float h0 = 0.f, dd = 0.f;
        for (int i = r; i < a.headdim * a.dstate; i += QB) {
            const int p = i / a.dstate, n = i % a.dstate;
            h0 += m.Gh[p * NS + n] * m.Hin[p * NS + n];
        }
        for (int i = r; i < QB * a.headdim; i += QB) {
            const int s = i / a.headdim, p = i % a.headdim;
            dd += m.dY[s * PS + p] * m.X[s * PS + p];
        }
        m.red[r] = h0;
        m.red[QB + r] = dd;
    }
}
// Thread 0: the decay gradient (reverse cumulative sum), ddt, and the dA and dD
// partials of this chunk.
__host__ __device__ inline void k5_decay(const BwdArgs &a, int c, int h, int b, int tid, const Smem &m) {
    if (tid != 0) return;
    const float lam = m.misc[0], Ah = a.A[h];
    float h0 = 0.f, dd = 0.f, ksum = 0.f;
    for (int r = 0; r < QB; ++r) {
        h0 += m.red[r];
        dd += m.red[QB + r];
        ksum += m.w[r] * m.Ksr[r];
    }
    h0 *= expf(lam);
    // colsum of E = dt_t * colsum of GL o XY
    float run = 0.f, dAp = 0.f;
    for (int t = QB - 1; t >= 0; --t) {
        float dacs = m.rowE[t] - m.d[t] * m.colG[t] + m.F[t] - m.w[t] * m.Ksr[t];
        if (t == QB - 1) dacs += h0 + ksum;
        run += dacs;  // dalpha[t] = sum_{t' >= t} dacs[t']
        const int tg = c * QB + t;
        if (tg < a.seqlen)
            a.ddt[ix_dt(a, b, tg, h)] = m.colG[t] + expf(lam - m.acs[t]) * m.Ksr[t] + Ah * run;
        dAp += m.d[t] * run;
    }
    a.dAp[ix_bh(a, b, h) * a.nchunks + c] = dAp;
    a.dDp[ix_bh(a, b, h) * a.nchunks + c] = dd;
}
// dx, and this head's share of dB and dC.
__host__ __device__ inline void k5_out(const BwdArgs &a, int c, int h, int b, int tid, const Smem &m) {
    const float Dh = a.D ? a.D[h] : 0.f;
    for (int i = tid; i < QB * a.headdim; i += NT) {
        const int s = i / a.headdim, p = i % a.headdim, t = c * QB + s;
        if (t >= a.seqlen) continue;
        float acc = 0.f, gb = 0.f;
        for (int l = s; l < QB; ++l) acc += m.GL[l * QS + s] * m.dY[l * PS + p];
        for (int n = 0; n < a.dstate; ++n) gb += m.Gh[p * NS + n] * m.Bs[s * NS + n];
        a.dx[ix_x(a, b, t, h, p)] = m.d[s] * acc + Dh * m.dY[s * PS + p] + m.w[s] * gb;
    }
    for (int i = tid; i < QB * a.dstate; i += NT) {
        const int s = i / a.dstate, n = i % a.dstate, t = c * QB + s;
        if (t >= a.seqlen) continue;
        float db = 0.f, dc = 0.f, xg = 0.f, yh = 0.f;
        for (int l = s; l < QB; ++l) db += m.K[l * QS + s] * m.Cs[l * NS + n];
        for (int r = 0; r <= s; ++r) dc += m.K[s * QS + r] * m.Bs[r * NS + n];
        for (int p = 0; p < a.headdim; ++p) {
            xg += m.X[s * PS + p] * m.Gh[p * NS + n];
            yh += m.dY[s * PS + p] * m.Hin[p * NS + n];
        }
        const size_t o = (((size_t)b * a.seqlen + t) * a.nheads + h) * a.dstate + n;
        a.dBh[o] = db + m.w[s] * xg;
        a.dCh[o] = dc + m.e[s] * yh;
    }
}

// ---------------------------------------------------- 6: sums over heads
// dB, dC: over the heads of each group (in head order); one thread per element.
__host__ __device__ inline void k6_group(const BwdArgs &a, size_t i) {
    const size_t per_t = (size_t)a.ngroups * a.dstate;
    const size_t bt = i / per_t, rem = i % per_t;
    const int g = (int)(rem / a.dstate), n = (int)(rem % a.dstate);
    const int hpg = a.nheads / a.ngroups;
    float sb = 0.f, sc = 0.f;
    for (int j = 0; j < hpg; ++j) {
        const size_t o = (bt * a.nheads + (size_t)g * hpg + j) * a.dstate + n;
        sb += a.dBh[o];
        sc += a.dCh[o];
    }
    a.dB[i] = sb;
    a.dC[i] = sc;
}
// dA[h], dD[h]: over batches and chunks (in order).
__host__ __device__ inline void k6_head(const BwdArgs &a, int h) {
    float sa = 0.f, sd = 0.f;
    for (int b = 0; b < a.batch; ++b)
        for (int c = 0; c < a.nchunks; ++c) {
            sa += a.dAp[ix_bh(a, b, h) * a.nchunks + c];
            sd += a.dDp[ix_bh(a, b, h) * a.nchunks + c];
        }
    a.dA[h] = sa;
    if (a.dD) a.dD[h] = sd;
}

}  // namespace bwd
}  // namespace ssd
