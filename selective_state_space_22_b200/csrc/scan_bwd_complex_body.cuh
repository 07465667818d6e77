// scan_bwd_complex_body.cuh -- the phases of the chunked backward scan, complex A.
//
// The complex (Mamba-3-Lite) variant of scan_bwd_body.cuh: A, B, C and the state
// are complex (interleaved float pairs), x, dt, D, y real.  The loss is
// L = sum_t <dy_t, y_t> + Re <dfinal, h_final> with y_t = Re(h_t C_t) + D x_t, and
// the gradient of a complex z = u + iv is dL/du + i dL/dv.  With acs the complex
// inclusive within-chunk cumulative sum of dt A, lam = acs[last], L[l][s] =
// exp(acs[l] - acs[s]) (l >= s), e_l = exp(acs[l]), w_s = exp(lam - acs[s]) dt_s:
//   Gh(previous chunk) = conj(exp(lam)) Gh + sum_l conj(e_l) dy_l conj(C_l)^T
//   dx_s = Re(sum_l (C_l.B_s) L[l][s] dt_s dy_l) + D dy_s + Re(conj(w_s) Gh conj(B_s))
//   dB_s = conj(sum_l K[l][s] C_l) + conj(w_s) Gh^T x_s ,  K[l][s] = L[l][s] dt_s (dy_l . x_s)
//   dC_l = conj(sum_s K[l][s] B_s + e_l h_in^T dy_l)
// and through acs, with E[l][s] = (C_l.B_s) K[l][s]:
//   dacs[t] = conj(sum_s E[t][s] - sum_l E[l][t] + e_t dy_t.(h_in C_t) - w_t x_t.(conj(Gh) B_t))
//             (+ conj(exp(lam) <conj(Gh), h_in> + sum_s w_s x_s.(conj(Gh) B_s)) at the last token)
//   dalpha = reverse cumulative sum of dacs;  ddt += Re(conj(dalpha) A);  dA += sum dt dalpha.
// (C_l.B_s = sum_n C_l[n] B_s[n], no conjugate, as in the forward readout.)  The
// chunk is 32 tokens so that the complex tiles fit in shared memory.  As in the
// real variant, every phase is a __host__ __device__ function of (block, thread),
// and the products are register-tiled: 256 threads as a 16 x 16 grid, each with
// a tile of 2 x 2 to 4 x 4 complex results, operands read from shared memory as
// 16-byte vectors (two complex values), rows strided 4 mod 32 words.
#pragma once

#include <math.h>
#include <stddef.h>
#include <stdint.h>

#ifndef __CUDACC__
#define __host__
#define __device__
#endif

// Read-only loads and unrolled loading loops on the device (see scan_bwd_body.cuh).
#ifdef __CUDA_ARCH__
#define BWDC_LDG(p) __ldg(p)
#define BWDC_UNROLL _Pragma("unroll 8")
#else
#define BWDC_LDG(p) (*(p))
#define BWDC_UNROLL
#endif

// On the device the operand rows come in as 16-byte asynchronous copies
// (cp.async, zero-filled past the sequence end or the row's width) when the rows
// are whole 16-byte units, so a thread has all its copies of a phase in flight
// at once instead of a few registers' worth; bwd_async_wait() at the end of the
// loading phase waits for them.  The host harness takes the scalar loops.
#ifndef SSD_BWD_ASYNC_DEFINED
#define SSD_BWD_ASYNC_DEFINED
#ifdef __CUDA_ARCH__
__device__ inline void bwd_cp16(float *dst, const float *src, bool valid) {
    const unsigned d = static_cast<unsigned>(__cvta_generic_to_shared(dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(d), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ inline void bwd_async_wait() { asm volatile("cp.async.wait_all;\n" ::: "memory"); }
#else
inline void bwd_async_wait() {}
#endif
// rows of `width` floats starting at src can be copied in 16-byte units
__host__ __device__ inline bool bwd_vec_rows(const float *src, int width) {
    return width % 4 == 0 && (reinterpret_cast<uintptr_t>(src) & 15) == 0;
}
#endif

namespace ssd {
namespace bwdc {

constexpr int QC = 32;        // tokens per chunk
constexpr int NT = 256;       // threads per block
constexpr int P_MAX = 64;     // head dim
constexpr int N_MAX = 64;     // complex state dim
constexpr int RED = 64;       // threads of the block reductions
// Row strides in floats: 4 more than a row, so rows stay 16-byte aligned and
// consecutive rows start 4 banks apart.
constexpr int PS = P_MAX + 4, NS = 2 * N_MAX + 4, QS2 = 2 * QC + 4, QS1 = QC + 4;
constexpr int PASS_GRP = 8;  // chunks whose loads a state pass issues together

struct c2 {
    float re, im;
};
__host__ __device__ inline c2 cmk(float r, float i) { return c2{r, i}; }
__host__ __device__ inline c2 cadd(c2 a, c2 b) { return c2{a.re + b.re, a.im + b.im}; }
__host__ __device__ inline c2 csub(c2 a, c2 b) { return c2{a.re - b.re, a.im - b.im}; }
__host__ __device__ inline c2 cmul(c2 a, c2 b) { return c2{a.re * b.re - a.im * b.im, a.re * b.im + a.im * b.re}; }
__host__ __device__ inline c2 cconj(c2 a) { return c2{a.re, -a.im}; }
__host__ __device__ inline c2 cscale(c2 a, float s) { return c2{a.re * s, a.im * s}; }
__host__ __device__ inline c2 cexpc(c2 z) {
    const float r = expf(z.re);
    return c2{r * cosf(z.im), r * sinf(z.im)};
}
__host__ __device__ inline c2 ld2(const float *p) { return c2{p[0], p[1]}; }
__host__ __device__ inline void st2(float *p, c2 v) {
    p[0] = v.re;
    p[1] = v.im;
}

struct BwdArgs {
    const float *x, *dt, *A, *B, *C, *D, *init, *dy, *dfinal;  // A, B, C, init, dfinal: float pairs
    float *dx, *ddt, *dA, *dB, *dC, *dD, *dinit;              // dA, dB, dC, dinit: float pairs
    int batch, seqlen, nheads, headdim, ngroups, dstate, nchunks;
    // workspace (complex regions are float pairs)
    float *acs;   // [b][h][nchunks * QC][2]
    float *lam;   // [b][h][nchunks][2]
    float *st;    // [b][h][nchunks][P*N][2]: chunk states, then the readout terms R
    float *hin;   // [b][h][nchunks][P*N][2]
    float *gh;    // [b][h][nchunks][P*N][2]
    float *dBh;   // [b][T][h][N][2]
    float *dCh;   // [b][T][h][N][2]
    float *dAp;   // [b][h][nchunks][2]
    float *dDp;   // [b][h][nchunks]
    int *dev_error;  // device error word (tensor-core phases' bounded waits)
};

__host__ __device__ inline size_t ws_floats(int batch, int seqlen, int nheads, int headdim, int dstate,
                                            int nchunks) {
    auto r4 = [](size_t v) { return (v + 3) / 4 * 4; };
    const size_t bh = (size_t)batch * nheads, pn = (size_t)headdim * dstate;
    return r4(2 * bh * nchunks * QC) + r4(2 * bh * nchunks) + 3 * r4(2 * bh * nchunks * pn) +
           2 * r4(2 * (size_t)batch * seqlen * nheads * dstate) + r4(2 * bh * nchunks) + r4(bh * nchunks);
}

__host__ __device__ inline void carve(BwdArgs &a, float *ws) {
    auto r4 = [](size_t v) { return (v + 3) / 4 * 4; };
    const size_t bh = (size_t)a.batch * a.nheads, pn = (size_t)a.headdim * a.dstate;
    float *p = ws;
    a.acs = p; p += r4(2 * bh * a.nchunks * QC);
    a.lam = p; p += r4(2 * bh * a.nchunks);
    a.st = p; p += r4(2 * bh * a.nchunks * pn);
    a.hin = p; p += r4(2 * bh * a.nchunks * pn);
    a.gh = p; p += r4(2 * bh * a.nchunks * pn);
    a.dBh = p; p += r4(2 * (size_t)a.batch * a.seqlen * a.nheads * a.dstate);
    a.dCh = p; p += r4(2 * (size_t)a.batch * a.seqlen * a.nheads * a.dstate);
    a.dAp = p; p += r4(2 * bh * a.nchunks);
    a.dDp = p;
}

// ------------------------------------------------------------- indexing
__host__ __device__ inline size_t ix_x(const BwdArgs &a, int b, int t, int h, int p) {
    return (((size_t)b * a.seqlen + t) * a.nheads + h) * a.headdim + p;
}
__host__ __device__ inline size_t ix_dt(const BwdArgs &a, int b, int t, int h) {
    return ((size_t)b * a.seqlen + t) * a.nheads + h;
}
// complex element index (multiply by 2 for the float offset)
__host__ __device__ inline size_t ix_bc(const BwdArgs &a, int b, int t, int g, int n) {
    return (((size_t)b * a.seqlen + t) * a.ngroups + g) * a.dstate + n;
}
__host__ __device__ inline size_t ix_bh(const BwdArgs &a, int b, int h) { return (size_t)b * a.nheads + h; }
__host__ __device__ inline size_t ix_pn(const BwdArgs &a, int b, int h, int c) {  // complex elements
    return (ix_bh(a, b, h) * a.nchunks + c) * ((size_t)a.headdim * a.dstate);
}
__host__ __device__ inline int group_of(const BwdArgs &a, int h) { return h / (a.nheads / a.ngroups); }

// ------------------------------------------------ shared-memory layout
// Arrays are zero beyond headdim / dstate, so the products run over P_MAX, N_MAX.
struct Smem {
    float *d;                    // [QC]
    float *acs, *e, *w;          // [QC][2]
    float *X, *dY;               // [QC][PS]
    float *Bs, *Cs;              // [QC][NS], complex n at 2n, 2n+1
    float *Hin, *Gh;             // [P_MAX][NS]
    float *GL, *K;               // [QC][QS2], complex s at 2s, 2s+1
    float *XY;                   // [QC][QS1]
    float *rowE, *colG, *F, *Ksr;  // [QC][2]
    float *red;                  // [3][RED]: <conj(Gh), h_in> re, im; dy.x
    float *part;                 // [2][QC][16][2]: per-thread-column terms of Ksr and F
    float *el;                   // [QC][2]: exp(lam - acs)
    float *misc;                 // [8]: lam; exp(lam) <conj(Gh), h_in>; dy.x
};
constexpr size_t SMEM_FLOATS = QC + 3 * 2 * QC + 2 * QC * PS + 2 * QC * NS + 2 * P_MAX * NS + 2 * QC * QS2 +
                               QC * QS1 + 4 * 2 * QC + 3 * RED + 2 * QC * 16 * 2 + 2 * QC + 8;
// The chunk-state phase uses the layout up to Bs, the readout phase up to Cs.
constexpr size_t SMEM_FLOATS_K1 = QC + 3 * 2 * QC + 2 * QC * PS + QC * NS;
constexpr size_t SMEM_FLOATS_K3 = QC + 3 * 2 * QC + 2 * QC * PS + 2 * QC * NS;
__host__ __device__ inline Smem smem_map(float *s) {
    Smem m;
    m.d = s; s += QC;
    m.acs = s; s += 2 * QC;
    m.e = s; s += 2 * QC;
    m.w = s; s += 2 * QC;
    m.X = s; s += QC * PS;
    m.dY = s; s += QC * PS;
    m.Bs = s; s += QC * NS;
    m.Cs = s; s += QC * NS;
    m.Hin = s; s += P_MAX * NS;
    m.Gh = s; s += P_MAX * NS;
    m.GL = s; s += QC * QS2;
    m.K = s; s += QC * QS2;
    m.XY = s; s += QC * QS1;
    m.rowE = s; s += 2 * QC;
    m.colG = s; s += 2 * QC;
    m.F = s; s += 2 * QC;
    m.Ksr = s; s += 2 * QC;
    m.red = s; s += 3 * RED;
    m.part = s; s += 2 * QC * 16 * 2;
    m.el = s; s += 2 * QC;
    m.misc = s;
    return m;
}

// ------------------------------------------------ shared loading phases
__host__ __device__ inline void load_dt(const BwdArgs &a, int c, int h, int b, int tid, const Smem &m) {
    for (int i = tid; i < QC; i += NT) {
        const int t = c * QC + i;
        m.d[i] = t < a.seqlen ? BWDC_LDG(a.dt + ix_dt(a, b, t, h)) : 0.f;
    }
}
__host__ __device__ inline void load_rows_p(const BwdArgs &a, const float *src, int c, int h, int b, int tid,
                                            float *dst) {
#ifdef __CUDA_ARCH__
    if (bwd_vec_rows(src, a.headdim)) {
        for (int i = tid; i < QC * (P_MAX / 4); i += NT) {
            const int s = i / (P_MAX / 4), p = 4 * (i % (P_MAX / 4)), t = c * QC + s;
            const bool v = t < a.seqlen && p < a.headdim;
            bwd_cp16(dst + s * PS + p, v ? src + ix_x(a, b, t, h, p) : src, v);
        }
        return;
    }
#endif
    BWDC_UNROLL
    for (int i = tid; i < QC * P_MAX; i += NT) {
        const int s = i / P_MAX, p = i % P_MAX, t = c * QC + s;
        dst[s * PS + p] = (t < a.seqlen && p < a.headdim) ? BWDC_LDG(src + ix_x(a, b, t, h, p)) : 0.f;
    }
}
// complex rows of B or C: [QC][N] pairs
__host__ __device__ inline void load_rows_n(const BwdArgs &a, const float *src, int c, int g, int b, int tid,
                                            float *dst) {
#ifdef __CUDA_ARCH__
    if (bwd_vec_rows(src, 2 * a.dstate)) {
        for (int i = tid; i < QC * (2 * N_MAX / 4); i += NT) {
            const int s = i / (2 * N_MAX / 4), f = 4 * (i % (2 * N_MAX / 4)), t = c * QC + s;
            const bool v = t < a.seqlen && f < 2 * a.dstate;
            bwd_cp16(dst + s * NS + f, v ? src + 2 * ix_bc(a, b, t, g, 0) + f : src, v);
        }
        return;
    }
#endif
    BWDC_UNROLL
    for (int i = tid; i < QC * 2 * N_MAX; i += NT) {
        const int s = i / (2 * N_MAX), f = i % (2 * N_MAX), t = c * QC + s;
        dst[s * NS + f] = (t < a.seqlen && f < 2 * a.dstate) ? BWDC_LDG(src + 2 * ix_bc(a, b, t, g, 0) + f) : 0.f;
    }
}
// a complex [P][N] block
__host__ __device__ inline void load_pn(const BwdArgs &a, const float *src, int tid, float *dst) {
#ifdef __CUDA_ARCH__
    if (bwd_vec_rows(src, 2 * a.dstate)) {
        for (int i = tid; i < P_MAX * (2 * N_MAX / 4); i += NT) {
            const int p = i / (2 * N_MAX / 4), f = 4 * (i % (2 * N_MAX / 4));
            const bool v = p < a.headdim && f < 2 * a.dstate;
            bwd_cp16(dst + p * NS + f, v ? src + (size_t)p * 2 * a.dstate + f : src, v);
        }
        return;
    }
#endif
    BWDC_UNROLL
    for (int i = tid; i < P_MAX * 2 * N_MAX; i += NT) {
        const int p = i / (2 * N_MAX), f = i % (2 * N_MAX);
        dst[p * NS + f] = (p < a.headdim && f < 2 * a.dstate) ? BWDC_LDG(src + (size_t)p * 2 * a.dstate + f) : 0.f;
    }
}
__host__ __device__ inline c2 sm2(const float *row, int k) { return c2{row[2 * k], row[2 * k + 1]}; }

// --------------------------------------------------- register tiles
struct alignas(16) f4 {
    float x, y, z, w;
};
__host__ __device__ inline f4 ld4(const float *p) { return *reinterpret_cast<const f4 *>(p); }
__host__ __device__ inline float comp(const f4 &v, int i) { return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w; }
// The complex columns of a thread's "n" tile: n(j) = 2 tc + (j & 1) + 32 (j >> 1),
// at float offset 4 tc + 2 (j & 1) + 64 (j >> 1) of a row.
__host__ __device__ inline int ncol(int tc, int j) { return 2 * tc + (j & 1) + 32 * (j >> 1); }
// acc[i][j] += a * v[j] for one real a and the four complex values of a row at
// float offsets 4 tc and 64 + 4 tc.
__host__ __device__ inline void axpy4(c2 (&acc)[4], float a, const float *row, int tc) {
    const f4 u = ld4(row + 4 * tc), v = ld4(row + 64 + 4 * tc);
    acc[0].re = fmaf(a, u.x, acc[0].re), acc[0].im = fmaf(a, u.y, acc[0].im);
    acc[1].re = fmaf(a, u.z, acc[1].re), acc[1].im = fmaf(a, u.w, acc[1].im);
    acc[2].re = fmaf(a, v.x, acc[2].re), acc[2].im = fmaf(a, v.y, acc[2].im);
    acc[3].re = fmaf(a, v.z, acc[3].re), acc[3].im = fmaf(a, v.w, acc[3].im);
}
// acc[j] += z * row[n(j)] for a complex z (no conjugate).
__host__ __device__ inline void czpy4(c2 (&acc)[4], c2 z, const float *row, int tc) {
    const f4 u = ld4(row + 4 * tc), v = ld4(row + 64 + 4 * tc);
    const c2 r[4] = {c2{u.x, u.y}, c2{u.z, u.w}, c2{v.x, v.y}, c2{v.z, v.w}};
    for (int j = 0; j < 4; ++j) acc[j] = cadd(acc[j], cmul(z, r[j]));
}
// Complex values n = 2 tc .. 2 tc + 1 and 2 tc + 32 .. 33 of a row (acc[0..3]) to a
// global row of `valid` complex values, 16 bytes at a time where aligned.
__host__ __device__ inline void store_n4(float *row, int tc, int valid, const c2 (&v)[4]) {
    for (int q = 0; q < 2; ++q) {
        const int n = 2 * tc + 32 * q;
        float *dst = row + 2 * n;
        if (n + 1 < valid && (reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
            *reinterpret_cast<f4 *>(dst) = f4{v[2 * q].re, v[2 * q].im, v[2 * q + 1].re, v[2 * q + 1].im};
        } else {
            if (n < valid) st2(dst, v[2 * q]);
            if (n + 1 < valid) st2(dst + 2, v[2 * q + 1]);
        }
    }
}
// out[p][n] = sum_k A[k][p] M[k][n] over k < QC for rows p = 4 tr .. 4 tr + 3 (A real,
// [QC][PS]) and the thread's four complex columns (M [QC][NS]), stored to a
// complex P x N array.
__host__ __device__ inline void tn_pn(const BwdArgs &a, const float *A, const float *M, float *dst, int tid) {
    const int r0 = 4 * (tid >> 4), tc = tid & 15;
    c2 acc[4][4];
    for (int i = 0; i < 4; ++i)
        for (int j = 0; j < 4; ++j) acc[i][j] = cmk(0.f, 0.f);
    for (int k = 0; k < QC; ++k) {
        const f4 av = ld4(A + k * PS + r0);
        for (int i = 0; i < 4; ++i) axpy4(acc[i], comp(av, i), M + k * NS, tc);
    }
    for (int i = 0; i < 4; ++i)
        if (r0 + i < a.headdim) store_n4(dst + 2 * (size_t)(r0 + i) * a.dstate, tc, a.dstate, acc[i]);
}

// ---------------------------------------------- 1: chunk states (forward)
__host__ __device__ inline void k1_load(const BwdArgs &a, int c, int h, int b, int tid, const Smem &m) {
    load_dt(a, c, h, b, tid, m);
    load_rows_p(a, a.x, c, h, b, tid, m.X);
    load_rows_n(a, a.B, c, group_of(a, h), b, tid, m.Bs);
    bwd_async_wait();
}
__host__ __device__ inline void k1_cumsum(const BwdArgs &a, int c, int h, int b, int tid, const Smem &m) {
    if (tid != 0) return;
    const c2 Ah = ld2(a.A + 2 * h);
    c2 v = cmk(0.f, 0.f);
    float *acs_g = a.acs + 2 * (ix_bh(a, b, h) * a.nchunks + c) * QC;
    for (int i = 0; i < QC; ++i) {
        v = cadd(v, cscale(Ah, m.d[i]));
        st2(m.acs + 2 * i, v);
        st2(acs_g + 2 * i, v);
    }
    st2(a.lam + 2 * (ix_bh(a, b, h) * a.nchunks + c), v);
    for (int i = 0; i < QC; ++i) st2(m.w + 2 * i, cscale(cexpc(csub(v, ld2(m.acs + 2 * i))), m.d[i]));
}
// B_s <- w_s B_s in place
__host__ __device__ inline void k1_scale(const BwdArgs &a, int tid, const Smem &m) {
    (void)a;
    for (int i = tid; i < QC * N_MAX; i += NT) {
        const int s = i / N_MAX, n = i % N_MAX;
        st2(m.Bs + s * NS + 2 * n, cmul(ld2(m.w + 2 * s), sm2(m.Bs + s * NS, n)));
    }
}
// S[p][n] = sum_s x_s[p] (w_s B_s[n])
__host__ __device__ inline void k1_state(const BwdArgs &a, int c, int h, int b, int tid, const Smem &m) {
    tn_pn(a, m.X, m.Bs, a.st + 2 * ix_pn(a, b, h, c), tid);
}

// ------------------------------------- 2: state entering each chunk (forward)
// Element i = blk * NT + tid of the P x N state of (batch b, head h).
__host__ __device__ inline void k2_pass(const BwdArgs &a, int blk, int h, int b, int tid) {
    const size_t pn = (size_t)a.headdim * a.dstate, i = (size_t)blk * NT + tid;
    if (i >= pn) return;
    c2 hv = a.init ? ld2(a.init + 2 * (ix_bh(a, b, h) * pn + i)) : cmk(0.f, 0.f);
    for (int c0 = 0; c0 < a.nchunks; c0 += PASS_GRP) {  // a group's loads in flight together
        c2 sv[PASS_GRP], lv[PASS_GRP];
        for (int j = 0; j < PASS_GRP; ++j)
            if (c0 + j < a.nchunks) {
                sv[j] = ld2(a.st + 2 * (ix_pn(a, b, h, c0 + j) + i));
                lv[j] = ld2(a.lam + 2 * (ix_bh(a, b, h) * a.nchunks + c0 + j));
            }
        for (int j = 0; j < PASS_GRP && c0 + j < a.nchunks; ++j) {
            st2(a.hin + 2 * (ix_pn(a, b, h, c0 + j) + i), hv);
            hv = cadd(cmul(cexpc(lv[j]), hv), sv[j]);
        }
    }
}

// -------------------- 3: readout terms R = sum_l conj(e_l) dy_l conj(C_l)^T
__host__ __device__ inline void k3_load(const BwdArgs &a, int c, int h, int b, int tid, const Smem &m) {
    const float *acs_g = a.acs + 2 * (ix_bh(a, b, h) * a.nchunks + c) * QC;
    for (int i = tid; i < QC; i += NT) st2(m.e + 2 * i, cexpc(ld2(acs_g + 2 * i)));
    load_rows_p(a, a.dy, c, h, b, tid, m.dY);
    load_rows_n(a, a.C, c, group_of(a, h), b, tid, m.Cs);
    bwd_async_wait();
}
// C_l <- conj(e_l C_l) in place
__host__ __device__ inline void k3_scale(const BwdArgs &a, int tid, const Smem &m) {
    (void)a;
    for (int i = tid; i < QC * N_MAX; i += NT) {
        const int l = i / N_MAX, n = i % N_MAX;
        st2(m.Cs + l * NS + 2 * n, cconj(cmul(ld2(m.e + 2 * l), sm2(m.Cs + l * NS, n))));
    }
}
__host__ __device__ inline void k3_r(const BwdArgs &a, int c, int h, int b, int tid, const Smem &m) {
    tn_pn(a, m.dY, m.Cs, a.st + 2 * ix_pn(a, b, h, c), tid);  // the chunk states were consumed by pass 2
}

// --------------------- 4: gradient of the state leaving each chunk (backward)
__host__ __device__ inline void k4_pass(const BwdArgs &a, int blk, int h, int b, int tid) {
    const size_t pn = (size_t)a.headdim * a.dstate, i = (size_t)blk * NT + tid;
    if (i >= pn) return;
    c2 gv = a.dfinal ? ld2(a.dfinal + 2 * (ix_bh(a, b, h) * pn + i)) : cmk(0.f, 0.f);
    for (int c0 = a.nchunks - 1; c0 >= 0; c0 -= PASS_GRP) {  // chunks c0, c0 - 1, ...
        c2 sv[PASS_GRP], lv[PASS_GRP];
        for (int j = 0; j < PASS_GRP; ++j)
            if (c0 - j >= 0) {
                sv[j] = ld2(a.st + 2 * (ix_pn(a, b, h, c0 - j) + i));
                lv[j] = ld2(a.lam + 2 * (ix_bh(a, b, h) * a.nchunks + c0 - j));
            }
        for (int j = 0; j < PASS_GRP && c0 - j >= 0; ++j) {
            st2(a.gh + 2 * (ix_pn(a, b, h, c0 - j) + i), gv);
            const c2 el = cexpc(lv[j]);
            gv = cadd(cmul(cconj(el), gv), sv[j]);
        }
    }
    if (a.dinit) st2(a.dinit + 2 * (ix_bh(a, b, h) * pn + i), gv);
}

// ------------------------------------------------ 5: gradients of one chunk
__host__ __device__ inline void k5_load(const BwdArgs &a, int c, int h, int b, int tid, const Smem &m) {
    const int g = group_of(a, h);
    load_dt(a, c, h, b, tid, m);
    const float *acs_g = a.acs + 2 * (ix_bh(a, b, h) * a.nchunks + c) * QC;
    const c2 lam = ld2(a.lam + 2 * (ix_bh(a, b, h) * a.nchunks + c));
    for (int i = tid; i < QC; i += NT) {
        const int t = c * QC + i;
        const float d = t < a.seqlen ? BWDC_LDG(a.dt + ix_dt(a, b, t, h)) : 0.f;
        const c2 ac = ld2(acs_g + 2 * i);
        st2(m.acs + 2 * i, ac);
        st2(m.e + 2 * i, cexpc(ac));
        const c2 wl = cexpc(csub(lam, ac));
        st2(m.el + 2 * i, wl);
        st2(m.w + 2 * i, cscale(wl, d));
    }
    if (tid == 0) st2(m.misc, lam);
    load_rows_p(a, a.x, c, h, b, tid, m.X);
    load_rows_p(a, a.dy, c, h, b, tid, m.dY);
    load_rows_n(a, a.B, c, g, b, tid, m.Bs);
    load_rows_n(a, a.C, c, g, b, tid, m.Cs);
    load_pn(a, a.hin + 2 * ix_pn(a, b, h, c), tid, m.Hin);
    load_pn(a, a.gh + 2 * ix_pn(a, b, h, c), tid, m.Gh);
    bwd_async_wait();
}
// GL = (C B^T) o L (causal), XY = dy x^T, K = L o dt_s o XY; thread tile rows
// l = 2 tr + i, columns s = tc + 16 j.
__host__ __device__ inline void k5_mats(const BwdArgs &a, int tid, const Smem &m) {
    (void)a;
    const int r0 = 2 * (tid >> 4), tc = tid & 15;
    c2 g[2][2];
    float xy[2][2];
    for (int i = 0; i < 2; ++i)
        for (int j = 0; j < 2; ++j) g[i][j] = cmk(0.f, 0.f), xy[i][j] = 0.f;
    for (int k = 0; k < 2 * N_MAX; k += 4) {  // two complex states per step
        f4 ca[2], bb[2];
        for (int i = 0; i < 2; ++i) ca[i] = ld4(m.Cs + (r0 + i) * NS + k);
        for (int j = 0; j < 2; ++j) bb[j] = ld4(m.Bs + (tc + 16 * j) * NS + k);
        for (int i = 0; i < 2; ++i)
            for (int j = 0; j < 2; ++j) {
                const f4 &u = ca[i], &v = bb[j];
                g[i][j].re = fmaf(u.x, v.x, fmaf(-u.y, v.y, fmaf(u.z, v.z, fmaf(-u.w, v.w, g[i][j].re))));
                g[i][j].im = fmaf(u.x, v.y, fmaf(u.y, v.x, fmaf(u.z, v.w, fmaf(u.w, v.z, g[i][j].im))));
            }
    }
    for (int p = 0; p < P_MAX; p += 4) {
        f4 ya[2], xb[2];
        for (int i = 0; i < 2; ++i) ya[i] = ld4(m.dY + (r0 + i) * PS + p);
        for (int j = 0; j < 2; ++j) xb[j] = ld4(m.X + (tc + 16 * j) * PS + p);
        for (int i = 0; i < 2; ++i)
            for (int j = 0; j < 2; ++j)
                xy[i][j] = fmaf(ya[i].x, xb[j].x, fmaf(ya[i].y, xb[j].y, fmaf(ya[i].z, xb[j].z, fmaf(ya[i].w, xb[j].w, xy[i][j]))));
    }
    for (int i = 0; i < 2; ++i)
        for (int j = 0; j < 2; ++j) {
            const int l = r0 + i, s = tc + 16 * j;
            m.XY[l * QS1 + s] = xy[i][j];
            if (l >= s) {
                const c2 L = cexpc(csub(ld2(m.acs + 2 * l), ld2(m.acs + 2 * s)));
                st2(m.GL + l * QS2 + 2 * s, cmul(g[i][j], L));
                st2(m.K + l * QS2 + 2 * s, cscale(L, m.d[s] * xy[i][j]));
            } else {
                st2(m.GL + l * QS2 + 2 * s, cmk(0.f, 0.f));
                st2(m.K + l * QS2 + 2 * s, cmk(0.f, 0.f));
            }
        }
}
__host__ __device__ inline void k5_tokens(const BwdArgs &a, int tid, const Smem &m) {
    if (tid < QC) {  // rows of E and columns of GL o XY
        const int t = tid;
        c2 re = cmk(0.f, 0.f), cg = cmk(0.f, 0.f);
        for (int s = 0; s < QC; ++s)
            re = cadd(re, cscale(ld2(m.GL + t * QS2 + 2 * s), m.XY[t * QS1 + s] * m.d[s]));
        for (int l = 0; l < QC; ++l) cg = cadd(cg, cscale(ld2(m.GL + l * QS2 + 2 * t), m.XY[l * QS1 + t]));
        st2(m.rowE + 2 * t, re);
        st2(m.colG + 2 * t, cg);
    } else if (tid >= 3 * QC && tid < 3 * QC + RED) {  // <conj(Gh), h_in> and dy . x, partial sums
        const int r = tid - 3 * QC;
        c2 h0 = cmk(0.f, 0.f);
        float dd = 0.f;
        for (int i = r; i < a.headdim * a.dstate; i += RED) {
            const int p = i / a.dstate, n = i % a.dstate;
            h0 = cadd(h0, cmul(cconj(sm2(m.Gh + p * NS, n)), sm2(m.Hin + p * NS, n)));
        }
        for (int i = r; i < QC * a.headdim; i += RED) {
            const int s = i / a.headdim, p = i % a.headdim;
            dd += m.dY[s * PS + p] * m.X[s * PS + p];
        }
        m.red[r] = h0.re;
        m.red[RED + r] = h0.im;
        m.red[2 * RED + r] = dd;
    }
}
// This head's dB and dC, with each thread's column share of Ksr and F:
//   xg = x Gh, yh = dy h_in (tiles rows 2 tr + i, complex columns n(j)),
//   dB_s = conj(sum_l K[l][s] C_l) + conj(w_s) xg_s,   Ksr[s] = sum_n B_s[n] conj(xg_s[n]),
//   dC_l = conj(sum_s K[l][s] B_s + e_l yh_l),          F[l] / e_l = sum_n C_l[n] yh_l[n].
__host__ __device__ inline void k5_bc(const BwdArgs &a, int c, int h, int b, int tid, const Smem &m) {
    const int r0 = 2 * (tid >> 4), tc = tid & 15;
    float *part_k = m.part, *part_f = m.part + QC * 16 * 2;
    {
        c2 acc[2][4];
        for (int i = 0; i < 2; ++i)
            for (int j = 0; j < 4; ++j) acc[i][j] = cmk(0.f, 0.f);
        for (int p = 0; p < P_MAX; p += 4) {  // x Gh
            f4 xa[2];
            for (int i = 0; i < 2; ++i) xa[i] = ld4(m.X + (r0 + i) * PS + p);
            for (int pp = 0; pp < 4; ++pp)
                for (int i = 0; i < 2; ++i) axpy4(acc[i], comp(xa[i], pp), m.Gh + (p + pp) * NS, tc);
        }
        c2 kc[2][4];
        for (int i = 0; i < 2; ++i) {
            const int s = r0 + i;
            c2 ks = cmk(0.f, 0.f);
            for (int j = 0; j < 4; ++j) {
                ks = cadd(ks, cmul(sm2(m.Bs + s * NS, ncol(tc, j)), cconj(acc[i][j])));
                kc[i][j] = cmk(0.f, 0.f);
            }
            st2(part_k + (s * 16 + tc) * 2, ks);
        }
        for (int l = r0; l < QC; ++l) {  // sum_l K[l][s] C_l, K[l][s] = 0 for l < s
            const f4 kv = ld4(m.K + l * QS2 + 2 * r0);
            czpy4(kc[0], c2{kv.x, kv.y}, m.Cs + l * NS, tc);
            czpy4(kc[1], c2{kv.z, kv.w}, m.Cs + l * NS, tc);
        }
        for (int i = 0; i < 2; ++i) {
            const int s = r0 + i, t = c * QC + s;
            if (t >= a.seqlen) continue;
            const c2 wc = cconj(ld2(m.w + 2 * s));
            c2 v[4];
            for (int j = 0; j < 4; ++j) v[j] = cadd(cconj(kc[i][j]), cmul(wc, acc[i][j]));
            store_n4(a.dBh + 2 * ((((size_t)b * a.seqlen + t) * a.nheads + h) * a.dstate), tc, a.dstate, v);
        }
    }
    {
        c2 acc[2][4];
        for (int i = 0; i < 2; ++i)
            for (int j = 0; j < 4; ++j) acc[i][j] = cmk(0.f, 0.f);
        for (int p = 0; p < P_MAX; p += 4) {  // dy h_in
            f4 ya[2];
            for (int i = 0; i < 2; ++i) ya[i] = ld4(m.dY + (r0 + i) * PS + p);
            for (int pp = 0; pp < 4; ++pp)
                for (int i = 0; i < 2; ++i) axpy4(acc[i], comp(ya[i], pp), m.Hin + (p + pp) * NS, tc);
        }
        for (int i = 0; i < 2; ++i) {
            const int l = r0 + i;
            c2 f = cmk(0.f, 0.f);
            const c2 el = ld2(m.e + 2 * l);
            for (int j = 0; j < 4; ++j) {
                f = cadd(f, cmul(sm2(m.Cs + l * NS, ncol(tc, j)), acc[i][j]));
                acc[i][j] = cmul(el, acc[i][j]);
            }
            st2(part_f + (l * 16 + tc) * 2, f);
        }
        for (int k = 0; k < r0 + 2; k += 2) {  // sum_s K[l][s] B_s, K[l][s] = 0 for s > l
            for (int i = 0; i < 2; ++i) {
                const f4 kv = ld4(m.K + (r0 + i) * QS2 + 2 * k);
                czpy4(acc[i], c2{kv.x, kv.y}, m.Bs + k * NS, tc);
                czpy4(acc[i], c2{kv.z, kv.w}, m.Bs + (k + 1) * NS, tc);
            }
        }
        for (int i = 0; i < 2; ++i) {
            const int l = r0 + i, t = c * QC + l;
            if (t >= a.seqlen) continue;
            c2 v[4];
            for (int j = 0; j < 4; ++j) v[j] = cconj(acc[i][j]);
            store_n4(a.dCh + 2 * ((((size_t)b * a.seqlen + t) * a.nheads + h) * a.dstate), tc, a.dstate, v);
        }
    }
}
// F and Ksr from their column shares (fixed order).
__host__ __device__ inline void k5_fk(const BwdArgs &a, int tid, const Smem &m) {
    (void)a;
    const float *part_k = m.part, *part_f = m.part + QC * 16 * 2;
    if (tid < QC) {
        c2 v = cmk(0.f, 0.f);
        for (int q = 0; q < 16; ++q) v = cadd(v, ld2(part_f + (tid * 16 + q) * 2));
        st2(m.F + 2 * tid, cmul(ld2(m.e + 2 * tid), v));
    } else if (tid < 2 * QC) {
        const int t = tid - QC;
        c2 v = cmk(0.f, 0.f);
        for (int q = 0; q < 16; ++q) v = cadd(v, ld2(part_k + (t * 16 + q) * 2));
        st2(m.Ksr + 2 * t, v);
    } else if (tid == 2 * QC) {  // the decay gradient's sums, off its one thread
        c2 h0 = cmk(0.f, 0.f);
        for (int r = 0; r < RED; ++r) h0 = cadd(h0, cmk(m.red[r], m.red[RED + r]));
        st2(m.misc + 2, cmul(cexpc(ld2(m.misc)), h0));
    } else if (tid == 3 * QC) {
        float dd = 0.f;
        for (int r = 0; r < RED; ++r) dd += m.red[2 * RED + r];
        m.misc[4] = dd;
    }
}
__host__ __device__ inline void k5_decay(const BwdArgs &a, int c, int h, int b, int tid, const Smem &m) {
    if (tid != 0) return;
    const c2 Ah = ld2(a.A + 2 * h), h0 = ld2(m.misc + 2);
    const float dd = m.misc[4];
    c2 ksum = cmk(0.f, 0.f);
    for (int t = 0; t < QC; ++t) ksum = cadd(ksum, cmul(ld2(m.w + 2 * t), ld2(m.Ksr + 2 * t)));
    c2 run = cmk(0.f, 0.f), dAp = cmk(0.f, 0.f);
    for (int t = QC - 1; t >= 0; --t) {
        // colsum of E = dt_t * colsum of GL o XY
        c2 inner = csub(ld2(m.rowE + 2 * t), cscale(ld2(m.colG + 2 * t), m.d[t]));
        inner = cadd(inner, ld2(m.F + 2 * t));
        inner = csub(inner, cmul(ld2(m.w + 2 * t), ld2(m.Ksr + 2 * t)));
        if (t == QC - 1) inner = cadd(inner, cadd(h0, ksum));
        run = cadd(run, cconj(inner));  // dalpha[t] = sum_{t' >= t} dacs[t']
        const int tg = c * QC + t;
        if (tg < a.seqlen) {
            const c2 wlam = ld2(m.el + 2 * t);
            a.ddt[ix_dt(a, b, tg, h)] =
                m.colG[2 * t] + cmul(wlam, ld2(m.Ksr + 2 * t)).re + cmul(cconj(run), Ah).re;
        }
        dAp = cadd(dAp, cscale(run, m.d[t]));
    }
    st2(a.dAp + 2 * (ix_bh(a, b, h) * a.nchunks + c), dAp);
    a.dDp[ix_bh(a, b, h) * a.nchunks + c] = dd;
}
// dx_s = dt_s sum_l Re(GL[l][s]) dy_l + D dy_s + Re(conj(w_s) sum_n conj(B_s[n]) Gh[.][n]),
// thread tile rows s = 2 tr + i, columns p = tc + 16 j.
__host__ __device__ inline void k5_dx(const BwdArgs &a, int c, int h, int b, int tid, const Smem &m) {
    const int r0 = 2 * (tid >> 4), tc = tid & 15;
    const float Dh = a.D ? a.D[h] : 0.f;
    float acc[2][4];
    c2 gb[2][4];
    for (int i = 0; i < 2; ++i)
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f, gb[i][j] = cmk(0.f, 0.f);
    for (int l = r0; l < QC; ++l) {  // GL[l][s] = 0 for l < s
        const f4 gl = ld4(m.GL + l * QS2 + 2 * r0);
        for (int j = 0; j < 4; ++j) {
            const float yv = m.dY[l * PS + tc + 16 * j];
            acc[0][j] = fmaf(gl.x, yv, acc[0][j]);
            acc[1][j] = fmaf(gl.z, yv, acc[1][j]);
        }
    }
    for (int k = 0; k < 2 * N_MAX; k += 4) {  // conj(B_s) . Gh[p], two complex states per step
        f4 ba[2], gv[4];
        for (int i = 0; i < 2; ++i) ba[i] = ld4(m.Bs + (r0 + i) * NS + k);
        for (int j = 0; j < 4; ++j) gv[j] = ld4(m.Gh + (tc + 16 * j) * NS + k);
        for (int i = 0; i < 2; ++i)
            for (int j = 0; j < 4; ++j) {
                const f4 &u = ba[i], &v = gv[j];
                gb[i][j].re = fmaf(u.x, v.x, fmaf(u.y, v.y, fmaf(u.z, v.z, fmaf(u.w, v.w, gb[i][j].re))));
                gb[i][j].im = fmaf(u.x, v.y, fmaf(-u.y, v.x, fmaf(u.z, v.w, fmaf(-u.w, v.z, gb[i][j].im))));
            }
    }
    for (int i = 0; i < 2; ++i) {
        const int s = r0 + i, t = c * QC + s;
        if (t >= a.seqlen) continue;
        const c2 ws = ld2(m.w + 2 * s);
        for (int j = 0; j < 4; ++j) {
            const int p = tc + 16 * j;
            if (p >= a.headdim) continue;
            a.dx[ix_x(a, b, t, h, p)] = m.d[s] * acc[i][j] + Dh * m.dY[s * PS + p] + ws.re * gb[i][j].re +
                                        ws.im * gb[i][j].im;
        }
    }
}

// ---------------------------------------------------- 6: sums over heads
__host__ __device__ inline void k6_group(const BwdArgs &a, size_t i) {  // i: complex element of dB / dC
    const size_t per_t = (size_t)a.ngroups * a.dstate;
    const size_t bt = i / per_t, rem = i % per_t;
    const int g = (int)(rem / a.dstate), n = (int)(rem % a.dstate);
    const int hpg = a.nheads / a.ngroups;
    c2 sb = cmk(0.f, 0.f), sc = cmk(0.f, 0.f);
    for (int j = 0; j < hpg; ++j) {
        const size_t o = 2 * ((bt * a.nheads + (size_t)g * hpg + j) * a.dstate + n);
        sb = cadd(sb, ld2(a.dBh + o));
        sc = cadd(sc, ld2(a.dCh + o));
    }
    st2(a.dB + 2 * i, sb);
    st2(a.dC + 2 * i, sc);
}
__host__ __device__ inline void k6_head(const BwdArgs &a, int h) {
    c2 sa = cmk(0.f, 0.f);
    float sd = 0.f;
    for (int b = 0; b < a.batch; ++b)
        for (int c = 0; c < a.nchunks; ++c) {
            sa = cadd(sa, ld2(a.dAp + 2 * (ix_bh(a, b, h) * a.nchunks + c)));
            sd += a.dDp[ix_bh(a, b, h) * a.nchunks + c];
        }
    st2(a.dA + 2 * h, sa);
    if (a.dD) a.dD[h] = sd;
}

}  // namespace bwdc
}  // namespace ssd
