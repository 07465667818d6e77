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
//
// The per-chunk products run as register-tiled matrix products on the CUDA
// cores: the 256 threads form a 16 x 16 grid, each owns a 4 x 4 or 4 x 8 tile of
// the result, and operands come from shared memory as 16-byte vectors (row
// strides of 4 mod 32 words keep every access pattern free of bank conflicts).
// Sums across threads go through a shared array of partial sums, added in a
// fixed order, so repeated calls stay bitwise equal.
#pragma once

#include <math.h>
#include <stddef.h>
#include <stdint.h>

#ifndef __CUDACC__
#define __host__
#define __device__
#endif

// The inputs and the workspace written by earlier launches are read-only while
// a phase runs; on the device they are read through the read-only path, which
// lets the compiler keep many rows' loads in flight ahead of the shared-memory
// stores of the loading loops.  BWD_UNROLL unrolls those loops on the device.
#ifdef __CUDA_ARCH__
#define BWD_LDG(p) __ldg(p)
#define BWD_UNROLL _Pragma("unroll 8")
#else
#define BWD_LDG(p) (*(p))
#define BWD_UNROLL
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
namespace bwd {

constexpr int QB = 64;       // tokens per chunk
constexpr int NT = 256;      // threads per block
constexpr int P_MAX = 64;    // head dim
constexpr int N_MAX = 128;   // state dim
// Shared-memory row strides: four floats longer than a row, so rows stay 16-byte
// aligned and consecutive rows start 4 banks apart.
constexpr int PS = P_MAX + 4, NS = N_MAX + 4, QS = QB + 4;
constexpr int PASS_GRP = 8;  // chunks whose loads a state pass issues together

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
    int *dev_error;  // device error word (tensor-core phases' bounded waits)
    float *gram;  // [b][g][nchunks][QB][QB]: C B^T of each chunk when the heads of a group share it, else null
};

// Workspace floats for one call (each region padded to 4 floats).
// Whether the heads of a group share one C B^T per chunk (computed once, by the
// group's own phase, and read by each head's per-chunk gradients).
__host__ __device__ inline bool shared_gram(int nheads, int ngroups) { return nheads / ngroups >= 2; }
__host__ __device__ inline size_t ws_floats(int batch, int seqlen, int nheads, int headdim, int ngroups, int dstate,
                                            int nchunks) {
    auto r4 = [](size_t v) { return (v + 3) / 4 * 4; };
    const size_t bh = (size_t)batch * nheads, pn = (size_t)headdim * dstate;
    const size_t gram = shared_gram(nheads, ngroups) ? (size_t)batch * ngroups * nchunks * QB * QB : 0;
    return r4(bh * nchunks * QB) + r4(bh * nchunks) + 3 * r4(bh * nchunks * pn) +
           2 * r4((size_t)batch * seqlen * nheads * dstate) + 2 * r4(bh * nchunks) + r4(gram);
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
    a.dDp = p; p += r4(bh * a.nchunks);
    a.gram = shared_gram(a.nheads, a.ngroups) ? p : nullptr;
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
// One layout serves every chunk kernel (fixed row strides PS, NS, QS).  Arrays
// are zero beyond headdim / dstate, so the products always run over P_MAX and
// N_MAX.
struct Smem {
    float *d, *acs, *e, *w;           // [QB]
    float *X, *dY;                    // [QB][PS]
    float *Bs, *Cs;                   // [QB][NS]
    float *Hin, *Gh;                  // [P_MAX][NS]
    float *GL, *XY, *K;               // [QB][QS]; XY later holds B Gh^T
    float *rowE, *colG, *F, *Ksr;     // [QB]
    float *red;                       // [2 * QB]
    float *part;                      // [QB][16]: partial row sums, one per thread column
    float *el;                        // [QB]: exp(lam - acs)
    float *misc;                      // [4]: lam, exp(lam) <Gh, h_in>, dy . x, sum_s w_s Ksr[s]
};
constexpr size_t SMEM_FLOATS = 4 * QB + 2 * QB * PS + 2 * QB * NS + 2 * P_MAX * NS + 3 * QB * QS +
                               4 * QB + 2 * QB + 16 * QB + QB + 4;
// The chunk-state phase uses the layout up to Bs, the readout phase up to Cs.
constexpr size_t SMEM_FLOATS_K1 = 4 * QB + 2 * QB * PS + QB * NS;
constexpr size_t SMEM_FLOATS_K3 = 4 * QB + 2 * QB * PS + 2 * QB * NS;
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
    m.part = s; s += 16 * QB;
    m.el = s; s += QB;
    m.misc = s;
    return m;
}

// ---------------------------------------------- register-tiled products
struct alignas(16) f4 {
    float x, y, z, w;
};
__host__ __device__ inline f4 ld4(const float *p) { return *reinterpret_cast<const f4 *>(p); }
__host__ __device__ inline float comp(const f4 &v, int i) { return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w; }

// Two fused multiply-adds on a pair of floats: one packed instruction on the
// device (fma.rn.f32x2, each lane rounded as fmaf), two fmaf on the host.
__host__ __device__ inline void fma_pair(float a, float b0, float b1, float &c0, float &c1) {
#ifdef __CUDA_ARCH__
    unsigned long long r;
    const float2 av = make_float2(a, a), bv = make_float2(b0, b1), cv = make_float2(c0, c1);
    asm("fma.rn.f32x2 %0, %1, %2, %3;"
        : "=l"(r)
        : "l"(*reinterpret_cast<const unsigned long long *>(&av)),
          "l"(*reinterpret_cast<const unsigned long long *>(&bv)),
          "l"(*reinterpret_cast<const unsigned long long *>(&cv)));
    const float2 rv = *reinterpret_cast<float2 *>(&r);
    c0 = rv.x;
    c1 = rv.y;
#else
    c0 = fmaf(a, b0, c0);
    c1 = fmaf(a, b1, c1);
#endif
}
// Two independent fused multiply-adds (a0 b0 + c0, a1 b1 + c1) as one packed
// instruction on the device, two fmaf on the host.
__host__ __device__ inline void fma_pairs(float a0, float a1, float b0, float b1, float &c0, float &c1) {
#ifdef __CUDA_ARCH__
    unsigned long long r;
    const float2 av = make_float2(a0, a1), bv = make_float2(b0, b1), cv = make_float2(c0, c1);
    asm("fma.rn.f32x2 %0, %1, %2, %3;"
        : "=l"(r)
        : "l"(*reinterpret_cast<const unsigned long long *>(&av)),
          "l"(*reinterpret_cast<const unsigned long long *>(&bv)),
          "l"(*reinterpret_cast<const unsigned long long *>(&cv)));
    const float2 rv = *reinterpret_cast<float2 *>(&r);
    c0 = rv.x;
    c1 = rv.y;
#else
    c0 = fmaf(a0, b0, c0);
    c1 = fmaf(a1, b1, c1);
#endif
}
// Thread (tr, tc) = (tid / 16, tid % 16) owns rows r0 = 4 tr .. 4 tr + 3.
// "nt": acc[i][j] += sum_k A[r0+i][k] B[tc+16j][k]   (both k-contiguous rows; k0, k1 multiples of 4)
// (The even and odd k run as the two lanes of packed float pairs, added at the end.)
template <int NJ>
__host__ __device__ inline void mm_nt(float (&acc)[4][NJ], const float *A, int lda, int r0, const float *B, int ldb,
                                      int tc, int k0, int k1) {
    float ev[4][NJ], od[4][NJ];
    for (int i = 0; i < 4; ++i)
        for (int j = 0; j < NJ; ++j) ev[i][j] = od[i][j] = 0.f;
    for (int k = k0; k < k1; k += 4) {
        f4 a[4], b[NJ];
        for (int i = 0; i < 4; ++i) a[i] = ld4(A + (r0 + i) * lda + k);
        for (int j = 0; j < NJ; ++j) b[j] = ld4(B + (tc + 16 * j) * ldb + k);
        for (int i = 0; i < 4; ++i)
            for (int j = 0; j < NJ; ++j) {
                fma_pairs(a[i].x, a[i].y, b[j].x, b[j].y, ev[i][j], od[i][j]);
                fma_pairs(a[i].z, a[i].w, b[j].z, b[j].w, ev[i][j], od[i][j]);
            }
    }
    for (int i = 0; i < 4; ++i)
        for (int j = 0; j < NJ; ++j) acc[i][j] += ev[i][j] + od[i][j];
}
// "tn": acc[i][j] += sum_k sc[k] A[k][r0+i] B[k][c(j)],  c(j) = 4 tc + j (+ 60 for j >= 4: 64 + 4 tc + j - 4)
// (sc may be null: no scaling)
template <int NJ>
__host__ __device__ inline void mm_tn(float (&acc)[4][NJ], const float *A, int lda, int r0, const float *sc,
                                      const float *B, int ldb, int tc, int k0, int k1) {
    for (int k = k0; k < k1; ++k) {
        f4 a = ld4(A + k * lda + r0);
        if (sc) {
            const float f = sc[k];
            a.x *= f, a.y *= f, a.z *= f, a.w *= f;
        }
        f4 b[NJ / 4];
        for (int q = 0; q < NJ / 4; ++q) b[q] = ld4(B + k * ldb + 64 * q + 4 * tc);
        for (int i = 0; i < 4; ++i)
            for (int q = 0; q < NJ / 4; ++q) {
                fma_pair(comp(a, i), b[q].x, b[q].y, acc[i][4 * q], acc[i][4 * q + 1]);
                fma_pair(comp(a, i), b[q].z, b[q].w, acc[i][4 * q + 2], acc[i][4 * q + 3]);
            }
    }
}
// "nn": acc[i][j] += sum_k A[r0+i][k] B[k][c(j)]   (k0, k1 multiples of 4)
template <int NJ>
__host__ __device__ inline void mm_nn(float (&acc)[4][NJ], const float *A, int lda, int r0, const float *B, int ldb,
                                      int tc, int k0, int k1) {
    for (int k = k0; k < k1; k += 4) {
        f4 a[4];
        for (int i = 0; i < 4; ++i) a[i] = ld4(A + (r0 + i) * lda + k);
        for (int kk = 0; kk < 4; ++kk) {
            f4 b[NJ / 4];
            for (int q = 0; q < NJ / 4; ++q) b[q] = ld4(B + (k + kk) * ldb + 64 * q + 4 * tc);
            for (int i = 0; i < 4; ++i)
                for (int q = 0; q < NJ / 4; ++q) {
                    fma_pair(comp(a[i], kk), b[q].x, b[q].y, acc[i][4 * q], acc[i][4 * q + 1]);
                    fma_pair(comp(a[i], kk), b[q].z, b[q].w, acc[i][4 * q + 2], acc[i][4 * q + 3]);
                }
        }
    }
}
template <int NJ> __host__ __device__ inline void zero(float (&acc)[4][NJ]) {
    for (int i = 0; i < 4; ++i)
        for (int j = 0; j < NJ; ++j) acc[i][j] = 0.f;
}
// Column of element j of a "tn"/"nn" tile.
__host__ __device__ inline int tile_col(int tc, int j) { return 64 * (j / 4) + 4 * tc + j % 4; }

// Four consecutive values to dst[0..3] of a row holding `valid` values from
// column col: one 16-byte store when all four are valid and aligned.
__host__ __device__ inline void store_row4(float *dst, int col, int valid, const float *v) {
    if (col + 3 < valid && (reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
        *reinterpret_cast<f4 *>(dst) = f4{v[0], v[1], v[2], v[3]};
    } else {
        for (int q = 0; q < 4; ++q)
            if (col + q < valid) dst[q] = v[q];
    }
}

// ------------------------------------------------ shared loading phases
// dt of the chunk (0 past the end), and x or dy [QB][P], B or C [QB][N]; zero
// past the sequence end and beyond headdim / dstate.
__host__ __device__ inline void load_dt(const BwdArgs &a, int c, int h, int b, int tid, const Smem &m) {
    for (int i = tid; i < QB; i += NT) {
        const int t = c * QB + i;
        m.d[i] = t < a.seqlen ? BWD_LDG(a.dt + ix_dt(a, b, t, h)) : 0.f;
    }
}
__host__ __device__ inline void load_rows_p(const BwdArgs &a, const float *src, int c, int h, int b, int tid,
                                            float *dst) {
#ifdef __CUDA_ARCH__
    if (bwd_vec_rows(src, a.headdim)) {
        for (int i = tid; i < QB * (P_MAX / 4); i += NT) {
            const int s = i / (P_MAX / 4), p = 4 * (i % (P_MAX / 4)), t = c * QB + s;
            const bool v = t < a.seqlen && p < a.headdim;
            bwd_cp16(dst + s * PS + p, v ? src + ix_x(a, b, t, h, p) : src, v);
        }
        return;
    }
#endif
    BWD_UNROLL
    for (int i = tid; i < QB * P_MAX; i += NT) {
        const int s = i / P_MAX, p = i % P_MAX, t = c * QB + s;
        dst[s * PS + p] = (t < a.seqlen && p < a.headdim) ? BWD_LDG(src + ix_x(a, b, t, h, p)) : 0.f;
    }
}
__host__ __device__ inline void load_rows_n(const BwdArgs &a, const float *src, int c, int g, int b, int tid,
                                            float *dst) {
#ifdef __CUDA_ARCH__
    if (bwd_vec_rows(src, a.dstate)) {
        for (int i = tid; i < QB * (N_MAX / 4); i += NT) {
            const int s = i / (N_MAX / 4), n = 4 * (i % (N_MAX / 4)), t = c * QB + s;
            const bool v = t < a.seqlen && n < a.dstate;
            bwd_cp16(dst + s * NS + n, v ? src + ix_bc(a, b, t, g, n) : src, v);
        }
        return;
    }
#endif
    BWD_UNROLL
    for (int i = tid; i < QB * N_MAX; i += NT) {
        const int s = i / N_MAX, n = i % N_MAX, t = c * QB + s;
        dst[s * NS + n] = (t < a.seqlen && n < a.dstate) ? BWD_LDG(src + ix_bc(a, b, t, g, n)) : 0.f;
    }
}
__host__ __device__ inline void load_pn(const BwdArgs &a, const float *src, int tid, float *dst) {
#ifdef __CUDA_ARCH__
    if (bwd_vec_rows(src, a.dstate)) {
        for (int i = tid; i < P_MAX * (N_MAX / 4); i += NT) {
            const int p = i / (N_MAX / 4), n = 4 * (i % (N_MAX / 4));
            const bool v = p < a.headdim && n < a.dstate;
            bwd_cp16(dst + p * NS + n, v ? src + (size_t)p * a.dstate + n : src, v);
        }
        return;
    }
#endif
    BWD_UNROLL
    for (int i = tid; i < P_MAX * N_MAX; i += NT) {
        const int p = i / N_MAX, n = i % N_MAX;
        dst[p * NS + n] = (p < a.headdim && n < a.dstate) ? BWD_LDG(src + (size_t)p * a.dstate + n) : 0.f;
    }
}
// A P x N tile (rows p = 4 tr + i, columns tile_col(tc, j)) to a row-major P x N
// array in global memory.
__host__ __device__ inline void store_pn(const BwdArgs &a, float *dst, int tid, const float (&acc)[4][8]) {
    const int r0 = 4 * (tid >> 4), tc = tid & 15;
    for (int i = 0; i < 4; ++i) {
        const int p = r0 + i;
        if (p >= a.headdim) continue;
        for (int q = 0; q < 2; ++q) {
            const int n0 = tile_col(tc, 4 * q);
            if (n0 < a.dstate) store_row4(dst + (size_t)p * a.dstate + n0, n0, a.dstate, &acc[i][4 * q]);
        }
    }
}

// ---------------------------------------------- 1: chunk states (forward)
__host__ __device__ inline void k1_load(const BwdArgs &a, int c, int h, int b, int tid, const Smem &m) {
    load_dt(a, c, h, b, tid, m);
    load_rows_p(a, a.x, c, h, b, tid, m.X);
    load_rows_n(a, a.B, c, group_of(a, h), b, tid, m.Bs);
    bwd_async_wait();
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
    a.lam[ix_bh(a, b, h) * a.nchunks + c] = v;
    for (int i = 0; i < QB; ++i) m.w[i] = expf(v - m.acs[i]) * m.d[i];
}
// S[p][n] = sum_s w_s x_s[p] B_s[n]
__host__ __device__ inline void k1_state(const BwdArgs &a, int c, int h, int b, int tid, const Smem &m) {
    float acc[4][8];
    zero(acc);
    mm_tn<8>(acc, m.X, PS, 4 * (tid >> 4), m.w, m.Bs, NS, tid & 15, 0, QB);
    store_pn(a, a.st + ix_pn(a, b, h, c), tid, acc);
}

// ------------------------------------- 2: state entering each chunk (forward)
// Element i = blk * NT + tid of the P x N state of (batch b, head h).
__host__ __device__ inline void k2_pass(const BwdArgs &a, int blk, int h, int b, int tid) {
    const size_t pn = (size_t)a.headdim * a.dstate, i = (size_t)blk * NT + tid;
    if (i >= pn) return;
    float hv = a.init ? a.init[ix_bh(a, b, h) * pn + i] : 0.f;
    for (int c0 = 0; c0 < a.nchunks; c0 += PASS_GRP) {  // a group's loads in flight together
        float sv[PASS_GRP], lv[PASS_GRP];
        for (int j = 0; j < PASS_GRP; ++j)
            if (c0 + j < a.nchunks) {
                sv[j] = BWD_LDG(a.st + ix_pn(a, b, h, c0 + j) + i);
                lv[j] = BWD_LDG(a.lam + ix_bh(a, b, h) * a.nchunks + c0 + j);
            }
        for (int j = 0; j < PASS_GRP && c0 + j < a.nchunks; ++j) {
            a.hin[ix_pn(a, b, h, c0 + j) + i] = hv;
            hv = expf(lv[j]) * hv + sv[j];
        }
    }
}

// ------------------------------- 3: readout terms R = sum_l e^{acs[l]} dy_l C_l^T
__host__ __device__ inline void k3_load(const BwdArgs &a, int c, int h, int b, int tid, const Smem &m) {
    const float *acs_g = a.acs + (ix_bh(a, b, h) * a.nchunks + c) * QB;
    for (int i = tid; i < QB; i += NT) m.e[i] = expf(BWD_LDG(acs_g + i));
    load_rows_p(a, a.dy, c, h, b, tid, m.dY);
    load_rows_n(a, a.C, c, group_of(a, h), b, tid, m.Cs);
    bwd_async_wait();
}
__host__ __device__ inline void k3_r(const BwdArgs &a, int c, int h, int b, int tid, const Smem &m) {
    float acc[4][8];
    zero(acc);
    mm_tn<8>(acc, m.dY, PS, 4 * (tid >> 4), m.e, m.Cs, NS, tid & 15, 0, QB);
    store_pn(a, a.st + ix_pn(a, b, h, c), tid, acc);  // the chunk states were consumed by pass 2
}

// --------------------- 4: gradient of the state leaving each chunk (backward)
__host__ __device__ inline void k4_pass(const BwdArgs &a, int blk, int h, int b, int tid) {
    const size_t pn = (size_t)a.headdim * a.dstate, i = (size_t)blk * NT + tid;
    if (i >= pn) return;
    float gv = a.dfinal ? a.dfinal[ix_bh(a, b, h) * pn + i] : 0.f;
    for (int c0 = a.nchunks - 1; c0 >= 0; c0 -= PASS_GRP) {  // chunks c0, c0 - 1, ...
        float sv[PASS_GRP], lv[PASS_GRP];
        for (int j = 0; j < PASS_GRP; ++j)
            if (c0 - j >= 0) {
                sv[j] = BWD_LDG(a.st + ix_pn(a, b, h, c0 - j) + i);
                lv[j] = BWD_LDG(a.lam + ix_bh(a, b, h) * a.nchunks + c0 - j);
            }
        for (int j = 0; j < PASS_GRP && c0 - j >= 0; ++j) {
            a.gh[ix_pn(a, b, h, c0 - j) + i] = gv;
            gv = expf(lv[j]) * gv + sv[j];
        }
    }
    if (a.dinit) a.dinit[ix_bh(a, b, h) * pn + i] = gv;
}

// --------------------------- 5a: C B^T of a chunk, once per (batch, group)
// When the heads of a group share B and C, G = C B^T of a chunk is the same for
// all of them: it is formed here once and the per-chunk gradients read it.
__host__ __device__ inline void kg_load(const BwdArgs &a, int c, int g, int b, int tid, const Smem &m) {
    load_rows_n(a, a.B, c, g, b, tid, m.Bs);
    load_rows_n(a, a.C, c, g, b, tid, m.Cs);
    bwd_async_wait();
}
__host__ __device__ inline void kg_gram(const BwdArgs &a, int c, int g, int b, int tid, const Smem &m) {
    const int r0 = 4 * (tid >> 4), tc = tid & 15;
    float acc[4][4];
    zero(acc);
    mm_nt<4>(acc, m.Cs, NS, r0, m.Bs, NS, tc, 0, N_MAX);
    float *dst = a.gram + (((size_t)b * a.ngroups + g) * a.nchunks + c) * QB * QB;
    for (int i = 0; i < 4; ++i)
        for (int j = 0; j < 4; ++j) dst[(r0 + i) * QB + tc + 16 * j] = acc[i][j];
}

// ------------------------------------------------ 5: gradients of one chunk
__host__ __device__ inline void k5_load(const BwdArgs &a, int c, int h, int b, int tid, const Smem &m) {
    const int g = group_of(a, h);
    load_dt(a, c, h, b, tid, m);
    const float *acs_g = a.acs + (ix_bh(a, b, h) * a.nchunks + c) * QB;
    const float lam = a.lam[ix_bh(a, b, h) * a.nchunks + c];
    for (int i = tid; i < QB; i += NT) {
        const int t = c * QB + i;
        const float d = t < a.seqlen ? BWD_LDG(a.dt + ix_dt(a, b, t, h)) : 0.f;
        const float ac = BWD_LDG(acs_g + i);
        m.acs[i] = ac;
        m.e[i] = expf(ac);
        m.el[i] = expf(lam - ac);
        m.w[i] = m.el[i] * d;
    }
    if (tid == 0) m.misc[0] = lam;
    load_rows_p(a, a.x, c, h, b, tid, m.X);
    load_rows_p(a, a.dy, c, h, b, tid, m.dY);
    load_rows_n(a, a.B, c, g, b, tid, m.Bs);
    load_rows_n(a, a.C, c, g, b, tid, m.Cs);
    load_pn(a, a.hin + ix_pn(a, b, h, c), tid, m.Hin);
    load_pn(a, a.gh + ix_pn(a, b, h, c), tid, m.Gh);
    if (a.gram) {  // the group's C B^T of this chunk, into GL (k5_mats turns it into GL in place)
        const float *gsrc = a.gram + (((size_t)b * a.ngroups + g) * a.nchunks + c) * QB * QB;
#ifdef __CUDA_ARCH__
        for (int i = tid; i < QB * QB / 4; i += NT)
            bwd_cp16(m.GL + (i / (QB / 4)) * QS + 4 * (i % (QB / 4)), gsrc + 4 * i, true);
#else
        for (int i = tid; i < QB * QB; i += NT) m.GL[(i / QB) * QS + i % QB] = gsrc[i];
#endif
    }
    bwd_async_wait();
}
// GL = (C B^T) o L (causal), XY = dy x^T, K = L o dt_s o XY; thread tile rows
// l = 4 tr + i, columns s = tc + 16 j.
__host__ __device__ inline void k5_mats(const BwdArgs &a, int tid, const Smem &m) {
    const int r0 = 4 * (tid >> 4), tc = tid & 15;
    float g[4][4], xy[4][4];
    zero(g);
    zero(xy);
    if (a.gram) {  // the group's C B^T, loaded into GL
        for (int i = 0; i < 4; ++i)
            for (int j = 0; j < 4; ++j) g[i][j] = m.GL[(r0 + i) * QS + tc + 16 * j];
    } else {
        mm_nt<4>(g, m.Cs, NS, r0, m.Bs, NS, tc, 0, N_MAX);
    }
    mm_nt<4>(xy, m.dY, PS, r0, m.X, PS, tc, 0, P_MAX);
    for (int i = 0; i < 4; ++i)
        for (int j = 0; j < 4; ++j) {
            const int l = r0 + i, s = tc + 16 * j;
            m.XY[l * QS + s] = xy[i][j];
            if (l >= s) {
                const float L = expf(m.acs[l] - m.acs[s]);
                m.GL[l * QS + s] = g[i][j] * L;
                m.K[l * QS + s] = L * m.d[s] * xy[i][j];
            } else {
                m.GL[l * QS + s] = 0.f;
                m.K[l * QS + s] = 0.f;
            }
        }
}
// Per token: the row sums of E = GL o XY o dt_s, the column sums of GL o XY; the
// last 128 threads reduce <Gh, h_in> and dy . x.  Rows are walked from a
// per-thread start so that the 32 lanes of a warp read 32 different banks.
__host__ __device__ inline void k5_tokens(const BwdArgs &a, int tid, const Smem &m) {
    (void)a;
    if (tid < QB) {
        const int t = tid;
        float re = 0.f;
        for (int q = 0; q < QB; ++q) {
            const int s = (q + t) & (QB - 1);
            re += m.GL[t * QS + s] * m.XY[t * QS + s] * m.d[s];
        }
        m.rowE[t] = re;
    } else if (tid < 2 * QB) {
        const int t = tid - QB;
        float cg = 0.f;
        for (int l = 0; l < QB; ++l) cg += m.GL[l * QS + t] * m.XY[l * QS + t];
        m.colG[t] = cg;
    } else if (tid < 3 * QB) {
        const int r = tid - 2 * QB;
        float h0 = 0.f;
        for (int i = r; i < P_MAX * N_MAX; i += QB) {
            const int p = i / N_MAX, n = i % N_MAX;
            h0 += m.Gh[p * NS + n] * m.Hin[p * NS + n];
        }
        m.red[r] = h0;
    } else {
        const int r = tid - 3 * QB;
        float dd = 0.f;
        for (int i = r; i < QB * P_MAX; i += QB) {
            const int s = i / P_MAX, p = i % P_MAX;
            dd += m.dY[s * PS + p] * m.X[s * PS + p];
        }
        m.red[QB + r] = dd;
    }
}
// GB = B Gh^T into the XY buffer (XY is no longer needed): rows s, columns p.
__host__ __device__ inline void k5_gb(const BwdArgs &a, int tid, const Smem &m) {
    (void)a;
    const int r0 = 4 * (tid >> 4), tc = tid & 15;
    float gb[4][4];
    zero(gb);
    mm_nt<4>(gb, m.Bs, NS, r0, m.Gh, NS, tc, 0, N_MAX);
    for (int i = 0; i < 4; ++i)
        for (int j = 0; j < 4; ++j) m.XY[(r0 + i) * QS + tc + 16 * j] = gb[i][j];
}
// This head's dB: dB_s = sum_l K[l][s] C_l + w_s (x_s Gh); with the partial sums
// of Ksr[s] = B_s . (x_s Gh) per thread column.
__host__ __device__ inline void k5_db(const BwdArgs &a, int c, int h, int b, int tid, const Smem &m) {
    const int r0 = 4 * (tid >> 4), tc = tid & 15;
    float acc[4][8];
    zero(acc);
    mm_nn<8>(acc, m.X, PS, r0, m.Gh, NS, tc, 0, P_MAX);  // x Gh
    for (int i = 0; i < 4; ++i) {
        const int s = r0 + i;
        float ks = 0.f;
        for (int j = 0; j < 8; ++j) ks = fmaf(m.Bs[s * NS + tile_col(tc, j)], acc[i][j], ks);
        m.part[s * 16 + tc] = ks;
        for (int j = 0; j < 8; ++j) acc[i][j] *= m.w[s];
    }
    mm_tn<8>(acc, m.K, QS, r0, nullptr, m.Cs, NS, tc, r0, QB);  // K[l][s] = 0 for l < s
    for (int i = 0; i < 4; ++i) {
        const int s = r0 + i, t = c * QB + s;
        if (t >= a.seqlen) continue;
        float *row = a.dBh + (((size_t)b * a.seqlen + t) * a.nheads + h) * a.dstate;
        for (int q = 0; q < 2; ++q) {
            const int n0 = tile_col(tc, 4 * q);
            if (n0 < a.dstate) store_row4(row + n0, n0, a.dstate, &acc[i][4 * q]);
        }
    }
}
// Ksr from its partial sums (fixed order).
__host__ __device__ inline void k5_ksr(const BwdArgs &a, int tid, const Smem &m) {
    (void)a;
    if (tid < QB) {
        float v = 0.f;
        for (int q = 0; q < 16; ++q) v += m.part[tid * 16 + q];
        m.Ksr[tid] = v;
    }
}
// This head's dC: dC_l = sum_s K[l][s] B_s + e_l (dy_l h_in); with the partial sums
// of F[l] / e_l = C_l . (dy_l h_in).
__host__ __device__ inline void k5_dc(const BwdArgs &a, int c, int h, int b, int tid, const Smem &m) {
    const int r0 = 4 * (tid >> 4), tc = tid & 15;
    float acc[4][8];
    zero(acc);
    mm_nn<8>(acc, m.dY, PS, r0, m.Hin, NS, tc, 0, P_MAX);  // dy h_in
    for (int i = 0; i < 4; ++i) {
        const int l = r0 + i;
        float f = 0.f;
        for (int j = 0; j < 8; ++j) f = fmaf(m.Cs[l * NS + tile_col(tc, j)], acc[i][j], f);
        m.part[l * 16 + tc] = f;
        for (int j = 0; j < 8; ++j) acc[i][j] *= m.e[l];
    }
    mm_nn<8>(acc, m.K, QS, r0, m.Bs, NS, tc, 0, r0 + 4);  // K[l][s] = 0 for s > l
    for (int i = 0; i < 4; ++i) {
        const int l = r0 + i, t = c * QB + l;
        if (t >= a.seqlen) continue;
        float *row = a.dCh + (((size_t)b * a.seqlen + t) * a.nheads + h) * a.dstate;
        for (int q = 0; q < 2; ++q) {
            const int n0 = tile_col(tc, 4 * q);
            if (n0 < a.dstate) store_row4(row + n0, n0, a.dstate, &acc[i][4 * q]);
        }
    }
}
// F from its partial sums; three other threads form the sums the decay gradient
// needs (each in token order), so that the one thread of k5_decay only runs the
// reverse cumulative sum.
__host__ __device__ inline void k5_f(const BwdArgs &a, int tid, const Smem &m) {
    (void)a;
    if (tid < QB) {
        float v = 0.f;
        for (int q = 0; q < 16; ++q) v += m.part[tid * 16 + q];
        m.F[tid] = m.e[tid] * v;
    } else if (tid == QB) {
        float h0 = 0.f;
        for (int r = 0; r < QB; ++r) h0 += m.red[r];
        m.misc[1] = h0 * expf(m.misc[0]);
    } else if (tid == QB + 32) {
        float dd = 0.f;
        for (int r = 0; r < QB; ++r) dd += m.red[QB + r];
        m.misc[2] = dd;
    } else if (tid == QB + 64) {
        float ksum = 0.f;
        for (int r = 0; r < QB; ++r) ksum += m.w[r] * m.Ksr[r];
        m.misc[3] = ksum;
    }
}
// Thread 0: the decay gradient (reverse cumulative sum), ddt, and the dA and dD
// partials of this chunk.
__host__ __device__ inline void k5_decay(const BwdArgs &a, int c, int h, int b, int tid, const Smem &m) {
    if (tid != 0) return;
    const float Ah = a.A[h], h0 = m.misc[1], dd = m.misc[2], ksum = m.misc[3];
    // colsum of E = dt_t * colsum of GL o XY
    float run = 0.f, dAp = 0.f;
    for (int t = QB - 1; t >= 0; --t) {
        float dacs = m.rowE[t] - m.d[t] * m.colG[t] + m.F[t] - m.w[t] * m.Ksr[t];
        if (t == QB - 1) dacs += h0 + ksum;
        run += dacs;  // dalpha[t] = sum_{t' >= t} dacs[t']
        const int tg = c * QB + t;
        if (tg < a.seqlen)
            a.ddt[ix_dt(a, b, tg, h)] = m.colG[t] + m.el[t] * m.Ksr[t] + Ah * run;
        dAp += m.d[t] * run;
    }
    a.dAp[ix_bh(a, b, h) * a.nchunks + c] = dAp;
    a.dDp[ix_bh(a, b, h) * a.nchunks + c] = dd;
}
// dx_s = dt_s sum_l GL[l][s] dy_l + D dy_s + w_s GB[s]  (rows s, columns p)
__host__ __device__ inline void k5_dx(const BwdArgs &a, int c, int h, int b, int tid, const Smem &m) {
    const int r0 = 4 * (tid >> 4), tc = tid & 15;
    const float Dh = a.D ? a.D[h] : 0.f;
    float acc[4][4];
    zero(acc);
    mm_tn<4>(acc, m.GL, QS, r0, nullptr, m.dY, PS, tc, r0, QB);  // GL[l][s] = 0 for l < s
    const int p0 = 4 * tc;
    if (p0 >= a.headdim) return;
    for (int i = 0; i < 4; ++i) {
        const int s = r0 + i, t = c * QB + s;
        if (t >= a.seqlen) continue;
        float v[4];
        for (int j = 0; j < 4; ++j)
            v[j] = m.d[s] * acc[i][j] + Dh * m.dY[s * PS + p0 + j] + m.w[s] * m.XY[s * QS + p0 + j];
        store_row4(a.dx + ix_x(a, b, t, h, p0), p0, a.headdim, v);
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
