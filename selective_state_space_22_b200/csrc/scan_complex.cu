// scan_complex.cu -- the complex chunked scan (one complex A per head) on CUDA
// cores, float32 arithmetic, by a phase rotation that makes every contraction
// real.
//
// With the cumulative log-decay of a chunk split into its real and imaginary
// parts, A_cs[l] = r_l + i theta_l, the decay between two tokens factors as
//
//   exp(A_cs[l] - A_cs[s]) = exp(r_l - r_s) * e^{i theta_l} * e^{-i theta_s}.
//
// Rotating each token's C and B by its own phase, C'_l = C_l e^{i theta_l} and
// B'_s = B_s e^{-i theta_s}, leaves a real decay magnitude, and because x is real
// only real parts are ever needed ("Block Anatomy, Numerical Stability &
// Scaling", Block Anatomy section 4.3-4.4 and 6: complex B, C and A, the real
// part of the output leaves the scan):
//
//   diagonal block  Re(G o L)[l, s] = exp(r_l - r_s) * Re(C'_l . B'_s)
//   chunk state     S[p, n] = e^{i Theta} sum_s exp(R - r_s) dt_s x_s[p] B'_s[n]
//   off-diagonal    Re(exp(A_cs[l]) C_l . h[p]) = exp(r_l) * Re(C'_l . h[p])
//
// (R + i Theta = the chunk's total log-decay).  Each Re(u . v) over N complex
// entries is one real dot product over 2N interleaved values,
// [u_re, -u_im] . [v_re, v_im], so all four contractions are real GEMMs with
// K = 2N, register-tiled below.  Three kernels, as in the real CUDA-core path:
// chunk state, the sequential state pass over chunks, and the chunk scan.
#include "cplx_view.cuh"
#include "ssd_internal.cuh"
#include "tc_ptx.cuh"

namespace ssd {
namespace {

constexpr int NT = 256;
constexpr int KC = 32;   // K-slice staged in shared memory
constexpr int KS = 64;   // tokens per chunk-state stage
constexpr int TL = 64;   // rows (tokens) per output tile
constexpr int TP = 64;   // head-dim columns per output tile
constexpr int TJ = 128;  // interleaved state values (2N) per chunk-state tile

struct CWs {  // the generic workspace layout with K = 2 (real and imaginary blocks)
    double *cs;
    double *lam;
    cf *S;
};

CWs carve_c(void *ws, const ScanArgs &a) {
    const size_t nbhc = (size_t)a.batch * a.nheads * a.nchunks;
    char *p = static_cast<char *>(ws);
    CWs w;
    w.cs = reinterpret_cast<double *>(p);
    p += align_up(nbhc * 2 * a.chunk * sizeof(double), 256);
    w.lam = reinterpret_cast<double *>(p);
    p += align_up(nbhc * 2 * sizeof(double), 256);
    w.S = reinterpret_cast<cf *>(p);
    return w;
}

// Inclusive prefix sum of v[0..Q) by one warp, in double.
__device__ void warp_scan_d(double *v, int Q) {
    const int lane = threadIdx.x & 31;
    double carry = 0.0;
    for (int base = 0; base < Q; base += 32) {
        double x = (base + lane < Q) ? v[base + lane] : 0.0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const double y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        x += carry;
        if (base + lane < Q) v[base + lane] = x;
        carry = __shfl_sync(0xffffffffu, x, 31);
    }
}

// dt of the chunk and its cumulative log-decay (real and imaginary parts, double)
// into shared memory; tokens past the sequence end get dt = 0.
template <typename T>
__device__ void chunk_log_decay(const ScanArgs &a, const CplxView<T> &v, int b, int h, int c, float *dts, double *cre,
                                double *cim) {
    const int Q = a.chunk, t0 = c * Q, valid = min(Q, a.seqlen - t0);
    const float Ar = a.A[2 * h], Ai = a.A[2 * h + 1];
    for (int s = threadIdx.x; s < Q; s += NT) {
        const float d = s < valid ? view_dt(v, (size_t)b * a.seqlen + t0 + s, h) : 0.f;
        dts[s] = d;
        cre[s] = (double)d * Ar;
        cim[s] = (double)d * Ai;
    }
    __syncthreads();
    if (threadIdx.x < 32)
        warp_scan_d(cre, Q);
    else if (threadIdx.x < 64)
        warp_scan_d(cim, Q);
    __syncthreads();
}

// ------------------------------------------------------------ 1. chunk state
// S[p, n] = e^{i Theta} sum_s w_s x_s[p] B'_s[n],  w_s = exp(R - r_s) dt_s.
// Block: one (batch, head, chunk) and a 64 x 128 tile of (p, interleaved n);
// thread: 4 p x 8 interleaved values, columns 4 tj .. 4 tj + 3 and 64 + 4 tj ..
// 64 + 4 tj + 3 (each 8-thread phase of a 128-bit shared load then reads 128
// contiguous bytes: no bank conflict).
template <typename T>
__global__ void __launch_bounds__(NT) cplx_chunk_state_kernel(ScanArgs a, CWs w, CplxView<T> v, int npt, int njt) {
    const int Q = a.chunk, H = a.nheads, P = a.headdim, N = a.dstate;
    const int c = blockIdx.x, h = blockIdx.y;
    const int b = blockIdx.z / (npt * njt), pt = (blockIdx.z / njt) % npt, jt = blockIdx.z % njt;
    const int g = h / (H / a.ngroups);
    const int t0 = c * Q, valid = min(Q, a.seqlen - t0);
    const int p0 = pt * TP, n0 = jt * (TJ / 2);

    extern __shared__ __align__(16) unsigned char smem_raw[];
    double *cre = reinterpret_cast<double *>(smem_raw);
    double *cim = cre + Q;
    float *dts = reinterpret_cast<float *>(cim + Q);
    float *wgt = dts + Q;
    float2 *rot = reinterpret_cast<float2 *>(wgt + Q);  // e^{-i theta_s}
    float *Xw = reinterpret_cast<float *>(rot + Q);     // [KS][TP]
    float *Bt = Xw + KS * TP;                           // [KS][TJ]

    chunk_log_decay(a, v, b, h, c, dts, cre, cim);
    const double R = cre[Q - 1], Th = cim[Q - 1];
    const size_t bhc = ((size_t)b * H + h) * a.nchunks + c;
    if (blockIdx.z % (npt * njt) == 0) {
        for (int s = threadIdx.x; s < Q; s += NT) {
            w.cs[(bhc * 2) * Q + s] = cre[s];
            w.cs[(bhc * 2 + 1) * Q + s] = cim[s];
        }
        if (threadIdx.x == 0) {
            w.lam[bhc * 2] = R;
            w.lam[bhc * 2 + 1] = Th;
        }
    }
    for (int s = threadIdx.x; s < Q; s += NT) {
        wgt[s] = (float)exp(R - cre[s]) * dts[s];
        double sn, cn;
        sincos(cim[s], &sn, &cn);
        rot[s] = make_float2((float)cn, (float)-sn);
    }
    __syncthreads();

    const int tp = threadIdx.x / 16, tj = threadIdx.x % 16;
    float acc[4][8];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
    for (int s0 = 0; s0 < valid; s0 += KS) {
        {  // all of a thread's loads are issued before its first shared-memory store
            constexpr int IX = KS * TP / NT, IB = KS * (TJ / 2) / NT;
            float xv[IX];
            cf bv[IB];
#pragma unroll
            for (int it = 0; it < IX; ++it) {
                const int i = threadIdx.x + it * NT, k = i / TP, p = i % TP, s = s0 + k;
                xv[it] = (s < valid && p0 + p < P) ? view_x(v, (size_t)b * a.seqlen + t0 + s, h, P, p0 + p) : 0.f;
            }
#pragma unroll
            for (int it = 0; it < IB; ++it) {
                const int i = threadIdx.x + it * NT, k = i / (TJ / 2), m = i % (TJ / 2), s = s0 + k;
                bv[it] = (s < valid && n0 + m < N) ? view_b(v, (size_t)b * a.seqlen + t0 + s, g, n0 + m) : cf{0.f, 0.f};
            }
#pragma unroll
            for (int it = 0; it < IX; ++it) {
                const int i = threadIdx.x + it * NT;
                Xw[i] = xv[it] * wgt[s0 + i / TP];
            }
#pragma unroll
            for (int it = 0; it < IB; ++it) {
                const int i = threadIdx.x + it * NT, k = i / (TJ / 2), m = i % (TJ / 2);
                const float2 r = rot[s0 + k];
                reinterpret_cast<float2 *>(Bt + k * TJ)[m] =
                    make_float2(bv[it].re * r.x - bv[it].im * r.y, bv[it].re * r.y + bv[it].im * r.x);
            }
        }
        __syncthreads();
#pragma unroll 8
        for (int k = 0; k < KS; ++k) {
            const float4 xa = *reinterpret_cast<const float4 *>(Xw + k * TP + 4 * tp);
            const float4 b0 = *reinterpret_cast<const float4 *>(Bt + k * TJ + 4 * tj);
            const float4 b1 = *reinterpret_cast<const float4 *>(Bt + k * TJ + 64 + 4 * tj);
            const float av[4] = {xa.x, xa.y, xa.z, xa.w};
            const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
        __syncthreads();
    }
    double st, ct;
    sincos(Th, &st, &ct);
    const float er = (float)ct, ei = (float)st;
    cf *S = w.S + bhc * (size_t)P * N;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int p = p0 + 4 * tp + i;
        if (p >= P) continue;
#pragma unroll
        for (int m = 0; m < 4; ++m) {  // complex columns 2 tj, 2 tj + 1, 32 + 2 tj, 32 + 2 tj + 1
            const int n = n0 + (m < 2 ? 2 * tj + m : 32 + 2 * tj + (m - 2));
            if (n >= N) continue;
            const float sr = acc[i][2 * m], si = acc[i][2 * m + 1];
            S[(size_t)p * N + n] = {er * sr - ei * si, er * si + ei * sr};
        }
    }
}

// ------------------------------------------------------------ 2. state pass
// h_c = exp(A_cs total of chunk c) h_{c-1} + S_c per state element, in place:
// S_c becomes the state entering chunk c; the last h is the final state.  The
// chunks' complex decay factors are computed once per block (NT chunks at a
// time) into shared memory; every thread stays to the end for the barriers.
__global__ void __launch_bounds__(NT, 4) cplx_state_pass_kernel(ScanArgs a, CWs w) {
    __shared__ cf fac[NT];
    ptx::grid_dep_wait();    // the chunk states are complete
    ptx::grid_dep_launch();  // the chunk scan may start its prologue
    const int PN = a.headdim * a.dstate;
    const int e = blockIdx.x * NT + threadIdx.x;
    const int h = blockIdx.y, b = blockIdx.z;
    const bool live = e < PN;
    const size_t bh = (size_t)b * a.nheads + h;
    cf run = {0.f, 0.f};
    if (live && a.init_state) run = reinterpret_cast<const cf *>(a.init_state)[bh * PN + e];
    constexpr int GRP = 16;  // chunk states loaded together, then folded in order
    for (int f0 = 0; f0 < a.nchunks; f0 += NT) {
        const int nf = min(NT, a.nchunks - f0);
        __syncthreads();  // the previous factors are no longer read
        if ((int)threadIdx.x < nf) {
            const size_t bhc = bh * a.nchunks + f0 + threadIdx.x;
            const float mag = expf((float)w.lam[bhc * 2]);
            float sn, cn;
            sincosf((float)w.lam[bhc * 2 + 1], &sn, &cn);
            fac[threadIdx.x] = {mag * cn, mag * sn};
        }
        __syncthreads();
        if (!live) continue;
        for (int c0 = 0; c0 < nf; c0 += GRP) {
            const int n = min(GRP, nf - c0);
            cf sv[GRP];
#pragma unroll
            for (int i = 0; i < GRP; ++i)
                if (i < n) sv[i] = w.S[(bh * a.nchunks + f0 + c0 + i) * PN + e];
#pragma unroll
            for (int i = 0; i < GRP; ++i) {
                if (i >= n) break;
                w.S[(bh * a.nchunks + f0 + c0 + i) * PN + e] = run;
                run = cfma(fac[c0 + i], run, sv[i]);
            }
        }
    }
    if (live && a.final_state) reinterpret_cast<cf *>(a.final_state)[bh * PN + e] = run;
}

// ------------------------------------------------------------- 3. chunk scan
// Block: one (batch, head, chunk), 64 rows l and 64 head-dim columns p;
// thread: 4 x 4 outputs.
//   y[l, p] = exp(r_l) Re(C'_l . h_in[p]) + sum_{s <= l} exp(r_l - r_s) dt_s Re(C'_l . B'_s) x_s[p] + D x_l[p]
// One (batch, head, chunk, 64-row tile, 64-column tile) of the chunk scan; the
// kernel below runs one per block, and the tensor-core chunk scan calls it for
// chunks whose decay is too steep for its factored form.  smem_raw: at least
// cplx_scan_tile_smem(Q) bytes.
template <typename T>
__device__ void cplx_scan_tile(const ScanArgs &a, const CWs &w, const CplxView<T> &v, int b, int h, int c, int rt,
                               int pt, unsigned char *smem_raw) {
    const int Q = a.chunk, H = a.nheads, P = a.headdim, N = a.dstate, K2 = 2 * N;
    const int g = h / (H / a.ngroups);
    const int t0 = c * Q, valid = min(Q, a.seqlen - t0);
    const int l0 = rt * TL;
    if (l0 >= valid) return;
    const int rows = min(TL, valid - l0);
    const int p0 = pt * TP;
    const size_t bhc = ((size_t)b * H + h) * a.nchunks + c;

    float *rr = reinterpret_cast<float *>(smem_raw);   // r_s (real cumulative log-decay)
    float *dts = rr + Q;
    float2 *ph = reinterpret_cast<float2 *>(dts + Q);  // e^{i theta_s}
    float *At = reinterpret_cast<float *>(ph + Q);     // [KC][TL]   [C'_re, -C'_im] of rows l
    float *Bt = At + KC * TL;                          // [KC][64]   [B'_re, B'_im] of tokens s, or h_in
    float *Ms = Bt + KC * 64;                          // [64 s][TL]
    float *Xs = Ms + 64 * TL;                          // [64 s][TP]

    for (int s = threadIdx.x; s < Q; s += NT) {
        rr[s] = (float)w.cs[(bhc * 2) * Q + s];
        double sn, cn;
        sincos(w.cs[(bhc * 2 + 1) * Q + s], &sn, &cn);
        ph[s] = make_float2((float)cn, (float)sn);
        dts[s] = s < valid ? view_dt(v, (size_t)b * a.seqlen + t0 + s, h) : 0.f;
    }
    __syncthreads();

    const int li = threadIdx.x / 16, pi = threadIdx.x % 16;
    // [C'_re, -C'_im] of row l, complex index n, into At[kk][l] (kk = 2 (n - n0))
    auto stage_c = [&](int kc) {
        for (int i = threadIdx.x; i < (KC / 2) * TL; i += NT) {
            const int l = i / (KC / 2), m = i % (KC / 2), n = kc / 2 + m;
            float vr = 0.f, vi = 0.f;
            if (l < rows && n < N) {
                const cf cv = view_c(v, (size_t)b * a.seqlen + t0 + l0 + l, g, n);
                const float2 e = ph[l0 + l];
                vr = cv.re * e.x - cv.im * e.y;
                vi = -(cv.re * e.y + cv.im * e.x);
            }
            At[(2 * m) * TL + l] = vr;
            At[(2 * m + 1) * TL + l] = vi;
        }
    };

    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

    // Off-diagonal: exp(r_l) Re(C'_l . h_in[p]) (skipped when h_in is zero).
    if (c > 0 || a.init_state) {
        const cf *hin = w.S + bhc * (size_t)P * N;
        for (int kc = 0; kc < K2; kc += KC) {
            stage_c(kc);
            for (int i = threadIdx.x; i < (KC / 2) * TP; i += NT) {
                const int p = i / (KC / 2), m = i % (KC / 2), n = kc / 2 + m;
                cf v = {0.f, 0.f};
                if (p0 + p < P && n < N) v = hin[(size_t)(p0 + p) * N + n];
                Bt[(2 * m) * 64 + p] = v.re;
                Bt[(2 * m + 1) * 64 + p] = v.im;
            }
            __syncthreads();
#pragma unroll 4
            for (int k = 0; k < KC; ++k) {
                const float4 av = *reinterpret_cast<const float4 *>(At + k * TL + 4 * li);
                const float4 bv = *reinterpret_cast<const float4 *>(Bt + k * 64 + 4 * pi);
                const float aa[4] = {av.x, av.y, av.z, av.w}, bb[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(aa[i], bb[j], acc[i][j]);
            }
            __syncthreads();
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float el = expf(rr[l0 + 4 * li + i]);
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] *= el;
        }
    }

    // Diagonal block, 64 source tokens at a time.
    const int s_end = l0 + rows;
    for (int s0 = 0; s0 < s_end; s0 += 64) {
        float gacc[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) gacc[i][j] = 0.f;
        for (int kc = 0; kc < K2; kc += KC) {
            stage_c(kc);
            for (int i = threadIdx.x; i < (KC / 2) * 64; i += NT) {
                const int s = i / (KC / 2), m = i % (KC / 2), n = kc / 2 + m;
                float vr = 0.f, vi = 0.f;
                if (s0 + s < valid && n < N) {
                    const cf bv = view_b(v, (size_t)b * a.seqlen + t0 + s0 + s, g, n);
                    const float2 e = ph[s0 + s];  // rotate by e^{-i theta_s}
                    vr = bv.re * e.x + bv.im * e.y;
                    vi = bv.im * e.x - bv.re * e.y;
                }
                Bt[(2 * m) * 64 + s] = vr;
                Bt[(2 * m + 1) * 64 + s] = vi;
            }
            __syncthreads();
#pragma unroll 4
            for (int k = 0; k < KC; ++k) {
                const float4 av = *reinterpret_cast<const float4 *>(At + k * TL + 4 * li);
                const float4 bv = *reinterpret_cast<const float4 *>(Bt + k * 64 + 4 * pi);
                const float aa[4] = {av.x, av.y, av.z, av.w}, bb[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) gacc[i][j] = fmaf(aa[i], bb[j], gacc[i][j]);
            }
            __syncthreads();
        }
        // M[l, s] = exp(r_l - r_s) dt_s Re(C'_l . B'_s), zero above the diagonal
#pragma unroll
        for (int i = 0; i < 4; ++i) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int l = l0 + 4 * li + i, s = s0 + 4 * pi + j;
                float m = 0.f;
                if (s <= l && s < valid && l < valid) m = gacc[i][j] * expf(rr[l] - rr[s]) * dts[s];
                Ms[(4 * pi + j) * TL + 4 * li + i] = m;
            }
        }
        for (int i = threadIdx.x; i < 64 * TP; i += NT) {
            const int s = i / TP, p = i % TP;
            Xs[i] = (s0 + s < valid && p0 + p < P) ? view_x(v, (size_t)b * a.seqlen + t0 + s0 + s, h, P, p0 + p) : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int s = 0; s < 64; ++s) {
            const float4 mv = *reinterpret_cast<const float4 *>(Ms + s * TL + 4 * li);
            const float4 xv = *reinterpret_cast<const float4 *>(Xs + s * TP + 4 * pi);
            const float mm[4] = {mv.x, mv.y, mv.z, mv.w}, xx[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(mm[i], xx[j], acc[i][j]);
        }
        __syncthreads();
    }

    float *yg = reinterpret_cast<float *>(a.y);
    const float Dh = a.D ? a.D[h] : 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int l = 4 * li + i;
        if (l >= rows) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int p = p0 + 4 * pi + j;
            if (p >= P) continue;
            const size_t idx = (((size_t)b * a.seqlen + t0 + l0 + l) * H + h) * P + p;
            yg[idx] = a.D ? fmaf(Dh, view_x(v, (size_t)b * a.seqlen + t0 + l0 + l, h, P, p), acc[i][j]) : acc[i][j];
        }
    }
    __syncthreads();  // the shared memory may be reused by the caller
}

template <typename T>
__global__ void __launch_bounds__(NT) cplx_chunk_scan_kernel(ScanArgs a, CWs w, CplxView<T> v, int nrt, int npt) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    cplx_scan_tile<T>(a, w, v, blockIdx.z / npt, blockIdx.y, blockIdx.x / nrt, blockIdx.x % nrt, blockIdx.z % npt,
                      smem_raw);
}

// The chunk scan for 2N <= 128: the rotated C of the block's 64 rows is staged
// once, in full K, and reused by the off-diagonal product and every source tile;
// each source tile stages its rotated B and x in one step.  Tiles in shared
// memory are [k][64] with rows padded to LD floats; K holds the real parts in
// rows 0-63 and the imaginary parts in rows 64-127 (zero past N).  A warp stages
// 8 state indices x 4 tokens at a time, so its 32 stores fall in 32 banks.
constexpr int LD = 68;
__device__ __forceinline__ void stage_index(int i, int &m, int &c) {  // i in [0, 4096) -> (m, c)
    const int lane = i & 31, blk = i >> 5;
    m = (blk & 7) * 8 + (lane & 7);
    c = (blk >> 3) * 4 + (lane >> 3);
}
template <typename T>
__global__ void __launch_bounds__(NT, 2) cplx_chunk_scan_n64_kernel(ScanArgs a, CWs w, CplxView<T> v, int nrt, int npt) {
    const int Q = a.chunk, H = a.nheads, P = a.headdim, N = a.dstate;
    const int rt = blockIdx.x % nrt, c = blockIdx.x / nrt;
    const int h = blockIdx.y;
    const int pt = blockIdx.z % npt, b = blockIdx.z / npt;
    const int g = h / (H / a.ngroups);
    const int t0 = c * Q, valid = min(Q, a.seqlen - t0);
    const int l0 = rt * TL;
    if (l0 >= valid) return;
    const int rows = min(TL, valid - l0);
    const int p0 = pt * TP;
    const size_t bhc = ((size_t)b * H + h) * a.nchunks + c;

    extern __shared__ __align__(16) unsigned char smem_raw[];
    float *rr = reinterpret_cast<float *>(smem_raw);
    float *dts = rr + Q;
    float2 *ph = reinterpret_cast<float2 *>(dts + Q);  // e^{i theta_s}
    float *Ch = reinterpret_cast<float *>(ph + Q);     // [128][LD]: [C'_re, -C'_im] of rows l
    float *Bs = Ch + 128 * LD;                         // [128][LD]: [B'_re, B'_im] of tokens s, or h_in
    float *Ms = Bs + 128 * LD;                         // [64 s][LD]
    float *Xs = Ms + 64 * LD;                          // [64 s][LD]

    for (int s = threadIdx.x; s < Q; s += NT) {
        rr[s] = (float)w.cs[(bhc * 2) * Q + s];
        double sn, cn;
        sincos(w.cs[(bhc * 2 + 1) * Q + s], &sn, &cn);
        ph[s] = make_float2((float)cn, (float)sn);
        dts[s] = s < valid ? view_dt(v, (size_t)b * a.seqlen + t0 + s, h) : 0.f;
    }
    __syncthreads();
    constexpr int IT = 64 * 64 / NT;  // staged elements per thread
    {
        cf cv[IT];
#pragma unroll
        for (int it = 0; it < IT; ++it) {
            int m, l;
            stage_index(threadIdx.x + it * NT, m, l);
            cv[it] = (l < rows && m < N) ? view_c(v, (size_t)b * a.seqlen + t0 + l0 + l, g, m) : cf{0.f, 0.f};
        }
#pragma unroll
        for (int it = 0; it < IT; ++it) {
            int m, l;
            stage_index(threadIdx.x + it * NT, m, l);
            const float2 e = ph[l0 + l];
            Ch[m * LD + l] = cv[it].re * e.x - cv[it].im * e.y;
            Ch[(64 + m) * LD + l] = -(cv[it].re * e.y + cv[it].im * e.x);
        }
    }

    const int li = threadIdx.x / 16, pi = threadIdx.x % 16;
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    // acc(l, j) += sum_k Ch[k][l] Tk[k][j] over the 2N interleaved values
    auto gemm_k = [&](const float *Tk, float (&o)[4][4]) {
#pragma unroll 8
        for (int k = 0; k < 128; ++k) {
            const float4 av = *reinterpret_cast<const float4 *>(Ch + k * LD + 4 * li);
            const float4 bv = *reinterpret_cast<const float4 *>(Tk + k * LD + 4 * pi);
            const float aa[4] = {av.x, av.y, av.z, av.w}, bb[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) o[i][j] = fmaf(aa[i], bb[j], o[i][j]);
        }
    };

    // Off-diagonal: exp(r_l) Re(C'_l . h_in[p]) (skipped when h_in is zero).
    if (c > 0 || a.init_state) {
        const cf *hin = w.S + bhc * (size_t)P * N;
        cf hv[IT];
#pragma unroll
        for (int it = 0; it < IT; ++it) {
            int m, q;
            stage_index(threadIdx.x + it * NT, m, q);
            hv[it] = (p0 + q < P && m < N) ? hin[(size_t)(p0 + q) * N + m] : cf{0.f, 0.f};
        }
#pragma unroll
        for (int it = 0; it < IT; ++it) {
            int m, q;
            stage_index(threadIdx.x + it * NT, m, q);
            Bs[m * LD + q] = hv[it].re;
            Bs[(64 + m) * LD + q] = hv[it].im;
        }
        __syncthreads();
        gemm_k(Bs, acc);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float el = expf(rr[l0 + 4 * li + i]);
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] *= el;
        }
        __syncthreads();
    }

    // Diagonal block, 64 source tokens at a time.
    const int s_end = l0 + rows;
    for (int s0 = 0; s0 < s_end; s0 += 64) {
        {
            cf bv[IT];
            float xv[IT];
#pragma unroll
            for (int it = 0; it < IT; ++it) {
                int m, sb;
                stage_index(threadIdx.x + it * NT, m, sb);
                bv[it] = (s0 + sb < valid && m < N) ? view_b(v, (size_t)b * a.seqlen + t0 + s0 + sb, g, m) : cf{0.f, 0.f};
                const int i = threadIdx.x + it * NT, s = i / TP, p = i % TP;  // x: p fastest
                xv[it] = (s0 + s < valid && p0 + p < P) ? view_x(v, (size_t)b * a.seqlen + t0 + s0 + s, h, P, p0 + p) : 0.f;
            }
#pragma unroll
            for (int it = 0; it < IT; ++it) {
                int m, sb;
                stage_index(threadIdx.x + it * NT, m, sb);
                const float2 e = ph[s0 + sb];  // rotate by e^{-i theta_s}
                Bs[m * LD + sb] = bv[it].re * e.x + bv[it].im * e.y;
                Bs[(64 + m) * LD + sb] = bv[it].im * e.x - bv[it].re * e.y;
                const int i = threadIdx.x + it * NT;
                Xs[(i / TP) * LD + i % TP] = xv[it];
            }
        }
        __syncthreads();
        float gacc[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) gacc[i][j] = 0.f;
        gemm_k(Bs, gacc);
        // M[l, s] = exp(r_l - r_s) dt_s Re(C'_l . B'_s), zero above the diagonal;
        // each source column's 4 rows go out as one float4
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int s = s0 + 4 * pi + j;
            float m4[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int l = l0 + 4 * li + i;
                m4[i] = (s <= l && s < valid && l < valid) ? gacc[i][j] * expf(rr[l] - rr[s]) * dts[s] : 0.f;
            }
            *reinterpret_cast<float4 *>(Ms + (4 * pi + j) * LD + 4 * li) = make_float4(m4[0], m4[1], m4[2], m4[3]);
        }
        __syncthreads();
#pragma unroll 8
        for (int s = 0; s < 64; ++s) {
            const float4 mv = *reinterpret_cast<const float4 *>(Ms + s * LD + 4 * li);
            const float4 xv = *reinterpret_cast<const float4 *>(Xs + s * LD + 4 * pi);
            const float mm[4] = {mv.x, mv.y, mv.z, mv.w}, xx[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(mm[i], xx[j], acc[i][j]);
        }
        __syncthreads();
    }

    float *yg = reinterpret_cast<float *>(a.y);
    const float Dh = a.D ? a.D[h] : 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int l = 4 * li + i;
        if (l >= rows) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int p = p0 + 4 * pi + j;
            if (p >= P) continue;
            const size_t idx = (((size_t)b * a.seqlen + t0 + l0 + l) * H + h) * P + p;
            yg[idx] = a.D ? fmaf(Dh, view_x(v, (size_t)b * a.seqlen + t0 + l0 + l, h, P, p), acc[i][j]) : acc[i][j];
        }
    }
}

#include "scan_complex_tc.cuh"

}  // namespace

// Launch with programmatic stream serialization: the kernel may begin while its
// predecessor in the stream is ending, and waits for it (grid_dep_wait) before
// it reads what the predecessor wrote.
template <typename... P, typename... Args>
cudaError_t launch_after(void (*kern)(P...), dim3 grid, int threads, size_t smem, cudaStream_t st, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

size_t cplx_scan_tile_smem(int Q) {
    return 2 * Q * sizeof(float) + Q * sizeof(float2) + (KC * TL + KC * 64 + 64 * TL + 64 * TP) * sizeof(float);
}

cudaError_t launch_cplx_state_pass(const ScanArgs &a, void *ws, cudaStream_t st) {
    const CWs w = carve_c(ws, a);
    const int PN = a.headdim * a.dstate;
    return launch_after(cplx_state_pass_kernel, dim3((PN + NT - 1) / NT, a.nheads, a.batch), NT, 0, st, a, w);
}

template <typename T>
cudaError_t launch_complex_cuda_cores(const ScanArgs &a, const CplxView<T> &v, void *ws, cudaStream_t st) {
    const CWs w = carve_c(ws, a);
    const int Q = a.chunk, P = a.headdim, N = a.dstate;
    cudaError_t e;

    const int npt = (P + TP - 1) / TP, njt = (2 * N + TJ - 1) / TJ;
    const size_t sm1 = 2 * Q * sizeof(double) + 2 * Q * sizeof(float) + Q * sizeof(float2) +
                       (KS * TP + KS * TJ) * sizeof(float);
    if ((e = cudaFuncSetAttribute(cplx_chunk_state_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)sm1)) != cudaSuccess)
        return e;
    cplx_chunk_state_kernel<T><<<dim3(a.nchunks, a.nheads, a.batch * npt * njt), NT, sm1, st>>>(a, w, v, npt, njt);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = launch_cplx_state_pass(a, ws, st)) != cudaSuccess) return e;

    const int nrt = (Q + TL - 1) / TL;
    if (N <= 64) {
        const size_t smf = 2 * Q * sizeof(float) + Q * sizeof(float2) + (2 * 128 + 2 * 64) * LD * sizeof(float);
        if ((e = cudaFuncSetAttribute(cplx_chunk_scan_n64_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)smf)) != cudaSuccess)
            return e;
        cplx_chunk_scan_n64_kernel<T><<<dim3(a.nchunks * nrt, a.nheads, a.batch * npt), NT, smf, st>>>(a, w, v, nrt,
                                                                                                       npt);
        return cudaGetLastError();
    }
    const size_t sm3 = cplx_scan_tile_smem(Q);
    if ((e = cudaFuncSetAttribute(cplx_chunk_scan_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)sm3)) != cudaSuccess)
        return e;
    cplx_chunk_scan_kernel<T><<<dim3(a.nchunks * nrt, a.nheads, a.batch * npt), NT, sm3, st>>>(a, w, v, nrt, npt);
    return cudaGetLastError();
}
bool cplx_tc_supported(int headdim, int dstate) { return headdim == 64 && dstate == 64; }

// The tensor-core path: chunk states (tcgen05), the state pass over chunks, the
// chunk scan (tcgen05; steep chunks on CUDA cores), in 128-token chunks.
template <typename T>
cudaError_t launch_complex_tc(const ScanArgs &a0, const CplxView<T> &v, void *ws, cudaStream_t st) {
    ScanArgs a = a0;
    a.chunk = ctc::QT;
    a.nchunks = (a.seqlen + ctc::QT - 1) / ctc::QT;
    const CWs w = carve_c(ws, a);
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(ctc::state_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  ctc::SMEM_STATE)) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(ctc::scan_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  ctc::SMEM_SCAN)) != cudaSuccess)
        return e;
    const dim3 grid(a.nchunks, a.nheads, a.batch);
    ctc::state_kernel<T><<<grid, ctc::NTH, ctc::SMEM_STATE, st>>>(a, w, v);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = launch_cplx_state_pass(a, ws, st)) != cudaSuccess) return e;
    return launch_after(ctc::scan_kernel<T>, grid, ctc::NTH, ctc::SMEM_SCAN, st, a, w, v);
}

template <typename T>
cudaError_t launch_complex_view(const ScanArgs &a, const CplxView<T> &v, void *ws, cudaStream_t st) {
    if (cplx_tc_supported(a.headdim, a.dstate)) return launch_complex_tc<T>(a, v, ws, st);
    return launch_complex_cuda_cores<T>(a, v, ws, st);
}

cudaError_t launch_complex_scan(const ScanArgs &a, void *ws, cudaStream_t st) {
    return launch_complex_view<float>(a, plain_view(a), ws, st);
}

cudaError_t launch_complex_packed(const ScanArgs &a, const void *proj, bool proj_bf16, const float *dt_bias, void *ws,
                                  cudaStream_t st) {
    if (proj_bf16)
        return launch_complex_view<__nv_bfloat16>(
            a, packed_view<__nv_bfloat16>(proj, dt_bias, a.nheads, a.headdim, a.dstate), ws, st);
    return launch_complex_view<float>(a, packed_view<float>(proj, dt_bias, a.nheads, a.headdim, a.dstate), ws, st);
}

}  // namespace ssd
