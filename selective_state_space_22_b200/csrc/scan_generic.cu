// scan_generic.cu -- chunked SSD scan on CUDA cores, float32 arithmetic.
//
// The chunkwise evaluation of "Block Anatomy, Numerical Stability & Scaling"
// (Numerical Stability, section 4), in three kernels:
//
//  1. chunk_state: per (batch, head, chunk) the inclusive within-chunk cumulative
//     log-decay A_cs = cumsum(dt * A) (kept in double so that the differences
//     A_cs[l] - A_cs[s] lose nothing), the chunk's total log-decay Lambda, and
//     the end-of-chunk state from a zero start,
//        S_c[p, n] = sum_s exp(Lambda - A_cs[s]) dt_s x_s[p] B_s[n].
//  2. state_pass: per state element, sequentially over chunks,
//        h_c = exp(Lambda_c) h_{c-1} + S_c        (h_{-1} = initial state),
//     overwriting S_c in place with the state that ENTERS chunk c; this is the
//     pages' strict-lower-triangular decay_chunk propagation evaluated as a
//     running product.  The last h_c is the final state.
//  3. chunk_scan: per (batch, head, chunk, 64-row tile, 64-column tile)
//        y[l, p] = sum_{s <= l} (C_l . B_s) exp(A_cs[l] - A_cs[s]) dt_s x_s[p]
//                  + exp(A_cs[l]) C_l . h_in[p, :] + D x_l[p].
//
// These serve the real variant in float32 and every shape the tensor-core
// kernel does not take (the complex variant has its own kernels).  A partial
// last chunk is handled by masking: tokens past seqlen contribute nothing and
// the final state is the state after the last real token.  Every exponent
// evaluated is a difference A_cs[l] - A_cs[s] with l >= s (or A_cs[l] itself),
// so for A <= 0 no exp can overflow.
#include "ssd_internal.cuh"

namespace ssd {
namespace {

constexpr int NT = 256;  // threads per block
constexpr int RT = 64;   // output rows (tokens) per scan tile
constexpr int PT = 64;   // headdim columns per scan tile
constexpr int KT = 32;   // dstate slice staged in shared memory
constexpr int ST = 64;   // source tokens per diagonal stage
constexpr int SS = 32;   // tokens per chunk-state stage
constexpr int OPT = 16;  // chunk-state outputs per thread

// B / C element of the io dtype, as float.
template <typename TIO> __device__ __forceinline__ float ld_bc(const void *base, size_t i) {
    return ld_f32(reinterpret_cast<const TIO *>(base) + i);
}

// Workspace regions (each 256-byte aligned; the complex kernels use the same
// layout with K = 2):
//   cs  [b][H][nc][K][Q] double   K = 1 here
//   lam [b][H][nc][K]    double
//   S   [b][H][nc][P][N] float
struct GenericWs {
    double *cs;
    double *lam;
    float *S;
};

GenericWs carve(void *ws, int batch, int nheads, int headdim, int dstate, int chunk, int nchunks,
                bool cplx) {
    const size_t K = cplx ? 2 : 1;
    const size_t nbhc = (size_t)batch * nheads * nchunks;
    char *p = static_cast<char *>(ws);
    GenericWs w;
    w.cs = reinterpret_cast<double *>(p);
    p += align_up(nbhc * K * chunk * sizeof(double), 256);
    w.lam = reinterpret_cast<double *>(p);
    p += align_up(nbhc * K * sizeof(double), 256);
    w.S = reinterpret_cast<float *>(p);
    return w;
}

// Warp 0 turns v[0..Q) into its inclusive prefix sum (double).
__device__ void warp0_inclusive_scan(double *v, int Q) {
    const int lane = threadIdx.x & 31;
    double carry = 0.0;
    for (int base = 0; base < Q; base += 32) {
        double x = (base + lane < Q) ? v[base + lane] : 0.0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            double y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        x += carry;
        if (base + lane < Q) v[base + lane] = x;
        carry = __shfl_sync(0xffffffffu, x, 31);
    }
}

// Shared prologue: dt and the cumulative log-decay of one chunk into shared
// memory.  Tokens past the end of the sequence get dt = 0 (decay 1, no input).
__device__ void load_chunk_decay(const ScanArgs &a, int b, int h, int c, float *dts, double *cs_re) {
    const int Q = a.chunk, t0 = c * Q;
    const int valid = min(Q, a.seqlen - t0);
    const float Ar = a.A[h];
    for (int s = threadIdx.x; s < Q; s += blockDim.x) {
        const float d = (s < valid) ? a.dt[((size_t)b * a.seqlen + t0 + s) * a.nheads + h] : 0.f;
        dts[s] = d;
        cs_re[s] = (double)d * (double)Ar;
    }
    __syncthreads();
    if (threadIdx.x < 32) warp0_inclusive_scan(cs_re, Q);
    __syncthreads();
}

// ------------------------------------------------------------ 1. chunk state
template <typename TIO>
__global__ void __launch_bounds__(NT) chunk_state_kernel(ScanArgs a, GenericWs w) {
    const int Q = a.chunk, H = a.nheads, P = a.headdim, N = a.dstate;
    const int PN = P * N;
    const int nsplit = (PN + NT * OPT - 1) / (NT * OPT);
    const int c = blockIdx.x, h = blockIdx.y;
    const int b = blockIdx.z / nsplit, split = blockIdx.z % nsplit;
    const int g = h / (H / a.ngroups);
    const int t0 = c * Q;
    const int K = 1;

    extern __shared__ __align__(16) unsigned char smem_raw[];
    double *cs_re = reinterpret_cast<double *>(smem_raw);
    float *dts = reinterpret_cast<float *>(cs_re + Q);
    float *ws_ = reinterpret_cast<float *>(dts + Q);  // per-token weight exp(Lambda - A_cs[s]) dt_s
    float *xw = ws_ + Q;                            // [SS][P]
    float *Bs = xw + SS * P;                        // [SS][N]

    load_chunk_decay(a, b, h, c, dts, cs_re);
    const double lam_re = cs_re[Q - 1];
    const size_t bhc = ((size_t)b * H + h) * a.nchunks + c;
    if (split == 0) {
        for (int s = threadIdx.x; s < Q; s += NT) {
            w.cs[(bhc * K) * Q + s] = cs_re[s];
        }
        if (threadIdx.x == 0) {
            w.lam[bhc * K] = lam_re;
        }
    }
    for (int s = threadIdx.x; s < Q; s += NT)
        ws_[s] = (float)exp(lam_re - cs_re[s]) * dts[s];
    __syncthreads();

    const int o0 = split * NT * OPT;
    float acc[OPT];
#pragma unroll
    for (int k = 0; k < OPT; ++k) acc[k] = 0.f;

    const int valid = min(Q, a.seqlen - t0);
    const TIO *xg = reinterpret_cast<const TIO *>(a.x);
    for (int s0 = 0; s0 < valid; s0 += SS) {
        const int sc = min(SS, valid - s0);
        for (int i = threadIdx.x; i < SS * P; i += NT) {
            int s = i / P, p = i % P;
            float v = 0.f;
            if (s < sc) {
                float xv = ld_f32(xg + (((size_t)b * a.seqlen + t0 + s0 + s) * H + h) * P + p);
                v = ws_[s0 + s] * xv;
            }
            xw[i] = v;
        }
        for (int i = threadIdx.x; i < SS * N; i += NT) {
            int s = i / N, n = i % N;
            Bs[i] = (s < sc) ? ld_bc<TIO>(a.B, (((size_t)b * a.seqlen + t0 + s0 + s) * a.ngroups + g) * N + n)
                             : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < OPT; ++k) {
            const int o = o0 + threadIdx.x + k * NT;
            if (o < PN) {
                const int p = o / N, n = o % N;
                float v = acc[k];
                for (int s = 0; s < sc; ++s) v = fmaf(xw[s * P + p], Bs[s * N + n], v);
                acc[k] = v;
            }
        }
        __syncthreads();
    }
    float *S = reinterpret_cast<float *>(w.S) + bhc * PN;
#pragma unroll
    for (int k = 0; k < OPT; ++k) {
        const int o = o0 + threadIdx.x + k * NT;
        if (o < PN) S[o] = acc[k];
    }
}

// ------------------------------------------------------------ 2. state pass
__global__ void __launch_bounds__(NT) state_pass_kernel(ScanArgs a, GenericWs w) {
    const int PN = a.headdim * a.dstate;
    const int e = blockIdx.x * NT + threadIdx.x;
    const int h = blockIdx.y, b = blockIdx.z;
    if (e >= PN) return;
    const int K = 1;
    const size_t bh = (size_t)b * a.nheads + h;
    float run = 0.f;
    if (a.init_state) run = reinterpret_cast<const float *>(a.init_state)[bh * PN + e];
    float *S = reinterpret_cast<float *>(w.S);
    for (int c = 0; c < a.nchunks; ++c) {
        const size_t bhc = bh * a.nchunks + c;
        float s = S[bhc * PN + e];
        S[bhc * PN + e] = run;  // the state entering chunk c
        const float dec = (float)exp(w.lam[bhc * K]);
        run = fmaf(dec, run, s);
    }
    if (a.final_state) reinterpret_cast<float *>(a.final_state)[bh * PN + e] = run;
}

// ------------------------------------------------------------- 3. chunk scan
template <typename TIO>
__global__ void __launch_bounds__(NT) chunk_scan_kernel(ScanArgs a, GenericWs w) {
    const int Q = a.chunk, H = a.nheads, P = a.headdim, N = a.dstate;
    const int nrt = (Q + RT - 1) / RT, npt = (P + PT - 1) / PT;
    const int rt = blockIdx.x % nrt, c = blockIdx.x / nrt;
    const int h = blockIdx.y;
    const int pt = blockIdx.z % npt, b = blockIdx.z / npt;
    const int g = h / (H / a.ngroups);
    const int t0 = c * Q;
    const int valid = min(Q, a.seqlen - t0);
    const int l0 = rt * RT;
    if (l0 >= valid) return;
    const int rows = min(RT, valid - l0);
    const int p0 = pt * PT;
    const int K = 1;
    const size_t bhc = ((size_t)b * H + h) * a.nchunks + c;

    extern __shared__ __align__(16) unsigned char smem_raw[];
    double *cs_re = reinterpret_cast<double *>(smem_raw);
    float *dts = reinterpret_cast<float *>(cs_re + Q);
    float *At = reinterpret_cast<float *>(dts + Q);  // [KT][RT]
    float *Bt = At + KT * RT;                      // [KT][64]
    float *Ms = reinterpret_cast<float *>(Bt + KT * 64);  // [ST][RT]
    float *Xs = Ms + ST * RT;                             // [ST][PT]

    for (int s = threadIdx.x; s < Q; s += NT) {
        cs_re[s] = w.cs[(bhc * K) * Q + s];
        dts[s] = (s < valid) ? a.dt[((size_t)b * a.seqlen + t0 + s) * H + h] : 0.f;
    }
    __syncthreads();

    const int li = threadIdx.x / 16, pi = threadIdx.x % 16;
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

    const TIO *xg = reinterpret_cast<const TIO *>(a.x);
    const size_t PN = (size_t)P * N;

    // Off-diagonal term: exp(A_cs[l]) C_l . h_in[p, :]  (skipped when h_in is 0).
    if (c > 0 || a.init_state) {
        const float *hin = reinterpret_cast<const float *>(w.S) + bhc * PN;
        for (int n0 = 0; n0 < N; n0 += KT) {
            for (int i = threadIdx.x; i < KT * RT; i += NT) {
                int l = i / KT, k = i % KT;
                float v = 0.f;
                if (l < rows && n0 + k < N) {
                    float cv = ld_bc<TIO>(a.C, (((size_t)b * a.seqlen + t0 + l0 + l) * a.ngroups + g) * N + n0 + k);
                    v = cv * (float)exp(cs_re[l0 + l]);
                }
                At[k * RT + l] = v;
            }
            for (int i = threadIdx.x; i < KT * PT; i += NT) {
                int p = i / KT, k = i % KT;
                Bt[k * 64 + p] = (p0 + p < P && n0 + k < N) ? hin[(size_t)(p0 + p) * N + n0 + k]
                                                            : 0.f;
            }
            __syncthreads();
#pragma unroll 4
            for (int k = 0; k < KT; ++k) {
                float av[4], bv[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) av[i] = At[k * RT + li * 4 + i];
#pragma unroll
                for (int j = 0; j < 4; ++j) bv[j] = Bt[k * 64 + pi * 4 + j];
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
            }
            __syncthreads();
        }
    }

    // Diagonal block: sum_{s <= l} Re((C_l . B_s) exp(A_cs[l] - A_cs[s])) dt_s x_s[p].
    const int s_end = l0 + rows;
    for (int s0 = 0; s0 < s_end; s0 += ST) {
        float gacc[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) gacc[i][j] = 0.f;
        for (int n0 = 0; n0 < N; n0 += KT) {
            for (int i = threadIdx.x; i < KT * RT; i += NT) {
                int l = i / KT, k = i % KT;
                At[k * RT + l] = (l < rows && n0 + k < N)
                    ? ld_bc<TIO>(a.C, (((size_t)b * a.seqlen + t0 + l0 + l) * a.ngroups + g) * N + n0 + k)
                    : 0.f;
            }
            for (int i = threadIdx.x; i < KT * ST; i += NT) {
                int s = i / KT, k = i % KT;
                Bt[k * 64 + s] = (s0 + s < valid && n0 + k < N)
                    ? ld_bc<TIO>(a.B, (((size_t)b * a.seqlen + t0 + s0 + s) * a.ngroups + g) * N + n0 + k)
                    : 0.f;
            }
            __syncthreads();
#pragma unroll 4
            for (int k = 0; k < KT; ++k) {
                float av[4], bv[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) av[i] = At[k * RT + li * 4 + i];
#pragma unroll
                for (int j = 0; j < 4; ++j) bv[j] = Bt[k * 64 + pi * 4 + j];
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) gacc[i][j] = fmaf(av[i], bv[j], gacc[i][j]);
            }
            __syncthreads();
        }
        // M[l, s] = Re(G[l, s] L[l, s]) dt_s, zero above the diagonal; thread (li, pi)
        // holds rows li*4.. and source tokens pi*4..
#pragma unroll
        for (int i = 0; i < 4; ++i) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int l = l0 + li * 4 + i, s = s0 + pi * 4 + j;
                float m = 0.f;
                if (s <= l && s < valid && l < valid) {
                    const float L = (float)exp(cs_re[l] - cs_re[s]);
                    m = gacc[i][j] * L * dts[s];
                }
                Ms[(pi * 4 + j) * RT + li * 4 + i] = m;
            }
        }
        for (int i = threadIdx.x; i < ST * PT; i += NT) {
            int s = i / PT, p = i % PT;
            Xs[i] = (s0 + s < valid && p0 + p < P)
                        ? ld_f32(xg + (((size_t)b * a.seqlen + t0 + s0 + s) * H + h) * P + p0 + p)
                        : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int s = 0; s < ST; ++s) {
            float mv[4], xv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) mv[i] = Ms[s * RT + li * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) xv[j] = Xs[s * PT + pi * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(mv[i], xv[j], acc[i][j]);
        }
        __syncthreads();
    }

    // Epilogue: + D x, store y.
    TIO *yg = reinterpret_cast<TIO *>(a.y);
    const float Dh = a.D ? a.D[h] : 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int l = li * 4 + i;
        if (l >= rows) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int p = p0 + pi * 4 + j;
            if (p >= P) continue;
            const size_t idx = (((size_t)b * a.seqlen + t0 + l0 + l) * H + h) * P + p;
            float v = acc[i][j];
            if (a.D) v = fmaf(Dh, ld_f32(xg + idx), v);
            st_f32(yg + idx, v);
        }
    }
}

template <typename TIO>
cudaError_t launch_typed(const ScanArgs &a, void *wsp, cudaStream_t st) {
    GenericWs w = carve(wsp, a.batch, a.nheads, a.headdim, a.dstate, a.chunk, a.nchunks, false);
    const int Q = a.chunk, P = a.headdim, N = a.dstate;
    const int PN = P * N;
    const int nsplit = (PN + NT * OPT - 1) / (NT * OPT);

    size_t sm1 = Q * sizeof(double) + Q * sizeof(float) + (Q + SS * (P + N)) * sizeof(float);
    auto k1 = chunk_state_kernel<TIO>;
    cudaError_t e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm1);
    if (e != cudaSuccess) return e;
    dim3 g1(a.nchunks, a.nheads, a.batch * nsplit);
    k1<<<g1, NT, sm1, st>>>(a, w);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    dim3 g2((PN + NT - 1) / NT, a.nheads, a.batch);
    state_pass_kernel<<<g2, NT, 0, st>>>(a, w);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (!a.y) return cudaSuccess;  // final state only

    size_t sm3 = Q * sizeof(double) + Q * sizeof(float) + (KT * RT + KT * 64) * sizeof(float) +
                 (ST * RT + ST * PT) * sizeof(float);
    auto k3 = chunk_scan_kernel<TIO>;
    e = cudaFuncSetAttribute(k3, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm3);
    if (e != cudaSuccess) return e;
    const int nrt = (Q + RT - 1) / RT, npt = (P + PT - 1) / PT;
    dim3 g3(a.nchunks * nrt, a.nheads, a.batch * npt);
    k3<<<g3, NT, sm3, st>>>(a, w);
    return cudaGetLastError();
}

}  // namespace

size_t generic_workspace_bytes(int batch, int nheads, int headdim, int dstate, int chunk,
                               int nchunks, bool cplx) {
    const size_t K = cplx ? 2 : 1;
    const size_t nbhc = (size_t)batch * nheads * nchunks;
    return align_up(nbhc * K * chunk * sizeof(double), 256) + align_up(nbhc * K * sizeof(double), 256) +
           align_up(nbhc * (size_t)headdim * dstate * K * sizeof(float), 256);
}

cudaError_t launch_generic_scan(const ScanArgs &a, bool cplx, bool bf16, void *ws, cudaStream_t st) {
    if (cplx) return launch_complex_scan(a, ws, st);
    if (bf16) return launch_typed<__nv_bfloat16>(a, ws, st);
    return launch_typed<float>(a, ws, st);
}

}  // namespace ssd
