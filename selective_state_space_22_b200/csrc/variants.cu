// variants.cu -- the two variants the pages name beside the Mamba-2 /
// Mamba-3-Lite scan ("Block Anatomy, Numerical Stability & Scaling", Block
// Anatomy sections 4.4 and 5.1; the "Mamba-50M" card).
//
// 1. The causal depthwise convolution that Mamba-1 and Mamba-2 run on the
//    projected input before the scan (kernel width K = 4):
//      out[t][c] = act(bias[c] + sum_k w[c][k] in[t - (K-1) + k][c]),
//    over the packed x | B | C channels of a Mamba-2 projection, written straight
//    into the scan's separate x, B and C tensors.  A thread slides a K-token
//    window along a run of tokens, so each input is read once (plus a K-1 token
//    halo per run, an L2 hit) and each output written once: HBM-bound.  Where
//    the channel ranges and pointers allow (K <= 4), a thread owns 16 bytes of
//    channels (8 bf16 or 4 float32) and moves them with one load and one store
//    per token; otherwise one channel per thread.
//
// 2. The Mamba-1 selective scan, one decay rate per state component:
//      h_t[n] = exp(dt_t[d] A[d][n]) h_{t-1}[n] + dt_t[d] B_t[n] x_t[d],
//      y_t[d] = sum_n C_t[n] h_t[n] + D[d] x_t[d].
//    With a decay per state the segsum decay is no longer one scalar per token
//    pair, so there is no chunked matrix form; the scan is sequential in time
//    and parallel over (batch, channel).  Four lanes share a channel, each with
//    N/4 of its states in registers, and add their parts of the readout with
//    two shuffles; a warp covers 8 consecutive channels, and B and C of a step
//    are one vector load per lane (the same for all channels of a group).
//    Bound by the N exponentials per channel and step (SFU), then by HBM.
#include "ssd_internal.cuh"

namespace ssd {
namespace {

template <typename T> __device__ __forceinline__ float ldf(const T *p) { return ld_f32<T>(p); }

constexpr int CONV_TT = 32;   // tokens per thread run
constexpr int CONV_MAXK = 8;

template <typename T>
__global__ void __launch_bounds__(128) conv1d_xbc_kernel(const T *__restrict__ in, const float *__restrict__ w,
                                                        const float *__restrict__ bias, const T *__restrict__ cinit,
                                                        T *__restrict__ xo, T *__restrict__ bo, T *__restrict__ co,
                                                        T *__restrict__ cfinal, int seqlen, int cx, int cb, int K,
                                                        int silu) {
    const int ctot = cx + 2 * cb;
    const int c = blockIdx.x * 128 + threadIdx.x;
    const int t0 = blockIdx.y * CONV_TT, b = blockIdx.z;
    if (c >= ctot || t0 >= seqlen) return;
    float wk[CONV_MAXK], win[CONV_MAXK];
#pragma unroll
    for (int k = 0; k < CONV_MAXK; ++k) {
        wk[k] = k < K ? w[(size_t)c * K + k] : 0.f;
        win[k] = 0.f;
    }
    const float bc = bias ? bias[c] : 0.f;
    // window: win[K-1-j] holds in[t - j]; prime it with tokens t0-K+1 .. t0-1
    const size_t rowb = (size_t)b * seqlen;
    for (int j = K - 1; j >= 1; --j) {
        const int s = t0 - j;
        float v = 0.f;
        if (s >= 0)
            v = ldf(in + (rowb + s) * ctot + c);
        else if (cinit)
            v = ldf(cinit + ((size_t)b * ctot + c) * (K - 1) + (K - 1) + s);
#pragma unroll
        for (int k = 0; k < CONV_MAXK - 1; ++k) win[k] = win[k + 1];
        win[K - 1] = v;
    }
    T *dst;
    int cc, cn;
    if (c < cx) {
        dst = xo, cc = c, cn = cx;
    } else if (c < cx + cb) {
        dst = bo, cc = c - cx, cn = cb;
    } else {
        dst = co, cc = c - cx - cb, cn = cb;
    }
    const int t1 = min(t0 + CONV_TT, seqlen);
    for (int t = t0; t < t1; ++t) {
#pragma unroll
        for (int k = 0; k < CONV_MAXK - 1; ++k) win[k] = win[k + 1];
        win[K - 1] = ldf(in + (rowb + t) * ctot + c);
        // shifting left by one each step keeps in[t - (K-1) + k] at win[k]
        float v = bc;
#pragma unroll
        for (int k = 0; k < CONV_MAXK; ++k)
            if (k < K) v = fmaf(wk[k], win[k], v);
        if (silu) v = v / (1.f + __expf(-v));
        st_f32(dst + (rowb + t) * cn + cc, v);
    }
    if (cfinal && t1 == seqlen)  // the last K-1 inputs, for a continued sequence
        for (int j = 0; j < K - 1; ++j) st_f32(cfinal + ((size_t)b * ctot + c) * (K - 1) + j, win[j + 1]);
}

// 16 bytes of T <-> floats.
template <typename T> struct Vec16;
template <> struct Vec16<float> {
    static constexpr int V = 4;
    static __device__ __forceinline__ void load(const float *p, float (&v)[4]) {
        const float4 q = *reinterpret_cast<const float4 *>(p);
        v[0] = q.x, v[1] = q.y, v[2] = q.z, v[3] = q.w;
    }
    static __device__ __forceinline__ void store(float *p, const float (&v)[4]) {
        *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
    }
};
template <> struct Vec16<__nv_bfloat16> {
    static constexpr int V = 8;
    static __device__ __forceinline__ void load(const __nv_bfloat16 *p, float (&v)[8]) {
        const uint4 q = *reinterpret_cast<const uint4 *>(p);
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            v[2 * e] = __uint_as_float(w[e] << 16);
            v[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
        }
    }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, const float (&v)[8]) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
            w[e] = *reinterpret_cast<const uint32_t *>(&h);
        }
        *reinterpret_cast<uint4 *>(p) = make_uint4(w[0], w[1], w[2], w[3]);
    }
};

constexpr int CONV_TV = 16;  // tokens per thread run (vector kernel)

// The convolution with one thread per 16 bytes of channels c0 .. c0+V-1 (all in
// one of the x, B, C ranges), K <= 4: the kernel is right-aligned into four taps,
// out[t] = bias + sum_{j<4} w4[j] in[t - 3 + j] with w4[j] = w[j - (4 - K)] (zero
// for j < 4 - K), so the window always holds the three tokens before t.
template <typename T>
__global__ void __launch_bounds__(128) conv1d_xbc_vec_kernel(const T *__restrict__ in, const float *__restrict__ w,
                                                            const float *__restrict__ bias,
                                                            const T *__restrict__ cinit, T *__restrict__ xo,
                                                            T *__restrict__ bo, T *__restrict__ co,
                                                            T *__restrict__ cfinal, int seqlen, int cx, int cb, int K,
                                                            int silu) {
    using IO = Vec16<T>;
    constexpr int V = IO::V;
    const int ctot = cx + 2 * cb;
    const int c0 = (blockIdx.x * 128 + threadIdx.x) * V;
    const int t0 = blockIdx.y * CONV_TV, b = blockIdx.z;
    if (c0 >= ctot || t0 >= seqlen) return;
    float wk[4][V], bc[V], win[3][V];
#pragma unroll
    for (int e = 0; e < V; ++e) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int k = j - (4 - K);
            wk[j][e] = k >= 0 ? w[(size_t)(c0 + e) * K + k] : 0.f;
        }
        bc[e] = bias ? bias[c0 + e] : 0.f;
    }
    const size_t rowb = (size_t)b * seqlen;
#pragma unroll
    for (int j = 0; j < 3; ++j) {  // win[j] = in[t0 - 3 + j]: the sequence, conv_init or zero
        const int s = t0 - 3 + j;
        if (s >= 0) {
            IO::load(in + (rowb + s) * ctot + c0, win[j]);
        } else {
#pragma unroll
            for (int e = 0; e < V; ++e)
                win[j][e] = (cinit && K - 1 + s >= 0) ? ldf(cinit + ((size_t)b * ctot + c0 + e) * (K - 1) + (K - 1) + s)
                                                      : 0.f;
        }
    }
    T *dst;
    int cc, cn;
    if (c0 < cx) {
        dst = xo, cc = c0, cn = cx;
    } else if (c0 < cx + cb) {
        dst = bo, cc = c0 - cx, cn = cb;
    } else {
        dst = co, cc = c0 - cx - cb, cn = cb;
    }
    const int t1 = min(t0 + CONV_TV, seqlen);
#pragma unroll
    for (int q = 0; q < CONV_TV; q += 4) {  // four tokens' loads in flight at a time
        float cur[4][V];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (t0 + q + i < t1) IO::load(in + (rowb + t0 + q + i) * ctot + c0, cur[i]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int t = t0 + q + i;
            if (t < t1) {
                float out[V];
#pragma unroll
                for (int e = 0; e < V; ++e) {
                    float v = fmaf(wk[0][e], win[0][e], bc[e]);
                    v = fmaf(wk[1][e], win[1][e], v);
                    v = fmaf(wk[2][e], win[2][e], v);
                    v = fmaf(wk[3][e], cur[i][e], v);
                    out[e] = silu ? v / (1.f + __expf(-v)) : v;
                    win[0][e] = win[1][e], win[1][e] = win[2][e], win[2][e] = cur[i][e];
                }
                IO::store(dst + (rowb + t) * cn + cc, out);
            }
        }
    }
    if (cfinal && t1 == seqlen)  // the last K-1 inputs, for a continued sequence
        for (int j = 0; j < K - 1; ++j)
#pragma unroll
            for (int e = 0; e < V; ++e)
                st_f32(cfinal + ((size_t)b * ctot + c0 + e) * (K - 1) + j, win[3 - (K - 1) + j][e]);
}

// Four lanes per channel: lane 4i + q of a warp holds states q*N/4 .. of channel
// 8w + i.  The exponent uses A pre-scaled by log2(e), so each state's decay is one
// multiply and one ex2.approx.
__device__ __forceinline__ float ex2_approx(float v) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
    return r;
}
template <typename T, int NQ> struct QLoad;  // NQ consecutive T -> floats
template <> struct QLoad<float, 1> {
    static __device__ __forceinline__ void load(const float *p, float (&v)[1]) { v[0] = *p; }
};
template <> struct QLoad<float, 2> {
    static __device__ __forceinline__ void load(const float *p, float (&v)[2]) {
        const float2 q = *reinterpret_cast<const float2 *>(p);
        v[0] = q.x, v[1] = q.y;
    }
};
template <int NQ> struct QLoadF {
    static __device__ __forceinline__ void load(const float *p, float (&v)[NQ]) {
#pragma unroll
        for (int i = 0; i < NQ; i += 4) {
            const float4 q = *reinterpret_cast<const float4 *>(p + i);
            v[i] = q.x, v[i + 1] = q.y, v[i + 2] = q.z, v[i + 3] = q.w;
        }
    }
};
template <> struct QLoad<float, 4> : QLoadF<4> {};
template <> struct QLoad<float, 8> : QLoadF<8> {};
template <> struct QLoad<__nv_bfloat16, 1> {
    static __device__ __forceinline__ void load(const __nv_bfloat16 *p, float (&v)[1]) { v[0] = __bfloat162float(*p); }
};
template <> struct QLoad<__nv_bfloat16, 2> {
    static __device__ __forceinline__ void load(const __nv_bfloat16 *p, float (&v)[2]) {
        const uint32_t q = *reinterpret_cast<const uint32_t *>(p);
        v[0] = __uint_as_float(q << 16), v[1] = __uint_as_float(q & 0xffff0000u);
    }
};
template <int NQ> struct QLoadB {
    static __device__ __forceinline__ void load(const __nv_bfloat16 *p, float (&v)[NQ]) {
#pragma unroll
        for (int i = 0; i < NQ; i += 4) {
            const uint2 q = *reinterpret_cast<const uint2 *>(p + i);
            v[i] = __uint_as_float(q.x << 16), v[i + 1] = __uint_as_float(q.x & 0xffff0000u);
            v[i + 2] = __uint_as_float(q.y << 16), v[i + 3] = __uint_as_float(q.y & 0xffff0000u);
        }
    }
};
template <> struct QLoad<__nv_bfloat16, 4> : QLoadB<4> {};
template <> struct QLoad<__nv_bfloat16, 8> : QLoadB<8> {};

template <typename T, int N>
__global__ void __launch_bounds__(128) selective_scan_q4_kernel(const T *__restrict__ x, const float *__restrict__ dt,
                                                               const float *__restrict__ A, const T *__restrict__ B,
                                                               const T *__restrict__ C, const float *__restrict__ D,
                                                               const float *__restrict__ h0, float *__restrict__ hT,
                                                               T *__restrict__ y, int seqlen, int channels,
                                                               int ngroups) {
    constexpr int NQ = N / 4;
    const int q = threadIdx.x & 3;
    const int d = blockIdx.x * 32 + (threadIdx.x >> 2), b = blockIdx.y;
    const bool live = d < channels;
    const int dc = live ? d : channels - 1;  // lanes past the end run a copy of the last channel, stores off
    const int g = dc / (channels / ngroups), n0 = q * NQ;
    float a2[NQ], h[NQ];
#pragma unroll
    for (int n = 0; n < NQ; ++n) {
        a2[n] = A[(size_t)dc * N + n0 + n] * 1.4426950408889634f;
        h[n] = h0 ? h0[((size_t)b * channels + dc) * N + n0 + n] : 0.f;
    }
    const float Dd = D ? D[dc] : 0.f;
    size_t row = (size_t)b * seqlen;
    // one step of look-ahead on every per-token load
    float xn = 0.f, dn = 0.f, bn[NQ], cn[NQ];
    if (seqlen > 0) {
        xn = ldf(x + row * channels + dc);
        dn = dt[row * channels + dc];
        QLoad<T, NQ>::load(B + (row * ngroups + g) * N + n0, bn);
        QLoad<T, NQ>::load(C + (row * ngroups + g) * N + n0, cn);
    }
    for (int t = 0; t < seqlen; ++t, ++row) {
        const float xt = xn, st = dn;
        float bt[NQ], ct[NQ];
#pragma unroll
        for (int n = 0; n < NQ; ++n) bt[n] = bn[n], ct[n] = cn[n];
        if (t + 1 < seqlen) {
            xn = ldf(x + (row + 1) * channels + dc);
            dn = dt[(row + 1) * channels + dc];
            QLoad<T, NQ>::load(B + ((row + 1) * ngroups + g) * N + n0, bn);
            QLoad<T, NQ>::load(C + ((row + 1) * ngroups + g) * N + n0, cn);
        }
        const float u = st * xt;
        float acc = 0.f;
#pragma unroll
        for (int n = 0; n < NQ; ++n) {
            h[n] = fmaf(ex2_approx(st * a2[n]), h[n], u * bt[n]);
            acc = fmaf(ct[n], h[n], acc);
        }
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        if (live && q == 0) st_f32(y + row * channels + d, fmaf(Dd, xt, acc));
    }
    if (hT && live)
#pragma unroll
        for (int n = 0; n < NQ; ++n) hT[((size_t)b * channels + d) * N + n0 + n] = h[n];
}

template <typename T, int N>
cudaError_t launch_sel(const void *x, const float *dt, const float *A, const void *B, const void *C, const float *D,
                       const float *h0, float *hT, void *y, int batch, int seqlen, int channels, int ngroups,
                       cudaStream_t st) {
    // The four-lane form reads each lane's N/4 states of B and C as one vector:
    // aligned when B and C are (the API asks for 16 bytes) and N/4 elements per lane.
    dim3 grid((channels + 31) / 32, batch);
    selective_scan_q4_kernel<T, N><<<grid, 128, 0, st>>>(static_cast<const T *>(x), dt, A, static_cast<const T *>(B),
                                                         static_cast<const T *>(C), D, h0, hT, static_cast<T *>(y),
                                                         seqlen, channels, ngroups);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_sel_n(const void *x, const float *dt, const float *A, const void *B, const void *C, const float *D,
                         const float *h0, float *hT, void *y, int batch, int seqlen, int channels, int ngroups,
                         int dstate, cudaStream_t st) {
    switch (dstate) {
    case 4: return launch_sel<T, 4>(x, dt, A, B, C, D, h0, hT, y, batch, seqlen, channels, ngroups, st);
    case 8: return launch_sel<T, 8>(x, dt, A, B, C, D, h0, hT, y, batch, seqlen, channels, ngroups, st);
    case 16: return launch_sel<T, 16>(x, dt, A, B, C, D, h0, hT, y, batch, seqlen, channels, ngroups, st);
    case 32: return launch_sel<T, 32>(x, dt, A, B, C, D, h0, hT, y, batch, seqlen, channels, ngroups, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace

bool selective_dstate_supported(int dstate) { return dstate == 4 || dstate == 8 || dstate == 16 || dstate == 32; }

cudaError_t launch_selective_scan(const void *x, const float *dt, const float *A, const void *B, const void *C,
                                  const float *D, const float *init_state, float *final_state, void *y, bool bf16,
                                  int batch, int seqlen, int channels, int ngroups, int dstate, cudaStream_t st) {
    if (bf16)
        return launch_sel_n<__nv_bfloat16>(x, dt, A, B, C, D, init_state, final_state, y, batch, seqlen, channels,
                                           ngroups, dstate, st);
    return launch_sel_n<float>(x, dt, A, B, C, D, init_state, final_state, y, batch, seqlen, channels, ngroups, dstate,
                               st);
}

cudaError_t launch_conv1d_xbc(const void *in, const float *w, const float *bias, const void *cinit, void *xo,
                              void *bo, void *co, void *cfinal, bool bf16, int batch, int seqlen, int cx, int cb,
                              int width, int silu, cudaStream_t st) {
    const int ctot = cx + 2 * cb;
    // 16-byte channel groups when no group straddles the x / B / C ranges and
    // every row and output base is 16-byte aligned (K <= 4).
    const int V = bf16 ? 8 : 4;
    auto al = [](const void *p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
    if (width <= 4 && cx % V == 0 && cb % V == 0 && al(in) && al(xo) && al(bo) && al(co)) {
        dim3 grid((ctot / V + 127) / 128, (seqlen + CONV_TV - 1) / CONV_TV, batch);
        if (bf16) {
            using T = __nv_bfloat16;
            conv1d_xbc_vec_kernel<T><<<grid, 128, 0, st>>>(
                static_cast<const T *>(in), w, bias, static_cast<const T *>(cinit), static_cast<T *>(xo),
                static_cast<T *>(bo), static_cast<T *>(co), static_cast<T *>(cfinal), seqlen, cx, cb, width, silu);
        } else {
            conv1d_xbc_vec_kernel<float><<<grid, 128, 0, st>>>(
                static_cast<const float *>(in), w, bias, static_cast<const float *>(cinit), static_cast<float *>(xo),
                static_cast<float *>(bo), static_cast<float *>(co), static_cast<float *>(cfinal), seqlen, cx, cb,
                width, silu);
        }
        return cudaGetLastError();
    }
    dim3 grid((ctot + 127) / 128, (seqlen + CONV_TT - 1) / CONV_TT, batch);
    if (bf16) {
        using T = __nv_bfloat16;
        conv1d_xbc_kernel<T><<<grid, 128, 0, st>>>(static_cast<const T *>(in), w, bias, static_cast<const T *>(cinit),
                                                    static_cast<T *>(xo), static_cast<T *>(bo), static_cast<T *>(co),
                                                    static_cast<T *>(cfinal), seqlen, cx, cb, width, silu);
    } else {
        conv1d_xbc_kernel<float><<<grid, 128, 0, st>>>(static_cast<const float *>(in), w, bias,
                                                        static_cast<const float *>(cinit), static_cast<float *>(xo),
                                                        static_cast<float *>(bo), static_cast<float *>(co),
                                                        static_cast<float *>(cfinal), seqlen, cx, cb, width, silu);
    }
    return cudaGetLastError();
}

}  // namespace ssd
