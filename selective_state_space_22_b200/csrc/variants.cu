// variants.cu -- the two variants the pages name beside the Mamba-2 /
// Mamba-3-Lite scan ("Block Anatomy, Numerical Stability & Scaling", Block
// Anatomy sections 4.4 and 5.1; the "Mamba-50M" card).
//
// 1. The causal depthwise convolution that Mamba-1 and Mamba-2 run on the
//    projected input before the scan (kernel width K = 4):
//      out[t][c] = act(bias[c] + sum_k w[c][k] in[t - (K-1) + k][c]),
//    over the packed x | B | C channels of a Mamba-2 projection, written straight
//    into the scan's separate x, B and C tensors.  One thread per channel slides
//    a K-token window along a run of TT tokens, so each input is read once (plus
//    a K-1 token halo per run) and each output written once: HBM-bound.
//
// 2. The Mamba-1 selective scan, one decay rate per state component:
//      h_t[n] = exp(dt_t[d] A[d][n]) h_{t-1}[n] + dt_t[d] B_t[n] x_t[d],
//      y_t[d] = sum_n C_t[n] h_t[n] + D[d] x_t[d].
//    With a decay per state the segsum decay is no longer one scalar per token
//    pair, so there is no chunked matrix form; the scan is sequential in time
//    and parallel over (batch, channel).  One lane owns one channel and its N
//    states in registers: a warp reads 32 consecutive channels' x and dt as
//    one line per step, B and C of the step are one broadcast line each.  Bound
//    by the N exponentials per channel and step (SFU), then by HBM.
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

template <typename T, int N>
__global__ void __launch_bounds__(128) selective_scan_kernel(const T *__restrict__ x, const float *__restrict__ dt,
                                                            const float *__restrict__ A, const T *__restrict__ B,
                                                            const T *__restrict__ C, const float *__restrict__ D,
                                                            const float *__restrict__ h0, float *__restrict__ hT,
                                                            T *__restrict__ y, int seqlen, int channels,
                                                            int ngroups) {
    const int d = blockIdx.x * 128 + threadIdx.x, b = blockIdx.y;
    if (d >= channels) return;
    const int g = d / (channels / ngroups);
    float a[N], h[N];
#pragma unroll
    for (int n = 0; n < N; ++n) {
        a[n] = A[(size_t)d * N + n];
        h[n] = h0 ? h0[((size_t)b * channels + d) * N + n] : 0.f;
    }
    const float Dd = D ? D[d] : 0.f;
    size_t row = (size_t)b * seqlen;
    // one step of look-ahead on the per-token loads
    float xn = seqlen > 0 ? ldf(x + row * channels + d) : 0.f;
    float dn = seqlen > 0 ? dt[row * channels + d] : 0.f;
    for (int t = 0; t < seqlen; ++t, ++row) {
        const float xt = xn, st = dn;
        if (t + 1 < seqlen) {
            xn = ldf(x + (row + 1) * channels + d);
            dn = dt[(row + 1) * channels + d];
        }
        const T *Bt = B + (row * ngroups + g) * N;
        const T *Ct = C + (row * ngroups + g) * N;
        const float u = st * xt;
        float acc = 0.f;
#pragma unroll
        for (int n = 0; n < N; ++n) {
            h[n] = fmaf(__expf(st * a[n]), h[n], u * ldf(Bt + n));
            acc = fmaf(ldf(Ct + n), h[n], acc);
        }
        st_f32(y + row * channels + d, fmaf(Dd, xt, acc));
    }
    if (hT)
#pragma unroll
        for (int n = 0; n < N; ++n) hT[((size_t)b * channels + d) * N + n] = h[n];
}

template <typename T, int N>
cudaError_t launch_sel(const void *x, const float *dt, const float *A, const void *B, const void *C, const float *D,
                       const float *h0, float *hT, void *y, int batch, int seqlen, int channels, int ngroups,
                       cudaStream_t st) {
    dim3 grid((channels + 127) / 128, batch);
    selective_scan_kernel<T, N><<<grid, 128, 0, st>>>(static_cast<const T *>(x), dt, A, static_cast<const T *>(B),
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
