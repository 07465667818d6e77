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
//    the channel ranges allow (K <= 4), a block copies a 256-channel x 32-token
//    tile into shared memory with asynchronous copies and each thread convolves
//    a channel pair from there; otherwise one channel per thread.
//
// 2. The Mamba-1 selective scan, one decay rate per state component:
//      h_t[n] = exp(dt_t[d] A[d][n]) h_{t-1}[n] + dt_t[d] B_t[n] x_t[d],
//      y_t[d] = sum_n C_t[n] h_t[n] + D[d] x_t[d].
//    With a decay per state the segsum decay is no longer one scalar per token
//    pair, so there is no chunked matrix form; the scan is sequential in time
//    and parallel over (batch, channel).  Where 64-channel blocks lie inside one
//    B/C group, two lanes share a channel (N/2 states each) and a block stages
//    x, dt, B and C of 32-token runs in shared memory; otherwise four lanes
//    share a channel and read global memory directly.  Either way the lanes of
//    a channel add their parts of the readout with shuffles.  Bound by the N
//    exponentials per channel and step (SFU), then by HBM.
#include "ssd_internal.cuh"

namespace ssd {
namespace {

template <typename T> __device__ __forceinline__ float ldf(const T *p) { return ld_f32<T>(p); }

// SiLU v / (1 + e^-v).  The exponent is capped at 80 so that the fast divide
// (exact to 2 ulp for divisors below 2^126) always sees a finite divisor; past
// the cap the quotient is below 1e-33 |v|.
__device__ __forceinline__ float silu_f(float v) { return __fdividef(v, 1.f + __expf(fminf(-v, 80.f))); }

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
        if (silu) v = silu_f(v);
        st_f32(dst + (rowb + t) * cn + cc, v);
    }
    if (cfinal && t1 == seqlen)  // the last K-1 inputs, for a continued sequence
        for (int j = 0; j < K - 1; ++j) st_f32(cfinal + ((size_t)b * ctot + c) * (K - 1) + j, win[j + 1]);
}

// Two consecutive channels of T <-> floats.
template <typename T> struct Pair;
template <> struct Pair<float> {
    static __device__ __forceinline__ float2 load(const float *p) { return *reinterpret_cast<const float2 *>(p); }
    static __device__ __forceinline__ void store(float *p, float2 v) { *reinterpret_cast<float2 *>(p) = v; }
};
template <> struct Pair<__nv_bfloat16> {
    static __device__ __forceinline__ float2 load(const __nv_bfloat16 *p) {
        const uint32_t r = *reinterpret_cast<const uint32_t *>(p);
        return make_float2(__uint_as_float(r << 16), __uint_as_float(r & 0xffff0000u));
    }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, float2 v) {
        *reinterpret_cast<__nv_bfloat162 *>(p) = __floats2bfloat162_rn(v.x, v.y);
    }
};

// Packed float32 pairs (sm_100): one instruction does both lanes, each lane
// rounded as the scalar fmaf / multiply would.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    unsigned long long r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;"
        : "=l"(r)
        : "l"(*reinterpret_cast<unsigned long long *>(&a)), "l"(*reinterpret_cast<unsigned long long *>(&b)),
          "l"(*reinterpret_cast<unsigned long long *>(&c)));
    return *reinterpret_cast<float2 *>(&r);
}
__device__ __forceinline__ float2 fmul2v(float2 a, float2 b) {
    unsigned long long r;
    asm("mul.rn.f32x2 %0, %1, %2;"
        : "=l"(r)
        : "l"(*reinterpret_cast<unsigned long long *>(&a)), "l"(*reinterpret_cast<unsigned long long *>(&b)));
    return *reinterpret_cast<float2 *>(&r);
}
// SiLU of a pair for bf16 outputs: v sigmoid(v) = v/2 (1 + tanh(v/2)) with the
// hardware tanh (relative error about 2^-11, below the 2^-9 rounding of the bf16
// result): one exponential-unit operation instead of two; the multiply and the
// fma packed.
__device__ __forceinline__ float2 silu2_bf16out(float2 v) {
    const float2 hv = fmul2v(make_float2(0.5f, 0.5f), v);
    float2 t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t.x) : "f"(hv.x));
    asm("tanh.approx.f32 %0, %1;" : "=f"(t.y) : "f"(hv.y));
    return ffma2(hv, t, hv);
}
template <typename T> __device__ __forceinline__ float2 silu2_out(float2 v);
template <> __device__ __forceinline__ float2 silu2_out<float>(float2 v) {
    return make_float2(silu_f(v.x), silu_f(v.y));
}
template <> __device__ __forceinline__ float2 silu2_out<__nv_bfloat16>(float2 v) { return silu2_bf16out(v); }

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(smem)),
                 "l"(gmem)
                 : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

constexpr int CONV_CH = 256;  // channels per block of the tiled kernel (128 threads x 2)
constexpr int CONV_TV = 32;   // tokens per block of the tiled kernel

// The convolution for a tile of 256 channels x 32 tokens, K <= 4.  The tile's
// input rows (and the three before it) are copied into shared memory with
// asynchronous 16-byte copies, which hold no registers while in flight, so a
// block has its whole tile in flight at once; then each thread convolves its
// channel pair (c0, c0 + 1), both in one of the x, B, C ranges, from shared
// memory.  The kernel is right-aligned into four taps,
// out[t] = bias + sum_{j<4} w4[j] in[t - 3 + j], w4[j] = w[j - (4 - K)] (zero for
// j < 4 - K), so the window always holds the three tokens before t.
template <typename T>
__global__ void __launch_bounds__(128) conv1d_xbc_tile_kernel(const T *__restrict__ in, const float *__restrict__ w,
                                                             const float *__restrict__ bias,
                                                             const T *__restrict__ cinit, T *__restrict__ xo,
                                                             T *__restrict__ bo, T *__restrict__ co,
                                                             T *__restrict__ cfinal, int seqlen, int cx, int cb, int K,
                                                             int silu) {
    using IO = Pair<T>;
    constexpr int E16 = 16 / (int)sizeof(T);  // elements per 16-byte copy
    __shared__ __align__(16) T tile[(CONV_TV + 3) * CONV_CH];
    const int ctot = cx + 2 * cb;
    const int cbase = blockIdx.x * CONV_CH, t0 = blockIdx.y * CONV_TV, b = blockIdx.z;
    const int nch = min(CONV_CH, ctot - cbase), n = min(CONV_TV, seqlen - t0);
    const size_t rowb = (size_t)b * seqlen;
    // rows r = 0 .. n + 2 hold tokens t0 - 3 + r; rows before the sequence are
    // filled per thread below
    const int cpr = nch / E16, r0 = t0 >= 3 ? 0 : 3 - t0;
    for (int u = threadIdx.x; u < (n + 3 - r0) * cpr; u += 128) {
        const int r = r0 + u / cpr, k = u % cpr;
        cp_async16(tile + r * CONV_CH + k * E16, in + (rowb + t0 - 3 + r) * ctot + cbase + k * E16);
    }
    const int c0 = cbase + 2 * threadIdx.x;
    float2 wk[4], bc = make_float2(0.f, 0.f);
    if (c0 < ctot) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int k = j - (4 - K);
            wk[j] = k >= 0 ? make_float2(w[(size_t)c0 * K + k], w[(size_t)(c0 + 1) * K + k]) : make_float2(0.f, 0.f);
        }
        if (bias) bc = make_float2(bias[c0], bias[c0 + 1]);
    }
    cp_async_wait_all();
    __syncthreads();
    if (c0 >= ctot) return;
    const T *col = tile + 2 * threadIdx.x;
    float2 win[3];
#pragma unroll
    for (int j = 0; j < 3; ++j) {  // win[j] = in[t0 - 3 + j]: the sequence, conv_init or zero
        const int s = t0 - 3 + j;
        if (s >= 0) {
            win[j] = IO::load(col + j * CONV_CH);
        } else if (cinit && K - 1 + s >= 0) {
            const T *ci = cinit + ((size_t)b * ctot + c0) * (K - 1) + (K - 1) + s;
            win[j] = make_float2(ldf(ci), ldf(ci + (K - 1)));
        } else {
            win[j] = make_float2(0.f, 0.f);
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
    T *pd = dst + (rowb + t0) * cn + cc;
#pragma unroll 4
    for (int i = 0; i < n; ++i) {
        const float2 cur = IO::load(col + (i + 3) * CONV_CH);
        float2 v = ffma2(wk[3], cur, ffma2(wk[2], win[2], ffma2(wk[1], win[1], ffma2(wk[0], win[0], bc))));
        if (silu) v = silu2_out<T>(v);
        IO::store(pd, v);
        pd += cn;
        win[0] = win[1], win[1] = win[2], win[2] = cur;
    }
    if (cfinal && t0 + n == seqlen)  // the last K-1 inputs, for a continued sequence
        for (int j = 0; j < K - 1; ++j) {
            const float2 v = win[3 - (K - 1) + j];
            st_f32(cfinal + ((size_t)b * ctot + c0) * (K - 1) + j, v.x);
            st_f32(cfinal + ((size_t)b * ctot + c0 + 1) * (K - 1) + j, v.y);
        }
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

constexpr int SEL_TT = 32;  // tokens per staged run
constexpr int SEL_CH = 64;  // channels per block (two lanes each)

// The selective scan for blocks of 64 channels that lie in one B/C group.  Two
// lanes share a channel, each with N/2 of its states in registers.  Runs of 32
// tokens (16 for float32 inputs with 32 states) of x, dt (64 channels) and B, C (the group's N states) are copied into
// shared memory as they are stored, with asynchronous 16-byte copies, double
// buffered: run r+1's copies are in flight while run r is computed, so no load
// latency sits between runs.  The recurrence reads B and C with vector shared
// loads (no address arithmetic in global memory), works on pairs of states with
// packed float32 instructions, and each run's y goes back as coalesced rows.
// Needs 16-byte aligned x, dt, B, C rows (checked by the launcher).
template <typename T> __device__ __forceinline__ void unpack8(const T *p, float (&v)[8]);
template <> __device__ __forceinline__ void unpack8<float>(const float *p, float (&v)[8]) {
    const float4 a = *reinterpret_cast<const float4 *>(p), b = *reinterpret_cast<const float4 *>(p + 4);
    v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w, v[4] = b.x, v[5] = b.y, v[6] = b.z, v[7] = b.w;
}
template <> __device__ __forceinline__ void unpack8<__nv_bfloat16>(const __nv_bfloat16 *p, float (&v)[8]) {
    const uint4 q = *reinterpret_cast<const uint4 *>(p);
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}
template <typename T> __device__ __forceinline__ float smem_f(const T *p) { return ld_f32<T>(p); }

template <typename T, int N>
__global__ void __launch_bounds__(128) selective_scan_tile_kernel(const T *__restrict__ x, const float *__restrict__ dt,
                                                                 const float *__restrict__ A, const T *__restrict__ B,
                                                                 const T *__restrict__ C, const float *__restrict__ D,
                                                                 const float *__restrict__ h0, float *__restrict__ hT,
                                                                 T *__restrict__ y, int seqlen, int channels,
                                                                 int ngroups) {
    constexpr int NH = N / 2;
    static_assert(NH % 8 == 0 || NH == 4, "states per lane read as 16-byte vectors");
    constexpr int XE = 16 / (int)sizeof(T);  // elements of x, B, C per 16-byte copy
    // tokens per run: 32, or 16 where two runs of float32 x, B and C with 32 states
    // would not fit in 48 KB of static shared memory
    constexpr int TT = (sizeof(T) == 4 && N >= 32) ? SEL_TT / 2 : SEL_TT;
    __shared__ __align__(16) T xs[2][TT][SEL_CH];
    __shared__ __align__(16) float ds[2][TT][SEL_CH];
    __shared__ __align__(16) T bs[2][TT][N], cs[2][TT][N];
    __shared__ float ys[TT][SEL_CH];
    const int tid = threadIdx.x, ch = tid >> 1, half = tid & 1;
    const int cbase = blockIdx.x * SEL_CH, b = blockIdx.y, d = cbase + ch;
    const int g = cbase / (channels / ngroups), n0 = half * NH;
    // Run r's copies into buffer r % 2 (rows past the sequence are not copied).
    auto copy_run = [&](int r) {
        const int t0 = r * TT, nt = min(TT, seqlen - t0), buf = r & 1;
        const size_t row0 = (size_t)b * seqlen + t0;
        for (int u = tid; u < nt * (SEL_CH / XE); u += 128) {
            const int i = u / (SEL_CH / XE), k = u % (SEL_CH / XE);
            cp_async16(&xs[buf][i][k * XE], x + (row0 + i) * channels + cbase + k * XE);
        }
        for (int u = tid; u < nt * (SEL_CH / 4); u += 128) {
            const int i = u / (SEL_CH / 4), k = u % (SEL_CH / 4);
            cp_async16(&ds[buf][i][k * 4], dt + (row0 + i) * channels + cbase + k * 4);
        }
        for (int u = tid; u < nt * (N / XE); u += 128) {
            const int i = u / (N / XE), k = u % (N / XE);
            const size_t o = ((row0 + i) * ngroups + g) * N + k * XE;
            cp_async16(&bs[buf][i][k * XE], B + o);
            cp_async16(&cs[buf][i][k * XE], C + o);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    const int nruns = (seqlen + TT - 1) / TT;
    if (nruns > 0) copy_run(0);
    float2 a2[NH / 2], h[NH / 2];
#pragma unroll
    for (int n = 0; n < NH / 2; ++n) {
        const size_t o = (size_t)d * N + n0 + 2 * n;
        a2[n] = make_float2(A[o] * 1.4426950408889634f, A[o + 1] * 1.4426950408889634f);
        const size_t oh = ((size_t)b * channels + d) * N + n0 + 2 * n;
        h[n] = h0 ? make_float2(h0[oh], h0[oh + 1]) : make_float2(0.f, 0.f);
    }
    const float Dd = D ? D[d] : 0.f;
    for (int r = 0; r < nruns; ++r) {
        const int t0 = r * TT, nt = min(TT, seqlen - t0), buf = r & 1;
        if (r + 1 < nruns) {
            copy_run(r + 1);  // into the buffer run r-1 used: its reads ended at the last barrier
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncthreads();  // run r's copies from every thread have landed
#pragma unroll 2
        for (int i = 0; i < nt; ++i) {
            const float xt = smem_f(&xs[buf][i][ch]), st = ds[buf][i][ch], u = st * xt;
            float bv[NH], cv[NH];
#pragma unroll
            for (int n = 0; n < NH; n += 8 < NH ? 8 : NH) {
                if constexpr (NH >= 8) {
                    float tb[8], tc[8];
                    unpack8<T>(&bs[buf][i][n0 + n], tb);
                    unpack8<T>(&cs[buf][i][n0 + n], tc);
#pragma unroll
                    for (int e = 0; e < 8; ++e) bv[n + e] = tb[e], cv[n + e] = tc[e];
                } else {
#pragma unroll
                    for (int e = 0; e < NH; ++e) bv[e] = smem_f(&bs[buf][i][n0 + e]), cv[e] = smem_f(&cs[buf][i][n0 + e]);
                }
            }
            const float2 st2 = make_float2(st, st), u2 = make_float2(u, u);
            float2 acc = make_float2(0.f, 0.f);
#pragma unroll
            for (int n = 0; n < NH / 2; ++n) {
                const float2 arg = fmul2v(st2, a2[n]);
                const float2 e = make_float2(ex2_approx(arg.x), ex2_approx(arg.y));
                h[n] = ffma2(e, h[n], fmul2v(u2, make_float2(bv[2 * n], bv[2 * n + 1])));
                acc = ffma2(make_float2(cv[2 * n], cv[2 * n + 1]), h[n], acc);
            }
            float accs = acc.x + acc.y;
            accs += __shfl_xor_sync(0xffffffffu, accs, 1);
            if (half == 0) ys[i][ch] = fmaf(Dd, xt, accs);
        }
        __syncthreads();  // ys complete; buffer buf is free for run r+2
        const size_t row0 = (size_t)b * seqlen + t0;
        for (int u = tid; u < nt * SEL_CH; u += 128) {
            const int i = u / SEL_CH, c = u % SEL_CH;
            st_f32(y + (row0 + i) * channels + cbase + c, ys[i][c]);
        }
    }
    if (hT)
#pragma unroll
        for (int n = 0; n < NH / 2; ++n) {
            const size_t oh = ((size_t)b * channels + d) * N + n0 + 2 * n;
            hT[oh] = h[n].x;
            hT[oh + 1] = h[n].y;
        }
}

template <typename T, int N>
cudaError_t launch_sel(const void *x, const float *dt, const float *A, const void *B, const void *C, const float *D,
                       const float *h0, float *hT, void *y, int batch, int seqlen, int channels, int ngroups,
                       cudaStream_t st) {
    // The four-lane form reads each lane's N/4 states of B and C as one vector:
    // aligned when B and C are (the API asks for 16 bytes) and N/4 elements per lane.
    if constexpr (N >= 8) {  // two lanes of N/2 >= 4 states (whole 16-byte reads)
        const bool aligned = ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(dt) |
                               reinterpret_cast<uintptr_t>(B) | reinterpret_cast<uintptr_t>(C)) & 15) == 0 &&
                             ((size_t)channels * sizeof(T)) % 16 == 0 && channels % 4 == 0 &&
                             ((size_t)N * sizeof(T)) % 16 == 0;
        if ((channels / ngroups) % SEL_CH == 0 && aligned) {  // every block inside one group
            dim3 grid(channels / SEL_CH, batch);
            selective_scan_tile_kernel<T, N><<<grid, 128, 0, st>>>(
                static_cast<const T *>(x), dt, A, static_cast<const T *>(B), static_cast<const T *>(C), D, h0, hT,
                static_cast<T *>(y), seqlen, channels, ngroups);
            return cudaGetLastError();
        }
    }
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
    // The tiled kernel when no channel pair straddles the x / B / C ranges, every
    // token row is a whole number of 16-byte copies (the API asks for 16-byte
    // aligned pointers) and K <= 4.
    const int e16 = bf16 ? 8 : 4;
    if (width <= 4 && cx % 2 == 0 && cb % 2 == 0 && ctot % e16 == 0) {
        dim3 grid((ctot + CONV_CH - 1) / CONV_CH, (seqlen + CONV_TV - 1) / CONV_TV, batch);
        if (bf16) {
            using T = __nv_bfloat16;
            conv1d_xbc_tile_kernel<T><<<grid, 128, 0, st>>>(
                static_cast<const T *>(in), w, bias, static_cast<const T *>(cinit), static_cast<T *>(xo),
                static_cast<T *>(bo), static_cast<T *>(co), static_cast<T *>(cfinal), seqlen, cx, cb, width, silu);
        } else {
            conv1d_xbc_tile_kernel<float><<<grid, 128, 0, st>>>(
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
