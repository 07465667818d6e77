// cplx_view.cuh -- how the complex scans read x, B, C and dt: strided views, so
// that the same kernels take the separate tensors of ssd_scan_fwd_complex or the
// packed projection output of ssd_scan_fwd_complex_packed.
//
// "Block Anatomy, Numerical Stability & Scaling", Block Anatomy section 4.1-4.3:
// the input projection of a Mamba-3-Lite block emits, per token, H(D + 4N + 1)
// values in head-major slices -- x (H*D), Re B, Im B, Re C, Im C (H*N each) and
// dt (H) -- and the block widens them to float32 and pairs the real and
// imaginary slices into complex64 B and C before the scan; Numerical Stability
// section 4 (_discretise) applies softplus to dt.  Read through a view, the scan
// does that unpacking in its own loads: no separate pass over HBM.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "ssd_internal.cuh"

namespace ssd {

template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

// Element (b, t, ...) of a view lives at base + (b * seqlen + t) * token_stride + ...
template <typename T> struct CplxView {
    const T *x;                  // x[b,t,h,p]   at bt * x_ts + h * P + p
    const T *bre, *bim;          // B[b,t,g,n]   at bt * bc_ts + g * bc_gs + n * bc_es (real, imaginary)
    const T *cre, *cim;          // C[b,t,g,n]   likewise
    const T *dt;                 // dt[b,t,h]    at bt * dt_ts + h
    long long x_ts, bc_ts, dt_ts;
    int bc_gs, bc_es;
    const float *dt_bias;        // dt + dt_bias[h] before softplus (nullable)
    int softplus;                // dt <- softplus(dt + dt_bias)
};

template <typename T>
__device__ __forceinline__ float view_x(const CplxView<T> &v, size_t bt, int h, int P, int p) {
    return to_f32<T>(v.x[bt * v.x_ts + (size_t)h * P + p]);
}
template <typename T> __device__ __forceinline__ cf view_b(const CplxView<T> &v, size_t bt, int g, int n) {
    const size_t o = bt * v.bc_ts + (size_t)g * v.bc_gs + (size_t)n * v.bc_es;
    return {to_f32<T>(v.bre[o]), to_f32<T>(v.bim[o])};
}
template <typename T> __device__ __forceinline__ cf view_c(const CplxView<T> &v, size_t bt, int g, int n) {
    const size_t o = bt * v.bc_ts + (size_t)g * v.bc_gs + (size_t)n * v.bc_es;
    return {to_f32<T>(v.cre[o]), to_f32<T>(v.cim[o])};
}
// softplus(u) = log(1 + e^u), computed as u + log1p(e^-u) for large u
__device__ __forceinline__ float softplus_f(float u) { return u > 15.f ? u + log1pf(__expf(-u)) : log1pf(__expf(u)); }
template <typename T> __device__ __forceinline__ float view_dt(const CplxView<T> &v, size_t bt, int h) {
    float d = to_f32<T>(v.dt[bt * v.dt_ts + h]);
    if (v.softplus) d = softplus_f(d + (v.dt_bias ? v.dt_bias[h] : 0.f));
    return d;
}

// The separate tensors of ssd_scan_fwd_complex: x, dt float32; B, C complex64
// (interleaved float pairs) [b, T, G, N].
inline CplxView<float> plain_view(const ScanArgs &a) {
    CplxView<float> v;
    v.x = static_cast<const float *>(a.x);
    v.bre = static_cast<const float *>(a.B);
    v.bim = v.bre + 1;
    v.cre = static_cast<const float *>(a.C);
    v.cim = v.cre + 1;
    v.dt = a.dt;
    v.x_ts = (long long)a.nheads * a.headdim;
    v.bc_ts = 2LL * a.ngroups * a.dstate;
    v.dt_ts = a.nheads;
    v.bc_gs = 2 * a.dstate;
    v.bc_es = 2;
    v.dt_bias = nullptr;
    v.softplus = 0;
    return v;
}

// The packed projection output [b, T, H (P + 4N + 1)] (one group per head).
template <typename T>
inline CplxView<T> packed_view(const void *proj, const float *dt_bias, int nheads, int headdim, int dstate) {
    const T *p = static_cast<const T *>(proj);
    const long long HP = (long long)nheads * headdim, HN = (long long)nheads * dstate;
    CplxView<T> v;
    v.x = p;
    v.bre = p + HP;
    v.bim = p + HP + HN;
    v.cre = p + HP + 2 * HN;
    v.cim = p + HP + 3 * HN;
    v.dt = p + HP + 4 * HN;
    v.x_ts = v.bc_ts = v.dt_ts = HP + 4 * HN + nheads;
    v.bc_gs = dstate;
    v.bc_es = 1;
    v.dt_bias = dt_bias;
    v.softplus = 1;
    return v;
}

}  // namespace ssd
