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
// The scan's inputs are read-only while it runs (outputs never alias them), so
// they are read through the read-only global path: besides the cache, that
// tells the compiler a load cannot alias the shared-memory stores of the
// staging loops, so loads of later rows can be issued ahead of them.
template <typename T> __device__ __forceinline__ float ldg_f32(const T *p) { return to_f32<T>(__ldg(p)); }

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
    int vec;                     // 16-byte loads of 4 states / 8 x values are aligned (set on the host)
};

template <typename T>
__device__ __forceinline__ float view_x(const CplxView<T> &v, size_t bt, int h, int P, int p) {
    return ldg_f32<T>(v.x + bt * v.x_ts + (size_t)h * P + p);
}
template <typename T> __device__ __forceinline__ cf view_b(const CplxView<T> &v, size_t bt, int g, int n) {
    const size_t o = bt * v.bc_ts + (size_t)g * v.bc_gs + (size_t)n * v.bc_es;
    return {ldg_f32<T>(v.bre + o), ldg_f32<T>(v.bim + o)};
}
template <typename T> __device__ __forceinline__ cf view_c(const CplxView<T> &v, size_t bt, int g, int n) {
    const size_t o = bt * v.bc_ts + (size_t)g * v.bc_gs + (size_t)n * v.bc_es;
    return {ldg_f32<T>(v.cre + o), ldg_f32<T>(v.cim + o)};
}
// Four consecutive states n0 .. n0+3 (n0 a multiple of 4) of B or C at one
// token: two 16-byte loads (interleaved float32) or one per part (split real
// and imaginary slices) when the view allows, else element by element.
template <typename T>
__device__ __forceinline__ void view_cplx4(const CplxView<T> &v, const T *re, const T *im, size_t bt, int g, int n0,
                                           cf (&out)[4]) {
    const size_t o = bt * v.bc_ts + (size_t)g * v.bc_gs + (size_t)n0 * v.bc_es;
    if (v.vec) {
        if constexpr (sizeof(T) == 4) {
            if (v.bc_es == 2) {  // (re, im) pairs
                const float4 a = __ldg(reinterpret_cast<const float4 *>(re + o));
                const float4 b = __ldg(reinterpret_cast<const float4 *>(re + o + 4));
                out[0] = {a.x, a.y}, out[1] = {a.z, a.w}, out[2] = {b.x, b.y}, out[3] = {b.z, b.w};
            } else {
                const float4 a = __ldg(reinterpret_cast<const float4 *>(re + o));
                const float4 b = __ldg(reinterpret_cast<const float4 *>(im + o));
                out[0] = {a.x, b.x}, out[1] = {a.y, b.y}, out[2] = {a.z, b.z}, out[3] = {a.w, b.w};
            }
        } else {  // bf16, split slices: 8 bytes per part
            const uint2 a = __ldg(reinterpret_cast<const uint2 *>(re + o));
            const uint2 b = __ldg(reinterpret_cast<const uint2 *>(im + o));
            out[0] = {__uint_as_float(a.x << 16), __uint_as_float(b.x << 16)};
            out[1] = {__uint_as_float(a.x & 0xffff0000u), __uint_as_float(b.x & 0xffff0000u)};
            out[2] = {__uint_as_float(a.y << 16), __uint_as_float(b.y << 16)};
            out[3] = {__uint_as_float(a.y & 0xffff0000u), __uint_as_float(b.y & 0xffff0000u)};
        }
        return;
    }
#pragma unroll
    for (int q = 0; q < 4; ++q)
        out[q] = {ldg_f32<T>(re + o + (size_t)q * v.bc_es), ldg_f32<T>(im + o + (size_t)q * v.bc_es)};
}
// Eight consecutive x values p0 .. p0+7 (p0 a multiple of 8) at one token and head.
template <typename T>
__device__ __forceinline__ void view_x8(const CplxView<T> &v, size_t bt, int h, int P, int p0, float (&out)[8]) {
    const T *px = v.x + bt * v.x_ts + (size_t)h * P + p0;
    if (v.vec) {
        if constexpr (sizeof(T) == 4) {
            const float4 a = __ldg(reinterpret_cast<const float4 *>(px)), b = __ldg(reinterpret_cast<const float4 *>(px + 4));
            out[0] = a.x, out[1] = a.y, out[2] = a.z, out[3] = a.w, out[4] = b.x, out[5] = b.y, out[6] = b.z,
            out[7] = b.w;
        } else {
            const uint4 a = __ldg(reinterpret_cast<const uint4 *>(px));
            const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                out[2 * e] = __uint_as_float(w[e] << 16);
                out[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
            }
        }
        return;
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) out[e] = ldg_f32<T>(px + e);
}

// softplus(u) = log(1 + e^u), computed as u + log1p(e^-u) for large u
__device__ __forceinline__ float softplus_f(float u) { return u > 15.f ? u + log1pf(__expf(-u)) : log1pf(__expf(u)); }
template <typename T> __device__ __forceinline__ float view_dt(const CplxView<T> &v, size_t bt, int h) {
    float d = ldg_f32<T>(v.dt + bt * v.dt_ts + h);
    if (v.softplus) d = softplus_f(d + (v.dt_bias ? __ldg(v.dt_bias + h) : 0.f));
    return d;
}

// Whether the vector loads above are aligned for every token, group and head:
// base pointers aligned to the load and every stride a multiple of it.  With
// interleaved pairs (bc_es == 2) the imaginary pointer is the real one plus a
// float and is never dereferenced by the vector path.
template <typename T> inline bool view_vec_ok(const CplxView<T> &v, int headdim, int dstate) {
    auto al = [](const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; };
    const long long xv = 16 / (long long)sizeof(T);  // x elements per 16-byte load
    const uintptr_t ba = 4 * sizeof(T);               // bytes per B/C load of one part (4 elements)
    const bool pairs = sizeof(T) == 4 && v.bc_es == 2;
    const bool bc_ok = pairs ? (al(v.bre, 16) && al(v.cre, 16))
                             : (v.bc_es == 1 && al(v.bre, ba) && al(v.bim, ba) && al(v.cre, ba) && al(v.cim, ba));
    return bc_ok && al(v.x, 16) && v.x_ts % xv == 0 && headdim % 8 == 0 && v.bc_ts % 4 == 0 &&
           v.bc_gs % 4 == 0 && dstate % 4 == 0;
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
    v.vec = view_vec_ok(v, a.headdim, a.dstate);
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
    v.vec = view_vec_ok(v, headdim, dstate);
    return v;
}

}  // namespace ssd
