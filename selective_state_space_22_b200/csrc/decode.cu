// decode.cu -- one recurrent step of the selective state-space model, in place.
//
//   state <- exp(dt A) state + dt x B^T ;  y = Re(state C) + D x
//
// The step is the body of the recurrence in the "Mamba-3-Lite" README (the
// recurrence section), applied once per generated token ("BitMamba 1B",
// "Context": inference per token).  It reads and writes the whole float32 state
// once, so it is bound by HBM bandwidth: each warp owns state rows
// (batch, head, p) of dstate elements, streams them with 128-bit loads and
// stores (evict-first: the state is touched once per step) and reduces the
// readout with warp shuffles.  B and C of a sequence are shared by all its heads
// and rows and stay in L1/L2.
#include "ssd_internal.cuh"

namespace ssd {
namespace {

constexpr int NT = 256;

__device__ __forceinline__ float4 ld_stream(const float4 *p) {
    float4 v;
    asm volatile("ld.global.cs.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p));
    return v;
}
__device__ __forceinline__ void st_stream(float4 *p, float4 v) {
    asm volatile("st.global.cs.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(v.x), "f"(v.y),
                 "f"(v.z), "f"(v.w)
                 : "memory");
}

template <typename TIO> __device__ __forceinline__ float4 ld4(const TIO *p);
template <> __device__ __forceinline__ float4 ld4<float>(const float *p) {
    return *reinterpret_cast<const float4 *>(p);
}
template <> __device__ __forceinline__ float4 ld4<__nv_bfloat16>(const __nv_bfloat16 *p) {
    uint2 u = *reinterpret_cast<const uint2 *>(p);
    float4 v;
    v.x = __uint_as_float(u.x << 16);
    v.y = __uint_as_float(u.x & 0xffff0000u);
    v.z = __uint_as_float(u.y << 16);
    v.w = __uint_as_float(u.y & 0xffff0000u);
    return v;
}

// Real step, dstate a multiple of 128.  One block per (batch, head): its index
// arithmetic, dt, the decay and D are computed once, and B and C (shared by the
// head's rows) once per warp.  A warp streams ROWS state rows at a time, lane j
// holding elements 4j..4j+3 of each 128-wide slice, so ROWS x 512 bytes of loads
// are in flight per warp before the first use.
template <typename TIO, int ROWS>
__global__ void __launch_bounds__(NT, 4) update_real_vec(float *__restrict__ state, const TIO *__restrict__ x,
                                                      const float *__restrict__ dt, const float *__restrict__ A,
                                                      const TIO *__restrict__ B, const TIO *__restrict__ C,
                                                      const float *__restrict__ D, TIO *__restrict__ y,
                                                      int nheads, int headdim, int ngroups, int dstate) {
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    const size_t bh = blockIdx.x;
    const int h = (int)(bh % (unsigned)nheads);
    const size_t b = bh / (unsigned)nheads;
    const int g = h / (nheads / ngroups);
    const float dtv = dt[bh];
    const float dec = __expf(dtv * A[h]);
    const float Dh = D ? D[h] : 0.f;
    const TIO *Bg = B + (b * ngroups + g) * dstate + lane * 4;
    const TIO *Cg = C + (b * ngroups + g) * dstate + lane * 4;
    float *st = state + bh * headdim * dstate + lane * 4;
    const TIO *xr = x + bh * headdim;
    TIO *yr = y + bh * headdim;
    for (int p0 = wib * ROWS; p0 < headdim; p0 += (NT / 32) * ROWS) {
        float yacc[ROWS], u[ROWS];
#pragma unroll
        for (int r = 0; r < ROWS; ++r) {
            yacc[r] = 0.f;
            u[r] = p0 + r < headdim ? dtv * ld_f32(xr + p0 + r) : 0.f;
        }
#pragma unroll 1
        for (int sl = 0; sl < dstate; sl += 128) {
            float4 hv[ROWS];
#pragma unroll
            for (int r = 0; r < ROWS; ++r)
                if (p0 + r < headdim) hv[r] = ld_stream(reinterpret_cast<const float4 *>(st + (size_t)(p0 + r) * dstate + sl));
            const float4 bv = ld4(Bg + sl), cv = ld4(Cg + sl);
#pragma unroll
            for (int r = 0; r < ROWS; ++r) {
                if (p0 + r >= headdim) continue;
                float4 h4 = hv[r];
                h4.x = fmaf(dec, h4.x, u[r] * bv.x);
                h4.y = fmaf(dec, h4.y, u[r] * bv.y);
                h4.z = fmaf(dec, h4.z, u[r] * bv.z);
                h4.w = fmaf(dec, h4.w, u[r] * bv.w);
                yacc[r] += h4.x * cv.x + h4.y * cv.y + h4.z * cv.z + h4.w * cv.w;
                st_stream(reinterpret_cast<float4 *>(st + (size_t)(p0 + r) * dstate + sl), h4);
            }
        }
#pragma unroll
        for (int r = 0; r < ROWS; ++r) {
            float part = yacc[r];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
            if (lane == 0 && p0 + r < headdim) st_f32(yr + p0 + r, part + Dh * ld_f32(xr + p0 + r));
        }
    }
}

// General step (any dstate), real or complex; one warp per state row.
template <typename TIO, bool CPLX>
__global__ void __launch_bounds__(NT) update_generic(float *__restrict__ state, const TIO *__restrict__ x,
                                                     const float *__restrict__ dt, const float *__restrict__ A,
                                                     const void *__restrict__ Bv, const void *__restrict__ Cv,
                                                     const float *__restrict__ D, TIO *__restrict__ y,
                                                     int batch, int nheads, int headdim, int ngroups,
                                                     int dstate) {
    const int lane = threadIdx.x & 31;
    const long row = (long)blockIdx.x * (NT / 32) + (threadIdx.x >> 5);
    const long nrows = (long)batch * nheads * headdim;
    if (row >= nrows) return;
    const long bh = row / headdim;
    const int h = (int)(bh % nheads);
    const long b = bh / nheads;
    const int g = h / (nheads / ngroups);
    const float d = dt[bh];
    const float xv = ld_f32(x + row);
    const float u = d * xv;
    float part = 0.f;
    if constexpr (CPLX) {
        const cf dec = cexp_d((double)d * A[2 * h], (double)d * A[2 * h + 1]);
        cf *st = reinterpret_cast<cf *>(state) + row * dstate;
        const cf *Bc = reinterpret_cast<const cf *>(Bv) + ((size_t)b * ngroups + g) * dstate;
        const cf *Cc = reinterpret_cast<const cf *>(Cv) + ((size_t)b * ngroups + g) * dstate;
        for (int n = lane; n < dstate; n += 32) {
            cf hv = cfma(dec, st[n], cscale(Bc[n], u));
            st[n] = hv;
            part += fmaf(hv.re, Cc[n].re, -hv.im * Cc[n].im);
        }
    } else {
        const float dec = __expf(d * A[h]);
        float *st = state + row * dstate;
        const TIO *Bt = reinterpret_cast<const TIO *>(Bv) + ((size_t)b * ngroups + g) * dstate;
        const TIO *Ct = reinterpret_cast<const TIO *>(Cv) + ((size_t)b * ngroups + g) * dstate;
        for (int n = lane; n < dstate; n += 32) {
            float hv = fmaf(dec, st[n], u * ld_f32(Bt + n));
            st[n] = hv;
            part = fmaf(hv, ld_f32(Ct + n), part);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (lane == 0) st_f32(y + row, part + (D ? D[h] * xv : 0.f));
}

template <typename TIO>
cudaError_t launch_real(float *state, const void *x, const float *dt, const float *A, const void *B,
                        const void *C, const float *D, void *y, int batch, int nheads, int headdim,
                        int ngroups, int dstate, cudaStream_t st) {
    const long nrows = (long)batch * nheads * headdim;
    if (dstate % 128 == 0) {
        update_real_vec<TIO, 4><<<(unsigned)((long)batch * nheads), NT, 0, st>>>(
            state, (const TIO *)x, dt, A, (const TIO *)B, (const TIO *)C, D, (TIO *)y, nheads, headdim,
            ngroups, dstate);
    } else {
        const long blocks = (nrows + NT / 32 - 1) / (NT / 32);
        update_generic<TIO, false><<<(unsigned)blocks, NT, 0, st>>>(
            state, (const TIO *)x, dt, A, B, C, D, (TIO *)y, batch, nheads, headdim, ngroups, dstate);
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_state_update(float *state, const void *x, const float *dt, const float *A,
                                const void *B, const void *C, const float *D, void *y, bool bf16,
                                bool cplx, int batch, int nheads, int headdim, int ngroups, int dstate,
                                cudaStream_t st) {
    if (cplx) {
        const long nrows = (long)batch * nheads * headdim;
        const long blocks = (nrows + NT / 32 - 1) / (NT / 32);
        update_generic<float, true><<<(unsigned)blocks, NT, 0, st>>>(
            state, (const float *)x, dt, A, B, C, D, (float *)y, batch, nheads, headdim, ngroups, dstate);
        return cudaGetLastError();
    }
    if (bf16)
        return launch_real<__nv_bfloat16>(state, x, dt, A, B, C, D, y, batch, nheads, headdim, ngroups,
                                          dstate, st);
    return launch_real<float>(state, x, dt, A, B, C, D, y, batch, nheads, headdim, ngroups, dstate, st);
}

// final_state = init_state (or zeros) for an empty sequence.
__global__ void copy_or_zero(const float *__restrict__ src, float *__restrict__ dst, size_t n) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
        dst[i] = src ? src[i] : 0.f;
}

cudaError_t launch_copy_or_zero_state(const float *init_state, float *final_state, size_t nfloats,
                                      cudaStream_t st) {
    if (nfloats == 0) return cudaSuccess;
    size_t blocks = (nfloats + 255) / 256;
    if (blocks > 4096) blocks = 4096;
    copy_or_zero<<<(unsigned)blocks, 256, 0, st>>>(init_state, final_state, nfloats);
    return cudaGetLastError();
}

}  // namespace ssd
