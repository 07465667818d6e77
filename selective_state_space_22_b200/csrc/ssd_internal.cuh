// ssd_internal.cuh -- types and helpers shared by the CUDA kernels of libssd.
//
// Nothing here is part of the public ABI (include/ssd.h is).  All kernels run
// on the stream the caller passes and read/write caller-owned device memory.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssd {

// ----------------------------------------------------------------- io types
template <typename T> __device__ __forceinline__ float ld_f32(const T *p);
template <> __device__ __forceinline__ float ld_f32<float>(const float *p) { return *p; }
template <> __device__ __forceinline__ float ld_f32<__nv_bfloat16>(const __nv_bfloat16 *p) {
    return __bfloat162float(*p);
}
template <typename T> __device__ __forceinline__ void st_f32(T *p, float v);
template <> __device__ __forceinline__ void st_f32<float>(float *p, float v) { *p = v; }
template <> __device__ __forceinline__ void st_f32<__nv_bfloat16>(__nv_bfloat16 *p, float v) {
    *p = __float2bfloat16_rn(v);
}

// ------------------------------------------------------------ complex floats
// Interleaved (re, im) pairs, the memory layout of complex64.
struct cf {
    float re, im;
};
__device__ __forceinline__ cf cmul(cf a, cf b) {
    return {fmaf(a.re, b.re, -a.im * b.im), fmaf(a.re, b.im, a.im * b.re)};
}
__device__ __forceinline__ cf cfma(cf a, cf b, cf c) {  // a*b + c
    return {fmaf(a.re, b.re, fmaf(-a.im, b.im, c.re)), fmaf(a.re, b.im, fmaf(a.im, b.re, c.im))};
}
__device__ __forceinline__ cf cscale(cf a, float s) { return {a.re * s, a.im * s}; }
__device__ __forceinline__ cf cadd(cf a, cf b) { return {a.re + b.re, a.im + b.im}; }

// exp(z) for a complex exponent z = (a, w) given in double: e^a (cos w, sin w).
__device__ __forceinline__ cf cexp_d(double a, double w) {
    float r = (float)exp(a);
    float s, c;
    sincosf((float)w, &s, &c);
    return {r * c, r * s};
}

// -------------------------------------------------------------- arguments
// One scan call as the kernels see it.  For the complex variant the complex
// tensors (A, B, C, states) are float pairs.
struct ScanArgs {
    const void *x;
    const float *dt;
    const float *A;
    const void *B;
    const void *C;
    const float *D;
    const float *init_state;
    float *final_state;
    void *y;
    int batch, seqlen, nheads, headdim, ngroups, dstate, chunk;
    int nchunks;
    int *dev_error;  // device error word (see ssd_get_device_status)
};

// Device error codes written to *dev_error (first writer wins).
enum : int { DEV_OK = 0, DEV_TIMEOUT = 1 };

// --------------------------------------------------------- kernel launchers
// Each returns cudaSuccess or the launch error; none synchronises.
size_t generic_workspace_bytes(int batch, int nheads, int headdim, int dstate, int chunk,
                               int nchunks, bool cplx);
// Complex scan (scan_complex.cu); same workspace layout and size as
// generic_workspace_bytes(..., cplx = true), with the chunk 128 when
// cplx_tc_supported (the tensor-core path evaluates 128-token chunks).
bool cplx_tc_supported(int headdim, int dstate);
cudaError_t launch_complex_scan(const ScanArgs &a, void *ws, cudaStream_t st);
// The same reading x, B, C and dt from the packed projection output
// [batch, seqlen, H (P + 4N + 1)] (float32 or bf16), dt = softplus(dt + dt_bias).
cudaError_t launch_complex_packed(const ScanArgs &a, const void *proj, bool proj_bf16, const float *dt_bias, void *ws,
                                  cudaStream_t st);
cudaError_t launch_generic_scan(const ScanArgs &a, bool cplx, bool bf16, void *ws,
                                cudaStream_t st);

// tcgen05 tensor-core scan (bf16 io, real A).
bool tc_supported(int headdim, int dstate, int seqlen);
size_t tc_workspace_bytes(int batch, int nheads);
cudaError_t launch_tc_scan(const ScanArgs &a, void *ws, cudaStream_t st);
int tc_kernel_launches(int batch, int nheads, int seqlen);
// Test only: with withhold != 0 the tensor-core kernel's producer issues no load,
// so every bounded wait runs out; wait_ns (0: the default) bounds each wait.
void set_tc_fault_injection(int withhold, unsigned long long wait_ns);

cudaError_t launch_state_update(float *state, const void *x, const float *dt, const float *A,
                                const void *B, const void *C, const float *D, void *y,
                                bool bf16, bool cplx, int batch, int nheads, int headdim,
                                int ngroups, int dstate, cudaStream_t st);

// Gradients of the real fp32 scan (scan_bwd.cu): headdim <= 64, dstate <= 128.
struct BwdCall {
    const float *x, *dt, *A, *B, *C, *D, *init_state, *dy, *dfinal;
    float *dx, *ddt, *dA, *dB, *dC, *dD, *dinit;
    int batch, seqlen, nheads, headdim, ngroups, dstate;
    int *dev_error;  // device error word
};
bool bwd_supported(int headdim, int dstate);
size_t bwd_workspace_bytes(int batch, int seqlen, int nheads, int headdim, int ngroups, int dstate);
cudaError_t launch_scan_bwd(const BwdCall &call, void *ws, cudaStream_t st);
// Complex variant: A, B, C, init_state, dfinal and dA, dB, dC, dinit are float
// pairs; headdim <= 64, dstate <= 64.
bool bwd_complex_supported(int headdim, int dstate);
size_t bwd_complex_workspace_bytes(int batch, int seqlen, int nheads, int headdim, int dstate);
cudaError_t launch_scan_bwd_complex(const BwdCall &call, void *ws, cudaStream_t st);

cudaError_t launch_copy_or_zero_state(const float *init_state, float *final_state,
                                      size_t nfloats, cudaStream_t st);

// Sequence split across devices (seqpar.cu): total log-decay of each (batch,
// head) over a slice, and the ordered fold of the slices' end states.
cudaError_t launch_log_decay_sum(const float *dt, const float *A, float *out, int batch, int seqlen, int nheads,
                                 cudaStream_t st);
cudaError_t launch_fold_states(const float *states, const float *lam, int nstates, float *out, int batch,
                               int nheads, int headdim, int dstate, cudaStream_t st);

// The variants (variants.cu): the causal conv1d prologue over packed x|B|C
// channels, and the Mamba-1 selective scan (dstate 4, 8, 16 or 32).
cudaError_t launch_conv1d_xbc(const void *in, const float *w, const float *bias, const void *cinit, void *xo,
                              void *bo, void *co, void *cfinal, bool bf16, int batch, int seqlen, int cx, int cb,
                              int width, int silu, cudaStream_t st);
bool selective_dstate_supported(int dstate);
cudaError_t launch_selective_scan(const void *x, const float *dt, const float *A, const void *B, const void *C,
                                  const float *D, const float *init_state, float *final_state, void *y, bool bf16,
                                  int batch, int seqlen, int channels, int ngroups, int dstate, cudaStream_t st);

// Sets the message ssd_last_error() returns on this host thread.
void set_last_error(const char *msg);

// The calling thread's current CUDA context (the driver's CUcontext, as an
// opaque pointer; NULL when there is none or the query is unavailable).  The
// per-device caches of device addresses and kernel attributes are keyed on it,
// so they are looked up again after the context changes (for example after
// cudaDeviceReset destroyed the primary context and a new one was created).
void *current_context();

static inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace ssd
