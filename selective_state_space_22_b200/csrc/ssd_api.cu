// ssd_api.cu -- the C ABI of libssd (declared in include/ssd.h).
//
// Host-side argument validation, workspace sizing, kernel selection and the
// device error word.  Every check happens before the first launch, so a
// non-OK status means nothing was enqueued.
#include <stdarg.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include <mutex>
#include <string>

#include "../../include/ssd.h"
#include "ssd_internal.cuh"

// First device-side error raised by a kernel of this library on this device
// (a bounded wait that gave up).  Read and cleared by ssd_get_device_status.
__device__ int g_ssd_device_error = 0;

namespace {

thread_local std::string g_last_error;

ssd_status fail(ssd_status s, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
ssd_status fail(ssd_status s, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return s;
}

ssd_status cuda_fail(cudaError_t e, const char *what) {
    return fail(SSD_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Device address of the error word in the current context, looked up once per
// (device, context) with that device current.
int *device_error_ptr(ssd_status *st) {
    struct Entry {
        void *ctx;
        int *ptr;
    };
    static Entry cache[64] = {};
    static std::mutex mu;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= 64) {
        *st = cuda_fail(e, "cudaGetDevice");
        return nullptr;
    }
    void *ctx = ssd::current_context();
    std::lock_guard<std::mutex> lk(mu);
    if (!cache[dev].ptr || cache[dev].ctx != ctx) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_ssd_device_error);
        if (e != cudaSuccess) {
            *st = cuda_fail(e, "cudaGetSymbolAddress(device error word)");
            return nullptr;
        }
        cache[dev] = Entry{ctx, static_cast<int *>(p)};
    }
    return cache[dev].ptr;
}

constexpr int kMaxHeaddim = 256;
constexpr int kMaxDstate = 256;

// Shape checks shared by the scans.
ssd_status check_scan_dims(int batch, int seqlen, int nheads, int headdim, int ngroups, int dstate,
                           int chunk) {
    if (batch < 0 || seqlen < 0)
        return fail(SSD_ERR_INVALID_ARG, "batch (%d) and seqlen (%d) must be >= 0", batch, seqlen);
    if (nheads <= 0 || headdim <= 0 || ngroups <= 0 || dstate <= 0)
        return fail(SSD_ERR_INVALID_ARG,
                    "nheads (%d), headdim (%d), ngroups (%d), dstate (%d) must be > 0", nheads,
                    headdim, ngroups, dstate);
    if (nheads % ngroups != 0)
        return fail(SSD_ERR_INVALID_ARG, "ngroups (%d) must divide nheads (%d)", ngroups, nheads);
    if (chunk != 64 && chunk != 128 && chunk != 256)
        return fail(SSD_ERR_INVALID_ARG, "chunk_size must be 64, 128 or 256 (got %d)", chunk);
    if (headdim > kMaxHeaddim || dstate > kMaxDstate)
        return fail(SSD_ERR_UNSUPPORTED, "headdim (%d) and dstate (%d) must be <= %d and %d",
                    headdim, dstate, kMaxHeaddim, kMaxDstate);
    if (nheads > 65535 || batch > 2048 || (long long)batch * seqlen > (1LL << 31))
        return fail(SSD_ERR_UNSUPPORTED, "sizes beyond the supported grid (batch <= 2048, "
                    "nheads <= 65535, batch*seqlen <= 2^31)");
    return SSD_OK;
}

struct Plan {
    bool tc;  // tcgen05 tensor-core kernel
    size_t ws;
    int launches;
};

Plan plan_scan(int batch, int seqlen, int nheads, int headdim, int ngroups, int dstate, int chunk,
               bool cplx, bool bf16) {
    Plan p{false, 0, 0};
    const int nchunks = seqlen > 0 ? (seqlen + chunk - 1) / chunk : 0;
    if (!cplx && bf16 && ssd::tc_supported(headdim, dstate, seqlen)) {
        p.tc = true;
        p.ws = ssd::tc_workspace_bytes(batch, nheads);
        p.launches = ssd::tc_kernel_launches(batch, nheads, seqlen);
        return p;
    }
    if (cplx && ssd::cplx_tc_supported(headdim, dstate)) {  // tensor-core path: 128-token chunks
        p.ws = ssd::generic_workspace_bytes(batch, nheads, headdim, dstate, 128, seqlen > 0 ? (seqlen + 127) / 128 : 0,
                                            true);
        p.launches = 3;
        return p;
    }
    p.ws = ssd::generic_workspace_bytes(batch, nheads, headdim, dstate, chunk, nchunks, cplx);
    p.launches = 3;
    return p;
}

ssd_status run_scan(const void *x, const float *dt, const float *A, const void *B, const void *C,
                    const float *D, const float *init_state, float *final_state, void *y, bool cplx,
                    bool bf16, int batch, int seqlen, int nheads, int headdim, int ngroups, int dstate,
                    int chunk, void *workspace, size_t workspace_bytes, void *stream) {
    ssd_status s = check_scan_dims(batch, seqlen, nheads, headdim, ngroups, dstate, chunk);
    if (s != SSD_OK) return s;
    const size_t state_floats = (size_t)batch * nheads * headdim * dstate * (cplx ? 2 : 1);
    const bool any_tokens = (size_t)batch * seqlen > 0;
    if (any_tokens) {
        if (!x || !dt || !A || !B || !C || (!y && !final_state))
            return fail(SSD_ERR_INVALID_ARG, "x, dt, A, B, C and y must be non-null");
        const void *ptrs[] = {x, dt, A, B, C, y, D, init_state, final_state};
        for (const void *p : ptrs)
            if (p && !aligned16(p)) return fail(SSD_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
    } else {
        if ((init_state && !aligned16(init_state)) || (final_state && !aligned16(final_state)))
            return fail(SSD_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (!any_tokens) {
        // No tokens: the final state is the initial one (or zeros).
        if (final_state && final_state != init_state) {
            cudaError_t e = ssd::launch_copy_or_zero_state(init_state, final_state, state_floats, st);
            if (e != cudaSuccess) return cuda_fail(e, "state copy launch");
        }
        return SSD_OK;
    }
    Plan pl = plan_scan(batch, seqlen, nheads, headdim, ngroups, dstate, chunk, cplx, bf16);
    if (pl.ws > 0) {
        if (!workspace)
            return fail(SSD_ERR_WORKSPACE, "workspace is NULL; %zu bytes are needed", pl.ws);
        if (workspace_bytes < pl.ws)
            return fail(SSD_ERR_WORKSPACE, "workspace of %zu bytes is too small; %zu are needed",
                        workspace_bytes, pl.ws);
        if (!aligned16(workspace)) return fail(SSD_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
    }
    int *dev_err = device_error_ptr(&s);
    if (!dev_err) return s;

    ssd::ScanArgs a;
    a.x = x;
    a.dt = dt;
    a.A = A;
    a.B = B;
    a.C = C;
    a.D = D;
    a.init_state = init_state;
    a.final_state = final_state;
    a.y = y;
    a.batch = batch;
    a.seqlen = seqlen;
    a.nheads = nheads;
    a.headdim = headdim;
    a.ngroups = ngroups;
    a.dstate = dstate;
    a.chunk = chunk;
    a.nchunks = (seqlen + chunk - 1) / chunk;
    a.dev_error = dev_err;
    cudaError_t e = pl.tc ? ssd::launch_tc_scan(a, workspace, st)
                          : ssd::launch_generic_scan(a, cplx, bf16, workspace, st);
    if (e != cudaSuccess) return cuda_fail(e, "scan launch");
    return SSD_OK;
}

// The state-only scan of one slice of a sequence: final state and total log-decay.
ssd_status run_final_state(const void *x, const float *dt, const float *A, const void *B, const float *init_state,
                           float *final_state, float *total_log_decay, bool bf16, int batch, int seqlen, int nheads,
                           int headdim, int ngroups, int dstate, int chunk, void *workspace, size_t workspace_bytes,
                           void *stream) {
    ssd_status s = check_scan_dims(batch, seqlen, nheads, headdim, ngroups, dstate, chunk);
    if (s != SSD_OK) return s;
    if (!final_state || !A) return fail(SSD_ERR_INVALID_ARG, "final_state and A are required");
    const bool any_tokens = (size_t)batch * seqlen > 0;
    if (any_tokens && (!x || !dt || !B)) return fail(SSD_ERR_INVALID_ARG, "x, dt and B must be non-null");
    const void *ptrs[] = {x, dt, A, B, init_state, final_state, total_log_decay};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return fail(SSD_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (total_log_decay) {
        cudaError_t e = any_tokens ? ssd::launch_log_decay_sum(dt, A, total_log_decay, batch, seqlen, nheads, st)
                                   : cudaMemsetAsync(total_log_decay, 0, (size_t)batch * nheads * sizeof(float), st);
        if (e != cudaSuccess) return cuda_fail(e, "log-decay sum launch");
    }
    // y = NULL selects the state-only form of the scan; C is never read then.
    return run_scan(x, dt, A, B, B, nullptr, init_state, final_state, nullptr, false, bf16, batch, seqlen, nheads,
                    headdim, ngroups, dstate, chunk, workspace, workspace_bytes, stream);
}

// The complex scan reading the packed projection output.
ssd_status run_scan_packed(const void *proj, bool proj_bf16, const float *dt_bias, const float *A, const float *D,
                           const float *init_state, float *final_state, float *y, int batch, int seqlen, int nheads,
                           int headdim, int dstate, int chunk, void *workspace, size_t workspace_bytes, void *stream) {
    ssd_status s = check_scan_dims(batch, seqlen, nheads, headdim, nheads, dstate, chunk);
    if (s != SSD_OK) return s;
    const bool any_tokens = (size_t)batch * seqlen > 0;
    if (any_tokens && (!proj || !A || !y)) return fail(SSD_ERR_INVALID_ARG, "proj, A and y must be non-null");
    const void *ptrs[] = {proj, dt_bias, A, D, init_state, final_state, y};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return fail(SSD_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (!any_tokens) {
        if (final_state && final_state != init_state) {
            cudaError_t e = ssd::launch_copy_or_zero_state(init_state, final_state,
                                                           (size_t)batch * nheads * headdim * dstate * 2, st);
            if (e != cudaSuccess) return cuda_fail(e, "state copy launch");
        }
        return SSD_OK;
    }
    Plan pl = plan_scan(batch, seqlen, nheads, headdim, nheads, dstate, chunk, true, false);
    if (!workspace) return fail(SSD_ERR_WORKSPACE, "workspace is NULL; %zu bytes are needed", pl.ws);
    if (workspace_bytes < pl.ws)
        return fail(SSD_ERR_WORKSPACE, "workspace of %zu bytes is too small; %zu are needed", workspace_bytes, pl.ws);
    if (!aligned16(workspace)) return fail(SSD_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
    int *dev_err = device_error_ptr(&s);
    if (!dev_err) return s;
    ssd::ScanArgs a{};
    a.A = A;
    a.D = D;
    a.init_state = init_state;
    a.final_state = final_state;
    a.y = y;
    a.batch = batch;
    a.seqlen = seqlen;
    a.nheads = nheads;
    a.headdim = headdim;
    a.ngroups = nheads;
    a.dstate = dstate;
    a.chunk = chunk;
    a.nchunks = (seqlen + chunk - 1) / chunk;
    a.dev_error = dev_err;
    cudaError_t e = ssd::launch_complex_packed(a, proj, proj_bf16, dt_bias, workspace, st);
    if (e != cudaSuccess) return cuda_fail(e, "scan launch");
    return SSD_OK;
}

ssd_status run_update(float *state, const void *x, const float *dt, const float *A, const void *B,
                      const void *C, const float *D, void *y, bool bf16, bool cplx, int batch,
                      int nheads, int headdim, int ngroups, int dstate, void *stream) {
    if (batch < 0)
        return fail(SSD_ERR_INVALID_ARG, "batch (%d) must be >= 0", batch);
    if (nheads <= 0 || headdim <= 0 || ngroups <= 0 || dstate <= 0)
        return fail(SSD_ERR_INVALID_ARG,
                    "nheads (%d), headdim (%d), ngroups (%d), dstate (%d) must be > 0", nheads,
                    headdim, ngroups, dstate);
    if (nheads % ngroups != 0)
        return fail(SSD_ERR_INVALID_ARG, "ngroups (%d) must divide nheads (%d)", ngroups, nheads);
    if ((long long)batch * nheads * headdim > (1LL << 36))
        return fail(SSD_ERR_UNSUPPORTED, "batch * nheads * headdim too large");
    if (batch == 0) return SSD_OK;
    if (!state || !x || !dt || !A || !B || !C || !y)
        return fail(SSD_ERR_INVALID_ARG, "state, x, dt, A, B, C and y must be non-null");
    const void *ptrs[] = {state, x, dt, A, B, C, y, D};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return fail(SSD_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
    cudaError_t e = ssd::launch_state_update(state, x, dt, A, B, C, D, y, bf16, cplx, batch, nheads,
                                             headdim, ngroups, dstate, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "state update launch");
    return SSD_OK;
}

bool valid_dtype(ssd_dtype d) { return d == SSD_F32 || d == SSD_BF16; }

}  // namespace

namespace ssd {
void set_last_error(const char *msg) { g_last_error = msg; }

void *current_context() {
    // cuCtxGetCurrent, fetched through the runtime so that libssd needs no link
    // against the driver library.
    typedef int (*GetCurrent)(void **);
    static GetCurrent fn = [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return (GetCurrent) nullptr;
        return reinterpret_cast<GetCurrent>(f);
    }();
    void *ctx = nullptr;
    if (!fn || fn(&ctx) != 0) return nullptr;
    return ctx;
}
}  // namespace ssd

// The backward scans (real or complex), after validation.
static ssd_status run_bwd(bool cplx, const float *x, const float *dt, const float *A, const float *B,
                          const float *C, const float *D, const float *init_state, const float *dy,
                          const float *dfinal, float *dx, float *ddt, float *dA, float *dB, float *dC,
                          float *dD, float *dinit, int batch, int seqlen, int nheads, int headdim,
                          int ngroups, int dstate, void *workspace, size_t workspace_bytes, void *stream) {
    ssd_status s = check_scan_dims(batch, seqlen, nheads, headdim, ngroups, dstate, 64);
    if (s != SSD_OK) return s;
    if (!cplx && !ssd::bwd_supported(headdim, dstate))
        return fail(SSD_ERR_UNSUPPORTED, "the backward scan takes headdim <= 64 and dstate <= 128 "
                    "(got %d and %d)", headdim, dstate);
    if (cplx && !ssd::bwd_complex_supported(headdim, dstate))
        return fail(SSD_ERR_UNSUPPORTED, "the complex backward scan takes headdim <= 64 and dstate <= 64 "
                    "(got %d and %d)", headdim, dstate);
    if (!A || !dA) return fail(SSD_ERR_INVALID_ARG, "A and dA are required");
    if ((long long)batch * seqlen > 0 && (!x || !dt || !B || !C || !dy || !dx || !ddt || !dB || !dC))
        return fail(SSD_ERR_INVALID_ARG, "x, dt, B, C, dy, dx, ddt, dB and dC are required");
    for (const void *p : {(const void *)x, (const void *)dt, (const void *)A, (const void *)B,
                          (const void *)C, (const void *)D, (const void *)init_state, (const void *)dy,
                          (const void *)dfinal, (const void *)dx, (const void *)ddt, (const void *)dA,
                          (const void *)dB, (const void *)dC, (const void *)dD, (const void *)dinit})
        if (p && !aligned16(p)) return fail(SSD_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
    if ((unsigned long long)batch * seqlen * ngroups * dstate / 256 >= (1ULL << 31))
        return fail(SSD_ERR_UNSUPPORTED, "batch * seqlen * ngroups * dstate is beyond the supported grid");
    const size_t need = cplx ? ssd::bwd_complex_workspace_bytes(batch, seqlen, nheads, headdim, dstate)
                             : ssd::bwd_workspace_bytes(batch, seqlen, nheads, headdim, ngroups, dstate);
    if (need > 0) {
        if (!workspace || workspace_bytes < need)
            return fail(SSD_ERR_WORKSPACE, "workspace of %zu bytes needed (got %zu)", need,
                        workspace ? workspace_bytes : (size_t)0);
        if (!aligned16(workspace)) return fail(SSD_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
    }
    int *dev_err = device_error_ptr(&s);
    if (!dev_err) return s;
    ssd::BwdCall call{x, dt, A, B, C, D, init_state, dy, dfinal, dx, ddt, dA, dB, dC, dD, dinit,
                      batch, seqlen, nheads, headdim, ngroups, dstate, dev_err};
    cudaError_t e = cplx ? ssd::launch_scan_bwd_complex(call, workspace, static_cast<cudaStream_t>(stream))
                         : ssd::launch_scan_bwd(call, workspace, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "launching the backward scan");
    return SSD_OK;
}

extern "C" {

size_t ssd_scan_workspace_size(int batch, int seqlen, int nheads, int headdim, int ngroups,
                               int dstate, int chunk_size, int is_complex, ssd_dtype io_dtype) {
    if (!valid_dtype(io_dtype)) return SSD_WORKSPACE_INVALID;
    if (check_scan_dims(batch, seqlen, nheads, headdim, ngroups, dstate, chunk_size) != SSD_OK)
        return SSD_WORKSPACE_INVALID;
    Plan pl = plan_scan(batch, seqlen, nheads, headdim, ngroups, dstate, chunk_size, is_complex != 0,
                        io_dtype == SSD_BF16);
    return pl.ws;
}

int ssd_scan_kernel_launches(int batch, int seqlen, int nheads, int headdim, int ngroups, int dstate,
                             int chunk_size, int is_complex, ssd_dtype io_dtype) {
    if (!valid_dtype(io_dtype)) return 0;
    if (check_scan_dims(batch, seqlen, nheads, headdim, ngroups, dstate, chunk_size) != SSD_OK)
        return 0;
    return plan_scan(batch, seqlen, nheads, headdim, ngroups, dstate, chunk_size, is_complex != 0,
                     io_dtype == SSD_BF16)
        .launches;
}

ssd_status ssd_scan_fwd(const void *x, const float *dt, const float *A, const void *B,
                        const void *C, const float *D, const float *init_state, float *final_state,
                        void *y, ssd_dtype io_dtype, int batch, int seqlen, int nheads, int headdim,
                        int ngroups, int dstate, int chunk_size, void *workspace,
                        size_t workspace_bytes, void *stream) {
    if (!valid_dtype(io_dtype)) return fail(SSD_ERR_INVALID_ARG, "io_dtype must be SSD_F32 or SSD_BF16");
    if (!y && (long long)batch * seqlen > 0) return fail(SSD_ERR_INVALID_ARG, "y must be non-null");
    return run_scan(x, dt, A, B, C, D, init_state, final_state, y, false, io_dtype == SSD_BF16, batch,
                    seqlen, nheads, headdim, ngroups, dstate, chunk_size, workspace, workspace_bytes,
                    stream);
}

ssd_status ssd_scan_final_state(const void *x, const float *dt, const float *A, const void *B,
                                const float *init_state, float *final_state, float *total_log_decay,
                                ssd_dtype io_dtype, int batch, int seqlen, int nheads, int headdim, int ngroups,
                                int dstate, int chunk_size, void *workspace, size_t workspace_bytes, void *stream) {
    if (!valid_dtype(io_dtype)) return fail(SSD_ERR_INVALID_ARG, "io_dtype must be SSD_F32 or SSD_BF16");
    return run_final_state(x, dt, A, B, init_state, final_state, total_log_decay, io_dtype == SSD_BF16, batch,
                           seqlen, nheads, headdim, ngroups, dstate, chunk_size, workspace, workspace_bytes, stream);
}

ssd_status ssd_fold_states(const float *states, const float *log_decay, int nstates, float *out, int batch,
                           int nheads, int headdim, int dstate, void *stream) {
    if (nstates <= 0 || batch < 0 || nheads <= 0 || headdim <= 0 || dstate <= 0)
        return fail(SSD_ERR_INVALID_ARG, "nstates, nheads, headdim and dstate must be > 0 and batch >= 0");
    if ((long long)batch * nheads * headdim * dstate * nstates > (1LL << 40))
        return fail(SSD_ERR_UNSUPPORTED, "states too large");
    if (batch == 0) return SSD_OK;
    if (!states || !out || (nstates > 1 && !log_decay))
        return fail(SSD_ERR_INVALID_ARG, "states, out (and log_decay when nstates > 1) must be non-null");
    for (const void *p : {(const void *)states, (const void *)log_decay, (const void *)out})
        if (p && !aligned16(p)) return fail(SSD_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
    cudaError_t e = ssd::launch_fold_states(states, log_decay, nstates, out, batch, nheads, headdim, dstate,
                                            static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "fold launch");
    return SSD_OK;
}

ssd_status ssd_scan_fwd_complex(const float *x, const float *dt, const float *A, const float *B,
                                const float *C, const float *D, const float *init_state,
                                float *final_state, float *y, int batch, int seqlen, int nheads,
                                int headdim, int ngroups, int dstate, int chunk_size, void *workspace,
                                size_t workspace_bytes, void *stream) {
    if (!y && (long long)batch * seqlen > 0) return fail(SSD_ERR_INVALID_ARG, "y must be non-null");
    return run_scan(x, dt, A, B, C, D, init_state, final_state, y, true, false, batch, seqlen, nheads,
                    headdim, ngroups, dstate, chunk_size, workspace, workspace_bytes, stream);
}

ssd_status ssd_scan_fwd_complex_packed(const void *proj, ssd_dtype proj_dtype, const float *dt_bias, const float *A,
                                       const float *D, const float *init_state, float *final_state, float *y,
                                       int batch, int seqlen, int nheads, int headdim, int dstate, int chunk_size,
                                       void *workspace, size_t workspace_bytes, void *stream) {
    if (!valid_dtype(proj_dtype)) return fail(SSD_ERR_INVALID_ARG, "proj_dtype must be SSD_F32 or SSD_BF16");
    return run_scan_packed(proj, proj_dtype == SSD_BF16, dt_bias, A, D, init_state, final_state, y, batch, seqlen,
                           nheads, headdim, dstate, chunk_size, workspace, workspace_bytes, stream);
}

ssd_status ssd_conv1d_xbc(const void *xbc, const float *weight, const float *bias, const void *conv_init,
                          void *x_out, void *B_out, void *C_out, void *conv_final, ssd_dtype io_dtype, int batch,
                          int seqlen, int x_channels, int bc_channels, int width, int silu, void *stream) {
    if (!valid_dtype(io_dtype)) return fail(SSD_ERR_INVALID_ARG, "io_dtype must be SSD_F32 or SSD_BF16");
    if (batch < 0 || seqlen < 0 || x_channels <= 0 || bc_channels < 0)
        return fail(SSD_ERR_INVALID_ARG, "batch and seqlen must be >= 0, x_channels > 0, bc_channels >= 0");
    if (width < 1 || width > 8) return fail(SSD_ERR_UNSUPPORTED, "width must be in 1..8 (got %d)", width);
    if ((long long)batch * seqlen > (1LL << 31) || batch > 65535 || (long long)x_channels + 2LL * bc_channels > (1 << 24))
        return fail(SSD_ERR_UNSUPPORTED, "sizes beyond the supported grid");
    if ((long long)batch * seqlen == 0) return SSD_OK;
    if (!xbc || !weight || !x_out || (bc_channels > 0 && (!B_out || !C_out)))
        return fail(SSD_ERR_INVALID_ARG, "xbc, weight, x_out, B_out and C_out must be non-null");
    for (const void *p : {(const void *)xbc, (const void *)weight, (const void *)bias, (const void *)conv_init,
                          (const void *)x_out, (const void *)B_out, (const void *)C_out, (const void *)conv_final})
        if (p && !aligned16(p)) return fail(SSD_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
    cudaError_t e = ssd::launch_conv1d_xbc(xbc, weight, bias, conv_init, x_out, B_out, C_out, conv_final,
                                           io_dtype == SSD_BF16, batch, seqlen, x_channels, bc_channels, width,
                                           silu != 0, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "conv1d launch");
    return SSD_OK;
}

ssd_status ssd_selective_scan(const void *x, const float *dt, const float *A, const void *B, const void *C,
                              const float *D, const float *init_state, float *final_state, void *y,
                              ssd_dtype io_dtype, int batch, int seqlen, int channels, int ngroups, int dstate,
                              void *stream) {
    if (!valid_dtype(io_dtype)) return fail(SSD_ERR_INVALID_ARG, "io_dtype must be SSD_F32 or SSD_BF16");
    if (batch < 0 || seqlen < 0 || channels <= 0 || ngroups <= 0 || dstate <= 0)
        return fail(SSD_ERR_INVALID_ARG, "batch, seqlen >= 0 and channels, ngroups, dstate > 0 required");
    if (channels % ngroups != 0)
        return fail(SSD_ERR_INVALID_ARG, "ngroups (%d) must divide channels (%d)", ngroups, channels);
    if (!ssd::selective_dstate_supported(dstate))
        return fail(SSD_ERR_UNSUPPORTED, "dstate must be 4, 8, 16 or 32 (got %d)", dstate);
    if (batch > 65535 || (long long)batch * seqlen > (1LL << 31))
        return fail(SSD_ERR_UNSUPPORTED, "sizes beyond the supported grid");
    if (batch == 0) return SSD_OK;
    if (!A || (seqlen > 0 && (!x || !dt || !B || !C || !y)))
        return fail(SSD_ERR_INVALID_ARG, "x, dt, A, B, C and y must be non-null");
    for (const void *p : {(const void *)x, (const void *)dt, (const void *)A, (const void *)B, (const void *)C,
                          (const void *)D, (const void *)init_state, (const void *)final_state, (const void *)y})
        if (p && !aligned16(p)) return fail(SSD_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (seqlen == 0) {
        e = final_state && final_state != init_state
                ? ssd::launch_copy_or_zero_state(init_state, final_state, (size_t)batch * channels * dstate, st)
                : cudaSuccess;
    } else {
        e = ssd::launch_selective_scan(x, dt, A, B, C, D, init_state, final_state, y, io_dtype == SSD_BF16, batch,
                                       seqlen, channels, ngroups, dstate, st);
    }
    if (e != cudaSuccess) return cuda_fail(e, "selective scan launch");
    return SSD_OK;
}

ssd_status ssd_state_update(float *state, const void *x, const float *dt, const float *A,
                            const void *B, const void *C, const float *D, void *y,
                            ssd_dtype io_dtype, int batch, int nheads, int headdim, int ngroups,
                            int dstate, void *stream) {
    if (!valid_dtype(io_dtype)) return fail(SSD_ERR_INVALID_ARG, "io_dtype must be SSD_F32 or SSD_BF16");
    return run_update(state, x, dt, A, B, C, D, y, io_dtype == SSD_BF16, false, batch, nheads, headdim,
                      ngroups, dstate, stream);
}

ssd_status ssd_state_update_complex(float *state, const float *x, const float *dt, const float *A,
                                    const float *B, const float *C, const float *D, float *y,
                                    int batch, int nheads, int headdim, int ngroups, int dstate,
                                    void *stream) {
    return run_update(state, x, dt, A, B, C, D, y, false, true, batch, nheads, headdim, ngroups,
                      dstate, stream);
}

size_t ssd_scan_bwd_workspace_size(int batch, int seqlen, int nheads, int headdim, int ngroups,
                                   int dstate) {
    if (check_scan_dims(batch, seqlen, nheads, headdim, ngroups, dstate, 64) != SSD_OK)
        return SSD_WORKSPACE_INVALID;
    if (!ssd::bwd_supported(headdim, dstate)) return SSD_WORKSPACE_INVALID;
    return ssd::bwd_workspace_bytes(batch, seqlen, nheads, headdim, ngroups, dstate);
}

size_t ssd_scan_bwd_complex_workspace_size(int batch, int seqlen, int nheads, int headdim, int ngroups,
                                           int dstate) {
    if (check_scan_dims(batch, seqlen, nheads, headdim, ngroups, dstate, 64) != SSD_OK)
        return SSD_WORKSPACE_INVALID;
    if (!ssd::bwd_complex_supported(headdim, dstate)) return SSD_WORKSPACE_INVALID;
    return ssd::bwd_complex_workspace_bytes(batch, seqlen, nheads, headdim, dstate);
}

ssd_status ssd_scan_bwd(const float *x, const float *dt, const float *A, const float *B,
                        const float *C, const float *D, const float *init_state, const float *dy,
                        const float *dfinal, float *dx, float *ddt, float *dA, float *dB, float *dC,
                        float *dD, float *dinit, int batch, int seqlen, int nheads, int headdim,
                        int ngroups, int dstate, void *workspace, size_t workspace_bytes, void *stream) {
    return run_bwd(false, x, dt, A, B, C, D, init_state, dy, dfinal, dx, ddt, dA, dB, dC, dD, dinit, batch,
                   seqlen, nheads, headdim, ngroups, dstate, workspace, workspace_bytes, stream);
}

ssd_status ssd_scan_bwd_complex(const float *x, const float *dt, const float *A, const float *B,
                                const float *C, const float *D, const float *init_state, const float *dy,
                                const float *dfinal, float *dx, float *ddt, float *dA, float *dB,
                                float *dC, float *dD, float *dinit, int batch, int seqlen, int nheads,
                                int headdim, int ngroups, int dstate, void *workspace,
                                size_t workspace_bytes, void *stream) {
    return run_bwd(true, x, dt, A, B, C, D, init_state, dy, dfinal, dx, ddt, dA, dB, dC, dD, dinit, batch,
                   seqlen, nheads, headdim, ngroups, dstate, workspace, workspace_bytes, stream);
}

ssd_status ssd_get_device_status(void *stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    int code = 0;
    e = cudaMemcpyFromSymbol(&code, g_ssd_device_error, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
    if (code == 0) return SSD_OK;
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_ssd_device_error, &zero, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "clearing the device error word");
    if (code == ssd::DEV_TIMEOUT)
        return fail(SSD_ERR_TIMEOUT, "a bounded inter-block wait gave up on the device; the "
                    "outputs of the call that raised it are invalid");
    return fail(SSD_ERR_CUDA, "device error code %d", code);
}

ssd_status ssd_debug_inject_stall(int withhold_first_load, unsigned long long wait_limit_ns) {
    ssd::set_tc_fault_injection(withhold_first_load, wait_limit_ns);
    return SSD_OK;
}

const char *ssd_last_error(void) { return g_last_error.c_str(); }

const char *ssd_version(void) { return "ssd-b200 0.1 (sm_100a)"; }

}  // extern "C"
