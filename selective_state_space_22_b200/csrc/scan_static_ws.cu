// scan_static_ws.cu -- ssd_scan_fwd_noalloc: the real scan for callers that
// cannot allocate device memory.
//
// Some callers have no way to hand the library a workspace.  A plugin loaded
// into a host application that owns all device memory (an inference server, a
// framework's custom-op slot) may be forbidden to call cudaMalloc after start-up;
// a real-time path may not afford an allocation's latency or its possible
// device-wide synchronisation; and a caller that never allocates must still get
// the scan's scratch from somewhere.  For them this entry point keeps its scratch
// in a fixed array that lives in the library's own device image: loading the
// library reserves it on every GPU that uses it, until the process exits, and no
// call ever allocates or frees anything.
//
// It runs the float32 CUDA-core scan (the same kernels ssd_scan_fwd uses for
// float32 inputs and for shapes the tensor-core kernel does not take), so its
// scratch holds, per (batch, head, chunk), the cumulative log-decays and one
// chunk state.  That bounds the problem size it accepts: see
// SSD_NOALLOC_SCRATCH_BYTES in include/ssd.h.
#include <stdarg.h>
#include <stdint.h>
#include <stdio.h>

#include <mutex>

#include "../../include/ssd.h"
#include "ssd_internal.cuh"

// The shared scratch.  Every call uses it from the start; calls that overlap on
// the GPU (different streams, or different host threads) race on it.
static __device__ __align__(256) unsigned char g_noalloc_scratch[SSD_NOALLOC_SCRATCH_BYTES];
// Device error word for this entry point's kernels (they never raise one).
static __device__ int g_noalloc_error = 0;

namespace {

// Errors are reported through ssd_last_error(), like every other entry point.
ssd_status set_msg(ssd_status s, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
ssd_status set_msg(ssd_status s, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    ssd::set_last_error(buf);
    return s;
}

// Device addresses of the two device globals, looked up once per (device,
// context) with that device current.  In host code the symbols themselves are
// host-side stand-ins and must never be handed to a kernel.
struct DevPtrs {
    void *ctx = nullptr;
    void *scratch = nullptr;
    int *err = nullptr;
};
DevPtrs g_ptrs[64];
std::mutex g_mu;

ssd_status device_ptrs(DevPtrs *out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return set_msg(SSD_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= 64) return set_msg(SSD_ERR_UNSUPPORTED, "device index %d out of range", dev);
    void *ctx = ssd::current_context();
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_ptrs[dev].scratch || g_ptrs[dev].ctx != ctx) {
        void *s = nullptr, *er = nullptr;
        e = cudaGetSymbolAddress(&s, g_noalloc_scratch);
        if (e != cudaSuccess)
            return set_msg(SSD_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
        e = cudaGetSymbolAddress(&er, g_noalloc_error);
        if (e != cudaSuccess)
            return set_msg(SSD_ERR_CUDA, "cudaGetSymbolAddress(error word): %s", cudaGetErrorString(e));
        g_ptrs[dev].ctx = ctx;
        g_ptrs[dev].scratch = s;
        g_ptrs[dev].err = static_cast<int *>(er);
    }
    *out = g_ptrs[dev];
    return SSD_OK;
}

bool al16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" ssd_status ssd_scan_fwd_noalloc(const void *x, const float *dt, const float *A, const void *B,
                                           const void *C, const float *D, const float *init_state,
                                           float *final_state, void *y, ssd_dtype io_dtype, int batch,
                                           int seqlen, int nheads, int headdim, int ngroups, int dstate,
                                           int chunk_size, void *stream) {
    if (io_dtype != SSD_F32 && io_dtype != SSD_BF16)
        return set_msg(SSD_ERR_INVALID_ARG, "io_dtype must be SSD_F32 or SSD_BF16");
    if (batch <= 0 || seqlen <= 0)
        return set_msg(SSD_ERR_INVALID_ARG, "batch (%d) and seqlen (%d) must be > 0", batch, seqlen);
    if (nheads <= 0 || headdim <= 0 || ngroups <= 0 || dstate <= 0)
        return set_msg(SSD_ERR_INVALID_ARG, "nheads, headdim, ngroups and dstate must be > 0");
    if (nheads % ngroups != 0)
        return set_msg(SSD_ERR_INVALID_ARG, "ngroups (%d) must divide nheads (%d)", ngroups, nheads);
    if (chunk_size != 64 && chunk_size != 128 && chunk_size != 256)
        return set_msg(SSD_ERR_INVALID_ARG, "chunk_size must be 64, 128 or 256 (got %d)", chunk_size);
    if (headdim > 256 || dstate > 256 || nheads > 65535 || batch > 2048)
        return set_msg(SSD_ERR_UNSUPPORTED, "headdim and dstate must be <= 256, nheads <= 65535, batch <= 2048");
    if (!x || !dt || !A || !B || !C || !y)
        return set_msg(SSD_ERR_INVALID_ARG, "x, dt, A, B, C and y must be non-null");
    const void *ptrs[] = {x, dt, A, B, C, y, D, init_state, final_state};
    for (const void *p : ptrs)
        if (p && !al16(p)) return set_msg(SSD_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
    const int nchunks = (seqlen + chunk_size - 1) / chunk_size;
    const size_t need = ssd::generic_workspace_bytes(batch, nheads, headdim, dstate, chunk_size, nchunks, false);
    if (need > (size_t)SSD_NOALLOC_SCRATCH_BYTES)
        return set_msg(SSD_ERR_WORKSPACE,
                       "these sizes need %zu bytes of scratch; ssd_scan_fwd_noalloc has %zu "
                       "(use ssd_scan_fwd with a caller-provided workspace)",
                       need, (size_t)SSD_NOALLOC_SCRATCH_BYTES);
    DevPtrs dp;
    ssd_status s = device_ptrs(&dp);
    if (s != SSD_OK) return s;

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
    a.chunk = chunk_size;
    a.nchunks = nchunks;
    a.dev_error = dp.err;
    // The kernels write every scratch value before reading it: nothing to clear.
    cudaError_t e = ssd::launch_generic_scan(a, false, io_dtype == SSD_BF16, dp.scratch,
                                             static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return set_msg(SSD_ERR_CUDA, "scan launch: %s", cudaGetErrorString(e));
    return SSD_OK;
}
