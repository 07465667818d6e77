// seqpar.cu -- the two small steps a sequence split across devices needs
// besides the scan itself.
//
// "Block Anatomy, Numerical Stability & Scaling" (Numerical Stability, section
// 4) carries a chunk's end state into every later chunk through the decay
// between them.  Cut a sequence into consecutive slices, one per device: slice
// j scanned from a zero state ends in S_j (slice 0 starts from the caller's
// initial state), and its total log-decay is Lam_j = A * sum of its dt.  The
// state entering slice r is then the ordered fold
//
//   h_0 = S_0,   h_j = exp(Lam_j) h_{j-1} + S_j,   entering state of slice r = h_{r-1},
//
// the inter-chunk recurrence applied at slice granularity.  Each device
// computes (S_j, Lam_j) with a state-only scan, the devices exchange them, and
// each folds the ones before it; its own slice is then scanned from that state.
//
//   log_decay_sum: Lam[b, h] = A[h] * sum_t dt[b, t, h]   (double accumulation)
//   fold_states:   the fold above, elementwise over [batch, heads, P, N]
#include "ssd_internal.cuh"

namespace ssd {
namespace {

// One block per (32 heads, batch); thread (x, y) sums tokens y, y + 8, ... of
// head h0 + x, so each row of 32 heads is read as one coalesced 128-byte line.
__global__ void __launch_bounds__(256) log_decay_sum_kernel(const float *__restrict__ dt, const float *__restrict__ A,
                                                           float *__restrict__ out, int seqlen, int nheads) {
    __shared__ double part[8][33];
    const int h = blockIdx.x * 32 + threadIdx.x, b = blockIdx.y;
    double acc = 0.0;
    if (h < nheads)
        for (int t = threadIdx.y; t < seqlen; t += 8) acc += dt[((size_t)b * seqlen + t) * nheads + h];
    part[threadIdx.y][threadIdx.x] = acc;
    __syncthreads();
    if (threadIdx.y == 0 && h < nheads) {
        double s = 0.0;
#pragma unroll
        for (int i = 0; i < 8; ++i) s += part[i][threadIdx.x];
        out[(size_t)b * nheads + h] = (float)(s * (double)A[h]);
    }
}

__global__ void fold_states_kernel(const float *__restrict__ states, const float *__restrict__ lam,
                                   int nstates, float *__restrict__ out, size_t n_per_state, int pn, size_t nbh) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n_per_state;
         i += (size_t)gridDim.x * blockDim.x) {
        const size_t bh = i / pn;
        float h = states[i];
        for (int j = 1; j < nstates; ++j) h = fmaf(__expf(lam[j * nbh + bh]), h, states[j * n_per_state + i]);
        out[i] = h;
    }
}

}  // namespace

cudaError_t launch_log_decay_sum(const float *dt, const float *A, float *out, int batch, int seqlen, int nheads,
                                 cudaStream_t st) {
    if (batch == 0 || nheads == 0) return cudaSuccess;
    dim3 grid((nheads + 31) / 32, batch), block(32, 8);
    log_decay_sum_kernel<<<grid, block, 0, st>>>(dt, A, out, seqlen, nheads);
    return cudaGetLastError();
}

cudaError_t launch_fold_states(const float *states, const float *lam, int nstates, float *out, int batch,
                               int nheads, int headdim, int dstate, cudaStream_t st) {
    const size_t nbh = (size_t)batch * nheads;
    const size_t n = nbh * headdim * dstate;
    if (n == 0) return cudaSuccess;
    size_t blocks = (n + 255) / 256;
    if (blocks > 8192) blocks = 8192;
    fold_states_kernel<<<(unsigned)blocks, 256, 0, st>>>(states, lam, nstates, out, n, headdim * dstate, nbh);
    return cudaGetLastError();
}

}  // namespace ssd
