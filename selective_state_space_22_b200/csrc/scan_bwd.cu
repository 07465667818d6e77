// scan_bwd.cu -- gradients of the real and complex scans (fp32), chunk by chunk.
//
// The arithmetic is in scan_bwd_body.cuh (and, for steps 1 and 3 at head dim 64,
// in the tcgen05 kernels of scan_bwd_tc.cuh); this file only launches it.  Six
// steps, seven launches (eight when the heads of a group share B and C: their
// C B^T per chunk is formed once, before step 5), run on the caller's stream:
//   1. chunk states S_c and the within-chunk cumulative decay      grid (chunks, heads, batch)
//   2. the state entering each chunk, h_in (a forward pass over chunks)   grid (heads, batch)
//   3. the readout terms R_c = sum_l exp(acs[l]) dy_l C_l^T         grid (chunks, heads, batch)
//   4. the gradient of the state leaving each chunk (a backward pass over
//      chunks), and dinit                                            grid (heads, batch)
//   5. dx, ddt and each head's dB, dC, dA, dD parts of one chunk    grid (chunks, heads, batch)
//   6. dB, dC summed over the heads of a group; dA, dD over batch and chunks
//      (two kernels)
// Sums run in a fixed order, so repeated calls give identical bits.  The complex
// variant (scan_bwd_complex_body.cuh) runs the same six steps on 32-token chunks.
#include <mutex>

#include "scan_bwd_body.cuh"
#include "scan_bwd_complex_body.cuh"
#include "scan_bwd_tc.cuh"
#include "ssd_internal.cuh"

namespace ssd {
namespace {

using namespace bwd;

constexpr size_t SMEM_BYTES = SMEM_FLOATS * sizeof(float);

__global__ void __launch_bounds__(NT) bwd_chunk_state(BwdArgs a) {
    extern __shared__ float sm[];
    const Smem m = smem_map(sm);
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
    k1_load(a, c, h, b, tid, m);
    __syncthreads();
    k1_cumsum(a, c, h, b, tid, m);
    __syncthreads();
    k1_state(a, c, h, b, tid, m);
}

__global__ void __launch_bounds__(NT) bwd_gram(BwdArgs a) {
    extern __shared__ float sm[];
    const Smem m = smem_map(sm);
    const int c = blockIdx.x, g = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
    kg_load(a, c, g, b, tid, m);
    __syncthreads();
    kg_gram(a, c, g, b, tid, m);
}

__global__ void __launch_bounds__(NT) bwd_state_fwd(BwdArgs a) {
    k2_pass(a, blockIdx.x, blockIdx.y, blockIdx.z, threadIdx.x);
}

__global__ void __launch_bounds__(NT) bwd_readout(BwdArgs a) {
    extern __shared__ float sm[];
    const Smem m = smem_map(sm);
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
    k3_load(a, c, h, b, tid, m);
    __syncthreads();
    k3_r(a, c, h, b, tid, m);
}

__global__ void __launch_bounds__(NT) bwd_state_bwd(BwdArgs a) {
    k4_pass(a, blockIdx.x, blockIdx.y, blockIdx.z, threadIdx.x);
}

__global__ void __launch_bounds__(NT) bwd_chunk_grad(BwdArgs a) {
    extern __shared__ float sm[];
    const Smem m = smem_map(sm);
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
    k5_load(a, c, h, b, tid, m);
    __syncthreads();
    k5_mats(a, tid, m);
    __syncthreads();
    k5_tokens(a, tid, m);
    __syncthreads();
    k5_gb(a, tid, m);
    __syncthreads();
    k5_db(a, c, h, b, tid, m);
    __syncthreads();
    k5_ksr(a, tid, m);
    __syncthreads();
    k5_dc(a, c, h, b, tid, m);
    __syncthreads();
    k5_f(a, tid, m);
    __syncthreads();
    k5_decay(a, c, h, b, tid, m);
    k5_dx(a, c, h, b, tid, m);
}

__global__ void __launch_bounds__(NT) bwd_group_sum(BwdArgs a, size_t total) {
    const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < total) k6_group(a, i);
}

__global__ void __launch_bounds__(NT) bwd_head_sum(BwdArgs a) {
    const int h = blockIdx.x * blockDim.x + threadIdx.x;
    if (h < a.nheads) k6_head(a, h);
}

// ------------------------------------------------------------- complex
constexpr size_t SMEM_BYTES_C = bwdc::SMEM_FLOATS * sizeof(float);

__global__ void __launch_bounds__(bwdc::NT) bwdc_chunk_state(bwdc::BwdArgs a) {
    extern __shared__ float sm[];
    const bwdc::Smem m = bwdc::smem_map(sm);
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
    bwdc::k1_load(a, c, h, b, tid, m);
    __syncthreads();
    bwdc::k1_cumsum(a, c, h, b, tid, m);
    __syncthreads();
    bwdc::k1_scale(a, tid, m);
    __syncthreads();
    bwdc::k1_state(a, c, h, b, tid, m);
}

__global__ void __launch_bounds__(bwdc::NT) bwdc_state_fwd(bwdc::BwdArgs a) {
    bwdc::k2_pass(a, blockIdx.x, blockIdx.y, blockIdx.z, threadIdx.x);
}

__global__ void __launch_bounds__(bwdc::NT) bwdc_readout(bwdc::BwdArgs a) {
    extern __shared__ float sm[];
    const bwdc::Smem m = bwdc::smem_map(sm);
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
    bwdc::k3_load(a, c, h, b, tid, m);
    __syncthreads();
    bwdc::k3_scale(a, tid, m);
    __syncthreads();
    bwdc::k3_r(a, c, h, b, tid, m);
}

__global__ void __launch_bounds__(bwdc::NT) bwdc_state_bwd(bwdc::BwdArgs a) {
    bwdc::k4_pass(a, blockIdx.x, blockIdx.y, blockIdx.z, threadIdx.x);
}

__global__ void __launch_bounds__(bwdc::NT) bwdc_chunk_grad(bwdc::BwdArgs a) {
    extern __shared__ float sm[];
    const bwdc::Smem m = bwdc::smem_map(sm);
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
    bwdc::k5_load(a, c, h, b, tid, m);
    __syncthreads();
    bwdc::k5_mats(a, tid, m);
    __syncthreads();
    bwdc::k5_tokens(a, tid, m);
    __syncthreads();
    bwdc::k5_bc(a, c, h, b, tid, m);
    __syncthreads();
    bwdc::k5_fk(a, tid, m);
    __syncthreads();
    bwdc::k5_decay(a, c, h, b, tid, m);
    bwdc::k5_dx(a, c, h, b, tid, m);
}

__global__ void __launch_bounds__(bwdc::NT) bwdc_group_sum(bwdc::BwdArgs a, size_t total) {
    const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < total) bwdc::k6_group(a, i);
}

__global__ void __launch_bounds__(bwdc::NT) bwdc_head_sum(bwdc::BwdArgs a) {
    const int h = blockIdx.x * blockDim.x + threadIdx.x;
    if (h < a.nheads) bwdc::k6_head(a, h);
}

// The shared-memory opt-in is per function, device and CUDA context: done[dev]
// holds the context it was last made in.
cudaError_t set_smem_attr(const void *const *fs, int nf, size_t bytes, void *(&done)[64]) {
    static std::mutex mu;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(mu);
    void *ctx = current_context();
    if (ctx && done[dev] == ctx) return cudaSuccess;
    for (int i = 0; i < nf; ++i) {
        e = cudaFuncSetAttribute(fs[i], cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
        if (e != cudaSuccess) return e;
    }
    done[dev] = ctx;
    return cudaSuccess;
}

}  // namespace

bool bwd_complex_supported(int headdim, int dstate) {
    return headdim >= 1 && headdim <= bwdc::P_MAX && dstate >= 1 && dstate <= bwdc::N_MAX;
}

size_t bwd_complex_workspace_bytes(int batch, int seqlen, int nheads, int headdim, int dstate) {
    const int nchunks = (seqlen + bwdc::QC - 1) / bwdc::QC;
    return bwdc::ws_floats(batch, seqlen, nheads, headdim, dstate, nchunks) * sizeof(float);
}

cudaError_t launch_scan_bwd_complex(const BwdCall &call, void *ws, cudaStream_t st) {
    bwdc::BwdArgs a{};
    a.x = call.x; a.dt = call.dt; a.A = call.A; a.B = call.B; a.C = call.C; a.D = call.D;
    a.init = call.init_state; a.dy = call.dy; a.dfinal = call.dfinal;
    a.dx = call.dx; a.ddt = call.ddt; a.dA = call.dA; a.dB = call.dB; a.dC = call.dC;
    a.dD = call.dD; a.dinit = call.dinit;
    a.batch = call.batch; a.seqlen = call.seqlen; a.nheads = call.nheads; a.headdim = call.headdim;
    a.ngroups = call.ngroups; a.dstate = call.dstate;
    a.nchunks = (call.seqlen + bwdc::QC - 1) / bwdc::QC;
    a.dev_error = call.dev_error;
    bwdc::carve(a, static_cast<float *>(ws));
    // head dim 64, 64 complex states: the chunk states and readout terms on tcgen05
    const bool tc = a.headdim == bwdtc::PD && a.dstate == bwdtc::NCX && a.dev_error;

    static void *attr_set[64] = {nullptr}, *attr_set_tc[64] = {nullptr};
    const void *fs[3] = {(const void *)bwdc_chunk_state, (const void *)bwdc_readout, (const void *)bwdc_chunk_grad};
    cudaError_t e = set_smem_attr(fs, 3, SMEM_BYTES_C, attr_set);
    if (e != cudaSuccess) return e;
    const void *ftc[2] = {(const void *)bwdtc::cplx_product_kernel<false>, (const void *)bwdtc::cplx_product_kernel<true>};
    if ((e = set_smem_attr(ftc, 2, bwdtc::CSMEM, attr_set_tc)) != cudaSuccess) return e;
    const int nt = bwdc::NT;
    const unsigned pn_blocks = (unsigned)(((size_t)a.headdim * a.dstate + nt - 1) / nt);
    if (a.batch > 0 && a.nchunks > 0) {
        const dim3 gc(a.nchunks, a.nheads, a.batch), gh(pn_blocks, a.nheads, a.batch);
        if (tc)
            bwdtc::cplx_product_kernel<false><<<gc, bwdtc::NTH, bwdtc::CSMEM, st>>>(a);
        else
            bwdc_chunk_state<<<gc, nt, bwdc::SMEM_FLOATS_K1 * sizeof(float), st>>>(a);
        bwdc_state_fwd<<<gh, nt, 0, st>>>(a);
        if (tc)
            bwdtc::cplx_product_kernel<true><<<gc, bwdtc::NTH, bwdtc::CSMEM, st>>>(a);
        else
            bwdc_readout<<<gc, nt, bwdc::SMEM_FLOATS_K3 * sizeof(float), st>>>(a);
        bwdc_state_bwd<<<gh, nt, 0, st>>>(a);
        bwdc_chunk_grad<<<gc, nt, SMEM_BYTES_C, st>>>(a);
        const size_t total = (size_t)a.batch * a.seqlen * a.ngroups * a.dstate;
        bwdc_group_sum<<<(unsigned)((total + nt - 1) / nt), nt, 0, st>>>(a, total);
    } else if (a.batch > 0) {  // empty sequences: dinit = dfinal (or zero)
        bwdc_state_bwd<<<dim3(pn_blocks, a.nheads, a.batch), nt, 0, st>>>(a);
    }
    bwdc_head_sum<<<(a.nheads + nt - 1) / nt, nt, 0, st>>>(a);
    return cudaGetLastError();
}

bool bwd_supported(int headdim, int dstate) {
    return headdim >= 1 && headdim <= P_MAX && dstate >= 1 && dstate <= N_MAX;
}

size_t bwd_workspace_bytes(int batch, int seqlen, int nheads, int headdim, int ngroups, int dstate) {
    const int nchunks = (seqlen + QB - 1) / QB;
    return ws_floats(batch, seqlen, nheads, headdim, ngroups, dstate, nchunks) * sizeof(float);
}

cudaError_t launch_scan_bwd(const BwdCall &call, void *ws, cudaStream_t st) {
    BwdArgs a{};
    a.x = call.x; a.dt = call.dt; a.A = call.A; a.B = call.B; a.C = call.C; a.D = call.D;
    a.init = call.init_state; a.dy = call.dy; a.dfinal = call.dfinal;
    a.dx = call.dx; a.ddt = call.ddt; a.dA = call.dA; a.dB = call.dB; a.dC = call.dC;
    a.dD = call.dD; a.dinit = call.dinit;
    a.batch = call.batch; a.seqlen = call.seqlen; a.nheads = call.nheads; a.headdim = call.headdim;
    a.ngroups = call.ngroups; a.dstate = call.dstate;
    a.nchunks = (call.seqlen + QB - 1) / QB;
    a.dev_error = call.dev_error;
    carve(a, static_cast<float *>(ws));
    // head dim 64, d_state 128: the chunk states and readout terms on tcgen05
    const bool tc = a.headdim == bwdtc::PD && a.dstate == bwdtc::ND && a.dev_error;

    // the shared-memory opt-in is per function, device and context
    static void *attr_ctx[64] = {nullptr};
    static std::mutex attr_mu;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    {
        std::lock_guard<std::mutex> lk(attr_mu);
        void *ctx = current_context();
        if (!ctx || attr_ctx[dev] != ctx) {
            for (const void *f : {(const void *)bwd_chunk_state, (const void *)bwd_readout,
                                  (const void *)bwd_chunk_grad, (const void *)bwd_gram}) {
                e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
                if (e != cudaSuccess) return e;
            }
            for (const void *f : {(const void *)bwdtc::chunk_product_kernel<false>,
                                  (const void *)bwdtc::chunk_product_kernel<true>}) {
                e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, bwdtc::SMEM);
                if (e != cudaSuccess) return e;
            }
            attr_ctx[dev] = ctx;
        }
    }
    const unsigned pn_blocks = (unsigned)(((size_t)a.headdim * a.dstate + NT - 1) / NT);
    if (a.batch > 0 && a.nchunks > 0) {
        const dim3 gc(a.nchunks, a.nheads, a.batch), gh(pn_blocks, a.nheads, a.batch);
        if (tc)
            bwdtc::chunk_product_kernel<false><<<gc, bwdtc::NTH, bwdtc::SMEM, st>>>(a);
        else
            bwd_chunk_state<<<gc, NT, SMEM_FLOATS_K1 * sizeof(float), st>>>(a);
        bwd_state_fwd<<<gh, NT, 0, st>>>(a);
        if (tc)
            bwdtc::chunk_product_kernel<true><<<gc, bwdtc::NTH, bwdtc::SMEM, st>>>(a);
        else
            bwd_readout<<<gc, NT, SMEM_FLOATS_K3 * sizeof(float), st>>>(a);
        bwd_state_bwd<<<gh, NT, 0, st>>>(a);
        if (a.gram) bwd_gram<<<dim3(a.nchunks, a.ngroups, a.batch), NT, SMEM_FLOATS_K3 * sizeof(float), st>>>(a);
        bwd_chunk_grad<<<gc, NT, SMEM_BYTES, st>>>(a);
        const size_t total = (size_t)a.batch * a.seqlen * a.ngroups * a.dstate;
        bwd_group_sum<<<(unsigned)((total + NT - 1) / NT), NT, 0, st>>>(a, total);
    } else if (a.batch > 0) {  // empty sequences: dinit = dfinal (or zero)
        bwd_state_bwd<<<dim3(pn_blocks, a.nheads, a.batch), NT, 0, st>>>(a);
    }
    bwd_head_sum<<<(a.nheads + NT - 1) / NT, NT, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace ssd
