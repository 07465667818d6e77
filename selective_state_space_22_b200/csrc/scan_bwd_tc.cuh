// scan_bwd_tc.cuh -- the two per-chunk contractions of the real backward that
// have the shape of a chunk state, on tcgen05 (sm_100a), for head dim 64 and
// d_state 128:
//   chunk state   S[p][n] = sum_s w_s x_s[p] B_s[n],  w_s = exp(lam - acs[s]) dt_s
//   readout       R[p][n] = sum_l e_l dy_l[p] C_l[n], e_l = exp(acs[l])
// ("Block Anatomy, Numerical Stability & Scaling", Numerical Stability section 4:
// the chunk states; section 5.3: the backward runs through the same exp products.)
// One CTA of 128 threads per (64-token chunk, head, batch).  The rows [tokens][n]
// (B or C) are the MMA's A operand, MN-major, and the scaled rows [tokens][p]
// (w x or e dy) its B operand, MN-major; M = n (128, the TMEM lanes), N = p (64
// columns), K = the chunk's 64 tokens.  Float32 accuracy from bf16 operands: each
// value is split into hi + lo (16 significant bits) and the product is
// hi.hi + hi.lo + lo.hi, accumulated in float32 in TMEM.  The chunk-state kernel
// also forms the chunk's cumulative decay (a warp scan) and writes acs and lam
// for the later phases.
#pragma once

#include <cuda_bf16.h>

#include "scan_bwd_body.cuh"
#include "scan_bwd_complex_body.cuh"
#include "ssd_internal.cuh"
#include "tc_ptx.cuh"

namespace ssd {
namespace bwdtc {

using namespace ptx;

constexpr int Q = bwd::QB;   // 64 tokens per chunk
constexpr int PD = 64;       // head dim of this path
constexpr int ND = 128;      // d_state of this path
constexpr int NTH = 128;
// Shared memory: the [tokens][n] rows as two 64-column halves of [64][128 B]
// (hi, then lo), the scaled [tokens][p] rows [64][128 B] (hi, then lo).
constexpr int O_AH = 0, O_AL = 16384, O_BH = 32768, O_BL = 40960, O_MISC = 49152;
constexpr int SMEM = O_MISC + 3 * Q * 4 + 64 + 1024;
constexpr uint32_t IDESC = idesc_bf16_f32(128, 64, 1, 1);
constexpr unsigned long long WAIT_NS = 1000000000ull;

// Byte offset of 16-byte chunk ch (8 bf16) of row r in a tile of 128-byte
// swizzled rows, the 64-column halves half_bytes apart.
__device__ __forceinline__ uint32_t swz(int r, int ch, int half_bytes) {
    return (uint32_t)((ch >> 3) * half_bytes + r * 128 + (((ch & 7) ^ (r & 7)) << 4));
}
// Eight floats -> bf16 hi and lo parts at sm + hi_off + o and sm + lo_off + o.
__device__ __forceinline__ void put_split8(uint8_t *sm, int hi_off, int lo_off, uint32_t o, const float (&v)[8]) {
    uint32_t h[4], l[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const __nv_bfloat162 hh = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
        const float2 hf = __bfloat1622float2(hh);
        const __nv_bfloat162 ll = __floats2bfloat162_rn(v[2 * e] - hf.x, v[2 * e + 1] - hf.y);
        h[e] = *reinterpret_cast<const uint32_t *>(&hh);
        l[e] = *reinterpret_cast<const uint32_t *>(&ll);
    }
    *reinterpret_cast<uint4 *>(sm + hi_off + o) = make_uint4(h[0], h[1], h[2], h[3]);
    *reinterpret_cast<uint4 *>(sm + lo_off + o) = make_uint4(l[0], l[1], l[2], l[3]);
}
__device__ __forceinline__ unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// READOUT = false: the chunk state (and acs, lam); true: the readout terms.
template <bool READOUT>
__global__ void __launch_bounds__(NTH) chunk_product_kernel(bwd::BwdArgs a) {
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = bwd::group_of(a, h), t0 = c * Q, valid = min(Q, a.seqlen - t0);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *scale = reinterpret_cast<float *>(sm + O_MISC);  // [Q]: w_s or e_l
    float *acs = scale + Q;                                  // [Q]
    float *wtot = acs + Q;                                   // [2]
    uint64_t *bar = reinterpret_cast<uint64_t *>(wtot + Q);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bar + 1);
    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tslot, 64);
        tmem_relinquish();
    }
    // Every row load of the chunk goes in flight first (into registers; nothing
    // below waits on them until the conversion), then the decays are formed.
    const float *rows_n = READOUT ? a.C : a.B;   // [tokens][n]: B or C
    const float *rows_p = READOUT ? a.dy : a.x;  // [tokens][p]: x or dy
    constexpr int IA = Q * 16 / NTH, IB = Q * 8 / NTH;
    float4 ra[IA][2], rb[IB][2];
#pragma unroll
    for (int it = 0; it < IA; ++it) {
        const int u = tid + it * NTH, r = u >> 4, ch = u & 15;
        ra[it][0] = ra[it][1] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (r < valid) {
            const float *src = rows_n + bwd::ix_bc(a, b, t0 + r, g, 8 * ch);
            ra[it][0] = __ldg(reinterpret_cast<const float4 *>(src));
            ra[it][1] = __ldg(reinterpret_cast<const float4 *>(src + 4));
        }
    }
#pragma unroll
    for (int it = 0; it < IB; ++it) {
        const int u = tid + it * NTH, r = u >> 3, ch = u & 7;
        rb[it][0] = rb[it][1] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (r < valid) {
            const float *src = rows_p + bwd::ix_x(a, b, t0 + r, h, 8 * ch);
            rb[it][0] = __ldg(reinterpret_cast<const float4 *>(src));
            rb[it][1] = __ldg(reinterpret_cast<const float4 *>(src + 4));
        }
    }
    const size_t bh = bwd::ix_bh(a, b, h);
    float *acs_g = a.acs + (bh * a.nchunks + c) * Q;
    if constexpr (!READOUT) {
        // cumulative decay of the chunk: warps 0 and 1 scan 32 tokens each
        float d = 0.f, v = 0.f;
        if (tid < Q) {
            d = tid < valid ? __ldg(a.dt + bwd::ix_dt(a, b, t0 + tid, h)) : 0.f;
            v = d * __ldg(a.A + h);
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += y;
            }
            if (lane == 31) wtot[warp] = v;
        }
        __syncthreads();
        if (tid < Q) {
            if (warp == 1) v += wtot[0];
            acs[tid] = v;
            acs_g[tid] = v;
        }
        __syncthreads();
        const float lam = acs[Q - 1];
        if (tid < Q) scale[tid] = expf(lam - v) * d;
        if (tid == 0) a.lam[bh * a.nchunks + c] = lam;
    } else {
        if (tid < Q) scale[tid] = expf(__ldg(acs_g + tid));
    }
    __syncthreads();
    // operands as bf16 hi/lo: the [tokens][n] rows, and the [tokens][p] rows scaled
    // by w (chunk state) or e (readout); rows past the sequence are zeros
#pragma unroll
    for (int it = 0; it < IA; ++it) {
        const int u = tid + it * NTH, r = u >> 4, ch = u & 15;
        const float4 x0 = ra[it][0], x1 = ra[it][1];
        const float v8[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
        put_split8(sm, O_AH, O_AL, swz(r, ch, Q * 128), v8);
    }
#pragma unroll
    for (int it = 0; it < IB; ++it) {
        const int u = tid + it * NTH, r = u >> 3, ch = u & 7;
        const float f = scale[r];
        const float4 x0 = rb[it][0], x1 = rb[it][1];
        const float v8[8] = {f * x0.x, f * x0.y, f * x0.z, f * x0.w, f * x1.x, f * x1.y, f * x1.z, f * x1.w};
        put_split8(sm, O_BH, O_BL, swz(r, ch, Q * 128), v8);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot, sb = smem_u32(sm);
    if (tid == 0) {
#pragma unroll 1
        for (int pass = 0; pass < 3; ++pass) {  // hi.hi + hi.lo + lo.hi
            const uint32_t aA = sb + (pass == 2 ? O_AL : O_AH), aB = sb + (pass == 1 ? O_BL : O_BH);
#pragma unroll 1
            for (int kk = 0; kk < Q / 16; ++kk)
                mma_ss(tmem, smem_desc_sw128(aA + kk * 2048, Q * 128, 1024), smem_desc_sw128(aB + kk * 2048, Q * 128, 1024),
                       IDESC, pass > 0 || kk > 0);
        }
        mma_commit(bar);
    }
    // bounded wait for the products (the device error word records a timeout)
    if (!mbar_try_wait(bar, 0)) {
        const unsigned long long w0 = globaltimer_ns();
        while (!mbar_try_wait(bar, 0))
            if (globaltimer_ns() - w0 > WAIT_NS) {
                atomicCAS(a.dev_error, 0, DEV_TIMEOUT);
                break;
            }
    }
    tc_fence_after();
    {  // TMEM lane n = 32 warp + lane, columns p -> S[p][n] (or R)
        const int n = 32 * warp + lane;
        float *out = a.st + bwd::ix_pn(a, b, h, c) + n;
#pragma unroll 1
        for (int cb = 0; cb < PD; cb += 32) {
            uint32_t r[32];
            tmem_ld32(tmem + ((uint32_t)(32 * warp) << 16) + cb, r);
#pragma unroll
            for (int i = 0; i < 32; ++i) out[(size_t)(cb + i) * ND] = __uint_as_float(r[i]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 64);
}

// ------------------------------------------------------------ complex variant
// The same two contractions for the complex head (head dim 64, 64 complex states,
// 32-token chunks), as one real product each: with the complex weight folded into
// the complex rows, S[p][n] = sum_s x_s[p] (w_s B_s[n]) and
// R[p][n] = sum_l dy_l[p] conj(e_l C_l[n]) take M = the 128 interleaved (re, im)
// values of n, N = p, K = the chunk's 32 tokens; TMEM lane k = 2n + (re, im) is
// float k of row p of the interleaved result.
constexpr int QCX = bwdc::QC;  // 32 tokens
constexpr int NCX = 64;        // complex states of this path
constexpr int C_AH = 0, C_AL = 8192, C_BH = 16384, C_BL = 20480, C_MISC = 24576;
constexpr int CSMEM = C_MISC + 6 * QCX * 4 + 64 + 1024;

template <bool READOUT>
__global__ void __launch_bounds__(NTH) cplx_product_kernel(bwdc::BwdArgs a) {
    using bwdc::c2;
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = bwdc::group_of(a, h), t0 = c * QCX, valid = min(QCX, a.seqlen - t0);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *wgt = reinterpret_cast<float *>(sm + C_MISC);  // [QCX][2]: w_s, or e_l
    uint64_t *bar = reinterpret_cast<uint64_t *>(wgt + 6 * QCX);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bar + 1);
    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tslot, 64);
        tmem_relinquish();
    }
    // every row load in flight first: the complex rows [tokens][2N] (B or C) and
    // the real rows [tokens][p] (x or dy)
    const float *rows_n = READOUT ? a.C : a.B;
    const float *rows_p = READOUT ? a.dy : a.x;
    constexpr int IA = QCX * 32 / NTH, IB = QCX * 16 / NTH;  // 16-byte loads per thread
    float4 ra[IA], rb[IB];
#pragma unroll
    for (int it = 0; it < IA; ++it) {
        const int u = tid + it * NTH, r = u >> 5, q = u & 31;
        ra[it] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (r < valid) ra[it] = __ldg(reinterpret_cast<const float4 *>(rows_n + 2 * bwdc::ix_bc(a, b, t0 + r, g, 0) + 4 * q));
    }
#pragma unroll
    for (int it = 0; it < IB; ++it) {
        const int u = tid + it * NTH, r = u >> 4, q = u & 15;
        rb[it] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (r < valid) rb[it] = __ldg(reinterpret_cast<const float4 *>(rows_p + bwdc::ix_x(a, b, t0 + r, h, 4 * q)));
    }
    const size_t bh = bwdc::ix_bh(a, b, h);
    float *acs_g = a.acs + 2 * (bh * a.nchunks + c) * QCX;
    if constexpr (!READOUT) {
        // complex cumulative decay of the chunk (one warp), lam, w_s = exp(lam - acs_s) dt_s
        if (warp == 0) {
            const float d = lane < valid ? __ldg(a.dt + bwdc::ix_dt(a, b, t0 + lane, h)) : 0.f;
            float vr = d * __ldg(a.A + 2 * h), vi = d * __ldg(a.A + 2 * h + 1);
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float yr = __shfl_up_sync(0xffffffffu, vr, o), yi = __shfl_up_sync(0xffffffffu, vi, o);
                if (lane >= o) vr += yr, vi += yi;
            }
            acs_g[2 * lane] = vr;
            acs_g[2 * lane + 1] = vi;
            const float lr = __shfl_sync(0xffffffffu, vr, 31), li = __shfl_sync(0xffffffffu, vi, 31);
            if (lane == 0) {
                a.lam[2 * (bh * a.nchunks + c)] = lr;
                a.lam[2 * (bh * a.nchunks + c) + 1] = li;
            }
            const c2 wl = bwdc::cscale(bwdc::cexpc(c2{lr - vr, li - vi}), d);
            wgt[2 * lane] = wl.re;
            wgt[2 * lane + 1] = wl.im;
        }
    } else {
        if (tid < QCX) {
            const c2 e = bwdc::cexpc(c2{__ldg(acs_g + 2 * tid), __ldg(acs_g + 2 * tid + 1)});
            wgt[2 * tid] = e.re;  // e_l; the weighted row is conjugated below
            wgt[2 * tid + 1] = e.im;
        }
    }
    __syncthreads();
    // operands as bf16 hi/lo, 128-byte swizzled: the weighted complex rows (two
    // 64-float halves) and the real rows
#pragma unroll
    for (int it = 0; it < IA; ++it) {
        const int u = tid + it * NTH, r = u >> 5, q = u & 31;  // floats 4q .. 4q+3 = complex 2q, 2q+1
        const c2 wr = c2{wgt[2 * r], wgt[2 * r + 1]};
        const float4 v = ra[it];
        c2 z0 = bwdc::cmul(wr, c2{v.x, v.y}), z1 = bwdc::cmul(wr, c2{v.z, v.w});
        if (READOUT) z0 = bwdc::cconj(z0), z1 = bwdc::cconj(z1);  // conj(e_l C_l)
        const float f4v[4] = {z0.re, z0.im, z1.re, z1.im};
        // two 16-byte chunks (8 bf16) per 8 floats: this thread's 4 floats are half a chunk
        const int ch = q >> 1, part = q & 1;
        const uint32_t o = swz(r, ch, QCX * 128) + 8 * part;
        uint32_t hw[2], lw[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const __nv_bfloat162 hh = __floats2bfloat162_rn(f4v[2 * e], f4v[2 * e + 1]);
            const float2 hf = __bfloat1622float2(hh);
            const __nv_bfloat162 ll = __floats2bfloat162_rn(f4v[2 * e] - hf.x, f4v[2 * e + 1] - hf.y);
            hw[e] = *reinterpret_cast<const uint32_t *>(&hh);
            lw[e] = *reinterpret_cast<const uint32_t *>(&ll);
        }
        *reinterpret_cast<uint2 *>(sm + C_AH + o) = make_uint2(hw[0], hw[1]);
        *reinterpret_cast<uint2 *>(sm + C_AL + o) = make_uint2(lw[0], lw[1]);
    }
#pragma unroll
    for (int it = 0; it < IB; ++it) {
        const int u = tid + it * NTH, r = u >> 4, q = u & 15;
        const float4 v = rb[it];
        const float f4v[4] = {v.x, v.y, v.z, v.w};
        const int ch = q >> 1, part = q & 1;
        const uint32_t o = swz(r, ch, QCX * 128) + 8 * part;
        uint32_t hw[2], lw[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const __nv_bfloat162 hh = __floats2bfloat162_rn(f4v[2 * e], f4v[2 * e + 1]);
            const float2 hf = __bfloat1622float2(hh);
            const __nv_bfloat162 ll = __floats2bfloat162_rn(f4v[2 * e] - hf.x, f4v[2 * e + 1] - hf.y);
            hw[e] = *reinterpret_cast<const uint32_t *>(&hh);
            lw[e] = *reinterpret_cast<const uint32_t *>(&ll);
        }
        *reinterpret_cast<uint2 *>(sm + C_BH + o) = make_uint2(hw[0], hw[1]);
        *reinterpret_cast<uint2 *>(sm + C_BL + o) = make_uint2(lw[0], lw[1]);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot, sb = smem_u32(sm);
    if (tid == 0) {
#pragma unroll 1
        for (int pass = 0; pass < 3; ++pass) {  // hi.hi + hi.lo + lo.hi
            const uint32_t aA = sb + (pass == 2 ? C_AL : C_AH), aB = sb + (pass == 1 ? C_BL : C_BH);
#pragma unroll 1
            for (int kk = 0; kk < QCX / 16; ++kk)
                mma_ss(tmem, smem_desc_sw128(aA + kk * 2048, QCX * 128, 1024),
                       smem_desc_sw128(aB + kk * 2048, QCX * 128, 1024), IDESC, pass > 0 || kk > 0);
        }
        mma_commit(bar);
    }
    if (!mbar_try_wait(bar, 0)) {
        const unsigned long long w0 = globaltimer_ns();
        while (!mbar_try_wait(bar, 0))
            if (globaltimer_ns() - w0 > WAIT_NS) {
                atomicCAS(a.dev_error, 0, DEV_TIMEOUT);
                break;
            }
    }
    tc_fence_after();
    {  // TMEM lane k = 2n + (re, im), columns p -> float k of row p of the [P][N] pairs
        const int k = 32 * warp + lane;
        float *out = a.st + 2 * bwdc::ix_pn(a, b, h, c) + k;
#pragma unroll 1
        for (int cb = 0; cb < PD; cb += 32) {
            uint32_t r[32];
            tmem_ld32(tmem + ((uint32_t)(32 * warp) << 16) + cb, r);
#pragma unroll
            for (int i = 0; i < 32; ++i) out[(size_t)(cb + i) * 2 * NCX] = __uint_as_float(r[i]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 64);
}

}  // namespace bwdtc
}  // namespace ssd
