// scan_complex_tc.cuh -- the complex chunked scan's two heavy steps on tcgen05
// tensor cores (included by scan_complex.cu, inside namespace ssd).
//
// The Mamba-3-Lite head (head dim 64, 64 complex states), 128-token chunks.
// Every contraction is a real product over the 2N = 128 interleaved (re, im)
// values, as in the CUDA-core kernels, with the complex decay folded into the
// operands:
//
//   chunk state   S = sum_s w_s x_s B_s,  w_s = exp(Lam - A_cs[s]) dt_s
//                 as B''^T X with B''_s = w_s B_s            (M = 2N, N = P, K = 128)
//   diagonal      Re(G o L)[l, s] = Re(C'_l . B'_s) with
//                 C'_l = C_l exp(A_cs[l] - rho), B'_s = B_s exp(rho - A_cs[s]) dt_s,
//                 rho = Re(Lam) / 2 on the real part only       (M = N = 128, K = 2N)
//   off-diagonal  Re(exp(A_cs[l]) C_l . h_in) = Re(C'_l . exp(rho) h_in)
//   y             = M X + C' h'^T,  M = that masked product + D on the diagonal
//
// ("Block Anatomy, Numerical Stability & Scaling", Block Anatomy 4.3-4.4 and 6;
// Numerical Stability 4.)  Each factor stays within exp(+-70) while the chunk's
// real log-decay span |Re Lam| is at most 140; steeper chunks run the CUDA-core
// per-element tile code instead.  The inputs are float32, and the tolerance asked
// of them is 1e-4, beyond bf16: every operand is split into bf16 hi + lo
// (hi = bf16(v), lo = bf16(v - hi), together 16 significant bits) and every
// product runs as hi.hi + hi.lo + lo.hi with float32 accumulation in TMEM.
namespace ctc {
using namespace ptx;

constexpr int QT = 128;         // tokens per chunk (tcgen05 M)
constexpr int NTH = 256;
constexpr double SPAN = 140.0;  // |Re Lam| bound of the factored form

// chunk scan: shared memory (1024-aligned tiles, 128-byte swizzled rows).  The
// contraction over k = 2N runs in two halves of 64, so each operand tile holds
// one half; X later reuses the C' tiles.  About 83 KB, so two CTAs share an SM.
constexpr int S_CH = 0, S_CL = 16384;       // C'  [128 l][64 k], hi and lo
constexpr int S_BH = 32768, S_BL = 49152;   // B'  [128 s][64 k]
constexpr int S_HH = 65536, S_HL = 73728;   // h'  [64 p][64 k]
constexpr int S_XH = 0, S_XL = 16384;       // X   [128 s][64 p], after the products have read C'
constexpr int S_MISC = 81920;
constexpr int SMEM_SCAN = S_MISC + QT * 16 + 64 + 1024;
static_assert(2 * (SMEM_SCAN + 1024) <= 233472, "two CTAs per SM");
// chunk state: B'' [64 s][128 k] and X [64 s][64 p], hi and lo: the contraction
// over the chunk's tokens runs in two halves of 64, so four CTAs share an SM.
constexpr int HT = 64;  // tokens per half
constexpr int A_BH = 0, A_BL = 16384, A_XH = 32768, A_XL = 40960, A_MISC = 49152;
constexpr int SMEM_STATE = A_MISC + QT * (16 + 4 + 8) + 64 + 1024;
static_assert(4 * (SMEM_STATE + 1024) <= 233472, "four CTAs per SM");

constexpr uint32_t IDESC_G = idesc_bf16_f32(128, 128, 0, 0);   // C' (K-major) x B' (K-major)
constexpr uint32_t IDESC_H = idesc_bf16_f32(128, 64, 0, 0);    // C' (K-major) x h' (K-major)
constexpr uint32_t IDESC_MX = idesc_bf16_f32(128, 64, 0, 1);   // M (TMEM) x X (MN-major)
constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 64, 1, 1);    // B''^T (MN-major) x X (MN-major)
constexpr unsigned long long WAIT_NS = 1000000000ull;

// Byte offset of 16-byte chunk ch (8 bf16) of a row in a tile of 128-byte
// swizzled rows; half_bytes = rows * 128 (the size of one 64-column half).
__device__ __forceinline__ uint32_t sw_off(int row, int ch, int half_bytes) {
    return (uint32_t)((ch >> 3) * half_bytes + row * 128 + (((ch & 7) ^ (row & 7)) << 4));
}
__device__ __forceinline__ uint32_t bf2_bits(__nv_bfloat162 v) { return *reinterpret_cast<uint32_t *>(&v); }
// Eight floats -> their bf16 hi and lo parts (v = hi + lo to 16 significant bits).
__device__ __forceinline__ void split8(const float (&v)[8], uint4 &hi, uint4 &lo) {
    uint32_t h[4], l[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const __nv_bfloat162 hh = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
        const float2 hf = __bfloat1622float2(hh);
        h[e] = bf2_bits(hh);
        l[e] = bf2_bits(__floats2bfloat162_rn(v[2 * e] - hf.x, v[2 * e + 1] - hf.y));
    }
    hi = make_uint4(h[0], h[1], h[2], h[3]);
    lo = make_uint4(l[0], l[1], l[2], l[3]);
}
__device__ __forceinline__ void put8(uint8_t *sm, int off_hi, int off_lo, uint32_t o, const float (&v)[8]) {
    uint4 hi, lo;
    split8(v, hi, lo);
    *reinterpret_cast<uint4 *>(sm + off_hi + o) = hi;
    *reinterpret_cast<uint4 *>(sm + off_lo + o) = lo;
}

__device__ __forceinline__ unsigned long long now_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}
// Bounded wait on phase 0 of an mbarrier; the device error word records a timeout.
__device__ bool wait_bounded(uint64_t *bar, uint32_t parity, int *err) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = now_ns();
    while (!mbar_try_wait(bar, parity))
        if (now_ns() - t0 > WAIT_NS) {
            atomicCAS(err, 0, DEV_TIMEOUT);
            return false;
        }
    return true;
}

// X of the chunk into shared memory as bf16 hi/lo rows [s][p].
template <typename T>
__device__ void stage_x(uint8_t *sm, int off_hi, int off_lo, const ScanArgs &a, const CplxView<T> &v, size_t bt0, int h,
                        int valid) {
#pragma unroll 4
    for (int it = 0; it < QT * 8 / NTH; ++it) {
        const int u = threadIdx.x + it * NTH, s = u >> 3, ch = u & 7;
        float val[8];
        if (s < valid) {
            view_x8(v, bt0 + s, h, a.headdim, 8 * ch, val);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) val[e] = 0.f;
        }
        put8(sm, off_hi, off_lo, sw_off(s, ch, QT * 128), val);
    }
}

// ------------------------------------------------------------ chunk state
template <typename T> __global__ void __launch_bounds__(NTH, 4) state_kernel(ScanArgs a, CWs w, CplxView<T> v) {
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z, H = a.nheads, P = a.headdim, N = a.dstate;
    const int g = h / (H / a.ngroups), t0 = c * QT, valid = min(QT, a.seqlen - t0);
    const size_t bhc = ((size_t)b * H + h) * a.nchunks + c, bt0 = (size_t)b * a.seqlen + t0;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float2 *wf = reinterpret_cast<float2 *>(sm + A_MISC);  // [128] complex weights
    float *dts = reinterpret_cast<float *>(wf + QT);
    double *cre = reinterpret_cast<double *>(dts + QT), *cim = cre + QT;
    uint64_t *bar = reinterpret_cast<uint64_t *>(cim + QT);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bar + 2);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tslot, 64);
        tmem_relinquish();
    }
    chunk_log_decay(a, v, b, h, c, dts, cre, cim);  // ends with a block barrier
    const double R = cre[QT - 1], Th = cim[QT - 1];
    // The chunk scan's per-token factors go to the chunk's log-decay slot (2 x 128
    // float2 in the place of 2 x 128 doubles): C' = exp(A_cs - rho) and
    // B' = exp(rho - A_cs) dt, rho = R / 2.  A chunk too steep for that form keeps
    // its cumulative log-decays there for the CUDA-core tile code.  Threads below
    // QT take C' and B', the others the chunk-state weights.
    const bool steep = fabs(R) > SPAN;
    float2 *fac = reinterpret_cast<float2 *>(w.cs + (bhc * 2) * QT);
    for (int u = tid; u < 2 * QT; u += NTH) {
        const int s = u & (QT - 1);
        double sn, cn;
        if (u >= QT) {
            sincos(Th - cim[s], &sn, &cn);
            const float m = (float)exp(R - cre[s]) * dts[s];
            wf[s] = make_float2(m * (float)cn, m * (float)sn);
        } else if (steep) {
            w.cs[(bhc * 2) * QT + s] = cre[s];
            w.cs[(bhc * 2 + 1) * QT + s] = cim[s];
        } else {
            const double rho = 0.5 * R;
            sincos(cim[s], &sn, &cn);
            const float ec = (float)exp(cre[s] - rho), eb = (float)exp(rho - cre[s]) * dts[s];
            fac[s] = make_float2(ec * (float)cn, ec * (float)sn);
            fac[QT + s] = make_float2(eb * (float)cn, -eb * (float)sn);
        }
    }
    if (tid == 0) {
        w.lam[bhc * 2] = R;
        w.lam[bhc * 2 + 1] = Th;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot, sb = smem_u32(sm);
#pragma unroll 1
    for (int th = 0; th < 2; ++th) {  // tokens 64 th .. 64 th + 63
        if (th == 1) {  // the first half's products have read the tiles
            wait_bounded(&bar[0], 0, a.dev_error);
            tc_fence_after();
        }
        // B''_s = w_s B_s as interleaved (re, im), rows s
#pragma unroll 4
        for (int it = 0; it < HT * 16 / NTH; ++it) {
            const int u = tid + it * NTH, sl = u >> 4, ch = u & 15, s = HT * th + sl;
            float val[8];
            cf bq[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
            if (s < valid) view_cplx4(v, v.bre, v.bim, bt0 + s, g, 4 * ch, bq);
            const float2 ws = wf[s];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const cf z = cmul(bq[q], cf{ws.x, ws.y});
                val[2 * q] = z.re;
                val[2 * q + 1] = z.im;
            }
            put8(sm, A_BH, A_BL, sw_off(sl, ch, HT * 128), val);
        }
        // X rows s as bf16 hi/lo
#pragma unroll 2
        for (int it = 0; it < HT * 8 / NTH; ++it) {
            const int u = tid + it * NTH, sl = u >> 3, ch = u & 7, s = HT * th + sl;
            float val[8];
            if (s < valid) {
                view_x8(v, bt0 + s, h, a.headdim, 8 * ch, val);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) val[e] = 0.f;
            }
            put8(sm, A_XH, A_XL, sw_off(sl, ch, HT * 128), val);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0) {
#pragma unroll 1
            for (int pass = 0; pass < 3; ++pass) {  // hi.hi + hi.lo + lo.hi
                const uint32_t aB = sb + (pass == 2 ? A_BL : A_BH), aX = sb + (pass == 1 ? A_XL : A_XH);
#pragma unroll 1
                for (int kk = 0; kk < HT / 16; ++kk)
                    mma_ss(tmem, smem_desc_sw128(aB + kk * 2048, HT * 128, 1024),
                           smem_desc_sw128(aX + kk * 2048, HT * 128, 1024), IDESC_S, th > 0 || pass > 0 || kk > 0);
            }
            mma_commit(&bar[th]);
        }
    }
    wait_bounded(&bar[1], 0, a.dev_error);
    tc_fence_after();
    {  // S[p][n] (complex) from TMEM lane k = 2n + (re, im), column p
        const int q = warp & 3, cb = 32 * (warp >> 2), k = 32 * q + lane;
        uint32_t r[32];
        tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + cb, r);
        float *S = reinterpret_cast<float *>(w.S + bhc * (size_t)P * N);
#pragma unroll
        for (int i = 0; i < 32; ++i) S[((size_t)(cb + i) * N + (k >> 1)) * 2 + (k & 1)] = __uint_as_float(r[i]);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 64);
}

// -------------------------------------------------------------- chunk scan
// TMEM (256 columns, so two CTAs share an SM): G in 0..127, overwritten in place
// by M's hi part (bf16 pairs, 0..63); y in 128..191; M's lo part in 192..255.
template <typename T>
__global__ void __launch_bounds__(NTH, 2) scan_kernel(ScanArgs a, CWs w, CplxView<T> v) {
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z, H = a.nheads, P = a.headdim, N = a.dstate;
    const int g = h / (H / a.ngroups), t0 = c * QT, valid = min(QT, a.seqlen - t0);
    const size_t bhc = ((size_t)b * H + h) * a.nchunks + c, bt0 = (size_t)b * a.seqlen + t0;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    // The first k half's C and B values go in flight before anything else: they
    // depend on nothing this kernel computes.
    constexpr int CBIT = QT * 8 / NTH;
    cf cq0[CBIT][4], bq0[CBIT][4];
#pragma unroll
    for (int it = 0; it < CBIT; ++it) {
        const int u = threadIdx.x + it * NTH, r = u >> 3, ch = u & 7;
#pragma unroll
        for (int q = 0; q < 4; ++q) cq0[it][q] = bq0[it][q] = cf{0.f, 0.f};
        if (r < valid) {
            view_cplx4(v, v.cre, v.cim, bt0 + r, g, 4 * ch, cq0[it]);
            view_cplx4(v, v.bre, v.bim, bt0 + r, g, 4 * ch, bq0[it]);
        }
    }
    const double Rr = w.lam[bhc * 2];
    if (fabs(Rr) > SPAN) {  // too steep for the factored form: the CUDA-core tile code
        grid_dep_wait();    // h_in is written by the state pass
        for (int rt = 0; rt * 64 < valid; ++rt) cplx_scan_tile<T>(a, w, v, b, h, c, rt, 0, sm);
        return;
    }
    float2 *fC = reinterpret_cast<float2 *>(sm + S_MISC), *fB = fC + QT;
    uint64_t *bars = reinterpret_cast<uint64_t *>(fB + QT);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + 3);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int i = 0; i < 3; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tslot, 256);
        tmem_relinquish();
    }
    const double rho = 0.5 * Rr;
    {  // C' and B' factors of the chunk, written by the chunk-state kernel
        const float2 *fac = reinterpret_cast<const float2 *>(w.cs + (bhc * 2) * QT);
        for (int u = tid; u < 2 * QT; u += NTH) fC[u] = __ldg(fac + u);  // fB = fC + QT
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *tslot, sb = smem_u32(sm);
    constexpr uint32_t COL_Y = 128, COL_MH = 0, COL_ML = 192;
    const float er = (float)exp(rho);
    const float *hin = reinterpret_cast<const float *>(w.S + bhc * (size_t)P * N);
    bool ok = true;
#pragma unroll
    for (int kh = 0; kh < 2; ++kh) {  // k = 64 kh .. 64 kh + 63: complex states 32 kh .. 32 kh + 31
        if (kh == 1) {  // the first half's products have read the tiles
            ok = wait_bounded(&bars[0], 0, a.dev_error) && ok;
            tc_fence_after();
        }
        // C' as (re, -im) and B' as (re, im), rows = tokens, 4 complex states per chunk of 8
#pragma unroll 4
        for (int it = 0; it < CBIT; ++it) {
            const int u = tid + it * NTH, r = u >> 3, cl = u & 7;
            float vc[8], vb[8];
            const float2 fc = fC[r], fb = fB[r];
            cf cq[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}}, bq[4] = {cq[0], cq[1], cq[2], cq[3]};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                cq[q] = cq0[it][q];
                bq[q] = bq0[it][q];
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const cf zc = cmul(cq[q], cf{fc.x, fc.y}), zb = cmul(bq[q], cf{fb.x, fb.y});
                vc[2 * q] = zc.re;
                vc[2 * q + 1] = -zc.im;
                vb[2 * q] = zb.re;
                vb[2 * q + 1] = zb.im;
            }
            const uint32_t o = sw_off(r, cl, QT * 128);
            put8(sm, S_CH, S_CL, o, vc);
            put8(sm, S_BH, S_BL, o, vb);
        }
        // h' = exp(rho) h_in as (re, im), rows p (h_in was written by earlier launches: read-only here;
        // the state pass that writes it may still be running until grid_dep_wait returns)
        if (kh == 0) grid_dep_wait();
#pragma unroll 2
        for (int it = 0; it < 64 * 8 / NTH; ++it) {
            const int u = tid + it * NTH, p = u >> 3, cl = u & 7, ch = 8 * kh + cl;
            float val[8];
            const float4 h0 = __ldg(reinterpret_cast<const float4 *>(hin + ((size_t)p * N + 4 * ch) * 2));
            const float4 h1 = __ldg(reinterpret_cast<const float4 *>(hin + ((size_t)p * N + 4 * ch) * 2 + 4));
            val[0] = er * h0.x, val[1] = er * h0.y, val[2] = er * h0.z, val[3] = er * h0.w;
            val[4] = er * h1.x, val[5] = er * h1.y, val[6] = er * h1.z, val[7] = er * h1.w;
            put8(sm, S_HH, S_HL, sw_off(p, cl, 64 * 128), val);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0) {
#pragma unroll 1
            for (int pass = 0; pass < 3; ++pass) {  // G = C' B'^T and y = C' h'^T, hi.hi + hi.lo + lo.hi
                const uint32_t aC = sb + (pass == 2 ? S_CL : S_CH), aB = sb + (pass == 1 ? S_BL : S_BH);
                const uint32_t aH = sb + (pass == 1 ? S_HL : S_HH);
#pragma unroll 1
                for (int kk = 0; kk < 4; ++kk) {
                    const uint32_t acc = kh > 0 || pass > 0 || kk > 0;
                    mma_ss(tm, smem_desc_sw128(aC + 32 * kk, 16, 1024), smem_desc_sw128(aB + 32 * kk, 16, 1024),
                           IDESC_G, acc);
                    mma_ss(tm + COL_Y, smem_desc_sw128(aC + 32 * kk, 16, 1024),
                           smem_desc_sw128(aH + 32 * kk, 16, 1024), IDESC_H, acc);
                }
            }
            mma_commit(&bars[kh]);
        }
        if (kh == 0) {  // the second half's C and B, in flight while the first half's products run
#pragma unroll
            for (int it = 0; it < CBIT; ++it) {
                const int u = tid + it * NTH, r = u >> 3, ch = 8 + (u & 7);
#pragma unroll
                for (int q = 0; q < 4; ++q) cq0[it][q] = bq0[it][q] = cf{0.f, 0.f};
                if (r < valid) {
                    view_cplx4(v, v.cre, v.cim, bt0 + r, g, 4 * ch, cq0[it]);
                    view_cplx4(v, v.bre, v.bim, bt0 + r, g, 4 * ch, bq0[it]);
                }
            }
        }
    }
    // Warps 4-7 load X of the chunk while the products run; it is written over
    // the C' tiles once they are done.
    constexpr int XIT = QT * 8 / (NTH - 128);
    float xr[XIT][8];
    if (warp >= 4) {
#pragma unroll
        for (int it = 0; it < XIT; ++it) {
            const int u = (tid - 128) + it * (NTH - 128), s = u >> 3, ch = u & 7;
            if (s < valid) {
                view_x8(v, bt0 + s, h, a.headdim, 8 * ch, xr[it]);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) xr[it][e] = 0.f;
            }
        }
    }
    ok = wait_bounded(&bars[1], 0, a.dev_error) && ok;  // every product of both halves is done
    tc_fence_after();
    if (warp < 4) {
        // M = the masked product + D on the diagonal, split into hi and lo, by the warp
        // of the rows' lane quadrant, blocks in order: M's hi block j lands on G
        // columns this thread has already read.
        const int q = warp;
        const uint32_t lo_ = (uint32_t)(32 * q) << 16;
        const float Dh = a.D ? a.D[h] : 0.f;
#pragma unroll 1
        for (int j = 0; j < 4; ++j) {
            uint32_t ph[16], pl[16];
            if (j > q) {
#pragma unroll
                for (int i = 0; i < 16; ++i) ph[i] = pl[i] = 0u;
            } else {
                uint32_t gr[32];
                tmem_ld32(tm + lo_ + 32 * j, gr);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    float m0 = __uint_as_float(gr[2 * i]), m1 = __uint_as_float(gr[2 * i + 1]);
                    if (j == q) {
                        m0 = (2 * i < lane) ? m0 : (2 * i == lane ? m0 + Dh : 0.f);
                        m1 = (2 * i + 1 < lane) ? m1 : (2 * i + 1 == lane ? m1 + Dh : 0.f);
                    }
                    const __nv_bfloat162 hh = __floats2bfloat162_rn(m0, m1);
                    const float2 hf2 = __bfloat1622float2(hh);
                    ph[i] = bf2_bits(hh);
                    pl[i] = bf2_bits(__floats2bfloat162_rn(m0 - hf2.x, m1 - hf2.y));
                }
            }
            tmem_st16(tm + lo_ + COL_MH + 16 * j, ph);
            tmem_st16(tm + lo_ + COL_ML + 16 * j, pl);
        }
        tmem_wait_st();
    } else {
        // X of the chunk as bf16 hi/lo rows [s][p], into the C' tiles
#pragma unroll
        for (int it = 0; it < XIT; ++it) {
            const int u = (tid - 128) + it * (NTH - 128), s = u >> 3, ch = u & 7;
            put8(sm, S_XH, S_XL, sw_off(s, ch, QT * 128), xr[it]);
        }
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
        if (ok) {
#pragma unroll 1
            for (int pass = 0; pass < 3; ++pass) {  // y += M X, hi.hi + hi.lo + lo.hi
                const uint32_t aM = tm + (pass == 2 ? COL_ML : COL_MH), aX = sb + (pass == 1 ? S_XL : S_XH);
#pragma unroll 1
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts(tm + COL_Y, aM + 8 * kk, smem_desc_sw128(aX + kk * 2048, 8192, 1024), IDESC_MX, 1);
            }
        }
        mma_commit(&bars[2]);
    }
    wait_bounded(&bars[2], 0, a.dev_error);
    tc_fence_after();
    {  // y rows: lane quadrant (warp & 3), columns 32 (warp >> 2) ..
        const int q = warp & 3, cb = 32 * (warp >> 2), l = 32 * q + lane;
        uint32_t r[32];
        tmem_ld32(tm + ((uint32_t)(32 * q) << 16) + COL_Y + cb, r);
        if (l < valid) {
            float *yrow = static_cast<float *>(a.y) + ((bt0 + l) * H + h) * P + cb;
#pragma unroll
            for (int i = 0; i < 8; ++i)
                reinterpret_cast<float4 *>(yrow)[i] = make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                                                  __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tm, 256);
}

}  // namespace ctc
