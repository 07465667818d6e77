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


// ------------------------------------------- helpers of the persistent kernel
// One k half of operands (bf16 hi/lo, 128-byte swizzled rows): C' and B' [128][64],
// h' [64][64].
constexpr int PS_CH = 0, PS_CL = 16384, PS_BH = 32768, PS_BL = 49152, PS_HH = 65536, PS_HL = 73728;
constexpr int P_STAGE = 81920;

// Bounded wait; once any wait of the CTA has run out (abort word set), every
// later wait gives up at once, so the kernel ends promptly.
__device__ bool pwait(uint64_t *bar, uint32_t parity, volatile int *abort_s, int *err) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = now_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (*abort_s) return false;
        if (now_ns() - t0 > WAIT_NS) {
            atomicCAS(err, 0, DEV_TIMEOUT);
            *abort_s = 1;
            return false;
        }
    }
    return true;
}

// Chunk `it` of the flattened (batch, head, chunk) order, chunks fastest.
struct PItem {
    int b, h, c, g, valid;
    size_t bhc, bt0;
};
__device__ __forceinline__ PItem p_item(const ScanArgs &a, int it) {
    PItem r;
    r.c = it % a.nchunks;
    r.h = (it / a.nchunks) % a.nheads;
    r.b = it / (a.nchunks * a.nheads);
    r.g = r.h / (a.nheads / a.ngroups);
    r.valid = min(QT, a.seqlen - r.c * QT);
    r.bhc = ((size_t)r.b * a.nheads + r.h) * a.nchunks + r.c;
    r.bt0 = (size_t)r.b * a.seqlen + (size_t)r.c * QT;
    return r;
}
__device__ __forceinline__ bool p_steep(const CWs &w, size_t bhc) { return fabs(__ldg(w.lam + bhc * 2)) > SPAN; }

// ------------------------------------------------- TMA-fed persistent chunk scan
// The chunk scan of scan_kernel for float32 inputs in the plain layout, one CTA
// per SM looping over chunks, the operands' raw float32 tiles brought in by TMA
// (no registers held while they are in flight) and converted shared -> shared:
//   warp 13     TMA producer: per chunk, four k quarters (C and B [128 t][32],
//               h_in [64 p][32] floats) and then X [128 t][64], each into one of
//               two 40 KB raw stages
//   warps 4-11  converters: each quarter -> bf16 hi/lo operands (C' and B' with
//               the per-token factors, h' = e^rho h_in; 64-byte swizzled rows of
//               32 k values) in one of two operand stages; X -> one of two
//               hi/lo buffers
//   warp 12     MMA issuer: G and C' h'^T of chunk j (four quarters), then M X of
//               chunk j-1
//   warps 0-3   lane quadrant q = warp of TMEM: the M build of chunk j, then y of
//               chunk j-1
// (Fourteen warps: at most four per SM sub-partition, 128 registers each.)
// Chunks too steep for the factored form are skipped by every role alike and
// done by steep_chunks_kernel.
constexpr int TNTH = 448;
constexpr int TW_CONV = 4, TW_MMA = 12, TW_TMA = 13;
constexpr int T_RAWSZ = 40960;             // C quarter 16 KB, B quarter 16 KB, h quarter 8 KB; or X 32 KB
constexpr int T_OP = 2 * T_RAWSZ;          // two operand stages of one k quarter each:
constexpr int Q_CH = 0, Q_CL = 8192, Q_BH = 16384, Q_BL = 24576, Q_HH = 32768, Q_HL = 36864, T_OPSZ = 40960;
constexpr int T_X = T_OP + 2 * T_OPSZ;     // two X buffers of 32 KB: hi [128][64], then lo
constexpr int T_XSZ = 32768;
constexpr int T_MISC = T_X + 2 * T_XSZ;
enum { TB_RAWF = 0, TB_RAWE = 2, TB_OPF = 4, TB_OPE = 6, TB_XF = 8, TB_XE = 10, TB_GDONE = 12, TB_MDONE = 14,
       TB_YDONE = 16, TB_FREE = 18, TB_DRAIN = 20, TB_N = 21 };
// Byte offset of 16-byte chunk c (of 4) of row `row` in a tile of 64-byte rows,
// 64-byte swizzle.
__device__ __forceinline__ uint32_t sw64_off(int row, int c) { return (uint32_t)(row * 64 + ((c ^ ((row >> 1) & 3)) << 4)); }
constexpr int SMEM_TMA = T_MISC + TB_N * 8 + 16 + 1024;
static_assert(SMEM_TMA <= 232448, "one CTA per SM");
static_assert(T_OP % 1024 == 0 && T_OPSZ % 1024 == 0 && T_X % 1024 == 0, "swizzled tiles are 1024-byte aligned");

// The CTA's chunks blockIdx.x, blockIdx.x + gridDim.x, ... that the factored form
// takes, in order; the next chunk's log-decay is loaded one step ahead, so no
// role waits on a global load at the top of its loop.
struct PIter {
    int it, n, step;
    double lam_next;
    const CWs *w;
    const ScanArgs *a;
    __device__ PIter(const ScanArgs &a_, const CWs &w_) : it(blockIdx.x), step(gridDim.x), w(&w_), a(&a_) {
        n = a_.batch * a_.nheads * a_.nchunks;
        lam_next = it < n ? __ldg(w_.lam + p_item(a_, it).bhc * 2) : 0.0;
    }
    // the next chunk the factored form takes (false when none is left)
    __device__ bool next(PItem &t, double &lam) {
        while (it < n) {
            const int cur = it;
            lam = lam_next;
            it += step;
            if (it < n) lam_next = __ldg(w->lam + p_item(*a, it).bhc * 2);
            if (fabs(lam) <= SPAN) {
                t = p_item(*a, cur);
                return true;
            }
        }
        return false;
    }
};

__global__ void __launch_bounds__(TNTH, 1)
    scan_tma_kernel(const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_b,
                    const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_h, ScanArgs a,
                    CWs w) {
    const int P = a.headdim, H = a.nheads;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + T_MISC);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + TB_N);
    volatile int *abort_s = reinterpret_cast<volatile int *>(tslot + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars[TB_RAWF + i], 1);    // the producer's expect_tx
            mbar_init(&bars[TB_RAWE + i], 256);  // the converter threads
            mbar_init(&bars[TB_GDONE + i], 1);
            mbar_init(&bars[TB_MDONE + i], 128);
            mbar_init(&bars[TB_YDONE + i], 1);
            mbar_init(&bars[TB_FREE + i], 128);
            mbar_init(&bars[TB_XF + i], 256);
            mbar_init(&bars[TB_XE + i], 1);
            mbar_init(&bars[TB_OPF + i], 256);
            mbar_init(&bars[TB_OPE + i], 1);
        }
        mbar_init(&bars[TB_DRAIN], 1);
        *abort_s = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tslot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot, sb = smem_u32(sm);
    constexpr uint32_t COL_Y = 128, COL_MH = 0, COL_ML = 192;

    if (warp == TW_TMA) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            int r = 0;  // raw stages issued
            bool h_ready = false;
            PIter items(a, w);
            PItem t;
            double lam;
            while (!*abort_s && items.next(t, lam)) {
                bool ok = true;
                for (int u = 0; u < 5 && ok; ++u) {
                    const int slot = r & 1;
                    ok = pwait(&bars[TB_RAWE + slot], ((r >> 1) & 1) ^ 1, abort_s, a.dev_error);
                    if (!ok) break;  // nothing more is issued after an abort
                    uint8_t *dst = sm + slot * T_RAWSZ;
                    uint64_t *full = &bars[TB_RAWF + slot];
                    if (u < 4) {
                        if (!h_ready) {  // h_in is written by the state pass
                            grid_dep_wait();
                            h_ready = true;
                        }
                        mbar_arrive_expect_tx(full, T_RAWSZ);
                        tma_load_4d(dst, &tm_c, full, 32 * u, t.g, t.c * QT, t.b);
                        tma_load_4d(dst + 16384, &tm_b, full, 32 * u, t.g, t.c * QT, t.b);
                        tma_load_2d(dst + 32768, &tm_h, full, 32 * u, (int)(t.bhc * P));
                    } else {
                        mbar_arrive_expect_tx(full, QT * 64 * 4);
                        tma_load_4d(dst, &tm_x, full, 0, t.h, t.c * QT, t.b);
                    }
                    ++r;
                }
                if (!ok) break;
            }
            // every load issued has landed before the CTA's shared memory is released
            for (int slot = 0; slot < 2; ++slot)
                if (r - 1 >= slot) {
                    const int kl = r - 1 - ((r - 1 - slot) & 1);
                    const unsigned long long t0 = now_ns();
                    while (!mbar_try_wait(&bars[TB_RAWF + slot], (kl >> 1) & 1))
                        if (now_ns() - t0 > WAIT_NS) {
                            atomicCAS(a.dev_error, 0, DEV_TIMEOUT);
                            break;
                        }
                }
        }
    } else if (warp >= TW_CONV && warp < TW_MMA) {
        // -------------------------------------------------------- converters
        const int ct = tid - TW_CONV * 32;  // 0..255
        int r = 0, j = 0;
        PIter items(a, w);
        PItem t;
        double lam;
        const int r0 = ct >> 2;  // this thread's rows of C' and B': r0 and r0 + 64 in every quarter
        while (items.next(t, lam)) {
            const float2 *fac = reinterpret_cast<const float2 *>(w.cs + (t.bhc * 2) * QT);  // C' then B' factors
            const float2 fcr[2] = {__ldg(fac + r0), __ldg(fac + r0 + 64)};
            const float2 fbr[2] = {__ldg(fac + QT + r0), __ldg(fac + QT + r0 + 64)};
            const float er = (float)exp(0.5 * lam);
#pragma unroll 1
            for (int q = 0; q < 4; ++q) {
                const int o = 4 * j + q, os = o & 1, slot = r & 1;
                uint8_t *op = sm + T_OP + os * T_OPSZ;
                pwait(&bars[TB_RAWF + slot], (r >> 1) & 1, abort_s, a.dev_error);
                pwait(&bars[TB_OPE + os], ((o >> 1) & 1) ^ 1, abort_s, a.dev_error);  // quarter o-2 is done
                const float *raw = reinterpret_cast<const float *>(sm + slot * T_RAWSZ);
#pragma unroll
                for (int i = 0; i < 2; ++i) {  // C' as (re, -im) and B' as (re, im), rows = tokens
                    const int u = ct + 256 * i, row = u >> 2, c = u & 3;
                    const float4 c0 = *reinterpret_cast<const float4 *>(raw + row * 32 + 8 * c);
                    const float4 c1 = *reinterpret_cast<const float4 *>(raw + row * 32 + 8 * c + 4);
                    const float4 b0 = *reinterpret_cast<const float4 *>(raw + 4096 + row * 32 + 8 * c);
                    const float4 b1 = *reinterpret_cast<const float4 *>(raw + 4096 + row * 32 + 8 * c + 4);
                    const cf cq[4] = {{c0.x, c0.y}, {c0.z, c0.w}, {c1.x, c1.y}, {c1.z, c1.w}};
                    const cf bq[4] = {{b0.x, b0.y}, {b0.z, b0.w}, {b1.x, b1.y}, {b1.z, b1.w}};
                    const float2 fc = fcr[i], fb = fbr[i];  // row = r0 + 64 i
                    float vc[8], vb[8];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const cf zc = cmul(cq[e], cf{fc.x, fc.y}), zb = cmul(bq[e], cf{fb.x, fb.y});
                        vc[2 * e] = zc.re;
                        vc[2 * e + 1] = -zc.im;
                        vb[2 * e] = zb.re;
                        vb[2 * e + 1] = zb.im;
                    }
                    const uint32_t so = sw64_off(row, c);
                    put8(op, Q_CH, Q_CL, so, vc);
                    put8(op, Q_BH, Q_BL, so, vb);
                }
                {  // h' = exp(rho) h_in, rows p
                    const int p = ct >> 2, c = ct & 3;
                    const float4 h0 = *reinterpret_cast<const float4 *>(raw + 8192 + p * 32 + 8 * c);
                    const float4 h1 = *reinterpret_cast<const float4 *>(raw + 8192 + p * 32 + 8 * c + 4);
                    float val[8] = {er * h0.x, er * h0.y, er * h0.z, er * h0.w,
                                    er * h1.x, er * h1.y, er * h1.z, er * h1.w};
                    put8(op, Q_HH, Q_HL, sw64_off(p, c), val);
                }
                fence_proxy_async_smem();
                mbar_arrive(&bars[TB_OPF + os]);
                mbar_arrive(&bars[TB_RAWE + slot]);
                ++r;
            }
            {  // X of the chunk, rows s (rows past the sequence arrive as zeros)
                const int slot = r & 1;
                pwait(&bars[TB_RAWF + slot], (r >> 1) & 1, abort_s, a.dev_error);
                const int xb = j & 1;
                pwait(&bars[TB_XE + xb], ((j >> 1) & 1) ^ 1, abort_s, a.dev_error);  // M X of chunk j-2 is done
                const float *raw = reinterpret_cast<const float *>(sm + slot * T_RAWSZ);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int u = ct + 256 * i, s_ = u >> 3, ch = u & 7;
                    const float4 x0 = *reinterpret_cast<const float4 *>(raw + s_ * 64 + 8 * ch);
                    const float4 x1 = *reinterpret_cast<const float4 *>(raw + s_ * 64 + 8 * ch + 4);
                    float val[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
                    put8(sm, T_X + xb * T_XSZ, T_X + xb * T_XSZ + 16384, sw_off(s_, ch, QT * 128), val);
                }
                fence_proxy_async_smem();
                mbar_arrive(&bars[TB_XF + xb]);
                mbar_arrive(&bars[TB_RAWE + slot]);
                ++r;
            }
            ++j;
        }
    } else if (warp == TW_MMA) {
        // -------------------------------------------------------- MMA issuer
        if (lane == 0) {
            auto mx = [&](int jj) {  // y += M X of chunk jj, once M and X are in place
                const int s = jj & 1;
                const uint32_t tm = tmem + 256 * s;
                pwait(&bars[TB_MDONE + s], (jj >> 1) & 1, abort_s, a.dev_error);
                const int xb = jj & 1;
                pwait(&bars[TB_XF + xb], (jj >> 1) & 1, abort_s, a.dev_error);
                tc_fence_after();
                const uint32_t xh = sb + T_X + xb * T_XSZ;
#pragma unroll 1
                for (int pass = 0; pass < 3; ++pass) {  // hi.hi + hi.lo + lo.hi
                    const uint32_t aM = tm + (pass == 2 ? COL_ML : COL_MH), aX = xh + (pass == 1 ? 16384 : 0);
#pragma unroll 1
                    for (int kk = 0; kk < 8; ++kk)
                        mma_ts(tm + COL_Y, aM + 8 * kk, smem_desc_sw128(aX + kk * 2048, 8192, 1024), IDESC_MX, 1);
                }
                mma_commit(&bars[TB_YDONE + s]);
                mma_commit(&bars[TB_XE + xb]);
            };
            int j = 0;
            PIter items(a, w);
            PItem t;
            double lam;
            while (items.next(t, lam)) {
                const int s = j & 1;
                const uint32_t tm = tmem + 256 * s;
                pwait(&bars[TB_FREE + s], ((j >> 1) & 1) ^ 1, abort_s, a.dev_error);  // y of chunk j-2 is out
#pragma unroll 1
                for (int q = 0; q < 4; ++q) {
                    const int o = 4 * j + q, os = o & 1;
                    const uint32_t st = sb + T_OP + os * T_OPSZ;
                    pwait(&bars[TB_OPF + os], (o >> 1) & 1, abort_s, a.dev_error);
                    tc_fence_after();
#pragma unroll 1
                    for (int pass = 0; pass < 3; ++pass) {  // G = C' B'^T and y = C' h'^T, hi.hi + hi.lo + lo.hi
                        const uint32_t aC = st + (pass == 2 ? Q_CL : Q_CH), aB = st + (pass == 1 ? Q_BL : Q_BH);
                        const uint32_t aH = st + (pass == 1 ? Q_HL : Q_HH);
#pragma unroll 1
                        for (int kk = 0; kk < 2; ++kk) {
                            const uint32_t acc = q > 0 || pass > 0 || kk > 0;
                            mma_ss(tm, smem_desc_sw64(aC + 32 * kk, 16, 512), smem_desc_sw64(aB + 32 * kk, 16, 512),
                                   IDESC_G, acc);
                            mma_ss(tm + COL_Y, smem_desc_sw64(aC + 32 * kk, 16, 512),
                                   smem_desc_sw64(aH + 32 * kk, 16, 512), IDESC_H, acc);
                        }
                    }
                    mma_commit(&bars[TB_OPE + os]);
                }
                mma_commit(&bars[TB_GDONE + s]);
                if (j > 0) mx(j - 1);
                ++j;
            }
            if (j > 0) mx(j - 1);
            mma_commit(&bars[TB_DRAIN]);  // everything this thread issued is done before TMEM is freed
            const unsigned long long t0 = now_ns();
            while (!mbar_try_wait(&bars[TB_DRAIN], 0))
                if (now_ns() - t0 > WAIT_NS) {
                    atomicCAS(a.dev_error, 0, DEV_TIMEOUT);
                    break;
                }
        }
    } else if (warp < TW_CONV) {
        // ----------------------------------------------- M build and epilogue
        const int qd = warp, l = 32 * qd + lane;
        const uint32_t lo_ = (uint32_t)(32 * qd) << 16;
        auto epilogue = [&](int jj, const PItem &t) {
            const int s = jj & 1;
            const uint32_t tm = tmem + 256 * s;
            pwait(&bars[TB_YDONE + s], (jj >> 1) & 1, abort_s, a.dev_error);
            tc_fence_after();
#pragma unroll 1
            for (int cb = 0; cb < 64; cb += 32) {
                uint32_t rr[32];
                tmem_ld32(tm + lo_ + COL_Y + cb, rr);
                if (l < t.valid) {
                    float *yrow = static_cast<float *>(a.y) + ((t.bt0 + l) * H + t.h) * P + cb;
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        reinterpret_cast<float4 *>(yrow)[i] =
                            make_float4(__uint_as_float(rr[4 * i]), __uint_as_float(rr[4 * i + 1]),
                                        __uint_as_float(rr[4 * i + 2]), __uint_as_float(rr[4 * i + 3]));
                }
            }
            tc_fence_before();
            mbar_arrive(&bars[TB_FREE + s]);
        };
        int j = 0;
        PItem prev{}, t;
        double lam;
        PIter items(a, w);
        while (items.next(t, lam)) {
            const int s = j & 1;
            const uint32_t tm = tmem + 256 * s;
            const float Dh = a.D ? __ldg(a.D + t.h) : 0.f;
            pwait(&bars[TB_GDONE + s], (j >> 1) & 1, abort_s, a.dev_error);
            tc_fence_after();
#pragma unroll 1
            for (int jb = 0; jb < 4; ++jb) {  // M = masked product + D on the diagonal, as scan_kernel
                uint32_t ph[16], pl[16];
                if (jb > qd) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) ph[i] = pl[i] = 0u;
                } else {
                    uint32_t gr[32];
                    tmem_ld32(tm + lo_ + 32 * jb, gr);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        float m0 = __uint_as_float(gr[2 * i]), m1 = __uint_as_float(gr[2 * i + 1]);
                        if (jb == qd) {
                            m0 = (2 * i < lane) ? m0 : (2 * i == lane ? m0 + Dh : 0.f);
                            m1 = (2 * i + 1 < lane) ? m1 : (2 * i + 1 == lane ? m1 + Dh : 0.f);
                        }
                        const __nv_bfloat162 hh = __floats2bfloat162_rn(m0, m1);
                        const float2 hf2 = __bfloat1622float2(hh);
                        ph[i] = bf2_bits(hh);
                        pl[i] = bf2_bits(__floats2bfloat162_rn(m0 - hf2.x, m1 - hf2.y));
                    }
                }
                tmem_st16(tm + lo_ + COL_MH + 16 * jb, ph);
                tmem_st16(tm + lo_ + COL_ML + 16 * jb, pl);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars[TB_MDONE + s]);
            if (j > 0) epilogue(j - 1, prev);
            prev = t;
            ++j;
        }
        if (j > 0) epilogue(j - 1, prev);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 512);
}


// ----------------------------------------------- TMA-fed persistent chunk states
// state_kernel for float32 inputs in the plain layout, one CTA per SM looping
// over chunks (steep ones included):
//   warp 13     TMA producer: per chunk, four token quarters of B [32 t][128 floats]
//               and X [32 t][64], each into one of three 24 KB raw stages
//   warps 0-3   chunk j's decays (thread = token: the cumulative log-decay in
//               double, the weights w_s of B'', the chunk scan's factors and Lambda
//               into the workspace), then the state S of chunk j-1 out of TMEM
//   warps 4-11  converters: each quarter -> B'' = w B and X as bf16 hi/lo
//               (128-byte swizzled rows) in one of two operand stages
//   warp 12     MMA issuer: S = B''^T X over the four quarters, three passes
// Two TMEM column sets of 64 hold two chunks' states.
constexpr int SNTH = 448;
constexpr int SW_CONV = 4, SW_MMA = 12, SW_TMA = 13;
constexpr int S_QT = 32;                  // tokens per quarter
constexpr int S_RAWSZ = 24576, S_NRAW = 3;  // B [32][128] 16 KB, X [32][64] 8 KB
constexpr int SO_BH = 0, SO_BL = 8192, SO_XH = 16384, SO_XL = 20480, S_OPSZ = 24576;
constexpr int S_OP = S_NRAW * S_RAWSZ;     // two operand stages
constexpr int S_WF = S_OP + 2 * S_OPSZ;    // weights [2][128] float2, then [4] double2 warp totals
constexpr int S_MISCB = S_WF + 2 * QT * 8 + 4 * 16 + 16;
enum { SB_RAWF = 0, SB_RAWE = 3, SB_OPF = 6, SB_OPE = 8, SB_WRDY = 10, SB_WFREE = 12, SB_SDONE = 14, SB_TFREE = 16,
       SB_DRAIN = 18, SB_N = 19 };
constexpr int SMEM_STMA = S_MISCB + SB_N * 8 + 16 + 1024;
static_assert(S_OP % 1024 == 0 && S_OPSZ % 1024 == 0, "swizzled tiles are 1024-byte aligned");
static_assert(SMEM_STMA <= 232448, "one CTA per SM");

__global__ void __launch_bounds__(SNTH, 1)
    state_tma_kernel(const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_x, ScanArgs a,
                     CWs w) {
    const int P = a.headdim, N = a.dstate, H = a.nheads;
    const int nitems = a.batch * H * a.nchunks;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float2 *wfs = reinterpret_cast<float2 *>(sm + S_WF);                 // [2][QT]
    double2 *wtot = reinterpret_cast<double2 *>(sm + S_WF + 2 * QT * 8);  // [4]
    double2 *last = wtot + 4;                                             // (R, Theta) of the chunk
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + S_MISCB);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + SB_N);
    volatile int *abort_s = reinterpret_cast<volatile int *>(tslot + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int i = 0; i < S_NRAW; ++i) {
            mbar_init(&bars[SB_RAWF + i], 1);
            mbar_init(&bars[SB_RAWE + i], 256);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars[SB_OPF + i], 256);
            mbar_init(&bars[SB_OPE + i], 1);
            mbar_init(&bars[SB_WRDY + i], 128);
            mbar_init(&bars[SB_WFREE + i], 256);
            mbar_init(&bars[SB_SDONE + i], 1);
            mbar_init(&bars[SB_TFREE + i], 128);
        }
        mbar_init(&bars[SB_DRAIN], 1);
        *abort_s = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tslot, 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot, sb = smem_u32(sm);

    if (warp == SW_TMA) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            int r = 0;
            bool ok = true;
            for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
                const PItem t = p_item(a, it);
                for (int tq = 0; tq < 4; ++tq) {
                    const int slot = r % S_NRAW;
                    ok = pwait(&bars[SB_RAWE + slot], ((r / S_NRAW) & 1) ^ 1, abort_s, a.dev_error);
                    if (!ok) break;  // nothing more is issued after an abort
                    uint8_t *dst = sm + slot * S_RAWSZ;
                    uint64_t *full = &bars[SB_RAWF + slot];
                    mbar_arrive_expect_tx(full, S_RAWSZ);
                    tma_load_4d(dst, &tm_b, full, 0, t.g, t.c * QT + S_QT * tq, t.b);
                    tma_load_4d(dst + 16384, &tm_x, full, 0, t.h, t.c * QT + S_QT * tq, t.b);
                    ++r;
                }
            }
            for (int slot = 0; slot < S_NRAW; ++slot)  // the last load of every slot has landed
                if (r - 1 >= slot) {
                    const int kl = r - 1 - (r - 1 - slot) % S_NRAW;
                    const unsigned long long t0 = now_ns();
                    while (!mbar_try_wait(&bars[SB_RAWF + slot], (kl / S_NRAW) & 1))
                        if (now_ns() - t0 > WAIT_NS) {
                            atomicCAS(a.dev_error, 0, DEV_TIMEOUT);
                            break;
                        }
                }
        }
    } else if (warp >= SW_CONV && warp < SW_MMA) {
        // -------------------------------------------------------- converters
        const int ct = tid - SW_CONV * 32;  // 0..255
        int r = 0, j = 0;
        for (int it = blockIdx.x; it < nitems; it += gridDim.x) {
            const int wb = j & 1;
            pwait(&bars[SB_WRDY + wb], (j >> 1) & 1, abort_s, a.dev_error);  // chunk j's weights
            const float2 *wf = wfs + wb * QT;
#pragma unroll 1
            for (int tq = 0; tq < 4; ++tq) {
                const int o = 4 * j + tq, os = o & 1, slot = r % S_NRAW;
                uint8_t *op = sm + S_OP + os * S_OPSZ;
                pwait(&bars[SB_RAWF + slot], (r / S_NRAW) & 1, abort_s, a.dev_error);
                pwait(&bars[SB_OPE + os], ((o >> 1) & 1) ^ 1, abort_s, a.dev_error);  // quarter o-2 is done
                const float *raw = reinterpret_cast<const float *>(sm + slot * S_RAWSZ);
#pragma unroll
                for (int i = 0; i < 2; ++i) {  // B''_s = w_s B_s as interleaved (re, im), rows s
                    const int u = ct + 256 * i, sl = u >> 4, ch = u & 15;
                    const float4 b0 = *reinterpret_cast<const float4 *>(raw + sl * 128 + 8 * ch);
                    const float4 b1 = *reinterpret_cast<const float4 *>(raw + sl * 128 + 8 * ch + 4);
                    const cf bq[4] = {{b0.x, b0.y}, {b0.z, b0.w}, {b1.x, b1.y}, {b1.z, b1.w}};
                    const float2 ws = wf[S_QT * tq + sl];
                    float val[8];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const cf z = cmul(bq[e], cf{ws.x, ws.y});
                        val[2 * e] = z.re;
                        val[2 * e + 1] = z.im;
                    }
                    put8(op, SO_BH, SO_BL, sw_off(sl, ch, S_QT * 128), val);
                }
                {  // X rows s as bf16 hi/lo
                    const int sl = ct >> 3, ch = ct & 7;
                    const float4 x0 = *reinterpret_cast<const float4 *>(raw + 4096 + sl * 64 + 8 * ch);
                    const float4 x1 = *reinterpret_cast<const float4 *>(raw + 4096 + sl * 64 + 8 * ch + 4);
                    float val[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
                    put8(op, SO_XH, SO_XL, sw_off(sl, ch, S_QT * 128), val);
                }
                fence_proxy_async_smem();
                mbar_arrive(&bars[SB_OPF + os]);
                mbar_arrive(&bars[SB_RAWE + slot]);
                ++r;
            }
            mbar_arrive(&bars[SB_WFREE + wb]);  // done with chunk j's weights
            ++j;
        }
    } else if (warp == SW_MMA) {
        // -------------------------------------------------------- MMA issuer
        if (lane == 0) {
            int j = 0;
            for (int it = blockIdx.x; it < nitems; it += gridDim.x) {
                const int s = j & 1;
                const uint32_t tm = tmem + 64 * s;
                pwait(&bars[SB_TFREE + s], ((j >> 1) & 1) ^ 1, abort_s, a.dev_error);  // S of chunk j-2 is out
#pragma unroll 1
                for (int tq = 0; tq < 4; ++tq) {
                    const int o = 4 * j + tq, os = o & 1;
                    const uint32_t st = sb + S_OP + os * S_OPSZ;
                    pwait(&bars[SB_OPF + os], (o >> 1) & 1, abort_s, a.dev_error);
                    tc_fence_after();
#pragma unroll 1
                    for (int pass = 0; pass < 3; ++pass) {  // hi.hi + hi.lo + lo.hi
                        const uint32_t aB = st + (pass == 2 ? SO_BL : SO_BH), aX = st + (pass == 1 ? SO_XL : SO_XH);
#pragma unroll 1
                        for (int kk = 0; kk < S_QT / 16; ++kk)
                            mma_ss(tm, smem_desc_sw128(aB + kk * 2048, S_QT * 128, 1024),
                                   smem_desc_sw128(aX + kk * 2048, S_QT * 128, 1024), IDESC_S,
                                   tq > 0 || pass > 0 || kk > 0);
                    }
                    mma_commit(&bars[SB_OPE + os]);
                }
                mma_commit(&bars[SB_SDONE + s]);
                ++j;
            }
            mma_commit(&bars[SB_DRAIN]);
            const unsigned long long t0 = now_ns();
            while (!mbar_try_wait(&bars[SB_DRAIN], 0))
                if (now_ns() - t0 > WAIT_NS) {
                    atomicCAS(a.dev_error, 0, DEV_TIMEOUT);
                    break;
                }
        }
    } else if (warp < SW_CONV) {
        // ------------------------------------- decays, then S of the chunk before
        const int sq = tid;  // token 0..127
        const int qd = warp;
        auto state_out = [&](int jj, size_t bhc) {  // S[p][n] (complex) from TMEM lane k = 2n + (re, im), column p
            const int s = jj & 1;
            pwait(&bars[SB_SDONE + s], (jj >> 1) & 1, abort_s, a.dev_error);
            tc_fence_after();
            const int k = 32 * qd + lane;
            float *S = reinterpret_cast<float *>(w.S + bhc * (size_t)P * N);
#pragma unroll 1
            for (int cb = 0; cb < 64; cb += 32) {
                uint32_t rr[32];
                tmem_ld32(tmem + 64 * s + ((uint32_t)(32 * qd) << 16) + cb, rr);
#pragma unroll
                for (int i = 0; i < 32; ++i) S[((size_t)(cb + i) * N + (k >> 1)) * 2 + (k & 1)] = __uint_as_float(rr[i]);
            }
            tc_fence_before();
            mbar_arrive(&bars[SB_TFREE + s]);
        };
        int j = 0;
        size_t prev_bhc = 0;
        for (int it = blockIdx.x; it < nitems; it += gridDim.x) {
            const PItem t = p_item(a, it);
            const int wb = j & 1;
            // the cumulative log-decay of the chunk in double (same sums, same order,
            // as chunk_log_decay: a warp scan per 32 tokens, then the totals before)
            const float Ar = a.A[2 * t.h], Ai = a.A[2 * t.h + 1];
            const float d = sq < t.valid ? a.dt[(t.bt0 + sq) * H + t.h] : 0.f;
            double vr = (double)d * Ar, vi = (double)d * Ai;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const double yr = __shfl_up_sync(0xffffffffu, vr, o), yi = __shfl_up_sync(0xffffffffu, vi, o);
                if (lane >= o) vr += yr, vi += yi;
            }
            if (lane == 31) wtot[qd] = make_double2(vr, vi);
            named_bar_sync(1, 128);
            if (qd > 0) {
                double pr = wtot[0].x, pi = wtot[0].y;
                for (int q = 1; q < qd; ++q) pr += wtot[q].x, pi += wtot[q].y;
                vr += pr, vi += pi;
            }
            if (sq == QT - 1) *last = make_double2(vr, vi);
            named_bar_sync(1, 128);
            const double R = last->x, Th = last->y;
            // weights of B'' (slot wb: the converters are done with chunk j-2's)
            pwait(&bars[SB_WFREE + wb], ((j >> 1) & 1) ^ 1, abort_s, a.dev_error);
            {
                double sn, cn;
                sincos(Th - vi, &sn, &cn);
                const float m = (float)exp(R - vr) * d;
                wfs[wb * QT + sq] = make_float2(m * (float)cn, m * (float)sn);
            }
            mbar_arrive(&bars[SB_WRDY + wb]);
            // the chunk scan's factors, or the log-decays of a steep chunk; Lambda
            float2 *fac = reinterpret_cast<float2 *>(w.cs + (t.bhc * 2) * QT);
            if (fabs(R) > SPAN) {
                w.cs[(t.bhc * 2) * QT + sq] = vr;
                w.cs[(t.bhc * 2 + 1) * QT + sq] = vi;
            } else {
                const double rho = 0.5 * R;
                double sn, cn;
                sincos(vi, &sn, &cn);
                const float ec = (float)exp(vr - rho), eb = (float)exp(rho - vr) * d;
                fac[sq] = make_float2(ec * (float)cn, ec * (float)sn);
                fac[QT + sq] = make_float2(eb * (float)cn, -eb * (float)sn);
            }
            if (sq == 0) {
                w.lam[t.bhc * 2] = R;
                w.lam[t.bhc * 2 + 1] = Th;
            }
            if (j > 0) state_out(j - 1, prev_bhc);
            prev_bhc = t.bhc;
            ++j;
        }
        if (j > 0) state_out(j - 1, prev_bhc);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 128);
}

// The chunks the factored form cannot take (|Re Lambda| > SPAN): the CUDA-core tile
// code, one CTA per chunk in a loop over all chunks.  smem: cplx_scan_tile_smem(QT).
template <typename T> __global__ void __launch_bounds__(NTH) steep_chunks_kernel(ScanArgs a, CWs w, CplxView<T> v) {
    extern __shared__ uint8_t smem_raw[];
    const int nitems = a.batch * a.nheads * a.nchunks;
    for (int it = blockIdx.x; it < nitems; it += gridDim.x) {
        const PItem t = p_item(a, it);
        if (!p_steep(w, t.bhc)) continue;
        for (int rt = 0; rt * 64 < t.valid; ++rt) cplx_scan_tile<T>(a, w, v, t.b, t.h, t.c, rt, 0, smem_raw);
    }
}

}  // namespace ctc
