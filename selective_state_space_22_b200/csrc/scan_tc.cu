// scan_tc.cu -- the chunked SSD scan as one persistent tcgen05 kernel (sm_100a).
//
// What it computes is the chunkwise evaluation of "Block Anatomy, Numerical
// Stability & Scaling" (Numerical Stability, section 4) for the real Mamba-2
// layout ("BitMamba 1B": one A per head, head dim 64, d_state 128), bf16 x/B/C/y
// with float32 decay, accumulation and state.  A tile is one (batch, head,
// 128-token chunk); the chunk is the MMA's M = 128.  Per tile:
//
//   A_cs = inclusive cumsum of dt*A over the chunk               (warp shuffles)
//   G    = C B^T                          128x128, K = 128        (tcgen05, TMEM)
//   M    = G o L o dt (+ D on the diagonal),  L[l,s] = exp(A_cs[l] - A_cs[s]), s <= l,
//          rewritten in place in TMEM as bf16                     (CUDA cores)
//   S    = B^T (exp(A_cs[last] - A_cs[s]) dt_s x_s)               (tcgen05: chunk state)
//   Y    = M X                            (D x enters through M's diagonal)
//   h_in = the state entering the chunk;   h_out = exp(A_cs[last]) h_in + S
//   y    = Y + exp(A_cs[l]) C h_in^T                              (tcgen05)
//
// Operands reach shared memory by TMA (128-byte swizzle, zero fill past the end
// of the sequence) and y leaves by a TMA store, which clips the ragged tail.
//
// Inter-chunk state passing.  The pages carry chunk c's end state into a later
// chunk z with exp(CD[z-1] - CD[c]) (a strict lower-triangular "decay_chunk"
// product).  Here the same quantity is a running state: h_out of one chunk is
// h_in of the next, updated in registers by the CTA that owns the sequence, so
// no state leaves the chip between chunks.  When there are fewer sequences than
// SMs, each sequence is cut into R runs of consecutive chunks and run r gets its
// own CTA.  That CTA first streams the chunks before its run through a
// state-only pass (W and the S MMA; no G, M or Y) to obtain its entering state,
// then scans its run in full.  CTAs never wait for one another, and the result
// does not depend on timing.
//
// Warp roles (10 warps): 0 TMA producer; 1 MMA issuer (G, S, M X); 2-5 "math"
// warpgroup (decay, W, M); 6-9 "state" warpgroup (state update, h_in^T, the
// C h_in^T MMA, the y epilogue).  Two input stages and two TMEM column sets let
// consecutive tiles overlap.
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "ssd_internal.cuh"
#include "tc_ptx.cuh"

namespace ssd {
namespace {

using namespace ptx;

constexpr int QT = 128;  // tokens per tile (tcgen05 M)
constexpr int PD = 64;   // head dim
constexpr int ND = 128;  // state dim
constexpr int MAX_RUNS = 16;

constexpr int NTH = 320;
constexpr int STATE_W0 = 6;  // warps 2-5 are the math warpgroup
constexpr uint32_t BAR_MATH = 1, BAR_STATE = 2;  // named barriers (128 threads each)

// TMEM: two column sets of 256 (consecutive tiles alternate).
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t COL_G = 0;    // G (f32, 128 cols), then M in place (bf16 pairs, 64 cols)
constexpr uint32_t COL_YD = 128; // M X                       (64 cols)
constexpr uint32_t COL_S = 192;  // chunk state, then C h^T   (64 cols)

// Shared memory: two input stages {C, B, X} and two W buffers.  Within a stage,
// X later holds h_in^T (once M X has read X) and C the y tile (once C h^T has
// read C).
constexpr int STAGE_BYTES = 81920;
constexpr int OFF_C = 0, OFF_B = 32768, OFF_X = 65536;
constexpr int OFF_W = 2 * STAGE_BYTES;
constexpr int OFF_MISC = OFF_W + 2 * 16384;
constexpr uint32_t LOAD_FULL = 2 * (QT * ND * 2) + QT * PD * 2;  // C, B, X
constexpr uint32_t LOAD_STATE = QT * ND * 2 + QT * PD * 2;       // B, X
enum {
    B_FULL = 0, B_EMPTY = 2, B_G = 4, B_S = 6, B_YD = 8, B_YO = 10,   // count 1 (TMA / commit / elected)
    B_CS = 12, B_W = 14, B_M = 16, B_FREE = 18, NBARS = 20            // count 128 (a warpgroup)
};
// misc: cs[2][128], dtv[2][128], bfac[2][128] floats, lam[2], wtot[4], bars, tmem base
constexpr int MISC_BYTES = 3 * 2 * QT * 4 + 8 + 16 + NBARS * 8 + 8;
constexpr int SMEM_ALLOC = OFF_MISC + MISC_BYTES + 1024;

constexpr uint32_t IDESC_G = idesc_bf16_f32(128, 128, 0, 0);   // C (K-major) x B (K-major)
constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 64, 1, 1);    // B^T (MN-major) x W (MN-major)
constexpr uint32_t IDESC_YD = idesc_bf16_f32(128, 64, 0, 1);   // M (TMEM) x X (MN-major)
constexpr uint32_t IDESC_YO = idesc_bf16_f32(128, 64, 0, 1);   // C (K-major) x h^T (MN-major)

constexpr unsigned long long WAIT_NS = 2000000000ull;  // 2 s bound on every wait

struct TcParams {
    const float *dt;
    const float *A;
    const float *D;
    const float *init_state;
    float *final_state;
    int seqlen, nheads, ngroups, nchunks, bH;
    int runs;                    // runs per sequence (1: whole sequences)
    int run_start[MAX_RUNS + 1]; // first chunk of each run; run_start[runs] = nchunks
    int *dev_error;
};

// CTA-local tile k -> (sequence, chunk, state-only?).  CTA i owns work items
// i, i + G, ...; item w is run (w % runs) of sequence (w / runs) and covers
// chunks 0 .. run_start[r+1]-1, those before run_start[r] state-only.
struct Tile {
    int c, bh, b, h, g, t0, valid;
    bool state_only;
};
__device__ __forceinline__ Tile decode_tile(const TcParams &p, int k) {
    Tile t;
    int w = blockIdx.x;
    while (true) {
        const int r = w % p.runs;
        const int n = p.run_start[r + 1];
        if (k < n) {
            t.c = k;
            t.bh = w / p.runs;
            t.state_only = k < p.run_start[r];
            break;
        }
        k -= n;
        w += gridDim.x;
    }
    t.b = t.bh / p.nheads;
    t.h = t.bh % p.nheads;
    t.g = t.h / (p.nheads / p.ngroups);
    t.t0 = t.c * QT;
    t.valid = min(QT, p.seqlen - t.t0);
    return t;
}
__device__ __forceinline__ int local_tiles(const TcParams &p) {
    int n = 0;
    for (int w = blockIdx.x; w < p.bH * p.runs; w += gridDim.x) n += p.run_start[w % p.runs + 1];
    return n;
}

__device__ __forceinline__ unsigned long long now_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Bounded wait on an mbarrier phase (the device error word is set on timeout).
__device__ void mbar_wait(uint64_t *bar, uint32_t parity, int *err) {
    if (mbar_try_wait(bar, parity)) return;
    const unsigned long long t0 = now_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (now_ns() - t0 > WAIT_NS) {
            atomicCAS(err, 0, DEV_TIMEOUT);
            return;
        }
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // .x (low half) = lo
    return *reinterpret_cast<uint32_t *>(&v);
}

// M for one 32-column block j of this thread's row (G block in gr): the causal
// mask on the diagonal block, D on the diagonal.
__device__ __forceinline__ void m_block(const uint32_t (&gr)[32], int j, int quad, int lane, float csl,
                                        const float *csk, const float *dtk, const float *bfk, float Dh,
                                        uint32_t (&packed)[16]) {
    const int r = 32 * j;
    const int lim = (j == quad) ? lane : 31;
    float L[32];
    if (fabsf(csk[r] - csk[r + 31]) <= 80.f) {
        // L[l, s] = exp(A_cs[l] - A_cs[r]) * (exp(A_cs[r] - A_cs[s]) dt_s): one exp per row
        const float a = __expf(csl - csk[r]);
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
            const float4 b4 = *reinterpret_cast<const float4 *>(bfk + r + i);
            L[i] = a * b4.x; L[i + 1] = a * b4.y; L[i + 2] = a * b4.z; L[i + 3] = a * b4.w;
        }
    } else {  // a wide decay range inside this block: one exp per element
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
            const float4 c4 = *reinterpret_cast<const float4 *>(csk + r + i);
            const float4 d4 = *reinterpret_cast<const float4 *>(dtk + r + i);
            L[i] = __expf(fminf(csl - c4.x, 0.f)) * d4.x;
            L[i + 1] = __expf(fminf(csl - c4.y, 0.f)) * d4.y;
            L[i + 2] = __expf(fminf(csl - c4.z, 0.f)) * d4.z;
            L[i + 3] = __expf(fminf(csl - c4.w, 0.f)) * d4.w;
        }
    }
    float m[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) m[i] = (i <= lim) ? __uint_as_float(gr[i]) * L[i] : 0.f;
    if (j == quad) {
#pragma unroll
        for (int i = 0; i < 32; ++i)
            if (i == lane) m[i] += Dh;
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) packed[i] = pack_bf16x2(m[2 * i], m[2 * i + 1]);
}

__global__ void __launch_bounds__(NTH, 1)
    ssd_scan_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
                       const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_y,
                       const TcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *cs = reinterpret_cast<float *>(sm + OFF_MISC);  // [2][128]
    float *dtv = cs + 2 * QT;                              // [2][128]
    float *bfac = dtv + 2 * QT;                            // [2][128]
    float *lam_s = bfac + 2 * QT;                          // [2]
    float *wtot = lam_s + 2;                               // [4]
    uint64_t *bars = reinterpret_cast<uint64_t *>(wtot + 4);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NBARS);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int i = 0; i < B_CS; ++i) mbar_init(&bars[i], 1);
        for (int i = B_CS; i < NBARS; ++i) mbar_init(&bars[i], 128);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int ntl = local_tiles(p);
    const uint32_t sbase = smem_u32(sm);
    int *err = p.dev_error;

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            for (int k = 0; k < ntl; ++k) {
                const Tile t = decode_tile(p, k);
                const int s = k & 1;
                mbar_wait(&bars[B_EMPTY + s], ((k >> 1) & 1) ^ 1, err);
                uint8_t *st = sm + s * STAGE_BYTES;
                uint64_t *full = &bars[B_FULL + s];
                mbar_arrive_expect_tx(full, t.state_only ? LOAD_STATE : LOAD_FULL);
                if (!t.state_only) {
                    tma_load_4d(st + OFF_C, &tm_c, full, 0, t.g, t.t0, t.b);
                    tma_load_4d(st + OFF_C + 16384, &tm_c, full, 64, t.g, t.t0, t.b);
                }
                tma_load_4d(st + OFF_B, &tm_b, full, 0, t.g, t.t0, t.b);
                tma_load_4d(st + OFF_B + 16384, &tm_b, full, 64, t.g, t.t0, t.b);
                tma_load_4d(st + OFF_X, &tm_x, full, 0, t.h, t.t0, t.b);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------- MMA issuer: G, S, M X
        if (lane == 0) {
            for (int k = 0; k < ntl; ++k) {
                const bool so = decode_tile(p, k).state_only;
                const int s = k & 1;
                const uint32_t par = (k >> 1) & 1, tm = tmem + 256 * s;
                const uint32_t aC = sbase + s * STAGE_BYTES + OFF_C, aB = sbase + s * STAGE_BYTES + OFF_B;
                const uint32_t aX = sbase + s * STAGE_BYTES + OFF_X, aW = sbase + OFF_W + s * 16384;
                mbar_wait(&bars[B_FULL + s], par, err);
                mbar_wait(&bars[B_FREE + s], par ^ 1, err);
                tc_fence_after();
                if (!so) {
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {  // G = C B^T
                        const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                        mma_ss(tm + COL_G, smem_desc_sw128(aC + off, 16, 1024), smem_desc_sw128(aB + off, 16, 1024),
                               IDESC_G, kk > 0);
                    }
                }
                mma_commit(&bars[B_G + s]);
                mbar_wait(&bars[B_W + s], par, err);
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)  // S = B^T W
                    mma_ss(tm + COL_S, smem_desc_sw128(aB + kk * 2048, 16384, 1024),
                           smem_desc_sw128(aW + kk * 2048, 8192, 1024), IDESC_S, kk > 0);
                mma_commit(&bars[B_S + s]);
                mbar_wait(&bars[B_M + s], par, err);
                tc_fence_after();
                if (!so) {
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)  // Y = M X
                        mma_ts(tm + COL_YD, tm + COL_G + 8 * kk, smem_desc_sw128(aX + kk * 2048, 8192, 1024),
                               IDESC_YD, kk > 0);
                }
                mma_commit(&bars[B_YD + s]);
            }
        }
    } else if (warp < STATE_W0) {
        // ------------------------------------------------ math warpgroup
        const int quad = warp & 3, row = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        Tile tn = ntl > 0 ? decode_tile(p, 0) : Tile{};
        float dn = (ntl > 0 && row < tn.valid) ? p.dt[((size_t)tn.b * p.seqlen + tn.t0 + row) * p.nheads + tn.h] : 0.f;
        for (int k = 0; k < ntl; ++k) {
            const Tile t = tn;
            const float d = dn;
            if (k + 1 < ntl) {  // next tile's dt, in flight while this tile is built
                tn = decode_tile(p, k + 1);
                dn = (row < tn.valid) ? p.dt[((size_t)tn.b * p.seqlen + tn.t0 + row) * p.nheads + tn.h] : 0.f;
            }
            const int s = k & 1;
            const uint32_t par = (k >> 1) & 1, tm = tmem + 256 * s + lane_off;
            float *csk = cs + s * QT, *dtk = dtv + s * QT, *bfk = bfac + s * QT;
            uint8_t *sx = sm + s * STAGE_BYTES + OFF_X, *sw = sm + OFF_W + s * 16384;
            const float Ah = p.A[t.h];
            const float Dh = p.D ? p.D[t.h] : 0.f;
            // The stage's data is here; through the stage handshake, the state
            // warpgroup is also done with this buffer set's values of tile k-2.
            mbar_wait(&bars[B_FULL + s], par, err);
            float v = d * Ah;  // inclusive cumsum of dt*A over the chunk
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += y;
            }
            if (lane == 31) wtot[quad] = v;
            named_bar_sync(BAR_MATH, 128);
            for (int w = 0; w < quad; ++w) v += wtot[w];
            csk[row] = v;
            dtk[row] = d;
            named_bar_sync(BAR_MATH, 128);
            const float lam = csk[QT - 1];
            if (row == 0) lam_s[s] = lam;
            bfk[row] = __expf(csk[row & ~31] - v) * d;  // exp(A_cs[r] - A_cs[s]) dt_s, r = s's 32-block start
            mbar_arrive(&bars[B_CS + s]);
            {  // W row = exp(lam - A_cs[row]) dt x_row (swizzled 16-byte chunks keep their places)
                const __nv_bfloat162 w2 = __float2bfloat162_rn(__expf(lam - v) * d);
                const uint4 *src = reinterpret_cast<const uint4 *>(sx + row * 128);
                uint4 *dst = reinterpret_cast<uint4 *>(sw + row * 128);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    uint4 q = src[j];
                    __nv_bfloat162 *u = reinterpret_cast<__nv_bfloat162 *>(&q);
#pragma unroll
                    for (int e = 0; e < 4; ++e) u[e] = __hmul2(u[e], w2);
                    dst[j] = q;
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(&bars[B_W + s]);
            // Every role waits on every phase of every barrier it watches, state-only
            // tiles included, so no waiter ever runs a phase ahead of a barrier.
            mbar_wait(&bars[B_G + s], par, err);
            if (t.state_only) {  // no M for a state-only tile
                mbar_arrive(&bars[B_M + s]);
                continue;
            }
            named_bar_sync(BAR_MATH, 128);  // bfac of every row written
            // M = G o L o dt (+ D on the diagonal), bf16 pairs, in place in TMEM.
            // Blocks above the diagonal are zero; the others load two at a time.
            tc_fence_after();
            {
                uint32_t pk[16];
                uint32_t g0[32], g1[32];
                if (quad >= 1) {
                    tmem_ld32x2(tm + COL_G, tm + COL_G + 32, g0, g1);
                    m_block(g0, 0, quad, lane, v, csk, dtk, bfk, Dh, pk);
                    tmem_st16(tm + COL_G, pk);
                    m_block(g1, 1, quad, lane, v, csk, dtk, bfk, Dh, pk);
                    tmem_st16(tm + COL_G + 16, pk);
                } else {
                    tmem_ld32(tm + COL_G, g0);
                    m_block(g0, 0, quad, lane, v, csk, dtk, bfk, Dh, pk);
                    tmem_st16(tm + COL_G, pk);
#pragma unroll
                    for (int i = 0; i < 16; ++i) pk[i] = 0u;
                    tmem_st16(tm + COL_G + 16, pk);
                }
                if (quad == 3) {
                    tmem_ld32x2(tm + COL_G + 64, tm + COL_G + 96, g0, g1);
                    m_block(g0, 2, quad, lane, v, csk, dtk, bfk, Dh, pk);
                    tmem_st16(tm + COL_G + 32, pk);
                    m_block(g1, 3, quad, lane, v, csk, dtk, bfk, Dh, pk);
                    tmem_st16(tm + COL_G + 48, pk);
                } else if (quad == 2) {
                    tmem_ld32(tm + COL_G + 64, g0);
                    m_block(g0, 2, quad, lane, v, csk, dtk, bfk, Dh, pk);
                    tmem_st16(tm + COL_G + 32, pk);
#pragma unroll
                    for (int i = 0; i < 16; ++i) pk[i] = 0u;
                    tmem_st16(tm + COL_G + 48, pk);
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i) pk[i] = 0u;
                    tmem_st16(tm + COL_G + 32, pk);
                    tmem_st16(tm + COL_G + 48, pk);
                }
                tmem_wait_st();
            }
            tc_fence_before();
            mbar_arrive(&bars[B_M + s]);
        }
    } else {
        // ----------------------------------------------- state warpgroup
        const int quad = warp & 3, row = quad * 32 + lane;
        const bool elected = (tid == STATE_W0 * 32);
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        float h[PD];  // the state carried from chunk to chunk: h[p] for state row n = row
        for (int k = 0; k < ntl; ++k) {
            const Tile t = decode_tile(p, k);
            const int s = k & 1;
            const uint32_t par = (k >> 1) & 1, tm = tmem + 256 * s + lane_off;
            if (t.c == 0) {
                if (p.init_state) {
                    const float *h0 = p.init_state + (size_t)t.bh * PD * ND + row;
#pragma unroll
                    for (int q = 0; q < PD; ++q) h[q] = h0[q * ND];
                } else {
#pragma unroll
                    for (int q = 0; q < PD; ++q) h[q] = 0.f;
                }
            }
            mbar_wait(&bars[B_CS + s], par, err);
            const float lam = lam_s[s];
            mbar_wait(&bars[B_S + s], par, err);
            // M X has read X once B_YD completes; X then takes h_in^T.
            mbar_wait(&bars[B_YD + s], par, err);
            tc_fence_after();
            {  // h_in^T (rows n, bf16, 128-byte swizzle) and h_out = exp(lam) h_in + S, 32 columns at a time
                uint8_t *sh = sm + s * STAGE_BYTES + OFF_X;
                const float el = __expf(lam);
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t r[32];
                    tmem_ld32(tm + COL_S + 32 * half, r);
                    if (!t.state_only) {
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const int b0 = 32 * half + 8 * q;
                            const int phys = (4 * half + q) ^ (row & 7);
                            *reinterpret_cast<uint4 *>(sh + row * 128 + phys * 16) =
                                make_uint4(pack_bf16x2(h[b0], h[b0 + 1]), pack_bf16x2(h[b0 + 2], h[b0 + 3]),
                                           pack_bf16x2(h[b0 + 4], h[b0 + 5]), pack_bf16x2(h[b0 + 6], h[b0 + 7]));
                        }
                    }
#pragma unroll
                    for (int q = 0; q < 32; ++q) h[32 * half + q] = fmaf(el, h[32 * half + q], __uint_as_float(r[q]));
                }
            }
            if (t.state_only) {  // no C h^T and no y: release the TMEM set and the stage
                tc_fence_before();
                if (elected) mbar_arrive(&bars[B_YO + s]);
                mbar_wait(&bars[B_YO + s], par, err);
                mbar_arrive(&bars[B_FREE + s]);
                if (elected) mbar_arrive(&bars[B_EMPTY + s]);
                continue;
            }
            if (t.c == p.nchunks - 1 && p.final_state) {
                float *fin = p.final_state + (size_t)t.bh * PD * ND + row;
#pragma unroll
                for (int q = 0; q < PD; ++q) fin[q * ND] = h[q];
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(BAR_STATE, 128);
            const uint32_t aC = sbase + s * STAGE_BYTES + OFF_C, aH = sbase + s * STAGE_BYTES + OFF_X;
            if (elected) {  // Y_off = C h_in^T
                tc_fence_after();
                const uint32_t tmo = tmem + 256 * s;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ss(tmo + COL_S, smem_desc_sw128(aC + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                           smem_desc_sw128(aH + kk * 2048, 8192, 1024), IDESC_YO, kk > 0);
                mma_commit(&bars[B_YO + s]);
            }
            // y = Y + exp(A_cs[l]) Y_off -> bf16 -> y tile over C -> TMA store
            mbar_wait(&bars[B_YO + s], par, err);
            tc_fence_after();
            uint8_t *sy = sm + s * STAGE_BYTES + OFF_C;
            const float e = __expf(cs[s * QT + row]);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t yd[32], yo[32];
                tmem_ld32x2(tm + COL_YD + 32 * half, tm + COL_S + 32 * half, yd, yo);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint32_t pk[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int e0 = 8 * q + 2 * i;
                        pk[i] = pack_bf16x2(fmaf(e, __uint_as_float(yo[e0]), __uint_as_float(yd[e0])),
                                            fmaf(e, __uint_as_float(yo[e0 + 1]), __uint_as_float(yd[e0 + 1])));
                    }
                    const int phys = (4 * half + q) ^ (row & 7);
                    *reinterpret_cast<uint4 *>(sy + row * 128 + phys * 16) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bars[B_FREE + s]);
            named_bar_sync(BAR_STATE, 128);
            if (elected) {
                tma_store_4d(&tm_y, sy, 0, t.h, t.t0, t.b);
                bulk_commit_group();
                bulk_wait_group_read0();  // the y tile has left the stage
                mbar_arrive(&bars[B_EMPTY + s]);
            }
        }
        if (elected) bulk_wait_group0();
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, TMEM_COLS);
}

// ------------------------------------------------------------------- host
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

cudaError_t get_encoder() {
    std::call_once(g_encode_once, [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    return g_encode ? cudaSuccess : cudaErrorNotSupported;
}

// 4-D bf16 tensor [d3][d2][d1][d0] (d0 contiguous), box 64 x 1 x 128 x 1, 128B swizzle.
cudaError_t make_map(CUtensorMap *m, const void *base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t d3) {
    cuuint64_t dims[4] = {d0, d1, d2, d3};
    cuuint64_t strides[3] = {d0 * 2, d0 * d1 * 2, d0 * d1 * d2 * 2};
    cuuint32_t box[4] = {64, 1, (cuuint32_t)QT, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

struct DevInfo {
    bool init = false;
    int sms = 0;
};
DevInfo g_dev[64];
std::mutex g_dev_mu;

// Split nchunks into `runs` runs so that every run's CTA has about the same
// work: run r streams its run_start[r] predecessors state-only (cost ALPHA per
// chunk relative to a full chunk) and then its own chunks in full.
void split_runs(int nchunks, int runs, int *start) {
    const double ALPHA = 0.35;
    auto last = [&](double K) {
        double x = 0;
        for (int r = 0; r < runs; ++r) x += K - ALPHA * x;
        return x;
    };
    double lo = 0, hi = nchunks;
    for (int it = 0; it < 60; ++it) {
        const double mid = 0.5 * (lo + hi);
        (last(mid) < nchunks ? lo : hi) = mid;
    }
    double x = 0;
    start[0] = 0;
    for (int r = 1; r < runs; ++r) {
        x += hi - ALPHA * x;
        start[r] = std::min(nchunks - (runs - r), std::max(start[r - 1] + 1, (int)(x + 0.5)));
    }
    start[runs] = nchunks;
}

}  // namespace

bool tc_supported(int headdim, int dstate, int seqlen) {
    return headdim == PD && dstate == ND && seqlen >= QT;
}

size_t tc_workspace_bytes(int, int) { return 0; }

int tc_kernel_launches() { return 1; }

cudaError_t launch_tc_scan(const ScanArgs &a, void *, cudaStream_t st) {
    cudaError_t e = get_encoder();
    if (e != cudaSuccess) return e;
    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    {
        std::lock_guard<std::mutex> lk(g_dev_mu);
        DevInfo &di = g_dev[dev];
        if (!di.init) {
            if ((e = cudaFuncSetAttribute(ssd_scan_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          SMEM_ALLOC)) != cudaSuccess)
                return e;
            if ((e = cudaDeviceGetAttribute(&di.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
            di.init = true;
        }
    }
    const DevInfo &di = g_dev[dev];

    CUtensorMap mx, mb, mc, my;
    if ((e = make_map(&mx, a.x, a.headdim, a.nheads, a.seqlen, a.batch)) != cudaSuccess) return e;
    if ((e = make_map(&mb, a.B, a.dstate, a.ngroups, a.seqlen, a.batch)) != cudaSuccess) return e;
    if ((e = make_map(&mc, a.C, a.dstate, a.ngroups, a.seqlen, a.batch)) != cudaSuccess) return e;
    if ((e = make_map(&my, a.y, a.headdim, a.nheads, a.seqlen, a.batch)) != cudaSuccess) return e;

    TcParams p;
    p.dt = a.dt;
    p.A = a.A;
    p.D = a.D;
    p.init_state = a.init_state;
    p.final_state = a.final_state;
    p.seqlen = a.seqlen;
    p.nheads = a.nheads;
    p.ngroups = a.ngroups;
    p.nchunks = (a.seqlen + QT - 1) / QT;
    p.bH = a.batch * a.nheads;
    // Whole sequences per CTA when there are enough of them to fill ~3/4 of the
    // SMs; otherwise runs, as many as the SMs allow.
    int runs = 1;
    if (4 * p.bH < 3 * di.sms) runs = std::max(1, std::min({di.sms / p.bH, p.nchunks, MAX_RUNS}));
    p.runs = runs;
    split_runs(p.nchunks, runs, p.run_start);
    p.dev_error = a.dev_error;

    const int items = p.bH * runs;
    const int grid = std::min(items, di.sms);  // one CTA per SM
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(NTH);
    cfg.dynamicSmemBytes = SMEM_ALLOC;
    cfg.stream = st;
    return cudaLaunchKernelEx(&cfg, ssd_scan_tc_kernel, mx, mb, mc, my, p);
}

}  // namespace ssd
