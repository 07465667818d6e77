// scan_tc.cu -- the chunked SSD scan as one persistent tcgen05 kernel (sm_100a).
//
// What it computes is the chunkwise evaluation of "Block Anatomy, Numerical
// Stability & Scaling" (Numerical Stability, section 4) for the real Mamba-2
// layout ("BitMamba 1B": one A per head, head dim 64, d_state 128), bf16 x/B/C/y
// with float32 decay, accumulation and state.  Each tile is one (batch, head,
// 128-token chunk); the chunk is the MMA's M = 128.  Per tile:
//
//   A_cs   = inclusive cumsum of dt*A over the chunk       (warp shuffles)
//   G      = C B^T                      128x128, K = 128    (tcgen05, TMEM)
//   M      = G o L o dt  (+ D on the diagonal), L[l,s] = exp(A_cs[l]-A_cs[s]) for s <= l,
//            rewritten in place in TMEM as bf16             (CUDA cores)
//   S      = B^T (exp(A_cs[last]-A_cs[s]) dt_s x_s)         (tcgen05; the chunk state)
//   Y      = M X                        (+ D x via M's diagonal)
//   h_in   = state entering the chunk, from a decoupled look-back over the
//            states published by earlier chunks of the same sequence
//   Y     += exp(A_cs[l]) C h_in^T                          (tcgen05)
//
// Operands reach shared memory by TMA (128-byte swizzle, zero fill past the end
// of the sequence) and y leaves by a TMA store, which clips the ragged tail.
//
// Inter-chunk state passing.  The pages propagate chunk c's end state into a
// later chunk z by exp(CD[z-1] - CD[c]) (a strict lower-triangular "decay_chunk"
// matrix).  Here every tile publishes, per sequence, into a small ring of slots
// in the workspace: first its local chunk state S_c with its log-decay Lambda_c
// (an "aggregate"), then, once it knows the state entering it, its inclusive
// state h_c = exp(Lambda_c) h_in + S_c (a "prefix").  A tile looks back over at
// most DEPTH predecessors, summing aggregates with the accumulated decay until
// it meets a prefix; so no tile waits for a chain of predecessors to finish in
// turn.  A slot is reused RING chunks later, and only after the tile that used
// it and every tile that may still read it have published their prefixes.
// Tiles are visited in chunk-major order by a cooperative (co-resident) grid,
// so every wait is on a tile with a smaller index and always ends; each wait is
// also bounded in time and reports SSD_ERR_TIMEOUT through the device error
// word instead of hanging.
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "ssd_internal.cuh"
#include "tc_ptx.cuh"

namespace ssd {
namespace {

using namespace ptx;

constexpr int QT = 128;   // tokens per tile (tcgen05 M)
constexpr int PD = 64;    // head dim
constexpr int ND = 128;   // state dim
constexpr int RING = 8;   // published-state slots per sequence (chunk-parallel mode)
constexpr int DEPTH = 2;  // look-back reads at most this many predecessors

// Warp roles: 0 TMA producer, 1 MMA issuer (G, S, M X), 2-5 "math" warpgroup
// (decay, W, M, y), 6-9 "state" warpgroup (inter-chunk state, h_in, C h_in^T).
// A warpgroup's warp w reaches TMEM lanes 32*(w%4)..+31, so each covers all 128.
constexpr int NTH = 320;
constexpr int MATH_W0 = 2, STATE_W0 = 6;
constexpr uint32_t BAR_MATH = 1, BAR_STATE = 2;  // named barriers (128 threads each)

// TMEM: two column sets of 256 (consecutive tiles alternate).
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t COL_G = 0;    // G (f32, 128 cols), then M in place (bf16 pairs, 64 cols)
constexpr uint32_t COL_YD = 128; // M X                       (64 cols)
constexpr uint32_t COL_S = 192;  // chunk state, then C h^T   (64 cols)

// Shared memory: two input stages {C, B, X} and two W / y buffers.
constexpr int STAGE_BYTES = 81920;
constexpr int OFF_C = 0, OFF_B = 32768, OFF_X = 65536;  // within a stage
constexpr int OFF_W = 2 * STAGE_BYTES;                  // 2 x 16 KB
constexpr int OFF_MISC = OFF_W + 2 * 16384;
constexpr uint32_t LOAD_BYTES = 2 * (QT * ND * 2) + QT * PD * 2;
enum {
    B_FULL = 0, B_EMPTY = 2, B_G = 4, B_S = 6, B_YD = 8, B_YO = 10,   // count 1 (TMA / commit)
    B_CS = 12, B_W = 14, B_M = 16, B_FREE = 18, NBARS = 20            // count 128 (warpgroup)
};
// misc: cs[2][128], dtv[2][128], bfac[2][128] floats, lam[2], wtot[4], bars, tmem base
constexpr int MISC_BYTES = 3 * 2 * QT * 4 + 8 + 16 + NBARS * 8 + 8;
constexpr int SMEM_ALLOC = OFF_MISC + MISC_BYTES + 1024;

constexpr uint32_t IDESC_G = idesc_bf16_f32(128, 128, 0, 0);   // C (K-major) x B (K-major)
constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 64, 1, 1);    // B^T (MN-major) x W (MN-major)
constexpr uint32_t IDESC_YD = idesc_bf16_f32(128, 64, 0, 1);   // M (TMEM) x X (MN-major)
constexpr uint32_t IDESC_YO = idesc_bf16_f32(128, 64, 0, 1);   // C (K-major) x h^T (MN-major)

enum : uint32_t { ST_AGG = 1, ST_PREFIX = 2 };
constexpr unsigned long long WAIT_NS = 2000000000ull;  // 2 s bound on every wait

struct TcParams {
    const float *dt;
    const float *A;
    const float *D;
    const float *init_state;
    float *final_state;
    uint32_t *flags;  // [bH][RING][ND]  (chunk << 2) | status, one per state row
    float *lam;       // [bH][RING][ND]  log-decay of the chunk in the slot
    float *agg;       // [bH][RING][ND][PD]   chunk state from a zero start
    float *pre;       // [bH][RING][ND][PD]   state after the chunk
    int seqlen, nheads, ngroups, nchunks, ntiles, bH;
    int resident;     // 1: each CTA owns whole sequences (state stays on chip)
    int *dev_error;
};

// Tile order.  Sequence-resident: CTA i takes sequences i, i+G, ... and walks
// each one's chunks in order.  Chunk-parallel: tiles are numbered chunk-major
// and dealt round-robin, so every wait is on a smaller tile number.
struct Tile {
    int c, bh, b, h, g, t0, valid;
};
__device__ __forceinline__ Tile decode_tile(const TcParams &p, int k) {
    Tile t;
    if (p.resident) {
        t.c = k % p.nchunks;
        t.bh = blockIdx.x + (k / p.nchunks) * gridDim.x;
    } else {
        const int tile = blockIdx.x + k * gridDim.x;
        t.c = tile / p.bH;
        t.bh = tile % p.bH;
    }
    t.b = t.bh / p.nheads;
    t.h = t.bh % p.nheads;
    t.g = t.h / (p.nheads / p.ngroups);
    t.t0 = t.c * QT;
    t.valid = min(QT, p.seqlen - t.t0);
    return t;
}
__device__ __forceinline__ int local_tiles(const TcParams &p) {
    if (p.resident) {
        const int nseq = (blockIdx.x < p.bH) ? (p.bH - 1 - blockIdx.x) / gridDim.x + 1 : 0;
        return nseq * p.nchunks;
    }
    return (blockIdx.x < p.ntiles) ? (p.ntiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
}

__device__ __forceinline__ unsigned long long now_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void report_timeout(int *err) { atomicCAS(err, 0, DEV_TIMEOUT); }

// Bounded wait on an mbarrier phase (the device error is set on timeout).
__device__ void mbar_wait(uint64_t *bar, uint32_t parity, int *err) {
    if (mbar_try_wait(bar, parity)) return;
    const unsigned long long t0 = now_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (now_ns() - t0 > WAIT_NS) {
            report_timeout(err);
            return;
        }
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // .x (low half) = lo
    return *reinterpret_cast<uint32_t *>(&v);
}

// This thread waits until its own flag *f satisfies `ready` (0 after a timeout).
template <typename Pred>
__device__ __forceinline__ uint32_t wait_flag(const uint32_t *f, Pred ready, int *err) {
    uint32_t v = ld_acquire_u32(f);
    if (ready(v)) return v;
    const unsigned long long t0 = now_ns();
    while (true) {
        __nanosleep(32);
        v = ld_acquire_u32(f);
        if (ready(v)) return v;
        if (now_ns() - t0 > WAIT_NS) {
            report_timeout(err);
            return 0;
        }
    }
}

// Chunk-parallel mode: the state entering chunk c for this thread's state row
// n, by a decoupled look-back that each row runs on its own (rows are
// independent: every flag, decay and 256-byte slot row belongs to one thread,
// and a release store orders the thread's own data before its flag).  On entry
// h holds S[n][:] of this chunk; on exit h holds h_in[:][n] and the chunk's
// prefix h_c = exp(lam) h_in + S has been published.
__device__ void lookback_row(const TcParams &p, const Tile &t, int n, float lam, float (&h)[PD],
                             float (&hin)[PD]) {
    const int c = t.c;
    const size_t ring0 = (size_t)t.bh * RING;
    const int slot = c % RING;
    const size_t fl = (ring0 + slot) * ND + n;  // this row's flag / lam index in the slot
    float *prow = p.pre + fl * PD;

    if (c >= RING) {  // slot reuse: its last user and possible readers have published prefixes
#pragma unroll
        for (int k = 0; k <= DEPTH; ++k) {
            const int j = c - RING + k;
            wait_flag(p.flags + (ring0 + j % RING) * ND + n, [j](uint32_t v) {
                return (int)(v >> 2) > j || ((int)(v >> 2) == j && (v & 3u) == ST_PREFIX);
            }, p.dev_error);
        }
    }

    if (c == 0) {
        if (p.init_state) {
            const float *h0 = p.init_state + (size_t)t.bh * PD * ND + n;
#pragma unroll
            for (int q = 0; q < PD; ++q) hin[q] = h0[q * ND];
        } else {
#pragma unroll
            for (int q = 0; q < PD; ++q) hin[q] = 0.f;
        }
    } else {
        const size_t fp = (ring0 + (c - 1) % RING) * ND + n;
        const uint32_t v0 = ld_acquire_u32(p.flags + fp);
        if (v0 == (((uint32_t)(c - 1) << 2) | ST_PREFIX)) {  // predecessor done: no aggregate needed
            const float *src = p.pre + fp * PD;
#pragma unroll
            for (int q = 0; q < PD; q += 4) {
                const float4 f = ld_cg_f4(src + q);
                hin[q] = f.x; hin[q + 1] = f.y; hin[q + 2] = f.z; hin[q + 3] = f.w;
            }
        } else {
            float *arow = p.agg + fl * PD;
#pragma unroll
            for (int q = 0; q < PD; q += 4) *reinterpret_cast<float4 *>(arow + q) = make_float4(h[q], h[q + 1], h[q + 2], h[q + 3]);
            p.lam[fl] = lam;
            st_release_u32(p.flags + fl, ((uint32_t)c << 2) | ST_AGG);
#pragma unroll
            for (int q = 0; q < PD; ++q) hin[q] = 0.f;
            float dec = 0.f;
            for (int j = c - 1; j >= 0; --j) {
                const size_t fj = (ring0 + j % RING) * ND + n;
                const bool need_prefix = (j == c - DEPTH) || (j == 0);
                const uint32_t v = wait_flag(p.flags + fj, [j, need_prefix](uint32_t v) {
                    return (int)(v >> 2) == j && ((v & 3u) == ST_PREFIX || (!need_prefix && (v & 3u) == ST_AGG));
                }, p.dev_error);
                const bool is_prefix = (v & 3u) == ST_PREFIX || v == 0;
                const float fd = __expf(dec);
                const float *src = (is_prefix ? p.pre : p.agg) + fj * PD;
#pragma unroll
                for (int q = 0; q < PD; q += 4) {
                    const float4 f = ld_cg_f4(src + q);
                    hin[q] = fmaf(fd, f.x, hin[q]);
                    hin[q + 1] = fmaf(fd, f.y, hin[q + 1]);
                    hin[q + 2] = fmaf(fd, f.z, hin[q + 2]);
                    hin[q + 3] = fmaf(fd, f.w, hin[q + 3]);
                }
                if (is_prefix) break;
                dec += __ldcg(p.lam + fj);
            }
        }
    }
    const float el = __expf(lam);
#pragma unroll
    for (int q = 0; q < PD; ++q) h[q] = fmaf(el, hin[q], h[q]);
#pragma unroll
    for (int q = 0; q < PD; q += 4) *reinterpret_cast<float4 *>(prow + q) = make_float4(h[q], h[q + 1], h[q + 2], h[q + 3]);
    st_release_u32(p.flags + fl, ((uint32_t)c << 2) | ST_PREFIX);
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
                mbar_arrive_expect_tx(&bars[B_FULL + s], LOAD_BYTES);
                tma_load_4d(st + OFF_C, &tm_c, &bars[B_FULL + s], 0, t.g, t.t0, t.b);
                tma_load_4d(st + OFF_C + 16384, &tm_c, &bars[B_FULL + s], 64, t.g, t.t0, t.b);
                tma_load_4d(st + OFF_B, &tm_b, &bars[B_FULL + s], 0, t.g, t.t0, t.b);
                tma_load_4d(st + OFF_B + 16384, &tm_b, &bars[B_FULL + s], 64, t.g, t.t0, t.b);
                tma_load_4d(st + OFF_X, &tm_x, &bars[B_FULL + s], 0, t.h, t.t0, t.b);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------- MMA issuer: G, S, M X
        if (lane == 0) {
            for (int k = 0; k < ntl; ++k) {
                const int s = k & 1;
                const uint32_t par = (k >> 1) & 1, tm = tmem + 256 * s;
                const uint32_t aC = sbase + s * STAGE_BYTES + OFF_C, aB = sbase + s * STAGE_BYTES + OFF_B;
                const uint32_t aX = sbase + s * STAGE_BYTES + OFF_X, aW = sbase + OFF_W + s * 16384;
                mbar_wait(&bars[B_FULL + s], par, err);
                mbar_wait(&bars[B_FREE + s], par ^ 1, err);
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {  // G = C B^T
                    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                    mma_ss(tm + COL_G, smem_desc_sw128(aC + off, 16, 1024), smem_desc_sw128(aB + off, 16, 1024),
                           IDESC_G, kk > 0);
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
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)  // Y = M X
                    mma_ts(tm + COL_YD, tm + COL_G + 8 * kk, smem_desc_sw128(aX + kk * 2048, 8192, 1024), IDESC_YD,
                           kk > 0);
                mma_commit(&bars[B_YD + s]);
            }
        }
    } else if (warp < STATE_W0) {
        // ------------------------------------------------ math warpgroup
        const int quad = warp & 3, row = quad * 32 + lane, mt = tid - MATH_W0 * 32;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        auto epilogue = [&](int j) {  // y = Y + exp(A_cs[l]) Y_off  -> TMA store
            const Tile t = decode_tile(p, j);
            const int s = j & 1;
            const uint32_t par = (j >> 1) & 1, tm = tmem + 256 * s + lane_off;
            uint8_t *sy = sm + OFF_W + s * 16384;
            mbar_wait(&bars[B_YO + s], par, err);
            tc_fence_after();
            const float e = __expf(cs[s * QT + row]);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t yd[32], yo[32];
                tmem_ld32(tm + COL_YD + 32 * half, yd);
                tmem_ld32(tm + COL_S + 32 * half, yo);
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
            named_bar_sync(BAR_MATH, 128);
            if (mt == 0) {
                tma_store_4d(&tm_y, sy, 0, t.h, t.t0, t.b);
                bulk_commit_group();
            }
            mbar_arrive(&bars[B_FREE + s]);
        };
        for (int k = 0; k < ntl; ++k) {
            const Tile t = decode_tile(p, k);
            const int s = k & 1;
            const uint32_t par = (k >> 1) & 1, tm = tmem + 256 * s + lane_off;
            float *csk = cs + s * QT, *dtk = dtv + s * QT, *bfk = bfac + s * QT;
            uint8_t *sx = sm + s * STAGE_BYTES + OFF_X, *sw = sm + OFF_W + s * 16384;
            const float d = (row < t.valid) ? p.dt[((size_t)t.b * p.seqlen + t.t0 + row) * p.nheads + t.h] : 0.f;
            const float Ah = p.A[t.h];
            const float Dh = p.D ? p.D[t.h] : 0.f;
            // The stage's data is here; through the stage handshake, the state
            // warpgroup is also done with this buffer set's decay values of tile k-2.
            mbar_wait(&bars[B_FULL + s], par, err);
            if (mt == 0) bulk_wait_group_read0();  // the y store of tile k-2 has read sw
            float v = d * Ah;                       // inclusive cumsum of dt*A over the chunk
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
            if (mt == 0) lam_s[s] = lam;
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
            named_bar_sync(BAR_MATH, 128);  // bfac of every row written
            // M = G o L o dt (+ D on the diagonal), bf16 pairs, in place in TMEM
            mbar_wait(&bars[B_G + s], par, err);
            tc_fence_after();
            {
                const float csl = v;
#pragma unroll 1
                for (int j = 0; j < 4; ++j) {
                    uint32_t packed[16];
                    if (j > quad) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) packed[i] = 0u;
                    } else {
                        uint32_t gr[32];
                        tmem_ld32(tm + COL_G + 32 * j, gr);
                        const int r = 32 * j;
                        const int lim = (j == quad) ? lane : 31;  // causal mask on the diagonal block
                        float L[32];
                        if (fabsf(csk[r] - csk[r + 31]) <= 80.f) {
                            // L[l, s] = exp(A_cs[l] - A_cs[r]) * (exp(A_cs[r] - A_cs[s]) dt_s): one exp per row
                            const float a = __expf(csl - csk[r]);
#pragma unroll
                            for (int i = 0; i < 32; i += 4) {
                                const float4 b4 = *reinterpret_cast<const float4 *>(bfk + r + i);
                                L[i] = a * b4.x; L[i + 1] = a * b4.y; L[i + 2] = a * b4.z; L[i + 3] = a * b4.w;
                            }
                        } else {  // a wide decay range in this block: one exp per element
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
                    tmem_st16(tm + COL_G + 16 * j, packed);
                }
                tmem_wait_st();
            }
            tc_fence_before();
            mbar_arrive(&bars[B_M + s]);
            if (k > 0) epilogue(k - 1);
        }
        if (ntl > 0) epilogue(ntl - 1);
        if (mt == 0) bulk_wait_group0();
    } else {
        // ----------------------------------------------- state warpgroup
        const int quad = warp & 3, row = quad * 32 + lane, st_t = tid - STATE_W0 * 32;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        float hcar[PD];  // sequence-resident mode: the state carried from chunk to chunk (row n)
        for (int k = 0; k < ntl; ++k) {
            const Tile t = decode_tile(p, k);
            const int s = k & 1;
            const uint32_t par = (k >> 1) & 1, tm = tmem + 256 * s + lane_off;
            mbar_wait(&bars[B_CS + s], par, err);
            const float lam = lam_s[s];
            mbar_wait(&bars[B_S + s], par, err);
            tc_fence_after();
            float sv[PD];
            {
                uint32_t r[32];
                tmem_ld32(tm + COL_S, r);
#pragma unroll
                for (int i = 0; i < 32; ++i) sv[i] = __uint_as_float(r[i]);
                tmem_ld32(tm + COL_S + 32, r);
#pragma unroll
                for (int i = 0; i < 32; ++i) sv[32 + i] = __uint_as_float(r[i]);
            }
            float hin[PD];
            if (p.resident) {
                if (t.c == 0) {
                    if (p.init_state) {
                        const float *h0 = p.init_state + (size_t)t.bh * PD * ND + row;
#pragma unroll
                        for (int q = 0; q < PD; ++q) hcar[q] = h0[q * ND];
                    } else {
#pragma unroll
                        for (int q = 0; q < PD; ++q) hcar[q] = 0.f;
                    }
                }
                const float el = __expf(lam);
#pragma unroll
                for (int q = 0; q < PD; ++q) {
                    hin[q] = hcar[q];
                    hcar[q] = fmaf(el, hcar[q], sv[q]);
                }
            } else {
                lookback_row(p, t, row, lam, sv, hin);
#pragma unroll
                for (int q = 0; q < PD; ++q) hcar[q] = sv[q];
            }
            if (t.c == p.nchunks - 1 && p.final_state) {
                float *fin = p.final_state + (size_t)t.bh * PD * ND + row;
#pragma unroll
                for (int q = 0; q < PD; ++q) fin[q * ND] = hcar[q];
            }
            // h_in^T (rows n, bf16, 128-byte swizzle) over X, once M X has read X
            mbar_wait(&bars[B_YD + s], par, err);
            uint8_t *sh = sm + s * STAGE_BYTES + OFF_X;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int phys = q ^ (row & 7);
                *reinterpret_cast<uint4 *>(sh + row * 128 + phys * 16) =
                    make_uint4(pack_bf16x2(hin[8 * q], hin[8 * q + 1]), pack_bf16x2(hin[8 * q + 2], hin[8 * q + 3]),
                               pack_bf16x2(hin[8 * q + 4], hin[8 * q + 5]), pack_bf16x2(hin[8 * q + 6], hin[8 * q + 7]));
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(BAR_STATE, 128);
            if (st_t == 0) {  // Y_off = C h_in^T, then the stage is free
                tc_fence_after();
                const uint32_t aC = sbase + s * STAGE_BYTES + OFF_C, aH = sbase + s * STAGE_BYTES + OFF_X;
                const uint32_t tmo = tmem + 256 * s;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ss(tmo + COL_S, smem_desc_sw128(aC + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                           smem_desc_sw128(aH + kk * 2048, 8192, 1024), IDESC_YO, kk > 0);
                mma_commit(&bars[B_YO + s]);
                mma_commit(&bars[B_EMPTY + s]);
            }
        }
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

struct TcWs {
    uint32_t *flags;
    float *lam, *agg, *pre;
    size_t flag_bytes;
};

TcWs carve_tc(void *ws, int bH) {
    TcWs w;
    char *p = static_cast<char *>(ws);
    w.flag_bytes = (size_t)bH * RING * ND * sizeof(uint32_t);
    w.flags = reinterpret_cast<uint32_t *>(p);
    p += align_up(w.flag_bytes, 256);
    w.lam = reinterpret_cast<float *>(p);
    p += align_up((size_t)bH * RING * ND * sizeof(float), 256);
    w.agg = reinterpret_cast<float *>(p);
    p += align_up((size_t)bH * RING * PD * ND * sizeof(float), 256);
    w.pre = reinterpret_cast<float *>(p);
    return w;
}

struct DevInfo {
    bool init = false;
    int sms = 0, per_sm = 0;
};
DevInfo g_dev[64];
std::mutex g_dev_mu;

}  // namespace

bool tc_supported(int headdim, int dstate, int seqlen) {
    return headdim == PD && dstate == ND && seqlen >= QT;
}

size_t tc_workspace_bytes(int batch, int nheads) {
    const size_t bH = (size_t)batch * nheads;
    return align_up(bH * RING * ND * sizeof(uint32_t), 256) + align_up(bH * RING * ND * sizeof(float), 256) +
           2 * align_up(bH * RING * PD * ND * sizeof(float), 256);
}

int tc_kernel_launches() { return 1; }

cudaError_t launch_tc_scan(const ScanArgs &a, void *ws, cudaStream_t st) {
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
            if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&di.per_sm, ssd_scan_tc_kernel, NTH,
                                                                   SMEM_ALLOC)) != cudaSuccess)
                return e;
            if (di.per_sm < 1) return cudaErrorLaunchOutOfResources;
            di.init = true;
        }
    }
    const DevInfo &di = g_dev[dev];

    CUtensorMap mx, mb, mc, my;
    if ((e = make_map(&mx, a.x, a.headdim, a.nheads, a.seqlen, a.batch)) != cudaSuccess) return e;
    if ((e = make_map(&mb, a.B, a.dstate, a.ngroups, a.seqlen, a.batch)) != cudaSuccess) return e;
    if ((e = make_map(&mc, a.C, a.dstate, a.ngroups, a.seqlen, a.batch)) != cudaSuccess) return e;
    if ((e = make_map(&my, a.y, a.headdim, a.nheads, a.seqlen, a.batch)) != cudaSuccess) return e;

    const int bH = a.batch * a.nheads;
    TcWs w = carve_tc(ws, bH);
    // With at least ~3/4 as many sequences as SMs, each CTA owns whole sequences
    // and keeps the state on chip; otherwise chunks are spread over all SMs and
    // the state passes through the look-back slots, which start empty.
    const bool resident = 4 * bH >= 3 * di.sms;
    if (!resident && (e = cudaMemsetAsync(w.flags, 0, w.flag_bytes, st)) != cudaSuccess) return e;

    TcParams p;
    p.dt = a.dt;
    p.A = a.A;
    p.D = a.D;
    p.init_state = a.init_state;
    p.final_state = a.final_state;
    p.flags = w.flags;
    p.lam = w.lam;
    p.agg = w.agg;
    p.pre = w.pre;
    p.seqlen = a.seqlen;
    p.nheads = a.nheads;
    p.ngroups = a.ngroups;
    p.nchunks = (a.seqlen + QT - 1) / QT;
    p.ntiles = p.nchunks * bH;
    p.bH = bH;
    p.resident = resident ? 1 : 0;
    p.dev_error = a.dev_error;

    const int grid = std::min(resident ? bH : p.ntiles, di.per_sm * di.sms);  // one CTA per SM
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(NTH);
    cfg.dynamicSmemBytes = SMEM_ALLOC;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, ssd_scan_tc_kernel, mx, mb, mc, my, p);
}

}  // namespace ssd
