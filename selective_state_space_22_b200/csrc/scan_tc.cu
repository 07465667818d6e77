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
constexpr int RING = 8;   // published-state slots per sequence
constexpr int DEPTH = 2;  // look-back reads at most this many predecessors

// Warp roles: 0 TMA producer, 1 MMA issuer, 2-5 "math" warpgroup (decay, W,
// M, y), 6-9 "state" warpgroup (look-back, publication, h_in).  A warpgroup's
// warp w reaches TMEM lanes 32*(w%4)..+31, so each covers all 128 lanes.
constexpr int NTH = 320;
constexpr int MATH_W0 = 2, STATE_W0 = 6;
constexpr uint32_t BAR_MATH = 1;  // named barrier of the math warpgroup (128 threads)

// TMEM: two column sets of 256 (tiles alternate between them).
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
    B_FULL = 0, B_EMPTY = 2, B_G = 4, B_S = 6, B_YD = 8, B_YO = 10,         // count 1
    B_CS = 12, B_W = 14, B_M = 16, B_H = 18, B_FREE = 20, NBARS = 22         // count 128
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
    uint32_t *flags;  // [bH][RING][4 warps]  (chunk << 2) | status
    float *lam;       // [bH][RING][4 warps]  log-decay of the chunk in the slot
    float *agg;       // [bH][RING][ND][PD]   chunk state from a zero start
    float *pre;       // [bH][RING][ND][PD]   state after the chunk
    int seqlen, nheads, ngroups, nchunks, ntiles, bH;
    int *dev_error;
};

struct Tile {
    int c, bh, b, h, g, t0, valid;
};
__device__ __forceinline__ Tile decode_tile(const TcParams &p, int k) {
    Tile t;
    const int tile = blockIdx.x + k * gridDim.x;
    t.c = tile / p.bH;
    t.bh = tile % p.bH;
    t.b = t.bh / p.nheads;
    t.h = t.bh % p.nheads;
    t.g = t.h / (p.nheads / p.ngroups);
    t.t0 = t.c * QT;
    t.valid = min(QT, p.seqlen - t.t0);
    return t;
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

// Lane 0 of a warp waits until *f satisfies `ready`; the value is broadcast
// (0 after a timeout, which is also reported).
template <typename Pred>
__device__ uint32_t warp_wait_flag(const uint32_t *f, Pred ready, int *err) {
    uint32_t v = 0;
    if ((threadIdx.x & 31) == 0) {
        v = ld_acquire_u32(f);
        if (!ready(v)) {
            const unsigned long long t0 = now_ns();
            while (true) {
                __nanosleep(32);
                v = ld_acquire_u32(f);
                if (ready(v)) break;
                if (now_ns() - t0 > WAIT_NS) {
                    report_timeout(err);
                    v = 0;
                    break;
                }
            }
        }
    }
    return __shfl_sync(0xffffffffu, v, 0);
}

__device__ __forceinline__ void ld_row64(const float *src, float (&v)[PD]) {
#pragma unroll
    for (int q = 0; q < PD; q += 4) {
        const float4 f = ld_cg_f4(src + q);
        v[q] = f.x; v[q + 1] = f.y; v[q + 2] = f.z; v[q + 3] = f.w;
    }
}
__device__ __forceinline__ void st_row64(float *dst, const float (&v)[PD]) {
#pragma unroll
    for (int q = 0; q < PD; q += 4) *reinterpret_cast<float4 *>(dst + q) = make_float4(v[q], v[q + 1], v[q + 2], v[q + 3]);
}

// State entering chunk c of sequence bh for this warp's 32 state rows (n = row),
// and publication of this chunk's prefix (and, when its predecessor's prefix is
// not there yet, first its aggregate).  s[] is S[n][:] of this thread's row;
// hp[] receives h_in[:][n].  Slot layout [n][p]: a row is 256 contiguous bytes.
__device__ void lookback(const TcParams &p, const Tile &t, int quad, int lane, float lam,
                         const float (&s)[PD], float (&hp)[PD]) {
    const int n = quad * 32 + lane;
    const int c = t.c;
    const size_t ring0 = (size_t)t.bh * RING;
    const int slot = c % RING;
    uint32_t *flag = p.flags + (ring0 + slot) * 4 + quad;
    const size_t row = (size_t)n * PD;

    if (c >= RING) {  // slot reuse: its last user and possible readers have published prefixes
        for (int k = 0; k <= DEPTH; ++k) {
            const int j = c - RING + k;
            warp_wait_flag(p.flags + (ring0 + j % RING) * 4 + quad, [j](uint32_t v) {
                return (int)(v >> 2) > j || ((int)(v >> 2) == j && (v & 3u) == ST_PREFIX);
            }, p.dev_error);
        }
    }

    if (c == 0) {
        if (p.init_state) {
            const float *h0 = p.init_state + (size_t)t.bh * PD * ND + n;
#pragma unroll
            for (int q = 0; q < PD; ++q) hp[q] = h0[q * ND];
        } else {
#pragma unroll
            for (int q = 0; q < PD; ++q) hp[q] = 0.f;
        }
    } else {
        const uint32_t *fprev = p.flags + (ring0 + (c - 1) % RING) * 4 + quad;
        uint32_t v0 = (lane == 0) ? ld_acquire_u32(fprev) : 0u;
        v0 = __shfl_sync(0xffffffffu, v0, 0);
        if (v0 == (((uint32_t)(c - 1) << 2) | ST_PREFIX)) {
            ld_row64(p.pre + (ring0 + (c - 1) % RING) * (ND * PD) + row, hp);  // fast path
        } else {
            st_row64(p.agg + (ring0 + slot) * (ND * PD) + row, s);
            if (lane == 0) p.lam[(ring0 + slot) * 4 + quad] = lam;
            __threadfence();
            __syncwarp();
            if (lane == 0) st_release_u32(flag, ((uint32_t)c << 2) | ST_AGG);
#pragma unroll
            for (int q = 0; q < PD; ++q) hp[q] = 0.f;
            float dec = 0.f;
            for (int j = c - 1; j >= 0; --j) {
                const int sj = j % RING;
                const bool need_prefix = (j == c - DEPTH) || (j == 0);
                const uint32_t v = warp_wait_flag(p.flags + (ring0 + sj) * 4 + quad, [j, need_prefix](uint32_t v) {
                    return (int)(v >> 2) == j && ((v & 3u) == ST_PREFIX || (!need_prefix && (v & 3u) == ST_AGG));
                }, p.dev_error);
                const bool is_prefix = (v & 3u) == ST_PREFIX || v == 0;
                const float fd = __expf(dec);
                const float *src = (is_prefix ? p.pre : p.agg) + (ring0 + sj) * (ND * PD) + row;
#pragma unroll
                for (int q = 0; q < PD; q += 4) {
                    const float4 f = ld_cg_f4(src + q);
                    hp[q] = fmaf(fd, f.x, hp[q]);
                    hp[q + 1] = fmaf(fd, f.y, hp[q + 1]);
                    hp[q + 2] = fmaf(fd, f.z, hp[q + 2]);
                    hp[q + 3] = fmaf(fd, f.w, hp[q + 3]);
                }
                if (is_prefix) break;
                dec += __ldcg(p.lam + (ring0 + sj) * 4 + quad);
            }
        }
    }

    const float el = __expf(lam);
    float hc[PD];
#pragma unroll
    for (int q = 0; q < PD; ++q) hc[q] = fmaf(el, hp[q], s[q]);
    st_row64(p.pre + (ring0 + slot) * (ND * PD) + row, hc);
    if ((c == p.nchunks - 1) && p.final_state) {
        float *fin = p.final_state + (size_t)t.bh * PD * ND + n;
#pragma unroll
        for (int q = 0; q < PD; ++q) fin[q * ND] = hc[q];
    }
    __threadfence();
    __syncwarp();
    if (lane == 0) st_release_u32(flag, ((uint32_t)c << 2) | ST_PREFIX);
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
    const int ntl = (blockIdx.x < p.ntiles) ? (p.ntiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
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
        // ------------------------------------------------------- MMA issuer
        if (lane == 0) {
            auto issue_yo = [&](int j) {
                const int s = j & 1;
                const uint32_t par = (j >> 1) & 1, tm = tmem + 256 * s;
                const uint32_t aC = sbase + s * STAGE_BYTES + OFF_C, aH = sbase + s * STAGE_BYTES + OFF_X;
                mbar_wait(&bars[B_H + s], par, err);
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_ss(tm + COL_S, smem_desc_sw128(aC + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024),
                           smem_desc_sw128(aH + k * 2048, 8192, 1024), IDESC_YO, k > 0);
                mma_commit(&bars[B_YO + s]);
                mma_commit(&bars[B_EMPTY + s]);
            };
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
                if (k > 0) issue_yo(k - 1);
            }
            if (ntl > 0) issue_yo(ntl - 1);
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
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    pk[i] = pack_bf16x2(fmaf(e, __uint_as_float(yo[2 * i]), __uint_as_float(yd[2 * i])),
                                        fmaf(e, __uint_as_float(yo[2 * i + 1]), __uint_as_float(yd[2 * i + 1])));
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int phys = (4 * half + q) ^ (row & 7);
                    *reinterpret_cast<uint4 *>(sy + row * 128 + phys * 16) =
                        make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
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
            // the stage's data is here, and (through the stage handshake) the
            // state warpgroup is done with this set's decay values of tile k-2
            mbar_wait(&bars[B_FULL + s], par, err);
            if (mt == 0) bulk_wait_group_read0();  // the y store of tile k-2 has read sw
            float v = d * Ah;
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
            bfk[row] = __expf(csk[row & ~31] - v) * d;
            mbar_arrive(&bars[B_CS + s]);
            {  // W row = exp(lam - A_cs[row]) dt x_row (swizzled 16-byte chunks keep their places)
                const float w = __expf(lam - v) * d;
                const uint4 *src = reinterpret_cast<const uint4 *>(sx + row * 128);
                uint4 *dst = reinterpret_cast<uint4 *>(sw + row * 128);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    uint4 q = src[j];
                    uint32_t *u = reinterpret_cast<uint32_t *>(&q);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&u[e]));
                        u[e] = pack_bf16x2(f.x * w, f.y * w);
                    }
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
                const float Dh = p.D ? p.D[t.h] : 0.f;
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
                        const bool direct = fabsf(csk[r] - csk[r + 31]) > 80.f;
                        const float a = __expf(csl - csk[r]);
                        float m[32];
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            const int sidx = r + i;
                            const float L = direct ? __expf(csl - csk[sidx]) * dtk[sidx] : a * bfk[sidx];
                            float mv = (sidx <= row) ? __uint_as_float(gr[i]) * L : 0.f;
                            if (sidx == row) mv += Dh;
                            m[i] = mv;
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
        const int quad = warp & 3, row = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
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
            float hp[PD];
            lookback(p, t, quad, lane, lam, sv, hp);
            // h_in^T (rows n, bf16, 128-byte swizzle) over X, once M X has read X
            mbar_wait(&bars[B_YD + s], par, err);
            uint8_t *sh = sm + s * STAGE_BYTES + OFF_X;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int phys = q ^ (row & 7);
                *reinterpret_cast<uint4 *>(sh + row * 128 + phys * 16) =
                    make_uint4(pack_bf16x2(hp[8 * q], hp[8 * q + 1]), pack_bf16x2(hp[8 * q + 2], hp[8 * q + 3]),
                               pack_bf16x2(hp[8 * q + 4], hp[8 * q + 5]), pack_bf16x2(hp[8 * q + 6], hp[8 * q + 7]));
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bars[B_H + s]);
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
    w.flag_bytes = (size_t)bH * RING * 4 * sizeof(uint32_t);
    w.flags = reinterpret_cast<uint32_t *>(p);
    p += align_up(w.flag_bytes, 256);
    w.lam = reinterpret_cast<float *>(p);
    p += align_up((size_t)bH * RING * 4 * sizeof(float), 256);
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
    return align_up(bH * RING * 4 * sizeof(uint32_t), 256) + align_up(bH * RING * 4 * sizeof(float), 256) +
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
    // The look-back protocol starts from empty slot flags.
    if ((e = cudaMemsetAsync(w.flags, 0, w.flag_bytes, st)) != cudaSuccess) return e;

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
    p.dev_error = a.dev_error;

    const int grid = std::min(p.ntiles, di.per_sm * di.sms);  // one CTA per SM
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
