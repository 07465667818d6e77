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
//   y    = M X + exp(A_cs[l]) C h_in^T                            (tcgen05)
//   h_out = exp(A_cs[last]) h_in + S
//
// D x enters through M's diagonal.  Operands reach shared memory by TMA
// (128-byte swizzle, zero fill past the end of the sequence); y is written from
// registers, rows past the end of the sequence skipped.
//
// Inter-chunk state passing.  The pages carry chunk c's end state into a later
// chunk z with exp(CD[z-1] - CD[c]) (a strict lower-triangular "decay_chunk"
// product).  Here the same quantity is a running state: h_out of one chunk is
// h_in of the next, updated in registers by the CTA that owns the sequence, so
// no state leaves the chip between chunks, and h_in of a chunk is ready before
// its data arrives.  When there are fewer sequences than SMs, each sequence is
// cut into R runs of consecutive chunks and run r gets its own CTA.  That CTA
// first streams the chunks before its run through a state-only pass (W and the
// S MMA; no G, M or y) to obtain its entering state, then scans its run in full.
// CTAs never wait for one another, and the result does not depend on timing.
//
// Warp roles (15 warps): 0 TMA producer; 1 MMA issuer for G and S; 14 MMA
// issuer for the two products of y; 2-5 "math" warpgroup (M); 6-9 "state"
// warpgroup (h_in^T, the state update); 10-13 "prep/epilogue" warpgroup (the
// cumulative decay and W of tile k, then y of tile k-1).  Hot loops are kept
// rolled: four roles share each SM sub-partition's instruction cache.  Two
// {C, B} slots, three X slots and two TMEM column sets let consecutive tiles
// overlap; a column set is released as soon as its y is out.  C h_in^T has its
// own columns, so it runs as soon as h_in^T is written, without waiting for the
// tile's state update.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
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

constexpr int NTH = 480;
constexpr int STATE_W0 = 6;     // warps 2-5: math warpgroup; 6-9: state warpgroup
constexpr int EPI_W0 = 10;      // warps 10-13: epilogue warpgroup
constexpr int Y_MMA_WARP = 14;  // issues the two products of y
constexpr uint32_t BAR_MATH = 1;  // named barrier of the math warpgroup (128 threads)

// TMEM: two column sets of 256 (consecutive tiles alternate).
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t COL_G = 0;    // G (f32, 128 cols), then M (bf16 pairs) in columns 0-63
constexpr uint32_t COL_YD = 64;  // M X, in G's second half once M is built   (64 cols)
constexpr uint32_t COL_YO = 128; // C h_in^T                                  (64 cols)
constexpr uint32_t COL_S = 192;  // chunk state                               (64 cols)

// Shared memory: C and B (released after G, S and C h^T) and X (released after W
// and M X) live in separate rings, two {C, B} slots of 64 KB and three X slots
// of 16 KB, so the loads of later tiles do not wait for this tile's M X; then
// one W buffer and one h_in^T buffer.
constexpr int CB_BYTES = 65536;
constexpr int OFF_C = 0, OFF_B = 32768;           // within a {C, B} slot
constexpr int OFF_XR = 2 * CB_BYTES;              // X ring [3][16 KB]
constexpr int X_SLOTS = 3;
constexpr int OFF_W = OFF_XR + X_SLOTS * 16384;
constexpr int OFF_H = OFF_W + 16384;              // one h_in^T buffer
constexpr int OFF_MISC = OFF_H + 16384;
constexpr uint32_t LOAD_CB = 2 * (QT * ND * 2);   // C, B
constexpr uint32_t LOAD_B = QT * ND * 2;          // B (state-only tiles)
constexpr uint32_t LOAD_X = QT * PD * 2;
enum {
    // count 1 (TMA bytes or an MMA commit); B_EMPTY ({C, B} slot free): 2, a
    // commit from each MMA issuer
    B_FULL = 0, B_EMPTY = 2, B_G = 4, B_S = 6, B_Y = 8, B_YO = 10,
    // the X ring; B_XEMPTY counts S's commit (S is issued once W has read X)
    // and M X's commit
    B_XFULL = 12, B_XEMPTY = 15,
    // count 128 (one warpgroup).  B_HW: h_in^T written; B_H: chunk state read
    B_CS = 18, B_W = 20, B_M = 22, B_H = 24, B_FREE = 26, B_HW = 28,
    // count 1: a final commit of each MMA issuer, so that it can wait for its own
    // MMAs before the CTA exits after an abort
    B_DRAIN = 30, NBARS = 32
};
// misc: cs[2][128], dtv[2][128], bfac[2][128] floats, lam[2], dh[2], wtot[4],
// the abort word (+ 7 spare ints), bars, tmem base
constexpr int MISC_BYTES = 3 * 2 * QT * 4 + 8 + 8 + 16 + 32 + NBARS * 8 + 8;
constexpr int SMEM_ALLOC = OFF_MISC + MISC_BYTES + 1024;

constexpr uint32_t IDESC_G = idesc_bf16_f32(128, 128, 0, 0);   // C (K-major) x B (K-major)
constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 64, 1, 1);    // B^T (MN-major) x W (MN-major)
constexpr uint32_t IDESC_YD = idesc_bf16_f32(128, 64, 0, 1);   // M (TMEM) x X (MN-major)
constexpr uint32_t IDESC_YO = idesc_bf16_f32(128, 64, 0, 1);   // C (K-major) x h^T (MN-major)

constexpr unsigned long long WAIT_NS = 1000000000ull;  // 1 s bound on every wait

struct TcParams {
    __nv_bfloat16 *y;
    const float *dt;
    const float *A;
    const float *D;
    const float *init_state;
    float *final_state;
    int seqlen, nheads, ngroups, nchunks, bH;
    int runs;                    // runs per sequence (1: whole sequences)
    int run_start[MAX_RUNS + 1]; // first chunk of each run; run_start[runs] = nchunks
    int *dev_error;
    unsigned long long wait_ns;  // bound on every wait (WAIT_NS unless a test shortens it)
    int withhold;                // test only: the producer issues no load, so every wait runs out
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

// Bounded wait on an mbarrier phase.  Returns false, without waiting further,
// once the CTA's abort word is set; a wait that runs out sets the device error
// word and the abort word.  After an abort the TMA producer stops at its first
// failed wait; every other role runs its remaining tiles with each wait giving
// up after 20 us (so the kernel ends within milliseconds),
// its shared-memory and TMEM accesses in bounds and its named barriers matched;
// the outputs are invalid and reported so.  Arrivals that then come early (MMA
// commits, warpgroup arrivals: plain counts, no transaction bytes) only complete
// barrier phases early.  At the end the TMA
// producer waits (bounded) for the last load of every slot and each MMA issuer
// for a commit of everything it issued, so nothing is in flight when the CTA
// frees TMEM and exits.  Only the first probe is inlined; the polling loop,
// which looks at the abort word once a wait has lasted 20 us, is one
// out-of-line copy, so that the many wait sites of the hot loops stay small.
__device__ __noinline__ bool mbar_wait_slow(uint64_t *bar, uint32_t parity, volatile int *abort_s, int *err,
                                            unsigned long long limit) {
    const unsigned long long t0 = now_ns();
    while (!mbar_try_wait(bar, parity)) {
        const unsigned long long waited = now_ns() - t0;
        if (waited > 20000) {  // the abort word is only looked at once a wait is long
            if (*abort_s) return false;
            if (waited > limit) {
                atomicCAS(err, 0, DEV_TIMEOUT);
                *abort_s = 1;
                return false;
            }
        }
    }
    return true;
}
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, const TcParams &p, volatile int *abort_s) {
    if (mbar_try_wait(bar, parity)) return true;
    return mbar_wait_slow(bar, parity, abort_s, p.dev_error, p.wait_ns);
}
// The same without the abort shortcut: how a role waits for its own TMA loads
// or MMAs to finish before the CTA exits (still bounded).
__device__ __noinline__ void mbar_wait_drain(uint64_t *bar, uint32_t parity, const TcParams &p,
                                             volatile int *abort_s) {
    const unsigned long long t0 = now_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (now_ns() - t0 > p.wait_ns) {
            atomicCAS(p.dev_error, 0, DEV_TIMEOUT);
            *abort_s = 1;
            return;
        }
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // .x (low half) = lo
    return *reinterpret_cast<uint32_t *>(&v);
}

// Decay factors of one 32-column block j for this thread's row l:
// L[s] = exp(A_cs[l] - A_cs[s]) dt_s, as pairs.
__device__ __forceinline__ void block_decay(int j, float csl, const float *csk, const float *dtk, const float *bfk,
                                           float2 (&L)[16]) {
    const int r = 32 * j;
    if (fabsf(csk[r] - csk[r + 31]) <= 80.f) {
        // exp(A_cs[l] - A_cs[r]) * (exp(A_cs[r] - A_cs[s]) dt_s): one exp per row
        const float a = __expf(csl - csk[r]);
        const float2 a2 = make_float2(a, a);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float4 b4 = *reinterpret_cast<const float4 *>(bfk + r + 4 * i);
            L[2 * i] = fmul2(a2, make_float2(b4.x, b4.y));
            L[2 * i + 1] = fmul2(a2, make_float2(b4.z, b4.w));
        }
    } else {  // a wide decay range inside this block: one exp per element
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float4 c4 = *reinterpret_cast<const float4 *>(csk + r + 4 * i);
            const float4 d4 = *reinterpret_cast<const float4 *>(dtk + r + 4 * i);
            L[2 * i] = make_float2(__expf(fminf(csl - c4.x, 0.f)) * d4.x, __expf(fminf(csl - c4.y, 0.f)) * d4.y);
            L[2 * i + 1] = make_float2(__expf(fminf(csl - c4.z, 0.f)) * d4.z, __expf(fminf(csl - c4.w, 0.f)) * d4.w);
        }
    }
}

// M = G o L for one block (G block in gr), bf16 pairs; on the diagonal block
// only s <= l is kept and D is added at s == l.
__device__ __forceinline__ void block_apply(const uint32_t (&gr)[32], const float2 (&L)[16], bool diag, int lane,
                                            float Dh, uint32_t (&packed)[16]) {
    if (!diag) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float2 m = fmul2(make_float2(__uint_as_float(gr[2 * i]), __uint_as_float(gr[2 * i + 1])), L[i]);
            packed[i] = pack_bf16x2(m.x, m.y);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float2 m = fmul2(make_float2(__uint_as_float(gr[2 * i]), __uint_as_float(gr[2 * i + 1])), L[i]);
            m.x = (2 * i < lane) ? m.x : (2 * i == lane ? m.x + Dh : 0.f);
            m.y = (2 * i + 1 < lane) ? m.y : (2 * i + 1 == lane ? m.y + Dh : 0.f);
            packed[i] = pack_bf16x2(m.x, m.y);
        }
    }
}

// One M block: TMEM load of G, decay factors computed while it is in flight,
// then M (bf16 pairs, 16 columns) written to columns 16j..16j+15.  The blocks of
// a row are built in order by the one thread that owns the row, and block j's
// columns belong to G blocks <= j, which that thread has already read.
__device__ __forceinline__ void m_block(uint32_t tm, int j, int quad, int lane, float csl, const float *csk,
                                        const float *dtk, const float *bfk, float Dh) {
    uint32_t pk[16];
    if (j > quad) {  // above the diagonal
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[i] = 0u;
    } else {
        uint32_t g[32];
        float2 L[16];
        tmem_ld32_nowait(tm + 32 * j, g);
        block_decay(j, csl, csk, dtk, bfk, L);
        tmem_wait_ld(g);
        block_apply(g, L, j == quad, lane, Dh, pk);
    }
    tmem_st16(tm + 16 * j, pk);
}

// Row scaling of a 128-byte swizzled shared-memory row (eight 16-byte chunks),
// src -> dst (may be the same row).  The factor is the same for the whole row,
// so the chunks are visited as j ^ key (key = row % 8): the eight rows a
// quarter-warp touches then fall on eight different bank groups.
__device__ __forceinline__ void scale_row(const uint8_t *src, uint8_t *dst, int key, __nv_bfloat162 f) {
    uint4 q[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) q[j] = reinterpret_cast<const uint4 *>(src)[j ^ key];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        __nv_bfloat162 *u = reinterpret_cast<__nv_bfloat162 *>(&q[j]);
#pragma unroll
        for (int e = 0; e < 4; ++e) u[e] = __hmul2(u[e], f);
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) reinterpret_cast<uint4 *>(dst)[j ^ key] = q[j];
}

// A state-only tile's W: the math warpgroup, which has no M to build for it,
// scales this thread's row of X into the C half of the tile's {C, B} slot.  Out of
// line, so that the M build's loop keeps its size.
__device__ __noinline__ void state_only_w_row(const uint8_t *x_row, uint8_t *w_row, int key, float f) {
    scale_row(x_row, w_row, key, __float2bfloat162_rn(f));
}

// SPLIT: the state-only form (no y: every tile state-only).  Then the math
// warpgroup, which has no M to build, builds each tile's W into the C half of the
// tile's {C, B} slot (TMA loads only B there), free once the tile two before has
// released the slot; W of one tile then does not wait for S of the one before, and
// the epilogue warpgroup only computes the decays (1.24 against 1.49 us per tile
// at T = 65536, 64 heads).  Otherwise the epilogue warpgroup builds every W, a
// run's state-only prefix included, into the one W buffer: the same change slowed
// the full tiles of a launch by 4-15%, more than the prefix gains.
template <bool SPLIT>
__global__ void __launch_bounds__(NTH, 1)
    ssd_scan_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
                       const __grid_constant__ CUtensorMap tm_c, const TcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *cs = reinterpret_cast<float *>(sm + OFF_MISC);  // [2][128]
    float *dtv = cs + 2 * QT;                              // [2][128]
    float *bfac = dtv + 2 * QT;                            // [2][128]
    float *lam_s = bfac + 2 * QT;                          // [2]
    float *dh_s = lam_s + 2;                               // [2]
    float *wtot = dh_s + 2;                                // [4]
    volatile int *abort_s = reinterpret_cast<volatile int *>(wtot + 4);  // [1]
    uint64_t *bars = reinterpret_cast<uint64_t *>(wtot + 12);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NBARS);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int i = 0; i < B_CS; ++i)
            mbar_init(&bars[i], (i == B_EMPTY || i == B_EMPTY + 1 || (i >= B_XEMPTY && i < B_XEMPTY + 3)) ? 2 : 1);
        for (int i = B_CS; i < B_DRAIN; ++i) mbar_init(&bars[i], 128);
        mbar_init(&bars[B_DRAIN], 1);
        mbar_init(&bars[B_DRAIN + 1], 1);
        *abort_s = 0;
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

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0 && !p.withhold) {
            // After an abort the producer stops issuing at its first failed wait, so
            // that a slot is never reloaded while its last load is in flight; ncb
            // and nx count the {C, B} and X loads issued (tiles 0 .. n - 1).
            int ncb = 0, nx = 0;
            for (int k = 0; k < ntl; ++k) {
                const Tile t = decode_tile(p, k);
                const int s = k & 1;
                if (!mbar_wait(&bars[B_EMPTY + s], ((k >> 1) & 1) ^ 1, p, abort_s)) break;
                uint8_t *st = sm + s * CB_BYTES;
                uint64_t *full = &bars[B_FULL + s];
                mbar_arrive_expect_tx(full, t.state_only ? LOAD_B : LOAD_CB);
                if (!t.state_only) {
                    tma_load_4d(st + OFF_C, &tm_c, full, 0, t.g, t.t0, t.b);
                    tma_load_4d(st + OFF_C + 16384, &tm_c, full, 64, t.g, t.t0, t.b);
                }
                tma_load_4d(st + OFF_B, &tm_b, full, 0, t.g, t.t0, t.b);
                tma_load_4d(st + OFF_B + 16384, &tm_b, full, 64, t.g, t.t0, t.b);
                ncb = k + 1;
                const int xs = k % X_SLOTS;
                if (!mbar_wait(&bars[B_XEMPTY + xs], ((k / X_SLOTS) & 1) ^ 1, p, abort_s)) break;
                mbar_arrive_expect_tx(&bars[B_XFULL + xs], LOAD_X);
                tma_load_4d(sm + OFF_XR + xs * 16384, &tm_x, &bars[B_XFULL + xs], 0, t.h, t.t0, t.b);
                nx = k + 1;
            }
            // Every load issued must have landed before the CTA's shared memory
            // is released (after an abort its consumer may never have waited).
            for (int s = 0; s < 2; ++s)  // the last tile loaded into each slot
                if (ncb - 1 >= s) {
                    const int kl = ncb - 1 - ((ncb - 1 - s) & 1);
                    mbar_wait_drain(&bars[B_FULL + s], (kl >> 1) & 1, p, abort_s);
                }
            for (int xs = 0; xs < X_SLOTS; ++xs)
                if (nx - 1 >= xs) {
                    const int kl = nx - 1 - (nx - 1 - xs) % X_SLOTS;
                    mbar_wait_drain(&bars[B_XFULL + xs], (kl / X_SLOTS) & 1, p, abort_s);
                }
        }
    } else if (warp == 1) {
        // ------------------------------------------- MMA issuer: G and S
        if (lane == 0) {
            for (int k = 0; k < ntl; ++k) {
                const bool so = decode_tile(p, k).state_only;
                const int s = k & 1;
                const uint32_t par = (k >> 1) & 1, tm = tmem + 256 * s;
                const uint32_t aC = sbase + s * CB_BYTES + OFF_C, aB = sbase + s * CB_BYTES + OFF_B;
                const uint32_t aW = (SPLIT && so) ? aC : sbase + OFF_W;
                mbar_wait(&bars[B_FULL + s], par, p, abort_s);
                mbar_wait(&bars[B_FREE + s], par ^ 1, p, abort_s);
                tc_fence_after();
                if (!so) {
#pragma unroll 1
                    for (int kk = 0; kk < 8; ++kk) {  // G = C B^T
                        const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                        mma_ss(tm + COL_G, smem_desc_sw128(aC + off, 16, 1024), smem_desc_sw128(aB + off, 16, 1024),
                               IDESC_G, kk > 0);
                    }
                }
                mma_commit(&bars[B_G + s]);
                mbar_wait(&bars[B_W + s], par, p, abort_s);
                // S's columns held the chunk state of tile k-2 until its state update
                if (k >= 2) mbar_wait(&bars[B_H + s], par ^ 1, p, abort_s);
                tc_fence_after();
#pragma unroll 1
                for (int kk = 0; kk < 8; ++kk)  // S = B^T W
                    mma_ss(tm + COL_S, smem_desc_sw128(aB + kk * 2048, 16384, 1024),
                           smem_desc_sw128(aW + kk * 2048, 8192, 1024), IDESC_S, kk > 0);
                mma_commit(&bars[B_S + s]);
                mma_commit(&bars[B_EMPTY + s]);  // G and S are done with the slot's B and C
                mma_commit(&bars[B_XEMPTY + k % X_SLOTS]);  // W (issued after W was built) is done with X
            }
            mma_commit(&bars[B_DRAIN]);  // this thread's MMAs are done before the CTA exits
            mbar_wait_drain(&bars[B_DRAIN], 0, p, abort_s);
        }
    } else if (warp == Y_MMA_WARP) {
        // --------------------------------- MMA issuer: C h_in^T and M X
        if (lane == 0) {
            for (int k = 0; k < ntl; ++k) {
                const bool so = decode_tile(p, k).state_only;
                const int s = k & 1;
                const uint32_t par = (k >> 1) & 1, tm = tmem + 256 * s;
                const int xs = k % X_SLOTS;
                const uint32_t aC = sbase + s * CB_BYTES + OFF_C, aX = sbase + OFF_XR + xs * 16384;
                const uint32_t aH = sbase + OFF_H;
                // G of this tile was issued after tile k-2's epilogue released the
                // set, so C h^T's columns are free; h_in^T of this tile is written.
                mbar_wait(&bars[B_G + s], par, p, abort_s);
                mbar_wait(&bars[B_HW + s], par, p, abort_s);
                tc_fence_after();
                if (!so) {
#pragma unroll 1
                    for (int kk = 0; kk < 8; ++kk)  // Y_off = C h_in^T
                        mma_ss(tm + COL_YO, smem_desc_sw128(aC + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                               smem_desc_sw128(aH + kk * 2048, 8192, 1024), IDESC_YO, kk > 0);
                }
                mma_commit(&bars[B_YO + s]);     // done with the h_in^T buffer
                mma_commit(&bars[B_EMPTY + s]);  // with G and S: done with the {C, B} slot
                mbar_wait(&bars[B_M + s], par, p, abort_s);
                mbar_wait(&bars[B_XFULL + xs], (k / X_SLOTS) & 1, p, abort_s);
                tc_fence_after();
                if (!so) {
#pragma unroll 1
                    for (int kk = 0; kk < 8; ++kk)  // Y = M X
                        mma_ts(tm + COL_YD, tm + COL_G + 8 * kk, smem_desc_sw128(aX + kk * 2048, 8192, 1024),
                               IDESC_YD, kk > 0);
                }
                mma_commit(&bars[B_Y + s]);
                mma_commit(&bars[B_XEMPTY + xs]);  // with the W threads: done with the X slot
            }
            mma_commit(&bars[B_DRAIN + 1]);
            mbar_wait_drain(&bars[B_DRAIN + 1], 0, p, abort_s);
        }
    } else if (warp < STATE_W0) {
        // ------------------------------------------------ math warpgroup
        // Per tile: M = G o L o dt (+ D on the diagonal), the four column blocks in
        // order, from the decays the prep/epilogue warpgroup put in shared memory.
        const int quad = warp & 3, row = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        for (int k = 0; k < ntl; ++k) {
            const bool so = decode_tile(p, k).state_only;
            const int s = k & 1;
            const uint32_t par = (k >> 1) & 1, tm = tmem + 256 * s + lane_off;
            const float *csk = cs + s * QT, *dtk = dtv + s * QT, *bfk = bfac + s * QT;
            mbar_wait(&bars[B_CS + s], par, p, abort_s);
            const float v = csk[row], Dh = dh_s[s];
            if constexpr (SPLIT) {
                if (so) {  // W of a state-only tile, into its slot's C half
                    const int xs = k % X_SLOTS;
                    mbar_wait(&bars[B_EMPTY + s], par ^ 1, p, abort_s);
                    mbar_wait(&bars[B_XFULL + xs], (k / X_SLOTS) & 1, p, abort_s);
                    state_only_w_row(sm + OFF_XR + xs * 16384 + row * 128, sm + s * CB_BYTES + OFF_C + row * 128,
                                     row & 7, __expf(csk[QT - 1] - v) * dtk[row]);
                    fence_proxy_async_smem();
                    mbar_arrive(&bars[B_W + s]);
                }
            }
            mbar_wait(&bars[B_G + s], par, p, abort_s);
            tc_fence_after();
            if (!so) {
#pragma unroll 1
                for (int j = 0; j < 4; ++j) m_block(tm + COL_G, j, quad, lane, v, csk, dtk, bfk, Dh);
                tmem_wait_st();
            }
            tc_fence_before();
            mbar_arrive(&bars[B_M + s]);
        }
    } else if (warp < EPI_W0) {
        // ----------------------------------------------- state warpgroup
        const int quad = warp & 3, row = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        float h[PD];  // the state carried from chunk to chunk: h[p] for state row n = row
        for (int k = 0; k < ntl; ++k) {
            const Tile t = decode_tile(p, k);
            const int s = k & 1;
            const uint32_t par = (k >> 1) & 1, tm = tmem + 256 * s + lane_off;
            mbar_wait(&bars[B_CS + s], par, p, abort_s);
            const float lam = lam_s[s];
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
            if (!t.state_only) {  // h_in^T (rows n, bf16, 128-byte swizzle)
                // the one buffer was last read by C h^T of tile k-1; waiting for
                // that (and not for this tile's G) lets C h^T go as early as it can
                if (k > 0) mbar_wait(&bars[B_YO + (s ^ 1)], ((k - 1) >> 1) & 1, p, abort_s);
                uint8_t *sh = sm + OFF_H;
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int phys = q ^ (row & 7);
                    *reinterpret_cast<uint4 *>(sh + row * 128 + phys * 16) =
                        make_uint4(pack_bf16x2(h[8 * q], h[8 * q + 1]), pack_bf16x2(h[8 * q + 2], h[8 * q + 3]),
                                   pack_bf16x2(h[8 * q + 4], h[8 * q + 5]), pack_bf16x2(h[8 * q + 6], h[8 * q + 7]));
                }
                fence_proxy_async_smem();
            }
            mbar_arrive(&bars[B_HW + s]);  // C h_in^T may go
            mbar_wait(&bars[B_S + s], par, p, abort_s);
            tc_fence_after();
            {  // h_out = exp(lam) h_in + S, 32 columns at a time
                const float el = __expf(lam);
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t r[32];
                    tmem_ld32(tm + COL_S + 32 * half, r);
#pragma unroll
                    for (int q = 0; q < 32; ++q) h[32 * half + q] = fmaf(el, h[32 * half + q], __uint_as_float(r[q]));
                }
            }
            tc_fence_before();
            mbar_arrive(&bars[B_H + s]);  // chunk state read: S of tile k+2 may overwrite it
            if (t.c == p.nchunks - 1 && p.final_state) {
                float *fin = p.final_state + (size_t)t.bh * PD * ND + row;
#pragma unroll
                for (int q = 0; q < PD; ++q) fin[q * ND] = h[q];
            }
        }
    } else if (warp < Y_MMA_WARP) {
        // --------------------------------------- prep / epilogue warpgroup
        // Step k: the cumulative decay and W of tile k, then y of tile k-1:
        //   y = M X + exp(A_cs[l]) C h_in^T, straight from TMEM to global memory.
        // Tile k's decays go to slot k % 2, last read for tile k-2: by its M and
        // its state update, both of which finished before tile k-2's y (waited
        // for in step k-1).
        const int quad = warp & 3, row = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        // The next tile's dt, A and D are loaded while this tile is built, so no
        // global-memory latency sits on the per-tile path.
        Tile tn = ntl > 0 ? decode_tile(p, 0) : Tile{};
        float dn = 0.f, An = 0.f, Dn = 0.f;
        if (ntl > 0) {
            dn = row < tn.valid ? p.dt[((size_t)tn.b * p.seqlen + tn.t0 + row) * p.nheads + tn.h] : 0.f;
            An = p.A[tn.h];
            Dn = p.D ? p.D[tn.h] : 0.f;
        }
        Tile prev{};  // tile k-1, whose y this step writes
        for (int k = 0; k <= ntl; ++k) {
            Tile cur{};
            if (k < ntl) {
                cur = tn;
                const float d = dn, Ah = An, Dh = Dn;
                if (k + 1 < ntl) {
                    tn = decode_tile(p, k + 1);
                    dn = (row < tn.valid) ? p.dt[((size_t)tn.b * p.seqlen + tn.t0 + row) * p.nheads + tn.h] : 0.f;
                    An = p.A[tn.h];
                    Dn = p.D ? p.D[tn.h] : 0.f;
                }
                const int s = k & 1;
                float *csk = cs + s * QT, *dtk = dtv + s * QT, *bfk = bfac + s * QT;
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
                if (row == 0) {
                    lam_s[s] = lam;
                    dh_s[s] = Dh;
                }
                bfk[row] = __expf(csk[row & ~31] - v) * d;  // exp(A_cs[r] - A_cs[s]) dt_s, r = s's 32-block start
                named_bar_sync(BAR_MATH, 128);  // every row's decays written
                mbar_arrive(&bars[B_CS + s]);
                // W (one buffer): the previous tile's S must have read it.  With SPLIT,
                // the math warpgroup builds a state-only tile's W.
                if (!(SPLIT && cur.state_only)) {
                    const int xs = k % X_SLOTS;
                    mbar_wait(&bars[B_XFULL + xs], (k / X_SLOTS) & 1, p, abort_s);
                    if (k > 0) mbar_wait(&bars[B_S + (s ^ 1)], ((k - 1) >> 1) & 1, p, abort_s);
                    // W row = exp(lam - A_cs[row]) dt x_row (a row keeps its swizzled chunk
                    // places).  W needs no TMEM lane, so the warp of lane quadrant 3, whose
                    // SM sub-partition also builds the most M blocks, skips it and the warp
                    // of quadrant 0 (the fewest) takes those rows too.
                    auto w_row = [&](int r) {
                        scale_row(sm + OFF_XR + xs * 16384 + r * 128, sm + OFF_W + r * 128, r & 7,
                                  __float2bfloat162_rn(__expf(lam - csk[r]) * dtk[r]));
                    };
                    if (quad != 3) w_row(row);
                    if (quad == 0) w_row(96 + lane);
                    fence_proxy_async_smem();
                    mbar_arrive(&bars[B_W + s]);
                }
            }
            if (k > 0) {  // y of tile k-1
                const int j = k - 1, s = j & 1;
                const uint32_t par = (j >> 1) & 1, tm = tmem + 256 * s + lane_off;
                const Tile t = prev;
                const float e = __expf(cs[s * QT + row]);
                mbar_wait(&bars[B_Y + s], par, p, abort_s);
                tc_fence_after();
                if (!t.state_only) {
                    __nv_bfloat16 *yrow = p.y + (((size_t)t.b * p.seqlen + t.t0 + row) * p.nheads + t.h) * PD;
#pragma unroll 1
                    for (int half = 0; half < 2; ++half) {
                        uint32_t yd[32], yo[32];
                        tmem_ld32x2(tm + COL_YD + 32 * half, tm + COL_YO + 32 * half, yd, yo);
                        if (row < t.valid) {
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                uint32_t pk[4];
#pragma unroll
                                for (int i = 0; i < 4; ++i) {
                                    const int e0 = 8 * q + 2 * i;
                                    pk[i] = pack_bf16x2(fmaf(e, __uint_as_float(yo[e0]), __uint_as_float(yd[e0])),
                                                        fmaf(e, __uint_as_float(yo[e0 + 1]), __uint_as_float(yd[e0 + 1])));
                                }
                                *reinterpret_cast<uint4 *>(yrow + 32 * half + 8 * q) =
                                    make_uint4(pk[0], pk[1], pk[2], pk[3]);
                            }
                        }
                    }
                }
                tc_fence_before();
                mbar_arrive(&bars[B_FREE + s]);
            }
            prev = cur;
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

struct DevInfo {
    bool init = false;
    void *ctx = nullptr;  // the context the kernel attribute was set in
    int sms = 0;
};
DevInfo g_dev[64];
std::mutex g_dev_mu;

// Test-only fault injection (set through ssd_debug_inject_stall).
std::atomic<int> g_withhold{0};
std::atomic<unsigned long long> g_wait_ns{0};

// Split nchunks into `runs` runs so that every run's CTA has about the same
// work: run r streams its run_start[r] predecessors state-only (cost ALPHA per
// chunk relative to a full chunk) and then its own chunks in full.  A state-only
// chunk costs about 0.65 of a full one: it is bound by the latency of its B and X
// loads through the two {C, B} slots, not by its work (measured: 1.7 against
// 2.6 us per chunk at T = 65536, 64 heads).
void split_runs(int nchunks, int runs, int *start) {
    const double ALPHA = 0.65;
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

void set_tc_fault_injection(int withhold, unsigned long long wait_ns) {
    g_wait_ns.store(wait_ns);
    g_withhold.store(withhold ? 1 : 0);
}

bool tc_supported(int headdim, int dstate, int seqlen) {
    return headdim == PD && dstate == ND && seqlen >= QT;
}

// Batch 1: the state between the two halves of the split above, and room for a
// copy of the initial state when the final state overwrites it.
size_t tc_workspace_bytes(int batch, int nheads) {
    return batch == 1 ? 2 * (size_t)nheads * PD * ND * sizeof(float) : 0;
}

namespace {
int device_sms() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        return 148;
    }
    return sms;
}
// Batch 1 with two runs per sequence takes the split (three launches).
bool batch1_split(int batch, int nheads, int seqlen, int sms) {
    const int bH = batch * nheads, nchunks = (seqlen + QT - 1) / QT;
    return batch == 1 && 4 * bH < 3 * sms && std::min({sms / bH, nchunks, MAX_RUNS}) == 2;
}
}  // namespace

int tc_kernel_launches(int batch, int nheads, int seqlen) {
    return batch1_split(batch, nheads, seqlen, device_sms()) ? 3 : 1;
}

namespace {

// One launch for the problem in a.  first > 0: each sequence is scanned over its
// first `first` chunks only, in full, as one run (no state-only prefix, no final
// state).  whole: one run per sequence whatever the SM count.  Otherwise runs
// are chosen as described at split_runs.
cudaError_t launch_one(const ScanArgs &a, cudaStream_t st, int sms, int first, bool whole) {
    cudaError_t e;
    CUtensorMap mx, mb, mc;
    if ((e = make_map(&mx, a.x, a.headdim, a.nheads, a.seqlen, a.batch)) != cudaSuccess) return e;
    if ((e = make_map(&mb, a.B, a.dstate, a.ngroups, a.seqlen, a.batch)) != cudaSuccess) return e;
    if ((e = make_map(&mc, a.C, a.dstate, a.ngroups, a.seqlen, a.batch)) != cudaSuccess) return e;

    TcParams p;
    p.y = static_cast<__nv_bfloat16 *>(a.y);
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
    if (!a.y) {
        // State-only form (no C, no y): every tile of every sequence state-only.
        p.run_start[0] = p.run_start[1] = p.nchunks;
    } else if (first > 0) {
        p.run_start[0] = 0;
        p.run_start[1] = first;
    } else {
        if (!whole && 4 * p.bH < 3 * sms) runs = std::max(1, std::min({sms / p.bH, p.nchunks, MAX_RUNS}));
        split_runs(p.nchunks, runs, p.run_start);
    }
    p.runs = runs;
    p.dev_error = a.dev_error;
    const unsigned long long wns = g_wait_ns.load();
    p.wait_ns = wns ? wns : WAIT_NS;
    p.withhold = g_withhold.load();

    const int items = p.bH * runs;
    const int grid = std::min(items, sms);  // one CTA per SM
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(NTH);
    cfg.dynamicSmemBytes = SMEM_ALLOC;
    cfg.stream = st;
    if (!a.y) return cudaLaunchKernelEx(&cfg, ssd_scan_tc_kernel<true>, mx, mb, mc, p);
    return cudaLaunchKernelEx(&cfg, ssd_scan_tc_kernel<false>, mx, mb, mc, p);
}

// A second stream and two events per device for the batch-1 split below.
struct SplitStream {
    void *ctx = nullptr;
    cudaStream_t s2 = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
};
SplitStream g_split[64];
std::mutex g_split_mu;

// Batch 1, two runs per sequence: instead of the second run replaying the first
// run's chunks inside the launch (a state-only tile costs 0.65 of a full one
// there), a second stream forms the state after the first `s` chunks with the
// state-only form (its own kernel instance: 1.24 against 2.54 us per tile at 64
// heads, alone) and then scans the rest from that state, while the first stream
// scans the first `s` chunks in full.  Each is a launch of one CTA per sequence,
// so the two streams run side by side.  s balances s full tiles against
// ALPHA_SO s state-only and (nchunks - s) full ones; side by side the state-only
// tiles cost more than alone, and 0.60 balanced best (T = 65536, 64 heads:
// 868 us, against 877 at 0.54, 890 at 0.49 and 901 at 0.66).
cudaError_t launch_batch1_split(const ScanArgs &a, float *h_split, cudaStream_t st, int sms, int dev) {
    const double ALPHA_SO = 0.60;
    const int nchunks = (a.seqlen + QT - 1) / QT;
    const int s = std::min(nchunks - 1, std::max(1, (int)(nchunks / (2.0 - ALPHA_SO) + 0.5)));
    cudaError_t e;
    SplitStream &ss = g_split[dev];
    void *ctx = current_context();
    if (ss.ctx != ctx || !ss.s2) {
        ss = SplitStream{};
        if ((e = cudaStreamCreateWithFlags(&ss.s2, cudaStreamNonBlocking)) != cudaSuccess) return e;
        if ((e = cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming)) != cudaSuccess) return e;
        if ((e = cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming)) != cudaSuccess) return e;
        ss.ctx = ctx;
    }
    // the second stream starts where the caller's stream is now
    if ((e = cudaEventRecord(ss.fork, st)) != cudaSuccess) return e;
    if ((e = cudaStreamWaitEvent(ss.s2, ss.fork, 0)) != cudaSuccess) return e;
    ScanArgs first = a;  // chunks 0 .. s-1 in full
    first.final_state = nullptr;
    if ((e = launch_one(first, st, sms, s, false)) != cudaSuccess) return e;
    ScanArgs prefix = a;  // the state after chunk s-1
    prefix.y = nullptr;
    prefix.seqlen = s * QT;
    prefix.final_state = h_split;
    if ((e = launch_one(prefix, ss.s2, sms, 0, false)) != cudaSuccess) return e;
    const size_t t0 = (size_t)s * QT;  // the rest, from that state (batch 1: plain pointer offsets)
    ScanArgs rest = a;
    rest.x = static_cast<const __nv_bfloat16 *>(a.x) + t0 * a.nheads * a.headdim;
    rest.dt = a.dt + t0 * a.nheads;
    rest.B = static_cast<const __nv_bfloat16 *>(a.B) + t0 * a.ngroups * a.dstate;
    rest.C = static_cast<const __nv_bfloat16 *>(a.C) + t0 * a.ngroups * a.dstate;
    rest.y = static_cast<__nv_bfloat16 *>(a.y) + t0 * a.nheads * a.headdim;
    rest.seqlen = a.seqlen - (int)t0;
    rest.init_state = h_split;
    if ((e = launch_one(rest, ss.s2, sms, 0, true)) != cudaSuccess) return e;
    if ((e = cudaEventRecord(ss.join, ss.s2)) != cudaSuccess) return e;
    return cudaStreamWaitEvent(st, ss.join, 0);
}

}  // namespace

cudaError_t launch_tc_scan(const ScanArgs &a, void *ws, cudaStream_t st) {
    cudaError_t e = get_encoder();
    if (e != cudaSuccess) return e;
    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    {
        std::lock_guard<std::mutex> lk(g_dev_mu);
        DevInfo &di = g_dev[dev];
        void *ctx = current_context();
        if (!di.init || di.ctx != ctx) {
            di.init = false;
            if ((e = cudaFuncSetAttribute(ssd_scan_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          SMEM_ALLOC)) != cudaSuccess)
                return e;
            if ((e = cudaFuncSetAttribute(ssd_scan_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          SMEM_ALLOC)) != cudaSuccess)
                return e;
            if ((e = cudaDeviceGetAttribute(&di.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
            di.ctx = ctx;
            di.init = true;
        }
    }
    const int sms = g_dev[dev].sms;
    if (a.y && ws && batch1_split(a.batch, a.nheads, a.seqlen, sms)) {
        // The second stream writes the final state while the first may still read
        // the initial one: when they overlap, both read a copy in the workspace.
        const size_t pn = (size_t)a.nheads * PD * ND;
        float *h_split = static_cast<float *>(ws), *h_copy = h_split + pn;
        ScanArgs b = a;
        if (a.init_state && a.final_state && a.final_state < a.init_state + pn && a.init_state < a.final_state + pn) {
            if ((e = cudaMemcpyAsync(h_copy, a.init_state, pn * sizeof(float), cudaMemcpyDeviceToDevice, st)) !=
                cudaSuccess)
                return e;
            b.init_state = h_copy;
        }
        std::lock_guard<std::mutex> lk(g_split_mu);
        return launch_batch1_split(b, h_split, st, sms, dev);
    }
    return launch_one(a, st, sms, 0, false);
}

}  // namespace ssd
