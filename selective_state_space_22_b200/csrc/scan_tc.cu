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
constexpr int NTH = 128;  // threads per CTA: 4 warps, one per TMEM lane quadrant
constexpr int RING = 8;   // published-state slots per sequence
constexpr int DEPTH = 3;  // look-back reads at most this many predecessors
constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t COL_G = 0;    // G (f32, 128 cols), then M in place (bf16 pairs, 64 cols)
constexpr uint32_t COL_YD = 128; // M X                       (64 cols)
constexpr uint32_t COL_S = 192;  // chunk state, then C h^T   (64 cols)
constexpr uint32_t LOAD_BYTES = 2 * (QT * ND * 2) + QT * PD * 2;

// Shared memory (offsets from a 1024-byte aligned base; every operand tile is
// rows of 128 bytes in the 128-byte swizzle pattern TMA writes).
constexpr int OFF_C = 0;          // C   [128 l][128 n]  two 64-column panels
constexpr int OFF_B = 32768;      // B   [128 s][128 n]  two panels
constexpr int OFF_X = 65536;      // X   [128 s][64 p];  later h_in^T bf16 [64 p][128 n]
constexpr int OFF_W = 81920;      // W = diag(w) X;      later the y tile
constexpr int OFF_MISC = 98304;   // cs, dt, column factors, warp sums, mbarriers, TMEM base
constexpr int MISC_BYTES = 3 * QT * 4 + 16 + 5 * 8 + 8;
constexpr int SMEM_ALLOC = OFF_MISC + MISC_BYTES + 1024;

constexpr uint32_t IDESC_G = idesc_bf16_f32(128, 128, 0, 0);   // C (K-major) x B (K-major)
constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 64, 1, 1);    // B^T (MN-major) x W (MN-major)
constexpr uint32_t IDESC_YD = idesc_bf16_f32(128, 64, 0, 1);   // M (TMEM) x X (MN-major)
constexpr uint32_t IDESC_YO = idesc_bf16_f32(128, 64, 0, 0);   // C (K-major) x h (K-major)

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
    float *agg;       // [bH][RING][PD][ND]
    float *pre;       // [bH][RING][PD][ND]
    int seqlen, nheads, ngroups, nchunks, ntiles, bH;
    int *dev_error;
};

__device__ __forceinline__ unsigned long long now_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void report_timeout(int *err) { atomicCAS(err, 0, DEV_TIMEOUT); }

// Bounded wait on an mbarrier phase; false (and the device error set) on timeout.
__device__ bool mbar_wait(uint64_t *bar, uint32_t parity, int *err) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = now_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (now_ns() - t0 > WAIT_NS) {
            report_timeout(err);
            return false;
        }
    }
    return true;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // .x (low half) = lo
    return *reinterpret_cast<uint32_t *>(&v);
}

// Lane 0 of a warp waits until *f satisfies `ready`; the value is broadcast.
template <typename Pred>
__device__ uint32_t warp_wait_flag(const uint32_t *f, Pred ready, int *err, bool &ok) {
    uint32_t v = 0;
    if ((threadIdx.x & 31) == 0) {
        v = ld_acquire_u32(f);
        if (!ready(v)) {
            const unsigned long long t0 = now_ns();
            while (true) {
                __nanosleep(64);
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
    v = __shfl_sync(0xffffffffu, v, 0);
    if (v == 0) ok = false;
    return v;
}

// State entering chunk c of sequence bh for this warp's 32 state rows (n), and
// publication of this chunk's aggregate and prefix.  s[] is the chunk state
// S[n][p] of this thread's row n; hp[] receives h_in[p][n].
__device__ void lookback(const TcParams &p, int bh, int c, int warp, int lane, float lam,
                         const float (&s)[PD], float (&hp)[PD], bool &ok) {
    const int n = warp * 32 + lane;
    const size_t ring0 = (size_t)bh * RING;
    const int slot = c % RING;
    uint32_t *flag = p.flags + (ring0 + slot) * 4 + warp;
    float *aggp = p.agg + (ring0 + slot) * (PD * ND) + n;
    float *prep = p.pre + (ring0 + slot) * (PD * ND) + n;

    // Reuse of this slot: the chunk that last used it (c - RING) and the chunks
    // that may still read it (up to c - RING + DEPTH) must all have published
    // their prefixes (a later chunk in their slot also proves it).
    if (c >= RING) {
        for (int k = 0; k <= DEPTH; ++k) {
            const int j = c - RING + k;
            const uint32_t *f = p.flags + (ring0 + j % RING) * 4 + warp;
            warp_wait_flag(f, [j](uint32_t v) {
                return (int)(v >> 2) > j || ((int)(v >> 2) == j && (v & 3u) == ST_PREFIX);
            }, p.dev_error, ok);
        }
    }

    if (c == 0) {
        if (p.init_state) {
            const float *h0 = p.init_state + (size_t)bh * PD * ND + n;
#pragma unroll
            for (int q = 0; q < PD; ++q) hp[q] = h0[q * ND];
        } else {
#pragma unroll
            for (int q = 0; q < PD; ++q) hp[q] = 0.f;
        }
    } else {
#pragma unroll
        for (int q = 0; q < PD; ++q) aggp[q * ND] = s[q];
        if (lane == 0) p.lam[(ring0 + slot) * 4 + warp] = lam;
        __threadfence();
        __syncwarp();
        if (lane == 0) st_release_u32(flag, ((uint32_t)c << 2) | ST_AGG);

#pragma unroll
        for (int q = 0; q < PD; ++q) hp[q] = 0.f;
        float dec = 0.f;
        for (int j = c - 1; j >= 0; --j) {
            const int sj = j % RING;
            const uint32_t *f = p.flags + (ring0 + sj) * 4 + warp;
            const bool need_prefix = (j == c - DEPTH) || (j == 0);
            const uint32_t v = warp_wait_flag(f, [j, need_prefix](uint32_t v) {
                return (int)(v >> 2) == j && ((v & 3u) == ST_PREFIX || (!need_prefix && (v & 3u) == ST_AGG));
            }, p.dev_error, ok);
            const bool is_prefix = (v & 3u) == ST_PREFIX || v == 0;
            const float fd = __expf(dec);
            const float *src = (is_prefix ? p.pre : p.agg) + (ring0 + sj) * (PD * ND) + n;
#pragma unroll
            for (int q = 0; q < PD; ++q) hp[q] = fmaf(fd, __ldcg(src + q * ND), hp[q]);
            if (is_prefix) break;
            dec += __ldcg(p.lam + (ring0 + sj) * 4 + warp);
        }
    }

    const float el = __expf(lam);
    const bool last = (c == p.nchunks - 1) && p.final_state;
    float *fin = last ? p.final_state + (size_t)bh * PD * ND + n : nullptr;
#pragma unroll
    for (int q = 0; q < PD; ++q) {
        const float hc = fmaf(el, hp[q], s[q]);
        prep[q * ND] = hc;
        if (last) fin[q * ND] = hc;
    }
    __threadfence();
    __syncwarp();
    if (lane == 0) st_release_u32(flag, ((uint32_t)c << 2) | ST_PREFIX);
}

__global__ void __launch_bounds__(NTH, 2)
    ssd_scan_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
                       const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_y,
                       const TcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sC = sm + OFF_C, *sB = sm + OFF_B, *sX = sm + OFF_X, *sW = sm + OFF_W;
    float *cs = reinterpret_cast<float *>(sm + OFF_MISC);
    float *dtv = cs + QT;
    float *bfac = dtv + QT;
    float *wtot = bfac + QT;
    uint64_t *bars = reinterpret_cast<uint64_t *>(wtot + 4);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 5);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int i = 0; i < 5; ++i) mbar_init(&bars[i], 1);
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
    const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);  // this warp's TMEM lane quadrant

    const int T = p.seqlen, H = p.nheads, hpg = p.nheads / p.ngroups;
    const uint32_t aC = smem_u32(sC), aB = smem_u32(sB), aX = smem_u32(sX), aW = smem_u32(sW);
    uint32_t ph = 0;
    bool ok = true;

    for (int tile = blockIdx.x; tile < p.ntiles; tile += gridDim.x) {
        const int c = tile / p.bH, bh = tile % p.bH;
        const int b = bh / H, h = bh % H, g = h / hpg;
        const int t0 = c * QT, valid = min(QT, T - t0);

        if (tid == 0) bulk_wait_group_read0();  // the previous y store has read sW
        if (!__syncthreads_and(ok)) break;      // a timed-out wait ends the CTA's work
        if (tid == 0) {
            mbar_arrive_expect_tx(&bars[0], LOAD_BYTES);
            tma_load_4d(sC, &tm_c, &bars[0], 0, g, t0, b);
            tma_load_4d(sC + 16384, &tm_c, &bars[0], 64, g, t0, b);
            tma_load_4d(sB, &tm_b, &bars[0], 0, g, t0, b);
            tma_load_4d(sB + 16384, &tm_b, &bars[0], 64, g, t0, b);
            tma_load_4d(sX, &tm_x, &bars[0], 0, h, t0, b);
        }

        // dt, dA = dt*A, inclusive cumulative sum over the chunk (row s = tid)
        const float d = (tid < valid) ? p.dt[((size_t)b * T + t0 + tid) * H + h] : 0.f;
        float v = d * p.A[h];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += y;
        }
        if (lane == 31) wtot[warp] = v;
        __syncthreads();
        for (int w = 0; w < warp; ++w) v += wtot[w];
        cs[tid] = v;
        dtv[tid] = d;
        __syncthreads();
        const float lam = cs[QT - 1];
        // exp(A_cs[r] - A_cs[s]) dt_s with r the first row of s's 32-row block
        bfac[tid] = __expf(cs[tid & ~31] - v) * d;

        if (!mbar_wait(&bars[0], ph, p.dev_error)) ok = false;

        if (tid == 0) {  // G = C B^T
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
                mma_ss(tmem + COL_G, smem_desc_sw128(aC + off, 16, 1024), smem_desc_sw128(aB + off, 16, 1024),
                       IDESC_G, k > 0);
            }
            mma_commit(&bars[1]);
        }

        {  // W row s = exp(lam - A_cs[s]) dt_s x_s  (rows keep their swizzled 16-byte chunks)
            const float w = __expf(lam - v) * d;
            const uint4 *src = reinterpret_cast<const uint4 *>(sX + tid * 128);
            uint4 *dst = reinterpret_cast<uint4 *>(sW + tid * 128);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                uint4 q = src[j];
                uint32_t *u = reinterpret_cast<uint32_t *>(&q);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    __nv_bfloat162 pr = *reinterpret_cast<__nv_bfloat162 *>(&u[e]);
                    float2 f = __bfloat1622float2(pr);
                    u[e] = pack_bf16x2(f.x * w, f.y * w);
                }
                dst[j] = q;
            }
        }
        fence_proxy_async_smem();
        __syncthreads();

        if (tid == 0) {  // S = B^T W (chunk state, rows n)
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < 8; ++k)
                mma_ss(tmem + COL_S, smem_desc_sw128(aB + k * 2048, 16384, 1024),
                       smem_desc_sw128(aW + k * 2048, 8192, 1024), IDESC_S, k > 0);
            mma_commit(&bars[2]);
        }

        // M = G o L o dt (+ D on the diagonal), bf16, in place in TMEM
        if (!mbar_wait(&bars[1], ph, p.dev_error)) ok = false;
        tc_fence_after();
        {
            const int l = tid;
            const float csl = v;
            const float Dh = p.D ? p.D[h] : 0.f;
#pragma unroll 1
            for (int j = 0; j < 4; ++j) {
                uint32_t packed[16];
                if (j > warp) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) packed[i] = 0u;
                } else {
                    uint32_t gr[32];
                    tmem_ld32(trow + COL_G + 32 * j, gr);
                    const int r = 32 * j;
                    const bool direct = fabsf(cs[r] - cs[r + 31]) > 80.f;
                    const float a = __expf(csl - cs[r]);
                    float m[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int s = r + i;
                        const float L = direct ? __expf(csl - cs[s]) * dtv[s] : a * bfac[s];
                        float mv = (s <= l) ? __uint_as_float(gr[i]) * L : 0.f;
                        if (s == l) mv += Dh;
                        m[i] = mv;
                    }
#pragma unroll
                    for (int i = 0; i < 16; ++i) packed[i] = pack_bf16x2(m[2 * i], m[2 * i + 1]);
                }
                tmem_st16(trow + COL_G + 16 * j, packed);
            }
            tmem_wait_st();
        }
        tc_fence_before();
        __syncthreads();

        if (tid == 0) {  // Y = M X
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < 8; ++k)
                mma_ts(tmem + COL_YD, tmem + COL_G + 8 * k, smem_desc_sw128(aX + k * 2048, 8192, 1024), IDESC_YD,
                       k > 0);
            mma_commit(&bars[3]);
        }

        // chunk state -> look-back -> state entering the chunk
        if (!mbar_wait(&bars[2], ph, p.dev_error)) ok = false;
        tc_fence_after();
        float s_reg[PD];
        {
            uint32_t r[32];
            tmem_ld32(trow + COL_S, r);
#pragma unroll
            for (int i = 0; i < 32; ++i) s_reg[i] = __uint_as_float(r[i]);
            tmem_ld32(trow + COL_S + 32, r);
#pragma unroll
            for (int i = 0; i < 32; ++i) s_reg[32 + i] = __uint_as_float(r[i]);
        }
        float hp[PD];
        lookback(p, bh, c, warp, lane, lam, s_reg, hp, ok);

        // h_in^T as bf16 (K-major, rows p, 128-byte swizzle) over X, once M X is done
        if (!mbar_wait(&bars[3], ph, p.dev_error)) ok = false;
        {
            const int n = tid;
            const uint32_t base = (n >> 6) * 8192 + (n & 7) * 2;
            const uint32_t chunk = (n & 63) >> 3;
#pragma unroll
            for (int q = 0; q < PD; ++q) {
                const uint32_t off = base + q * 128 + ((chunk ^ (q & 7)) << 4);
                *reinterpret_cast<__nv_bfloat16 *>(sX + off) = __float2bfloat16_rn(hp[q]);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        if (tid == 0) {  // Y_off = C h_in^T
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t aoff = (k >> 2) * 16384 + (k & 3) * 32;
                const uint32_t boff = (k >> 2) * 8192 + (k & 3) * 32;
                mma_ss(tmem + COL_S, smem_desc_sw128(aC + aoff, 16, 1024), smem_desc_sw128(aX + boff, 16, 1024),
                       IDESC_YO, k > 0);
            }
            mma_commit(&bars[4]);
        }
        if (!mbar_wait(&bars[4], ph, p.dev_error)) ok = false;
        tc_fence_after();

        {  // y = Y + exp(A_cs[l]) Y_off -> bf16 -> y tile (rows l, 128-byte swizzle)
            const float e = __expf(v);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t yd[32], yo[32];
                tmem_ld32(trow + COL_YD + 32 * half, yd);
                tmem_ld32(trow + COL_S + 32 * half, yo);
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    pk[i] = pack_bf16x2(fmaf(e, __uint_as_float(yo[2 * i]), __uint_as_float(yd[2 * i])),
                                        fmaf(e, __uint_as_float(yo[2 * i + 1]), __uint_as_float(yd[2 * i + 1])));
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int chunk = 4 * half + q;
                    const int phys = chunk ^ (tid & 7);
                    *reinterpret_cast<uint4 *>(sW + tid * 128 + phys * 16) =
                        make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tma_store_4d(&tm_y, sW, 0, h, t0, b);
            bulk_commit_group();
        }
        ph ^= 1;
    }

    if (tid == 0) bulk_wait_group0();
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

    const int grid = std::min(p.ntiles, di.per_sm * di.sms);
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
