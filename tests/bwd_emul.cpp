// CPU run of the backward kernels' phases (test infrastructure only).
//
// Each block of every kernel is run here thread by thread, phase by phase, with
// a full barrier between phases -- the same functions the CUDA kernels call
// between __syncthreads().  Shared memory is filled with NaN before each block
// so that reading anything the block did not write shows up in the result.
#include <cmath>
#include <limits>
#include <vector>

#include "scan_bwd_body.cuh"
#include "scan_bwd_complex_body.cuh"


extern "C" int emulate_scan_bwd_real(const float *x, const float *dt, const float *A, const float *B,
                                const float *C, const float *D, const float *init, const float *dy,
                                const float *dfinal, float *dx, float *ddt, float *dA, float *dB,
                                float *dC, float *dD, float *dinit, int batch, int seqlen, int nheads,
                                int headdim, int ngroups, int dstate) {
    using namespace ssd::bwd;
    if (headdim < 1 || headdim > P_MAX || dstate < 1 || dstate > N_MAX || nheads % ngroups) return -1;
    BwdArgs a{};
    a.x = x; a.dt = dt; a.A = A; a.B = B; a.C = C; a.D = D; a.init = init; a.dy = dy; a.dfinal = dfinal;
    a.dx = dx; a.ddt = ddt; a.dA = dA; a.dB = dB; a.dC = dC; a.dD = dD; a.dinit = dinit;
    a.batch = batch; a.seqlen = seqlen; a.nheads = nheads; a.headdim = headdim; a.ngroups = ngroups;
    a.dstate = dstate;
    a.nchunks = (seqlen + QB - 1) / QB;
    std::vector<float> ws(ws_floats(batch, seqlen, nheads, headdim, ngroups, dstate, a.nchunks) + 4,
                          std::numeric_limits<float>::quiet_NaN());
    carve(a, ws.data());
    // Each chunk kernel gets exactly the shared memory its launch asks for, so
    // that an access past it shows up under AddressSanitizer.
    std::vector<float> sm(SMEM_FLOATS), sm1(SMEM_FLOATS_K1), sm3(SMEM_FLOATS_K3);
    const Smem m = smem_map(sm.data()), m1 = smem_map(sm1.data()), m3 = smem_map(sm3.data());
    auto fresh = [&] {
        for (auto *v : {&sm, &sm1, &sm3}) std::fill(v->begin(), v->end(), std::numeric_limits<float>::quiet_NaN());
    };
    auto each = [&](auto &&f) { for (int tid = 0; tid < NT; ++tid) f(tid); };
    const int pn_blocks = (headdim * dstate + NT - 1) / NT;

    if (batch > 0 && a.nchunks > 0) {
        for (int b = 0; b < batch; ++b)
            for (int h = 0; h < nheads; ++h)
                for (int c = 0; c < a.nchunks; ++c) {
                    fresh();
                    each([&](int t) { k1_load(a, c, h, b, t, m1); });
                    each([&](int t) { k1_cumsum(a, c, h, b, t, m1); });
                    each([&](int t) { k1_state(a, c, h, b, t, m1); });
                }
        for (int b = 0; b < batch; ++b)
            for (int h = 0; h < nheads; ++h)
                for (int blk = 0; blk < pn_blocks; ++blk) each([&](int t) { k2_pass(a, blk, h, b, t); });
        for (int b = 0; b < batch; ++b)
            for (int h = 0; h < nheads; ++h)
                for (int c = 0; c < a.nchunks; ++c) {
                    fresh();
                    each([&](int t) { k3_load(a, c, h, b, t, m3); });
                    each([&](int t) { k3_r(a, c, h, b, t, m3); });
                }
        for (int b = 0; b < batch; ++b)
            for (int h = 0; h < nheads; ++h)
                for (int blk = 0; blk < pn_blocks; ++blk) each([&](int t) { k4_pass(a, blk, h, b, t); });
        if (a.gram)
            for (int b = 0; b < batch; ++b)
                for (int g = 0; g < ngroups; ++g)
                    for (int c = 0; c < a.nchunks; ++c) {
                        fresh();
                        each([&](int t) { kg_load(a, c, g, b, t, m3); });
                        each([&](int t) { kg_gram(a, c, g, b, t, m3); });
                    }
        for (int b = 0; b < batch; ++b)
            for (int h = 0; h < nheads; ++h)
                for (int c = 0; c < a.nchunks; ++c) {
                    fresh();
                    each([&](int t) { k5_load(a, c, h, b, t, m); });
                    each([&](int t) { k5_mats(a, t, m); });
                    each([&](int t) { k5_tokens(a, t, m); });
                    each([&](int t) { k5_gb(a, t, m); });
                    each([&](int t) { k5_db(a, c, h, b, t, m); });
                    each([&](int t) { k5_ksr(a, t, m); });
                    each([&](int t) { k5_dc(a, c, h, b, t, m); });
                    each([&](int t) { k5_f(a, t, m); });
                    each([&](int t) {
                        k5_decay(a, c, h, b, t, m);
                        k5_dx(a, c, h, b, t, m);
                    });
                }
        const size_t total = (size_t)batch * seqlen * ngroups * dstate;
        for (size_t i = 0; i < total; ++i) k6_group(a, i);
    } else if (batch > 0) {
        for (int b = 0; b < batch; ++b)
            for (int h = 0; h < nheads; ++h)
                for (int blk = 0; blk < pn_blocks; ++blk) each([&](int t) { k4_pass(a, blk, h, b, t); });
    }
    for (int h = 0; h < nheads; ++h) k6_head(a, h);
    return 0;
}

// The complex variant: A, B, C, init, dfinal and dA, dB, dC, dinit are float pairs.
extern "C" int emulate_scan_bwd_complex(const float *x, const float *dt, const float *A, const float *B,
                                        const float *C, const float *D, const float *init, const float *dy,
                                        const float *dfinal, float *dx, float *ddt, float *dA, float *dB,
                                        float *dC, float *dD, float *dinit, int batch, int seqlen,
                                        int nheads, int headdim, int ngroups, int dstate) {
    using namespace ssd::bwdc;
    if (headdim < 1 || headdim > P_MAX || dstate < 1 || dstate > N_MAX || nheads % ngroups) return -1;
    BwdArgs a{};
    a.x = x; a.dt = dt; a.A = A; a.B = B; a.C = C; a.D = D; a.init = init; a.dy = dy; a.dfinal = dfinal;
    a.dx = dx; a.ddt = ddt; a.dA = dA; a.dB = dB; a.dC = dC; a.dD = dD; a.dinit = dinit;
    a.batch = batch; a.seqlen = seqlen; a.nheads = nheads; a.headdim = headdim; a.ngroups = ngroups;
    a.dstate = dstate;
    a.nchunks = (seqlen + QC - 1) / QC;
    std::vector<float> ws(ws_floats(batch, seqlen, nheads, headdim, dstate, a.nchunks) + 4,
                          std::numeric_limits<float>::quiet_NaN());
    carve(a, ws.data());
    std::vector<float> sm(SMEM_FLOATS), sm1(SMEM_FLOATS_K1), sm3(SMEM_FLOATS_K3);
    const Smem m = smem_map(sm.data()), m1 = smem_map(sm1.data()), m3 = smem_map(sm3.data());
    auto fresh = [&] {
        for (auto *v : {&sm, &sm1, &sm3}) std::fill(v->begin(), v->end(), std::numeric_limits<float>::quiet_NaN());
    };
    auto each = [&](auto &&f) { for (int tid = 0; tid < NT; ++tid) f(tid); };
    const int pn_blocks = (headdim * dstate + NT - 1) / NT;

    if (batch > 0 && a.nchunks > 0) {
        for (int b = 0; b < batch; ++b)
            for (int h = 0; h < nheads; ++h)
                for (int c = 0; c < a.nchunks; ++c) {
                    fresh();
                    each([&](int t) { k1_load(a, c, h, b, t, m1); });
                    each([&](int t) { k1_cumsum(a, c, h, b, t, m1); });
                    each([&](int t) { k1_scale(a, t, m1); });
                    each([&](int t) { k1_state(a, c, h, b, t, m1); });
                }
        for (int b = 0; b < batch; ++b)
            for (int h = 0; h < nheads; ++h)
                for (int blk = 0; blk < pn_blocks; ++blk) each([&](int t) { k2_pass(a, blk, h, b, t); });
        for (int b = 0; b < batch; ++b)
            for (int h = 0; h < nheads; ++h)
                for (int c = 0; c < a.nchunks; ++c) {
                    fresh();
                    each([&](int t) { k3_load(a, c, h, b, t, m3); });
                    each([&](int t) { k3_scale(a, t, m3); });
                    each([&](int t) { k3_r(a, c, h, b, t, m3); });
                }
        for (int b = 0; b < batch; ++b)
            for (int h = 0; h < nheads; ++h)
                for (int blk = 0; blk < pn_blocks; ++blk) each([&](int t) { k4_pass(a, blk, h, b, t); });
        for (int b = 0; b < batch; ++b)
            for (int h = 0; h < nheads; ++h)
                for (int c = 0; c < a.nchunks; ++c) {
                    fresh();
                    each([&](int t) { k5_load(a, c, h, b, t, m); });
                    each([&](int t) { k5_mats(a, t, m); });
                    each([&](int t) { k5_tokens(a, t, m); });
                    each([&](int t) { k5_bc(a, c, h, b, t, m); });
                    each([&](int t) { k5_fk(a, t, m); });
                    each([&](int t) {
                        k5_decay(a, c, h, b, t, m);
                        k5_dx(a, c, h, b, t, m);
                    });
                }
        const size_t total = (size_t)batch * seqlen * ngroups * dstate;
        for (size_t i = 0; i < total; ++i) k6_group(a, i);
    } else if (batch > 0) {
        for (int b = 0; b < batch; ++b)
            for (int h = 0; h < nheads; ++h)
                for (int blk = 0; blk < pn_blocks; ++blk) each([&](int t) { k4_pass(a, blk, h, b, t); });
    }
    for (int h = 0; h < nheads; ++h) k6_head(a, h);
    return 0;
}
