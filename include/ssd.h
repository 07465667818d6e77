/*
 * ssd.h -- C ABI of the B200 selective state-space (SSD) scan library, libssd.so.
 *
 * The operation (all three entry points evaluate the same recurrence):
 *
 *   h_t = exp(dt_t * A_h) * h_{t-1} + dt_t * x_t B_t^T          (state P x N per head)
 *   y_t = Re( h_t C_t ) + D_h * x_t                             (output P per head)
 *
 * Sources: "Mamba-3-Lite" README, the section on the classical (real) Mamba-2
 * recurrence and its complex promotion; "Block Anatomy, Numerical Stability &
 * Scaling" -- Block Anatomy section 3 (the interface: (B,T,H,D)-shaped inputs in,
 * a (B,T,H,D) real output out), section 4.3 (x and dt stay float32, B and C are
 * complex64), section 4.4 (one complex A per head, decay exp(softplus(dt) A)),
 * section 6 (the real part of the output leaves the scan; the state starts at
 * zero); Numerical Stability section 4 (the chunkwise form: within-chunk decay
 * exp(segsum(dt A)) and the inter-chunk propagation).  "BitMamba 1B" (Portuguese
 * edition, "Contexto") gives the Mamba-2 layer shape: 64 heads, d_state 128,
 * d_inner 4096 (head dim 64), one real A per head.
 *
 * Conventions shared by every entry point
 *  - Every tensor pointer is a DEVICE pointer to contiguous row-major memory,
 *    16-byte aligned.  The caller owns all memory; nothing is allocated, freed
 *    or retained by the library.
 *  - Work is enqueued on `stream` (a cudaStream_t passed as void*; NULL is the
 *    legacy default stream) and is asynchronous: a returned SSD_OK means the
 *    launch was accepted, not that it finished.
 *  - Arguments are validated on the host before any launch; on a non-OK status
 *    nothing was launched and ssd_last_error() describes why.
 *  - dt is the step size AFTER softplus and dt_bias (the library applies no
 *    softplus).  Head h reads group h / (nheads / ngroups) of B and C.
 *  - The input is injected as dt_t * x_t B_t^T and the output reads the state
 *    after that step's update.
 *  - Complex tensors are interleaved (re, im) float pairs, the memory layout of
 *    a complex64 tensor.  The complex output is the real part only.
 *  - Outputs never alias inputs, except: final_state may equal init_state, and
 *    ssd_state_update updates `state` in place.
 *  - Device addresses the library caches (its error word, the no-alloc scratch)
 *    and kernel attributes are kept per (device, current CUDA context) and looked
 *    up again when the context changes.  Work enqueued before a cudaDeviceReset
 *    must not be waited on with ssd_get_device_status afterwards.
 */
#ifndef SSD_B200_H
#define SSD_B200_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SSD_OK = 0,
    SSD_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size; nothing launched */
    SSD_ERR_UNSUPPORTED = 2,   /* valid arguments this build has no kernel for */
    SSD_ERR_CUDA = 3,          /* a CUDA runtime call failed (launch or query) */
    SSD_ERR_TIMEOUT = 4,       /* a bounded inter-block wait gave up (device-side) */
    SSD_ERR_WORKSPACE = 5      /* workspace NULL or smaller than ssd_scan_workspace_size */
} ssd_status;

typedef enum {
    SSD_F32 = 0,   /* float32 */
    SSD_BF16 = 1   /* bfloat16 */
} ssd_dtype;

/* Returned by ssd_scan_workspace_size for sizes that no scan accepts. */
#define SSD_WORKSPACE_INVALID ((size_t)-1)

/*
 * Workspace bytes that ssd_scan_fwd / ssd_scan_fwd_complex need for these sizes:
 * 0 when the selected kernel needs none (then the workspace argument may be
 * NULL), SSD_WORKSPACE_INVALID when the sizes are invalid.  The workspace needs
 * no initialisation: every value is written before it is read.  One workspace
 * may not be used by two calls that can run at the same time (different
 * streams): they would race.
 */
size_t ssd_scan_workspace_size(int batch, int seqlen, int nheads, int headdim,
                               int ngroups, int dstate, int chunk_size,
                               int is_complex, ssd_dtype io_dtype);

/*
 * Number of kernels that one ssd_scan_fwd / ssd_scan_fwd_complex call with these
 * sizes enqueues when seqlen > 0 (0 for invalid sizes).  For capture planning
 * and launch accounting; it launches nothing.
 */
int ssd_scan_kernel_launches(int batch, int seqlen, int nheads, int headdim, int ngroups,
                             int dstate, int chunk_size, int is_complex, ssd_dtype io_dtype);

/*
 * Real chunked scan (Mamba-2 layout, one real A per head).
 *
 *  x           [batch, seqlen, nheads, headdim]  io_dtype
 *  dt          [batch, seqlen, nheads]           float32, > 0 (post-softplus)
 *  A           [nheads]                          float32, expected <= 0
 *  B, C        [batch, seqlen, ngroups, dstate]  io_dtype
 *  D           [nheads] float32, or NULL for no skip term
 *  init_state  [batch, nheads, headdim, dstate] float32, or NULL for zeros
 *  final_state [batch, nheads, headdim, dstate] float32, or NULL to skip
 *  y           [batch, seqlen, nheads, headdim]  io_dtype (output)
 *  chunk_size  chunk length of the chunkwise evaluation: 64, 128 or 256.  The
 *              result does not depend on it beyond rounding.
 *  workspace   device scratch of at least ssd_scan_workspace_size(...) bytes.
 *
 * seqlen may be 0 (then y is empty and final_state = init_state, or zeros) and
 * need not be a multiple of chunk_size.  io_dtype SSD_BF16 with headdim 64,
 * dstate 128 and seqlen >= 128 runs the tcgen05 tensor-core kernel: one launch,
 * no workspace, bitwise reproducible.  With batch 1 it takes a workspace of
 * nheads * headdim * dstate * 4 bytes: when each sequence is cut in two (fewer
 * sequences than SMs), the state between the halves is formed by a state-only
 * launch on an internal second stream while the caller's stream scans the first
 * half (three launches, joined back to the caller's stream before the call's work
 * ends; the same bits as the one-launch form).  The first such call on a device
 * creates that stream and two events, so it should come before any stream capture.  It evaluates 128-token chunks
 * (its MMA tile height) whatever chunk_size says.  Every other combination runs the
 * float32 CUDA-core kernels (three launches, a workspace), which honour
 * chunk_size.  State and accumulation are float32 in both.
 */
ssd_status ssd_scan_fwd(const void *x, const float *dt, const float *A,
                        const void *B, const void *C, const float *D,
                        const float *init_state, float *final_state, void *y,
                        ssd_dtype io_dtype, int batch, int seqlen, int nheads,
                        int headdim, int ngroups, int dstate, int chunk_size,
                        void *workspace, size_t workspace_bytes, void *stream);

/*
 * Complex chunked scan (Mamba-3-Lite layout, one complex A per head).
 *
 *  x           [batch, seqlen, nheads, headdim]       float32 (real)
 *  dt          [batch, seqlen, nheads]                float32
 *  A           [nheads] complex (float pairs), Re A expected <= 0
 *  B, C        [batch, seqlen, ngroups, dstate] complex
 *  D           [nheads] float32 or NULL
 *  init_state  [batch, nheads, headdim, dstate] complex, or NULL for zeros
 *  final_state [batch, nheads, headdim, dstate] complex, or NULL
 *  y           [batch, seqlen, nheads, headdim] float32 = Re(h_t C_t) + D x_t
 *
 * Three launches and a workspace (ssd_scan_workspace_size with is_complex = 1):
 * chunk states, the state pass over chunks, the chunk scan.  Every contraction
 * is a real product over the 2 dstate interleaved (re, im) values, with the
 * complex decay folded into C and B.  headdim 64 and dstate 64 (the Mamba-3-Lite
 * head) run the chunk states and chunk scan on tcgen05 tensor cores in
 * 128-token chunks, with each float32 operand split into bf16 hi and lo parts
 * and three products per contraction (float32 accumulation; about 1e-5 of the
 * float32 result), and chunks whose real log-decay spans more than 140 on
 * CUDA cores; other sizes run float32 CUDA-core kernels that honour chunk_size.
 * State and accumulation are float32 (complex64).  Other arguments as
 * ssd_scan_fwd.
 */
ssd_status ssd_scan_fwd_complex(const float *x, const float *dt, const float *A,
                                const float *B, const float *C, const float *D,
                                const float *init_state, float *final_state, float *y,
                                int batch, int seqlen, int nheads, int headdim,
                                int ngroups, int dstate, int chunk_size,
                                void *workspace, size_t workspace_bytes, void *stream);

/*
 * The complex scan reading the packed input-projection output directly.
 *
 * "Block Anatomy, Numerical Stability & Scaling", Block Anatomy section 4.1-4.3:
 * a Mamba-3-Lite block's projection emits per token W = H (D + 4N + 1) values in
 * head-major slices, in this order: x (H*D), Re B (H*N), Im B (H*N), Re C
 * (H*N), Im C (H*N), dt (H); Numerical Stability section 4 (_discretise) applies
 * softplus to dt.  This call reads those slices in place (float32 or bf16,
 * widened exactly), pairs the real and imaginary parts, and computes
 * dt = softplus(dt_raw + dt_bias[h]) inside the scan's own loads, so the
 * separate unpacking pass of the block (the float32 copies and the complex64
 * B and C) never touches HBM.  The result equals ssd_scan_fwd_complex given the
 * unpacked tensors.
 *
 *  proj        [batch, seqlen, W] in proj_dtype, W = nheads (headdim + 4 dstate + 1)
 *  dt_bias     [nheads] float32 added before the softplus, or NULL for none
 *  A, D, init_state, final_state, y, chunk_size, workspace: as ssd_scan_fwd_complex,
 *  with one group per head (ngroups = nheads; workspace from
 *  ssd_scan_workspace_size(batch, seqlen, nheads, headdim, nheads, dstate,
 *  chunk_size, 1, SSD_F32)).
 */
ssd_status ssd_scan_fwd_complex_packed(const void *proj, ssd_dtype proj_dtype,
                                       const float *dt_bias, const float *A, const float *D,
                                       const float *init_state, float *final_state, float *y,
                                       int batch, int seqlen, int nheads, int headdim,
                                       int dstate, int chunk_size, void *workspace,
                                       size_t workspace_bytes, void *stream);

/*
 * Sequence split across devices, step 1: the final state of a slice of the
 * sequence, and its total log-decay, without its outputs.
 *
 * "Block Anatomy, Numerical Stability & Scaling" (Numerical Stability, section
 * 4) carries each chunk's end state into later chunks through the decay between
 * them; the same holds for consecutive slices of a sequence held by different
 * devices.  A device scans its slice from a zero state (the first slice from
 * the caller's initial state) with this call, which runs the state part of the
 * scan only (cumulative decay, chunk states, state passing; no C, no y).
 *
 *  x, dt, A, B, init_state, io_dtype, sizes, chunk_size, workspace: as
 *    ssd_scan_fwd (same workspace size).
 *  final_state      [batch, nheads, headdim, dstate] float32, required.
 *  total_log_decay  [batch, nheads] float32 = A[h] * sum over the slice of
 *    dt[b, t, h] (summed in double), or NULL.
 * For seqlen 0 the final state is init_state (or zeros) and the log-decay 0.
 */
ssd_status ssd_scan_final_state(const void *x, const float *dt, const float *A,
                                const void *B, const float *init_state,
                                float *final_state, float *total_log_decay,
                                ssd_dtype io_dtype, int batch, int seqlen, int nheads,
                                int headdim, int ngroups, int dstate, int chunk_size,
                                void *workspace, size_t workspace_bytes, void *stream);

/*
 * Sequence split across devices, step 2: the state entering a slice.
 *
 * Given the final states S_0 .. S_{n-1} of the n slices before it (S_0 from the
 * caller's initial state, the others from zero) and their total log-decays,
 * out = h_{n-1} with h_0 = S_0 and h_j = exp(log_decay_j) h_{j-1} + S_j, the
 * inter-chunk recurrence of the pages applied per slice.  Elementwise, float32.
 *
 *  states     [nstates, batch, nheads, headdim, dstate] float32
 *  log_decay  [nstates, batch, nheads] float32 (entry 0 unused; may be NULL
 *             when nstates == 1)
 *  out        [batch, nheads, headdim, dstate] float32 (may not alias states)
 */
ssd_status ssd_fold_states(const float *states, const float *log_decay, int nstates,
                           float *out, int batch, int nheads, int headdim, int dstate,
                           void *stream);

/*
 * The causal depthwise convolution Mamba-1 and Mamba-2 run before the scan
 * ("Block Anatomy, Numerical Stability & Scaling", Block Anatomy section 5.1:
 * each channel at position t becomes a learned combination of positions
 * t-K+1 .. t, K = 4), over the packed x | B | C channels of a Mamba-2 input
 * projection, written straight into the scan's separate inputs:
 *
 *   out[b,t,c] = act(bias[c] + sum_{k<K} weight[c,k] * xbc[b, t-K+1+k, c])
 *
 * with act the identity, or SiLU v / (1 + exp(-v)) when silu != 0 (the pages
 * name the convolution only; Mamba-2 follows it with SiLU).  Positions before
 * t = 0 read conv_init (the last K-1 inputs of a preceding part of the same
 * sequence) or zero.
 *
 *  xbc        [batch, seqlen, x_channels + 2 bc_channels]  io_dtype
 *  weight     [x_channels + 2 bc_channels, width] float32; bias the same
 *             channels, float32, or NULL
 *  conv_init  [batch, x_channels + 2 bc_channels, width - 1] io_dtype, or NULL
 *  x_out      [batch, seqlen, x_channels] io_dtype (channels 0 .. x_channels-1;
 *             for the scan: [batch, seqlen, nheads, headdim])
 *  B_out, C_out [batch, seqlen, bc_channels] io_dtype (the next two channel
 *             ranges; for the scan: [batch, seqlen, ngroups, dstate])
 *  conv_final [batch, x_channels + 2 bc_channels, width - 1] io_dtype, or NULL:
 *             the last width-1 inputs, the conv_init of a continuation
 *  width      1 .. 8.
 * Float32 arithmetic; one read of every input, one write of every output.
 */
ssd_status ssd_conv1d_xbc(const void *xbc, const float *weight, const float *bias,
                          const void *conv_init, void *x_out, void *B_out, void *C_out,
                          void *conv_final, ssd_dtype io_dtype, int batch, int seqlen,
                          int x_channels, int bc_channels, int width, int silu, void *stream);

/*
 * The Mamba-1 selective scan: one decay rate per state component ("Block
 * Anatomy, Numerical Stability & Scaling", Block Anatomy section 4.4: A of shape
 * (H, N); the "Mamba-50M" card: a Mamba selective-SSM language model).  Each
 * channel d has its own step and dstate states:
 *
 *   h_t[n] = exp(dt_t[d] A[d,n]) h_{t-1}[n] + dt_t[d] B_t[n] x_t[d]
 *   y_t[d] = sum_n C_t[n] h_t[n] + D[d] x_t[d]
 *
 *  x, y        [batch, seqlen, channels]  io_dtype
 *  dt          [batch, seqlen, channels]  float32 (after softplus and bias)
 *  A           [channels, dstate]         float32
 *  B, C        [batch, seqlen, ngroups, dstate]  io_dtype; channel d reads group
 *              d / (channels / ngroups)
 *  D           [channels] float32 or NULL
 *  init_state, final_state [batch, channels, dstate] float32 or NULL
 *  dstate      4, 8, 16 or 32 (SSD_ERR_UNSUPPORTED otherwise).
 * Sequential in time (the per-state decay has no chunked matrix form),
 * parallel over (batch, channel): one launch, no workspace, float32 state.
 */
ssd_status ssd_selective_scan(const void *x, const float *dt, const float *A, const void *B,
                              const void *C, const float *D, const float *init_state,
                              float *final_state, void *y, ssd_dtype io_dtype, int batch,
                              int seqlen, int channels, int ngroups, int dstate, void *stream);

/*
 * One recurrent decoding step, in place on the state (real variant):
 *   state <- exp(dt A) state + dt x B^T ;  y = state C + D x
 *
 *  state [batch, nheads, headdim, dstate] float32, read and overwritten
 *  x     [batch, nheads, headdim]  io_dtype
 *  dt    [batch, nheads]           float32
 *  A     [nheads] float32;  B, C [batch, ngroups, dstate] io_dtype
 *  D     [nheads] float32 or NULL;  y [batch, nheads, headdim] io_dtype (output)
 *
 * Needs no workspace.  "batch" is the number of sequences decoded together.
 */
ssd_status ssd_state_update(float *state, const void *x, const float *dt,
                            const float *A, const void *B, const void *C,
                            const float *D, void *y, ssd_dtype io_dtype, int batch,
                            int nheads, int headdim, int ngroups, int dstate,
                            void *stream);

/* The complex decoding step: state, A, B, C complex; x, dt, D, y float32. */
ssd_status ssd_state_update_complex(float *state, const float *x, const float *dt,
                                    const float *A, const float *B, const float *C,
                                    const float *D, float *y, int batch, int nheads,
                                    int headdim, int ngroups, int dstate, void *stream);

/*
 * Gradients of the real scan, float32, for training through it.
 *
 * The loss is L = sum_t <dy_t, y_t> + <dfinal, final_state>: dy and dfinal are
 * the gradients arriving at the outputs y and final_state of ssd_scan_fwd.  The
 * pages train through the scan ("Block Anatomy, Numerical Stability & Scaling",
 * Numerical Stability section 5.3: the backward differentiates the products of
 * the exp factors) but print no backward formula; this is the chain rule through
 * the recurrence above, evaluated in 64-token chunks.
 *
 * Inputs (float32, as ssd_scan_fwd with io_dtype SSD_F32):
 *  x [batch, seqlen, nheads, headdim], dt [batch, seqlen, nheads], A [nheads],
 *  B, C [batch, seqlen, ngroups, dstate], D [nheads] or NULL,
 *  init_state [batch, nheads, headdim, dstate] or NULL (zeros),
 *  dy [batch, seqlen, nheads, headdim], dfinal [batch, nheads, headdim, dstate]
 *  or NULL (zeros).
 * Outputs (float32, every element written):
 *  dx, ddt, dA [nheads], dB and dC [batch, seqlen, ngroups, dstate] (summed over
 *  the heads of each group), dD [nheads] or NULL (not computed),
 *  dinit [batch, nheads, headdim, dstate] or NULL (not computed).  dD is the
 *  gradient for D whether or not D was given.
 *
 * Limits: headdim <= 64 and dstate <= 128 (SSD_ERR_UNSUPPORTED otherwise).  Runs
 * in seven launches (eight when heads share a group: C B^T once per group and
 * chunk); with headdim 64 and dstate 128 the chunk states and the
 * readout terms are tcgen05 products (bf16 hi/lo, three products, float32
 * accumulation), the rest CUDA cores.  Sums are taken in a fixed order, so
 * repeated calls give identical bits.  The workspace (ssd_scan_bwd_workspace_size bytes,
 * caller-owned, 16-byte aligned, no initialisation needed) holds the chunk
 * states, the state gradients and per-head partial sums; it grows with
 * batch * nheads * ceil(seqlen / 64) * headdim * dstate * 12 bytes plus
 * batch * seqlen * nheads * dstate * 8 bytes, plus, when the heads of a group
 * share B and C (nheads / ngroups >= 2), each chunk's C B^T once per group:
 * batch * ngroups * ceil(seqlen / 64) * 16 KB.  SSD_ERR_WORKSPACE when it is NULL
 * or too small.
 */
size_t ssd_scan_bwd_workspace_size(int batch, int seqlen, int nheads, int headdim,
                                   int ngroups, int dstate);

ssd_status ssd_scan_bwd(const float *x, const float *dt, const float *A, const float *B,
                        const float *C, const float *D, const float *init_state,
                        const float *dy, const float *dfinal, float *dx, float *ddt,
                        float *dA, float *dB, float *dC, float *dD, float *dinit,
                        int batch, int seqlen, int nheads, int headdim, int ngroups,
                        int dstate, void *workspace, size_t workspace_bytes, void *stream);

/*
 * Gradients of the complex scan (the Mamba-3-Lite variant), float32.
 *
 * The loss is L = sum_t <dy_t, y_t> + Re <dfinal, final_state> with
 * y_t = Re(h_t C_t) + D x_t.  A [nheads], B and C [batch, seqlen, ngroups, dstate],
 * init_state and dfinal [batch, nheads, headdim, dstate] are complex (interleaved
 * float pairs), as are the outputs dA, dB, dC and dinit; x, dt, D, dy, dx, ddt
 * and dD are float32.  For a complex z = u + iv the gradient written is
 * dL/du + i dL/dv.  Limits: headdim <= 64 and dstate <= 64; the chunk is 32
 * tokens.  With headdim 64 and dstate 64 the chunk states and readout terms are
 * tcgen05 products, as in ssd_scan_bwd.  Workspace from
 * ssd_scan_bwd_complex_workspace_size.  Everything else as ssd_scan_bwd.
 */
size_t ssd_scan_bwd_complex_workspace_size(int batch, int seqlen, int nheads, int headdim,
                                           int ngroups, int dstate);

ssd_status ssd_scan_bwd_complex(const float *x, const float *dt, const float *A,
                                const float *B, const float *C, const float *D,
                                const float *init_state, const float *dy, const float *dfinal,
                                float *dx, float *ddt, float *dA, float *dB, float *dC,
                                float *dD, float *dinit, int batch, int seqlen, int nheads,
                                int headdim, int ngroups, int dstate, void *workspace,
                                size_t workspace_bytes, void *stream);

/*
 * Waits for `stream`, then reports and clears an error that a kernel raised on
 * the device since the last call on this device (SSD_ERR_TIMEOUT when one of the
 * tensor-core kernel's bounded waits between its warp roles gave up after 1 s;
 * the kernel then stops at once and the outputs of that call are invalid), or a
 * CUDA error from the stream.
 * SSD_OK when there was none.
 */
ssd_status ssd_get_device_status(void *stream);

/*
 * Size of the fixed scratch array behind ssd_scan_fwd_noalloc (16 MiB).  Every
 * GPU that loads this library holds it until the process exits.
 */
#define SSD_NOALLOC_SCRATCH_BYTES (16u << 20)

/*
 * ssd_scan_fwd_noalloc -- the real scan for callers that cannot allocate.
 *
 * (The pages have no counterpart to this entry point.)  Some callers cannot call
 * cudaMalloc or hand over a workspace: a plugin inside a host application that
 * owns all device memory, a path where an allocation's latency or implicit
 * synchronisation is not acceptable.  This variant takes the same arguments as
 * ssd_scan_fwd minus the workspace, and keeps its scratch in a fixed device
 * array of SSD_NOALLOC_SCRATCH_BYTES inside the library.  It allocates and frees
 * nothing, ever.
 *
 *  - It runs the float32 CUDA-core scan (for bf16 or float32 io).  Sizes whose
 *    scratch exceeds SSD_NOALLOC_SCRATCH_BYTES are rejected with
 *    SSD_ERR_WORKSPACE before anything is launched.  The scratch needed is
 *    batch * nheads * ceil(seqlen / chunk_size) * (headdim * dstate * 4 +
 *    chunk_size * 8 + 8) bytes plus up to 768 bytes of alignment padding.
 *    batch and seqlen must be > 0.
 *  - The first call on a device (and the first after the current CUDA context
 *    changed, e.g. after cudaDeviceReset) looks up the array's device address,
 *    with that device current; make that first call before any stream capture.
 *  - All calls share the one array, and each call overwrites it: calls whose
 *    work can overlap on the GPU (other streams, other host threads) race and
 *    give wrong results.  Serialise them.
 *  - Errors are reported by the return status and ssd_last_error().
 */
ssd_status ssd_scan_fwd_noalloc(const void *x, const float *dt, const float *A,
                                const void *B, const void *C, const float *D,
                                const float *init_state, float *final_state, void *y,
                                ssd_dtype io_dtype, int batch, int seqlen, int nheads,
                                int headdim, int ngroups, int dstate, int chunk_size,
                                void *stream);

/*
 * Test hook for the failure path (not for production use).  The pages have no
 * counterpart: it exists so that a test can make the tensor-core kernel's
 * bounded waits run out without faulting anything.
 *
 * With withhold_first_load != 0, every tensor-core scan launched afterwards (on
 * any thread) has its load producer issue no load at all; every other role of
 * the kernel then waits for data that never comes, gives up after
 * wait_limit_ns nanoseconds (0: the default bound of 1 s), and the kernel
 * leaves at once.  Its outputs are then invalid and the next
 * ssd_get_device_status reports SSD_ERR_TIMEOUT.  withhold_first_load = 0
 * restores normal operation; wait_limit_ns then still bounds each wait (0: the
 * default).  Always returns SSD_OK.
 */
ssd_status ssd_debug_inject_stall(int withhold_first_load, unsigned long long wait_limit_ns);

/* Message for the last non-OK status returned on the calling host thread. */
const char *ssd_last_error(void);

/* Library version string. */
const char *ssd_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SSD_B200_H */
