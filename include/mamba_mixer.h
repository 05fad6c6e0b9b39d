/*
 * mamba_mixer.h -- C ABI of the B200 (sm_100a) Mamba mixer core.
 *
 * Two operations, both asynchronous on a CUDA stream the caller chooses:
 *
 *   mamba_mixer_fwd      selective-scan forward over a whole sequence (prefill)
 *   mamba_state_update   the one-token state update used in decode
 *
 * the same two with the RMSNorm of B_t and C_t fused in:
 *   mamba_mixer_fwd_normed, mamba_state_update_normed
 *
 * two more ways into the forward beyond the plain call:
 *   mamba_mixer_fwd_noalloc  no workspace argument (a fixed scratch array inside the library)
 *   mamba_mixer_fwd_host     activations in host memory, copies overlapped with the compute
 * the producers either side of the scan, on the tensor cores (tcgen05):
 *   mamba_proj_matmul           out = A W^T, a projection (bf16 operands, fp32 accumulation)
 *   mamba_mixer_fwd_projected   conv -> x_proj -> [dt_low | B | C] (+RMSNorm) -> dt_proj -> scan
 * the Mamba-2 and Mamba-3 forms of the scan:
 *   mamba_ssd_fwd            Mamba-2 prefill (scalar decay per head, chunked products on the tensor cores)
 *   mamba_ssd_state_update   Mamba-2 one-token step (decode), in place on the state
 *   mamba_m3_fwd             Mamba-3 prefill (trapezoid rule, complex state, 1/2/4 inputs per state)
 *   mamba_m3_state_update    Mamba-3 one-token step (decode), in place on the state
 *
 * and two status readers:
 *   mamba_check_status       did the last forward on this workspace complete? (per call)
 *   mamba_mixer_fault_status has any kernel on this device given up a bounded wait? (sticky)
 *
 * What they compute.  The Jamba hybrid SSM-Transformer lesson (section "SSM in
 * one page") gives the recurrence h_t = A h_{t-1} + B x_t, y_t = C h_t, notes
 * that y_t needs only h_{t-1} and x_t (constant memory, O(1) per token), and
 * that Mamba makes A, B and C data-dependent ("selective").  Its "Mamba-3"
 * section describes Mamba's convolution as an outer convolution on x_t ahead of
 * the recurrence; the reproduction blog's kernel-profile section names Delta as
 * the parameter that sets the state's decay.  The mixer-core problem statement
 * fixes the remaining form, which this library implements per channel d and
 * state index n:
 *
 *   u_t      = SiLU(conv_b[d] + sum_{k<W} conv_w[d,k] * x_{t-W+1+k})
 *   Delta_t  = softplus(dt_t + dt_bias[d])
 *   h_t[n]   = exp(Delta_t * A[d,n]) * h_{t-1}[n] + Delta_t * B_t[n] * u_t
 *   y_t      = (sum_n C_t[n] * h_t[n] + Dskip[d] * u_t) * SiLU(z_t)
 *
 * with x_{t<0} taken from the carried conv window, conv_w[d, W-1] applied to
 * the current token, one (B_t, C_t) group shared by all channels of a
 * sequence, and A passed directly (negative entries), not as log(-A).
 *
 * Conventions for every entry point:
 *   - Pointers are device (or managed) addresses, 16-byte aligned, dense
 *     row-major with the last dimension contiguous -- except the activations
 *     of mamba_mixer_fwd_host, which are host addresses.
 *   - "act" tensors hold MM_F32 floats or MM_BF16 bfloat16 values; parameters
 *     and the SSM state are always fp32.
 *   - Supported sizes: d_state == 16, d_conv == 4, d_inner a multiple of 8.
 *   - Validation happens on the host before anything is launched; a rejected
 *     call launches nothing and writes nothing.  A launch failure reported by
 *     the CUDA runtime returns MM_ERR_CUDA (the runtime's error is cleared).
 *   - The library allocates no device memory; the caller passes every buffer
 *     and scratch area.  Its only device state between calls is the device
 *     fault word and the fixed scratch array of mamba_mixer_fwd_noalloc.
 *     Calls only enqueue work: results are valid once the stream reaches them.
 *     A call starts after all earlier work in its stream and is complete
 *     before later work starts.  Within a time-chunked forward call, the
 *     second launch overlaps the first's tail (programmatic dependent launch).
 *   - Kernels never assert or trap.
 */
#ifndef MAMBA_MIXER_H
#define MAMBA_MIXER_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum mm_status {
    MM_OK = 0,
    MM_ERR_NULL = 1,        /* a required pointer is NULL                            */
    MM_ERR_SHAPE = 2,       /* a size is negative, zero where it must not be, or too big */
    MM_ERR_ALIGN = 3,       /* a pointer is not 16-byte aligned                      */
    MM_ERR_DTYPE = 4,       /* unknown activation dtype                              */
    MM_ERR_ALIAS = 5,       /* an output overlaps an input or another output         */
    MM_ERR_UNSUPPORTED = 6, /* d_state != 16, d_conv != 4, or d_inner % 8 != 0       */
    MM_ERR_CUDA = 7,        /* the CUDA runtime reported an error at launch          */
    MM_ERR_DEVICE = 8,      /* no usable sm_100 device is current                    */
    MM_ERR_WORKSPACE = 9,   /* workspace missing or smaller than the size this call needs */
    MM_ERR_SCRATCH_LIMIT = 10, /* mamba_mixer_fwd_noalloc: sizes need more than its built-in scratch */
    MM_ERR_TIMEOUT = 11,    /* mamba_check_status / mamba_mixer_fault_status: a kernel gave up a
                               bounded wait (its bulk copies, or a chunk summary never written) */
    MM_ERR_ARG = 12,        /* an argument value out of range (norm_eps not positive and finite) */
    MM_ERR_BOUNDS = 13      /* debug build only: a kernel skipped an access outside its buffer */
} mm_status;

typedef enum mm_dtype {
    MM_F32 = 0,   /* IEEE binary32 */
    MM_BF16 = 1   /* bfloat16      */
} mm_dtype;

/*
 * Selective-scan forward (prefill) for `batch` sequences of `seqlen` tokens.
 *
 * Inputs (act = activation dtype):
 *   xz             [batch, seqlen, 2*d_inner] act   x = xz[..., :d_inner], z = xz[..., d_inner:]
 *   conv_w         [d_inner, d_conv]          fp32  conv_w[d, d_conv-1] multiplies the current token
 *   conv_b         [d_inner]                  fp32  or NULL (= 0)
 *   dt             [batch, seqlen, d_inner]   act   step input before the bias
 *   dt_bias        [d_inner]                  fp32
 *   A              [d_inner, d_state]         fp32  (negative for a decaying state)
 *   Bm, Cm         [batch, seqlen, d_state]   act   shared by all channels of a sequence
 *   Dskip          [d_inner]                  fp32  or NULL (= 0)
 *   h0             [batch, d_inner, d_state]  fp32  initial state, or NULL (= 0)
 *   conv_state_in  [batch, d_inner, d_conv-1] act   the d_conv-1 raw x preceding token 0,
 *                                                   oldest first, or NULL (= 0)
 * Outputs:
 *   y              [batch, seqlen, d_inner]   act   rounded to nearest even for bf16
 *   h_last         [batch, d_inner, d_state]  fp32  state after the last token (h0 if seqlen == 0)
 *   conv_state_out [batch, d_inner, d_conv-1] act   the last d_conv-1 raw x, oldest first
 *                                                   (shifted in from conv_state_in when
 *                                                   seqlen < d_conv-1)
 * Passing (h_last, conv_state_out) of one call as (h0, conv_state_in) of the
 * next continues the sequence exactly; outputs may not overlap inputs, so
 * carry through two buffer sets (MM_ERR_ALIAS otherwise).
 *
 * workspace / workspace_bytes: device scratch of at least
 * mamba_mixer_workspace_size(...) bytes for the same sizes, 16-byte aligned
 * (MM_ERR_WORKSPACE when missing or smaller).  Its first 256 bytes hold the
 * call's status, which mamba_check_status reads.  When a sequence has too few
 * channels to fill the GPU, the forward splits it into time chunks: a first
 * launch stores each chunk's end state (run from a zero state) and total step
 * size there, and a second launch starts every chunk from the exact carried
 * state.  The caller owns the workspace; its contents need not be initialised
 * and are not needed after the call, except for the status; calls that share
 * one must not overlap in time.  It may not overlap any input or output
 * (MM_ERR_ALIAS).
 * stream: a cudaStream_t (NULL = the legacy default stream).
 * batch == 0 is a no-op.  seqlen == 0 writes h_last and conv_state_out only.
 * Length bound (MM_ERR_SHAPE, and a workspace size of 0, beyond it): one
 * sequence's xz rows, seqlen x 2 d_inner elements, must span less than 2^40
 * bytes (the bulk tensor copy's stride limit), and seqlen <= 2^30.  In bf16
 * at d_inner 8192 that is up to 2^25 - 1 tokens; run longer sequences as
 * several calls, carrying (h_last, conv_state_out).
 */
mm_status mamba_mixer_fwd(const void* xz, const float* conv_w, const float* conv_b,
                          const void* dt, const float* dt_bias, const float* A,
                          const void* Bm, const void* Cm, const float* Dskip,
                          const float* h0, const void* conv_state_in,
                          void* y, float* h_last, void* conv_state_out,
                          int64_t batch, int64_t seqlen, int64_t d_inner,
                          int64_t d_state, int64_t d_conv, mm_dtype act,
                          void* workspace, size_t workspace_bytes, void* stream);

/*
 * mamba_mixer_fwd with an RMSNorm of the selective parameters fused in.
 * The Jamba deep-dive report lists RMSNorm inside the Mamba layer among its
 * standard components, and its large-scale-stability section applies it to
 * the layer's internal activations; the pages do not say which.  This library
 * takes B_t and C_t, the activations that enter the recurrence, and
 * normalises each over its d_state entries before it is used:
 *
 *   B_t[n] <- B_t[n] * b_norm_w[n] / sqrt(mean_n B_t[n]^2 + norm_eps)
 *   C_t[n] <- C_t[n] * c_norm_w[n] / sqrt(mean_n C_t[n]^2 + norm_eps)
 *
 * b_norm_w, c_norm_w: [d_state] fp32 device weights, 16-byte aligned; NULL =
 * that input is used as it is (both NULL = mamba_mixer_fwd).  norm_eps must
 * be positive and finite when a weight is given (MM_ERR_ARG otherwise).  The
 * norm is computed in fp32 as each tile of B/C is staged; the inputs are not
 * modified.  Everything else is as mamba_mixer_fwd, including the workspace.
 */
mm_status mamba_mixer_fwd_normed(const void* xz, const float* conv_w, const float* conv_b,
                                 const void* dt, const float* dt_bias, const float* A,
                                 const void* Bm, const void* Cm, const float* Dskip,
                                 const float* h0, const void* conv_state_in,
                                 void* y, float* h_last, void* conv_state_out,
                                 int64_t batch, int64_t seqlen, int64_t d_inner,
                                 int64_t d_state, int64_t d_conv, mm_dtype act,
                                 const float* b_norm_w, const float* c_norm_w, float norm_eps,
                                 void* workspace, size_t workspace_bytes, void* stream);

/*
 * mamba_mixer_fwd without a workspace argument, for callers that cannot
 * allocate device memory.  No counterpart in the paper: it is a calling
 * convenience of this library, not part of the method.
 *
 * Who needs it: a host program that links only this C library and has no
 * device allocator of its own, and serving processes whose device memory is
 * planned in full before they start (weights, per-sequence SSM and conv
 * state) and that do not allocate on the request path.  Both can still pass
 * the inputs and outputs they already own; only the forward's scratch (the
 * carried chunk states of a time-split sequence) has nowhere to come from.
 *
 * The scratch is a fixed MAMBA_MIXER_NOALLOC_SCRATCH_BYTES array in the
 * library's device image: every GPU that loads the library holds it until
 * the process exits.  Sizes whose scratch would not fit (see
 * mamba_mixer_workspace_size) return MM_ERR_SCRATCH_LIMIT before anything is
 * launched; with the default launch plan every size fits.
 *
 * The first call in each CUDA context (a device's primary context, or one
 * the caller made current) looks up the array's device address in that
 * context and keeps it, keyed by the context's unique id, so a context made
 * after cudaDeviceReset gets a lookup of its own; make that first call before
 * any stream capture.  All calls on a device share the one array and nothing
 * in it is kept between calls (each call writes every scratch value it later
 * reads), but calls that overlap on the GPU -- on different streams, or from
 * different threads -- race on it and give wrong results: serialise them.
 * The status of the last call is read with mamba_check_status(NULL, stream).
 * Arguments, outputs and errors are otherwise those of mamba_mixer_fwd, and
 * every argument check of mamba_mixer_fwd comes before the scratch-size check.
 */
#define MAMBA_MIXER_NOALLOC_SCRATCH_BYTES (8u << 20)
mm_status mamba_mixer_fwd_noalloc(const void* xz, const float* conv_w, const float* conv_b,
                                  const void* dt, const float* dt_bias, const float* A,
                                  const void* Bm, const void* Cm, const float* Dskip,
                                  const float* h0, const void* conv_state_in,
                                  void* y, float* h_last, void* conv_state_out,
                                  int64_t batch, int64_t seqlen, int64_t d_inner,
                                  int64_t d_state, int64_t d_conv, mm_dtype act, void* stream);

/* Bytes of device workspace mamba_mixer_fwd needs for these sizes: at least
 * 256 (the status) for every valid size, 0 for invalid sizes.  A function of
 * its arguments, of the SM count of the current device (148, a B200's, when
 * no device is usable) and of the MAMBA_MIXER_CHUNKS tuning variable; none of
 * these may change between this call and the forward that uses the result.
 * MAMBA_MIXER_CHUNKS=K (a positive integer) forces K time chunks per sequence
 * instead of the launch plan's choice, capped at one chunk per 32-token tile;
 * the result is the same up to fp32 rounding.  It is a tuning and test knob.
 * Two more such knobs select slower code paths, for comparison only, and
 * leave the results the same up to fp32 rounding:
 * MAMBA_MIXER_GENERIC_WIDTH=1 runs the forward's any-width kernels where the
 * 256-channel CTA would run one compiled for that width, and
 * MAMBA_MIXER_GEMM_ROW_STORES=1 makes the projection GEMM write bf16 outputs
 * with per-thread row stores instead of staged bulk tensor stores. */
size_t mamba_mixer_workspace_size(int64_t batch, int64_t seqlen, int64_t d_inner,
                                  int64_t d_state, int64_t d_conv, mm_dtype act);

/*
 * The forward (mamba_mixer_fwd) on activations held in HOST memory, for a
 * caller whose sequence is not yet on the device.  The per-channel
 * parameters (conv_w, conv_b, dt_bias, A, Dskip) are DEVICE pointers, as in
 * mamba_mixer_fwd; everything else is a HOST pointer with the same shape and
 * meaning:
 *   in : xz, dt, Bm, Cm; h0 and conv_state_in (or NULL = zeros)
 *   out: y, h_last, conv_state_out
 * The sequence is cut into pieces along L.  Each piece's inputs are copied
 * to the device on `h2d_stream`, the forward runs on it on `stream` with the
 * state (h and the conv window) carried from the previous piece on the
 * device, and its y is copied back on `d2h_stream`; two staging slots let the
 * copies of one piece overlap the compute of its neighbours.  The result is
 * the forward of the whole sequence (it differs from one mamba_mixer_fwd
 * call only by where the time is split, i.e. by fp32 rounding).
 *
 * Host buffers should be page-locked (cudaHostAlloc / cudaHostRegister) for
 * the copies to overlap; pageable memory is correct but serialises.
 * `workspace` is DEVICE memory of at least
 * mamba_mixer_host_workspace_size(...) bytes, 16-byte aligned; it holds the
 * staging slots, the carried state and the forward's own scratch.  The
 * library allocates no memory.  The three streams may be the same stream
 * (no overlap) and may be NULL (the legacy default stream).
 * Asynchronous: when it returns, all work is queued and `stream` waits for
 * the last copy back, so synchronising `stream` makes every output valid.
 * Host buffers must stay alive and unmodified until then.  Errors as
 * mamba_mixer_fwd; sizes are validated before anything is queued.  The
 * length bound of mamba_mixer_fwd applies to each piece (about an eighth of
 * the sequence), not to the whole sequence.  Every piece records a failure
 * in the workspace's status under the call's one epoch:
 * mamba_check_status(workspace, stream) after the call reports whether any
 * piece gave up.  The device parameters may not overlap the workspace
 * (MM_ERR_ALIAS).
 */
mm_status mamba_mixer_fwd_host(const void* xz, const float* conv_w, const float* conv_b,
                               const void* dt, const float* dt_bias, const float* A,
                               const void* Bm, const void* Cm, const float* Dskip,
                               const float* h0, const void* conv_state_in,
                               void* y, float* h_last, void* conv_state_out,
                               int64_t batch, int64_t seqlen, int64_t d_inner,
                               int64_t d_state, int64_t d_conv, mm_dtype act,
                               void* workspace, size_t workspace_bytes,
                               void* stream, void* h2d_stream, void* d2h_stream);

/* Bytes of device workspace mamba_mixer_fwd_host needs for these sizes (0 for
 * invalid sizes). */
size_t mamba_mixer_host_workspace_size(int64_t batch, int64_t seqlen, int64_t d_inner,
                                       int64_t d_state, int64_t d_conv, mm_dtype act);

/*
 * One-token state update (decode) for n_layers independent stacked Mamba
 * layers at batch `batch`, updating the carried state in place.
 *
 *   x, z, dt       [n_layers, batch, d_inner]          act   the new token's inputs
 *   conv_w         [n_layers, d_inner, d_conv]         fp32
 *   conv_b         [n_layers, d_inner]                 fp32  or NULL (= 0)
 *   dt_bias        [n_layers, d_inner]                 fp32
 *   Dskip          [n_layers, d_inner]                 fp32  or NULL (= 0)
 *   A              [n_layers, d_inner, d_state]        fp32
 *   Bm, Cm         [n_layers, batch, d_state]          act
 *   ssm_state      [n_layers, batch, d_inner, d_state] fp32  in: h_{t-1}; out: h_t
 *   conv_state     [n_layers, batch, d_inner, d_conv-1] act  in: the d_conv-1 previous raw x,
 *                                                            oldest first; out: shifted by one
 *                                                            with x appended
 *   y              [n_layers, batch, d_inner]          act
 * This is the forward's step for one token (same arithmetic), so a prefill
 * followed by decode steps equals one longer prefill.  In-place by contract;
 * y may not overlap any other argument (MM_ERR_ALIAS).
 */
mm_status mamba_state_update(const void* x, const void* z, const void* dt,
                             const float* conv_w, const float* conv_b,
                             const float* dt_bias, const float* Dskip, const float* A,
                             const void* Bm, const void* Cm,
                             float* ssm_state, void* conv_state, void* y,
                             int64_t n_layers, int64_t batch, int64_t d_inner,
                             int64_t d_state, int64_t d_conv, mm_dtype act, void* stream);

/*
 * mamba_state_update with each (layer, batch) row's B and C normalised as in
 * mamba_mixer_fwd_normed, so decode continues a normed prefill exactly.
 * b_norm_w, c_norm_w: [n_layers, d_state] fp32 (one weight row per layer), or
 * NULL; norm_eps positive and finite when a weight is given (MM_ERR_ARG).
 */
mm_status mamba_state_update_normed(const void* x, const void* z, const void* dt,
                                    const float* conv_w, const float* conv_b,
                                    const float* dt_bias, const float* Dskip, const float* A,
                                    const void* Bm, const void* Cm,
                                    float* ssm_state, void* conv_state, void* y,
                                    int64_t n_layers, int64_t batch, int64_t d_inner,
                                    int64_t d_state, int64_t d_conv, mm_dtype act,
                                    const float* b_norm_w, const float* c_norm_w, float norm_eps,
                                    void* stream);

/*
 * Status of the last forward call that ran on `workspace` (the workspace of
 * mamba_mixer_fwd or mamba_mixer_fwd_host; NULL = the fixed scratch of
 * mamba_mixer_fwd_noalloc in the current context).  Waits for `stream` to
 * finish (the status is device memory written by the call's kernels), so it
 * cannot be recorded in a stream capture.  Returns MM_ERR_TIMEOUT if a kernel
 * of that call gave up a bounded wait -- on its own bulk copies, or because a
 * chunk summary it starts from was never written (the kernel then writes no
 * output, so y and the carried state of that call are not valid) -- MM_OK if
 * it completed, MM_ERR_CUDA if the status could not be read, MM_ERR_ALIGN for
 * a workspace that is not 16-byte aligned.  The status belongs to one call:
 * a later call on the same workspace replaces it.
 */
mm_status mamba_check_status(const void* workspace, void* stream);

/*
 * Device fault word of the library on the current device.  Every wait of a
 * kernel on its own bulk copies is bounded; a kernel that gives up (a copy
 * that never lands -- not expected on working hardware) sets this word,
 * skips its remaining work and exits instead of hanging.  Returns
 * MM_ERR_TIMEOUT if the word is set, MM_OK if not; clears it when `reset` is
 * non-zero.  Synchronises with the device (reads device memory).
 * Test hooks: the environment variable MAMBA_MIXER_WAIT_LIMIT sets the number
 * of wait attempts (0 makes the forward give up at once) and
 * MAMBA_MIXER_SUMMARY_WAIT_LIMIT the same for the summary pass of a
 * time-chunked forward alone (its chunk summaries then go missing);
 * MAMBA_MIXER_TEST_LAUNCH_FAIL=1 makes every forward launch ask for more
 * shared memory than a CTA may have, so the runtime rejects it on the host
 * and the call returns MM_ERR_CUDA (nothing reaches the GPU).
 */
mm_status mamba_mixer_fault_status(int reset);

/*
 * Projection product on the tensor cores: out[m, n] = sum_k A[m, k] W[n, k],
 * bf16 operands, fp32 accumulation (tcgen05.mma, operands staged by TMA,
 * accumulator in tensor memory).  The projections either side of the scan
 * are such products: the JAMBA hybrid-model blog names x_proj and dt_proj,
 * and the Jamba reproduction blog's LoRA section the low-rank Delta
 * projection.
 *   A    [M, K] bf16, row-major          W   [N, K] bf16 (one row per output feature)
 *   out  [M, N] fp32 (out_dtype MM_F32) or bf16 (MM_BF16, rounded to nearest even)
 * K and N must be multiples of 8 (16-byte rows; MM_ERR_UNSUPPORTED), M, N, K
 * below 2^31.  workspace: at least mamba_proj_matmul_workspace_size(M, N, K)
 * bytes (the call's status, read by mamba_check_status).  M == 0 is a no-op.
 * out may not overlap A, W or the workspace (MM_ERR_ALIAS).
 */
mm_status mamba_proj_matmul(const void* A, const void* W, void* out, int64_t M, int64_t N, int64_t K,
                            mm_dtype out_dtype, void* workspace, size_t workspace_bytes, void* stream);
size_t mamba_proj_matmul_workspace_size(int64_t M, int64_t N, int64_t K);

/*
 * The mixer with its producers, in the order the method runs them (bf16
 * activations only: the products run on the tensor cores):
 *
 *   u      = SiLU(conv_b + causal depthwise conv(x))                [B, L, D]
 *   x_dbl  = u W_x^T                        W_x [R + 2 N, D] bf16   [B, L, R + 2N]
 *   dt_low, B_t, C_t = x_dbl[:R], x_dbl[R:R+N], x_dbl[R+N:]
 *            each RMS-normalised over its own width when its weight is given
 *            (dt_norm_w [R], b_norm_w / c_norm_w [N] fp32; NULL = not normalised)
 *   dt     = dt_low W_dt^T                  W_dt [D, R] bf16        [B, L, D]
 *   y, h_last, conv_state_out = the selective scan of mamba_mixer_fwd on
 *            (x, z, dt, B, C) with conv_w, conv_b, dt_bias, A, Dskip, h0,
 *            conv_state_in as there.
 *
 * R = dt_rank, a multiple of 32 up to 1024; d_state == 16; d_conv == 4;
 * d_inner a multiple of 64.  The pages name the projections (JAMBA hybrid-model
 * blog: x_proj, dt_proj; reproduction blog: the low-rank Delta projection)
 * but give no rank; the standard choice, ceil(hidden / 16) = 256 at hidden
 * 4096, is what the tests and the benchmark use.  workspace: at least
 * mamba_mixer_projected_workspace_size(...) bytes; it holds the scan's own
 * workspace (with the call's status, first) and the intermediates u, x_proj's
 * split-K partials, dt_low, B, C and dt.  The weights and every caller buffer
 * may not overlap it (MM_ERR_ALIAS).  Errors otherwise as mamba_mixer_fwd.
 */
mm_status mamba_mixer_fwd_projected(const void* xz, const float* conv_w, const float* conv_b,
                                    const void* W_x, const void* W_dt, const float* dt_bias, const float* A,
                                    const float* Dskip, const float* h0, const void* conv_state_in,
                                    const float* dt_norm_w, const float* b_norm_w, const float* c_norm_w,
                                    float norm_eps, void* y, float* h_last, void* conv_state_out,
                                    int64_t batch, int64_t seqlen, int64_t d_inner, int64_t d_state,
                                    int64_t dt_rank, int64_t d_conv, mm_dtype act,
                                    void* workspace, size_t workspace_bytes, void* stream);
size_t mamba_mixer_projected_workspace_size(int64_t batch, int64_t seqlen, int64_t d_inner, int64_t d_state,
                                            int64_t dt_rank, int64_t d_conv, mm_dtype act);
/* Byte offsets, within that workspace, of the intermediates a call leaves
 * there (valid once its stream has reached the end of the call): offsets[0]
 * u [B, L, D], [1] dt_low [B, L, R], [2] B_t [B, L, N], [3] C_t [B, L, N],
 * [4] dt [B, L, D], all bf16 row-major.  For inspection and tests; the
 * forward itself does not need them afterwards. */
mm_status mamba_mixer_projected_layout(int64_t batch, int64_t seqlen, int64_t d_inner, int64_t d_state,
                                       int64_t dt_rank, int64_t d_conv, size_t offsets[5]);

/*
 * The Mamba-2 form of the selective scan, prefill (bf16 activations, fp32
 * state; the products run on the tensor cores).  The Jamba lesson's "SSM in
 * one page" section: Mamba-2 simplified the state matrix -- to a scalar times
 * the identity per head -- and its "Mamba-3" section: Mamba-2 discretises
 * with Euler's rule.  For head h of H (P = headdim channels, c = h P + p),
 * group g = h / (H / groups) and every token t:
 *
 *   Delta_t  = softplus(dt_t[h] + dt_bias[h])
 *   s_t[p,n] = exp(Delta_t A[h]) s_{t-1}[p,n] + Delta_t B_t[g,n] x_t[c]
 *   y_t[c]   = (sum_n C_t[g,n] s_t[p,n] + D[h] x_t[c]) * SiLU(z_t[c])   (no gate if z is NULL)
 *
 * computed chunk by chunk (128 tokens) as dense products -- the same sums,
 * regrouped.  x is the layer's input after its convolution.
 *
 *   x, z           [batch, seqlen, heads*headdim]   bf16  (z may be NULL)
 *   dt             [batch, seqlen, heads]           bf16  before dt_bias and softplus
 *   dt_bias        [heads]                          fp32  or NULL (= 0)
 *   A              [heads]                          fp32  negative
 *   Bm, Cm         [batch, seqlen, groups, d_state] bf16
 *   Dskip          [heads]                          fp32  or NULL (= 0)
 *   h0             [batch, heads, headdim, d_state] fp32  or NULL (= 0)
 *   y              [batch, seqlen, heads*headdim]   bf16  output
 *   h_last         [batch, heads, headdim, d_state] fp32  output: the state after the last token
 *
 * Supported: headdim == 64, d_state == 128 (MM_ERR_UNSUPPORTED otherwise);
 * heads a multiple of groups, both positive (MM_ERR_SHAPE).  Every pointer
 * 16-byte aligned (MM_ERR_ALIGN); y and h_last may not overlap an input or
 * each other (MM_ERR_ALIAS).  workspace: at least
 * mamba_ssd_workspace_size(...) bytes, 16-byte aligned, overlapping no other
 * argument; its first 256 bytes hold the call's status for
 * mamba_check_status.  seqlen == 0 writes h_last = h0 (or zeros).  Runs on
 * `stream`; the library allocates nothing.  Errors otherwise as
 * mamba_mixer_fwd.
 */
mm_status mamba_ssd_fwd(const void* x, const void* z, const void* dt, const float* dt_bias, const float* A,
                        const void* Bm, const void* Cm, const float* Dskip, const float* h0,
                        void* y, float* h_last,
                        int64_t batch, int64_t seqlen, int64_t heads, int64_t headdim, int64_t d_state,
                        int64_t groups, void* workspace, size_t workspace_bytes, void* stream);
/* Workspace bytes of mamba_ssd_fwd for these sizes (0 if they are not
 * supported): the status header, the fp32 state each chunk adds from zero,
 * the state entering each chunk (as two bf16 parts) and each chunk's total
 * decay. */
size_t mamba_ssd_workspace_size(int64_t batch, int64_t seqlen, int64_t heads, int64_t headdim, int64_t d_state,
                                int64_t groups);

/*
 * One token of the Mamba-2 form (decode), in place on the state: the
 * recurrence of mamba_ssd_fwd above for a single token, with the state the
 * previous call (prefill or decode) left as h_last:
 *
 *   Delta    = softplus(dt[h] + dt_bias[h])
 *   s[p,n]   = exp(Delta A[h]) s[p,n] + Delta B[g,n] x[c]
 *   y[c]     = (sum_n C[g,n] s[p,n] + D[h] x[c]) * SiLU(z[c])   (no gate if z is NULL)
 *
 *   x, z           [batch, heads*headdim]            bf16  (z may be NULL)
 *   dt             [batch, heads]                    bf16  before dt_bias and softplus
 *   dt_bias        [heads]                           fp32  or NULL (= 0)
 *   A              [heads]                           fp32  negative
 *   Bm, Cm         [batch, groups, d_state]          bf16
 *   Dskip          [heads]                           fp32  or NULL (= 0)
 *   state          [batch, heads, headdim, d_state]  fp32  read and overwritten
 *   y              [batch, heads*headdim]            bf16  output
 *
 * The same results as mamba_ssd_fwd with seqlen 1, h0 = state and h_last =
 * state, up to rounding order.  Supported: headdim == 64, d_state == 128
 * (MM_ERR_UNSUPPORTED otherwise); heads a multiple of groups, both positive,
 * batch <= 65535 (MM_ERR_SHAPE).  Every pointer 16-byte aligned
 * (MM_ERR_ALIGN); state and y may not overlap an input or each other
 * (MM_ERR_ALIAS).  No workspace and no wait: one launch of one CTA per (head,
 * sequence) on `stream`.  batch == 0 is a no-op.  Errors otherwise as
 * mamba_state_update.
 */
mm_status mamba_ssd_state_update(const void* x, const void* z, const void* dt, const float* dt_bias,
                                 const float* A, const void* Bm, const void* Cm, const float* Dskip,
                                 float* state, void* y,
                                 int64_t batch, int64_t heads, int64_t headdim, int64_t d_state, int64_t groups,
                                 void* stream);

/*
 * The Mamba-3 form of the selective scan, prefill (bf16 activations, fp32
 * state and arithmetic).  The Jamba lesson's "Mamba-3" section names three
 * changes over Mamba-2: an exponential-trapezoidal discretisation, whose
 * conv-like rule acts on the state input inside the recurrence; a complex
 * state, equivalent to a data-dependent rotary embedding; and multi-input
 * multi-output (MIMO) projections.  The section gives no formula; the
 * readings: per head h, group g = h / (H / groups), channel c = h P + p and
 * state pair k (d_state entries 2k, 2k+1 = real and imaginary part),
 *
 *   Delta_t  = softplus(dt_t[h] + dt_bias[h]);   lambda_t = trap_t[h] (1/2 when trap is NULL)
 *   a_t[k]   = exp(Delta_t A[h]) (cos(Delta_t theta[h,k]) + i sin(Delta_t theta[h,k]))
 *   u_t[k]   = sum_r (B_t[r,g,2k] + i B_t[r,g,2k+1]) x_t[r,c]     (rank inputs r share the state)
 *   s_t[k]   = a_t[k] (s_{t-1}[k] + (1 - lambda_t) Delta_t u_{t-1}[k]) + lambda_t Delta_t u_t[k]
 *   y_t[r,c] = (sum_k Re(conj(C_t[r,g,k]) s_t[k]) + D[h] x_t[r,c]) * SiLU(z_t[r,c])   (no gate if z is NULL)
 *
 * lambda = 1 gives Euler's rule (the Mamba-2 step), 1/2 the trapezoid.
 * u_{-1} is the input of the token before the call, from x_prev and B_prev
 * (zero when both are NULL): a sequence split into calls continues exactly
 * when each call passes the previous call's h_last as h0 and its last token's
 * x and B rows as x_prev and B_prev.
 *
 *   x, z           [batch, seqlen, rank, heads*headdim]          bf16  (z may be NULL)
 *   dt, trap       [batch, seqlen, heads]                        bf16  (trap may be NULL)
 *   dt_bias        [heads] fp32 or NULL;  A [heads] fp32 (negative)
 *   theta          [heads, d_state/2]                            fp32  rotation frequencies
 *   Bm, Cm         [batch, seqlen, rank, groups, d_state]        bf16
 *   Dskip          [heads] fp32 or NULL
 *   h0             [batch, heads, headdim, d_state]              fp32  or NULL (= 0)
 *   x_prev         [batch, rank, heads*headdim]                  bf16  or NULL (together with B_prev)
 *   B_prev         [batch, rank, groups, d_state]                bf16  or NULL
 *   y              [batch, seqlen, rank, heads*headdim]          bf16  output
 *   h_last         [batch, heads, headdim, d_state]              fp32  output
 *
 * Supported: headdim == 64, d_state == 16, rank 1, 2 or 4, an even number
 * of heads (MM_ERR_UNSUPPORTED otherwise); heads a multiple of groups
 * (MM_ERR_SHAPE).  x_prev and B_prev are given together or not at all
 * (MM_ERR_NULL).  Every pointer 16-byte aligned (MM_ERR_ALIGN); y and h_last
 * may not overlap an input or each other (MM_ERR_ALIAS).  workspace: at least
 * mamba_m3_workspace_size(...) bytes (the chunk end states of a sequence cut
 * in time), 16-byte aligned, overlapping no other argument; its first 256
 * bytes hold the call's status for mamba_check_status.  seqlen == 0 writes
 * h_last = h0 (or zeros).  Runs on `stream`; the library allocates nothing.
 */
mm_status mamba_m3_fwd(const void* x, const void* z, const void* dt, const void* trap, const float* dt_bias,
                       const float* A, const float* theta, const void* Bm, const void* Cm, const float* Dskip,
                       const float* h0, const void* x_prev, const void* B_prev, void* y, float* h_last,
                       int64_t batch, int64_t seqlen, int64_t rank, int64_t heads, int64_t headdim,
                       int64_t d_state, int64_t groups, void* workspace, size_t workspace_bytes, void* stream);
/* Workspace bytes of mamba_m3_fwd for these sizes (0 if not supported). */
size_t mamba_m3_workspace_size(int64_t batch, int64_t seqlen, int64_t rank, int64_t heads, int64_t headdim,
                               int64_t d_state, int64_t groups);

/*
 * One token of the Mamba-3 form (decode), in place on the state: the
 * recurrence of mamba_m3_fwd above for a single token t, with the state the
 * previous call left as h_last and the previous token's input:
 *
 *   s[k]   = a_t[k] (s[k] + (1 - lambda_t) Delta_t u_prev[k]) + lambda_t Delta_t u_t[k]
 *   y[r,c] = (sum_k Re(conj(C_t[r,g,k]) s[k]) + D[h] x_t[r,c]) * SiLU(z_t[r,c])
 *
 * with a_t, u_t, Delta_t and lambda_t as defined there and u_prev the input
 * of the token before (x_prev, B_prev; zero when both are NULL).  A decode
 * loop passes, at each step, the previous step's x and B rows as x_prev and
 * B_prev.
 *
 *   x, z           [batch, rank, heads*headdim]     bf16  (z may be NULL)
 *   dt, trap       [batch, heads]                   bf16  (trap may be NULL: 1/2)
 *   dt_bias        [heads] fp32 or NULL;  A [heads] fp32 (negative)
 *   theta          [heads, d_state/2]               fp32
 *   Bm, Cm         [batch, rank, groups, d_state]   bf16
 *   Dskip          [heads] fp32 or NULL
 *   state          [batch, heads, headdim, d_state] fp32  read and overwritten
 *   x_prev, B_prev [batch, rank, heads*headdim], [batch, rank, groups, d_state]  bf16  or both NULL
 *   y              [batch, rank, heads*headdim]     bf16  output
 *
 * The same results as mamba_m3_fwd with seqlen 1, h0 = state and h_last =
 * state, up to rounding order.  Supported sizes and errors as mamba_m3_fwd
 * (no workspace, no wait); state and y may not overlap an input or each other
 * (MM_ERR_ALIAS).  One launch on `stream`; batch == 0 is a no-op.
 */
mm_status mamba_m3_state_update(const void* x, const void* z, const void* dt, const void* trap, const float* dt_bias,
                                const float* A, const float* theta, const void* Bm, const void* Cm,
                                const float* Dskip, float* state, const void* x_prev, const void* B_prev, void* y,
                                int64_t batch, int64_t rank, int64_t heads, int64_t headdim, int64_t d_state,
                                int64_t groups, void* stream);

/* A static, human-readable name for a status code. */
const char* mamba_status_string(mm_status status);

/* ABI version of this header (incremented on any signature change). */
int mamba_mixer_abi_version(void);

#define MAMBA_MIXER_ABI_VERSION 8

#ifdef __cplusplus
}
#endif

#endif /* MAMBA_MIXER_H */
