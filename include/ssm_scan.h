/*
 * ssm_scan.h: C ABI of the B200 (sm_100a) selective-scan library
 * (libssmscan.so): the fused forward pass, the same with the causal
 * convolution fused in front, the batched decode step, the backward pass, and
 * a no-allocation forward for callers that cannot allocate.
 *
 * The operation is the selective state-space recurrence (Mamba-1 / S6) as
 * the page "Mamba: Linear-Time Sequence Modeling with Selective State Spaces"
 * (www.abhik.ai/papers/mamba) states it, section "Original paper, equations
 * and runnable CPU code":
 *   row "1. Produce coefficients from the locally mixed input":
 *       delta = softplus(delta_raw + delta_bias),   A = -exp(A_log)
 *   row "2. Retain, write and read each channel's state":
 *       a[t,e,n] = exp(delta[t,e] * A[e,n])
 *       h[t,e,n] = a[t,e,n] * h[t-1,e,n] + delta[t,e] * B[t,n] * x[t,e]
 *       y[t,e]   = sum_n C[t,n] * h[t,e,n] + D[e] * x[t,e]
 *     (read after the update; an optional incoming state continues an
 *     earlier prefix; the write is delta*B*x, not the exact zero-order-hold
 *     integral)
 *   row "5. Put the selective operator inside the complete mixer":
 *       y <- y * SiLU(z)      (after D*x is included)
 * per batch b, expanded channel e, state coordinate n. B and C are shared by
 * every channel ("In the pinned mamba_simple block, B and C have shape
 * [b, T, N] and are shared across the expanded channels", section "The input
 * changes the coefficients, while A stays learned"). The final state h_L is
 * returned; the states of the other steps are never written to memory (the
 * fused, on-chip evaluation the same page describes in "Compose the updates
 * instead of waiting for every state").
 *
 * Conventions for every call:
 *   - Pointers named x, delta, z, B, C, y point to DEVICE memory of the
 *     activation dtype (SSM_F32: float, SSM_BF16: bfloat16). A_log, D,
 *     delta_bias, h0, h_last point to DEVICE memory of float32.
 *   - All tensors are dense, row-major (C order), with these shapes:
 *         x, delta, z, y : [batch, seqlen, dim]       dim = E, contiguous
 *         B, C           : [batch, seqlen, dstate]    dstate = N
 *         A_log          : [dim, dstate]
 *         D, delta_bias  : [dim]
 *         h0, h_last     : [batch, dim, dstate]       (float32)
 *   - Ownership: the caller owns every buffer. The library keeps no pointer
 *     after a call returns. Work is ASYNCHRONOUS on `stream` (a cudaStream_t;
 *     NULL means the legacy default stream): buffers must stay valid and
 *     unmodified until the stream has passed the call.
 *   - Errors: every call returns an int status (SSM_OK or a negative code)
 *     and never aborts or throws. Argument errors are found on the host
 *     before anything is launched. A failed launch returns SSM_ERR_CUDA.
 *   - Thread safety: a handle may be used by one host thread at a time, and
 *     carries at most one in-flight call on any stream at a time when it
 *     needs workspace (long sequences with few channels; shapes whose
 *     channel tiles do not divide evenly over the SMs, which run on
 *     persistent blocks handing chunks over; the backward pass's
 *     checkpoints). Different handles are independent.
 *   - CUDA graphs: ssm_scan_step, ssm_scan_fwd and ssm_scan_fwd_conv only
 *     enqueue memsets and kernels once their workspace exists, so their
 *     calls can be captured into a graph and replayed, split sequences
 *     included (each call clears its own publication flags on the stream),
 *     and so can the persistent-block scan (it clears its ticket and
 *     hand-over flags the same way).
 *     Calls that grow a workspace do so on their first use with that shape:
 *     make that call before capturing.
 */
#ifndef SSM_SCAN_H
#define SSM_SCAN_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define SSM_API __attribute__((visibility("default")))
#else
#define SSM_API
#endif

struct CUstream_st; /* cudaStream_t is `struct CUstream_st *` */

typedef struct ssm_scan_s *ssm_scan_t;

typedef struct {
    int64_t batch;  /* b  > 0 */
    int64_t seqlen; /* L  > 0 */
    int64_t dim;    /* E  > 0, expanded channels */
    int64_t dstate; /* N  in 1..64 */
} ssm_scan_dims;

/* Activation dtype (x, delta, z, B, C and y). */
enum { SSM_F32 = 0, SSM_BF16 = 1 };

/*
 * flags:
 *   SSM_DELTA_SOFTPLUS: delta = softplus(delta + delta_bias), else delta + bias.
 *   SSM_WRITE_ZOH: the write is the exact zero-order-hold input map
 *     Bbar = (delta A)^-1 (exp(delta A) - 1) delta B, i.e. per state
 *     expm1(delta A[e,n]) / A[e,n] * B[t,n] * x[t,e] (delta * B * x when
 *     A = 0), instead of the default delta * B * x ("Mamba: Linear-Time
 *     Sequence Modeling with Selective State Spaces", nadeemcite summary,
 *     section "Core Idea"; the abhik page, "There is a discretization detail
 *     worth keeping explicit").
 */
enum { SSM_DELTA_SOFTPLUS = 1u << 0, SSM_WRITE_ZOH = 1u << 1 };

/*
 * Training pair (the states are still recomputed on the way back, as section
 * "Compose the updates instead of waiting for every state" of the abhik page
 * describes; only the sparse checkpoints the backward starts from are kept):
 *   SSM_SAVE_CHECKPOINTS (ssm_scan_fwd only): the forward also writes the
 *     state before every 8th step into the handle's checkpoint workspace,
 *     which it grows on first use (b * ceil(L / 8) * dim * dstate floats;
 *     SSM_ERR_NOMEM if it cannot: make that call before capturing a graph).
 *     The call then runs unsplit (one block per sequence and channel tile),
 *     needs the chunked variant's shapes (dstate 4, 8 or 16, 8 or 16 for
 *     bfloat16; dim * element size a multiple of 16 bytes; 16-byte aligned
 *     x, delta, z, B, C: SSM_ERR_UNSUPPORTED otherwise) and does not combine
 *     with ssm_scan_fwd_conv (SSM_ERR_INVALID). The handle remembers the
 *     shape, dtype and flags the checkpoints belong to.
 *   SSM_REUSE_CHECKPOINTS (ssm_scan_bwd only): skip the backward's own
 *     checkpointing forward and start from the checkpoints the last
 *     SSM_SAVE_CHECKPOINTS forward on this handle wrote. Its shape, dtype and
 *     SSM_DELTA_SOFTPLUS / SSM_WRITE_ZOH flags must match this call's
 *     (SSM_ERR_INVALID otherwise, also when there are none, or when a
 *     backward without this flag has overwritten them since); its inputs
 *     (x, delta, A_log, B, h0, delta_bias) must be this call's, which the
 *     library cannot check. The gradients are the ones the same call without
 *     the flag returns.
 */
enum { SSM_SAVE_CHECKPOINTS = 1u << 2, SSM_REUSE_CHECKPOINTS = 1u << 3 };

/*
 * SSM_DETERMINISTIC (ssm_scan_bwd only): the gradients summed over channels
 * or steps (dB, dC, dA_log, dD, ddelta_bias) are bitwise the same on every
 * run. Without it they are added with float32 atomics, whose order varies
 * (a relative run-to-run spread far below the float32 rounding of the
 * oracle comparison). With it, each thread block writes its share to a
 * partial array the handle grows (2 * ceil(dim / G) * batch * seqlen *
 * dstate + batch * dim * (dstate + 2) floats, G = 16, 32 or 64 channels for
 * dstate 16, 8 or 4; SSM_ERR_NOMEM if it cannot) and fixed-order sums of
 * those arrays follow on `stream`. The per-element gradients are
 * deterministic either way.
 */
enum { SSM_DETERMINISTIC = 1u << 4 };

/* Status codes. */
enum {
    SSM_OK = 0,
    SSM_ERR_INVALID = -1,     /* NULL required pointer, bad size or flag  */
    SSM_ERR_UNSUPPORTED = -2, /* dtype or dstate outside what is built   */
    SSM_ERR_ALIGN = -3,       /* pointer misaligned for its element type */
    SSM_ERR_ARCH = -4,        /* device is not compute capability 10.0   */
    SSM_ERR_CUDA = -5,        /* a CUDA runtime call failed              */
    SSM_ERR_TIMEOUT = -6,     /* a bounded inter-block wait gave up      */
    SSM_ERR_NOMEM = -7        /* workspace or handle allocation failed   */
};

/* Kernel variant selection (ssm_scan_set_variant). AUTO picks by shape. */
enum {
    SSM_VARIANT_AUTO = 0,
    SSM_VARIANT_SEQUENTIAL = 1, /* one thread per (b, e), any shape        */
    SSM_VARIANT_CHUNKED = 2     /* staged tiles, warp-level scan, fused    */
};

/*
 * ssm_scan_create: make a handle bound to CUDA device `device`.
 * Checks that the device has compute capability 10.0 (B200, sm_100a) and
 * caches its multiprocessor count. Allocates no device memory.
 * Returns SSM_OK and writes *out; SSM_ERR_INVALID if out is NULL or device is
 * out of range; SSM_ERR_ARCH on another architecture; SSM_ERR_CUDA if the
 * runtime cannot be queried; SSM_ERR_NOMEM if the host allocation fails.
 */
SSM_API int ssm_scan_create(ssm_scan_t *out, int device);

/*
 * ssm_scan_destroy: release the handle and any workspace it grew. Waits for
 * nothing: the caller must ensure no call using the handle is still in
 * flight. NULL is accepted and ignored (SSM_OK).
 */
SSM_API int ssm_scan_destroy(ssm_scan_t h);

/*
 * ssm_scan_fwd: the fused selective-scan forward pass (see the file header
 * for the recurrence and layouts).
 *   x, delta, B, C, A_log, y : required (non-NULL).
 *   D          : NULL means no direct path (D = 0).
 *   z          : NULL means no gate.
 *   delta_bias : NULL means a zero bias.
 *   h0         : NULL means a zero incoming state.
 *   h_last     : NULL means the final state is not written.
 *   flags      : SSM_DELTA_SOFTPLUS and/or SSM_WRITE_ZOH; other bits are
 *                SSM_ERR_INVALID.
 *   dtype      : SSM_F32 or SSM_BF16 (activations and y).
 * y must not overlap any input. Pointers must be aligned to their element
 * size (SSM_ERR_ALIGN otherwise). Launches on `stream` and returns without
 * waiting. The handle's device must be current on the calling thread.
 */
SSM_API int ssm_scan_fwd(ssm_scan_t h, const void *x, const void *delta,
                 const float *A_log, const void *B, const void *C,
                 const float *D, const void *z, const float *delta_bias,
                 uint32_t flags, const float *h0, void *y, float *h_last,
                 ssm_scan_dims dims, int dtype, struct CUstream_st *stream);

/*
 * ssm_scan_fwd_conv: ssm_scan_fwd with the causal depthwise convolution and
 * SiLU that produce x fused in front ("Mamba: Linear-Time Sequence Modeling
 * with Selective State Spaces", www.abhik.ai/papers/mamba, section "Original
 * paper, equations and runnable CPU code", row "4. Add causal local context
 * before selecting coefficients", and row "5. Put the selective operator
 * inside the complete mixer"):
 *     x[b, t, e] = SiLU(conv_bias[e] + sum_{k<K} conv_weight[e, k] *
 *                       v[b, t - K + 1 + k, e]),  v = 0 before t = 0,
 * then the scan of ssm_scan_fwd on x (D x and the gate use this x). x is
 * formed in registers; it is never written to memory.
 *   v           : [batch, seqlen, dim] activation dtype, required.
 *   conv_weight : [dim, conv_width] float32, required (SSM_ERR_INVALID).
 *   conv_bias   : [dim] float32, NULL means zero.
 *   conv_width  : K, 1..SSM_SCAN_CONV_MAX_WIDTH (else SSM_ERR_INVALID).
 * Everything else, and every error, as for ssm_scan_fwd.
 */
#define SSM_SCAN_CONV_MAX_WIDTH 4
SSM_API int ssm_scan_fwd_conv(ssm_scan_t h, const void *v,
                              const float *conv_weight, const float *conv_bias,
                              int conv_width, const void *delta,
                              const float *A_log, const void *B, const void *C,
                              const float *D, const void *z,
                              const float *delta_bias, uint32_t flags,
                              const float *h0, void *y, float *h_last,
                              ssm_scan_dims dims, int dtype,
                              struct CUstream_st *stream);

/*
 * ssm_scan_bwd: the backward pass of ssm_scan_fwd: the gradients of
 *     loss = sum(dy * y) + sum(dh_last * h_last)
 * with respect to every input, by reverse-mode differentiation of the
 * recurrence ("Mamba: Linear-Time Sequence Modeling with Selective State
 * Spaces", www.abhik.ai/papers/mamba, section "Original paper, equations and
 * runnable CPU code", rows 1, 2 and 5; the states are recomputed on the way
 * back rather than stored, as section "Compose the updates instead of
 * waiting for every state" describes). Two launches on `stream`: the forward
 * with a state checkpoint every 8 steps into a workspace the handle grows
 * (b * ceil(L / 8) * dim * dstate floats; SSM_ERR_NOMEM if it cannot), then
 * a reverse sweep from those checkpoints. With SSM_REUSE_CHECKPOINTS (see
 * above), only the reverse sweep, from the training forward's checkpoints.
 *   inputs     : as ssm_scan_fwd (x, delta, A_log, B, C, D, z, delta_bias,
 *                flags, h0); dy [batch, seqlen, dim] activation dtype,
 *                required; dh_last [batch, dim, dstate] float32 or NULL (0).
 *   dx, ddelta : [batch, seqlen, dim] activation dtype, required; ddelta is
 *                the gradient of the raw step (before bias and softplus).
 *   dz         : [batch, seqlen, dim] activation dtype; required with z.
 *   dB, dC     : [batch, seqlen, dstate] float32, required (sums over the
 *                channels).
 *   dA_log     : [dim, dstate] float32, required (sum over the batch).
 *   dD, ddelta_bias : [dim] float32; required with D / delta_bias.
 *   dh0        : [batch, dim, dstate] float32 or NULL (not written).
 * The summed outputs are cleared by the call. dstate must be 4, 8 or 16
 * (8 or 16 for bfloat16), dim * element size a multiple of 16 bytes, and x,
 * delta, z, dy, B, C, A_log, h0, dh_last, dB, dC, dh0 16-byte aligned
 * (SSM_ERR_UNSUPPORTED / SSM_ERR_ALIGN otherwise). Outputs must not overlap
 * inputs. Other errors as for ssm_scan_fwd.
 */
SSM_API int ssm_scan_bwd(ssm_scan_t h, const void *x, const void *delta,
                         const float *A_log, const void *B, const void *C,
                         const float *D, const void *z,
                         const float *delta_bias, uint32_t flags,
                         const float *h0, const void *dy,
                         const float *dh_last, void *dx, void *ddelta,
                         float *dA_log, float *dB, float *dC, float *dD,
                         void *dz, float *ddelta_bias, float *dh0,
                         ssm_scan_dims dims, int dtype,
                         struct CUstream_st *stream);

/*
 * ssm_scan_set_variant: force a kernel variant for later calls on this
 * handle (SSM_VARIANT_*), or SSM_VARIANT_AUTO to choose by shape.
 * `segments` > 1 asks the chunked variant to split every sequence into that
 * many independent pieces joined by the inter-block carry (0 = automatic,
 * 1 = never split). A forced variant that cannot run a given shape makes
 * ssm_scan_fwd return SSM_ERR_UNSUPPORTED. Returns SSM_ERR_INVALID for an
 * unknown variant or a negative segment count.
 */
SSM_API int ssm_scan_set_variant(ssm_scan_t h, int variant, int segments);

/*
 * ssm_scan_set_time_blocks: for the chunked variant, how many lanes of a warp
 * share one channel's time axis (1, 2, 4 or 8: each takes a block of
 * consecutive steps, and the blocks are joined by a warp-shuffle scan of
 * their affine maps), or 0 to choose by shape. Returns SSM_ERR_INVALID for
 * other values. A value a shape cannot use is reported by ssm_scan_fwd as
 * SSM_ERR_UNSUPPORTED.
 */
SSM_API int ssm_scan_set_time_blocks(ssm_scan_t h, int time_blocks);

/*
 * ssm_scan_set_debug: testing hook. `flags` bit 0 makes the first piece of
 * every split sequence skip its publication, so that the bounded wait of its
 * successor runs out: that call then reports SSM_ERR_TIMEOUT through
 * ssm_scan_sync_status and its outputs are invalid. Bit 1 makes
 * ssm_scan_step use its per-thread-load kernel where it would use the
 * bulk-copy one. `spin_limit` bounds every wait between thread blocks and
 * every wait for a bulk copy (in polls of roughly 1 us each; 0 restores the
 * default of 10^6 polls, about one second). Returns SSM_ERR_INVALID for a
 * NULL handle.
 */
SSM_API int ssm_scan_set_debug(ssm_scan_t h, unsigned flags,
                               unsigned spin_limit);

/*
 * ssm_scan_last_variant: the variant (SSM_VARIANT_*) and segment count the
 * most recent successful ssm_scan_fwd on this handle launched. Either output
 * pointer may be NULL.
 */
SSM_API int ssm_scan_last_variant(ssm_scan_t h, int *variant, int *segments);

/*
 * ssm_scan_sync_status: wait for `stream`, then report device-side status of
 * the calls made on this handle since the previous sync: SSM_ERR_TIMEOUT if a
 * bounded wait between thread blocks gave up (its results are then invalid),
 * SSM_ERR_CUDA on an asynchronous CUDA error, else SSM_OK. Resets the status.
 */
SSM_API int ssm_scan_sync_status(ssm_scan_t h, struct CUstream_st *stream);

/*
 * ssm_scan_step: one decode step for `dims.batch` sequences at once, updating
 * the convolution buffer and the state in place ("Mamba: Linear-Time Sequence
 * Modeling with Selective State Spaces", www.abhik.ai/papers/mamba, section
 * "Original paper, equations and runnable CPU code", row "6. Carry both
 * buffers to the next token", with the causal convolution of row "4. Add
 * causal local context before selecting coefficients"):
 *     conv_state <- shift left by one sample, append x_new
 *     x     = SiLU(sum_k conv_state[k] * conv_weight[e, k] + conv_bias[e])
 *     delta = softplus(delta_raw + delta_bias)   (SSM_DELTA_SOFTPLUS)
 *     state <- exp(delta A) * state + delta * B * x  (or the SSM_WRITE_ZOH write)
 *     y     = (sum_n C[n] * state[n] + D[e] * x) * SiLU(z)
 * Layouts (dense, row-major): x_new, delta, z, y: [batch, dim] activation
 * dtype; conv_state: [batch, dim, conv_width] activation dtype (oldest sample
 * first); conv_weight: [dim, conv_width] float32; conv_bias, D, delta_bias:
 * [dim] float32; A_log: [dim, dstate] float32; B, C: [batch, dstate]
 * activation dtype; state: [batch, dim, dstate] float32.
 *   conv_state : NULL skips the convolution (x = x_new); otherwise
 *                conv_weight is required and 1 <= conv_width <= 8.
 *   conv_bias, D, z, delta_bias : NULL means absent (0 / no gate).
 *   dims.seqlen must be 1; dims.dstate is 1..64.
 * state, conv_state and y must not overlap each other or any input. Launches
 * on `stream` without waiting. Errors as for ssm_scan_fwd.
 * For dstate 4, 8 or 16 (rows of B and C of at least 16 bytes), dim * element
 * size a multiple of 16 bytes and every buffer 16-byte aligned, each block's
 * state, inputs, conv buffers and y move as bulk copies between global and
 * shared memory; its waits for them are bounded, and one that gives up is
 * reported as SSM_ERR_TIMEOUT by ssm_scan_sync_status (the state is then
 * partly updated). The blocks of each 128-channel column take batch rows from
 * a counter in the handle's control block, cleared on `stream` before each
 * launch, so a handle runs one step at a time (one stream, or calls ordered
 * between streams). Other shapes use per-thread loads. The first call on a
 * handle allocates its 4 KiB control block on `stream`: make it before
 * capturing the step into a CUDA graph.
 */
SSM_API int ssm_scan_step(ssm_scan_t h, const void *x_new, void *conv_state,
                          const float *conv_weight, const float *conv_bias,
                          int conv_width, const void *delta,
                          const float *delta_bias, const float *A_log,
                          const void *B, const void *C, const float *D,
                          const void *z, uint32_t flags, float *state, void *y,
                          ssm_scan_dims dims, int dtype,
                          struct CUstream_st *stream);

/*
 * ssm_scan_fwd_static_scratch: the forward pass of ssm_scan_fwd for callers
 * that cannot allocate device memory. The source pages have no counterpart:
 * this entry exists for users of the library, not for the method.
 * Examples are a serving loop whose memory pool already holds the whole
 * device, or a plug-in whose host fixes its memory budget up front. For
 * such callers a cudaMalloc either fails or synchronizes the device at a bad
 * moment, and ssm_scan_fwd may grow a workspace when it splits sequences.
 *
 * This call allocates nothing. The split-sequence workspace is a fixed 8 MiB
 * device array inside the library, held by every GPU that loads the library
 * until the process exits.
 *   device   : CUDA device of every pointer; it must be current.
 *   segments : pieces per sequence: 0 chooses by shape, 1 never splits, and
 *              a larger value forces that count.
 *   status   : a device int the caller has zeroed, or NULL. A split call
 *              sets it to 1 if a bounded wait between thread blocks gave
 *              up; the outputs are then invalid. With status NULL the call
 *              never splits (segments 0 then means 1, and segments > 1
 *              returns SSM_ERR_INVALID), so no such wait can go unreported.
 *   flags    : SSM_DELTA_SOFTPLUS and SSM_WRITE_ZOH, as for ssm_scan_fwd
 *              (SSM_SAVE_CHECKPOINTS: SSM_ERR_INVALID, there is no handle).
 *   the rest : as for ssm_scan_fwd. Additionally dstate is 4, 8 or 16,
 *              dim * element size is a multiple of 16 bytes, and x, delta,
 *              z, B, C are 16-byte aligned (else SSM_ERR_UNSUPPORTED or
 *              SSM_ERR_ALIGN).
 * A split workspace that does not fit in the array returns
 * SSM_ERR_UNSUPPORTED before anything is launched. It needs
 * batch x pieces x dim x dstate x 12 bytes plus flags.
 * The first call on a device looks up the array's device address and clears
 * it, which synchronizes that device: make that first call before any stream
 * capture. Every call shares the one array, which keeps the last call's
 * contents; a split call clears its launch ticket and publication flags on
 * the stream before its kernel. Calls that overlap on the GPU race, so
 * callers on several streams or host threads must serialize them.
 */
SSM_API int ssm_scan_fwd_static_scratch(
    int device, const void *x, const void *delta, const float *A_log,
    const void *B, const void *C, const float *D, const void *z,
    const float *delta_bias, uint32_t flags, const float *h0, void *y,
    float *h_last, ssm_scan_dims dims, int dtype, int segments, int *status,
    struct CUstream_st *stream);

/* ssm_scan_status_string: static English text for a status code. */
/*
 * ssm_measure_ex2_rate: the measured throughput of the SFU's exp2 on `device`
 * (MUFU.EX2 operations per second, all SMs, at whatever clock the device runs):
 * a kernel of independent exp2 chains, 2048 threads per SM, timed over five
 * launches of about 2e11 operations (about 40 ms). The scan's roofline divides its
 * one-exp-per-element count by this unit; the pages have no counterpart, it
 * confirms the rate the roofline derives from the SM count, 16 ex2 per clock per
 * SM and the clock. Allocates 4 bytes of device memory and synchronizes the
 * device. Returns SSM_ERR_INVALID for a NULL output or a bad device,
 * SSM_ERR_CUDA on a runtime error.
 */
SSM_API int ssm_measure_ex2_rate(int device, double *ex2_per_second);

SSM_API const char *ssm_scan_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* SSM_SCAN_H */
