/*
 * ssm.h -- C ABI of libssm.so, a B200 (sm_100a) selective-scan library.
 *
 * Three operations:
 *
 *  ssm_scan_fwd    Mamba S6 selective scan, one direction.
 *                  Defined by the discrete recurrence of the Mamba2 page
 *                  ("手写简化版Mamba2", intelliparadigm.com) sec. 2.2 with the
 *                  Bbar ~= dt*B approximation, the per-step scan of sec. 4.3
 *                  and the D skip + SiLU gate of sec. 4.4:
 *                    dt[b,t,d]  = softplus(delta[b,t,d] + delta_bias[d])
 *                                 (plain delta + delta_bias if delta_softplus = 0)
 *                    h[n]       = exp(dt * A[d,n]) * h[n] + dt * B[b,t,n] * x[b,t,d]
 *                    out[b,t,d] = (sum_n C[b,t,n] h[n] + D[d] x[b,t,d]) * silu(z[b,t,d])
 *                  h starts at zero; reverse = 1 runs t = L-1 .. 0.
 *
 *  bidir_scan_fwd  Vision-Mamba bidirectional scan (the Vim reproduction page,
 *                  news.rkmt.cn, sec. 3.1-3.2): a forward scan and a reversed
 *                  scan, each with its own delta_bias, A, B, C, D, z, on shared
 *                  x and delta; out = forward result + reversed result, both at
 *                  the original positions.  Both directions are computed in one
 *                  launch over a single pass of HBM.
 *
 *  ssd_chunk_fwd   Mamba2 SSD (Mamba2 page sec. 3.1-3.2): the same recurrence
 *                  with A a scalar per head, computed chunk by chunk -- matrix
 *                  products (tensor cores) inside each chunk and the chunk state
 *                  passed on between chunks.
 *
 * Conventions shared by all entry points
 *  - Every tensor argument is a DEVICE pointer to a contiguous row-major array
 *    (last index fastest) on the current CUDA device.  The caller owns all
 *    memory, including the workspace; the library allocates nothing and keeps
 *    no state between calls.
 *  - x, delta, z, B, C and out have the element type dims->dtype (SSM_F32 or
 *    SSM_BF16).  delta_bias, A, D and last_state are always float32.
 *  - Every pointer must be 16-byte aligned; dim (S6) must be a multiple of 4
 *    for SSM_F32 and of 8 for SSM_BF16.  Otherwise SSM_ERR_MISALIGNED.
 *  - out must not overlap any input.  last_state is written, not accumulated.
 *  - All arithmetic is float32 (the state, dt, exp(dt*A)); bf16 inputs are
 *    widened exactly and the output is rounded to nearest even.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream) and thread-safe.  All arguments are validated before
 *    anything is launched; on an error nothing is launched and the return
 *    value says why.  SSM_ERR_CUDA means a launch failed (the CUDA error is
 *    then sticky in the caller's context as usual).
 *  - A zero batch, seqlen or dim is a valid empty call: the tensor pointers
 *    may then be NULL, nothing is launched, and last_state (if given and of
 *    non-zero size) is zero-filled.
 */
#ifndef SSM_B200_SSM_H
#define SSM_B200_SSM_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SSM_API __attribute__((visibility("default")))
#else
#define SSM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { SSM_F32 = 0, SSM_BF16 = 1 } ssm_dtype;

typedef enum {
    SSM_OK = 0,
    SSM_ERR_INVALID_ARG = 1,         /* NULL required pointer, negative size, NULL dims */
    SSM_ERR_UNSUPPORTED_SHAPE = 2,   /* dstate outside 1..16 (S6); SSD shape not supported */
    SSM_ERR_MISALIGNED = 3,          /* pointer not 16-byte aligned / dim not a vector multiple */
    SSM_ERR_UNSUPPORTED_DTYPE = 4,   /* dtype not SSM_F32 / SSM_BF16 (SSD: SSM_BF16 only) */
    SSM_ERR_WORKSPACE_TOO_SMALL = 5, /* workspace_bytes < the *_workspace_size() value */
    SSM_ERR_CUDA = 6,                /* a CUDA launch or runtime call failed */
    SSM_ERR_DEVICE_TIMEOUT = 7       /* a bounded device-side wait gave up (see ssm_check_device) */
} ssm_status;

/* S6 problem size.  dtype is an ssm_dtype value. */
typedef struct {
    int64_t batch;   /* B */
    int64_t seqlen;  /* L */
    int64_t dim;     /* D, channels (d_inner) */
    int64_t dstate;  /* N, 1..16 */
    int32_t dtype;
} ssm_dims;

/* Parameters of one scan direction (bidir_scan_fwd). */
typedef struct {
    const float *delta_bias; /* (D) float32, or NULL for no bias              */
    const float *A;          /* (D, N) float32, required                       */
    const void *B;           /* (B, L, N) dtype, required; shared by channels  */
    const void *C;           /* (B, L, N) dtype, required; shared by channels  */
    const float *D;          /* (D) float32, or NULL for no skip term          */
    const void *z;           /* (B, L, D) dtype, or NULL for no gate           */
    float *last_state;       /* (B, D, N) float32 output, or NULL              */
} ssm_dir_params;

/*
 * Bytes of device workspace ssm_scan_fwd needs for `dims` (0 if none).  The
 * value depends only on dims.  Returns 0 for invalid dims.
 */
SSM_API size_t ssm_scan_workspace_size(const ssm_dims *dims);

/*
 * S6 scan, one direction.
 *   x, delta   (B, L, D) dtype, required
 *   delta_bias (D) float32 or NULL;  delta_softplus: 1 = apply softplus
 *   A          (D, N) float32, required (any values; A < 0 keeps it stable)
 *   B, C       (B, L, N) dtype, required
 *   D          (D) float32 or NULL;  z (B, L, D) dtype or NULL
 *   reverse    0 = t ascending, 1 = t descending (outputs stay at their t)
 *   out        (B, L, D) dtype, written
 *   last_state (B, D, N) float32 or NULL: the state after the last step
 *              (after t = L-1 forward, after t = 0 reversed)
 *   workspace  device scratch of at least ssm_scan_workspace_size(dims)
 *              bytes (may be NULL when that size is 0); contents on entry
 *              are ignored, contents on return are unspecified.
 */
SSM_API ssm_status ssm_scan_fwd(const ssm_dims *dims, const void *x, const void *delta,
                        const float *delta_bias, int delta_softplus, const float *A,
                        const void *B, const void *C, const float *D, const void *z,
                        int reverse, void *out, float *last_state, void *workspace,
                        size_t workspace_bytes, void *stream);

/*
 * ssm_scan_fwd started from a given state.  The recurrence depends only on
 * the previous h (Mamba2 page, sec. 4.3; sec. 5.2 for inference from a
 * stored state), so a long sequence can run in pieces, each piece's
 * last_state handed to the next as its initial_state.
 *   initial_state  (B, D, N) float32 or NULL (zero): h before the first step
 *                  (before t = 0, or before t = L-1 when reversed).  It may
 *                  be the same buffer as last_state (updated in place).
 * Other arguments, workspace and errors as for ssm_scan_fwd.  With L = 0 the
 * last state is the initial state.
 */
SSM_API ssm_status ssm_scan_fwd_state(const ssm_dims *dims, const void *x, const void *delta,
                                      const float *delta_bias, int delta_softplus, const float *A,
                                      const void *B, const void *C, const float *D, const void *z,
                                      int reverse, const float *initial_state, void *out,
                                      float *last_state, void *workspace, size_t workspace_bytes,
                                      void *stream);

/*
 * One decode step for every (batch, channel): the recurrent inference form
 * of the Mamba2 page, sec. 5.2 -- the scan's step of sec. 4.3 - 4.4 applied
 * once to a stored state:
 *   dt = softplus(delta + bias);  state = exp(dt A) state + dt B x;
 *   out = (C state + D x) silu(z)
 * dims: seqlen must be 1 (SSM_ERR_UNSUPPORTED_SHAPE otherwise); batch, dim,
 *   dstate and dtype as for ssm_scan_fwd.
 *   x, delta, z  (B, D) dtype (z may be NULL: no gate)
 *   B, C         (B, N) dtype
 *   A (D, N), delta_bias (D) or NULL, D (D) or NULL: float32
 *   state        (B, D, N) float32, read and written in place
 *   out          (B, D) dtype, written
 * No workspace.  All pointers 16-byte aligned; asynchronous on stream.
 */
SSM_API ssm_status ssm_step(const ssm_dims *dims, const void *x, const void *delta,
                            const float *delta_bias, int delta_softplus, const float *A,
                            const void *B, const void *C, const float *D, const void *z,
                            float *state, void *out, void *stream);

/* Bytes of the scratch array that ssm_scan_fwd_noalloc draws from. */
#define SSM_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)

/*
 * ssm_scan_fwd for callers that cannot allocate device memory when they run
 * the scan -- for example a plugin inside an inference engine that receives
 * only its tensors and a stream at enqueue time, or a serving loop that
 * allows no allocation after start-up.  The pages have no counterpart to
 * this entry point; it is a convenience of this library.
 *
 * Arguments and results are those of ssm_scan_fwd without the workspace.
 * The scratch comes from one array of SSM_NOALLOC_SCRATCH_BYTES that the
 * library keeps on every GPU that loads it, until the process exits.  A
 * problem that needs more (ssm_scan_workspace_size(dims) larger than
 * SSM_NOALLOC_SCRATCH_BYTES) returns SSM_ERR_WORKSPACE_TOO_SMALL before
 * anything runs.  The first call on each device looks up the array's device
 * address with a CUDA runtime call; make that first call before any stream
 * capture.  The address is kept for the life of the process: after a
 * cudaDeviceReset (or any teardown of the device's primary context) this
 * entry point must not be called again in that process.  All calls share the
 * array: nothing in it needs to start at zero, but calls whose kernels
 * overlap on the GPU (other streams, other host threads) race on it.
 * Allocates nothing.
 */
SSM_API ssm_status ssm_scan_fwd_noalloc(const ssm_dims *dims, const void *x, const void *delta,
                                        const float *delta_bias, int delta_softplus,
                                        const float *A, const void *B, const void *C,
                                        const float *D, const void *z, int reverse, void *out,
                                        float *last_state, void *stream);

/* Bytes of device workspace bidir_scan_fwd needs for `dims` (0 if none). */
SSM_API size_t bidir_scan_workspace_size(const ssm_dims *dims);

/*
 * Vision-Mamba bidirectional scan:
 *   out = S6(x, delta, fwd, reverse = 0) + S6(x, delta, bwd, reverse = 1)
 * with x, delta (B, L, D) shared; fwd and bwd each as described for
 * ssm_dir_params (their last_state fields are optional outputs).
 * fwd and bwd must be non-NULL, and either both or neither have a gate z
 * (SSM_ERR_INVALID_ARG otherwise); out (B, L, D) dtype is written.
 */
SSM_API ssm_status bidir_scan_fwd(const ssm_dims *dims, const void *x, const void *delta,
                          int delta_softplus, const ssm_dir_params *fwd,
                          const ssm_dir_params *bwd, void *out, void *workspace,
                          size_t workspace_bytes, void *stream);

/*
 * ssm_scan_fwd_state and bidir_scan_fwd with the exact zero-order-hold
 * discretisation of the Mamba2 page, sec. 2.2, in place of its dt B
 * approximation: x is held constant over each step and h' = A h + B x is
 * integrated exactly, so per state
 *   h_t = exp(dt a) h_{t-1} + ((exp(dt a) - 1) / a) B_t x_t
 * (the limit dt B_t x_t where a = 0).  On the GPU the coefficient is
 * (e - 1) / a from the step's own exponential e where |dt a| >= 1/16, and
 * the series dt (1 + u/2 + u^2/6 + u^3/24), u = dt a, below that (where
 * e - 1 would cancel).
 * Arguments, layouts, workspace (ssm_scan_workspace_size /
 * bidir_scan_workspace_size of the same dims) and errors as for
 * ssm_scan_fwd_state and bidir_scan_fwd, and:
 *   dims->dstate must be 16 and dims->batch at most 65535
 *   (SSM_ERR_UNSUPPORTED_SHAPE otherwise): these run only on the layout
 *   that splits each channel's 16 states over two or four threads, in one
 *   pass without segments, so long sequences over few channels (where the
 *   dt B scans cut the sequence into segments) run several times slower.
 * Forward scans only: the backward, checkpointing, ordered, conv and decode
 * entry points use dt B.
 */
SSM_API ssm_status ssm_scan_fwd_zoh(const ssm_dims *dims, const void *x, const void *delta,
                                   const float *delta_bias, int delta_softplus, const float *A,
                                   const void *B, const void *C, const float *D, const void *z,
                                   int reverse, const float *initial_state, void *out,
                                   float *last_state, void *workspace, size_t workspace_bytes,
                                   void *stream);
SSM_API ssm_status bidir_scan_fwd_zoh(const ssm_dims *dims, const void *x, const void *delta,
                                     int delta_softplus, const ssm_dir_params *fwd,
                                     const ssm_dir_params *bwd, void *out, void *workspace,
                                     size_t workspace_bytes, void *stream);

/*
 * How ssm_scan_fwd (bidirectional = 0) or bidir_scan_fwd (bidirectional = 1)
 * runs a problem of these sizes.  The pages have no counterpart: this is a
 * query of the library's own launch plan, for callers sizing work and for
 * tests.
 *   segments           (out, may be NULL) the number of pieces the sequence
 *                      is cut into for parallelism (1: one pass; more: the
 *                      chunked scan with state hand-off of the Mamba2 page,
 *                      sec. 3.2, run as summary, carry and main passes)
 *   channels_per_lane  (out, may be NULL) 1 or 2: channels one GPU thread owns;
 *                      -2 or -4: that many threads share each channel, each
 *                      holding an equal share of its 16 states (one pass, no
 *                      segments; N = 16 only).  With -2 the last batch rows
 *                      may take four threads per channel in the same launch,
 *                      where that evens out the launch's last round of warps.
 * Host-only, makes no CUDA call.  Returns the status the scan entry points
 * give for invalid dims; an empty problem reports 1 segment.
 */
SSM_API ssm_status ssm_scan_plan(const ssm_dims *dims, int bidirectional, int *segments,
                                 int *channels_per_lane);

/*
 * S6 along a given order of the positions, with an optional token mask:
 * the row, column, cross (several orders, summed by the caller) and
 * centre-out spiral scans of the Samba (sec. 3.1) and Mamba-YOLO
 * (sec. 1.2, 4.4) pages, and the masked-token bypass of the Samba page's
 * pyramid-mask module (sec. 2).
 *   order  (L) int32, 4-byte aligned, a permutation of 0..L-1 shared by the
 *          batch, or NULL (0..L-1): step i reads and writes position
 *          order[i] (order[L-1-i] when reversed).  An entry outside [0, L)
 *          is treated as its own step index and makes ssm_check_device
 *          return SSM_ERR_INVALID_ARG; repeated entries give unspecified
 *          results.
 *   mask   (B, L) bytes indexed by position, or NULL: 0 bypasses the token
 *          -- the state passes through unchanged and out at that position
 *          is 0 (for the bidirectional form, in both directions).
 * Other arguments, workspace and errors as for ssm_scan_fwd.
 */
SSM_API ssm_status ssm_scan_fwd_ordered(const ssm_dims *dims, const void *x, const void *delta,
                                        const float *delta_bias, int delta_softplus, const float *A,
                                        const void *B, const void *C, const float *D, const void *z,
                                        int reverse, const int32_t *order, const unsigned char *mask,
                                        void *out, float *last_state, void *workspace,
                                        size_t workspace_bytes, void *stream);

/* bidir_scan_fwd along an order (the forward parameters scan it, the
 * backward ones scan it reversed), with the token mask above. */
SSM_API ssm_status bidir_scan_fwd_ordered(const ssm_dims *dims, const void *x, const void *delta,
                                          int delta_softplus, const ssm_dir_params *fwd,
                                          const ssm_dir_params *bwd, const int32_t *order,
                                          const unsigned char *mask, void *out, void *workspace,
                                          size_t workspace_bytes, void *stream);

/*
 * The depthwise causal conv1d that precedes the scan (the Mamba2 page's
 * block, sec. 4.4 listing: one kernel per channel, padding width-1, the
 * first L outputs kept; the Vim page, sec. 2: a short kernel before the
 * scan to mix neighbouring tokens), optionally followed by SiLU:
 *   u[t, d] = act(bias[d] + sum_{k < width} weight[d, k] x_in[t - (width-1) + k, d])
 * with t counted along the scan direction (a reversed scan convolves the
 * flipped sequence) and x_in = 0 before the first step.
 */
typedef struct {
    const float *weight;   /* (D, width) float32, required */
    const float *bias;     /* (D) float32, or NULL */
    int32_t width;         /* 1..4 (SSM_ERR_UNSUPPORTED_SHAPE otherwise) */
    int32_t silu;          /* 1: u = silu(conv), 0: u = conv */
} ssm_conv_params;

/*
 * ssm_scan_fwd on u = conv(x_in) computed inside the scan: x_in (B, L, D)
 * dtype replaces x, and the scan and its D skip both use u.  Other
 * arguments, workspace and errors as for ssm_scan_fwd.
 */
SSM_API ssm_status ssm_scan_fwd_conv(const ssm_dims *dims, const void *x_in, const ssm_conv_params *conv,
                                     const void *delta, const float *delta_bias, int delta_softplus,
                                     const float *A, const void *B, const void *C, const float *D,
                                     const void *z, int reverse, void *out, float *last_state,
                                     void *workspace, size_t workspace_bytes, void *stream);

/* bidir_scan_fwd on x_in, each direction convolving it with its own conv
 * along its own scan direction (as each Vim direction has its own conv). */
SSM_API ssm_status bidir_scan_fwd_conv(const ssm_dims *dims, const void *x_in, const void *delta,
                                       int delta_softplus, const ssm_dir_params *fwd,
                                       const ssm_dir_params *bwd, const ssm_conv_params *conv_fwd,
                                       const ssm_conv_params *conv_bwd, void *out, void *workspace,
                                       size_t workspace_bytes, void *stream);

/* Bytes of device workspace ssm_scan_bwd needs for `dims` (0 for invalid dims). */
SSM_API size_t ssm_scan_bwd_workspace_size(const ssm_dims *dims);

/*
 * Gradients of ssm_scan_fwd (same dims and inputs, same reverse flag) for
 * an incoming gradient dout of out -- the training use of the Mamba2 page,
 * sec. 5.1, which backpropagates through the scan.  The states are
 * recomputed (a forward pass stores h every 4 steps in the workspace), so
 * nothing from the forward call is needed.  All gradients are float32:
 *   dout            (B, L, D) dtype, required
 *   dx, ddelta      (B, L, D), required, written
 *   dA (D, N), dB, dC (B, L, N): required, written
 *   dD (D), dz (B, L, D), ddelta_bias (D): required when D, z, delta_bias
 *                   are given (else ignored), written
 * ddelta is the gradient of the raw delta (through the softplus when
 * delta_softplus is set).  dB, dC sum over the channels, dA, dD and
 * ddelta_bias over the batch and the sequence.  Workspace:
 * ssm_scan_bwd_workspace_size(dims) bytes.  Errors as for ssm_scan_fwd.
 */
SSM_API ssm_status ssm_scan_bwd(const ssm_dims *dims, const void *x, const void *delta,
                                const float *delta_bias, int delta_softplus, const float *A,
                                const void *B, const void *C, const float *D, const void *z,
                                int reverse, const void *dout, float *dx, float *ddelta, float *dA,
                                float *dB, float *dC, float *dD, float *dz, float *ddelta_bias,
                                void *workspace, size_t workspace_bytes, void *stream);

/* Gradients of one direction's parameters (bidir_scan_bwd), float32. */
typedef struct {
    float *dA;            /* (D, N), required */
    float *dB, *dC;       /* (B, L, N), required */
    float *dD;            /* (D): required when the direction has D */
    float *dz;            /* (B, L, D): required when the direction has z */
    float *ddelta_bias;   /* (D): required when the direction has delta_bias */
} ssm_dir_grads;

/*
 * Gradients of bidir_scan_fwd for an incoming gradient dout (B, L, D) dtype:
 * dx and ddelta (B, L, D) float32 sum both directions (x and delta are
 * shared); each direction's parameter gradients go to its ssm_dir_grads.
 * Same workspace as ssm_scan_bwd (ssm_scan_bwd_workspace_size); errors as
 * for ssm_scan_bwd.
 */
SSM_API ssm_status bidir_scan_bwd(const ssm_dims *dims, const void *x, const void *delta,
                                  int delta_softplus, const ssm_dir_params *fwd,
                                  const ssm_dir_params *bwd, const void *dout, float *dx, float *ddelta,
                                  const ssm_dir_grads *grad_fwd, const ssm_dir_grads *grad_bwd,
                                  void *workspace, size_t workspace_bytes, void *stream);

/*
 * Training pair that skips the backward's recompute of the states.  The
 * backward above rebuilds the state entering every 4-step chunk with a
 * forward pass of its own (the recompute the Mamba2 page, sec. 5.1, suggests
 * instead of keeping every step); a training loop runs the forward scan
 * anyway, so the checkpointing forward below stores those states while it
 * scans, and the checkpointed backward reads them instead of recomputing.
 *
 * Checkpoint array of one direction: the state entering every 4-step chunk
 * of that direction's scan order (chunk 0's is zero), (B, ceil(L / 4), D, NS)
 * float32 with NS = N rounded up to 4, 8 or 16 (padding states zero),
 * ssm_scan_ckpt_size(dims) bytes, caller-owned, 16-byte aligned.  It is only
 * meaningful for the same dims, inputs and direction; a backward given an
 * array of another call computes wrong gradients (the library cannot tell).
 * When the plan cuts the sequence into segments, the entering state of each
 * segment comes from the carry pass, so the checkpoints (and the gradients
 * from them) can differ from the recomputed ones in the last bits.
 */
SSM_API size_t ssm_scan_ckpt_size(const ssm_dims *dims);

/* ssm_scan_fwd that also writes the checkpoint array `ckpt` (required when
 * the problem is not empty).  Errors as for ssm_scan_fwd. */
SSM_API ssm_status ssm_scan_fwd_ckpt(const ssm_dims *dims, const void *x, const void *delta,
                                     const float *delta_bias, int delta_softplus, const float *A,
                                     const void *B, const void *C, const float *D, const void *z,
                                     int reverse, void *out, float *last_state, float *ckpt,
                                     void *workspace, size_t workspace_bytes, void *stream);

/* bidir_scan_fwd that also writes each direction's checkpoint array
 * (ckpt_fwd for the forward scan, ckpt_bwd for the reversed one; both
 * required when the problem is not empty). */
SSM_API ssm_status bidir_scan_fwd_ckpt(const ssm_dims *dims, const void *x, const void *delta,
                                       int delta_softplus, const ssm_dir_params *fwd,
                                       const ssm_dir_params *bwd, void *out, float *ckpt_fwd,
                                       float *ckpt_bwd, void *workspace, size_t workspace_bytes,
                                       void *stream);

/* ssm_scan_bwd from the checkpoints of ssm_scan_fwd_ckpt (same dims,
 * inputs and reverse flag): no workspace, no recompute pass.  Errors as for
 * ssm_scan_bwd; a NULL ckpt is SSM_ERR_INVALID_ARG. */
SSM_API ssm_status ssm_scan_bwd_ckpt(const ssm_dims *dims, const void *x, const void *delta,
                                     const float *delta_bias, int delta_softplus, const float *A,
                                     const void *B, const void *C, const float *D, const void *z,
                                     int reverse, const void *dout, float *dx, float *ddelta, float *dA,
                                     float *dB, float *dC, float *dD, float *dz, float *ddelta_bias,
                                     const float *ckpt, void *stream);

/* bidir_scan_bwd from the checkpoints of bidir_scan_fwd_ckpt. */
SSM_API ssm_status bidir_scan_bwd_ckpt(const ssm_dims *dims, const void *x, const void *delta,
                                       int delta_softplus, const ssm_dir_params *fwd,
                                       const ssm_dir_params *bwd, const void *dout, float *dx,
                                       float *ddelta, const ssm_dir_grads *grad_fwd,
                                       const ssm_dir_grads *grad_bwd, const float *ckpt_fwd,
                                       const float *ckpt_bwd, void *stream);

/* SSD problem size.  Supported: dtype SSM_BF16, headdim 64, dstate 128,
 * chunk 64, seqlen any value >= 0 (a short last chunk is handled). */
typedef struct {
    int64_t batch;    /* B */
    int64_t seqlen;   /* L */
    int64_t nheads;   /* H */
    int64_t headdim;  /* P */
    int64_t dstate;   /* N */
    int64_t chunk;    /* Q, tokens per chunk */
    int32_t dtype;
} ssd_dims;

/* Bytes of device workspace ssd_chunk_fwd needs for `dims` (0 if none). */
SSM_API size_t ssd_chunk_workspace_size(const ssd_dims *dims);

/*
 * Mamba2 SSD chunked scan (Mamba2 page sec. 3.2), equal to the sequential
 * recurrence with A[d, n] = A[h] for every channel d = (h, p) of head h:
 *   x, z       (B, L, H, P) dtype (z may be NULL: no gate)
 *   delta      (B, L, H) dtype;  delta_bias (H) float32 or NULL
 *   A          (H) float32;  D (H) float32 or NULL
 *   B, C       (B, L, N) dtype, shared by all heads
 *   out        (B, L, H, P) dtype, written
 *   last_state (B, H, P, N) float32 or NULL
 */
SSM_API ssm_status ssd_chunk_fwd(const ssd_dims *dims, const void *x, const void *delta,
                         const float *delta_bias, int delta_softplus, const float *A,
                         const void *B, const void *C, const float *D, const void *z,
                         void *out, float *last_state, void *workspace,
                         size_t workspace_bytes, void *stream);

/*
 * Waits for `stream`, then reports (and clears) the library's device-side
 * error words: SSM_ERR_DEVICE_TIMEOUT if a bounded wait inside a kernel gave
 * up since the last check, SSM_ERR_INVALID_ARG if a scan order held an
 * index outside [0, L), SSM_ERR_CUDA if the stream reports a CUDA error,
 * SSM_OK otherwise.  Blocking; meant for tests and debugging.
 */
SSM_API ssm_status ssm_check_device(void *stream);

/*
 * Test hook for the device-timeout path (the pages have no counterpart; it
 * exists so that a test can make a bounded device wait run out without
 * faulting or hanging the GPU).  SSD calls enqueued after it, in this
 * process, run with every pipeline wait limited to `wait_limit` polls
 * (0 restores the default of 1 << 20) and, if `withhold_chunk` >= 0, with
 * the producer warp never signalling that chunk's dt, so the consumers' wait
 * for it runs out: such a call still completes (its outputs are undefined,
 * every copy and MMA it issued is waited for, its tensor memory is freed)
 * and the next ssm_check_device returns SSM_ERR_DEVICE_TIMEOUT.
 * ssm_debug_ssd_stall(-1, 0) restores normal calls.  Process-wide and not
 * synchronised with calls on other threads: for tests only.
 */
SSM_API void ssm_debug_ssd_stall(int withhold_chunk, unsigned wait_limit);

/*
 * Test hook for the choice between the thread layouts of the plain S6 scans
 * (ssm_scan_fwd, ssm_scan_fwd_state, ssm_scan_fwd_noalloc, bidir_scan_fwd and
 * the checkpointing forwards; the pages have no counterpart).  With N = 16 those calls
 * either give each GPU thread one or two whole channels (cutting long
 * sequences into segments), or split each channel's 16 states over four or
 * over two threads in one pass; a cost model fitted to measured B200
 * timings picks the fastest for the sizes (mode 0, the default).  Mode 1
 * makes calls enqueued after it, in this process, always take the first
 * layout, mode 2 four threads per channel and mode 3 two whenever N = 16;
 * ssm_scan_plan reports what the calls take.  The backward passes with
 * N = 16 split each channel's states over four threads unless mode 1 is
 * set (then one thread per channel).
 * The two layouts sum the readout in different orders, so results agree to
 * rounding, not bit for bit.  Returns SSM_ERR_INVALID_ARG for another mode.
 * Process-wide and not synchronised with calls on other threads: for tests.
 */
SSM_API ssm_status ssm_debug_s6_mapping(int mode);

/* Static, human-readable name of a status code. */
SSM_API const char *ssm_status_string(ssm_status status);

/* Library ABI version (major * 10000 + minor * 100 + patch). */
SSM_API int ssm_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SSM_B200_SSM_H */
