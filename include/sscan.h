/*
 * sscan.h -- C ABI of the B200 (sm_100a) selective-scan forward library
 * (libsscan.so).
 *
 * The operation ("tm_ssm_selective" (Transformer Math page on selective
 * SSMs), section "Discretization becomes a per-token operation"; the
 * selective_scan reference loop of "12. Selective State Space"; shapes from
 * "Mamba & Mamba-2 Architecture", section 1): for every batch row b, channel
 * d and state n, with the step delta = delta[b,t,d] and x = u[b,t,d],
 *
 *     Abar       = exp(delta * A[d,n])                     (zero-order hold of A)
 *     Bbar u     = delta * B[b,t,n] * x                    (Euler, the default)
 *                | (exp(delta*A[d,n]) - 1) / A[d,n] * B[b,t,n] * x   (SSCAN_ZOH)
 *     h[b,d,n]   = Abar * h[b,d,n] + Bbar u                (h before t = 0: h0, or 0)
 *     y[b,t,d]   = sum_n C[b,t,n] * h[b,d,n]               (state after token t)
 *     h_final[b,d,n] = h after the last token
 *
 * The [B,L,D,N] state sequence is never written to memory: each (b,d) state
 * row lives in registers ("Selective State-Space Models (Mamba) and
 * Hardware-Aware Scans", section 3, kernel fusion and SRAM residency).
 *
 * Layout.  Every tensor is dense row-major (C order), in device memory:
 *     u, delta, y : [B][L][D]   dtype of the plan (fp32 or bf16)
 *     B, C        : [B][L][N]   dtype of the plan
 *     A           : [D][N]      fp32 (the pages' A = -exp(A_log), diagonal)
 *     h0, h_final : [B][D][N]   fp32 (the state is always kept in fp32)
 * Every pointer must be 16-byte aligned.  The state and all arithmetic are
 * fp32; a bf16 plan widens its inputs exactly and rounds y to nearest-even.
 *
 * Ownership.  The caller owns every buffer passed in (inputs, outputs and
 * the workspace).  A plan owns its host-side description and one 4-byte
 * device status word that it allocates at creation and frees on destroy.
 *
 * Streams and errors.  sscan_forward enqueues its work on the caller's
 * stream and returns without synchronising.  Every entry point returns an
 * SSCAN_* status: argument problems are reported before anything is
 * launched; a failed launch gives SSCAN_ERR_CUDA.  Conditions only the
 * device can see (a bounded wait that gave up) are latched in the plan's
 * status word and read back with sscan_get_status.
 *
 * CUDA graphs.  A launch of the chained or tiled schedules (sscan_plan_describe
 * says "kernel=chained" or "kernel=tiled") tags its carry flags with a tag the
 * host picks per call,
 * so a graph that captured it would replay the same tag and could read a
 * carried state left by an earlier replay: do not replay such calls from a
 * graph.  The decode, step and generic schedules keep no state between
 * launches and may be captured.
 *
 * Aliasing.  y must not overlap any input.  h_final may be the same buffer
 * as h0 (each state row is read before it is written, by the same thread).
 *
 * Thread safety.  A plan may be used from one host thread at a time; calls
 * with distinct plans are independent.
 */
#ifndef SSCAN_H
#define SSCAN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SSCAN_API __attribute__((visibility("default")))
#else
#define SSCAN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct sscan_plan *sscan_plan_t;

/* dtype of u, delta, B, C and y */
enum { SSCAN_F32 = 0, SSCAN_BF16 = 1 };

/* flags */
enum {
    /* exact zero-order-hold input term (exp(delta*A)-1)/A * B * u instead of
     * the Euler term delta * B * u ("tm_ssm_selective", section
     * "Discretization becomes a per-token operation") */
    SSCAN_ZOH = 1u << 0,
    /* fused prologue: the scan uses delta' = softplus(delta + delta_bias[d])
     * = log(1 + exp(delta + delta_bias[d])) instead of delta, i.e. delta is
     * the raw projection Linear_D(u_t) and the bias d_bias of
     * "tm_ssm_selective", section "The mechanism: parameters as functions of
     * the input" (Delta_t = softplus(d_bias + Linear_D(u_t))) */
    SSCAN_DELTA_SOFTPLUS = 1u << 1
};

/* status codes */
enum {
    SSCAN_OK = 0,
    SSCAN_ERR_INVALID = 1,      /* bad size, null pointer, overlapping output, bad flag */
    SSCAN_ERR_UNSUPPORTED = 2,  /* N outside {16, 32, 64}, or no usable CUDA device */
    SSCAN_ERR_ALIGN = 3,        /* a pointer is not 16-byte aligned */
    SSCAN_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
    SSCAN_ERR_TIMEOUT = 5,      /* device side: a bounded wait for another block gave up */
    SSCAN_ERR_WORKSPACE = 6     /* workspace missing, misaligned or too small */
};

/* Create a plan for one problem shape on the current CUDA device.
 *   B, L, D  batch rows, tokens, channels (B, D >= 1; L >= 0)
 *   N        state size per channel, one of 16, 32, 64 (the pages use 16;
 *            "12. Selective State Space" discusses 64 and 128)
 *   dtype    SSCAN_F32 or SSCAN_BF16
 *   flags    0 or any of SSCAN_ZOH, SSCAN_DELTA_SOFTPLUS
 * On success *plan receives the plan and SSCAN_OK is returned; otherwise
 * *plan is set to NULL.  Sizes are validated before any CUDA call, so
 * SSCAN_ERR_INVALID / SSCAN_ERR_UNSUPPORTED come back without a device. */
SSCAN_API int sscan_plan_create(sscan_plan_t *plan, int64_t B, int64_t L, int64_t D, int64_t N,
                      int dtype, uint32_t flags);

/* Release a plan (NULL is ignored).  Not stream-ordered: no forward call of
 * this plan may still be running. */
SSCAN_API void sscan_plan_destroy(sscan_plan_t plan);

/* Bytes of device workspace sscan_forward needs for this plan (0 when the
 * chosen schedule needs none).  The workspace must be 256-byte aligned. */
SSCAN_API size_t sscan_workspace_bytes(sscan_plan_t plan);

/* Enqueue the forward pass on `stream` (a cudaStream_t; NULL = legacy default).
 *   u, delta        [B][L][D], plan dtype
 *   A               [D][N] fp32
 *   B, C            [B][L][N], plan dtype
 *   h0              [B][D][N] fp32, or NULL for a zero initial state
 *   y               [B][L][D], plan dtype (output)
 *   h_final         [B][D][N] fp32 (output), or NULL to skip it
 *   workspace       sscan_workspace_bytes(plan) bytes, or NULL when that is 0
 * Returns SSCAN_OK once the work is enqueued. */
SSCAN_API int sscan_forward(sscan_plan_t plan, const void *u, const void *delta, const float *A,
                  const void *B, const void *C, const float *h0, void *y, float *h_final,
                  void *workspace, void *stream);

/* sscan_forward with the fused prologue and epilogue of the Mamba block:
 *   delta_bias      [D] fp32 added to delta before use (and before softplus
 *                   when the plan has SSCAN_DELTA_SOFTPLUS), or NULL
 *   z               [B][L][D], plan dtype: the output is y * silu(z),
 *                   silu(z) = z / (1 + exp(-z)), or NULL for no gate
 *                   ("Selective State-Space Models (Mamba) and Hardware-Aware
 *                   Scans", section 4: the block's second branch gates the
 *                   SSM output multiplicatively)
 * h_final is the state of the scan (the gate acts on y only).  All other
 * arguments, the ownership (caller-owned device buffers, nothing retained)
 * and the errors are those of sscan_forward; delta_bias and z must be
 * 16-byte aligned and must not overlap y or h_final.  sscan_forward is this
 * call with delta_bias = z = NULL. */
SSCAN_API int sscan_forward_gated(sscan_plan_t plan, const void *u, const void *delta, const float *A,
                        const void *B, const void *C, const float *h0, const float *delta_bias,
                        const void *z, void *y, float *h_final, void *workspace, void *stream);

/* Bytes of device workspace sscan_forward_host needs for this plan (always
 * > 0; 0 only when plan is NULL or host memory ran out).  The workspace must
 * be 256-byte aligned.  It holds two buffer slots of one piece's inputs and
 * outputs (the slot for z is reserved whether or not a call passes z), A, the
 * bias, the state (carried, or the piece's rows') and the pieces' scan
 * workspaces. */
SSCAN_API size_t sscan_host_workspace_bytes(sscan_plan_t plan);

/* sscan_forward_gated on HOST buffers: the arguments and their layouts are
 * those of sscan_forward_gated, except that u, delta, A, B, C, h0,
 * delta_bias, z, y and h_final live in host memory (page-locked memory lets
 * the copies overlap; any memory cudaMemcpy accepts works), need no
 * alignment, and `workspace` is device memory of
 * sscan_host_workspace_bytes(plan) bytes.  The call cuts the problem into
 * pieces: at most 8 along L (multiples of 64 tokens, the last one shorter; the
 * state carried between pieces in the workspace: a piece's h_final is the
 * next piece's h0, exactly the split-call resume of sscan_forward) or, when L
 * is below 512 tokens and B >= 2, 2 along the independent batch rows.  For each
 * piece it copies the inputs to the device, scans and copies y (and, along B,
 * the rows' h_final) back; with two buffer slots, the host-to-device copy of
 * piece k+1 and the device-to-host copy of piece k-1 run while piece k is
 * scanned.  The results equal one sscan_forward_gated call on the whole
 * problem.
 * Streams: the work starts after what is already queued on `stream`, and
 * `stream` waits for all of it (copies included) before anything queued
 * later, so synchronising `stream` makes y and h_final readable; the call
 * itself returns without synchronising.  The plan creates two internal
 * streams and a few events on its first host call (freed with the plan).
 * Ownership and errors as for sscan_forward_gated (the aliasing rules apply
 * to the host buffers; a workspace that overlaps one gives
 * SSCAN_ERR_WORKSPACE); device-side waits of the pieces are latched in the
 * plan's status word (sscan_get_status). */
SSCAN_API int sscan_forward_host(sscan_plan_t plan, const void *u, const void *delta, const float *A,
                                 const void *B, const void *C, const float *h0, const float *delta_bias,
                                 const void *z, void *y, float *h_final, void *workspace, void *stream);

/* Backward pass of the forward: gradients of a loss given dy = dLoss/dy and
 * optionally dh_final = dLoss/dh_final, by the chain rule through
 * h_t = Abar_t h_{t-1} + beta_t u_t, y_t = C_t . h_t, the states recomputed
 * from checkpoints rather than stored ("Selective State-Space Models (Mamba)
 * and Hardware-Aware Scans", section 3, backward-pass recomputation).
 * Shape-based (no plan):
 *   B, L, D, N, dtype, flags  as for sscan_plan_create (N = 16, 32 or 64; flags
 *                           SSCAN_ZOH and SSCAN_DELTA_SOFTPLUS as in the forward)
 *   u, delta, A, B_in, C_in, h0  the forward's inputs (as for sscan_forward;
 *                           delta is the raw step when SSCAN_DELTA_SOFTPLUS is set)
 *   dy                      [B][L][D], dtype
 *   dh_final                [B][D][N] fp32, or NULL (zero)
 *   du, ddelta              [B][L][D], dtype (output; ddelta is the gradient of
 *                           the delta passed in, i.e. of the raw step when fused)
 *   dA                      [D][N] fp32 (output; summed over batch and time)
 *   dB, dC                  [B][L][N] fp32 (output; summed over channels)
 *   dh0                     [B][D][N] fp32 (output), or NULL to skip it
 *   workspace               sscan_backward_workspace_bytes(B, L, D, N) bytes
 *                           (the state checkpoints and the per-block partial
 *                           sums of dB and dC), 16-byte aligned
 * All pointers are caller-owned device memory; nothing is retained.  dA and
 * the bias gradient are accumulated with fp32 atomics, so their last bits
 * depend on the order of arrival; dB and dC are sums in a fixed order.  Two
 * kernels are enqueued.  Errors as for sscan_forward (SSCAN_ERR_UNSUPPORTED for N
 * outside {16, 32, 64}).  sscan_backward is sscan_backward_gated without a
 * bias and a gate. */
SSCAN_API size_t sscan_backward_workspace_bytes(int64_t B, int64_t L, int64_t D, int64_t N);
SSCAN_API int sscan_backward(int64_t B, int64_t L, int64_t D, int64_t N, int dtype, uint32_t flags, const void *u,
                   const void *delta, const float *A, const void *B_in, const void *C_in, const float *h0,
                   const void *dy, const float *dh_final, void *du, void *ddelta, float *dA, float *dB, float *dC,
                   float *dh0, void *workspace, void *stream);

/* Backward pass of sscan_forward_gated (the fused prologue delta' =
 * softplus(delta + delta_bias) and gate y' = y silu(z)): the arguments of
 * sscan_backward plus
 *   delta_bias              [D] fp32 as passed to the forward, or NULL
 *   z                       [B][L][D], dtype, the forward's gate, or NULL
 *   ddelta_bias             [D] fp32 (output, summed over batch and time;
 *                           required when delta_bias is given, else NULL)
 *   dz                      [B][L][D], dtype (output; required when z is given)
 * dy is the gradient of the gated output y'; ddelta the gradient of the raw
 * delta.  By the chain rule around the plain backward: the scan's output
 * gradient is dy silu(z), dz = dy ys silu'(z) with ys the scan's output
 * (recomputed), ddelta_raw = ddelta' sigmoid(delta + delta_bias) under
 * softplus ("Selective State-Space Models (Mamba) and Hardware-Aware Scans",
 * section 4, the gate; "tm_ssm_selective", "The mechanism: parameters as
 * functions of the input", the softplus step). */
SSCAN_API int sscan_backward_gated(int64_t B, int64_t L, int64_t D, int64_t N, int dtype, uint32_t flags,
                                   const void *u, const void *delta, const float *A, const void *B_in,
                                   const void *C_in, const float *h0, const float *delta_bias, const void *z,
                                   const void *dy, const float *dh_final, void *du, void *ddelta, float *dA,
                                   float *dB, float *dC, float *dh0, float *ddelta_bias, void *dz,
                                   void *workspace, void *stream);

/* Mamba-2 state-space-duality (SSD) forward ("Mamba & Mamba-2 Architecture",
 * section 3, "Mamba-2 and State Space Duality (SSD)"): one scalar transition
 * per head, a_t = exp(delta[b,t,h] * A[h]); B and C shared by all heads; per
 * batch row b and head h, with Bbar_s = delta[b,s,h] * B[b,s,:],
 *
 *     y[b,t,h,:]    = sum_{s <= t} (C[b,t,:] . Bbar_s) (prod_{k=s+1..t} a_k) x[b,s,h,:]
 *                     + (prod_{k <= t} a_k) C[b,t,:] h0[b,h]          (Y = (M o C Bbar^T) X)
 *     h_final[b,h]  = sum_s (prod_{k > s} a_k) Bbar_s^T x[b,s,h,:] + (prod_k a_k) h0[b,h]
 *
 * computed block by block (128 tokens) on the tensor cores: the intra-block
 * matrix times X, the inter-block term from the carried state, and the state
 * passing between blocks.  Shape-based (no plan, no workspace):
 *   B, L, H     batch rows, tokens, heads (B, H >= 1; L >= 0)
 *   P, N        head dimension and state size; P = 64, N = 128 are compiled in
 *               (others: SSCAN_ERR_UNSUPPORTED)
 *   x           [B][L][H][P] bf16
 *   delta       [B][L][H] fp32, the step after softplus (>= 0)
 *   A           [H] fp32 (A <= 0, the decay per unit step)
 *   B_in, C_in  [B][L][N] bf16
 *   h0          [B][H][N][P] fp32, or NULL for a zero initial state
 *   y           [B][L][H][P] bf16 (output; round to nearest even)
 *   h_final     [B][H][N][P] fp32 (output), or NULL; may be the same buffer as h0
 *   status      a device int the kernel ORs error bits into when one of its
 *               bounded waits gives up (y and h_final then incomplete), or NULL
 * Every pointer is caller-owned device memory, 16-byte aligned (status: 4);
 * nothing is retained and nothing is allocated.  Asynchronous on `stream`.
 * Arithmetic: bf16 MMA operands (x, B, C as given; the intra-block matrix, the
 * carried state and the decay-weighted x rounded to bf16 as operands), fp32
 * accumulation, fp32 state and decays.  Errors as for sscan_forward. */
SSCAN_API int sscan_ssd_forward(int64_t B, int64_t L, int64_t H, int64_t P, int64_t N, const void *x,
                                const float *delta, const float *A, const void *B_in, const void *C_in,
                                const float *h0, void *y, float *h_final, int *status, void *stream);

/* Wait for `stream`, then read and clear the plan's device status word.
 * Returns SSCAN_OK, SSCAN_ERR_TIMEOUT, or SSCAN_ERR_CUDA. */
SSCAN_API int sscan_get_status(sscan_plan_t plan, void *stream);

/* Static description of a status code. */
SSCAN_API const char *sscan_status_string(int status);

/* Describe the schedule the plan chose (states per thread, threads per
 * channel, time chunks, grid) into buf (NUL-terminated, truncated to len).
 * Returns the number of characters the full description needs. */
SSCAN_API int sscan_plan_describe(sscan_plan_t plan, char *buf, size_t len);

/* Library version, major*10000 + minor*100 + patch. */
SSCAN_API int sscan_version(void);

/* The forward pass for callers that must not allocate device memory.  There is
 * no counterpart in the pages: this is a deployment convenience.
 *
 * Who needs it: code that runs where cudaMalloc is unavailable or unwelcome,
 * e.g. a host that has handed all device memory to its own pool, or a
 * latency-critical call site that cannot afford an allocation (which may
 * synchronise the device).  Such callers still own and pass every input and
 * output buffer; what they cannot provide is the plan (its status word) and
 * the scratch workspace that sscan_forward needs for some shapes.
 *
 * This entry point allocates nothing.  It takes the shape directly (same
 * meaning and limits as sscan_plan_create), the same buffers as sscan_forward
 * and a stream, chooses the same schedule a plan would, and uses as scratch a
 * fixed 32 MiB array compiled into the library (every GPU that loads the
 * library holds it until the process exits).  Shapes whose workspace does not
 * fit return SSCAN_ERR_WORKSPACE without launching.
 *
 * The first call on a device looks up the array's device address on that
 * device (the current one); make that first call before capturing any stream
 * work.  Every call shares the one array: its contents persist between calls,
 * the parts that must start at zero are cleared on the caller's stream at the
 * start of each call, and calls whose work overlaps on the GPU (other streams,
 * other host threads) race on it.  The return value reports argument and
 * launch errors; what only the device can see (a bounded wait that gave up,
 * leaving part of y and h_final unwritten) is latched in a status word inside
 * the array, which each call clears at its start: read it with
 * sscan_noalloc_status after the call and before the next one. */
SSCAN_API int sscan_forward_noalloc(int64_t B, int64_t L, int64_t D, int64_t N, int dtype,
                                    uint32_t flags, const void *u, const void *delta, const float *A,
                                    const void *B_in, const void *C_in, const float *h0, void *y,
                                    float *h_final, void *stream);

/* Status of the last sscan_forward_noalloc call on the current device: waits for
 * `stream` (the stream that call used), reads and clears the device status word
 * in the library's fixed array.  Allocates nothing.  Returns SSCAN_OK,
 * SSCAN_ERR_TIMEOUT (a device wait of that call gave up: its y and h_final are
 * incomplete) or SSCAN_ERR_CUDA. */
SSCAN_API int sscan_noalloc_status(void *stream);

#ifdef __cplusplus
}
#endif

#endif /* SSCAN_H */
