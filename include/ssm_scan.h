/*
 * ssm_scan.h -- C ABI of the B200 (sm_100a) selective diagonal scan library.
 *
 * The operation (per batch row b and head h) is the linear-transition
 * state-space recurrence
 *      h_t = A_t h_{t-1} + B_t u_t,      y_t = C_t h_t + D u_t
 * of "When a Diagonal State Is Not Enough" (sungsoo.github.io), Part 01
 * "Definition" and Part 03 "Selective SSM and masked linear attention", in
 * the HybridMamba / SSD-MIMO form of "Diagonal Equivalence in State Space
 * Models" (abstract; kongchang.com "From MIMO to HybridMamba"):
 *
 *  - state H_t is N x P per head, N = n_real + 2 * n_pairs: n_real real
 *    coordinates with per-coordinate decay (Mamba-1 style) followed by
 *    n_pairs complex coordinates stored as (re, im) row pairs and evolved by
 *    real 2x2 decay-rotation blocks (Mamba-3 style); P channels share one
 *    transition (Mamba-2-style heads);
 *  - A_t = exp(dt_t a) on real rows and exp(dt_t a_j) R(dt_t theta_j) on pair
 *    j, R(phi) = [[cos, -sin], [sin, cos]], a = -exp(A_log);
 *  - two-endpoint (exponential-trapezoidal) write, sungsoo.github.io Part 05:
 *        H_t = A_t (H_{t-1} + beta_t W_{t-1}) + gamma_t W_t,   W_t = B_t u_t,
 *        gamma_t = lam_t dt_t,  beta_t = (1 - lam_t) dt_t
 *    (two_endpoint = 0 means lam = 1: the Euler write of Mamba-1/2);
 *  - SSD-MIMO routing (sungsoo.github.io Part 03 "SISO and MIMO"): u_t is
 *    R x P, B_t is N x R, C_t is O x N; D is used only when O == R.
 *  Mamba-1, Mamba-2 and Mamba-3-SISO configurations are special cases.
 *
 * Memory: the caller owns every buffer.  The library allocates no device or
 * host memory and launches only on the caller's stream.  All pointers are
 * device pointers unless stated otherwise.
 *
 * Errors: every entry point returns SSM_OK (0) or a negative SSM_ERR_* code
 * and never aborts; ssm_scan_last_error() gives a message for the calling
 * thread.  Launches are asynchronous: a fault inside a kernel surfaces as
 * SSM_ERR_CUDA from a later call or from the caller's own synchronisation.
 */
#ifndef SSM_SCAN_H
#define SSM_SCAN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SSM_SCAN_ABI_VERSION 3

#if defined(__GNUC__)
#define SSM_API __attribute__((visibility("default")))
#else
#define SSM_API
#endif

enum ssm_status {
    SSM_OK = 0,
    SSM_ERR_ARG = -1,         /* bad descriptor, null required pointer, size mismatch */
    SSM_ERR_UNSUPPORTED = -2, /* valid problem outside what the kernels implement */
    SSM_ERR_ALIGN = -3,       /* pointer or stride alignment the kernels need is not met */
    SSM_ERR_CUDA = -4,        /* a CUDA runtime call or a kernel launch failed */
    SSM_ERR_TIMEOUT = -5,     /* a bounded device-side wait gave up (see ssm_scan_poll_device_error) */
    SSM_ERR_WORKSPACE = -6    /* workspace missing or smaller than ssm_scan_workspace_size() */
};

enum ssm_dtype { SSM_F32 = 0, SSM_BF16 = 1 };
enum ssm_decay_mode { SSM_DECAY_PER_HEAD = 0, SSM_DECAY_PER_COORD = 1 };
/* Rotation angle of pair j at step t: SSM_ANGLE_STATIC phi = dt_t theta[h][j]
 * (a fixed frequency scaled by the step), SSM_ANGLE_PER_TOKEN phi =
 * theta[b][t][h][j] (a data-dependent angle per token, the complex state of
 * Mamba-3 written as 2x2 rotations, sungsoo.github.io Part 05). */
enum ssm_angle_mode { SSM_ANGLE_STATIC = 0, SSM_ANGLE_PER_TOKEN = 1 };
/* Write of step t: SSM_DISC_EULER scales W_t = B_t u_t by dt_t (the two-endpoint
 * form when two_endpoint == 1); SSM_DISC_ZOH is the exact zero-order hold
 * ("State Space Models", robocikowo.com, glossary item 2): with the input held
 * over the step, mode m (rate lam = a, or a + i omega on a pair) receives
 * ((e^{dt lam} - 1) / lam) W_t, complex on a pair (= dt phi1(dt a + i phi),
 * phi1(z) = (e^z - 1) / z, phi the step's rotation angle). */
enum ssm_discretization { SSM_DISC_EULER = 0, SSM_DISC_ZOH = 1 };
/* SSM_PASS_FWD: a forward that keeps what ssm_scan_bwd_saved reads;
 * SSM_PASS_FWD_INFER: a forward only (smaller workspace). */
enum ssm_pass { SSM_PASS_FWD = 0, SSM_PASS_BWD = 1, SSM_PASS_FWD_INFER = 2 };

/*
 * Problem descriptor.  Tensor layouts (innermost last):
 *   x, dx      [batch][seqlen][nheads][rank_in][headdim]
 *   y, dy      [batch][seqlen][nheads][rank_out][headdim]
 *   B, dB      [batch][seqlen][ngroups][rank_in][N]     B_t[n][r] = B[b][t][g][r][n]
 *   C, dC      [batch][seqlen][ngroups][rank_out][N]    C_t[o][n] = C[b][t][g][o][n]
 *   dt, lambda, ddt, dlambda   [batch][seqlen][nheads]
 *   A_log, dA_log  fp32 [nheads][n_decay], n_decay = 1 (SSM_DECAY_PER_HEAD) or
 *                  n_real + n_pairs (SSM_DECAY_PER_COORD: real rows, then pairs)
 *   theta, dtheta  fp32 [nheads][n_pairs]   rotation frequency of each pair
 *                  (SSM_ANGLE_STATIC), or fp32 [batch][seqlen][nheads][n_pairs],
 *                  dense, the angle of each pair at each token (SSM_ANGLE_PER_TOKEN)
 *   D, dD          fp32 [nheads]
 *   h0, hT, prev_write, last_write, dh0, dprev_write  fp32 [batch][nheads][N][headdim]
 * Head h reads group g = h / (nheads / ngroups).  State rows: the n_real real
 * rows first, then pair j as rows n_real + 2j (re) and n_real + 2j + 1 (im).
 * The two innermost dimensions of x/y/B/C are dense; the three outer ones
 * (batch, time, head-or-group) use the element strides below, which also
 * apply to the matching gradient tensor.  dt/lambda use their own strides.
 * ssm_desc_set_contiguous() fills every stride for dense tensors.
 */
typedef struct ssm_desc {
    int64_t batch, seqlen, nheads, headdim, ngroups;
    int32_t n_real, n_pairs;
    int32_t rank_in, rank_out;  /* R, O; SISO is 1, 1 */
    int32_t chunk;              /* kernel choice, results equal up to rounding: 0 = library choice,
                                   1 = token-by-token recurrent kernels, other values = the
                                   chunked tensor-core kernels where supported.  A per-head
                                   decay without rotation pairs (bf16, headdim 64, 64 or 128
                                   state rows, rank_in == rank_out in {1, 2, 4}) takes the
                                   scalar-decay chain, 128 / rank_in tokens per chunk, with no
                                   range condition.  Other shapes with bf16, headdim 64,
                                   rank 1 and 64 or 128 state rows take the 64-token
                                   per-coordinate chain.  That chain folds
                                   each mode's decay into the operands around 16-token
                                   sub-block references, which needs
                                   |A| * log2(e) * (sum of dt over any 16 aligned tokens)
                                   <= 100 for the largest |A| of the head; the call checks
                                   this on the device and, where it fails, the recurrent
                                   kernels (launched behind the same device-side check)
                                   produce the result instead */
    int32_t decay_mode;         /* enum ssm_decay_mode */
    int32_t two_endpoint;       /* 0: lambda not read (lam = 1); 1: lambda used */
    int32_t dtype_io;           /* enum ssm_dtype of x, dt, B, C, lambda, y and of their gradients */
    int64_t stride_x[3], stride_y[3], stride_B[3], stride_C[3], stride_dt[3], stride_lambda[3];
    int32_t angle_mode;         /* enum ssm_angle_mode (ignored when n_pairs == 0) */
    int32_t n_static;           /* 0 <= n_static <= n_real: the first n_static real rows are
                                   static, with the transition exp(a_n) at every step whatever
                                   dt_t (HybridMamba's real static rows next to its real and
                                   complex dynamic ones, sungsoo.github.io Part 08 item 3);
                                   their write is that of every row.  n_static > 0 is taken
                                   by the token-by-token recurrent kernels */
    int32_t discretization;     /* enum ssm_discretization.  SSM_DISC_ZOH needs two_endpoint == 0
                                   and n_static == 0, and is taken by the recurrent kernels */
    int32_t reserved_;          /* must be 0 */
} ssm_desc_t;

/* Fill every stride of *d for dense tensors of the sizes already set. */
SSM_API void ssm_desc_set_contiguous(ssm_desc_t *d);

/*
 * Bytes of device workspace that ssm_scan_fwd (pass = SSM_PASS_FWD for a
 * training forward whose workspace a later ssm_scan_bwd_saved reads;
 * SSM_PASS_FWD_INFER for a forward alone, which is all ssm_scan_fwd requires)
 * or ssm_scan_bwd (pass = SSM_PASS_BWD) needs for this descriptor; 0 means
 * the workspace pointer may be NULL.  ssm_scan_fwd given at least the
 * SSM_PASS_FWD size also writes the per-chunk products the backward reuses.  Returns 0 for an invalid descriptor (the
 * compute call then reports the error).  The workspace must be 256-byte
 * aligned; its contents need not be initialised and are clobbered.
 * The SSM_PASS_BWD size is that of the kernels the call takes when every
 * tensor base is 16-byte aligned (as allocators return them).  A backward
 * whose tensors are not falls back to the recurrent kernels, which can need
 * more: it then fails with SSM_ERR_WORKSPACE, and the message gives the size.
 */
SSM_API size_t ssm_scan_workspace_size(const ssm_desc_t *d, int pass);

/*
 * Forward scan.  Reads x, dt, A_log, theta (may be NULL when n_pairs == 0),
 * B, C, D (may be NULL when rank_in != rank_out), lambda (ignored when
 * two_endpoint == 0), h0 and prev_write (NULL = zero initial state and zero
 * left endpoint).  Writes y and, when non-NULL, hT = H_{L-1} and
 * last_write = W_{L-1} = B_{L-1} u_{L-1}; passing (hT, last_write) as
 * (h0, prev_write) of the next call continues the sequence exactly.  y may be
 * NULL (a state-only forward: hT / last_write only; the per-coordinate
 * tensor-core chain then builds every chunk's state at once and needs the
 * SSM_PASS_FWD workspace size).
 * stream is a cudaStream_t (NULL = legacy default stream).
 */
SSM_API int ssm_scan_fwd(const ssm_desc_t *d, const void *x, const void *dt, const float *A_log,
                 const float *theta, const void *B, const void *C, const float *D,
                 const void *lambda, const float *h0, const float *prev_write, void *y,
                 float *hT, float *last_write, void *workspace, size_t workspace_bytes,
                 void *stream);

/*
 * Forward scan followed by the mixer's output gate (the pages' fused kernel
 * merges the state update with the gating and output projection of the mixer:
 * "Diagonal Equivalence in State Space Models", kongchang.com, the
 * kernel-performance paragraph; the gate's form is read as Mamba's):
 *     y_gated = y * silu(z),   silu(z) = z / (1 + e^{-z}),
 * with z in y's layout and strides (dtype_io).  Inputs and hT / last_write as
 * ssm_scan_fwd; y_pre (may be NULL) receives the pre-gate y, which
 * ssm_gate_bwd needs.  The scan writes y to y_gated and one elementwise pass
 * gates it in place right after, while y is still in L2 (inside the
 * instruction-bound tensor-core epilogue the gate was measured slower).  Same
 * workspace as ssm_scan_fwd.
 */
SSM_API int ssm_scan_fwd_gated(const ssm_desc_t *d, const void *x, const void *dt,
                               const float *A_log, const float *theta, const void *B,
                               const void *C, const float *D, const void *lambda,
                               const float *h0, const float *prev_write, const void *z,
                               void *y_gated, void *y_pre, float *hT, float *last_write,
                               void *workspace, size_t workspace_bytes, void *stream);

/*
 * Gradient through the output gate, for the upstream gradient dy_gated of
 * y_gated: dy = dy_gated * silu(z) (the dy of ssm_scan_bwd) and
 * dz = dy_gated * y_pre * sigmoid(z) (1 + z (1 - sigmoid(z))); all in y's
 * layout and dtype_io.  dy may alias dy_gated.
 */
SSM_API int ssm_gate_bwd(const ssm_desc_t *d, const void *z, const void *y_pre,
                         const void *dy_gated, void *dy, void *dz, void *stream);

/*
 * Backward scan: gradients of sum(dy * y) with respect to every input of
 * ssm_scan_fwd, recomputing the forward states (nothing is saved between the
 * calls).  Inputs as for ssm_scan_fwd plus dy.  Outputs dx, ddt, dB, dC (in
 * dtype_io), dA_log, dD (fp32), dtheta (fp32; may be NULL when n_pairs == 0),
 * dlambda (dtype_io; may be NULL, and is not written when two_endpoint == 0),
 * dh0 and dprev_write (fp32; may be NULL).  Gradients are written, not
 * accumulated; group-shared dB/dC sum the heads of their group, and the
 * per-head parameter gradients sum the batch, in a fixed order (deterministic).
 */
SSM_API int ssm_scan_bwd(const ssm_desc_t *d, const void *x, const void *dt, const float *A_log,
                 const float *theta, const void *B, const void *C, const float *D,
                 const void *lambda, const float *h0, const float *prev_write, const void *dy,
                 void *dx, void *ddt, float *dA_log, float *dtheta, void *dB, void *dC,
                 float *dD, void *dlambda, float *dh0, float *dprev_write, void *workspace,
                 size_t workspace_bytes, void *stream);

/*
 * Backward that reuses the forward's chunk states: identical to ssm_scan_bwd,
 * except that fwd_workspace is the workspace of a preceding ssm_scan_fwd call
 * with the same descriptor and the same inputs (x, dt, A_log, theta, B, C, D,
 * lambda, h0, prev_write; dy may differ), left unchanged since.  The tensor-core backward then reads
 * the states entering every 64-token chunk from it instead of recomputing them
 * (the training step "forward saving chunk states, then backward").  For
 * descriptors whose forward needs no workspace it behaves as ssm_scan_bwd.
 * Reading a workspace from other inputs gives wrong gradients; nothing checks
 * it.  fwd_workspace must not be NULL and must hold
 * ssm_scan_workspace_size(d, SSM_PASS_FWD) bytes (a training forward),
 * 256-byte aligned.
 */
SSM_API int ssm_scan_bwd_saved(const ssm_desc_t *d, const void *x, const void *dt,
                               const float *A_log, const float *theta, const void *B,
                               const void *C, const float *D, const void *lambda,
                               const float *h0, const float *prev_write, const void *dy, void *dx,
                               void *ddt, float *dA_log, float *dtheta, void *dB, void *dC,
                               float *dD, void *dlambda, float *dh0, float *dprev_write,
                               const void *fwd_workspace, size_t fwd_workspace_bytes,
                               void *workspace, size_t workspace_bytes, void *stream);

/*
 * Allocation-free backward (no counterpart in the paper; a library service).
 * Same inputs, outputs and results as ssm_scan_bwd, but it takes no
 * workspace: its scratch is a fixed 32 MiB array inside the library
 * (SSM_NOALLOC_SCRATCH_BYTES), which every GPU that loads the library keeps
 * until the process exits.  It is meant for callers that cannot or must not
 * call cudaMalloc themselves -- for example code running inside a host
 * framework that owns all device memory through its own pool, or a
 * latency-critical path where allocating (and the synchronisation a later
 * cudaFree brings) is not allowed.  The call itself allocates nothing.
 *
 *  - Problems whose backward workspace (ssm_scan_workspace_size with
 *    SSM_PASS_BWD) exceeds SSM_NOALLOC_SCRATCH_BYTES are rejected with
 *    SSM_ERR_WORKSPACE before any launch.
 *  - The first call on a device looks up the array's device address with
 *    that device current (a one-time set-up per device); make that first
 *    call before any stream capture.
 *  - All calls on a device share the one array and it keeps the last call's
 *    contents.  Nothing in it has to start at zero (every scratch byte the
 *    backward reads is written earlier in the same call), but calls whose
 *    kernels overlap on the GPU (different streams, or several host threads)
 *    race on it: serialise them.
 */
#define SSM_NOALLOC_SCRATCH_BYTES (32u << 20)
SSM_API int ssm_scan_bwd_noalloc(const ssm_desc_t *d, const void *x, const void *dt,
                                 const float *A_log, const float *theta, const void *B,
                                 const void *C, const float *D, const void *lambda,
                                 const float *h0, const float *prev_write, const void *dy,
                                 void *dx, void *ddt, float *dA_log, float *dtheta, void *dB,
                                 void *dC, float *dD, void *dlambda, float *dh0,
                                 float *dprev_write, void *stream);

/*
 * One recurrent step (autoregressive decoding): the recurrence of
 * ssm_scan_fwd for a single token, with the state kept by the caller
 * ("State Space Models", robocikowo.com: glossary item 2, the discretised
 * recurrence, and the complexity entry, constant memory per token in
 * autoregressive inference).  For every (batch row, head):
 *     h <- A_t (h + beta_t w) + gamma_t W_t,   W_t = B_t u_t,   w <- W_t
 *     y_t = C_t h + D u_t
 * With SSM_ANGLE_PER_TOKEN, theta is the token's angles, fp32
 * [batch][nheads][n_pairs].
 * h and w are fp32 [batch][nheads][N][headdim], read and overwritten in
 * place: h holds H_{t-1} on entry and H_t on return; w holds the previous
 * write W_{t-1} on entry and W_t on return.  w may be NULL when
 * two_endpoint == 0 (then nothing is read from or written to it).
 * The token's x, dt, B, C, lambda and y use the layouts and strides of
 * ssm_scan_fwd with time index 0; d->seqlen must be 1.  Starting from
 * h = h0, w = prev_write and calling this once per token gives the y, hT and
 * last_write of ssm_scan_fwd over the sequence up to rounding.  rank_in and
 * rank_out up to 8.  No workspace; errors as ssm_scan_fwd.
 */
SSM_API int ssm_scan_step(const ssm_desc_t *d, const void *x, const void *dt, const float *A_log,
                          const float *theta, const void *B, const void *C, const float *D,
                          const void *lambda, float *h, float *w, void *y, void *stream);

/*
 * Pre-activations of the scan's step size and two-endpoint weight (the
 * positivity maps in front of ssm_scan_fwd; the pages give the log-uniform
 * initialisation of the step, "State Space Models", robocikowo.com; the maps
 * themselves are the reading the workloads use):
 *     dt[b][t][h] = softplus(z[b][t][h] + dt_bias[h])
 *     lambda[b][t][h] = sigmoid(lambda_logit[b][t][h])   (two_endpoint == 1)
 * z and dt use d's dt layout and strides, lambda_logit and lambda its lambda
 * layout; all in dtype_io, dt_bias fp32 [nheads].  lambda_logit / lambda may
 * be NULL when two_endpoint == 0.  The outputs may alias the inputs.
 * seqlen may be anything (one elementwise pass).
 */
SSM_API int ssm_preact_fwd(const ssm_desc_t *d, const void *z, const float *dt_bias,
                           const void *lambda_logit, void *dt, void *lambda, void *stream);

/*
 * Gradients through the pre-activations, from ddt and dlambda (as written by
 * ssm_scan_bwd):  dz = ddt * sigmoid(z + dt_bias),
 * ddt_bias[h] = sum over (b, t) of the dz returned (in dtype_io; fp32 sum, written, fixed
 * summation order),
 * dlambda_logit = dlambda * lambda (1 - lambda).  dz may alias ddt and
 * dlambda_logit may alias dlambda; ddt_bias may be NULL; the lambda pointers
 * may be NULL when two_endpoint == 0.
 */
SSM_API int ssm_preact_bwd(const ssm_desc_t *d, const void *z, const float *dt_bias,
                           const void *lambda_logit, const void *ddt, const void *dlambda,
                           void *dz, float *ddt_bias, void *dlambda_logit, void *stream);

/*
 * Sequence sharding (context parallelism).  A sequence split into nseg
 * consecutive segments (one per rank, or processed one after another) is
 * scanned exactly by scanning every segment and exchanging per-segment
 * boundary values.  The recurrence is linear in its state (sungsoo.github.io,
 * Part 03: the chunked form composes the state carried between chunks the same
 * way), so with Phi_k the product of segment k's transitions and beta_0(k) the
 * left-endpoint weight of its first token:
 *     forward:  K_in(0) = h0, W_in(0) = prev_write,
 *               K_in(k+1) = Phi_k (K_in(k) + beta_0(k) W_in(k)) + hT_loc(k),
 *               W_in(k+1) = last write of segment k,
 *     where hT_loc(k) is segment k's end state scanned from zero (h0 = 0,
 *     prev_write = 0); scanning segment k again from (K_in(k), W_in(k)) gives
 *     its exact y and hT.
 *     backward: dK_end(nseg-1) = dhT (NULL = 0),
 *               dK_end(k) = dh0_loc(k+1) + Phi_{k+1}^T dK_end(k+1),
 *               dW_end(k) = beta_0(k+1) dK_end(k)   (0 for the last segment),
 *     where dh0_loc(k+1) is the dh0 of segment k+1's backward with no end
 *     adjoint; segment k's backward with end adjoint dK_end(k) gives its exact
 *     gradients once dW_end(k) is added to its last token's write
 *     (ssm_cp_write_adjoint), and the per-head parameter gradients are the sums
 *     over segments.
 * The end adjoint enters a segment's backward through ssm_cp_tail_rows(d)
 * trailing rows of its buffers (ssm_cp_fill_tail): the backward runs over
 * seqlen + tail rows with the same strides.  Every call below takes the
 * segment's own descriptor (seqlen = the segment's length, strides of its
 * buffers).  Layouts: states [B][H][N][P] fp32; phi [B][H][n_real + n_pairs][2]
 * fp32 (re, im; im = 0 on a real row); beta0 [B][H] fp32; a gathered array
 * ("_all") stacks nseg of them, segment k at index k.
 */

/* Trailing rows ssm_cp_fill_tail writes: N (fp32 I/O) or 2 N (bf16: the end
 * adjoint as bf16 value + remainder).  -1 for a bad descriptor. */
SSM_API int ssm_cp_tail_rows(const ssm_desc_t *d);

/* phi and beta0 of the segment described by d (its dt, lambda, theta: the
 * same inputs as ssm_scan_fwd).  n_pairs up to 64. */
SSM_API int ssm_cp_segment_transition(const ssm_desc_t *d, const void *dt, const float *A_log,
                                      const float *theta, const void *lambda, float *phi,
                                      float *beta0, void *stream);

/* K_in(seg) -> h_in and W_in(seg) -> w_in from the gathered hT_loc / last
 * writes / phi / beta0 of the segments before seg, starting from h0 /
 * prev_write (NULL = zero).  The gathered arrays are not read when seg == 0. */
SSM_API int ssm_cp_state_combine(const ssm_desc_t *d, int nseg, int seg, const float *hT_all,
                                 const float *wT_all, const float *phi_all,
                                 const float *beta0_all, const float *h0, const float *w0,
                                 float *h_in, float *w_in, void *stream);

/* dK_end(seg) -> dh_end and dW_end(seg) -> dw_end from the gathered dh0_loc /
 * phi / beta0 of the segments after seg and the adjoint dhT of the whole
 * sequence's final state (NULL = zero).  The gathered arrays are not read when
 * seg == nseg - 1. */
SSM_API int ssm_cp_adjoint_combine(const ssm_desc_t *d, int nseg, int seg, const float *dh0_all,
                                   const float *phi_all, const float *beta0_all,
                                   const float *dhT, float *dh_end, float *dw_end, void *stream);

/* Writes the trailing rows t = seqlen .. seqlen + tail - 1 of the segment's
 * x, dt, B, C, lambda (two_endpoint) and dy buffers (which must hold them at
 * the descriptor's strides): dt, x and B zero, lambda 1, so the state passes
 * through unchanged; C row 0 of trailing token s N + k is the unit vector e_k
 * and its dy row 0 carries part s of dh_end[:, k, :] (NULL = zero).  A
 * backward over seqlen + tail tokens then has dh_end as the adjoint of the
 * segment's end state, and the trailing rows add nothing to the parameter
 * gradients (they are weighted by dt or x).  A forward over the seqlen + tail
 * rows after this call gives the segment's own y and hT unchanged (its last
 * write is the trailing rows' zero write; the segment's own is that of its
 * local forward), and since calls with another dh_end change only dy, the
 * backwards may read that forward's workspace (ssm_scan_bwd_saved).  With x,
 * dt, B, C and lambda all NULL only the dy rows are written (the other rows as
 * an earlier call left them).  Not for per-token angles or static rows
 * (SSM_ERR_UNSUPPORTED). */
SSM_API int ssm_cp_fill_tail(const ssm_desc_t *d, void *x, void *dt, void *B, void *C,
                             void *lambda, void *dy, const float *dh_end, void *stream);

/* Adds dw_end, the adjoint of the segment's last write W_{L-1} = B_{L-1} u_{L-1},
 * to dx and dB of its last token (dx += B^T dw_end per head, dB += the group's
 * sum of dw_end u^T); dx / dB as written by ssm_scan_bwd. */
SSM_API int ssm_cp_write_adjoint(const ssm_desc_t *d, const void *x, const void *B,
                                 const float *dw_end, void *dx, void *dB, void *stream);

/* Message describing the last failing call on this host thread ("" if none). */
SSM_API const char *ssm_scan_last_error(void);

/*
 * Synchronise `stream` and report device-side errors raised by bounded waits
 * inside the kernels since the previous poll (SSM_ERR_TIMEOUT), or a sticky
 * CUDA error (SSM_ERR_CUDA).  Clears the device error word.
 */
SSM_API int ssm_scan_poll_device_error(void *stream);

/*
 * Per-kernel device timing (used by the benchmark).  ssm_scan_profile_start
 * opens a session on the calling host thread and creates up to
 * `max_launches` + 64 CUDA events up front; until ssm_scan_profile_stop, every
 * kernel that ssm_scan_fwd / ssm_scan_bwd launch is bracketed by events
 * recorded on the caller's stream (launches past the capacity are not timed).
 * ssm_scan_profile_stop waits for the events, writes one entry per distinct
 * kernel in first-launch order -- its name (NUL-terminated, truncated to
 * name_len bytes, into names + i * name_len), launch count and summed device
 * milliseconds -- destroys the events and returns the number of entries
 * (at most max_kernels) or a negative status.
 */
SSM_API int ssm_scan_profile_start(int max_launches);
SSM_API int ssm_scan_profile_stop(char *names, int name_len, int *counts, double *total_ms,
                                  int max_kernels);

/*
 * Failure-path diagnostic (the pages have no counterpart).  The chained
 * tensor-core kernels wait, on the device, for the chunk before (forward) or
 * after (backward) to publish its carry; each such wait polls at most this
 * many times (default 2^22, about half a second) before it gives up.  A wait
 * that gives up stops every kernel of that call early (its outputs are then
 * undefined), and the next ssm_scan_poll_device_error reports SSM_ERR_TIMEOUT;
 * later calls are unaffected.  0 makes every such wait give up at once: tests
 * use it to exercise the timeout path without a fault.  Applies to calls made
 * after it returns (the value is read when a call is issued).  Returns the
 * previous limit, or SSM_ERR_ARG for a negative value.
 */
SSM_API int64_t ssm_scan_set_wait_limit(int64_t polls);

/* SSM_SCAN_ABI_VERSION of the loaded library. */
SSM_API int ssm_scan_abi_version(void);

/*
 * Which kernels produced the result of the last ssm_scan_fwd / ssm_scan_bwd
 * call made on the calling host thread: synchronises `stream` (the stream of
 * that call) and returns SSM_ROUTE_CHUNKED (tensor-core chain),
 * SSM_ROUTE_RANGE_FALLBACK (chunk-eligible call whose inputs failed the
 * device-side range check, taken by the recurrent kernels),
 * SSM_ROUTE_RECURRENT (recurrent kernels chosen on the host: chunk = 1 or a
 * shape the chunked kernels do not take), SSM_ROUTE_SSD (per-head decay,
 * bf16, head dim 64, 64 or 128 state rows, no rotation pairs, rank_in ==
 * rank_out in {1, 2, 4}), SSM_ROUTE_CHANNEL (the Mamba-1 channel scan), or a
 * negative status (no call yet,
 * or the gate word cannot be read).  A diagnostic for tests and tuning; the
 * pages have no counterpart.
 */
enum ssm_route {
    SSM_ROUTE_CHUNKED = 0,
    SSM_ROUTE_RANGE_FALLBACK = 1,
    SSM_ROUTE_RECURRENT = 2,
    SSM_ROUTE_SSD = 3,  /* tensor-core chain of a per-head (scalar) decay: masked linear
                           attention with an exact segment-sum mask, 128 / R tokens per chunk */
    SSM_ROUTE_CHANNEL = 4 /* channel scan: head dim 1 (Mamba-1 channels), 8 or 16 real state
                             rows, groups of a multiple of 64 channels, bf16 */
};
SSM_API int ssm_scan_last_route(void *stream);

#ifdef __cplusplus
}
#endif
#endif /* SSM_SCAN_H */
