/*
 * mambascan.h -- C ABI of the B200 (sm_100a) selective-scan (S6) library.
 *
 * Two operations of the Mamba selective state-space layer:
 *
 *  mamba_scan_fwd      the fused selective scan over a whole sequence
 *  mamba_state_update  the single-token state update used for decoding
 *
 * and, beside them, the convolution prologue, the trapezoidal (Mamba-3) rule,
 * the backward pass and the Mamba-2 chunked SSD forward (mamba_ssd_fwd,
 * documented with its own arguments further down). The first two compute,
 * per channel row (b, d) and state index n < dstate,
 *
 *   delta   = delta_raw + delta_bias[d]            (bias, if given, added first)
 *   delta   = log(1 + exp(delta))                  if delta_softplus (identity above 20)
 *   h[n]    = exp(delta * A[d,n]) * h[n] + delta * B[n] * x      (first-order Bbar)
 *   y       = sum_n C[n] * h[n] + D[d] * x                        (after the update)
 *   y       = y * z * sigmoid(z)                                  if z is given
 *
 * as defined on the pages this library follows:
 *  - "Notas sobre Mamba", section "O mecanismo de seleção (S6)": input
 *    dependent B_t, C_t and delta_t = softplus(Linear(x_t) + bias); diagonal
 *    A = -exp(A_log); h_t = Abar_t h_{t-1} + Bbar_t x_t, y_t = C_t^T h_t;
 *    Abar = exp(delta A), Bbar = delta B.
 *  - "Notas sobre Mamba", section "Preliminares": the implementation uses the
 *    first-order Bbar_t = delta_t B_t rather than the full ZOH expression.
 *  - "Notas sobre Mamba", section "A varredura paralela ciente do hardware":
 *    the recurrence is an associative scan over the pairs (Abar_t, Bbar_t x_t);
 *    discretised parameters and the N-dimensional state stay on chip and only
 *    the output is written back.
 *  - "Mamba-2 e State Space Duality (SSD)", section "Como o Mamba-1 alcançou
 *    complexidade linear": y_t = C_t h_t + D x_t and the decode step.
 *  - "Notas sobre Mamba", section "O bloco Mamba": the S6 output is gated by
 *    SiLU of the second branch z.
 *
 * Conventions shared by every entry point:
 *  - All tensor pointers are DEVICE pointers, allocated and owned by the
 *    caller. The library allocates nothing and keeps no state between calls
 *    beyond a per-device cache of device properties (and the fixed scratch
 *    array of mamba_scan_fwd_noalloc, below).
 *  - Strides are in ELEMENTS of the tensor's own type. The innermost axis
 *    (L for the scan, dstate for states, dim for decode vectors) must be
 *    contiguous (stride 1).
 *  - `in_dtype` (ms_dtype) is the type of u/x, delta, B, C, z and y. A, D,
 *    delta_bias and all states are float32. Arithmetic is float32.
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and nothing synchronises. A status other than MS_OK means that
 *    nothing was launched, except MS_ERR_CUDA, which reports a launch error
 *    (kernels already queued by the same call may have run). Faults that
 *    happen while a kernel runs surface at the caller's next synchronisation.
 *  - Outputs must not alias inputs (the decode state is updated in place and
 *    is the one in/out argument).
 *  - Calls are thread safe; concurrent calls on different streams must not
 *    share output or workspace buffers.
 */
#ifndef MAMBASCAN_H
#define MAMBASCAN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MAMBASCAN_ABI_VERSION 2
/* Largest state size N supported by the kernels. */
#define MS_MAX_DSTATE 16

typedef enum ms_status {
    MS_OK = 0,
    MS_ERR_INVALID_ARG = 1,  /* null pointer, non-positive size, bad stride, bad enum   */
    MS_ERR_UNSUPPORTED = 2,  /* valid but outside what the kernels support (dstate>16)   */
    MS_ERR_ALIGNMENT = 3,    /* a pointer is not aligned to its element size             */
    MS_ERR_CUDA = 4,         /* a CUDA runtime call or kernel launch failed              */
    MS_ERR_TIMEOUT = 5,      /* a bounded device wait gave up (reported in a status word)  */
    MS_ERR_WORKSPACE = 6     /* workspace missing or smaller than the size asked for      */
} ms_status;

typedef enum ms_dtype {
    MS_F32 = 0,
    MS_BF16 = 1
} ms_dtype;

/*
 * Arguments of the selective scan forward.
 *
 *   u, delta, z, y : (batch, dim, seqlen), L contiguous, strides
 *                    (*_batch_stride, *_dim_stride). z may be NULL (no gate).
 *   B, C           : (batch, dstate, seqlen), L contiguous, strides
 *                    (*_batch_stride, *_state_stride); shared by every channel d.
 *   A              : (dim, dstate) float32, contiguous. Usually -exp(A_log).
 *   D, delta_bias  : (dim) float32, or NULL for zero.
 *   initial_state  : (batch, dim, dstate) float32 contiguous, or NULL for zero.
 *   final_state    : (batch, dim, dstate) float32 contiguous, or NULL (not written).
 *   force_segments : 0 = automatic. >0 splits the sequence of every row into
 *                    that many segments joined by the multi-block carry pass
 *                    (the count is capped at the number of 16-step blocks).
 */
typedef struct ms_scan_args {
    int64_t batch, dim, dstate, seqlen;
    int32_t in_dtype;
    int32_t delta_softplus;

    const void *u;      int64_t u_batch_stride, u_dim_stride;
    const void *delta;  int64_t delta_batch_stride, delta_dim_stride;
    const void *B;      int64_t B_batch_stride, B_state_stride;
    const void *C;      int64_t C_batch_stride, C_state_stride;
    const void *z;      int64_t z_batch_stride, z_dim_stride;
    void *y;            int64_t y_batch_stride, y_dim_stride;

    const float *A;
    const float *D;
    const float *delta_bias;
    const float *initial_state;
    float *final_state;

    int32_t force_segments;
    int32_t reserved;   /* must be 0 */
} ms_scan_args;

/*
 * Arguments of the single-token state update (decode).
 *
 *   state          : (batch, dim, dstate) float32, dstate contiguous, strides
 *                    (state_batch_stride, state_dim_stride). Updated IN PLACE.
 *   x, delta, z, y : (batch, dim), dim contiguous, batch stride *_batch_stride.
 *                    z may be NULL.
 *   B, C           : (batch, dstate), dstate contiguous, batch stride *_batch_stride.
 *   A              : (dim, dstate) float32 contiguous; D, delta_bias: (dim) or NULL.
 */
typedef struct ms_update_args {
    int64_t batch, dim, dstate;
    int32_t in_dtype;
    int32_t delta_softplus;

    float *state;       int64_t state_batch_stride, state_dim_stride;
    const void *x;      int64_t x_batch_stride;
    const void *delta;  int64_t delta_batch_stride;
    const void *B;      int64_t B_batch_stride;
    const void *C;      int64_t C_batch_stride;
    const void *z;      int64_t z_batch_stride;
    void *y;            int64_t y_batch_stride;

    const float *A;
    const float *D;
    const float *delta_bias;
} ms_update_args;

/* Human-readable name of a status code (static string, never NULL). */
const char *mamba_status_string(int status);

/* Message of the last MS_ERR_CUDA / MS_ERR_INVALID_ARG on this thread (static
 * thread-local buffer, never NULL, "" if none). */
const char *mamba_last_error(void);

/* MAMBASCAN_ABI_VERSION of the loaded library. */
int mamba_abi_version(void);

/*
 * Bytes of device workspace that mamba_scan_fwd needs for these arguments
 * (written to *bytes; 0 when the plan neither splits the sequence into
 * segments nor uses the persistent schedule described at
 * mamba_scan_fwd_with_plan).
 * Validates the arguments like mamba_scan_fwd, without touching the device
 * memory they point to. The caller allocates the workspace (256-byte aligned)
 * and may reuse it across calls on one stream.
 */
ms_status mamba_scan_workspace_size(const ms_scan_args *args, size_t *bytes);

/*
 * Selective scan forward: y for every (b, d, t) and, if requested, the state
 * after the last step. The expanded (batch, dim, seqlen, dstate) state is
 * never written to memory. `workspace` may be NULL when the size query gave 0.
 * Errors: MS_ERR_INVALID_ARG, MS_ERR_UNSUPPORTED (dstate > 16),
 * MS_ERR_ALIGNMENT (a pointer not aligned to its element type),
 * MS_ERR_WORKSPACE, MS_ERR_CUDA.
 */
ms_status mamba_scan_fwd(const ms_scan_args *args, void *workspace, size_t workspace_bytes,
                         void *stream);

/*
 * Single-token selective state update: state <- exp(delta A) state + delta B x
 * in place, then y = C . state + D x (times silu(z)). One launch; no workspace.
 * Errors: as mamba_scan_fwd, without MS_ERR_WORKSPACE.
 */
ms_status mamba_state_update(const ms_update_args *args, void *stream);

/*
 * Launch plan of a scan: which compiled kernel configuration runs it and how
 * the work is cut. mamba_scan_plan_query returns the plan mamba_scan_fwd
 * would use; mamba_scan_fwd_with_plan runs a caller-chosen plan (for tuning
 * and for testing every configuration). Fields marked "out" are filled by the
 * library and ignored on input.
 */
typedef struct ms_scan_plan {
    int32_t config;          /* index of the kernel configuration, 0 .. mamba_scan_num_configs()-1 */
    int32_t warps_per_cta;   /* chunked: 2 .. max_warps; sequential: exactly max_warps (4)         */
    int32_t segments;        /* pieces the sequence of every row is cut into (>= 1)               */
    int32_t lanes;           /* out: chunked: lanes per row pair; sequential: lanes per row        */
    int64_t segment_len;     /* out: time steps per segment                                      */
    uint64_t workspace_bytes;/* out: workspace the plan needs                                    */
    int32_t ctas;            /* sequential kernels: 0 = one CTA per unit of rows (batch entry x
                                block of rows); > 0 = persistent schedule over this many CTAs
                                (below); chunked kernels: 0                                      */
    int32_t reserved;        /* must be 0                                                        */
} ms_scan_plan;

/* Number of compiled scan kernel configurations. */
int mamba_scan_num_configs(void);

/*
 * Properties of configuration `config`.
 *  - Chunked kernels (kind 0): lanes per row pair, state indices per pass
 *    (0 = the fully unrolled pipelined kernel, dstate 16 only; 1; 2) and the
 *    largest CTA in warps (plans take 2 .. max_warps warps and any number of
 *    segments).
 *  - Sequential kernels (kind 1): lanes per row, states per lane (16 / lanes)
 *    and the fixed CTA size in warps (4); plans take exactly that many warps
 *    and one segment, and need no workspace unless they ask for the
 *    persistent schedule (ctas > 0).
 * Returns MS_ERR_INVALID_ARG for an unknown index.
 */
ms_status mamba_scan_config_info(int config, int *lanes, int *states_per_pass, int *max_warps);

/*
 * Kind of configuration `config` (written to *kind): 0 = chunked kernel (each
 * row's time axis is split across lanes and joined by a scan), 1 = sequential
 * kernel (each lane runs the recurrence step by step for some of a row's
 * states). Returns MS_ERR_INVALID_ARG for an unknown index or NULL kind.
 */
ms_status mamba_scan_config_kind(int config, int *kind);

/* The plan mamba_scan_fwd would run for these arguments (validates like it). */
ms_status mamba_scan_plan_query(const ms_scan_args *args, ms_scan_plan *plan);

/* Bytes of workspace (*bytes) that mamba_scan_fwd_with_plan needs to run
 * `plan` on these arguments; MS_ERR_UNSUPPORTED if the plan cannot run them. */
ms_status mamba_scan_plan_workspace_size(const ms_scan_args *args, const ms_scan_plan *plan, size_t *bytes);

/*
 * mamba_scan_fwd with the launch plan fixed by the caller. The plan is
 * checked (index, CTA size, shared memory, segments <= number of chunks, and
 * that the configuration can run these arguments: the pipelined kernels need
 * dstate 16, and kernels with more than one state per pass need 16-byte
 * aligned rows); an unusable plan returns MS_ERR_UNSUPPORTED and launches
 * nothing. Same results as mamba_scan_fwd up to float32 rounding order.
 *
 * Persistent schedule (sequential kernels, plan->ctas > 0). The rows are cut
 * into units (one batch entry x the CTA's block of rows) and every unit's
 * sequence into chunks of 16 steps; the chunks of all units, unit after
 * unit, are divided into plan->ctas equal ranges, one per CTA, so every SM
 * does the same share of the recurrence whatever the number of rows. A unit
 * whose chunks fall into two ranges is started by one CTA, which leaves its
 * state in the workspace, and continued by the next CTA from that state (the
 * recurrence itself is unchanged: no step is computed twice). plan->ctas may
 * not exceed the number of units nor the CTAs the device can hold at once;
 * the launch is cooperative, so all of them run concurrently. The workspace
 * (mamba_scan_plan_workspace_size) starts with a status word, an int32 that
 * the call clears and the kernel sets to MS_ERR_TIMEOUT if a CTA gave up
 * waiting (about 4 s) for the state it continues from (the outputs are then
 * wrong); flags and states follow. The automatic plan uses this schedule when
 * it balances the SMs better than one CTA per unit.
 */
ms_status mamba_scan_fwd_with_plan(const ms_scan_args *args, const ms_scan_plan *plan, void *workspace,
                                   size_t workspace_bytes, void *stream);

/* ---- Convolution prologue ------------------------------------------------
 * The Mamba block ("Notas sobre Mamba", section "O bloco Mamba", block
 * diagram) puts a short depthwise convolution and a SiLU on the x branch
 * before the selective SSM; "Mamba-2 e State Space Duality (SSD)" configures
 * its width as d_conv = 4. The pages print no formula; the library computes
 * the causal depthwise convolution, one filter per channel d, with zero input
 * before t = 0:
 *     u[b,d,t] = act( bias[d] + sum_{k<width} weight[d,k] * x[b,d,t-width+1+k] )
 * with act = SiLU (or the identity), weight[d,width-1] on the current input,
 * and u is the SSM input of the scan (its D u skip term included). */
#define MS_MAX_CONV_WIDTH 4

typedef struct ms_conv1d_args {
    const float *weight;   /* (dim, width) float32, contiguous, required                  */
    const float *bias;     /* (dim) float32, or NULL (no bias)                            */
    int32_t width;         /* taps, 1 .. MS_MAX_CONV_WIDTH                                */
    int32_t silu;          /* 1: act = SiLU; 0: act = identity                            */
} ms_conv1d_args;

/*
 * Convolution prologue fused into the selective scan: args->u holds x, the
 * convolution input ((batch, dim, seqlen), the layout and dtype of u); every
 * other argument means what it means for mamba_scan_fwd. u itself is never
 * written to memory. Runs on the sequential kernels with 2 or 4 lanes per row,
 * in one segment, with no workspace (mamba_conv_scan_fwd_ws below takes one,
 * for the persistent schedule). `plan` is NULL (automatic) or one of those
 * configurations (warps_per_cta = max_warps, segments = 1, ctas 0). The caller owns
 * every buffer; the call enqueues one kernel on `stream`.
 * Errors: as mamba_scan_fwd; MS_ERR_INVALID_ARG for a NULL conv or weight or a
 * silu flag other than 0/1, or width < 1; MS_ERR_UNSUPPORTED for width >
 * MS_MAX_CONV_WIDTH, force_segments > 1, or a plan that cannot fuse the
 * prologue; MS_ERR_ALIGNMENT for a misaligned weight or bias.
 */
ms_status mamba_conv_scan_fwd(const ms_scan_args *args, const ms_conv1d_args *conv,
                              const ms_scan_plan *plan, void *stream);

/*
 * The same with a caller-owned device workspace (256-byte aligned), which
 * lets the automatic plan (plan NULL) or the caller's plan (ctas > 0) use the
 * persistent schedule of the sequential kernels: the chunks of all rows cut
 * evenly over the SMs, a row's state handed between CTAs through the
 * workspace. mamba_conv_scan_workspace_size reports the bytes the plan the
 * call would run needs (0: none; the workspace pointer may then be NULL).
 * Errors as mamba_conv_scan_fwd, plus MS_ERR_WORKSPACE for a missing or short
 * workspace and MS_ERR_ALIGNMENT for a misaligned one; a persistent launch
 * whose carry wait runs out leaves MS_ERR_TIMEOUT in the workspace's status
 * word (see mamba_scan_fwd_with_plan).
 */
ms_status mamba_conv_scan_workspace_size(const ms_scan_args *args, const ms_conv1d_args *conv,
                                         const ms_scan_plan *plan, size_t *bytes);
ms_status mamba_conv_scan_fwd_ws(const ms_scan_args *args, const ms_conv1d_args *conv, const ms_scan_plan *plan,
                                 void *workspace, size_t workspace_bytes, void *stream);

/*
 * Decode step with the convolution prologue: args->x is the new convolution
 * input. conv_state (batch, dim, width) in the input dtype (element strides
 * conv_state_batch_stride and conv_state_dim_stride; the width axis is
 * contiguous) holds each row's last `width` inputs, oldest first; it is
 * updated in place (the oldest input dropped, x appended), then u =
 * act(bias + weight . conv_state) is the input of the state update
 * (mamba_state_update with u for x). A zero conv_state is the state of a
 * sequence that has not started, matching the scan's zero input before t = 0.
 * Errors: as mamba_state_update; MS_ERR_INVALID_ARG for a NULL conv, weight or
 * conv_state, negative strides, silu other than 0/1 or width < 1;
 * MS_ERR_UNSUPPORTED for width > MS_MAX_CONV_WIDTH; MS_ERR_ALIGNMENT for a
 * pointer not aligned to its element size.
 */
ms_status mamba_conv_state_update(const ms_update_args *args, const ms_conv1d_args *conv, void *conv_state,
                                  int64_t conv_state_batch_stride, int64_t conv_state_dim_stride,
                                  void *stream);

/*
 * Exponential-trapezoidal selective scan (Mamba-3; "Notas sobre Mamba",
 * section "Recorrência trapezoidal"):
 *     h_t = alpha_t h_{t-1} + beta_t B_{t-1} u_{t-1} + gamma_t B_t u_t,
 *     alpha_t = exp(delta_t A), beta_t = (1 - lambda_t) delta_t alpha_t,
 *     gamma_t = lambda_t delta_t,  lambda_t = sigmoid(lambda_raw_t),
 * with B_{-1} u_{-1} = 0, and the readout, skip term and gate of
 * mamba_scan_fwd. lambda_raw is (batch, dim, seqlen) in the input dtype, one
 * value per (b, d, t), contiguous along t, with element strides
 * lambda_batch_stride and lambda_dim_stride. lambda = 1 everywhere is the
 * exponential-Euler scan of mamba_scan_fwd. A nonzero initial state is the
 * state before t = 0; the previous-input term still starts at zero. Runs on the
 * sequential kernels with 2 or 4 lanes per row, in one segment, with no
 * workspace; `plan` is NULL (automatic) or one of those configurations without
 * CTAs (ctas 0).
 * Errors: as mamba_scan_fwd; MS_ERR_INVALID_ARG for a NULL lambda_raw or
 * negative strides; MS_ERR_UNSUPPORTED for force_segments > 1 or a plan that
 * cannot run the rule; MS_ERR_ALIGNMENT for a misaligned lambda_raw.
 */
ms_status mamba_trap_scan_fwd(const ms_scan_args *args, const void *lambda_raw, int64_t lambda_batch_stride,
                              int64_t lambda_dim_stride, const ms_scan_plan *plan, void *stream);

/*
 * The same with a caller-owned device workspace (256-byte aligned), which
 * lets the automatic plan (plan NULL) or the caller's plan (ctas > 0) use the
 * persistent schedule of the sequential kernels (a row's state handed between
 * CTAs through the workspace; the CTA that takes a row over reads B at the
 * step before its first one from B itself).
 * mamba_trap_scan_workspace_size reports the bytes the plan the call would run
 * needs (0: none; the workspace pointer may then be NULL). Errors as
 * mamba_trap_scan_fwd, plus MS_ERR_WORKSPACE for a missing or short workspace
 * and MS_ERR_ALIGNMENT for a misaligned one; a persistent launch whose carry
 * wait runs out leaves MS_ERR_TIMEOUT in the workspace's status word (see
 * mamba_scan_fwd_with_plan).
 */
ms_status mamba_trap_scan_workspace_size(const ms_scan_args *args, const void *lambda_raw,
                                         int64_t lambda_batch_stride, int64_t lambda_dim_stride,
                                         const ms_scan_plan *plan, size_t *bytes);
ms_status mamba_trap_scan_fwd_ws(const ms_scan_args *args, const void *lambda_raw, int64_t lambda_batch_stride,
                                 int64_t lambda_dim_stride, const ms_scan_plan *plan, void *workspace,
                                 size_t workspace_bytes, void *stream);

/* ---- Backward pass ---------------------------------------------------------
 * Gradients of the selective scan for the loss sum(y dy) + sum(h_T dh_T)
 * ("Notas sobre Mamba", section "A varredura paralela ciente do hardware":
 * the backward pass recomputes the states instead of storing them). The
 * forward's arguments come in an ms_scan_args (its y and final_state are not
 * used); the gradients come out here. Layouts: dy, du, ddelta, dz as u
 * (batch, dim, seqlen) in the input dtype, contiguous along t; ddelta is the
 * gradient w.r.t. the raw delta (through the softplus and the bias). dB and
 * dC are (batch, dstate, seqlen) float32, contiguous (summed over dim, since B
 * and C are shared across channels); dA is (dim, dstate), dD and
 * ddelta_bias (dim), summed over the batch; dinitial_state and dfinal_state
 * are (batch, dim, dstate) float32, contiguous. dA, dB, dC, dD and
 * ddelta_bias are written (zeroed by the call, then accumulated). */
typedef struct ms_scan_bwd_args {
    const void *dy;          int64_t dy_batch_stride, dy_dim_stride;            /* required */
    const float *dfinal_state;                                                /* or NULL (zero) */
    void *du;                int64_t du_batch_stride, du_dim_stride;            /* required */
    void *ddelta;            int64_t ddelta_batch_stride, ddelta_dim_stride;    /* required */
    void *dz;                int64_t dz_batch_stride, dz_dim_stride;            /* required iff z */
    float *dA;                                                                /* required */
    float *dB, *dC;                                                           /* required */
    float *dD;                                                                /* required iff D */
    float *ddelta_bias;                                                       /* required iff delta_bias */
    float *dinitial_state;                                                    /* or NULL */
} ms_scan_bwd_args;

/* Device workspace for mamba_scan_bwd (the states at every 8-step checkpoint:
 * batch * dim * ceil(seqlen / 8) * 16 floats). */
ms_status mamba_scan_bwd_workspace_size(const ms_scan_args *args, size_t *bytes);

/*
 * Backward pass: one kernel launch (after clearing the accumulated outputs)
 * on `stream`. The caller owns every buffer, the workspace included (256-byte
 * aligned). Errors: as mamba_scan_fwd for the forward arguments;
 * MS_ERR_INVALID_ARG for a NULL bwd, a missing required gradient or negative
 * strides; MS_ERR_ALIGNMENT for misaligned pointers; MS_ERR_WORKSPACE for a
 * missing or short workspace.
 */
ms_status mamba_scan_bwd(const ms_scan_args *args, const ms_scan_bwd_args *bwd, void *workspace,
                         size_t workspace_bytes, void *stream);

/*
 * Training pair with the checkpoints kept from the forward ("Notas sobre
 * Mamba", section "A varredura paralela ciente do hardware": the backward
 * recomputes the states; here it recomputes them from the forward's states at
 * every 8th step instead of sweeping the sequence a second time).
 *
 * mamba_scan_fwd_checkpointed: mamba_scan_fwd, and in addition the state after
 * every 8th step (t = 7, 15, ...) of every (batch, dim) row goes to
 * `checkpoints`: (batch * dim, ceil(seqlen / 8), 16) float32 (states past
 * dstate unspecified), caller-owned, 256-byte aligned, at least the size
 * mamba_scan_bwd_workspace_size reports (checkpoint_bytes). Only the sequential
 * kernels write them: MS_ERR_UNSUPPORTED when the plan for the arguments is a
 * chunked kernel (force_segments > 1, or very few rows). `workspace` is the
 * forward's own, as for mamba_scan_fwd. Other errors as mamba_scan_fwd, plus
 * MS_ERR_INVALID_ARG for NULL checkpoints, MS_ERR_WORKSPACE for a short
 * buffer, MS_ERR_ALIGNMENT for a misaligned one.
 *
 * mamba_scan_bwd_checkpointed: mamba_scan_bwd with the checkpoints of a
 * mamba_scan_fwd_checkpointed call on the same arguments (same u, delta, A, B,
 * C, D, z, delta_bias, initial_state and flags) in place of the workspace; it
 * only reads them. Errors as mamba_scan_bwd (MS_ERR_WORKSPACE for a short
 * buffer).
 */
ms_status mamba_scan_fwd_checkpointed(const ms_scan_args *args, float *checkpoints, size_t checkpoint_bytes,
                                      void *workspace, size_t workspace_bytes, void *stream);
ms_status mamba_scan_bwd_checkpointed(const ms_scan_args *args, const ms_scan_bwd_args *bwd,
                                      const float *checkpoints, size_t checkpoint_bytes, void *stream);

/* ---- Mamba-2 scalar-decay SSM (structured state space duality, SSD) --------
 * Per batch b and head h, sequentially in t, on a state H of 64 x 128 values
 * (headdim x dstate):
 *     delta = dt[b,t,h] + dt_bias[h];  delta = log(1 + exp(delta)) if dt_softplus
 *     H     = exp(delta A[h]) H + (delta x[b,t,h,:]) B[b,t,g,:]^T
 *     y[b,t,h,:] = H C[b,t,g,:] + D[h] x[b,t,h,:];  y *= z sigmoid(z) if z
 * with g = h / (nheads / ngroups). Sources: "Notas sobre Mamba", section "A
 * forma dual: atenção mascarada" (Abar_t = a_t I and the recurrent form of
 * its check) and section "O algoritmo SSD" (diagonal blocks by the quadratic
 * form, off-diagonal blocks by passing a state from block to block);
 * "Mamba-2 e State Space Duality (SSD)", sections "A teoria do State Space
 * Duality (SSD) no Mamba-2" (decay exp(sum delta_k a_k)) and "O algoritmo de
 * decomposição em blocos do SSD" (fixed blocks, tensor cores inside a block,
 * a recurrent scan of block states between blocks).
 *
 * Layouts (element strides; the listed inner axes are contiguous):
 *   x, z, y : (batch, seqlen, nheads, 64) bf16, head and headdim axes contiguous
 *   dt      : (batch, seqlen, nheads) bf16, head axis contiguous
 *   B, C    : (batch, seqlen, ngroups, 128) bf16, group and state axes contiguous
 *   A       : (nheads) float32, usually -exp(A_log); D, dt_bias: (nheads) or NULL
 *   initial_state, final_state : (batch, nheads, 64, 128) float32 contiguous, or NULL
 * Only bf16 inputs, headdim 64 and dstate 128 are supported. The batch and
 * token strides of x, z, y, B and C must be multiples of 8 elements and their
 * base pointers 16-byte aligned (the kernel moves them in 16-byte pieces and
 * through tensor maps); x's token stride must be at least nheads * 64 and the
 * token stride of B and C at least ngroups * 128.
 */
#define MS_SSD_HEADDIM 64
#define MS_SSD_DSTATE 128
typedef struct ms_ssd_args {
    int64_t batch, seqlen, nheads, ngroups;
    int32_t in_dtype;        /* MS_BF16 */
    int32_t dt_softplus;

    const void *x;      int64_t x_batch_stride, x_token_stride;
    const void *dt;     int64_t dt_batch_stride, dt_token_stride;
    const void *B;      int64_t B_batch_stride, B_token_stride;
    const void *C;      int64_t C_batch_stride, C_token_stride;
    const void *z;      int64_t z_batch_stride, z_token_stride;    /* z may be NULL */
    void *y;            int64_t y_batch_stride, y_token_stride;

    const float *A;
    const float *D;
    const float *dt_bias;
    const float *initial_state;
    float *final_state;

    /* Limit of each of the kernel's internal pipeline waits, in microseconds;
     * 0 = the default of about one second. */
    uint32_t wait_limit_us;
    /* Fault-injection hook for tests of the timeout path: k > 0 makes the
     * kernel withhold the loads of block k - 1 (of every (batch, head)), so
     * the wait for them runs out and the status word reports MS_ERR_TIMEOUT;
     * no load or product of that block is ever issued, so nothing is left in
     * flight. 0 = normal operation. */
    int32_t withhold_block;
} ms_ssd_args;

/* Smallest device workspace of mamba_ssd_fwd: a status word (int32 at offset
 * 0). Enough for one CTA per (batch, head); see mamba_ssd_workspace_size. */
#define MS_SSD_WORKSPACE_BYTES 256

/*
 * Workspace bytes with which mamba_ssd_fwd takes its best schedule for these
 * arguments on the current device (at least MS_SSD_WORKSPACE_BYTES). When
 * there are more (batch, head) pairs than SMs and they would leave the last
 * wave partly empty, that is the persistent schedule: one resident CTA per SM,
 * the chunks of all pairs cut evenly over them, and a pair's state handed
 * from one CTA to the next through the workspace (status word, one flag per
 * CTA, then 64 x 128 floats per CTA). Errors as mamba_ssd_fwd's argument checks;
 * MS_ERR_INVALID_ARG for a NULL bytes.
 */
ms_status mamba_ssd_workspace_size(const ms_ssd_args *args, size_t *bytes);

/*
 * SSD forward: one kernel launch on `stream` (after clearing the status word
 * and, for the persistent schedule, the flags). A CTA walks a sequence in
 * blocks of 128 tokens: one CTA per (batch, head), or, with a workspace of at
 * least mamba_ssd_workspace_size bytes that asks for it, the persistent
 * schedule (a cooperative launch). The block products run on the tensor cores
 * in bf16 with fp32 accumulation; the state passed between blocks stays in
 * fp32 (on chip, or in the workspace between two CTAs). The caller owns the
 * workspace (at least MS_SSD_WORKSPACE_BYTES, 16-byte aligned). After
 * synchronizing, its first int32 is 0 when the kernel finished normally,
 * MS_ERR_TIMEOUT when one of the kernel's internal waits (pipeline, or the
 * hand-over between CTAs) gave up after about a second (the outputs are then
 * incomplete), or MS_ERR_ALIGNMENT when the kernel's shared memory window was
 * not 1024-byte aligned (nothing was computed).
 * The tensor maps the kernel reads through are encoded on the host by the
 * driver's encoder, looked up once per process. Errors: MS_ERR_INVALID_ARG
 * for NULL or negative sizes, strides or pointers, or nheads not a multiple
 * of ngroups; MS_ERR_UNSUPPORTED for a dtype other than bf16 or a driver
 * without tensor-map support; MS_ERR_ALIGNMENT for misaligned pointers or
 * strides; MS_ERR_WORKSPACE for a missing or short workspace; MS_ERR_CUDA for
 * a failed launch.
 */
ms_status mamba_ssd_fwd(const ms_ssd_args *args, void *workspace, size_t workspace_bytes, void *stream);

/* ---- Measurement helper -----------------------------------------------------
 * Measured throughput of one arithmetic unit on the current device, the
 * denominators of the scan's roofline (the pages bound the selective scan by
 * the non-tensor units: "Mamba-2 e State Space Duality (SSD)", section "O
 * gargalo de hardware no scan associativo do Mamba-1"). unit: 0 = ex2.approx
 * (the MUFU exponential every element of the scan takes), 1 = tanh.approx
 * (MUFU), 2 = float32 FMA, 3 = packed f32x2 FMA (two results per
 * instruction). Every SM runs 32 warps of 16 independent dependency chains.
 * Writes results per second (*ops_per_s, from CUDA events around one launch
 * after a warm-up launch) and per clock per SM (*ops_per_clk_per_sm, from the
 * SM cycle counter). `scratch` is 256 bytes of caller-owned device memory,
 * 256-byte aligned (overwritten). Unlike the compute entry points this call is
 * synchronous: it returns after synchronizing `stream`. Errors:
 * MS_ERR_INVALID_ARG (unit outside 0..3, NULL scratch or outputs),
 * MS_ERR_ALIGNMENT (misaligned scratch), MS_ERR_CUDA. */
ms_status mamba_probe_unit_throughput(int unit, void *scratch, double *ops_per_s, double *ops_per_clk_per_sm,
                                      void *stream);

/* Size of the device array behind mamba_scan_fwd_noalloc (8 MiB per GPU). */
#define MS_NOALLOC_SCRATCH_BYTES (8u << 20)

/*
 * mamba_scan_fwd_noalloc -- the same selective scan forward as mamba_scan_fwd
 * for callers that cannot allocate device memory: a plugin inside a host
 * application that owns every device allocation and passes in only its
 * tensors, or a path on which cudaMalloc is off limits because it can stall
 * the whole device. (The pages this library follows have no counterpart; this
 * entry point exists for those callers.)
 *
 * The workspace that mamba_scan_fwd takes from its caller (the multi-block
 * carry, or the persistent schedule's status word, flags and handed-over
 * states) lives here in a fixed device array of MS_NOALLOC_SCRATCH_BYTES,
 * which every GPU that loads the library holds until the process exits. The
 * call allocates nothing. Inputs and outputs are the caller's, exactly as for
 * mamba_scan_fwd.
 *  - The first call on a device looks up the array's device address on that
 *    (current) device; make that first call before any stream capture.
 *  - All calls on a device share the array and it keeps the last call's
 *    contents; the call itself clears (on the stream, before its kernel) the
 *    part that must start at zero and writes every other entry before reading
 *    it, so the caller clears nothing, but calls whose kernels overlap on the
 *    GPU (unordered streams) race on it and give wrong results.
 *  - Calls that would need more scratch than the array holds (the size
 *    mamba_scan_workspace_size reports exceeds MS_NOALLOC_SCRATCH_BYTES) are
 *    rejected with MS_ERR_WORKSPACE and launch nothing.
 * Errors: as mamba_scan_fwd.
 */
ms_status mamba_scan_fwd_noalloc(const ms_scan_args *args, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* MAMBASCAN_H */
