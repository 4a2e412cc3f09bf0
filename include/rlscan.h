/*
 * rlscan.h -- C ABI of librlscan: RL credit-assignment estimators as one
 * segmented first-order linear recurrence, computed by fused CUDA kernels on
 * NVIDIA B200 (sm_100a).
 *
 * What is computed.  "rl-triton: High-Performance Triton GPU Kernels for
 * Reinforcement Learning Credit Assignment" (gist.science technical summary),
 * Methodologie 1 "Unified Algebraic Framework": every estimator below is the
 * backward recurrence A_t = alpha_t + beta_t * A_{t+1} (or its forward-time
 * mirror), solved as an associative scan over pairs with the combine
 * (alpha_B, beta_B) (+) (alpha_A, beta_A) = (alpha_B + beta_B alpha_A,
 * beta_A beta_B).  Methodologie 2 "Fused Triton Kernels": each call builds
 * its per-step coefficients on chip from the raw rollout inputs and reads and
 * writes every element of HBM once.  The pages name the seven estimators (same
 * title, arxivlens page, Abstract); the formula of each is its original
 * paper's and is stated with its entry point.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Layout.  Per-step arrays are row-major [N, T] with T contiguous (one row per
 *   environment, the pages' [num_envs, seq_len] tensors, Probleemstelling),
 *   except for the "_tm" entry points, which take them time-major [T, N].
 *   Retrace's q and pi are [N, T, A] with A contiguous.  Per-row arrays
 *   (bootstrap, init_trace) are [N].
 * Types.  Values are float32 (bfloat16 bit patterns for the "_bf16" entry
 *   points), integers and actions int32, flags uint8 with nonzero meaning true
 *   (the byte layout of torch.bool).
 * Pointers.  Every pointer is a device-accessible address (device, managed or
 *   mapped pinned host memory) on the current CUDA device.  Float and int32
 *   arrays must be 4-byte aligned.  32-byte alignment of every per-step array
 *   (8-byte for flag arrays; Retrace: 16 and 4) selects the vectorised path,
 *   anything else the scalar path with the same results.  The caller owns
 *   every buffer.
 *   Outputs must not overlap any input or each other (in-place use is refused:
 *   the kernels read neighbouring steps).
 * Episode boundaries (same page, Methodologie 3 "Expliciete Boundary
 *   Semantiek").  terminated[t] != 0: the transition out of step t ended the
 *   episode naturally, its successor value is 0.  truncated[t] != 0: the
 *   episode was cut after step t and trunc_value[t] holds the value of the
 *   true final observation, which replaces the successor value.  The window
 *   end t = T-1 takes bootstrap[n] as successor value, once, in the local term
 *   of step T-1.  Termination wins when both flags are set.  `terminated` may
 *   be NULL (no step terminates).  `truncated` may be NULL (no truncation);
 *   then `trunc_value` is ignored and may be NULL.
 *   Nothing crosses a boundary or a row.
 * Sizes.  N >= 0, T >= 0; N == 0 or T == 0 is a no-op returning RLSCAN_OK
 *   (pointers may then be NULL).  T * max(A, 1) <= 2^30 per row.  Calls with
 *   more than 2^30 steps are split into several launches by rows.
 * Scalars.  gamma, lambda, rho_bar, c_bar must be finite; rho_bar, c_bar > 0.
 * Streams.  Every call is asynchronous on `stream` (NULL = legacy default
 *   stream).  Calls on different streams may run concurrently.
 * Scratch.  Rows that fit one thread block (up to about 4096 steps; Retrace
 *   512 or 1024) need none: each block owns whole rows.  Longer rows are
 *   split into chunks that thread blocks draw from a ticket counter and that
 *   hand their carries to one another; counter and carries live in a small
 *   per-(device, stream) workspace the library allocates on the first such
 *   call on that stream and keeps until rlscan_release_workspaces().
 *   Allocation is not allowed while `stream` is being captured into a CUDA
 *   graph: make one call of the same or larger size on that stream (or call
 *   rlscan_reserve_workspace) before capturing.
 * Errors.  Invalid arguments are reported synchronously and launch nothing.
 *   Conditions only the device can see (a carry hand-off that timed out, an
 *   action index outside [0, A)) are recorded in a per-device status word
 *   that rlscan_sync_status() returns and clears; the kernels never trap.
 */
#ifndef RLSCAN_H
#define RLSCAN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define RLSCAN_ABI_VERSION 1

/* Same type as cudaStream_t. */
typedef struct CUstream_st *rlscan_stream_t;

typedef enum rlscan_status {
  RLSCAN_OK = 0,
  RLSCAN_ERR_INVALID_ARG = 1, /* bad size, NULL mandatory pointer, misalignment, non-finite scalar,
                                 host memory the device cannot read, action index out of range */
  RLSCAN_ERR_OVERLAP = 2,     /* an output overlaps an input or another output */
  RLSCAN_ERR_LAUNCH = 3,      /* the kernel launch failed (cudaGetLastError after launch) */
  RLSCAN_ERR_TIMEOUT = 4,     /* a thread block gave up waiting for its successor's carry */
  RLSCAN_ERR_NOMEM = 5,       /* workspace allocation failed */
  RLSCAN_ERR_CUDA = 6,        /* another CUDA runtime error (no device, sync failure, ...) */
  RLSCAN_ERR_CAPTURE = 7,     /* workspace would have to grow while the stream is being captured */
  RLSCAN_ERR_TOO_LARGE = 8    /* the problem exceeds rlscan_gae_noalloc's fixed scratch */
} rlscan_status;

/* ---------------------------------------------------------------------------
 * Generalized Advantage Estimation (Schulman et al. 2016; named by the pages,
 * arxivlens Abstract).  Backward in t:
 *   delta_t = r_t + gamma * nv_t - v_t,   nv_t = v_{t+1} inside an episode,
 *   A_t = delta_t + gamma * lambda * A_{t+1}   (cut at a boundary),
 *   advantages = A, returns = A + v.
 * Inputs  rewards, values [N,T]; bootstrap [N]; terminated [N,T];
 *         truncated [N,T] (nullable), trunc_value [N,T] (read only where truncated).
 * Outputs advantages [N,T]; returns [N,T] (nullable: not written).
 * ------------------------------------------------------------------------- */
rlscan_status rlscan_gae(const float *rewards, const float *values, const float *bootstrap,
                         const uint8_t *terminated, const uint8_t *truncated,
                         const float *trunc_value, float *advantages, float *returns, int64_t N,
                         int64_t T, float gamma, float lambda, rlscan_stream_t stream);

/* ---------------------------------------------------------------------------
 * GAE with bfloat16 I/O (reduced-precision storage; the pages hint at format
 * limits, gist.science technical summary, Resultaten).  Same arguments
 * and checks as rlscan_gae, but every real array -- rewards, values,
 * bootstrap, trunc_value, advantages, returns -- holds bfloat16 values
 * (passed as their uint16_t bit patterns, 2-byte aligned).  The arithmetic is
 * fp32: inputs widen exactly, the scan runs in fp32, and each output is
 * rounded to the nearest bfloat16 (ties to even), so it differs from rlscan_gae
 * on the widened inputs by at most one rounding to 8 significant bits (2^-8
 * relative) plus the fp32 scan error.  9 bytes per step instead of 17.
 * ------------------------------------------------------------------------- */
rlscan_status rlscan_gae_bf16(const uint16_t *rewards, const uint16_t *values, const uint16_t *bootstrap,
                              const uint8_t *terminated, const uint8_t *truncated, const uint16_t *trunc_value,
                              uint16_t *advantages, uint16_t *returns, int64_t N, int64_t T, float gamma,
                              float lambda, rlscan_stream_t stream);

/* ---------------------------------------------------------------------------
 * GAE without any device allocation.  The paper has no counterpart: this is a
 * deployment variant of rlscan_gae for callers that must not allocate device
 * memory -- for example code that runs while its stream is being captured
 * into a CUDA graph (allocation is not a capturable operation), processes in
 * which another allocator already owns the device's free memory, and
 * latency-critical loops that cannot afford the device-wide synchronisation
 * an allocation may cause.  Arguments, layout and results are exactly
 * rlscan_gae's.
 *
 * Scratch.  Rows longer than one thread block's chunk hand carries between
 * blocks through scratch that here lives in a fixed array compiled into the
 * library (2 MiB + 16 bytes of device memory on every GPU that loads it, held
 * until the process exits), instead of a workspace allocated per stream.
 * - Limit: N * T <= 2^27 steps; larger calls return RLSCAN_ERR_TOO_LARGE and
 *   launch nothing.
 * - The first call on a device resolves the array's device address on that
 *   device (cudaGetSymbolAddress); make that first call before capturing any
 *   stream into a graph.
 * - Every call clears the part of the array it uses (one cudaMemsetAsync on
 *   `stream`) before its kernel, and every call on a device shares the same
 *   array: calls whose kernels can overlap on the GPU (different streams
 *   without ordering between them) race on it.  Order them on one stream or
 *   with events.
 * ------------------------------------------------------------------------- */
rlscan_status rlscan_gae_noalloc(const float *rewards, const float *values, const float *bootstrap,
                                 const uint8_t *terminated, const uint8_t *truncated,
                                 const float *trunc_value, float *advantages, float *returns,
                                 int64_t N, int64_t T, float gamma, float lambda,
                                 rlscan_stream_t stream);

/* ---------------------------------------------------------------------------
 * V-trace (Espeholt et al. 2018, IMPALA; named by the pages), with the trace
 * coefficient scaled by lambda.  Backward in t:
 *   rho_t = min(rho_bar, exp(log_rhos_t)),  c_t = lambda * min(c_bar, exp(log_rhos_t)),
 *   vs_t - v_t = rho_t (r_t + gamma nv_t - v_t) + gamma c_t (vs_{t+1} - v_{t+1})  (cut at a boundary),
 *   pg_advantages_t = rho_t (r_t + gamma * (vs_{t+1} inside an episode, else nv_t) - v_t).
 * Inputs  log_rhos, rewards, values [N,T]; bootstrap [N]; flags as for GAE.
 * Outputs vs [N,T]; pg_advantages [N,T] (nullable).
 * ------------------------------------------------------------------------- */
rlscan_status rlscan_vtrace(const float *log_rhos, const float *rewards, const float *values,
                            const float *bootstrap, const uint8_t *terminated,
                            const uint8_t *truncated, const float *trunc_value, float *vs,
                            float *pg_advantages, int64_t N, int64_t T, float gamma, float lambda,
                            float rho_bar, float c_bar, rlscan_stream_t stream);

/* ---------------------------------------------------------------------------
 * Retrace(lambda) (Munos et al. 2016; named by the pages, whose results note
 * its heavier per-step work from loading action probabilities).  Backward in t:
 *   E_t = sum_a pi[t,a] q[t,a],  q_t = q[t, actions_t],
 *   c_t = lambda * min(1, pi[t, actions_t] / mu_a_t),
 *   Qret_t = r_t + gamma (E_{t+1} - c_{t+1} q_{t+1} + c_{t+1} Qret_{t+1})  inside an episode,
 *   Qret_t = r_t + gamma nv_t at a boundary, where bootstrap[n] and trunc_value
 *   are expected values E_pi Q of the successor state.
 * Inputs  q, pi [N,T,A]; mu_a (behaviour probability of the taken action),
 *         actions (int32 in [0, A)), rewards [N,T]; bootstrap [N]; flags as for GAE.
 * Output  q_ret [N,T].
 * An action outside [0, A) is not read through; it sets RLSCAN_ERR_INVALID_ARG
 * in the device status and that step uses q_t = pi_t(a_t) = 0.
 * ------------------------------------------------------------------------- */
rlscan_status rlscan_retrace(const float *q, const float *pi, const float *mu_a,
                             const int32_t *actions, const float *rewards, const float *bootstrap,
                             const uint8_t *terminated, const uint8_t *truncated,
                             const float *trunc_value, float *q_ret, int64_t N, int64_t T,
                             int64_t A, float gamma, float lambda, rlscan_stream_t stream);

/* ---------------------------------------------------------------------------
 * TD(lambda) returns (lambda-returns).  Backward in t:
 *   G_t = r_t + gamma ((1 - lambda) v_{t+1} + lambda G_{t+1})  inside an episode,
 *   G_t = r_t + gamma nv_t at a boundary.
 * Inputs as for GAE.  Output returns [N,T].
 * ------------------------------------------------------------------------- */
rlscan_status rlscan_td_lambda(const float *rewards, const float *values, const float *bootstrap,
                               const uint8_t *terminated, const uint8_t *truncated,
                               const float *trunc_value, float *returns, int64_t N, int64_t T,
                               float gamma, float lambda, rlscan_stream_t stream);

/* ---------------------------------------------------------------------------
 * Discounted return.  Backward in t: G_t = r_t + gamma * (G_{t+1} inside an
 * episode, else nv_t).  bootstrap is nullable (NULL = 0 at the window end).
 * Output returns [N,T].
 * ------------------------------------------------------------------------- */
rlscan_status rlscan_discounted_return(const float *rewards, const float *bootstrap,
                                       const uint8_t *terminated, const uint8_t *truncated,
                                       const float *trunc_value, float *returns, int64_t N,
                                       int64_t T, float gamma, rlscan_stream_t stream);

/* ---------------------------------------------------------------------------
 * Accumulating eligibility trace, the forward-time mirror of the recurrence
 * (gist.science technical summary, Methodologie 1).  Forward in t:
 *   e_t = g_t + gamma lambda e_{t-1},  e_{-1} = init_trace[n] (nullable: 0),
 * restarting (e_{t-1} := 0) after a step with terminated or truncated set.
 * Inputs  inputs (g) [N,T]; init_trace [N]; terminated [N,T]; truncated [N,T] (nullable).
 * Output  traces [N,T].
 * ------------------------------------------------------------------------- */
rlscan_status rlscan_elig_trace(const float *inputs, const float *init_trace,
                                const uint8_t *terminated, const uint8_t *truncated,
                                float *traces, int64_t N, int64_t T, float gamma, float lambda,
                                rlscan_stream_t stream);

/* ---------------------------------------------------------------------------
 * Episodic inclusive prefix sum.  Forward in t: S_t = x_t + S_{t-1}, S_{-1} = 0,
 * restarting after a done step.  int32 two's-complement arithmetic (wraps
 * modulo 2^32); results are exact, independent of the launch configuration.
 * Inputs  x [N,T] int32; terminated [N,T]; truncated [N,T] (nullable).
 * Output  out [N,T] int32.
 * ------------------------------------------------------------------------- */
rlscan_status rlscan_episodic_prefix_sum(const int32_t *x, const uint8_t *terminated,
                                         const uint8_t *truncated, int32_t *out, int64_t N,
                                         int64_t T, rlscan_stream_t stream);

/* ---------------------------------------------------------------------------
 * Generic affine scan: the recurrence every estimator above specialises
 * (gist.science technical summary, Methodologie 1: A_t = alpha_t +
 * beta_t A_{t+1} and its forward-time mirror), with the coefficients given
 * instead of built.  In scan order -- t = 0..T-1, or t = T-1..0 when
 * `reverse` is 1 --
 *   x_t = b_t + a_t * x_prev,
 * where x_prev is the previous step in scan order, or init[n] for the row's
 * first step (init nullable: 0).  reset[t] != 0 cuts the dependency:
 * x_t = b_t (reset nullable: no resets).  Rows are independent.
 * Inputs  a, b [N,T] float32; reset [N,T] uint8 (nullable); init [N] (nullable).
 * Output  x [N,T] float32.
 * Errors  RLSCAN_ERR_INVALID_ARG also for reverse other than 0 or 1.
 * ------------------------------------------------------------------------- */
rlscan_status rlscan_affine_scan(const float *a, const float *b, const uint8_t *reset, const float *init,
                                 float *x, int64_t N, int64_t T, int32_t reverse, rlscan_stream_t stream);

/* ---------------------------------------------------------------------------
 * rlscan_affine_scan with bfloat16 storage (bf16 I/O): a, b, init and x hold
 * bfloat16 values (IEEE binary32 truncated to its top 16 bits, passed as
 * uint16_t), reset is uint8 as above.  Arithmetic is fp32 in registers; each
 * x_t is rounded to bf16 (round to nearest, ties to even; 8 significant
 * bits) when stored, so |x - exact| <= 2^-8 |x| plus the fp32 error.  Half
 * the bytes of the fp32
 * call.  Vectorised when a, b and x are 16-byte aligned.
 * ------------------------------------------------------------------------- */
rlscan_status rlscan_affine_scan_bf16(const uint16_t *a, const uint16_t *b, const uint8_t *reset,
                                      const uint16_t *init, uint16_t *x, int64_t N, int64_t T, int32_t reverse,
                                      rlscan_stream_t stream);

/* ---------------------------------------------------------------------------
 * Gradient of rlscan_affine_scan (its adjoint), for a loss L whose direct
 * derivative with respect to x_t is dy_t.  `x` is the forward call's output
 * and `reverse` its direction.  The chain rule through the recurrence is an
 * affine scan in the opposite direction: with nxt(t) / prv(t) the following
 * / preceding step in the forward scan's order,
 *   g_t      = dy_t + a_nxt(t) g_nxt(t)   (0 term if nxt(t) resets or is absent)
 *   db_t     = g_t                                          dL/db
 *   da_t     = g_t * x_prv(t), x_prv = init[n] at the first step, 0 where reset
 *   dinit[n] = a_first g_first, 0 if the first step resets  dL/dinit
 * Inputs  a, x, dy [N,T] float32; reset [N,T] (nullable); init [N] (nullable).
 * Output  db [N,T]; da [N,T] (nullable); dinit [N] (nullable).
 * ------------------------------------------------------------------------- */
rlscan_status rlscan_affine_scan_grad(const float *a, const float *x, const float *dy, const uint8_t *reset,
                                      const float *init, float *da, float *db, float *dinit, int64_t N,
                                      int64_t T, int32_t reverse, rlscan_stream_t stream);

/* ---------------------------------------------------------------------------
 * Time-major layout (the memory-layout option of the rl-triton API page,
 * Hugging Face model card, "Key Features": contiguous vs strided).  Each call
 * below takes the same arguments, applies the same checks and computes the
 * same values as the row-major call of the same name without "_tm", but every
 * per-step array is time-major [T,N]: element (t, n) at t * N + n, so each time
 * step is one contiguous run of the N environments (the layout of rollout
 * buffers filled one vectorised environment step at a time).  Per-environment
 * arrays (bootstrap, init_trace, init) stay [N].  Retrace and the bf16 and
 * adjoint scans are row-major only.
 * - Limits: N <= 2^26 and fewer than 2^31 thread-block chunks (T / 64 times
 *   N / 32, roughly); larger calls return RLSCAN_ERR_INVALID_ARG.
 * - Scratch: windows longer than one block's chunk (64 steps) hand carries
 *   along T through the stream's workspace, 16 bytes per environment per
 *   chunk (rlscan_query_plan_tm reports it).
 * - RLSCAN_OPT_FORCE_LOOKBACK applies (shorter chunks, so carries chain even
 *   for short windows); RLSCAN_OPT_FORCE_BLOCK and _FORCE_SCALAR do not (256
 *   threads, one scalar access per step and array, any alignment of 4 bytes).
 * ------------------------------------------------------------------------- */
rlscan_status rlscan_gae_tm(const float *rewards, const float *values, const float *bootstrap,
                            const uint8_t *terminated, const uint8_t *truncated, const float *trunc_value,
                            float *advantages, float *returns, int64_t N, int64_t T, float gamma, float lambda,
                            rlscan_stream_t stream);
rlscan_status rlscan_vtrace_tm(const float *log_rhos, const float *rewards, const float *values,
                               const float *bootstrap, const uint8_t *terminated, const uint8_t *truncated,
                               const float *trunc_value, float *vs, float *pg_advantages, int64_t N, int64_t T,
                               float gamma, float lambda, float rho_bar, float c_bar, rlscan_stream_t stream);
rlscan_status rlscan_td_lambda_tm(const float *rewards, const float *values, const float *bootstrap,
                                  const uint8_t *terminated, const uint8_t *truncated, const float *trunc_value,
                                  float *returns, int64_t N, int64_t T, float gamma, float lambda,
                                  rlscan_stream_t stream);
rlscan_status rlscan_discounted_return_tm(const float *rewards, const float *bootstrap, const uint8_t *terminated,
                                          const uint8_t *truncated, const float *trunc_value, float *returns,
                                          int64_t N, int64_t T, float gamma, rlscan_stream_t stream);
rlscan_status rlscan_elig_trace_tm(const float *inputs, const float *init_trace, const uint8_t *terminated,
                                   const uint8_t *truncated, float *traces, int64_t N, int64_t T, float gamma,
                                   float lambda, rlscan_stream_t stream);
rlscan_status rlscan_episodic_prefix_sum_tm(const int32_t *x, const uint8_t *terminated, const uint8_t *truncated,
                                            int32_t *out, int64_t N, int64_t T, rlscan_stream_t stream);
rlscan_status rlscan_affine_scan_tm(const float *a, const float *b, const uint8_t *reset, const float *init,
                                    float *x, int64_t N, int64_t T, int32_t reverse, rlscan_stream_t stream);

/* ---------------------------------------------------------------------------
 * Status, workspace and configuration.
 * ------------------------------------------------------------------------- */

/* Synchronize `stream`, then return and clear the device-side status of the
 * current device (RLSCAN_OK, RLSCAN_ERR_TIMEOUT or RLSCAN_ERR_INVALID_ARG).
 * The status word is per device and shared by all streams on it; the first
 * recorded error wins.  A CUDA error while synchronizing gives RLSCAN_ERR_CUDA. */
rlscan_status rlscan_sync_status(rlscan_stream_t stream);

/* Human-readable name of a status code (static string, never NULL). */
const char *rlscan_status_string(rlscan_status status);

/* Free every workspace the library allocated (all devices and streams).  The
 * caller must ensure no rlscan work is in flight. */
void rlscan_release_workspaces(void);

/* Make sure the workspace of (current device, `stream`) holds at least
 * `bytes` (as reported by rlscan_query_plan's workspace_bytes), allocating it
 * now.  Call before capturing work on `stream` into a CUDA graph.
 * RLSCAN_ERR_CAPTURE if the stream is capturing and the workspace is too small. */
rlscan_status rlscan_reserve_workspace(int64_t bytes, rlscan_stream_t stream);

/* ABI version this library was built with (RLSCAN_ABI_VERSION). */
int rlscan_abi_version(void);

typedef enum rlscan_estimator {
  RLSCAN_EST_GAE = 0,
  RLSCAN_EST_VTRACE = 1,
  RLSCAN_EST_RETRACE = 2,
  RLSCAN_EST_TD_LAMBDA = 3,
  RLSCAN_EST_DISCOUNTED_RETURN = 4,
  RLSCAN_EST_ELIG_TRACE = 5,
  RLSCAN_EST_EPISODIC_PREFIX_SUM = 6,
  RLSCAN_EST_AFFINE_SCAN = 7,
  RLSCAN_EST_AFFINE_SCAN_GRAD = 8,
  RLSCAN_EST_AFFINE_SCAN_BF16 = 9,
  RLSCAN_EST_GAE_BF16 = 10
} rlscan_estimator;

/* How a call of the given shape is executed (no device work, no allocation). */
typedef struct rlscan_plan_info {
  int32_t block_threads;    /* threads per thread block */
  int32_t chunk_steps;      /* steps one thread block scans */
  int32_t lookback;         /* 1: blocks chain their carries through the workspace */
  int32_t launches;         /* kernel launches the call makes (row slices) */
  int64_t chunks;           /* chunks over all launches: groups of whole rows (walked by
                               resident blocks) or, with look-back, pieces of
                               chunk_steps steps drawn by ticket */
  int64_t workspace_bytes;  /* workspace the call needs on its stream */
} rlscan_plan_info;

rlscan_status rlscan_query_plan(rlscan_estimator estimator, int64_t N, int64_t T, int64_t A,
                                rlscan_plan_info *info);
/* The same for the time-major calls (estimators with a "_tm" entry point;
 * others give RLSCAN_ERR_INVALID_ARG).  chunks counts thread blocks, each a
 * chunk of chunk_steps steps: K steps x up to 8 time slices x 32 environments
 * per column group. */
rlscan_status rlscan_query_plan_tm(rlscan_estimator estimator, int64_t N, int64_t T, rlscan_plan_info *info);

/* Process-wide options (all default 0 unless stated). */
typedef enum rlscan_option {
  RLSCAN_OPT_LOOKBACK_TIMEOUT_NS = 1, /* carry wait limit per block, default 1e9 (1 s) */
  RLSCAN_OPT_FORCE_LOOKBACK = 2,      /* 1: chain carries even where blocks hold whole rows */
  RLSCAN_OPT_FORCE_BLOCK = 3,         /* 0: auto; else threads per block (a multiple of 64
                                         from 128 to 512; Retrace takes 128 or 256 and
                                         ignores other values) */
  RLSCAN_OPT_FORCE_SCALAR = 4,        /* 1: take the scalar (unvectorised) load path */
  RLSCAN_OPT_CHECK_POINTERS = 5,      /* default 1: reject host memory the device cannot read */
  RLSCAN_OPT_TEST_STARVE_LOOKBACK = 6, /* test only, 1: the first block never publishes its
                                          carry, so its predecessors time out */
  RLSCAN_OPT_PDL = 7                   /* default 1: programmatic dependent launch, so a kernel
                                          can be scheduled while the previous kernel on the
                                          stream drains (it waits for it before any access) */
} rlscan_option;

rlscan_status rlscan_set_option(rlscan_option option, int64_t value);
int64_t rlscan_get_option(rlscan_option option);

#ifdef __cplusplus
}
#endif

#endif /* RLSCAN_H */
