/*
 * race_attn.h — C ABI of the RACE attention library (librace_attn.so).
 *
 * RACE attention estimates attention under the sharpened angular kernel
 *     sim(q, k) = (1 - arccos(qhat . khat) / pi)^P
 * with L repeated arrays of P-bit signed-random-projection buckets (R = 2^P) and
 * soft hashing.  Sources, by page title:
 *   [JA]  "RACE Attention: 長系列トレーニングのための厳密な線形時間アテンションの技術的概要"
 *         (gist.science, Japanese technical overview), §2.1 core idea (sim equation,
 *         soft bucketization, bucket aggregation, reconstruction), §2.2 (differentiable
 *         soft assignment with temperature; prefix-sum kernels for causal masking;
 *         complexity O(L N R d)).
 *   [IT]  "RACE Attention: A Strictly Linear-Time Attention for Long-Sequence
 *         Training" (gist.science, Italian technical summary), §2 (random projections
 *         softened by a softmax over the hypercube vertices; per-bucket mass and value
 *         sums; normalised weighted mean), §3 (causal and non-causal kernels).
 *   [ABS] "Replacing Softmax Similarity with a Sharpened Angular Similarity ..."
 *         (arXiv 2510.04008 abstract): forward-backward of a multi-head attention layer.
 *
 * The operation, fixed exactly:
 *     xhat = x / max(|x|_2, 1e-12)
 *     u_l  = W_l^T xhat                         (W: [L, d, P], plane p of table l = W[l,:,p])
 *     p_l  = softmax_b(<c_b, u_l> / tau)        (b = 0..R-1, c_bp = +1 iff bit p of b is set)
 *     phi  = concat_l p_l / sqrt(L)             ([L*R] per vector)
 *     o_i  = sum_{j in J(i)} (phi(q_i).phi(k_j)) v_j / sum_{j in J(i)} phi(q_i).phi(k_j)
 *     J(i) = all j (non-causal) or j <= i (causal, inclusive).
 *
 * Layouts.  q, k, v, out, dout, dq, dk, dv are dense row-major [H][N][d] with
 * H = batch * heads.  W and dW are dense float32, [L][d][P] shared by every head (the
 * spec-form calls), or [H][L][d][P] with one set of planes per head (race_args_t
 * .w_per_head).  den is [H][N] float32.  phi dumps are [H][N][L*R].
 *
 * Pointers.  Every tensor pointer is a DEVICE pointer on the current CUDA device,
 * except where an entry point says "host".  Tensor pointers must be 16-byte aligned.
 * The caller owns every buffer; the library keeps no pointer after a call returns.
 *
 * Execution.  Calls enqueue work on `stream` and return without synchronising
 * (cudaStream_t; NULL is the legacy default stream).  They never print, abort or
 * exit.  Argument errors are reported before anything is enqueued.
 *
 * Threads and state.  The compute calls keep no host state between calls: several
 * host threads may call them at once, each with its own workspace (race_args_t
 * .workspace, or the library's own allocation).  State shared by the whole process:
 * the device status flag (one word per device, raised by any call on it and read and
 * cleared by race_device_status), the static scratch of race_forward_noalloc (see
 * there), the launch counter (atomic), the profiling registry of race_timing_* (a
 * mutex guards it; while recording is on every launch of every thread adds events to
 * it), and two values fixed at the first call: the driver entry point used to build
 * TMA descriptors and the RACE_NVTX switch.
 *
 * Supported sizes: d = 64; 1 <= P <= 8; L >= 1 with L * 2^P <= 16384; N >= 1;
 * H >= 1; tau finite and > 0.  Other d values give RACE_ERR_UNSUPPORTED.
 */
#ifndef RACE_ATTN_H
#define RACE_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t. */
typedef struct CUstream_st *race_stream_t;

typedef enum {
  RACE_OK = 0,
  RACE_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size, bad tau          */
  RACE_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. d != 64)             */
  RACE_ERR_WORKSPACE = 3,     /* caller workspace too small or allocation failed     */
  RACE_ERR_CUDA = 4,          /* a CUDA runtime call or a launch failed              */
  RACE_ERR_DEVICE_STATUS = 5, /* a kernel raised its device status flag (a bounded  */
                              /* wait gave up, or an index check failed)             */
  RACE_ERR_SCRATCH_LIMIT = 6  /* race_forward_noalloc: the problem needs more scratch */
                              /* than RACE_NOALLOC_SCRATCH_BYTES                     */
} race_status_t;

typedef enum { RACE_BF16 = 0, RACE_FP32 = 1 } race_dtype_t;

/* Which kernels a call may use.  AUTO picks the tensor-core (tcgen05) path for
 * bf16 inputs where it exists and the CUDA-core path otherwise.  SIMT forces the
 * CUDA-core kernels (always available; the only path for fp32).  TENSOR forces the
 * tensor-core kernels and fails with RACE_ERR_UNSUPPORTED where they do not apply.
 * The tensor-core kernels cover bf16 inputs with 6 <= P <= 8 and N < 2^31 - 128, and
 *   forward:  L * 2^P a multiple of 128;
 *   backward: L * 2^P a multiple of 256 and L * P <= 256.
 * Every other shape runs on the CUDA-core kernels under AUTO. */
typedef enum { RACE_IMPL_AUTO = 0, RACE_IMPL_SIMT = 1, RACE_IMPL_TENSOR = 2 } race_impl_t;

/* Full argument set of the *_ex entry points. */
typedef struct {
  int64_t N;                 /* sequence length                                        */
  int H;                     /* batch * heads                                          */
  int d;                     /* head dimension (64)                                    */
  int L;                     /* number of hash tables                                  */
  int P;                     /* hyperplanes per table; R = 2^P buckets                 */
  float tau;                 /* soft-hash temperature (the pages' beta is 1/tau)       */
  int causal;                /* 0: all keys; 1: keys j <= i                            */
  race_dtype_t dtype;        /* element type of q, k, v, dout                          */
  race_dtype_t out_dtype;    /* element type of out (forward writes, backward reads)   */
  int chunk;                 /* advisory tokens per chunk: 0 or a positive multiple of  */
                             /* 32 (others: RACE_ERR_INVALID_ARG).  The tensor-core     */
                             /* kernels always run 128-token chunks and the CUDA-core   */
                             /* kernels 32-token tiles; results do not depend on it     */
  void *workspace;           /* device scratch of >= workspace_bytes, or NULL: the      */
  size_t workspace_bytes;    /* library then allocates stream-ordered scratch itself    */
  float *den;                /* optional [H][N]: forward writes den_i =                 */
                             /* sum_j phi(q_i).phi(k_j); backward reads it (NULL: the   */
                             /* backward recomputes it)                                 */
  race_impl_t impl;          /* kernel family, see race_impl_t                          */
  race_dtype_t grad_dtype;   /* element type of dq, dk, dv written by the backward      */
                             /* (bf16 or float32, for either input dtype; float32 keeps */
                             /* the gradients free of a final bf16 rounding)            */
  int w_per_head;            /* 0: W and dW are [L][d][P], shared by every head (dW the */
                             /* sum over heads); 1: W and dW are [H][L][d][P], one set  */
                             /* of hash planes per head                                 */
} race_args_t;

/* Fill `a` with the defaults of the spec-form calls: bf16 in, out and gradients,
 * chunk 0, no workspace, no den, RACE_IMPL_AUTO. */
void race_args_init(race_args_t *a, int64_t N, int H, int d, int L, int P, float tau,
                    int causal);

/* ---------------------------------------------------------------------------------
 * race_forward — RACE attention forward, bf16 q/k/v/out, float32 W.
 * Soft hash, bucket aggregation (S = sum phi(k) v^T, z = sum phi(k)), readout and
 * normalisation: [JA] §2.1 (soft bucketization, bucket aggregation, reconstruction),
 * causal prefix sums: [JA] §2.2.  Allocates stream-ordered scratch on `stream`
 * (cudaMallocAsync / cudaFreeAsync).
 * Returns RACE_OK, RACE_ERR_INVALID_ARG, RACE_ERR_UNSUPPORTED, RACE_ERR_WORKSPACE or
 * RACE_ERR_CUDA.
 * ------------------------------------------------------------------------------ */
race_status_t race_forward(const void *q, const void *k, const void *v, const float *W,
                           void *out, int64_t N, int H, int d, int L, int P, float tau,
                           int causal, race_stream_t stream);

/* ---------------------------------------------------------------------------------
 * race_backward — gradients of sum(out * dout) with respect to q, k, v and W
 * (differentiable soft assignment, [JA] §2.2 and [IT] §3 item 4; the formulas are the
 * chain rule of the forward).  bf16 q/k/v/out/dout/dq/dk/dv; dW float32, OVERWRITTEN
 * with the sum over all heads and tokens.  `out` must be the forward's output for the
 * same inputs.  den is recomputed.  Scratch as in race_forward.
 * ------------------------------------------------------------------------------ */
race_status_t race_backward(const void *q, const void *k, const void *v, const float *W,
                            const void *out, const void *dout, void *dq, void *dk,
                            void *dv, float *dW, int64_t N, int H, int d, int L, int P,
                            float tau, int causal, race_stream_t stream);

/* Extended forms: every option in `a` (dtypes, chunk, caller workspace, den, impl). */
race_status_t race_forward_ex(const void *q, const void *k, const void *v, const float *W,
                              void *out, const race_args_t *a, race_stream_t stream);
race_status_t race_backward_ex(const void *q, const void *k, const void *v,
                               const float *W, const void *out, const void *dout,
                               void *dq, void *dk, void *dv, float *dW,
                               const race_args_t *a, race_stream_t stream);

/* ---------------------------------------------------------------------------------
 * race_forward_noalloc — the forward of race_forward_ex computed without allocating
 * any memory.  The paper has no counterpart: this is a deployment aid for callers that
 * cannot allocate device memory at call time, e.g. a serving process that reserves
 * all free HBM for its caches at start-up (any later cudaMalloc fails or fragments the
 * reservation) or a latency-bound loop that must not enter the allocator, which can
 * synchronise or grow its pool.
 *
 * Arguments, layouts and results are those of race_forward_ex; a->workspace and
 * a->workspace_bytes are ignored.  The scratch is instead one fixed device array of
 * RACE_NOALLOC_SCRATCH_BYTES that is part of the library's loaded module (one per
 * device).  No cudaMalloc, cudaMallocAsync or other allocating routine is called; the
 * call clears the parts of the array that must start at zero on `stream` itself.
 *
 * Set-up: every call looks up the array's device address on the current device (so a
 * device reset cannot leave a stale address behind); the first call on a device may
 * load the module there.  Make that first call before any stream capture begins.
 *
 * Concurrency: all calls on one device share the array.  Calls that can overlap in
 * time (different streams, or different host threads without ordering) race on it and
 * give wrong results; order them on one stream.
 *
 * Errors: RACE_ERR_SCRATCH_LIMIT, before any device work, when
 * race_workspace_size(a, 0) exceeds RACE_NOALLOC_SCRATCH_BYTES; RACE_ERR_CUDA when the
 * address look-up fails; otherwise the statuses of race_forward_ex.
 * ------------------------------------------------------------------------------ */
#define RACE_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)
race_status_t race_forward_noalloc(const void *q, const void *k, const void *v,
                                   const float *W, void *out, const race_args_t *a,
                                   race_stream_t stream);

/* ---------------------------------------------------------------------------------
 * race_forward_stream — the forward of race_forward_ex over a block of N new tokens that
 * continues earlier blocks of the same sequences: every query also attends to all keys of
 * the earlier blocks through their carried sketch state, which the call updates.  This is
 * the state carry of decoding (N = 1 per call) and of chunked prefill; the pages name an
 * efficient KV cache at inference as a use of the sketch ([JA] §6; the state is the
 * bucket aggregation of [JA] §2.1 and the causal prefix of [JA] §2.2).
 *
 * State layout: float32 [H][L * 2^P][65], row l * 2^P + b of head h holding
 *     sum over earlier keys j of p_{l,b}(k_j) * [v_j | 1]
 * with p_l = softmax_b(<c_b, W_l^T khat_j>/tau) the unscaled corner probabilities (phi =
 * p / sqrt(L)): columns 0..63 value sums, column 64 the mass.  (H * L * 2^P * 65 floats;
 * with per-head planes each head's state uses its own planes.)
 * state_in: the state before the block (NULL: all zero, the start of a sequence).
 * state_out: receives the state after the block (NULL: not written); it may be the same
 * buffer as state_in.  Both must be 16-byte aligned device pointers.
 * a->causal = 1: keys j <= i within the block plus every earlier key; a->causal = 0: every
 * key of the block plus every earlier key.  Other arguments, results and errors as
 * race_forward_ex; the scratch need is race_workspace_size(a, 0).
 * ------------------------------------------------------------------------------ */
race_status_t race_forward_stream(const void *q, const void *k, const void *v,
                                  const float *W, void *out, const float *state_in,
                                  float *state_out, const race_args_t *a,
                                  race_stream_t stream);

/* ---------------------------------------------------------------------------------
 * race_hard_forward — classic RACE with hard hashes, the tau -> 0 limit of the soft
 * estimator: repeated arrays of counts ([JA] §2.1 count estimators and bucket
 * aggregation; [KO] §2: L tables of P-bit buckets).  With h_l(x) the P-bit bucket whose
 * bit p is 1 when W_l[:,p] . x >= 0 (decided in float32),
 *     A_ij = number of tables l with h_l(q_i) == h_l(k_j)      (j in J(i))
 *     out_i = sum_j A_ij v_j / sum_j A_ij,  and out_i = 0 when no key collides.
 * counts (nullable, int32 [H][N], device): receives sum_j A_ij, exact.  tau is ignored;
 * other arguments and layouts as race_forward_ex (P <= 8).  Scratch as race_forward_ex
 * with the size given by race_hard_workspace_size.
 * ------------------------------------------------------------------------------ */
race_status_t race_hard_forward(const void *q, const void *k, const void *v, const float *W,
                                void *out, int *counts, const race_args_t *a,
                                race_stream_t stream);
race_status_t race_hard_workspace_size(const race_args_t *a, size_t *bytes);

/* race_hard_hash — the bucket ids alone: ids[h][n][l] = h_l(x_hn) as uint8 (device),
 * for x of a->dtype [H][N][d]. */
race_status_t race_hard_hash(const void *x, const float *W, uint8_t *ids, const race_args_t *a,
                             race_stream_t stream);

/* Scratch bytes the *_ex calls need for `a` (backward != 0: the backward).  Writes 0
 * and returns an error status for invalid or unsupported arguments.  Host only; no
 * device work. */
race_status_t race_workspace_size(const race_args_t *a, int backward, size_t *bytes);

/* ---------------------------------------------------------------------------------
 * race_hash — the feature map alone: L2 normalisation, the d x (L*P) projection and
 * the softmax over the 2^P corners, phi = concat_l p_l / sqrt(L) ([JA] §2.1 soft
 * bucketization; [IT] §2 item 2).  x: [H][N][d] of a->dtype; phi: [H][N][L*2^P] of
 * a->out_dtype (bf16 or float32).  Uses a->N, H, d, L, P, tau only.  Writes
 * H*N*L*2^P elements: meant for checks and small problems.
 * ------------------------------------------------------------------------------ */
race_status_t race_hash(const void *x, const float *W, void *phi, const race_args_t *a,
                        race_stream_t stream);

/* Synchronises `stream`, then reports and clears this device's status flag, which a
 * kernel raises when a bounded wait gives up or an index check fails.  *flags (may be
 * NULL) receives the raw flag bits.  Returns RACE_OK or RACE_ERR_DEVICE_STATUS (or
 * RACE_ERR_CUDA). */
race_status_t race_device_status(race_stream_t stream, uint32_t *flags);

/* ---------------------------------------------------------------------------------
 * race_selftest_wait_timeout — exercises the failure path of the library's kernels
 * without any fault: one kernel (a single warp; no TMA copy, no MMA) waits on an
 * mbarrier phase that nothing completes, through the same bounded-wait routine the
 * tensor-core kernels use, with a limit of `limit_cycles` SM clock cycles
 * (1 <= limit_cycles <= 2e9, the kernels' own limit; about 1e6 is half a millisecond).
 * The wait gives up, raises the timeout bit (1) of the device status flag and the
 * kernel returns, so the context stays usable.  Synchronises `stream`; *timed_out
 * (host, may be NULL) receives 1 when every lane gave up.  The flag stays raised for
 * race_device_status to report (RACE_ERR_DEVICE_STATUS) and clear.
 * Returns RACE_OK, RACE_ERR_INVALID_ARG or RACE_ERR_CUDA.
 * ------------------------------------------------------------------------------ */
race_status_t race_selftest_wait_timeout(int64_t limit_cycles, int *timed_out,
                                         race_stream_t stream);

/* Static description of a status code. */
const char *race_status_string(race_status_t s);

/* Library version as major*10000 + minor*100 + patch. */
int race_version(void);

/* ---------------------------------------------------------------------------------
 * Profiling aids (host only).
 * race_timing_enable(1) clears the per-kernel totals and makes every later kernel
 * launch of the library record a CUDA event before and after it on its own stream;
 * race_timing_enable(0) stops recording.  race_timing_report(i, ...) gives the i-th
 * kernel seen while recording was on: its name (valid until the next
 * race_timing_enable), the summed device time in milliseconds and the number of
 * launches; it waits for the recorded events.  It returns RACE_ERR_INVALID_ARG once i
 * is past the last kernel.  race_launch_count() is the number of kernel launches the
 * library has issued in this process.
 * ------------------------------------------------------------------------------ */
race_status_t race_timing_enable(int on);
race_status_t race_timing_report(int i, const char **name, double *total_ms,
                                 int64_t *launches);
int64_t race_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* RACE_ATTN_H */
