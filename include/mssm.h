/*
 * mssm.h - C ABI of the B200 (sm_100a) Mamba-1 selective scan library (libmssm.so).
 *
 * The library computes, on one GPU, the forward selective scan of a Mamba-1
 * layer and its one-token decode counterpart:
 *
 *   delta_t   = softplus(delta_raw_t + bias_d)          (softplus and bias optional)
 *   A_bar_tn  = exp(delta_t * A_dn)
 *   h_tn      = A_bar_tn * h_(t-1)n + delta_t * B_tn * u_t          (h_(-1) = 0)
 *               (optionally the zero-order-hold input term and a given h_(-1))
 *   y_t       = sum_n C_tn * h_tn + D_d * u_t                       (D optional)
 *   out_t     = y_t * silu(z_t)                                     (z optional)
 *
 * Sources (web pages, by title and section):
 *  - "Linear Attention vs Softmax Attention: Can RWKV or Mamba Replace
 *    Transformers?": section Core Concepts, item 3 (Selective State Space
 *    Models: the continuous system and its discretisation A_bar = exp(Delta A));
 *    section Implementation (the listed SelectiveSSMLayer: softplus step size,
 *    A = -exp(A_log), the sequential loop with B_bar = Delta B from a zero state,
 *    readout C.h + D x, output multiplied by silu of the gate branch); section
 *    How It Works (the fused scan: inputs read once, only y written back).
 *  - "State Space Models in Large Language Models: How Mamba, S4, and Selective
 *    Recurrence Challenge Transformer Attention": sections Discretization
 *    (recurrent view, one O(1) step per token) and Dynamic Parameterization
 *    (Delta_t = Softplus(Parameter + Linear(x_t))).
 *  - "Mamba selective state space" (chenyuan1125.github.io), section
 *    "Selectivity Removes the Convolution Shortcut; Scan Restores Parallelism":
 *    each position is the affine map (A_bar_t, B_bar_t x_t); neighbouring maps
 *    compose associatively, which is what lets the length be split into chunks
 *    whose carries are combined.
 *
 * Conventions shared by every entry point
 *  - Tensors are described by mssm_tensor: a DEVICE pointer plus shape and
 *    strides in ELEMENTS.  The caller owns all memory; the library never frees
 *    or retains a caller pointer beyond the call.
 *  - Supported dtype mixes: everything fp32; or bf16 for u/delta/B/C/z/out
 *    (x/dt/B/C/z/out for decode) with fp32 A, D, bias and state.
 *  - The state size N must be 16 (MSSM_ERR_UNSUPPORTED otherwise).
 *  - Sizes: Bt, D and L each below 2^31, and the number of rows (Bt * D, or the
 *    sequence count * D for packed sequences) below 2^31 (MSSM_ERR_UNSUPPORTED
 *    otherwise).
 *  - The innermost (length) dimension of u/delta/z/out/B/C must have stride 1.
 *  - All calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream).  Argument errors are reported synchronously, before
 *    anything is launched; launch failures map to MSSM_ERR_CUDA.  A detailed
 *    message for the last error on the calling thread is available from
 *    mssm_last_error().
 *  - Outputs must not alias inputs; decode `state` is the only in-place tensor.
 *  - The current CUDA device must be the device that holds the tensors.
 */
#ifndef MSSM_H
#define MSSM_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MSSM_F32 = 0,
    MSSM_BF16 = 1,
    MSSM_I32 = 2  /* index tensors only (cu_seqlens) */
} mssm_dtype;

typedef enum {
    MSSM_OK = 0,
    MSSM_ERR_INVALID_ARG = 1, /* null required pointer, bad shape/stride/dtype combination */
    MSSM_ERR_UNSUPPORTED = 2, /* valid but not implemented here (N != 16, misaligned rows, ...) */
    MSSM_ERR_CUDA = 3,        /* a CUDA runtime call or a kernel launch failed */
    MSSM_ERR_TIMEOUT = 4      /* a bounded device-side wait gave up (see mssm_get_error) */
} mssm_status;

typedef struct {
    void *data;         /* device pointer; must be 16-byte aligned for the vector paths */
    int32_t dtype;      /* mssm_dtype */
    int32_t ndim;       /* 1..4 */
    int64_t shape[4];   /* sizes, outermost first */
    int64_t stride[4];  /* strides in elements, outermost first */
} mssm_tensor;

/*
 * Forward selective scan (prefill / training forward), fused:
 * softplus + discretisation + recurrence + readout + D skip + silu(z) gate +
 * store, plus the final state.  The B x D x L x N state never touches memory.
 *
 *   u          [Bt, D, L]  bf16|f32      the scan input (the conv branch output)
 *   delta      [Bt, D, L]  dtype of u    the step before softplus (delta_raw)
 *   A          [D, N]      f32           state matrix (diagonal per channel)
 *   B, C       [Bt, N, L]  dtype of u    input/readout projections, shared by channels
 *   D          [D]         f32 or NULL   skip weight (NULL: no skip)
 *   z          [Bt, D, L]  dtype of u, or NULL (NULL: no gate)
 *   delta_bias [D]         f32 or NULL   added to delta before softplus
 *   softplus_flag          1: delta = softplus(delta + bias); 0: delta = delta + bias
 *   out        [Bt, D, L]  dtype of u    written
 *   last_state [Bt, D, N]  f32 or NULL   h after the last step, written (n stride 1)
 *   stream                 cudaStream_t
 *
 * Initial state is zero.  Bt*D == 0 is a no-op; L == 0 writes a zero
 * last_state.  Long sequences are split into chunks: a first kernel summarises
 * every chunk but the last (its total step and its end state from zero), the
 * last CTA of each row tile to finish folds those summaries into carried
 * states, and a second kernel runs each chunk from its carried state.  No CTA
 * ever waits on another.  The summaries live in a per-device workspace owned
 * by the library: allocated with cudaMalloc on the first call that needs it
 * (grown when a larger problem needs more, which synchronises the device) and
 * freed by mssm_shutdown().  Calls that use the workspace must not overlap on
 * the GPU (different streams of one device); run them on one stream or order
 * them with events.  A first call of the largest size before any stream
 * capture keeps allocation out of captured work.  Shapes with many row tiles
 * instead use a persistent kernel that runs each tile's chunks in order
 * (MSSM_ERR_TIMEOUT from mssm_get_error if one of its bounded waits gave up).
 */
mssm_status mssm_selective_scan_fwd(const mssm_tensor *u, const mssm_tensor *delta,
                                    const mssm_tensor *A, const mssm_tensor *B,
                                    const mssm_tensor *C, const mssm_tensor *D,
                                    const mssm_tensor *z, const mssm_tensor *delta_bias,
                                    int softplus_flag, mssm_tensor *out,
                                    mssm_tensor *last_state, void *stream);

/* Discretisation of the input term (mssm_selective_scan_fwd_ex, mssm_state_update_ex). */
typedef enum {
    MSSM_DISC_EULER = 0, /* B_bar = delta * B: the listed layer's loop ("Linear Attention vs
                            Softmax Attention ...", section Implementation); the default */
    MSSM_DISC_ZOH = 1    /* B_bar = (exp(delta A) - 1) / A * B per state: the zero-order hold
                            of the same page's Core Concepts, item 3, and of "State Space Models
                            in Large Language Models ...", section Discretization, for diagonal
                            A; delta * B where A = 0 (the limit) */
} mssm_discretization;

/*
 * Optional inputs of mssm_selective_scan_fwd_ex.  Set struct_size to
 * sizeof(mssm_scan_ext); fields may be appended in later versions.
 *   discretization  mssm_discretization
 *   h0              [S, D, N] f32, n stride 1: the state before the first step of each
 *                   sequence (NULL: zero), e.g. the last_state of the previous piece of
 *                   a sequence processed in parts (prefill in pieces, resume).  S = Bt,
 *                   or the number of packed sequences.  Must not alias out or last_state.
 *   cu_seqlens      [S + 1] int32 DEVICE tensor, or NULL: packed variable-length
 *                   sequences.  u, delta, z, out are then [1, D, T] and B, C [1, N, T];
 *                   sequence s covers steps cu_seqlens[s] .. cu_seqlens[s+1] - 1, starts
 *                   from h0[s] (or zero), and its final state goes to last_state[s]
 *                   ([S, D, N]).  Offsets must be non-decreasing within [0, T].
 *   max_seqlen      host value >= every sequence length (used to plan the launch; only
 *                   read with cu_seqlens).  Offsets outside [0, T], decreasing offsets
 *                   or a longer sequence are clamped on the device and reported as
 *                   MSSM_ERR_INVALID_ARG by mssm_get_error; the outputs are then undefined.
 * The packed layout is the one the listed layer's batch would take with its padding
 * removed; a sequence boundary resets the state, as if each sequence were its own batch
 * row (the pages' scan has no state across batch rows).
 */
typedef struct {
    int32_t struct_size;
    int32_t discretization;
    const mssm_tensor *h0;
    const mssm_tensor *cu_seqlens;
    int64_t max_seqlen;
} mssm_scan_ext;

/*
 * mssm_selective_scan_fwd_ex: mssm_selective_scan_fwd with the options of `ext`
 * (NULL: none, i.e. the plain call).  Same arguments, results, workspace and
 * errors otherwise; an invalid ext (struct_size too small, unknown
 * discretization, h0 of the wrong shape, dtype or n stride, h0 aliasing an
 * output) is MSSM_ERR_INVALID_ARG.  With h0 given, the scan equals running the
 * recurrence from h0: splitting a sequence at any step and passing the first
 * part's last_state as the second part's h0 reproduces the whole-sequence call.
 */
mssm_status mssm_selective_scan_fwd_ex(const mssm_tensor *u, const mssm_tensor *delta,
                                       const mssm_tensor *A, const mssm_tensor *B,
                                       const mssm_tensor *C, const mssm_tensor *D,
                                       const mssm_tensor *z, const mssm_tensor *delta_bias,
                                       int softplus_flag, const mssm_scan_ext *ext,
                                       mssm_tensor *out, mssm_tensor *last_state, void *stream);

/*
 * mssm_selective_scan_fwd_noalloc: the same scan, same arguments and results,
 * for callers that cannot allocate device memory during the call.  Examples: a
 * host application whose device memory is entirely owned by its own allocator
 * or a pre-reserved pool, or a loop that cannot afford cudaMalloc's implicit
 * device-wide synchronisation.  (The pages describe no such entry point; it is
 * a property of this library's boundary, not of the method.)
 *
 * It never calls cudaMalloc, cudaFree or any allocating routine.  When a long
 * sequence is split into chunks, the chunk summaries go to a fixed 8 MiB array
 * compiled into the library's device image, present on every GPU that loads
 * the library until the process exits.  A problem whose summaries need more
 * than 8 MiB (about (chunks - 1) x Bt x D x 68 bytes) is rejected with
 * MSSM_ERR_UNSUPPORTED and a message naming the size; problems that are not
 * split use no scratch at all.
 *
 * The first call on each device looks up the array's device address (with that
 * device current) and caches it; make that first call before any stream
 * capture.  Every call shares the one array and finds in it what the previous
 * call left: each call zeroes the arrival counters it needs (one small
 * cudaMemsetAsync on `stream`).  Calls that overlap on the GPU race on the
 * array; issue them on one stream or order them with events.
 */
mssm_status mssm_selective_scan_fwd_noalloc(const mssm_tensor *u, const mssm_tensor *delta,
                                            const mssm_tensor *A, const mssm_tensor *B,
                                            const mssm_tensor *C, const mssm_tensor *D,
                                            const mssm_tensor *z, const mssm_tensor *delta_bias,
                                            int softplus_flag, mssm_tensor *out,
                                            mssm_tensor *last_state, void *stream);

/*
 * One-token selective state update (decode), state updated IN PLACE:
 *
 *   state [Bt, D, N] f32   read and written (n stride 1)
 *   x, dt [Bt, D]          bf16|f32; dt is the step before softplus (delta_raw)
 *   A     [D, N] f32
 *   B, C  [Bt, N]          dtype of x
 *   D     [D] f32 or NULL; z [Bt, D] dtype of x or NULL
 *   out   [Bt, D]          dtype of x, written
 *
 * This entry point applies delta = softplus(dt) (no bias).  The same step as
 * one iteration of mssm_selective_scan_fwd's recurrence ("State Space Models
 * in Large Language Models ...", section Discretization, recurrent view).
 * When `state` is one contiguous 16-byte-aligned [Bt*D][16] range (and the
 * per-row inputs are aligned runs), a persistent kernel streams each (batch,
 * 128-channel block) tile and its inputs through shared memory with bulk
 * copies (see MSSM_OPT_DECODE_PATH); its bounded waits report
 * MSSM_ERR_TIMEOUT through mssm_get_error if they ever give up.
 */
mssm_status mssm_state_update(mssm_tensor *state, const mssm_tensor *x, const mssm_tensor *dt,
                              const mssm_tensor *A, const mssm_tensor *B, const mssm_tensor *C,
                              const mssm_tensor *D, const mssm_tensor *z, mssm_tensor *out,
                              void *stream);

/*
 * As mssm_state_update, with an optional per-channel dt_bias [D] f32 (NULL: none),
 * an explicit softplus flag and the discretisation (mssm_discretization), so
 * that a sequence of decode steps reproduces mssm_selective_scan_fwd_ex called
 * with the same bias, flag and discretisation.
 */
mssm_status mssm_state_update_ex(mssm_tensor *state, const mssm_tensor *x,
                                 const mssm_tensor *dt, const mssm_tensor *A,
                                 const mssm_tensor *B, const mssm_tensor *C,
                                 const mssm_tensor *D, const mssm_tensor *z,
                                 const mssm_tensor *dt_bias, int softplus_flag,
                                 int discretization, mssm_tensor *out, void *stream);

/*
 * Backward of mssm_selective_scan_fwd (Euler discretisation, zero initial state,
 * no packed sequences): the gradients of Loss with respect to every input, given
 * dout = dLoss/dout.  The states are recomputed, never stored: one pass of chunk
 * summaries, both ways, gives every chunk's start state and incoming dLoss/dh
 * (chunks of 64 steps, or 32 from 1024 row tiles of 32 channels on), and every
 * chunk then sweeps its recomputed states backwards ("Mamba
 * selective state space", the hardware-aware scan: intermediates are recomputed in
 * the backward pass).
 *   inputs     as for mssm_selective_scan_fwd, plus dout [Bt, D, L] dtype of u
 *   du, ddelta [Bt, D, L] dtype of u, written (ddelta: with respect to delta before
 *              the bias and softplus)
 *   dz         [Bt, D, L] dtype of u, written; given exactly when z is
 *   dA         [D, N] f32; dB, dC [Bt, N, L] f32 (summed over channels);
 *   dD, ddelta_bias [D] f32, given exactly when D / delta_bias are
 * The f32 gradients must be dense; they are zeroed and accumulated with atomic
 * adds, so their rounding order is not fixed.  Uses a per-device workspace of
 * 49 floats per chunk and row (about 196 x L / 64 bytes per row, twice that with
 * 32-step chunks), grown with cudaMalloc on demand (which synchronises the device)
 * and freed by mssm_shutdown().  L may reach 65535 x 64 steps.
 */
mssm_status mssm_selective_scan_bwd(const mssm_tensor *u, const mssm_tensor *delta, const mssm_tensor *A,
                                    const mssm_tensor *B, const mssm_tensor *C, const mssm_tensor *D,
                                    const mssm_tensor *z, const mssm_tensor *delta_bias, int softplus_flag,
                                    const mssm_tensor *dout, mssm_tensor *du, mssm_tensor *ddelta,
                                    mssm_tensor *dA, mssm_tensor *dB, mssm_tensor *dC, mssm_tensor *dD,
                                    mssm_tensor *dz, mssm_tensor *ddelta_bias, void *stream);

/*
 * Causal depthwise conv1d + SiLU: the step that produces the scan's input u from
 * the in-projection's x branch ("Linear Attention vs Softmax Attention ...",
 * section Implementation: the listed layer's grouped Conv1d with one group per
 * channel, kernel size K, padding K - 1, the output truncated to the first L
 * steps, then SiLU):
 *
 *   out[b,d,t] = act(bias[d] + sum_{k<K} weight[d,k] * x[b,d,t-(K-1)+k]),  x = 0 before t = 0
 *
 *   x, out      [Bt, D, L]  bf16|f32 (same dtype), L stride 1; out must not alias x
 *   weight      [D, K] f32, 1 <= K <= 4;   bias [D] f32 or NULL
 *   cu_seqlens  NULL, or [S + 1] int32 DEVICE offsets of packed sequences in a
 *               [1, D, T] x (as in mssm_scan_ext): every sequence sees zeros before
 *               its own first step; out outside every sequence is left unwritten
 *   max_seqlen  host bound on the sequence lengths (read only with cu_seqlens)
 *   silu_flag   1: act = SiLU, 0: identity
 * Inconsistent offsets are clamped and reported by mssm_get_error
 * (MSSM_ERR_INVALID_ARG).  The output is written in the scan's u layout.
 */
mssm_status mssm_causal_conv1d_fwd(const mssm_tensor *x, const mssm_tensor *weight, const mssm_tensor *bias,
                                   const mssm_tensor *cu_seqlens, int64_t max_seqlen, int silu_flag,
                                   mssm_tensor *out, void *stream);

/*
 * One decode step of the same conv, conv_state updated IN PLACE:
 *   conv_state [Bt, D, K-1]  dtype of x: the previous K-1 inputs, oldest first
 *   x, out     [Bt, D]       bf16|f32
 *   weight [D, K] f32 with 2 <= K <= 4;  bias [D] f32 or NULL
 * out = act(bias + sum_k weight[d,k] * window[k]) over window = [conv_state, x];
 * conv_state then drops its oldest input and appends x.  Steps from a zero state
 * reproduce mssm_causal_conv1d_fwd step by step.
 */
mssm_status mssm_causal_conv1d_update(mssm_tensor *conv_state, const mssm_tensor *x, const mssm_tensor *weight,
                                      const mssm_tensor *bias, int silu_flag, mssm_tensor *out, void *stream);

/* Static, human-readable name of a status code. */
const char *mssm_status_string(mssm_status status);

/* Detailed message of the last non-OK status returned on the calling thread ("" if none). */
const char *mssm_last_error(void);

/*
 * Synchronises `stream` and reports an asynchronous failure of the work queued
 * on it: MSSM_ERR_CUDA (with the CUDA error text in mssm_last_error());
 * MSSM_ERR_TIMEOUT when a bounded device-side wait gave up since the last call
 * (the decode kernels wait, with an iteration limit, for their own bulk copies
 * and on giving up leave that tile's state rows unchanged; the chained scan
 * schedule waits for the previous chunk's carried state and on giving up runs
 * the chunk from zero); MSSM_ERR_INVALID_ARG when a scan met inconsistent
 * cu_seqlens.  Clears the device error word.  No kernel waits on the host.
 */
mssm_status mssm_get_error(void *stream);

/*
 * Tuning / diagnostic options (process-wide; take effect on the next call):
 *   MSSM_OPT_FORCE_GENERAL_A (value 0/1): when 1, never use the structured-A
 *     path (A[d,n] == (n+1) * A[d,0] exactly, which computes exp(delta*A[d,n])
 *     as powers of one exponential); every state then takes its own exponential.
 *   MSSM_OPT_CHUNK_LEN (value 0, or a positive multiple of 64): length of the
 *     chunks a sequence is split into (a value >= L means no split); 0 restores
 *     the automatic choice.
 *   MSSM_OPT_SCHEDULE (value 0..5): 0 automatic; otherwise force a schedule of
 *     mssm_scan_plan (value = schedule + 1: 1 forward only, no split; 2 summaries
 *     + forward; 3 chained; 4 fused single pass; 5 split chunks).  A forced split
 *     schedule needs L > 64; otherwise the plan falls back to forward only.  The
 *     fused and split-chunk schedules take plain batches only, and the split-chunk
 *     schedule chunk lengths that are multiples of 256 (4 sub-segments of whole
 *     64-step blocks); otherwise the plan falls back to forward only.
 *   MSSM_OPT_KERNEL_TIMING (value 0/1): when 1, every kernel launch is bracketed
 *     by two CUDA events recorded on the caller's stream (see mssm_kernel_stats).
 *   MSSM_OPT_DECODE_PATH (value 0..3): the state-update kernel.  0 automatic:
 *     the first of 1, 2, 3 whose layout conditions hold.  1 persistent streaming
 *     kernel (per warp a block of 32 channels and a ring of bulk-copied tiles);
 *     needs the state as one contiguous, 16-byte aligned [Bt, D, 16] range, x,
 *     dt and z with unit channel stride and 16-byte aligned batch rows, D a
 *     multiple of 8 (bf16) or 4 (f32), and B, C with unit n stride and 16-byte
 *     aligned batch rows.  2 one bulk-copied tile of 256 rows per CTA; needs the
 *     contiguous state.  3 one thread per row, any layout.  A forced path whose
 *     conditions fail falls back to the next one that holds.
 *   MSSM_OPT_ROWS_PER_CTA (value 0, 32, 64 or 128): channels per row tile of the
 *     scan plan; 0 automatic.  With one channel per thread a tile is one CTA of
 *     32 or 64 threads; with two channels per thread (bf16 I/O only) a 64- or
 *     128-channel tile is a CTA of 32 or 64 threads.  The chained, fused and
 *     split-chunk schedules take tiles of one warp (32 channels, or 64 with two
 *     per thread).
 *   MSSM_OPT_ROWS_PER_THREAD (value 0, 1 or 2): channels each thread of the scan
 *     kernels keeps in registers (each step's B and C are then read once for
 *     all of them); 0 automatic.  Two per thread exist for bf16 I/O only; for
 *     fp32 I/O a forced 2 means 1.
 *   MSSM_OPT_TEST_HOOKS (value 0/1, for testing failure detection only): when 1,
 *     the chained scan schedule publishes no carried states, so every chunk after
 *     the first gives up its bounded wait (about 0.5 s), runs from a zero state
 *     and sets the device error word; mssm_get_error then reports
 *     MSSM_ERR_TIMEOUT.  No fault, trap or unbounded wait is involved.
 * Unknown options or invalid values return MSSM_ERR_INVALID_ARG.
 */
typedef enum {
    MSSM_OPT_FORCE_GENERAL_A = 1,
    MSSM_OPT_CHUNK_LEN = 2,
    MSSM_OPT_KERNEL_TIMING = 3,
    MSSM_OPT_SCHEDULE = 4,
    MSSM_OPT_DECODE_PATH = 5,
    MSSM_OPT_TEST_HOOKS = 6,
    MSSM_OPT_ROWS_PER_CTA = 7,
    MSSM_OPT_ROWS_PER_THREAD = 8
} mssm_option;
mssm_status mssm_set_option(int option, int64_t value);

/*
 * Host-only query of the launch plan mssm_selective_scan_fwd would use for a
 * [Bt, D, L] problem with bf16 I/O on a GPU with sm_count SMs (sm_count <= 0:
 * the current device, or 148 when there is none): channels per row tile (32, 64
 * or 128), chunk length,
 * number of chunks (1 = no split) and schedule: 0 = one forward kernel,
 * 1 = chunk-summary kernel + forward kernel, 2 = persistent chained forward
 * kernel (chunks of a tile run in order, each starting from the state the
 * previous one published), 3 = fused single pass (one persistent kernel: every
 * chunk summarises itself, looks back over the published summaries of the
 * chunks before it for its start state, then runs forward), 4 = split chunks
 * (one persistent kernel of 4-warp CTAs: the warps summarise the 4 sub-segments
 * of a chunk, combine the summaries in shared memory with the chunk's incoming
 * state, which the previous chunk hands over, and sweep their sub-segments
 * forward).  Honours MSSM_OPT_CHUNK_LEN.  Launches nothing; any
 * output pointer may be NULL.
 */
mssm_status mssm_scan_plan(int64_t Bt, int64_t D, int64_t L, int sm_count, int *rows_per_cta,
                           int64_t *chunk_len, int64_t *n_chunks, int *schedule);

/*
 * The same query for S packed sequences of at most max_seqlen steps summing to
 * total_len (the T of mssm_scan_ext.cu_seqlens; total_len < 0: S full sequences).
 */
mssm_status mssm_scan_plan_packed(int64_t S, int64_t D, int64_t max_seqlen, int64_t total_len, int sm_count,
                                  int *rows_per_cta, int64_t *chunk_len, int64_t *n_chunks, int *schedule);

/* The full launch plan of a scan (mssm_scan_plan_query). */
typedef struct {
    int32_t struct_size;      /* sizeof(mssm_scan_plan_info), set by the caller */
    int32_t schedule;         /* 0..4, as mssm_scan_plan reports it */
    int32_t rows_per_cta;     /* channels per row tile: 32, 64 or 128 */
    int32_t rows_per_thread;  /* channels per thread: 1 or 2 (2: bf16 I/O only) */
    int64_t chunk_len;        /* steps per chunk of the length split */
    int64_t n_chunks;         /* chunks per sequence (1 = no split) */
    int32_t grid;             /* persistent CTAs of the chained and fused schedules, else 0 */
    int32_t reserved;
} mssm_scan_plan_info;

/*
 * The plan mssm_selective_scan_fwd (and _ex) would use for S sequences of at
 * most max_seqlen steps (total_len: their summed length for packed sequences,
 * < 0 for S full sequences) of D channels with I/O dtype io_dtype (MSSM_F32 or
 * MSSM_BF16) on a GPU with sm_count SMs (<= 0: the current device, or 148).
 * Honours the tuning options below.  Host only; launches nothing.  Returns
 * MSSM_ERR_INVALID_ARG for a null info, a struct_size below this version's
 * size, negative sizes or another dtype.
 */
mssm_status mssm_scan_plan_query(int64_t S, int64_t D, int64_t max_seqlen, int64_t total_len, int io_dtype,
                                 int sm_count, mssm_scan_plan_info *info);

/* Kernel kinds counted by mssm_kernel_stats. */
typedef enum {
    MSSM_KERNEL_SCAN_CHUNK_STATE = 0, /* chunk summaries + carry fold (split scans only) */
    MSSM_KERNEL_SCAN_OUT = 1,         /* forward sweep with fused epilogue */
    MSSM_KERNEL_STATE_UPDATE = 2,     /* decode step */
    MSSM_KERNEL_CONV = 3,             /* causal conv1d (prefill and decode step) */
    MSSM_KERNEL_SCAN_BWD = 4,         /* backward scan (both of its passes) */
    MSSM_KERNEL_KINDS = 5
} mssm_kernel_kind;

/*
 * Diagnostics: per kernel kind, the number of launches issued so far
 * (`launches`), and, for launches made while MSSM_OPT_KERNEL_TIMING was on, how
 * many were timed (`timed`) and their summed device duration in ms (`ms`).
 * Waits for the pending timing events.  Any output pointer may be NULL (each
 * non-NULL one is an array of MSSM_KERNEL_KINDS).  reset != 0 zeroes the
 * counters afterwards.
 */
mssm_status mssm_kernel_stats(int64_t *launches, int64_t *timed, double *ms, int reset);

/*
 * Frees the library's per-device workspaces and forgets the device addresses it
 * cached (of the no-allocation scratch array and of the error word).  Call it
 * with no work in flight, and before any cudaDeviceReset: a reset unloads the
 * library's device module, and addresses cached from before it would be stale.
 * The library may be used again afterwards; it looks the addresses up anew.
 */
mssm_status mssm_shutdown(void);

/* Library version, "major.minor.patch". */
const char *mssm_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MSSM_H */
