/*
 * sparse_attn.h -- C ABI of the structured sparse causal attention library
 * (sm_100a / B200).
 *
 * The operation ("Depth-Staggered Fibonacci Spacing for Sparse Attention:
 * Static Schedules Beat Learned Dilation and Extrapolate Where Dense
 * Attention Fails", C. A. Capps; technical summary, section "Methodology"):
 * for every layer l, batch b, head h and query position i, attention over
 *   - the dense causal window  j = i, i-1, ..., i-W+1       ("Attended set"),
 *   - S sink keys             j = 0 .. S-1 with j <= i     (optional),
 *   - one member per offset f_k (the Fibonacci ladder 1, 2, 3, 5, ..., 987 by
 *     default), at distance d_k = alpha_l * f_k             ("Scaling"),
 *     linearly interpolated between rows when d_k is not an integer, with RoPE
 *     applied to K (and Q) before the gather               ("Implementation").
 * Exact arithmetic conventions (the library's reading of what the page leaves
 * open):
 *   d_k = fp32 product alpha_l * (float)f_k;  lo = floor(d_k);  w = d_k - lo;
 *   offset k exists for query i iff i - ceil(d_k) >= 0;
 *   key_k = (1-w) RoPE(K)[i-lo] + w RoPE(K)[i-lo-1], value_k likewise from V
 *   (the second row is not read when w == 0);
 *   q_hat_i = scale * RoPE(Q)[i]; score = q_hat_i . key; one softmax over all
 *   members (duplicates are separate members); O_i = sum_m p_m value_m;
 *   LSE_i = log sum_m exp(score_m);
 *   RoPE: rotate-half pairs (j, j + D/2), angle pos * rope_base^(-2j/D), taken
 *   in double precision and rounded to fp32;
 *   an offset whose d_k lies outside [0, 2^24) (negative or NaN alpha, or one
 *   so large that the product overflows the range) has no defined row: the
 *   whole layer's outputs become NaN (no row is read for it).
 *
 * Tensors.  Q, K, V, O, dO, dQ, dK, dV are contiguous [L][B][H][T][D] arrays
 * (D innermost) of the element type params.dtype, in DEVICE memory, 16-byte
 * aligned.  LSE is a device fp32 [L][B][H][T] array; alpha and dalpha are
 * device fp32 [L] arrays (these three need 4-byte alignment).  Accumulation is
 * always fp32.
 *
 * Ownership.  The caller owns every buffer it passes (inputs, outputs and the
 * workspace) and keeps them alive until the work queued on `stream` has
 * finished.  On the first call for a given (device, T, D, rope_base) the
 * library computes a RoPE cos/sin table on the device and keeps it, in memory
 * it allocates once and releases at process exit; no other call allocates.
 *
 * Streams and errors.  Every call only enqueues kernels on `stream` (a
 * cudaStream_t passed as void*, NULL = the legacy default stream) and returns
 * without waiting.  Argument errors are detected on the host before anything
 * is enqueued and return SA_ERR_INVALID_ARG / SA_ERR_UNSUPPORTED /
 * SA_ERR_WORKSPACE; a failed launch returns SA_ERR_CUDA.  Nothing throws
 * across this boundary and no call aborts the process.
 */
#ifndef SPARSE_ATTN_H
#define SPARSE_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SA_OK = 0,
  SA_ERR_INVALID_ARG = 1,  /* null pointer, bad shape, misaligned, f_k < 1, ... */
  SA_ERR_UNSUPPORTED = 2,  /* valid but not built: D not in {16,32,64,128}, ... */
  SA_ERR_WORKSPACE = 3,    /* workspace smaller than sparse_attn_workspace_size() */
  SA_ERR_CUDA = 4,         /* a CUDA runtime call or a launch failed */
  SA_ERR_INTERNAL = 5
} sa_status;

typedef enum { SA_DTYPE_F32 = 0, SA_DTYPE_BF16 = 1 } sa_dtype;

/* Problem description.  All fields are read during the call only. */
typedef struct {
  int32_t L, B, H, T, D;   /* layers, batch, heads, sequence length, head dim   */
  int32_t window;          /* W >= 1: keys i-W+1 .. i (the query itself included) */
  int32_t n_offsets;       /* 0 .. SA_MAX_OFFSETS                                 */
  const int32_t* offsets;  /* HOST array of n_offsets values f_k >= 1 (may be
                              NULL when n_offsets == 0); copied during the call  */
  int32_t n_sinks;         /* S >= 0: keys 0 .. S-1 always attended (when j <= i) */
  float rope_base;         /* > 0, e.g. 10000                                     */
  float scale;             /* score scale; <= 0 selects 1/sqrt(D)                 */
  sa_dtype dtype;          /* element type of Q, K, V, O, dO, dQ, dK, dV          */
} sa_params;

#define SA_MAX_OFFSETS 32
#define SA_MAX_SINKS 16

/*
 * Bytes of device workspace that sparse_attn_fwd (backward = 0) or
 * sparse_attn_bwd (backward = 1) needs for these params; 0 when none.
 * Returns 0 as well for invalid params (the call itself then reports why).
 */
size_t sparse_attn_workspace_size(const sa_params* p, int backward);

/*
 * Forward: O and (when lse != NULL) LSE for all L layers in one call.
 *   q, k, v : device [L][B][H][T][D], dtype p->dtype           (read)
 *   alpha   : device fp32 [L], the per-layer offset scale       (read)
 *   o       : device [L][B][H][T][D], dtype p->dtype            (written)
 *   lse     : device fp32 [L][B][H][T] or NULL                  (written)
 *   workspace / workspace_bytes: device scratch of at least
 *             sparse_attn_workspace_size(p, 0) bytes, 16-byte aligned (may be
 *             NULL if 0).  The bf16 / D = 64 path keeps the RoPE-rotated keys
 *             there (L*B*H*T*D 16-bit values); other configurations need none.
 * Source: "Depth-Staggered Fibonacci Spacing for Sparse Attention",
 * Methodology -- "Attended set", "Scaling", "Implementation".
 */
sa_status sparse_attn_fwd(const sa_params* p, const void* q, const void* k, const void* v,
                          const float* alpha, void* o, float* lse,
                          void* workspace, size_t workspace_bytes, void* stream);

/*
 * Backward of sparse_attn_fwd for the upstream gradient dout.
 *   q, k, v, o, dout : device [L][B][H][T][D], dtype p->dtype   (read)
 *   lse              : device fp32 [L][B][H][T] from the forward (read)
 *   alpha            : device fp32 [L]                          (read)
 *   dq, dk, dv       : device [L][B][H][T][D], dtype p->dtype   (overwritten)
 *   dalpha           : device fp32 [L], overwritten with
 *                      sum over (b, h, i, k) of dLoss/dw_k * f_k, the gradient
 *                      to alpha through the interpolation weight w_k (floor
 *                      held fixed: at an integer d_k this is the derivative
 *                      from above; a second row i-lo-1 < 0 contributes 0).
 *   workspace        : at least sparse_attn_workspace_size(p, 1) bytes.
 * No atomics: every output element is written by exactly one thread and the
 * per-layer dalpha is summed in a fixed order, so results are deterministic.
 * Source: same passages; the page states that the interpolation lets
 * gradients reach alpha ("Implementation") and trains alpha per layer
 * ("Experimental variables", learned schedule).
 */
sa_status sparse_attn_bwd(const sa_params* p, const void* q, const void* k, const void* v,
                          const void* o, const float* lse, const void* dout,
                          const float* alpha, void* dq, void* dk, void* dv, float* dalpha,
                          void* workspace, size_t workspace_bytes, void* stream);

/*
 * Training pair: a forward that also saves what the backward would otherwise
 * recompute, and the backward that consumes it.  This is activation saving
 * (the paper has no counterpart; its training runs a forward and a backward
 * per step): the forward keeps, in the caller's `context` buffer,
 *   - the RoPE-rotated keys (fp16 of RoPE(K) / 256, [L][B][H][T][D]),
 *   - the rotated, scaled queries (fp16 of RoPE(Q) * scale / 256, same layout),
 *   - every member's softmax probability (window lags 0..W-1 unfolded, sinks,
 *     offsets in the order of p->offsets sorted ascending), fp32
 *     [L*B*H][W+S+n_offsets][T],
 *   - every offset's row-score difference score(row i-lo-1) - score(row i-lo),
 *     fp32 [L*B*H][n_offsets][T],
 * and sparse_attn_bwd_ctx then skips the score pass and both rotation pre-passes.
 * Results equal sparse_attn_fwd / sparse_attn_bwd up to fp32 rounding order.
 *
 * sparse_attn_context_size: bytes of the context for these params; 0 when
 * the configuration has no staged kernels (dtype other than bf16 or D != 64):
 * the two calls then return SA_ERR_UNSUPPORTED (use sparse_attn_fwd/_bwd).
 * sparse_attn_fwd_train: arguments as sparse_attn_fwd, plus the context
 * (device, >= sparse_attn_context_size bytes, 16-byte aligned; written).
 * sparse_attn_bwd_ctx: arguments as sparse_attn_bwd plus the context written
 * by sparse_attn_fwd_train for the same q, k, v, alpha and params (read; lse
 * may be NULL); its workspace is sparse_attn_workspace_size(p, 1) bytes.
 * Both run the staged kernels whatever sparse_attn_force_general says.
 */
size_t sparse_attn_context_size(const sa_params* p);
sa_status sparse_attn_fwd_train(const sa_params* p, const void* q, const void* k, const void* v,
                                const float* alpha, void* o, float* lse, void* context,
                                size_t context_bytes, void* stream);
sa_status sparse_attn_bwd_ctx(const sa_params* p, const void* q, const void* k, const void* v,
                              const void* o, const float* lse, const void* dout,
                              const float* alpha, const void* context, void* dq, void* dk,
                              void* dv, float* dalpha, void* workspace, size_t workspace_bytes,
                              void* stream);

/*
 * Log-prior on the offset members.  "pi-Attention: Periodic Sparse
 * Transformers for Efficient Long-Context Modeling" (Core components, dynamic
 * adaptive fusion) merges its local and skip logits into one softmax by adding
 * a log-prior in the log domain.  A softmax ignores a shift common to all of a
 * query's members, so only the difference of the two priors matters.  Here
 * one value beta_i per query is added to the score of every offset member of
 * query i.  The window and the sinks get 0.  beta_i = ln 2 weighs each offset
 * member as if it were listed twice; beta_i -> -inf removes the offsets.
 *   beta  : device fp32 [L][B][H][T]                              (read)
 *   dbeta : device fp32 [L][B][H][T], overwritten with
 *           dLoss/dbeta_i = sum over query i's offset members of dLoss/dscore
 *                                                                 (written)
 * sparse_attn_fwd_prior: arguments as sparse_attn_fwd plus beta. context
 *   NULL runs the plain forward, with the same kernel choice as
 *   sparse_attn_fwd. A non-NULL context runs the training forward (as
 *   sparse_attn_fwd_train): the saved probabilities include the prior, and
 *   workspace is unused.
 * sparse_attn_bwd_prior: arguments as sparse_attn_bwd plus beta (the
 *   forward's), an optional context (from sparse_attn_fwd_prior with the same
 *   beta; lse may then be NULL) and dbeta.
 * beta, dbeta: non-NULL, 4-byte aligned, else SA_ERR_INVALID_ARG.  Decode
 * takes the prior through sparse_attn_decode_prior; the allocation-free
 * forward takes none.
 */
sa_status sparse_attn_fwd_prior(const sa_params* p, const void* q, const void* k, const void* v,
                                const float* alpha, const float* beta, void* o, float* lse,
                                void* workspace, size_t workspace_bytes, void* context,
                                size_t context_bytes, void* stream);
sa_status sparse_attn_bwd_prior(const sa_params* p, const void* q, const void* k, const void* v,
                                const void* o, const float* lse, const void* dout,
                                const float* alpha, const float* beta, const void* context,
                                void* dq, void* dk, void* dv, float* dalpha, float* dbeta,
                                void* workspace, size_t workspace_bytes, void* stream);

/*
 * Single-token decode with a KV cache: for every (layer, batch, head), the
 * attention output of one new query at position `pos` against the cache rows
 * 0..pos (the new token's own K/V row, at pos, included).  The result equals
 * row `pos` of sparse_attn_fwd on the first pos + 1 rows with that query in
 * row pos.  Source: the attended set, scaling and interpolation of
 * "Depth-Staggered Fibonacci Spacing for Sparse Attention" (Methodology);
 * the page measures inference latency for this gather (Results, efficiency).
 *   p->T     : the cache length (rows allocated per unit); 0 <= pos < p->T
 *   q        : device [L][B][H][D], unrotated (rotated at pos here)     (read)
 *   k, v     : device [L][B][H][p->T][D] caches; only the rows the query
 *              attends are read (window, sinks, offset rows; all <= pos)  (read)
 *   alpha    : device fp32 [L]                                           (read)
 *   o        : device [L][B][H][D], dtype p->dtype                     (written)
 *   lse      : device fp32 [L][B][H] or NULL                           (written)
 * Any dtype and head dim of sparse_attn_fwd; no workspace.  Returns
 * SA_ERR_INVALID_ARG for pos outside [0, p->T) and SA_ERR_UNSUPPORTED for a
 * window above 256.
 */
sa_status sparse_attn_decode(const sa_params* p, int32_t pos, const void* q, const void* k,
                             const void* v, const float* alpha, void* o, float* lse,
                             void* stream);
/*
 * Decode with the log-prior of sparse_attn_fwd_prior: beta is the new
 * queries' prior, device fp32 [L][B][H], added to the score of each of their
 * offset members. NULL means none, as in sparse_attn_decode.
 */
sa_status sparse_attn_decode_prior(const sa_params* p, int32_t pos, const void* q, const void* k,
                                   const void* v, const float* alpha, const float* beta, void* o,
                                   float* lse, void* stream);

/*
 * Learned-alpha parametrisation.  The page trains "one free parameter theta
 * per layer, initialised at alpha = 1" and constrains alpha to [0.5, 1.5]
 * (Methodology: scaling; experimental variables); it does not give the map.
 * The map used here: alpha = 0.5 + sigmoid(theta), so theta = 0 gives
 * alpha = 1 and every theta lands inside the interval.
 *   sparse_attn_alpha_from_theta: alpha[l] = 0.5 + 1 / (1 + exp(-theta[l]))
 *   sparse_attn_dtheta: dtheta[l] = dalpha[l] * s (1 - s), s = sigmoid(theta[l])
 *     (dalpha as written by sparse_attn_bwd / sparse_attn_bwd_ctx).
 * theta, alpha, dalpha, dtheta: device fp32 [L], 4-byte aligned; fp32 math
 * with the CUDA exponential.  One launch each on `stream`.
 */
sa_status sparse_attn_alpha_from_theta(int32_t L, const float* theta, float* alpha,
                                       void* stream);
sa_status sparse_attn_dtheta(int32_t L, const float* theta, const float* dalpha, float* dtheta,
                             void* stream);

/*
 * Forward that allocates no device memory.  The paper has no counterpart: this
 * entry point exists for callers that cannot let a library call cudaMalloc --
 * applications whose device memory belongs to a pooling allocator that must
 * account for every byte, and embedders or latency-critical services that
 * forbid allocation after start-up.  It computes what sparse_attn_fwd
 * computes (same arguments minus the workspace), to within the same parity
 * tolerances but not bit for bit: with no workspace for rotated keys, bf16 /
 * D = 64 problems with windows up to 256 run the staged CUDA-core kernel with
 * the keys rotated in shared memory (sparse_attn_fwd may choose the
 * tensor-core kernel there), and all others the general kernels.  Its only
 * scratch, the RoPE cos/sin table, lives in a fixed file-scope device array
 * of SA_NOALLOC_SCRATCH_BYTES (8 MiB) that every GPU loading this library
 * holds until the process exits.
 *   Limit: T * (D/2) * 8 bytes must fit in SA_NOALLOC_SCRATCH_BYTES (for D=64,
 *   T <= 32768); larger problems return SA_ERR_UNSUPPORTED before any work.
 *   Set-up: the first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture.
 *   Sharing: every call on a device uses the same array and rewrites the part
 *   it needs on `stream` before reading it; calls that overlap on the GPU
 *   (for example on two streams) race on the array and must be serialised by
 *   the caller.
 * It calls no cudaMalloc, cudaFree or other allocating routine.
 */
#define SA_NOALLOC_SCRATCH_BYTES (8u << 20)
sa_status sparse_attn_fwd_noalloc(const sa_params* p, const void* q, const void* k,
                                  const void* v, const float* alpha, void* o, float* lse,
                                  void* stream);

/*
 * Device error word of the staged kernels.  Reading synchronises with the
 * device; with clear != 0 the word is reset.  Returns -1 on a CUDA error.
 *   bit 0: a bounded wait for a staging copy gave up (the kernel then left
 *          its outputs incomplete and returned rather than wait without end);
 *   bit 1: a row index outside the rows staged in shared memory, or a staging
 *          round larger than its ring -- checked only by the bounds-checking
 *          build (compiled with SA_DEBUG_BOUNDS), which records and skips the
 *          access;
 *   bit 2: a finite input beyond the range of the staged 16-bit operands:
 *          |RoPE(K)| / 256 (and, in the backward, |RoPE(Q)| * scale / 256)
 *          above 65504, i.e. rotated key or scaled query elements beyond about
 *          1.68e7; for the tensor-core forward also |RoPE(Q)| * scale above
 *          65504.  Outputs of such a call are not valid.
 */
int32_t sparse_attn_device_error(int clear);

/*
 * Diagnostics of the bounded waits (process wide, for tests):
 * sparse_attn_set_wait_limit sets how many SM clocks a staging wait waits
 * before it gives up (<= 0: the default, 1e9 clocks, about half a second).
 * With sparse_attn_plant_stall(1), every CTA of later staged launches expects
 * 16 bytes more in its first staging round than any copy delivers, so that
 * round's wait runs out: bit 0 of the device error word is set and the kernel
 * returns without finishing its outputs.  Nothing faults and nothing waits
 * beyond the limit.  Off (0) by default.
 */
void sparse_attn_set_wait_limit(long long clocks);
void sparse_attn_plant_stall(int on);

/*
 * Diagnostics: throughput probe of the fp32 FMA pipe, the peak of the ALU
 * roofline of the CUDA-core kernels (the paper has no counterpart).  Launches
 * `blocks` CTAs of `threads` threads (32..256, a multiple of 32); each thread
 * runs 8 independent register-only FMA chains of `iters` steps, scalar
 * fma.rn.f32 (packed = 0) or packed fma.rn.f32x2 (packed != 0), then writes one
 * float to out[blocks * threads] (device).  FLOPs per launch:
 * blocks * threads * iters * 8 * 2 * (packed ? 2 : 1).  The caller times it
 * (CUDA events on `stream`).  Returns SA_ERR_INVALID_ARG for bad sizes.
 */
sa_status sparse_attn_diag_fma_probe(int32_t blocks, int32_t threads, int32_t iters,
                                     int32_t packed, float* out, void* stream);

/* Static, NUL-terminated description of a status code. */
const char* sparse_attn_status_string(sa_status s);

/* Number of kernel launches the most recent successful fwd/bwd call on this
 * host thread enqueued (a diagnostic for counting launches). */
int32_t sparse_attn_last_launch_count(void);

/*
 * Diagnostics: with on != 0, every later call runs the general kernels (any
 * dtype and head dim) even where a specialised kernel exists (bf16, D = 64).
 * Process wide; off by default.  Used to test the two paths against each other.
 */
void sparse_attn_force_general(int on);

/*
 * Diagnostics: which bf16 / D = 64 forward kernel sparse_attn_fwd runs.
 * 0 (default): the faster for the configuration, as measured on B200: the
 * tensor-core kernel for windows of 48 or more, except where its shared
 * memory would leave it one CTA per SM while the CUDA-core kernel keeps two;
 * otherwise the CUDA-core kernel.  1: the CUDA-core staged kernel; 2: the
 * warp-level (mma.sync) tensor-core kernel where it applies (at most 16
 * sinks); 3: the fifth-generation tensor-core kernel (tcgen05 GEMMs for the
 * window band and the sinks, accumulators in tensor memory, offset members on
 * the CUDA cores) where it applies (at most 16 sinks, band plus sinks at most
 * 256 rows: W <= 113 with sinks, W <= 129 without), else as 0.  Other values
 * mean 0.  Process wide; sparse_attn_force_general takes precedence.
 */
void sparse_attn_select_forward(int which);

/*
 * Kernel tracing (diagnostics).  While enabled (on != 0), every kernel the
 * library enqueues is bracketed by two CUDA events recorded on the same
 * stream.  sparse_attn_trace_read waits for all recorded events, writes up to
 * `max` entries (static kernel name, total milliseconds, launch count), returns
 * the number of distinct kernels, and clears the record.  Tracing is process
 * wide and off by default; it costs two event records per launch.
 */
void sparse_attn_trace_enable(int on);
int32_t sparse_attn_trace_read(int32_t max, const char** names, double* total_ms,
                               int32_t* counts);

#ifdef __cplusplus
}
#endif

#endif /* SPARSE_ATTN_H */
