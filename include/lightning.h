/*
 * lightning.h: C ABI of liblightning, lightning attention for NVIDIA B200 (sm_100a).
 *
 * Lightning attention is causal linear attention with a per-head exponential
 * decay, computed tile by tile ("MiniMax-01: Scaling Foundation Models with
 * Lightning Attention | Summary", section 2.2 Linear Attention: masked
 * attention inside a tile, an accumulated key-value state for the tiles
 * before it; and section 3.3 for the inference kernels). For every head h with
 * slope s_h >= 0 and decay lam_h = exp(-s_h), and every token i:
 *
 *     O_i   = sum_{j <= i} lam_h^(i-j) (q_i . k_j) v_j
 *     state = sum_j lam_h^(N-1-j) k_j^T v_j            state[a][b], a: key dim, b: value dim
 *
 * There is no normalization, SiLU or gating inside the operator (the page's
 * derivation leaves them out as well).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - All tensor pointers are DEVICE pointers owned by the caller, 16-byte
 *   aligned, dense and row-major. The library never allocates device memory;
 *   scratch space is the caller's `workspace`.
 * - Shapes: q, k, v, o are [B][H][N][d] (head dim d = d_k = d_v); packed
 *   variable-length inputs are [H][total][d]; states are [B][H][d][d] fp32.
 * - `slopes` is a device fp32 array [H] (s_h, finite, >= 0: not checked,
 *   since checking needs a device read).
 * - dtypes: LA_BF16 inputs take LA_BF16 or LA_F32 outputs; LA_F32 inputs take
 *   LA_F32 outputs. Accumulation and states are always fp32.
 * - d must be 64 or 128.
 * - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *   default stream) and returns a synchronous status: argument errors are
 *   found before anything is launched. A device-side error (a bounded wait
 *   that timed out) is recorded in the workspace status word and read back by
 *   la_read_device_status().
 * - Calls that share a workspace must not overlap on the GPU.
 */
#ifndef LIGHTNING_H
#define LIGHTNING_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LA_API __attribute__((visibility("default")))

typedef struct CUstream_st* la_stream_t; /* same type as cudaStream_t */

typedef enum {
    LA_OK = 0,
    LA_ERR_INVALID_ARG = -1, /* null pointer, bad shape, misaligned pointer */
    LA_ERR_UNSUPPORTED = -2, /* valid request this build does not handle (e.g. d = 96) */
    LA_ERR_CUDA = -3,        /* a CUDA launch or runtime call failed */
    LA_ERR_TIMEOUT = -4,     /* device side: a bounded wait gave up */
    LA_ERR_WORKSPACE = -5    /* workspace missing or smaller than la_workspace_bytes() */
} la_status;

typedef enum { LA_BF16 = 0, LA_F32 = 1 } la_dtype;

/*
 * Size limits of every prefill, backward and mixed-step call (larger requests
 * return LA_ERR_UNSUPPORTED before anything is launched): N, or the packed
 * total, at most LA_MAX_TOKENS tokens (token coordinates are 32-bit in the
 * tensor-memory copies); B*H, or num_seqs*H, at most LA_MAX_PROBLEMS.
 */
#define LA_MAX_TOKENS ((long long)2147483647 - 256)
#define LA_MAX_PROBLEMS ((long long)1 << 28)

typedef enum {
    LA_OP_PREFILL = 0,
    LA_OP_PREFILL_VARLEN = 1,
    LA_OP_DECODE = 2,
    LA_OP_BACKWARD = 3
} la_op;

/*
 * Bytes of workspace an operation needs (0 for decode). For LA_OP_PREFILL and
 * LA_OP_BACKWARD pass B, H, N, d; for LA_OP_PREFILL_VARLEN pass H, total
 * tokens, d and num_seqs (B is ignored). The size depends only on these
 * arguments, the input dtype and the current tuning (la_set_tuning), never on
 * data. Returns 0 for invalid arguments.
 */
LA_API size_t la_workspace_bytes(int op, int B, int H, long long N_or_total, int d, int num_seqs,
                                 int in_t);

/*
 * Prefill: O and the final state for [B][H][N][d] inputs.
 * ("MiniMax-01 ... | Summary", section 2.2: tiles of the sequence, an
 * intra-tile masked product and an inter-tile product against the
 * accumulated state, which is updated after each tile.)
 *   q, k, v    in   [B][H][N][d], dtype in_t
 *   slopes     in   [H] fp32
 *   o          out  [B][H][N][d], dtype out_t
 *   state_out  out  [B][H][d][d] fp32, state after the last token; may be NULL
 *   workspace  scratch of at least la_workspace_bytes(LA_OP_PREFILL, ...) bytes
 * N may be 0 (then only state_out, all zeros, is written).
 */
LA_API int la_prefill(const void* q, const void* k, const void* v, const float* slopes, void* o,
                      float* state_out, int B, int H, long long N, int d, int in_t, int out_t,
                      void* workspace, size_t ws_bytes, la_stream_t stream);

/*
 * The final state alone, without outputs: the state of a prefix to cache
 * ("MiniMax-01 ... | Summary", section 3: cached prefixes that later inputs
 * continue from), or a chunk's local state in a sequence-parallel prefill
 * (section 3.2, LASP+). For every (sequence, head):
 *     state = lam^N S_in + sum_j lam^(N-1-j) k_j^T v_j
 *   k, v       in   [B][H][N][d], dtype in_t (no queries are needed)
 *   state_in   in   [B][H][d][d] fp32, or NULL for a zero state; may be the
 *                   same array as state_out
 *   state_out  out  [B][H][d][d] fp32, not NULL
 *   workspace  at least la_workspace_bytes(LA_OP_PREFILL, ...) bytes
 * Errors as for la_prefill. On the bf16 path it costs the state-update part
 * of a prefill: K and V are read once, no scores are formed.
 */
LA_API int la_prefill_state(const void* k, const void* v, const float* slopes,
                            const float* state_in, float* state_out, int B, int H, long long N,
                            int d, int in_t, void* workspace, size_t ws_bytes, la_stream_t stream);

/*
 * Prefill over packed variable-length sequences ("MiniMax-01 ... | Summary",
 * section 3.2: data packing concatenates samples; the state restarts at every
 * sample boundary). Sequence s covers tokens [cu_seqlens[s], cu_seqlens[s+1])
 * of the packed [H][total][d] tensors; it is never padded.
 *   cu_seqlens in   device int32 [num_seqs + 1], cu_seqlens[0] = 0, non-decreasing,
 *                   cu_seqlens[num_seqs] = total (not checked: needs a device read)
 *   state_out  out  [num_seqs][H][d][d] fp32, may be NULL
 * A zero-length sequence produces no rows and a zero state. num_seqs == 0 with
 * total > 0 is LA_ERR_INVALID_ARG (tokens that belong to no sequence).
 */
LA_API int la_prefill_varlen(const int* cu_seqlens, int num_seqs, const void* q, const void* k,
                             const void* v, const float* slopes, void* o, float* state_out, int H,
                             long long total, int d, int in_t, int out_t, void* workspace,
                             size_t ws_bytes, la_stream_t stream);

/*
 * Prefill continued from an incoming state: the inputs are the tokens that
 * follow a prefix whose state is already known (a cached prefix, or the
 * previous piece of a prefill cut into pieces; "MiniMax-01 ... | Summary",
 * section 3: inference inputs with cached prefixes that reuse the earlier
 * segments' computation, and section 3.3's batches of cached inputs). With
 * S_in the state after the prefix, for every (sequence, head):
 *     O_i   = lam^(i+1) q_i S_in + sum_{j <= i} lam^(i-j) (q_i . k_j) v_j
 *     state = lam^N S_in + sum_j lam^(N-1-j) k_j^T v_j
 * so that prefill(prefix) followed by this call on the rest gives the rows
 * and the final state of one prefill over the whole sequence.
 *   state_in   in   [B][H][d][d] fp32, not NULL; may be the same array as
 *                   state_out (the state is then advanced in place); any
 *                   other overlap with an output is undefined
 * Every other argument, result and error is as for la_prefill (N may be 0:
 * state_out then receives state_in).
 */
LA_API int la_prefill_with_state(const void* q, const void* k, const void* v,
                                 const float* slopes, const float* state_in, void* o,
                                 float* state_out, int B, int H, long long N, int d, int in_t,
                                 int out_t, void* workspace, size_t ws_bytes, la_stream_t stream);

/*
 * la_prefill_varlen continued from one incoming state per (sequence, head):
 *   state_in   in   [num_seqs][H][d][d] fp32, not NULL unless num_seqs == 0;
 *                   may be the same array as state_out
 * The operator per sequence is that of la_prefill_with_state; a zero-length
 * sequence's final state is its incoming state. Every other argument, result
 * and error is as for la_prefill_varlen; the workspace size is that of
 * LA_OP_PREFILL_VARLEN.
 */
LA_API int la_prefill_varlen_with_state(const int* cu_seqlens, int num_seqs, const void* q,
                                        const void* k, const void* v, const float* slopes,
                                        const float* state_in, void* o, float* state_out, int H,
                                        long long total, int d, int in_t, int out_t,
                                        void* workspace, size_t ws_bytes, la_stream_t stream);

/*
 * One decode step for a batch of B sequences ("MiniMax-01 ... | Summary",
 * section 3.3: the memory-bound single-token step, fused into one kernel):
 *     S <- lam_h S + k^T v     then     o = q S
 * (the new token is included in its own output).
 *   q, k, v      in      [B][H][d], dtype in_t
 *   state_inout  in/out  [B][H][d][d] fp32, updated in place
 *   o            out     [B][H][d], dtype out_t
 */
LA_API int la_decode(const void* q, const void* k, const void* v, const float* slopes,
                     float* state_inout, void* o, int B, int H, int d, int in_t, int out_t,
                     la_stream_t stream);

/*
 * One step over a batch of cached inputs of mixed lengths, with prefill and
 * decoding separated ("MiniMax-01 ... | Summary", section 3.3, Separated
 * Prefill and Decoding Execution: single-token inputs and longer inputs go to
 * different kernels on separate CUDA streams). Sequence s of the packed batch
 * continues from its state states[s] and covers tokens
 * [cu_seqlens[s], cu_seqlens[s+1]):
 *   - one-token sequences: the decode step (la_decode) on decode_stream;
 *   - longer sequences: the prefill from their states
 *     (la_prefill_varlen_with_state) on prefill_stream;
 *   - empty sequences: nothing (their states stay as they are).
 * The result is that of la_prefill_varlen_with_state over the whole batch.
 *   cu_seqlens  in      device int32 [num_seqs + 1] (as for la_prefill_varlen)
 *   q, k, v     in      [H][total][d], dtype in_t
 *   states      in/out  [num_seqs][H][d][d] fp32, advanced in place (NULL only when
 *                       num_seqs == 0)
 *   o           out     [H][total][d], dtype out_t
 *   workspace   at least la_workspace_bytes(LA_OP_PREFILL_VARLEN, ...) bytes;
 *               used on prefill_stream only (read its device status there)
 * The two parts touch disjoint rows and states. The call orders neither
 * stream after the other: the caller makes both wait for the work that
 * produced the inputs and waits for both before reading the outputs. The
 * streams may be the same stream (then the parts run one after the other).
 */
LA_API int la_mixed_step(const int* cu_seqlens, int num_seqs, const void* q, const void* k,
                         const void* v, const float* slopes, float* states, void* o, int H,
                         long long total, int d, int in_t, int out_t, void* workspace,
                         size_t ws_bytes, la_stream_t prefill_stream, la_stream_t decode_stream);

/* Most chunks (ranks) la_state_prefix takes. */
#define LA_MAX_CHUNKS 64

/*
 * Global prefix of a sequence-parallel prefill ("MiniMax-01 ... | Summary",
 * section 3.2, LASP+: the sequence is cut into R consecutive chunks, one per
 * rank; each rank summarizes its chunk locally, the summaries are gathered
 * (one all-gather), and each rank builds the state before its chunk). With
 * S_p the state of chunk p alone (la_prefill's state_out on that chunk) and
 * n_p its length:
 *     out = S_in(r) = sum_{p<r} lam^(n_{p+1} + ... + n_{r-1}) S_p
 * the state after chunks 0..r-1, which la_prefill_with_state then continues
 * from for chunk r (r = 0 gives zeros; r = R gives the whole sequence's state).
 *   states  in   [R][B][H][d][d] fp32 device, the gathered local states
 *   slopes  in   [H] fp32 device
 *   lens    in   HOST int64 [R], chunk lengths (>= 0)
 *   R, r    1 <= R <= LA_MAX_CHUNKS, 0 <= r <= R
 *   out     out  [B][H][d][d] fp32 device, must not overlap states
 * No workspace.
 */
LA_API int la_state_prefix(const float* states, const float* slopes, const long long* lens, int R,
                           int r, int B, int H, int d, float* out, la_stream_t stream);

/*
 * Output normalization and gate, the step after the operator ("MiniMax-01 ...
 * | Summary", section 2.2: the linear-attention output passes through a
 * normalization, and the blocks gate it; the page gives neither form). This
 * library takes an RMS normalization over all H*d features of a token and a
 * sigmoid gate, and turns the head-major output into token-major rows:
 *     r_{b,n}          = 1 / sqrt( mean_{h,c} O[b][h][n][c]^2 + eps )
 *     Y[b][n][h d + c] = w[h d + c] * O[b][h][n][c] * r_{b,n} * sigmoid(G[b][n][h d + c])
 *   o       in   [B][H][N][d], dtype o_t (the prefill's output; varlen: B = 1, N = total)
 *   gate    in   [B][N][H*d], dtype y_t
 *   weight  in   [H*d] fp32
 *   eps     in   >= 0 and finite
 *   y       out  [B][N][H*d], dtype y_t; must not overlap o or gate
 * LA_ERR_UNSUPPORTED when H*d > 16384 or B*N > LA_MAX_TOKENS. No workspace;
 * N may be 0.
 */
LA_API int la_output_norm_gate(const void* o, const void* gate, const float* weight, float eps,
                               void* y, int B, int H, long long N, int d, int o_t, int y_t,
                               la_stream_t stream);

/*
 * Gradients of L = <dO, O> with respect to q, k and v for [B][H][N][d]
 * inputs (the pages state no backward pass; these are the derivatives of the
 * operator above):
 *     dQ_i = sum_{j<=i} lam^(i-j) (dO_i . v_j) k_j
 *     dK_j = sum_{i>=j} lam^(i-j) (dO_i . v_j) q_i
 *     dV_j = sum_{i>=j} lam^(i-j) (q_i . k_j) dO_i
 *   dO, q, k, v  in   dtype in_t
 *   dq, dk, dv   out  dtype out_t
 * No gradient is produced for slopes or for an incoming state.
 */
LA_API int la_backward(const void* dO, const void* q, const void* k, const void* v,
                       const float* slopes, void* dq, void* dk, void* dv, int B, int H,
                       long long N, int d, int in_t, int out_t, void* workspace, size_t ws_bytes,
                       la_stream_t stream);

/* Human-readable name of a status code (static string). */
LA_API const char* la_status_string(int status);

/*
 * Synchronizes `stream`, then returns the device-side status recorded in
 * `workspace` by the last call that used it (LA_OK, or LA_ERR_TIMEOUT when a
 * bounded inter-CTA wait gave up; that call's outputs are then invalid).
 */
LA_API int la_read_device_status(const void* workspace, la_stream_t stream);

/*
 * Process-wide tuning, for invariance tests and experiments (0 = default).
 *   block_tokens    tile length C of the fp32 path: 32, 64 or 128
 *   segment_tokens  tokens per chunk of the chunk-parallel state scan of the
 *                   bf16 path: a multiple of 128, or 0 for automatic
 * Not thread-safe with concurrent calls. Returns LA_ERR_INVALID_ARG for bad values.
 */
LA_API int la_set_tuning(int block_tokens, int segment_tokens);
LA_API int la_get_tuning(int* block_tokens, int* segment_tokens);

/* Number of kernels the last call on this host thread launched (for accounting). */
LA_API int la_last_launch_count(void);

/*
 * Test-only fault injection for the chunk-parallel state scan of the bf16
 * path, set on the host (process-wide, not thread-safe with concurrent calls).
 *   skip_publish   non-zero: segments never signal that their prefix state is
 *                  ready, so every later segment's bounded wait runs out
 *   wait_limit_us  bound of that wait in microseconds (0 = default, 2 s)
 * An expired wait is reported as LA_ERR_TIMEOUT by la_read_device_status;
 * the outputs of that call are then invalid, the CUDA context stays usable.
 * Call la_set_fault_injection(0, 0) to restore normal operation.
 */
LA_API int la_set_fault_injection(int skip_publish, int wait_limit_us);

/*
 * Size in bytes of the scratch array built into the library for
 * la_prefill_noalloc (16 MiB).
 */
#define LA_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)

/*
 * la_prefill without a caller-supplied workspace. The pages have no
 * counterpart: this entry point exists for callers that cannot allocate
 * device memory (a C or embedded host program without a device allocator, a
 * plugin whose host application forbids allocations after start-up, a
 * latency-critical loop that must not call cudaMalloc).
 *
 * Same arguments, results and errors as la_prefill, minus the workspace.
 * A device-side error of the call (a bounded wait of the state scan that gave
 * up) is written into the built-in scratch, not into a caller's workspace:
 * read it with la_noalloc_device_status. The scratch is a fixed array of LA_NOALLOC_SCRATCH_BYTES in device memory that
 * every GPU which loads the library holds until the process exits. Requests
 * whose la_workspace_bytes(LA_OP_PREFILL, ...) exceeds that size are refused
 * with LA_ERR_WORKSPACE before any GPU work (for bf16 inputs with d = 128 the
 * scratch covers up to 127 (sequence, head) pairs, B*H; the fp32 path needs
 * only a few hundred bytes).
 *
 * The first call on a device looks up the array's device address (with that
 * device current); make that first call before any stream capture. The
 * function allocates nothing (no cudaMalloc, cudaFree or allocating library
 * routine). All calls share the one array, which keeps the last call's
 * contents; each call clears what must start at zero on its own stream. Calls
 * that overlap on the GPU (other streams, other host threads) race on the
 * array: serialize them.
 */
LA_API int la_prefill_noalloc(const void* q, const void* k, const void* v, const float* slopes,
                              void* o, float* state_out, int B, int H, long long N, int d,
                              int in_t, int out_t, la_stream_t stream);

/*
 * Device-side status of the last la_prefill_noalloc on the current device.
 * This is la_read_device_status for the built-in scratch, and has no
 * counterpart on the pages either. It synchronizes `stream` (the stream the
 * call ran on), then copies the status word out of the scratch into host
 * memory: LA_OK, or LA_ERR_TIMEOUT when a bounded wait of the state scan gave
 * up (that call's outputs are then invalid; the context stays usable).
 * Returns LA_ERR_CUDA if the synchronization or the copy fails. Allocates
 * nothing. A later la_prefill_noalloc on the device overwrites the word.
 */
LA_API int la_noalloc_device_status(la_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* LIGHTNING_H */
