/*
 * specverify.h -- C ABI of the B200 (sm_100a) speculative-decoding
 * verification sampler, libspecverify.so.
 *
 * What the calls compute ("Accelerating Sonar through speculation",
 * Perplexity 2025, section "Speculative decoding": after the draft stage come
 * the acceptance stage and the target-generation stage; section
 * "Target-Draft": acceptance compares the full draft and target
 * distributions, and the target always yields one more set of logits after
 * the accepted drafts; "Speculative decoding explained", section "Draft and
 * verification loop": a draft is accepted outright when the target is at
 * least as confident, otherwise with a probability that falls as the gap
 * grows, and a rejected draft is replaced by a token drawn from an adjusted
 * distribution, which keeps the target's output distribution exactly).
 * The exact rule, as in Leviathan, Kalman & Matias, "Fast inference from
 * transformers via speculative decoding": accept draft x with probability
 * min(1, p(x)/q(x)); at the first rejection resample from
 * norm(max(0, p - q)); if nothing is rejected, sample the bonus token from
 * the last target row.
 *
 * Notation: B requests, k drafts per request, V vocabulary entries, T
 * temperature.  p_j = softmax(target_row_j / T), q_j = softmax(draft_row_j / T).
 *
 * Conventions shared by every call:
 *   - Every pointer argument is caller-owned DEVICE memory (global memory of
 *     the current device), except where a comment says otherwise.  The
 *     library makes no allocation at run time and never synchronises: all
 *     work is enqueued on `stream` and the outputs are valid when the
 *     stream reaches that point.  Apart from launch settings cached per
 *     device, it keeps no state between calls; the one exception is
 *     spec_verify_linear_noalloc, whose calls share a static device array
 *     (see there).
 *   - Logit tensors are row-major [B][rows][row_stride] of fp32 or bf16.
 *     Only columns [0, V) of a row are read as vocabulary.  row_stride * the
 *     element size must be a multiple of 16 bytes and every logit base
 *     pointer 16-byte aligned (the kernels move rows in 16-byte vectors).
 *   - Random numbers: Philox4x32-10 (Salmon et al., SC'11) with key
 *     (seed low 32 bits, seed high 32 bits) and counter (request, position,
 *     purpose, offset); u = (first output word >> 8) * 2^-24.  Purposes:
 *     0 = accept test, 1 = final sample.  Equal (seed, offset) give equal
 *     results; advance `offset` between calls for fresh randomness.
 *   - Return value: SPEC_OK, or a negative code detected on the host before
 *     anything is enqueued (SPEC_ECUDA: a launch failed; earlier kernels of
 *     the same call may have run).
 *   - Input errors the host cannot see (a token outside [0, V), a malformed
 *     parent array, a NaN logit, a row with no finite normaliser) are
 *     reported per request: that request's out_tokens and accepted_len are
 *     all -1 and the matching SPEC_STATUS_* bit is OR-ed into *status when
 *     status is non-NULL.  The kernels never trap.
 */
#ifndef SPECVERIFY_H
#define SPECVERIFY_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SPECVERIFY_API __attribute__((visibility("default")))
#else
#define SPECVERIFY_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* The CUDA runtime's stream handle; repeated here so that the header needs
 * no CUDA include.  Pass 0 for the legacy default stream. */
typedef struct CUstream_st *cudaStream_t;

typedef enum { SPEC_F32 = 0, SPEC_BF16 = 1 } spec_dtype_t;

enum {
    SPEC_OK = 0,
    SPEC_EINVAL = -1,        /* a size, count, temperature or NULL pointer is invalid   */
    SPEC_EALIGN = -2,        /* a logit base or the row pitch is not 16-byte aligned    */
    SPEC_EUNSUPPORTED = -3,  /* a size beyond the documented limits                      */
    SPEC_ECUDA = -4,         /* a CUDA launch or query failed                            */
    SPEC_EWORKSPACE = -5     /* workspace NULL, misaligned or smaller than required      */
};

/* Bits OR-ed into *status (device int32) by the kernels. */
enum {
    SPEC_STATUS_TOKEN = 1,   /* a draft or node token outside [0, V)                     */
    SPEC_STATUS_TREE = 2,    /* parents[0] != -1, parents[i] not in [0, i), or a node
                                deeper than max_depth                                    */
    SPEC_STATUS_LOGIT = 4,   /* a NaN logit, or a row with no finite normaliser
                                (+inf present, or every entry -inf)                      */
    SPEC_STATUS_TIMEOUT = 8, /* spec_verify_linear: a warp gave up waiting (about a
                                second) for another step of the same call; requests not
                                yet complete keep out_tokens and accepted_len at -1.
                                The call is a cooperative launch (all of its blocks
                                resident at once, else SPEC_ECUDA), so this is not
                                expected; spec_verify_debug_wait_expiry provokes it.    */
    SPEC_STATUS_CAPACITY = 16 /* spec_plug_tokens: a sequence buffer without room for
                                the tokens to append (or a negative length)             */
};

/* Limits checked on the host. */
#define SPEC_MAX_K 32
#define SPEC_MAX_NODES 1024

/*
 * Bytes of device workspace a call needs for `batch` requests with
 * `rows_per_req` logit rows each (linear: 2k+1; greedy with a workspace:
 * k+1; tree: 2*num_nodes) over a vocabulary of `vocab` entries.  The
 * workspace holds per-row partial normalisers (or partial argmaxes),
 * per-request decisions, counters and the draw's partial sums.  It must be
 * 256-byte aligned; it needs no initialisation (each call first clears, on
 * its stream, what it counts with) and its contents are undefined between
 * calls.  Two calls that may run concurrently need two workspaces.
 * Returns 0 for invalid arguments.
 */
SPECVERIFY_API size_t spec_verify_workspace_size(int batch, int rows_per_req, int vocab);

/* Static text for a return code (never NULL). */
SPECVERIFY_API const char *spec_verify_strerror(int code);

/*
 * Linear stochastic verification.
 *   target_logits [B][k+1][row_stride]: row j is the target distribution for
 *                 the token after draft j-1 (row 0: after the committed
 *                 prefix; row k: the bonus row).
 *   draft_logits  [B][k][row_stride]: row j is the draft distribution that
 *                 draft token j was drawn from.
 *   draft_tokens  [B][k] int32.
 *   1 <= k <= SPEC_MAX_K, V >= 1, row_stride >= V, temperature > 0 finite.
 * For each request: n = the first j whose test u_j * q_j(x_j) < p_j(x_j)
 * fails (u_j = U(seed, b, j, 0, offset)), or k.  If n < k the token at n is
 * drawn from max(0, p_n - q_n) (renormalised; if that mass is exactly zero,
 * from p_n); if n == k from p_k, both by inverse CDF with
 * u = U(seed, b, n, 1, offset): the smallest v whose running sum of weights
 * exceeds u times the total.
 * Outputs: out_tokens [B][k+1] = x_0..x_{n-1}, the sampled token, then -1;
 *          accepted_len [B] = n;
 *          dbg_logp, dbg_logq [B][k] (nullable, fp32): log p_j(x_j), log q_j(x_j);
 *          status (nullable, one int32): error bits, OR-ed in.
 * workspace: at least spec_verify_workspace_size(B, 2k+1, V) bytes.
 */
SPECVERIFY_API int spec_verify_linear(const void *target_logits, const void *draft_logits, spec_dtype_t dtype,
                       int64_t row_stride, const int32_t *draft_tokens, int batch, int k,
                       int vocab, float temperature, uint64_t seed, uint32_t offset,
                       int32_t *out_tokens, int32_t *accepted_len, float *dbg_logp,
                       float *dbg_logq, int32_t *status, void *workspace,
                       size_t workspace_bytes, cudaStream_t stream);

/*
 * spec_verify_linear without a workspace argument, for callers that cannot
 * allocate device memory: a plugin whose host framework owns the device
 * pool and hands out no workspace, or a serving loop that forbids
 * cudaMalloc once running.  The pages have no counterpart of this call; it
 * is a packaging convenience.  Inputs, outputs, results and error codes are
 * those of spec_verify_linear.  Its scratch is one static device array of
 * SPEC_NOALLOC_SCRATCH_BYTES compiled into the library, which every GPU that
 * loads the library holds until the process exits; the call itself
 * allocates nothing.  A request that needs more scratch than that
 * (spec_verify_workspace_size(B, 2k+1, V) > SPEC_NOALLOC_SCRATCH_BYTES)
 * returns SPEC_EUNSUPPORTED before anything is enqueued (an invalid argument
 * still returns the code spec_verify_linear gives it: those checks run
 * first).  The first call on a device, made with that device current, looks
 * up the array's device address and caches it for the life of the process;
 * make it before any stream capture starts.  The cached address is stale
 * after cudaDeviceReset (or any teardown of the device's primary context):
 * do not reset a device while calls of this library may still be made on
 * it.  All calls on a device share the array: each clears what must start
 * at zero, but calls that overlap on the GPU race and must be serialised by
 * the caller.
 */
#define SPEC_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)
SPECVERIFY_API int spec_verify_linear_noalloc(const void *target_logits, const void *draft_logits,
                                              spec_dtype_t dtype, int64_t row_stride,
                                              const int32_t *draft_tokens, int batch, int k,
                                              int vocab, float temperature, uint64_t seed,
                                              uint32_t offset, int32_t *out_tokens,
                                              int32_t *accepted_len, float *dbg_logp,
                                              float *dbg_logq, int32_t *status,
                                              cudaStream_t stream);

/*
 * Greedy (argmax-match) verification ("Accelerating Sonar through
 * speculation", section "Target-Draft": the draft emits its top token at
 * each step).  g_j = argmax_v target_logits[b][j][v] over [0, V), ties to the
 * lowest index; n = first j < k with draft_tokens[b][j] != g_j, else k.
 * Outputs: out_tokens [B][k+1] = x_0..x_{n-1}, g_n, then -1; accepted_len [B] = n.
 * Draft logits are not read and the temperature does not apply.
 * workspace: NULL, or at least spec_verify_workspace_size(B, k+1, V) bytes,
 *   256-byte aligned (else SPEC_EWORKSPACE; workspace_bytes is ignored when
 *   workspace is NULL).  Both forms give identical outputs.  With a
 *   workspace the rows are streamed in fixed-size items whose partial
 *   (max, argmax) records the workspace holds, then merged per row: the
 *   faster form.  Without one, a thread-block cluster merges each request's
 *   argmax in distributed shared memory, for callers that cannot provide
 *   device memory.  A workspace must not be shared by calls that may overlap.
 */
SPECVERIFY_API int spec_verify_greedy(const void *target_logits, spec_dtype_t dtype, int64_t row_stride,
                       const int32_t *draft_tokens, int batch, int k, int vocab,
                       int32_t *out_tokens, int32_t *accepted_len, int32_t *status,
                       void *workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Tree verification ("Accelerating Sonar through speculation", section
 * "EAGLE": drafts form a tree of top-K candidates; the longest acceptable
 * sequence is kept and one target token is appended).
 *   target_logits [B][N][row_stride]: row i = target distribution of the
 *                 token after node i.
 *   draft_logits  [B][N][row_stride]: row i = draft distribution node i's
 *                 children were drawn from; NULL when stochastic == 0; only
 *                 rows of nodes that have children are read.
 *   node_tokens   [B][N] int32: token of node i (entry 0, the root, ignored).
 *   parents       [B][N] int32: parents[0] == -1, 0 <= parents[i] < i.
 *   1 <= N <= SPEC_MAX_NODES, 1 <= max_depth, every node depth <= max_depth.
 * stochastic = 0 (greedy) or 1 (independent tests): node i >= 1 is
 * accepted when its parent is accepted and its test passes:
 *   greedy:     node_tokens[i] == argmax(target row parents[i]);
 *   stochastic: u * q_par(t) < p_par(t) with u = U(seed, b, i-1, 0, offset)
 *               (position i-1 is the node's draft index, so a chain tree
 *               draws exactly the numbers of spec_verify_linear).
 * d = the deepest accepted node, ties to the lowest index (d = 0 when none).
 * Outputs: out_tokens [B][max_depth+1] = tokens of the nodes on the path
 *          root->d (root excluded), then a bonus token from target row d
 *          (greedy: its argmax; stochastic: inverse CDF of p_d with
 *          u = U(seed, b, d, 1, offset)), then -1;
 *          accepted_len [B] = depth(d);
 *          out_path_nodes [B][max_depth+1] (nullable): node at depth 0..depth(d)
 *          (entry 0 = 0, the root), then -1.
 * The stochastic == 1 test has no residual step: it does not keep the
 * target distribution exactly (a variant that trades the guarantee for
 * simplicity, as "Speculative decoding explained" allows).
 * stochastic = 2 (distribution-exact): the single-draft rule of
 * "Speculative decoding explained" (section "Draft and verification loop")
 * applied to one sibling after another.  Walk from the root; at node u the
 * children are tested in index order, child c (token t) with
 * u_c = U(seed, b, c-1, 0, offset): accepted when u_c * q_u(t) < p(t), with
 * p the current distribution (first the target row of u) and q_u draft row
 * u; an accepted child becomes the node (p = its target row); a rejected
 * child replaces p by norm(max(0, p - q_u)) (a zero mass leaves p unchanged).
 * With no child left, the token is drawn from p by inverse CDF with
 * U(seed, b, u, 1, offset); d = that final node.  The outputs are as above.
 * When every node's children are independent draws from its draft row, the
 * emitted tokens follow the target's distribution exactly.
 * workspace: at least spec_verify_workspace_size(B, 2*N, V) bytes.
 */
SPECVERIFY_API int spec_verify_tree(const void *target_logits, const void *draft_logits, spec_dtype_t dtype,
                     int64_t row_stride, const int32_t *node_tokens, const int32_t *parents,
                     int batch, int num_nodes, int max_depth, int vocab, int stochastic,
                     float temperature, uint64_t seed, uint32_t offset, int32_t *out_tokens,
                     int32_t *accepted_len, int32_t *out_path_nodes, int32_t *status,
                     void *workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Greedy verification that reads only the rows its result depends on.
 * Same definition and outputs as spec_verify_greedy (greedy) and
 * spec_verify_tree with stochastic == 0 (tree): "Accelerating Sonar through
 * speculation", sections "Target-Draft" and "EAGLE" -- a node is kept when
 * its parent is kept and its token is the argmax of the parent's target row,
 * and the output is the deepest kept path plus the argmax after it.  Only
 * the rows of kept nodes (and the root) decide that output, so these calls
 * walk from the root and read exactly those rows: spec_verify_greedy_walk
 * reads target rows 0..n of each request (n + 1 of k + 1 rows),
 * spec_verify_tree_greedy_walk one row per kept node.  Each level costs a
 * dependent step, so they pay off when few drafts are kept.
 * Arguments, layouts, limits and outputs are those of spec_verify_greedy and
 * spec_verify_tree (draft logits, temperature, seed and offset do not
 * apply; no workspace).  Input errors are reported as there, with one
 * difference: a NaN logit is detected only in a row the walk reads (a NaN
 * in a row of a rejected node cannot change the result and is not seen).
 * Malformed parents, a node deeper than max_depth and out-of-range tokens
 * are detected for every node, as in the full calls.
 */
SPECVERIFY_API int spec_verify_greedy_walk(const void *target_logits, spec_dtype_t dtype,
                                           int64_t row_stride, const int32_t *draft_tokens,
                                           int batch, int k, int vocab, int32_t *out_tokens,
                                           int32_t *accepted_len, int32_t *status,
                                           cudaStream_t stream);

SPECVERIFY_API int spec_verify_tree_greedy_walk(const void *target_logits, spec_dtype_t dtype,
                                                int64_t row_stride, const int32_t *node_tokens,
                                                const int32_t *parents, int batch, int num_nodes,
                                                int max_depth, int vocab, int32_t *out_tokens,
                                                int32_t *accepted_len, int32_t *out_path_nodes,
                                                int32_t *status, cudaStream_t stream);

/*
 * The next step's input tokens, written on the device ("Accelerating Sonar
 * through speculation", section "MTP schedule for one token": a kernel plugs
 * the next target tokens into their positions, so the accepted count need not
 * reach the CPU before the next step; section "MTP": the draft reads the
 * target's input tokens shifted one position left of its hidden states).
 *   in_tokens    [B][k+1]: this step's target input tokens (position 0: the
 *                last committed token; positions 1..k: the drafts).
 *   out_tokens   [B][k+1], accepted_len [B]: a verification's outputs
 *                (spec_verify_linear or spec_verify_greedy; n = accepted_len).
 *   next_tokens  [B][k+1] (nullable): next[i] = in[i+1] for i < k, except
 *                next[n] = out[n] (the drawn token plugged at its position);
 *                next[k] = out[n] when n < k (a pad).  Positions after n
 *                hold drafts past the first rejection: a don't-care that the
 *                next draft run processes and discards.
 *   seq_tokens   [B][capacity], seq_len [B] (both NULL or both non-NULL; in
 *                place): out[0..n] is appended at seq_tokens[b][seq_len[b]..]
 *                and seq_len[b] grows by n + 1.
 * A request with accepted_len -1 (an error the verification reported) is
 * left alone (next row all -1, sequence unchanged); accepted_len outside
 * [-1, k] does the same and sets SPEC_STATUS_TOKEN; a sequence without room
 * for n + 1 tokens (or with a negative length) is left unchanged and sets
 * SPEC_STATUS_CAPACITY (next is still written).  1 <= k <= SPEC_MAX_K.
 * No host synchronisation; one small kernel on `stream`.
 */
SPECVERIFY_API int spec_plug_tokens(const int32_t *in_tokens, const int32_t *out_tokens,
                                    const int32_t *accepted_len, int batch, int k,
                                    int32_t *next_tokens, int32_t *seq_tokens, int32_t *seq_len,
                                    int capacity, int32_t *status, cudaStream_t stream);

/*
 * Vocabulary-sharded verification ("Accelerating Sonar through speculation",
 * section "Draft-target schedule": the target runs tensor-parallel over a
 * group of ranks; with its output projection split by vocabulary, rank w
 * holds columns [bounds[w], bounds[w+1]) of every logit row).  The rule is
 * that of spec_verify_linear / spec_verify_greedy; these calls are the
 * per-rank steps between which the caller exchanges the small results
 * across the ranks (all-gather, all-reduce max).  Every cross-rank merge
 * runs in rank order inside the kernels, so all ranks compute identical
 * values.  Local logit tensors are [B][rows][row_stride] holding the rank's
 * columns (vocab_lo <= v < vocab_hi as local index v - vocab_lo;
 * row_stride >= vocab_hi - vocab_lo; 16-byte pitch and bases as elsewhere).
 * Sequence (linear): row_stats -> all-gather(max, sum, probe) -> decide ->
 * draw_sums(no norm_parts) -> all-gather -> draw_sums(norm_parts) ->
 * all-gather -> draw_pick -> all-reduce max(token) -> emit.
 * Sequence (greedy): row_stats(draft NULL) -> all-gather(max, arg) ->
 * decide_greedy.  No host synchronisation; errors as spec_verify_linear.
 *
 * spec_shard_row_stats: per row of this rank's columns (linear: target rows
 *   0..k then draft rows 0..k-1, R = 2k+1; greedy, draft_logits NULL: target
 *   rows 0..k, R = k+1): row_max [B][R] (NaN when a NaN is present), and
 *   either row_sum [B][R] (fp64 sum of exp((l - max)/T)) and probe [B][k][2]
 *   (target and draft logit at draft token j if this rank holds it, else
 *   NaN), or row_argmax [B][R] (global index of the lowest maximal entry;
 *   INT32_MAX when every entry is -inf).
 * spec_shard_decide: inputs gathered over the W = shards ranks:
 *   row_max_all [W][B][2k+1], row_sum_all [W][B][2k+1],
 *   probe_all [W][B][k][2], bounds [W+1] (device int32).  Merges each row
 *   (max; sum of s_w exp((m_w - max)/T)), tests the drafts as
 *   spec_verify_linear, writes out_tokens (the drawn slot left -1),
 *   accepted_len and draw [B][6] (fp64: mode, n, maxima, u) for the next steps.
 * spec_shard_decide_greedy: row_max_all, row_argmax_all [W][B][k+1]; writes
 *   the complete greedy outputs.
 * spec_shard_draw_sums: sums [B][2] (fp64) over this rank's columns of each
 *   request's draw rows: with norm_parts NULL, (sum e, sum f) of the draw's
 *   target and draft rows; with norm_parts = the ranks' first sums
 *   [shards][B][2], (mass of the draw weights, sum e), the weights being
 *   max(0, e/S_t - f/S_d) (residual) or e (target row).
 * spec_shard_draw_pick: with the ranks' first and second sums gathered, the
 *   rank whose part of the running mass (rank order) holds u * Z writes the
 *   drawn token (global index, inverse CDF inside its columns) into
 *   token [B]; other ranks write -1 (a residual whose mass vanished in
 *   rounding draws from the target row, as spec_verify_linear).
 * spec_shard_emit: out_tokens[b][n] = token[b] for each request that draws.
 */
SPECVERIFY_API int spec_shard_row_stats(const void *target_logits, const void *draft_logits,
                                        spec_dtype_t dtype, int64_t row_stride,
                                        const int32_t *draft_tokens, int batch, int k, int vocab_lo,
                                        int vocab_hi, float temperature, float *row_max,
                                        double *row_sum, int32_t *row_argmax, float *probe,
                                        cudaStream_t stream);
SPECVERIFY_API int spec_shard_decide(const float *row_max_all, const double *row_sum_all,
                                     const float *probe_all, const int32_t *bounds, int shards,
                                     const int32_t *draft_tokens, int batch, int k, int vocab,
                                     float temperature, uint64_t seed, uint32_t offset,
                                     int32_t *out_tokens, int32_t *accepted_len, double *draw,
                                     int32_t *status, cudaStream_t stream);
SPECVERIFY_API int spec_shard_decide_greedy(const float *row_max_all, const int32_t *row_argmax_all,
                                            int shards, const int32_t *draft_tokens, int batch, int k,
                                            int vocab, int32_t *out_tokens, int32_t *accepted_len,
                                            int32_t *status, cudaStream_t stream);
SPECVERIFY_API int spec_shard_draw_sums(const void *target_logits, const void *draft_logits,
                                        spec_dtype_t dtype, int64_t row_stride, int batch, int k,
                                        int vocab_lo, int vocab_hi, float temperature,
                                        const double *draw, const double *norm_parts, int shards,
                                        double *sums, cudaStream_t stream);
SPECVERIFY_API int spec_shard_draw_pick(const void *target_logits, const void *draft_logits,
                                        spec_dtype_t dtype, int64_t row_stride, int batch, int k,
                                        int vocab_lo, int vocab_hi, float temperature,
                                        const double *draw, const double *norm_parts,
                                        const double *mass_parts, int shards, int shard_index,
                                        int32_t *token, cudaStream_t stream);
SPECVERIFY_API int spec_shard_emit(const int32_t *token, const double *draw, int batch, int k,
                                   int32_t *out_tokens, cudaStream_t stream);

/*
 * Diagnostic: the bounded waits of spec_verify_linear, made to expire.
 * Arguments as spec_verify_linear (no seed, offset or debug outputs), plus
 * poll_limit in [1, SPEC_DEBUG_MAX_POLLS]: the number of polls (each at
 * most about 2 us) after which a waiting warp gives up.  The pass-1 step
 * of this call stores no partial normaliser, so every decide step waits
 * until its limit, then reports SPEC_STATUS_TIMEOUT into *status
 * (required here) and the kernel returns; every request keeps
 * out_tokens and accepted_len at -1.  Lets a caller check that an expired
 * wait ends the kernel with an error status rather than a hang.
 */
#define SPEC_DEBUG_MAX_POLLS 4096u
SPECVERIFY_API int spec_verify_debug_wait_expiry(const void *target_logits, const void *draft_logits,
                                                 spec_dtype_t dtype, int64_t row_stride,
                                                 const int32_t *draft_tokens, int batch, int k,
                                                 int vocab, float temperature, uint32_t poll_limit,
                                                 int32_t *out_tokens, int32_t *accepted_len,
                                                 int32_t *status, void *workspace,
                                                 size_t workspace_bytes, cudaStream_t stream);

/*
 * Diagnostic: the uniforms the kernels draw.  out [batch][count] (device,
 * double) = U(seed, b, first_position + i, purpose, offset).  Lets a caller
 * check the device Philox stream against an independent implementation.
 */
SPECVERIFY_API int spec_verify_debug_uniforms(uint64_t seed, uint32_t offset, uint32_t purpose, int batch,
                               int count, int first_position, double *out,
                               cudaStream_t stream);

/*
 * Diagnostic: the kernels' base-2 exponentials, out[i] = 2^z[i] for
 * z[i] <= 0 (device arrays of n doubles).  kind 0: fp64, table driven
 * (Tang's method; results below 2^-1020 are 0); kind 1: fp32 polynomial on
 * the FMA pipe (input rounded to fp32; results below 2^-125 are 0);
 * kind 2: fp32 special-function unit (ex2.approx).  Lets a caller check
 * their accuracy.
 */
SPECVERIFY_API int spec_verify_debug_exp2(const double *z, double *out, int n, int kind,
                                          cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SPECVERIFY_H */
