/*
 * ts_verify.h -- C ABI of libtsverify.so, the B200 (sm_100a) implementation
 * of TokenSwift's per-step verification path.
 *
 * TokenSwift accelerates ultra-long generation by drafting several tokens,
 * verifying them in one tree-structured pass over the full KV cache, keeping
 * the longest valid candidate, penalising recently generated tokens, and
 * drafting over a partial KV cache that keeps the initial tokens plus the
 * most important ones ("TokenSwift - A framework for accelerating the
 * generation of ultra-long text", aiboss88.com, section "TokenSwift's
 * technical principles"; "From Hours to Minutes: Lossless Acceleration of
 * Ultra-Long Sequence Generation up to 100K Tokens", arxivlens.com,
 * "Technical Contribution").  This library implements the three kernels of
 * that step (with a fused form in which the verify attention hands the root
 * node's scores to the select) and, as host code, the n-gram reuse table;
 * the model around them (projections, LM head, draft heads) is the
 * caller's.
 *
 * Conventions for every entry point
 *  - Memory: the caller owns every buffer.  The library never allocates,
 *    frees or synchronises (except ts_workspace_status, which says so).
 *    "device" pointers are CUDA device memory on the current device.
 *  - Streams: `stream` is a cudaStream_t passed as void*; NULL is the legacy
 *    default stream.  Calls are asynchronous with respect to the host.
 *  - Errors: arguments are validated on the host before anything is
 *    launched; an invalid call returns a non-zero ts_status and launches
 *    nothing.  A launch failure returns TS_ERR_CUDA.  Conditions that only
 *    the device can see (a window id outside the vocabulary, an expired
 *    bounded wait) are recorded in the workspace's status word, read by
 *    ts_workspace_status().
 *  - Workspace: sized by the matching *_workspace_size() call, at least
 *    256-byte aligned, zero-filled once by the caller before first use.
 *    Every call returns the counters and tickets it relies on to zero
 *    before it ends; the rest of the workspace is scratch that each call
 *    writes before it reads.  After a call that recorded a device-side
 *    error in the status word, zero-fill the workspace again.
 *    Concurrent calls need distinct workspaces.
 *  - bf16 tensors are raw IEEE bfloat16 bit patterns; every device pointer
 *    must be 16-byte aligned.
 *  - No C++ exception crosses this interface.
 */
#ifndef TS_VERIFY_H
#define TS_VERIFY_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TS_API __attribute__((visibility("default")))
#else
#define TS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    TS_OK = 0,
    TS_ERR_INVALID_ARG = 1, /* a host-checked argument is invalid */
    TS_ERR_UNSUPPORTED = 2, /* valid, but outside what this build supports */
    TS_ERR_WORKSPACE = 3,   /* workspace missing, too small or misaligned */
    TS_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed */
    TS_ERR_TIMEOUT = 5,     /* device: a bounded wait expired (status word) */
    TS_ERR_DEVICE_ARG = 6,  /* device: invalid data seen on the device (status word) */
    TS_ERR_SCRATCH_LIMIT = 7 /* needs more scratch than ts_tree_verify_attn_noalloc holds */
} ts_status;

/* Largest draft tree, in nodes (ancestor sets are 64-bit masks). */
#define TS_MAX_TREE 64
/* query heads per KV head supported by the importance select */
#define TS_MAX_SELECT_GROUP 8

/* Static description of a status code; never NULL. */
TS_API const char *ts_status_string(int status);

/* Library ABI version (major * 100 + minor). */
TS_API int ts_version(void);

/*
 * Tree-masked attention of the draft-tree queries over the full KV cache.
 *
 * Source: tree-based multi-candidate verification ("TokenSwift's technical
 * principles", aiboss88.com; tencent article, parallel-verification figure:
 * candidates go through the model with the full KV cache under tree-based
 * attention; arxivlens "Technical Contribution": a 3-ary tree).
 *
 * For tree node i and query head h (KV head g = h / (Hq / Hkv)):
 *   out[i,h,:] = sum_j softmax_j(scale * q[i,h,:] . k[g,j,:]) v[g,j,:]
 * over j in [0, n_ctx) and j = n_ctx + a for every node a on the root path
 * of i (i included).  The tree tail rows [n_ctx, n_ctx + n_tree) of the
 * cache hold the tree nodes' own K/V, node a at row n_ctx + a.
 *
 *  q            device bf16 [n_tree, Hq, D], contiguous (node-major).
 *  k_cache      device bf16 [Hkv, kv_cap, D], contiguous; rows [0, n_ctx)
 *               context, [n_ctx, n_ctx + n_tree) the tree tail, rows beyond
 *               are not read.
 *  v_cache      same layout as k_cache.
 *  kv_cap       rows per KV head in the cache, >= n_ctx + n_tree.
 *  n_heads_q, n_heads_kv, head_dim
 *               Hq % Hkv == 0; head_dim is 64 or 128.
 *  n_ctx        context length, >= 0 (0: the tree attends only to itself).
 *  n_tree       tree nodes, 1 .. TS_MAX_TREE.
 *  parent       HOST int32 [n_tree]: parent[0] = -1, 0 <= parent[i] < i
 *               (BFS/topological order).  Read before the call returns.
 *  softmax_scale  finite, usually 1/sqrt(D).
 *  out          device fp32 [n_tree, Hq, D], written entirely.
 *  workspace    device, >= ts_tree_verify_attn_workspace_size(...) bytes.
 *
 * With head_dim 128 and n_ctx >= 2048 the split-KV kernel hands tiles to
 * its splits at run time, so two calls on the same inputs may fold the
 * weights in a different fp32 order (and, rarely, round one weight to bf16
 * the other way): results agree to about 1e-4, not bit for bit.  That kernel is one cooperative launch (every CTA
 * resident at once, one per SM); a launch the device cannot co-schedule
 * returns TS_ERR_CUDA.
 */
TS_API size_t ts_tree_verify_attn_workspace_size(int n_heads_q, int n_heads_kv, int head_dim,
                                          int n_ctx, int n_tree);
TS_API int ts_tree_verify_attn(const void *q, const void *k_cache, const void *v_cache, int64_t kv_cap,
                        int n_heads_q, int n_heads_kv, int head_dim, int n_ctx, int n_tree,
                        const int32_t *parent, float softmax_scale, float *out,
                        void *workspace, size_t workspace_bytes, void *stream);

/*
 * ts_tree_verify_attn without a workspace argument, for callers that cannot
 * allocate device memory (the TokenSwift pages have no counterpart; this is
 * an interface convenience).  Some callers may not call cudaMalloc where
 * they run attention: code whose device memory is all owned by another
 * runtime's allocator or a fixed, pre-planned budget, or code that must not
 * block on an allocation.  They pass inputs and outputs as for
 * ts_tree_verify_attn; the split-KV scratch comes from a static device array
 * of TS_NOALLOC_SCRATCH_BYTES inside the library, taken on each device that
 * calls this entry point and held until the process exits.  Nothing is
 * allocated and no allocating routine is called.
 *
 *  - Limit: a problem whose ts_tree_verify_attn_workspace_size() exceeds
 *    TS_NOALLOC_SCRATCH_BYTES is rejected with TS_ERR_SCRATCH_LIMIT before
 *    anything is launched (16 MiB covers, e.g., 32/8 heads, D 128, a 40-node
 *    tree up to about 73 million context positions: the scratch holds the
 *    split partials and one byte per 128-position tile and KV head).
 *  - Set-up: the first call on a device (and the first after that device's
 *    context was reset) looks up the array's device address
 *    (cudaGetSymbolAddress, with the device current) and keeps it for that
 *    context; make that first call outside any stream capture.
 *  - Sharing: every call on a device uses the same array and it keeps the
 *    last call's contents; each call clears the part that must start at
 *    zero.  Calls whose work overlaps on the GPU (different streams, no
 *    ordering between them) race on the array and give wrong results:
 *    order them, or use ts_tree_verify_attn with separate workspaces.
 *  - Errors: every argument is checked on the host first, with the same
 *    results as ts_tree_verify_attn (an invalid call queues nothing);
 *    TS_ERR_SCRATCH_LIMIT as above.  Conditions only the device can see (an
 *    expired bounded wait) go to the status word of the array, which no
 *    call clears: read and clear it with ts_noalloc_status.
 */
#define TS_NOALLOC_SCRATCH_BYTES (16u << 20)
TS_API int ts_tree_verify_attn_noalloc(const void *q, const void *k_cache, const void *v_cache,
                                       int64_t kv_cap, int n_heads_q, int n_heads_kv,
                                       int head_dim, int n_ctx, int n_tree,
                                       const int32_t *parent, float softmax_scale, float *out,
                                       void *stream);

/*
 * Device-side status of ts_tree_verify_attn_noalloc calls on the current
 * device (no counterpart on the pages): waits for the work queued on
 * `stream` (synchronises it), then returns TS_OK or the first device-side
 * error those calls recorded since the status was last cleared, and clears
 * it when `clear` is non-zero.  TS_ERR_CUDA if the read fails.
 */
TS_API int ts_noalloc_status(void *stream, int clear);

/*
 * Failure-detection self-test of the no-alloc scratch (no counterpart on the
 * pages; diagnostic only): sets the array's hand-off tickets to non-zero
 * values, as a call that ended early on the device could leave them, then
 * launches the bounded-wait self-test of ts_selftest_bounded_wait on the
 * array's header, so that about one second later TS_ERR_TIMEOUT is in the
 * status word ts_noalloc_status reads.  The next ts_tree_verify_attn_noalloc
 * call still computes correctly and leaves that status in place.
 */
TS_API int ts_noalloc_selftest(void *stream);

/*
 * Dynamic partial-KV update: importance scores, sink + top-budget selection
 * and the gather into the compact draft cache.
 *
 * Source: "TokenSwift's technical principles" (aiboss88.com): the initial
 * KV cache is retained and the rest is replaced in order of token
 * importance; tencent article 动态KV缓存更新: the partial cache is updated
 * dynamically to cut KV load time; the draft model is the target model run
 * with that partial cache (无损的输出质量).
 *
 *   score[g,n] = (1/G) sum_{h in group g} softmax_n(scale * q_last[h] . k[g,n])
 * over n in [0, n_ctx).  Per KV head g the kept set is [0, n_sink) plus the
 * `budget` highest scores of [n_sink, n_ctx) (equal scores: lower position
 * first), listed in ascending position; n_keep = min(n_ctx, n_sink+budget).
 *
 *  q_last       device bf16 [Hq, D] (the root node's query rows).
 *  k_cache, v_cache, kv_cap, n_heads_q, n_heads_kv, head_dim
 *               as for ts_tree_verify_attn; only rows [0, n_ctx) are read.
 *  n_ctx        >= 1.   n_sink, budget >= 0.
 *  softmax_scale  finite.
 *  scores_out   device fp32 [Hkv, n_ctx], or NULL (not returned).
 *  idx_out      device int32 [Hkv, n_keep], ascending positions.
 *  k_partial, v_partial
 *               device bf16 [Hkv, partial_cap, D]; rows [0, n_keep) are
 *               written with the kept rows, in idx_out order.
 *  partial_cap  >= n_keep.
 */
TS_API size_t ts_kv_importance_select_workspace_size(int n_heads_q, int n_heads_kv, int head_dim,
                                              int n_ctx);
TS_API int ts_kv_importance_select(const void *q_last, const void *k_cache, const void *v_cache,
                            int64_t kv_cap, int n_heads_q, int n_heads_kv, int head_dim,
                            int n_ctx, int n_sink, int budget, float softmax_scale,
                            float *scores_out, int32_t *idx_out, void *k_partial,
                            void *v_partial, int64_t partial_cap, void *workspace,
                            size_t workspace_bytes, void *stream);

/*
 * The same verify attention, also leaving the root node's scores for the
 * importance select: root_scores_out[h][n] = log2(e) * softmax_scale *
 * q[0][h] . k[h / G][n] for n in [0, n_ctx), fp32 [n_heads_q, n_ctx]
 * (device, 4-byte aligned; 16-byte aligned when n_ctx is a multiple of 4,
 * for ts_kv_select_from_scores).  The root's query rows are the ones the
 * importance score is defined on, and the verify pass computes these
 * products anyway: handing them to ts_kv_select_from_scores spares the
 * select's own pass over K.  G = n_heads_q / n_heads_kv must be at most
 * TS_MAX_SELECT_GROUP (else TS_ERR_UNSUPPORTED).  Every other argument, the
 * workspace and `out` are as for ts_tree_verify_attn, and `out` is the
 * same.
 */
TS_API int ts_tree_verify_attn_root_scores(const void *q, const void *k_cache,
                                           const void *v_cache, int64_t kv_cap, int n_heads_q,
                                           int n_heads_kv, int head_dim, int n_ctx, int n_tree,
                                           const int32_t *parent, float softmax_scale,
                                           float *out, float *root_scores_out, void *workspace,
                                           size_t workspace_bytes, void *stream);

/*
 * The partial-KV update of ts_kv_importance_select from root scores given
 * by the caller (as left by ts_tree_verify_attn_root_scores): the group-mean
 * softmax over [0, n_ctx) of root_scores (base 2), then the same sink +
 * top-budget selection and gather.  root_scores: device fp32 [n_heads_q,
 * n_ctx], read only.  The other arguments are as for
 * ts_kv_importance_select (no query rows, no scale); the workspace needs
 * ts_kv_select_from_scores_workspace_size(n_heads_q, n_heads_kv, n_ctx)
 * bytes for the current device (0 for an invalid shape): per-chunk head
 * statistics, the importance scores when scores_out is NULL, per-head
 * histograms and counters, and a candidate list of up to n_ctx entries per
 * KV head.
 */
TS_API size_t ts_kv_select_from_scores_workspace_size(int n_heads_q, int n_heads_kv, int n_ctx);
TS_API int ts_kv_select_from_scores(const float *root_scores, const void *k_cache,
                                    const void *v_cache, int64_t kv_cap, int n_heads_q,
                                    int n_heads_kv, int head_dim, int n_ctx, int n_sink,
                                    int budget, float *scores_out, int32_t *idx_out,
                                    void *k_partial, void *v_partial, int64_t partial_cap,
                                    void *workspace, size_t workspace_bytes, void *stream);

/*
 * Contextual penalty, per-node target argmax and the longest accepted path.
 *
 * Source: "TokenSwift's technical principles" (aiboss88.com): a penalty on
 * recently generated tokens; the longest valid candidate is the output;
 * tencent article 上下文惩罚 and the figure text (the longest valid candidate,
 * e.g. "is the father of", is kept).
 *
 * For every id in the window (a set), a positive logit is divided by
 * `penalty` and a non-positive one multiplied by it (binary32,
 * round-to-nearest).  argmax[i] is the largest penalised logit of node i,
 * ties to the lowest id, NaN counted as -inf.  The root is valid; a draft
 * node is valid when its parent is valid and its token equals the argmax at
 * its parent (it is what greedy decoding would have produced).  The accepted
 * path is the root path of the deepest valid node, equal depths going to
 * the lowest node index.
 *
 *  logits       device fp32 [n_tree, vocab]; not modified.
 *  n_tree       1 .. TS_MAX_TREE.   vocab 1 .. 16,777,216 (above:
 *               TS_ERR_UNSUPPORTED).
 *  window       device int32 [window_len] (may be NULL when window_len is
 *               0); ids outside [0, vocab) are ignored and flagged as
 *               TS_ERR_DEVICE_ARG in the status word.
 *  penalty      finite, > 0.
 *  parent       HOST int32 [n_tree], as for ts_tree_verify_attn.
 *  tree_tokens  device int32 [n_tree]; tree_tokens[0] (the root) is unused.
 *  argmax_out   device int32 [n_tree], or NULL.
 *  accept_out   device int32 [2 + n_tree]: {L, bonus, path[0..L]} where L
 *               is the number of accepted draft nodes, path[0] = 0 is the
 *               root, and bonus = argmax at path[L]; entries past path[L]
 *               are set to -1.
 */
TS_API size_t ts_penalize_accept_workspace_size(int n_tree, int vocab);
TS_API int ts_penalize_accept(const float *logits, int n_tree, int vocab, const int32_t *window,
                       int window_len, float penalty, const int32_t *parent,
                       const int32_t *tree_tokens, int32_t *argmax_out, int32_t *accept_out,
                       void *workspace, size_t workspace_bytes, void *stream);

/*
 * ts_penalize_accept with the method's two randomised / contextual options
 * ("TokenSwift's technical principles", aiboss88.com: "Contextual penalty
 * strategy" -- the penalty falls on recently generated tokens -- and
 * tree-based verification -- the longest valid candidate is selected at
 * random).  flags = 0 gives exactly ts_penalize_accept.
 *
 *  TS_PENALIZE_PATH_TOKENS  node i's window is `window` together with the
 *               tokens of the draft nodes on i's root path (i included; the
 *               root's entry of tree_tokens is not read): the tokens that
 *               precede the one node i's logits predict.  A draft token
 *               outside [0, vocab) is ignored and flagged TS_ERR_DEVICE_ARG.
 *  TS_ACCEPT_RANDOM_TIE     of the c deepest valid nodes, in ascending
 *               index order, the one at position (random mod c) is kept
 *               (instead of the first).  `random` is a random 64-bit
 *               integer drawn by the caller; it is read only with this flag.
 * Every other argument, the workspace and the outputs are as for
 * ts_penalize_accept.  Unknown flag bits: TS_ERR_INVALID_ARG.
 */
#define TS_PENALIZE_PATH_TOKENS 1u
#define TS_ACCEPT_RANDOM_TIE 2u
TS_API int ts_penalize_accept_ex(const float *logits, int n_tree, int vocab,
                                 const int32_t *window, int window_len, float penalty,
                                 const int32_t *parent, const int32_t *tree_tokens,
                                 unsigned flags, uint64_t random, int32_t *argmax_out,
                                 int32_t *accept_out, void *workspace, size_t workspace_bytes,
                                 void *stream);

/*
 * ts_penalize_accept_ex with temperature acceptance: the target token of
 * every node is a draw from softmax(penalised logits / temperature) rather
 * than its argmax ("TokenSwift's technical principles", aiboss88.com,
 * tree-based verification: the output stays lossless -- every accepted
 * token is what the target model itself would have sampled after the tokens
 * before it -- and gains diversity).  The draw is the Gumbel-max rule:
 * target[i] is the id maximising
 *
 *     score = penalised[i][id] / temperature + gumbel[i][id]
 *
 * computed in binary32 with round-to-nearest, one rounding per operation
 * (the quotient, then the sum; never fused), ties to the lowest id, a NaN
 * score counting as -inf.  With gumbel holding independent standard Gumbel
 * draws (-log(-log u), u uniform on (0, 1)) the result is distributed
 * exactly as that softmax.  A draft node is valid when its parent is valid
 * and its token equals target[parent]; the accepted path and the flags are
 * as for ts_penalize_accept_ex, with target in place of argmax (bonus =
 * target at path[L]).  Temperature 1 with all-zero noise gives exactly
 * ts_penalize_accept_ex.
 *
 *  gumbel       device fp32 [n_tree, vocab], 16-byte aligned; not
 *               modified.  The caller draws it (and owns the generator).
 *  temperature  finite, > 0.
 *  vocab        1 .. 8,388,608 (above: TS_ERR_UNSUPPORTED).
 *  target_out   device int32 [n_tree], or NULL.
 * The other arguments, the workspace (ts_penalize_accept_workspace_size)
 * and the errors are as for ts_penalize_accept_ex; a NULL or misaligned
 * gumbel or a bad temperature: TS_ERR_INVALID_ARG.  The call reads
 * 2 * n_tree * vocab * 4 bytes (logits and noise, each once).
 */
TS_API int ts_penalize_sample_accept(const float *logits, const float *gumbel, float temperature,
                                     int n_tree, int vocab, const int32_t *window,
                                     int window_len, float penalty, const int32_t *parent,
                                     const int32_t *tree_tokens, unsigned flags, uint64_t random,
                                     int32_t *target_out, int32_t *accept_out, void *workspace,
                                     size_t workspace_bytes, void *stream);

/*
 * Commit of the accepted path: the tree rows of the nodes on the accepted
 * path move to the context end, in path order, in both caches, so that the
 * next step's context is n_ctx + L + 1 contiguous rows (tencent article,
 * parallel-verification figure: the longest valid candidate is kept and
 * updates the state for the next step).  For j = 1 .. L, row n_ctx + j of
 * every KV head takes row n_ctx + path[j] (row n_ctx is the root already);
 * other rows are not touched.  The path is read on the device, so the call
 * can follow ts_penalize_accept on the same stream with no host round trip.
 *
 *  k_cache, v_cache  device bf16 [Hkv, kv_cap, D], modified in place.
 *  kv_cap, n_heads_kv, head_dim  as for ts_tree_verify_attn (D 64 or 128).
 *  n_ctx, n_tree     the verified step's context length and tree size;
 *                    n_ctx + n_tree <= kv_cap.
 *  accept            device int32 [2 + n_tree] as written by
 *                    ts_penalize_accept: {L, bonus, path[0..L]}.  A result
 *                    that is not a root path (L outside [0, n_tree), path[0]
 *                    not 0, nodes not increasing or out of range) moves
 *                    nothing and is flagged TS_ERR_DEVICE_ARG.
 *  workspace         device, >= 256 bytes (the status header), 256-byte
 *                    aligned, zero-filled.
 */
TS_API int ts_kv_commit_path(void *k_cache, void *v_cache, int64_t kv_cap, int n_heads_kv,
                             int head_dim, int n_ctx, int n_tree, const int32_t *accept,
                             void *workspace, size_t workspace_bytes, void *stream);

/*
 * n-gram reuse table.  TokenSwift drafts with the frequencies of the
 * n-grams already generated: phrases that occurred often are retrieved and
 * reused as draft candidates, and the table is updated with the tokens
 * each verification accepts ("TokenSwift - A framework for accelerating
 * the generation of ultra-long text", aiboss88.com, "Parallel generation
 * of multiple tokens and token reuse"; "TokenSwift ... 从小时到分钟",
 * cloud.tencent.com, the parallel-verification step of the method figure).
 * The pages fix neither n nor the retrieval rule; this table counts every
 * run of n consecutive tokens of the generated text (2 <= n <= 8) and
 * returns, for a prefix of p tokens (1 <= p <= n-1), the most frequent
 * n-grams that start with it: count descending, ties by continuation in
 * ascending token order.  p = 1 gives whole-phrase continuations of a
 * token; p = n-1 gives the next-token counts after the last n-1 tokens.
 *
 * Host code on caller-owned HOST memory: one contiguous buffer of
 * ts_ngram_table_bytes(n, capacity) = 64 + 216 * capacity bytes, 8-byte
 * aligned, holding a header, `capacity` n-gram slots (open addressing,
 * linear probing) and two indices of `capacity` entries each, which chain
 * the n-grams by first token and by first n-1 tokens and keep each
 * chain's best 16 in order.  A top-k with k <= 16 for p = 1 or p = n-1
 * reads that list; a larger k, or another p, walks a chain.  The table
 * holds at most capacity - max(1, capacity/8) distinct n-grams.  Calls on
 * one table must not overlap (no internal locking).  Tokens are
 * non-negative int32 ids.
 *
 *  ts_ngram_table_bytes  bytes for (n, capacity); 0 if n is outside [2, 8]
 *                        or capacity is not a power of two in [2, 2^31].
 *  ts_ngram_init         formats `table` (table_bytes must be at least the
 *                        size above) as an empty table.
 *  ts_ngram_update       counts the n-grams of `text` that END at one of its
 *                        last n_new positions (text[0, text_len) is the
 *                        tail of the generated text; pass at least the n-1
 *                        tokens before the new ones so that n-grams which
 *                        straddle them are counted).  All or nothing: if
 *                        the distinct n-grams not yet present would exceed
 *                        the fill limit, nothing changes and
 *                        TS_ERR_WORKSPACE is returned.  A negative token in
 *                        the scanned range is TS_ERR_INVALID_ARG.
 *  ts_ngram_topk_prefix  the k (1 <= k <= 4096) most frequent n-grams that
 *                        start with prefix[0..p): their n-p continuation
 *                        tokens into cont_out [k, n-p] and counts into
 *                        count_out [k]; *n_found = how many exist (<= k);
 *                        rows past that get tokens -1 and count 0.
 *  ts_ngram_topk         ts_ngram_topk_prefix with the one-token prefix
 *                        `first` (cont_out [k, n-1]).
 *  ts_ngram_count        occurrences of one n-gram (gram[0..n)); 0 if absent.
 *  ts_ngram_size         distinct n-grams held and total n-grams counted.
 * Errors: TS_ERR_INVALID_ARG for NULL pointers, an unformatted table, a
 * table_bytes smaller than the table, or out-of-range sizes.
 */
TS_API size_t ts_ngram_table_bytes(int n, int64_t capacity);
TS_API int ts_ngram_init(void *table, size_t table_bytes, int n, int64_t capacity);
TS_API int ts_ngram_update(void *table, size_t table_bytes, const int32_t *text,
                           int64_t text_len, int64_t n_new);
TS_API int ts_ngram_topk_prefix(const void *table, size_t table_bytes, const int32_t *prefix,
                                int p, int k, int32_t *cont_out, int64_t *count_out,
                                int *n_found);
TS_API int ts_ngram_topk(const void *table, size_t table_bytes, int32_t first, int k,
                         int32_t *cont_out, int64_t *count_out, int *n_found);
TS_API int ts_ngram_count(const void *table, size_t table_bytes, const int32_t *gram,
                          int64_t *count);
TS_API int ts_ngram_size(const void *table, size_t table_bytes, int64_t *distinct,
                         int64_t *total);

/*
 * Number of kernels this library has launched in this process (all
 * devices, all entry points); a diagnostic for counting launches.
 */
TS_API unsigned long long ts_kernel_launch_count(void);

/*
 * Failure-detection self-test.  Every pipeline wait in this library's
 * kernels is bounded (about one second of SM clock); a wait that runs out
 * records TS_ERR_TIMEOUT in the workspace status word and the kernel ends
 * without trapping, so the context stays usable.  This call launches one
 * small CTA that takes that same bounded wait on a barrier nothing ever
 * completes: about one second later it has recorded TS_ERR_TIMEOUT in
 * `workspace` (read it with ts_workspace_status).  Diagnostic only; no
 * page of the method has a counterpart.
 *  workspace    device, >= 256 bytes, 256-byte aligned, zero-filled.
 */
TS_API int ts_selftest_bounded_wait(void *workspace, size_t workspace_bytes, void *stream);

/*
 * Reads the status word of a workspace after the work queued on `stream`
 * has finished (this call synchronises `stream`).  Returns TS_OK or the
 * first device-side error recorded since the last clear; clears the word
 * when `clear` is non-zero.  Returns TS_ERR_CUDA if the copy fails.
 */
TS_API int ts_workspace_status(const void *workspace, void *stream, int clear);

#ifdef __cplusplus
}
#endif
#endif /* TS_VERIFY_H */
