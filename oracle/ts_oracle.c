/*
 * ts_oracle.c -- plain, slow, fp64 CPU oracle for the TokenSwift per-step
 * verification path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library calls, links or
 * loads this file; only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark do.  It shares no code, header, table or helper with the
 * CUDA path.  Every function is the plain definition of what the method
 * computes, written out with loops: no blocking, no splitting, no online
 * softmax, no reordering beyond what the definition states.  The one
 * concession to speed is an OpenMP "parallel for" over independent output
 * rows, which changes no arithmetic.
 *
 * Sources (the TokenSwift write-ups):
 *  - "TokenSwift - A framework for accelerating the generation of ultra-long
 *    text" (aiboss88.com), section "TokenSwift's technical principles":
 *    tree-based multi-candidate verification, the dynamic KV cache update
 *    (keep the initial cache, replace the rest by token importance), and the
 *    contextual penalty on recently generated tokens.
 *  - "90分钟生成10万Token..." (cloud.tencent.com), section 技术原理
 *    (动态KV缓存更新, 上下文惩罚) and the parallel-verification figure text:
 *    candidates are run against the full KV cache and the longest valid
 *    sequence is kept.
 *  - "From Hours to Minutes: Lossless Acceleration of Ultra-Long Sequence
 *    Generation up to 100K Tokens" (arxivlens.com), "Technical Contribution":
 *    a simple 3-ary tree in tree attention, KV compression, contextual
 *    penalty.
 *
 * Readings of points the pages leave open are stated at each function.
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* bf16 is the upper half of an IEEE binary32; widening is exact. */
static double bf16_value(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* A parent array is a tree in BFS order: parent[0] = -1, 0 <= parent[i] < i. */
static int tree_is_valid(const int32_t *parent, int n_tree)
{
    if (n_tree < 1 || parent[0] != -1)
        return 0;
    for (int i = 1; i < n_tree; ++i)
        if (parent[i] < 0 || parent[i] >= i)
            return 0;
    return 1;
}

/*
 * Tree-masked attention of draft-tree node `node`, query head `h`.
 *
 * Definition (tree-based verification against the full KV cache, aiboss88
 * "technical principles"; tencent parallel-verification figure): node i sees
 * every context position [0, n_ctx) and, in the tree tail [n_ctx, n_ctx+T),
 * exactly the positions of the nodes on its root path, itself included --
 * the tokens that would precede it in ordinary autoregressive decoding.
 * Query head h reads KV head h / (Hq / Hkv) (grouped-query attention).
 *
 *   s_j   = scale * sum_d q[node,h,d] * k[g,j,d]
 *   out_d = sum_j exp(s_j - max s) v[g,j,d] / sum_j exp(s_j - max s)
 *
 * Reading: the root (node 0) is the last accepted token; its K/V row sits at
 * the first tail position and the context excludes it.
 */
static void attend_one(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                       int64_t kv_cap, int n_heads_q, int n_heads_kv, int head_dim,
                       int n_ctx, int n_tree, const int32_t *parent, double scale,
                       int node, int h, double *out)
{
    const int group = n_heads_q / n_heads_kv;
    const int g = h / group;
    const uint16_t *qrow = q + ((int64_t)node * n_heads_q + h) * head_dim;
    const uint16_t *kh = k + (int64_t)g * kv_cap * head_dim;
    const uint16_t *vh = v + (int64_t)g * kv_cap * head_dim;

    /* visible positions: the context, then the root path of `node` */
    int64_t n_vis = n_ctx;
    int64_t *pos = (int64_t *)malloc(sizeof(int64_t) * (size_t)(n_ctx + n_tree));
    double *s = (double *)malloc(sizeof(double) * (size_t)(n_ctx + n_tree));
    for (int64_t j = 0; j < n_ctx; ++j)
        pos[j] = j;
    for (int a = node; a >= 0; a = parent[a])
        pos[n_vis++] = (int64_t)n_ctx + a;

    double m = -INFINITY;
    for (int64_t t = 0; t < n_vis; ++t) {
        const uint16_t *krow = kh + pos[t] * head_dim;
        double dot = 0.0;
        for (int d = 0; d < head_dim; ++d)
            dot += bf16_value(qrow[d]) * bf16_value(krow[d]);
        s[t] = scale * dot;
        if (s[t] > m)
            m = s[t];
    }
    double z = 0.0;
    for (int64_t t = 0; t < n_vis; ++t) {
        s[t] = exp(s[t] - m);
        z += s[t];
    }
    for (int d = 0; d < head_dim; ++d)
        out[d] = 0.0;
    for (int64_t t = 0; t < n_vis; ++t) {
        const uint16_t *vrow = vh + pos[t] * head_dim;
        for (int d = 0; d < head_dim; ++d)
            out[d] += s[t] * bf16_value(vrow[d]);
    }
    for (int d = 0; d < head_dim; ++d)
        out[d] /= z;
    free(pos);
    free(s);
}

static int attn_args_ok(int64_t kv_cap, int n_heads_q, int n_heads_kv, int head_dim,
                        int n_ctx, int n_tree, const int32_t *parent)
{
    if (n_heads_q < 1 || n_heads_kv < 1 || head_dim < 1 || n_heads_q % n_heads_kv)
        return 0;
    if (n_ctx < 0 || !tree_is_valid(parent, n_tree))
        return 0;
    return kv_cap >= (int64_t)n_ctx + n_tree;
}

/* All outputs: out is fp64 [T, Hq, D].  Returns 0, or -1 on invalid input. */
int tso_tree_verify_attn(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                         int64_t kv_cap, int n_heads_q, int n_heads_kv, int head_dim,
                         int n_ctx, int n_tree, const int32_t *parent, double scale,
                         double *out)
{
    if (!attn_args_ok(kv_cap, n_heads_q, n_heads_kv, head_dim, n_ctx, n_tree, parent))
        return -1;
    const int rows = n_tree * n_heads_q;
#pragma omp parallel for schedule(dynamic)
    for (int r = 0; r < rows; ++r)
        attend_one(q, k, v, kv_cap, n_heads_q, n_heads_kv, head_dim, n_ctx, n_tree, parent,
                   scale, r / n_heads_q, r % n_heads_q, out + (int64_t)r * head_dim);
    return 0;
}

/* Selected outputs only: row r is (node[r], head[r]); out is fp64 [n_rows, D]. */
int tso_tree_verify_attn_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                              int64_t kv_cap, int n_heads_q, int n_heads_kv, int head_dim,
                              int n_ctx, int n_tree, const int32_t *parent, double scale,
                              const int32_t *node, const int32_t *head, int n_rows,
                              double *out)
{
    if (!attn_args_ok(kv_cap, n_heads_q, n_heads_kv, head_dim, n_ctx, n_tree, parent))
        return -1;
    for (int r = 0; r < n_rows; ++r)
        if (node[r] < 0 || node[r] >= n_tree || head[r] < 0 || head[r] >= n_heads_q)
            return -1;
#pragma omp parallel for schedule(dynamic)
    for (int r = 0; r < n_rows; ++r)
        attend_one(q, k, v, kv_cap, n_heads_q, n_heads_kv, head_dim, n_ctx, n_tree, parent,
                   scale, node[r], head[r], out + (int64_t)r * head_dim);
    return 0;
}

/*
 * Token importance for the dynamic partial-KV update (aiboss88 "technical
 * principles": the cache after the initial tokens is replaced in order of
 * token importance; tencent 动态KV缓存更新).  The pages do not print the
 * score; the one used here is the softmax attention weight of the last
 * query over the context, averaged over the query heads of each KV group:
 *
 *   score[g,n] = (1/G) sum_{h in group g} exp(s_hn - m_h) / sum_n' exp(s_hn' - m_h)
 *   s_hn = scale * q_last[h] . k[g,n],   n, n' in [0, n_ctx)
 *
 * Readings: q_last is the root (node 0) query, [Hq, D]; the softmax spans
 * the whole context, sinks included, and excludes the tree tail.
 * scores: fp64 [Hkv, n_ctx].
 */
int tso_importance_scores(const uint16_t *q_last, const uint16_t *k, int64_t kv_cap,
                          int n_heads_q, int n_heads_kv, int head_dim, int n_ctx,
                          double scale, double *scores)
{
    if (n_heads_q < 1 || n_heads_kv < 1 || n_heads_q % n_heads_kv || n_ctx < 0 ||
        kv_cap < n_ctx)
        return -1;
    const int group = n_heads_q / n_heads_kv;
#pragma omp parallel for
    for (int g = 0; g < n_heads_kv; ++g) {
        double *sc = scores + (int64_t)g * n_ctx;
        double *s = (double *)malloc(sizeof(double) * (size_t)(n_ctx > 0 ? n_ctx : 1));
        for (int n = 0; n < n_ctx; ++n)
            sc[n] = 0.0;
        for (int h = g * group; h < (g + 1) * group; ++h) {
            const uint16_t *qrow = q_last + (int64_t)h * head_dim;
            double m = -INFINITY;
            for (int n = 0; n < n_ctx; ++n) {
                const uint16_t *krow = k + ((int64_t)g * kv_cap + n) * head_dim;
                double dot = 0.0;
                for (int d = 0; d < head_dim; ++d)
                    dot += bf16_value(qrow[d]) * bf16_value(krow[d]);
                s[n] = scale * dot;
                if (s[n] > m)
                    m = s[n];
            }
            double z = 0.0;
            for (int n = 0; n < n_ctx; ++n) {
                s[n] = exp(s[n] - m);
                z += s[n];
            }
            for (int n = 0; n < n_ctx; ++n)
                sc[n] += s[n] / z / (double)group;
        }
        free(s);
    }
    return 0;
}

typedef struct {
    double score;
    int32_t pos;
} cand_t;

/* higher score first; equal scores: lower position first */
static int cand_cmp(const void *a, const void *b)
{
    const cand_t *x = (const cand_t *)a, *y = (const cand_t *)b;
    if (x->score > y->score)
        return -1;
    if (x->score < y->score)
        return 1;
    return (x->pos > y->pos) - (x->pos < y->pos);
}

static int int_cmp(const void *a, const void *b)
{
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

/*
 * Retained set of the partial cache for each KV head (aiboss88 "technical
 * principles": keep the initial KV cache, replace the later part by
 * importance).  Readings: the first n_sink positions are always kept and
 * are not candidates; of [n_sink, n_ctx) the `budget` highest-scoring
 * positions are kept, equal scores going to the lower position; if
 * n_ctx <= n_sink + budget everything is kept; the list is ascending.
 * idx: [Hkv, n_keep] with n_keep = min(n_ctx, n_sink + budget).
 * Returns n_keep, or -1 on invalid input.
 */
int tso_select_topk(const double *scores, int n_heads_kv, int n_ctx, int n_sink, int budget,
                    int32_t *idx)
{
    if (n_heads_kv < 1 || n_ctx < 0 || n_sink < 0 || budget < 0)
        return -1;
    int64_t want = (int64_t)n_sink + budget;
    const int n_keep = want < n_ctx ? (int)want : n_ctx;
    for (int g = 0; g < n_heads_kv; ++g) {
        int32_t *out = idx + (int64_t)g * n_keep;
        if (n_keep == n_ctx) {
            for (int n = 0; n < n_ctx; ++n)
                out[n] = n;
            continue;
        }
        const double *sc = scores + (int64_t)g * n_ctx;
        const int n_cand = n_ctx - n_sink;
        cand_t *c = (cand_t *)malloc(sizeof(cand_t) * (size_t)(n_cand > 0 ? n_cand : 1));
        for (int t = 0; t < n_cand; ++t) {
            c[t].score = sc[n_sink + t];
            c[t].pos = n_sink + t;
        }
        qsort(c, (size_t)n_cand, sizeof(cand_t), cand_cmp);
        int w = 0;
        for (int n = 0; n < n_sink; ++n)
            out[w++] = n;
        for (int t = 0; t < budget; ++t)
            out[w++] = c[t].pos;
        qsort(out, (size_t)n_keep, sizeof(int32_t), int_cmp);
        free(c);
    }
    return n_keep;
}

/* Copy the retained rows into the compact draft cache [Hkv, partial_cap, D]. */
int tso_gather_rows(const uint16_t *src, int64_t kv_cap, int n_heads_kv, int head_dim,
                    const int32_t *idx, int n_keep, uint16_t *dst, int64_t partial_cap)
{
    if (partial_cap < n_keep)
        return -1;
    for (int g = 0; g < n_heads_kv; ++g)
        for (int t = 0; t < n_keep; ++t) {
            int32_t n = idx[(int64_t)g * n_keep + t];
            if (n < 0 || n >= kv_cap)
                return -1;
            memcpy(dst + ((int64_t)g * partial_cap + t) * head_dim,
                   src + ((int64_t)g * kv_cap + n) * head_dim, sizeof(uint16_t) * head_dim);
        }
    return 0;
}

/*
 * Contextual penalty, then the target argmax of every tree node
 * (aiboss88 "technical principles": a penalty on recently generated tokens;
 * tencent 上下文惩罚: generation probabilities are adjusted).
 *
 * For each id in the window (a set: an id listed twice is penalised once),
 * a positive logit is divided by the penalty and a non-positive one is
 * multiplied by it; other logits are unchanged.  The arithmetic is binary32
 * with round-to-nearest, as the path computes it, so that the integer
 * decision (the argmax) is taken in the same precision on both sides.
 * argmax: the largest penalised logit, ties to the lowest id; a NaN counts
 * as -inf.  Returns 0, or -1 on invalid input (an id outside [0, V)).
 */
int tso_penalize_argmax(const float *logits, int n_tree, int vocab, const int32_t *window,
                        int window_len, float penalty, int32_t *argmax, float *penalized)
{
    if (n_tree < 0 || vocab < 1 || window_len < 0 || !(penalty > 0.0f))
        return -1;
    unsigned char *in_window = (unsigned char *)calloc((size_t)vocab, 1);
    for (int w = 0; w < window_len; ++w) {
        if (window[w] < 0 || window[w] >= vocab) {
            free(in_window);
            return -1;
        }
        in_window[window[w]] = 1;
    }
    for (int i = 0; i < n_tree; ++i) {
        float best = -INFINITY;
        int32_t best_id = 0;
        for (int id = 0; id < vocab; ++id) {
            float x = logits[(int64_t)i * vocab + id];
            if (in_window[id])
                x = x > 0.0f ? x / penalty : x * penalty;
            if (penalized)
                penalized[(int64_t)i * vocab + id] = x;
            if (x != x)
                x = -INFINITY;
            if (x > best) {
                best = x;
                best_id = id;
            }
        }
        argmax[i] = best_id;
    }
    free(in_window);
    return 0;
}

/*
 * Longest accepted path (aiboss88 "technical principles": the longest valid
 * candidate is kept; tencent figure text: the longest valid candidate, e.g.
 * "is the father of", is the output).  Greedy reading: the root is valid; a
 * draft node is valid when its parent is valid and its token equals the
 * target argmax at its parent, so a valid path is exactly what ordinary
 * greedy decoding would have produced.  The output is the root path of the
 * deepest valid node; equal depths go to the lowest node index.
 *
 * out (int32[2 + T]): out[0] = accepted draft nodes L (the depth of that
 * node), out[1] = bonus token (the argmax at that node), out[2 .. 2+L] = the
 * path's node indices starting with the root 0.  Returns L, or -1 on
 * invalid input.
 */
int tso_accept_longest(const int32_t *parent, const int32_t *tokens, const int32_t *argmax,
                       int n_tree, int32_t *out)
{
    if (!tree_is_valid(parent, n_tree))
        return -1;
    int *valid = (int *)malloc(sizeof(int) * (size_t)n_tree);
    int *depth = (int *)malloc(sizeof(int) * (size_t)n_tree);
    valid[0] = 1;
    depth[0] = 0;
    int best = 0;
    for (int i = 1; i < n_tree; ++i) {
        int p = parent[i];
        valid[i] = valid[p] && tokens[i] == argmax[p];
        depth[i] = depth[p] + 1;
        if (valid[i] && depth[i] > depth[best])
            best = i;
    }
    const int len = depth[best];
    int node = best;
    for (int t = len; t >= 0; --t) {
        out[2 + t] = node;
        node = parent[node];
    }
    out[0] = len;
    out[1] = argmax[best];
    free(valid);
    free(depth);
    return len;
}

/*
 * Contextual penalty with each node's own draft path in its window, then
 * the target argmax of every tree node (aiboss88 "Contextual penalty
 * strategy": the penalty falls on recently generated tokens).  The logits of
 * node i give the token that would follow i, and the tokens most recently
 * generated before it are those of i's own draft path.  Reading: node i's
 * window is the caller's window together with the tokens of the draft nodes
 * on i's root path (i included; the root, the last accepted token, is
 * already in the caller's window and its entry of `tokens` is not read),
 * taken as one set.  Penalty and argmax rules as in tso_penalize_argmax.
 * Returns 0, or -1 on invalid input (a window id or a draft token outside
 * [0, V), or an invalid tree).
 */
int tso_penalize_argmax_path(const float *logits, int n_tree, int vocab, const int32_t *window,
                             int window_len, float penalty, const int32_t *parent,
                             const int32_t *tokens, int32_t *argmax, float *penalized)
{
    if (n_tree < 1 || vocab < 1 || window_len < 0 || !(penalty > 0.0f) ||
        !tree_is_valid(parent, n_tree))
        return -1;
    for (int i = 1; i < n_tree; ++i)
        if (tokens[i] < 0 || tokens[i] >= vocab)
            return -1;
    unsigned char *in_window = (unsigned char *)calloc((size_t)vocab, 1);
    for (int w = 0; w < window_len; ++w) {
        if (window[w] < 0 || window[w] >= vocab) {
            free(in_window);
            return -1;
        }
        in_window[window[w]] = 1;
    }
    unsigned char *mark = (unsigned char *)malloc((size_t)vocab);
    for (int i = 0; i < n_tree; ++i) {
        memcpy(mark, in_window, (size_t)vocab);
        for (int a = i; a != 0; a = parent[a])
            mark[tokens[a]] = 1;
        float best = -INFINITY;
        int32_t best_id = 0;
        for (int id = 0; id < vocab; ++id) {
            float x = logits[(int64_t)i * vocab + id];
            if (mark[id])
                x = (x > 0.0f) ? (x / penalty) : (x * penalty);
            if (penalized)
                penalized[(int64_t)i * vocab + id] = x;
            if (x != x)
                x = -INFINITY;
            if (best < x) {
                best = x;
                best_id = id;
            }
        }
        argmax[i] = best_id;
    }
    free(mark);
    free(in_window);
    return 0;
}

/*
 * Longest accepted path with a random choice among equally long valid paths
 * (aiboss88 "Tree-based multi-candidate token verification": the longest
 * valid n-gram is selected at random).  Validity as in tso_accept_longest.
 * Reading: the deepest valid nodes are listed in ascending index (BFS)
 * order; with c of them, the one at position (r mod c) is kept, r being a
 * random 64-bit integer the caller draws.  Output as tso_accept_longest.
 * Returns L, or -1 on invalid input.
 */
int tso_accept_longest_random(const int32_t *parent, const int32_t *tokens,
                              const int32_t *argmax, int n_tree, uint64_t r, int32_t *out)
{
    if (!tree_is_valid(parent, n_tree))
        return -1;
    int *valid = (int *)malloc(sizeof(int) * (size_t)n_tree);
    int *depth = (int *)malloc(sizeof(int) * (size_t)n_tree);
    valid[0] = 1;
    depth[0] = 0;
    int deepest = 0;
    for (int i = 1; i < n_tree; ++i) {
        int p = parent[i];
        valid[i] = tokens[i] == argmax[p] && valid[p];
        depth[i] = depth[p] + 1;
        if (valid[i] && depth[i] > deepest)
            deepest = depth[i];
    }
    int count = 0;
    for (int i = 0; i < n_tree; ++i)
        count += valid[i] && depth[i] == deepest;
    int pick = (int)(r % (uint64_t)count), best = 0;
    for (int i = 0; i < n_tree; ++i)
        if (valid[i] && depth[i] == deepest && pick-- == 0) {
            best = i;
            break;
        }
    const int len = depth[best];
    int node = best;
    for (int t = len; t >= 0; --t) {
        out[2 + t] = node;
        node = parent[node];
    }
    out[0] = len;
    out[1] = argmax[best];
    free(valid);
    free(depth);
    return len;
}

/*
 * Temperature acceptance: the target token of every tree node is a draw from
 * the tempered distribution softmax(penalised logits / temperature) instead
 * of its argmax (aiboss88 "Tree-based multi-candidate token verification":
 * the output stays lossless, i.e. distributed as the target model's own
 * sampling, while the choice gains diversity).  Reading: the draw is the
 * Gumbel-max rule -- the id maximising penalised / temperature + g, with
 * g[i][id] independent standard Gumbel noise drawn by the caller -- whose
 * result is distributed exactly as that softmax.  A draft node is then valid
 * when its parent is valid and its token equals the draw at its parent, so
 * every accepted token is the target's own sample given the tokens before
 * it; acceptance itself is tso_accept_longest (or _random) with the draws in
 * place of the argmax.
 *
 * `penalized` is the fp32 output of tso_penalize_argmax (or _path).  Each
 * node's score is computed in binary32, round-to-nearest, one rounding per
 * operation: the quotient, then the sum with g, so that the integer decision
 * is taken in the same precision as the path takes it.  The draw is the
 * largest score, ties to the lowest id, a NaN counting as -inf.  Returns 0,
 * or -1 when the temperature is not a finite positive number.
 */
int tso_sample_targets(const float *penalized, const float *gumbel, int n_tree, int vocab,
                       float temperature, int32_t *target)
{
    if (n_tree < 0 || vocab < 1 || !(temperature > 0.0f) || !(temperature <= FLT_MAX))
        return -1;
    for (int i = 0; i < n_tree; ++i) {
        float best = -INFINITY;
        int32_t best_id = 0;
        for (int id = 0; id < vocab; ++id) {
            const int64_t at = (int64_t)i * vocab + id;
            float z = penalized[at] / temperature;
            z = z + gumbel[at];
            if (z != z)
                z = -INFINITY;
            if (best < z) {
                best = z;
                best_id = id;
            }
        }
        target[i] = best_id;
    }
    return 0;
}

/*
 * Commit of the accepted path into the cache (tencent parallel-verification
 * figure: the candidates are verified against the full KV cache, the
 * longest valid one is kept and the state is updated for the next step).
 * The tree's K/V rows sit at n_ctx + node; after acceptance the accepted
 * path's rows become the next context rows in path order: row n_ctx + j
 * takes the row of path node path[j], j = 0 .. L (path[0] = 0, the root, at
 * n_ctx already).  Rows past n_ctx + L are left as they were.  `accept` is
 * the int32 {L, bonus, path[0..L]} of tso_accept_longest.  Operates on one
 * cache (K or V) [Hkv, kv_cap, D] in place.  Returns 0, or -1 on invalid
 * input.
 */
int tso_kv_commit_path(uint16_t *cache, int64_t kv_cap, int n_heads_kv, int head_dim, int n_ctx,
                       int n_tree, const int32_t *accept)
{
    const int len = accept[0];
    if (len < 0 || len >= n_tree || (int64_t)n_ctx + n_tree > kv_cap)
        return -1;
    for (int j = 0; j <= len; ++j)
        if (accept[2 + j] < j || accept[2 + j] >= n_tree)
            return -1;
    uint16_t *rows = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)(len + 1) * head_dim);
    for (int g = 0; g < n_heads_kv; ++g) {
        uint16_t *base = cache + (int64_t)g * kv_cap * head_dim;
        /* every source row is read before any row is written */
        for (int j = 0; j <= len; ++j)
            memcpy(rows + (size_t)j * head_dim, base + ((int64_t)n_ctx + accept[2 + j]) * head_dim,
                   sizeof(uint16_t) * head_dim);
        for (int j = 0; j <= len; ++j)
            memcpy(base + ((int64_t)n_ctx + j) * head_dim, rows + (size_t)j * head_dim,
                   sizeof(uint16_t) * head_dim);
    }
    free(rows);
    return 0;
}
