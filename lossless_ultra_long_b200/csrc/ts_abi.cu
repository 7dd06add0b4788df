// ts_abi.cu -- the extern "C" entry points of libtsverify.so: argument
// validation, workspace sizing and launches.  Declarations and contracts
// are in include/ts_verify.h.
#include <math.h>
#include <string.h>

#include <atomic>

#include "ts_internal.cuh"

namespace ts {
static std::atomic<unsigned long long> g_launches{0};
void count_launches(unsigned n) { g_launches.fetch_add(n, std::memory_order_relaxed); }
}  // namespace ts

namespace ts {
int current_num_sms()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        cudaGetLastError();  // no device here: plan for a full B200
        return 148;
    }
    return n;
}
}  // namespace ts

namespace {

using ts::current_num_sms;

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool tree_ok(const int32_t *parent, int n_tree)
{
    if (!parent || n_tree < 1 || n_tree > TS_MAX_TREE || parent[0] != -1)
        return false;
    for (int i = 1; i < n_tree; ++i)
        if (parent[i] < 0 || parent[i] >= i)
            return false;
    return true;
}

bool shape_ok(int n_heads_q, int n_heads_kv, int head_dim)
{
    return n_heads_q >= 1 && n_heads_kv >= 1 && n_heads_q % n_heads_kv == 0 &&
           n_heads_q <= 1024;
}

bool head_dim_supported(int head_dim) { return head_dim == 64 || head_dim == 128; }

int workspace_ok(void *ws, size_t bytes, size_t need)
{
    if (!ws || !aligned(ws, 256) || bytes < need)
        return 0;
    return 1;
}

}  // namespace

extern "C" {

const char *ts_status_string(int status)
{
    switch (status) {
    case TS_OK: return "ok";
    case TS_ERR_INVALID_ARG: return "invalid argument";
    case TS_ERR_UNSUPPORTED: return "unsupported configuration";
    case TS_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case TS_ERR_CUDA: return "CUDA runtime error";
    case TS_ERR_TIMEOUT: return "device wait timed out";
    case TS_ERR_DEVICE_ARG: return "invalid data seen on the device";
    case TS_ERR_SCRATCH_LIMIT: return "problem needs more scratch than the no-alloc entry point holds";
    default: return "unknown status";
    }
}

int ts_version(void) { return 100; }

unsigned long long ts_kernel_launch_count(void) { return ts::g_launches.load(); }

size_t ts_tree_verify_attn_workspace_size(int n_heads_q, int n_heads_kv, int head_dim, int n_ctx,
                                          int n_tree)
{
    if (!shape_ok(n_heads_q, n_heads_kv, head_dim) || !head_dim_supported(head_dim) ||
        n_ctx < 0 || n_tree < 1 || n_tree > TS_MAX_TREE)
        return 0;
    return ts::attn_workspace_bytes(n_heads_q, n_heads_kv, head_dim, n_ctx, n_tree,
                                    current_num_sms());
}

extern "C++" {
namespace ts {

int attn_validate(const void *q, const void *k_cache, const void *v_cache, int64_t kv_cap,
                  int n_heads_q, int n_heads_kv, int head_dim, int n_ctx, int n_tree,
                  const int32_t *parent, float softmax_scale, const float *out)
{
    if (!q || !k_cache || !v_cache || !out || !shape_ok(n_heads_q, n_heads_kv, head_dim))
        return TS_ERR_INVALID_ARG;
    if (n_ctx < 0 || n_tree < 1 || n_tree > TS_MAX_TREE || !tree_ok(parent, n_tree))
        return TS_ERR_INVALID_ARG;
    if ((int64_t)n_ctx + n_tree > kv_cap || (int64_t)n_ctx + n_tree > INT32_MAX - 1024)
        return TS_ERR_INVALID_ARG;
    if (!isfinite(softmax_scale))
        return TS_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 16))
        return TS_ERR_INVALID_ARG;
    if (!head_dim_supported(head_dim))
        return TS_ERR_UNSUPPORTED;
    return TS_OK;
}

}  // namespace ts
}  // extern "C++"

namespace {

int attn_call(const void *q, const void *k_cache, const void *v_cache, int64_t kv_cap,
              int n_heads_q, int n_heads_kv, int head_dim, int n_ctx, int n_tree,
              const int32_t *parent, float softmax_scale, float *out, float *root_scores,
              void *workspace, size_t workspace_bytes, void *stream)
{
    const int st = ts::attn_validate(q, k_cache, v_cache, kv_cap, n_heads_q, n_heads_kv,
                                     head_dim, n_ctx, n_tree, parent, softmax_scale, out);
    if (st != TS_OK)
        return st;
    const int sms = current_num_sms();
    const size_t need = ts::attn_workspace_bytes(n_heads_q, n_heads_kv, head_dim, n_ctx, n_tree, sms);
    if (!workspace_ok(workspace, workspace_bytes, need))
        return TS_ERR_WORKSPACE;

    ts::TreeMasks masks;
    memset(&masks, 0, sizeof masks);
    for (int i = 0; i < n_tree; ++i)
        masks.anc[i] = (i ? masks.anc[parent[i]] : 0ull) | (1ull << i);

    ts::AttnArgs a;
    a.q = static_cast<const __nv_bfloat16 *>(q);
    a.k = static_cast<const __nv_bfloat16 *>(k_cache);
    a.v = static_cast<const __nv_bfloat16 *>(v_cache);
    a.out = out;
    a.kv_cap = kv_cap;
    a.n_heads_q = n_heads_q;
    a.n_heads_kv = n_heads_kv;
    a.head_dim = head_dim;
    a.n_ctx = n_ctx;
    a.n_tree = n_tree;
    a.scale_log2 = softmax_scale * 1.4426950408889634f;
    a.workspace = workspace;
    a.workspace_bytes = workspace_bytes;
    a.root_scores = root_scores;
    const cudaError_t e = ts::attn_launch(a, masks, sms, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TS_OK : TS_ERR_CUDA;
}

}  // namespace

int ts_tree_verify_attn(const void *q, const void *k_cache, const void *v_cache, int64_t kv_cap,
                        int n_heads_q, int n_heads_kv, int head_dim, int n_ctx, int n_tree,
                        const int32_t *parent, float softmax_scale, float *out,
                        void *workspace, size_t workspace_bytes, void *stream)
{
    return attn_call(q, k_cache, v_cache, kv_cap, n_heads_q, n_heads_kv, head_dim, n_ctx,
                     n_tree, parent, softmax_scale, out, nullptr, workspace, workspace_bytes,
                     stream);
}

int ts_tree_verify_attn_root_scores(const void *q, const void *k_cache, const void *v_cache,
                                    int64_t kv_cap, int n_heads_q, int n_heads_kv, int head_dim,
                                    int n_ctx, int n_tree, const int32_t *parent,
                                    float softmax_scale, float *out, float *root_scores_out,
                                    void *workspace, size_t workspace_bytes, void *stream)
{
    if (!root_scores_out || !aligned(root_scores_out, 4))
        return TS_ERR_INVALID_ARG;
    if (shape_ok(n_heads_q, n_heads_kv, head_dim) && n_heads_q / n_heads_kv > TS_MAX_SELECT_GROUP)
        return TS_ERR_UNSUPPORTED;
    return attn_call(q, k_cache, v_cache, kv_cap, n_heads_q, n_heads_kv, head_dim, n_ctx,
                     n_tree, parent, softmax_scale, out, root_scores_out, workspace,
                     workspace_bytes, stream);
}

size_t ts_kv_importance_select_workspace_size(int n_heads_q, int n_heads_kv, int head_dim,
                                              int n_ctx)
{
    if (!shape_ok(n_heads_q, n_heads_kv, head_dim) || !head_dim_supported(head_dim) || n_ctx < 1)
        return 0;
    return ts::select_workspace_bytes(n_heads_q, n_heads_kv, head_dim, n_ctx, current_num_sms());
}

int ts_kv_importance_select(const void *q_last, const void *k_cache, const void *v_cache,
                            int64_t kv_cap, int n_heads_q, int n_heads_kv, int head_dim,
                            int n_ctx, int n_sink, int budget, float softmax_scale,
                            float *scores_out, int32_t *idx_out, void *k_partial,
                            void *v_partial, int64_t partial_cap, void *workspace,
                            size_t workspace_bytes, void *stream)
{
    if (!q_last || !k_cache || !v_cache || !idx_out || !k_partial || !v_partial)
        return TS_ERR_INVALID_ARG;
    if (!shape_ok(n_heads_q, n_heads_kv, head_dim) || n_ctx < 1 || n_sink < 0 || budget < 0)
        return TS_ERR_INVALID_ARG;
    if ((int64_t)n_ctx > kv_cap || !isfinite(softmax_scale))
        return TS_ERR_INVALID_ARG;
    const int64_t want = (int64_t)n_sink + budget;
    const int n_keep = want < n_ctx ? (int)want : n_ctx;
    if (partial_cap < n_keep)
        return TS_ERR_INVALID_ARG;
    if (!aligned(q_last, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(k_partial, 16) || !aligned(v_partial, 16) || !aligned(idx_out, 4) ||
        (scores_out && !aligned(scores_out, 4)))
        return TS_ERR_INVALID_ARG;
    if (!head_dim_supported(head_dim) || !ts::select_supported(n_heads_q, n_heads_kv, head_dim, n_ctx))
        return TS_ERR_UNSUPPORTED;
    const int sms = current_num_sms();
    const size_t need = ts::select_workspace_bytes(n_heads_q, n_heads_kv, head_dim, n_ctx, sms);
    if (!workspace_ok(workspace, workspace_bytes, need))
        return TS_ERR_WORKSPACE;

    ts::SelectArgs a = {};
    a.q_last = static_cast<const __nv_bfloat16 *>(q_last);
    a.k = static_cast<const __nv_bfloat16 *>(k_cache);
    a.v = static_cast<const __nv_bfloat16 *>(v_cache);
    a.kv_cap = kv_cap;
    a.n_heads_q = n_heads_q;
    a.n_heads_kv = n_heads_kv;
    a.head_dim = head_dim;
    a.n_ctx = n_ctx;
    a.n_sink = n_sink;
    a.budget = budget;
    a.scale_log2 = softmax_scale * 1.4426950408889634f;
    a.scores_out = scores_out;
    a.idx_out = idx_out;
    a.k_partial = static_cast<__nv_bfloat16 *>(k_partial);
    a.v_partial = static_cast<__nv_bfloat16 *>(v_partial);
    a.partial_cap = partial_cap;
    a.workspace = workspace;
    a.workspace_bytes = workspace_bytes;
    const cudaError_t e = ts::select_launch(a, sms, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TS_OK : TS_ERR_CUDA;
}

size_t ts_kv_select_from_scores_workspace_size(int n_heads_q, int n_heads_kv, int n_ctx)
{
    if (!shape_ok(n_heads_q, n_heads_kv, 64) || n_ctx < 1)
        return 0;
    return ts::select_from_scores_workspace_bytes(n_heads_q, n_heads_kv, n_ctx, current_num_sms());
}

int ts_kv_select_from_scores(const float *root_scores, const void *k_cache, const void *v_cache,
                             int64_t kv_cap, int n_heads_q, int n_heads_kv, int head_dim,
                             int n_ctx, int n_sink, int budget, float *scores_out,
                             int32_t *idx_out, void *k_partial, void *v_partial,
                             int64_t partial_cap, void *workspace, size_t workspace_bytes,
                             void *stream)
{
    if (!root_scores || !k_cache || !v_cache || !idx_out || !k_partial || !v_partial)
        return TS_ERR_INVALID_ARG;
    if (!shape_ok(n_heads_q, n_heads_kv, head_dim) || n_ctx < 1 || n_sink < 0 || budget < 0)
        return TS_ERR_INVALID_ARG;
    if ((int64_t)n_ctx > kv_cap)
        return TS_ERR_INVALID_ARG;
    const int64_t want = (int64_t)n_sink + budget;
    const int n_keep = want < n_ctx ? (int)want : n_ctx;
    if (partial_cap < n_keep)
        return TS_ERR_INVALID_ARG;
    if (!aligned(root_scores, 4) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(k_partial, 16) || !aligned(v_partial, 16) || !aligned(idx_out, 4) ||
        (scores_out && !aligned(scores_out, 4)))
        return TS_ERR_INVALID_ARG;
    // the score rows are read 16 bytes at a time when n_ctx is a multiple of 4
    if ((n_ctx & 3) == 0 && !aligned(root_scores, 16))
        return TS_ERR_INVALID_ARG;
    if (!head_dim_supported(head_dim) || !ts::select_supported(n_heads_q, n_heads_kv, head_dim, n_ctx))
        return TS_ERR_UNSUPPORTED;
    const int sms = current_num_sms();
    if (!workspace_ok(workspace, workspace_bytes,
                      ts::select_from_scores_workspace_bytes(n_heads_q, n_heads_kv, n_ctx, sms)))
        return TS_ERR_WORKSPACE;

    ts::SelectArgs a = {};
    a.k = static_cast<const __nv_bfloat16 *>(k_cache);
    a.v = static_cast<const __nv_bfloat16 *>(v_cache);
    a.kv_cap = kv_cap;
    a.n_heads_q = n_heads_q;
    a.n_heads_kv = n_heads_kv;
    a.head_dim = head_dim;
    a.n_ctx = n_ctx;
    a.n_sink = n_sink;
    a.budget = budget;
    a.scores_out = scores_out;
    a.idx_out = idx_out;
    a.k_partial = static_cast<__nv_bfloat16 *>(k_partial);
    a.v_partial = static_cast<__nv_bfloat16 *>(v_partial);
    a.partial_cap = partial_cap;
    a.workspace = workspace;
    a.workspace_bytes = workspace_bytes;
    a.root_scores = root_scores;
    const cudaError_t e = ts::select_launch(a, sms, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TS_OK : TS_ERR_CUDA;
}

size_t ts_penalize_accept_workspace_size(int n_tree, int vocab)
{
    if (n_tree < 1 || n_tree > TS_MAX_TREE || vocab < 1)
        return 0;
    return ts::penalize_workspace_bytes(n_tree, vocab);
}

int ts_penalize_accept(const float *logits, int n_tree, int vocab, const int32_t *window,
                       int window_len, float penalty, const int32_t *parent,
                       const int32_t *tree_tokens, int32_t *argmax_out, int32_t *accept_out,
                       void *workspace, size_t workspace_bytes, void *stream)
{
    return ts_penalize_accept_ex(logits, n_tree, vocab, window, window_len, penalty, parent,
                                 tree_tokens, 0u, 0ull, argmax_out, accept_out, workspace,
                                 workspace_bytes, stream);
}

namespace {

// Both penalty entry points: gumbel == NULL takes the argmax, otherwise the
// temperature draw.
int penalize_accept_impl(const float *logits, const float *gumbel, float temperature,
                         int n_tree, int vocab, const int32_t *window, int window_len,
                         float penalty, const int32_t *parent, const int32_t *tree_tokens,
                         unsigned flags, uint64_t random, int32_t *argmax_out,
                         int32_t *accept_out, void *workspace, size_t workspace_bytes,
                         void *stream)
{
    if ((flags & ~(unsigned)(TS_PENALIZE_PATH_TOKENS | TS_ACCEPT_RANDOM_TIE)) != 0)
        return TS_ERR_INVALID_ARG;
    if (!logits || !tree_tokens || !accept_out || n_tree < 1 || n_tree > TS_MAX_TREE || vocab < 1)
        return TS_ERR_INVALID_ARG;
    if (window_len < 0 || (window_len > 0 && !window) || !(penalty > 0.0f) || !isfinite(penalty))
        return TS_ERR_INVALID_ARG;
    if (!tree_ok(parent, n_tree))
        return TS_ERR_INVALID_ARG;
    if (vocab > ts::penalize_max_vocab(gumbel != nullptr))
        return TS_ERR_UNSUPPORTED;
    if (!aligned(logits, 16) || !aligned(tree_tokens, 4) || !aligned(accept_out, 4) ||
        (window && !aligned(window, 4)) || (argmax_out && !aligned(argmax_out, 4)))
        return TS_ERR_INVALID_ARG;
    if (!workspace_ok(workspace, workspace_bytes, ts::penalize_workspace_bytes(n_tree, vocab)))
        return TS_ERR_WORKSPACE;

    ts::TreeParents tp;
    memset(&tp, 0, sizeof tp);
    for (int i = 0; i < n_tree; ++i)
        tp.parent[i] = static_cast<int8_t>(parent[i]);
    ts::PenalizeArgs a;
    a.logits = logits;
    a.n_tree = n_tree;
    a.vocab = vocab;
    a.window = window;
    a.window_len = window_len;
    a.penalty = penalty;
    a.tree_tokens = tree_tokens;
    a.argmax_out = argmax_out;
    a.accept_out = accept_out;
    a.workspace = workspace;
    a.workspace_bytes = workspace_bytes;
    a.flags = flags;
    a.random = random;
    a.gumbel = gumbel;
    a.temperature = temperature;
    const cudaError_t e =
        ts::penalize_launch(a, tp, current_num_sms(), static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TS_OK : TS_ERR_CUDA;
}

}  // namespace

int ts_penalize_accept_ex(const float *logits, int n_tree, int vocab, const int32_t *window,
                          int window_len, float penalty, const int32_t *parent,
                          const int32_t *tree_tokens, unsigned flags, uint64_t random,
                          int32_t *argmax_out, int32_t *accept_out, void *workspace,
                          size_t workspace_bytes, void *stream)
{
    return penalize_accept_impl(logits, nullptr, 1.0f, n_tree, vocab, window, window_len,
                                penalty, parent, tree_tokens, flags, random, argmax_out,
                                accept_out, workspace, workspace_bytes, stream);
}

int ts_penalize_sample_accept(const float *logits, const float *gumbel, float temperature,
                              int n_tree, int vocab, const int32_t *window, int window_len,
                              float penalty, const int32_t *parent, const int32_t *tree_tokens,
                              unsigned flags, uint64_t random, int32_t *target_out,
                              int32_t *accept_out, void *workspace, size_t workspace_bytes,
                              void *stream)
{
    if (!gumbel || !aligned(gumbel, 16) || !(temperature > 0.0f) || !isfinite(temperature))
        return TS_ERR_INVALID_ARG;
    return penalize_accept_impl(logits, gumbel, temperature, n_tree, vocab, window, window_len,
                                penalty, parent, tree_tokens, flags, random, target_out,
                                accept_out, workspace, workspace_bytes, stream);
}

int ts_kv_commit_path(void *k_cache, void *v_cache, int64_t kv_cap, int n_heads_kv,
                      int head_dim, int n_ctx, int n_tree, const int32_t *accept,
                      void *workspace, size_t workspace_bytes, void *stream)
{
    if (!k_cache || !v_cache || !accept || n_heads_kv < 1 || n_ctx < 0 || n_tree < 1 ||
        n_tree > TS_MAX_TREE)
        return TS_ERR_INVALID_ARG;
    if ((int64_t)n_ctx + n_tree > kv_cap)
        return TS_ERR_INVALID_ARG;
    if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(accept, 4))
        return TS_ERR_INVALID_ARG;
    if (!head_dim_supported(head_dim))
        return TS_ERR_UNSUPPORTED;
    if (!workspace_ok(workspace, workspace_bytes, ts::kHeaderBytes))
        return TS_ERR_WORKSPACE;
    ts::CommitArgs a;
    a.k = static_cast<__nv_bfloat16 *>(k_cache);
    a.v = static_cast<__nv_bfloat16 *>(v_cache);
    a.kv_cap = kv_cap;
    a.n_heads_kv = n_heads_kv;
    a.head_dim = head_dim;
    a.n_ctx = n_ctx;
    a.n_tree = n_tree;
    a.accept = accept;
    a.workspace = workspace;
    const cudaError_t e = ts::commit_launch(a, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TS_OK : TS_ERR_CUDA;
}

int ts_selftest_bounded_wait(void *workspace, size_t workspace_bytes, void *stream)
{
    if (!workspace_ok(workspace, workspace_bytes, ts::kHeaderBytes))
        return TS_ERR_WORKSPACE;
    const cudaError_t e =
        ts::selftest_bounded_wait_launch(workspace, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TS_OK : TS_ERR_CUDA;
}

int ts_workspace_status(const void *workspace, void *stream, int clear)
{
    if (!workspace)
        return TS_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t word = 0;
    if (cudaMemcpyAsync(&word, workspace, sizeof word, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return TS_ERR_CUDA;
    if (clear && word) {
        const uint32_t zero = 0;
        if (cudaMemcpyAsync(const_cast<void *>(workspace), &zero, sizeof zero,
                            cudaMemcpyHostToDevice, s) != cudaSuccess ||
            cudaStreamSynchronize(s) != cudaSuccess)
            return TS_ERR_CUDA;
    }
    return static_cast<int>(word);
}

}  // extern "C"
