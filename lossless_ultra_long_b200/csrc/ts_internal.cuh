// ts_internal.cuh -- shared definitions of the libtsverify kernels (not part
// of the public interface; the C ABI is include/ts_verify.h).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "ts_verify.h"

namespace ts {

// ---------------------------------------------------------------- workspace
// Every workspace starts with this header.  `status` collects device-side
// errors (ts_status codes, first one wins); the tickets serve "last CTA does
// the epilogue" hand-offs and are returned to zero by the CTA that takes
// the last ticket.
struct WorkspaceHeader {
    uint32_t status;
    uint32_t tickets[63];
};
static_assert(sizeof(WorkspaceHeader) == 256, "header is one 256-byte line");
constexpr size_t kHeaderBytes = sizeof(WorkspaceHeader);

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Host-side count of kernel launches issued by the library.
void count_launches(unsigned n);

// Launch with programmatic stream serialization: the kernel may be
// scheduled while the previous kernel on the stream is still running; it
// must call griddepcontrol.wait before it touches that kernel's results (and
// on every path, so that its own completion implies its predecessor's).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
    if (e == cudaSuccess)
        e = cudaGetLastError();
    if (e == cudaSuccess)
        count_launches(1);
    return e;
}

__device__ __forceinline__ void record_status(WorkspaceHeader *ws, uint32_t code)
{
    atomicCAS(&ws->status, 0u, code);
}

// Ancestor sets of the draft tree, bit a of anc[i] set iff node a is on the
// root path of node i (i included).  Passed by value as a kernel parameter.
struct TreeMasks {
    unsigned long long anc[TS_MAX_TREE];
};

struct TreeParents {
    int8_t parent[TS_MAX_TREE];
};

// ------------------------------------------------------------ launch entry
struct AttnArgs {
    const __nv_bfloat16 *q;
    const __nv_bfloat16 *k;
    const __nv_bfloat16 *v;
    float *out;
    int64_t kv_cap;
    int n_heads_q, n_heads_kv, head_dim;
    int n_ctx, n_tree;
    float scale_log2;   // softmax_scale * log2(e)
    void *workspace;
    size_t workspace_bytes;
    // optional: the root node's scores over the context, base 2
    // (scale_log2 * q[0, h] . k[g, n]), fp32 [Hq, n_ctx]; null if not wanted
    float *root_scores;
};

size_t attn_workspace_bytes(int n_heads_q, int n_heads_kv, int head_dim, int n_ctx, int n_tree,
                            int num_sms);
// Leading bytes of that workspace (header included) that must be zero when
// a call starts (every call leaves them zero, unless it recorded a
// device-side error).
size_t attn_workspace_zeroed_bytes(int n_heads_q, int n_heads_kv, int head_dim, int n_ctx,
                                   int n_tree, int num_sms);
// SM count of the current device (148 when none can be queried).
int current_num_sms();
// Host-side checks of a verify-attention call's arguments (everything but
// the workspace): TS_OK or the status the call returns.
int attn_validate(const void *q, const void *k_cache, const void *v_cache, int64_t kv_cap,
                  int n_heads_q, int n_heads_kv, int head_dim, int n_ctx, int n_tree,
                  const int32_t *parent, float softmax_scale, const float *out);
cudaError_t attn_launch(const AttnArgs &a, const TreeMasks &masks, int num_sms,
                        cudaStream_t stream);

struct SelectArgs {
    const __nv_bfloat16 *q_last;
    const __nv_bfloat16 *k;
    const __nv_bfloat16 *v;
    int64_t kv_cap;
    int n_heads_q, n_heads_kv, head_dim;
    int n_ctx, n_sink, budget;
    float scale_log2;
    float *scores_out;
    int32_t *idx_out;
    __nv_bfloat16 *k_partial;
    __nv_bfloat16 *v_partial;
    int64_t partial_cap;
    void *workspace;
    size_t workspace_bytes;
    // optional: base-2 root scores fp32 [Hq, n_ctx] computed elsewhere (by
    // the verify attention); when set, the score pass is skipped and q_last
    // and scale_log2 are unused
    const float *root_scores;
};

size_t select_workspace_bytes(int n_heads_q, int n_heads_kv, int head_dim, int n_ctx,
                              int num_sms);
size_t select_from_scores_workspace_bytes(int n_heads_q, int n_heads_kv, int n_ctx, int num_sms);
int select_supported(int n_heads_q, int n_heads_kv, int head_dim, int n_ctx);
cudaError_t select_launch(const SelectArgs &a, int num_sms, cudaStream_t stream);
// The score pass alone: base-2 root scores fp32 [Hq, n_ctx] into `out`.
cudaError_t select_score_pass_launch(const SelectArgs &a, float *out, int num_sms,
                                     cudaStream_t stream);

// One CTA waits, with the kernels' bounded wait, on a barrier nothing
// completes; the wait records TS_ERR_TIMEOUT after its bound.
cudaError_t selftest_bounded_wait_launch(void *workspace, cudaStream_t stream);

struct PenalizeArgs {
    const float *logits;
    int n_tree, vocab;
    const int32_t *window;
    int window_len;
    float penalty;
    const int32_t *tree_tokens;
    int32_t *argmax_out;
    int32_t *accept_out;
    void *workspace;
    size_t workspace_bytes;
    unsigned flags;              // TS_PENALIZE_PATH_TOKENS | TS_ACCEPT_RANDOM_TIE
    unsigned long long random;   // r of the random choice among the deepest valid nodes
    const float *gumbel;         // [n_tree, vocab] noise of the temperature draw, or null (argmax)
    float temperature;           // read only with gumbel
};

// Commit of the accepted path's tree rows into the context (one cache pair).
struct CommitArgs {
    __nv_bfloat16 *k;
    __nv_bfloat16 *v;
    int64_t kv_cap;
    int n_heads_kv, head_dim, n_ctx, n_tree;
    const int32_t *accept;   // device {L, bonus, path[0..L]}
    void *workspace;
};
cudaError_t commit_launch(const CommitArgs &a, cudaStream_t stream);

size_t penalize_workspace_bytes(int n_tree, int vocab);
// Largest vocabulary one penalty launch covers (its splits times the
// longest slice a CTA stages); `sample`: with the temperature draw's noise.
int penalize_max_vocab(bool sample);
cudaError_t penalize_launch(const PenalizeArgs &a, const TreeParents &parents, int num_sms,
                            cudaStream_t stream);

}  // namespace ts
