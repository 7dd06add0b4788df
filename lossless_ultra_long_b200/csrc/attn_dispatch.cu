// attn_dispatch.cu -- picks the tree-verify attention kernel for a shape.
//
// head_dim 128, a context of at least kTcMinContext positions and a
// positive softmax scale run on a tcgen05 kernel: the 128-position-tile one
// up to 192 query rows per KV head (G * T), the 64-position-tile one up to
// 224.  Everything else (head_dim 64, larger groups or trees, short
// contexts) runs on the general mma.sync kernel.  The workspace size covers
// whichever kernel a launch picks.
#include "attn_common.cuh"

namespace ts {

size_t attn_workspace_bytes(int n_heads_q, int n_heads_kv, int head_dim, int n_ctx, int n_tree,
                            int num_sms)
{
    // large enough for whichever kernel the launch picks
    size_t bytes = attn_mma_workspace_bytes(n_heads_q, n_heads_kv, head_dim, n_ctx, n_tree, num_sms);
    auto take = [&](const AttnPlan &p) {
        const size_t tc = kHeaderBytes +
                          align_up(attn_exact_partial_bytes(p.n_split, n_heads_q, n_tree), 256);
        bytes = tc > bytes ? tc : bytes;
    };
    if (attn_t128_eligible(n_heads_q, n_heads_kv, head_dim, n_ctx, n_tree)) {
        const size_t t128 = attn_t128_workspace_bytes(n_heads_q, n_heads_kv, n_ctx, n_tree, num_sms);
        bytes = t128 > bytes ? t128 : bytes;
    }
    if (attn_tc_eligible(n_heads_q, n_heads_kv, head_dim, n_ctx, n_tree))
        take(attn_tc_plan(n_heads_q, n_heads_kv, n_ctx, n_tree, num_sms));
    return bytes;
}

cudaError_t attn_launch(const AttnArgs &a, const TreeMasks &masks, int num_sms,
                        cudaStream_t stream)
{
    cudaError_t e;
    if (a.scale_log2 > 0.f &&
        attn_t128_eligible(a.n_heads_q, a.n_heads_kv, a.head_dim, a.n_ctx, a.n_tree)) {
        if (a.root_scores == nullptr || attn_t128_leaves_root_scores(a))
            return attn_t128_launch(a, masks, num_sms, stream);   // leaves root scores itself
        AttnArgs b = a;
        b.root_scores = nullptr;
        e = attn_t128_launch(b, masks, num_sms, stream);
    } else if (a.scale_log2 > 0.f &&
               attn_tc_eligible(a.n_heads_q, a.n_heads_kv, a.head_dim, a.n_ctx, a.n_tree)) {
        e = attn_tc_launch(a, masks, num_sms, stream);
    } else {
        e = attn_mma_launch(a, masks, num_sms, stream);
    }
    if (e != cudaSuccess || a.root_scores == nullptr || a.n_ctx == 0)
        return e;
    // the other kernels (and the 128-position one on trees of fewer than
    // four nodes) do not leave root scores: the select's score pass does
    SelectArgs sa = {};
    sa.q_last = a.q;   // node 0's rows [Hq, D]
    sa.k = a.k;
    sa.v = a.v;
    sa.kv_cap = a.kv_cap;
    sa.n_heads_q = a.n_heads_q;
    sa.n_heads_kv = a.n_heads_kv;
    sa.head_dim = a.head_dim;
    sa.n_ctx = a.n_ctx;
    sa.scale_log2 = a.scale_log2;
    sa.workspace = a.workspace;
    sa.workspace_bytes = a.workspace_bytes;
    return select_score_pass_launch(sa, a.root_scores, num_sms, stream);
}

}  // namespace ts
