// attn_dispatch.cu -- picks the tree-verify attention kernel for a shape.
//
// head_dim 128, at most 256 query rows per KV head (G * T) and a context of
// at least kTcMinContext positions run on the tcgen05 kernel; everything
// else (head_dim 64, larger groups or trees, short contexts) on the general
// mma.sync kernel.  The choice depends only on the shape, so the workspace
// size query and the launch always agree.
#include "attn_common.cuh"

namespace ts {

size_t attn_workspace_bytes(int n_heads_q, int n_heads_kv, int head_dim, int n_ctx, int n_tree,
                            int num_sms)
{
    if (attn_tc_eligible(n_heads_q, n_heads_kv, head_dim, n_ctx, n_tree)) {
        const AttnPlan p = attn_tc_plan(n_heads_q, n_heads_kv, n_ctx, n_tree, num_sms);
        return kHeaderBytes + align_up(attn_partial_bytes(p.n_split, n_heads_q, head_dim, n_tree),
                                       256);
    }
    return attn_mma_workspace_bytes(n_heads_q, n_heads_kv, head_dim, n_ctx, n_tree, num_sms);
}

cudaError_t attn_launch(const AttnArgs &a, const TreeMasks &masks, int num_sms,
                        cudaStream_t stream)
{
    if (attn_tc_eligible(a.n_heads_q, a.n_heads_kv, a.head_dim, a.n_ctx, a.n_tree))
        return attn_tc_launch(a, masks, num_sms, stream);
    return attn_mma_launch(a, masks, num_sms, stream);
}

}  // namespace ts
