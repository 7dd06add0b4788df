// attn_dispatch.cu -- picks the tree-verify attention kernel for a shape.
//
// head_dim 128, a context of at least kTcMinContext positions and a
// positive softmax scale run on the tcgen05 kernel with 128-position tiles
// (up to 192 query rows per KV head in one CTA, more in groups of tree nodes
// of at most 128 rows).  Everything else (head_dim 64, groups over 128
// heads, short contexts) runs on the general mma.sync kernel.  The
// workspace size covers whichever kernel a launch picks.
#include <mutex>

#include "attn_common.cuh"

namespace ts {

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000,
                                             cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        else
            cudaGetLastError();
    });
    return fn;
}

bool encode_kv_map(CUtensorMap *m, const void *ptr, int rows, int64_t kv_cap, int n_heads_kv,
                   int box_rows, int head_dim)
{
    auto enc = tensor_map_encoder();
    if (!enc)
        return false;
    const cuuint64_t dims[3] = {(cuuint64_t)head_dim, (cuuint64_t)rows, (cuuint64_t)n_heads_kv};
    const cuuint64_t strides[2] = {(cuuint64_t)head_dim * 2, (cuuint64_t)kv_cap * head_dim * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t attn_workspace_bytes(int n_heads_q, int n_heads_kv, int head_dim, int n_ctx, int n_tree,
                            int num_sms)
{
    // large enough for whichever kernel the launch picks
    size_t bytes = attn_mma_workspace_bytes(n_heads_q, n_heads_kv, head_dim, n_ctx, n_tree, num_sms);
    if (attn_t128_eligible(n_heads_q, n_heads_kv, head_dim, n_ctx, n_tree)) {
        const size_t t128 = attn_t128_workspace_bytes(n_heads_q, n_heads_kv, n_ctx, n_tree, num_sms);
        bytes = t128 > bytes ? t128 : bytes;
    }
    return bytes;
}

size_t attn_workspace_zeroed_bytes(int n_heads_q, int n_heads_kv, int head_dim, int n_ctx,
                                   int n_tree, int num_sms)
{
    size_t bytes = kHeaderBytes;
    if (attn_t128_eligible(n_heads_q, n_heads_kv, head_dim, n_ctx, n_tree)) {
        const size_t t128 = attn_t128_zeroed_bytes(n_heads_q, n_heads_kv, n_ctx, n_tree, num_sms);
        bytes = t128 > bytes ? t128 : bytes;
    }
    return bytes;
}

cudaError_t attn_launch(const AttnArgs &a, const TreeMasks &masks, int num_sms,
                        cudaStream_t stream)
{
    cudaError_t e;
    if (a.scale_log2 > 0.f &&
        attn_t128_eligible(a.n_heads_q, a.n_heads_kv, a.head_dim, a.n_ctx, a.n_tree) &&
        attn_t128_fits(a.n_heads_q, a.n_heads_kv, a.n_ctx, a.n_tree, num_sms)) {
        if (a.root_scores == nullptr || attn_t128_leaves_root_scores(a))
            return attn_t128_launch(a, masks, num_sms, stream);   // leaves root scores itself
        AttnArgs b = a;
        b.root_scores = nullptr;
        e = attn_t128_launch(b, masks, num_sms, stream);
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
