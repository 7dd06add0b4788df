// attn_common.cuh -- pieces shared by the two tree-verify attention kernels
// (tcgen05 and mma.sync) and the dispatch between them.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include "ts_internal.cuh"

namespace ts {

struct AttnPlan {
    int n_split;          // KV splits per head
    int tiles_per_split;  // KV tiles each split streams
    int node_groups = 1;      // tree-node groups, one CTA each per (split, head)
    int nodes_per_group = 0;  // nodes of each group (the last may have fewer)
};

// The tcgen05 kernel feeds P to the PV product as one bf16 value; that is
// exact enough (<= 1e-4 class) once attention is spread over thousands of
// positions.  Shorter contexts, where a few weights can dominate, go to the
// mma.sync kernel, which splits P into two bf16 parts.
constexpr int kTcMinContext = 2048;

// Split partials share one layout: acc fp32 [n_split, T*Hq, D] after the
// workspace header, then (m, l) fp32 [n_split, T*Hq, 2]; m is in log2 units.
inline size_t attn_partial_bytes(int n_split, int n_heads_q, int head_dim, int n_tree)
{
    return (size_t)n_split * n_tree * n_heads_q * (head_dim + 2) * sizeof(float);
}
cudaError_t attn_combine_launch(const AttnArgs &a, int n_split, cudaStream_t stream);

size_t attn_mma_workspace_bytes(int n_heads_q, int n_heads_kv, int head_dim, int n_ctx,
                                int n_tree, int num_sms);
cudaError_t attn_mma_launch(const AttnArgs &a, const TreeMasks &masks, int num_sms,
                            cudaStream_t stream);

// Tensor map over a bf16 [Hkv, kv_cap, head_dim] cache viewed as 3-D (d,
// position, head), 128-byte swizzle, boxes of 64 columns x box_rows
// positions; positions at or past `rows` read as zeros.
bool encode_kv_map(CUtensorMap *m, const void *ptr, int rows, int64_t kv_cap, int n_heads_kv,
                   int box_rows, int head_dim = 128);

// Split partials of the tcgen05 kernels (head_dim 128): acc fp32
// [n_split, T*Hq, 128] after the workspace header, then (m, l, q, 0) fp32
// [n_split, T*Hq, 4]: m in log2 units, l the sum of the bf16-rounded
// weights relative to 2^m, q the sum of their squares.  The combine folds them; it recomputes exactly (fp32, CUDA
// cores) every split whose int32 flag [n_split, Hkv] is set (flags may be
// null: none), and the heavy splits of rows whose weight sits on too few
// positions for bf16 weights.  split_positions: KV positions per split.
size_t attn_exact_partial_bytes(int n_split, int n_heads_q, int n_tree);
// flags: n_flag_groups int32 per (split, KV head), any of them set flags
// the split of that head.
cudaError_t attn_exact_combine_launch(const AttnArgs &a, const TreeMasks &masks, int n_split,
                                      int split_positions, const int32_t *flags,
                                      int n_flag_groups, cudaStream_t stream);

// 128-position tiles, softmax spread over the four SM sub-partitions; up to
// 192 query rows per KV head in one CTA, more split into groups of tree
// nodes with one CTA each.
bool attn_t128_eligible(int n_heads_q, int n_heads_kv, int head_dim, int n_ctx, int n_tree);
AttnPlan attn_t128_plan(int n_heads_q, int n_heads_kv, int n_ctx, int n_tree, int num_sms);
size_t attn_t128_workspace_bytes(int n_heads_q, int n_heads_kv, int n_ctx, int n_tree, int num_sms);
cudaError_t attn_t128_launch(const AttnArgs &a, const TreeMasks &masks, int num_sms,
                             cudaStream_t stream);
// whether that kernel writes a.root_scores itself (G <= 8 root rows inside
// the first 16 TMEM lanes); otherwise it ignores them
bool attn_t128_leaves_root_scores(const AttnArgs &a);

}  // namespace ts
