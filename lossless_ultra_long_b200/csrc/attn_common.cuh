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

// 128-position tiles, softmax spread over the four SM sub-partitions; up to
// 192 query rows per KV head in one CTA, more split into groups of tree
// nodes with one CTA each.  The splits of a (head, group) take KV tiles at
// run time and fold their partials themselves (one cooperative launch).
bool attn_t128_eligible(int n_heads_q, int n_heads_kv, int head_dim, int n_ctx, int n_tree);
AttnPlan attn_t128_plan(int n_heads_q, int n_heads_kv, int n_ctx, int n_tree, int num_sms);
// whether its grid (one CTA per SM, all resident: a cooperative launch) fits
// the device; more (KV head, node group) pairs than SMs go to the other kernel
bool attn_t128_fits(int n_heads_q, int n_heads_kv, int n_ctx, int n_tree, int num_sms);
size_t attn_t128_workspace_bytes(int n_heads_q, int n_heads_kv, int n_ctx, int n_tree, int num_sms);
// leading bytes of that workspace (header included) that must be zero when
// a call starts; every call leaves them so
size_t attn_t128_zeroed_bytes(int n_heads_q, int n_heads_kv, int n_ctx, int n_tree, int num_sms);
cudaError_t attn_t128_launch(const AttnArgs &a, const TreeMasks &masks, int num_sms,
                             cudaStream_t stream);
// whether that kernel writes a.root_scores itself (G <= 8 root rows inside
// the first 16 TMEM lanes); otherwise it ignores them
bool attn_t128_leaves_root_scores(const AttnArgs &a);

}  // namespace ts
