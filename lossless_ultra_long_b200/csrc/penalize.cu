// penalize.cu -- contextual penalty, per-node argmax and longest accepted
// path in one launch.
//
// TokenSwift (aiboss88.com), "TokenSwift's technical principles": a penalty
// on recently generated tokens; the longest valid candidate of the tree is
// kept.  Tencent article: 上下文惩罚 and the parallel-verification figure
// (the worked example keeps "is the father of", the longest valid candidate).
//
// Grid (vocab chunks, tree nodes).  Each CTA marks the window ids that fall
// in its chunk in a shared-memory bitmap, streams its slice of the logits
// row with 16-byte loads, penalises marked ids (binary32 divide / multiply,
// round-to-nearest) and reduces (value, id) with warp shuffles, ties to the
// lower id.  Its result goes to the workspace; the CTA that takes the last
// ticket reduces every node's chunks, writes the argmax, and walks the tree.
// The logits are read exactly once; HBM traffic is T * V * 4 bytes.
#include <float.h>
#include <limits.h>

#include "ts_internal.cuh"

namespace ts {
namespace {

constexpr int kThreads = 256;
constexpr int kChunk = 8192;            // vocab entries per CTA
constexpr int kBitWords = kChunk / 32;

struct Best {
    float v;
    int i;
};

__device__ __forceinline__ bool beats(float v1, int i1, float v2, int i2)
{
    return v1 > v2 || (v1 == v2 && i1 < i2);
}

__device__ __forceinline__ void consider(Best &b, float x, int id)
{
    if (x != x)
        x = -INFINITY;
    if (beats(x, id, b.v, b.i)) {
        b.v = x;
        b.i = id;
    }
}

__device__ __forceinline__ Best warp_best(Best b)
{
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        float ov = __shfl_xor_sync(0xffffffffu, b.v, off);
        int oi = __shfl_xor_sync(0xffffffffu, b.i, off);
        if (beats(ov, oi, b.v, b.i)) {
            b.v = ov;
            b.i = oi;
        }
    }
    return b;
}

__device__ __forceinline__ float penalise(float x, float p)
{
    return x > 0.0f ? __fdiv_rn(x, p) : __fmul_rn(x, p);
}

__global__ void __launch_bounds__(kThreads)
penalize_accept_kernel(PenalizeArgs a, TreeParents tree, int n_chunks)
{
    __shared__ uint32_t bits[kBitWords];
    __shared__ Best warp_res[kThreads / 32];
    __shared__ int am[TS_MAX_TREE];
    __shared__ int is_last;

    WorkspaceHeader *hdr = reinterpret_cast<WorkspaceHeader *>(a.workspace);
    Best *part = reinterpret_cast<Best *>(reinterpret_cast<char *>(a.workspace) + kHeaderBytes);

    const int tid = threadIdx.x;
    const int node = blockIdx.y;
    const int v0 = blockIdx.x * kChunk;
    const int v1 = min(v0 + kChunk, a.vocab);

    for (int w = tid; w < kBitWords; w += kThreads)
        bits[w] = 0u;
    __syncthreads();
    for (int w = tid; w < a.window_len; w += kThreads) {
        const int id = a.window[w];
        if (id < 0 || id >= a.vocab) {
            if (blockIdx.x == 0 && node == 0)
                record_status(hdr, TS_ERR_DEVICE_ARG);
            continue;
        }
        if (id >= v0 && id < v1)
            atomicOr(&bits[(id - v0) >> 5], 1u << ((id - v0) & 31));
    }
    __syncthreads();

    const float *row = a.logits + (int64_t)node * a.vocab;
    const float p = a.penalty;
    Best b{-INFINITY, INT_MAX};
    if ((a.vocab & 3) == 0) {
        // all of this thread's 16-byte loads are issued before any is used
        constexpr int kPer = kChunk / (kThreads * 4);
        float4 x4[kPer];
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
            const int v = v0 + (u * kThreads + tid) * 4;
            x4[u] = v < v1 ? __ldcs(reinterpret_cast<const float4 *>(row + v))
                           : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
        }
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
            const int v = v0 + (u * kThreads + tid) * 4;
            if (v >= v1)
                continue;
            const uint32_t word = bits[(v - v0) >> 5] >> ((v - v0) & 31);
            float x[4] = {x4[u].x, x4[u].y, x4[u].z, x4[u].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                float y = ((word >> e) & 1u) ? penalise(x[e], p) : x[e];
                consider(b, y, v + e);
            }
        }
    } else {
        for (int v = v0 + tid; v < v1; v += kThreads) {
            float x = __ldcs(row + v);
            if ((bits[(v - v0) >> 5] >> ((v - v0) & 31)) & 1u)
                x = penalise(x, p);
            consider(b, x, v);
        }
    }
    b = warp_best(b);
    if ((tid & 31) == 0)
        warp_res[tid >> 5] = b;
    __syncthreads();
    if (tid < 32) {
        Best c = tid < kThreads / 32 ? warp_res[tid] : Best{-INFINITY, INT_MAX};
        c = warp_best(c);
        if (tid == 0) {
            part[node * n_chunks + blockIdx.x] = c;
            __threadfence();
            const unsigned total = gridDim.x * gridDim.y;
            is_last = atomicAdd(&hdr->tickets[0], 1u) == total - 1;
        }
    }
    __syncthreads();
    if (!is_last)
        return;

    // ---- epilogue: the last CTA sees every chunk's result
    __threadfence();
    const int warp = tid >> 5, lane = tid & 31;
    for (int n = warp; n < a.n_tree; n += kThreads / 32) {
        Best c{-INFINITY, INT_MAX};
        for (int ch = lane; ch < n_chunks; ch += 32) {
            Best q;
            q.v = __ldcg(&part[n * n_chunks + ch].v);
            q.i = __ldcg(&part[n * n_chunks + ch].i);
            if (beats(q.v, q.i, c.v, c.i))
                c = q;
        }
        c = warp_best(c);
        if (lane == 0) {
            am[n] = c.i;
            if (a.argmax_out)
                a.argmax_out[n] = c.i;
        }
    }
    __shared__ int tok[TS_MAX_TREE];
    for (int i = tid; i < a.n_tree; i += kThreads)
        tok[i] = a.tree_tokens[i];
    __syncthreads();
    if (tid == 0) {
        // valid[i]: parent valid and token == argmax at the parent
        unsigned long long valid = 1ull;
        int depth[TS_MAX_TREE];
        depth[0] = 0;
        int best = 0;
        for (int i = 1; i < a.n_tree; ++i) {
            const int pa = tree.parent[i];
            depth[i] = depth[pa] + 1;
            const bool ok = ((valid >> pa) & 1ull) && tok[i] == am[pa];
            if (ok) {
                valid |= 1ull << i;
                if (depth[i] > depth[best])
                    best = i;
            }
        }
        const int len = depth[best];
        int32_t *out = a.accept_out;
        out[0] = len;
        out[1] = am[best];
        for (int t = len + 1; t < a.n_tree; ++t)
            out[2 + t] = -1;
        int nd = best;
        for (int t = len; t >= 0; --t) {
            out[2 + t] = nd;
            nd = tree.parent[nd];
        }
        hdr->tickets[0] = 0u;
    }
}

}  // namespace

size_t penalize_workspace_bytes(int n_tree, int vocab)
{
    const size_t n_chunks = (size_t)(vocab + kChunk - 1) / kChunk;
    return kHeaderBytes + align_up(n_chunks * (size_t)n_tree * sizeof(Best), 256);
}

cudaError_t penalize_launch(const PenalizeArgs &a, const TreeParents &parents,
                            cudaStream_t stream)
{
    const int n_chunks = (a.vocab + kChunk - 1) / kChunk;
    dim3 grid(n_chunks, a.n_tree);
    penalize_accept_kernel<<<grid, kThreads, 0, stream>>>(a, parents, n_chunks);
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess)
        count_launches(1);
    return e;
}

}  // namespace ts
