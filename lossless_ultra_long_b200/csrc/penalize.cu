// penalize.cu -- contextual penalty, per-node argmax and longest accepted
// path in one launch.
//
// TokenSwift (aiboss88.com), "TokenSwift's technical principles": a penalty
// on recently generated tokens; the longest valid candidate of the tree is
// kept.  Tencent article: 上下文惩罚 and the parallel-verification figure
// (the worked example keeps "is the father of", the longest valid candidate).
//
// Grid (vocab splits, tree nodes), sized to one wave of resident CTAs.  Each
// CTA starts one bulk asynchronous copy of its slice of the logits row into
// shared memory, marks the window ids that fall in the slice in a
// shared-memory bitmap while it is in flight, then penalises marked ids
// (binary32 divide / multiply, round-to-nearest) and reduces (value, id)
// with warp shuffles, ties to the lower id.  Its result goes to the workspace; the CTA that
// takes the last ticket reduces every node's splits, writes the argmax, and
// walks the tree.  The logits are read exactly once: T * V * 4 bytes.
// Options (flags): the tokens of a node's own draft path join its window
// (aiboss88, "Contextual penalty strategy": the recently generated tokens),
// and the kept node is drawn among the deepest valid ones with a
// caller-given random integer (aiboss88, tree-based verification: the
// longest valid candidate is selected at random).  With caller-drawn
// Gumbel noise (the kSample instance) each node's target token is the
// draw from softmax(penalised / temperature) by the Gumbel-max rule -- the
// largest penalised / temperature + g, in binary32 -- instead of the
// argmax; the noise slice is bulk-copied beside the logits slice, so that
// instance reads 2 * T * V * 4 bytes.
#include <float.h>
#include <limits.h>

#include "sm100.cuh"
#include "ts_internal.cuh"

namespace ts {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxChunk = 16384;               // vocab entries per CTA, at most (64 KB)
constexpr int kBitWords = kMaxChunk / 32;
constexpr int kMaxSplits = 1024;

// Vocab entries per CTA (a multiple of 4): enough splits per node for one
// wave of resident CTAs (ctas_per_sm on each SM), no more than max_chunk
// entries each.
int penalize_chunk(int n_tree, int vocab, int num_sms, int ctas_per_sm, int max_chunk)
{
    int splits = (ctas_per_sm * num_sms) / (n_tree > 0 ? n_tree : 1);
    const int need = (vocab + max_chunk - 1) / max_chunk;
    splits = splits < need ? need : splits;
    splits = splits > kMaxSplits ? kMaxSplits : (splits < 1 ? 1 : splits);
    int chunk = (vocab + splits - 1) / splits;
    chunk = (chunk + 3) / 4 * 4;
    return chunk < 4 ? 4 : chunk;
}

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

// 64-bit key ordered like beats(): order-preserving bits of the value
// (NaN already mapped to -inf by consider, zero's sign dropped), then the
// complemented id
__device__ __forceinline__ unsigned long long best_key(Best b)
{
    // -0 and +0 compare equal, so they must share one key (ties by id)
    const uint32_t u = b.v == 0.f ? 0u : __float_as_uint(b.v);
    const uint32_t ord = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return ((unsigned long long)ord << 32) | (uint32_t)~(uint32_t)b.i;
}

__device__ __forceinline__ float penalise(float x, float p)
{
    return x > 0.0f ? __fdiv_rn(x, p) : __fmul_rn(x, p);
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes,
                                          uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n"
        ::"r"(dst), "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// The score a node's id competes with: the penalised logit, or with the
// temperature draw that divided by the temperature plus the id's noise
// (one binary32 rounding per operation, never fused).
template <bool kSample>
__device__ __forceinline__ float draw_score(float y, float t, float g)
{
    if constexpr (kSample)
        return __fadd_rn(__fdiv_rn(y, t), g);
    else
        return y;
}

template <bool kSample>
__global__ void __launch_bounds__(kThreads)
penalize_accept_kernel(PenalizeArgs a, TreeParents tree, int chunk, int n_chunks)
{
    // this CTA's slice of the logits row, then (kSample) the same slice of
    // the noise row at xs + chunk
    extern __shared__ __align__(16) float xs[];
    __shared__ uint32_t bits[kBitWords];
    __shared__ Best warp_res[kThreads / 32];
    __shared__ int am[TS_MAX_TREE];
    __shared__ int is_last;
    __shared__ uint64_t landed;
    __shared__ uint32_t abort_flag;

    WorkspaceHeader *hdr = reinterpret_cast<WorkspaceHeader *>(a.workspace);
    Best *part = reinterpret_cast<Best *>(reinterpret_cast<char *>(a.workspace) + kHeaderBytes);

    const int tid = threadIdx.x;
    const int node = blockIdx.y;
    const int v0 = blockIdx.x * chunk;
    const int v1 = min(v0 + chunk, a.vocab);
    const float *row = a.logits + (int64_t)node * a.vocab;
    const float *grow = kSample ? a.gumbel + (int64_t)node * a.vocab : nullptr;
    // rows and slices start on 16-byte boundaries and end on whole vectors
    const bool vec = (a.vocab & 3) == 0 && (reinterpret_cast<uintptr_t>(a.logits) & 15) == 0;

    if (vec && tid == 0) {
        sm100::mbar_init(sm100::smem_addr(&landed), 1);
        abort_flag = 0u;
        sm100::fence_mbar_init();
        const uint32_t bytes = (uint32_t)(v1 - v0) * 4u;
        sm100::mbar_arrive_expect_tx(sm100::smem_addr(&landed), kSample ? 2u * bytes : bytes);
        bulk_load(sm100::smem_addr(xs), row + v0, bytes, sm100::smem_addr(&landed));
        if constexpr (kSample)   // chunk is a multiple of 4: 16-byte aligned
            bulk_load(sm100::smem_addr(xs + chunk), grow + v0, bytes,
                      sm100::smem_addr(&landed));
    }
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
    if ((a.flags & TS_PENALIZE_PATH_TOKENS) && tid == 0) {
        // the tokens of this node's draft path (the root's entry excluded)
        // join its window
        for (int n = node; n > 0; n = tree.parent[n]) {
            const int id = a.tree_tokens[n];
            if (id < 0 || id >= a.vocab) {
                if (blockIdx.x == 0)
                    record_status(hdr, TS_ERR_DEVICE_ARG);
                continue;
            }
            if (id >= v0 && id < v1)
                atomicOr(&bits[(id - v0) >> 5], 1u << ((id - v0) & 31));
        }
    }
    __syncthreads();

    const float p = a.penalty;
    const float temp = a.temperature;
    Best b{-INFINITY, INT_MAX};
    if (vec) {
        if (sm100::wait_bounded(sm100::smem_addr(&landed), 0, &abort_flag, hdr)) {
            // two independent running bests (even and odd lanes of each
            // vector) halve the compare chain
            const float4 *x4 = reinterpret_cast<const float4 *>(xs);
            const float4 *g4 = reinterpret_cast<const float4 *>(xs + chunk);
            Best b2{-INFINITY, INT_MAX};
            for (int u = tid; u < (v1 - v0) / 4; u += kThreads) {
                const float4 q = x4[u];
                float4 gq = make_float4(0.f, 0.f, 0.f, 0.f);
                if constexpr (kSample)
                    gq = g4[u];
                const uint32_t word = bits[u >> 3] >> ((u & 7) * 4);
                const float x[4] = {q.x, q.y, q.z, q.w};
                const float g[4] = {gq.x, gq.y, gq.z, gq.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float y = ((word >> e) & 1u) ? penalise(x[e], p) : x[e];
                    consider(e & 1 ? b2 : b, draw_score<kSample>(y, temp, g[e]),
                             v0 + 4 * u + e);
                }
            }
            if (beats(b2.v, b2.i, b.v, b.i))
                b = b2;
        }
    } else {
        for (int v = v0 + tid; v < v1; v += kThreads) {
            float x = __ldcs(row + v);
            if ((bits[(v - v0) >> 5] >> ((v - v0) & 31)) & 1u)
                x = penalise(x, p);
            consider(b, draw_score<kSample>(x, temp, kSample ? __ldcs(grow + v) : 0.f), v);
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
    // every (node, split) result is loaded in one round and folded into its
    // node with a 64-bit max whose order is that of beats(): the float's
    // order-preserving bits above the complemented id (larger value, then
    // lower id)
    __shared__ unsigned long long node_key[TS_MAX_TREE];
    for (int n = tid; n < a.n_tree; n += kThreads)
        node_key[n] = 0ull;
    __syncthreads();
    {
        const int total = a.n_tree * n_chunks;
        constexpr int kL = 8;   // results per thread in flight
        for (int base = 0; base < total; base += kThreads * kL) {
            Best q[kL];
#pragma unroll
            for (int u = 0; u < kL; ++u) {
                const int k = base + u * kThreads + tid;
                if (k < total) {
                    q[u].v = __ldcg(&part[k].v);
                    q[u].i = __ldcg(&part[k].i);
                }
            }
#pragma unroll
            for (int u = 0; u < kL; ++u) {
                const int k = base + u * kThreads + tid;
                if (k < total)
                    atomicMax(&node_key[k / n_chunks], best_key(q[u]));
            }
        }
    }
    __syncthreads();
    for (int n = tid; n < a.n_tree; n += kThreads) {
        const int id = (int)~(uint32_t)node_key[n];
        am[n] = id;
        if (a.argmax_out)
            a.argmax_out[n] = id;
    }
    __shared__ int tok[TS_MAX_TREE], par[TS_MAX_TREE];
    for (int i = tid; i < a.n_tree; i += kThreads) {
        tok[i] = a.tree_tokens[i];
        par[i] = tree.parent[i];
    }
    __syncthreads();
    // Each node checks its own root path: valid when every node on it
    // carries the argmax at its parent.  The kept node is the deepest valid
    // one, ties to the lowest index: the largest (depth << 8 | 255 - i).
    // With the random choice, the deepest valid nodes are also listed (one
    // bit per node) and the (r mod c)-th of them in index order is kept.
    __shared__ int best_key[2];
    __shared__ unsigned deepest[2];
    int my_depth = -1;
    if (tid < 2 * 32) {
        int key = -1;
        if (tid < a.n_tree) {
            int i = tid, d = 0;
            bool ok = true;
            while (i != 0) {
                const int pa = par[i];
                ok = ok && tok[i] == am[pa];
                i = pa;
                ++d;
            }
            if (ok) {
                key = (d << 8) | (255 - tid);
                my_depth = d;
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            key = max(key, __shfl_xor_sync(0xffffffffu, key, off));
        if ((tid & 31) == 0)
            best_key[tid >> 5] = key;
    }
    __syncthreads();
    if (tid < 2 * 32) {
        const int len = max(best_key[0], best_key[1]) >> 8;
        const unsigned m = __ballot_sync(0xffffffffu, my_depth == len);
        if ((tid & 31) == 0)
            deepest[tid >> 5] = m;
    }
    __syncthreads();
    if (tid == 0) {
        const int key = max(best_key[0], best_key[1]);
        int best = 255 - (key & 255);
        const int len = key >> 8;
        if (a.flags & TS_ACCEPT_RANDOM_TIE) {
            unsigned long long m = ((unsigned long long)deepest[1] << 32) | deepest[0];
            const int c = __popcll(m);
            for (int k = (int)(a.random % (unsigned long long)c); k > 0; --k)
                m &= m - 1;   // drop the lowest set bit
            best = __ffsll((long long)m) - 1;
        }
        int32_t *out = a.accept_out;
        out[0] = len;
        out[1] = am[best];
        for (int t = len + 1; t < a.n_tree; ++t)
            out[2 + t] = -1;
        int nd = best;
        for (int t = len; t >= 0; --t) {
            out[2 + t] = nd;
            nd = par[nd];
        }
        hdr->tickets[0] = 0u;
    }
}

}  // namespace

int penalize_max_vocab(bool sample)
{
    return (sample ? kMaxChunk / 2 : kMaxChunk) * kMaxSplits;
}

size_t penalize_workspace_bytes(int n_tree, int vocab)
{
    // room for the most splits any device gives (per-split results)
    return kHeaderBytes + align_up((size_t)kMaxSplits * n_tree * sizeof(Best), 256);
}

namespace {

template <bool kSample>
cudaError_t penalize_launch_as(const PenalizeArgs &a, const TreeParents &parents, int num_sms,
                               cudaStream_t stream)
{
    // dynamic shared memory: the logits slice, and the noise slice beside
    // it; with two slices each is half as long, so that a CTA holds the same
    // 64 KB and as many CTAs stay resident per SM
    constexpr int kSlices = kSample ? 2 : 1;
    constexpr int kSliceMax = kMaxChunk / kSlices;
    static int per_sm = 0;
    if (per_sm == 0) {
        int n = 0;
        if (cudaFuncSetAttribute(penalize_accept_kernel<kSample>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kSlices * kSliceMax * (int)sizeof(float)) != cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, penalize_accept_kernel<kSample>,
                                                          kThreads,
                                                          kSlices * kSliceMax * sizeof(float)) !=
                cudaSuccess ||
            n < 1) {
            cudaGetLastError();
            n = 1;
        }
        per_sm = n;
    }
    const int chunk = penalize_chunk(a.n_tree, a.vocab, num_sms, per_sm, kSliceMax);
    const int n_chunks = (a.vocab + chunk - 1) / chunk;
    dim3 grid(n_chunks, a.n_tree);
    penalize_accept_kernel<kSample>
        <<<grid, kThreads, (size_t)kSlices * chunk * sizeof(float), stream>>>(a, parents, chunk,
                                                                             n_chunks);
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess)
        count_launches(1);
    return e;
}

}  // namespace

cudaError_t penalize_launch(const PenalizeArgs &a, const TreeParents &parents, int num_sms,
                            cudaStream_t stream)
{
    return a.gumbel ? penalize_launch_as<true>(a, parents, num_sms, stream)
                    : penalize_launch_as<false>(a, parents, num_sms, stream);
}

}  // namespace ts
