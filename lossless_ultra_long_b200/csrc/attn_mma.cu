// attn_mma.cu -- split-KV tree-verify attention on warp-level mma.sync.
//
// Tree-based verification runs every draft-tree node's query against the
// full KV cache, each node seeing the context plus its own root path
// (TokenSwift, aiboss88.com, "TokenSwift's technical principles"; tencent
// article, parallel-verification figure).  This file is the general kernel:
// any head_dim in {64, 128}, any group size and tree size.
//
// Work split (flash-decoding): grid (splits, Hkv, row blocks).  A CTA owns
// one KV head, a contiguous range of 64-token KV tiles and up to 16 warps of
// 16 query rows each; rows of a KV head are (node, head-in-group) pairs, so
// all G*T rows that share the head stream its K/V exactly once per split.
// K/V tiles are staged in shared memory by cp.async (16-byte, XOR-swizzled
// rows) in a three-stage ring; QK^T and PV run on mma.m16n8k16 bf16 with
// fp32 accumulators (P enters PV as two bf16 parts, so PV keeps ~16
// significant bits of P); the softmax is the online (running max / sum) form in
// base 2.  Only tiles that reach the tree tail evaluate the ancestor mask.
// Each split writes an unnormalised partial (acc, m, l) that a combine
// kernel merges across splits with a log-sum-exp rescale; a single-split
// launch normalises in place instead.
#include <math.h>

#include "attn_common.cuh"

namespace ts {
namespace {

constexpr int kTile = 64;        // KV positions per pipeline stage
constexpr int kStages = 3;
constexpr int kMaxWarps = 12;    // 192 query rows per CTA

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid)
{
    const int n = valid ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(n));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                        uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                          uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// (lo, hi) floats -> bf16x2 of their rounding, and bf16x2 of the remainders
__device__ __forceinline__ void split_bf16(float lo, float hi, uint32_t &big, uint32_t &small)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    const float2 back = __bfloat1622float2(h);
    __nv_bfloat162 r = __floats2bfloat162_rn(lo - back.x, hi - back.y);
    big = *reinterpret_cast<uint32_t *>(&h);
    small = *reinterpret_cast<uint32_t *>(&r);
}

// byte offset of 16-byte chunk `c` of tile row `r` (rows of D bf16)
template <int D>
__device__ __forceinline__ uint32_t swz(int r, int c)
{
    return static_cast<uint32_t>(r * (D * 2) + ((c ^ (r & 7)) << 4));
}

template <int D>
struct Plan {
    static constexpr int kChunks = D / 8;                       // 16-byte chunks per row
    static constexpr int kStageBytes = kTile * D * 2;           // one of K or V
    static constexpr int kSmem = kStages * 2 * kStageBytes;
};

template <int D>
__global__ void __launch_bounds__(kMaxWarps * 32, 1)
attn_split_kernel(AttnArgs a, TreeMasks masks, int tiles_per_split, int n_split)
{
    extern __shared__ __align__(128) unsigned char smem[];
    constexpr int CH = Plan<D>::kChunks;
    constexpr int SB = Plan<D>::kStageBytes;

    const int split = blockIdx.x;
    const int g = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nthreads = blockDim.x;
    const int G = a.n_heads_q / a.n_heads_kv;
    const int R = G * a.n_tree;
    const int total = a.n_ctx + a.n_tree;
    const int n_tiles_all = (total + kTile - 1) / kTile;
    const int t_begin = split * tiles_per_split;
    const int t_end = min(t_begin + tiles_per_split, n_tiles_all);
    const int n_tiles = t_end - t_begin;

    const __nv_bfloat16 *kh = a.k + (int64_t)g * a.kv_cap * D;
    const __nv_bfloat16 *vh = a.v + (int64_t)g * a.kv_cap * D;
    const uint32_t sbase = smem_u32(smem);

    auto load_tile = [&](int t_local, int stage) {
        const int pos0 = (t_begin + t_local) * kTile;
        const uint32_t ks = sbase + stage * 2 * SB, vs = ks + SB;
        for (int c = threadIdx.x; c < kTile * CH; c += nthreads) {
            const int r = c / CH, ch = c % CH;
            const int pos = pos0 + r;
            const bool ok = pos < total;
            const int64_t off = (int64_t)(ok ? pos : 0) * D + ch * 8;
            cp_async16(ks + swz<D>(r, ch), kh + off, ok);
            cp_async16(vs + swz<D>(r, ch), vh + off, ok);
        }
    };

#pragma unroll
    for (int s = 0; s < kStages - 1; ++s) {
        if (s < n_tiles)
            load_tile(s, s);
        cp_async_commit();
    }

    // ---- this warp's 16 rows: Q fragments stay in registers
    const int row_base = blockIdx.z * blockDim.x / 2 + warp * 16;  // 16 rows per warp
    const int qr = lane >> 2, qc = (lane & 3) * 2;
    int rnode[2], rhead[2];
    bool rvalid[2];
#pragma unroll
    for (int hi = 0; hi < 2; ++hi) {
        const int r = row_base + qr + hi * 8;
        rvalid[hi] = r < R;
        const int rr = rvalid[hi] ? r : 0;
        rnode[hi] = rr / G;
        rhead[hi] = g * G + rr % G;
    }
    uint32_t qa[D / 16][4];
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
        for (int hi = 0; hi < 2; ++hi) {
            const __nv_bfloat16 *qrow =
                a.q + ((int64_t)rnode[hi] * a.n_heads_q + rhead[hi]) * D + kk * 16 + qc;
            uint32_t lo = rvalid[hi] ? *reinterpret_cast<const uint32_t *>(qrow) : 0u;
            uint32_t up = rvalid[hi] ? *reinterpret_cast<const uint32_t *>(qrow + 8) : 0u;
            qa[kk][hi] = lo;
            qa[kk][2 + hi] = up;
        }
    }
    const unsigned long long anc0 = masks.anc[rnode[0]], anc1 = masks.anc[rnode[1]];

    float o[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i)
        o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};

    for (int t = 0; t < n_tiles; ++t) {
        cp_async_wait<kStages - 2>();
        __syncthreads();
        if (t + kStages - 1 < n_tiles)
            load_tile(t + kStages - 1, (t + kStages - 1) % kStages);
        cp_async_commit();

        const int stage = t % kStages;
        const uint32_t ks = sbase + stage * 2 * SB, vs = ks + SB;
        const int mrow = lane & 7, mat = lane >> 3;

        float s[kTile / 8][4];
#pragma unroll
        for (int i = 0; i < kTile / 8; ++i)
            s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
            for (int np = 0; np < kTile / 16; ++np) {
                uint32_t b0, b1, b2, b3;
                const int tok = np * 16 + (mat >> 1) * 8 + mrow;
                ldsm_x4(ks + swz<D>(tok, kk * 2 + (mat & 1)), b0, b1, b2, b3);
                mma_bf16(s[2 * np], qa[kk], b0, b1);
                mma_bf16(s[2 * np + 1], qa[kk], b2, b3);
            }
        }

        // scale to base 2, mask, online softmax
        const int pos0 = (t_begin + t) * kTile;
        const bool edge = pos0 + kTile > a.n_ctx;
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int nt = 0; nt < kTile / 8; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                float x = s[nt][e] * a.scale_log2;
                if (edge) {
                    const int pos = pos0 + nt * 8 + qc + (e & 1);
                    if (pos >= total) {
                        x = -INFINITY;
                    } else if (pos >= a.n_ctx) {
                        const unsigned long long anc = (e >> 1) ? anc1 : anc0;
                        if (!((anc >> (pos - a.n_ctx)) & 1ull))
                            x = -INFINITY;
                    }
                }
                s[nt][e] = x;
                mx[e >> 1] = fmaxf(mx[e >> 1], x);
            }
        }
        float corr[2], mref[2];
#pragma unroll
        for (int hi = 0; hi < 2; ++hi) {
            mx[hi] = fmaxf(mx[hi], __shfl_xor_sync(0xffffffffu, mx[hi], 1));
            mx[hi] = fmaxf(mx[hi], __shfl_xor_sync(0xffffffffu, mx[hi], 2));
            const float m_new = fmaxf(m_run[hi], mx[hi]);
            mref[hi] = m_new == -INFINITY ? 0.f : m_new;
            corr[hi] = exp2f(m_run[hi] - mref[hi]);
            m_run[hi] = m_new;
            l_run[hi] *= corr[hi];
        }
#pragma unroll
        for (int nt = 0; nt < kTile / 8; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float p = exp2f(s[nt][e] - mref[e >> 1]);
                s[nt][e] = p;
                l_run[e >> 1] += p;
            }
        }
#pragma unroll
        for (int dt = 0; dt < D / 8; ++dt) {
            o[dt][0] *= corr[0];
            o[dt][1] *= corr[0];
            o[dt][2] *= corr[1];
            o[dt][3] *= corr[1];
        }

        // O += P V, with P = P_hi + P_lo (two bf16 parts, ~16 significant
        // bits) so that few, large weights keep fp32-level accuracy
#pragma unroll
        for (int kt = 0; kt < kTile / 16; ++kt) {
            uint32_t pa[4], pl[4];
            split_bf16(s[2 * kt][0], s[2 * kt][1], pa[0], pl[0]);
            split_bf16(s[2 * kt][2], s[2 * kt][3], pa[1], pl[1]);
            split_bf16(s[2 * kt + 1][0], s[2 * kt + 1][1], pa[2], pl[2]);
            split_bf16(s[2 * kt + 1][2], s[2 * kt + 1][3], pa[3], pl[3]);
#pragma unroll
            for (int dp = 0; dp < D / 16; ++dp) {
                uint32_t b0, b1, b2, b3;
                const int tok = kt * 16 + (mat & 1) * 8 + mrow;
                ldsm_x4_t(vs + swz<D>(tok, dp * 2 + (mat >> 1)), b0, b1, b2, b3);
                mma_bf16(o[2 * dp], pa, b0, b1);
                mma_bf16(o[2 * dp + 1], pa, b2, b3);
                mma_bf16(o[2 * dp], pl, b0, b1);
                mma_bf16(o[2 * dp + 1], pl, b2, b3);
            }
        }
    }
    cp_async_wait<0>();

    // ---- epilogue
#pragma unroll
    for (int hi = 0; hi < 2; ++hi) {
        l_run[hi] += __shfl_xor_sync(0xffffffffu, l_run[hi], 1);
        l_run[hi] += __shfl_xor_sync(0xffffffffu, l_run[hi], 2);
    }
    const int rows_all = a.n_tree * a.n_heads_q;
    float *ws_o = reinterpret_cast<float *>(reinterpret_cast<char *>(a.workspace) + kHeaderBytes);
    float *ws_ml = ws_o + (size_t)n_split * rows_all * D;
#pragma unroll
    for (int hi = 0; hi < 2; ++hi) {
        if (!rvalid[hi])
            continue;
        const int orow = rnode[hi] * a.n_heads_q + rhead[hi];
        if (n_split == 1) {
            const float inv = 1.f / l_run[hi];
            float *dst = a.out + (int64_t)orow * D;
#pragma unroll
            for (int dt = 0; dt < D / 8; ++dt)
                *reinterpret_cast<float2 *>(dst + dt * 8 + qc) =
                    make_float2(o[dt][2 * hi] * inv, o[dt][2 * hi + 1] * inv);
        } else {
            float *dst = ws_o + ((size_t)split * rows_all + orow) * D;
#pragma unroll
            for (int dt = 0; dt < D / 8; ++dt)
                *reinterpret_cast<float2 *>(dst + dt * 8 + qc) =
                    make_float2(o[dt][2 * hi], o[dt][2 * hi + 1]);
            if ((lane & 3) == 0)
                *reinterpret_cast<float2 *>(ws_ml + ((size_t)split * rows_all + orow) * 2) =
                    make_float2(m_run[hi], l_run[hi]);
        }
    }
}

// One warp per output row: out = sum_s 2^(m_s - M) acc_s / sum_s 2^(m_s - M) l_s.
template <int D>
__global__ void __launch_bounds__(256)
attn_combine_kernel(const float *__restrict__ ws_o, const float *__restrict__ ws_ml, float *out,
                    int rows_all, int n_split)
{
    const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows_all)
        return;
    float M = -INFINITY;
    for (int s = 0; s < n_split; ++s)
        M = fmaxf(M, __ldcg(ws_ml + ((size_t)s * rows_all + row) * 2));
    constexpr int PER = D / 32;
    float acc[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e)
        acc[e] = 0.f;
    float L = 0.f;
    // splits in batches of kB: the batch's loads are in flight together
    constexpr int kB = 6;
    for (int s0 = 0; s0 < n_split; s0 += kB) {
        float2 ml[kB];
        float x[kB][PER];
#pragma unroll
        for (int u = 0; u < kB; ++u) {
            const int s = s0 + u;
            if (s < n_split) {
                ml[u] = __ldcg(reinterpret_cast<const float2 *>(ws_ml + ((size_t)s * rows_all + row) * 2));
                const float *src = ws_o + ((size_t)s * rows_all + row) * D + lane * PER;
                if constexpr (PER == 4) {
                    const float4 v = __ldcg(reinterpret_cast<const float4 *>(src));
                    x[u][0] = v.x; x[u][1] = v.y; x[u][2] = v.z; x[u][3] = v.w;
                } else {
                    const float2 v = __ldcg(reinterpret_cast<const float2 *>(src));
                    x[u][0] = v.x; x[u][1] = v.y;
                }
            } else {
                ml[u] = make_float2(-INFINITY, 0.f);
#pragma unroll
                for (int e = 0; e < PER; ++e)
                    x[u][e] = 0.f;
            }
        }
#pragma unroll
        for (int u = 0; u < kB; ++u) {
            const float w = ml[u].x == -INFINITY ? 0.f : exp2f(ml[u].x - M);
            L += w * ml[u].y;
#pragma unroll
            for (int e = 0; e < PER; ++e)
                acc[e] += w * x[u][e];
        }
    }
    const float inv = 1.f / L;
    float *dst = out + (size_t)row * D + lane * PER;
    if constexpr (PER == 4)
        *reinterpret_cast<float4 *>(dst) = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv,
                                                       acc[3] * inv);
    else
        *reinterpret_cast<float2 *>(dst) = make_float2(acc[0] * inv, acc[1] * inv);
}

struct SplitPlan {
    int warps, row_blocks, n_split, tiles_per_split;
};

SplitPlan make_plan(int n_heads_q, int n_heads_kv, int n_ctx, int n_tree, int num_sms)
{
    SplitPlan p;
    const int R = (n_heads_q / n_heads_kv) * n_tree;
    const int warps_needed = (R + 15) / 16;
    p.row_blocks = (warps_needed + kMaxWarps - 1) / kMaxWarps;
    p.warps = (warps_needed + p.row_blocks - 1) / p.row_blocks;
    const int ctas_per_sm = p.warps <= 6 ? 2 : 1;
    const int n_tiles = (n_ctx + n_tree + kTile - 1) / kTile;
    int want = (num_sms * ctas_per_sm) / (n_heads_kv * p.row_blocks);
    want = want < 1 ? 1 : (want > n_tiles ? n_tiles : want);
    p.tiles_per_split = (n_tiles + want - 1) / want;
    p.n_split = (n_tiles + p.tiles_per_split - 1) / p.tiles_per_split;
    return p;
}

template <int D>
cudaError_t launch_d(const AttnArgs &a, const TreeMasks &masks, const SplitPlan &p,
                     cudaStream_t stream)
{
    const int smem = Plan<D>::kSmem;
    static const cudaError_t attr = cudaFuncSetAttribute(
        attn_split_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (attr != cudaSuccess)
        return attr;
    dim3 grid(p.n_split, a.n_heads_kv, p.row_blocks);
    attn_split_kernel<D><<<grid, p.warps * 32, smem, stream>>>(a, masks, p.tiles_per_split,
                                                               p.n_split);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return e;
    count_launches(1);
    if (p.n_split == 1)
        return e;
    return attn_combine_launch(a, p.n_split, stream);
}

}  // namespace

cudaError_t attn_combine_launch(const AttnArgs &a, int n_split, cudaStream_t stream)
{
    const int rows_all = a.n_tree * a.n_heads_q;
    const float *ws_o = reinterpret_cast<const float *>(
        reinterpret_cast<const char *>(a.workspace) + kHeaderBytes);
    const float *ws_ml = ws_o + (size_t)n_split * rows_all * a.head_dim;
    if (a.head_dim == 128)
        attn_combine_kernel<128><<<(rows_all + 7) / 8, 256, 0, stream>>>(ws_o, ws_ml, a.out,
                                                                         rows_all, n_split);
    else
        attn_combine_kernel<64><<<(rows_all + 7) / 8, 256, 0, stream>>>(ws_o, ws_ml, a.out,
                                                                        rows_all, n_split);
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess)
        count_launches(1);
    return e;
}

size_t attn_mma_workspace_bytes(int n_heads_q, int n_heads_kv, int head_dim, int n_ctx,
                                int n_tree, int num_sms)
{
    const SplitPlan p = make_plan(n_heads_q, n_heads_kv, n_ctx, n_tree, num_sms);
    return kHeaderBytes + align_up(attn_partial_bytes(p.n_split, n_heads_q, head_dim, n_tree), 256);
}

cudaError_t attn_mma_launch(const AttnArgs &a, const TreeMasks &masks, int num_sms,
                            cudaStream_t stream)
{
    const SplitPlan p = make_plan(a.n_heads_q, a.n_heads_kv, a.n_ctx, a.n_tree, num_sms);
    return a.head_dim == 128 ? launch_d<128>(a, masks, p, stream)
                             : launch_d<64>(a, masks, p, stream);
}

}  // namespace ts
