// attn_tc.cu -- split-KV tree-verify attention on the 5th-generation tensor
// cores (tcgen05, TMEM accumulators, TMA-fed shared memory).
//
// Tree-based verification runs every draft-tree node's query against the
// full KV cache, each node seeing the context plus its own root path
// (TokenSwift, aiboss88.com, "TokenSwift's technical principles"; tencent
// article, parallel-verification figure; arxivlens "Technical
// Contribution": a 3-ary tree).  For one KV head the G*T query rows
// (node-major, then the group's heads) form one or two 128-row blocks that
// every KV tile of the split serves, so K/V are streamed from HBM once.
//
// CTA = (split, KV head), 12 warps, one CTA per SM:
//   warp 0      TMA producer: K and V tiles of 64 positions (two 64-column
//               boxes each, 128-byte swizzle) into a ring of stages.  The
//               tensor map's row extent is n_ctx + T, so rows past the tree
//               tail arrive as zeros.
//   warp 1      allocates TMEM; one lane issues every tcgen05.mma:
//                 S_b(t)  = Q_b K(t)^T   (M 128, N 64,  K 128; smem x smem)
//                 O_b    += P_b(t) V(t)  (M 128, N 128, K 64;  tmem x smem)
//               S is double-buffered so QK of tile t+1 overlaps the
//               softmax of tile t.
//   warps 4-11  softmax, one thread per query row (TMEM lane): loads S,
//               scales to base 2, applies the ancestor mask on tiles that
//               reach the tree tail, exponentiates against a per-row
//               reference max and writes P as bf16 back over S for the PV
//               product.  The reference only moves (rescaling O and l in
//               place) when a tile's max exceeds it by more than 2^8, so
//               the common tile needs no O traffic; l sums the bf16-rounded
//               P so the normalisation matches what PV used.
// TMEM columns: O_b at [128 b, 128 b + 128); S_b(buf) at 128 NB + 64 (2b + buf).
// Each split leaves an unnormalised partial (acc, m, l) for the combine
// kernel, or normalises in place when it is the only split.
//
// Every wait on an mbarrier is bounded (about a second): on expiry the
// kernel records TS_ERR_TIMEOUT in the workspace status word, all roles
// leave their loops, and TMEM is freed before the CTA exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

#include <mutex>

#include "attn_common.cuh"
#include "sm100.cuh"

namespace ts {
namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kTileN = 64;                      // KV positions per tile
constexpr int kBlockM = 128;                    // query rows per MMA block
constexpr int kBoxBytes = kTileN * 64 * 2;      // one 64-column box of a tile: 8 KB
constexpr int kStageBytes = 4 * kBoxBytes;      // K lo, K hi, V lo, V hi
constexpr int kQBlockBytes = kBlockM * kD * 2;  // 32 KB
constexpr int kThreads = 384;
constexpr int kFirstSoftmaxWarp = 4;

template <int NB>
struct TcCfg {
    static constexpr int kStages = NB == 2 ? 4 : 5;
    static constexpr int kTmemCols = NB == 2 ? 512 : 256;
    static constexpr int kSCol0 = 128 * NB;
    static constexpr size_t kSmemBytes =
        1024 + (size_t)NB * kQBlockBytes + (size_t)kStages * kStageBytes + 256;
};

struct TcBarriers {
    uint64_t full[5];
    uint64_t empty[5];
    uint64_t s_full[2][2];
    uint64_t p_full[2][2];
    uint64_t o_done[2];
    uint64_t o_final[2];
    uint64_t drain;
    uint32_t tmem_base;
    uint32_t abort;
};
static_assert(sizeof(TcBarriers) <= 256, "barrier block");

constexpr uint32_t kIdescQK = idesc_bf16(kBlockM, kTileN, 0, 0);
constexpr uint32_t kIdescPV = idesc_bf16(kBlockM, kD, 0, 1);

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi, float &sum)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    const float2 back = __bfloat1622float2(h);
    sum += back.x + back.y;
    return *reinterpret_cast<uint32_t *>(&h);
}

template <int NB>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
               AttnArgs a, TreeMasks masks, int tiles_per_split, int n_split)
{
    using Cfg = TcCfg<NB>;
    constexpr int S = Cfg::kStages;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *base = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char *sQ = base;
    unsigned char *sKV = base + NB * kQBlockBytes;
    TcBarriers *bar = reinterpret_cast<TcBarriers *>(sKV + S * kStageBytes);
    WorkspaceHeader *hdr = reinterpret_cast<WorkspaceHeader *>(a.workspace);
    volatile uint32_t *abort = &bar->abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int split = blockIdx.x, g = blockIdx.y;
    const int G = a.n_heads_q / a.n_heads_kv;
    const int R = G * a.n_tree;
    const int total = a.n_ctx + a.n_tree;
    const int n_tiles_all = (total + kTileN - 1) / kTileN;
    const int t_begin = split * tiles_per_split;
    const int n_tiles = min(t_begin + tiles_per_split, n_tiles_all) - t_begin;

    // softmax warps with at least one real row, per block
    int active_warps[2];
#pragma unroll
    for (int b = 0; b < 2; ++b) {
        const int rows = min(max(R - b * kBlockM, 0), kBlockM);
        active_warps[b] = (rows + 31) / 32;
    }

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(smem_addr(&bar->full[s]), 1);
            mbar_init(smem_addr(&bar->empty[s]), 1);
        }
        for (int b = 0; b < NB; ++b) {
            for (int u = 0; u < 2; ++u) {
                mbar_init(smem_addr(&bar->s_full[b][u]), 1);
                mbar_init(smem_addr(&bar->p_full[b][u]), active_warps[b]);
            }
            mbar_init(smem_addr(&bar->o_done[b]), 1);
            mbar_init(smem_addr(&bar->o_final[b]), 1);
        }
        mbar_init(smem_addr(&bar->drain), 1);
        bar->abort = 0u;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_addr(&bar->tmem_base), Cfg::kTmemCols);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmap_k);
        prefetch_tmap(&tmap_v);
    }

    // Q rows of this KV head into 128-byte-swizzled K-major blocks:
    // row r (node r / G, head g*G + r % G), 16-byte chunk c of the row.
    for (int idx = threadIdx.x; idx < NB * kBlockM * (kD / 8); idx += kThreads) {
        const int r = idx / (kD / 8), c = idx % (kD / 8);
        uint4 val = make_uint4(0u, 0u, 0u, 0u);
        if (r < R) {
            const int node = r / G, h = g * G + r % G;
            val = *reinterpret_cast<const uint4 *>(a.q + ((int64_t)node * a.n_heads_q + h) * kD +
                                                   c * 8);
        }
        const int blk = r / kBlockM, rr = r % kBlockM, half = c / 8, cc = c % 8;
        unsigned char *dst = sQ + blk * kQBlockBytes + half * (kBlockM * 128) + rr * 128 +
                             ((cc ^ (rr & 7)) << 4);
        *reinterpret_cast<uint4 *>(dst) = val;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bar->tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            int issued = 0;
            for (int t = 0; t < n_tiles; ++t) {
                const int s = t % S;
                if (t >= S &&
                    !wait_bounded(smem_addr(&bar->empty[s]), ((t / S) & 1) ^ 1, abort, hdr))
                    break;
                const uint32_t fb = smem_addr(&bar->full[s]);
                mbar_arrive_expect_tx(fb, kStageBytes);
                const uint32_t dst = smem_addr(sKV + s * kStageBytes);
                const int pos0 = (t_begin + t) * kTileN;
                tma_load_3d(dst, &tmap_k, 0, pos0, g, fb);
                tma_load_3d(dst + kBoxBytes, &tmap_k, 64, pos0, g, fb);
                tma_load_3d(dst + 2 * kBoxBytes, &tmap_v, 0, pos0, g, fb);
                tma_load_3d(dst + 3 * kBoxBytes, &tmap_v, 64, pos0, g, fb);
                issued = t + 1;
            }
            if (*abort) {
                // let our own copies land before the CTA exits
                for (int t = max(0, issued - S); t < issued; ++t)
                    wait_drain(smem_addr(&bar->full[t % S]), (t / S) & 1);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t q_base = smem_addr(sQ);
            bool ok = true;
            for (int t = 0; t <= n_tiles && ok; ++t) {
                if (t < n_tiles) {
                    const int s = t % S;
                    if (!wait_bounded(smem_addr(&bar->full[s]), (t / S) & 1, abort, hdr)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t k_base = smem_addr(sKV + s * kStageBytes);
#pragma unroll
                    for (int b = 0; b < NB; ++b) {
                        const uint32_t d_col = tmem + Cfg::kSCol0 + 64 * (2 * b + (t & 1));
#pragma unroll
                        for (int kk = 0; kk < kD / 16; ++kk) {
                            const uint32_t koff = (kk >> 2) * kBoxBytes + (kk & 3) * 32;
                            const uint32_t qoff = b * kQBlockBytes + (kk >> 2) * (kBlockM * 128) +
                                                  (kk & 3) * 32;
                            mma_ss(d_col, sdesc_sw128(q_base + qoff, 16, 1024),
                                   sdesc_sw128(k_base + koff, 16, 1024), kIdescQK, kk > 0);
                        }
                        mma_commit(smem_addr(&bar->s_full[b][t & 1]));
                    }
                }
                if (t >= 1) {
                    const int u = t - 1, s = u % S;
                    const uint32_t v_base = smem_addr(sKV + s * kStageBytes + 2 * kBoxBytes);
#pragma unroll
                    for (int b = 0; b < NB; ++b) {
                        if (!wait_bounded(smem_addr(&bar->p_full[b][u & 1]), (u >> 1) & 1, abort,
                                          hdr)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t o_col = tmem + 128 * b;
                        const uint32_t p_col = tmem + Cfg::kSCol0 + 64 * (2 * b + (u & 1));
#pragma unroll
                        for (int kk = 0; kk < kTileN / 16; ++kk)
                            mma_ts(o_col, p_col + kk * 8,
                                   sdesc_sw128(v_base + kk * 2048, kBoxBytes, 1024), kIdescPV,
                                   (u > 0 || kk > 0) ? 1u : 0u);
                        mma_commit(smem_addr(&bar->o_done[b]));
                        if (u == n_tiles - 1)
                            mma_commit(smem_addr(&bar->o_final[b]));
                    }
                    if (ok)
                        mma_commit(smem_addr(&bar->empty[s]));
                }
            }
            // every MMA issued above has finished before TMEM is released
            mma_commit(smem_addr(&bar->drain));
            wait_drain(smem_addr(&bar->drain), 0);
        }
    } else if (warp >= kFirstSoftmaxWarp) {
        // ---------------------------------------------------------- softmax
        const int b = (warp - kFirstSoftmaxWarp) / 4;
        const int quarter = warp & 3;
        if (b < NB && quarter < active_warps[b]) {
            const int lane_row = quarter * 32 + lane;
            const int r = b * kBlockM + lane_row;
            const bool valid = r < R;
            const int rr = valid ? r : 0;
            const int node = rr / G, h = g * G + rr % G;
            const unsigned long long anc = masks.anc[node];
            const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
            const uint32_t o_addr = tmem + lane_off + 128 * b;
            float m_ref = -INFINITY, l = 0.f;
            bool ok = true;
            for (int t = 0; t < n_tiles; ++t) {
                const int buf = t & 1;
                if (!warp_wait_bounded(smem_addr(&bar->s_full[b][buf]), (t >> 1) & 1, abort,
                                       hdr)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t s_addr = tmem + lane_off + Cfg::kSCol0 + 64 * (2 * b + buf);
                uint32_t raw[2][32];
                tmem_ld32(s_addr, raw[0]);
                tmem_ld32(s_addr + 32, raw[1]);
                float x[64];
                float mx = -INFINITY;
                const int pos0 = (t_begin + t) * kTileN;
                if (pos0 + kTileN <= a.n_ctx) {
#pragma unroll
                    for (int j = 0; j < 64; ++j) {
                        x[j] = __uint_as_float(raw[j >> 5][j & 31]) * a.scale_log2;
                        mx = fmaxf(mx, x[j]);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 64; ++j) {
                        const int pos = pos0 + j;
                        float v = __uint_as_float(raw[j >> 5][j & 31]) * a.scale_log2;
                        if (pos >= total)
                            v = -INFINITY;
                        else if (pos >= a.n_ctx && !((anc >> (pos - a.n_ctx)) & 1ull))
                            v = -INFINITY;
                        x[j] = v;
                        mx = fmaxf(mx, v);
                    }
                }
                // move the reference max only when this tile exceeds it by > 2^8
                const bool need = mx > m_ref + 8.0f;
                if (__any_sync(0xffffffffu, need)) {
                    const float m_new = need ? mx : m_ref;
                    const float f = (m_ref == -INFINITY) ? 0.f : exp2f(m_ref - m_new);
                    l *= f;
                    if (t > 0) {
                        // S(t) is committed after PV(t-2) was issued, so
                        // o_done has completed t-1 or t phases here: parity
                        // (t-1) tells them apart
                        if (!warp_wait_bounded(smem_addr(&bar->o_done[b]), (t - 1) & 1, abort,
                                               hdr)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            uint32_t o[32];
                            tmem_ld32(o_addr + 32 * c, o);
#pragma unroll
                            for (int j = 0; j < 32; ++j)
                                o[j] = __float_as_uint(__uint_as_float(o[j]) * f);
                            tmem_st32(o_addr + 32 * c, o);
                        }
                        tmem_st_wait();
                    }
                    m_ref = m_new;
                }
                const float m_use = m_ref == -INFINITY ? 0.f : m_ref;
                uint32_t pk[32];
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    pk[j] = pack_bf16x2(exp2f(x[2 * j] - m_use), exp2f(x[2 * j + 1] - m_use), l);
                tmem_st32(s_addr, pk);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(smem_addr(&bar->p_full[b][buf]));
            }
            // o_done alone cannot say whether the last PV has landed: when the
            // softmax finishes its last tile, PV(n-2) may still be queued
            // (QK of a tile is issued before PV of the previous one), and a
            // parity wait cannot tell n-2 completions from n.  o_final is
            // committed once, after the last PV of this block.
            if (ok && n_tiles > 0 &&
                warp_wait_bounded(smem_addr(&bar->o_final[b]), 0, abort, hdr)) {
                tc_fence_after();
                const int rows_all = a.n_tree * a.n_heads_q;
                const int orow = node * a.n_heads_q + h;
                float *ws_o = reinterpret_cast<float *>(reinterpret_cast<char *>(a.workspace) +
                                                        kHeaderBytes);
                float *ws_ml = ws_o + (size_t)n_split * rows_all * kD;
                const float inv = (n_split == 1 && l > 0.f) ? 1.f / l : 1.f;
                float *dst = n_split == 1 ? a.out + (size_t)orow * kD
                                          : ws_o + ((size_t)split * rows_all + orow) * kD;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t o[32];
                    tmem_ld32(o_addr + 32 * c, o);
                    if (valid) {
#pragma unroll
                        for (int j = 0; j < 32; j += 4)
                            *reinterpret_cast<float4 *>(dst + 32 * c + j) = make_float4(
                                __uint_as_float(o[j]) * inv, __uint_as_float(o[j + 1]) * inv,
                                __uint_as_float(o[j + 2]) * inv, __uint_as_float(o[j + 3]) * inv);
                    }
                }
                if (valid && n_split > 1)
                    *reinterpret_cast<float2 *>(ws_ml + ((size_t)split * rows_all + orow) * 2) =
                        make_float2(m_ref, l);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, Cfg::kTmemCols);
    }
}

// ------------------------------------------------------------------- host
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

// [Hkv, kv_cap, D] bf16 viewed as 3-D (d, position, head); positions past
// `rows` read as zeros.
bool encode_kv_map(CUtensorMap *m, const void *ptr, int rows, int64_t kv_cap, int n_heads_kv)
{
    auto enc = tensor_map_encoder();
    if (!enc)
        return false;
    const cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)rows, (cuuint64_t)n_heads_kv};
    const cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)kv_cap * kD * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)kTileN, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NB>
cudaError_t launch_nb(const AttnArgs &a, const TreeMasks &masks, const AttnPlan &p,
                      cudaStream_t stream)
{
    CUtensorMap mk, mv;
    const int rows = a.n_ctx + a.n_tree;
    if (!encode_kv_map(&mk, a.k, rows, a.kv_cap, a.n_heads_kv) ||
        !encode_kv_map(&mv, a.v, rows, a.kv_cap, a.n_heads_kv))
        return cudaErrorInvalidValue;
    const size_t smem = TcCfg<NB>::kSmemBytes;
    static const cudaError_t attr = cudaFuncSetAttribute(
        attn_tc_kernel<NB>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (attr != cudaSuccess)
        return attr;
    attn_tc_kernel<NB><<<dim3(p.n_split, a.n_heads_kv), kThreads, smem, stream>>>(
        mk, mv, a, masks, p.tiles_per_split, p.n_split);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return e;
    count_launches(1);
    if (p.n_split == 1)
        return cudaSuccess;
    return attn_combine_launch(a, p.n_split, stream);
}

}  // namespace

bool attn_tc_eligible(int n_heads_q, int n_heads_kv, int head_dim, int n_ctx, int n_tree)
{
    const int rows = (n_heads_q / n_heads_kv) * n_tree;
    return head_dim == kD && rows <= 2 * kBlockM && n_ctx >= kTcMinContext;
}

AttnPlan attn_tc_plan(int n_heads_q, int n_heads_kv, int n_ctx, int n_tree, int num_sms)
{
    AttnPlan p;
    const int n_tiles = (n_ctx + n_tree + kTileN - 1) / kTileN;
    int want = num_sms / n_heads_kv;
    want = want < 1 ? 1 : (want > n_tiles ? n_tiles : want);
    p.tiles_per_split = (n_tiles + want - 1) / want;
    p.n_split = (n_tiles + p.tiles_per_split - 1) / p.tiles_per_split;
    (void)n_heads_q;
    return p;
}

cudaError_t attn_tc_launch(const AttnArgs &a, const TreeMasks &masks, int num_sms,
                           cudaStream_t stream)
{
    const AttnPlan p = attn_tc_plan(a.n_heads_q, a.n_heads_kv, a.n_ctx, a.n_tree, num_sms);
    const int rows = (a.n_heads_q / a.n_heads_kv) * a.n_tree;
    return rows > kBlockM ? launch_nb<2>(a, masks, p, stream) : launch_nb<1>(a, masks, p, stream);
}

}  // namespace ts
