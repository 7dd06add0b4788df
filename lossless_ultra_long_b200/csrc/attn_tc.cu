// attn_tc.cu -- split-KV tree-verify attention on the 5th-generation tensor
// cores (tcgen05, TMEM accumulators, TMA-fed shared memory).
//
// Tree-based verification runs every draft-tree node's query against the
// full KV cache, each node seeing the context plus its own root path
// (TokenSwift, aiboss88.com, "TokenSwift's technical principles"; tencent
// article, parallel-verification figure; arxivlens "Technical
// Contribution": a 3-ary tree).  For one KV head the R = G*T query rows
// (node-major, then the group's heads) share every KV tile, so K/V are
// streamed from HBM once per split.
//
// The two products run in the orientations the tensor core executes at
// full rate (an MMA instruction costs about the same below N = 128, and an
// MN-major B operand runs at about half rate):
//   S_b  = Q_b K^T      rows on M (128-row blocks b), N = 64 positions,
//                       both operands K-major in shared memory;
//   O^T += V^T P^T      head dim on M, all R rows on N (padded to 16),
//                       V^T is the TMA tile read MN-major, P^T K-major.
// P^T is written to shared memory by the softmax threads, one row each.
//
// CTA = (split, KV head), 12 warps, one CTA per SM:
//   warps 0, 2  TMA producers for K and for V: 64-position tiles (two
//               64-column boxes each, 128-byte swizzle) into two rings.  The
//               tensor map's row extent is n_ctx + T, so rows past the tree
//               tail arrive as zeros.
//   warp 1      allocates TMEM; one lane issues every tcgen05.mma.  S is
//               double-buffered so QK of tile t+1 overlaps the softmax of t.
//   warps 4..   softmax, one thread per query row (TMEM lane of its block):
//               scale to base 2, ancestor mask on tiles that reach the tree
//               tail, exponentiate against a per-row reference max, write
//               the bf16 P^T row.  The reference only moves when a tile's
//               max exceeds it by more than 2^8; then warps 4-7 (which
//               between them see all 128 TMEM lanes, i.e. all of D) rescale
//               the affected O^T columns before the next PV.  l sums the
//               bf16-rounded P so the normalisation matches what PV used.
// TMEM: O^T in columns [0, R_pad); S_b(buf) at kSCol0 + 64 (2b + buf).
// Each split leaves an unnormalised partial (acc, m, l) for the combine
// kernel, or normalises in place when it is the only split.
//
// Every wait is on an mbarrier and bounded (about a second): on expiry the
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
constexpr int kBlockM = 128;                    // query rows per QK block
constexpr int kBoxBytes = kTileN * 64 * 2;      // one 64-column box of a tile: 8 KB
constexpr int kHalfStageBytes = 2 * kBoxBytes;  // K (or V) of a tile: lo and hi boxes
constexpr int kQBlockBytes = kBlockM * kD * 2;  // 32 KB
constexpr int kThreads = 384;
constexpr int kFirstSoftmaxWarp = 4;
constexpr int kMaxStages = 8;
constexpr int kMaxRows = 256;
constexpr size_t kSmemLimit = 232448;           // dynamic shared memory per CTA

struct TcBarriers {
    uint64_t full_k[kMaxStages];
    uint64_t empty_k[kMaxStages];
    uint64_t full_v[kMaxStages];
    uint64_t empty_v[kMaxStages];
    uint64_t s_full[2][2];     // QK of a block landed in S(buf)
    uint64_t sm_sync[2];       // every softmax warp finished a tile
    uint64_t p_full[2];        // P^T(buf) written and O^T corrected
    uint64_t o_done;           // one commit per PV
    uint64_t o_final;          // committed once, after the last PV
    uint64_t drain;
    uint32_t tmem_base;
    uint32_t abort;
    int32_t rescale_tile[2];   // tile index + 1 when that tile moved a row's max
};

struct TcAux {
    float factor[2][kMaxRows];  // per-row O^T rescale factor of the tile
    float l[kMaxRows];
    float m[kMaxRows];
    TcBarriers bar;
};
constexpr size_t kAuxBytes = (sizeof(TcAux) + 1023) / 1024 * 1024;

struct TcLayout {
    int r_pad;       // rows rounded up to 16: N of the PV product
    int stages_k, stages_v;
    size_t p_off, k_off, v_off, aux_off, smem_bytes;
};

__host__ __device__ inline TcLayout tc_layout(int nb, int rows)
{
    TcLayout L;
    L.r_pad = (rows + 15) / 16 * 16;
    L.p_off = (size_t)nb * kQBlockBytes;
    L.k_off = L.p_off + 2 * (size_t)L.r_pad * 128;
    const size_t fixed = 1024 + L.k_off + kAuxBytes;
    int halves = (int)((kSmemLimit - fixed) / kHalfStageBytes);
    halves = halves > 2 * kMaxStages ? 2 * kMaxStages : halves;
    // V is consumed one softmax later than K, but both need a tile or two of
    // look-ahead beyond the one in use
    L.stages_v = halves * 3 / 7 < 2 ? 2 : halves * 3 / 7;
    L.stages_k = halves - L.stages_v;
    L.stages_k = L.stages_k > kMaxStages ? kMaxStages : L.stages_k;
    L.v_off = L.k_off + (size_t)L.stages_k * kHalfStageBytes;
    L.aux_off = L.v_off + (size_t)L.stages_v * kHalfStageBytes;
    L.smem_bytes = 1024 + L.aux_off + kAuxBytes;
    return L;
}

// P = 2^(x * scale - m) for the 64 scores of one row, packed to bf16 pairs;
// returns the sum of the rounded values (what the PV product will use).
// POLY: one pair in four goes through the FMA-pipe polynomial instead of
// MUFU ex2 (masked tiles, whose -inf scores the polynomial clamps instead of
// zeroing, use MUFU only).
template <bool POLY>
__device__ __forceinline__ float exp_pack_tile(const float (&x)[64], float scale, float neg_m,
                                               uint32_t (&pk)[32])
{
    const uint64_t sc2 = pack2(scale, scale);
    const uint64_t nm2 = pack2(neg_m, neg_m);
    uint64_t y[32];
#pragma unroll
    for (int j = 0; j < 32; ++j)
        y[j] = fma2(pack2(x[2 * j], x[2 * j + 1]), sc2, nm2);
    uint64_t ls2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        float e0, e1;
        if (POLY && (j & 3) == 3) {
            unpack2(exp2_poly2(y[j]), e0, e1);
        } else {
            float y0, y1;
            unpack2(y[j], y0, y1);
            e0 = ex2(y0);
            e1 = ex2(y1);
        }
        __nv_bfloat162 h = __floats2bfloat162_rn(e0, e1);
        const uint32_t hb = *reinterpret_cast<uint32_t *>(&h);
        pk[j] = hb;
        ls2[j & 3] = add2(ls2[j & 3],
                          pack2(__uint_as_float(hb << 16), __uint_as_float(hb & 0xFFFF0000u)));
    }
    const uint64_t s01 = add2(add2(ls2[0], ls2[1]), add2(ls2[2], ls2[3]));
    float a0, a1;
    unpack2(s01, a0, a1);
    return a0 + a1;
}

template <int NB>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
               AttnArgs a, TreeMasks masks, int tiles_per_split, int n_split)
{
    constexpr int kSCol0 = NB == 2 ? 256 : 128;
    constexpr int kTmemCols = NB == 2 ? 512 : 256;
    constexpr int kSoftmaxWarps = 4 * NB;

    const int G = a.n_heads_q / a.n_heads_kv;
    const int R = G * a.n_tree;
    const TcLayout lay = tc_layout(NB, R);
    const int SK = lay.stages_k, SV = lay.stages_v, r_pad = lay.r_pad;

    extern __shared__ unsigned char smem_raw[];
    unsigned char *base = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char *sQ = base;
    unsigned char *sP = base + lay.p_off;
    unsigned char *sK = base + lay.k_off;
    unsigned char *sV = base + lay.v_off;
    TcAux *aux = reinterpret_cast<TcAux *>(base + lay.aux_off);
    TcBarriers *bar = &aux->bar;
    WorkspaceHeader *hdr = reinterpret_cast<WorkspaceHeader *>(a.workspace);
    volatile uint32_t *abort = &bar->abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int split = blockIdx.x, g = blockIdx.y;
    const int total = a.n_ctx + a.n_tree;
    const int n_tiles_all = (total + kTileN - 1) / kTileN;
    const int t_begin = split * tiles_per_split;
    const int n_tiles = min(t_begin + tiles_per_split, n_tiles_all) - t_begin;

    // softmax warps that take part in the per-tile sync: those with rows,
    // and warps 4-7, which rescale and write out O^T
    int sync_warps = 0;
    for (int w = 0; w < kSoftmaxWarps; ++w)
        sync_warps += (w < 4) || ((w / 4) * kBlockM + (w % 4) * 32 < R);

    if (threadIdx.x == 0) {
        for (int s = 0; s < SK; ++s) {
            mbar_init(smem_addr(&bar->full_k[s]), 1);
            mbar_init(smem_addr(&bar->empty_k[s]), 1);
        }
        for (int s = 0; s < SV; ++s) {
            mbar_init(smem_addr(&bar->full_v[s]), 1);
            mbar_init(smem_addr(&bar->empty_v[s]), 1);
        }
        for (int u = 0; u < 2; ++u) {
            for (int b = 0; b < NB; ++b)
                mbar_init(smem_addr(&bar->s_full[b][u]), 1);
            mbar_init(smem_addr(&bar->sm_sync[u]), sync_warps);
            mbar_init(smem_addr(&bar->p_full[u]), 4);
            bar->rescale_tile[u] = 0;
        }
        mbar_init(smem_addr(&bar->o_done), 1);
        mbar_init(smem_addr(&bar->o_final), 1);
        mbar_init(smem_addr(&bar->drain), 1);
        bar->abort = 0u;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_addr(&bar->tmem_base), kTmemCols);
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

    if (warp == 0 || warp == 2) {
        // ----------------------------------------- TMA producers (K, V)
        if (lane == 0) {
            const bool is_k = warp == 0;
            const int ns = is_k ? SK : SV;
            uint64_t *full = is_k ? bar->full_k : bar->full_v;
            uint64_t *empty = is_k ? bar->empty_k : bar->empty_v;
            unsigned char *ring = is_k ? sK : sV;
            const void *tmap = is_k ? static_cast<const void *>(&tmap_k)
                                    : static_cast<const void *>(&tmap_v);
            int issued = 0;
            for (int t = 0; t < n_tiles; ++t) {
                const int s = t % ns;
                if (t >= ns &&
                    !wait_bounded(smem_addr(&empty[s]), ((t / ns) & 1) ^ 1, abort, hdr))
                    break;
                const uint32_t fb = smem_addr(&full[s]);
                mbar_arrive_expect_tx(fb, kHalfStageBytes);
                const uint32_t dst = smem_addr(ring + s * kHalfStageBytes);
                const int pos0 = (t_begin + t) * kTileN;
                tma_load_3d(dst, tmap, 0, pos0, g, fb);
                tma_load_3d(dst + kBoxBytes, tmap, 64, pos0, g, fb);
                issued = t + 1;
            }
            if (*abort) {
                // let our own copies land before the CTA exits
                for (int t = max(0, issued - ns); t < issued; ++t)
                    wait_drain(smem_addr(&full[t % ns]), (t / ns) & 1);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16(kBlockM, kTileN, 0, 0);
            const uint32_t idesc_pv = idesc_bf16(kD, r_pad, 1, 0);
            // Descriptors are built once; per MMA only the start-address
            // field moves (address / 16 in the low bits, no carry out of it
            // inside shared memory).
            uint64_t qd[NB][8];
#pragma unroll
            for (int b = 0; b < NB; ++b)
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    qd[b][kk] = sdesc_sw128(smem_addr(sQ) + b * kQBlockBytes +
                                                (kk >> 2) * (kBlockM * 128) + (kk & 3) * 32,
                                            16, 1024);
            const uint64_t kd0 = sdesc_sw128(smem_addr(sK), 16, 1024);
            const uint64_t vd0 = sdesc_sw128(smem_addr(sV), kBoxBytes, 1024);
            const uint64_t pd0 = sdesc_sw128(smem_addr(sP), 16, 1024);
            constexpr uint64_t kStageStep = kHalfStageBytes >> 4;
            bool ok = true;
            for (int t = 0; t <= n_tiles && ok; ++t) {
                if (t < n_tiles) {
                    const int s = t % SK;
                    if (!wait_bounded(smem_addr(&bar->full_k[s]), (t / SK) & 1, abort, hdr)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t kd = kd0 + (uint64_t)s * kStageStep;
#pragma unroll
                    for (int b = 0; b < NB; ++b) {
                        const uint32_t d_col = tmem + kSCol0 + 64 * (2 * b + (t & 1));
                        mma_ss_c<0>(d_col, qd[b][0], kd, idesc_qk);
#pragma unroll
                        for (int kk = 1; kk < kD / 16; ++kk)
                            mma_ss_c<1>(d_col, qd[b][kk],
                                        kd + (((kk >> 2) * kBoxBytes + (kk & 3) * 32) >> 4),
                                        idesc_qk);
                        mma_commit(smem_addr(&bar->s_full[b][t & 1]));
                    }
                    mma_commit(smem_addr(&bar->empty_k[s]));
                }
                if (t >= 1) {
                    const int u = t - 1, s = u % SV;
                    if (!wait_bounded(smem_addr(&bar->full_v[s]), (u / SV) & 1, abort, hdr) ||
                        !wait_bounded(smem_addr(&bar->p_full[u & 1]), (u >> 1) & 1, abort, hdr)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t vd = vd0 + (uint64_t)s * kStageStep;
                    const uint64_t pd = pd0 + (uint64_t)((u & 1) * r_pad * 128 >> 4);
                    if (u == 0)
                        mma_ss_c<0>(tmem, vd, pd, idesc_pv);
                    else
                        mma_ss_c<1>(tmem, vd, pd, idesc_pv);
#pragma unroll
                    for (int kk = 1; kk < kTileN / 16; ++kk)
                        mma_ss_c<1>(tmem, vd + kk * (2048 >> 4), pd + kk * (32 >> 4), idesc_pv);
                    mma_commit(smem_addr(&bar->o_done));
                    if (u == n_tiles - 1)
                        mma_commit(smem_addr(&bar->o_final));
                    mma_commit(smem_addr(&bar->empty_v[s]));
                }
            }
            // every MMA issued above has finished before TMEM is released
            mma_commit(smem_addr(&bar->drain));
            wait_drain(smem_addr(&bar->drain), 0);
        }
    } else if (warp >= kFirstSoftmaxWarp && warp < kFirstSoftmaxWarp + kSoftmaxWarps &&
               ((warp - kFirstSoftmaxWarp) < 4 ||
                (warp - kFirstSoftmaxWarp) / 4 * kBlockM + (warp & 3) * 32 < R)) {
        // ---------------------------------------------------------- softmax
        const int b = (warp - kFirstSoftmaxWarp) / 4;
        const int quarter = warp & 3;
        const bool corrector = b == 0;   // warps 4-7: all 128 lanes between them
        const bool active = b * kBlockM + quarter * 32 < R;
        const int r = b * kBlockM + quarter * 32 + lane;
        const int rr = r < R ? r : 0;
        const int node = rr / G;
        const unsigned long long anc = masks.anc[node];
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        float m_ref = -INFINITY, l = 0.f;
        bool ok = true;
        for (int t = 0; t < n_tiles; ++t) {
            const int buf = t & 1;
            if (active) {
                if (!warp_wait_bounded(smem_addr(&bar->s_full[b][buf]), (t >> 1) & 1, abort,
                                       hdr)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint32_t raw[64];
                tmem_ld64(tmem + lane_off + kSCol0 + 64 * (2 * b + buf), raw);
                // raw scores; the scale (> 0) is applied inside the exponent
                float x[64];
                const int pos0 = (t_begin + t) * kTileN;
                const bool edge = pos0 + kTileN > a.n_ctx;
                if (!edge) {
#pragma unroll
                    for (int j = 0; j < 64; ++j)
                        x[j] = __uint_as_float(raw[j]);
                } else {
#pragma unroll
                    for (int j = 0; j < 64; ++j) {
                        const int pos = pos0 + j;
                        const bool seen = pos < total &&
                                          (pos < a.n_ctx || ((anc >> (pos - a.n_ctx)) & 1ull));
                        x[j] = seen ? __uint_as_float(raw[j]) : -INFINITY;
                    }
                }
                float pm[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    pm[e] = max3f(x[e], x[e + 8], x[e + 16]);
                    pm[e] = max3f(pm[e], x[e + 24], x[e + 32]);
                    pm[e] = max3f(pm[e], x[e + 40], x[e + 48]);
                    pm[e] = fmaxf(pm[e], x[e + 56]);
                }
                const float mx = max3f(max3f(pm[0], pm[1], pm[2]), max3f(pm[3], pm[4], pm[5]),
                                       fmaxf(pm[6], pm[7])) *
                                 a.scale_log2;
                // move the reference max only when this tile exceeds it by > 2^8
                float f = 1.f;
                const bool need = mx > m_ref + 8.0f;
                if (need) {
                    f = (m_ref == -INFINITY) ? 0.f : ex2(m_ref - mx);
                    m_ref = mx;
                    l *= f;
                }
                aux->factor[buf][r] = f;
                if (__any_sync(0xffffffffu, need) && lane == 0)
                    bar->rescale_tile[buf] = t + 1;
                const float neg_m = m_ref == -INFINITY ? 0.f : -m_ref;
                uint32_t pk[32];
                // the choice of exponent paths is hoisted out of the unrolled
                // loop so that each version is straight-line code
                if (edge)
                    l += exp_pack_tile<false>(x, a.scale_log2, neg_m, pk);
                else
                    l += exp_pack_tile<true>(x, a.scale_log2, neg_m, pk);
                // P^T row r: 64 bf16 = one 128-byte swizzled row of the K-major tile
                unsigned char *prow = sP + buf * r_pad * 128 + (r >> 3) * 1024 + (r & 7) * 128;
                if (r < r_pad) {
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        *reinterpret_cast<uint4 *>(prow + ((c ^ (r & 7)) << 4)) =
                            make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
                }
                fence_proxy_async_smem();
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(smem_addr(&bar->sm_sync[buf]));
            if (corrector) {
                if (!warp_wait_bounded(smem_addr(&bar->sm_sync[buf]), (t >> 1) & 1, abort, hdr)) {
                    ok = false;
                    break;
                }
                if (t > 0 && bar->rescale_tile[buf] == t + 1) {
                    // S(t) was committed after PV(t-2) was issued, so o_done has
                    // completed t-1 or t phases: parity (t-1) tells them apart
                    if (!warp_wait_bounded(smem_addr(&bar->o_done), (t - 1) & 1, abort, hdr)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    for (int c = 0; c < r_pad; c += 32) {
                        uint32_t o[32];
                        tmem_ld32(tmem + lane_off + c, o);
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            o[j] = __float_as_uint(__uint_as_float(o[j]) *
                                                   aux->factor[buf][c + j]);
                        tmem_st32(tmem + lane_off + c, o);
                    }
                    tmem_st_wait();
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(smem_addr(&bar->p_full[buf]));
            }
        }

        // ---- epilogue: row owners publish (m, l); warps 4-7 write O^T out
        if (ok) {
            const int rows_all = a.n_tree * a.n_heads_q;
            float *ws_o =
                reinterpret_cast<float *>(reinterpret_cast<char *>(a.workspace) + kHeaderBytes);
            float *ws_ml = ws_o + (size_t)n_split * rows_all * kD;
            if (active && r < R) {
                aux->l[r] = l;
                if (n_split > 1) {
                    const int orow = node * a.n_heads_q + g * G + r % G;
                    *reinterpret_cast<float2 *>(ws_ml + ((size_t)split * rows_all + orow) * 2) =
                        make_float2(m_ref, l);
                }
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(smem_addr(&bar->sm_sync[n_tiles & 1]));
            if (corrector &&
                warp_wait_bounded(smem_addr(&bar->sm_sync[n_tiles & 1]), (n_tiles >> 1) & 1,
                                  abort, hdr) &&
                warp_wait_bounded(smem_addr(&bar->o_final), 0, abort, hdr)) {
                tc_fence_after();
                const int d = quarter * 32 + lane;
                for (int c = 0; c < r_pad; c += 32) {
                    uint32_t o[32];
                    tmem_ld32(tmem + lane_off + c, o);
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int rw = c + j;
                        if (rw < R) {
                            const int orow = (rw / G) * a.n_heads_q + g * G + rw % G;
                            const float v = __uint_as_float(o[j]);
                            if (n_split == 1)
                                a.out[(size_t)orow * kD + d] = v / aux->l[rw];
                            else
                                ws_o[((size_t)split * rows_all + orow) * kD + d] = v;
                        }
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
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
    const TcLayout lay = tc_layout(NB, (a.n_heads_q / a.n_heads_kv) * a.n_tree);
    const size_t smem = lay.smem_bytes;
    static const cudaError_t attr = cudaFuncSetAttribute(
        attn_tc_kernel<NB>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemLimit);
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
    return head_dim == kD && rows <= kMaxRows && n_ctx >= kTcMinContext;
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
