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
//   S_b  = Q_b K^T      rows on M (128-row blocks b), N = 64 positions;
//                       Q_b is held in TMEM (loaded once), K is K-major in
//                       shared memory;
//   O^T += V^T P^T      head dim on M, all R rows on N (padded to 16),
//                       V^T is the TMA tile read MN-major, P^T K-major.
// P^T is written to shared memory by the softmax threads, one row each.
// Shared-memory bandwidth (about 128 B/clk for tensor-core operand reads)
// is the scarce resource at these shapes, which is why Q lives in TMEM
// rather than being re-read from shared memory by every QK instruction.
//
// CTA = (split, KV head), 15 warps, one CTA per SM:
//   warps 0, 2  TMA producers for K and for V: 64-position tiles (two
//               64-column boxes each, 128-byte swizzle) into two rings.  The
//               tensor map's row extent is n_ctx + T, so rows past the tree
//               tail arrive as zeros.
//   warp 1      allocates TMEM; one lane issues every tcgen05.mma.  A
//               block's S is released as soon as its softmax warps have
//               loaded it into registers, so QK of tile t+1 overlaps the
//               softmax arithmetic of tile t.
//   warps 4-7, 12-14  softmax, one thread per query row (a TMEM lane of
//               its block; block 0 rows on warps 4-7, block 1 rows on 12-14):
//               scale to base 2, ancestor mask on tiles that reach the tree
//               tail, exponentiate against a per-row reference max, write
//               the bf16 P^T row.  l sums the bf16-rounded P so the
//               normalisation matches what PV used.
//   warps 8-11  correctors: between them they see all 128 TMEM lanes, i.e.
//               all of D.  After every softmax warp has finished a tile they
//               release it to PV; when a row's reference max moved (only
//               when a tile's max exceeds it by more than 2^8) they first
//               rescale that row's O^T column.  At the end they write O^T.
// TMEM: O^T in [0, kOCols), Q_b in 64 columns from kQCol0, S_b in 64
// columns from kSCol0.
// Each split leaves an unnormalised partial (acc, m, l, q) for the combine
// kernel; q is the sum of the squared bf16 weights, so that the combine can
// recompute exactly the rows whose weight sits on too few positions for one
// bf16 rounding of P each.
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
constexpr int kThreads = 480;    // 15 warps
constexpr int kMaxStages = 8;
constexpr int kMaxRows = 224;    // block 1 has softmax warps 12-14 only
constexpr size_t kSmemLimit = 232448;           // dynamic shared memory per CTA

struct TcBarriers {
    uint64_t full_k[kMaxStages];
    uint64_t empty_k[kMaxStages];
    uint64_t full_v[kMaxStages];
    uint64_t empty_v[kMaxStages];
    uint64_t s_full[2];        // QK of a block landed in its S
    uint64_t s_free[2];        // that block's softmax warps hold S in registers
    uint64_t sm_sync[2];       // every softmax warp finished a tile
    uint64_t p_full[2];        // P^T(buf) written and O^T corrected
    uint64_t pv_done[2];       // PV of a tile whose P^T sat in buffer (t & 1) finished
    uint64_t o_final;          // committed once, after the last PV
    uint64_t drain[2];         // each issuing thread's own MMAs, before TMEM is freed
    uint32_t tmem_base;
    uint32_t abort;
    int32_t rescale_tile[2];   // tile index + 1 when that tile moved a row's max
};

struct TcAux {
    float factor[2][256];  // per-row O^T rescale factor of the tile (32-column reads)
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
    (void)nb;
    L.p_off = 0;
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
__device__ __forceinline__ float exp_pack_tile(const float (&x)[64], float scale, float neg_m,
                                               uint32_t (&pk)[32], float &sq)
{
    const uint64_t sc2 = pack2(scale, scale);
    const uint64_t nm2 = pack2(neg_m, neg_m);
    uint64_t y[32];
#pragma unroll
    for (int j = 0; j < 32; ++j)
        y[j] = fma2(pack2(x[2 * j], x[2 * j + 1]), sc2, nm2);
    uint64_t ls2[4] = {0ull, 0ull, 0ull, 0ull}, qs2[2] = {0ull, 0ull};
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        float y0, y1;
        unpack2(y[j], y0, y1);
        __nv_bfloat162 h = __floats2bfloat162_rn(ex2(y0), ex2(y1));
        const uint32_t hb = *reinterpret_cast<uint32_t *>(&h);
        pk[j] = hb;
        const uint64_t e2 = pack2(__uint_as_float(hb << 16), __uint_as_float(hb & 0xFFFF0000u));
        ls2[j & 3] = add2(ls2[j & 3], e2);
        qs2[j & 1] = fma2(e2, e2, qs2[j & 1]);
    }
    const uint64_t s01 = add2(add2(ls2[0], ls2[1]), add2(ls2[2], ls2[3]));
    const uint64_t q01 = add2(qs2[0], qs2[1]);
    float a0, a1;
    unpack2(q01, a0, a1);
    sq = a0 + a1;
    unpack2(s01, a0, a1);
    return a0 + a1;
}

template <int NB>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
               AttnArgs a, TreeMasks masks, int tiles_per_split, int n_split)
{
    constexpr int kOCols = NB == 2 ? 256 : 128;
    constexpr int kQCol0 = kOCols;
    constexpr int kSCol0 = kQCol0 + 64 * NB;
    constexpr int kTmemCols = NB == 2 ? 512 : 256;

    const int G = a.n_heads_q / a.n_heads_kv;
    const int R = G * a.n_tree;
    const TcLayout lay = tc_layout(NB, R);
    const int SK = lay.stages_k, SV = lay.stages_v, r_pad = lay.r_pad;

    extern __shared__ unsigned char smem_raw[];
    unsigned char *base = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
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

    // softmax warps with rows: they arrive once per tile on sm_sync, and on
    // their block's s_free
    int sync_warps = 0, block_warps[2] = {0, 0};
    for (int w = 0; w < 4 * NB && w < 7; ++w) {
        const int has = (w / 4) * kBlockM + (w % 4) * 32 < R;
        sync_warps += has;
        block_warps[w / 4] += has;
    }

    if (threadIdx.x == 0) {
        for (int s = 0; s < SK; ++s) {
            mbar_init(smem_addr(&bar->full_k[s]), 1);
            mbar_init(smem_addr(&bar->empty_k[s]), 1);
        }
        for (int s = 0; s < SV; ++s) {
            mbar_init(smem_addr(&bar->full_v[s]), 1);
            mbar_init(smem_addr(&bar->empty_v[s]), 1);
        }
        for (int b = 0; b < NB; ++b) {
            mbar_init(smem_addr(&bar->s_full[b]), 1);
            mbar_init(smem_addr(&bar->s_free[b]), block_warps[b]);
        }
        for (int u = 0; u < 2; ++u) {
            mbar_init(smem_addr(&bar->sm_sync[u]), sync_warps);
            mbar_init(smem_addr(&bar->p_full[u]), 4);
            bar->rescale_tile[u] = 0;
        }
        mbar_init(smem_addr(&bar->pv_done[0]), 1);
        mbar_init(smem_addr(&bar->pv_done[1]), 1);
        mbar_init(smem_addr(&bar->o_final), 1);
        mbar_init(smem_addr(&bar->drain[0]), 1);
        mbar_init(smem_addr(&bar->drain[1]), 1);
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

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bar->tmem_base;

    // Q rows of this KV head into TMEM, as the A operand of QK: the thread
    // owning query row r (node r / G, head g*G + r % G) writes its 128 bf16
    // as 64 packed columns of its block's lane.
    if ((warp >= 4 && warp < 8) || (NB == 2 && warp >= 12)) {
        const int b = warp < 8 ? 0 : 1;
        const int quarter = warp & 3;
        if (b * kBlockM + quarter * 32 < R) {
            const int r = b * kBlockM + quarter * 32 + lane;
            uint32_t qv[64];
            if (r < R) {
                const uint4 *src = reinterpret_cast<const uint4 *>(
                    a.q + ((int64_t)(r / G) * a.n_heads_q + g * G + r % G) * kD);
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const uint4 u = src[c];
                    qv[4 * c] = u.x;
                    qv[4 * c + 1] = u.y;
                    qv[4 * c + 2] = u.z;
                    qv[4 * c + 3] = u.w;
                }
            } else {
#pragma unroll
                for (int c = 0; c < 64; ++c)
                    qv[c] = 0u;
            }
            const uint32_t qa = tmem + ((uint32_t)(quarter * 32) << 16) + kQCol0 + 64 * b;
            uint32_t (&q0)[32] = *reinterpret_cast<uint32_t (*)[32]>(&qv[0]);
            uint32_t (&q1)[32] = *reinterpret_cast<uint32_t (*)[32]>(&qv[32]);
            tmem_st32(qa, q0);
            tmem_st32(qa + 32, q1);
            tmem_st_wait();
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

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
    } else if (warp == 1 || warp == 3) {
        // --------------------------------------------- MMA issuers: QK, PV
        // Two threads feed the tensor core, so that one issues while the
        // other waits; each commits (and at the end drains) its own MMAs.
        if (lane == 0) {
            // Descriptors are built once; per MMA only the start-address
            // field moves (address / 16 in the low bits, no carry out of it
            // inside shared memory).
            constexpr uint64_t kStageStep = kHalfStageBytes >> 4;
            if (warp == 1) {
                constexpr uint32_t idesc_qk = idesc_bf16(kBlockM, kTileN, 0, 0);
                const uint64_t kd0 = sdesc_sw128(smem_addr(sK), 16, 1024);
                for (int t = 0; t < n_tiles; ++t) {
                    const int s = t % SK;
                    if (!wait_bounded(smem_addr(&bar->full_k[s]), (t / SK) & 1, abort, hdr))
                        break;
                    tc_fence_after();
                    const uint64_t kd = kd0 + (uint64_t)s * kStageStep;
                    bool ok = true;
#pragma unroll
                    for (int b = 0; b < NB; ++b) {
                        // S_b is reused: its softmax warps must hold S(t-1)
                        if (t > 0 &&
                            !wait_bounded(smem_addr(&bar->s_free[b]), (t - 1) & 1, abort, hdr)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t d_col = tmem + kSCol0 + 64 * b;
                        const uint32_t q_col = tmem + kQCol0 + 64 * b;
                        mma_ts_c<0>(d_col, q_col, kd, idesc_qk);
#pragma unroll
                        for (int kk = 1; kk < kD / 16; ++kk)
                            mma_ts_c<1>(d_col, q_col + kk * 8,
                                        kd + (((kk >> 2) * kBoxBytes + (kk & 3) * 32) >> 4),
                                        idesc_qk);
                        mma_commit(smem_addr(&bar->s_full[b]));
                    }
                    if (!ok)
                        break;
                    mma_commit(smem_addr(&bar->empty_k[s]));
                }
            } else {
                const uint32_t idesc_pv = idesc_bf16(kD, r_pad, 1, 0);
                const uint64_t vd0 = sdesc_sw128(smem_addr(sV), kBoxBytes, 1024);
                const uint64_t pd0 = sdesc_sw128(smem_addr(sP), 16, 1024);
                for (int t = 0; t < n_tiles; ++t) {
                    const int s = t % SV;
                    if (!wait_bounded(smem_addr(&bar->full_v[s]), (t / SV) & 1, abort, hdr) ||
                        !wait_bounded(smem_addr(&bar->p_full[t & 1]), (t >> 1) & 1, abort, hdr))
                        break;
                    tc_fence_after();
                    const uint64_t vd = vd0 + (uint64_t)s * kStageStep;
                    const uint64_t pd = pd0 + (uint64_t)((t & 1) * r_pad * 128 >> 4);
                    if (t == 0)
                        mma_ss_c<0>(tmem, vd, pd, idesc_pv);
                    else
                        mma_ss_c<1>(tmem, vd, pd, idesc_pv);
#pragma unroll
                    for (int kk = 1; kk < kTileN / 16; ++kk)
                        mma_ss_c<1>(tmem, vd + kk * (2048 >> 4), pd + kk * (32 >> 4), idesc_pv);
                    mma_commit(smem_addr(&bar->pv_done[t & 1]));
                    if (t == n_tiles - 1)
                        mma_commit(smem_addr(&bar->o_final));
                    mma_commit(smem_addr(&bar->empty_v[s]));
                }
            }
            // every MMA this thread issued has finished before TMEM is released
            const int dn = warp == 1 ? 0 : 1;
            mma_commit(smem_addr(&bar->drain[dn]));
            wait_drain(smem_addr(&bar->drain[dn]), 0);
        }
    } else if ((warp >= 4 && warp < 8) || (NB == 2 && warp >= 12)) {
        // ---------------------------------------------------------- softmax
        const int b = warp < 8 ? 0 : 1;
        const int quarter = warp & 3;
        const int r = b * kBlockM + quarter * 32 + lane;
        if (b * kBlockM + quarter * 32 < R) {
            const int rr = r < R ? r : 0;
            const int node = rr / G;
            const unsigned long long anc = masks.anc[node];
            const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
            // q: the sum of the squared rounded weights, rescaled with l
            // (each weight is at most 2^8, so it cannot overflow)
            float m_ref = -INFINITY, l = 0.f, q = 0.f;
            bool ok = true;
            for (int t = 0; t < n_tiles; ++t) {
                const int buf = t & 1;
                if (!warp_wait_bounded(smem_addr(&bar->s_full[b]), t & 1, abort, hdr)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint32_t raw[64];
                tmem_ld64(tmem + lane_off + kSCol0 + 64 * b, raw);
                // S is in registers: QK of the next tile may overwrite it
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(smem_addr(&bar->s_free[b]));
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
                    q *= f * f;
                }
                aux->factor[buf][r] = f;
                if (__any_sync(0xffffffffu, need) && lane == 0)
                    bar->rescale_tile[buf] = t + 1;
                const float neg_m = m_ref == -INFINITY ? 0.f : -m_ref;
                uint32_t pk[32];
                float dq;
                l += exp_pack_tile(x, a.scale_log2, neg_m, pk, dq);
                q += dq;
                // P^T(t) reuses the buffer of P^T(t-2): PV(t-2) must be done.
                // PV(t-4), the buffer's previous user, finished before this
                // warp wrote P^T(t-2), so pv_done[buf] has exactly one phase
                // that can still be open
                if (t >= 2 &&
                    !warp_wait_bounded(smem_addr(&bar->pv_done[buf]), ((t - 2) >> 1) & 1, abort,
                                       hdr)) {
                    ok = false;
                    break;
                }
                // P^T row r: 64 bf16 = one 128-byte swizzled row of the K-major tile
                unsigned char *prow = sP + buf * r_pad * 128 + (r >> 3) * 1024 + (r & 7) * 128;
                if (r < r_pad) {
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        *reinterpret_cast<uint4 *>(prow + ((c ^ (r & 7)) << 4)) =
                            make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(smem_addr(&bar->sm_sync[buf]));
            }
            // publish (m, l) for the correctors' epilogue
            if (ok) {
                const int rows_all = a.n_tree * a.n_heads_q;
                float *ws_ml = reinterpret_cast<float *>(reinterpret_cast<char *>(a.workspace) +
                                                         kHeaderBytes) +
                               (size_t)n_split * rows_all * kD;
                if (r < R) {
                    const int orow = node * a.n_heads_q + g * G + r % G;
                    *reinterpret_cast<float4 *>(ws_ml + ((size_t)split * rows_all + orow) * 4) =
                        make_float4(m_ref, l, q, 0.f);
                }
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(smem_addr(&bar->sm_sync[n_tiles & 1]));
            }
        }
    } else if (warp >= 8 && warp < 12) {
        // -------------------------------------------------------- correctors
        const int quarter = warp & 3;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        bool ok = true;
        for (int t = 0; t < n_tiles; ++t) {
            const int buf = t & 1;
            if (!warp_wait_bounded(smem_addr(&bar->sm_sync[buf]), (t >> 1) & 1, abort, hdr)) {
                ok = false;
                break;
            }
            if (t > 0 && bar->rescale_tile[buf] == t + 1) {
                // PV(t-1) must be done.  Every softmax warp waited for
                // PV(t-2) before writing P^T(t), and PV runs in order, so
                // PV(t-3) is done too: pv_done[(t-1) & 1] has one open phase
                if (!warp_wait_bounded(smem_addr(&bar->pv_done[(t - 1) & 1]), ((t - 1) >> 1) & 1,
                                       abort, hdr)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int c = 0; c < r_pad; c += 32) {
                    uint32_t o[32];
                    tmem_ld32(tmem + lane_off + c, o);
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        o[j] = __float_as_uint(__uint_as_float(o[j]) * aux->factor[buf][c + j]);
                    tmem_st32(tmem + lane_off + c, o);
                }
                tmem_st_wait();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(smem_addr(&bar->p_full[buf]));
        }
        // ---- epilogue: O^T (D on lanes, query rows on columns) to out / partials
        if (ok &&
            warp_wait_bounded(smem_addr(&bar->sm_sync[n_tiles & 1]), (n_tiles >> 1) & 1, abort,
                              hdr) &&
            warp_wait_bounded(smem_addr(&bar->o_final), 0, abort, hdr)) {
            tc_fence_after();
            const int rows_all = a.n_tree * a.n_heads_q;
            float *ws_o =
                reinterpret_cast<float *>(reinterpret_cast<char *>(a.workspace) + kHeaderBytes);
            const int d = quarter * 32 + lane;
            for (int c = 0; c < r_pad; c += 32) {
                uint32_t o[32];
                tmem_ld32(tmem + lane_off + c, o);
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int rw = c + j;
                    if (rw < R) {
                        const int orow = (rw / G) * a.n_heads_q + g * G + rw % G;
                        ws_o[((size_t)split * rows_all + orow) * kD + d] = __uint_as_float(o[j]);
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
template <int NB>
cudaError_t launch_nb(const AttnArgs &a, const TreeMasks &masks, const AttnPlan &p,
                      cudaStream_t stream)
{
    CUtensorMap mk, mv;
    const int rows = a.n_ctx + a.n_tree;
    if (!encode_kv_map(&mk, a.k, rows, a.kv_cap, a.n_heads_kv, kTileN) ||
        !encode_kv_map(&mv, a.v, rows, a.kv_cap, a.n_heads_kv, kTileN))
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
    // no overflow flags: the reference max moves with the scores
    return attn_exact_combine_launch(a, masks, p.n_split, p.tiles_per_split * kTileN, nullptr,
                                     stream);
}

}  // namespace

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
