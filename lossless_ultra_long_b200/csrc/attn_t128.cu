// attn_t128.cu -- split-KV tree-verify attention on the 5th-generation tensor
// cores with 128-position KV tiles and the softmax spread evenly over the
// four SM sub-partitions.
//
// Tree-based verification runs every draft-tree node's query against the
// full KV cache, each node seeing the context plus its own root path
// (TokenSwift, aiboss88.com, "TokenSwift's technical principles"; tencent
// article, parallel-verification figure; arxivlens "Technical
// Contribution": a 3-ary tree).  For one KV head the R = G*T query rows
// (node-major, then the group's heads) share every KV tile, so K/V are
// streamed from HBM once per split.
//
// Products (orientations the tensor core runs at full rate):
//   S_b  = Q_b K^T     query rows on M (128-lane blocks b), N = 128 positions.
//                      Block 0's Q sits in TMEM; block 1's (rows 128..R-1)
//                      in shared memory.
//   O^T += V^T P^T     head dim on M, the R rows on N (padded to 16); V^T is
//                      the TMA tile read MN-major, P^T is K-major.
// An MMA below N = 128 costs about as much as one at N = 128, so a 128-wide
// tile needs half the QK instructions of a 64-wide one.
//
// Query rows are spread over the TMEM lane quarters: block b's rows are cut
// into four runs of rq_b = ceil(R_b / 4); run q sits in lanes 32q..32q+rq_b-1.
// A warp can only reach its own lane quarter (its sub-partition), so this
// gives every sub-partition the same share of the exponentials.  A softmax
// warp owns a unit of 16 lanes of one block and reads it with the 16x256b
// TMEM shape: four threads per row, 32 of the tile's 128 scores each, two
// rows per thread (lanes t/4 and 8 + t/4 of the unit).
//
// CTA = (split, KV head), 16 warps, one CTA per SM:
//   warp 3      one lane is the TMA producer of K and V (two 64-column boxes
//               of 128 positions per tile, 128-byte swizzle), K one tile
//               ahead of V.  The map's row extent is n_ctx + T, so rows past
//               the tree tail arrive as zeros.  It starts as soon as the
//               barriers exist, while the other warps put the query rows in
//               place, so HBM is busy from the first microsecond.
//   warp 0      when the call asks for the root node's scores and all of
//               them sit in TMEM lane quarter 0 (the warp's own quarter),
//               reads them out of S_0 each tile and stores them, so that no
//               softmax warp carries that work; otherwise idle.
//   warp 1      allocates TMEM; one lane issues the QK MMAs.  A block's S is
//               released as soon as its softmax warps hold it in registers.
//   warp 2      one lane issues the PV MMAs.
//   warps 4-15  softmax, unit j = (warp - 4) / 4 of lane quarter warp % 4:
//               scale to base 2, ancestor mask on tiles that reach the tree
//               tail, exponentiate against a per-row reference max, write
//               the bf16 P^T rows.  l sums the bf16-rounded P so the
//               normalisation matches what PV used.  At the end they read
//               O^T (their lane quarters together cover all of D) into the
//               freed K/V ring in output-row order and send each node's G
//               rows to the workspace with one bulk copy: per-row stores
//               from every SM at once took several microseconds per CTA,
//               on the critical path of each split.
// TMEM: O^T in [0, 192), Q_0 in [192, 256), S_0 in [256, 384), S_1 in
// [384, 512).
//
// The reference max of a row is fixed at the first tile where the row sees
// anything, and never moves, so the softmax warps need no per-tile
// agreement with each other and no per-tile maximum at all.  fp32 has room
// for it: a row's weights are at most its sum l, and while l <= 2^63 the
// accumulated O^T stays below 2^63 * max|V|, far from overflow (a score
// rise of about 44 nats inside one split would be needed to exceed it).  A
// split in which some row's l ends above 2^63 (or not a number) raises a
// flag; the combine kernel then recomputes that split's partial for the
// affected head exactly (fp32, online softmax on CUDA cores) instead of
// reading it.
// Each split leaves an unnormalised partial (acc, m, l, q) and its flag;
// the combine kernel always runs.
//
// P enters the PV product as one bf16 value and l sums those same rounded
// values, so a row's output is an exact weighted mean of V with weights
// perturbed by at most one bf16 rounding each.  Spread over many positions
// those perturbations average out (the error falls like 1/sqrt of the
// effective number of positions); on a row whose weight sits on a handful
// of positions they do not.  The kernel therefore also keeps q, the sum of
// the squared rounded weights, so that l^2 / q is the row's effective
// number of positions.  The combine recomputes exactly (fp32, CUDA cores)
// the splits that carry the weight of any row whose count over all splits
// is below kNeffMin.
//
// Every wait is on an mbarrier and bounded (about a second): on expiry the
// kernel records TS_ERR_TIMEOUT in the workspace status word, all roles
// leave their loops, and TMEM is freed before the CTA exits.
#include <math.h>

#include "attn_common.cuh"
#include "sm100.cuh"

namespace ts {
namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kTileN = 128;                  // KV positions per tile
constexpr int kBlockM = 128;                 // query rows per QK block (TMEM lanes)
constexpr int kBoxBytes = kTileN * 64 * 2;   // one 64-column box of a tile: 16 KB
constexpr int kStageBytes = 2 * kBoxBytes;   // K (or V) of a tile
constexpr int kThreads = 512;                // 16 warps
constexpr int kMaxStages = 4;
constexpr int kMaxRows = 192;
constexpr int kQCol = 192;                   // Q of block 0: 128 bf16 = 64 columns per lane
constexpr int kSCol = 256;                   // S_b: 128 columns from kSCol + 128 b
constexpr int kTmemCols = 512;
constexpr int kQ1Bytes = kBlockM * kD * 2;   // Q of block 1 in shared memory: 32 KB
constexpr float kMaxRowSum = 9.223372036854775808e18f;   // 2^63: bound on a row's weight sum
// Rows whose effective number of attended positions is below this are
// recomputed exactly.  With each weight perturbed by one bf16 rounding
// (relative spread 2^-8 / sqrt(3)), the output error of a row with n
// effective positions has a standard deviation of about
// 2^-8 / sqrt(3) * rms|v - o| / sqrt(n); at n = 64 and |v - o| ~ 1.4
// (bf16 N(0,1) values) that is 4e-4, so even the largest of many such
// errors stays inside 2e-3.
constexpr float kNeffMin = 64.f;
constexpr size_t kSmemLimit = 232448;        // dynamic shared memory per CTA
static_assert(kBlockM % 32 == 0, "a 32-column O^T chunk lies inside one query block");
constexpr int kBarQuery = 1;                 // named barrier: query rows in place
constexpr int kBarOut = 2;                   // named barrier: O^T staged in shared memory
constexpr int kBarQLoads = 3;                // named barrier: the query loads are issued
constexpr int kQLoadThreads = 32 * 9;        // warps 4-11 arrive, the producer warp waits

struct Bars {
    uint64_t full_k[kMaxStages];
    uint64_t empty_k[kMaxStages];
    uint64_t full_v[kMaxStages];
    uint64_t empty_v[kMaxStages];
    uint64_t s_full[2];   // QK of block b landed in S_b
    uint64_t s_free[2];   // block b's softmax warps hold S_b in registers
    uint64_t sm_done;     // every softmax warp wrote its P^T rows
    uint64_t pv_done;     // one commit per PV
    uint64_t pv_issued[2];  // PV(t) is in the tensor queue (slot t & 1)
    uint64_t o_final;     // committed once, after the last PV
    uint64_t drain[2];    // each issuing thread's own MMAs, before TMEM is freed
    uint32_t tmem_base;
    uint32_t abort;
    int32_t overflow;     // some row exceeded its reference max by the headroom
};

struct Aux {
    Bars bar;
};
constexpr size_t kAuxBytes = (sizeof(Aux) + 1023) / 1024 * 1024;

struct Layout {
    int r_pad;  // rows rounded up to 16: N of the PV product
    int stages_k, stages_v;
    bool o_staged;  // the freed K/V ring holds every O row (fp32) for the write-out
    size_t q1_off, p_off, k_off, v_off, aux_off, rs_off, smem_bytes;
};

// Rows per TMEM lane quarter in block 0 (rows 0..min(R, 128) - 1 cut into
// four equal runs).
__host__ __device__ inline int t128_rq0(int rows) { return ((rows < kBlockM ? rows : kBlockM) + 3) / 4; }

// With two blocks, block 1 holds rows 0..R1-1 (R1 = R - 128) and block 0
// rows R1..R-1, so that the root node's rows sit in block 1, whose softmax
// warps carry a quarter of a block-0 warp's exponentials at 160 rows.  P^T
// row (and O^T column) n is block-0 row n for n < 128, block-1 row n - 128.
__host__ __device__ inline int t128_row_of(int n, int R)
{
    return R > kBlockM ? (n < kBlockM ? (R - kBlockM) + n : n - kBlockM) : n;
}

// Whether warp 0 reads the root node's scores out of TMEM (one block: the G
// root rows are TMEM lanes 0..G-1 of S_0, inside lanes 0..15, i.e. G <= 8
// and G <= rq0).
__host__ __device__ inline bool t128_rs_warp0(const AttnArgs &a, int T)
{
    const int G = a.n_heads_q / a.n_heads_kv;
    const int R = G * T;
    return a.root_scores != nullptr && R <= kBlockM && G <= 8 && G <= t128_rq0(R);
}

// Whether the block-1 softmax warp of lane quarter 0 stores the root node's
// scores (two blocks: block 1's first quarter run, rows 0..rq1-1, holds the
// G root rows when G <= rq1 and G <= 8, i.e. they are its first 16 lanes).
__host__ __device__ inline bool t128_rs_block1(const AttnArgs &a, int T)
{
    const int G = a.n_heads_q / a.n_heads_kv;
    const int R = G * T;
    const int rq1 = (R - kBlockM + 3) / 4;
    return a.root_scores != nullptr && R > kBlockM && G <= 8 && G <= rq1;
}

// Shared memory that stages the root node's scores for bulk copies (two
// tiles of the G root rows) when block 1 stores them and every row starts
// on a 16-byte boundary; 0 otherwise (plain stores, or warp 0).
__host__ __device__ inline int t128_rs_bytes(const AttnArgs &a, int T)
{
    const bool bulk = t128_rs_block1(a, T) &&
                      (reinterpret_cast<uintptr_t>(a.root_scores) & 15) == 0 &&
                      (a.n_ctx & 3) == 0;
    return bulk ? 2 * (a.n_heads_q / a.n_heads_kv) * kTileN * 4 : 0;
}

__host__ __device__ inline Layout t128_layout(int rows, int rs_bytes)
{
    Layout L;
    L.r_pad = (rows + 15) / 16 * 16;
    L.q1_off = 0;
    L.p_off = rows > kBlockM ? kQ1Bytes : 0;
    // P^T: positions 0-63 then 64-127, each r_pad rows of 128 bytes; then
    // 1 KB that rows past the query rows are written to
    L.k_off = L.p_off + (size_t)L.r_pad * 256 + 1024;
    const size_t fixed = 1024 + L.k_off + kAuxBytes + rs_bytes;
    int stages = (int)((kSmemLimit - fixed) / kStageBytes);
    stages = stages > 2 * kMaxStages ? 2 * kMaxStages : stages;
    L.stages_v = 2;
    L.stages_k = stages - 2 > kMaxStages ? kMaxStages : stages - 2;
    L.v_off = L.k_off + (size_t)L.stages_k * kStageBytes;
    L.o_staged = (size_t)rows * kD * 4 <= (size_t)(L.stages_k + L.stages_v) * kStageBytes;
    L.aux_off = L.v_off + (size_t)L.stages_v * kStageBytes;
    L.rs_off = L.aux_off + kAuxBytes;
    L.smem_bytes = 1024 + L.rs_off + rs_bytes;
    return L;
}

// P = 2^(x * scale - m) for the 32 scores a thread holds of row A
// (registers r[4j], r[4j + 1], j = 0..15) and, when TWO, of row B
// (r[4j + 2], r[4j + 3]), packed to bf16 pairs; adds the sums of the rounded
// values (what the PV product will use) to lA and lB, and their squares to
// qA and qB.  Both rows advance together, so each score register is dead
// once its pair is packed.
template <bool TWO>
__device__ __forceinline__ void exp_pack_rows(const uint32_t (&r)[64], float scale, float neg_mA,
                                              float neg_mB, uint32_t (&pA)[16],
                                              uint32_t (&pB)[16], float &lA, float &lB,
                                              float &qA, float &qB)
{
    const uint64_t sc2 = pack2(scale, scale);
    const uint64_t nA2 = pack2(neg_mA, neg_mA);
    const uint64_t nB2 = pack2(neg_mB, neg_mB);
    uint64_t sA = 0ull, sB = 0ull, wA = 0ull, wB = 0ull;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
#pragma unroll
        for (int h = 0; h < (TWO ? 2 : 1); ++h) {
            const uint64_t y = fma2(pack2(__uint_as_float(r[4 * j + 2 * h]),
                                          __uint_as_float(r[4 * j + 2 * h + 1])),
                                    sc2, h ? nB2 : nA2);
            float y0, y1;
            unpack2(y, y0, y1);
            __nv_bfloat162 hv = __floats2bfloat162_rn(ex2(y0), ex2(y1));
            const uint32_t hb = *reinterpret_cast<uint32_t *>(&hv);
            const uint64_t e2 =
                pack2(__uint_as_float(hb << 16), __uint_as_float(hb & 0xFFFF0000u));
            if (h) {
                pB[j] = hb;
                sB = add2(sB, e2);
                wB = fma2(e2, e2, wB);
            } else {
                pA[j] = hb;
                sA = add2(sA, e2);
                wA = fma2(e2, e2, wA);
            }
        }
    }
    // a split whose rows keep l <= 2^63 has every sum of squares <= l^2 <=
    // 2^126, inside the fp32 range (a larger l flags the split anyway)
    float a0, a1;
    unpack2(sA, a0, a1);
    lA += a0 + a1;
    unpack2(wA, a0, a1);
    qA += a0 + a1;
    if (TWO) {
        unpack2(sB, a0, a1);
        lB += a0 + a1;
        unpack2(wB, a0, a1);
        qB += a0 + a1;
    }
}

// Row maximum of the 32 scores a thread holds of one row.
__device__ __forceinline__ float row_max(const uint32_t (&r)[64], int e)
{
    float m[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        m[u] = max3f(__uint_as_float(r[4 * u + e]), __uint_as_float(r[4 * u + e + 1]),
                     __uint_as_float(r[4 * (u + 4) + e]));
        m[u] = max3f(m[u], __uint_as_float(r[4 * (u + 4) + e + 1]),
                     __uint_as_float(r[4 * (u + 8) + e]));
        m[u] = max3f(m[u], __uint_as_float(r[4 * (u + 8) + e + 1]),
                     __uint_as_float(r[4 * (u + 12) + e]));
        m[u] = fmaxf(m[u], __uint_as_float(r[4 * (u + 12) + e + 1]));
    }
    return fmaxf(max3f(m[0], m[1], m[2]), m[3]);
}

// Eight rows' P (one half of a 16-lane unit: rows nbase + r, r = 0..7, of
// which the first n_valid are query rows) into the K-major,
// 128-byte-swizzled P^T tile.  pk[j] of thread t holds positions
// 8j + 2(t%4), +1 of row t/4: the m8n8 fragment of matrix j, so four
// stmatrix instructions write the 16 matrices, each row a 16-byte chunk.
// Rows past n_valid go to the scratch kilobyte instead, so they cannot land
// on another lane quarter's rows.
__device__ __forceinline__ void store_p_half(uint32_t p_addr, uint32_t scratch, int nbase,
                                             int n_valid, int r_pad, int lane,
                                             const uint32_t (&pk)[16])
{
    const int r = lane & 7, n = nbase + r;
    const bool valid = r < n_valid;
    const uint32_t row = p_addr + (uint32_t)((n >> 3) * 1024 + (n & 7) * 128);
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const int j = 4 * m + (lane >> 3);
        const uint32_t addr = valid ? row + (uint32_t)((j >> 3) * (r_pad * 128) +
                                                       (((j & 7) ^ (n & 7)) << 4))
                                    : scratch + (uint32_t)(lane << 4);
        stmatrix_x4(addr, pk[4 * m], pk[4 * m + 1], pk[4 * m + 2], pk[4 * m + 3]);
    }
}

__global__ void __launch_bounds__(kThreads, 1)
attn_t128_kernel(const __grid_constant__ CUtensorMap tmap_k,
                 const __grid_constant__ CUtensorMap tmap_v, AttnArgs a, TreeMasks masks,
                 int tiles_per_split, int n_split, int nodes_per_group, int32_t *flags)
{
    const int G = a.n_heads_q / a.n_heads_kv;
    // node group blockIdx.z: tree nodes node0 .. node0 + T - 1 (global node
    // indices), its rows m = local node * G + head in group
    const int node0 = blockIdx.z * nodes_per_group;
    const int T = min(nodes_per_group, a.n_tree - node0);
    if (node0 != 0)
        a.root_scores = nullptr;   // the root node's rows live in group 0
    const int R = G * T;
    const int NB = R > kBlockM ? 2 : 1;
    const int R0 = R < kBlockM ? R : kBlockM, R1 = R - R0;
    const int rq0 = (R0 + 3) / 4, rq1 = (R1 + 3) / 4;  // rows per lane quarter
    const int u0 = (rq0 + 15) / 16, u1 = (rq1 + 15) / 16;
    const int U = u0 + u1;  // softmax warps per lane quarter (at most 3)
    const bool rs_warp0 = t128_rs_warp0(a, T);
    const int rs_bytes = t128_rs_bytes(a, T);
    const Layout lay = t128_layout(R, rs_bytes);
    const int SK = lay.stages_k, SV = lay.stages_v, r_pad = lay.r_pad;

    extern __shared__ unsigned char smem_raw[];
    unsigned char *base = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char *sQ1 = base + lay.q1_off;
    unsigned char *sP = base + lay.p_off;
    unsigned char *sK = base + lay.k_off;
    unsigned char *sV = base + lay.v_off;
    Aux *aux = reinterpret_cast<Aux *>(base + lay.aux_off);
    Bars *bar = &aux->bar;
    WorkspaceHeader *hdr = reinterpret_cast<WorkspaceHeader *>(a.workspace);
    volatile uint32_t *abort = &bar->abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int split = blockIdx.x, g = blockIdx.y;
    const int total = a.n_ctx + a.n_tree;
    const int n_tiles_all = (total + kTileN - 1) / kTileN;
    const int t_begin = split * tiles_per_split;
    const int n_tiles = min(t_begin + tiles_per_split, n_tiles_all) - t_begin;

    if (threadIdx.x == 0) {
        for (int s = 0; s < SK; ++s) {
            mbar_init(smem_addr(&bar->full_k[s]), 1);
            mbar_init(smem_addr(&bar->empty_k[s]), 1);
        }
        for (int s = 0; s < SV; ++s) {
            mbar_init(smem_addr(&bar->full_v[s]), 1);
            mbar_init(smem_addr(&bar->empty_v[s]), 1);
        }
        mbar_init(smem_addr(&bar->s_full[0]), 1);
        mbar_init(smem_addr(&bar->s_full[1]), 1);
        mbar_init(smem_addr(&bar->s_free[0]), 4 * u0 + (rs_warp0 ? 1 : 0));
        mbar_init(smem_addr(&bar->s_free[1]), u1 > 0 ? 4 * u1 : 1);
        mbar_init(smem_addr(&bar->sm_done), 4 * U);
        mbar_init(smem_addr(&bar->pv_done), 1);
        mbar_init(smem_addr(&bar->pv_issued[0]), 1);
        mbar_init(smem_addr(&bar->pv_issued[1]), 1);
        mbar_init(smem_addr(&bar->o_final), 1);
        mbar_init(smem_addr(&bar->drain[0]), 1);
        mbar_init(smem_addr(&bar->drain[1]), 1);
        bar->abort = 0u;
        bar->overflow = 0;
        fence_mbar_init();
        // the combine kernel may take the SMs this grid leaves idle (and
        // then each SM a split frees) and wait there for this grid's end
        launch_dependents();
    }
    if (warp == 1) {
        tmem_alloc(smem_addr(&bar->tmem_base), kTmemCols);
        tmem_relinquish();
    }
    if (warp == 3 && lane == 0) {
        prefetch_tmap(&tmap_k);
        prefetch_tmap(&tmap_v);
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bar->tmem_base;
    // The TMA producer (warp 3) starts streaming K and V as soon as the
    // query rows' loads are on their way (ahead of the K/V requests, so
    // that they are not queued behind a whole ring of tiles from every
    // CTA); the other warps put the query rows in place meanwhile and meet
    // at a named barrier of their own.

    // Query rows of this KV head into place: row n = node * G + (head - g*G).
    // Block 0 (rows 0..R0-1) into TMEM lanes (warps 4-7, 32x32b stores);
    // block 1 (rows 128..R-1) into the shared-memory A tile (warps 8-11).
    auto q_row = [&](int n) {
        return reinterpret_cast<const uint4 *>(
            a.q + ((int64_t)(node0 + n / G) * a.n_heads_q + g * G + n % G) * kD);
    };
    if (warp == 3) {
        // producer: below, without the query barrier
    } else if (warp >= 4 && warp < 8) {
        const int q = warp & 3;
        const int n = q * rq0 + lane;
        const bool valid = lane < rq0 && n < R0;
        uint32_t qv[64];
        if (valid) {
            const uint4 *src = q_row(t128_row_of(n, R));
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const uint4 u = __ldg(src + c);
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
        named_bar_arrive(kBarQLoads, kQLoadThreads);
        const uint32_t qa = tmem + ((uint32_t)(q * 32) << 16) + kQCol;
        uint32_t (&q0)[32] = *reinterpret_cast<uint32_t (*)[32]>(&qv[0]);
        uint32_t (&q1)[32] = *reinterpret_cast<uint32_t (*)[32]>(&qv[32]);
        tmem_st32(qa, q0);
        tmem_st32(qa + 32, q1);
        tmem_st_wait();
    } else if (NB == 2 && warp >= 8 && warp < 12) {
        const int q = warp & 3;
        const int m = q * 32 + lane;  // A-tile row = TMEM lane of S_1
        const int n = kBlockM + q * rq1 + lane;
        const bool valid = lane < rq1 && n < R;
        const uint4 *src = valid ? q_row(t128_row_of(n, R)) : nullptr;
        // every load in flight before the first store (the stores could
        // alias the loads as far as the compiler knows)
        uint4 u[16];
#pragma unroll
        for (int c = 0; c < 16; ++c)
            u[c] = valid ? __ldg(src + c) : make_uint4(0u, 0u, 0u, 0u);
        named_bar_arrive(kBarQLoads, kQLoadThreads);
#pragma unroll
        for (int c = 0; c < 16; ++c)
            *reinterpret_cast<uint4 *>(sQ1 + (c >> 3) * kBoxBytes + (m >> 3) * 1024 +
                                       (m & 7) * 128 + (((c & 7) ^ (m & 7)) << 4)) = u[c];
        fence_proxy_async_smem();
    } else if (warp >= 8 && warp < 12) {
        named_bar_arrive(kBarQLoads, kQLoadThreads);   // one block: no rows to load
    }
    if (warp != 3) {
        tc_fence_before();
        named_bar_sync(kBarQuery, kThreads - 32);
        tc_fence_after();
    }

    if (warp == 3) {
        // ------------------------------------ TMA producer (K one tile ahead)
        named_bar_sync(kBarQLoads, kQLoadThreads);
        if (lane == 0) {
            int nk = 0, nv = 0;   // tiles issued so far
            // step i issues K(i), then V(i - 1): K is consumed a whole softmax
            // pass before V, and each load waits only for its own ring slot
            for (int i = 0; i <= n_tiles; ++i) {
                bool ok = true;
#pragma unroll 1
                for (int which = 0; which < 2 && ok; ++which) {
                    const bool is_k = which == 0;
                    const int t = is_k ? i : i - 1;
                    if (t < 0 || t >= n_tiles)
                        continue;
                    const int ns = is_k ? SK : SV;
                    const int s = t % ns;
                    uint64_t *full = is_k ? bar->full_k : bar->full_v;
                    uint64_t *empty = is_k ? bar->empty_k : bar->empty_v;
                    if (t >= ns &&
                        !wait_bounded(smem_addr(&empty[s]), ((t / ns) & 1) ^ 1, abort, hdr)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_addr(&full[s]);
                    mbar_arrive_expect_tx(fb, kStageBytes);
                    const uint32_t dst = smem_addr((is_k ? sK : sV) + s * kStageBytes);
                    const void *tmap = is_k ? static_cast<const void *>(&tmap_k)
                                            : static_cast<const void *>(&tmap_v);
                    const int pos0 = (t_begin + t) * kTileN;
                    tma_load_3d(dst, tmap, 0, pos0, g, fb);
                    tma_load_3d(dst + kBoxBytes, tmap, 64, pos0, g, fb);
                    if (is_k)
                        nk = t + 1;
                    else
                        nv = t + 1;
                }
                if (!ok)
                    break;
            }
            if (*abort) {
                // let our own copies land before the CTA exits
                for (int t = max(0, nk - SK); t < nk; ++t)
                    wait_drain(smem_addr(&bar->full_k[t % SK]), (t / SK) & 1);
                for (int t = max(0, nv - SV); t < nv; ++t)
                    wait_drain(smem_addr(&bar->full_v[t % SV]), (t / SV) & 1);
            }
        }
    } else if (warp == 0) {
        // --------------------------- root node's scores out of S_0 (lanes 0..G-1)
        if (rs_warp0) {
            // one block only; one 16x256b load of lanes 0..15, the shape the softmax warps
            // use: thread t holds lane t/4 (and 8 + t/4) at columns
            // 8j + 2(t%4) + {0, 1}, so threads 0..4G-1 hold the G root rows
            const int r = lane >> 2;          // root row of this thread (lanes 0..7)
            const bool mine = r < G;
            const int c0 = 2 * (lane & 3);
            float *dst_row = a.root_scores + (size_t)(g * G + (mine ? r : 0)) * a.n_ctx;
            const bool vec = ((reinterpret_cast<uintptr_t>(a.root_scores) | (uintptr_t)a.n_ctx * 4) &
                              7) == 0;
            for (int t = 0; t < n_tiles; ++t) {
                if (!warp_wait_bounded(smem_addr(&bar->s_full[0]), t & 1, abort, hdr))
                    break;
                tc_fence_after();
                const int pos0 = (t_begin + t) * kTileN;
                uint32_t rr[64];
                if (pos0 < a.n_ctx)
                    tmem_ld16x256_x16(tmem + kSCol, rr);
                // S_0 is read: QK of the next tile may overwrite it
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(smem_addr(&bar->s_free[0]));
                if (pos0 >= a.n_ctx || !mine)
                    continue;   // a tile of the tree tail only, or not a root lane
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) {
                    const int p = pos0 + 8 * jj + c0;
                    const float x0 = __uint_as_float(rr[4 * jj]) * a.scale_log2;
                    const float x1 = __uint_as_float(rr[4 * jj + 1]) * a.scale_log2;
                    if (vec && p + 1 < a.n_ctx) {
                        *reinterpret_cast<float2 *>(dst_row + p) = make_float2(x0, x1);
                    } else {
                        if (p < a.n_ctx)
                            dst_row[p] = x0;
                        if (p + 1 < a.n_ctx)
                            dst_row[p + 1] = x1;
                    }
                }
            }
        }
    } else if (warp == 1 || warp == 2) {
        // --------------------------------------------- MMA issuers: QK, PV
        if (lane == 0) {
            constexpr uint64_t kStageStep = kStageBytes >> 4;
            if (warp == 1) {
                const uint32_t idesc = idesc_bf16(kBlockM, kTileN, 0, 0);
                const uint64_t kd0 = sdesc_sw128(smem_addr(sK), 16, 1024);
                const uint64_t qd0 = sdesc_sw128(smem_addr(sQ1), 16, 1024);
                for (int t = 0; t < n_tiles; ++t) {
                    const int s = t % SK;
                    if (!wait_bounded(smem_addr(&bar->full_k[s]), (t / SK) & 1, abort, hdr))
                        break;
                    // QK(t) enters the tensor queue after PV(t-2): the softmax
                    // warps wait for PV(t-2) before writing P^T(t-1), while
                    // S(t) is only read after they finish tile t-1.  PV(t)
                    // needs S(t), so slot t & 1 has one open phase here.
                    if (t >= 2 && !wait_bounded(smem_addr(&bar->pv_issued[t & 1]),
                                                ((t - 2) >> 1) & 1, abort, hdr))
                        break;
                    const uint64_t kd = kd0 + (uint64_t)s * kStageStep;
                    bool ok = true;
                    for (int b = 0; b < NB; ++b) {
                        // S_b is reused: its softmax warps must hold S_b(t-1)
                        if (t > 0 &&
                            !wait_bounded(smem_addr(&bar->s_free[b]), (t - 1) & 1, abort, hdr)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t d_col = tmem + kSCol + 128 * b;
                        if (b == 0) {
                            mma_ts_c<0>(d_col, tmem + kQCol, kd, idesc);
#pragma unroll
                            for (int kk = 1; kk < kD / 16; ++kk)
                                mma_ts_c<1>(d_col, tmem + kQCol + kk * 8,
                                            kd + (((kk >> 2) * kBoxBytes + (kk & 3) * 32) >> 4),
                                            idesc);
                        } else {
                            mma_ss_c<0>(d_col, qd0, kd, idesc);
#pragma unroll
                            for (int kk = 1; kk < kD / 16; ++kk) {
                                const uint64_t off = ((kk >> 2) * kBoxBytes + (kk & 3) * 32) >> 4;
                                mma_ss_c<1>(d_col, qd0 + off, kd + off, idesc);
                            }
                        }
                        mma_commit(smem_addr(&bar->s_full[b]));
                    }
                    if (!ok)
                        break;
                    mma_commit(smem_addr(&bar->empty_k[s]));
                }
            } else {
                const uint32_t idesc = idesc_bf16(kD, r_pad, 1, 0);
                const uint64_t vd0 = sdesc_sw128(smem_addr(sV), kBoxBytes, 1024);
                const uint64_t pd0 = sdesc_sw128(smem_addr(sP), 16, 1024);
                const uint32_t p_half = (uint32_t)r_pad * 128;
                for (int t = 0; t < n_tiles; ++t) {
                    const int s = t % SV;
                    if (!wait_bounded(smem_addr(&bar->full_v[s]), (t / SV) & 1, abort, hdr) ||
                        !wait_bounded(smem_addr(&bar->sm_done), t & 1, abort, hdr))
                        break;
                    tc_fence_after();
                    const uint64_t vd = vd0 + (uint64_t)s * kStageStep;
                    if (t == 0)
                        mma_ss_c<0>(tmem, vd, pd0, idesc);
                    else
                        mma_ss_c<1>(tmem, vd, pd0, idesc);
#pragma unroll
                    for (int kk = 1; kk < kTileN / 16; ++kk)
                        mma_ss_c<1>(tmem, vd + ((kk * 2048) >> 4),
                                    pd0 + (((kk >> 2) * p_half + (kk & 3) * 32) >> 4), idesc);
                    mma_commit(smem_addr(&bar->pv_done));
                    if (t == n_tiles - 1)
                        mma_commit(smem_addr(&bar->o_final));
                    mma_commit(smem_addr(&bar->empty_v[s]));
                    mbar_arrive(smem_addr(&bar->pv_issued[t & 1]));
                }
            }
            // every MMA this thread issued has finished before TMEM is released
            const int dn = warp - 1;
            mma_commit(smem_addr(&bar->drain[dn]));
            wait_drain(smem_addr(&bar->drain[dn]), 0);
        }
    } else if (warp >= 4 && (warp - 4) / 4 < U) {
        // ---------------------------------------------------------- softmax
        const int q = warp & 3, j = (warp - 4) >> 2;
        const int b = j < u0 ? 0 : 1;
        const int lb = 16 * (b == 0 ? j : j - u0);  // unit's first lane in the quarter
        const int Rb = b == 0 ? R0 : R1, rqb = b == 0 ? rq0 : rq1;
        const int iA = lb + (lane >> 2), iB = iA + 8;
        const bool vA = iA < rqb && q * rqb + iA < Rb;
        const bool vB = iB < rqb && q * rqb + iB < Rb;
        const bool hasA = __any_sync(0xffffffffu, vA), hasB = __any_sync(0xffffffffu, vB);
        const int nA = kBlockM * b + q * rqb + iA, nB = nA + 8;
        const uint32_t s_addr = tmem + ((uint32_t)(32 * q + lb) << 16) + kSCol + 128 * b;
        const uint32_t o_lane = (uint32_t)(32 * q) << 16;
        const int c0 = 2 * (lane & 3);
        // P^T rows of this unit: half A is nbase + 0..7, half B nbase + 8..15;
        // the valid ones are those inside the quarter's run and the block
        const int nbase = kBlockM * b + q * rqb + lb;
        const int nvA = max(0, min(8, min(rqb - lb, Rb - q * rqb - lb)));
        const int nvB = max(0, min(8, min(rqb - lb - 8, Rb - q * rqb - lb - 8)));
        const uint32_t p_addr = smem_addr(sP);
        const uint32_t p_scratch = p_addr + (uint32_t)r_pad * 256;
        float mA = -INFINITY, mB = -INFINITY, lA = 0.f, lB = 0.f, qA = 0.f, qB = 0.f;
        // root rows (rows 0..G-1) held by this thread and this warp (block 1
        // only); the first lane of a row's quad copies its staged scores out
        const bool rootA = b == 1 && vA && t128_row_of(nA, R) < G;
        const bool rootB = b == 1 && vB && t128_row_of(nB, R) < G;
        const bool rs_warp = t128_rs_block1(a, T) && __any_sync(0xffffffffu, rootA || rootB);
        const bool rs_issue = rs_bytes != 0 && (lane & 3) == 0 && (rootA || rootB);
        bool ok = true;
        for (int t = 0; t < n_tiles; ++t) {
            if (!warp_wait_bounded(smem_addr(&bar->s_full[b]), t & 1, abort, hdr)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t r[64];
            tmem_ld16x256_x16(s_addr, r);
            // S is in registers: QK of the next tile may overwrite it
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(smem_addr(&bar->s_free[b]));
            // raw scores; the scale (> 0) is applied inside the exponent
            const int pos0 = (t_begin + t) * kTileN;
            // the root node's rows leave their context scores, base 2, for the
            // importance select
            if (rs_warp && pos0 < a.n_ctx) {
                if (rs_bytes != 0) {
                    // staged in shared memory (one buffer per tile parity) and
                    // written out by bulk copies, so that no global store sits
                    // ahead of this warp's barrier arrivals
                    const uint32_t buf =
                        smem_addr(base + lay.rs_off) + (uint32_t)((t & 1) * G * kTileN * 4);
                    if (rs_issue)
                        bulk_wait_read<1>();   // the copy out of this buffer two tiles ago
                    __syncwarp();
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        if (h ? rootB : rootA) {
                            const uint32_t row = buf + (uint32_t)(t128_row_of(h ? nB : nA, R) *
                                                                      kTileN * 4 +
                                                                  c0 * 4);
#pragma unroll
                            for (int jj = 0; jj < 16; ++jj)
                                st_shared_v2(row + 32 * jj,
                                             __float_as_uint(__uint_as_float(r[4 * jj + 2 * h]) *
                                                             a.scale_log2),
                                             __float_as_uint(__uint_as_float(r[4 * jj + 2 * h + 1]) *
                                                             a.scale_log2));
                        }
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (rs_issue) {
                        const uint32_t bytes = (uint32_t)min(kTileN, a.n_ctx - pos0) * 4;
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int m = t128_row_of(h ? nB : nA, R);
                            if (h ? rootB : rootA)
                                bulk_store(a.root_scores + (size_t)(g * G + m) * a.n_ctx + pos0,
                                           buf + (uint32_t)(m * kTileN * 4), bytes);
                        }
                        bulk_commit();
                    }
                } else {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        if (h ? rootB : rootA) {
                            float *dst = a.root_scores +
                                         (size_t)(g * G + t128_row_of(h ? nB : nA, R)) * a.n_ctx;
#pragma unroll
                            for (int jj = 0; jj < 16; ++jj)
#pragma unroll
                                for (int e = 0; e < 2; ++e) {
                                    const int pos = pos0 + 8 * jj + c0 + e;
                                    if (pos < a.n_ctx)
                                        dst[pos] =
                                            __uint_as_float(r[4 * jj + 2 * h + e]) * a.scale_log2;
                                }
                        }
                    }
                }
            }
            if (pos0 + kTileN > a.n_ctx) {
                // visibility of this thread's 32 positions (entry k = 2 jj + e
                // is position pos0 + 8 jj + c0 + e) for its two rows
                const unsigned long long ancA = masks.anc[node0 + (vA ? t128_row_of(nA, R) / G : 0)];
                const unsigned long long ancB = masks.anc[node0 + (vB ? t128_row_of(nB, R) / G : 0)];
                uint32_t visA = 0u, visB = 0u;
#pragma unroll 1
                for (int k = 0; k < 32; ++k) {
                    const int pos = pos0 + 8 * (k >> 1) + c0 + (k & 1);
                    const int tp = pos - a.n_ctx;
                    const bool in = pos < total;
                    visA |= (uint32_t)(in && (tp < 0 || ((ancA >> tp) & 1ull))) << k;
                    visB |= (uint32_t)(in && (tp < 0 || ((ancB >> tp) & 1ull))) << k;
                }
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                    if (!((visA >> k) & 1u))
                        r[4 * (k >> 1) + (k & 1)] = __float_as_uint(-INFINITY);
                    if (!((visB >> k) & 1u))
                        r[4 * (k >> 1) + 2 + (k & 1)] = __float_as_uint(-INFINITY);
                }
            }
            // a row that has seen nothing yet takes this tile's max as its
            // reference (its O^T column and l are still zero); afterwards
            // the maxima are not needed
            if (__any_sync(0xffffffffu, mA == -INFINITY || mB == -INFINITY)) {
                const float xA = row_max(r, 0) * a.scale_log2;
                const float xB = row_max(r, 2) * a.scale_log2;
                float yA = fmaxf(xA, __shfl_xor_sync(0xffffffffu, xA, 1));
                float yB = fmaxf(xB, __shfl_xor_sync(0xffffffffu, xB, 1));
                yA = fmaxf(yA, __shfl_xor_sync(0xffffffffu, yA, 2));
                yB = fmaxf(yB, __shfl_xor_sync(0xffffffffu, yB, 2));
                if (mA == -INFINITY)
                    mA = yA;
                if (mB == -INFINITY)
                    mB = yB;
            }

            uint32_t pA[16], pB[16];
            {
                const float nmA = mA == -INFINITY ? 0.f : -mA;
                const float nmB = mB == -INFINITY ? 0.f : -mB;
                if (hasB)
                    exp_pack_rows<true>(r, a.scale_log2, nmA, nmB, pA, pB, lA, lB, qA, qB);
                else if (hasA)
                    exp_pack_rows<false>(r, a.scale_log2, nmA, nmB, pA, pB, lA, lB, qA, qB);
            }
            // P^T is free once PV(t-1) is done.  This warp saw PV(t-2) done
            // before writing P^T(t-1), and PV(t) waits for this warp, so
            // pv_done has one open phase here.
            if (t > 0 &&
                !warp_wait_bounded(smem_addr(&bar->pv_done), (t - 1) & 1, abort, hdr)) {
                ok = false;
                break;
            }
            if (hasA)
                store_p_half(p_addr, p_scratch, nbase, nvA, r_pad, lane, pA);
            if (hasB)
                store_p_half(p_addr, p_scratch, nbase + 8, nvB, r_pad, lane, pB);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(smem_addr(&bar->sm_done));
        }
        if (rs_issue)
            bulk_wait_all();   // shared memory must outlive the copies out of it
        // ---- (m, l) of each row (four threads' partial sums), then O^T
#pragma unroll
        for (int o = 1; o <= 2; o <<= 1) {
            lA += __shfl_xor_sync(0xffffffffu, lA, o);
            lB += __shfl_xor_sync(0xffffffffu, lB, o);
            qA += __shfl_xor_sync(0xffffffffu, qA, o);
            qB += __shfl_xor_sync(0xffffffffu, qB, o);
        }
        // every weight of a row is at most its sum: a sum past 2^63 (or not a
        // number) flags the split for the exact recompute
        const bool over = (vA && !(lA <= kMaxRowSum)) || (vB && !(lB <= kMaxRowSum));
        if (__any_sync(0xffffffffu, over) && lane == 0)
            bar->overflow = 1;
        const int rows_all = a.n_tree * a.n_heads_q;
        float *ws_o =
            reinterpret_cast<float *>(reinterpret_cast<char *>(a.workspace) + kHeaderBytes);
        float *ws_ml = ws_o + (size_t)n_split * rows_all * kD;
        // P^T row n -> output row of the head group
        auto orow_of = [&](int n) {
            const int m = t128_row_of(n, R);
            return (node0 + m / G) * a.n_heads_q + g * G + m % G;
        };
        if (ok && (lane & 3) == 0) {
            if (vA)
                *reinterpret_cast<float4 *>(ws_ml + ((size_t)split * rows_all + orow_of(nA)) * 4) =
                    make_float4(mA, lA, qA, 0.f);
            if (vB)
                *reinterpret_cast<float4 *>(ws_ml + ((size_t)split * rows_all + orow_of(nB)) * 4) =
                    make_float4(mB, lB, qB, 0.f);
        }
        // O^T out of TMEM.  Once the last PV is done the K/V ring is free:
        // the rows are staged there in output order (row m = node * G + the
        // head's index in the group, 512 bytes each), so that each node's G
        // rows leave as one contiguous bulk copy instead of many small
        // stores.
        const bool have_o = ok && warp_wait_bounded(smem_addr(&bar->o_final), 0, abort, hdr);
        const int d = 32 * q + lane;
        if (have_o) {
            tc_fence_after();
            const bool staged = lay.o_staged;
            for (int c = 32 * j; c < r_pad; c += 32 * U) {
                uint32_t o[32];
                tmem_ld32(tmem + o_lane + c, o);
                const int nv = min(32, R - c);   // query rows among P^T rows c .. c+31
                if (staged) {
                    // a 32-row chunk lies inside one block, where the output
                    // row is the P^T row plus a constant
                    float *dst = reinterpret_cast<float *>(sK) + (size_t)t128_row_of(c, R) * kD + d;
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj)
                        if (jj < nv)
                            dst[jj * kD] = __uint_as_float(o[jj]);
                } else {
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj)
                        if (jj < nv)
                            ws_o[((size_t)split * rows_all + orow_of(c + jj)) * kD + d] =
                                __uint_as_float(o[jj]);
                }
            }
        }
        if (lay.o_staged) {
            fence_proxy_async_smem();
            named_bar_sync(kBarOut, 128 * U);   // every softmax warp, whatever its path
            // a warp that gave up set the abort flag before this barrier
            if (!*abort && lane == 0) {
                const int sw = warp - 4;   // 0 .. 4U-1
                for (int node = sw; node < T; node += 4 * U)
                    bulk_store(ws_o + ((size_t)split * rows_all + (size_t)(node0 + node) * a.n_heads_q + g * G) * kD,
                               smem_addr(sK) + (uint32_t)(node * G * kD * 4), (uint32_t)(G * kD * 4));
                bulk_commit();
                bulk_wait_all();   // the ring must outlive the copies out of it
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    if (threadIdx.x == 0)
        flags[(split * a.n_heads_kv + g) * gridDim.z + blockIdx.z] = bar->overflow;
}

// One split's partial (m, l, acc) of one query row, recomputed exactly in
// fp32 from K and V by an online softmax over the split's visible
// positions.  One warp; lane holds head dims 4 lane .. 4 lane + 3.  Used
// only for splits whose flag says the kernel's fixed reference max ran out
// of headroom, and for the splits that carry the weight of a row whose
// weight sits on too few positions for one bf16 rounding of P.
__device__ void split_partial_exact(const AttnArgs &a, unsigned long long anc, int g,
                                    const float (&q4)[4], int p0, int p1, float &m, float &l,
                                    float (&acc)[4])
{
    constexpr int kU = 8;   // positions per step: their loads and reductions overlap
    const int lane = threadIdx.x & 31;
    const __nv_bfloat16 *kh = a.k + (size_t)g * a.kv_cap * kD + 4 * lane;
    const __nv_bfloat16 *vh = a.v + (size_t)g * a.kv_cap * kD + 4 * lane;
    m = -INFINITY;
    l = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e)
        acc[e] = 0.f;
    for (int pos0 = p0; pos0 < p1; pos0 += kU) {
        float sc[kU];
        bool seen[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int pos = pos0 + u;
            const int tp = pos - a.n_ctx;
            seen[u] = pos < p1 && (tp < 0 || ((anc >> tp) & 1ull));
            const uint2 kb = seen[u] ? *reinterpret_cast<const uint2 *>(kh + (size_t)pos * kD)
                                     : make_uint2(0u, 0u);
            const float2 k01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&kb.x));
            const float2 k23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&kb.y));
            sc[u] = q4[0] * k01.x + q4[1] * k01.y + q4[2] * k23.x + q4[3] * k23.y;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
#pragma unroll
            for (int u = 0; u < kU; ++u)
                sc[u] += __shfl_xor_sync(0xffffffffu, sc[u], o);
        float mx = -INFINITY;
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            sc[u] = seen[u] ? sc[u] * a.scale_log2 : -INFINITY;
            mx = fmaxf(mx, sc[u]);
        }
        if (mx == -INFINITY)
            continue;
        if (mx > m) {
            const float f = m == -INFINITY ? 0.f : exp2f(m - mx);
            l *= f;
#pragma unroll
            for (int e = 0; e < 4; ++e)
                acc[e] *= f;
            m = mx;
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            if (!seen[u])
                continue;
            const float pw = exp2f(sc[u] - m);
            const uint2 vb = *reinterpret_cast<const uint2 *>(vh + (size_t)(pos0 + u) * kD);
            const float2 v01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&vb.x));
            const float2 v23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&vb.y));
            l += pw;
            acc[0] += pw * v01.x;
            acc[1] += pw * v01.y;
            acc[2] += pw * v23.x;
            acc[3] += pw * v23.y;
        }
    }
}

// One warp per output row: out = sum_s 2^(m_s - M) acc_s / sum_s 2^(m_s - M) l_s
// over the splits' partials.  Recomputed exactly instead of read: splits
// flagged for overflow, and, on a row whose effective number of positions
// may be below kNeffMin (L^2 < kNeffMin * sum_s c_s^2 q_s with c_s =
// 2^(m_s - M)), every split s whose c_s^2 q_s is above L^2 / (kNeffMin *
// n_split) -- the remaining splits then add up to a bound of at least
// kNeffMin on their own.
__global__ void __launch_bounds__(256)
attn_t128_combine_kernel(AttnArgs a, TreeMasks masks, int n_split, int split_positions,
                         const int32_t *__restrict__ flags, int n_flag_groups)
{
    const int rows_all = a.n_tree * a.n_heads_q;
    const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    // launched early (programmatic dependent launch): the split partials
    // are complete only once the split grid has finished
    grid_dependency_wait();
    if (row >= rows_all)
        return;
    const int head = row % a.n_heads_q, node = row / a.n_heads_q;
    const int g = head / (a.n_heads_q / a.n_heads_kv);
    const float *ws_o =
        reinterpret_cast<const float *>(reinterpret_cast<const char *>(a.workspace) + kHeaderBytes);
    const float *ws_ml = ws_o + (size_t)n_split * rows_all * kD;
    auto mlq_of = [&](int s) {
        return __ldcg(reinterpret_cast<const float4 *>(ws_ml + ((size_t)s * rows_all + row) * 4));
    };

    // One round trip for the common case (at most kFastSplits splits): lane
    // s reads split s's (m, l, q) and flag while every lane also reads its
    // four columns of every split's acc, all loads in flight together.
    auto flagged = [&](int s) {
        if (flags == nullptr)
            return false;
        bool f = false;
        for (int z = 0; z < n_flag_groups; ++z)
            f = f || flags[(s * a.n_heads_kv + g) * n_flag_groups + z] != 0;
        return f;
    };
    constexpr int kFastSplits = 24;
    const bool fast = n_split <= kFastSplits;
    float4 xs[kFastSplits];
    float4 my = make_float4(-INFINITY, 0.f, 0.f, 0.f);
    bool my_f = false;
    if (fast) {
        if (lane < n_split) {
            my = mlq_of(lane);
            my_f = flagged(lane);
        }
#pragma unroll
        for (int u = 0; u < kFastSplits; ++u)
            xs[u] = u < n_split ? __ldcg(reinterpret_cast<const float4 *>(
                                      ws_o + ((size_t)u * rows_all + row) * kD + 4 * lane))
                                : make_float4(0.f, 0.f, 0.f, 0.f);
    }

    // M, and L and the bound's denominator, over the splits that are not
    // flagged
    bool any = false;
    float M = -INFINITY;
    if (fast) {
        any = my_f;
        if (!my_f)
            M = my.x;
    } else {
        for (int s = lane; s < n_split; s += 32) {
            const bool f = flagged(s);
            any |= f;
            if (!f)
                M = fmaxf(M, mlq_of(s).x);
        }
    }
    any = __any_sync(0xffffffffu, any);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    // L^2 and the q sums reach 2^126 times the splits squared: the count is
    // formed in fp64
    double Lp = 0.0, Qp = 0.0;
    if (M != -INFINITY) {
        if (fast) {
            if (!my_f && my.x != -INFINITY) {
                const double c = (double)exp2f(my.x - M);
                Lp = c * (double)my.y;
                Qp = c * c * (double)my.z;
            }
        } else {
            for (int s = lane; s < n_split; s += 32) {
                if (flagged(s))
                    continue;
                const float4 x = mlq_of(s);
                const double c = x.x == -INFINITY ? 0.0 : (double)exp2f(x.x - M);
                Lp += c * (double)x.y;
                Qp += c * c * (double)x.z;
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        Lp += __shfl_xor_sync(0xffffffffu, Lp, o);
        Qp += __shfl_xor_sync(0xffffffffu, Qp, o);
    }
    const bool peaked = Lp * Lp < (double)kNeffMin * Qp;   // uniform across the warp
    const double heavy = Lp * Lp / ((double)kNeffMin * n_split);

    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    float L = 0.f;
    if (!any && !peaked && fast) {
        // every partial is used as it is: lane s's weight 2^(m_s - M) and
        // its weighted l, passed to every lane
        const float w_my = my.x == -INFINITY ? 0.f : exp2f(my.x - M);
        const float wl_my = w_my * my.y;
#pragma unroll
        for (int u = 0; u < kFastSplits; ++u) {
            if (u >= n_split)
                break;
            const float w = __shfl_sync(0xffffffffu, w_my, u);
            L += __shfl_sync(0xffffffffu, wl_my, u);
            acc[0] += w * xs[u].x;
            acc[1] += w * xs[u].y;
            acc[2] += w * xs[u].z;
            acc[3] += w * xs[u].w;
        }
    } else if (!any && !peaked) {
        // every partial is used as it is; M is known, so the splits are
        // summed in batches of kB whose loads are in flight together
        constexpr int kB = 9;
        for (int s0 = 0; s0 < n_split; s0 += kB) {
            float4 mlq[kB], x[kB];
#pragma unroll
            for (int u = 0; u < kB; ++u) {
                const int s = s0 + u;
                if (s < n_split) {
                    mlq[u] = mlq_of(s);
                    x[u] = __ldcg(reinterpret_cast<const float4 *>(
                        ws_o + ((size_t)s * rows_all + row) * kD + 4 * lane));
                } else {
                    mlq[u] = make_float4(-INFINITY, 0.f, 0.f, 0.f);
                    x[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
#pragma unroll
            for (int u = 0; u < kB; ++u) {
                const float w = mlq[u].x == -INFINITY ? 0.f : exp2f(mlq[u].x - M);
                L += w * mlq[u].y;
                acc[0] += w * x[u].x;
                acc[1] += w * x[u].y;
                acc[2] += w * x[u].z;
                acc[3] += w * x[u].w;
            }
        }
    } else {
        // fold the splits one by one into a running (Mr, L, acc), the
        // flagged and the heavy ones recomputed
        const uint2 qb = *reinterpret_cast<const uint2 *>(a.q + (size_t)row * kD + 4 * lane);
        const float2 q01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&qb.x));
        const float2 q23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&qb.y));
        const float q4[4] = {q01.x, q01.y, q23.x, q23.y};
        const int total = a.n_ctx + a.n_tree;
        float Mr = -INFINITY;
        for (int s = 0; s < n_split; ++s) {
            float ms, ls, as[4];
            const float4 x4 = mlq_of(s);
            bool exact = flagged(s);
            if (!exact && peaked && x4.x != -INFINITY) {
                const double c = (double)exp2f(x4.x - M);
                exact = c * c * (double)x4.z > heavy;
            }
            if (exact) {
                const int p0 = s * split_positions;
                const int p1 = min(p0 + split_positions, total);
                split_partial_exact(a, masks.anc[node], g, q4, p0, p1, ms, ls, as);
            } else {
                const float4 x = __ldcg(reinterpret_cast<const float4 *>(
                    ws_o + ((size_t)s * rows_all + row) * kD + 4 * lane));
                ms = x4.x;
                ls = x4.y;
                as[0] = x.x;
                as[1] = x.y;
                as[2] = x.z;
                as[3] = x.w;
            }
            if (ms == -INFINITY)
                continue;
            const float Mn = fmaxf(Mr, ms);
            const float fa = Mr == -INFINITY ? 0.f : exp2f(Mr - Mn);
            const float fb = exp2f(ms - Mn);
            L = L * fa + ls * fb;
#pragma unroll
            for (int e = 0; e < 4; ++e)
                acc[e] = acc[e] * fa + as[e] * fb;
            Mr = Mn;
        }
    }
    const float inv = 1.f / L;
    *reinterpret_cast<float4 *>(a.out + (size_t)row * kD + 4 * lane) =
        make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
}

// Split partials (acc fp32 [n_split, T*Hq, D], then (m, l, q, 0) fp32
// [n_split, T*Hq, 4]) after the header, then one int32 overflow flag per
// (split, KV head).

size_t flags_offset(int n_split, int n_heads_q, int n_tree)
{
    return kHeaderBytes + align_up(attn_exact_partial_bytes(n_split, n_heads_q, n_tree), 256);
}

}  // namespace

size_t attn_t128_workspace_bytes(int n_heads_q, int n_heads_kv, int n_ctx, int n_tree, int num_sms)
{
    const AttnPlan p = attn_t128_plan(n_heads_q, n_heads_kv, n_ctx, n_tree, num_sms);
    return flags_offset(p.n_split, n_heads_q, n_tree) +
           align_up((size_t)p.n_split * n_heads_kv * p.node_groups * sizeof(int32_t), 256);
}

bool attn_t128_eligible(int n_heads_q, int n_heads_kv, int head_dim, int n_ctx, int n_tree)
{
    // a CTA takes whole tree nodes: one node's G rows must fit one block
    const int G = n_heads_q / n_heads_kv;
    return head_dim == kD && G <= kBlockM && n_ctx >= kTcMinContext;
}

AttnPlan attn_t128_plan(int n_heads_q, int n_heads_kv, int n_ctx, int n_tree, int num_sms)
{
    AttnPlan p;
    const int G = n_heads_q / n_heads_kv;
    const int rows = G * n_tree;
    // up to kMaxRows rows in one CTA; beyond that, groups of nodes of at
    // most kBlockM rows (one 128-lane block each), one CTA per group
    p.node_groups = rows <= kMaxRows ? 1 : (rows + kBlockM - 1) / kBlockM;
    p.nodes_per_group = (n_tree + p.node_groups - 1) / p.node_groups;
    p.node_groups = (n_tree + p.nodes_per_group - 1) / p.nodes_per_group;
    const int n_tiles = (n_ctx + n_tree + kTileN - 1) / kTileN;
    int want = num_sms / (n_heads_kv * p.node_groups);
    want = want < 1 ? 1 : (want > n_tiles ? n_tiles : want);
    p.tiles_per_split = (n_tiles + want - 1) / want;
    p.n_split = (n_tiles + p.tiles_per_split - 1) / p.tiles_per_split;
    return p;
}

cudaError_t attn_t128_launch(const AttnArgs &a, const TreeMasks &masks, int num_sms,
                             cudaStream_t stream)
{
    const AttnPlan p = attn_t128_plan(a.n_heads_q, a.n_heads_kv, a.n_ctx, a.n_tree, num_sms);
    CUtensorMap mk, mv;
    const int rows = a.n_ctx + a.n_tree;
    if (!encode_kv_map(&mk, a.k, rows, a.kv_cap, a.n_heads_kv, kTileN) ||
        !encode_kv_map(&mv, a.v, rows, a.kv_cap, a.n_heads_kv, kTileN))
        return cudaErrorInvalidValue;
    // the first node group is the largest and holds the root node
    const int T0 = p.nodes_per_group;
    const Layout lay = t128_layout((a.n_heads_q / a.n_heads_kv) * T0, t128_rs_bytes(a, T0));
    static const cudaError_t attr = cudaFuncSetAttribute(
        attn_t128_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemLimit);
    if (attr != cudaSuccess)
        return attr;
    int32_t *flags = reinterpret_cast<int32_t *>(
        reinterpret_cast<char *>(a.workspace) + flags_offset(p.n_split, a.n_heads_q, a.n_tree));
    cudaError_t e;
    if (p.node_groups > 1 && p.node_groups <= 8) {
        // the node groups of one (split, head) stream the same K/V tiles: as
        // one cluster they start together on one GPC, so that the second
        // read of each tile finds it in L2
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(p.n_split, a.n_heads_kv, p.node_groups);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = lay.smem_bytes;
        cfg.stream = stream;
        cudaLaunchAttribute attr_c[1];
        attr_c[0].id = cudaLaunchAttributeClusterDimension;
        attr_c[0].val.clusterDim.x = 1;
        attr_c[0].val.clusterDim.y = 1;
        attr_c[0].val.clusterDim.z = p.node_groups;
        cfg.attrs = attr_c;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, attn_t128_kernel, mk, mv, a, masks, p.tiles_per_split,
                               p.n_split, p.nodes_per_group, flags);
        if (e == cudaSuccess)
            e = cudaGetLastError();
    } else {
        attn_t128_kernel<<<dim3(p.n_split, a.n_heads_kv, p.node_groups), kThreads, lay.smem_bytes,
                           stream>>>(mk, mv, a, masks, p.tiles_per_split, p.n_split,
                                     p.nodes_per_group, flags);
        e = cudaGetLastError();
    }
    if (e != cudaSuccess)
        return e;
    count_launches(1);
    return attn_exact_combine_launch(a, masks, p.n_split, p.tiles_per_split * kTileN, flags,
                                     p.node_groups, stream);
}

bool attn_t128_leaves_root_scores(const AttnArgs &a)
{
    const AttnPlan p = attn_t128_plan(a.n_heads_q, a.n_heads_kv, a.n_ctx, a.n_tree, 148);
    return t128_rs_warp0(a, p.nodes_per_group) || t128_rs_block1(a, p.nodes_per_group);
}

size_t attn_exact_partial_bytes(int n_split, int n_heads_q, int n_tree)
{
    return (size_t)n_split * n_tree * n_heads_q * (kD + 4) * sizeof(float);
}

cudaError_t attn_exact_combine_launch(const AttnArgs &a, const TreeMasks &masks, int n_split,
                                      int split_positions, const int32_t *flags,
                                      int n_flag_groups, cudaStream_t stream)
{
    const int rows_all = a.n_tree * a.n_heads_q;
    return launch_pdl(attn_t128_combine_kernel, dim3((rows_all + 7) / 8), dim3(256), 0, stream, a,
                      masks, n_split, split_positions, flags, n_flag_groups);
}

}  // namespace ts
