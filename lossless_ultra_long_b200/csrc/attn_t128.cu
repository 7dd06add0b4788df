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
// CTA = (split, KV head, node group), 16 warps, one CTA per SM:
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
// anything (that tile's max rounded up to an integer, in log2 units), and
// never moves, so the softmax warps need no per-tile agreement with each
// other and no per-tile maximum at all.  Being an integer, it scales every
// weight by an exact power of two: the bf16-rounded weight of a position is
// almost always the same whichever split streams it (the fp32 exponent
// argument, formed against the split's reference, can round across a bf16
// boundary the other way), so the run-time hand-out of tiles to splits
// moves results by fp32 summation order and such rare flips (~1e-4).  fp32 has room
// for it: a row's weights are at most its sum l, and while l <= 2^63 the
// accumulated O^T stays below 2^63 * max|V|, far from overflow (a score
// rise of about 44 nats inside one split would be needed to exceed it).  A
// split in which some row's l ends above 2^63 (or not a number) raises a
// flag; the combine then recomputes that split's partial for the affected
// head exactly (fp32, online softmax on CUDA cores) instead of reading it.
//
// Work split: n_split CTAs per (KV head, node group), one per SM.  Each
// starts on its own KV tile and then takes the next untaken tile of its
// (head, group) from a counter in the workspace, so that splits which HBM
// serves faster take more tiles and all end together (a fixed cut left the
// slowest split several microseconds behind the mean).  An owner map
// records which split streamed each tile.  Each split leaves an
// unnormalised partial (acc, m, l, q) and its flag, counts itself in, and
// once all splits of its (head, group) have arrived (the launch is
// cooperative, so they are all resident) folds every n_split-th output row
// of the group; no second kernel runs.
//
// P enters the PV product as one bf16 value while l sums the fp32 weights
// (as FlashAttention kernels do), so a row's output is sum bf16(p) v /
// sum p: every weight perturbed by at most one bf16 rounding (relative
// 2^-8), the normalisation by none.  Spread over many positions those
// perturbations average out (the error falls like rms|v| / sqrt of the
// effective number of positions); on a row whose weight sits on a handful
// of positions they do not.  The kernel therefore also keeps q, the sum of
// the squared weights, so that l^2 / q is the row's effective number of
// positions.  The combine recomputes exactly (fp32, CUDA cores)
// the splits that carry the weight of any row whose count over all splits
// is below kNeffMin.
//
// Every wait is bounded (about a second): on expiry the kernel records
// TS_ERR_TIMEOUT in the workspace status word, all roles leave their loops,
// and TMEM is freed before the CTA exits.
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
// 2^-8 / sqrt(3) * rms|v| / sqrt(n); at n = 64 and rms|v| ~ 1 (bf16
// N(0,1) values) that is 2.8e-4, so even the largest of many such errors
// stays inside 2e-3.
constexpr float kNeffMin = 64.f;
constexpr size_t kSmemLimit = 232448;        // dynamic shared memory per CTA
static_assert(kBlockM % 32 == 0, "a 32-column O^T chunk lies inside one query block");
constexpr int kBarQuery = 1;                 // named barrier: query rows in place
constexpr int kBarOut = 2;                   // named barrier: O^T staged in shared memory
constexpr int kBarQLoads = 3;                // named barrier: the query loads are issued
constexpr int kQLoadThreads = 32 * 9;        // warps 4-11 arrive, the producer warp waits
constexpr int kTileRing = 16;                // entries of the tile-index ring (> K/V lead)

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
    // tile index of the CTA's t-th tile at [t % kTileRing], -1 after its
    // last: written by the producer before the arrival on full_k of slot
    // t, read by every role after its own wait for tile t
    volatile int32_t tile_of[kTileRing];
    uint32_t tmem_base;
    uint32_t abort;
    int32_t overflow;     // some row exceeded its reference max by the headroom
};

struct Aux {
    Bars bar;
    unsigned long long anc[TS_MAX_TREE];   // the tree's ancestor masks, read on the tail tiles
};
constexpr size_t kAuxBytes = (sizeof(Aux) + 1023) / 1024 * 1024;

struct Layout {
    int r_pad;  // rows rounded up to 16: N of the PV product
    int stages_k, stages_v;
    bool o_staged;  // the freed K/V ring holds every O row (fp32) for the write-out
    size_t q1_off, p_off, k_off, v_off, aux_off, smem_bytes;
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

// Whether warp 0 reads the root node's scores out of TMEM: they are rows
// 0..G-1, which sit in the first lane-quarter run of the last block (block
// 0 alone, or block 1: rows 0..rq_b-1 are TMEM lanes 0..rq_b-1), so the G
// root rows are lanes 0..G-1, inside the first 16 lanes when G <= 8 and
// G <= rq_b.  Warp 0 can read lane quarter 0, and is otherwise idle.
__host__ __device__ inline bool t128_rs_warp0(const AttnArgs &a, int T)
{
    const int G = a.n_heads_q / a.n_heads_kv;
    const int R = G * T;
    const int rq = R > kBlockM ? (R - kBlockM + 3) / 4 : t128_rq0(R);
    return a.root_scores != nullptr && G <= 8 && G <= rq;
}

__host__ __device__ inline Layout t128_layout(int rows)
{
    Layout L;
    L.r_pad = (rows + 15) / 16 * 16;
    L.q1_off = 0;
    L.p_off = rows > kBlockM ? kQ1Bytes : 0;
    // P^T: positions 0-63 then 64-127, each r_pad rows of 128 bytes; then
    // 1 KB that rows past the query rows are written to
    L.k_off = L.p_off + (size_t)L.r_pad * 256 + 1024;
    const size_t fixed = 1024 + L.k_off + kAuxBytes;
    int stages = (int)((kSmemLimit - fixed) / kStageBytes);
    stages = stages > 2 * kMaxStages ? 2 * kMaxStages : stages;
    L.stages_v = 2;
    L.stages_k = stages - 2 > kMaxStages ? kMaxStages : stages - 2;
    L.v_off = L.k_off + (size_t)L.stages_k * kStageBytes;
    L.o_staged = (size_t)rows * kD * 4 <= (size_t)(L.stages_k + L.stages_v) * kStageBytes;
    L.aux_off = L.v_off + (size_t)L.stages_v * kStageBytes;
    L.smem_bytes = 1024 + L.aux_off + kAuxBytes;
    return L;
}

// Visibility of a thread's 32 positions of a tile that reaches the tree tail
// (entry k = 2 jj + e is position pos0 + 8 jj + c0 + e) for a row with
// ancestor mask anc: the tile's 128 positions as two 64-bit words (bit p
// set iff position pos0 + p is a context position, p < d = n_ctx - pos0, or
// a node of the row's root path, tree bit p - d of anc), shifted down by c0,
// then bits 8 jj + e gathered into bit 2 jj + e.
__device__ __noinline__ uint32_t t128_tail_vis(unsigned long long anc, int d, int n_tree, int c0)
{
    const unsigned long long tree = n_tree >= 64 ? anc : (anc & ((1ull << n_tree) - 1ull));
    uint32_t vis = 0u;
#pragma unroll
    for (int w = 0; w < 2; ++w) {
        const int nctx = min(max(d - 64 * w, 0), 64);
        unsigned long long m = nctx == 64 ? ~0ull : ((1ull << nctx) - 1ull);
        const int sft = 64 * w - d;   // tree bit of the word's bit 0
        if (sft >= 0) {
            if (sft < 64)
                m |= tree >> sft;
        } else if (-sft < 64) {
            m |= tree << (-sft);
        }
        // bits 8 j and 8 j + 1 (j = 0..7) of the shifted word -> bits 2 j, 2 j + 1
        unsigned long long x = (m >> c0) & 0x0303030303030303ull;
        x = (x | (x >> 6)) & 0x000F000F000F000Full;
        x = (x | (x >> 12)) & 0x000000FF000000FFull;
        x = (x | (x >> 24)) & 0xFFFFull;
        vis |= (uint32_t)x << (16 * w);
    }
    return vis;
}

// P = 2^(x * scale - m) for the 32 scores a thread holds of row A
// (registers r[4j], r[4j + 1], j = 0..15) and, when TWO, of row B
// (r[4j + 2], r[4j + 3]), packed to bf16 pairs for the PV product; adds the
// fp32 weights to lA and lB and their squares to qA and qB (summing the
// rounded bf16 values instead costs two more instructions a pair, on the
// path every tile waits for).  Both rows advance together, so each score
// register is dead once its pair is packed.
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
            const float x0 = ex2(y0), x1 = ex2(y1);
            __nv_bfloat162 hv = __floats2bfloat162_rn(x0, x1);
            const uint32_t hb = *reinterpret_cast<uint32_t *>(&hv);
            const uint64_t e2 = pack2(x0, x1);
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

// The kernel's workspace, after the 256-byte header.
struct T128Sync {
    int32_t *sync;    // [Hkv * groups][4]: tile counter, arrivals, finished combines, unused;
                      // zero when a call starts, and again when it ends
    float *part;      // split partials: acc fp32 [n_split][T*Hq][128], then
                      // (m, l, q, 0) fp32 [n_split][T*Hq][4]
    int32_t *flags;   // [n_split][Hkv * groups]: the split's reference max ran out of headroom
    uint8_t *owner;   // [Hkv * groups][n_tiles]: the split that streamed each tile
};

// Adds positions p0 .. p1-1 of one query row to a running exact partial
// (m, l, acc) of one split: fp32 online softmax on CUDA cores, one warp,
// lane holding head dims 4 lane .. 4 lane + 3.  Used only for splits whose
// flag says the fixed reference max ran out of headroom, and for the splits
// that carry the weight of a row whose weight sits on too few positions for
// one bf16 rounding of P.
__device__ void split_partial_exact(const AttnArgs &a, unsigned long long anc, int g,
                                    const float (&q4)[4], int p0, int p1, float &m, float &l,
                                    float (&acc)[4])
{
    constexpr int kU = 8;   // positions per step: their loads and reductions overlap
    const int lane = threadIdx.x & 31;
    const __nv_bfloat16 *kh = a.k + (size_t)g * a.kv_cap * kD + 4 * lane;
    const __nv_bfloat16 *vh = a.v + (size_t)g * a.kv_cap * kD + 4 * lane;
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

// One output row, by one warp: out = sum_s 2^(m_s - M) acc_s / sum_s
// 2^(m_s - M) l_s over the n_split partials of its (KV head, node group)
// gz.  Recomputed exactly instead of read: splits flagged for overflow,
// and, on a row whose effective number of positions may be below kNeffMin
// (L^2 < kNeffMin * sum_s c_s^2 q_s with c_s = 2^(m_s - M)), every split s
// whose c_s^2 q_s is above L^2 / (kNeffMin * n_split) -- the remaining
// splits then add up to a bound of at least kNeffMin on their own.  A
// recomputed split covers the tiles the owner map gives it.
__device__ __forceinline__ void t128_combine_row(const AttnArgs &a, const TreeMasks &masks, int row,
                                              int g, int gz, int n_gz, int n_split,
                                              const T128Sync &sy)
{
    const int rows_all = a.n_tree * a.n_heads_q;
    const int lane = threadIdx.x & 31;
    const int node = row / a.n_heads_q;
    const int32_t *flags = sy.flags;
    const float *ws_o = sy.part;
    const float *ws_ml = ws_o + (size_t)n_split * rows_all * kD;
    auto mlq_of = [&](int s) {
        return __ldcg(reinterpret_cast<const float4 *>(ws_ml + ((size_t)s * rows_all + row) * 4));
    };
    auto flagged = [&](int s) { return __ldcg(flags + (size_t)s * n_gz + gz) != 0; };

    // The common case (at most 2 kHalf splits): lane s reads split s's
    // (m, l, q) and flag while every lane also reads its four columns of the
    // acc of the first kHalf splits, all in flight together; the rest
    // follow once M is known (two halves keep the registers below the
    // kernel's budget).
    constexpr int kHalf = 12;
    const bool fast = n_split <= 2 * kHalf;
    float4 xs[kHalf];
    float4 my = make_float4(-INFINITY, 0.f, 0.f, 0.f);
    bool my_f = false;
    if (fast) {
        if (lane < n_split) {
            my = mlq_of(lane);
            my_f = flagged(lane);
        }
#pragma unroll
        for (int u = 0; u < kHalf; ++u)
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
        for (int h = 0; h < 2 && h * kHalf < n_split; ++h) {
            if (h == 1) {
#pragma unroll
                for (int u = 0; u < kHalf; ++u)
                    xs[u] = kHalf + u < n_split
                                ? __ldcg(reinterpret_cast<const float4 *>(
                                      ws_o + ((size_t)(kHalf + u) * rows_all + row) * kD + 4 * lane))
                                : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < kHalf; ++u) {
                const int sp = h * kHalf + u;
                if (sp >= n_split)
                    break;
                const float w = __shfl_sync(0xffffffffu, w_my, sp);
                L += __shfl_sync(0xffffffffu, wl_my, sp);
                acc[0] += w * xs[u].x;
                acc[1] += w * xs[u].y;
                acc[2] += w * xs[u].z;
                acc[3] += w * xs[u].w;
            }
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
        const int n_tiles_all = (total + kTileN - 1) / kTileN;
        const uint8_t *own = sy.owner + (size_t)gz * n_tiles_all;
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
                ms = -INFINITY;
                ls = 0.f;
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    as[e] = 0.f;
                // the tiles this split streamed, 32 owner entries at a time
                for (int t0 = 0; t0 < n_tiles_all; t0 += 32) {
                    const int t = t0 + lane;
                    uint32_t bits = __ballot_sync(0xffffffffu, t < n_tiles_all && own[t] == s);
                    while (bits) {
                        const int tt = t0 + __ffs(bits) - 1;
                        bits &= bits - 1;
                        split_partial_exact(a, masks.anc[node], g, q4, tt * kTileN,
                                            min(tt * kTileN + kTileN, total), ms, ls, as);
                    }
                }
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

// Bounded wait until the int32 at p (written by other CTAs) reaches
// target, read with gpu-scope acquire; on expiry raises *abort and records
// TS_ERR_TIMEOUT.
__device__ __forceinline__ bool wait_count_bounded(const int32_t *p, int target,
                                                   volatile uint32_t *abort, WorkspaceHeader *ws)
{
    const long long t0 = clock64();
    for (;;) {
        int32_t v;
        asm volatile("ld.acquire.gpu.global.b32 %0, [%1];\n" : "=r"(v) : "l"(p) : "memory");
        if (v >= target)
            return true;
        if (clock64() - t0 > kWaitCycles) {
            *abort = 1u;
            record_status(ws, TS_ERR_TIMEOUT);
            return false;
        }
        __nanosleep(128);
    }
}

__global__ void __launch_bounds__(kThreads, 1)
attn_t128_kernel(const __grid_constant__ CUtensorMap tmap_k,
                 const __grid_constant__ CUtensorMap tmap_v, AttnArgs a, TreeMasks masks,
                 int n_split, int nodes_per_group, T128Sync sy)
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
    const Layout lay = t128_layout(R);
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
    // (KV head, node group) of this CTA: its splits share one tile counter
    // and one arrival count (sy.sync + 4 gz)
    const int gz = g * gridDim.z + blockIdx.z;

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
        // warp 0 also reads S of the last block when it stores the root scores
        mbar_init(smem_addr(&bar->s_free[0]), 4 * u0 + (rs_warp0 && NB == 1 ? 1 : 0));
        mbar_init(smem_addr(&bar->s_free[1]), (u1 > 0 ? 4 * u1 : 1) + (rs_warp0 && NB == 2 ? 1 : 0));
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
        // the next kernel in the stream, when launched as a programmatic
        // dependent, may take the SMs this grid leaves idle (and then each SM
        // a split frees) and wait there for this grid's end
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
    // launched as a programmatic dependent: everything above (barriers,
    // TMEM, tensor maps) overlaps the previous kernel's tail; what follows
    // reads its results (the query rows, the cache, the workspace counters)
    grid_dependency_wait();
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
    } else if (warp == 0) {
        // the ancestor masks into shared memory: the tail tiles read them per
        // thread, which the kernel-parameter bank would serialise
        for (int i = lane; i < a.n_tree; i += 32)
            aux->anc[i] = masks.anc[i];
    }
    if (warp != 3) {
        tc_fence_before();
        named_bar_sync(kBarQuery, kThreads - 32);
        tc_fence_after();
    }

    if (warp == 3) {
        // ------------------------------------ TMA producer (K one tile ahead)
        // Tiles are handed out at run time, from the end of the cache
        // backwards: the split's own tile (n_tiles - 1 - split) first, then
        // tile n_tiles - 1 - (n_split + k) for the k-th increment of the
        // (head, group) counter, so that the splits of a head end together
        // however HBM serves them, and the tree-tail tile (the one with
        // ancestor masks) is taken first rather than last.  Each taken tile
        // is recorded in the owner map (for the exact recompute of a split).
        named_bar_sync(kBarQLoads, kQLoadThreads);
        if (lane == 0) {
            int nk = 0, nv = 0;   // tiles issued so far
            int uk = 0, uv = 0;   // ring entries used (the end marker included)
            // k-th tile handed out -> its index (k < 0 once none is left)
            auto tile_at = [&](int k) { return n_tiles_all - 1 - k; };
            int32_t *ctr = sy.sync + 4 * gz;
            int cur = tile_at(split);
            int nxt = tile_at(n_split + atomicAdd(&ctr[0], 1));   // used one step later
            int kend = -1;        // ring index of the end marker
            uint8_t *owner = sy.owner + (size_t)gz * n_tiles_all;
            // K and V are read once per call: their L2 lines go first, so
            // that the partials, the root scores and what the next kernels
            // read stay in L2
            const uint64_t pol = l2_evict_first_policy();
            // step i issues K(i), then V(i - 1): K is consumed a whole softmax
            // pass before V, and each load waits only for its own ring slot
            for (int i = 0;; ++i) {
                if (kend < 0) {
                    const int s = i % SK;
                    if (i >= SK &&
                        !wait_bounded(smem_addr(&bar->empty_k[s]), ((i / SK) & 1) ^ 1, abort, hdr))
                        break;
                    const uint32_t fb = smem_addr(&bar->full_k[s]);
                    if (cur >= 0) {
                        bar->tile_of[i % kTileRing] = cur;
                        owner[cur] = (uint8_t)split;
                        mbar_arrive_expect_tx(fb, kStageBytes);
                        const uint32_t dst = smem_addr(sK + s * kStageBytes);
                        tma_load_3d_hint(dst, &tmap_k, 0, cur * kTileN, g, fb, pol);
                        tma_load_3d_hint(dst + kBoxBytes, &tmap_k, 64, cur * kTileN, g, fb, pol);
                        nk = uk = i + 1;
                        cur = nxt;
                        if (cur >= 0)
                            nxt = tile_at(n_split + atomicAdd(&ctr[0], 1));
                    } else {
                        // no tile left: the QK issuer passes the marker on
                        bar->tile_of[i % kTileRing] = -1;
                        mbar_arrive(fb);
                        kend = i;
                        uk = i + 1;
                    }
                }
                if (i >= 1) {
                    const int t = i - 1, s = t % SV;
                    if (t >= SV &&
                        !wait_bounded(smem_addr(&bar->empty_v[s]), ((t / SV) & 1) ^ 1, abort, hdr))
                        break;
                    const uint32_t fb = smem_addr(&bar->full_v[s]);
                    if (t == kend) {
                        mbar_arrive(fb);   // the PV issuer's end
                        uv = t + 1;
                        break;
                    }
                    mbar_arrive_expect_tx(fb, kStageBytes);
                    const uint32_t dst = smem_addr(sV + s * kStageBytes);
                    const int pos0 = bar->tile_of[t % kTileRing] * kTileN;
                    tma_load_3d_hint(dst, &tmap_v, 0, pos0, g, fb, pol);
                    tma_load_3d_hint(dst + kBoxBytes, &tmap_v, 64, pos0, g, fb, pol);
                    nv = uv = t + 1;
                }
            }
            if (*abort) {
                // let our own copies land before the CTA exits (those whose
                // ring slot no later entry has taken)
                for (int t = max(0, uk - SK); t < nk; ++t)
                    wait_drain(smem_addr(&bar->full_k[t % SK]), (t / SK) & 1);
                for (int t = max(0, uv - SV); t < nv; ++t)
                    wait_drain(smem_addr(&bar->full_v[t % SV]), (t / SV) & 1);
            }
        }
    } else if (warp == 0) {
        // ------------------- root node's scores out of S_b, b the last block (lanes 0..G-1)
        if (rs_warp0) {
            // one 16x256b load of lanes 0..15, the shape the softmax warps
            // use: thread t holds lane t/4 (and 8 + t/4) at columns
            // 8j + 2(t%4) + {0, 1}, so threads 0..4G-1 hold the G root rows
            const int bl = NB - 1;
            const int r = lane >> 2;          // root row of this thread (lanes 0..7)
            const bool mine = r < G;
            const int c0 = 2 * (lane & 3);
            float *dst_row = a.root_scores + (size_t)(g * G + (mine ? r : 0)) * a.n_ctx;
            const bool vec = ((reinterpret_cast<uintptr_t>(a.root_scores) | (uintptr_t)a.n_ctx * 4) &
                              7) == 0;
            for (int t = 0;; ++t) {
                if (!warp_wait_bounded(smem_addr(&bar->s_full[bl]), t & 1, abort, hdr))
                    break;
                const int tile = bar->tile_of[t % kTileRing];
                if (tile < 0)
                    break;
                tc_fence_after();
                const int pos0 = tile * kTileN;
                uint32_t rr[64];
                if (pos0 < a.n_ctx)
                    tmem_ld16x256_x16(tmem + kSCol + 128 * bl, rr);
                // S_b is read: QK of the next tile may overwrite it
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(smem_addr(&bar->s_free[bl]));
                if (pos0 >= a.n_ctx || !mine)
                    continue;   // a tile of the tree tail only, or not a root lane
                if (vec && pos0 + kTileN <= a.n_ctx) {
                    // a whole context tile: no bounds, one 8-byte store per pair
                    float2 *dst2 = reinterpret_cast<float2 *>(dst_row + pos0 + c0);
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj)
                        dst2[4 * jj] = make_float2(__uint_as_float(rr[4 * jj]) * a.scale_log2,
                                                   __uint_as_float(rr[4 * jj + 1]) * a.scale_log2);
                    continue;
                }
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
                for (int t = 0;; ++t) {
                    const int s = t % SK;
                    if (!wait_bounded(smem_addr(&bar->full_k[s]), (t / SK) & 1, abort, hdr))
                        break;
                    if (bar->tile_of[t % kTileRing] < 0) {
                        // no tile left: the readers of each S_b learn it from
                        // a plain arrival, once they hold S_b(t-1)
                        for (int b = 0; b < NB; ++b) {
                            if (t > 0 &&
                                !wait_bounded(smem_addr(&bar->s_free[b]), (t - 1) & 1, abort, hdr))
                                break;
                            mbar_arrive(smem_addr(&bar->s_full[b]));
                        }
                        break;
                    }
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
                for (int t = 0;; ++t) {
                    const int s = t % SV;
                    if (!wait_bounded(smem_addr(&bar->full_v[s]), (t / SV) & 1, abort, hdr))
                        break;
                    if (bar->tile_of[t % kTileRing] < 0) {
                        mma_commit(smem_addr(&bar->o_final));   // after the last PV
                        break;
                    }
                    if (!wait_bounded(smem_addr(&bar->sm_done), t & 1, abort, hdr))
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
        bool ok = true;
        for (int t = 0;; ++t) {
            if (!warp_wait_bounded(smem_addr(&bar->s_full[b]), t & 1, abort, hdr)) {
                ok = false;
                break;
            }
            const int tile = bar->tile_of[t % kTileRing];
            if (tile < 0)
                break;
            tc_fence_after();
            uint32_t r[64];
            tmem_ld16x256_x16(s_addr, r);
            // S is in registers: QK of the next tile may overwrite it
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(smem_addr(&bar->s_free[b]));
            // raw scores; the scale (> 0) is applied inside the exponent
            const int pos0 = tile * kTileN;
            if (pos0 + kTileN > a.n_ctx) {
                // visibility of this thread's 32 positions (entry k = 2 jj + e
                // is position pos0 + 8 jj + c0 + e) for its two rows
                const uint32_t visA =
                    t128_tail_vis(aux->anc[node0 + (vA ? t128_row_of(nA, R) / G : 0)],
                                  a.n_ctx - pos0, a.n_tree, c0);
                const uint32_t visB =
                    t128_tail_vis(aux->anc[node0 + (vB ? t128_row_of(nB, R) / G : 0)],
                                  a.n_ctx - pos0, a.n_tree, c0);
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                    if (!((visA >> k) & 1u))
                        r[4 * (k >> 1) + (k & 1)] = __float_as_uint(-INFINITY);
                    if (!((visB >> k) & 1u))
                        r[4 * (k >> 1) + 2 + (k & 1)] = __float_as_uint(-INFINITY);
                }
            }
            // a row that has seen nothing yet takes this tile's max, rounded
            // up to an integer, as its reference (its O^T column and l are
            // still zero); afterwards the maxima are not needed
            if (__any_sync(0xffffffffu, mA == -INFINITY || mB == -INFINITY)) {
                const float xA = row_max(r, 0) * a.scale_log2;
                const float xB = row_max(r, 2) * a.scale_log2;
                float yA = fmaxf(xA, __shfl_xor_sync(0xffffffffu, xA, 1));
                float yB = fmaxf(xB, __shfl_xor_sync(0xffffffffu, xB, 1));
                yA = fmaxf(yA, __shfl_xor_sync(0xffffffffu, yA, 2));
                yB = fmaxf(yB, __shfl_xor_sync(0xffffffffu, yB, 2));
                if (mA == -INFINITY)
                    mA = ceilf(yA);
                if (mB == -INFINITY)
                    mB = ceilf(yB);
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
        float *ws_o = sy.part;
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
                // the copies' writes, made by the async proxy, before the
                // arrival below publishes them to the other splits
                fence_proxy_async_global();
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }

    // ---- combine.  Once every split of this (head, group) has arrived,
    // each folds its share of the group's rows (rows split, split +
    // n_split, ...; one warp each).  The launch is cooperative, so all
    // splits are resident and the wait ends.
    const int n_gz = a.n_heads_kv * gridDim.z;
    int32_t *ctr = sy.sync + 4 * gz;
    if (threadIdx.x == 0) {
        sy.flags[(size_t)split * n_gz + gz] = bar->overflow;
        __threadfence();   // partials, flag and owner entries before the arrival
        atomicAdd(&ctr[1], 1);
        wait_count_bounded(&ctr[1], n_split, abort, hdr);
    }
    __syncthreads();
    if (!*abort) {
        for (int m = split + warp * n_split; m < R; m += (kThreads / 32) * n_split)
            t128_combine_row(a, masks, (node0 + m / G) * a.n_heads_q + g * G + m % G, g, gz, n_gz,
                             n_split, sy);
    }
    __syncthreads();
    if (threadIdx.x == 0 && atomicAdd(&ctr[2], 1) == n_split - 1) {
        // every split of the group is past its wait and done taking tiles:
        // the counters go back to zero for the next call
        atomicExch(&ctr[0], 0);
        atomicExch(&ctr[1], 0);
        atomicExch(&ctr[2], 0);
    }
}

struct T128WsLayout {
    size_t sync, part, flags, owner, total;
};

// header | counters (zero between calls) | partials | flags | owner map
T128WsLayout t128_ws_layout(const AttnPlan &p, int n_heads_q, int n_heads_kv, int n_ctx,
                            int n_tree)
{
    const size_t n_gz = (size_t)n_heads_kv * p.node_groups;
    const size_t n_tiles = (size_t)(n_ctx + n_tree + kTileN - 1) / kTileN;
    T128WsLayout L;
    L.sync = kHeaderBytes;
    L.part = L.sync + align_up(n_gz * 4 * sizeof(int32_t), 256);
    L.flags = L.part + align_up((size_t)p.n_split * n_tree * n_heads_q * (kD + 4) * sizeof(float), 256);
    L.owner = L.flags + align_up((size_t)p.n_split * n_gz * sizeof(int32_t), 256);
    L.total = L.owner + align_up(n_gz * n_tiles, 256);
    return L;
}

}  // namespace

size_t attn_t128_workspace_bytes(int n_heads_q, int n_heads_kv, int n_ctx, int n_tree, int num_sms)
{
    const AttnPlan p = attn_t128_plan(n_heads_q, n_heads_kv, n_ctx, n_tree, num_sms);
    return t128_ws_layout(p, n_heads_q, n_heads_kv, n_ctx, n_tree).total;
}

size_t attn_t128_zeroed_bytes(int n_heads_q, int n_heads_kv, int n_ctx, int n_tree, int num_sms)
{
    const AttnPlan p = attn_t128_plan(n_heads_q, n_heads_kv, n_ctx, n_tree, num_sms);
    return t128_ws_layout(p, n_heads_q, n_heads_kv, n_ctx, n_tree).part;
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
    // one CTA per SM; the splits of a (head, group) take tiles at run time,
    // each starting with its own, so there are at most as many as tiles
    // (and at most 255: the owner map holds a byte per tile)
    const int n_tiles = (n_ctx + n_tree + kTileN - 1) / kTileN;
    int want = num_sms / (n_heads_kv * p.node_groups);
    want = want < 1 ? 1 : want;
    want = want > n_tiles ? n_tiles : want;
    p.n_split = want > 255 ? 255 : want;
    p.tiles_per_split = (n_tiles + p.n_split - 1) / p.n_split;   // on average
    return p;
}

bool attn_t128_fits(int n_heads_q, int n_heads_kv, int n_ctx, int n_tree, int num_sms)
{
    const AttnPlan p = attn_t128_plan(n_heads_q, n_heads_kv, n_ctx, n_tree, num_sms);
    return (long long)p.n_split * n_heads_kv * p.node_groups <= num_sms;
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
    const Layout lay = t128_layout((a.n_heads_q / a.n_heads_kv) * T0);
    static const cudaError_t attr = cudaFuncSetAttribute(
        attn_t128_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemLimit);
    if (attr != cudaSuccess)
        return attr;
    const T128WsLayout wl = t128_ws_layout(p, a.n_heads_q, a.n_heads_kv, a.n_ctx, a.n_tree);
    char *ws = reinterpret_cast<char *>(a.workspace);
    T128Sync sy;
    sy.sync = reinterpret_cast<int32_t *>(ws + wl.sync);
    sy.part = reinterpret_cast<float *>(ws + wl.part);
    sy.flags = reinterpret_cast<int32_t *>(ws + wl.flags);
    sy.owner = reinterpret_cast<uint8_t *>(ws + wl.owner);
    // cooperative: the splits of a head wait for one another before the
    // combine, so every CTA must be resident at once (one per SM)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.n_split, a.n_heads_kv, p.node_groups);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = lay.smem_bytes;
    cfg.stream = stream;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeCooperative;
    at[0].val.cooperative = 1;
    // and a programmatic dependent of the kernel before it in the stream
    at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 2;
    cudaError_t e = cudaLaunchKernelEx(&cfg, attn_t128_kernel, mk, mv, a, masks, p.n_split,
                                       p.nodes_per_group, sy);
    if (e == cudaSuccess)
        e = cudaGetLastError();
    if (e != cudaSuccess)
        return e;
    count_launches(1);
    return cudaSuccess;
}

bool attn_t128_leaves_root_scores(const AttnArgs &a)
{
    const AttnPlan p = attn_t128_plan(a.n_heads_q, a.n_heads_kv, a.n_ctx, a.n_tree, 148);
    return t128_rs_warp0(a, p.nodes_per_group);
}

}  // namespace ts
