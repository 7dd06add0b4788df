// select.cu -- dynamic partial-KV update: importance score, sink + top-budget
// selection, and the gather into the compact draft cache.
//
// TokenSwift (aiboss88.com), "TokenSwift's technical principles": the
// initial KV cache is kept and the rest is replaced in order of token
// importance; tencent article 动态KV缓存更新: the partial cache is refreshed
// during generation; 无损的输出质量: the draft model is the target model with
// that partial cache.
//
// Pass 1 (grid: chunks x Hkv): s[h,n] = log2(e) * scale * q_last[h] . k[g,n]
//   for the G query heads of KV head g, on the tensor cores: per 16 keys a
//   warp runs D/16 mma.sync m16n8k16 (bf16 in, fp32 accumulate) with the
//   keys as the 16 rows of A, read from a 128-byte-swizzled TMA tile with
//   ldmatrix, and the group's query rows as the 8 columns of B, held in
//   registers.  A CTA streams its chunk of key rows through a 4-stage ring
//   of 64-row tiles (one producer lane, four MMA warps).  Writes s (fp32
//   [Hq, n_ctx]) and a running (max, sum 2^(s-max)) per head and chunk.
//   K is read once: Hkv * n_ctx * D * 2 bytes.
// Selection (grids of chunks x Hkv, about two CTAs per SM, every head at
//   once; each kernel a programmatic dependent of the one before):
//   1. per chunk, each head's (max, sum 2^(s-max)) -- only when the scores
//      come from the caller; the score pass leaves them itself;
//   2. the importance score[n] = (1/G) sum_h 2^(s[h,n] - M_h) / Z_h of the
//      chunk's positions, written out, and a 4096-bin histogram of the top
//      bits of the candidates' scores (non-negative floats order as their
//      bit patterns), summed per head in global memory;
//   3. per chunk, the bin holding the budget-th largest candidate (from the
//      head's histogram), the candidates above it counted and those in it
//      listed (score bits, position);
//   4. per chunk, the exact budget-th largest score among the listed ones
//      (two radix passes over the remaining 19 bits; every chunk of a head
//      does this on its own, a few hundred keys) and the chunk's offset;
//      then its kept positions -- sinks, every score above the threshold,
//      and the first scores equal to it in position order, so equal scores
//      go to the lower position -- written in ascending order and their
//      K/V rows copied with 16-byte loads.
#include <math.h>

#include "attn_common.cuh"
#include "sm100.cuh"
#include "ts_internal.cuh"

namespace ts {
namespace {

constexpr int kMaxGroup = TS_MAX_SELECT_GROUP;

// ------------------------------------------------------------------ pass 1
constexpr int kP1Rows = 64;     // key rows per pipeline stage
constexpr int kP1Stages = 4;
constexpr int kP1Warps = 4;     // MMA warps, 16 keys of a tile each; warp 4 loads
constexpr int kP1Threads = 32 * (kP1Warps + 1);
constexpr int kP1BoxBytes = kP1Rows * 128;   // 64 rows x 64 columns of bf16

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t (&r)[4])
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

// d += a (16x16, row-major) * b (16x8, column-major), bf16 in, fp32 accumulate
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int D>
__global__ void __launch_bounds__(kP1Threads)
score_logits_kernel(const __grid_constant__ CUtensorMap tmap_k, SelectArgs a, int chunk,
                    int n_chunks, float *s_out, float2 *part_out)
{
    using namespace sm100;
    constexpr int kBoxes = D / 64;
    constexpr int kStageBytes = kBoxes * kP1BoxBytes;

    extern __shared__ unsigned char p1_raw[];
    unsigned char *ring = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(p1_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t full[kP1Stages], empty[kP1Stages];
    __shared__ uint32_t abort_flag;
    __shared__ float red_m[kP1Warps * 32][2], red_l[kP1Warps * 32][2];

    const int g = blockIdx.y;
    const int c = blockIdx.x;
    const int G = a.n_heads_q / a.n_heads_kv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int n0 = c * chunk;
    const int n1 = min(n0 + chunk, a.n_ctx);
    const int n_tiles = (n1 - n0 + kP1Rows - 1) / kP1Rows;
    WorkspaceHeader *hdr = reinterpret_cast<WorkspaceHeader *>(a.workspace);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kP1Stages; ++s) {
            mbar_init(smem_addr(&full[s]), 1);
            mbar_init(smem_addr(&empty[s]), kP1Warps);
        }
        abort_flag = 0u;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kP1Warps) {
        // ------------------------------------------------------- producer
        if (lane == 0) {
            int issued = 0;
            for (int t = 0; t < n_tiles; ++t) {
                const int s = t % kP1Stages;
                if (t >= kP1Stages && !wait_bounded(smem_addr(&empty[s]),
                                                    ((t / kP1Stages) & 1) ^ 1, &abort_flag, hdr))
                    break;
                const uint32_t fb = smem_addr(&full[s]);
                mbar_arrive_expect_tx(fb, kStageBytes);
#pragma unroll
                for (int b = 0; b < kBoxes; ++b)
                    tma_load_3d(smem_addr(ring + s * kStageBytes + b * kP1BoxBytes), &tmap_k, 64 * b,
                                n0 + t * kP1Rows, g, fb);
                issued = t + 1;
            }
            if (abort_flag)
                for (int t = max(0, issued - kP1Stages); t < issued; ++t)
                    wait_drain(smem_addr(&full[t % kP1Stages]), (t / kP1Stages) & 1);
        }
    } else {
        // ------------------------------------------------------ MMA warps
        // B = Q_group^T: column n = query head g*G + n (zero past G); the
        // fragment of k-step kk holds q[n][16kk + 2(lane%4) + {0,1}] and
        // q[n][16kk + 8 + 2(lane%4) + {0,1}] for n = lane / 4
        const int hq = lane >> 2;
        uint32_t bq[D / 16][2];
        const uint32_t *qrow = reinterpret_cast<const uint32_t *>(
            a.q_last + (int64_t)(g * G + (hq < G ? hq : 0)) * D);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            bq[kk][0] = hq < G ? qrow[8 * kk + (lane & 3)] : 0u;
            bq[kk][1] = hq < G ? qrow[8 * kk + 4 + (lane & 3)] : 0u;
        }
        // this lane's ldmatrix row (of the warp's 16 keys) and 8-column half
        const int lr = warp * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
        const int lh = lane >> 4;
        // accumulator (key, head) of this lane: keys lane/4 and lane/4 + 8,
        // heads 2(lane%4) and 2(lane%4) + 1
        const int h0 = 2 * (lane & 3);
        float run_m[2] = {-INFINITY, -INFINITY}, run_l[2] = {0.f, 0.f};
        for (int t = 0; t < n_tiles; ++t) {
            const int s = t % kP1Stages;
            if (!warp_wait_bounded(smem_addr(&full[s]), (t / kP1Stages) & 1, &abort_flag, hdr))
                break;
            const uint32_t stage = smem_addr(ring + s * kStageBytes);
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const int ch = (kk & 3) * 2 + lh;   // 16-byte chunk within the 128-byte row
                uint32_t af[4];
                ldmatrix_x4(stage + (kk >> 2) * kP1BoxBytes + lr * 128 + ((ch ^ (lr & 7)) << 4), af);
                mma_16816(acc, af, bq[kk][0], bq[kk][1]);
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(smem_addr(&empty[s]));
            const int nk = n0 + t * kP1Rows + warp * 16 + (lane >> 2);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int n = nk + 8 * (e >> 1), h = h0 + (e & 1);
                if (h < G && n < n1) {
                    const float sv = acc[e] * a.scale_log2;
                    s_out[(int64_t)(g * G + h) * a.n_ctx + n] = sv;
                    const float m_new = fmaxf(run_m[e & 1], sv);
                    run_l[e & 1] = run_l[e & 1] * exp2f(run_m[e & 1] - m_new) + exp2f(sv - m_new);
                    run_m[e & 1] = m_new;
                }
            }
        }
        red_m[threadIdx.x][0] = run_m[0];
        red_m[threadIdx.x][1] = run_m[1];
        red_l[threadIdx.x][0] = run_l[0];
        red_l[threadIdx.x][1] = run_l[1];
    }
    __syncthreads();
    // merge the running (max, sum) of every lane that holds head h
    if (part_out != nullptr && threadIdx.x < G) {
        const int h = threadIdx.x, e = h & 1;
        float M = -INFINITY;
        for (int t = 0; t < kP1Warps * 32; ++t)
            if (2 * (t & 3) == (h & ~1))
                M = fmaxf(M, red_m[t][e]);
        float L = 0.f;
        for (int t = 0; t < kP1Warps * 32; ++t)
            if (2 * (t & 3) == (h & ~1) && red_m[t][e] != -INFINITY)
                L += red_l[t][e] * exp2f(red_m[t][e] - M);
        part_out[(size_t)(g * G + h) * n_chunks + c] = make_float2(M, L);
    }
}

// ------------------------------------------------------ the selection pipeline
// Importance, threshold, compaction and gather for every KV head at once,
// in five short kernels over (chunk of positions, KV head) grids that cover
// the GPU.  Key of a position: the bit pattern of its importance, a sum of
// non-negative terms, so keys order as the values do.
constexpr int kSelThreads = 512;
constexpr int kBins0 = 4096;   // first-level bins: key bits 30..19
constexpr int kShift0 = 19;
constexpr int kMaxChunks = 256;
constexpr int kMaxChunkLen = 48 * 1024;   // a chunk's kept positions are listed in shared memory
static_assert(kMaxChunkLen < 65536, "per-chunk counts are packed in 16 bits");
static_assert(kMaxChunks <= kSelThreads, "one chunk per thread in the offset scan");
static_assert(kMaxGroup <= kSelThreads / 32, "one warp per head in the statistics merge");

enum SelMode { kSelect = 0, kKeepAll = 1, kSinksOnly = 2 };

struct SelInfo {
    int digit0;    // the bin of the budget-th largest candidate key
    int need0;     // how many keys of that bin are kept
};

struct SelWs {
    float2 *part;      // [Hq, n_parts] per-chunk (max, sum 2^(s - max)) of each head
    int n_parts;
    float *imp;        // [Hkv, n_ctx] importance (scores_out or workspace)
    int *hist;         // [Hkv, kBins0] candidate keys per top-bits bin
    SelInfo *info;     // [Hkv]
    int2 *cnt;         // [Hkv, NC] per chunk: keys above the threshold bin, keys in it
    uint2 *cand;       // [Hkv, n_ctx] (key, position) of the threshold bin's keys,
                       // each chunk's from its own first position on
};

struct SelGeom {
    int nc;      // chunks per head
    int chunk;   // positions per chunk (a multiple of 4)
};

__device__ __forceinline__ float warp_max(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}

__device__ __forceinline__ float warp_sum(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

__device__ __forceinline__ int warp_isum(int x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Exclusive scan of one int per thread over the block (any multiple of 32
// threads up to 1024); returns the block total.  scratch: 65 ints.
__device__ int block_exclusive_scan(int x, int *scratch, int &excl)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o)
            incl += y;
    }
    if (lane == 31)
        scratch[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int nw = blockDim.x / 32;
        const int w = lane < nw ? scratch[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o)
                wi += y;
        }
        if (lane < nw)
            scratch[32 + lane] = wi - w;
        if (lane == nw - 1)
            scratch[64] = wi;
    }
    __syncthreads();
    excl = scratch[32 + warp] + incl - x;
    const int total = scratch[64];
    __syncthreads();
    return total;
}

// Kernel 1 (scores given by the caller): per (chunk, KV head), each head of
// the group's (max, sum of 2^(s - max)) over the chunk.  Every head's loads
// of a round are in flight together; one reduction serves all heads.
template <int GM>
__global__ void __launch_bounds__(kSelThreads)
sel_stats_kernel(SelectArgs a, SelGeom geo, SelWs ws)
{
    __shared__ float2 red[kSelThreads / 32][GM];
    const int c = blockIdx.x, g = blockIdx.y;
    const int G = a.n_heads_q / a.n_heads_kv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int N = a.n_ctx;
    const int p0 = min(c * geo.chunk, N), p1 = min(p0 + geo.chunk, N);
    sm100::launch_dependents();
    sm100::grid_dependency_wait();   // the scores come from the previous kernel
    float m[GM], l[GM];
#pragma unroll
    for (int h = 0; h < GM; ++h) {
        m[h] = -INFINITY;
        l[h] = 0.f;
    }
    auto add = [&](int h, float x) {   // online (max, sum) of one head
        if (x > m[h]) {
            l[h] = (m[h] == -INFINITY ? 0.f : l[h] * exp2f(m[h] - x)) + 1.f;
            m[h] = x;
        } else if (x != -INFINITY) {
            l[h] += exp2f(x - m[h]);
        }
    };
    if ((N & 3) == 0) {
        // 16-byte rows (the caller's rows are 16-byte aligned then)
        constexpr int kU = 8 / GM;   // float4 per head and thread in flight
        const int v0 = p0 / 4, v1 = p1 / 4;
        for (int vb = v0 + tid; vb < v1; vb += kU * kSelThreads) {
            float4 x[GM][kU];
#pragma unroll
            for (int h = 0; h < GM; ++h)
#pragma unroll
                for (int u = 0; u < kU; ++u) {
                    const int vi = vb + u * kSelThreads;
                    x[h][u] = h < G && vi < v1
                                  ? __ldcg(reinterpret_cast<const float4 *>(
                                               a.root_scores + (size_t)(g * G + h) * N) + vi)
                                  : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
                }
#pragma unroll
            for (int h = 0; h < GM; ++h) {
                float mx = -INFINITY;
#pragma unroll
                for (int u = 0; u < kU; ++u)
                    mx = fmaxf(mx, fmaxf(fmaxf(x[h][u].x, x[h][u].y), fmaxf(x[h][u].z, x[h][u].w)));
                if (mx == -INFINITY)
                    continue;
                if (mx > m[h]) {
                    l[h] = m[h] == -INFINITY ? 0.f : l[h] * exp2f(m[h] - mx);
                    m[h] = mx;
                }
                float acc = 0.f;
#pragma unroll
                for (int u = 0; u < kU; ++u)
                    acc += exp2f(x[h][u].x - m[h]) + exp2f(x[h][u].y - m[h]) +
                           exp2f(x[h][u].z - m[h]) + exp2f(x[h][u].w - m[h]);
                l[h] += acc;
            }
        }
    } else {
        for (int n = p0 + tid; n < p1; n += kSelThreads)
#pragma unroll
            for (int h = 0; h < GM; ++h)
                if (h < G)
                    add(h, __ldcg(a.root_scores + (size_t)(g * G + h) * N + n));
    }
    // warp, then CTA: the max, then the sums rescaled to it
#pragma unroll
    for (int h = 0; h < GM; ++h) {
        const float wm = warp_max(m[h]);
        const float wl = warp_sum(m[h] == -INFINITY ? 0.f : l[h] * exp2f(m[h] - wm));
        if (lane == 0)
            red[warp][h] = make_float2(wm, wl);
    }
    __syncthreads();
    if (warp < G) {
        const float2 r = lane < kSelThreads / 32 ? red[lane][warp] : make_float2(-INFINITY, 0.f);
        const float M = warp_max(r.x);
        const float L = warp_sum(r.x == -INFINITY ? 0.f : r.y * exp2f(r.x - M));
        if (lane == 0)
            ws.part[(size_t)(g * G + warp) * ws.n_parts + c] = make_float2(M, L);
    }
}

// Kernel 2: importance of the chunk's positions (group mean of the heads'
// softmax weights), written out, and a histogram of the candidate keys'
// top 12 bits added into the head's global histogram.  The score loads are
// issued before the head statistics are merged, so that both are in flight
// together.
template <int GM>
__global__ void __launch_bounds__(kSelThreads, GM == 4 ? 2 : 1)
sel_keys_kernel(SelectArgs a, SelGeom geo, SelWs ws, const float *__restrict__ s_all, int mode,
                int vec)
{
    __shared__ int hist[kBins0];
    __shared__ float head_m[GM], head_w[GM];
    const int c = blockIdx.x, g = blockIdx.y;
    const int G = a.n_heads_q / a.n_heads_kv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int N = a.n_ctx;
    const int p0 = min(c * geo.chunk, N), p1 = min(p0 + geo.chunk, N);
    const bool do_hist = mode == kSelect;
    for (int b = tid; b < kBins0; b += kSelThreads)
        hist[b] = 0;
    sm100::launch_dependents();
    sm100::grid_dependency_wait();   // statistics and scores of the previous kernels
    // one shared-memory atomic per key (grouping a warp's equal bins with
    // a match instruction first measured slower)
    auto hist_add = [&](bool in, uint32_t key) {
        if (in)
            atomicAdd(&hist[key >> kShift0], 1);
    };
    float *imp = ws.imp + (size_t)g * N;
    constexpr int kR = 8 / GM;   // rounds of four positions per thread in flight
    const int span = vec ? 4 * kSelThreads : kSelThreads;   // positions per round
    const int rounds = (p1 - p0 + span - 1) / span;
    float4 sv[kR][GM];
    auto load = [&](int it0) {
#pragma unroll
        for (int r = 0; r < kR; ++r) {
            if (vec) {
                const int nb = p0 + 4 * (tid + (it0 + r) * kSelThreads);
#pragma unroll
                for (int h = 0; h < GM; ++h)
                    sv[r][h] = h < G && it0 + r < rounds && nb < p1
                                   ? __ldcg(reinterpret_cast<const float4 *>(
                                         s_all + (size_t)(g * G + h) * N + nb))
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
            } else {
                const int n = p0 + tid + (it0 + r) * kSelThreads;
#pragma unroll
                for (int h = 0; h < GM; ++h)
                    sv[r][h].x = h < G && it0 + r < rounds && n < p1
                                     ? __ldcg(s_all + (size_t)(g * G + h) * N + n)
                                     : 0.f;
            }
        }
    };
    load(0);
    if (warp < G) {
        const float2 *pp = ws.part + (size_t)(g * G + warp) * ws.n_parts;
        float M = -INFINITY;
        float2 mine[2];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int i = lane + 32 * k;
            mine[k] = i < ws.n_parts ? __ldcg(pp + i) : make_float2(-INFINITY, 0.f);
        }
        for (int i = lane + 64; i < ws.n_parts; i += 32)
            M = fmaxf(M, __ldcg(pp + i).x);
#pragma unroll
        for (int k = 0; k < 2; ++k)
            M = fmaxf(M, mine[k].x);
        M = warp_max(M);
        float L = 0.f;
#pragma unroll
        for (int k = 0; k < 2; ++k)
            if (mine[k].x != -INFINITY)
                L += mine[k].y * exp2f(mine[k].x - M);
        for (int i = lane + 64; i < ws.n_parts; i += 32) {
            const float2 x = __ldcg(pp + i);
            if (x.x != -INFINITY)
                L += x.y * exp2f(x.x - M);
        }
        L = warp_sum(L);
        if (lane == 0) {
            head_m[warp] = M;
            head_w[warp] = 1.f / ((float)G * L);
        }
    }
    __syncthreads();
    float hm[GM], hw[GM];
#pragma unroll
    for (int h = 0; h < GM; ++h) {
        hm[h] = h < G ? head_m[h] : 0.f;
        hw[h] = h < G ? head_w[h] : 0.f;
    }
    for (int it0 = 0; it0 < rounds; it0 += kR) {
        if (it0 > 0)
            load(it0);
#pragma unroll
        for (int r = 0; r < kR; ++r) {
            if (it0 + r >= rounds)
                break;   // uniform: every lane has the same rounds
            if (vec) {
                const int nb = p0 + 4 * (tid + (it0 + r) * kSelThreads);
                const bool live = nb < p1;
                float sc[4] = {0.f, 0.f, 0.f, 0.f};
                if (live) {
#pragma unroll
                    for (int h = 0; h < GM; ++h)
                        if (h < G) {
                            sc[0] += exp2f(sv[r][h].x - hm[h]) * hw[h];
                            sc[1] += exp2f(sv[r][h].y - hm[h]) * hw[h];
                            sc[2] += exp2f(sv[r][h].z - hm[h]) * hw[h];
                            sc[3] += exp2f(sv[r][h].w - hm[h]) * hw[h];
                        }
                    *reinterpret_cast<float4 *>(imp + nb) = make_float4(sc[0], sc[1], sc[2], sc[3]);
                }
                if (do_hist)
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        hist_add(live && nb + e >= a.n_sink, __float_as_uint(sc[e]));
            } else {
                const int n = p0 + tid + (it0 + r) * kSelThreads;
                float sc = 0.f;
                if (n < p1) {
#pragma unroll
                    for (int h = 0; h < GM; ++h)
                        if (h < G)
                            sc += exp2f(sv[r][h].x - hm[h]) * hw[h];
                    imp[n] = sc;
                }
                if (do_hist)
                    hist_add(n < p1 && n >= a.n_sink, __float_as_uint(sc));
            }
        }
    }
    if (!do_hist)
        return;
    __syncthreads();
    int *ghist = ws.hist + (size_t)g * kBins0;
    for (int b = tid; b < kBins0; b += kSelThreads)
        if (hist[b] != 0)
            atomicAdd(&ghist[b], hist[b]);
}

// The threshold bin of head g from its global histogram: the bin b with
// (candidates in higher bins) < budget <= (that count + its own).  Thread t
// holds bins 4095 - 8t .. 4088 - 8t (descending).  found: 2 ints.
__device__ void find_digit0(const int *ghist, int budget, int *scan, int *found)
{
    const int tid = threadIdx.x;
    int x[8];
    int sum = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        x[k] = __ldcg(&ghist[kBins0 - 1 - (8 * tid + k)]);
        sum += x[k];
    }
    int above;
    block_exclusive_scan(sum, scan, above);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        if (above < budget && budget <= above + x[k]) {
            found[0] = kBins0 - 1 - (8 * tid + k);
            found[1] = budget - above;
        }
        above += x[k];
    }
    __syncthreads();
}

// Kernel 3: per chunk, the threshold bin (found by every chunk from the
// head's histogram), the candidate keys above it counted and those in it
// listed at the chunk's own place in the candidate array.
constexpr int kCandPer = 8;   // positions per thread and batch
__global__ void __launch_bounds__(kSelThreads)
sel_cand_kernel(SelectArgs a, SelGeom geo, SelWs ws)
{
    __shared__ int scan[72];
    __shared__ int found[2];
    __shared__ int red[kSelThreads / 32];
    const int c = blockIdx.x, g = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int N = a.n_ctx;
    const int p0 = min(c * geo.chunk, N), p1 = min(p0 + geo.chunk, N);
    const float *imp = ws.imp + (size_t)g * N;
    uint2 *cand = ws.cand + (size_t)g * N + p0;
    const int batches = (p1 - p0 + kCandPer * kSelThreads - 1) / (kCandPer * kSelThreads);
    uint32_t key[kCandPer];
    sm100::launch_dependents();
    sm100::grid_dependency_wait();   // importance and histogram of the previous kernel
    auto load = [&](int bt) {
#pragma unroll
        for (int i = 0; i < kCandPer; ++i) {
            const int n = p0 + tid + (bt * kCandPer + i) * kSelThreads;
            key[i] = n < p1 && n >= a.n_sink ? __float_as_uint(__ldcg(imp + n)) : 0xFFFFFFFFu;
        }
    };
    load(0);   // in flight while the histogram is read
    if (tid == 0)
        found[0] = -1;
    find_digit0(ws.hist + (size_t)g * kBins0, a.budget, scan, found);
    const int digit0 = found[0];
    if (c == 0 && tid == 0) {
        ws.info[g].digit0 = digit0;
        ws.info[g].need0 = found[1];
    }
    int n_above = 0, base = 0;
    for (int bt = 0; bt < batches; ++bt) {
        if (bt > 0)
            load(bt);
        int hits = 0;
#pragma unroll
        for (int i = 0; i < kCandPer; ++i) {
            if (key[i] == 0xFFFFFFFFu)
                continue;   // outside the chunk, or a sink (scores are finite)
            const int bin = (int)(key[i] >> kShift0);
            n_above += bin > digit0;
            hits += bin == digit0;
        }
        int before;
        const int total = block_exclusive_scan(hits, scan, before);
        int k = base + before;
#pragma unroll
        for (int i = 0; i < kCandPer; ++i)
            if (key[i] != 0xFFFFFFFFu && (int)(key[i] >> kShift0) == digit0)
                cand[k++] = make_uint2(key[i], (uint32_t)(p0 + tid + (bt * kCandPer + i) * kSelThreads));
        base += total;
    }
    n_above = warp_isum(n_above);
    if (lane == 0)
        red[warp] = n_above;
    __syncthreads();
    if (warp == 0) {
        int v = lane < kSelThreads / 32 ? red[lane] : 0;
        v = warp_isum(v);
        if (lane == 0)
            ws.cnt[(size_t)g * geo.nc + c] = make_int2(v, base);
    }
}

// The exact threshold of head g and the offsets of chunk c, computed by
// every chunk of the head on its own (a few hundred candidates in the
// threshold bin, typically): the budget-th largest key among the
// candidates (two radix passes over their low 19 bits, on a copy in shared
// memory when it fits), then per chunk the number of kept positions before
// it and of equal-to-threshold keys before it.
constexpr int kCandSmem = 8 * 1024;   // candidates held in shared memory at most (64 KB)

struct ThreshShared {
    int hist[1024];
    int scan[72];
    int found[2];
    uint32_t small[32];        // the keys of a thinly filled second-level bin
    int n_small;
    int seg[kMaxChunks];       // candidate offsets of the chunks
    int gtc[kMaxChunks], eqc[kMaxChunks];
    int2 ci;                   // this chunk: kept before it, equal-to-T keys before it
    uint32_t T;                // the budget-th largest candidate key
    int need_eq;               // keys equal to T that are kept (lowest positions first)
};

// Block-wide exact threshold over the n_cand candidates get(0 .. n_cand-1)
// of bin digit0: a radix pass over bits 18..9 (1024 bins); if the bin it
// finds holds at most 32 keys, warp 0 ranks them directly, else a second
// pass over bits 8..0.  Then per chunk the candidates above T and equal to
// T (sh.gtc, sh.eqc).  Leaves sh.T and sh.need_eq.
template <typename Get>
__device__ __forceinline__ void block_radix_threshold(Get get, int n_cand, int digit0, int need,
                                                      const SelGeom &geo, ThreshShared &sh)
{
    const int tid = threadIdx.x, lane = tid & 31;
    uint32_t prefix = (uint32_t)digit0 << kShift0;
    uint32_t pmask = 0xFFFFFFFFu << kShift0;
    bool done = false;
    for (int pass = 0; pass < 2 && !done; ++pass) {
        const int shift = pass == 0 ? 9 : 0;
        const int nb = pass == 0 ? 1024 : 512;
        const uint32_t dmask = (uint32_t)nb - 1;
        for (int b = tid; b < 1024; b += kSelThreads)
            sh.hist[b] = 0;
        if (tid == 0)
            sh.n_small = 0;
        __syncthreads();
        for (int i = tid; i < n_cand; i += kSelThreads) {
            const uint32_t key = get(i).x;
            if ((key & pmask) == prefix)
                atomicAdd(&sh.hist[(key >> shift) & dmask], 1);
        }
        __syncthreads();
        // thread t holds bins nb-1-2t, nb-2-2t (descending)
        int x0 = 0, x1 = 0;
        if (2 * tid < nb) {
            x0 = sh.hist[nb - 1 - 2 * tid];
            x1 = sh.hist[nb - 2 - 2 * tid];
        }
        int above;
        block_exclusive_scan(x0 + x1, sh.scan, above);
        if (2 * tid < nb) {
            if (above < need && need <= above + x0) {
                sh.found[0] = nb - 1 - 2 * tid;
                sh.found[1] = above;
            } else if (above + x0 < need && need <= above + x0 + x1) {
                sh.found[0] = nb - 2 - 2 * tid;
                sh.found[1] = above + x0;
            }
        }
        __syncthreads();
        const int digit = sh.found[0];
        prefix |= (uint32_t)digit << shift;
        pmask |= dmask << shift;
        need -= sh.found[1];
        if (pass == 0 && sh.hist[digit] <= 32) {
            // few keys share the 22-bit prefix: list them and rank them in
            // one warp
            for (int i = tid; i < n_cand; i += kSelThreads) {
                const uint32_t key = get(i).x;
                if ((key & pmask) == prefix)
                    sh.small[atomicAdd(&sh.n_small, 1)] = key;
            }
            __syncthreads();
            if (tid < 32) {
                const int m = sh.n_small;
                const uint32_t mine = lane < m ? sh.small[lane] : 0u;
                int gt = 0, ge = 0;
                for (int j = 0; j < m; ++j) {
                    const uint32_t kj = __shfl_sync(0xffffffffu, mine, j);
                    gt += kj > mine;
                    ge += kj >= mine;
                }
                if (lane < m && gt < need && need <= ge) {
                    sh.T = mine;   // every writer holds the same key
                    sh.need_eq = need - gt;
                }
            }
            done = true;
        } else if (pass == 1 && tid == 0) {
            sh.T = prefix;
            sh.need_eq = need;
        }
        __syncthreads();
    }
    const uint32_t T = sh.T;
    for (int i = tid; i < n_cand; i += kSelThreads) {
        const uint2 kp = get(i);
        const int ch = (int)kp.y / geo.chunk;
        if (kp.x > T)
            atomicAdd(&sh.gtc[ch], 1);
        else if (kp.x == T)
            atomicAdd(&sh.eqc[ch], 1);
    }
    __syncthreads();
}

// The exact threshold of head g and the offsets of chunk c, found by every
// chunk of the head on its own with the whole CTA (a few hundred
// candidates in the threshold bin, typically).
// The per-chunk counts (this thread's chunk), digit0 and need0 come loaded.
__device__ void sel_threshold(const SelectArgs &a, const SelGeom &geo, const SelWs &ws, int mode,
                              int g, int c, uint2 *cs, int cand_cap, ThreshShared &sh, int2 cn,
                              int digit0, int need0)
{
    const int tid = threadIdx.x;
    const int N = a.n_ctx;
    const bool sel = mode == kSelect;
    const bool live = tid < geo.nc;
    int seg_before;
    const int n_cand = block_exclusive_scan(cn.y, sh.scan, seg_before);
    if (live) {
        sh.seg[tid] = seg_before;
        sh.gtc[tid] = 0;
        sh.eqc[tid] = 0;
    }
    if (tid == 0) {
        sh.T = 0xFFFFFFFFu;   // nothing at or above: no candidate kept
        sh.need_eq = 0;
    }
    __syncthreads();
    const uint2 *gcand = ws.cand + (size_t)g * N;
    // candidate i: chunk ch = the last with seg[ch] <= i, at its own place
    auto cand_at = [&](int i) -> uint2 {
        int lo = 0, hi = geo.nc - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (sh.seg[mid] <= i)
                lo = mid;
            else
                hi = mid - 1;
        }
        return __ldcg(gcand + (size_t)lo * geo.chunk + (i - sh.seg[lo]));
    };
    if (sel) {
        if (n_cand <= cand_cap) {
            for (int i0 = 0; i0 < n_cand; i0 += 4 * kSelThreads) {
                uint2 v[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int i = i0 + tid + k * kSelThreads;
                    v[k] = i < n_cand ? cand_at(i) : make_uint2(0u, 0u);
                }
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int i = i0 + tid + k * kSelThreads;
                    if (i < n_cand)
                        cs[i] = v[k];
                }
            }
            __syncthreads();
            // one code path per source of the candidates
            block_radix_threshold([&](int i) { return cs[i]; }, n_cand, digit0, need0, geo, sh);
        } else {
            block_radix_threshold([&](int i) { return cand_at(i); }, n_cand, digit0, need0, geo,
                                  sh);
        }
    }
    // kept before chunk ch: sinks before it, keys above T before it, and of
    // the equal keys the first need_eq in position order.  One chunk per
    // thread: scan the equal counts, then the kept counts.
    const int need_eq = sh.need_eq;
    const int ch = tid;
    const int my_eq = live && sel ? sh.eqc[ch] : 0;
    int eq_before;
    block_exclusive_scan(my_eq, sh.scan, eq_before);
    int k = 0;
    if (live) {
        const int q0 = ch * geo.chunk, q1 = min(q0 + geo.chunk, N);
        if (mode == kKeepAll) {
            k = max(0, q1 - q0);
        } else {
            k = max(0, min(q1, a.n_sink) - q0);
            if (sel)
                k += cn.x + sh.gtc[ch] + max(0, min(need_eq - eq_before, my_eq));
        }
    }
    int kept_before;
    block_exclusive_scan(k, sh.scan, kept_before);
    if (ch == c)
        sh.ci = make_int2(kept_before, eq_before);
    __syncthreads();
}

// Kernel 4: each chunk finds its head's threshold and its own offset, then
// writes its kept positions in ascending order from that offset and copies
// their K and V rows into the partial cache.  The first chunk of a head
// leaves the head's histogram zero for the next call.
constexpr int kGatherPer = 8;   // positions per thread held in registers
template <int D>
__global__ void __launch_bounds__(kSelThreads, 2)
sel_gather_kernel(SelectArgs a, SelGeom geo, SelWs ws, int mode, int cand_cap)
{
    extern __shared__ uint2 dyn[];   // cand_cap candidates, then this chunk's kept positions
    __shared__ ThreshShared sh;
    __shared__ int n_rows;
    uint2 *cs = dyn;
    int *list = reinterpret_cast<int *>(dyn + cand_cap);
    const int c = blockIdx.x, g = blockIdx.y;
    const int tid = threadIdx.x;
    const int N = a.n_ctx;
    const int p0 = min(c * geo.chunk, N), p1 = min(p0 + geo.chunk, N);
    const float *imp = ws.imp + (size_t)g * N;
    sm100::launch_dependents();
    sm100::grid_dependency_wait();   // candidates and counts of the previous kernel
    const bool sel = mode == kSelect;
    // the threshold's inputs first, so that they are not queued behind the
    // chunk's keys
    const int2 cn = tid < geo.nc && sel ? __ldcg(&ws.cnt[(size_t)g * geo.nc + tid])
                                        : make_int2(0, 0);
    const int digit0 = sel ? __ldcg(&ws.info[g].digit0) : 0;
    const int need0 = sel ? __ldcg(&ws.info[g].need0) : 0;
    // warp w owns positions [s0, s1) of the chunk, read coalesced in rounds
    // of 32: position s0 + 32 r + lane
    const int warp = tid >> 5, lane = tid & 31;
    const int rounds = (p1 - p0 + kSelThreads - 1) / kSelThreads;
    const int s0 = min(p0 + warp * 32 * rounds, p1), s1 = min(s0 + 32 * rounds, p1);
    const bool in_regs = rounds <= kGatherPer && sel;
    uint32_t key[kGatherPer];
    if (in_regs) {
#pragma unroll
        for (int r = 0; r < kGatherPer; ++r) {
            const int n = s0 + 32 * r + lane;
            key[r] = r < rounds && n < s1 ? __float_as_uint(__ldcg(imp + n)) : 0u;
        }
    }
    sel_threshold(a, geo, ws, mode, g, c, cs, cand_cap, sh, cn, digit0, need0);
    if (c == 0 && sel) {
        int *ghist = ws.hist + (size_t)g * kBins0;
        for (int b = tid; b < kBins0; b += kSelThreads)
            ghist[b] = 0;
    }
    const int2 ci = sh.ci;
    const uint32_t T = sh.T;
    const int need_eq = sh.need_eq;
    const int64_t want = (int64_t)a.n_sink + a.budget;
    const int n_keep = want < N ? (int)want : N;
    // 0 dropped, 1 kept, 2 equal to T
    auto cls = [&](int r) -> int {
        const int n = s0 + 32 * r + lane;
        if (n >= s1)
            return 0;
        if (mode == kKeepAll || n < a.n_sink)
            return 1;
        if (!sel)
            return 0;
        const uint32_t k = in_regs ? key[r] : __float_as_uint(__ldcg(imp + n));
        return k > T ? 1 : (k == T ? 2 : 0);
    };
    // the warp's counts, then one scan over the warps (both counts packed:
    // a chunk has at most kMaxChunkLen < 2^16 positions)
    int n_sure = 0, n_eq = 0;
    if (in_regs) {
#pragma unroll
        for (int r = 0; r < kGatherPer; ++r) {
            const int k = r < rounds ? cls(r) : 0;
            n_sure += __popc(__ballot_sync(0xffffffffu, k == 1));
            n_eq += __popc(__ballot_sync(0xffffffffu, k == 2));
        }
    } else {
        for (int r = 0; r < rounds; ++r) {
            const int k = cls(r);
            n_sure += __popc(__ballot_sync(0xffffffffu, k == 1));
            n_eq += __popc(__ballot_sync(0xffffffffu, k == 2));
        }
    }
    int packed_before;
    block_exclusive_scan(lane == 0 ? (n_sure | (n_eq << 16)) : 0, sh.scan, packed_before);
    packed_before = __shfl_sync(0xffffffffu, packed_before, 0);
    const int sure_before = packed_before & 0xFFFF, eq_before = packed_before >> 16;
    // equal keys are kept in position order: the first need_eq of the head
    int eqb = ci.y + eq_before;   // equal keys before this round's lane 0
    int slot = sure_before + max(0, min(need_eq, eqb)) - max(0, min(need_eq, ci.y));
    int32_t *idx = a.idx_out + (size_t)g * n_keep;
    const unsigned lt = (1u << lane) - 1u;
    auto place = [&](int r, int k) {
        const unsigned eqm = __ballot_sync(0xffffffffu, k == 2);
        const bool kept = k == 1 || (k == 2 && eqb + __popc(eqm & lt) < need_eq);
        const unsigned km = __ballot_sync(0xffffffffu, kept);
        if (kept) {
            const int my = slot + __popc(km & lt);
            const int out = ci.x + my;
            const int n = s0 + 32 * r + lane;
            if (out < n_keep) {
                idx[out] = n;
                list[my] = n;
            } else {
                record_status(reinterpret_cast<WorkspaceHeader *>(a.workspace), TS_ERR_DEVICE_ARG);
            }
        }
        eqb += __popc(eqm);
        slot += __popc(km);
    };
    if (in_regs) {
#pragma unroll
        for (int r = 0; r < kGatherPer; ++r)
            if (r < rounds)
                place(r, cls(r));
    } else {
        for (int r = 0; r < rounds; ++r)
            place(r, cls(r));
    }
    // rows: the chunk's kept count is the last thread's end slot
    if (tid == kSelThreads - 1)
        n_rows = min(slot, n_keep - ci.x);
    __syncthreads();
    const int rows = n_rows;
    constexpr int LPR = D / 8;   // lanes per row, 16 bytes each
    const __nv_bfloat16 *kh = a.k + (int64_t)g * a.kv_cap * D;
    const __nv_bfloat16 *vh = a.v + (int64_t)g * a.kv_cap * D;
    __nv_bfloat16 *kp = a.k_partial + (int64_t)g * a.partial_cap * D;
    __nv_bfloat16 *vp = a.v_partial + (int64_t)g * a.partial_cap * D;
    const int rows_per_pass = kSelThreads / LPR;
    const int li = tid % LPR;
    constexpr int kG = 4;   // rows per thread per step, loads in flight together
    for (int t0 = tid / LPR; t0 < rows; t0 += rows_per_pass * kG) {
        uint4 kv[kG], vv[kG];
        int nn[kG];
#pragma unroll
        for (int u = 0; u < kG; ++u) {
            const int t = t0 + u * rows_per_pass;
            nn[u] = t < rows ? list[t] : -1;
            const int r = nn[u] >= 0 ? nn[u] : 0;
            kv[u] = *reinterpret_cast<const uint4 *>(kh + (int64_t)r * D + li * 8);
            vv[u] = *reinterpret_cast<const uint4 *>(vh + (int64_t)r * D + li * 8);
        }
#pragma unroll
        for (int u = 0; u < kG; ++u) {
            const int t = t0 + u * rows_per_pass;
            if (nn[u] >= 0) {
                *reinterpret_cast<uint4 *>(kp + (int64_t)(ci.x + t) * D + li * 8) = kv[u];
                *reinterpret_cast<uint4 *>(vp + (int64_t)(ci.x + t) * D + li * 8) = vv[u];
            }
        }
    }
}

// --------------------------------------------------------------------- host
struct SelPlan {
    int p1_chunk, p1_chunks;   // the score pass's chunks (its partials)
    SelGeom geo;               // the selection's chunks
};

SelPlan make_sel_plan(int n_heads_kv, int n_ctx, int num_sms)
{
    SelPlan p;
    // score pass: three 64 KB-ring CTAs fit an SM, one wave over all heads
    int want = (num_sms * 3) / n_heads_kv;
    want = want < 1 ? 1 : want;
    int chunk = (n_ctx + want - 1) / want;
    chunk = chunk < 512 ? 512 : chunk;
    p.p1_chunk = chunk;
    p.p1_chunks = (n_ctx + chunk - 1) / chunk;
    // selection: about two CTAs per SM over all heads, chunks of at least
    // 1024 positions, a multiple of 4, at most kMaxChunks per head
    int nc = (2 * num_sms) / n_heads_kv;
    nc = nc < 1 ? 1 : nc;
    const int max_nc = (n_ctx + 1023) / 1024;
    nc = nc > max_nc ? max_nc : nc;
    const int min_nc = (n_ctx + kMaxChunkLen - 1) / kMaxChunkLen;
    nc = nc < min_nc ? min_nc : nc;
    nc = nc > kMaxChunks ? kMaxChunks : nc;
    int sc = ((n_ctx + nc - 1) / nc + 3) / 4 * 4;
    p.geo.chunk = sc;
    p.geo.nc = (n_ctx + sc - 1) / sc;
    return p;
}

// Workspace: header, [score pass: s fp32 [Hq, n_ctx]], partials, importance,
// histograms, info, per-chunk counts and offsets, candidates.
struct SelOffsets {
    size_t s, part, imp, hist, info, cnt, cand, total;
};

SelOffsets sel_offsets(int n_heads_q, int n_heads_kv, int n_ctx, const SelPlan &p,
                       bool score_pass)
{
    SelOffsets o;
    size_t at = kHeaderBytes;
    auto take = [&](size_t bytes) {
        const size_t r = at;
        at = align_up(at + bytes, 256);
        return r;
    };
    const int n_parts = score_pass ? p.p1_chunks : p.geo.nc;
    o.s = take(score_pass ? (size_t)n_heads_q * n_ctx * sizeof(float) : 0);
    o.part = take((size_t)n_heads_q * n_parts * sizeof(float2));
    o.imp = take((size_t)n_heads_kv * n_ctx * sizeof(float));
    o.hist = take((size_t)n_heads_kv * kBins0 * sizeof(int));
    o.info = take((size_t)n_heads_kv * sizeof(SelInfo));
    o.cnt = take((size_t)n_heads_kv * p.geo.nc * sizeof(int2));
    o.cand = take((size_t)n_heads_kv * n_ctx * sizeof(uint2));
    o.total = at;
    return o;
}

template <int D>
cudaError_t launch_p1(const SelectArgs &a, const SelPlan &p, float *s_out, float2 *part_out,
                      cudaStream_t stream)
{
    CUtensorMap mk;
    if (!encode_kv_map(&mk, a.k, a.n_ctx, a.kv_cap, a.n_heads_kv, kP1Rows, D))
        return cudaErrorInvalidValue;
    constexpr int smem = 1024 + kP1Stages * (D / 64) * kP1BoxBytes;
    static const cudaError_t attr = cudaFuncSetAttribute(
        score_logits_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (attr != cudaSuccess)
        return attr;
    dim3 grid(p.p1_chunks, a.n_heads_kv);
    score_logits_kernel<D><<<grid, kP1Threads, smem, stream>>>(mk, a, p.p1_chunk, p.p1_chunks,
                                                                s_out, part_out);
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess)
        count_launches(1);
    return e;
}

template <int D>
cudaError_t launch_d(const SelectArgs &a, const SelPlan &p, cudaStream_t stream)
{
    const bool score_pass = a.root_scores == nullptr;
    const SelOffsets o = sel_offsets(a.n_heads_q, a.n_heads_kv, a.n_ctx, p, score_pass);
    char *w = reinterpret_cast<char *>(a.workspace);
    SelWs ws;
    ws.part = reinterpret_cast<float2 *>(w + o.part);
    ws.n_parts = score_pass ? p.p1_chunks : p.geo.nc;
    ws.imp = a.scores_out ? a.scores_out : reinterpret_cast<float *>(w + o.imp);
    ws.hist = reinterpret_cast<int *>(w + o.hist);
    ws.info = reinterpret_cast<SelInfo *>(w + o.info);
    ws.cnt = reinterpret_cast<int2 *>(w + o.cnt);
    ws.cand = reinterpret_cast<uint2 *>(w + o.cand);
    const int64_t want = (int64_t)a.n_sink + a.budget;
    const int mode = want >= a.n_ctx ? kKeepAll : (a.budget == 0 ? kSinksOnly : kSelect);
    const dim3 grid(p.geo.nc, a.n_heads_kv);

    // scores: the caller's (then their per-chunk statistics here), or the
    // score pass into the workspace (which leaves the statistics itself)
    const float *s_all = a.root_scores;
    const int G = a.n_heads_q / a.n_heads_kv;
    const int GM = G <= 1 ? 1 : (G <= 2 ? 2 : (G <= 4 ? 4 : 8));
    const dim3 block(kSelThreads);
    cudaError_t e;
    // every kernel of the pipeline is launched as a programmatic dependent
    // of the one before (it waits for it before reading its results)
    if (score_pass) {
        float *s_ws = reinterpret_cast<float *>(w + o.s);
        e = launch_p1<D>(a, p, s_ws, ws.part, stream);
        if (e != cudaSuccess)
            return e;
        s_all = s_ws;
    } else {
        e = GM == 1   ? launch_pdl(sel_stats_kernel<1>, grid, block, 0, stream, a, p.geo, ws)
            : GM == 2 ? launch_pdl(sel_stats_kernel<2>, grid, block, 0, stream, a, p.geo, ws)
            : GM == 4 ? launch_pdl(sel_stats_kernel<4>, grid, block, 0, stream, a, p.geo, ws)
                      : launch_pdl(sel_stats_kernel<8>, grid, block, 0, stream, a, p.geo, ws);
        if (e != cudaSuccess)
            return e;
    }
    // 16-byte loads and stores when every row starts on a 16-byte boundary
    const int vec = (a.n_ctx & 3) == 0 && reinterpret_cast<uintptr_t>(s_all) % 16 == 0 &&
                    reinterpret_cast<uintptr_t>(ws.imp) % 16 == 0;
    e = GM == 1   ? launch_pdl(sel_keys_kernel<1>, grid, block, 0, stream, a, p.geo, ws, s_all, mode, vec)
        : GM == 2 ? launch_pdl(sel_keys_kernel<2>, grid, block, 0, stream, a, p.geo, ws, s_all, mode, vec)
        : GM == 4 ? launch_pdl(sel_keys_kernel<4>, grid, block, 0, stream, a, p.geo, ws, s_all, mode, vec)
                  : launch_pdl(sel_keys_kernel<8>, grid, block, 0, stream, a, p.geo, ws, s_all, mode, vec);
    if (e != cudaSuccess)
        return e;
    if (mode == kSelect) {
        e = launch_pdl(sel_cand_kernel, grid, block, 0, stream, a, p.geo, ws);
        if (e != cudaSuccess)
            return e;
    }
    // dynamic shared memory: the candidates (as many as fit beside the
    // chunk's list, up to kCandSmem), then the list
    const size_t list_bytes = (size_t)p.geo.chunk * sizeof(int);
    constexpr size_t kDynMax = 96 * 1024;   // two CTAs per SM with the static part
    size_t cap = list_bytes < kDynMax ? (kDynMax - list_bytes) / sizeof(uint2) : 0;
    cap = cap > (size_t)kCandSmem ? (size_t)kCandSmem : cap;
    const int cand_cap = (int)cap;
    const size_t dyn = (size_t)cand_cap * sizeof(uint2) + list_bytes;
    static const cudaError_t attr = cudaFuncSetAttribute(
        sel_gather_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    if (attr != cudaSuccess)
        return attr;
    e = launch_pdl(sel_gather_kernel<D>, grid, block, dyn, stream, a, p.geo, ws, mode, cand_cap);
    if (e != cudaSuccess)
        return e;
    return cudaSuccess;
}

}  // namespace

cudaError_t select_score_pass_launch(const SelectArgs &a, float *out, int num_sms,
                                     cudaStream_t stream)
{
    const SelPlan p = make_sel_plan(a.n_heads_kv, a.n_ctx, num_sms);
    return a.head_dim == 128 ? launch_p1<128>(a, p, out, nullptr, stream)
                             : launch_p1<64>(a, p, out, nullptr, stream);
}

int select_supported(int n_heads_q, int n_heads_kv, int head_dim, int n_ctx)
{
    const int G = n_heads_q / n_heads_kv;
    if (G > kMaxGroup)
        return 0;
    if (head_dim == 64 && G > 8)
        return 0;
    // a chunk's kept positions are listed in shared memory
    const SelPlan p = make_sel_plan(n_heads_kv, n_ctx, 148);
    return p.geo.chunk <= kMaxChunkLen;
}

size_t select_workspace_bytes(int n_heads_q, int n_heads_kv, int head_dim, int n_ctx,
                              int num_sms)
{
    (void)head_dim;
    const SelPlan p = make_sel_plan(n_heads_kv, n_ctx, num_sms);
    return sel_offsets(n_heads_q, n_heads_kv, n_ctx, p, true).total;
}

size_t select_from_scores_workspace_bytes(int n_heads_q, int n_heads_kv, int n_ctx, int num_sms)
{
    const SelPlan p = make_sel_plan(n_heads_kv, n_ctx, num_sms);
    return sel_offsets(n_heads_q, n_heads_kv, n_ctx, p, false).total;
}

cudaError_t select_launch(const SelectArgs &a, int num_sms, cudaStream_t stream)
{
    const SelPlan p = make_sel_plan(a.n_heads_kv, a.n_ctx, num_sms);
    return a.head_dim == 128 ? launch_d<128>(a, p, stream) : launch_d<64>(a, p, stream);
}

}  // namespace ts
