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
//   once):
//   1. per chunk, each head's (max, sum 2^(s-max)) -- only when the scores
//      come from the caller; the score pass leaves them itself;
//   2. the importance score[n] = (1/G) sum_h 2^(s[h,n] - M_h) / Z_h of the
//      chunk's positions, written out, and a 4096-bin histogram of the top
//      bits of the candidates' scores (non-negative floats order as their
//      bit patterns), summed per head in global memory; the last chunk of a
//      head to finish finds the bin holding the budget-th largest candidate;
//   3. per chunk, the candidates above that bin are counted and those in it
//      listed (score bits, position);
//   4. one CTA per head finds the exact budget-th largest score among the
//      listed ones (two radix passes over the remaining 19 bits) and, per
//      chunk, how many positions are kept before it;
//   5. per chunk, the kept positions -- sinks, every score above the
//      threshold, and the first scores equal to it in position order, so
//      equal scores go to the lower position -- are written in ascending
//      order from the chunk's offset and their K/V rows copied with 16-byte
//      loads.
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
static_assert(kMaxChunks <= kSelThreads, "one chunk per thread in the offset scan");
static_assert(kMaxGroup <= kSelThreads / 32, "one warp per head in the statistics merge");

enum SelMode { kSelect = 0, kKeepAll = 1, kSinksOnly = 2 };

struct SelInfo {
    int digit0;    // the bin of the budget-th largest candidate key
    int need0;     // how many keys of that bin are kept
    int n_cand;    // keys of that bin, appended to the candidate list
    uint32_t T;    // the budget-th largest candidate key
    int need_eq;   // how many keys equal to T are kept (lowest positions first)
    int pad[3];
};

struct SelWs {
    float2 *part;      // [Hq, n_parts] per-chunk (max, sum 2^(s - max)) of each head
    int n_parts;
    float *imp;        // [Hkv, n_ctx] importance (scores_out or workspace)
    int *hist;         // [Hkv, kBins0]
    int *tick;         // [Hkv]
    SelInfo *info;     // [Hkv]
    int *above;        // [Hkv, NC] candidate keys above the threshold bin, per chunk
    int2 *chunk;       // [Hkv, NC] (kept before the chunk, equal-to-T keys before it)
    uint2 *cand;       // [Hkv, n_ctx] (key, position) of the threshold bin's keys
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
// the group's (max, sum of 2^(s - max)) over the chunk.
__global__ void __launch_bounds__(kSelThreads)
sel_stats_kernel(SelectArgs a, SelGeom geo, SelWs ws)
{
    __shared__ float2 red[kSelThreads / 32];
    const int c = blockIdx.x, g = blockIdx.y;
    const int G = a.n_heads_q / a.n_heads_kv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int N = a.n_ctx;
    const int p0 = min(c * geo.chunk, N), p1 = min(p0 + geo.chunk, N);
    for (int h = 0; h < G; ++h) {
        const float *row = a.root_scores + (size_t)(g * G + h) * N;
        float m = -INFINITY, l = 0.f;
        if ((N & 3) == 0) {
            // the chunk is a multiple of 4 positions: 16-byte loads, all of
            // this thread's loads in flight together
            constexpr int kU = 8;
            const int v0 = p0 / 4, v1 = p1 / 4;
            for (int vb = v0 + tid; vb < v1; vb += kU * kSelThreads) {
                float4 x[kU];
#pragma unroll
                for (int u = 0; u < kU; ++u) {
                    const int vi = vb + u * kSelThreads;
                    x[u] = vi < v1 ? __ldcg(reinterpret_cast<const float4 *>(row) + vi)
                                   : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
                }
                float mx = -INFINITY;
#pragma unroll
                for (int u = 0; u < kU; ++u)
                    mx = fmaxf(mx, fmaxf(fmaxf(x[u].x, x[u].y), fmaxf(x[u].z, x[u].w)));
                if (mx == -INFINITY)
                    continue;
                if (mx > m) {
                    l = m == -INFINITY ? 0.f : l * exp2f(m - mx);
                    m = mx;
                }
                float acc = 0.f;
#pragma unroll
                for (int u = 0; u < kU; ++u)
                    acc += exp2f(x[u].x - m) + exp2f(x[u].y - m) + exp2f(x[u].z - m) +
                           exp2f(x[u].w - m);
                l += acc;
            }
        } else {
            for (int n = p0 + tid; n < p1; n += kSelThreads) {
                const float x = __ldcg(row + n);
                if (x > m) {
                    l = (m == -INFINITY ? 0.f : l * exp2f(m - x)) + 1.f;
                    m = x;
                } else if (x != -INFINITY) {
                    l += exp2f(x - m);
                }
            }
        }
        // CTA: max, then the sums rescaled to it
        const float wm = warp_max(m);
        float wl = warp_sum(m == -INFINITY ? 0.f : l * exp2f(m - wm));
        if (lane == 0)
            red[warp] = make_float2(wm, wl);
        __syncthreads();
        if (warp == 0) {
            const float2 r = lane < kSelThreads / 32 ? red[lane] : make_float2(-INFINITY, 0.f);
            const float M = warp_max(r.x);
            const float L = warp_sum(r.x == -INFINITY ? 0.f : r.y * exp2f(r.x - M));
            if (lane == 0)
                ws.part[(size_t)(g * G + h) * ws.n_parts + c] = make_float2(M, L);
        }
        __syncthreads();
    }
}

// Kernel 2: importance of the chunk's positions (group mean of the heads'
// softmax weights), written out; a histogram of the candidate keys' top 12
// bits, summed over the head's chunks; the last chunk of a head to finish
// finds the bin holding the budget-th largest candidate.
__global__ void __launch_bounds__(kSelThreads, 2)
sel_keys_kernel(SelectArgs a, SelGeom geo, SelWs ws, const float *__restrict__ s_all, int mode,
                int vec)
{
    __shared__ int hist[kBins0];
    __shared__ float head_m[kMaxGroup], head_w[kMaxGroup];
    __shared__ int scan[72];
    __shared__ int is_last;
    __shared__ int found[2];
    const int c = blockIdx.x, g = blockIdx.y;
    const int G = a.n_heads_q / a.n_heads_kv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int N = a.n_ctx;
    const int p0 = min(c * geo.chunk, N), p1 = min(p0 + geo.chunk, N);
    const bool do_hist = mode == kSelect;
    for (int b = tid; b < kBins0; b += kSelThreads)
        hist[b] = 0;
    if (warp < G) {
        const float2 *pp = ws.part + (size_t)(g * G + warp) * ws.n_parts;
        float M = -INFINITY;
        for (int i = lane; i < ws.n_parts; i += 32)
            M = fmaxf(M, pp[i].x);
        M = warp_max(M);
        float L = 0.f;
        for (int i = lane; i < ws.n_parts; i += 32)
            if (pp[i].x != -INFINITY)
                L += pp[i].y * exp2f(pp[i].x - M);
        L = warp_sum(L);
        if (lane == 0) {
            head_m[warp] = M;
            head_w[warp] = 1.f / ((float)G * L);
        }
    }
    __syncthreads();
    float hm[kMaxGroup], hw[kMaxGroup];
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) {
        hm[h] = h < G ? head_m[h] : 0.f;
        hw[h] = h < G ? head_w[h] : 0.f;
    }
    // lanes with equal bins add once, by their leader (positive scores
    // share their leading bits, so many lanes of a warp hit the same bin)
    auto hist_add = [&](bool in, uint32_t key) {
        const unsigned act = __ballot_sync(0xffffffffu, in);
        if (in) {
            const uint32_t bin = key >> kShift0;
            const unsigned same = __match_any_sync(act, bin);
            if (lane == __ffs(same) - 1)
                atomicAdd(&hist[bin], __popc(same));
        }
    };
    float *imp = ws.imp + (size_t)g * N;
    if (vec) {
        // four positions per thread and round; two CTAs per SM keep enough
        // loads in flight
        constexpr int kR = 1;
        const int rounds = (p1 - p0 + 4 * kSelThreads - 1) / (4 * kSelThreads);
        for (int it0 = 0; it0 < rounds; it0 += kR) {
            float4 sv[kR][kMaxGroup];
#pragma unroll
            for (int r = 0; r < kR; ++r) {
                const int nb = p0 + 4 * (tid + (it0 + r) * kSelThreads);
#pragma unroll
                for (int h = 0; h < kMaxGroup; ++h)
                    if (h < G)
                        sv[r][h] = nb < p1 ? __ldcg(reinterpret_cast<const float4 *>(
                                                 s_all + (size_t)(g * G + h) * N + nb))
                                           : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int r = 0; r < kR; ++r) {
                if (it0 + r >= rounds)
                    break;   // uniform: every lane has the same rounds
                const int nb = p0 + 4 * (tid + (it0 + r) * kSelThreads);
                const bool live = nb < p1;
                float sc[4] = {0.f, 0.f, 0.f, 0.f};
                if (live) {
#pragma unroll
                    for (int h = 0; h < kMaxGroup; ++h)
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
            }
        }
    } else {
        const int rounds = (p1 - p0 + kSelThreads - 1) / kSelThreads;
        for (int it = 0; it < rounds; ++it) {
            const int n = p0 + tid + it * kSelThreads;
            float sc = 0.f;
            if (n < p1) {
                for (int h = 0; h < G; ++h)
                    sc += exp2f(__ldcg(s_all + (size_t)(g * G + h) * N + n) - hm[h]) * hw[h];
                imp[n] = sc;
            }
            if (do_hist)
                hist_add(n < p1 && n >= a.n_sink, __float_as_uint(sc));
        }
    }
    if (!do_hist)
        return;
    __syncthreads();
    int *ghist = ws.hist + (size_t)g * kBins0;
    for (int b = tid; b < kBins0; b += kSelThreads)
        if (hist[b] != 0)
            atomicAdd(&ghist[b], hist[b]);
    __threadfence();
    __syncthreads();
    if (tid == 0)
        is_last = atomicAdd(&ws.tick[g], 1) == geo.nc - 1;
    __syncthreads();
    if (!is_last)
        return;
    __threadfence();
    // every chunk of this head has added its histogram: the digit is the
    // bin b with (keys in higher bins) < budget <= (that count + its keys).
    // Thread t holds bins 4095 - 8t .. 4088 - 8t (descending).
    int x[8];
    int sum = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        x[k] = __ldcg(&ghist[kBins0 - 1 - (8 * tid + k)]);
        sum += x[k];
    }
    int above;
    block_exclusive_scan(sum, scan, above);
    if (tid == 0)
        found[0] = -1;
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        if (above < a.budget && a.budget <= above + x[k]) {
            found[0] = kBins0 - 1 - (8 * tid + k);
            found[1] = a.budget - above;
        }
        above += x[k];
    }
    __syncthreads();
    if (tid == 0) {
        ws.info[g].digit0 = found[0];
        ws.info[g].need0 = found[1];
        ws.tick[g] = 0;
    }
    // the histogram is left zero for the next call
    for (int b = tid; b < kBins0; b += kSelThreads)
        ghist[b] = 0;
}

// Kernel 3: per chunk, the candidate keys above the threshold bin are
// counted and those in it are appended (key, position) to the head's list.
__global__ void __launch_bounds__(kSelThreads)
sel_cand_kernel(SelectArgs a, SelGeom geo, SelWs ws)
{
    __shared__ int red[kSelThreads / 32];
    const int c = blockIdx.x, g = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int N = a.n_ctx;
    const int p0 = min(c * geo.chunk, N), p1 = min(p0 + geo.chunk, N);
    const int digit0 = __ldcg(&ws.info[g].digit0);
    const float *imp = ws.imp + (size_t)g * N;
    uint2 *cand = ws.cand + (size_t)g * N;
    int n_above = 0;
    const int rounds = (p1 - p0 + kSelThreads - 1) / kSelThreads;
    for (int it = 0; it < rounds; ++it) {
        const int n = p0 + tid + it * kSelThreads;
        const bool in = n < p1 && n >= a.n_sink;
        const uint32_t key = in ? __float_as_uint(__ldcg(imp + n)) : 0u;
        const int bin = (int)(key >> kShift0);
        n_above += in && bin > digit0;
        const bool hit = in && bin == digit0;
        const unsigned m = __ballot_sync(0xffffffffu, hit);
        if (m) {
            int base = 0;
            if (lane == 0)
                base = atomicAdd(&ws.info[g].n_cand, __popc(m));
            base = __shfl_sync(0xffffffffu, base, 0);
            if (hit)
                cand[base + __popc(m & ((1u << lane) - 1u))] = make_uint2(key, (uint32_t)n);
        }
    }
    n_above = warp_isum(n_above);
    if (lane == 0)
        red[warp] = n_above;
    __syncthreads();
    if (warp == 0) {
        int v = lane < kSelThreads / 32 ? red[lane] : 0;
        v = warp_isum(v);
        if (lane == 0)
            ws.above[(size_t)g * geo.nc + c] = v;
    }
}

// Kernel 4, one CTA per KV head: the exact budget-th largest key among the
// candidates (two radix passes over their low 19 bits), then per chunk the
// number of kept positions before it and of equal-to-threshold keys before
// it, so that each chunk can place its kept positions on its own.
__global__ void __launch_bounds__(kSelThreads)
sel_thresh_kernel(SelectArgs a, SelGeom geo, SelWs ws, int mode)
{
    __shared__ int hist[1024];
    __shared__ int scan[72];
    __shared__ int found[2];
    __shared__ int gtc[kMaxChunks], eqc[kMaxChunks];
    const int g = blockIdx.x;
    const int tid = threadIdx.x;
    const int N = a.n_ctx;
    SelInfo *inf = &ws.info[g];
    uint32_t T = 0xFFFFFFFFu;   // nothing at or above: no candidate kept
    int need_eq = 0;
    int n_cand = 0;
    if (mode == kSelect) {
        n_cand = __ldcg(&inf->n_cand);
        const int digit0 = __ldcg(&inf->digit0);
        int need = __ldcg(&inf->need0);
        const uint2 *cand = ws.cand + (size_t)g * N;
        uint32_t prefix = (uint32_t)digit0 << kShift0;
        uint32_t pmask = 0xFFFFFFFFu << kShift0;
        for (int pass = 0; pass < 2; ++pass) {
            const int shift = pass == 0 ? 9 : 0;
            const int nb = pass == 0 ? 1024 : 512;
            const uint32_t dmask = (uint32_t)nb - 1;
            for (int b = tid; b < 1024; b += kSelThreads)
                hist[b] = 0;
            __syncthreads();
            for (int i = tid; i < n_cand; i += kSelThreads) {
                const uint32_t key = __ldcg(&cand[i].x);
                if ((key & pmask) == prefix)
                    atomicAdd(&hist[(key >> shift) & dmask], 1);
            }
            __syncthreads();
            // thread t holds bins nb-1-2t, nb-2-2t (descending)
            int x0 = 0, x1 = 0;
            if (2 * tid < nb) {
                x0 = hist[nb - 1 - 2 * tid];
                x1 = hist[nb - 2 - 2 * tid];
            }
            int above;
            block_exclusive_scan(x0 + x1, scan, above);
            if (2 * tid < nb) {
                if (above < need && need <= above + x0) {
                    found[0] = nb - 1 - 2 * tid;
                    found[1] = above;
                } else if (above + x0 < need && need <= above + x0 + x1) {
                    found[0] = nb - 2 - 2 * tid;
                    found[1] = above + x0;
                }
            }
            __syncthreads();
            prefix |= (uint32_t)found[0] << shift;
            pmask |= dmask << shift;
            need -= found[1];
            __syncthreads();
        }
        T = prefix;
        need_eq = need;
    }
    // per chunk: candidates above T and equal to T
    for (int i = tid; i < geo.nc; i += kSelThreads) {
        gtc[i] = 0;
        eqc[i] = 0;
    }
    __syncthreads();
    if (mode == kSelect) {
        const uint2 *cand = ws.cand + (size_t)g * N;
        for (int i = tid; i < n_cand; i += kSelThreads) {
            const uint2 kp = __ldcg(&cand[i]);
            const int ch = (int)kp.y / geo.chunk;
            if (kp.x > T)
                atomicAdd(&gtc[ch], 1);
            else if (kp.x == T)
                atomicAdd(&eqc[ch], 1);
        }
    }
    __syncthreads();
    // kept before chunk c: sinks before it, keys above T before it, and of
    // the equal keys the first need_eq in position order.  One chunk per
    // thread (nc <= kMaxChunks <= kSelThreads): scan the equal counts, then
    // the kept counts.
    const int ch = tid;
    const bool live = ch < geo.nc;
    const int my_eq = live && mode == kSelect ? eqc[ch] : 0;
    int eq_before;
    block_exclusive_scan(my_eq, scan, eq_before);
    int k = 0;
    if (live) {
        const int q0 = ch * geo.chunk, q1 = min(q0 + geo.chunk, N);
        if (mode == kKeepAll) {
            k = max(0, q1 - q0);
        } else {
            k = max(0, min(q1, a.n_sink) - q0);
            if (mode == kSelect)
                k += __ldcg(&ws.above[(size_t)g * geo.nc + ch]) + gtc[ch] +
                     max(0, min(need_eq - eq_before, eqc[ch]));
        }
    }
    int kept_before;
    block_exclusive_scan(k, scan, kept_before);
    if (live)
        ws.chunk[(size_t)g * geo.nc + ch] = make_int2(kept_before, eq_before);
    if (tid == 0) {
        inf->T = T;
        inf->need_eq = need_eq;
        inf->n_cand = 0;   // the list is empty again for the next call
    }
}

// Kernel 5: each chunk writes its kept positions in ascending order from
// its offset and copies their K and V rows into the partial cache.
template <int D>
__global__ void __launch_bounds__(kSelThreads)
sel_gather_kernel(SelectArgs a, SelGeom geo, SelWs ws, int mode)
{
    extern __shared__ int list[];   // this chunk's kept positions
    __shared__ int scan[72];
    const int c = blockIdx.x, g = blockIdx.y;
    const int tid = threadIdx.x;
    const int N = a.n_ctx;
    const int p0 = min(c * geo.chunk, N), p1 = min(p0 + geo.chunk, N);
    const int2 ci = __ldcg(&ws.chunk[(size_t)g * geo.nc + c]);
    const uint32_t T = __ldcg(&ws.info[g].T);
    const int need_eq = __ldcg(&ws.info[g].need_eq);
    const float *imp = ws.imp + (size_t)g * N;
    const int64_t want = (int64_t)a.n_sink + a.budget;
    const int n_keep = want < N ? (int)want : N;
    // each thread a contiguous run of the chunk
    const int per = (p1 - p0 + kSelThreads - 1) / kSelThreads;
    const int q0 = p0 + tid * per, q1 = min(q0 + per, p1);
    auto cls = [&](int n) -> int {   // 0 dropped, 1 kept, 2 equal to T
        if (mode == kKeepAll || n < a.n_sink)
            return 1;
        if (mode != kSelect)
            return 0;
        const uint32_t key = __float_as_uint(__ldcg(imp + n));
        return key > T ? 1 : (key == T ? 2 : 0);
    };
    int n_sure = 0, n_eq = 0;
    for (int n = q0; n < q1; ++n) {
        const int k = cls(n);
        n_sure += k == 1;
        n_eq += k == 2;
    }
    int sure_before, eq_before;
    block_exclusive_scan(n_sure, scan, sure_before);
    block_exclusive_scan(n_eq, scan, eq_before);
    // equal keys are kept in position order: the first need_eq of the head
    const int eqb = ci.y + eq_before;
    int slot = sure_before + max(0, min(need_eq, eqb)) - max(0, min(need_eq, ci.y));
    int eq_rank = eqb;
    int32_t *idx = a.idx_out + (size_t)g * n_keep;
    for (int n = q0; n < q1; ++n) {
        const int k = cls(n);
        const bool kept = k == 1 || (k == 2 && eq_rank++ < need_eq);
        if (kept) {
            const int out = ci.x + slot;
            if (out < n_keep) {
                idx[out] = n;
                list[slot] = n;
            } else {
                record_status(reinterpret_cast<WorkspaceHeader *>(a.workspace), TS_ERR_DEVICE_ARG);
            }
            ++slot;
        }
    }
    __syncthreads();
    // rows: the chunk's kept count is the last thread's end slot
    __shared__ int n_rows;
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
    constexpr int kG = 8;   // rows per thread per step, loads in flight together
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
// histogram, tickets, info, per-chunk counts, candidates.
struct SelOffsets {
    size_t s, part, imp, hist, tick, info, above, chunk, cand, total;
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
    o.tick = take((size_t)n_heads_kv * sizeof(int));
    o.info = take((size_t)n_heads_kv * sizeof(SelInfo));
    o.above = take((size_t)n_heads_kv * p.geo.nc * sizeof(int));
    o.chunk = take((size_t)n_heads_kv * p.geo.nc * sizeof(int2));
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
    ws.tick = reinterpret_cast<int *>(w + o.tick);
    ws.info = reinterpret_cast<SelInfo *>(w + o.info);
    ws.above = reinterpret_cast<int *>(w + o.above);
    ws.chunk = reinterpret_cast<int2 *>(w + o.chunk);
    ws.cand = reinterpret_cast<uint2 *>(w + o.cand);
    const int64_t want = (int64_t)a.n_sink + a.budget;
    const int mode = want >= a.n_ctx ? kKeepAll : (a.budget == 0 ? kSinksOnly : kSelect);
    const dim3 grid(p.geo.nc, a.n_heads_kv);

    // scores: the caller's (then their per-chunk statistics here), or the
    // score pass into the workspace (which leaves the statistics itself)
    const float *s_all = a.root_scores;
    cudaError_t e;
    if (score_pass) {
        float *s_ws = reinterpret_cast<float *>(w + o.s);
        e = launch_p1<D>(a, p, s_ws, ws.part, stream);
        if (e != cudaSuccess)
            return e;
        s_all = s_ws;
    } else {
        sel_stats_kernel<<<grid, kSelThreads, 0, stream>>>(a, p.geo, ws);
        if ((e = cudaGetLastError()) != cudaSuccess)
            return e;
        count_launches(1);
    }
    // 16-byte loads and stores when every row starts on a 16-byte boundary
    const int vec = (a.n_ctx & 3) == 0 && reinterpret_cast<uintptr_t>(s_all) % 16 == 0 &&
                    reinterpret_cast<uintptr_t>(ws.imp) % 16 == 0;
    sel_keys_kernel<<<grid, kSelThreads, 0, stream>>>(a, p.geo, ws, s_all, mode, vec);
    if ((e = cudaGetLastError()) != cudaSuccess)
        return e;
    count_launches(1);
    if (mode == kSelect) {
        sel_cand_kernel<<<grid, kSelThreads, 0, stream>>>(a, p.geo, ws);
        if ((e = cudaGetLastError()) != cudaSuccess)
            return e;
        count_launches(1);
    }
    sel_thresh_kernel<<<a.n_heads_kv, kSelThreads, 0, stream>>>(a, p.geo, ws, mode);
    if ((e = cudaGetLastError()) != cudaSuccess)
        return e;
    count_launches(1);
    const size_t list_bytes = (size_t)p.geo.chunk * sizeof(int);
    static const cudaError_t attr = cudaFuncSetAttribute(
        sel_gather_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    if (attr != cudaSuccess)
        return attr;
    sel_gather_kernel<D><<<grid, kSelThreads, list_bytes, stream>>>(a, p.geo, ws, mode);
    if ((e = cudaGetLastError()) != cudaSuccess)
        return e;
    count_launches(1);
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
