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
// Pass 2 (one 8-CTA cluster per KV head): merges the chunk partials into
//   the softmax max / normaliser of each head, forms
//   score[n] = (1/G) sum_h 2^(s[h,n] - M_h) / Z_h for its slice of
//   positions, keeps the order-preserving bit pattern of every score in
//   shared memory, and finds the budget-th largest candidate exactly with a
//   4 x 8-bit radix select whose histograms are summed over the cluster
//   through distributed shared memory.  Positions are then compacted in
//   ascending order (sinks, every key above the threshold, and the first
//   keys equal to it in position order, so equal scores go to the lower
//   position) and the kept K/V rows are copied with 16-byte loads.
#include <cooperative_groups.h>
#include <math.h>

#include "attn_common.cuh"
#include "sm100.cuh"
#include "ts_internal.cuh"

namespace cg = cooperative_groups;

namespace ts {
namespace {

constexpr int kClusterCtas = 8;
constexpr int kP2Threads = 512;
constexpr int kMaxSlice = 48 * 1024;   // positions per CTA held in shared memory
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

// ------------------------------------------------------------------ pass 2
__device__ __forceinline__ uint32_t order_key(float f)
{
    const uint32_t b = __float_as_uint(f);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// exclusive scan of one int per thread over the block; returns the total
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
        int w = lane < nw ? scratch[lane] : 0;
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

// Radix select of the budget-th largest key in three passes over the
// key bits: 11, 11 and 10 bits from the top.
constexpr int kRadixBins = 2048;
constexpr int kRadixPasses = 3;
__host__ __device__ constexpr int radix_shift(int pass) { return pass == 0 ? 21 : pass == 1 ? 10 : 0; }
__host__ __device__ constexpr uint32_t radix_mask(int pass) { return pass == 2 ? 1023u : 2047u; }

struct alignas(16) P2Shared {
    int hist[2][kRadixBins];   // pass p uses hist[p & 1]
    int scan[72];
    float head_w[kMaxGroup];   // 1 / (G * Z_h)
    float head_m[kMaxGroup];
    float2 slice_ml[kMaxGroup];  // this CTA's (max, sum) per head over its slice
    float2 warp_ml[kP2Threads / 32][kMaxGroup];  // each warp's (max, sum) per head
    int counts[4];             // [0] equal-to-threshold, [1] kept
    int bcast[4];
};

template <int D>
__global__ void __launch_bounds__(kP2Threads, 1)
select_gather_kernel(SelectArgs a, int n_chunks, int slice, const float *__restrict__ s_all)
{
    cg::cluster_group cluster = cg::this_cluster();
    extern __shared__ __align__(16) unsigned char dsm[];
    P2Shared &sh = *reinterpret_cast<P2Shared *>(dsm);
    uint32_t *keys = reinterpret_cast<uint32_t *>(dsm + sizeof(P2Shared));

    const int rank = (int)cluster.block_rank();
    const int n_ranks = (int)cluster.num_blocks();
    const int g = blockIdx.y;
    const int G = a.n_heads_q / a.n_heads_kv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int N = a.n_ctx;
    const int p0 = min(rank * slice, N), p1 = min(p0 + slice, N);
    const int64_t want = (int64_t)a.n_sink + a.budget;
    const bool keep_all = want >= N;
    const int n_keep = keep_all ? N : (int)want;

    const float2 *part = reinterpret_cast<const float2 *>(
        reinterpret_cast<const char *>(a.workspace) + kHeaderBytes +
        (size_t)a.n_heads_q * N * sizeof(float));

    // softmax max / normaliser per head of the group: from the score pass's
    // per-chunk partials, or, for scores given by the caller, from this
    // cluster's own pass over them (each CTA its slice, summed across ranks)
    if (a.root_scores != nullptr) {
        // every thread folds its positions of the slice into a running
        // (max, sum of 2^(s - max)) per head in one pass; then the warp, the
        // CTA and the cluster combine the pairs
        float rm[kMaxGroup], rl[kMaxGroup];
#pragma unroll
        for (int h = 0; h < kMaxGroup; ++h) {
            rm[h] = -INFINITY;
            rl[h] = 0.f;
        }
        auto fold = [](float &m, float &l, float x) {
            if (x > m) {
                l = (m == -INFINITY ? 0.f : l * exp2f(m - x)) + 1.f;
                m = x;
            } else if (x != -INFINITY) {
                l += exp2f(x - m);
            }
        };
        if ((N & 3) == 0) {
            // one head at a time, eight 16-byte loads in flight per thread
            constexpr int kU = 8;
            const int v0 = p0 / 4, v1 = p1 / 4;
#pragma unroll
            for (int h = 0; h < kMaxGroup; ++h) {
                if (h >= G)
                    continue;
                const float4 *row = reinterpret_cast<const float4 *>(s_all + (size_t)(g * G + h) * N);
                for (int vb = v0 + tid; vb < v1; vb += kU * kP2Threads) {
                    float4 sv[kU];
#pragma unroll
                    for (int u = 0; u < kU; ++u) {
                        const int vi = vb + u * kP2Threads;
                        sv[u] = vi < v1 ? __ldcg(row + vi)
                                        : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
                    }
                    float mx = -INFINITY;
#pragma unroll
                    for (int u = 0; u < kU; ++u)
                        mx = fmaxf(mx, fmaxf(fmaxf(sv[u].x, sv[u].y), fmaxf(sv[u].z, sv[u].w)));
                    if (mx == -INFINITY)
                        continue;
                    if (mx > rm[h]) {
                        rl[h] = rm[h] == -INFINITY ? 0.f : rl[h] * exp2f(rm[h] - mx);
                        rm[h] = mx;
                    }
                    float acc = 0.f;
#pragma unroll
                    for (int u = 0; u < kU; ++u)
                        acc += exp2f(sv[u].x - rm[h]) + exp2f(sv[u].y - rm[h]) +
                               exp2f(sv[u].z - rm[h]) + exp2f(sv[u].w - rm[h]);
                    rl[h] += acc;
                }
            }
        } else {
            for (int n = p0 + tid; n < p1; n += kP2Threads)
#pragma unroll
                for (int h = 0; h < kMaxGroup; ++h)
                    if (h < G)
                        fold(rm[h], rl[h], __ldcg(s_all + (size_t)(g * G + h) * N + n));
        }
        // warp: pairwise merge of (m, l)
#pragma unroll
        for (int h = 0; h < kMaxGroup; ++h) {
            if (h >= G)
                continue;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float om = __shfl_xor_sync(0xffffffffu, rm[h], o);
                const float ol = __shfl_xor_sync(0xffffffffu, rl[h], o);
                const float mm = fmaxf(rm[h], om);
                if (mm != -INFINITY) {
                    rl[h] = (rm[h] == -INFINITY ? 0.f : rl[h] * exp2f(rm[h] - mm)) +
                            (om == -INFINITY ? 0.f : ol * exp2f(om - mm));
                    rm[h] = mm;
                }
            }
            if (lane == 0)
                sh.warp_ml[warp][h] = make_float2(rm[h], rl[h]);
        }
        __syncthreads();
        // CTA: one warp per head over the 16 warps' pairs
        if (warp < G) {
            const float2 x = lane < kP2Threads / 32 ? sh.warp_ml[lane][warp]
                                                    : make_float2(-INFINITY, 0.f);
            float m = x.x;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            float l = (m == -INFINITY || x.x == -INFINITY) ? 0.f : x.y * exp2f(x.x - m);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                l += __shfl_xor_sync(0xffffffffu, l, o);
            if (lane == 0)
                sh.slice_ml[warp] = make_float2(m, l);
        }
        cluster.sync();
        if (warp < G) {
            float M = -INFINITY;
            float2 part_r[kClusterCtas];
#pragma unroll
            for (int r = 0; r < kClusterCtas; ++r) {
                part_r[r] = r < n_ranks ? cluster.map_shared_rank(&sh.slice_ml[0], r)[warp]
                                        : make_float2(-INFINITY, 0.f);
                M = fmaxf(M, part_r[r].x);
            }
            float L = 0.f;
#pragma unroll
            for (int r = 0; r < kClusterCtas; ++r)
                if (part_r[r].x != -INFINITY)
                    L += part_r[r].y * exp2f(part_r[r].x - M);
            if (lane == 0) {
                sh.head_m[warp] = M;
                sh.head_w[warp] = 1.f / ((float)G * L);
            }
        }
    } else if (warp < G) {
        const float2 *pp = part + (size_t)(g * G + warp) * n_chunks;
        float M = -INFINITY;
        for (int c = lane; c < n_chunks; c += 32)
            M = fmaxf(M, pp[c].x);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        float L = 0.f;
        for (int c = lane; c < n_chunks; c += 32)
            if (pp[c].x != -INFINITY)
                L += pp[c].y * exp2f(pp[c].x - M);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            L += __shfl_xor_sync(0xffffffffu, L, o);
        if (lane == 0) {
            sh.head_m[warp] = M;
            sh.head_w[warp] = 1.f / ((float)G * L);
        }
    }
    __syncthreads();

    const bool do_select = !keep_all && a.budget > 0;
    // the first radix pass's histogram is built while the keys are formed
    for (int b = tid; b < kRadixBins; b += kP2Threads)
        sh.hist[0][b] = 0;
    __syncthreads();
    // adds one to the pass's bin of each candidate key (positions >= n_sink)
    // whose higher digits match `prefix`; lanes with equal bins add once, by
    // their leader (positive scores share their leading bits, so most lanes
    // of a warp hit the same bin)
    auto hist_add = [&](int *hist, bool in, uint32_t key, uint32_t prefix, uint32_t pmask,
                        int pass) {
        const bool hit = in && (key & pmask) == prefix;
        const unsigned act = __ballot_sync(0xffffffffu, hit);
        if (hit) {
            const uint32_t bin = (key >> radix_shift(pass)) & radix_mask(pass);
            const unsigned same = __match_any_sync(act, bin);
            if (lane == __ffs(same) - 1)
                atomicAdd(&hist[bin], __popc(same));
        }
    };

    // scores of this slice -> order-preserving keys in shared memory
    if ((N & 3) == 0) {
        // four consecutive positions per thread, one 16-byte load per head
        // (the slice is a multiple of 4, so p0 and p1 are too); every lane
        // of a warp runs the same number of rounds
        // two rounds per step, so that 2 G 16-byte loads are in flight
        constexpr int kR = 2;
        const int rounds = (p1 - p0 + 4 * kP2Threads - 1) / (4 * kP2Threads);
        float hm[kMaxGroup], hw[kMaxGroup];
#pragma unroll
        for (int h = 0; h < kMaxGroup; ++h) {
            hm[h] = h < G ? sh.head_m[h] : 0.f;
            hw[h] = h < G ? sh.head_w[h] : 0.f;
        }
        for (int it0 = 0; it0 < rounds; it0 += kR) {
            float4 sv[kR][kMaxGroup];
#pragma unroll
            for (int r = 0; r < kR; ++r) {
                const int nb = p0 + 4 * (tid + (it0 + r) * kP2Threads);
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
                const int nb = p0 + 4 * (tid + (it0 + r) * kP2Threads);
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
                }
                uint32_t kk[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    kk[e] = order_key(sc[e]);
                if (live) {
                    *reinterpret_cast<uint4 *>(&keys[nb - p0]) =
                        make_uint4(kk[0], kk[1], kk[2], kk[3]);
                    if (a.scores_out)
                        *reinterpret_cast<float4 *>(a.scores_out + (size_t)g * N + nb) =
                            make_float4(sc[0], sc[1], sc[2], sc[3]);
                }
                if (do_select)
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        hist_add(sh.hist[0], live && nb + e >= a.n_sink, kk[e], 0u, 0u, 0);
            }
        }
    } else {
        // eight positions per thread per step so their loads are in flight together
        constexpr int kU = 8;
        const int rounds = (p1 - p0 + kP2Threads * kU - 1) / (kP2Threads * kU);
        for (int it = 0; it < rounds; ++it) {
            const int nb = p0 + tid + it * kP2Threads * kU;
            float sc[kU];
#pragma unroll
            for (int u = 0; u < kU; ++u)
                sc[u] = 0.f;
            for (int h = 0; h < G; ++h) {
                const float *row = s_all + (size_t)(g * G + h) * N;
                float sv[kU];
#pragma unroll
                for (int u = 0; u < kU; ++u) {
                    const int n = nb + u * kP2Threads;
                    sv[u] = n < p1 ? __ldcg(row + n) : 0.f;
                }
#pragma unroll
                for (int u = 0; u < kU; ++u)
                    sc[u] += exp2f(sv[u] - sh.head_m[h]) * sh.head_w[h];
            }
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int n = nb + u * kP2Threads;
                const uint32_t key = order_key(sc[u]);
                if (n < p1) {
                    keys[n - p0] = key;
                    if (a.scores_out)
                        a.scores_out[(size_t)g * N + n] = sc[u];
                }
                if (do_select)
                    hist_add(sh.hist[0], n < p1 && n >= a.n_sink, key, 0u, 0u, 0);
            }
        }
    }
    __syncthreads();

    // exact radix select of the budget-th largest key over [n_sink, N):
    // three passes (11, 11, 10 bits), histograms summed over the cluster
    // through distributed shared memory
    uint32_t prefix = 0u, pmask = 0u;
    int need = a.budget;
    if (do_select) {
        const int c0 = max(p0, a.n_sink);
        for (int pass = 0; pass < kRadixPasses; ++pass) {
            int *hist = sh.hist[pass & 1];
            if (pass > 0) {
                // this buffer was last read by other CTAs two passes ago,
                // before they reached the previous pass's cluster barrier
                for (int b = tid; b < kRadixBins; b += kP2Threads)
                    hist[b] = 0;
                __syncthreads();
                for (int nb = c0 - (c0 - p0) % 32; nb < p1; nb += kP2Threads) {
                    const int n = nb + tid;
                    const bool in = n >= c0 && n < p1;
                    hist_add(hist, in, in ? keys[n - p0] : 0u, prefix, pmask, pass);
                }
            }
            cluster.sync();
            // thread t looks at bins 4t .. 4t + 3 from the top (bin
            // 2047 - 4t - k): an exclusive scan over t counts the keys in
            // higher bins; the digit is the bin with (keys above it) < need
            // <= (that count + its own keys)
            const int nbins = (int)radix_mask(pass) + 1;
            int x[4] = {0, 0, 0, 0};
            if (4 * tid < nbins) {
                // bins nbins-4-4t .. nbins-1-4t: one 16-byte read per rank,
                // all ranks' reads in flight together
                const int q = (nbins - 4 - 4 * tid) / 4;
                int4 v[kClusterCtas];
#pragma unroll
                for (int r = 0; r < kClusterCtas; ++r)
                    v[r] = r < n_ranks
                               ? reinterpret_cast<const int4 *>(cluster.map_shared_rank(hist, r))[q]
                               : make_int4(0, 0, 0, 0);
#pragma unroll
                for (int r = 0; r < kClusterCtas; ++r) {
                    x[0] += v[r].w;
                    x[1] += v[r].z;
                    x[2] += v[r].y;
                    x[3] += v[r].x;
                }
            }
            int above;
            block_exclusive_scan(x[0] + x[1] + x[2] + x[3], sh.scan, above);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int b = nbins - 1 - (4 * tid + k);
                if (b >= 0 && above < need && need <= above + x[k]) {
                    sh.bcast[0] = b;
                    sh.bcast[1] = above;
                }
                above += x[k];
            }
            __syncthreads();   // the digit is in bcast
            const int d = sh.bcast[0];
            need -= sh.bcast[1];
            prefix |= (uint32_t)d << radix_shift(pass);
            pmask |= radix_mask(pass) << radix_shift(pass);
            __syncthreads();
        }
    }
    // prefix is now the threshold key; `need` keys equal to it are kept

    // positions of this slice: how many equal the threshold (candidates only)
    const int per_thread = (p1 - p0 + kP2Threads - 1) / kP2Threads;
    const int q0 = p0 + tid * per_thread, q1 = min(q0 + per_thread, p1);
    int my_eq = 0;
    if (do_select)
        for (int n = max(q0, a.n_sink); n < q1; ++n)
            my_eq += keys[n - p0] == prefix;
    int eq_excl;
    const int eq_total = block_exclusive_scan(my_eq, sh.scan, eq_excl);
    if (tid == 0)
        sh.counts[0] = eq_total;
    cluster.sync();
    int eq_before = 0;
    for (int r = 0; r < rank; ++r)
        eq_before += *cluster.map_shared_rank(&sh.counts[0], r);

    // kept flags -> counts -> ascending slots
    auto kept = [&](int n, int &eq_rank) -> bool {
        if (keep_all || n < a.n_sink)
            return true;
        if (!do_select)
            return false;
        const uint32_t key = keys[n - p0];
        if (key > prefix)
            return true;
        if (key == prefix)
            return eq_rank++ < need;
        return false;
    };
    int my_kept = 0;
    {
        int eq_rank = eq_before + eq_excl;
        for (int n = q0; n < q1; ++n)
            my_kept += kept(n, eq_rank);
    }
    int kept_excl;
    const int kept_total = block_exclusive_scan(my_kept, sh.scan, kept_excl);
    if (tid == 0)
        sh.counts[1] = kept_total;
    cluster.sync();
    int kept_before = 0;
    for (int r = 0; r < rank; ++r)
        kept_before += *cluster.map_shared_rank(&sh.counts[1], r);
    cluster.sync();   // no CTA may exit while others read its shared memory

    // write indices; reuse the key slots of kept positions to list them
    int32_t *idx = a.idx_out + (size_t)g * n_keep;
    {
        int eq_rank = eq_before + eq_excl;
        int slot = kept_before + kept_excl;
        for (int n = q0; n < q1; ++n)
            if (kept(n, eq_rank)) {
                if (slot < n_keep)
                    idx[slot] = n;
                else
                    record_status(reinterpret_cast<WorkspaceHeader *>(a.workspace),
                                  TS_ERR_DEVICE_ARG);
                ++slot;
            }
    }
    __syncthreads();

    // gather: kept rows of this slice are idx[kept_before .. kept_before + kept_total)
    constexpr int LPR = D / 8;   // lanes per row, 16 bytes each
    const __nv_bfloat16 *kh = a.k + (int64_t)g * a.kv_cap * D;
    const __nv_bfloat16 *vh = a.v + (int64_t)g * a.kv_cap * D;
    __nv_bfloat16 *kp = a.k_partial + (int64_t)g * a.partial_cap * D;
    __nv_bfloat16 *vp = a.v_partial + (int64_t)g * a.partial_cap * D;
    const int rows_per_pass = kP2Threads / LPR;
    const int li = tid % LPR;
    __threadfence_block();
    const int my_rows = min(kept_total, n_keep - kept_before);
    // eight rows per thread per step: their K and V loads are in flight together
    constexpr int kG = 8;
    for (int t0 = tid / LPR; t0 < my_rows; t0 += rows_per_pass * kG) {
        uint4 kv[kG], vv[kG];
        int slot[kG];
        bool ok[kG];
#pragma unroll
        for (int u = 0; u < kG; ++u) {
            const int t = t0 + u * rows_per_pass;
            slot[u] = kept_before + t;
            const int n = t < my_rows ? __ldcg(&idx[slot[u]]) : -1;
            ok[u] = n >= 0 && n < N;
            const int nn = ok[u] ? n : 0;
            kv[u] = *reinterpret_cast<const uint4 *>(kh + (int64_t)nn * D + li * 8);
            vv[u] = *reinterpret_cast<const uint4 *>(vh + (int64_t)nn * D + li * 8);
        }
#pragma unroll
        for (int u = 0; u < kG; ++u)
            if (ok[u]) {
                *reinterpret_cast<uint4 *>(kp + (int64_t)slot[u] * D + li * 8) = kv[u];
                *reinterpret_cast<uint4 *>(vp + (int64_t)slot[u] * D + li * 8) = vv[u];
            }
    }
}

struct SelPlan {
    int chunk, n_chunks, slice;
};

SelPlan make_sel_plan(int n_heads_kv, int n_ctx, int num_sms)
{
    SelPlan p;
    // three 64 KB-ring CTAs fit an SM: one wave of them over all heads
    // (rounded down, so that no CTA waits for a second wave)
    int want = (num_sms * 3) / n_heads_kv;
    want = want < 1 ? 1 : want;
    const int min_chunk = 512;
    int chunk = (n_ctx + want - 1) / want;
    chunk = chunk < min_chunk ? min_chunk : chunk;
    p.chunk = chunk;
    p.n_chunks = (n_ctx + chunk - 1) / chunk;
    p.slice = ((n_ctx + kClusterCtas - 1) / kClusterCtas + 3) / 4 * 4;
    return p;
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
    dim3 grid(p.n_chunks, a.n_heads_kv);
    score_logits_kernel<D><<<grid, kP1Threads, smem, stream>>>(mk, a, p.chunk, p.n_chunks, s_out,
                                                                part_out);
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess)
        count_launches(1);
    return e;
}

template <int D>
cudaError_t launch_d(const SelectArgs &a, const SelPlan &p, cudaStream_t stream)
{
    // scores from the caller, or the score pass into the workspace
    const float *s_all = a.root_scores;
    cudaError_t e = cudaSuccess;
    if (s_all == nullptr) {
        float *s_ws =
            reinterpret_cast<float *>(reinterpret_cast<char *>(a.workspace) + kHeaderBytes);
        e = launch_p1<D>(a, p, s_ws, reinterpret_cast<float2 *>(s_ws + (size_t)a.n_heads_q * a.n_ctx),
                         stream);
        if (e != cudaSuccess)
            return e;
        s_all = s_ws;
    }

    const size_t smem = sizeof(P2Shared) + (size_t)p.slice * sizeof(uint32_t);
    static const cudaError_t attr_ok = cudaFuncSetAttribute(
        select_gather_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
        (int)(sizeof(P2Shared) + (size_t)kMaxSlice * sizeof(uint32_t)));
    if (attr_ok != cudaSuccess)
        return attr_ok;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kClusterCtas, a.n_heads_kv, 1);
    cfg.blockDim = dim3(kP2Threads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kClusterCtas;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, select_gather_kernel<D>, a, p.n_chunks, p.slice, s_all);
    if (e == cudaSuccess)
        count_launches(1);
    return e;
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
    return ((n_ctx + kClusterCtas - 1) / kClusterCtas + 3) / 4 * 4 <= kMaxSlice;
}

size_t select_workspace_bytes(int n_heads_q, int n_heads_kv, int head_dim, int n_ctx,
                              int num_sms)
{
    (void)head_dim;
    const SelPlan p = make_sel_plan(n_heads_kv, n_ctx, num_sms);
    const size_t s_bytes = (size_t)n_heads_q * n_ctx * sizeof(float);
    const size_t part = (size_t)n_heads_q * p.n_chunks * 2 * sizeof(float);
    return kHeaderBytes + align_up(s_bytes + part, 256);
}

cudaError_t select_launch(const SelectArgs &a, int num_sms, cudaStream_t stream)
{
    const SelPlan p = make_sel_plan(a.n_heads_kv, a.n_ctx, num_sms);
    return a.head_dim == 128 ? launch_d<128>(a, p, stream) : launch_d<64>(a, p, stream);
}

}  // namespace ts
