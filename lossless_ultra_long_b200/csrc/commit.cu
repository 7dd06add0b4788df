// commit.cu -- the accepted path's K/V rows become the next context rows
// (ts_kv_commit_path).
//
// After verification the longest valid candidate is kept and the state is
// updated for the next step (tencent article, parallel-verification figure:
// candidates are verified against the full KV cache, the longest valid one
// is kept).  The tree's rows sit at n_ctx + node; the accepted path's rows
// must end up at n_ctx + 0 .. n_ctx + L in path order, so that the next
// step's context is n_ctx + L + 1 rows long and contiguous.  The path is
// read on the device from the acceptance result, so no host round trip is
// needed between acceptance and commit.
//
// Grid (KV head, cache): one CTA moves the L rows of one head of K or of V.
// A row's target n_ctx + j can be another row's source (path [0, 2, 5]:
// row 2 moves to 1 and row 5 to 2), so every moved row is first read into
// shared memory and only then written.  Row j = 0 is the root, already in
// place.  An acceptance result that is not a root path of the tree (L or a
// node out of range, nodes not increasing) moves nothing and records
// TS_ERR_DEVICE_ARG in the workspace status word.
#include "ts_internal.cuh"

namespace ts {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxChunks = TS_MAX_TREE * 16;   // 16-byte chunks of the moved rows (D <= 128)

__global__ void __launch_bounds__(kThreads)
kv_commit_kernel(CommitArgs a)
{
    __shared__ uint4 rows[kMaxChunks];
    __shared__ int path[TS_MAX_TREE];
    __shared__ int len;
    const int tid = threadIdx.x;
    const int g = blockIdx.x;
    __nv_bfloat16 *base = (blockIdx.y ? a.v : a.k) + (int64_t)g * a.kv_cap * a.head_dim;
    if (tid == 0) {
        int L = a.accept[0];
        bool ok = L >= 0 && L < a.n_tree;
        for (int j = 0; ok && j <= L; ++j) {
            const int n = a.accept[2 + j];
            ok = n >= j && n < a.n_tree && (j == 0 ? n == 0 : n > path[j - 1]);
            path[j] = n;
        }
        if (!ok) {
            L = 0;
            if (g == 0 && blockIdx.y == 0)
                record_status(reinterpret_cast<WorkspaceHeader *>(a.workspace),
                              TS_ERR_DEVICE_ARG);
        }
        len = L;
    }
    __syncthreads();
    const int L = len;
    if (L == 0)
        return;
    const int cpr = a.head_dim / 8;   // 16-byte chunks per row
    const int n = L * cpr;            // rows j = 1 .. L
    for (int c = tid; c < n; c += kThreads) {
        const int j = 1 + c / cpr, e = c % cpr;
        rows[c] = *reinterpret_cast<const uint4 *>(base + ((int64_t)a.n_ctx + path[j]) * a.head_dim +
                                                   8 * e);
    }
    __syncthreads();
    for (int c = tid; c < n; c += kThreads) {
        const int j = 1 + c / cpr, e = c % cpr;
        *reinterpret_cast<uint4 *>(base + ((int64_t)a.n_ctx + j) * a.head_dim + 8 * e) = rows[c];
    }
}

}  // namespace

cudaError_t commit_launch(const CommitArgs &a, cudaStream_t stream)
{
    kv_commit_kernel<<<dim3(a.n_heads_kv, 2), kThreads, 0, stream>>>(a);
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess)
        count_launches(1);
    return e;
}

}  // namespace ts
