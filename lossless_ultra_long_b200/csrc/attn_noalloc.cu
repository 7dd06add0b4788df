// attn_noalloc.cu -- ts_tree_verify_attn_noalloc: tree-verify attention for
// callers that cannot allocate device memory.
//
// Some callers may not call cudaMalloc (or any allocating routine) at the
// point where they run attention: code running under a memory manager that
// owns every device allocation (a plugin inside another runtime, an
// inference server with a fixed pre-planned budget), or code on a path that
// must never block on the allocator.  They still own inputs and outputs,
// but cannot provide the split-KV scratch (the workspace) that
// ts_tree_verify_attn takes.  This entry point supplies that scratch from a
// file-scope device array of fixed size instead.
//
// The array lives in this translation unit only, so its memory is taken on
// a device only once the library's module for this file is loaded there
// (first use of this entry point); it is then held until the process exits.
#include <mutex>

#include "ts_internal.cuh"

namespace {

__device__ __align__(256) unsigned char g_noalloc_scratch[TS_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 128;
std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  In host code
// the array's name is only a host-side stand-in, so the address is looked up
// once per device with cudaGetSymbolAddress and cached.
cudaError_t scratch_address(void **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= kMaxDevices)
        return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess)
            return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" int ts_tree_verify_attn_noalloc(const void *q, const void *k_cache,
                                           const void *v_cache, int64_t kv_cap, int n_heads_q,
                                           int n_heads_kv, int head_dim, int n_ctx, int n_tree,
                                           const int32_t *parent, float softmax_scale,
                                           float *out, void *stream)
{
    const size_t need =
        ts_tree_verify_attn_workspace_size(n_heads_q, n_heads_kv, head_dim, n_ctx, n_tree);
    if (need > (size_t)TS_NOALLOC_SCRATCH_BYTES)
        return TS_ERR_SCRATCH_LIMIT;
    void *scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) {
        cudaGetLastError();
        return TS_ERR_CUDA;
    }
    // the array keeps the previous call's contents: the header (status word
    // and hand-off tickets) must start at zero
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(scratch, 0, ts::kHeaderBytes, s) != cudaSuccess) {
        cudaGetLastError();
        return TS_ERR_CUDA;
    }
    return ts_tree_verify_attn(q, k_cache, v_cache, kv_cap, n_heads_q, n_heads_kv, head_dim,
                               n_ctx, n_tree, parent, softmax_scale, out, scratch,
                               (size_t)TS_NOALLOC_SCRATCH_BYTES, stream);
}
