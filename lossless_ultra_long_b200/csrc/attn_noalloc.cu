// attn_noalloc.cu -- ts_tree_verify_attn_noalloc: tree-verify attention for
// callers that cannot allocate device memory; ts_noalloc_status, which
// reads the device-side status those calls leave; and ts_noalloc_selftest,
// the failure-detection self-test on that scratch.
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
// a device once the library's module is loaded there; it is then held until
// the process exits.  Like every workspace it starts with the 256-byte
// header whose first word collects device-side errors (a bounded wait that
// ran out, for one).  The caller cannot see the array, so ts_noalloc_status
// reads that word for it; each call clears the rest of the header but keeps
// the word, so an error stays visible until the caller clears it.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "ts_internal.cuh"

namespace {

__device__ __align__(256) unsigned char g_noalloc_scratch[TS_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 128;
std::mutex g_mu;
struct Slot {
    unsigned long long ctx_id;   // context the address belongs to (0: none yet)
    void *ptr;
};
Slot g_slot[kMaxDevices] = {};

// The current context's process-unique id (cuCtxGetId), or 0 when the
// driver cannot say; an id is never reused, so a context created after a
// cudaDeviceReset gets a new one.
unsigned long long current_context_id()
{
    static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
    static PFN_cuCtxGetId_v12000 get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 4000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
        p = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx ||
        get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

// Device address of the scratch array on the current device.  In host code
// the array's name is only a host-side stand-in, so the address is looked up
// with cudaGetSymbolAddress, with the device current, once per device and
// context (again after the device's context was reset).
cudaError_t scratch_address(void **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= kMaxDevices)
        return cudaErrorInvalidDevice;
    // 0 before the device's context exists: then the lookup below creates
    // it, and the next call records its id
    const unsigned long long id = current_context_id();
    std::lock_guard<std::mutex> lock(g_mu);
    Slot &slot = g_slot[dev];
    if (!slot.ptr || id == 0 || slot.ctx_id != id) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess)
            return e;
        slot.ptr = p;
        slot.ctx_id = id;
    }
    *out = slot.ptr;
    return cudaSuccess;
}

}  // namespace

extern "C" int ts_tree_verify_attn_noalloc(const void *q, const void *k_cache,
                                           const void *v_cache, int64_t kv_cap, int n_heads_q,
                                           int n_heads_kv, int head_dim, int n_ctx, int n_tree,
                                           const int32_t *parent, float softmax_scale,
                                           float *out, void *stream)
{
    // everything is checked on the host before anything is queued
    const int st = ts::attn_validate(q, k_cache, v_cache, kv_cap, n_heads_q, n_heads_kv,
                                     head_dim, n_ctx, n_tree, parent, softmax_scale, out);
    if (st != TS_OK)
        return st;
    const size_t need =
        ts_tree_verify_attn_workspace_size(n_heads_q, n_heads_kv, head_dim, n_ctx, n_tree);
    if (need == 0)
        return TS_ERR_INVALID_ARG;
    if (need > (size_t)TS_NOALLOC_SCRATCH_BYTES)
        return TS_ERR_SCRATCH_LIMIT;
    void *scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) {
        cudaGetLastError();
        return TS_ERR_CUDA;
    }
    // the array keeps the previous call's contents: the hand-off tickets
    // and the kernel's counters must start at zero; the status word is kept
    // until the caller clears it
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t zeroed = ts::attn_workspace_zeroed_bytes(n_heads_q, n_heads_kv, head_dim, n_ctx,
                                                          n_tree, ts::current_num_sms());
    if (cudaMemsetAsync(static_cast<unsigned char *>(scratch) + sizeof(uint32_t), 0,
                        zeroed - sizeof(uint32_t), s) != cudaSuccess) {
        cudaGetLastError();
        return TS_ERR_CUDA;
    }
    return ts_tree_verify_attn(q, k_cache, v_cache, kv_cap, n_heads_q, n_heads_kv, head_dim,
                               n_ctx, n_tree, parent, softmax_scale, out, scratch,
                               (size_t)TS_NOALLOC_SCRATCH_BYTES, stream);
}

extern "C" int ts_noalloc_status(void *stream, int clear)
{
    void *scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) {
        cudaGetLastError();
        return TS_ERR_CUDA;
    }
    return ts_workspace_status(scratch, stream, clear);
}

extern "C" int ts_noalloc_selftest(void *stream)
{
    void *scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) {
        cudaGetLastError();
        return TS_ERR_CUDA;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // leave the hand-off tickets non-zero, as a call that ended early on the
    // device could, then let the bounded wait run out on the array's header
    if (cudaMemsetAsync(static_cast<unsigned char *>(scratch) + sizeof(uint32_t), 0xFF,
                        ts::kHeaderBytes - sizeof(uint32_t), s) != cudaSuccess ||
        ts::selftest_bounded_wait_launch(scratch, s) != cudaSuccess) {
        cudaGetLastError();
        return TS_ERR_CUDA;
    }
    return TS_OK;
}
