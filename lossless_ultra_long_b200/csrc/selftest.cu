// selftest.cu -- the bounded device wait, made to run out on purpose
// (ts_selftest_bounded_wait).
//
// Every pipeline wait in the library's kernels (TMA stages, MMA commits,
// softmax hand-offs) is an mbarrier wait bounded by about one second of SM
// clock; when it runs out the kernel records TS_ERR_TIMEOUT in the
// workspace status word, every role leaves its loop and the kernel ends, so
// the context stays usable.  This kernel takes that same wait on a barrier
// that nothing ever completes: one thread, one barrier of count 1, no
// arrival.  It ends after the bound with the status recorded; nothing
// traps, faults or spins without limit.
#include "sm100.cuh"
#include "ts_internal.cuh"

namespace ts {
namespace {

__global__ void __launch_bounds__(32) bounded_wait_selftest_kernel(WorkspaceHeader *ws)
{
    __shared__ uint64_t never;
    __shared__ uint32_t abort_flag;
    if (threadIdx.x == 0) {
        sm100::mbar_init(sm100::smem_addr(&never), 1);
        abort_flag = 0u;
        sm100::fence_mbar_init();
        // phase 0 of `never` would complete on one arrival; none comes
        sm100::wait_bounded(sm100::smem_addr(&never), 0, &abort_flag, ws);
    }
}

}  // namespace

cudaError_t selftest_bounded_wait_launch(void *workspace, cudaStream_t stream)
{
    bounded_wait_selftest_kernel<<<1, 32, 0, stream>>>(
        reinterpret_cast<WorkspaceHeader *>(workspace));
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess)
        count_launches(1);
    return e;
}

}  // namespace ts
