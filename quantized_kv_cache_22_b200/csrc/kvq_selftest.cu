// kvq_selftest.cu -- self-test of the failure-detection primitive the kernels use.
//
// Every wait of the library's kernels is a bounded mbarrier wait
// (mbar_wait_bounded): after its limit of wall time it gives up, the kernel
// records KVQ_ERR_TIMEOUT in the workspace status word, drains and returns, so
// the context stays usable.  This launch runs that primitive on a barrier that
// nothing ever completes, so that the give-up path can be exercised on a GPU
// without a fault, a trap or a hang.
#include "kvq_internal.h"
#include "kvq_ptx.cuh"
#include "../../include/kvq.h"

namespace kvq {
namespace {

__global__ void __launch_bounds__(32) bounded_wait_selftest_kernel(int *status, uint64_t limit_ns)
{
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);        // one arrival expected; none is ever made
        abort_flag = 0;
        fence_mbar_init();
        // phase 0 never completes: the wait gives up after limit_ns
        if (!mbar_wait_bounded(&bar, 0u, &abort_flag, limit_ns)) atomicExch(status, KVQ_ERR_TIMEOUT);
    }
}

}  // namespace

cudaError_t launch_bounded_wait_selftest(int *status, uint64_t limit_ns, cudaStream_t stream)
{
    (void)cudaGetLastError();   // drop a stale, already-reported error of an earlier call
    bounded_wait_selftest_kernel<<<1, 32, 0, stream>>>(status, limit_ns);
    return cudaGetLastError();
}

}  // namespace kvq
