// Diagnostic kernel for tests of the failure path (moe_debug_wait_timeout).
//
// Every pipeline in this library waits on mbarriers with a bounded wait that
// gives up after about a second and records MOE_ERR_TIMEOUT in the pack's
// error word.  This kernel is such a wait whose producer never delivers: one
// thread waits on an mbarrier that nothing arrives on, through the same
// helper, and records the timeout when it gives up.  It issues no copies and
// no tensor-core work, so it has nothing to drain, and the context stays
// usable for the forwards that follow.
#include <cuda_runtime.h>

#include "moe_internal.cuh"
#include "tc_common.cuh"

namespace moe {
namespace {

__global__ void __launch_bounds__(32) wait_probe_kernel(int32_t *err)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    tc::mbar_init(&bar, 1);  // one expected arrival, which never comes
    tc::fence_mbar_init();
    if (!tc::mbar_wait(&bar, 0)) atomicExch(err, (int)MOE_ERR_TIMEOUT);
}

}  // namespace

cudaError_t launch_wait_probe(int32_t *err, cudaStream_t s)
{
    wait_probe_kernel<<<1, 32, 0, s>>>(err);
    return cudaGetLastError();
}

}  // namespace moe
