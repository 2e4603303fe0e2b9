// selftest.cu -- a kernel whose pipeline wait runs out on purpose, so that the timeout path
// every kernel shares (bounded mbarrier wait -> device error word -> TMEM freed -> clean exit)
// can be exercised on a real GPU without faulting it.  Nothing ever arrives at the barrier it
// waits on; the wait gives up after `limit_ns`, the CTA frees its tensor memory and returns,
// and the context stays usable.
#include "internal.h"
#include "sm100.cuh"

namespace bsa {
namespace {

__global__ void __launch_bounds__(32, 1) wait_timeout_kernel(unsigned* err, uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncwarp();
    tmem_alloc(&tmem_slot, 32);
    tmem_relinquish();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;
    if (threadIdx.x == 0) mbar_wait_slow(&bar, 0, &abort_flag, err, limit_ns);  // never completes
    __syncwarp();
    tc_fence_before();
    tmem_dealloc(tmem, 32);
}

}  // namespace

cudaError_t launch_wait_timeout_selftest(unsigned* err, uint64_t limit_ns, cudaStream_t s) {
    wait_timeout_kernel<<<1, 32, 0, s>>>(err, limit_ns);
    return cudaGetLastError();
}

}  // namespace bsa
