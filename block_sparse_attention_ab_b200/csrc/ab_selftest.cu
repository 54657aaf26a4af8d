// ab_selftest.cu -- test entry points (see include/ab_attn.h): ab_selftest_bounded_wait
// exercises the bounded mbarrier wait that every pipeline of the library relies on,
// without a GPU fault; ab_selftest_force_counter_slot steers the next attention call
// onto a chosen claim slot.
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/ab_attn.h"
#include "ab_device.cuh"
#include "ab_kernels.h"

namespace {

// One CTA of 64 threads: thread 0 initialises an mbarrier expecting one arrival; with
// `complete` set, thread 0 arrives; then every thread waits on phase 0 with the given
// limit, exactly as a pipeline role does. Without the arrival nothing completes the
// phase, the waits give up after limit_ns, raise AB_FLAG_TIMEOUT and return.
__global__ void bounded_wait_kernel(int *flag, int *done, uint64_t limit_ns, int complete)
{
    __shared__ uint64_t bar;
    __shared__ volatile int abort_flag;
    if (threadIdx.x == 0) {
        ab::mbar_init(&bar, 1);
        abort_flag = 0;
        ab::fence_barrier_init();
    }
    __syncthreads();
    if (complete && threadIdx.x == 0) ab::mbar_arrive(&bar);
    const bool ok = ab::mbar_wait(&bar, 0, &abort_flag, flag, limit_ns);
    __syncthreads();
    if (threadIdx.x == 0) *done = ok ? 1 : 2;
}

}  // namespace

extern "C" ab_status ab_selftest_bounded_wait(int limit_us, int complete, int *dev_flag,
                                              int *dev_done, void *stream)
{
    if (!dev_flag || !dev_done) return AB_ERR_NULL;
    if (limit_us < 1 || limit_us > 1000000) return AB_ERR_RANGE;
    bounded_wait_kernel<<<1, 64, 0, (cudaStream_t)stream>>>(
        dev_flag, dev_done, (uint64_t)limit_us * 1000ull, complete ? 1 : 0);
    return ab::status_of(cudaGetLastError());
}

extern "C" ab_status ab_selftest_force_counter_slot(int slot)
{
    if (slot < 0 || slot >= 4096) return AB_ERR_RANGE;
    ab::force_next_counter_slot(slot);
    return AB_OK;
}
