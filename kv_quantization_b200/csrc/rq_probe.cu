// rq_probe.cu -- a self-test of the bounded-wait failure path.
//
// Every mbarrier wait in the tensor-core kernels gives up after a bounded
// number of polls, records kErrTimeout in the library's device error word and
// unwinds (the CTA's threads agree on the failure, free their TMEM and
// return) instead of hanging the GPU.  In a healthy kernel no wait ever runs
// out, so this probe makes one run out on purpose, with nothing else in
// flight: one CTA allocates TMEM, waits with a short limit on an mbarrier no
// thread or copy ever arrives on, unwinds the same way and frees the TMEM.
#include <cstdint>

#include "rq_kernels.h"
#include "sm100.cuh"

namespace rq {

__global__ void __launch_bounds__(64, 1) bounded_wait_probe_kernel(uint32_t polls)
{
    __shared__ __align__(8) uint64_t bar;
    __shared__ uint32_t tmem_slot;
    const int warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);          // expects one arrival; none ever comes
        fence_barrier_init();
    }
    if (warp == 0) tmem_alloc(&tmem_slot, 32);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;
    bool ok = true;
    if (threadIdx.x == 32) ok = mbar_wait_limit(&bar, 0u, polls);
    // uniform unwind: every thread learns of the failure before the TMEM goes
    (void)__syncthreads_or(!ok);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 32);
}

cudaError_t launch_wait_probe(uint32_t polls, cudaStream_t st)
{
    bounded_wait_probe_kernel<<<1, 64, 0, st>>>(polls);
    note_launch("bounded_wait_probe_kernel");
    return cudaGetLastError();
}

}  // namespace rq
