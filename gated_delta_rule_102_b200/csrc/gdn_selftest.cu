// Self-test of the bounded waits every kernel of the library uses: one thread waits on
// an mbarrier phase that nothing completes, with a short limit, and must give up and
// report GDN_DEVICE_ERR_TIMEOUT through the error flag, leaving the context usable. No
// copy is in flight and the wait ends by construction (it is bounded by the SM's cycle
// counter), so the failure is made without faulting or hanging the GPU.
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdn_device.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

__global__ void wait_timeout_selftest_kernel(uint64_t limit_cycles, int32_t* err_flag, unsigned long long* cycles) {
    __shared__ uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);  // one arrival expected; none is ever made
    mbar_init_fence();
    const long long t0 = clock64();
    const bool ok = mbar_wait_bounded(&bar, 0, limit_cycles);
    if (cycles) *cycles = (unsigned long long)(clock64() - t0);
    if (!ok && err_flag) atomicOr(err_flag, GDN_DEVICE_ERR_TIMEOUT_BIT);
}

}  // namespace

cudaError_t launch_wait_selftest(uint64_t limit_cycles, int32_t* err_flag, unsigned long long* cycles,
                                 cudaStream_t stream) {
    wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(limit_cycles, err_flag, cycles);
    return cudaGetLastError();
}

}  // namespace gdn
