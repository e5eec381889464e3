// Self-test of the bounded waits every kernel of the library uses (no counterpart on the
// pages): one CTA waits on an mbarrier that nothing ever completes, with the same helper and
// the same give-up path as the GEMM pipelines, only with a short limit.  The wait runs out,
// raises the shared abort flag and the device error word, and the kernel returns: the context
// stays usable and nvfp4lora_device_status reports NVFP4LORA_ERR_DEVICE_TIMEOUT.
#pragma once

#include <cstdint>

#include "ptx.cuh"

namespace nvfp4lora {

__global__ void __launch_bounds__(32, 1) wait_timeout_selftest_kernel(unsigned long long limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);          // one arrival would complete phase 0; none comes
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, limit_ns);
    __syncthreads();
}

}  // namespace nvfp4lora
