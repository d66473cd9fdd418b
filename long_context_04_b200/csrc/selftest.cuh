// Self-test of the device-side failure path: one wait that can never complete.
//
// Every wait in the library's kernels is bounded: after its limit it records
// DEV_TIMEOUT in the per-device status word and the kernel returns, so that the
// host learns of it from la_get_device_status and the context stays usable.  This
// kernel exercises exactly that path with nothing else in flight (no copies, no
// MMAs): thread 0 waits on an mbarrier that nothing arrives on, gives up after the
// limit, records the fault and returns.
#pragma once

#include "la_device.cuh"

namespace la {

__global__ void __launch_bounds__(32) selftest_wait_kernel(unsigned long long limit_ns) {
    __shared__ uint64_t never;
    if (threadIdx.x == 0) {
        mbar_init(&never, 1);
        fence_mbarrier_init_cluster();
    }
    __syncwarp();
    if (threadIdx.x == 0 && !mbar_wait(&never, 0u, nullptr, limit_ns)) record_fault(DEV_TIMEOUT);
    __syncwarp();
}

}  // namespace la
