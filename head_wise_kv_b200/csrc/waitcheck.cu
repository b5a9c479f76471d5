// Diagnostic for the bounded waits: one warp waits on an mbarrier that
// nothing will complete, with the same bounded-wait helper every pipeline
// wait of the attention kernels uses, and on giving up sets
// DUO_STATUS_WAIT_TIMEOUT as their timeout paths do.  It lets a test make a
// wait run out on the device (no fault, no trap, no unbounded spin) and
// check that the status reaches the host and the context stays usable.
#include <cuda_runtime.h>
#include <stdint.h>

#include "duo_internal.cuh"

namespace duo {

namespace {

__global__ void __launch_bounds__(32) wait_check_kernel(int32_t* status, unsigned long long limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(smem_addr(&bar), 1);   // one arrival completes a phase; none comes
        fence_mbar_init();
    }
    __syncwarp();
    int ok = 1;
    if (threadIdx.x == 0) ok = mbar_wait(smem_addr(&bar), 0, limit_ns) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!ok && threadIdx.x == 0) set_status(status, DUO_STATUS_WAIT_TIMEOUT);
}

}  // namespace

cudaError_t launch_wait_check(int32_t* status, unsigned long long limit_ns, cudaStream_t s) {
    wait_check_kernel<<<1, 32, 0, s>>>(status, limit_ns);
    return cudaGetLastError();
}

}  // namespace duo
