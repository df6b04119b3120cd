// gdla_selftest.cu - GPU self-test of the failure path shared by every
// bounded wait of the kernels: a wait on an mbarrier that nothing arrives on
// runs out, records its site in the device failure word and returns.
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdla.h"
#include "gdla_ptx.cuh"

namespace gdla {

__global__ void __launch_bounds__(32, 1) gdla_selftest_wait_kernel() {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncwarp();
    // Phase 0 never completes (its one expected arrival never comes).
    if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, &abort_flag, GDLA_SELFTEST_SITE);
}

}  // namespace gdla

extern "C" GDLA_API gdla_status_t gdla_selftest_wait_timeout(void *stream) {
    gdla::gdla_selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>();
    return cudaPeekAtLastError() == cudaSuccess ? GDLA_OK : GDLA_ERR_CUDA;
}
