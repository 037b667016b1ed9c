// kda_selftest.cuh -- a diagnostic for the failure-reporting path.
//
// Every pipeline wait in the prefill is bounded: when a phase does not
// complete within its limit, the wait gives up, the kernel sets
// KDA_ERR_TIMEOUT in the per-device status word and returns, and the context
// stays usable.  This kernel exercises exactly that, without any fault: its
// single waiting thread uses the same bounded wait on a barrier that nothing
// ever arrives on, with a caller-chosen short limit.
#pragma once

#include "kda_common.cuh"
#include "sm100_ptx.cuh"
#include "../../include/kda.h"

namespace kda {

__global__ void __launch_bounds__(32)
selftest_wait_timeout_kernel(unsigned long long limit_cycles) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        sm100::mbar_init(&bar, 1);
        abort_flag = 0;
        sm100::fence_mbar_init();
    }
    __syncthreads();
    // Phase 0 of a fresh barrier completes only after one arrival; none comes.
    if (threadIdx.x == 0 &&
        !sm100::mbar_wait(&bar, 0, reinterpret_cast<volatile int *>(&abort_flag), limit_cycles))
        raise_error(kErrTimeout);
}

}  // namespace kda

extern "C" KDA_API kda_status kda_selftest_wait_timeout(uint64_t limit_cycles, void *stream) {
    if (limit_cycles == 0 || limit_cycles > (1ull << 32)) return KDA_ERR_INVALID_ARGUMENT;
    kda::selftest_wait_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        (unsigned long long)limit_cycles);
    return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}
