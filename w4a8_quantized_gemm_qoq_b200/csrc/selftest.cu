// qoq_watchdog_selftest: exercises the bounded waits that every pipeline role
// of the GEMM uses, on a device, without any fault: one thread waits on an
// mbarrier phase that never completes, another on a global flag that nothing
// sets. Each wait must give up after its limit and record QOQ_ERR_TIMEOUT
// with its wait site, block and detail in a status block of the same layout
// as the GEMM workspace's status words, after which the kernel returns.
#include <cuda_runtime.h>
#include <stdint.h>

#include "qoq_device.cuh"
#include "qoq_internal.h"

namespace qoq {
namespace {

// status: [0..3] the mbarrier wait's record, [8..11] the flag wait's record,
// [16] the flag that nothing sets.
__global__ void __launch_bounds__(64, 1) watchdog_selftest_kernel(int32_t *status, unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_a, abort_b;
    if (threadIdx.x == 0) {
        abort_a = 0;
        abort_b = 0;
        mbar_init(&bar, 1);   // one arrival expected; none ever comes
        mbar_fence_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const Watchdog wd{&abort_a, status};
        wait_bounded(&bar, 0u, wd, kSiteDequantFull, 1, (uint64_t)limit_ns);
    } else if (threadIdx.x == 32) {
        const Watchdog wd{&abort_b, status + 8};
        wait_flag_bounded(status + 16, wd, 2, (uint64_t)limit_ns);
    }
}

}  // namespace
}  // namespace qoq

extern "C" qoq_status qoq_watchdog_selftest(int32_t *status, int64_t limit_ns, void *stream) {
    if (status == nullptr || limit_ns <= 0 || limit_ns > 2000000000LL) return QOQ_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(status) & 15u) return QOQ_ERR_ALIGNMENT;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(status, 0, 32 * sizeof(int32_t), s) != cudaSuccess) return QOQ_ERR_CUDA;
    qoq::watchdog_selftest_kernel<<<1, 64, 0, s>>>(status, (unsigned long long)limit_ns);
    return cudaGetLastError() == cudaSuccess ? QOQ_OK : QOQ_ERR_CUDA;
}
