// selftest.cu -- the bounded device-side wait, exercised on purpose (failure detection).
//
// Every wait in the library's kernels is an mbarrier try-wait polled against %globaltimer
// with a deadline; when the deadline passes, the kernel records MOE_ERR_DEVICE_TIMEOUT in
// the workspace status word, drains what it has in flight and returns. This kernel runs the
// same wait on a barrier that nothing ever arrives on, so that tests can check the timeout
// path end to end (status recorded, kernel returns, context usable) without a fault.
#include "common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace moe {
namespace {

__global__ void __launch_bounds__(32) selftest_wait_kernel(int* status, uint64_t ns) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncwarp();
    if (!mbar_wait(&bar, 0, gtimer() + ns) && threadIdx.x == 0) set_status(status, MOE_ERR_DEVICE_TIMEOUT);
}

}  // namespace
}  // namespace moe

extern "C" MOE_API moe_status moe_selftest_bounded_wait(void* ws, int64_t timeout_ns, moe_stream_t stream) {
    if (!ws || timeout_ns <= 0 || timeout_ns > 1000000000) return MOE_ERR_INVALID_ARGUMENT;
    moe::selftest_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(static_cast<int*>(ws), uint64_t(timeout_ns));
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
