// selftest.cu -- the bounded device-side waits, exercised on purpose (failure detection).
//
// Every wait in the library's kernels is polled against %globaltimer with a deadline: an
// mbarrier try-wait (tensor-core kernel) or an acquire load of a grid-barrier counter (the
// persistent decode kernel). When the deadline passes, the kernel records
// MOE_ERR_DEVICE_TIMEOUT in the workspace status word, drains what it has in flight and
// returns. These kernels run the same waits on a barrier that can never complete, so that
// tests can check the timeout path end to end (status recorded, kernel returns, context
// usable) without a fault.
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

// One block arrives at a grid barrier that needs two arrivals: the wait gives up at the
// deadline and records the timeout; the counter is put back to zero afterwards.
__global__ void __launch_bounds__(32) selftest_grid_kernel(int* status, unsigned* ctr, uint64_t ns) {
    __shared__ int flag;
    grid_barrier(ctr, 2u, gtimer() + ns, status, &flag);
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        *ctr = 0;
    }
}

}  // namespace
}  // namespace moe

extern "C" MOE_API moe_status moe_selftest_bounded_wait(void* ws, int64_t timeout_ns, moe_stream_t stream) {
    if (!ws || timeout_ns <= 0 || timeout_ns > 1000000000) return MOE_ERR_INVALID_ARGUMENT;
    moe::selftest_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(static_cast<int*>(ws), uint64_t(timeout_ns));
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" MOE_API moe_status moe_selftest_grid_wait(void* ws, int64_t timeout_ns, moe_stream_t stream) {
    if (!ws || timeout_ns <= 0 || timeout_ns > 1000000000) return MOE_ERR_INVALID_ARGUMENT;
    char* base = static_cast<char*>(ws);
    moe::selftest_grid_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(
        reinterpret_cast<int*>(base), reinterpret_cast<unsigned*>(base + moe::kSelftestBarOffset), uint64_t(timeout_ns));
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
