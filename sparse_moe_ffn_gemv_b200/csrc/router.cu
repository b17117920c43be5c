// router.cu -- scoring, select-only bias, top-k and combine weights (a2): one warp per token.
#include "topk_dev.cuh"

namespace moe {

namespace {

__global__ void __launch_bounds__(256) topk_kernel(TopkArgs a) {
    pdl_begin();
    const int64_t t = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    if (t < a.T) topk_token(a, t);
}

}  // namespace

cudaError_t launch_topk(const TopkArgs& a, cudaStream_t s) {
    if (a.T == 0) return cudaSuccess;
    const int64_t threads = a.T * 32;
    const unsigned grid = unsigned((threads + 255) / 256);
    { const cudaError_t e_ = launch_pdl(topk_kernel, dim3(grid), dim3(256), 0, s, a); if (e_ != cudaSuccess) return e_; }
    return cudaGetLastError();
}

}  // namespace moe
