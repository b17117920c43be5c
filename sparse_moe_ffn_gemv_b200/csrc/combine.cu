// combine.cu -- routed/shared combine (a7) and the latent RMSNorm (a8).
//
// Klear PR item 2: y = y_experts * coef[0] + shared * coef[1] (blend); ferrox
// latent_moe.rs: output = routed_out + shared (add), and
// combined = rms_norm(combined) with a [latent] weight before up_proj.
#include <cuda_fp16.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

// Four consecutive routed values of token t, columns 4*c4 .. 4*c4+3: the sum of the
// token's nsum rows (fp32 rows, or bf16 rows as the tensor-core down GEMM writes them).
template <typename RT>
__device__ __forceinline__ float4 load4(const RT* p);
template <> __device__ __forceinline__ float4 load4<float>(const float* p) {
    return *reinterpret_cast<const float4*>(p);
}
template <> __device__ __forceinline__ float4 load4<__nv_bfloat16>(const __nv_bfloat16* p) {
    const uint2 w = *reinterpret_cast<const uint2*>(p);
    return make_float4(bf16lo(w.x), bf16hi(w.x), bf16lo(w.y), bf16hi(w.y));
}

template <typename RT>
__device__ __forceinline__ float4 routed_sum(const RT* __restrict__ rows, int nsum, int64_t t, int64_t c4, int H4) {
    const RT* p = rows + ((t * nsum) * H4 + c4) * 4;
    float4 r = load4<RT>(p);
    for (int j = 1; j < nsum; ++j) {
        const float4 v = load4<RT>(p + int64_t(j) * H4 * 4);
        r.x += v.x; r.y += v.y; r.z += v.z; r.w += v.w;
    }
    return r;
}

// Four consecutive outputs in one vector store: 16 bytes of fp32 or 8 bytes of bf16.
__device__ __forceinline__ void store4(float* o, float4 r) { *reinterpret_cast<float4*>(o) = r; }
__device__ __forceinline__ void store4(__nv_bfloat16* o, float4 r) {
    const __nv_bfloat162 a = __floats2bfloat162_rn(r.x, r.y), b = __floats2bfloat162_rn(r.z, r.w);
    *reinterpret_cast<uint2*>(o) = make_uint2(*reinterpret_cast<const uint32_t*>(&a), *reinterpret_cast<const uint32_t*>(&b));
}

template <typename AT, typename RT>
__global__ void __launch_bounds__(256) combine_kernel(const RT* __restrict__ rows, int nsum,
                                                      const float* __restrict__ s_acc,
                                                      const float* __restrict__ coef, int mode,
                                                      int64_t T, int H, AT* __restrict__ y) {
    pdl_begin();
    const int H4 = H / 4;
    const int64_t n4 = T * H4;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
         i += int64_t(gridDim.x) * blockDim.x) {
        const int64_t t = i / H4;
        float4 r = routed_sum<RT>(rows, nsum, t, i - t * H4, H4);
        if (mode != MOE_SHARED_NONE) {
            const float4 sv = reinterpret_cast<const float4*>(s_acc)[i];
            if (mode == MOE_SHARED_ADD) {
                r.x += sv.x; r.y += sv.y; r.z += sv.z; r.w += sv.w;
            } else {
                const float c0 = coef[2 * t], c1 = coef[2 * t + 1];
                r.x = r.x * c0 + sv.x * c1;
                r.y = r.y * c0 + sv.y * c1;
                r.z = r.z * c0 + sv.z * c1;
                r.w = r.w * c0 + sv.w * c1;
            }
        }
        store4(y + i * 4, r);
    }
}

template <typename AT, typename RT>
__global__ void __launch_bounds__(256) rmsnorm_kernel(const RT* __restrict__ rows, int nsum,
                                                      const AT* __restrict__ gamma, float eps,
                                                      int L, AT* __restrict__ out) {
    pdl_begin();
    extern __shared__ float rsum[];   // the routed sum of this token, L floats
    __shared__ float red[8];
    const int64_t t = blockIdx.x;
    const int L4 = L / 4;
    float ss = 0.f;
    for (int c4 = threadIdx.x; c4 < L4; c4 += blockDim.x) {
        const float4 v = routed_sum<RT>(rows, nsum, t, c4, L4);
        reinterpret_cast<float4*>(rsum)[c4] = v;
        ss = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, ss))));
    }
    const float* row = rsum;
    ss = warp_sum(ss);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) tot += red[w];
    const float inv = rsqrtf(tot / float(L) + eps);
    for (int c = threadIdx.x; c < L; c += blockDim.x)
        out[t * L + c] = from_f<AT>(row[c] * inv * to_f<AT>(gamma[c]));
}

// Eight bf16 values -> eight fp16 values per thread (exact within fp16's range).
__global__ void __launch_bounds__(256) to_f16_kernel(const uint4* __restrict__ src, int64_t n8, uint4* __restrict__ dst) {
    pdl_begin();
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n8; i += int64_t(gridDim.x) * blockDim.x) {
        float f[8];
        unpack8(src[i], f);
        uint32_t h[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            __half2 v = __floats2half2_rn(f[2 * j], f[2 * j + 1]);
            h[j] = *reinterpret_cast<uint32_t*>(&v);
        }
        dst[i] = make_uint4(h[0], h[1], h[2], h[3]);
    }
}

template <typename RT>
cudaError_t launch_combine_t(const RT* rows, int nsum, const float* s_acc, const float* coef, int mode, int64_t T,
                             int H, void* y, int act_dtype, cudaStream_t s, bool out_f32) {
    const int64_t n4 = T * H / 4;
    const unsigned grid = unsigned(std::min<int64_t>((n4 + 255) / 256, 148 * 16));
    cudaError_t e;
    if (act_dtype == kF32 || out_f32)
        e = launch_pdl(combine_kernel<float, RT>, dim3(grid), dim3(256), 0, s, rows, nsum, s_acc, coef, mode, T, H,
                       static_cast<float*>(y));
    else
        e = launch_pdl(combine_kernel<__nv_bfloat16, RT>, dim3(grid), dim3(256), 0, s, rows, nsum, s_acc, coef, mode,
                       T, H, static_cast<__nv_bfloat16*>(y));
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <typename AT, typename RT>
cudaError_t launch_rmsnorm_t(const RT* rows, int nsum, const void* gamma, float eps, int64_t T, int L, void* out,
                             cudaStream_t s) {
    const size_t smem = size_t(L) * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(rmsnorm_kernel<AT, RT>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
    e = launch_pdl(rmsnorm_kernel<AT, RT>, dim3(unsigned(T)), dim3(256), smem, s, rows, nsum,
                   static_cast<const AT*>(gamma), eps, L, static_cast<AT*>(out));
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_combine(const void* rows, int rows_dtype, int nsum, const float* s_acc, const float* coef,
                           int mode, int64_t T, int H, void* y, int act_dtype, cudaStream_t s, bool out_f32) {
    if (T == 0) return cudaSuccess;
    if (rows_dtype == kBF16)
        return launch_combine_t(static_cast<const __nv_bfloat16*>(rows), nsum, s_acc, coef, mode, T, H, y, act_dtype,
                                s, out_f32);
    return launch_combine_t(static_cast<const float*>(rows), nsum, s_acc, coef, mode, T, H, y, act_dtype, s, out_f32);
}

cudaError_t launch_to_f16(const void* src, int64_t n, void* dst, cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    const int64_t n8 = n / 8;
    const unsigned grid = unsigned(std::min<int64_t>((n8 + 255) / 256, 148 * 8));
    const cudaError_t e = launch_pdl(to_f16_kernel, dim3(grid), dim3(256), 0, s, static_cast<const uint4*>(src), n8,
                                     static_cast<uint4*>(dst));
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_rmsnorm(const void* rows, int rows_dtype, int nsum, const void* gamma, float eps, int64_t T,
                           int L, void* out, int act_dtype, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    if (act_dtype == kF32)
        return launch_rmsnorm_t<float>(static_cast<const float*>(rows), nsum, gamma, eps, T, L, out, s);
    if (rows_dtype == kBF16)
        return launch_rmsnorm_t<__nv_bfloat16>(static_cast<const __nv_bfloat16*>(rows), nsum, gamma, eps, T, L, out, s);
    return launch_rmsnorm_t<__nv_bfloat16>(static_cast<const float*>(rows), nsum, gamma, eps, T, L, out, s);
}

}  // namespace moe
