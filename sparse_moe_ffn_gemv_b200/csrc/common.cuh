// common.cuh -- internal helpers shared by the library's CUDA sources.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>

#include <utility>

#include "moe.h"

namespace moe {

constexpr int kWarp = 32;
constexpr int kMaxTopK = 16;
constexpr int kMaxExperts = 512;

// Weight formats / act dtypes (same integers as enum moe_dtype).
constexpr int kF32 = MOE_DTYPE_F32;
constexpr int kBF16 = MOE_DTYPE_BF16;
constexpr int kQ4 = MOE_DTYPE_Q4_AFFINE;
constexpr int kMX4 = MOE_DTYPE_MXFP4;

// ---------------------------------------------------------------- workspace
// Every call carves its scratch out of the caller's workspace at fixed
// 256-byte-aligned offsets that depend only on (config, max_tokens).
struct WsLayout {
    size_t status;       // int32 status word (+ pad)
    size_t logits;       // f32 [T, ld_logits]: E router logits, then 2 coefficient logits
    size_t topk_idx;     // int32 [T, k]
    size_t topk_w;       // f32 [T, k]
    size_t coef;         // f32 [T, 2]
    size_t offsets;      // int32 [E + 1]
    size_t sorted_slot;  // int32 [T * k]
    size_t slot_pos;     // int32 [T * k]
    size_t active;       // int32 [E + 1]: n_active, then the active expert ids
    size_t chunk_hist;   // int32 [E, n_chunks]: slots per expert in each permutation chunk
    size_t h;            // act [T * k, I]: routed intermediate, sorted order
    size_t hs;           // act [T, Is]: shared intermediate
    size_t y_acc;        // f32 [T, K]: routed sum
    size_t s_acc;        // f32 [T, H]: shared expert output
    size_t z;            // act [T, L]: latent input of the experts
    size_t nrm;          // act [T, L]: normalised latent
    size_t tiles;        // int32 tile list of the tensor-core path
    size_t uperm;        // [T * k, K]: routed token rows in sorted order (fp16 for 4-bit affine)
    size_t x16;          // fp16 [T, H]: x as the fp16 token operand (4-bit dense planes)
    size_t n16;          // fp16 [T, L]: the normalised latent likewise
    size_t total;
    int ld_logits;
    int n_chunks;
    int64_t T;
};

// Byte offset, within the workspace's 256-byte status region, of the decode kernel's three
// grid-barrier counters (every launch leaves them at zero).
constexpr size_t kDecodeBarOffset = 16;
// ... and of the counter the grid-barrier self test waits on.
constexpr size_t kSelftestBarOffset = 32;

constexpr int kPermChunk = 2048;   // slots per permutation chunk (fixed-scratch permutation)
constexpr int kPermChunkWs = 2048;  // slots per chunk when the workspace holds the histograms (512 measured slower)

inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }
inline int act_bytes(const moe_config& c) { return c.act_dtype == kF32 ? 4 : 2; }
inline int expert_in(const moe_config& c) { return c.latent_dim ? c.latent_dim : c.hidden; }

// Upper bound of tensor-core tiles for the routed gate/up and down GEMMs.
int64_t max_routed_tiles(const moe_config& c, int64_t T);

WsLayout ws_layout(const moe_config& c, int64_t T);

// ---------------------------------------------------------------- device helpers
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ void unpack8(const uint4 v, float (&f)[8]) {
    f[0] = bf16lo(v.x); f[1] = bf16hi(v.x); f[2] = bf16lo(v.y); f[3] = bf16hi(v.y);
    f[4] = bf16lo(v.z); f[5] = bf16hi(v.z); f[6] = bf16lo(v.w); f[7] = bf16hi(v.w);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

template <typename AT> __device__ __forceinline__ float to_f(AT v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) {
    return __bfloat162float(v);
}
template <typename AT> __device__ __forceinline__ AT from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}

// MXFP4 (OCP Microscaling Formats v1.0). An E2M1 code's exponent and mantissa bits, placed
// at the bottom of a float's exponent field, give exactly the element value times 2^-126
// (exponent field 0 is the format's subnormal, and so it is for the float): one exact
// multiply restores it. The E8M0 block scale byte s is 2^(s - 127).
__device__ __forceinline__ float e2m1_value(uint32_t code) {
    const float mag = __uint_as_float((code & 7u) << 22) * 0x1p126f;
    return __uint_as_float(__float_as_uint(mag) | ((code & 8u) << 28));
}
__device__ __forceinline__ float e8m0_value(uint32_t s) {
    return __uint_as_float(s ? (s << 23) : 0x00400000u);  // 255 (NaN in the format) -> inf
}

// SwiGLU / clamped SwiGLU on fp32 pre-activations.
__device__ __forceinline__ float act_apply(int act, float g, float v, float limit, float alpha) {
    if (act == MOE_ACT_SWIGLU) return g / (1.0f + expf(-g)) * v;
    float gc = fminf(g, limit);
    float vc = fminf(fmaxf(v, -limit), limit);
    return gc / (1.0f + expf(-alpha * gc)) * (vc + 1.0f);
}

// Programmatic dependent launch: every kernel first lets the next kernel in the stream
// begin launching, then waits until the previous kernel's results are complete and
// visible. Touching no memory before the wait keeps plain stream-order semantics while the
// launch latency of each kernel overlaps the tail of the one before.
__device__ __forceinline__ void pdl_begin() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Sticky device status word (first error wins).
__device__ __forceinline__ void set_status(int* status, int code) {
    if (status) atomicCAS(status, 0, code);
}

// Host: launch a kernel that begins with pdl_begin(); programmatic dependent launch is
// allowed only when MOE_PDL=1 (it measured slower here: dependents holding SM resources
// while they wait delay the previous kernel's tail).
inline bool pdl_enabled() {  // measured slower on B200 for these kernels: off unless MOE_PDL=1
    const char* e = getenv("MOE_PDL");
    return e && e[0] == '1';
}
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

}  // namespace moe
