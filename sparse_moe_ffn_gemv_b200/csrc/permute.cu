// permute.cu -- token permutation into per-expert groups (a3).
//
// A stable counting sort of the T*k slots by expert id: per-chunk histograms,
// an exclusive prefix over experts (and over earlier chunks of the same
// expert), then every slot's destination = its expert's base + the number of
// earlier slots of the same expert. Within a 512-slot step, ranks come from
// warp match masks plus per-warp counts in shared memory, so equal experts keep
// ascending slot order. Also emits the compact list of experts that received
// tokens, which the expert kernels use to skip empty experts.
#include <cuda.h>
#include <cuda_fp16.h>

#include <mutex>

#include "permute_dev.cuh"

namespace moe {

namespace {

constexpr int kPlaceThreads = 512;
constexpr int kPlaceWarps = kPlaceThreads / 32;

__global__ void __launch_bounds__(256) hist_kernel(PermuteArgs a) {
    pdl_begin();
    __shared__ int hist[kPermE];
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    const int64_t s0 = int64_t(blockIdx.x) * a.chunk;
    const int64_t s1 = min(a.S, s0 + a.chunk);
    for (int64_t s = s0 + threadIdx.x; s < s1; s += blockDim.x) {
        const int e = a.idx[s];
        if (e >= 0 && e < a.E) atomicAdd(&hist[e], 1);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < a.E; e += blockDim.x)
        a.chunk_hist[int64_t(e) * a.n_chunks + blockIdx.x] = hist[e];  // expert-major
}

__global__ void __launch_bounds__(kPlaceThreads) place_kernel(PermuteArgs a) {
    pdl_begin();
    __shared__ PlaceSmem<kPlaceThreads> sm;
    place_chunk<kPlaceThreads>(a, blockIdx.x, sm);
}

// Compact list of the experts that hold tokens, from offsets [E + 1]
// (moe_grouped_ffn called with a caller-made permutation).
__global__ void __launch_bounds__(kPlaceThreads) active_kernel(const int32_t* offsets, int E, int32_t* active) {
    pdl_begin();
    __shared__ int flags[kPermE];
    __shared__ int warp_tot[kPlaceWarps + 1];
    const int tid = threadIdx.x;
    const int f = (tid < E && offsets[tid + 1] > offsets[tid]) ? 1 : 0;
    if (tid < E) flags[tid] = f;
    __syncthreads();
    const int n = block_exclusive_scan<kPlaceThreads>(flags, E, warp_tot);
    if (tid < E && f) active[1 + flags[tid]] = tid;
    if (tid == 0) active[0] = n;
}

__global__ void __launch_bounds__(kPlaceThreads) tile_start_kernel(const int32_t* offsets, int E, int bn,
                                                                 int32_t* tile_start) {
    pdl_begin();
    __shared__ int v[kPermE];
    __shared__ int warp_tot[kPlaceWarps + 1];
    const int tid = threadIdx.x;
    if (tid < E) v[tid] = (offsets[tid + 1] - offsets[tid] + bn - 1) / bn;
    __syncthreads();
    const int n = block_exclusive_scan<kPlaceThreads>(v, E, warp_tot);
    if (tid < E) tile_start[tid] = v[tid];
    if (tid == 0) tile_start[E] = n;
}

// One warp per destination row, 16-byte vectors; only sorted positions in [*lo, *hi) when
// those bounds are given (a range of experts). F16: the bf16 rows are written as fp16
// (exact within fp16's range), the token operand of 4-bit affine weights.
template <bool F16>
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint4* __restrict__ src, int vpr,
                                                          const int32_t* __restrict__ sorted_slot, int k,
                                                          int64_t S, uint4* __restrict__ dst,
                                                          const int32_t* lo, const int32_t* hi) {
    pdl_begin();
    const int lane = threadIdx.x & 31;
    const int64_t p = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    if (p >= S || (lo && (p < *lo || p >= *hi))) return;
    const int64_t row = sorted_slot[p] / k;
    const uint4* s = src + row * vpr;
    uint4* d = dst + p * vpr;
    for (int c = lane; c < vpr; c += 32) {
        if constexpr (F16) {
            float f[8];
            unpack8(s[c], f);
            uint32_t h[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                __half2 v = __floats2half2_rn(f[2 * j], f[2 * j + 1]);
                h[j] = *reinterpret_cast<uint32_t*>(&v);
            }
            d[c] = make_uint4(h[0], h[1], h[2], h[3]);
        } else {
            d[c] = s[c];
        }
    }
}

}  // namespace

cudaError_t launch_gather_rows(const void* src, int K, const int32_t* sorted_slot, int k, int64_t S, void* dst,
                               cudaStream_t s, const int32_t* lo, const int32_t* hi, bool to_f16) {
    if (S == 0) return cudaSuccess;
    const int vpr = K * 2 / 16;
    const unsigned grid = unsigned((S * 32 + 255) / 256);
    auto kern = to_f16 ? gather_rows_kernel<true> : gather_rows_kernel<false>;
    const cudaError_t e = launch_pdl(kern, dim3(grid), dim3(256), 0, s, static_cast<const uint4*>(src), vpr, sorted_slot,
                                     k, S, static_cast<uint4*>(dst), lo, hi);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_tile_start(const int32_t* offsets, int E, int tile_bn, int32_t* tile_start, cudaStream_t s) {
    { const cudaError_t e_ = launch_pdl(tile_start_kernel, dim3(1), dim3(kPlaceThreads), 0, s, offsets, E, tile_bn, tile_start); if (e_ != cudaSuccess) return e_; }
    return cudaGetLastError();
}

cudaError_t launch_active_list(const int32_t* offsets, int E, int32_t* active, cudaStream_t s) {
    { const cudaError_t e_ = launch_pdl(active_kernel, dim3(1), dim3(kPlaceThreads), 0, s, offsets, E, active); if (e_ != cudaSuccess) return e_; }
    return cudaGetLastError();
}

cudaError_t launch_permute(const PermuteArgs& a, cudaStream_t s) {
    if (a.S == 0) return cudaSuccess;
    if (a.n_chunks > 1) {
        { const cudaError_t e_ = launch_pdl(hist_kernel, dim3(a.n_chunks), dim3(256), 0, s, a); if (e_ != cudaSuccess) return e_; }
        cudaError_t err = cudaGetLastError();
        if (err != cudaSuccess) return err;
    }
    { const cudaError_t e_ = launch_pdl(place_kernel, dim3(a.n_chunks), dim3(kPlaceThreads), 0, s, a); if (e_ != cudaSuccess) return e_; }
    return cudaGetLastError();
}

// ---------------------------------------------------------------- permutation without a workspace
// Scratch of moe_permute_noalloc: [status word, padded to 256 B][active list, 513 ints,
// padded to 2304 B][per-chunk histograms, 512 experts x 32 chunks, expert-major]. Every GPU that loads
// the library holds it until the process exits.
namespace {
constexpr int kNoAllocMaxSlots = 65536;
constexpr int kNoAllocMaxExperts = kPermE;
constexpr size_t kNoAllocStatus = 0;
constexpr size_t kNoAllocActive = 256;
constexpr size_t kNoAllocHist = 256 + 2304;
constexpr size_t kNoAllocBytes = kNoAllocHist + size_t(kNoAllocMaxSlots / kPermChunk) * kNoAllocMaxExperts * 4;
static_assert(kNoAllocBytes == 68096, "documented size of the fixed scratch");
static_assert((kNoAllocMaxExperts + 1) * 4 <= 2304, "active list fits its region");
}  // namespace

static __device__ __align__(256) unsigned char g_permute_scratch[kNoAllocBytes];

namespace {
// The current context's unique id (0 if no context is current or the driver lacks the call).
unsigned long long current_context_id() {
    using GetCurrentFn = CUresult (*)(CUcontext*);
    using GetIdFn = CUresult (*)(CUcontext, unsigned long long*);
    static GetCurrentFn get_current = nullptr;
    static GetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<GetCurrentFn>(p);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<GetIdFn>(p);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current && get_id && get_current(&ctx) == CUDA_SUCCESS && ctx && get_id(ctx, &id) == CUDA_SUCCESS)
        return id;
    return 0;
}

// Device address of g_permute_scratch on the current device, looked up once per device and
// context: a context created after a device reset gets its address looked up again.
cudaError_t permute_scratch(void** out) {
    constexpr int kMaxDevices = 64;
    static void* addr[kMaxDevices] = {};
    static unsigned long long ctx_of[kMaxDevices] = {};
    static std::mutex mu;
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    const unsigned long long ctx = current_context_id();
    if (!addr[dev] || ctx == 0 || ctx != ctx_of[dev]) {
        void* p = nullptr;
        err = cudaGetSymbolAddress(&p, g_permute_scratch);  // also makes the device's context current
        if (err != cudaSuccess) return err;
        addr[dev] = p;
        ctx_of[dev] = current_context_id();
    }
    *out = addr[dev];
    return cudaSuccess;
}
}  // namespace

}  // namespace moe

extern "C" moe_status moe_permute_noalloc(const moe_config* cfg, const int32_t* topk_idx, int64_t T,
                                          int32_t* expert_offsets, int32_t* sorted_slot, int32_t* slot_pos,
                                          int32_t* device_status, moe_stream_t stream) {
    using namespace moe;
    const moe_status vs = moe_config_validate(cfg);
    if (vs != MOE_OK) return vs;
    if (T < 0) return MOE_ERR_INVALID_ARGUMENT;
    if (T == 0) return MOE_OK;
    if (T * int64_t(cfg->top_k) > kNoAllocMaxSlots || cfg->num_experts > kNoAllocMaxExperts)
        return MOE_ERR_SHAPE_OVERFLOW;
    const void* ptrs[] = {topk_idx, expert_offsets, sorted_slot, slot_pos};
    for (const void* q : ptrs)
        if (!q || (reinterpret_cast<uintptr_t>(q) & 15u)) return MOE_ERR_INVALID_ARGUMENT;
    if (device_status && (reinterpret_cast<uintptr_t>(device_status) & 3u)) return MOE_ERR_INVALID_ARGUMENT;
    void* scratch = nullptr;
    if (permute_scratch(&scratch) != cudaSuccess) return MOE_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    char* base = static_cast<char*>(scratch);
    int* status = device_status ? reinterpret_cast<int*>(device_status) : reinterpret_cast<int*>(base + kNoAllocStatus);
    // the status word must start at zero; histograms and the active list are rewritten in full
    if (!device_status && cudaMemsetAsync(status, 0, sizeof(int), s) != cudaSuccess) return MOE_ERR_CUDA;
    PermuteArgs p;
    p.idx = topk_idx;
    p.S = T * cfg->top_k;
    p.E = cfg->num_experts;
    p.offsets = expert_offsets;
    p.sorted_slot = sorted_slot;
    p.slot_pos = slot_pos;
    p.active = reinterpret_cast<int32_t*>(base + kNoAllocActive);
    p.chunk_hist = reinterpret_cast<int32_t*>(base + kNoAllocHist);
    p.chunk = kPermChunk;
    p.n_chunks = int((p.S + kPermChunk - 1) / kPermChunk);
    p.status = status;
    return launch_permute(p, s) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
