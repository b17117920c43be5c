// gemv.cu -- weight-streaming expert and projection kernels for small batches.
//
// When a group holds few tokens (decode-sized batches), the block is bound by
// reading each activated weight once from HBM. These kernels stream weight
// rows with 16-byte non-allocating loads (one warp per output row, several
// loads in flight per lane), keep the group's tokens in shared memory, and
// accumulate in fp32 on the CUDA cores. Tensor cores would idle at these
// shapes.
//
// Expert shape: down(act(gate(u), up(u))) with [out, in] weights (ferrox
// KimiExpertWeights::forward); gate_up applied then down weighted by the
// routing weights and summed per token (libmir-metal execute, Native arm:
// mxfp4_gate_up then mxfp4_down with routing.weights); 4-bit affine planes
// dequantised on the fly, w = scale * q + bias per group (mlxcel issue #974).
#include <algorithm>

#include "gemv_dev.cuh"

namespace moe {

namespace {

constexpr int kRowsPerBlock = 8;  // one warp per weight row / intermediate unit
constexpr int kThreads = kRowsPerBlock * 32;

template <typename AT>
__device__ __forceinline__ float ld_act(const void* p, int64_t i) {
    return to_f<AT>(reinterpret_cast<const AT*>(p)[i]);
}

// One block of 8 intermediate units of one group: h[p, i] = act(gate_i . u_p, up_i . u_p).
template <int WF>
__device__ void gateup_group(const GateUpArgs& a, bool shared, int e, int unit0, int64_t p0,
                             int64_t cnt, int K, int I, typename Fmt<WF>::AT* us, float* xsum) {
    using AT = typename Fmt<WF>::AT;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i = unit0 + warp;
    const bool live = i < I;
    const char* rows[2];
    QRow q[2] = {{nullptr, nullptr, nullptr}, {nullptr, nullptr, nullptr}};
    const int64_t rb = row_bytes<WF>(K);
    if (shared) {
        rows[0] = reinterpret_cast<const char*>(a.sg_w) + int64_t(live ? i : 0) * rb;
        rows[1] = reinterpret_cast<const char*>(a.su_w) + int64_t(live ? i : 0) * rb;
        if constexpr (WF == kQ4) {  // 4-bit shared planes
            const int64_t ng = K / a.s_group, r0 = live ? i : 0;
            q[0] = {reinterpret_cast<const __nv_bfloat16*>(a.sg_s) + r0 * ng,
                    reinterpret_cast<const __nv_bfloat16*>(a.sg_z) + r0 * ng, nullptr};
            q[1] = {reinterpret_cast<const __nv_bfloat16*>(a.su_s) + r0 * ng,
                    reinterpret_cast<const __nv_bfloat16*>(a.su_z) + r0 * ng, nullptr};
        }
    } else if (a.interleaved) {  // one plane: rows 2i (gate) and 2i + 1 (up), companions alike
        const int64_t r0 = int64_t(e) * 2 * I + 2 * int64_t(live ? i : 0);
        rows[0] = reinterpret_cast<const char*>(a.gate_up_w) + r0 * rb;
        rows[1] = rows[0] + rb;
        if constexpr (WF == kQ4) {
            const int64_t ng = K / a.group_size;
            q[0] = {reinterpret_cast<const __nv_bfloat16*>(a.gate_s) + r0 * ng,
                    reinterpret_cast<const __nv_bfloat16*>(a.gate_z) + r0 * ng, nullptr};
            q[1] = {q[0].s + ng, q[0].z + ng, nullptr};
        } else if constexpr (WF == kMX4) {
            q[0] = {nullptr, nullptr, reinterpret_cast<const uint8_t*>(a.gate_s) + r0 * (K / 32)};
            q[1] = {nullptr, nullptr, q[0].e8 + K / 32};
        }
    } else {
        const int64_t r0 = int64_t(e) * I + (live ? i : 0);
        rows[0] = reinterpret_cast<const char*>(a.gate_w) + r0 * rb;
        rows[1] = reinterpret_cast<const char*>(a.up_w) + r0 * rb;
        if constexpr (WF == kQ4) {
            const int64_t ng = K / a.group_size;
            q[0] = {reinterpret_cast<const __nv_bfloat16*>(a.gate_s) + r0 * ng,
                    reinterpret_cast<const __nv_bfloat16*>(a.gate_z) + r0 * ng, nullptr};
            q[1] = {reinterpret_cast<const __nv_bfloat16*>(a.up_s) + r0 * ng,
                    reinterpret_cast<const __nv_bfloat16*>(a.up_z) + r0 * ng, nullptr};
        } else if constexpr (WF == kMX4) {
            q[0] = {nullptr, nullptr, reinterpret_cast<const uint8_t*>(a.gate_s) + r0 * (K / 32)};
            q[1] = {nullptr, nullptr, reinterpret_cast<const uint8_t*>(a.up_s) + r0 * (K / 32)};
        }
    }
    float bg = 0.f, bu = 0.f;
    if (!shared && a.has_bias && live) {
        if (a.interleaved) {
            bg = ld_act<AT>(a.gate_up_b, int64_t(e) * 2 * I + 2 * i);
            bu = ld_act<AT>(a.gate_up_b, int64_t(e) * 2 * I + 2 * i + 1);
        } else {
            bg = ld_act<AT>(a.gate_b, int64_t(e) * I + i);
            bu = ld_act<AT>(a.up_b, int64_t(e) * I + i);
        }
    }
    const void* src = shared ? a.xs : a.u;
    AT* dst = reinterpret_cast<AT*>(shared ? a.hs : a.h);
    for (int64_t c = 0; c < cnt; c += kTT) {
        const int tt = int(cnt - c < kTT ? cnt - c : kTT);
        __syncthreads();
        stage_tokens<WF>(src, K, p0 + c, tt, shared ? nullptr : a.sorted_slot, a.k, us, xsum);
        __syncthreads();
        if (!live) continue;
        float acc[2][kTT];
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
            for (int t = 0; t < kTT; ++t) acc[r][t] = 0.f;
        dot_rows<WF, 2>(rows, q, K, shared ? a.s_group : a.group_size, us, xsum, tt, acc);
        reduce_acc<WF>(acc, 2, tt);
#pragma unroll
        for (int t = 0; t < kTT; ++t) {
            if (t < tt && lane == t)
                dst[(p0 + c + t) * I + i] = from_f<AT>(act_apply(a.act, acc[0][t] + bg, acc[1][t] + bu,
                                                                 a.limit, a.alpha));
        }
    }
}

template <int WF>
__device__ __forceinline__ void gateup_blocks(const GateUpArgs& a) {
    pdl_begin();
    constexpr int WFD = is_4bit<WF>() ? kBF16 : WF;  // the shared expert is dense
    using AT = typename Fmt<WF>::AT;
    extern __shared__ uint4 smem_raw[];
    AT* us = reinterpret_cast<AT*>(smem_raw);
    const int sblocks = a.shared_I ? (a.shared_I + kRowsPerBlock - 1) / kRowsPerBlock : 0;
    int b = blockIdx.x;
    if (b < sblocks) {
        if constexpr (WF != kF32) {
            if (a.sg_s) {  // 4-bit shared planes
                gateup_group<kQ4>(a, true, -1, b * kRowsPerBlock, 0, a.T, a.Hs, a.shared_I, us,
                                  reinterpret_cast<float*>(us + int64_t(kTT) * a.Hs));
                return;
            }
        }
        gateup_group<WFD>(a, true, -1, b * kRowsPerBlock, 0, a.T, a.Hs, a.shared_I, us, nullptr);
        return;
    }
    b -= sblocks;
    const int ublocks = (a.I + kRowsPerBlock - 1) / kRowsPerBlock;
    const int ai = b / ublocks;
    if (ai >= a.active[0]) return;
    const int e = a.active[1 + ai];
    const int64_t p0 = a.offsets[e];
    const int64_t cnt = a.offsets[e + 1] - p0;
    float* xsum = reinterpret_cast<float*>(us + int64_t(kTT) * a.K);
    gateup_group<WF>(a, false, e, (b - ai * ublocks) * kRowsPerBlock, p0, cnt, a.K, a.I, us, xsum);
}

template <int WF>
__global__ void __launch_bounds__(kThreads) gateup_gemv_kernel(GateUpArgs a) { gateup_blocks<WF>(a); }
// 4-bit affine weights: the word-at-a-time dequantisation fits three blocks per SM (80
// registers), which measured faster for single-token decode than two without the bound.
__global__ void __launch_bounds__(kThreads, 3) gateup_gemv_q4_kernel(GateUpArgs a) { gateup_blocks<kQ4>(a); }
template <int WF> constexpr void (*gateup_kernel())(GateUpArgs) {
    if constexpr (WF == kQ4) return &gateup_gemv_q4_kernel;
    else return &gateup_gemv_kernel<WF>;
}

// One block of 8 * NR output rows of one group's down projection, NR rows per warp.
template <int WF, int NR>
__device__ void down_group(const DownArgs& a, bool shared, int e, int row0, int64_t p0, int64_t cnt,
                           int I, int R, typename Fmt<WF>::AT* us, float* xsum) {
    using AT = typename Fmt<WF>::AT;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rbase = row0 + warp * NR;
    const int64_t rb = row_bytes<WF>(I);
    const char* rows[NR];
    QRow q[NR];
    float bd[NR];
    bool live[NR];
#pragma unroll
    for (int i = 0; i < NR; ++i) {
        const int r = rbase + i;
        live[i] = r < R;
        q[i] = {nullptr, nullptr, nullptr};
        bd[i] = 0.f;
        if (shared) {
            rows[i] = reinterpret_cast<const char*>(a.sd_w) + int64_t(live[i] ? r : 0) * rb;
            if constexpr (WF == kQ4) {  // 4-bit shared down plane
                const int64_t ng = I / a.s_group;
                q[i] = {reinterpret_cast<const __nv_bfloat16*>(a.sd_s) + int64_t(live[i] ? r : 0) * ng,
                        reinterpret_cast<const __nv_bfloat16*>(a.sd_z) + int64_t(live[i] ? r : 0) * ng, nullptr};
            }
        } else {
            const int64_t gr = int64_t(e) * R + (live[i] ? r : 0);
            rows[i] = reinterpret_cast<const char*>(a.down_w) + gr * rb;
            if constexpr (WF == kQ4) {
                const int64_t ng = I / a.group_size;
                q[i] = {reinterpret_cast<const __nv_bfloat16*>(a.down_s) + gr * ng,
                        reinterpret_cast<const __nv_bfloat16*>(a.down_z) + gr * ng, nullptr};
            } else if constexpr (WF == kMX4) {
                q[i] = {nullptr, nullptr, reinterpret_cast<const uint8_t*>(a.down_s) + gr * (I / 32)};
            }
            if (a.has_bias && live[i]) bd[i] = ld_act<AT>(a.down_b, gr);
        }
    }
    const bool any = live[0];
    const void* src = shared ? a.hs : a.h;
    for (int64_t c = 0; c < cnt; c += kTT) {
        const int tt = int(cnt - c < kTT ? cnt - c : kTT);
        __syncthreads();
        stage_tokens<WF>(src, I, p0 + c, tt, nullptr, 1, us, xsum);
        __syncthreads();
        if (!any) continue;
        float acc[NR][kTT];
#pragma unroll
        for (int i = 0; i < NR; ++i)
#pragma unroll
            for (int t = 0; t < kTT; ++t) acc[i][t] = 0.f;
        dot_rows<WF, NR>(rows, q, I, shared ? a.s_group : a.group_size, us, xsum, tt, acc);
#pragma unroll
        for (int i = 0; i < NR; ++i)
#pragma unroll
            for (int t = 0; t < kTT; ++t) {
                if (t >= tt) break;
                acc[i][t] = warp_sum(acc[i][t]);
            }
#pragma unroll
        for (int i = 0; i < NR; ++i) {
            if (!live[i]) continue;
            const int r = rbase + i;
#pragma unroll
            for (int t = 0; t < kTT; ++t) {
                if (t < tt && lane == t) {
                    const int64_t p = p0 + c + t;
                    if (shared) {
                        a.s_acc[p * a.Hs + r] = acc[i][t];
                    } else {
                        const int slot = a.sorted_slot[p];
                        const int64_t token = slot / a.k;
                        atomicAdd(a.y_acc + token * R + r, a.topk_w[slot] * (acc[i][t] + bd[i]));
                    }
                }
            }
        }
    }
}

template <int WF>
__global__ void __launch_bounds__(kThreads) down_gemv_kernel(DownArgs a) {
    pdl_begin();
    constexpr int WFD = is_4bit<WF>() ? kBF16 : WF;
    using AT = typename Fmt<WF>::AT;
    extern __shared__ uint4 smem_raw[];
    AT* us = reinterpret_cast<AT*>(smem_raw);
    constexpr int NR = Fmt<WF>::DR, RR = kRowsPerBlock * NR;  // rows per warp / per block (both parts)
    const int sblocks = a.shared_I ? (a.Hs + RR - 1) / RR : 0;
    int b = blockIdx.x;
    if (b < sblocks) {
        if constexpr (WF != kF32) {
            if (a.sd_s) {  // 4-bit shared down plane: one row per warp, blocks of RR rows
#pragma unroll 1
                for (int r0 = b * RR; r0 < min(a.Hs, (b + 1) * RR); r0 += kRowsPerBlock)
                    down_group<kQ4, 1>(a, true, -1, r0, 0, a.T, a.shared_I, a.Hs, us,
                                       reinterpret_cast<float*>(us + int64_t(kTT) * a.shared_I));
                return;
            }
        }
        down_group<WFD, NR>(a, true, -1, b * RR, 0, a.T, a.shared_I, a.Hs, us, nullptr);
        return;
    }
    b -= sblocks;
    const int rblocks = (a.K + RR - 1) / RR;
    const int ai = b / rblocks;
    if (ai >= a.active[0]) return;
    const int e = a.active[1 + ai];
    const int64_t p0 = a.offsets[e];
    const int64_t cnt = a.offsets[e + 1] - p0;
    float* xsum = reinterpret_cast<float*>(us + int64_t(kTT) * a.I);
    down_group<WF, NR>(a, false, e, (b - ai * rblocks) * RR, p0, cnt, a.I, a.K, us, xsum);
}

template <typename AT, bool Q>
__global__ void __launch_bounds__(kThreads) dense_gemv_kernel(DenseGemvArgs a) {
    pdl_begin();
    constexpr int WF = sizeof(AT) == 4 ? kF32 : kBF16;
    extern __shared__ uint4 smem_raw[];
    AT* us = reinterpret_cast<AT*>(smem_raw);
    float* xsum = reinterpret_cast<float*>(us + int64_t(kTT) * a.K);  // Q: sums per 32 of each token
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = blockIdx.x * kRowsPerBlock + warp;
    const int rows = a.rows0 + a.rows1;
    const bool live = r < rows;
    const int64_t p0 = int64_t(blockIdx.y) * kTT;
    const int tt = int(a.T - p0 < kTT ? a.T - p0 : kTT);
    if constexpr (Q) stage_tokens<kQ4>(a.u, a.K, p0, tt, nullptr, 1, us, xsum);
    else stage_tokens<WF>(a.u, a.K, p0, tt, nullptr, 1, us, nullptr);
    __syncthreads();
    if (!live) return;
    const int rr = r < a.rows0 ? r : r - a.rows0;
    const void* W = r < a.rows0 ? a.W0 : a.W1;
    const void* bias = r < a.rows0 ? a.b0 : a.b1;
    float acc[1][kTT];
#pragma unroll
    for (int t = 0; t < kTT; ++t) acc[0][t] = 0.f;
    if (Q && r < a.rows0) {  // a 4-bit affine row of W0
        const int64_t ng = a.K / a.group0;
        const char* rowp[1] = {reinterpret_cast<const char*>(W) + int64_t(rr) * row_bytes<kQ4>(a.K)};
        const QRow q[1] = {{reinterpret_cast<const __nv_bfloat16*>(a.s0) + rr * ng,
                            reinterpret_cast<const __nv_bfloat16*>(a.z0) + rr * ng, nullptr}};
        if constexpr (Q) dot_rows<kQ4, 1>(rowp, q, a.K, a.group0, us, xsum, tt, acc);
    } else {
        const char* rowp[1] = {reinterpret_cast<const char*>(W) + int64_t(rr) * row_bytes<WF>(a.K)};
        const QRow q[1] = {{nullptr, nullptr, nullptr}};
        dot_rows<WF, 1>(rowp, q, a.K, 64, us, nullptr, tt, acc);
    }
    const float b = bias ? ld_act<AT>(bias, rr) : 0.f;
#pragma unroll
    for (int t = 0; t < kTT; ++t) {
        if (t >= tt) break;
        acc[0][t] = warp_sum(acc[0][t]);
    }
#pragma unroll
    for (int t = 0; t < kTT; ++t) {
        if (t < tt && lane == t) {
            const int64_t p = p0 + t;
            float v = acc[0][t] + b;
            if (a.addend) v += a.addend[p * a.ld_add + r];
            if (a.out_f32) reinterpret_cast<float*>(a.out)[p * a.ld_out + r] = v;
            else reinterpret_cast<AT*>(a.out)[p * a.ld_out + r] = from_f<AT>(v);
        }
    }
}

template <typename KernelT>
cudaError_t set_smem(KernelT kernel, size_t bytes) {
    if (bytes <= 48 * 1024) return cudaSuccess;
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes));
}

size_t stage_bytes(int wf, int K) {
    const size_t act = wf == kF32 ? 4 : 2;
    size_t b = size_t(kTT) * K * act;
    if (wf == kQ4) b += size_t(kTT) * (K / 32) * sizeof(float);
    return b;
}

template <int WF>
cudaError_t launch_gateup_t(const GateUpArgs& a, cudaStream_t s) {
    constexpr int WFD = is_4bit<WF>() ? kBF16 : WF;
    const size_t smem = std::max(stage_bytes(WF, a.K), a.shared_I ? stage_bytes(a.sg_s ? kQ4 : WFD, a.Hs) : size_t(0));
    cudaError_t err = set_smem(gateup_kernel<WF>(), smem);
    if (err != cudaSuccess) return err;
    const int64_t sblocks = a.shared_I ? (a.shared_I + kRowsPerBlock - 1) / kRowsPerBlock : 0;
    const int64_t rblocks = int64_t(a.routed_groups) * ((a.I + kRowsPerBlock - 1) / kRowsPerBlock);
    const int64_t grid = sblocks + rblocks;
    if (grid == 0) return cudaSuccess;
    { const cudaError_t e_ = launch_pdl(gateup_kernel<WF>(), dim3(unsigned(grid)), dim3(kThreads), smem, s, a); if (e_ != cudaSuccess) return e_; }
    return cudaGetLastError();
}

template <int WF>
cudaError_t launch_down_t(const DownArgs& a, cudaStream_t s) {
    constexpr int WFD = is_4bit<WF>() ? kBF16 : WF;
    const size_t smem = std::max(stage_bytes(WF, a.I), a.shared_I ? stage_bytes(a.sd_s ? kQ4 : WFD, a.shared_I) : size_t(0));
    cudaError_t err = set_smem(down_gemv_kernel<WF>, smem);
    if (err != cudaSuccess) return err;
    constexpr int RR = kRowsPerBlock * Fmt<WF>::DR;
    const int64_t sblocks = a.shared_I ? (a.Hs + RR - 1) / RR : 0;
    const int64_t rblocks = int64_t(a.routed_groups) * ((a.K + RR - 1) / RR);
    const int64_t grid = sblocks + rblocks;
    if (grid == 0) return cudaSuccess;
    { const cudaError_t e_ = launch_pdl(down_gemv_kernel<WF>, dim3(unsigned(grid)), dim3(kThreads), smem, s, a); if (e_ != cudaSuccess) return e_; }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gateup_gemv(const GateUpArgs& a, cudaStream_t s) {
    switch (a.wf) {
        case kF32: return launch_gateup_t<kF32>(a, s);
        case kBF16: return launch_gateup_t<kBF16>(a, s);
        case kQ4: return launch_gateup_t<kQ4>(a, s);
        case kMX4: return launch_gateup_t<kMX4>(a, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_down_gemv(const DownArgs& a, cudaStream_t s) {
    switch (a.wf) {
        case kF32: return launch_down_t<kF32>(a, s);
        case kBF16: return launch_down_t<kBF16>(a, s);
        case kQ4: return launch_down_t<kQ4>(a, s);
        case kMX4: return launch_down_t<kMX4>(a, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_dense_gemv(const DenseGemvArgs& a, cudaStream_t s) {
    const int rows = a.rows0 + a.rows1;
    if (a.T == 0 || rows == 0) return cudaSuccess;
    const dim3 grid(unsigned((rows + kRowsPerBlock - 1) / kRowsPerBlock), unsigned((a.T + kTT - 1) / kTT));
    if (grid.y > 65535u) return cudaErrorInvalidConfiguration;
    cudaError_t err;
    if (a.act_dtype == kF32) {
        const size_t smem = stage_bytes(kF32, a.K);
        if ((err = set_smem(dense_gemv_kernel<float, false>, smem)) != cudaSuccess) return err;
        { const cudaError_t e_ = launch_pdl(dense_gemv_kernel<float, false>, dim3(grid), dim3(kThreads), smem, s, a); if (e_ != cudaSuccess) return e_; }
    } else if (a.s0) {  // 4-bit affine W0
        const size_t smem = stage_bytes(kQ4, a.K);
        if ((err = set_smem(dense_gemv_kernel<__nv_bfloat16, true>, smem)) != cudaSuccess) return err;
        { const cudaError_t e_ = launch_pdl(dense_gemv_kernel<__nv_bfloat16, true>, dim3(grid), dim3(kThreads), smem, s, a); if (e_ != cudaSuccess) return e_; }
    } else {
        const size_t smem = stage_bytes(kBF16, a.K);
        if ((err = set_smem(dense_gemv_kernel<__nv_bfloat16, false>, smem)) != cudaSuccess) return err;
        { const cudaError_t e_ = launch_pdl(dense_gemv_kernel<__nv_bfloat16, false>, dim3(grid), dim3(kThreads), smem, s, a); if (e_ != cudaSuccess) return e_; }
    }
    return cudaGetLastError();
}

}  // namespace moe
