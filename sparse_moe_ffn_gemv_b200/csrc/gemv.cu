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

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int kTT = 8;        // tokens staged per pass
constexpr int kRowsPerBlock = 8;  // one warp per weight row / intermediate unit
constexpr int kThreads = kRowsPerBlock * 32;

template <int WF> struct Fmt;
// VE: weights per 16-byte vector; U: vectors per row in flight per lane; DR: down-projection
// rows per warp (two short rows keep more bytes in flight; with the 4-bit dequantisation's
// registers one row per warp keeps more warps resident, which measured faster).
template <> struct Fmt<kF32> { using AT = float; static constexpr int VE = 4, U = 4, DR = 2; };
template <> struct Fmt<kBF16> { using AT = __nv_bfloat16; static constexpr int VE = 8, U = 4, DR = 2; };
template <> struct Fmt<kQ4> { using AT = __nv_bfloat16; static constexpr int VE = 32, U = 2, DR = 1; };
template <> struct Fmt<kMX4> { using AT = __nv_bfloat16; static constexpr int VE = 32, U = 2, DR = 1; };
template <int WF> constexpr bool is_4bit() { return WF == kQ4 || WF == kMX4; }

// Row pointer of a weight matrix row in a given format (bytes per row).
template <int WF> __host__ __device__ __forceinline__ int64_t row_bytes(int K) {
    return WF == kF32 ? int64_t(K) * 4 : (WF == kBF16 ? int64_t(K) * 2 : int64_t(K) / 2);
}

struct QRow {  // 4-bit companions of one row
    const __nv_bfloat16* s;  // affine: bf16 scale per group
    const __nv_bfloat16* z;  // affine: bf16 bias per group
    const uint8_t* e8;       // MXFP4: E8M0 scale byte per block of 32
};

// acc[r][t] += sum_c W_r[c] * u_t[c] for NR rows and tt (<= kTT) staged tokens.
template <int WF, int NR>
__device__ __forceinline__ void dot_rows(const char* const (&rows)[NR], const QRow (&q)[NR], int K,
                                         int group_size, const typename Fmt<WF>::AT* us,
                                         const float* xsum, int tt, float (&acc)[NR][kTT]) {
    using F = Fmt<WF>;
    using AT = typename F::AT;
    const int lane = threadIdx.x & 31;
    const int nvec = K / F::VE;
    for (int base = lane; base < nvec; base += 32 * F::U) {
        uint4 wv[NR][F::U];
#pragma unroll
        for (int u = 0; u < F::U; ++u) {
            const int v = base + 32 * u;
#pragma unroll
            for (int r = 0; r < NR; ++r)
                wv[r][u] = v < nvec ? ld_stream16(rows[r] + int64_t(v) * 16) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < F::U; ++u) {
            const int v = base + 32 * u;
            if (v >= nvec) break;
            const int c0 = v * F::VE;
            if constexpr (WF == kBF16) {
                float wf[NR][8];
#pragma unroll
                for (int r = 0; r < NR; ++r) unpack8(wv[r][u], wf[r]);
#pragma unroll
                for (int t = 0; t < kTT; ++t) {
                    if (t >= tt) break;
                    float xf[8];
                    unpack8(*reinterpret_cast<const uint4*>(us + int64_t(t) * K + c0), xf);
#pragma unroll
                    for (int r = 0; r < NR; ++r)
#pragma unroll
                        for (int j = 0; j < 8; ++j) acc[r][t] = fmaf(wf[r][j], xf[j], acc[r][t]);
                }
            } else if constexpr (WF == kF32) {
#pragma unroll
                for (int t = 0; t < kTT; ++t) {
                    if (t >= tt) break;
                    const float4 xv = *reinterpret_cast<const float4*>(us + int64_t(t) * K + c0);
#pragma unroll
                    for (int r = 0; r < NR; ++r) {
                        acc[r][t] = fmaf(__uint_as_float(wv[r][u].x), xv.x, acc[r][t]);
                        acc[r][t] = fmaf(__uint_as_float(wv[r][u].y), xv.y, acc[r][t]);
                        acc[r][t] = fmaf(__uint_as_float(wv[r][u].z), xv.z, acc[r][t]);
                        acc[r][t] = fmaf(__uint_as_float(wv[r][u].w), xv.w, acc[r][t]);
                    }
                }
            } else if constexpr (WF == kMX4) {  // one vector = one block of 32: sum_j e_j x_j times 2^(s-127)
                float qf[NR][32], sc[NR];
#pragma unroll
                for (int r = 0; r < NR; ++r) {
                    sc[r] = e8m0_value(q[r].e8[v]);
                    const uint32_t words[4] = {wv[r][u].x, wv[r][u].y, wv[r][u].z, wv[r][u].w};
#pragma unroll
                    for (int i = 0; i < 4; ++i)
#pragma unroll
                        for (int n = 0; n < 8; ++n) qf[r][i * 8 + n] = e2m1_value(words[i] >> (4 * n));
                }
#pragma unroll
                for (int t = 0; t < kTT; ++t) {
                    if (t >= tt) break;
                    float dq[NR];
#pragma unroll
                    for (int r = 0; r < NR; ++r) dq[r] = 0.f;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        float xf[8];
                        unpack8(*reinterpret_cast<const uint4*>(us + int64_t(t) * K + c0 + 8 * i), xf);
#pragma unroll
                        for (int r = 0; r < NR; ++r)
#pragma unroll
                            for (int n = 0; n < 8; ++n) dq[r] = fmaf(qf[r][i * 8 + n], xf[n], dq[r]);
                    }
#pragma unroll
                    for (int r = 0; r < NR; ++r) acc[r][t] = fmaf(sc[r], dq[r], acc[r][t]);
                }
            } else {  // 4-bit affine: sum_j (s q_j + b) x_j = s * sum_j q_j x_j + b * sum_j x_j
                // Decoded one 32-bit word (8 codes) at a time, so that only 8 codes per row are
                // live beside the per-token partial sums (fewer registers, more resident warps).
                float dq[NR][kTT];
#pragma unroll
                for (int r = 0; r < NR; ++r)
#pragma unroll
                    for (int t = 0; t < kTT; ++t) dq[r][t] = 0.f;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float qf[NR][8];
#pragma unroll
                    for (int r = 0; r < NR; ++r) {
                        const uint32_t word = i == 0 ? wv[r][u].x : i == 1 ? wv[r][u].y : i == 2 ? wv[r][u].z : wv[r][u].w;
#pragma unroll
                        for (int n = 0; n < 8; ++n)  // the code q in [0, 15] as a float, exactly: (2^23 + q) - 2^23
                            qf[r][n] = __uint_as_float(0x4B000000u | ((word >> (4 * n)) & 0xFu)) - 8388608.0f;
                    }
#pragma unroll
                    for (int t = 0; t < kTT; ++t) {
                        if (t >= tt) break;
                        float xf[8];
                        unpack8(*reinterpret_cast<const uint4*>(us + int64_t(t) * K + c0 + 8 * i), xf);
#pragma unroll
                        for (int r = 0; r < NR; ++r)
#pragma unroll
                            for (int n = 0; n < 8; ++n) dq[r][t] = fmaf(qf[r][n], xf[n], dq[r][t]);
                    }
                }
                const int grp = c0 / group_size;
#pragma unroll
                for (int r = 0; r < NR; ++r) {
                    const float sc = __bfloat162float(q[r].s[grp]);
                    const float bi = __bfloat162float(q[r].z[grp]);
#pragma unroll
                    for (int t = 0; t < kTT; ++t) {
                        if (t >= tt) break;
                        acc[r][t] = fmaf(sc, dq[r][t], fmaf(bi, xsum[t * (K / 32) + v], acc[r][t]));
                    }
                }
            }
        }
    }
}

// Stage tokens [p0, p0 + tt) of a group into shared memory (rows of K act values);
// for 4-bit weights also the per-32 sums of each staged row.
template <int WF>
__device__ __forceinline__ void stage_tokens(const void* src, int K, int64_t p0, int tt,
                                             const int32_t* sorted_slot, int k,
                                             typename Fmt<WF>::AT* us, float* xsum) {
    using AT = typename Fmt<WF>::AT;
    const int vpr = K * int(sizeof(AT)) / 16;  // 16-byte vectors per row
    for (int i = threadIdx.x; i < tt * vpr; i += blockDim.x) {
        const int t = i / vpr, c = i - t * vpr;
        const int64_t p = p0 + t;
        const int64_t row = sorted_slot ? int64_t(sorted_slot[p] / k) : p;
        reinterpret_cast<uint4*>(us)[int64_t(t) * vpr + c] =
            reinterpret_cast<const uint4*>(src)[row * vpr + c];
    }
    if constexpr (WF == kQ4) {
        __syncthreads();
        const int nv = K / 32;
        for (int i = threadIdx.x; i < tt * nv; i += blockDim.x) {
            const int t = i / nv, v = i - t * nv;
            const uint4* p = reinterpret_cast<const uint4*>(us + int64_t(t) * K + v * 32);
            float s = 0.f;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float f[8];
                unpack8(p[j], f);
#pragma unroll
                for (int n = 0; n < 8; ++n) s += f[n];
            }
            xsum[i] = s;
        }
    }
}

template <int WF>
__device__ __forceinline__ void reduce_acc(float (&acc)[2][kTT], int nr, int tt) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        if (r >= nr) break;
#pragma unroll
        for (int t = 0; t < kTT; ++t) {
            if (t >= tt) break;
            acc[r][t] = warp_sum(acc[r][t]);
        }
    }
}

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
        dot_rows<WF, 2>(rows, q, K, a.group_size, us, xsum, tt, acc);
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
        dot_rows<WF, NR>(rows, q, I, a.group_size, us, xsum, tt, acc);
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

template <typename AT>
__global__ void __launch_bounds__(kThreads) dense_gemv_kernel(DenseGemvArgs a) {
    pdl_begin();
    constexpr int WF = sizeof(AT) == 4 ? kF32 : kBF16;
    extern __shared__ uint4 smem_raw[];
    AT* us = reinterpret_cast<AT*>(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = blockIdx.x * kRowsPerBlock + warp;
    const int rows = a.rows0 + a.rows1;
    const bool live = r < rows;
    const int64_t p0 = int64_t(blockIdx.y) * kTT;
    const int tt = int(a.T - p0 < kTT ? a.T - p0 : kTT);
    stage_tokens<WF>(a.u, a.K, p0, tt, nullptr, 1, us, nullptr);
    __syncthreads();
    if (!live) return;
    const int rr = r < a.rows0 ? r : r - a.rows0;
    const void* W = r < a.rows0 ? a.W0 : a.W1;
    const void* bias = r < a.rows0 ? a.b0 : a.b1;
    const char* rowp[1] = {reinterpret_cast<const char*>(W) + int64_t(rr) * row_bytes<WF>(a.K)};
    QRow q[1] = {{nullptr, nullptr, nullptr}};
    float acc[1][kTT];
#pragma unroll
    for (int t = 0; t < kTT; ++t) acc[0][t] = 0.f;
    dot_rows<WF, 1>(rowp, q, a.K, 64, us, nullptr, tt, acc);
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
    const size_t smem = std::max(stage_bytes(WF, a.K), a.shared_I ? stage_bytes(WFD, a.Hs) : size_t(0));
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
    const size_t smem = std::max(stage_bytes(WF, a.I), a.shared_I ? stage_bytes(WFD, a.shared_I) : size_t(0));
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
        if ((err = set_smem(dense_gemv_kernel<float>, smem)) != cudaSuccess) return err;
        { const cudaError_t e_ = launch_pdl(dense_gemv_kernel<float>, dim3(grid), dim3(kThreads), smem, s, a); if (e_ != cudaSuccess) return e_; }
    } else {
        const size_t smem = stage_bytes(kBF16, a.K);
        if ((err = set_smem(dense_gemv_kernel<__nv_bfloat16>, smem)) != cudaSuccess) return err;
        { const cudaError_t e_ = launch_pdl(dense_gemv_kernel<__nv_bfloat16>, dim3(grid), dim3(kThreads), smem, s, a); if (e_ != cudaSuccess) return e_; }
    }
    return cudaGetLastError();
}

}  // namespace moe
