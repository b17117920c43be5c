// gemv_dev.cuh -- weight-streaming dot products shared by the CUDA-core expert kernels and
// the persistent decode kernel.
//
// A warp streams NR weight rows with 16-byte non-allocating loads (several vectors in flight
// per lane) and dots them with up to kTT tokens staged in shared memory, accumulating in
// fp32. Formats: f32, bf16, 4-bit affine (w = scale * q + bias per group; mlxcel issue #974)
// and MXFP4 (OCP MX v1.0 E2M1 codes with an E8M0 scale per 32).
#pragma once

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kTT = 8;        // tokens staged per pass

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

// acc[r][t] += sum_c W_r[c] * u_t[c] for NR rows and tt (<= kTT) staged tokens; u_t is row
// t of `us` (rows of K values), or row tl[t] when a token list is given. U: 16-byte vectors
// per row in flight per lane.
template <int WF, int NR, int TT = kTT, int U = Fmt<WF>::U>
__device__ __forceinline__ void dot_rows(const char* const (&rows)[NR], const QRow (&q)[NR], int K,
                                         int group_size, const typename Fmt<WF>::AT* us,
                                         const float* xsum, int tt, float (&acc)[NR][TT],
                                         const int* tl = nullptr) {
    using F = Fmt<WF>;
    using AT = typename F::AT;
    const int lane = threadIdx.x & 31;
    const int nvec = K / F::VE;
    for (int base = lane; base < nvec; base += 32 * U) {
        uint4 wv[NR][U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int v = base + 32 * u;
#pragma unroll
            for (int r = 0; r < NR; ++r)
                wv[r][u] = v < nvec ? ld_stream16(rows[r] + int64_t(v) * 16) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int v = base + 32 * u;
            if (v >= nvec) break;
            const int c0 = v * F::VE;
            if constexpr (WF == kBF16) {
                float wf[NR][8];
#pragma unroll
                for (int r = 0; r < NR; ++r) unpack8(wv[r][u], wf[r]);
#pragma unroll
                for (int t = 0; t < TT; ++t) {
                    if (t >= tt) break;
                    float xf[8];
                    unpack8(*reinterpret_cast<const uint4*>(us + int64_t(tl ? tl[t] : t) * K + c0), xf);
#pragma unroll
                    for (int r = 0; r < NR; ++r)
#pragma unroll
                        for (int j = 0; j < 8; ++j) acc[r][t] = fmaf(wf[r][j], xf[j], acc[r][t]);
                }
            } else if constexpr (WF == kF32) {
#pragma unroll
                for (int t = 0; t < TT; ++t) {
                    if (t >= tt) break;
                    const float4 xv = *reinterpret_cast<const float4*>(us + int64_t(tl ? tl[t] : t) * K + c0);
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
                for (int t = 0; t < TT; ++t) {
                    if (t >= tt) break;
                    float dq[NR];
#pragma unroll
                    for (int r = 0; r < NR; ++r) dq[r] = 0.f;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        float xf[8];
                        unpack8(*reinterpret_cast<const uint4*>(us + int64_t(tl ? tl[t] : t) * K + c0 + 8 * i), xf);
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
                float dq[NR][TT];
#pragma unroll
                for (int r = 0; r < NR; ++r)
#pragma unroll
                    for (int t = 0; t < TT; ++t) dq[r][t] = 0.f;
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
                    for (int t = 0; t < TT; ++t) {
                        if (t >= tt) break;
                        float xf[8];
                        unpack8(*reinterpret_cast<const uint4*>(us + int64_t(tl ? tl[t] : t) * K + c0 + 8 * i), xf);
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
                    for (int t = 0; t < TT; ++t) {
                        if (t >= tt) break;
                        acc[r][t] = fmaf(sc, dq[r][t], fmaf(bi, xsum[(tl ? tl[t] : t) * (K / 32) + v], acc[r][t]));
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

}  // namespace
}  // namespace moe
