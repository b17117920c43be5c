// gemv.cu -- weight-streaming expert and projection kernels for small batches.
//
// When a group holds few tokens (decode-sized batches), the block is bound by
// reading each activated weight once from HBM. Every warp streams its own weight
// rows with 16-byte non-allocating loads, up to 16 loads in flight per lane, and
// takes several rows at once when rows are short. There is no shared-memory
// staging and no block barrier: a warp starts loading weights at once, and reads
// the few token vectors it multiplies through L1. Accumulation is fp32 on the CUDA
// cores; tensor cores would idle at these shapes.
//
// Expert shape: down(act(gate(u), up(u))) with [out, in] weights (ferrox
// KimiExpertWeights::forward); gate_up applied, then down weighted by the routing
// weights and summed per token (libmir-metal execute, Native arm: mxfp4_gate_up
// then mxfp4_down with routing.weights); 4-bit affine planes dequantised on the
// fly, w = scale * q + bias per group (mlxcel issue #974).
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int kTT = 8;        // tokens multiplied per pass over a weight row
constexpr int kWarps = 8;     // warps per block
constexpr int kThreads = kWarps * 32;
constexpr int kInFlight = 16; // 16-byte weight loads in flight per lane

template <int WF> struct Fmt;
template <> struct Fmt<kF32> { using AT = float; static constexpr int VE = 4; };
template <> struct Fmt<kBF16> { using AT = __nv_bfloat16; static constexpr int VE = 8; };
template <> struct Fmt<kQ4> { using AT = __nv_bfloat16; static constexpr int VE = 32; };

// Bytes of one weight row of K inputs in a given format.
template <int WF> __host__ __device__ __forceinline__ int64_t row_bytes(int K) {
    return WF == kF32 ? int64_t(K) * 4 : (WF == kBF16 ? int64_t(K) * 2 : int64_t(K) / 2);
}

struct QRow {  // 4-bit companions of one row: bf16 scale / bias per group
    const __nv_bfloat16* s;
    const __nv_bfloat16* z;
};

__device__ __forceinline__ uint4 ld_act16(const void* p) {  // token vectors: cached in L1
    return *reinterpret_cast<const uint4*>(p);
}

// acc[r][t] += sum_c W_r[c] * u_t[c] over the K inputs, for NR rows and tt (<= kTT)
// tokens whose rows start at tok[t] (act dtype, K elements each).
template <int WF, int NR>
__device__ __forceinline__ void stream_rows(const char* const (&rows)[NR], const QRow (&q)[NR], int K,
                                            int group_size, const char* const (&tok)[kTT], int tt,
                                            float (&acc)[NR][kTT]) {
    using F = Fmt<WF>;
    // vectors per row per batch (a 4-bit vector carries 32 weights: fewer suffice)
    constexpr int IN_FLIGHT = WF == kQ4 ? kInFlight / 2 : kInFlight;
    constexpr int U = (IN_FLIGHT / NR) > 0 ? (IN_FLIGHT / NR) : 1;
    constexpr int AB = sizeof(typename F::AT);
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
            const int64_t cb = int64_t(v) * F::VE * AB;  // byte offset of this vector's inputs
            if constexpr (WF == kBF16) {
                float wf[NR][8];
#pragma unroll
                for (int r = 0; r < NR; ++r) unpack8(wv[r][u], wf[r]);
#pragma unroll
                for (int t = 0; t < kTT; ++t) {
                    if (t >= tt) break;
                    float xf[8];
                    unpack8(ld_act16(tok[t] + cb), xf);
#pragma unroll
                    for (int r = 0; r < NR; ++r)
#pragma unroll
                        for (int j = 0; j < 8; ++j) acc[r][t] = fmaf(wf[r][j], xf[j], acc[r][t]);
                }
            } else if constexpr (WF == kF32) {
#pragma unroll
                for (int t = 0; t < kTT; ++t) {
                    if (t >= tt) break;
                    const uint4 xv = ld_act16(tok[t] + cb);
                    const float x0 = __uint_as_float(xv.x), x1 = __uint_as_float(xv.y);
                    const float x2 = __uint_as_float(xv.z), x3 = __uint_as_float(xv.w);
#pragma unroll
                    for (int r = 0; r < NR; ++r) {
                        acc[r][t] = fmaf(__uint_as_float(wv[r][u].x), x0, acc[r][t]);
                        acc[r][t] = fmaf(__uint_as_float(wv[r][u].y), x1, acc[r][t]);
                        acc[r][t] = fmaf(__uint_as_float(wv[r][u].z), x2, acc[r][t]);
                        acc[r][t] = fmaf(__uint_as_float(wv[r][u].w), x3, acc[r][t]);
                    }
                }
            } else {  // 4-bit affine: sum_j (s q_j + b) x_j = s * sum_j q_j x_j + b * sum_j x_j
                const int grp = (v * 32) / group_size;
                float sc[NR], bi[NR];
#pragma unroll
                for (int r = 0; r < NR; ++r) {
                    sc[r] = __bfloat162float(q[r].s[grp]);
                    bi[r] = __bfloat162float(q[r].z[grp]);
                }
#pragma unroll
                for (int t = 0; t < kTT; ++t) {
                    if (t >= tt) break;
                    float dq[NR];
#pragma unroll
                    for (int r = 0; r < NR; ++r) dq[r] = 0.f;
                    float xs = 0.f;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        float xf[8];
                        unpack8(ld_act16(tok[t] + cb + 16 * i), xf);
#pragma unroll
                        for (int n = 0; n < 8; ++n) xs += xf[n];
#pragma unroll
                        for (int r = 0; r < NR; ++r) {
                            const uint32_t word = i == 0 ? wv[r][u].x : i == 1 ? wv[r][u].y : i == 2 ? wv[r][u].z : wv[r][u].w;
#pragma unroll
                            for (int n = 0; n < 8; ++n) {
                                const float qv = __uint_as_float(0x4B000000u | ((word >> (4 * n)) & 0xFu)) - 8388608.0f;
                                dq[r] = fmaf(qv, xf[n], dq[r]);
                            }
                        }
                    }
#pragma unroll
                    for (int r = 0; r < NR; ++r) acc[r][t] = fmaf(sc[r], dq[r], fmaf(bi[r], xs, acc[r][t]));
                }
            }
        }
    }
}

template <int NR>
__device__ __forceinline__ void zero_acc(float (&acc)[NR][kTT]) {
#pragma unroll
    for (int r = 0; r < NR; ++r)
#pragma unroll
        for (int t = 0; t < kTT; ++t) acc[r][t] = 0.f;
}

template <int NR>
__device__ __forceinline__ void reduce_acc(float (&acc)[NR][kTT], int tt) {
#pragma unroll
    for (int r = 0; r < NR; ++r)
#pragma unroll
        for (int t = 0; t < kTT; ++t)
            if (t < tt) acc[r][t] = warp_sum(acc[r][t]);
}

template <typename AT>
__device__ __forceinline__ float ld_act(const void* p, int64_t i) {
    return to_f<AT>(reinterpret_cast<const AT*>(p)[i]);
}

// Gate/up of UPW intermediate units per warp (rows: gate_0, up_0, gate_1, up_1, ...):
// h[p, i] = act(gate_i . u_p + bg, up_i . u_p + bu) for the group's tokens.
template <int WF, int UPW>
__device__ __forceinline__ void gateup_units(const GateUpArgs& a, bool shared, int e, int unit0, int64_t p0,
                                             int64_t cnt, int K, int I) {
    using AT = typename Fmt<WF>::AT;
    constexpr int NR = 2 * UPW;
    const int lane = threadIdx.x & 31;
    const int64_t rb = row_bytes<WF>(K);
    const char* rows[NR];
    QRow q[NR];
    float bias[NR];
#pragma unroll
    for (int j = 0; j < UPW; ++j) {
        const int i = min(unit0 + j, I - 1);  // a warp past the end re-reads a valid row, stores nothing
        q[2 * j] = q[2 * j + 1] = {nullptr, nullptr};
        bias[2 * j] = bias[2 * j + 1] = 0.f;
        if (shared) {
            rows[2 * j] = reinterpret_cast<const char*>(a.sg_w) + int64_t(i) * rb;
            rows[2 * j + 1] = reinterpret_cast<const char*>(a.su_w) + int64_t(i) * rb;
        } else if (a.interleaved) {
            const int64_t r0 = int64_t(e) * 2 * I + 2 * int64_t(i);
            rows[2 * j] = reinterpret_cast<const char*>(a.gate_up_w) + r0 * rb;
            rows[2 * j + 1] = rows[2 * j] + rb;
            if (a.has_bias) {
                bias[2 * j] = ld_act<AT>(a.gate_up_b, r0);
                bias[2 * j + 1] = ld_act<AT>(a.gate_up_b, r0 + 1);
            }
        } else {
            const int64_t r0 = int64_t(e) * I + i;
            rows[2 * j] = reinterpret_cast<const char*>(a.gate_w) + r0 * rb;
            rows[2 * j + 1] = reinterpret_cast<const char*>(a.up_w) + r0 * rb;
            if constexpr (WF == kQ4) {
                const int64_t ng = K / a.group_size;
                q[2 * j] = {reinterpret_cast<const __nv_bfloat16*>(a.gate_s) + r0 * ng,
                            reinterpret_cast<const __nv_bfloat16*>(a.gate_z) + r0 * ng};
                q[2 * j + 1] = {reinterpret_cast<const __nv_bfloat16*>(a.up_s) + r0 * ng,
                                reinterpret_cast<const __nv_bfloat16*>(a.up_z) + r0 * ng};
            }
            if (a.has_bias) {
                bias[2 * j] = ld_act<AT>(a.gate_b, r0);
                bias[2 * j + 1] = ld_act<AT>(a.up_b, r0);
            }
        }
    }
    const char* src = static_cast<const char*>(shared ? a.xs : a.u);
    AT* dst = reinterpret_cast<AT*>(shared ? a.hs : a.h);
    const int64_t tok_bytes = int64_t(K) * sizeof(AT);
    for (int64_t c = 0; c < cnt; c += kTT) {
        const int tt = int(cnt - c < kTT ? cnt - c : kTT);
        const char* tok[kTT];
#pragma unroll
        for (int t = 0; t < kTT; ++t) {
            const int64_t p = p0 + c + (t < tt ? t : 0);
            const int64_t row = shared ? p : int64_t(a.sorted_slot[p] / a.k);
            tok[t] = src + row * tok_bytes;
        }
        float acc[NR][kTT];
        zero_acc<NR>(acc);
        stream_rows<WF, NR>(rows, q, K, a.group_size, tok, tt, acc);
        reduce_acc<NR>(acc, tt);
#pragma unroll
        for (int j = 0; j < UPW; ++j)
#pragma unroll
            for (int t = 0; t < kTT; ++t)
                if (t < tt && lane == j * kTT + t && unit0 + j < I)
                    dst[(p0 + c + t) * I + unit0 + j] = from_f<AT>(
                        act_apply(a.act, acc[2 * j][t] + bias[2 * j], acc[2 * j + 1][t] + bias[2 * j + 1],
                                  a.limit, a.alpha));
    }
}

template <int WF, int UPW>
__global__ void __launch_bounds__(kThreads) gateup_gemv_kernel(GateUpArgs a) {
    constexpr int WFD = (WF == kQ4) ? kBF16 : WF;  // the shared expert is dense
    constexpr int UPB = kWarps * UPW;              // units per block
    const int warp = threadIdx.x >> 5;
    const int sblocks = a.shared_I ? (a.shared_I + UPB - 1) / UPB : 0;
    int b = blockIdx.x;
    if (b < sblocks) {
        const int unit0 = b * UPB + warp * UPW;
        if (unit0 < a.shared_I) gateup_units<WFD, UPW>(a, true, -1, unit0, 0, a.T, a.Hs, a.shared_I);
        return;
    }
    b -= sblocks;
    const int ublocks = (a.I + UPB - 1) / UPB;
    const int ai = b / ublocks;
    if (ai >= a.active[0]) return;
    const int unit0 = (b - ai * ublocks) * UPB + warp * UPW;
    if (unit0 >= a.I) return;
    const int e = a.active[1 + ai];
    const int64_t p0 = a.offsets[e];
    gateup_units<WF, UPW>(a, false, e, unit0, p0, a.offsets[e + 1] - p0, a.K, a.I);
}

// Down projection of RW output rows per warp for one group.
template <int WF, int RW>
__device__ __forceinline__ void down_rows(const DownArgs& a, bool shared, int e, int row0, int64_t p0,
                                          int64_t cnt, int I, int R) {
    using AT = typename Fmt<WF>::AT;
    const int lane = threadIdx.x & 31;
    const int64_t rb = row_bytes<WF>(I);
    const char* rows[RW];
    QRow q[RW];
    float bd[RW];
#pragma unroll
    for (int j = 0; j < RW; ++j) {
        const int r = min(row0 + j, R - 1);
        q[j] = {nullptr, nullptr};
        bd[j] = 0.f;
        if (shared) {
            rows[j] = reinterpret_cast<const char*>(a.sd_w) + int64_t(r) * rb;
        } else {
            const int64_t gr = int64_t(e) * R + r;
            rows[j] = reinterpret_cast<const char*>(a.down_w) + gr * rb;
            if constexpr (WF == kQ4) {
                const int64_t ng = I / a.group_size;
                q[j] = {reinterpret_cast<const __nv_bfloat16*>(a.down_s) + gr * ng,
                        reinterpret_cast<const __nv_bfloat16*>(a.down_z) + gr * ng};
            }
            if (a.has_bias) bd[j] = ld_act<AT>(a.down_b, gr);
        }
    }
    const char* src = static_cast<const char*>(shared ? a.hs : a.h);
    const int64_t tok_bytes = int64_t(I) * sizeof(AT);
    for (int64_t c = 0; c < cnt; c += kTT) {
        const int tt = int(cnt - c < kTT ? cnt - c : kTT);
        const char* tok[kTT];
#pragma unroll
        for (int t = 0; t < kTT; ++t) tok[t] = src + (p0 + c + (t < tt ? t : 0)) * tok_bytes;
        float acc[RW][kTT];
        zero_acc<RW>(acc);
        stream_rows<WF, RW>(rows, q, I, a.group_size, tok, tt, acc);
        reduce_acc<RW>(acc, tt);
#pragma unroll
        for (int j = 0; j < RW; ++j)
#pragma unroll
            for (int t = 0; t < kTT; ++t)
                if (t < tt && lane == j * kTT + t && row0 + j < R) {
                    const int64_t p = p0 + c + t;
                    const int r = row0 + j;
                    if (shared) {
                        a.s_acc[p * a.Hs + r] = acc[j][t];
                    } else {
                        const int slot = a.sorted_slot[p];
                        atomicAdd(a.y_acc + int64_t(slot / a.k) * R + r, a.topk_w[slot] * (acc[j][t] + bd[j]));
                    }
                }
    }
}

template <int WF, int RW>
__global__ void __launch_bounds__(kThreads) down_gemv_kernel(DownArgs a) {
    constexpr int WFD = (WF == kQ4) ? kBF16 : WF;
    constexpr int RPB = kWarps * RW;  // rows per block
    const int warp = threadIdx.x >> 5;
    const int sblocks = a.shared_I ? (a.Hs + RPB - 1) / RPB : 0;
    int b = blockIdx.x;
    if (b < sblocks) {
        const int row0 = b * RPB + warp * RW;
        if (row0 < a.Hs) down_rows<WFD, RW>(a, true, -1, row0, 0, a.T, a.shared_I, a.Hs);
        return;
    }
    b -= sblocks;
    const int rblocks = (a.K + RPB - 1) / RPB;
    const int ai = b / rblocks;
    if (ai >= a.active[0]) return;
    const int row0 = (b - ai * rblocks) * RPB + warp * RW;
    if (row0 >= a.K) return;
    const int e = a.active[1 + ai];
    const int64_t p0 = a.offsets[e];
    down_rows<WF, RW>(a, false, e, row0, p0, a.offsets[e + 1] - p0, a.I, a.K);
}

// out[t, r] = W[r] . u[t] (+ bias) (+ addend) for RW rows per warp and kTT tokens per block row.
template <typename AT, int RW>
__global__ void __launch_bounds__(kThreads) dense_gemv_kernel(DenseGemvArgs a) {
    constexpr int WF = sizeof(AT) == 4 ? kF32 : kBF16;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rows_total = a.rows0 + a.rows1;
    const int row0 = (blockIdx.x * kWarps + warp) * RW;
    if (row0 >= rows_total) return;
    const int64_t p0 = int64_t(blockIdx.y) * kTT;
    const int tt = int(a.T - p0 < kTT ? a.T - p0 : kTT);
    const char* rows[RW];
    QRow q[RW];
    float bias[RW];
#pragma unroll
    for (int j = 0; j < RW; ++j) {
        const int r = min(row0 + j, rows_total - 1);
        const bool first = r < a.rows0;
        const int rr = first ? r : r - a.rows0;
        rows[j] = reinterpret_cast<const char*>(first ? a.W0 : a.W1) + int64_t(rr) * row_bytes<WF>(a.K);
        q[j] = {nullptr, nullptr};
        const void* b = first ? a.b0 : a.b1;
        bias[j] = b ? ld_act<AT>(b, rr) : 0.f;
    }
    const char* tok[kTT];
#pragma unroll
    for (int t = 0; t < kTT; ++t)
        tok[t] = static_cast<const char*>(a.u) + (p0 + (t < tt ? t : 0)) * int64_t(a.K) * sizeof(AT);
    float acc[RW][kTT];
    zero_acc<RW>(acc);
    stream_rows<WF, RW>(rows, q, a.K, 64, tok, tt, acc);
    reduce_acc<RW>(acc, tt);
#pragma unroll
    for (int j = 0; j < RW; ++j)
#pragma unroll
        for (int t = 0; t < kTT; ++t)
            if (t < tt && lane == j * kTT + t && row0 + j < rows_total) {
                const int64_t p = p0 + t;
                const int r = row0 + j;
                float v = acc[j][t] + bias[j];
                if (a.addend) v += a.addend[p * a.ld_add + r];
                if (a.out_f32) reinterpret_cast<float*>(a.out)[p * a.ld_out + r] = v;
                else reinterpret_cast<AT*>(a.out)[p * a.ld_out + r] = from_f<AT>(v);
            }
}

// Rows per warp for rows of `nvec` 16-byte vectors: enough rows to keep ~16 loads in flight.
int rows_per_warp(int64_t row_bytes_) {
    const int64_t per_lane = (row_bytes_ / 16 + 31) / 32;
    if (per_lane <= 4) return 4;
    if (per_lane <= 8) return 2;
    return 1;
}

}  // namespace

cudaError_t launch_gateup_gemv(const GateUpArgs& a, cudaStream_t s) {
    const int wfd = a.wf == kQ4 ? kBF16 : a.wf;
    // units per warp: two when one unit's gate+up rows would leave fewer than 8 loads in flight
    const int64_t rbytes = a.wf == kF32 ? int64_t(a.K) * 4 : a.wf == kBF16 ? int64_t(a.K) * 2 : a.K / 2;
    const int upw = rows_per_warp(rbytes) >= 4 ? 2 : 1;
    (void)wfd;
    const int upb = kWarps * upw;
    const int64_t sblocks = a.shared_I ? (a.shared_I + upb - 1) / upb : 0;
    const int64_t grid = sblocks + int64_t(a.routed_groups) * ((a.I + upb - 1) / upb);
    if (grid == 0) return cudaSuccess;
#define MOE_GU(WFV, UPWV) gateup_gemv_kernel<WFV, UPWV><<<unsigned(grid), kThreads, 0, s>>>(a)
    if (a.wf == kF32) { if (upw == 2) MOE_GU(kF32, 2); else MOE_GU(kF32, 1); }
    else if (a.wf == kBF16) { if (upw == 2) MOE_GU(kBF16, 2); else MOE_GU(kBF16, 1); }
    else { if (upw == 2) MOE_GU(kQ4, 2); else MOE_GU(kQ4, 1); }
#undef MOE_GU
    return cudaGetLastError();
}

cudaError_t launch_down_gemv(const DownArgs& a, cudaStream_t s) {
    const int64_t rbytes = a.wf == kF32 ? int64_t(a.I) * 4 : a.wf == kBF16 ? int64_t(a.I) * 2 : a.I / 2;
    const int rw = rows_per_warp(rbytes);
    const int rpb = kWarps * rw;
    const int64_t sblocks = a.shared_I ? (a.Hs + rpb - 1) / rpb : 0;
    const int64_t grid = sblocks + int64_t(a.routed_groups) * ((a.K + rpb - 1) / rpb);
    if (grid == 0) return cudaSuccess;
#define MOE_DN(WFV) \
    do { if (rw == 4) down_gemv_kernel<WFV, 4><<<unsigned(grid), kThreads, 0, s>>>(a); \
         else if (rw == 2) down_gemv_kernel<WFV, 2><<<unsigned(grid), kThreads, 0, s>>>(a); \
         else down_gemv_kernel<WFV, 1><<<unsigned(grid), kThreads, 0, s>>>(a); } while (0)
    if (a.wf == kF32) MOE_DN(kF32);
    else if (a.wf == kBF16) MOE_DN(kBF16);
    else MOE_DN(kQ4);
#undef MOE_DN
    return cudaGetLastError();
}

cudaError_t launch_dense_gemv(const DenseGemvArgs& a, cudaStream_t s) {
    const int rows = a.rows0 + a.rows1;
    if (a.T == 0 || rows == 0) return cudaSuccess;
    const int ab = a.act_dtype == kF32 ? 4 : 2;
    const int rw = rows_per_warp(int64_t(a.K) * ab);
    const int rpb = kWarps * rw;
    const dim3 grid(unsigned((rows + rpb - 1) / rpb), unsigned((a.T + kTT - 1) / kTT));
    if (grid.y > 65535u) return cudaErrorInvalidConfiguration;
#define MOE_DG(AT) \
    do { if (rw == 4) dense_gemv_kernel<AT, 4><<<grid, kThreads, 0, s>>>(a); \
         else if (rw == 2) dense_gemv_kernel<AT, 2><<<grid, kThreads, 0, s>>>(a); \
         else dense_gemv_kernel<AT, 1><<<grid, kThreads, 0, s>>>(a); } while (0)
    if (a.act_dtype == kF32) MOE_DG(float);
    else MOE_DG(__nv_bfloat16);
#undef MOE_DG
    return cudaGetLastError();
}

}  // namespace moe
