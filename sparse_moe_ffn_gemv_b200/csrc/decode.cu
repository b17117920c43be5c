// decode.cu -- the whole block for a decode-sized batch (T <= 8 tokens) in one launch.
//
// At a few tokens the block is bound by reading the activated weights once from HBM, and
// a chain of short kernels (router, top-k, gate/up, down, combine) loses most of its time to
// the start and tail of each launch. Here one cooperative launch of one 512-thread block
// per SM runs three phases separated by grid barriers:
//   A  the router and coefficient-head rows (fp32 logits) and the shared expert's gate/up
//      units (Klear PR item 2: the shared expert reads the block input x; neither depends
//      on the routing, so they start at once);
//   B  every block takes the top-k of the T tokens itself (Klear PR item 3: sigmoid of fp32
//      logits, select-only bias, unbiased weights, norm_topk_prob; libmir-metal
//      router_top_k_unit for softmax over the top-k logits), sorts the T*k slots by expert,
//      and the grid streams the routed gate/up units of the distinct experts (one weight
//      row pair per warp item, dotted with the tokens routed to that expert);
//   C  each block owns a contiguous range of output rows: it stages every slot's
//      intermediate vector, streams the down rows of its range for every distinct expert
//      and for the shared expert, and writes y = y_r | y_r + s | c0 y_r + c1 s for its
//      rows (libmir-metal execute: down weighted by routing.weights and summed; ferrox
//      KimiExpertWeights::forward: down(act(gate, up))).
// (An L2 prefetch of each block's phase-C down rows issued at the start of phase B
// measured slower: Klear, one token, 47.1 vs 45.1 us without it.)
// Every grid-barrier wait is bounded by %globaltimer: a wait that gives up records
// MOE_ERR_DEVICE_TIMEOUT in the status word, and the block skips the remaining phases.
// The last block to finish resets the barrier counters, so the next launch starts from 0.
#include <algorithm>

#include "gemv_dev.cuh"
#include "ptx.cuh"
#include "topk_dev.cuh"

namespace moe {

namespace {

constexpr int kDecThreads = 512;
constexpr int kDecWarps = kDecThreads / kWarp;
constexpr int kDecMaxSlots = kTT * kMaxTopK;  // T * k slots at most
constexpr int kDecRowsMax = 64;               // output rows a block owns at most
constexpr uint64_t kDecWaitNs = 2000000000ull;  // 2 s bound on a grid-barrier wait
constexpr size_t kDecSmemMax = 200 * 1024;

struct DecSmem {
    int32_t sidx[kDecMaxSlots];  // expert of slot s = t * k + j
    float sw[kDecMaxSlots];      // combine weight of slot s
    float scoef[kTT * 2];        // blend coefficients of each token
    int sorted[kDecMaxSlots];    // slots sorted by expert, ascending slot within an expert
    int head[kDecMaxSlots];      // 1: first slot of its expert
    int lt[kDecMaxSlots];        // slots whose expert is smaller than slot s's
    int dexp[kDecMaxSlots];      // distinct experts, ascending
    int doff[kDecMaxSlots + 1];  // their ranges in `sorted`
    int n_d;                     // number of distinct experts
    int flag;
    float sstat[2 * kTT];        // softmax over all experts: each token's max and 1 / sum
    float ssel[kMaxExperts];     // select-only biases, staged in phase A
    float acc_r[kDecRowsMax][kTT];  // routed sum of the block's rows
    float acc_s[kDecRowsMax][kTT];  // shared expert output of the block's rows
};

// Byte offset of the top-k keys in the dynamic shared memory: after the T staged token rows
// (bf16) and, for 4-bit planes, their per-32 sums; 16-byte aligned.
__host__ __device__ __forceinline__ size_t dec_keys_offset(int T, int H, bool sums) {
    return (size_t(T) * H * 2 + (sums ? size_t(T) * (H / 32) * 4 : 0) + 15) & ~size_t(15);
}

__device__ __forceinline__ float bf16_ld(const void* p, int64_t i) {
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
}

// Copy n16 16-byte vectors from global (through L2: another block wrote them) to shared.
__device__ __forceinline__ void copy_cg(uint4* dst, const void* src, int64_t n16) {
    const uint4* s = reinterpret_cast<const uint4*>(src);
    for (int64_t i = threadIdx.x; i < n16; i += blockDim.x) dst[i] = __ldcg(s + i);
}

// Rows per warp item and 16-byte vectors in flight per row and lane. With one token the
// accumulators are few: phases A and B take two rows (one gate/up unit) per item with a whole
// 2048-wide bf16 row in flight per lane pair of loads (U = 8: one round trip per item), phase
// C four down rows. With up to 8 tokens: two rows everywhere. Every phase of one format uses
// the same shape, so that it runs the same code.
template <int WF, int TT> struct DecShape {
    static constexpr bool ONE = TT == 1;
    static constexpr int RR = 2;                                    // router / coefficient rows
    static constexpr int SU = 1;                                    // shared gate/up units
    static constexpr int BU = 1;                                    // routed gate/up units
    static constexpr int UA = ONE ? 8 : Fmt<kBF16>::U;              // bf16 rows, phases A and B
    static constexpr int UB = (ONE && WF == kBF16) ? 8 : Fmt<WF>::U;  // routed gate/up rows
    static constexpr int DN = (ONE && WF == kBF16) ? 4 : 2;         // routed down rows
    static constexpr int SN = ONE ? 4 : 2;                          // shared down rows
    static constexpr int UC = Fmt<WF>::U;                           // routed down rows, phase C
};

// acc[r][t] = sum over the row of W_r . u_t, reduced over the warp (every lane holds it).
template <int WF, int NR, int TT, int U = Fmt<WF>::U>
__device__ __forceinline__ void dot_reduce(const char* const (&rows)[NR], const QRow (&q)[NR], int K, int gs,
                                           const __nv_bfloat16* us, const float* usum, int tt, float (&acc)[NR][TT],
                                           const int* tl = nullptr) {
#pragma unroll
    for (int r = 0; r < NR; ++r)
#pragma unroll
        for (int t = 0; t < TT; ++t) acc[r][t] = 0.f;
    dot_rows<WF, NR, TT, U>(rows, q, K, gs, us, usum, tt, acc, tl);
#pragma unroll
    for (int r = 0; r < NR; ++r)
#pragma unroll
        for (int t = 0; t < TT; ++t) {
            if (t >= tt) break;
            acc[r][t] = warp_sum(acc[r][t]);
        }
}

// One out-of-line copy of the dot product per (format, rows, tokens): every call site of
// every phase runs the same instructions. The kernel runs each phase once per SM after an L2
// flush could have evicted its code, so distinct instructions cost instruction-cache misses;
// the call's argument traffic (a few words of local memory) is paid once per item.
template <int WF, int NR, int TT, int U = Fmt<WF>::U>
__device__ __noinline__ void dec_dot(const char* const* rows, const QRow* q, int K, int gs,
                                     const __nv_bfloat16* us, const float* usum, int tt, const int* tl,
                                     float* out) {
    const char* r[NR];
    QRow qq[NR];
#pragma unroll
    for (int j = 0; j < NR; ++j) {
        r[j] = rows[j];
        qq[j] = q[j];
    }
    float acc[NR][TT];
    dot_reduce<WF, NR, TT, U>(r, qq, K, gs, us, usum, tt, acc, tl);
#pragma unroll
    for (int j = 0; j < NR; ++j)
#pragma unroll
        for (int t = 0; t < TT; ++t) out[j * TT + t] = acc[j][t];
}

template <int WF, int TT>
__global__ void __launch_bounds__(kDecThreads, 1) decode_kernel(const DecodeArgs a) {
    using AT = __nv_bfloat16;
    using Sh = DecShape<WF, TT>;
    constexpr int DN = Sh::DN, SN = Sh::SN, RR = Sh::RR, SU = Sh::SU, BU = Sh::BU;
    constexpr int UA = Sh::UA, UB = Sh::UB, UC = Sh::UC;
    extern __shared__ uint4 dsm[];
    __shared__ DecSmem sm;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T = a.T, H = a.H, k = a.k, I = a.I, Is = a.Is, S = T * k, E = a.E;
    // grid-wide warp index, SM-major: item i goes to warp i / grid of SM i % grid, so that a
    // phase with fewer items than warps, or a partial last round, is spread over every SM
    const int gw = warp * gridDim.x + blockIdx.x, nw = gridDim.x * kDecWarps;
    const uint64_t deadline = gtimer() + kDecWaitNs;
    const int RB = (H + gridDim.x - 1) / gridDim.x;  // output rows per block
    const int r0 = min(H, int(blockIdx.x) * RB), r1 = min(H, r0 + RB), nr = r1 - r0;
    const bool blend = a.shared_mode == MOE_SHARED_BLEND;
    const int64_t drb = row_bytes<WF>(I);  // bytes of one routed down row
    const int dg = a.dense_group;
    const bool dq = a.dense_q4 != 0;
    const int64_t dhb = dq ? H / 2 : int64_t(H) * 2;   // bytes of a router / shared gate/up row
    const int64_t srb = dq ? Is / 2 : int64_t(Is) * 2;  // bytes of one shared down row
    auto dense_q = [&](const void* sc, const void* bi, int64_t row, int cols) -> QRow {
        if (!dq) return QRow{nullptr, nullptr, nullptr};
        const int64_t ng = cols / dg;
        return QRow{static_cast<const __nv_bfloat16*>(sc) + row * ng, static_cast<const __nv_bfloat16*>(bi) + row * ng,
                    nullptr};
    };

    // ------------------------------------------------------------ phase A
    AT* xs = reinterpret_cast<AT*>(dsm);
    float* xsum = reinterpret_cast<float*>(xs + int64_t(T) * H);  // 4-bit affine: sums per 32
    // selection keys of the top-k (phase B), after the staged tokens and their sums
    uint64_t* skeys = reinterpret_cast<uint64_t*>(dsm) + dec_keys_offset(T, H, WF == kQ4 || dq) / 8;
    if (a.has_sel)
        for (int e = threadIdx.x; e < E; e += blockDim.x) sm.ssel[e] = __ldg(a.sel_bias + e);
    if (WF == kQ4 || dq) stage_tokens<kQ4>(a.x, H, 0, T, nullptr, 1, xs, xsum);
    else stage_tokens<kBF16>(a.x, H, 0, T, nullptr, 1, xs, nullptr);
    __syncthreads();
    {
        const int n_rg = (E + RR - 1) / RR;           // router row groups
        const int n_cf = blend ? 2 : 0;                // coefficient rows (bf16)
        const int n_sh = Is ? (Is + SU - 1) / SU : 0;  // shared gate/up unit groups
        for (int it = gw; it < n_rg + n_cf + n_sh; it += nw) {
            if (it < n_rg) {  // RR router rows -> fp32 logits of every token
                const char* rows[RR];
                QRow q[RR];
#pragma unroll
                for (int j = 0; j < RR; ++j) {
                    const int e = min(it * RR + j, E - 1);
                    rows[j] = static_cast<const char*>(a.router_w) + int64_t(e) * dhb;
                    q[j] = dense_q(a.router_s, a.router_z, e, H);
                }
                float acc[RR * TT];
                if (dq) dec_dot<kQ4, RR, TT>(rows, q, H, dg, xs, xsum, T, nullptr, acc);
                else dec_dot<kBF16, RR, TT, UA>(rows, q, H, 64, xs, nullptr, T, nullptr, acc);
#pragma unroll
                for (int j = 0; j < RR; ++j) {
                    const int e = it * RR + j;
                    const float b = a.router_b ? bf16_ld(a.router_b, min(e, E - 1)) : 0.f;
#pragma unroll
                    for (int t = 0; t < TT; ++t)
                        if (t < T && e < E && lane == t) a.logits[int64_t(t) * a.ld_logits + e] = acc[j * TT + t] + b;
                }
            } else if (it < n_rg + n_cf) {  // one coefficient-head row (bf16), in the router's item shape
                const int c = it - n_rg;
                const char* rows[RR];
                QRow q[RR];
#pragma unroll
                for (int j = 0; j < RR; ++j) {
                    rows[j] = static_cast<const char*>(a.coef_w) + int64_t(c) * H * 2;
                    q[j] = QRow{nullptr, nullptr, nullptr};
                }
                float acc[RR * TT];
                dec_dot<kBF16, RR, TT, UA>(rows, q, H, 64, xs, nullptr, T, nullptr, acc);
                const float b = bf16_ld(a.coef_b, c);
#pragma unroll
                for (int t = 0; t < TT; ++t)
                    if (t < T && lane == t) a.logits[int64_t(t) * a.ld_logits + E + c] = acc[t] + b;
            } else {  // SU shared gate/up units
                const int i0 = (it - n_rg - n_cf) * SU;
                const char* rows[2 * SU];
                QRow q[2 * SU];
#pragma unroll
                for (int j = 0; j < SU; ++j) {
                    const int i = min(i0 + j, Is - 1);
                    rows[j] = static_cast<const char*>(a.sg_w) + int64_t(i) * dhb;
                    rows[SU + j] = static_cast<const char*>(a.su_w) + int64_t(i) * dhb;
                    q[j] = dense_q(a.sg_s, a.sg_z, i, H);
                    q[SU + j] = dense_q(a.su_s, a.su_z, i, H);
                }
                float acc[2 * SU * TT];
                if (dq) dec_dot<kQ4, 2 * SU, TT>(rows, q, H, dg, xs, xsum, T, nullptr, acc);
                else dec_dot<kBF16, 2 * SU, TT, UA>(rows, q, H, 64, xs, nullptr, T, nullptr, acc);
#pragma unroll
                for (int j = 0; j < SU; ++j)
#pragma unroll
                    for (int t = 0; t < TT; ++t)
                        if (t < T && i0 + j < Is && lane == t)
                            reinterpret_cast<AT*>(a.hs)[int64_t(t) * Is + i0 + j] = __float2bfloat16_rn(
                                act_apply(a.act, acc[j * TT + t], acc[(SU + j) * TT + t], a.limit, a.alpha));
            }
        }
    }
    bool ok = grid_barrier(&a.bar[0], gridDim.x, deadline, a.status, &sm.flag);

    // ------------------------------------------------------------ phase B
    if (ok) {
        {  // top-k of the T tokens, identical in every block
            TopkArgs ta;
            ta.logits = a.logits; ta.ld = a.ld_logits; ta.T = T; ta.E = E; ta.k = k;
            ta.scoring = a.scoring; ta.norm = a.norm; ta.has_sel = a.has_sel; ta.sel_bias = a.sel_bias;
            ta.blend = blend ? 1 : 0;
            ta.idx = sm.sidx; ta.w = sm.sw; ta.coef = sm.scoef;
            topk_block(ta, skeys, sm.sstat, sm.ssel, reinterpret_cast<float*>(skeys + T * E));
        }
        __syncthreads();
        // stable counting sort of the S slots by expert (a token's k experts are distinct,
        // so an expert holds at most T slots)
        const int s = threadIdx.x;
        int e = 0, lt = 0, eqb = 0;
        if (s < S) {
            e = sm.sidx[s];
            for (int u = 0; u < S; ++u) {
                const int f = sm.sidx[u];
                lt += f < e ? 1 : 0;
                eqb += (f == e && u < s) ? 1 : 0;
            }
            sm.sorted[lt + eqb] = s;
            sm.head[s] = eqb == 0 ? 1 : 0;
            sm.lt[s] = lt;
        }
        const int n_d = __syncthreads_count(s < S && eqb == 0);
        if (s < S && eqb == 0) {
            int d = 0;
            for (int u = 0; u < S; ++u) d += (sm.head[u] && sm.sidx[u] < e) ? 1 : 0;
            sm.dexp[d] = e;
            sm.doff[d] = lt;
        }
        if (threadIdx.x == 0) {
            sm.doff[n_d] = S;
            sm.n_d = n_d;
        }
        __syncthreads();
        // routed gate/up: BU units (gate + up rows) of one distinct expert per warp item
        const int ub = (I + BU - 1) / BU;
        const int64_t rbh = row_bytes<WF>(H);
        for (int it = gw; it < n_d * ub; it += nw) {
            const int d = it / ub, i0 = (it - d * ub) * BU;
            const int ex = sm.dexp[d];
            const int sb = sm.doff[d], cnt = sm.doff[d + 1] - sb;
            int tl[TT];
#pragma unroll
            for (int j = 0; j < TT; ++j) tl[j] = j < cnt ? sm.sorted[sb + j] / k : 0;
            const char* rows[2 * BU];
            QRow q[2 * BU];
            float bg[BU], bu[BU];
#pragma unroll
            for (int j = 0; j < BU; ++j) {
                const int i = min(i0 + j, I - 1);
                int64_t g0, g1;  // plane rows of the gate and the up weights
                if (a.interleaved) {
                    g0 = int64_t(ex) * 2 * I + 2 * i;
                    g1 = g0 + 1;
                    rows[j] = static_cast<const char*>(a.gate_up_w) + g0 * rbh;
                    rows[BU + j] = rows[j] + rbh;
                } else {
                    g0 = g1 = int64_t(ex) * I + i;
                    rows[j] = static_cast<const char*>(a.gate_w) + g0 * rbh;
                    rows[BU + j] = static_cast<const char*>(a.up_w) + g1 * rbh;
                }
                q[j] = q[BU + j] = QRow{nullptr, nullptr, nullptr};
                if constexpr (WF == kQ4) {
                    const int64_t ng = H / a.group_size;
                    const __nv_bfloat16* s0 = static_cast<const __nv_bfloat16*>(a.gate_s);
                    const __nv_bfloat16* z0 = static_cast<const __nv_bfloat16*>(a.gate_z);
                    const __nv_bfloat16* s1 = static_cast<const __nv_bfloat16*>(a.interleaved ? a.gate_s : a.up_s);
                    const __nv_bfloat16* z1 = static_cast<const __nv_bfloat16*>(a.interleaved ? a.gate_z : a.up_z);
                    q[j] = {s0 + g0 * ng, z0 + g0 * ng, nullptr};
                    q[BU + j] = {s1 + g1 * ng, z1 + g1 * ng, nullptr};
                } else if constexpr (WF == kMX4) {
                    const uint8_t* s0 = static_cast<const uint8_t*>(a.gate_s);
                    const uint8_t* s1 = static_cast<const uint8_t*>(a.interleaved ? a.gate_s : a.up_s);
                    q[j] = {nullptr, nullptr, s0 + g0 * (H / 32)};
                    q[BU + j] = {nullptr, nullptr, s1 + g1 * (H / 32)};
                }
                bg[j] = bu[j] = 0.f;
                if (a.has_bias) {
                    if (a.interleaved) {
                        bg[j] = bf16_ld(a.gate_up_b, int64_t(ex) * 2 * I + 2 * i);
                        bu[j] = bf16_ld(a.gate_up_b, int64_t(ex) * 2 * I + 2 * i + 1);
                    } else {
                        bg[j] = bf16_ld(a.gate_b, int64_t(ex) * I + i);
                        bu[j] = bf16_ld(a.up_b, int64_t(ex) * I + i);
                    }
                }
            }
            float acc[2 * BU * TT];
            dec_dot<WF, 2 * BU, TT, UB>(rows, q, H, a.group_size, xs, xsum, cnt, tl, acc);
#pragma unroll
            for (int j = 0; j < BU; ++j)
#pragma unroll
                for (int t = 0; t < TT; ++t)
                    if (t < cnt && i0 + j < I && lane == t)
                        reinterpret_cast<AT*>(a.h)[int64_t(sm.sorted[sb + t]) * I + i0 + j] = __float2bfloat16_rn(
                            act_apply(a.act, acc[j * TT + t] + bg[j], acc[(BU + j) * TT + t] + bu[j], a.limit, a.alpha));
        }
        ok = grid_barrier(&a.bar[1], gridDim.x, deadline, a.status, &sm.flag);
    }

    // ------------------------------------------------------------ phase C
    if (ok) {
        const int n_d = sm.n_d;
        AT* hsm = reinterpret_cast<AT*>(dsm);                          // [S, I] by slot
        float* hsum = reinterpret_cast<float*>(hsm + int64_t(S) * I);  // 4-bit affine: sums per 32
        AT* hss = reinterpret_cast<AT*>(hsum + (WF == kQ4 ? int64_t(S) * (I / 32) : 0));  // [T, Is]
        float* hssum = reinterpret_cast<float*>(hss + int64_t(T) * Is);  // 4-bit shared down: sums per 32
        copy_cg(reinterpret_cast<uint4*>(hsm), a.h, int64_t(S) * I / 8);
        if (Is) copy_cg(reinterpret_cast<uint4*>(hss), a.hs, int64_t(T) * Is / 8);
        for (int i = threadIdx.x; i < nr * kTT; i += blockDim.x) {
            sm.acc_r[i / kTT][i % kTT] = 0.f;
            sm.acc_s[i / kTT][i % kTT] = 0.f;
        }
        __syncthreads();
        auto sums32 = [&](const AT* rowsrc, int nrows, int cols, float* dst) {  // per-32 sums of rows
            const int nv = cols / 32;
            for (int i = threadIdx.x; i < nrows * nv; i += blockDim.x) {
                const uint4* p = reinterpret_cast<const uint4*>(rowsrc + int64_t(i / nv) * cols + (i % nv) * 32);
                float sum = 0.f;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    float f[8];
                    unpack8(p[j], f);
#pragma unroll
                    for (int n = 0; n < 8; ++n) sum += f[n];
                }
                dst[i] = sum;
            }
        };
        if (dq && Is) sums32(hss, T, Is, hssum);
        if (WF == kQ4) sums32(hsm, S, I, hsum);
        if (WF == kQ4 || (dq && Is)) __syncthreads();
        const int nq = (nr + DN - 1) / DN, nsq = (nr + SN - 1) / SN;
        const int n_items = n_d * nq + (Is ? nsq : 0);
        for (int it = warp; it < n_items; it += kDecWarps) {
            if (it < n_d * nq) {  // DN down rows of one distinct expert
                const int d = it / nq, qq = it - d * nq;
                const int ex = sm.dexp[d];
                const int sb = sm.doff[d], cnt = sm.doff[d + 1] - sb;
                int tl[TT];
#pragma unroll
                for (int j = 0; j < TT; ++j) tl[j] = j < cnt ? sm.sorted[sb + j] : 0;  // slot rows of hsm
                const char* rows[DN];
                QRow q[DN];
                float bd[DN];
#pragma unroll
                for (int jr = 0; jr < DN; ++jr) {
                    const int r = min(r0 + qq * DN + jr, r1 - 1);
                    const int64_t gr = int64_t(ex) * H + r;
                    rows[jr] = static_cast<const char*>(a.down_w) + gr * drb;
                    q[jr] = {nullptr, nullptr, nullptr};
                    if constexpr (WF == kQ4) {
                        const int64_t ng = I / a.group_size;
                        q[jr] = {static_cast<const __nv_bfloat16*>(a.down_s) + gr * ng,
                                 static_cast<const __nv_bfloat16*>(a.down_z) + gr * ng, nullptr};
                    } else if constexpr (WF == kMX4) {
                        q[jr] = {nullptr, nullptr, static_cast<const uint8_t*>(a.down_s) + gr * (I / 32)};
                    }
                    bd[jr] = a.has_bias ? bf16_ld(a.down_b, gr) : 0.f;
                }
                float acc[DN * TT];
                dec_dot<WF, DN, TT, UC>(rows, q, I, a.group_size, hsm, hsum, cnt, tl, acc);
#pragma unroll
                for (int jr = 0; jr < DN; ++jr)
#pragma unroll
                    for (int j = 0; j < TT; ++j) {
                        const int rl = qq * DN + jr;
                        if (j < cnt && lane == 0 && rl < nr) {
                            const int slot = tl[j];
                            atomicAdd(&sm.acc_r[rl][slot / k], sm.sw[slot] * (acc[jr * TT + j] + bd[jr]));
                        }
                    }
            } else {  // SN rows of the shared expert's down projection, every token
                const int qq = it - n_d * nq;
                const char* rows[SN];
                QRow q[SN];
#pragma unroll
                for (int jr = 0; jr < SN; ++jr) {
                    const int64_t r = min(r0 + qq * SN + jr, r1 - 1);
                    rows[jr] = static_cast<const char*>(a.sd_w) + r * srb;
                    q[jr] = dense_q(a.sd_s, a.sd_z, r, Is);
                }
                float acc[SN * TT];
                if (dq) dec_dot<kQ4, SN, TT>(rows, q, Is, dg, hss, hssum, T, nullptr, acc);
                else dec_dot<kBF16, SN, TT>(rows, q, Is, 64, hss, nullptr, T, nullptr, acc);
#pragma unroll
                for (int jr = 0; jr < SN; ++jr)
#pragma unroll
                    for (int t = 0; t < TT; ++t) {
                        const int rl = qq * SN + jr;
                        if (t < T && lane == 0 && rl < nr) sm.acc_s[rl][t] = acc[jr * TT + t];
                    }
            }
        }
        __syncthreads();
        // y = y_r | y_r + s | c0 y_r + c1 s for the block's rows (Klear PR item 2)
        for (int i = threadIdx.x; i < T * nr; i += blockDim.x) {
            const int t = i / nr, rl = i - t * nr;
            const float yr = sm.acc_r[rl][t], sv = sm.acc_s[rl][t];
            float v = yr;
            if (a.shared_mode == MOE_SHARED_ADD) v = yr + sv;
            else if (blend) v = yr * sm.scoef[2 * t] + sv * sm.scoef[2 * t + 1];
            reinterpret_cast<AT*>(a.y)[int64_t(t) * H + r0 + rl] = __float2bfloat16_rn(v);
        }
    }

    // the last block out resets the barrier counters for the next launch
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(&a.bar[2], 1u) == gridDim.x - 1) {
            a.bar[0] = 0;
            a.bar[1] = 0;
            __threadfence();
            a.bar[2] = 0;
        }
    }
}

template <int WF>
cudaError_t launch_decode_t(const DecodeArgs& a, size_t smem, cudaStream_t s) {
    auto kern = a.T == 1 ? decode_kernel<WF, 1> : decode_kernel<WF, kTT>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (err != cudaSuccess) return err;
    int dev = 0, sms = 0, per_sm = 0;
    if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
    if ((err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return err;
    if ((err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kDecThreads, smem)) != cudaSuccess)
        return err;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const int grid = sms * std::min(per_sm, 1);  // one block per SM: every block is resident
    if ((a.H + grid - 1) / grid > kDecRowsMax) return cudaErrorInvalidConfiguration;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kDecThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;  // co-residency of all blocks (grid barriers)
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    err = cudaLaunchKernelEx(&cfg, kern, a);
    if (err != cudaSuccess) return err;
    return cudaGetLastError();
}

}  // namespace

size_t decode_smem_bytes(const DecodeArgs& a) {
    if (a.T < 1 || a.T > kTT || a.k > kMaxTopK || a.E > kMaxExperts) return 0;
    if (a.wf != kBF16 && a.wf != kQ4 && a.wf != kMX4) return 0;
    const size_t S = size_t(a.T) * a.k;
    const bool q4 = a.wf == kQ4;
    const size_t pa = dec_keys_offset(a.T, a.H, q4 || a.dense_q4) + size_t(a.T) * a.E * 12;  // keys + logits
    const size_t pc = S * a.I * 2 + (q4 ? S * (a.I / 32) * 4 : 0) + size_t(a.T) * a.Is * 2 +
                      (a.dense_q4 ? size_t(a.T) * (a.Is / 32) * 4 : 0);
    const size_t need = (std::max(pa, pc) + 15) & ~size_t(15);
    return need <= kDecSmemMax ? need : 0;
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s) {
    const size_t smem = decode_smem_bytes(a);
    if (smem == 0) return cudaErrorInvalidValue;
    switch (a.wf) {
        case kBF16: return launch_decode_t<kBF16>(a, smem, s);
        case kQ4: return launch_decode_t<kQ4>(a, smem, s);
        case kMX4: return launch_decode_t<kMX4>(a, smem, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace moe
