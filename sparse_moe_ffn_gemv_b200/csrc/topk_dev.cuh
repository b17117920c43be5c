// topk_dev.cuh -- scoring, select-only bias, top-k and combine weights of one token (a2).
//
// One warp per token over the fp32 router logits (Klear PR item 3: sigmoid of fp32 logits,
// the expert bias added to a copy used only for selection, the returned scores gathered
// unbiased, norm_topk_prob; libmir-metal ClampedRoutedExperts::forward:
// router_top_k_unit(top_k), i.e. softmax over the selected logits; softmax over all experts
// otherwise). The 2-way blend coefficients (Klear PR item 2) are the softmax of the two
// logits stored after the E router logits. Logits are read through L2 (__ldcg): another
// block of the same launch may have written them.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kPerLane = kMaxExperts / kWarp;  // 16 experts per lane at most

// Order-preserving packing of (selection key, expert): a larger key wins, and among
// equal keys the lower expert index wins (its complement is larger).
__device__ __forceinline__ uint64_t pack_key(float key, int e) {
    uint32_t u = __float_as_uint(key);
    u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return (uint64_t(u) << 32) | uint32_t(0xFFFFFFFFu - uint32_t(e));
}

__device__ __forceinline__ uint64_t warp_max_u64(uint64_t v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const uint64_t w = __shfl_xor_sync(0xffffffffu, v, o);
        v = w > v ? w : v;
    }
    return v;
}

// Selection key of one expert: its score (sigmoid, softmax over all experts with the token's
// max m and 1 / sum, or the raw logit) plus the select-only bias, packed with the index.
__device__ __forceinline__ uint64_t select_key(const TopkArgs& a, float logit, float sb, int e, float m,
                                               float inv_sum) {
    float score = logit;
    if (a.scoring == MOE_SCORING_SOFTMAX_ALL) score = expf(logit - m) * inv_sum;
    else if (a.scoring == MOE_SCORING_SIGMOID) score = 1.0f / (1.0f + expf(-logit));
    return pack_key(score + sb, e);
}

// Combine weights of token t from its choices (lane j < k holds the j-th chosen expert my_e
// and its logit my_l), then the writes: indices, weights, blend coefficients, and for one
// token its slot permutation and the cleared rows.
__device__ __forceinline__ void finish_token(const TopkArgs& a, int64_t t, int my_e, float my_l, float m,
                                             float inv_sum) {
    const int lane = threadIdx.x & 31;
    const float* lg = a.logits + t * a.ld;
    const int E = a.E;
    // combine weights: unbiased scores of the chosen experts, or softmax over their logits
    const bool mine = lane < a.k;
    float w;
    if (a.scoring == MOE_SCORING_SOFTMAX_TOPK) {
        const float mm = warp_max(my_l);
        const float ex = mine ? expf(my_l - mm) : 0.f;
        w = ex / warp_sum(ex);
    } else if (a.scoring == MOE_SCORING_SOFTMAX_ALL) {
        w = mine ? expf(my_l - m) * inv_sum : 0.f;
    } else if (a.scoring == MOE_SCORING_SIGMOID) {
        w = mine ? 1.0f / (1.0f + expf(-my_l)) : 0.f;
    } else {
        w = mine ? my_l : 0.f;
    }
    if (a.norm) w = w / warp_sum(w);
    if (mine) {
        a.idx[t * a.k + lane] = my_e;
        a.w[t * a.k + lane] = w;
    }
    if (a.blend && lane == 0) {
        const float c0 = __ldcg(lg + E), c1 = __ldcg(lg + E + 1);
        const float cm = fmaxf(c0, c1);
        const float e0 = expf(c0 - cm), e1 = expf(c1 - cm);
        a.coef[t * 2 + 0] = e0 / (e0 + e1);
        a.coef[t * 2 + 1] = e1 / (e0 + e1);
    }
    if (a.p_offsets) {
        // One token (t == 0): its k slots sorted by expert. The experts of a token's top-k
        // are distinct, so a slot's rank is the number of chosen experts below its own.
        int ek[kMaxTopK];
#pragma unroll
        for (int q = 0; q < kMaxTopK; ++q) ek[q] = q < a.k ? __shfl_sync(0xffffffffu, my_e, q) : 0x7fffffff;
        if (mine) {
            int rank = 0;
#pragma unroll
            for (int q = 0; q < kMaxTopK; ++q) rank += ek[q] < my_e ? 1 : 0;
            a.p_sorted[rank] = lane;
            a.p_slot_pos[lane] = rank;
            a.p_active[1 + rank] = my_e;
        }
        for (int e = lane; e <= a.E; e += 32) {
            int below = 0;
#pragma unroll
            for (int q = 0; q < kMaxTopK; ++q) below += ek[q] < e ? 1 : 0;
            a.p_offsets[e] = below;
            if (a.p_tiles) a.p_tiles[e] = below;  // one token per active expert: one tile each
        }
        if (lane == 0) a.p_active[0] = a.k;
    }
    if (a.zero) {
        float4* z = reinterpret_cast<float4*>(a.zero + t * a.zero_cols);
        for (int64_t c = lane; c < a.zero_cols / 4; c += 32) z[c] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

// Top-k, combine weights and blend coefficients of token t, computed by one warp with the
// keys in registers (the top-k kernel: one warp per token of a batch).
__device__ __forceinline__ void topk_token(const TopkArgs& a, int64_t t) {
    const int lane = threadIdx.x & 31;
    const float* lg = a.logits + t * a.ld;
    const int E = a.E;

    // this lane's experts: lane, lane + 32, ...; logits and select-only biases loaded together
    float l[kPerLane], sb[kPerLane];
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) {
        const int e = lane + 32 * i;
        l[i] = e < E ? __ldcg(lg + e) : -INFINITY;
        sb[i] = (e < E && a.has_sel) ? __ldg(a.sel_bias + e) : 0.f;
    }
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) m = fmaxf(m, l[i]);
    float inv_sum = 1.f;
    if (a.scoring == MOE_SCORING_SOFTMAX_ALL) {
        m = warp_max(m);
        float sum = 0.f;
#pragma unroll
        for (int i = 0; i < kPerLane; ++i)
            if (lane + 32 * i < E) sum += expf(l[i] - m);
        inv_sum = 1.0f / warp_sum(sum);
    }
    uint64_t packed[kPerLane];
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) {
        const int e = lane + 32 * i;
        packed[i] = 0;  // below every real key
        if (e < E) packed[i] = select_key(a, l[i], sb[i], e, m, inv_sum);
    }
    // k rounds of a warp arg-max; lane j keeps the j-th choice and its logit (from the
    // registers of the lane that owns the expert)
    int my_e = -1;
    float my_l = -INFINITY;
    for (int j = 0; j < a.k; ++j) {
        uint64_t best = 0;
#pragma unroll
        for (int i = 0; i < kPerLane; ++i) best = packed[i] > best ? packed[i] : best;
        best = warp_max_u64(best);
        float won = 0.f;
#pragma unroll
        for (int i = 0; i < kPerLane; ++i)
            if (packed[i] == best) {
                packed[i] = 0;
                won = l[i];
            }
        const int e = int(0xFFFFFFFFu - uint32_t(best & 0xFFFFFFFFu));
        won = __shfl_sync(0xffffffffu, won, e & 31);
        if (lane == j) {
            my_e = e;
            my_l = won;
        }
    }
    finish_token(a, t, my_e, my_l, m, inv_sum);
}

// The same top-k for the T (<= 8) tokens of a decode batch, by one whole block, with the keys
// in shared memory (skeys: T * E words) and rolled loops: the decode kernel runs this once
// per SM, with the instruction caches cold, so few distinct instructions matter more than
// registers. Same keys, tie-breaking and arithmetic as topk_token (identical results).
// ssel: the select-only biases already staged in shared memory (or null: read from global);
// slog: T * E floats of shared memory that keep the logits for the combine weights.
// Every thread of the block calls it; warp t < T finishes token t.
__device__ __forceinline__ void topk_block(const TopkArgs& a, uint64_t* skeys, float* sstat, const float* ssel,
                                           float* slog) {
    const int T = int(a.T), E = a.E;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (a.scoring == MOE_SCORING_SOFTMAX_ALL) {  // each token's max and 1 / sum, lane order as above
        if (warp < T) {
            const float* lg = a.logits + int64_t(warp) * a.ld;
            float m = -INFINITY;
#pragma unroll 1
            for (int e = lane; e < E; e += 32) m = fmaxf(m, __ldcg(lg + e));
            m = warp_max(m);
            float sum = 0.f;
#pragma unroll 1
            for (int e = lane; e < E; e += 32) sum += expf(__ldcg(lg + e) - m);
            sum = warp_sum(sum);
            if (lane == 0) {
                sstat[2 * warp] = m;
                sstat[2 * warp + 1] = 1.0f / sum;
            }
        }
        __syncthreads();
    }
#pragma unroll 1
    for (int i = threadIdx.x; i < T * E; i += blockDim.x) {
        const int t = i / E, e = i - t * E;
        const bool sa = a.scoring == MOE_SCORING_SOFTMAX_ALL;
        const float l = __ldcg(a.logits + int64_t(t) * a.ld + e);
        const float sb = a.has_sel ? (ssel ? ssel[e] : __ldg(a.sel_bias + e)) : 0.f;
        slog[i] = l;
        skeys[i] = select_key(a, l, sb, e, sa ? sstat[2 * t] : 0.f, sa ? sstat[2 * t + 1] : 1.f);
    }
    __syncthreads();
    if (warp >= T) return;
    uint64_t* kt = skeys + int64_t(warp) * E;
    int my_e = -1;
#pragma unroll 1
    for (int j = 0; j < a.k; ++j) {
        uint64_t best = 0;
#pragma unroll 1
        for (int e = lane; e < E; e += 32) {
            const uint64_t v = kt[e];
            best = v > best ? v : best;
        }
        best = warp_max_u64(best);
        const int e = int(0xFFFFFFFFu - uint32_t(best & 0xFFFFFFFFu));
        if (lane == (e & 31)) kt[e] = 0;  // the expert's owner lane takes it out
        __syncwarp();
        if (lane == j) my_e = e;
    }
    const float my_l = lane < a.k ? slog[warp * E + my_e] : -INFINITY;
    const bool sa = a.scoring == MOE_SCORING_SOFTMAX_ALL;
    finish_token(a, warp, my_e, my_l, sa ? sstat[2 * warp] : 0.f, sa ? sstat[2 * warp + 1] : 1.f);
}

}  // namespace
}  // namespace moe
