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

// Top-k, combine weights and blend coefficients of token t, computed by one warp.
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
    auto score_of = [&](float logit) {
        if (a.scoring == MOE_SCORING_SOFTMAX_ALL) return expf(logit - m) * inv_sum;
        if (a.scoring == MOE_SCORING_SIGMOID) return 1.0f / (1.0f + expf(-logit));
        return logit;
    };
    uint64_t packed[kPerLane];
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) {
        const int e = lane + 32 * i;
        packed[i] = 0;  // below every real key
        if (e < E) packed[i] = pack_key(score_of(l[i]) + sb[i], e);
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
    // combine weights: unbiased scores of the chosen experts, or softmax over their logits
    const bool mine = lane < a.k;
    float w;
    if (a.scoring == MOE_SCORING_SOFTMAX_TOPK) {
        const float mm = warp_max(my_l);
        const float ex = mine ? expf(my_l - mm) : 0.f;
        w = ex / warp_sum(ex);
    } else {
        w = mine ? score_of(my_l) : 0.f;
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

}  // namespace
}  // namespace moe
