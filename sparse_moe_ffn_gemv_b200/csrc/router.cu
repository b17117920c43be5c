// router.cu -- scoring, select-only bias, top-k and combine weights (a2).
//
// One warp per token over the fp32 router logits (Klear PR item 3: sigmoid of
// fp32 logits, the expert bias added to a copy used only for selection, the
// returned scores gathered unbiased, norm_topk_prob; libmir-metal
// ClampedRoutedExperts::forward: router_top_k_unit(top_k), i.e. softmax over
// the selected logits; softmax over all experts otherwise). The 2-way blend
// coefficients (Klear PR item 2) are the softmax of the two logits stored
// after the E router logits.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int kPerLane = kMaxExperts / kWarp;  // 16 experts per lane at most

__global__ void __launch_bounds__(256) topk_kernel(TopkArgs a) {
    const int lane = threadIdx.x & 31;
    const int64_t t = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    if (t >= a.T) return;
    const float* lg = a.logits + t * a.ld;
    const int E = a.E;
    const int nper = (E + 31) >> 5;

    float score[kPerLane], key[kPerLane];
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) {
        const int e = lane + 32 * i;
        score[i] = (i < nper && e < E) ? lg[e] : -INFINITY;
        m = fmaxf(m, score[i]);
    }
    if (a.scoring == MOE_SCORING_SOFTMAX_ALL) {
        m = warp_max(m);
        float sum = 0.f;
#pragma unroll
        for (int i = 0; i < kPerLane; ++i) {
            const int e = lane + 32 * i;
            score[i] = (i < nper && e < E) ? expf(score[i] - m) : 0.f;
            sum += score[i];
        }
        sum = warp_sum(sum);
        const float inv = 1.0f / sum;
#pragma unroll
        for (int i = 0; i < kPerLane; ++i) score[i] *= inv;
    } else if (a.scoring == MOE_SCORING_SIGMOID) {
#pragma unroll
        for (int i = 0; i < kPerLane; ++i) score[i] = 1.0f / (1.0f + expf(-score[i]));
    }
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) {
        const int e = lane + 32 * i;
        const bool valid = i < nper && e < E;
        key[i] = valid ? score[i] + (a.has_sel ? a.sel_bias[e] : 0.f) : -INFINITY;
    }

    // k rounds of a warp arg-max; equal keys rank the lower expert index first.
    uint32_t taken = 0;
    int sel[kMaxTopK];
    float sel_score[kMaxTopK];
    for (int j = 0; j < a.k; ++j) {
        float bk = -INFINITY;
        int be = 0x7fffffff;
        float bs = 0.f;
#pragma unroll
        for (int i = 0; i < kPerLane; ++i) {
            const int e = lane + 32 * i;
            if (i < nper && e < E && !((taken >> i) & 1u) && key[i] > bk) {
                bk = key[i];
                be = e;
                bs = score[i];
            }
        }
        // an untaken valid key of -inf (impossible for finite logits) never beats be
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ok = __shfl_xor_sync(0xffffffffu, bk, o);
            const int oe = __shfl_xor_sync(0xffffffffu, be, o);
            const float os = __shfl_xor_sync(0xffffffffu, bs, o);
            if (ok > bk || (ok == bk && oe < be)) {
                bk = ok;
                be = oe;
                bs = os;
            }
        }
        if ((be & 31) == lane) taken |= 1u << (be >> 5);
        sel[j] = be;
        sel_score[j] = bs;
    }

    float w[kMaxTopK];
    if (a.scoring == MOE_SCORING_SOFTMAX_TOPK) {
        float mm = -INFINITY;
        for (int j = 0; j < a.k; ++j) mm = fmaxf(mm, sel_score[j]);
        float sum = 0.f;
        for (int j = 0; j < a.k; ++j) {
            w[j] = expf(sel_score[j] - mm);
            sum += w[j];
        }
        for (int j = 0; j < a.k; ++j) w[j] /= sum;
    } else {
        for (int j = 0; j < a.k; ++j) w[j] = sel_score[j];
    }
    if (a.norm) {
        float sum = 0.f;
        for (int j = 0; j < a.k; ++j) sum += w[j];
        for (int j = 0; j < a.k; ++j) w[j] /= sum;
    }
    for (int j = 0; j < a.k; ++j) {
        if (lane == j) {
            a.idx[t * a.k + j] = sel[j];
            a.w[t * a.k + j] = w[j];
        }
    }
    if (a.blend && lane == 0) {
        const float c0 = lg[E], c1 = lg[E + 1];
        const float cm = fmaxf(c0, c1);
        const float e0 = expf(c0 - cm), e1 = expf(c1 - cm);
        a.coef[t * 2 + 0] = e0 / (e0 + e1);
        a.coef[t * 2 + 1] = e1 / (e0 + e1);
    }
    if (a.zero) {
        float4* z = reinterpret_cast<float4*>(a.zero + t * a.zero_cols);
        for (int64_t c = lane; c < a.zero_cols / 4; c += 32) z[c] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

}  // namespace

cudaError_t launch_topk(const TopkArgs& a, cudaStream_t s) {
    if (a.T == 0) return cudaSuccess;
    const int64_t threads = a.T * 32;
    const unsigned grid = unsigned((threads + 255) / 256);
    topk_kernel<<<grid, 256, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace moe
