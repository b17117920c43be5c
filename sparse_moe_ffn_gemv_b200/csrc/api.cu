// api.cu -- the C ABI: host-side validation, workspace layout and launch order.
//
// Every check that the host can make runs before the first launch (Klear PR
// "Other guards": zero checks before divisibility, k within 1..=E, positive
// finite eps, a blend without its coefficient head rejected; mlxcel issue #974:
// quantisation parameters bounded where they enter, errors returned instead of
// an abort crossing the boundary).
#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>

#include "common.cuh"
#include "internal.h"

namespace moe {

int64_t max_routed_tiles(const moe_config& c, int64_t T) {
    const int64_t S = T * c.top_k;
    return (S + kTcBN - 1) / kTcBN + std::min<int64_t>(c.num_experts, S);  // the smaller tile height
}

WsLayout ws_layout(const moe_config& c, int64_t T) {
    WsLayout L{};
    size_t off = 0;
    auto take = [&](int64_t bytes) {
        const size_t o = off;
        off = align256(off + size_t(bytes > 0 ? bytes : 0));
        return o;
    };
    const int64_t E = c.num_experts, k = c.top_k, I = c.intermediate, H = c.hidden;
    const int64_t K = expert_in(c), Ld = c.latent_dim, Is = c.shared_intermediate;
    const int64_t ab = act_bytes(c);
    L.T = T;
    L.ld_logits = int((E + 2 + 3) & ~int64_t(3));
    L.n_chunks = int((T * k + kPermChunkWs - 1) / kPermChunkWs);
    L.status = take(256);
    L.logits = take(T * L.ld_logits * 4);
    L.topk_idx = take(T * k * 4);
    L.topk_w = take(T * k * 4);
    L.coef = take(T * 2 * 4);
    L.offsets = take((E + 1) * 4);
    L.sorted_slot = take(T * k * 4);
    L.slot_pos = take(T * k * 4);
    L.active = take((E + 1) * 4);
    L.chunk_hist = take(int64_t(L.n_chunks > 0 ? L.n_chunks : 1) * E * 4);
    L.h = take(T * k * I * ab);
    L.hs = take(T * Is * ab);
    L.y_acc = take(T * K * 4);
    L.s_acc = take(c.shared_mode != MOE_SHARED_NONE ? T * H * 4 : 0);
    L.z = take(Ld ? T * Ld * ab : 0);
    L.nrm = take(Ld ? T * Ld * ab : 0);
    L.tiles = take((E + 1) * 4);
    L.uperm = take(c.act_dtype == MOE_DTYPE_BF16 ? T * k * K * 2 : 0);
    // fp16 copies of the dense token operands of 4-bit dense planes on the tensor cores
    const bool dq = c.dense_format == MOE_DTYPE_Q4_AFFINE;
    L.x16 = take(dq ? T * H * 2 : 0);
    L.n16 = take(Ld && dq ? T * Ld * 2 : 0);
    L.total = off;
    return L;
}

}  // namespace moe

using namespace moe;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool finite_pos(float v) { return std::isfinite(v) && v > 0.f; }

bool dense_q4(const moe_config* c) { return c->dense_format == MOE_DTYPE_Q4_AFFINE; }

// Token rows per tensor-core tile. 128 in launches that dequantise 4-bit weights (their
// shared memory holds the packed-weight ring as well) and on small bf16 batches (four stages
// of weights in flight per SM, where the launch streams weights for a few tokens); 256 on
// large bf16 batches, where a weight tile then serves twice the token rows (an expert with
// 129..256 routed rows reads its weights once instead of twice). The expert launches carry
// the routed and the shared problem, the dense launches one projection. Wide tiles keep one
// accumulator set (the epilogue of a tile no longer overlaps the next tile's main loop), so
// they pay only where most experts hold more than 128 routed rows (measured: latent block at
// 8192 tokens, 170 rows per expert on average, expert gate/up 2.97 -> 2.63 ms; Klear at 4096
// tokens, 128 on average, block 0.71 -> 0.78 ms), and in dense launches that still give
// every SM two tiles or more (a router of 384 rows at 8192 tokens has 64 wide tiles: 84 ->
// 113 us).
int expert_bn(const moe_config* c, int64_t T) {
    const bool q = c->weight_format == MOE_DTYPE_Q4_AFFINE || c->weight_format == MOE_DTYPE_MXFP4 || dense_q4(c);
    return !q && T * c->top_k >= 160 * int64_t(c->num_experts) ? kTcBNWide : kTcBN;
}
int dense_bn(const moe_config* c, int64_t T, int M) {
    const int64_t wide_tiles = int64_t((M + kTcRows - 1) / kTcRows) * ((T + kTcBNWide - 1) / kTcBNWide);
    return !dense_q4(c) && wide_tiles >= 2 * int64_t(device_sm_count()) ? kTcBNWide : kTcBN;
}

// Weight operand(s) of a dense (one-group) tensor-core problem: bf16 [M, K], or 4-bit affine
// words [M, K / 8] with bf16 scales / biases per dense_group_size columns (the second
// operand w1 only in gate/up mode).
bool tc_dense_weights(const moe_config* c, TcProblem& p, CUtensorMap* m0, CUtensorMap* m1, const void* w0,
                      const void* s0, const void* z0, const void* w1, const void* s1, const void* z1, int M, int K) {
    if (dense_q4(c)) {
        p.q4 = 1;
        p.mx = 0;
        p.group_size = c->dense_group_size;
        p.qs0 = s0; p.qz0 = z0; p.qs1 = s1; p.qz1 = z1;
        return tc_q4_weight_map(m0, w0, 1, M, K) && (!w1 || tc_q4_weight_map(m1, w1, 1, M, K));
    }
    return tc_weight_map(m0, w0, 1, M, K, false) && (!w1 || tc_weight_map(m1, w1, 1, M, K, false));
}


moe_status validate_config(const moe_config* c) {
    if (!c) return MOE_ERR_INVALID_ARGUMENT;
    // zero / sign checks first, divisibility afterwards
    if (c->hidden <= 0 || c->num_experts <= 0 || c->top_k <= 0 || c->intermediate <= 0)
        return MOE_ERR_INVALID_ARGUMENT;
    if (c->top_k > c->num_experts || c->top_k > kMaxTopK || c->num_experts > kMaxExperts)
        return MOE_ERR_INVALID_ARGUMENT;
    if (c->scoring < MOE_SCORING_SOFTMAX_ALL || c->scoring > MOE_SCORING_SOFTMAX_TOPK)
        return MOE_ERR_INVALID_ARGUMENT;
    if (c->activation != MOE_ACT_SWIGLU && c->activation != MOE_ACT_SWIGLU_CLAMPED)
        return MOE_ERR_INVALID_ARGUMENT;
    if (c->shared_mode < MOE_SHARED_NONE || c->shared_mode > MOE_SHARED_BLEND) return MOE_ERR_INVALID_ARGUMENT;
    if (c->act_dtype != MOE_DTYPE_F32 && c->act_dtype != MOE_DTYPE_BF16) return MOE_ERR_INVALID_ARGUMENT;
    if (c->weight_format < MOE_DTYPE_F32 || c->weight_format > MOE_DTYPE_MXFP4)
        return MOE_ERR_INVALID_ARGUMENT;
    if (c->shared_intermediate < 0 || c->latent_dim < 0) return MOE_ERR_INVALID_ARGUMENT;
    if ((c->shared_mode == MOE_SHARED_NONE) != (c->shared_intermediate == 0)) return MOE_ERR_INVALID_ARGUMENT;
    if (c->latent_use_norm && !c->latent_dim) return MOE_ERR_INVALID_ARGUMENT;
    if (c->latent_use_norm && !finite_pos(c->rms_eps)) return MOE_ERR_INVALID_ARGUMENT;
    if (c->activation == MOE_ACT_SWIGLU_CLAMPED &&
        (!finite_pos(c->swiglu_limit) || !std::isfinite(c->swiglu_alpha)))
        return MOE_ERR_INVALID_ARGUMENT;
    // routed_scaling_factor: declared by some checkpoints, never applied (Klear PR item 3)
    if (c->routed_scaling_factor != 1.0f) return MOE_ERR_UNSUPPORTED;
    // weight format <-> activation dtype
    if ((c->weight_format == MOE_DTYPE_F32) != (c->act_dtype == MOE_DTYPE_F32)) return MOE_ERR_UNSUPPORTED;
    const int K = expert_in(*c);
    if (c->weight_format == MOE_DTYPE_Q4_AFFINE) {
        if (c->bits != 4) return MOE_ERR_INVALID_QUANTIZATION;
        if (c->group_size != 32 && c->group_size != 64 && c->group_size != 128)
            return MOE_ERR_INVALID_QUANTIZATION;
        if (K % c->group_size != 0 || c->intermediate % c->group_size != 0)
            return MOE_ERR_INVALID_QUANTIZATION;
    }
    if (c->weight_format == MOE_DTYPE_MXFP4) {  // OCP MX: blocks of 32 elements, 4-bit E2M1
        if (c->bits != 4 || c->group_size != 32) return MOE_ERR_INVALID_QUANTIZATION;
        if (K % 64 != 0 || c->intermediate % 64 != 0) return MOE_ERR_INVALID_QUANTIZATION;
    }
    // 4-bit dense planes (router, shared expert, latent projections)
    if (c->dense_format != 0 && c->dense_format != MOE_DTYPE_Q4_AFFINE) return MOE_ERR_INVALID_ARGUMENT;
    if (c->dense_format == MOE_DTYPE_Q4_AFFINE) {
        if (c->act_dtype != MOE_DTYPE_BF16) return MOE_ERR_UNSUPPORTED;
        const int g = c->dense_group_size;
        if (g != 32 && g != 64 && g != 128) return MOE_ERR_INVALID_QUANTIZATION;
        if (c->hidden % g || c->shared_intermediate % g || c->latent_dim % g) return MOE_ERR_INVALID_QUANTIZATION;
    }
    // 16-byte rows
    const int q = c->act_dtype == MOE_DTYPE_F32 ? 4 : 8;
    if (c->hidden % q || c->intermediate % q || K % q || c->shared_intermediate % q) return MOE_ERR_INVALID_ARGUMENT;
    // sizes of the stacked planes must fit the index arithmetic
    const int64_t plane = int64_t(c->num_experts) * 2 * c->intermediate * K;
    if (plane / c->num_experts / 2 / c->intermediate != K || plane > (int64_t(1) << 46))
        return MOE_ERR_SHAPE_OVERFLOW;
    return MOE_OK;
}

moe_status validate_weights(const moe_config* c, const moe_weights* w) {
    if (!w) return MOE_ERR_INVALID_ARGUMENT;
    auto need = [](const void* p) { return p != nullptr; };
    if (!need(w->router_w)) return MOE_ERR_MISSING_TENSOR;
    if (c->has_router_bias && !need(w->router_b)) return MOE_ERR_MISSING_TENSOR;
    if (c->has_selection_bias && !need(w->selection_bias)) return MOE_ERR_MISSING_TENSOR;
    if (c->shared_mode == MOE_SHARED_BLEND && (!need(w->coef_w) || !need(w->coef_b))) return MOE_ERR_MISSING_TENSOR;
    if (c->gate_up_interleaved) {
        if (!need(w->gate_up_w)) return MOE_ERR_MISSING_TENSOR;
        if (c->has_expert_bias && !need(w->gate_up_b)) return MOE_ERR_MISSING_TENSOR;
    } else {
        if (!need(w->gate_w) || !need(w->up_w)) return MOE_ERR_MISSING_TENSOR;
        if (c->has_expert_bias && (!need(w->gate_b) || !need(w->up_b))) return MOE_ERR_MISSING_TENSOR;
    }
    if (!need(w->down_w)) return MOE_ERR_MISSING_TENSOR;
    if (c->has_expert_bias && !need(w->down_b)) return MOE_ERR_MISSING_TENSOR;
    // 4-bit companions: scales (and Q4 biases) of each routed plane; an interleaved gate_up
    // plane carries its own (gate_up_s / gate_up_z, libmir-metal ExpertLayout::Native)
    const bool il = c->gate_up_interleaved;
    if (c->weight_format == MOE_DTYPE_Q4_AFFINE) {
        const void* q[] = {il ? w->gate_up_s : w->gate_s, il ? w->gate_up_z : w->gate_z,
                           il ? w->gate_up_s : w->up_s, il ? w->gate_up_z : w->up_z, w->down_s, w->down_z};
        for (const void* p : q)
            if (!need(p)) return MOE_ERR_MISSING_TENSOR;
    }
    if (c->weight_format == MOE_DTYPE_MXFP4 &&
        (!need(il ? w->gate_up_s : w->gate_s) || !need(il ? w->gate_up_s : w->up_s) || !need(w->down_s)))
        return MOE_ERR_MISSING_TENSOR;
    if (c->shared_mode != MOE_SHARED_NONE &&
        (!need(w->shared_gate_w) || !need(w->shared_up_w) || !need(w->shared_down_w)))
        return MOE_ERR_MISSING_TENSOR;
    if (c->latent_dim && (!need(w->latent_down_w) || !need(w->latent_up_w))) return MOE_ERR_MISSING_TENSOR;
    if (c->latent_use_norm && !need(w->latent_norm_w)) return MOE_ERR_MISSING_TENSOR;
    if (c->dense_format == MOE_DTYPE_Q4_AFFINE) {
        if (!need(w->router_s) || !need(w->router_z)) return MOE_ERR_MISSING_TENSOR;
        if (c->shared_mode != MOE_SHARED_NONE &&
            (!need(w->shared_gate_s) || !need(w->shared_gate_z) || !need(w->shared_up_s) || !need(w->shared_up_z) ||
             !need(w->shared_down_s) || !need(w->shared_down_z)))
            return MOE_ERR_MISSING_TENSOR;
        if (c->latent_dim &&
            (!need(w->latent_down_s) || !need(w->latent_down_z) || !need(w->latent_up_s) || !need(w->latent_up_z)))
            return MOE_ERR_MISSING_TENSOR;
    }
    const void* all[] = {w->router_w, w->router_b, w->selection_bias, w->coef_w, w->coef_b,
                         w->gate_w, w->up_w, w->gate_up_w, w->gate_b, w->up_b, w->gate_up_b,
                         w->down_w, w->down_b, w->gate_s, w->gate_z, w->up_s, w->up_z,
                         w->down_s, w->down_z, w->shared_gate_w, w->shared_up_w, w->shared_down_w,
                         w->latent_down_w, w->latent_up_w, w->latent_norm_w, w->gate_up_s, w->gate_up_z,
                         w->router_s, w->router_z, w->shared_gate_s, w->shared_gate_z, w->shared_up_s,
                         w->shared_up_z, w->shared_down_s, w->shared_down_z, w->latent_down_s, w->latent_down_z,
                         w->latent_up_s, w->latent_up_z};
    for (const void* p : all)
        if (p && !aligned16(p)) return MOE_ERR_INVALID_ARGUMENT;
    return MOE_OK;
}

moe_status check_tokens(const moe_config* c, int64_t T) {
    if (T < 0) return MOE_ERR_INVALID_ARGUMENT;
    const int64_t Kmax = std::max(std::max<int64_t>(c->hidden, c->intermediate), std::max<int64_t>(expert_in(*c), c->shared_intermediate));
    if (T > (int64_t(1) << 26) || T * c->top_k >= (int64_t(1) << 31) || T * c->top_k * Kmax >= (int64_t(1) << 46))
        return MOE_ERR_SHAPE_OVERFLOW;
    return MOE_OK;
}

moe_status check_ptr(const void* p) {
    if (!p) return MOE_ERR_INVALID_ARGUMENT;
    return aligned16(p) ? MOE_OK : MOE_ERR_INVALID_ARGUMENT;
}

// Which engine runs a GEMM: weight-streaming CUDA-core kernels (few tokens per
// weight row) or the tcgen05 tensor-core kernel (many). MOE_PATH=gemv|tc forces one
// where both are possible (used by the tests to cross-check the two).
enum { kPathAuto = 0, kPathGemv = 1, kPathTc = 2, kPathDecode = 3 };
int path_override() {
    const char* e = getenv("MOE_PATH");
    if (!e) return kPathAuto;
    if (!strcmp(e, "gemv")) return kPathGemv;
    if (!strcmp(e, "tc")) return kPathTc;
    if (!strcmp(e, "decode")) return kPathDecode;
    return kPathAuto;
}
bool dense_tc(const moe_config* c, int64_t T, int K) {
    if (c->act_dtype != MOE_DTYPE_BF16 || K % 64 != 0) return false;
    const int o = path_override();
    return o == kPathTc || (o == kPathAuto && T >= 64);
}
// The routed experts go to the tensor cores once there are about E/4 slots: measured on
// B200, the TMA-fed tcgen05 kernel streams the activated weights faster than the CUDA-core
// kernels from there on, although most tiles then hold only a few tokens (Klear shape:
// 8 tokens 149 vs 157 us, 64 tokens 279 vs 627 us; at 4 tokens the CUDA cores win).
bool routed_tc(const moe_config* c, int64_t T) {
    if (c->act_dtype != MOE_DTYPE_BF16 || c->weight_format == MOE_DTYPE_F32) return false;
    if (expert_in(*c) % 64 != 0 || c->intermediate % 64 != 0) return false;
    const int o = path_override();
    return o == kPathTc || (o == kPathAuto && 4 * T * c->top_k >= int64_t(c->num_experts));
}

// The whole block as one persistent launch (csrc/decode.cu) for up to 8 tokens without a
// latent projection, bf16 activations and bf16 / 4-bit routed planes; MOE_PATH=gemv or tc
// selects the multi-kernel engines instead.
DecodeArgs decode_args(const moe_config* c, const moe_weights* w, const void* x, int64_t T, void* y, void* ws,
                       const WsLayout& L) {
    DecodeArgs d;
    d.T = int(T); d.H = c->hidden; d.E = c->num_experts; d.k = c->top_k; d.I = c->intermediate;
    d.Is = c->shared_intermediate;
    d.wf = c->weight_format; d.interleaved = c->gate_up_interleaved; d.has_bias = c->has_expert_bias;
    d.group_size = c->group_size;
    d.act = c->activation; d.limit = c->swiglu_limit; d.alpha = c->swiglu_alpha;
    d.scoring = c->scoring; d.norm = c->norm_topk_prob; d.has_sel = c->has_selection_bias;
    d.shared_mode = c->shared_mode;
    d.router_w = w->router_w; d.router_b = c->has_router_bias ? w->router_b : nullptr;
    if (c->shared_mode == MOE_SHARED_BLEND) { d.coef_w = w->coef_w; d.coef_b = w->coef_b; }
    d.sel_bias = static_cast<const float*>(w->selection_bias);
    d.gate_w = w->gate_w; d.up_w = w->up_w; d.gate_up_w = w->gate_up_w;
    d.gate_s = c->gate_up_interleaved ? w->gate_up_s : w->gate_s;
    d.gate_z = c->gate_up_interleaved ? w->gate_up_z : w->gate_z;
    d.up_s = w->up_s; d.up_z = w->up_z;
    d.gate_b = w->gate_b; d.up_b = w->up_b; d.gate_up_b = w->gate_up_b;
    d.down_w = w->down_w; d.down_s = w->down_s; d.down_z = w->down_z; d.down_b = w->down_b;
    if (c->shared_mode != MOE_SHARED_NONE) { d.sg_w = w->shared_gate_w; d.su_w = w->shared_up_w; d.sd_w = w->shared_down_w; }
    if (dense_q4(c)) {
        d.dense_q4 = 1;
        d.dense_group = c->dense_group_size;
        d.router_s = w->router_s; d.router_z = w->router_z;
        d.sg_s = w->shared_gate_s; d.sg_z = w->shared_gate_z; d.su_s = w->shared_up_s; d.su_z = w->shared_up_z;
        d.sd_s = w->shared_down_s; d.sd_z = w->shared_down_z;
    }
    d.x = x; d.y = y;
    d.logits = reinterpret_cast<float*>(static_cast<char*>(ws) + L.logits); d.ld_logits = L.ld_logits;
    d.h = static_cast<char*>(ws) + L.h;
    d.hs = static_cast<char*>(ws) + L.hs;
    d.status = reinterpret_cast<int*>(static_cast<char*>(ws) + L.status);
    d.bar = reinterpret_cast<unsigned*>(static_cast<char*>(ws) + L.status + kDecodeBarOffset);
    return d;
}

// Chosen where it measured faster than both other engines on B200 (graph replay, L2
// flushed): a single token (Klear bf16 47 vs 62 / 72 us, clamped MXFP4 62 vs 88 / 133 us),
// and two tokens with bf16 weights (Klear 74 vs 86 / 82 us). From there on the tensor-core
// kernel streams the weights faster (Klear 4 tokens: 115 vs 111 us; 8 tokens: 176 vs 129 us;
// clamped MXFP4 8 tokens: 432 vs 361 us).
bool use_decode(const moe_config* c, int64_t T, const DecodeArgs& d) {
    if (c->latent_dim || c->act_dtype != MOE_DTYPE_BF16 || c->weight_format == MOE_DTYPE_F32) return false;
    const int o = path_override();
    if (o == kPathGemv || o == kPathTc) return false;
    if (T < 1 || T > 8 || decode_smem_bytes(d) == 0) return false;
    return o == kPathDecode || T == 1 || (T == 2 && c->weight_format == MOE_DTYPE_BF16);
}

#define MOE_CHECK(expr)                          \
    do {                                         \
        const moe_status _s = (expr);            \
        if (_s != MOE_OK) return _s;             \
    } while (0)
#define MOE_CUDA(expr)                                  \
    do {                                                \
        if ((expr) != cudaSuccess) return MOE_ERR_CUDA; \
    } while (0)

// Common preamble of every computing call: config, weights, tokens, workspace.
moe_status prelude(const moe_config* c, const moe_weights* w, int64_t T, void* ws, size_t ws_bytes,
                   WsLayout* L) {
    MOE_CHECK(validate_config(c));
    if (w) MOE_CHECK(validate_weights(c, w));
    MOE_CHECK(check_tokens(c, T));
    if (T == 0) return MOE_OK;
    MOE_CHECK(check_ptr(ws));
    *L = ws_layout(*c, T);
    if (ws_bytes < L->total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    return MOE_OK;
}

template <typename P> P* at(void* ws, size_t off) { return reinterpret_cast<P*>(static_cast<char*>(ws) + off); }

// a1 + a2
// The router's dense GEMV: E router rows (+ 2 coefficient rows for the blend) -> fp32 logits.
DenseGemvArgs router_args(const moe_config* c, const moe_weights* w, const void* x, int64_t T, void* ws,
                          const WsLayout& L) {
    const bool blend = c->shared_mode == MOE_SHARED_BLEND;
    DenseGemvArgs r;
    r.W0 = w->router_w;
    r.b0 = c->has_router_bias ? w->router_b : nullptr;
    r.rows0 = c->num_experts;
    if (blend) {
        r.W1 = w->coef_w;
        r.b1 = w->coef_b;
        r.rows1 = 2;
    }
    r.u = x;
    r.T = T;
    r.K = c->hidden;
    r.out = at<float>(ws, L.logits);
    r.ld_out = L.ld_logits;
    r.out_f32 = 1;
    r.act_dtype = c->act_dtype;
    if (dense_q4(c)) {
        r.s0 = w->router_s;
        r.z0 = w->router_z;
        r.group0 = c->dense_group_size;
    }
    return r;
}

TopkArgs topk_args(const moe_config* c, const moe_weights* w, int64_t T, int32_t* idx, float* wts, float* coef,
                   void* ws, const WsLayout& L) {
    TopkArgs t;
    t.logits = at<float>(ws, L.logits);
    t.ld = L.ld_logits;
    t.T = T;
    t.E = c->num_experts;
    t.k = c->top_k;
    t.scoring = c->scoring;
    t.norm = c->norm_topk_prob;
    t.has_sel = c->has_selection_bias;
    t.sel_bias = static_cast<const float*>(w->selection_bias);
    t.blend = c->shared_mode == MOE_SHARED_BLEND;
    t.idx = idx;
    t.w = wts;
    t.coef = coef;
    return t;
}

// Where the top-k warp writes the permutation of a single token (moe_block_forward, T == 1).
struct PermOut {
    int32_t *offsets = nullptr, *sorted_slot = nullptr, *slot_pos = nullptr, *active = nullptr, *tiles = nullptr;
};

moe_status run_route(const moe_config* c, const moe_weights* w, const void* x, int64_t T, int32_t* idx,
                     float* wts, float* coef, float* zero, int64_t zero_cols, void* ws, const WsLayout& L,
                     cudaStream_t s, const PermOut* perm = nullptr) {
    const bool blend = c->shared_mode == MOE_SHARED_BLEND;
    const DenseGemvArgs r = router_args(c, w, x, T, ws, L);
    // a 4-bit router stays on the weight-streaming kernel at every size: it dequantises exactly
    // in fp32 (s * sum q x + b * sum x), while the tensor cores would round each weight, and
    // the selection keys decide integer expert choices
    if (dense_tc(c, T, c->hidden) && !dense_q4(c)) {
        TcParams P;
        const int np = blend ? 2 : 1;
        for (int i = 0; i < np; ++i) {
            TcProblem& p = P.p[i];
            p.mode = kEpiStoreF32;
            p.M = i == 0 ? c->num_experts : 2;
            p.K = c->hidden;
            p.m_blocks = (p.M + kTcRows - 1) / kTcRows;
            p.rows = int(T);
            p.bn = dense_bn(c, T, c->num_experts);  // both problems: one tile height
            p.n_tiles = int((T + p.bn - 1) / p.bn);
            p.bias0 = i == 0 ? r.b0 : r.b1;
            p.out = at<float>(ws, L.logits) + (i == 0 ? 0 : c->num_experts);
            p.ld_out = L.ld_logits;
            const bool wok = i == 0 ? tc_dense_weights(c, p, &P.a0[i], nullptr, r.W0, w->router_s, w->router_z, nullptr,
                                                       nullptr, nullptr, p.M, c->hidden)
                                    : tc_weight_map(&P.a0[i], r.W1, 1, p.M, c->hidden, false);  // blend head: act dtype
            if (!wok || !tc_token_map(P.b[i], x, T, c->hidden, p.bn)) return MOE_ERR_CUDA;
        }
        P.nprob = np;
        P.status = at<int>(ws, L.status);
        const int64_t tiles = int64_t(P.p[0].m_blocks) * P.p[0].n_tiles + (np > 1 ? P.p[1].n_tiles : 0);
        MOE_CUDA(launch_tc_gemm(P, false, tiles, s));
    } else {
        MOE_CUDA(launch_dense_gemv(r, s));
    }
    TopkArgs t = topk_args(c, w, T, idx, wts, coef, ws, L);
    t.zero = zero;
    t.zero_cols = zero_cols;
    if (perm && T == 1) {
        t.p_offsets = perm->offsets;
        t.p_sorted = perm->sorted_slot;
        t.p_slot_pos = perm->slot_pos;
        t.p_active = perm->active;
        t.p_tiles = perm->tiles;
    }
    MOE_CUDA(launch_topk(t, s));
    return MOE_OK;
}

// a3
moe_status run_permute(const moe_config* c, const int32_t* idx, int64_t T, int32_t* offsets,
                       int32_t* sorted_slot, int32_t* slot_pos, void* ws, const WsLayout& L, cudaStream_t s,
                       bool tc_tiles) {
    PermuteArgs p;
    p.idx = idx;
    p.S = T * c->top_k;
    p.E = c->num_experts;
    p.offsets = offsets;
    p.sorted_slot = sorted_slot;
    p.slot_pos = slot_pos;
    p.active = at<int32_t>(ws, L.active);
    p.chunk_hist = at<int32_t>(ws, L.chunk_hist);
    p.chunk = kPermChunkWs;
    p.n_chunks = L.n_chunks;
    p.status = at<int>(ws, L.status);
    if (tc_tiles) {
        p.tile_bn = expert_bn(c, T);
        p.tile_start = at<int32_t>(ws, L.tiles);
    }
    MOE_CUDA(launch_permute(p, s));
    return MOE_OK;
}

// The routed experts a call runs: [e0, e0 + ne). The routed planes of moe_weights hold
// exactly these experts (plane g = expert e0 + g); offsets / sorted_slot stay the full
// permutation's, and only the slots of these experts are read.
struct ExpertRange {
    int e0 = 0, ne = 0;
};

// Tensor-core part of a4 + a5 (+ a6): the routed groups (rtc) and/or the shared expert (stc).
// The routed down GEMM's epilogue multiplies each slot's output row by its routing weight
// and adds it into the token's fp32 routed sum y_acc, which must be zero on entry.
moe_status run_experts_tc(const moe_config* c, const moe_weights* w, const void* u, const void* x, int64_t T,
                          const int32_t* offsets, const int32_t* sorted_slot, const float* topk_w,
                          float* y_acc, bool rtc, bool stc, ExpertRange rg, void* ws, const WsLayout& L,
                          cudaStream_t s) {
    const int K = expert_in(*c), I = c->intermediate, E = rg.ne, k = c->top_k, H = c->hidden;
    const int32_t* goff = offsets ? offsets + rg.e0 : nullptr;  // the range's offsets [ne + 1]
    // 4-bit affine problems run on fp16 operands: fp16 copies of their token inputs
    const bool aff = rtc && c->weight_format == MOE_DTYPE_Q4_AFFINE, dq = stc && dense_q4(c);
    void* x16 = at<void>(ws, L.x16);
    const int Is = c->shared_intermediate;
    const int64_t S = T * k;
    const int BN = expert_bn(c, T);
    const int64_t n_dense = (T + BN - 1) / BN;
    void* uperm = at<void>(ws, L.uperm);
    // the routed token rows in sorted order (fp16 for 4-bit affine weights)
    if (rtc) MOE_CUDA(launch_gather_rows(u, K, sorted_slot, k, S, uperm, s, goff, goff + E, aff));
    if (dq) MOE_CUDA(launch_to_f16(x, T * H, x16, s));
    void* h = at<void>(ws, L.h);
    void* hs = at<void>(ws, L.hs);
    const int32_t* tiles = at<int32_t>(ws, L.tiles);
    {  // gate/up + activation
        TcParams P;
        int np = 0;
        int64_t max_tiles = 0;
        if (stc) {
            TcProblem& p = P.p[np];
            p.mode = kEpiGateUp;
            p.M = Is; p.K = H; p.m_blocks = (Is + kTcRowsGateUp - 1) / kTcRowsGateUp;
            p.rows = int(T); p.n_tiles = int(n_dense); p.bn = BN;
            p.out = hs; p.ld_out = Is;
            p.out_f16 = dq ? 1 : 0;  // fp16 hs for the fp16 shared down GEMM
            if (!tc_dense_weights(c, p, &P.a0[np], &P.a1[np], w->shared_gate_w, w->shared_gate_s, w->shared_gate_z,
                                  w->shared_up_w, w->shared_up_s, w->shared_up_z, Is, H) ||
                !tc_token_map(P.b[np], dq ? x16 : x, T, H, BN))
                return MOE_ERR_CUDA;
            max_tiles += int64_t(p.m_blocks) * p.n_tiles;
            ++np;
        }
        if (rtc) {
            TcProblem& p = P.p[np];
            p.mode = kEpiGateUp;
            p.M = I; p.K = K; p.m_blocks = (I + kTcRowsGateUp - 1) / kTcRowsGateUp;
            p.grouped = 1; p.num_groups = E; p.offsets = goff; p.tile_start = tiles; p.bn = BN;
            p.out = h; p.ld_out = I;
            p.interleaved = c->gate_up_interleaved;  // bf16 / f32 planes: one 4-D map
            if (c->has_expert_bias) {
                if (c->gate_up_interleaved) {
                    p.bias0 = w->gate_up_b;
                    p.bias_interleaved = 1;
                } else {
                    p.bias0 = w->gate_b;
                    p.bias1 = w->up_b;
                }
            }
            bool ok;
            if (c->weight_format == MOE_DTYPE_Q4_AFFINE || c->weight_format == MOE_DTYPE_MXFP4) {
                // packed 4-bit codes, dequantised in the main loop
                p.q4 = 1;
                p.mx = c->weight_format == MOE_DTYPE_MXFP4;
                p.group_size = c->group_size;
                if (c->gate_up_interleaved) {
                    // one [E, 2I, K] plane: gate rows 2i and up rows 2i + 1 through two maps
                    // that step over every other row; the companions interleave the same way
                    const int64_t ng = K / c->group_size;
                    const int64_t sb = p.mx ? 1 : 2;  // bytes per scale
                    p.interleaved = 0;
                    p.qrow_step = 2;
                    p.qs0 = w->gate_up_s;
                    p.qs1 = static_cast<const char*>(w->gate_up_s) + ng * sb;
                    p.qz0 = p.mx ? nullptr : w->gate_up_z;
                    p.qz1 = p.mx ? nullptr : static_cast<const char*>(w->gate_up_z) + ng * 2;
                    const char* gu = static_cast<const char*>(w->gate_up_w);
                    ok = tc_q4_weight_map(&P.a0[np], gu, E, I, K, 2) &&
                         tc_q4_weight_map(&P.a1[np], gu + int64_t(K) / 2, E, I, K, 2);
                } else {
                    p.qs0 = w->gate_s; p.qz0 = w->gate_z; p.qs1 = w->up_s; p.qz1 = w->up_z;
                    ok = tc_q4_weight_map(&P.a0[np], w->gate_w, E, I, K) &&
                         tc_q4_weight_map(&P.a1[np], w->up_w, E, I, K);
                }
            } else if (c->gate_up_interleaved) {
                ok = tc_weight_map(&P.a0[np], w->gate_up_w, E, I, K, true);
            } else {
                ok = tc_weight_map(&P.a0[np], w->gate_w, E, I, K, false) &&
                     tc_weight_map(&P.a1[np], w->up_w, E, I, K, false);
            }
            p.out_f16 = aff ? 1 : 0;  // fp16 h for the fp16 routed down GEMM
            if (!ok || !tc_token_map(P.b[np], uperm, S, K, BN)) return MOE_ERR_CUDA;
            max_tiles += int64_t(p.m_blocks) * max_routed_tiles(*c, T);
            ++np;
        }
        P.nprob = np;
        P.status = at<int>(ws, L.status);
        P.act = c->activation;
        P.limit = c->swiglu_limit;
        P.alpha = c->swiglu_alpha;
        MOE_CUDA(launch_tc_gemm(P, true, max_tiles, s));
    }
    {  // down (+ weighted scatter into the routed sum)
        TcParams P;
        int np = 0;
        int64_t max_tiles = 0;
        if (stc) {
            TcProblem& p = P.p[np];
            p.mode = kEpiStoreF32;
            p.M = H; p.K = Is; p.m_blocks = (H + kTcRows - 1) / kTcRows;
            p.rows = int(T); p.n_tiles = int(n_dense); p.bn = BN;
            p.out = at<float>(ws, L.s_acc); p.ld_out = H;
            if (!tc_dense_weights(c, p, &P.a0[np], nullptr, w->shared_down_w, w->shared_down_s, w->shared_down_z,
                                  nullptr, nullptr, nullptr, H, Is) ||
                !tc_token_map(P.b[np], hs, T, Is, BN))
                return MOE_ERR_CUDA;
            max_tiles += int64_t(p.m_blocks) * p.n_tiles;
            ++np;
        }
        if (rtc) {
            TcProblem& p = P.p[np];
            p.mode = kEpiScatterAdd;
            p.M = K; p.K = I; p.m_blocks = (K + kTcRows - 1) / kTcRows;
            p.grouped = 1; p.num_groups = E; p.offsets = goff; p.tile_start = tiles; p.bn = BN;
            p.sorted_slot = sorted_slot; p.topk_w = topk_w; p.k = k;
            p.bias0 = c->has_expert_bias ? w->down_b : nullptr;
            p.out = y_acc; p.ld_out = K;
            bool ok;
            if (c->weight_format == MOE_DTYPE_Q4_AFFINE || c->weight_format == MOE_DTYPE_MXFP4) {
                p.q4 = 1;
                p.mx = c->weight_format == MOE_DTYPE_MXFP4;
                p.group_size = c->group_size;
                p.qs0 = w->down_s; p.qz0 = w->down_z;
                ok = tc_q4_weight_map(&P.a0[np], w->down_w, E, K, I);
            } else {
                ok = tc_weight_map(&P.a0[np], w->down_w, E, K, I, false);
            }
            if (!ok || !tc_token_map(P.b[np], h, S, I, BN)) return MOE_ERR_CUDA;
            max_tiles += int64_t(p.m_blocks) * max_routed_tiles(*c, T);
            ++np;
        }
        P.nprob = np;
        P.status = at<int>(ws, L.status);
        MOE_CUDA(launch_tc_gemm(P, false, max_tiles, s));
    }
    return MOE_OK;
}

// Where the routed sum lives after run_experts: token t's sum is the sum of rows
// [t*nsum, (t+1)*nsum) of `rows` (width K).
struct RoutedSum {
    const void* rows = nullptr;
    int nsum = 1;
    int dtype = MOE_DTYPE_F32;
};

// a4 + a5 (+ a6 when with_shared). y_acc must be zero on entry: both engines add each
// slot's weighted output into its token's row.
moe_status run_experts(const moe_config* c, const moe_weights* w, const void* u, const void* x, int64_t T,
                       const int32_t* offsets, const int32_t* sorted_slot, const float* topk_w,
                       float* y_acc, bool with_routed, bool with_shared, void* ws, const WsLayout& L,
                       cudaStream_t s, RoutedSum* sum, ExpertRange rg = ExpertRange{}) {
    if (rg.ne == 0) rg.ne = c->num_experts;
    const int K = expert_in(*c);
    const bool sh = with_shared && c->shared_mode != MOE_SHARED_NONE;
    const bool rtc = with_routed && routed_tc(c, T);
    // the shared expert joins the routed tensor-core launches whenever those run
    const bool stc = sh && c->shared_intermediate % 64 == 0 && c->hidden % 64 == 0 &&
                     c->act_dtype == MOE_DTYPE_BF16 && (dense_tc(c, T, c->hidden) || rtc);
    if (sum) {
        sum->rows = y_acc;
        sum->nsum = 1;
        sum->dtype = MOE_DTYPE_F32;
    }
    if (rtc || stc)
        MOE_CHECK(run_experts_tc(c, w, u, x, T, offsets, sorted_slot, topk_w, y_acc, rtc, stc, rg, ws, L, s));
    const int64_t groups = (with_routed && !rtc) ? std::min<int64_t>(rg.ne, T * c->top_k) : 0;
    if (groups == 0 && (!sh || stc)) return MOE_OK;
    GateUpArgs g;
    g.wf = c->weight_format;
    g.interleaved = c->gate_up_interleaved;
    g.has_bias = c->has_expert_bias;
    g.group_size = c->group_size;
    g.gate_w = w->gate_w; g.up_w = w->up_w; g.gate_up_w = w->gate_up_w;
    g.gate_s = c->gate_up_interleaved ? w->gate_up_s : w->gate_s;
    g.gate_z = c->gate_up_interleaved ? w->gate_up_z : w->gate_z;
    g.up_s = w->up_s; g.up_z = w->up_z;
    g.gate_b = w->gate_b; g.up_b = w->up_b; g.gate_up_b = w->gate_up_b;
    g.offsets = offsets ? offsets + rg.e0 : nullptr;
    g.sorted_slot = sorted_slot;
    g.active = at<int32_t>(ws, L.active);
    g.k = c->top_k;
    g.I = c->intermediate;
    g.K = K;
    g.routed_groups = int(groups);
    g.u = u;
    g.h = at<void>(ws, L.h);
    if (sh && !stc) {
        g.sg_w = w->shared_gate_w;
        g.su_w = w->shared_up_w;
        g.shared_I = c->shared_intermediate;
        g.Hs = c->hidden;
        g.xs = x;
        g.hs = at<void>(ws, L.hs);
        if (dense_q4(c)) {
            g.sg_s = w->shared_gate_s; g.sg_z = w->shared_gate_z;
            g.su_s = w->shared_up_s; g.su_z = w->shared_up_z;
            g.s_group = c->dense_group_size;
        }
    }
    g.T = T;
    g.act = c->activation;
    g.limit = c->swiglu_limit;
    g.alpha = c->swiglu_alpha;
    MOE_CUDA(launch_gateup_gemv(g, s));
    DownArgs d;
    d.wf = c->weight_format;
    d.has_bias = c->has_expert_bias;
    d.group_size = c->group_size;
    d.down_w = w->down_w; d.down_s = w->down_s; d.down_z = w->down_z; d.down_b = w->down_b;
    d.offsets = offsets ? offsets + rg.e0 : nullptr;
    d.sorted_slot = sorted_slot;
    d.active = at<int32_t>(ws, L.active);
    d.topk_w = topk_w;
    d.k = c->top_k;
    d.I = c->intermediate;
    d.K = K;
    d.routed_groups = int(groups);
    d.h = at<void>(ws, L.h);
    d.y_acc = y_acc;
    if (sh && !stc) {
        d.sd_w = w->shared_down_w;
        d.shared_I = c->shared_intermediate;
        d.Hs = c->hidden;
        d.hs = at<void>(ws, L.hs);
        d.s_acc = at<float>(ws, L.s_acc);
        if (dense_q4(c)) {
            d.sd_s = w->shared_down_s; d.sd_z = w->shared_down_z;
            d.s_group = c->dense_group_size;
        }
    }
    d.T = T;
    MOE_CUDA(launch_down_gemv(d, s));
    return MOE_OK;
}

// a8 (first half): z = x Wdp^T
moe_status run_latent_down(const moe_config* c, const moe_weights* w, const void* x, int64_t T, void* z,
                           void* ws, const WsLayout& L, cudaStream_t s) {
    int* status = at<int>(ws, L.status);
    DenseGemvArgs r;
    r.W0 = w->latent_down_w;
    r.rows0 = c->latent_dim;
    r.u = x;
    r.T = T;
    r.K = c->hidden;
    r.out = z;
    r.ld_out = c->latent_dim;
    r.out_f32 = 0;
    r.act_dtype = c->act_dtype;
    if (dense_q4(c)) {
        r.s0 = w->latent_down_s;
        r.z0 = w->latent_down_z;
        r.group0 = c->dense_group_size;
    }
    if (dense_tc(c, T, c->hidden) && c->latent_dim % 64 == 0) {
        TcParams P;
        TcProblem& p = P.p[0];
        p.mode = kEpiStoreAct;
        p.M = c->latent_dim; p.K = c->hidden; p.m_blocks = (p.M + kTcRows - 1) / kTcRows;
        p.bn = dense_bn(c, T, p.M);
        p.rows = int(T); p.n_tiles = int((T + p.bn - 1) / p.bn);
        p.out = z; p.ld_out = c->latent_dim;
        const void* xt = x;
        if (dense_q4(c)) {  // fp16 operands
            xt = static_cast<char*>(ws) + L.x16;
            MOE_CUDA(launch_to_f16(x, T * c->hidden, const_cast<void*>(xt), s));
        }
        if (!tc_dense_weights(c, p, &P.a0[0], nullptr, w->latent_down_w, w->latent_down_s, w->latent_down_z, nullptr,
                              nullptr, nullptr, p.M, p.K) ||
            !tc_token_map(P.b[0], xt, T, p.K, p.bn))
            return MOE_ERR_CUDA;
        P.nprob = 1;
        P.status = status;
        MOE_CUDA(launch_tc_gemm(P, false, int64_t(p.m_blocks) * p.n_tiles, s));
        return MOE_OK;
    }
    MOE_CUDA(launch_dense_gemv(r, s));
    return MOE_OK;
}

// a7 (and the tail of a8): s_acc already holds the shared expert when shared_mode != NONE.
moe_status run_output(const moe_config* c, const moe_weights* w, RoutedSum rs, const float* coef,
                      int64_t T, void* y, void* ws, const WsLayout& L, cudaStream_t s) {
    const float* s_acc = c->shared_mode != MOE_SHARED_NONE ? at<float>(ws, L.s_acc) : nullptr;
    if (!c->latent_dim) {
        MOE_CUDA(launch_combine(rs.rows, rs.dtype, rs.nsum, s_acc, coef, c->shared_mode, T, c->hidden, y, c->act_dtype, s));
        return MOE_OK;
    }
    const void* n = nullptr;
    if (c->latent_use_norm) {
        MOE_CUDA(launch_rmsnorm(rs.rows, rs.dtype, rs.nsum, w->latent_norm_w, c->rms_eps, T, c->latent_dim,
                                at<void>(ws, L.nrm), c->act_dtype, s));
    } else {
        // no norm: the routed latent sum rounded to the activation dtype
        MOE_CUDA(launch_combine(rs.rows, rs.dtype, rs.nsum, nullptr, nullptr, MOE_SHARED_NONE, T, c->latent_dim,
                                at<void>(ws, L.nrm), c->act_dtype, s));
    }
    n = at<void>(ws, L.nrm);
    if (c->shared_mode == MOE_SHARED_BLEND) return MOE_ERR_UNSUPPORTED;  // rejected earlier
    DenseGemvArgs r;
    r.W0 = w->latent_up_w;
    r.rows0 = c->hidden;
    r.u = n;
    r.T = T;
    r.K = c->latent_dim;
    r.out = y;
    r.ld_out = c->hidden;
    r.out_f32 = c->act_dtype == MOE_DTYPE_F32;
    r.addend = s_acc;
    r.ld_add = c->hidden;
    r.act_dtype = c->act_dtype;
    if (dense_q4(c)) {
        r.s0 = w->latent_up_s;
        r.z0 = w->latent_up_z;
        r.group0 = c->dense_group_size;
    }
    if (dense_tc(c, T, c->latent_dim) && c->hidden % 64 == 0) {
        TcParams P;
        TcProblem& p = P.p[0];
        p.mode = kEpiStoreAct;
        p.M = c->hidden; p.K = c->latent_dim; p.m_blocks = (p.M + kTcRows - 1) / kTcRows;
        p.bn = dense_bn(c, T, p.M);
        p.rows = int(T); p.n_tiles = int((T + p.bn - 1) / p.bn);
        p.out = y; p.ld_out = c->hidden;
        p.addend = s_acc; p.ld_add = c->hidden;
        const void* nt = n;
        if (dense_q4(c)) {  // fp16 operands
            nt = at<void>(ws, L.n16);
            MOE_CUDA(launch_to_f16(n, T * c->latent_dim, const_cast<void*>(nt), s));
        }
        if (!tc_dense_weights(c, p, &P.a0[0], nullptr, w->latent_up_w, w->latent_up_s, w->latent_up_z, nullptr,
                              nullptr, nullptr, p.M, p.K) ||
            !tc_token_map(P.b[0], nt, T, p.K, p.bn))
            return MOE_ERR_CUDA;
        P.nprob = 1;
        P.status = at<int>(ws, L.status);
        MOE_CUDA(launch_tc_gemm(P, false, int64_t(p.m_blocks) * p.n_tiles, s));
        return MOE_OK;
    }
    MOE_CUDA(launch_dense_gemv(r, s));
    return MOE_OK;
}

}  // namespace

extern "C" {

moe_status moe_config_validate(const moe_config* cfg) {
    MOE_CHECK(validate_config(cfg));
    if (cfg->latent_dim && cfg->shared_mode == MOE_SHARED_BLEND) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

moe_status moe_weights_validate(const moe_config* cfg, const moe_weights* w) {
    MOE_CHECK(moe_config_validate(cfg));
    return validate_weights(cfg, w);
}

moe_status moe_workspace_size(const moe_config* cfg, int64_t max_tokens, size_t* bytes) {
    MOE_CHECK(moe_config_validate(cfg));
    if (!bytes) return MOE_ERR_INVALID_ARGUMENT;
    MOE_CHECK(check_tokens(cfg, max_tokens));
    *bytes = ws_layout(*cfg, max_tokens).total;
    return MOE_OK;
}

moe_status moe_route(const moe_config* cfg, const moe_weights* w, const void* x, int64_t T, int32_t* topk_idx,
                     float* topk_w, float* coef, void* ws, size_t ws_bytes, moe_stream_t stream) {
    MOE_CHECK(moe_config_validate(cfg));
    WsLayout L;
    MOE_CHECK(prelude(cfg, w, T, ws, ws_bytes, &L));
    if (T == 0) return MOE_OK;
    MOE_CHECK(check_ptr(x));
    MOE_CHECK(check_ptr(topk_idx));
    MOE_CHECK(check_ptr(topk_w));
    if (cfg->shared_mode == MOE_SHARED_BLEND) MOE_CHECK(check_ptr(coef));
    return run_route(cfg, w, x, T, topk_idx, topk_w, coef, nullptr, 0, ws, L, (cudaStream_t)stream);
}

moe_status moe_permute(const moe_config* cfg, const int32_t* topk_idx, int64_t T, int32_t* expert_offsets,
                       int32_t* sorted_slot, int32_t* slot_pos, void* ws, size_t ws_bytes, moe_stream_t stream) {
    MOE_CHECK(moe_config_validate(cfg));
    WsLayout L;
    MOE_CHECK(prelude(cfg, nullptr, T, ws, ws_bytes, &L));
    if (T == 0) return MOE_OK;
    MOE_CHECK(check_ptr(topk_idx));
    MOE_CHECK(check_ptr(expert_offsets));
    MOE_CHECK(check_ptr(sorted_slot));
    MOE_CHECK(check_ptr(slot_pos));
    return run_permute(cfg, topk_idx, T, expert_offsets, sorted_slot, slot_pos, ws, L, (cudaStream_t)stream,
                       false);
}

}  // extern "C"

namespace {
moe_status grouped_ffn_range(const moe_config* cfg, const moe_weights* w, const void* u, int64_t T,
                             const int32_t* expert_offsets, const int32_t* sorted_slot, const float* topk_w,
                             ExpertRange rg, float* y_acc, void* ws, size_t ws_bytes, moe_stream_t stream) {
    MOE_CHECK(moe_config_validate(cfg));
    WsLayout L;
    MOE_CHECK(prelude(cfg, w, T, ws, ws_bytes, &L));
    if (T == 0) return MOE_OK;
    MOE_CHECK(check_ptr(u));
    MOE_CHECK(check_ptr(expert_offsets));
    MOE_CHECK(check_ptr(sorted_slot));
    MOE_CHECK(check_ptr(topk_w));
    MOE_CHECK(check_ptr(y_acc));
    cudaStream_t s = (cudaStream_t)stream;
    MOE_CUDA(cudaMemsetAsync(y_acc, 0, size_t(T) * expert_in(*cfg) * sizeof(float), s));
    MOE_CUDA(launch_active_list(expert_offsets + rg.e0, rg.ne, at<int32_t>(ws, L.active), s));
    if (routed_tc(cfg, T))
        MOE_CUDA(launch_tile_start(expert_offsets + rg.e0, rg.ne, expert_bn(cfg, T), at<int32_t>(ws, L.tiles), s));
    return run_experts(cfg, w, u, nullptr, T, expert_offsets, sorted_slot, topk_w, y_acc, true, false, ws, L, s,
                       nullptr, rg);
}
}  // namespace

extern "C" {

moe_status moe_grouped_ffn(const moe_config* cfg, const moe_weights* w, const void* u, int64_t T,
                           const int32_t* expert_offsets, const int32_t* sorted_slot, const float* topk_w,
                           float* y_acc, void* ws, size_t ws_bytes, moe_stream_t stream) {
    if (!cfg) return MOE_ERR_INVALID_ARGUMENT;
    return grouped_ffn_range(cfg, w, u, T, expert_offsets, sorted_slot, topk_w, ExpertRange{0, cfg->num_experts},
                             y_acc, ws, ws_bytes, stream);
}

moe_status moe_grouped_ffn_experts(const moe_config* cfg, const moe_weights* w, const void* u, int64_t T,
                                   const int32_t* expert_offsets, const int32_t* sorted_slot, const float* topk_w,
                                   int32_t expert_begin, int32_t expert_end, float* y_acc, void* ws,
                                   size_t ws_bytes, moe_stream_t stream) {
    MOE_CHECK(moe_config_validate(cfg));
    if (expert_begin < 0 || expert_end <= expert_begin || expert_end > cfg->num_experts)
        return MOE_ERR_INVALID_ARGUMENT;
    return grouped_ffn_range(cfg, w, u, T, expert_offsets, sorted_slot, topk_w,
                             ExpertRange{expert_begin, expert_end - expert_begin}, y_acc, ws, ws_bytes, stream);
}

moe_status moe_latent_down(const moe_config* cfg, const moe_weights* w, const void* x, int64_t T, void* z,
                           void* ws, size_t ws_bytes, moe_stream_t stream) {
    MOE_CHECK(moe_config_validate(cfg));
    if (!cfg->latent_dim) return MOE_ERR_INVALID_ARGUMENT;
    WsLayout L;
    MOE_CHECK(prelude(cfg, w, T, ws, ws_bytes, &L));
    if (T == 0) return MOE_OK;
    MOE_CHECK(check_ptr(x));
    MOE_CHECK(check_ptr(z));
    return run_latent_down(cfg, w, x, T, z, ws, L, (cudaStream_t)stream);
}

moe_status moe_combine(const moe_config* cfg, const moe_weights* w, const float* y_acc, const void* x,
                       const float* coef, int64_t T, void* y, void* ws, size_t ws_bytes, moe_stream_t stream) {
    MOE_CHECK(moe_config_validate(cfg));
    WsLayout L;
    MOE_CHECK(prelude(cfg, w, T, ws, ws_bytes, &L));
    if (T == 0) return MOE_OK;
    MOE_CHECK(check_ptr(y_acc));
    MOE_CHECK(check_ptr(x));
    MOE_CHECK(check_ptr(y));
    if (cfg->shared_mode == MOE_SHARED_BLEND) MOE_CHECK(check_ptr(coef));
    cudaStream_t s = (cudaStream_t)stream;
    if (cfg->shared_mode != MOE_SHARED_NONE)
        MOE_CHECK(run_experts(cfg, w, nullptr, x, T, nullptr, nullptr, nullptr, nullptr, false, true, ws, L, s,
                              nullptr));
    RoutedSum rs;
    rs.rows = y_acc;
    return run_output(cfg, w, rs, coef, T, y, ws, L, s);
}

moe_status moe_block_forward(const moe_config* cfg, const moe_weights* w, const void* x, int64_t T, void* y,
                             void* ws, size_t ws_bytes, moe_stream_t stream) {
    MOE_CHECK(moe_config_validate(cfg));
    WsLayout L;
    MOE_CHECK(prelude(cfg, w, T, ws, ws_bytes, &L));
    if (T == 0) return MOE_OK;
    MOE_CHECK(check_ptr(x));
    MOE_CHECK(check_ptr(y));
    cudaStream_t s = (cudaStream_t)stream;
    {
        const DecodeArgs d = decode_args(cfg, w, x, T, y, ws, L);
        if (use_decode(cfg, T, d)) {
            MOE_CUDA(launch_decode(d, s));
            return MOE_OK;
        }
    }
    const int K = expert_in(*cfg);
    float* y_acc = at<float>(ws, L.y_acc);
    int32_t* idx = at<int32_t>(ws, L.topk_idx);
    float* wts = at<float>(ws, L.topk_w);
    float* coef = at<float>(ws, L.coef);
    const bool rtc = routed_tc(cfg, T);
    const void* u = cfg->latent_dim ? at<void>(ws, L.z) : x;
    int32_t* offsets = at<int32_t>(ws, L.offsets);
    int32_t* sorted_slot = at<int32_t>(ws, L.sorted_slot);
    // both engines add every slot's weighted output into y_acc: its rows are cleared by the
    // router; a single token's permutation comes from the top-k warp itself
    PermOut perm;
    perm.offsets = offsets;
    perm.sorted_slot = sorted_slot;
    perm.slot_pos = at<int32_t>(ws, L.slot_pos);
    perm.active = at<int32_t>(ws, L.active);
    perm.tiles = rtc ? at<int32_t>(ws, L.tiles) : nullptr;
    MOE_CHECK(run_route(cfg, w, x, T, idx, wts, coef, y_acc, K, ws, L, s, &perm));
    if (cfg->latent_dim) MOE_CHECK(run_latent_down(cfg, w, x, T, at<void>(ws, L.z), ws, L, s));
    if (T > 1) MOE_CHECK(run_permute(cfg, idx, T, offsets, sorted_slot, at<int32_t>(ws, L.slot_pos), ws, L, s, rtc));
    RoutedSum rs;
    MOE_CHECK(run_experts(cfg, w, u, x, T, offsets, sorted_slot, wts, y_acc, true, true, ws, L, s, &rs));
    return run_output(cfg, w, rs, coef, T, y, ws, L, s);
}

moe_status moe_read_device_status(void* ws, moe_stream_t stream) {
    if (!ws) return MOE_ERR_INVALID_ARGUMENT;
    int status = 0;
    cudaStream_t s = (cudaStream_t)stream;
    MOE_CUDA(cudaMemcpyAsync(&status, ws, sizeof(int), cudaMemcpyDeviceToHost, s));
    MOE_CUDA(cudaStreamSynchronize(s));
    MOE_CUDA(cudaMemsetAsync(ws, 0, sizeof(int), s));
    MOE_CUDA(cudaStreamSynchronize(s));
    if (status == MOE_ERR_DEVICE_CHECK || status == MOE_ERR_DEVICE_TIMEOUT) return moe_status(status);
    return status == 0 ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_clear_device_status(void* ws, moe_stream_t stream) {
    if (!ws) return MOE_ERR_INVALID_ARGUMENT;
    MOE_CUDA(cudaMemsetAsync(ws, 0, 256, (cudaStream_t)stream));
    return MOE_OK;
}

const char* moe_status_string(moe_status s) {
    switch (s) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARGUMENT: return "invalid argument";
        case MOE_ERR_SHAPE_OVERFLOW: return "shape overflow";
        case MOE_ERR_INVALID_QUANTIZATION: return "invalid quantization parameters";
        case MOE_ERR_MISSING_TENSOR: return "missing tensor";
        case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
        case MOE_ERR_CUDA: return "CUDA error";
        case MOE_ERR_DEVICE_CHECK: return "device-side check failed (expert id out of range)";
        case MOE_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
        case MOE_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    }
    return "unknown status";
}

}  // extern "C"
