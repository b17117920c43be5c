/*
 * moe_oracle.c -- plain fp64 CPU oracle of the sparse MoE FFN block forward.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg load this library. It shares no code, header, table or
 * constant with the CUDA library, and it never calls it.
 *
 * Everything is evaluated one token at a time, in double precision, from the
 * stored tensors converted exactly to double (bf16 and f32 are exact in
 * double; 4-bit affine weights are dequantised exactly as scale*q + bias).
 * No blocking, no fusion, no reordering: each step is the plain definition.
 *
 * Sources (page title, section):
 *  - Klear sparse MoE family PR (mlxcel #1044), item 2: the shared expert is
 *    blended by a per-token 2-way softmax of a [2, hidden] coefficient head
 *    with a [2] bias; coefficient index 0 weights the routed mixture, index 1
 *    the shared expert.
 *  - same PR, item 3: routing is the sigmoid of fp32 router logits; the
 *    expert bias is added to a copy used only to select experts, the combine
 *    weights are the unbiased sigmoid scores of the selected experts,
 *    norm_topk_prob divides them by their sum, and the declared
 *    routed_scaling_factor is not applied.
 *  - libmir-metal clamped_routed/experts/mod.rs, ClampedRoutedExperts::forward:
 *    router -> router_top_k_unit(top_k) (softmax over the selected logits) ->
 *    gate_up with a clamp limit and biases -> down weighted by the routing
 *    weights and summed; ExpertLayout::DenseFused's interleaved gate_up.
 *  - ferrox latent_moe.rs, module doc and kimi_latent_moe_forward: routing on
 *    the full hidden, latent = down_proj(hidden), experts in latent space,
 *    combined = sum_i w_i * expert_i(latent), rms_norm iff use_norm,
 *    up_proj, then + shared_expert(hidden). KimiExpertWeights::forward gives
 *    the expert shape down(act(gate(x), up(x))) with [out, in] weights.
 *  - mlxcel issue #974, "What exists": stacked switch_mlp expert planes and
 *    the affine 4-bit mode (weight, scales, biases, group_size 64, bits 4).
 *  - libmir-metal clamped_routed/experts/mod.rs, the split/u32 MXFP4 layout
 *    (gate, up and down blocks, each with scales and a bias); the element and
 *    scale encodings are not on the pages and come from the public OCP
 *    Microscaling Formats (MX) Specification v1.0: blocks of 32 elements, each
 *    element FP4 E2M1 (sign, 2 exponent bits with bias 1, 1 mantissa bit,
 *    subnormal when the exponent field is 0), one shared E8M0 scale per block
 *    (2^(byte - 127); byte 255 is NaN). ExpertLayout::Native's single gate_up
 *    plane (blocks, scales, bias) is read as the interleaved gate_up: row 2i
 *    gate, 2i+1 up, its scales / biases in the same row order.
 *
 * Readings where the pages are silent (each listed in the design notes):
 *  - SwiGLU is silu(g) * v with silu(g) = g / (1 + e^-g).
 *  - Clamped SwiGLU: g' = min(g, limit), v' = clamp(v, -limit, limit),
 *    out = g' * sigmoid(alpha * g') * (v' + 1); linear biases enter before it.
 *  - Interleaved gate_up: row 2i is gate_i, row 2i+1 is up_i (bias likewise).
 *  - Top-k: descending selection key, exact ties go to the lower index.
 *  - 4-bit word layout: element j of a row at bits 4*(j mod 8) of word j/8;
 *    w = scale * q + bias per group of group_size consecutive inputs.
 *  - RMSNorm: v / sqrt(mean(v^2) + eps) * gamma.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_SOFTMAX_ALL = 0, ORC_SIGMOID = 1, ORC_SOFTMAX_TOPK = 2 };
enum { ORC_SWIGLU = 0, ORC_SWIGLU_CLAMPED = 1 };
enum { ORC_F32 = 0, ORC_BF16 = 1, ORC_Q4 = 2, ORC_MXFP4 = 3 };
enum { ORC_SHARED_NONE = 0, ORC_SHARED_ADD = 1, ORC_SHARED_BLEND = 2 };

typedef struct {
    int32_t hidden, num_experts, top_k, intermediate;
    int32_t scoring, norm_topk_prob;
    double routed_scaling_factor;
    int32_t activation;
    double swiglu_limit, swiglu_alpha;
    int32_t gate_up_interleaved, has_expert_bias, has_router_bias, has_selection_bias;
    int32_t act_dtype, weight_format, group_size;
    int32_t shared_mode, shared_intermediate;
    int32_t latent_dim, latent_use_norm;
    double rms_eps;
    int32_t dense_weight_format;  /* router, shared and latent planes: act dtype or Q4 */
    int32_t dense_group_size;     /* Q4 group of those planes                          */
} orc_config;

/* Host pointers to the stored tensors. Dense tensors are in the activation
 * dtype (f32 or bf16 bit patterns), except selection_bias which is f32.
 * Routed expert planes are in weight_format; for 4-bit, *_w are the packed
 * words and *_s / *_z the bf16 per-group scales / biases. */
typedef struct {
    const void *router_w, *router_b, *selection_bias, *coef_w, *coef_b;
    const void *gate_w, *up_w, *gate_up_w, *gate_b, *up_b, *gate_up_b, *down_w, *down_b;
    const void *gate_s, *gate_z, *up_s, *up_z, *down_s, *down_z;
    const void *shared_gate_w, *shared_up_w, *shared_down_w;
    const void *latent_down_w, *latent_up_w, *latent_norm_w;
    const void *gate_up_s, *gate_up_z;  /* 4-bit interleaved gate_up plane */
    /* 4-bit dense planes: bf16 scales / biases [rows, cols / dense_group_size] */
    const void *router_s, *router_z, *shared_gate_s, *shared_gate_z, *shared_up_s, *shared_up_z;
    const void *shared_down_s, *shared_down_z, *latent_down_s, *latent_down_z;
    const void *latent_up_s, *latent_up_z;
} orc_weights;

static double bf16_bits_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Element i of a dense tensor stored as f32 or bf16. */
static double dense_at(const void *p, int32_t dtype, int64_t i)
{
    if (dtype == ORC_F32) return (double)((const float *)p)[i];
    return bf16_bits_to_double(((const uint16_t *)p)[i]);
}

/* Exact dequantisation of one 4-bit affine weight W[row, col] of a plane
 * with `cols` inputs per row (row counts across stacked experts). */
double orc_dequant_q4(const uint32_t *q, const uint16_t *scales, const uint16_t *biases,
                      int64_t cols, int32_t group_size, int64_t row, int64_t col)
{
    uint32_t word = q[row * (cols / 8) + col / 8];
    int code = (int)((word >> (4 * (col % 8))) & 0xFu);
    int64_t groups = cols / group_size;
    double s = bf16_bits_to_double(scales[row * groups + col / group_size]);
    double b = bf16_bits_to_double(biases[row * groups + col / group_size]);
    return s * (double)code + b;
}

/* One MXFP4 weight W[row, col]: the E2M1 element value times its block's
 * E8M0 scale, 32 elements per block (OCP MX v1.0). The element value is the
 * format's definition written out: exponent field e, mantissa bit m, and
 * (-1)^sign * 2^(e-1) * (1 + m/2) for e > 0, (-1)^sign * m/2 for e = 0. */
double orc_dequant_mxfp4(const uint32_t *q, const uint8_t *scales, int64_t cols, int64_t row, int64_t col)
{
    uint32_t word = q[row * (cols / 8) + col / 8];
    int code = (int)((word >> (4 * (col % 8))) & 0xFu);
    int e = (code >> 1) & 3, m = code & 1;
    double v = e > 0 ? ldexp(1.0 + 0.5 * m, e - 1) : 0.5 * m;
    if (code & 8) v = -v;
    int sbyte = scales[row * (cols / 32) + col / 32];
    if (sbyte == 255) return NAN;
    return ldexp(v, sbyte - 127);
}

/* W[e, r, c] of a stacked routed-expert plane [E, rows, cols]. */
static double plane_at(const orc_config *cfg, const void *w, const void *s, const void *z,
                       int64_t rows, int64_t cols, int64_t e, int64_t r, int64_t c)
{
    int64_t row = e * rows + r;
    if (cfg->weight_format == ORC_Q4)
        return orc_dequant_q4((const uint32_t *)w, (const uint16_t *)s, (const uint16_t *)z,
                              cols, cfg->group_size, row, c);
    if (cfg->weight_format == ORC_MXFP4)
        return orc_dequant_mxfp4((const uint32_t *)w, (const uint8_t *)s, cols, row, c);
    return dense_at(w, cfg->weight_format, row * cols + c);
}

double orc_activation(int32_t act, double g, double v, double limit, double alpha)
{
    if (act == ORC_SWIGLU) return g / (1.0 + exp(-g)) * v;
    double gc = g < limit ? g : limit;
    double vc = v < -limit ? -limit : (v > limit ? limit : v);
    return gc / (1.0 + exp(-alpha * gc)) * (vc + 1.0);
}

/* W[r, c] of a dense (non-routed) [rows, cols] plane: the activation dtype, or
 * 4-bit affine words with bf16 scales / biases per dense_group_size columns (a
 * 4-bit checkpoint quantises its dense projections too: mlxcel issue #974's
 * Jamba study, models/jamba-v0.1-4bit's quantised dense projections). */
static double dense_plane_at(const orc_config *cfg, const void *w, const void *s, const void *z,
                             int64_t cols, int64_t r, int64_t c)
{
    if (cfg->dense_weight_format == ORC_Q4)
        return orc_dequant_q4((const uint32_t *)w, (const uint16_t *)s, (const uint16_t *)z,
                              cols, cfg->dense_group_size, r, c);
    return dense_at(w, cfg->act_dtype, r * cols + c);
}

/* y[r] = sum_c W[r, c] * v[c] for a dense [rows, cols] plane. */
static void dense_matvec(const orc_config *cfg, const void *W, const void *S, const void *Z,
                         int64_t rows, int64_t cols, const double *v, double *y)
{
    for (int64_t r = 0; r < rows; ++r) {
        double acc = 0.0;
        for (int64_t c = 0; c < cols; ++c) acc += dense_plane_at(cfg, W, S, Z, cols, r, c) * v[c];
        y[r] = acc;
    }
}

/* One routed expert: out = Wd[e] * act(Wg[e] u + bg, Wu[e] u + bu) + bd. */
static void routed_expert(const orc_config *cfg, const orc_weights *w, int64_t e,
                          const double *u, double *out, double *h)
{
    const int64_t K = cfg->latent_dim ? cfg->latent_dim : cfg->hidden;
    const int64_t I = cfg->intermediate;
    const int32_t ad = cfg->act_dtype;
    for (int64_t i = 0; i < I; ++i) {
        double g = 0.0, v = 0.0;
        for (int64_t c = 0; c < K; ++c) {
            double wg, wu;
            if (cfg->gate_up_interleaved) {
                wg = plane_at(cfg, w->gate_up_w, w->gate_up_s, w->gate_up_z, 2 * I, K, e, 2 * i, c);
                wu = plane_at(cfg, w->gate_up_w, w->gate_up_s, w->gate_up_z, 2 * I, K, e, 2 * i + 1, c);
            } else {
                wg = plane_at(cfg, w->gate_w, w->gate_s, w->gate_z, I, K, e, i, c);
                wu = plane_at(cfg, w->up_w, w->up_s, w->up_z, I, K, e, i, c);
            }
            g += wg * u[c];
            v += wu * u[c];
        }
        if (cfg->has_expert_bias) {
            if (cfg->gate_up_interleaved) {
                g += dense_at(w->gate_up_b, ad, e * 2 * I + 2 * i);
                v += dense_at(w->gate_up_b, ad, e * 2 * I + 2 * i + 1);
            } else {
                g += dense_at(w->gate_b, ad, e * I + i);
                v += dense_at(w->up_b, ad, e * I + i);
            }
        }
        h[i] = orc_activation(cfg->activation, g, v, cfg->swiglu_limit, cfg->swiglu_alpha);
    }
    for (int64_t r = 0; r < K; ++r) {
        double acc = 0.0;
        for (int64_t i = 0; i < I; ++i)
            acc += plane_at(cfg, w->down_w, w->down_s, w->down_z, K, I, e, r, i) * h[i];
        if (cfg->has_expert_bias) acc += dense_at(w->down_b, ad, e * K + r);
        out[r] = acc;
    }
}

/* The shared expert on the full hidden: down(act(gate x, up x)), no biases. */
static void shared_expert(const orc_config *cfg, const orc_weights *w, const double *x,
                          double *out, double *h)
{
    const int64_t H = cfg->hidden, Is = cfg->shared_intermediate;
    for (int64_t i = 0; i < Is; ++i) {
        double g = 0.0, v = 0.0;
        for (int64_t c = 0; c < H; ++c) {
            g += dense_plane_at(cfg, w->shared_gate_w, w->shared_gate_s, w->shared_gate_z, H, i, c) * x[c];
            v += dense_plane_at(cfg, w->shared_up_w, w->shared_up_s, w->shared_up_z, H, i, c) * x[c];
        }
        h[i] = orc_activation(cfg->activation, g, v, cfg->swiglu_limit, cfg->swiglu_alpha);
    }
    dense_matvec(cfg, w->shared_down_w, w->shared_down_s, w->shared_down_z, H, Is, h, out);
}

/* Router for one token: logits, selection keys, the chosen experts (or the
 * caller's `forced` set) and their combine weights. */
static void route_token(const orc_config *cfg, const orc_weights *w, const double *x,
                        const int32_t *forced, double *logits, double *keys, double *score,
                        int32_t *idx, double *wts)
{
    const int64_t H = cfg->hidden, E = cfg->num_experts, k = cfg->top_k;
    const int32_t ad = cfg->act_dtype;
    for (int64_t e = 0; e < E; ++e) {
        double acc = 0.0;
        for (int64_t c = 0; c < H; ++c)
            acc += dense_plane_at(cfg, w->router_w, w->router_s, w->router_z, H, e, c) * x[c];
        if (cfg->has_router_bias) acc += dense_at(w->router_b, ad, e);
        logits[e] = acc;
    }
    if (cfg->scoring == ORC_SOFTMAX_ALL) {
        double m = logits[0], sum = 0.0;
        for (int64_t e = 1; e < E; ++e) if (logits[e] > m) m = logits[e];
        for (int64_t e = 0; e < E; ++e) { score[e] = exp(logits[e] - m); sum += score[e]; }
        for (int64_t e = 0; e < E; ++e) score[e] /= sum;
    } else if (cfg->scoring == ORC_SIGMOID) {
        for (int64_t e = 0; e < E; ++e) score[e] = 1.0 / (1.0 + exp(-logits[e]));
    } else {
        for (int64_t e = 0; e < E; ++e) score[e] = logits[e];
    }
    for (int64_t e = 0; e < E; ++e) {
        keys[e] = score[e];
        if (cfg->has_selection_bias) keys[e] += (double)((const float *)w->selection_bias)[e];
    }
    if (forced) {
        for (int64_t j = 0; j < k; ++j) idx[j] = forced[j];
    } else {
        char *taken = (char *)calloc((size_t)E, 1);
        for (int64_t j = 0; j < k; ++j) {
            int64_t best = -1;
            for (int64_t e = 0; e < E; ++e)
                if (!taken[e] && (best < 0 || keys[e] > keys[best])) best = e;
            taken[best] = 1;
            idx[j] = (int32_t)best;
        }
        free(taken);
    }
    if (cfg->scoring == ORC_SOFTMAX_TOPK) {
        double m = logits[idx[0]], sum = 0.0;
        for (int64_t j = 1; j < k; ++j) if (logits[idx[j]] > m) m = logits[idx[j]];
        for (int64_t j = 0; j < k; ++j) { wts[j] = exp(logits[idx[j]] - m); sum += wts[j]; }
        for (int64_t j = 0; j < k; ++j) wts[j] /= sum;
    } else {
        for (int64_t j = 0; j < k; ++j) wts[j] = score[idx[j]];
    }
    if (cfg->norm_topk_prob) {
        double sum = 0.0;
        for (int64_t j = 0; j < k; ++j) sum += wts[j];
        for (int64_t j = 0; j < k; ++j) wts[j] /= sum;
    }
    for (int64_t j = 0; j < k; ++j) wts[j] *= cfg->routed_scaling_factor;
}

/* The whole block for one token x (already in double). y == NULL routes only. */
static void token_forward(const orc_config *cfg, const orc_weights *w, const double *x,
                          const int32_t *forced, double *y, int32_t *idx, double *wts,
                          double *coef, double *keys, double *logits_out)
{
    const int64_t H = cfg->hidden, E = cfg->num_experts, k = cfg->top_k;
    const int64_t K = cfg->latent_dim ? cfg->latent_dim : cfg->hidden;
    const int64_t I = cfg->intermediate, Is = cfg->shared_intermediate;
    const int32_t ad = cfg->act_dtype;
    int64_t hmax = I > Is ? I : Is;
    double *logits = (double *)malloc(sizeof(double) * (size_t)E);
    double *key = (double *)malloc(sizeof(double) * (size_t)E);
    double *score = (double *)malloc(sizeof(double) * (size_t)E);
    route_token(cfg, w, x, forced, logits, key, score, idx, wts);
    if (keys) memcpy(keys, key, sizeof(double) * (size_t)E);
    if (logits_out) memcpy(logits_out, logits, sizeof(double) * (size_t)E);
    if (coef && cfg->shared_mode == ORC_SHARED_BLEND) {
        double c[2];
        for (int j = 0; j < 2; ++j) {
            double acc = 0.0;
            for (int64_t h = 0; h < H; ++h) acc += dense_at(w->coef_w, ad, j * H + h) * x[h];
            c[j] = acc + dense_at(w->coef_b, ad, j);
        }
        double m = c[0] > c[1] ? c[0] : c[1];
        double e0 = exp(c[0] - m), e1 = exp(c[1] - m);
        coef[0] = e0 / (e0 + e1);
        coef[1] = e1 / (e0 + e1);
    } else if (coef) {
        coef[0] = coef[1] = 0.0;
    }
    if (y) {
        double *u = (double *)malloc(sizeof(double) * (size_t)K);
        double *acc = (double *)calloc((size_t)K, sizeof(double));
        double *o = (double *)malloc(sizeof(double) * (size_t)K);
        double *hb = (double *)malloc(sizeof(double) * (size_t)hmax);
        double *yr = (double *)malloc(sizeof(double) * (size_t)H);
        if (cfg->latent_dim) dense_matvec(cfg, w->latent_down_w, w->latent_down_s, w->latent_down_z, K, H, x, u);
        else memcpy(u, x, sizeof(double) * (size_t)K);
        for (int64_t j = 0; j < k; ++j) {
            routed_expert(cfg, w, idx[j], u, o, hb);
            for (int64_t r = 0; r < K; ++r) acc[r] += wts[j] * o[r];
        }
        if (cfg->latent_dim) {
            if (cfg->latent_use_norm) {
                double ss = 0.0;
                for (int64_t r = 0; r < K; ++r) ss += acc[r] * acc[r];
                double inv = 1.0 / sqrt(ss / (double)K + cfg->rms_eps);
                for (int64_t r = 0; r < K; ++r)
                    acc[r] = acc[r] * inv * dense_at(w->latent_norm_w, ad, r);
            }
            dense_matvec(cfg, w->latent_up_w, w->latent_up_s, w->latent_up_z, H, K, acc, yr);
        } else {
            memcpy(yr, acc, sizeof(double) * (size_t)H);
        }
        if (cfg->shared_mode == ORC_SHARED_NONE) {
            memcpy(y, yr, sizeof(double) * (size_t)H);
        } else {
            double *s = (double *)malloc(sizeof(double) * (size_t)H);
            shared_expert(cfg, w, x, s, hb);
            if (cfg->shared_mode == ORC_SHARED_ADD) {
                for (int64_t h = 0; h < H; ++h) y[h] = yr[h] + s[h];
            } else {
                double c[2];
                if (coef) { c[0] = coef[0]; c[1] = coef[1]; }
                else {
                    for (int j = 0; j < 2; ++j) {
                        double a = 0.0;
                        for (int64_t h = 0; h < H; ++h) a += dense_at(w->coef_w, ad, j * H + h) * x[h];
                        c[j] = a + dense_at(w->coef_b, ad, j);
                    }
                    double m = c[0] > c[1] ? c[0] : c[1];
                    double e0 = exp(c[0] - m), e1 = exp(c[1] - m);
                    c[0] = e0 / (e0 + e1);
                    c[1] = e1 / (e0 + e1);
                }
                for (int64_t h = 0; h < H; ++h) y[h] = yr[h] * c[0] + s[h] * c[1];
            }
            free(s);
        }
        free(u); free(acc); free(o); free(hb); free(yr);
    }
    free(logits); free(key); free(score);
}

static void load_token(const orc_config *cfg, const void *x, int64_t t, double *xt)
{
    for (int64_t h = 0; h < cfg->hidden; ++h)
        xt[h] = dense_at(x, cfg->act_dtype, t * cfg->hidden + h);
}

int orc_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* The block forward for the tokens listed in `tokens` (n of them) of a batch
 * x [T, hidden]. Outputs are indexed by list position. y == NULL routes only.
 * coef, keys and logits may be NULL. Returns 0, or -1 on a bad token id. */
int orc_forward(const orc_config *cfg, const orc_weights *w, const void *x, int64_t T,
                const int64_t *tokens, int64_t n, double *y, int32_t *idx, double *wts,
                double *coef, double *keys, double *logits, int32_t threads)
{
    const int64_t H = cfg->hidden, E = cfg->num_experts, k = cfg->top_k;
    for (int64_t i = 0; i < n; ++i)
        if (tokens[i] < 0 || tokens[i] >= T) return -1;
    (void)threads;
#pragma omp parallel for schedule(dynamic, 1) num_threads(threads > 0 ? threads : orc_max_threads())
    for (int64_t i = 0; i < n; ++i) {
        double *xt = (double *)malloc(sizeof(double) * (size_t)H);
        load_token(cfg, x, tokens[i], xt);
        token_forward(cfg, w, xt, NULL, y ? y + i * H : NULL, idx + i * k, wts + i * k,
                      coef ? coef + i * 2 : NULL, keys ? keys + i * E : NULL,
                      logits ? logits + i * E : NULL);
        free(xt);
    }
    return 0;
}

/* Token t evaluated with a caller-given expert set idx[k] (weights follow the
 * same scoring rule, restricted to that set). Used where near-ties make more
 * than one expert set correct. */
int orc_forward_with_indices(const orc_config *cfg, const orc_weights *w, const void *x,
                             int64_t T, int64_t t, const int32_t *forced, double *y,
                             double *wts)
{
    if (t < 0 || t >= T) return -1;
    for (int64_t j = 0; j < cfg->top_k; ++j)
        if (forced[j] < 0 || forced[j] >= cfg->num_experts) return -1;
    double *xt = (double *)malloc(sizeof(double) * (size_t)cfg->hidden);
    int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * (size_t)cfg->top_k);
    load_token(cfg, x, t, xt);
    token_forward(cfg, w, xt, forced, y, idx, wts, NULL, NULL, NULL);
    free(xt); free(idx);
    return 0;
}

/* Permutation of slots (slot s = t*k + j) into per-expert groups: a stable
 * counting sort by expert id. offsets[E+1] is the exclusive prefix sum of the
 * per-expert counts, sorted_slot lists the slots of expert 0, then 1, ..., in
 * ascending slot order, and slot_pos is its inverse. */
void orc_permute(const int32_t *idx, int64_t T, int32_t k, int32_t E, int32_t *offsets,
                 int32_t *sorted_slot, int32_t *slot_pos)
{
    int64_t S = T * (int64_t)k;
    int32_t *cursor = (int32_t *)calloc((size_t)E, sizeof(int32_t));
    for (int32_t e = 0; e <= E; ++e) offsets[e] = 0;
    for (int64_t s = 0; s < S; ++s) offsets[idx[s] + 1] += 1;
    for (int32_t e = 0; e < E; ++e) offsets[e + 1] += offsets[e];
    for (int32_t e = 0; e < E; ++e) cursor[e] = offsets[e];
    for (int64_t s = 0; s < S; ++s) {
        int32_t e = idx[s];
        sorted_slot[cursor[e]] = (int32_t)s;
        slot_pos[s] = cursor[e];
        cursor[e] += 1;
    }
    free(cursor);
}
