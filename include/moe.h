/*
 * moe.h -- C ABI of the sparse Mixture-of-Experts FFN block forward on B200.
 *
 * The block (Klear sparse MoE family PR, items 2-3; libmir-metal
 * clamped_routed/experts/mod.rs, ClampedRoutedExperts::forward/execute;
 * ferrox latent_moe.rs, kimi_latent_moe_forward):
 *
 *   logits = x Wr^T (+ b_r)                           router, fp32 logits
 *   scores = softmax(logits) | sigmoid(logits) | logits   (per `scoring`)
 *   keys   = scores (+ selection_bias)                    select-only bias
 *   idx    = top-k(keys), descending, ties -> lower expert index
 *   w      = scores[idx] | softmax(logits[idx]); optionally w /= sum(w)
 *   u      = x, or z = x Wdp^T for the latent variant
 *   y_r    = sum_j w_j * Wd[e_j] act(Wg[e_j] u + bg, Wu[e_j] u + bu) (+ bd)
 *   latent: y_r = Wup (rmsnorm(y_r) * gamma)
 *   y      = y_r | y_r + s | y_r * c0 + s * c1,   s = shared expert(x),
 *            (c0, c1) = softmax(x Wc^T + b_c)
 *
 * Conventions for every call:
 *  - All pointers are DEVICE pointers unless stated otherwise. The caller
 *    allocates, owns and frees every buffer, the workspace included; the
 *    library never allocates device memory, never frees, and keeps no pointer
 *    after a call returns. The one exception is moe_permute_noalloc, whose
 *    scratch is a fixed device array inside the library (see its declaration:
 *    its size, and the race between calls that overlap on the GPU).
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *    stream). T (the token count) is the product of the input's leading dims;
 *    T == 0 returns MOE_OK and launches nothing.
 *  - Errors are returned as moe_status, never thrown and never aborted across
 *    this boundary (mlxcel issue #974: an exception crossing an FFI boundary is
 *    an uncatchable abort). Everything checkable on the host is checked before
 *    the first launch, so a failed call launched nothing.
 *  - Row-major layouts; weights are [out, in] (ferrox KimiExpertWeights:
 *    w1 gate [ffn, in], w2 down [in, ffn], w3 up [ffn, in]) and routed experts
 *    are stacked [E, out, in] (mlxcel issue #974, switch_mlp planes).
 *  - Every device pointer must be 16-byte aligned and every row length in
 *    bytes a multiple of 16 (hidden, intermediate, latent and shared widths
 *    multiples of 8 for bf16, of 4 for f32).
 *
 * Library: libmoe_b200.so (sm_100a). Thread-safe: calls keep no global device
 * state, except moe_permute_noalloc's fixed scratch array, which all of its calls
 * share (calls of it that overlap on the GPU race; serialise them).
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; declared here so that callers need no CUDA header. */
typedef struct CUstream_st *moe_stream_t;

typedef enum moe_status {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARGUMENT = 1,     /* NULL/misaligned pointer, bad enum, bad size  */
    MOE_ERR_SHAPE_OVERFLOW = 2,       /* a size product overflows the index types     */
    MOE_ERR_INVALID_QUANTIZATION = 3, /* bits / group_size not supported              */
    MOE_ERR_MISSING_TENSOR = 4,       /* a tensor the config needs is NULL            */
    MOE_ERR_UNSUPPORTED = 5,          /* valid on the pages, not built here           */
    MOE_ERR_CUDA = 6,                 /* a CUDA launch/runtime call failed            */
    MOE_ERR_DEVICE_CHECK = 7,         /* a kernel found an out-of-range expert id     */
    MOE_ERR_DEVICE_TIMEOUT = 8,       /* a bounded device wait gave up                */
    MOE_ERR_WORKSPACE_TOO_SMALL = 9   /* ws_bytes below moe_workspace_size(cfg, T)    */
} moe_status;

enum moe_scoring {
    MOE_SCORING_SOFTMAX_ALL = 0,   /* softmax over all E logits, then top-k            */
    MOE_SCORING_SIGMOID = 1,       /* sigmoid of fp32 logits (Klear PR item 3)          */
    MOE_SCORING_SOFTMAX_TOPK = 2   /* top-k logits, softmax over the k (router_top_k_unit) */
};
enum moe_activation {
    MOE_ACT_SWIGLU = 0,            /* silu(g) * v                                       */
    MOE_ACT_SWIGLU_CLAMPED = 1     /* g'=min(g,limit), v'=clamp(v,-limit,limit),
                                      g' * sigmoid(alpha g') * (v' + 1)                 */
};
enum moe_dtype {
    MOE_DTYPE_F32 = 0,
    MOE_DTYPE_BF16 = 1,
    MOE_DTYPE_Q4_AFFINE = 2,       /* weights only: packed 4-bit codes + bf16 scale/bias */
    MOE_DTYPE_MXFP4 = 3            /* weights only: E2M1 codes + an E8M0 scale per 32
                                      elements (OCP Microscaling Formats v1.0)          */
};
enum moe_shared_mode {
    MOE_SHARED_NONE = 0,
    MOE_SHARED_ADD = 1,            /* y = y_r + s (ferrox latent_moe.rs)                */
    MOE_SHARED_BLEND = 2           /* y = y_r * c0 + s * c1 (Klear PR item 2)           */
};

/* Plain-data description of one block. Checked by moe_config_validate. */
typedef struct moe_config {
    int32_t hidden;                /* H                                                 */
    int32_t num_experts;           /* E                                                 */
    int32_t top_k;                 /* k, 1 <= k <= E, k <= 16                           */
    int32_t intermediate;          /* I, routed expert intermediate width               */
    int32_t scoring;               /* enum moe_scoring                                  */
    int32_t norm_topk_prob;        /* 1: w /= sum(w) over the k                         */
    float routed_scaling_factor;   /* must be 1.0 (Klear PR item 3: not applied)        */
    int32_t activation;            /* enum moe_activation                               */
    float swiglu_limit;            /* clamp limit (clamped only), finite > 0            */
    float swiglu_alpha;            /* sigmoid slope (clamped only), finite              */
    int32_t gate_up_interleaved;   /* 1: one [E, 2I, K] plane, row 2i gate, 2i+1 up     */
    int32_t has_expert_bias;       /* 1: gate/up and down linear biases                 */
    int32_t has_router_bias;       /* 1: router bias b_r [E]                            */
    int32_t has_selection_bias;    /* 1: select-only bias [E] (f32)                     */
    int32_t act_dtype;             /* MOE_DTYPE_F32 or MOE_DTYPE_BF16: x, y and every
                                      non-routed weight                                 */
    int32_t weight_format;         /* routed planes: F32 (needs act F32), BF16, Q4_AFFINE,
                                      MXFP4 (both need act BF16)                        */
    int32_t group_size;            /* Q4: 32, 64 or 128; MXFP4: 32                      */
    int32_t bits;                  /* Q4 and MXFP4: 4                                   */
    int32_t shared_mode;           /* enum moe_shared_mode                              */
    int32_t shared_intermediate;   /* Is (> 0 iff shared_mode != NONE)                  */
    int32_t latent_dim;            /* L; 0 = no latent projection                       */
    int32_t latent_use_norm;       /* 1: RMSNorm of the combined latent                 */
    float rms_eps;                 /* RMSNorm epsilon, finite > 0                       */
    int32_t dense_format;          /* router, shared-expert and latent planes: 0 = in
                                      act_dtype, MOE_DTYPE_Q4_AFFINE = 4-bit affine (needs
                                      act BF16; the 2-row blend head stays in act_dtype)  */
    int32_t dense_group_size;      /* Q4 group of those planes: 32, 64 or 128           */
} moe_config;

/*
 * Device pointers to the block's tensors (NULL where the config does not use
 * them). Dense tensors are in act_dtype except selection_bias (f32).
 *   router_w [E, H]   router_b [E]   selection_bias [E] f32
 *   coef_w [2, H]     coef_b [2]                                (BLEND)
 *   gate_w, up_w [E, I, K]  or  gate_up_w [E, 2I, K]            K = L or H
 *   down_w [E, K, I]
 *   gate_b, up_b [E, I] or gate_up_b [E, 2I];  down_b [E, K]    (expert bias)
 *   Q4: gate_w/up_w/down_w hold uint32 words [E, rows, cols/8] (element j of a
 *       row at bits 4*(j mod 8) of word j/8), gate_s/up_s/down_s the bf16
 *       scales and gate_z/up_z/down_z the bf16 biases [E, rows, cols/group];
 *       weight = scale * q + bias.
 *   MXFP4: the same uint32 words, each code an E2M1 element (bit 3 sign, bits
 *       2..1 exponent, bit 0 mantissa: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6);
 *       gate_s/up_s/down_s hold one uint8 E8M0 scale per 32 elements
 *       [E, rows, cols/32], weight = element * 2^(scale - 127); the _z fields are
 *       unused. A scale byte of 255 (NaN in the format) gives non-finite weights.
 *   4-bit with gate_up_interleaved (libmir-metal ExpertLayout::Native: one
 *       gate_up block plane with its scales and bias): gate_up_w holds the
 *       words of the [E, 2I, K] plane (row 2i gate, 2i+1 up), gate_up_s (and,
 *       for Q4, gate_up_z) its companions [E, 2I, K/group] in the same row
 *       order; gate_s/gate_z/up_s/up_z are unused.
 *   shared_gate_w, shared_up_w [Is, H]; shared_down_w [H, Is]
 *   latent_down_w [L, H]; latent_up_w [H, L]; latent_norm_w [L]
 *   dense_format Q4 (a 4-bit checkpoint quantises its dense projections too; mlxcel issue
 *       #974, the Jamba study): router_w, shared_*_w and latent_down_w / latent_up_w hold
 *       uint32 words [rows, cols/8] like the routed Q4 planes, and <plane>_s / <plane>_z
 *       (router_s, router_z, shared_gate_s, ...) their bf16 scales and biases
 *       [rows, cols/dense_group_size]. coef_w / coef_b and latent_norm_w stay in act_dtype.
 */
typedef struct moe_weights {
    const void *router_w, *router_b, *selection_bias, *coef_w, *coef_b;
    const void *gate_w, *up_w, *gate_up_w, *gate_b, *up_b, *gate_up_b, *down_w, *down_b;
    const void *gate_s, *gate_z, *up_s, *up_z, *down_s, *down_z;
    const void *shared_gate_w, *shared_up_w, *shared_down_w;
    const void *latent_down_w, *latent_up_w, *latent_norm_w;
    const void *gate_up_s, *gate_up_z;  /* 4-bit interleaved gate_up plane: its scales / biases */
    const void *router_s, *router_z;    /* dense_format Q4: scales / biases of each dense plane */
    const void *shared_gate_s, *shared_gate_z, *shared_up_s, *shared_up_z, *shared_down_s, *shared_down_z;
    const void *latent_down_s, *latent_down_z, *latent_up_s, *latent_up_z;
} moe_weights;

/* Checks a config on the host (Klear PR "Other guards": zero checks before
 * divisibility, 1 <= k <= E, finite positive eps; mlxcel issue #974: bits and
 * group_size bounded before use). No device work. */
MOE_API moe_status moe_config_validate(const moe_config *cfg);

/* Checks that every tensor the config needs is present (MOE_ERR_MISSING_TENSOR,
 * e.g. a blend without its coefficient head) and 16-byte aligned. Host only. */
MOE_API moe_status moe_weights_validate(const moe_config *cfg, const moe_weights *w);

/* Bytes of workspace needed for up to max_tokens tokens (the same value serves
 * every call below). *bytes is written on MOE_OK only. Host only. */
MOE_API moe_status moe_workspace_size(const moe_config *cfg, int64_t max_tokens, size_t *bytes);

/* Router (a1 + a2): fp32 logits of x [T, H], scoring, select-only bias, top-k
 * and the combine weights; for BLEND also the 2-way coefficients.
 * Writes topk_idx [T, k] int32 (descending selection key, ties to the lower
 * index), topk_w [T, k] f32, coef [T, 2] f32 (BLEND; may be NULL otherwise).
 * Klear PR item 3; libmir-metal forward: router -> router_top_k_unit. */
MOE_API moe_status moe_route(const moe_config *cfg, const moe_weights *w, const void *x, int64_t T,
                     int32_t *topk_idx, float *topk_w, float *coef,
                     void *ws, size_t ws_bytes, moe_stream_t stream);

/* Permutation (a3): groups the T*k slots (slot s = t*k + j) by expert with a
 * stable counting sort. Writes expert_offsets [E+1] (exclusive prefix of the
 * per-expert counts), sorted_slot [T*k] (expert 0's slots ascending, then
 * expert 1's, ...) and slot_pos [T*k] (its inverse). An expert id outside
 * [0, E) sets MOE_ERR_DEVICE_CHECK in the workspace status word (see
 * moe_read_device_status) and that slot is dropped. */
MOE_API moe_status moe_permute(const moe_config *cfg, const int32_t *topk_idx, int64_t T,
                       int32_t *expert_offsets, int32_t *sorted_slot, int32_t *slot_pos,
                       void *ws, size_t ws_bytes, moe_stream_t stream);

/* Routed experts (a4 + a5): y_acc [T, K] f32 = sum over each token's k slots of
 * topk_w[slot] * expert(u[token]) with u [T, K] in act_dtype (K = L for the
 * latent variant, else H). Overwrites y_acc. The expert_offsets / sorted_slot
 * inputs are moe_permute's outputs for the same topk_idx.
 * libmir-metal execute (gate_up then down weighted by routing.weights);
 * ferrox kimi_latent_moe_forward (combined += w * expert(latent)).
 * Engine: the tcgen05 tensor-core kernel once 4*T*k >= E (bf16 activations,
 * K and I multiples of 64), else the CUDA-core weight-streaming kernels; the
 * environment variable MOE_PATH=gemv or MOE_PATH=tc forces one of them, for
 * the router and latent projections too (read at every call). MOE_PDL=1 enables programmatic dependent launch between the
 * kernels (off by default: it measured slower). */
MOE_API moe_status moe_grouped_ffn(const moe_config *cfg, const moe_weights *w, const void *u, int64_t T,
                           const int32_t *expert_offsets, const int32_t *sorted_slot,
                           const float *topk_w, float *y_acc,
                           void *ws, size_t ws_bytes, moe_stream_t stream);

/* Routed experts of one contiguous expert range (expert-parallel sharding; the pages run
 * the block on one device, so this call has no counterpart there). Computes what
 * moe_grouped_ffn computes, restricted to experts [expert_begin, expert_end): y_acc [T, K]
 * f32 = sum over each token's slots routed to those experts of topk_w[slot] *
 * expert(u[token]), zero where a token has none. The routed planes of `w` (gate/up/down,
 * their biases and 4-bit companions) hold ONLY these experts, stacked from expert_begin
 * (plane g is expert expert_begin + g); the dense planes are as for moe_grouped_ffn.
 * expert_offsets / sorted_slot / topk_w are the full permutation of all E experts, as
 * moe_permute writes it. The partial sums of ranges that cover [0, E) add up to
 * moe_grouped_ffn's result (one range per GPU, followed by a reduce-scatter of y_acc over
 * the token dimension). 0 <= expert_begin < expert_end <= E, else MOE_ERR_INVALID_ARGUMENT.
 * Overwrites y_acc. */
MOE_API moe_status moe_grouped_ffn_experts(const moe_config *cfg, const moe_weights *w, const void *u, int64_t T,
                                   const int32_t *expert_offsets, const int32_t *sorted_slot,
                                   const float *topk_w, int32_t expert_begin, int32_t expert_end,
                                   float *y_acc, void *ws, size_t ws_bytes, moe_stream_t stream);

/* Latent down projection (first half of a8): z [T, L] (act_dtype) = x Wdp^T.
 * ferrox kimi_latent_moe_forward: latent = down_proj(hidden). */
MOE_API moe_status moe_latent_down(const moe_config *cfg, const moe_weights *w, const void *x, int64_t T,
                           void *z, void *ws, size_t ws_bytes, moe_stream_t stream);

/* Combine (a6 + a7, and the tail of a8): from the routed sum y_acc [T, K] f32,
 * computes the shared expert on x, then y [T, H] (act_dtype) = y_r, y_r + s or
 * y_r * coef[:, 0] + s * coef[:, 1]; for the latent variant y_r = Wup
 * (rmsnorm(y_acc) * gamma) first. coef [T, 2] is moe_route's (BLEND only).
 * Klear PR item 2; ferrox kimi_latent_moe_forward (rms_norm, up_proj, + shared). */
MOE_API moe_status moe_combine(const moe_config *cfg, const moe_weights *w, const float *y_acc,
                       const void *x, const float *coef, int64_t T, void *y,
                       void *ws, size_t ws_bytes, moe_stream_t stream);

/* The whole block: y [T, H] = block(x [T, H]), act_dtype in and out. The engine is chosen
 * by the batch: one cooperative decode launch for one token (two with bf16 weights; no
 * latent projection, bf16 activations), the CUDA-core weight-streaming kernels for few
 * slots per expert, the tensor-core kernels from about E / 4 slots on (environment variable
 * MOE_PATH=gemv | tc | decode forces one engine where it can run). */
MOE_API moe_status moe_block_forward(const moe_config *cfg, const moe_weights *w, const void *x,
                             int64_t T, void *y, void *ws, size_t ws_bytes, moe_stream_t stream);

/* Permutation without a workspace (no counterpart on the pages: an addition for
 * callers that cannot allocate device memory). Some callers may not call cudaMalloc at
 * the point where they route tokens: a serving loop that reserved all of its device
 * memory up front and may not grow it, a host that owns the allocator and exposes none to
 * plug-ins, or code recorded into a CUDA graph while the allocation would break the
 * capture. This variant computes exactly what moe_permute computes, keeping its scratch
 * (status word, active-expert list, per-chunk histograms, 68,096 bytes) in one fixed
 * device array inside the library, which every GPU that loads the library holds until the
 * process exits. Limits: T * top_k <= 65,536 slots and num_experts <= 512, else
 * MOE_ERR_SHAPE_OVERFLOW before any launch. The caller still passes every input and
 * output. device_status (optional, caller-owned int32 on the device, zeroed by the caller)
 * receives MOE_ERR_DEVICE_CHECK on an out-of-range expert id, and passing it is the only
 * way to observe that check: with device_status NULL the bad slot is still dropped, but
 * the error goes to a word inside the fixed array that no call reads. No call allocates
 * or frees anything. The first call on each device (and the first after the device's
 * context was replaced, e.g. by cudaDeviceReset) looks up the array's device address
 * with that device current: make that first call before any stream capture. All calls
 * share the one array
 * and leave their contents in it, so calls that overlap on the GPU (different streams
 * without ordering, or different host threads) race: serialise them. */
MOE_API moe_status moe_permute_noalloc(const moe_config *cfg, const int32_t *topk_idx, int64_t T,
                                       int32_t *expert_offsets, int32_t *sorted_slot, int32_t *slot_pos,
                                       int32_t *device_status, moe_stream_t stream);

/* Synchronises `stream`, returns the status word that device-side checks
 * write into the workspace (MOE_OK, MOE_ERR_DEVICE_CHECK or
 * MOE_ERR_DEVICE_TIMEOUT) and clears it. The first 256 bytes of a workspace
 * hold this word and a launch counter that every call leaves at zero: a new
 * workspace must be zero-filled (or cleared with moe_clear_device_status)
 * before its first use. The same region holds the grid-barrier counters of the persistent
 * decode kernel, which every launch also leaves at zero. */
MOE_API moe_status moe_read_device_status(void *ws, moe_stream_t stream);

/* Clears the workspace's 256-byte status region, asynchronously on `stream`. */
MOE_API moe_status moe_clear_device_status(void *ws, moe_stream_t stream);

/* Failure-detection self test: one CTA waits on an mbarrier that nothing ever
 * completes, with the bounded wait every kernel of the library uses (a
 * %globaltimer deadline of timeout_ns, 0 < timeout_ns <= 1e9). When it gives up
 * it records MOE_ERR_DEVICE_TIMEOUT in the status word of `ws` (read it with
 * moe_read_device_status) and returns; nothing traps or hangs. Asynchronous on
 * `stream`; MOE_ERR_INVALID_ARGUMENT for a NULL ws or an out-of-range timeout. */
MOE_API moe_status moe_selftest_bounded_wait(void *ws, int64_t timeout_ns, moe_stream_t stream);

/* Failure-detection self test of the grid barrier the persistent decode kernel uses
 * between its phases (moe_block_forward on a decode-sized batch): one block arrives at a
 * barrier that needs two arrivals and polls it with the same %globaltimer deadline
 * (timeout_ns, 0 < timeout_ns <= 1e9); when it gives up it records
 * MOE_ERR_DEVICE_TIMEOUT in the status word of `ws` and returns, and the counter is put
 * back to zero. Asynchronous on `stream`; MOE_ERR_INVALID_ARGUMENT for a NULL ws or an
 * out-of-range timeout. */
MOE_API moe_status moe_selftest_grid_wait(void *ws, int64_t timeout_ns, moe_stream_t stream);

/* Static, NUL-terminated description of a status code. */
MOE_API const char *moe_status_string(moe_status status);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
