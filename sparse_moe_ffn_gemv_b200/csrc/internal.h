// internal.h -- host-side launchers shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include "moe.h"

namespace moe {

// out[t, r] = sum_c W[r, c] u[t, c] (+ bias[r]) (+ addend[t, r]) for the rows of
// W0 followed by the rows of W1 (the router and the coefficient head share a pass).
struct DenseGemvArgs {
    const void* W0 = nullptr; const void* b0 = nullptr; int rows0 = 0;
    const void* W1 = nullptr; const void* b1 = nullptr; int rows1 = 0;
    const void* u = nullptr; int64_t T = 0; int K = 0;
    void* out = nullptr; int ld_out = 0; int out_f32 = 0;
    const float* addend = nullptr; int ld_add = 0;
    int act_dtype = MOE_DTYPE_BF16;
    // W0 4-bit affine when s0 is set: words [rows0, K / 8], bf16 scales / biases [rows0, K / group0]
    const void *s0 = nullptr, *z0 = nullptr; int group0 = 64;
};
cudaError_t launch_dense_gemv(const DenseGemvArgs& a, cudaStream_t s);

struct TopkArgs {
    const float* logits = nullptr; int ld = 0; int64_t T = 0;
    int E = 0, k = 0, scoring = 0, norm = 0, has_sel = 0, blend = 0;
    const float* sel_bias = nullptr;
    int32_t* idx = nullptr; float* w = nullptr; float* coef = nullptr;
    float* zero = nullptr; int64_t zero_cols = 0;  // rows of this buffer are cleared per token
    // T == 1 only: the warp also writes the permutation of the token's k slots (offsets
    // [E + 1], sorted slots, their inverse, the active list and, if set, the tile prefix)
    int32_t *p_offsets = nullptr, *p_sorted = nullptr, *p_slot_pos = nullptr, *p_active = nullptr;
    int32_t* p_tiles = nullptr;
};
cudaError_t launch_topk(const TopkArgs& a, cudaStream_t s);

struct PermuteArgs {
    const int32_t* idx = nullptr; int64_t S = 0; int E = 0;
    int32_t* offsets = nullptr; int32_t* sorted_slot = nullptr; int32_t* slot_pos = nullptr;
    int32_t* active = nullptr; int32_t* chunk_hist = nullptr; int n_chunks = 0;
    int chunk = 2048;                // slots per chunk (one block each); n_chunks = ceil(S / chunk)
    int* status = nullptr;
    int tile_bn = 0;                 // > 0: also write tile_start[E + 1], the exclusive prefix
    int32_t* tile_start = nullptr;   //      of ceil(count_e / tile_bn) (tensor-core tile list)
};
cudaError_t launch_permute(const PermuteArgs& a, cudaStream_t s);
// active[0] = number of experts with tokens, active[1..] their ids, from offsets [E + 1].
cudaError_t launch_active_list(const int32_t* offsets, int E, int32_t* active, cudaStream_t s);

// dst[p, :] = src[sorted_slot[p] / k, :] for p < S (rows of K bf16): expert inputs in
// sorted order for the tensor-core path; with lo / hi (device pointers) only *lo <= p < *hi;
// to_f16: written as fp16.
cudaError_t launch_gather_rows(const void* src, int K, const int32_t* sorted_slot, int k, int64_t S,
                               void* dst, cudaStream_t s, const int32_t* lo = nullptr, const int32_t* hi = nullptr,
                               bool to_f16 = false);
// tile_start from offsets (moe_grouped_ffn called with a caller-made permutation).
cudaError_t launch_tile_start(const int32_t* offsets, int E, int tile_bn, int32_t* tile_start, cudaStream_t s);

// Routed + shared gate/up on CUDA cores: h = act(Wg u + bg, Wu u + bu).
struct GateUpArgs {
    int wf = MOE_DTYPE_BF16, interleaved = 0, has_bias = 0, group_size = 64;
    const void *gate_w = nullptr, *up_w = nullptr, *gate_up_w = nullptr;
    // 4-bit companions; with interleaved planes gate_s / gate_z are those of gate_up_w
    // ([E, 2I, K / group], the plane's row order)
    const void *gate_s = nullptr, *gate_z = nullptr, *up_s = nullptr, *up_z = nullptr;
    const void *gate_b = nullptr, *up_b = nullptr, *gate_up_b = nullptr;
    const int32_t *offsets = nullptr, *sorted_slot = nullptr, *active = nullptr;
    int k = 1, I = 0, K = 0, routed_groups = 0;  // routed_groups: bound on active experts
    const void* u = nullptr; void* h = nullptr;
    // shared expert (dense group over all T tokens), shared_I == 0 disables it
    const void *sg_w = nullptr, *su_w = nullptr; int shared_I = 0, Hs = 0;
    const void* xs = nullptr; void* hs = nullptr;
    // 4-bit shared planes when sg_s is set (bf16 scales / biases per s_group columns)
    const void *sg_s = nullptr, *sg_z = nullptr, *su_s = nullptr, *su_z = nullptr; int s_group = 64;
    int64_t T = 0;
    int act = 0; float limit = 7.f, alpha = 1.702f;
};
cudaError_t launch_gateup_gemv(const GateUpArgs& a, cudaStream_t s);

// Routed + shared down on CUDA cores: y_acc[token] += w * (Wd h + bd); s_acc = Wsd hs.
struct DownArgs {
    int wf = MOE_DTYPE_BF16, has_bias = 0, group_size = 64;
    const void *down_w = nullptr, *down_s = nullptr, *down_z = nullptr, *down_b = nullptr;
    const int32_t *offsets = nullptr, *sorted_slot = nullptr, *active = nullptr;
    const float* topk_w = nullptr;
    int k = 1, I = 0, K = 0, routed_groups = 0;
    const void* h = nullptr; float* y_acc = nullptr;
    const void* sd_w = nullptr; int shared_I = 0, Hs = 0; const void* hs = nullptr;
    float* s_acc = nullptr;
    const void *sd_s = nullptr, *sd_z = nullptr; int s_group = 64;  // 4-bit shared down plane
    int64_t T = 0;
};
cudaError_t launch_down_gemv(const DownArgs& a, cudaStream_t s);

// The routed sum of token t is the sum of rows [t*nsum, (t+1)*nsum) of `rows` (width H,
// fp32 or bf16 as rows_dtype says): nsum = 1 for an accumulated [T, H] buffer, nsum = k
// for per-slot weighted rows. y = r | r + s | c0 r + c1 s, stored in act dtype (or f32
// when out_f32).
cudaError_t launch_combine(const void* rows, int rows_dtype, int nsum, const float* s_acc, const float* coef,
                           int mode, int64_t T, int H, void* y, int act_dtype, cudaStream_t s, bool out_f32 = false);
// nrm = r / sqrt(mean(r^2) + eps) * gamma (act dtype), r the routed sum as above (width L).
cudaError_t launch_rmsnorm(const void* rows, int rows_dtype, int nsum, const void* gamma, float eps, int64_t T,
                           int L, void* out, int act_dtype, cudaStream_t s);

// ------------------------------------------------------------------ persistent decode kernel
// The whole block for a decode-sized batch (T <= 8, no latent projection) in one cooperative
// launch: router + coefficient rows and the shared expert's gate/up, a grid barrier, top-k
// and the routed gate/up, a grid barrier, then the routed and shared down rows with the
// weighted combine and the blend, each block owning a contiguous range of output rows.
struct DecodeArgs {
    int T = 0, H = 0, E = 0, k = 0, I = 0, Is = 0;
    int wf = MOE_DTYPE_BF16, interleaved = 0, has_bias = 0, group_size = 64;
    int act = 0; float limit = 7.f, alpha = 1.702f;
    int scoring = 0, norm = 0, has_sel = 0, shared_mode = 0;
    const void *router_w = nullptr, *router_b = nullptr, *coef_w = nullptr, *coef_b = nullptr;
    const float* sel_bias = nullptr;
    const void *gate_w = nullptr, *up_w = nullptr, *gate_up_w = nullptr;
    const void *gate_s = nullptr, *gate_z = nullptr, *up_s = nullptr, *up_z = nullptr;
    const void *gate_b = nullptr, *up_b = nullptr, *gate_up_b = nullptr;
    const void *down_w = nullptr, *down_s = nullptr, *down_z = nullptr, *down_b = nullptr;
    const void *sg_w = nullptr, *su_w = nullptr, *sd_w = nullptr;
    // 4-bit router and shared planes (dense_q4): bf16 scales / biases per dense_group columns
    int dense_q4 = 0, dense_group = 64;
    const void *router_s = nullptr, *router_z = nullptr;
    const void *sg_s = nullptr, *sg_z = nullptr, *su_s = nullptr, *su_z = nullptr, *sd_s = nullptr, *sd_z = nullptr;
    const void* x = nullptr; void* y = nullptr;
    float* logits = nullptr; int ld_logits = 0;   // workspace: fp32 router + coefficient logits
    void* h = nullptr;                            // workspace: bf16 [T * k, I] by slot
    void* hs = nullptr;                           // workspace: bf16 [T, Is]
    unsigned* bar = nullptr;                      // workspace: three zeroed counters
    int* status = nullptr;
};
// Dynamic shared memory the decode kernel needs for a config and T (0 if it cannot run it).
size_t decode_smem_bytes(const DecodeArgs& a);
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s);

// ------------------------------------------------------------------ tensor-core GEMM
int device_sm_count();          // SMs of the current device (148 if the query fails)
constexpr int kTcBN = 128;       // token rows per tile (4-bit weights, small batches)
constexpr int kTcBNWide = 256;   // token rows per tile of bf16 launches on large batches
constexpr int kTcRowsGateUp = 128;  // intermediate units per gate/up tile (gate + up rows)
constexpr int kTcRows = 256;        // output rows per tile of the other GEMMs
enum { kEpiGateUp = 0, kEpiScatterAdd = 1, kEpiStoreF32 = 2, kEpiStoreAct = 3 };

// One GEMM problem of a tensor-core launch: D[M rows, tokens] = W[M, K] . U[tokens, K]^T.
struct TcProblem {
    int mode = kEpiStoreF32;
    int M = 0, K = 0, m_blocks = 0;        // m_blocks = ceil(M / rows per tile)
    int grouped = 0;                       // 1: expert groups (offsets / tile_start), 0: one dense group
    int rows = 0, n_tiles = 0;             // dense: token rows and their tiles
    int bn = kTcBN;                        // token rows per tile (the kernel's; checked at launch)
    int band = 0;                          // dense: token tiles per band of the tile order (set at launch)
    int num_groups = 0;
    const int32_t* offsets = nullptr;      // [E + 1] sorted-row offsets of the groups
    const int32_t* tile_start = nullptr;   // [E + 1] prefix of token tiles per group
    const int32_t* sorted_slot = nullptr;  // scatter-add: sorted row -> slot (token = slot / k)
    const float* topk_w = nullptr;         // scatter-add: slot -> combine weight
    int k = 1;
    const void* bias0 = nullptr;           // bf16 [groups, M] (or [groups, 2M] interleaved gate/up)
    const void* bias1 = nullptr;           // bf16 [groups, M] (up bias, separate layout)
    int bias_interleaved = 0, interleaved = 0;
    void* out = nullptr; int ld_out = 0;
    const float* addend = nullptr; int ld_add = 0;
    // 4-bit affine weights (tc_q4_weight_map planes): bf16 scales / biases [groups, M, K / group_size]
    // of the first (gate or single) and second (up) weight plane
    int q4 = 0, group_size = 64;
    const void *qs0 = nullptr, *qz0 = nullptr, *qs1 = nullptr, *qz1 = nullptr;
    int mx = 0;  // with q4 = 1: MXFP4 codes, qs0 / qs1 the E8M0 scale bytes [groups, M, K / 32]
    int qrow_step = 1;  // companion rows per unit: 2 for an interleaved gate_up plane, whose
                        // up companions start one row after qs0 / qz0 (qs1 / qz1 = that row)
    // 4-bit affine weights run the MMA on fp16 operands (the dequantised s * q + b rounds to
    // 11 significant bits; bf16 keeps 8): the token operand of such a problem is fp16, and
    // out_f16 makes a gate/up problem write its h in fp16 for the fp16 down GEMM after it.
    int out_f16 = 0;
};

struct alignas(64) TcParams {
    TcParams() {  // unused tensor maps stay zero; the problems keep their defaults
        memset(static_cast<void*>(a0), 0, sizeof(a0));
        memset(static_cast<void*>(a1), 0, sizeof(a1));
        memset(static_cast<void*>(b), 0, sizeof(b));
    }
    CUtensorMap a0[2];  // weights (gate / single)
    CUtensorMap a1[2];  // weights (up), gate/up mode with separate planes
    CUtensorMap b[2][5];  // tokens, boxes of 16, 32, 64, 128 and 256 rows (a tile loads the smallest
                          // box that holds its valid tokens)
    TcProblem p[2];
    int nprob = 0;
    int* status = nullptr;
    int act = 0;
    float limit = 7.f, alpha = 1.702f;
};

bool tc_weight_map(CUtensorMap* m, const void* w, int E, int R, int K, bool interleaved);
// Packed 4-bit weight operand: [E, R, K / 8] uint32 words (8 codes each), one 64-wide K block
// (8 words) x 128 rows per box, no swizzle (the kernel's dequantising warps read it).
// row_step 2 views every other row of an interleaved [E, 2R, K / 8] plane from w (gate rows;
// pass w advanced by one row for the up rows).
bool tc_q4_weight_map(CUtensorMap* m, const void* w, int E, int R, int K, int row_step = 1);
// Five maps m[0..4] of the token operand [rows, K] bf16, boxes of 16, 32, 64, 128, 256 rows (<= bn).
bool tc_token_map(CUtensorMap* m, const void* u, int64_t rows, int K, int bn);
// dst[i] = fp16(src[i]) for n bf16 values (exact within fp16's range), n % 8 == 0.
cudaError_t launch_to_f16(const void* src, int64_t n, void* dst, cudaStream_t s);
cudaError_t launch_tc_gemm(TcParams& P, bool gateup, int64_t max_tiles, cudaStream_t s);

}  // namespace moe
