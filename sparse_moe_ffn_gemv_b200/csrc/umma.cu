// umma.cu -- tensor-core (tcgen05 / TMEM) grouped GEMM fed by TMA, for prefill-sized batches.
//
// D[128 token rows, 256 weight rows] = U[tokens, K] . W[rows, K]^T per tile: the tokens
// are the MMA's M side and the tile's 256 weight rows (128 gate + 128 up rows, or 256
// output rows) its N side, so that one 128 x 256 x 16 MMA per K step reads 12 KB of shared
// memory (a 128 x 128 pair of MMAs sharing the token tile would read 16 KB for the same
// work). Every expert group is padded only to the token tile, and each weight tile is read
// from HBM once and shared by the token tiles of its group through L2 (those tiles run at
// about the same time; dense problems walk their tiles in bands of token tiles so that the
// tiles running together share token tiles and weight blocks).
//
// One persistent CTA (or CTA pair) per SM (pair of SMs), warp-specialised:
//   warp 0      TMA producer: weight tile(s) + token tile per 64-wide K block into a
//               STAGES-deep shared-memory ring (128-byte swizzle)
//   warp 1      MMA issuer (one thread): tcgen05.mma kind::f16, bf16 x bf16 -> fp32 in
//               TMEM, M = 128 token rows x N = 256 weight rows
//   warps 2..9  epilogue (two warps per TMEM lane quarter, each half of the columns; one
//               token row per thread): tcgen05.ld, then SwiGLU / clamped SwiGLU -> bf16 h
//               (gate/up: gate and up of a unit are columns u and 128 + u), the weighted
//               combine (down: the slot's output row times its routing weight reduced
//               into the token's fp32 routed sum with 16-byte vector reductions), or a
//               plain store, each thread writing contiguous 16-byte vectors
//   4-bit weights: warps 2..5 epilogue (one per TMEM lane quarter, all 256 columns) and
//   warps 6..21 dequantisation: the producer loads the packed words, these warps write
//               w = scale * q + bias (fp16; MXFP4: bf16) into the swizzled operand layout
//               the MMA reads (mlxcel issue #974: affine 4-bit, per-group scale and bias). With 4-bit weights the shared memory holds two rings: a deep
//               one of small slots (the two packed tiles + the token tile of a K block)
//               that TMA fills far ahead, and a shallow one of bf16 operand tiles that
//               the dequantising warps fill and the MMA drains, so that load latency,
//               dequantisation and MMA overlap instead of sharing one stage
// Tiles of 128 token rows keep two accumulator sets in TMEM, so the epilogue of one tile
// overlaps the main loop of the next; bf16 launches on large batches use tiles of 256 token
// rows, which read each weight tile once for up to 256 routed rows: in grouped launches one
// CTA per tile (two MMAs per K step sharing the weight tile, the second skipped when the tile
// holds at most 128 rows, one accumulator set of 2 x 256 columns), in dense launches a
// cluster of two CTAs per tile (PAIR: each CTA holds 128 token rows and one 128-row weight
// tile, the leader issues tcgen05.mma.cta_group::2 with M = 256, N = 256 over both CTAs'
// shared memory, two accumulator sets of 256 columns per CTA).
// Every mbarrier wait is bounded by %globaltimer; a wait that gives up records
// MOE_ERR_DEVICE_TIMEOUT in the status word, drains its own outstanding copies / MMAs and
// returns, and TMEM is always freed.
//
// Block math (libmir-metal execute: gate_up with biases and limit, then down weighted by
// routing.weights and summed; ferrox KimiExpertWeights::forward: down(act(gate, up))).
#include <cuda.h>

#include <algorithm>
#include <mutex>
#include <type_traits>

#include <cuda_fp16.h>

#include "common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace moe {

namespace {

constexpr int kBM = 128;          // weight rows per MMA (M)
constexpr int kBK = 64;           // K per stage: one 128-byte swizzle atom of bf16
// 4-bit weights: 16 dequantising warps, one thread per (weight tile, row, half of the K
// block). With 8 warps (one whole row each) a warp took about 1100 cycles per K block, twice
// the MMA's 512: two warps per SM sub-partition could not hide the shared-memory and fence
// latencies of their chain.
constexpr int kDqThreads = 512;
constexpr int kDqParts = kDqThreads / (2 * kBM);  // parts of a K block per weight row
constexpr int kDqWords = 8 / kDqParts;             // packed words (8 codes each) per thread
constexpr int kDqTiles = 1;                        // weight tiles per dequantising thread
constexpr int kEpiThreads = 256;
constexpr int kPkBytes = kBM * kBK / 2;  // packed 4-bit weight tile: 128 rows x 32 bytes
constexpr int kMaxGroups = 512;   // expert groups whose tile table fits in shared memory
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s bound on any single wait

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* m) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups 1024 B apart.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr) {
    return uint64_t((saddr & 0x3FFFFu) >> 4) | (uint64_t(1) << 16) | (uint64_t(1024 >> 4) << 32) |
           (uint64_t(1) << 46) | (uint64_t(2) << 61);
}
// Instruction descriptor: kind::f16, A = B = bf16, D = f32, both K-major, M = 128, N = n.
__host__ __device__ constexpr uint32_t idesc_bf16(int n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(n >> 3) << 17) | (uint32_t(kBM >> 4) << 24);
}
// The same with A = B = fp16 (4-bit affine weights).
__host__ __device__ constexpr uint32_t idesc_f16(int n) {
    return (1u << 4) | (uint32_t(n >> 3) << 17) | (uint32_t(kBM >> 4) << 24);
}

__device__ __forceinline__ void umma(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(su32(bar))
                 : "memory");
}
// CTA pair: M = 256 rows (128 in each CTA's shared memory and TMEM), N = 256 (each CTA holds
// half of the N-side operand), issued by the pair's leader.
__host__ __device__ constexpr uint32_t idesc_bf16_pair() {
    return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(256 >> 3) << 17) | (uint32_t(256 >> 4) << 24);
}
__device__ __forceinline__ void umma_pair(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
// Arrive on the mbarrier at the same shared-memory offset in both CTAs of the pair once the
// leader's MMAs issued so far have completed.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            su32(bar)),
        "h"(uint16_t(3))
        : "memory");
}
// Issue an N-column TMEM load (N = 16 or 32) without waiting; the registers are valid only
// after tmem_ld_wait on the same array (which also keeps the compiler from using them early).
template <int N>
__device__ __forceinline__ void tmem_ld_issue(uint32_t taddr, uint32_t (&r)[N]) {
    static_assert(N == 16 || N == 32, "16 or 32 columns");
    if constexpr (N == 32) {
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
            "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
            : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
              "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
              "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
              "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
              "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
            : "r"(taddr));
    } else {
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
            : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
              "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
              "=r"(r[15])
            : "r"(taddr));
    }
}
template <int N>
__device__ __forceinline__ void tmem_ld_wait(uint32_t (&r)[N]) {
    if constexpr (N == 32) {
        asm volatile("tcgen05.wait::ld.sync.aligned;"
                     : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                       "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                       "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]),
                       "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]),
                       "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
                     :
                     : "memory");
    } else {
        asm volatile("tcgen05.wait::ld.sync.aligned;"
                     : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                       "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                       "+r"(r[14]), "+r"(r[15])
                     :
                     : "memory");
    }
}

// Where one tile lives.
struct TileInfo {
    int prob;      // problem index
    int group;     // expert id (grouped) or 0
    int mb;        // weight-row block
    int row0;      // first B row (sorted position or token) of the tile
    int nvalid;    // valid token columns
    int ntt;       // token tiles that share this tile's weight block (of its group)
};

// Tile tables of the (at most one) grouped problem, copied to shared memory at start.
struct GroupTables {
    int ts[kMaxGroups + 1];   // tile_start
    int off[kMaxGroups + 1];  // offsets
};

__device__ __forceinline__ int problem_tiles(const TcProblem& p, const GroupTables& g) {
    if (p.grouped) return g.ts[p.num_groups] * p.m_blocks;
    return p.n_tiles * p.m_blocks;
}

__device__ __forceinline__ TileInfo decode_tile(const TcParams& P, const GroupTables& gt, int tile, int t0) {
    TileInfo ti;
    int local = tile;
    ti.prob = 0;
    if (P.nprob > 1 && tile >= t0) {
        ti.prob = 1;
        local = tile - t0;
    }
    const TcProblem& p = P.p[ti.prob];
    if (!p.grouped) {
        // dense: bands of `band` token tiles, every weight-row block of a token tile in turn,
        // so that the tiles running at the same time share a few token tiles and every weight
        // block (each read about once per band from HBM, the rest from L2)
        ti.group = 0;
        int nb;
        if (p.band > 0) {
            const int bsz = p.band * p.m_blocks;
            const int band = local / bsz, within = local - band * bsz;
            nb = band * p.band + within / p.m_blocks;
            ti.mb = within - (within / p.m_blocks) * p.m_blocks;
        } else {
            ti.mb = local / p.n_tiles;
            nb = local - ti.mb * p.n_tiles;
        }
        ti.row0 = nb * p.bn;
        ti.nvalid = min(p.bn, p.rows - ti.row0);
        ti.ntt = p.n_tiles;
        return ti;
    }
    // largest e with tile_start[e] * m_blocks <= local (that expert is non-empty)
    int lo = 0, hi = p.num_groups - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (gt.ts[mid] * p.m_blocks <= local) lo = mid;
        else hi = mid - 1;
    }
    const int e = lo;
    const int ts = gt.ts[e];
    const int nbe = gt.ts[e + 1] - ts;
    const int l = local - ts * p.m_blocks;
    ti.group = e;
    ti.mb = l / nbe;
    const int nb = l - ti.mb * nbe;
    const int off = gt.off[e];
    const int cnt = gt.off[e + 1] - off;
    ti.row0 = off + nb * p.bn;
    ti.nvalid = min(p.bn, cnt - nb * p.bn);
    ti.ntt = nbe;
    return ti;
}

// Every tile carries two 128-row weight operands that share one token tile: the gate and
// up rows of 128 intermediate units (gate/up), or 256 consecutive output rows (others).
// bf16 weights: STAGES stages of [A0 | A1 | B]. 4-bit weights: STAGES load slots of
// [packed 0 | packed 1 | B] (TMA), then ASTAGES operand slots of [A0 | A1] (dequantised).
// PAIR: a cluster of two CTAs shares each 256-token tile: CTA r holds token rows
// 128 r .. 128 r + 127 and weight tile r (the gate or the up rows, or output rows
// 128 r .. 128 r + 127), and the leader's M = 256, N = 256 MMAs read both CTAs' operands.
template <bool GATEUP, int BN, int STAGES, bool Q4 = false, bool PAIR = false>
struct TcShape {
    static constexpr int A_BYTES = kBM * kBK * 2;                // 16 KB: one 128-row weight tile
    static constexpr int B_BYTES = (PAIR ? kBM : BN) * kBK * 2;  // this CTA's token tile
    static constexpr int ASTAGES = Q4 ? 2 : 0;                   // dequantised operand slots
    static constexpr int NA = PAIR ? 1 : 2;                      // weight tiles per CTA and stage
    static constexpr int B_OFF = Q4 ? 2 * kPkBytes : NA * A_BYTES;  // token tile within a stage
    static constexpr int STAGE_BYTES = Q4 ? 2 * kPkBytes + B_BYTES : NA * A_BYTES + B_BYTES;
    static constexpr int ARING_OFF = STAGES * STAGE_BYTES;       // operand ring (4-bit only)
    static constexpr int RING_BYTES = STAGES * STAGE_BYTES + ASTAGES * 2 * A_BYTES;
    // epilogue warps: 8, or 4 beside the dequantising warps, which keeps the 4-bit block at
    // 14 warps, at most 4 per SM sub-partition and so 128 registers per thread
    static constexpr int EPI = Q4 ? 128 : kEpiThreads;
    static constexpr int DQ_BASE = 64 + EPI;                     // first dequantising thread
    static constexpr int THREADS = 64 + EPI + (Q4 ? kDqThreads : 0);
    // TMEM: one 128 x 256 fp32 accumulator per 128 token rows of a tile; 128-row tiles keep
    // two accumulator sets (the epilogue of one tile overlaps the next tile's main loop),
    // 256-row tiles one set of two (512 columns either way)
    static constexpr int MH = PAIR ? 1 : BN / kBM;               // 128-row token halves per CTA tile
    static constexpr int NBUF = MH == 1 ? 2 : 1;                 // accumulator sets
    static constexpr int ACC_COLS = 2 * kBM;                     // columns of one accumulator
    static constexpr int TMEM_COLS = ACC_COLS * MH * NBUF;
    static constexpr int ROWS = GATEUP ? kBM : 2 * kBM;          // weight rows per tile
    // epilogue layout: the warps of each token half cover its 128 rows (lane quarters) and
    // the 256 columns in NH column halves each
    static constexpr int EPI_WARPS_PER_HALF = EPI / 32 / MH;
    static constexpr int NH = EPI_WARPS_PER_HALF == 4 ? 2 : 1;
    static constexpr int BIAS_BYTES = (EPI / 32) * 128 * NH * 4;
    static constexpr int SMEM = RING_BYTES + 1024 /*align*/ + 256 /*barriers*/ + int(sizeof(GroupTables)) + BIAS_BYTES;
    static_assert(TMEM_COLS == 512, "TMEM columns");
    static_assert(BN == 128 || (BN == 256 && !Q4), "token tile");
    static_assert(!PAIR || (BN == 256 && !Q4), "CTA pairs: bf16, 256-token tiles");
    static_assert(EPI_WARPS_PER_HALF == 4 || EPI_WARPS_PER_HALF == 8, "epilogue warps");
    static_assert(STAGE_BYTES % 1024 == 0 && B_OFF % 1024 == 0, "swizzle atoms stay 1 KB aligned");
    static_assert((2 * STAGES + 5 + 2 * ASTAGES) * 8 + 4 <= 256, "barriers fit their region");
    static_assert(SMEM <= 232448, "dynamic shared memory per block");
};

// SwiGLU / clamped SwiGLU with the fast exponential (the result is rounded to bf16).
__device__ __forceinline__ float act_fast(int act, float g, float v, float limit, float alpha) {
    if (act == MOE_ACT_SWIGLU) return __fdividef(g, 1.0f + __expf(-g)) * v;
    const float gc = fminf(g, limit);
    const float vc = fminf(fmaxf(v, -limit), limit);
    return __fdividef(gc, 1.0f + __expf(-alpha * gc)) * (vc + 1.0f);
}

// Fire-and-forget add of four consecutive fp32 values in global memory (16-byte aligned).
// The routed sums are the target of every slot's reduction, spread over the whole launch:
// they carry an L2 evict-last hint so that the streamed weights and token rows do not push
// them out between the reductions of their token's slots.
__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d, uint64_t pol) {
    asm volatile("red.global.add.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p), "f"(a), "f"(b), "f"(c),
                 "f"(d), "l"(pol)
                 : "memory");
}

__device__ __forceinline__ float bf16_at(const void* p, int64_t i) {
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
}

// Eight 4-bit codes (element j in bits 4j..4j+3 of the word) -> eight fp16 weights
// w = s * q + b, one rounding each. A code q becomes the exact fp16 1024 + q by OR-ing it into
// the mantissa of 1024.0 (two codes per 32-bit pair: the pair (q_i, q_i+4) comes from the same
// nibble position of both halves), PRMT puts neighbours together, and q = (1024 + q) - 1024 is
// exact before the single-rounding fma.
__device__ __forceinline__ uint4 dequant8_f16(uint32_t w, __half2 s2, __half2 b2) {
    const uint32_t p0 = (w & 0x000F000Fu) | 0x64006400u;          // (q0, q4)
    const uint32_t p1 = ((w >> 4) & 0x000F000Fu) | 0x64006400u;   // (q1, q5)
    const uint32_t p2 = ((w >> 8) & 0x000F000Fu) | 0x64006400u;   // (q2, q6)
    const uint32_t p3 = ((w >> 12) & 0x000F000Fu) | 0x64006400u;  // (q3, q7)
    const uint32_t o[4] = {__byte_perm(p0, p1, 0x5410), __byte_perm(p2, p3, 0x5410),
                           __byte_perm(p0, p1, 0x7632), __byte_perm(p2, p3, 0x7632)};
    const __half2 off = __floats2half2_rn(1024.0f, 1024.0f);
    uint32_t r[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __half2 q = __hsub2(*reinterpret_cast<const __half2*>(&o[i]), off);
        const __half2 v = __hfma2(q, s2, b2);
        r[i] = *reinterpret_cast<const uint32_t*>(&v);
    }
    return make_uint4(r[0], r[1], r[2], r[3]);
}

// Eight MXFP4 codes (OCP MX v1.0 E2M1, element j in bits 4j..4j+3) -> eight bf16 weights
// element * 2^(block scale). A code's exponent and mantissa bits placed at the bottom of a
// bf16 exponent field give exactly the element times 2^-126 (subnormal at exponent 0, as in
// the format); two exact power-of-two multiplies (2^126, then the block scale) finish.
__device__ __forceinline__ uint4 dequant8_mx(uint32_t w, __nv_bfloat162 scale2) {
    uint32_t p[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {  // (code_i, code_i+4) as bf16 bit patterns
        const uint32_t c = (w >> (4 * i)) & 0x000F000Fu;
        p[i] = ((c & 0x00080008u) << 12) | ((c & 0x00070007u) << 6);
    }
    const uint32_t o[4] = {__byte_perm(p[0], p[1], 0x5410), __byte_perm(p[2], p[3], 0x5410),
                           __byte_perm(p[0], p[1], 0x7632), __byte_perm(p[2], p[3], 0x7632)};
    const __nv_bfloat162 two126 = __halves2bfloat162(__ushort_as_bfloat16(0x7E80), __ushort_as_bfloat16(0x7E80));
    uint32_t r[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 v = __hmul2(__hmul2(*reinterpret_cast<const __nv_bfloat162*>(&o[i]), two126), scale2);
        r[i] = *reinterpret_cast<const uint32_t*>(&v);
    }
    return make_uint4(r[0], r[1], r[2], r[3]);
}

// Byte offset of row r's 16-byte chunk c (8 bf16 of one 64-wide K block) in a 128-row
// operand tile with the 128-byte swizzle the MMA descriptor expects (8-row atoms of 1 KB,
// chunk index XOR row within the atom).
__device__ __forceinline__ uint32_t sw128_offset(int r, int c) {
    return uint32_t((r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4));
}

// The two bf16 weight tiles of K block kc of a tile, by TMA, completing on `bar`.
template <bool GATEUP>
__device__ __forceinline__ void load_a_bf16(uint8_t* dst, const TcParams& P, const TileInfo& ti, int mrow, int kc,
                                            uint64_t* bar, uint64_t pol) {
    constexpr int A_BYTES = kBM * kBK * 2;
    if (!GATEUP) {  // rows [mrow, mrow + 128) and [mrow + 128, mrow + 256)
        tma_3d(dst, &P.a0[ti.prob], bar, kc, mrow, ti.group, pol);
        tma_3d(dst + A_BYTES, &P.a0[ti.prob], bar, kc, mrow + kBM, ti.group, pol);
    } else if (P.p[ti.prob].interleaved) {  // [E, I, 2, K]: plane 0 = gate rows, 1 = up rows
        tma_4d(dst, &P.a0[ti.prob], bar, kc, 0, mrow, ti.group, pol);
        tma_4d(dst + A_BYTES, &P.a0[ti.prob], bar, kc, 1, mrow, ti.group, pol);
    } else {
        tma_3d(dst, &P.a0[ti.prob], bar, kc, mrow, ti.group, pol);
        tma_3d(dst + A_BYTES, &P.a1[ti.prob], bar, kc, mrow, ti.group, pol);
    }
}

// CTA pair: this CTA's one weight tile of K block kc (rank 0: gate rows or output rows
// [mrow, mrow + 128); rank 1: up rows or [mrow + 128, mrow + 256)), completing on the
// leader's barrier at cluster address bar.
template <bool GATEUP>
__device__ __forceinline__ void load_a_pair(uint8_t* dst, const TcParams& P, const TileInfo& ti, int mrow, int kc,
                                            uint32_t rank, uint32_t bar, uint64_t pol) {
    if (!GATEUP) tma_3d_pair(dst, &P.a0[ti.prob], bar, kc, mrow + kBM * int(rank), ti.group, pol);
    else if (P.p[ti.prob].interleaved) tma_4d_pair(dst, &P.a0[ti.prob], bar, kc, int(rank), mrow, ti.group, pol);
    else tma_3d_pair(dst, rank ? &P.a1[ti.prob] : &P.a0[ti.prob], bar, kc, mrow, ti.group, pol);
}

template <bool GATEUP, int BN, int STAGES, bool Q4, bool PAIR>
__global__ void __launch_bounds__(TcShape<GATEUP, BN, STAGES, Q4, PAIR>::THREADS, 1)
    tc_gemm_kernel(const __grid_constant__ TcParams P) {
    using S = TcShape<GATEUP, BN, STAGES, Q4, PAIR>;
    constexpr int AS = S::ASTAGES > 0 ? S::ASTAGES : 1;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::RING_BYTES);
    uint64_t* empty = full + STAGES;
    uint64_t* acc_full = empty + STAGES;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* drain = acc_empty + 2;
    uint64_t* dq = drain + 1;       // 4-bit: operand slot filled (dequantised or loaded)
    uint64_t* aempty = dq + AS;     // 4-bit: operand slot consumed by the MMA
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(aempty + AS);
    GroupTables& gt = *reinterpret_cast<GroupTables*>(smem + S::RING_BYTES + 256);
    float* sbias = reinterpret_cast<float*>(&gt + 1);  // epilogue: 128 column biases per warp

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // CTA pairs: rank in the pair (0 = leader: issues the MMAs, owns the full / acc_empty
    // barriers) and the pair's tile stride; single CTAs: rank 0, one tile per CTA
    const uint32_t crank = PAIR ? cluster_rank() : 0u;
    const int tile0 = PAIR ? int(blockIdx.x >> 1) : int(blockIdx.x);
    const int tstep = PAIR ? int(gridDim.x >> 1) : int(gridDim.x);
    if (warp == 0) {
        if constexpr (PAIR) {
            asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(tmem_slot)),
                         "r"(uint32_t(S::TMEM_COLS)));
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
        } else {
            asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(tmem_slot)),
                         "r"(uint32_t(S::TMEM_COLS)));
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
        }
    }
    if (warp == 1 && lane == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], (PAIR ? 2 : 1) * S::EPI / 32);  // one arrive per epilogue warp (of the pair)
        }
        mbar_init(drain, 1);
        if (Q4)
            for (int st = 0; st < S::ASTAGES; ++st) {
                mbar_init(&dq[st], kDqThreads / 32);  // one arrive per dequantising warp
                mbar_init(&aempty[st], 1);            // one MMA commit
            }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 2 && lane == 0) {
        for (int i = 0; i < P.nprob; ++i) {
            prefetch_tmap(&P.a0[i]);
            if (GATEUP && !P.p[i].interleaved) prefetch_tmap(&P.a1[i]);
            for (int v = 0; v < 5; ++v) prefetch_tmap(&P.b[i][v]);
        }
    }
    pdl_begin();  // everything above touches no memory that earlier kernels write
    for (int i = 0; i < P.nprob; ++i) {
        if (!P.p[i].grouped) continue;
        for (int e = threadIdx.x; e <= P.p[i].num_groups; e += blockDim.x) {
            gt.ts[e] = P.p[i].tile_start[e];
            gt.off[e] = P.p[i].offsets[e];
        }
    }
    tc_fence_before();
    __syncthreads();
    if constexpr (PAIR) cluster_sync();  // the peer's barriers are initialised before any remote use
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int t0 = problem_tiles(P.p[0], gt);
    const int total = t0 + (P.nprob > 1 ? problem_tiles(P.p[1], gt) : 0);
    const uint64_t deadline = gtimer() + kWaitNs;
    bool timed_out = false;

    if (warp == 0) {
        // -------------------------------------------------------------- TMA producer (one warp)
        // bf16: both weight tiles + the token tile of each K block into one stage.
        // 4-bit: the two packed tiles + the token tile into one load slot (the
        // dequantising warps bring bf16 tiles into the operand ring themselves).
        // Lane 0 waits for the slot, arms its barrier and issues the loads.
        uint32_t stage = 0, phase = 0;
        uint32_t armed = 0;  // bit s: stage s was filled at least once
        uint32_t last_par = 0;
        const uint64_t pol_w = policy_evict_first(), pol_n = policy_evict_normal(), pol_t = policy_evict_last();
        for (int tile = tile0; tile < total && !timed_out; tile += tstep) {
            const TileInfo ti = decode_tile(P, gt, tile, t0);
            const uint64_t pw = ti.ntt > 1 ? pol_n : pol_w;  // weights shared by several token tiles
            // token rows: a dense batch is re-read by every weight-row block (kept); routed rows
            // are re-read only by their expert's blocks, which run at about the same time
            const TcProblem& p = P.p[ti.prob];
            const uint64_t pt = p.grouped ? pol_n : pol_t;
            const int nk = p.K / kBK;
            const int mrow = ti.mb * S::ROWS;
            // token rows: the smallest box (16, 32, 64, 128, 256 rows) that holds the valid tokens
            // (CTA pairs: of this CTA's 128-row half; the leader's barrier counts both halves)
            auto box_of = [](int nv) { return nv <= 16 ? 0 : nv <= 32 ? 1 : nv <= 64 ? 2 : nv <= 128 ? 3 : 4; };
            auto half_nv = [&](uint32_t r) { return max(0, min(kBM, ti.nvalid - kBM * int(r))); };
            const int bv = box_of(PAIR ? half_nv(crank) : ti.nvalid);
            const uint32_t b_bytes = uint32_t(min(BN, 16 << bv)) * kBK * 2;
            const uint32_t pair_tx = PAIR ? 2u * S::A_BYTES + (uint32_t(16 << box_of(half_nv(0))) +
                                                               uint32_t(16 << box_of(half_nv(1)))) * kBK * 2
                                          : 0u;
            for (int kb = 0; kb < nk; ++kb) {
                int ok = 1;
                if (lane == 0) ok = mbar_wait(&empty[stage], phase ^ 1u, deadline) ? 1 : 0;
                if (!__shfl_sync(0xffffffffu, ok, 0)) {
                    timed_out = true;
                    break;
                }
                uint8_t* sb = smem + stage * S::STAGE_BYTES;
                const int kc = kb * kBK;
                if (lane == 0) {
                    if constexpr (Q4) {
                        if (p.q4) {  // packed words of the two weight tiles (8 words per K block)
                            mbar_expect_tx(&full[stage], 2 * kPkBytes + b_bytes);
                            tma_3d(sb, &P.a0[ti.prob], &full[stage], kb * 8, mrow, ti.group, pw);
                            if (!GATEUP)
                                tma_3d(sb + kPkBytes, &P.a0[ti.prob], &full[stage], kb * 8, mrow + kBM, ti.group, pw);
                            else
                                tma_3d(sb + kPkBytes, &P.a1[ti.prob], &full[stage], kb * 8, mrow, ti.group, pw);
                        } else {
                            mbar_expect_tx(&full[stage], b_bytes);
                        }
                    } else if constexpr (PAIR) {
                        // this CTA's weight tile and token half; the bytes complete on the
                        // leader's barrier, which the leader arms with the pair's total
                        const uint32_t fb = mapa_shared(&full[stage], 0);
                        if (crank == 0) mbar_expect_tx(&full[stage], pair_tx);
                        load_a_pair<GATEUP>(sb, P, ti, mrow, kc, crank, fb, pw);
                        tma_2d_pair(sb + S::B_OFF, &P.b[ti.prob][bv], fb, kc, ti.row0 + kBM * int(crank), pt);
                    } else {
                        mbar_expect_tx(&full[stage], 2 * S::A_BYTES + b_bytes);
                        load_a_bf16<GATEUP>(sb, P, ti, mrow, kc, &full[stage], pw);
                    }
                    if constexpr (!PAIR) tma_2d(sb + S::B_OFF, &P.b[ti.prob][bv], &full[stage], kc, ti.row0, pt);
                }
                armed |= 1u << stage;
                last_par = (last_par & ~(1u << stage)) | (phase << stage);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        // drain: every copy this warp issued has landed before the CTA can exit (CTA pairs:
        // the leader's MMA has consumed it, which it does only once both halves landed)
        if (lane == 0) {
            const uint64_t dl2 = gtimer() + kWaitNs;
            for (int s = 0; s < STAGES; ++s)
                if ((armed >> s) & 1u) mbar_wait(PAIR ? &empty[s] : &full[s], (last_par >> s) & 1u, dl2);
            if (timed_out) set_status(P.status, MOE_ERR_DEVICE_TIMEOUT);
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0 && crank == 0) {
            // ---------------------------------------------------------- MMA issuer (pairs: the leader's)
            uint32_t stage = 0, phase = 0, it = 0;
            uint32_t astage = 0, aphase = 0;
            // M = 128 token rows, N = 256 weight rows; fp16 operands for 4-bit affine weights
            constexpr uint32_t idesc_b = idesc_bf16(2 * kBM), idesc_h = idesc_f16(2 * kBM);
            for (int tile = tile0; tile < total && !timed_out; tile += tstep, ++it) {
                const TileInfo ti = decode_tile(P, gt, tile, t0);
                const TcProblem& p = P.p[ti.prob];
                const uint32_t ab = it % S::NBUF, aph = (it / S::NBUF) & 1u;
                if (!mbar_wait(&acc_empty[ab], aph ^ 1u, deadline)) {
                    timed_out = true;
                    break;
                }
                tc_fence_after();
                const uint32_t d0 = tmem_base + ab * S::MH * S::ACC_COLS;
                const int nh = S::MH == 2 && ti.nvalid > kBM ? 2 : 1;  // token halves with valid rows
                const uint32_t idesc = PAIR ? idesc_bf16_pair() : (Q4 && p.q4 && !p.mx) ? idesc_h : idesc_b;
                const int nk = p.K / kBK;
                for (int kb = 0; kb < nk; ++kb) {
                    // 4-bit: the operand slot is complete once the dequantising warps have
                    // filled it, which they do only after the load slot (token tile) landed
                    if (!mbar_wait(Q4 ? &dq[astage] : &full[stage], Q4 ? aphase : phase, deadline)) {
                        timed_out = true;
                        break;
                    }
                    tc_fence_after();
                    // the two 128-row weight tiles lie back to back: one 256-row operand
                    const uint32_t sw = Q4 ? su32(smem + S::ARING_OFF + astage * 2 * S::A_BYTES)
                                           : su32(smem + stage * S::STAGE_BYTES);
                    const uint32_t st = su32(smem + stage * S::STAGE_BYTES + S::B_OFF);
#pragma unroll
                    for (int k = 0; k < kBK / 16; ++k) {
                        const uint32_t acc = (kb > 0 || k > 0) ? 1u : 0u;
                        if constexpr (PAIR) umma_pair(d0, smem_desc(st + k * 32), smem_desc(sw + k * 32), idesc, acc);
                        else umma(d0, smem_desc(st + k * 32), smem_desc(sw + k * 32), idesc, acc);
                        if (S::MH == 2 && nh == 2)  // token rows 128..255 (16 KB further), same weights
                            umma(d0 + S::ACC_COLS, smem_desc(st + kBM * 128 + k * 32), smem_desc(sw + k * 32), idesc, acc);
                    }
                    if constexpr (PAIR) umma_commit_pair(&empty[stage]);  // both CTAs' slots
                    else umma_commit(&empty[stage]);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                    if constexpr (Q4) {
                        umma_commit(&aempty[astage]);
                        if (++astage == uint32_t(S::ASTAGES)) {
                            astage = 0;
                            aphase ^= 1u;
                        }
                    }
                }
                if (timed_out) break;
                if constexpr (PAIR) umma_commit_pair(&acc_full[ab]);  // both CTAs' epilogues
                else umma_commit(&acc_full[ab]);
            }
            // drain: all MMAs issued by this thread have completed
            if constexpr (PAIR) umma_commit_pair(drain);
            else umma_commit(drain);
            mbar_wait(drain, 0, gtimer() + kWaitNs);
            if (timed_out) set_status(P.status, MOE_ERR_DEVICE_TIMEOUT);
        }
    } else if (Q4 && int(threadIdx.x) >= S::DQ_BASE) {
        // ---------------------------------------------------------- dequantisation warps
        // Thread d dequantises row d % 128 of weight tile (d / 128) % 2, part d / 256 of the
        // K block (kDqWords packed words: one 16-byte load from the load slot, kDqWords
        // swizzled 16-byte stores into the operand slot); a warp's threads share tile and
        // part. Its (scale, bias) pairs are loaded eight K blocks ahead. A bf16 tile in the
        // same launch (the shared expert) gets its operand slot filled by TMA, issued by the
        // first dequantising thread.
        constexpr int DT = kDqTiles;
        const int d = threadIdx.x - S::DQ_BASE;
        const int drow = d & (kBM - 1), a0 = (d / kBM) & 1, part = d / (2 * kBM);
        const bool leader = d == 0;
        uint32_t stage = 0, phase = 0;
        uint32_t astage = 0, aphase = 0;
        uint32_t a_armed = 0, a_last = 0;  // leader: operand slots it filled by TMA
        const uint64_t pol_w = policy_evict_first(), pol_n = policy_evict_normal();
        auto next = [&]() {
            if (++stage == STAGES) {
                stage = 0;
                phase ^= 1u;
            }
            if (++astage == uint32_t(S::ASTAGES)) {
                astage = 0;
                aphase ^= 1u;
            }
        };
        for (int tile = tile0; tile < total && !timed_out; tile += tstep) {
            const TileInfo ti = decode_tile(P, gt, tile, t0);
            const uint64_t pw = ti.ntt > 1 ? pol_n : pol_w;  // weights shared by several token tiles
            const TcProblem& p = P.p[ti.prob];
            const int nk = p.K / kBK;
            const int mrow = ti.mb * S::ROWS;
            if (!p.q4) {  // bf16 tile: the leader loads both weight tiles into the operand slot
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(&full[stage], phase, deadline) || !mbar_wait(&aempty[astage], aphase ^ 1u, deadline)) {
                        timed_out = true;
                        break;
                    }
                    __syncwarp();
                    if (leader) {
                        mbar_expect_tx(&dq[astage], 2 * S::A_BYTES);  // counts as this warp's arrive
                        load_a_bf16<GATEUP>(smem + S::ARING_OFF + astage * 2 * S::A_BYTES, P, ti, mrow, kb * kBK,
                                            &dq[astage], pw);
                        a_armed |= 1u << astage;
                        a_last = (a_last & ~(1u << astage)) | (aphase << astage);
                    } else if (lane == 0) {
                        mbar_arrive(&dq[astage]);
                    }
                    next();
                }
                continue;
            }
            const int ng = p.K / p.group_size;
            // this thread's row of each of its weight tiles in the scale / bias planes (rows
            // past M read row M - 1: their results are discarded); byte addresses: bf16 scales
            // and biases, or MXFP4's one-byte scales and no biases
            const unsigned char* sp[DT];
            const unsigned char* zp[DT];
#pragma unroll
            for (int ai = 0; ai < DT; ++ai) {
                const int a = a0 + ai;
                const int r = min(mrow + (GATEUP ? 0 : a * kBM) + drow, p.M - 1);
                const int64_t off = (int64_t(ti.group) * p.M + r) * p.qrow_step * ng;
                sp[ai] = static_cast<const unsigned char*>((GATEUP && a == 1) ? p.qs1 : p.qs0) + off * (p.mx ? 1 : 2);
                zp[ai] = p.mx ? nullptr : static_cast<const unsigned char*>((GATEUP && a == 1) ? p.qz1 : p.qz0) + off * 2;
            }
            // (scale, bias) of each tile for the two 32-wide halves of K block kb. The raw words
            // are loaded kPre blocks ahead into a register ring whose slots are indexed
            // statically (the K loop is unrolled kPre times), and converted only when their
            // block is dequantised, so that no instruction waits on a load issued since.
            // Group 32: one 32-bit word holds the two groups of the block (scales, then
            // biases; MXFP4: a 16-bit word of the two E8M0 bytes); larger groups: one 16-bit
            // value serves both halves.
            const bool two = p.group_size == 32;
            auto run = [&](auto mx_tag) {
            constexpr bool MX = decltype(mx_tag)::value;
            auto load_raw = [&](int kb, uint32_t (&rs)[DT], uint32_t (&rz)[DT]) {
                const int g = (kb * kBK) / p.group_size;
#pragma unroll
                for (int ai = 0; ai < DT; ++ai) {
                    if constexpr (MX) {
                        rs[ai] = __ldg(reinterpret_cast<const unsigned short*>(sp[ai] + g));
                        rz[ai] = 0;
                    } else if (two) {
                        rs[ai] = __ldg(reinterpret_cast<const unsigned int*>(sp[ai]) + g / 2);
                        rz[ai] = __ldg(reinterpret_cast<const unsigned int*>(zp[ai]) + g / 2);
                    } else {
                        rs[ai] = __ldg(reinterpret_cast<const unsigned short*>(sp[ai]) + g);
                        rz[ai] = __ldg(reinterpret_cast<const unsigned short*>(zp[ai]) + g);
                    }
                }
            };
            // raw words -> the pair used by the dequantisation of half h: (scale, bias) as an
            // fp16 pair in one 32-bit register, or MXFP4's 2^(byte - 127) twice as bf16
            auto convert = [&](const uint32_t (&rs)[DT], const uint32_t (&rz)[DT], __nv_bfloat162 (&o)[DT][2]) {
#pragma unroll
                for (int ai = 0; ai < DT; ++ai)
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        if constexpr (MX) {
                            const uint32_t sbyte = (rs[ai] >> (8 * h)) & 0xFFu;
                            const __nv_bfloat16 sc = __ushort_as_bfloat16(uint16_t(sbyte ? (sbyte << 7) : 0x0040u));
                            o[ai][h] = __halves2bfloat162(sc, sc);
                        } else {
                            const int sh = (two && h == 1) ? 16 : 0;
                            const __half2 sz = __floats2half2_rn(
                                __bfloat162float(__ushort_as_bfloat16(uint16_t(rs[ai] >> sh))),
                                __bfloat162float(__ushort_as_bfloat16(uint16_t(rz[ai] >> sh))));
                            o[ai][h] = *reinterpret_cast<const __nv_bfloat162*>(&sz);
                        }
                    }
            };
            constexpr int kPre = 8;
            uint32_t rs[kPre][DT], rz[kPre][DT];
#pragma unroll
            for (int j = 0; j < kPre; ++j)
                if (j < nk) load_raw(j, rs[j], rz[j]);
            for (int kb0 = 0; kb0 < nk && !timed_out; kb0 += kPre) {
#pragma unroll
            for (int j = 0; j < kPre; ++j) {
                const int kb = kb0 + j;
                if (kb >= nk) break;
                __nv_bfloat162 q0[DT][2];
                convert(rs[j], rz[j], q0);
                if (kb + kPre < nk) load_raw(kb + kPre, rs[j], rz[j]);  // this slot's next block
                if (!mbar_wait(&full[stage], phase, deadline) || !mbar_wait(&aempty[astage], aphase ^ 1u, deadline)) {
                    timed_out = true;
                    break;
                }
                // this slot's last use is no longer the leader's copy (the MMA consumed it
                // before the slot came free), so the exit drain must not wait on that phase
                if (leader) a_armed &= ~(1u << astage);
                const uint8_t* lb = smem + stage * S::STAGE_BYTES;
                uint8_t* ob = smem + S::ARING_OFF + astage * 2 * S::A_BYTES;
#pragma unroll
                for (int ai = 0; ai < DT; ++ai) {
                    const int a = a0 + ai;
                    static_assert(kDqWords == 4, "one 16-byte load of packed words per thread");
                    const uint4 w0 = *reinterpret_cast<const uint4*>(lb + a * kPkBytes + drow * 32 + part * 16);
                    const uint32_t words[4] = {w0.x, w0.y, w0.z, w0.w};
#pragma unroll
                    for (int j = 0; j < kDqWords; ++j) {
                        const int c = part * kDqWords + j;  // 16-byte chunk (8 K values) of the row
                        const __nv_bfloat162 sbv = q0[ai][c >> 2];
                        uint4 v;
                        if constexpr (MX) {
                            v = dequant8_mx(words[j], sbv);
                        } else {
                            const __half2 sz = *reinterpret_cast<const __half2*>(&sbv);
                            v = dequant8_f16(words[j], __low2half2(sz), __high2half2(sz));
                        }
                        *reinterpret_cast<uint4*>(ob + a * S::A_BYTES + sw128_offset(drow, c)) = v;
                    }
                }
                // generic-proxy writes, read next by the tensor cores (async proxy)
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(&dq[astage]);
                next();
            }
            }
            };
            if (p.mx) run(std::true_type{});
            else run(std::false_type{});
        }
        // drain: the operand loads the leader issued have landed before the CTA can exit
        // (only slots whose last use was such a load: a later 4-bit use of the slot moved its
        // barrier on, and waiting for the old parity would wait for a phase that never comes)
        if (leader) {
            const uint64_t dl2 = gtimer() + kWaitNs;
            for (int s = 0; s < S::ASTAGES; ++s)
                if ((a_armed >> s) & 1u) mbar_wait(&dq[s], (a_last >> s) & 1u, dl2);
        }
        if (timed_out) set_status(P.status, MOE_ERR_DEVICE_TIMEOUT);
    } else {
        // -------------------------------------------------------------- epilogue (256 threads)
        // Accumulator lane = token row of the tile, column = weight row. The two warps of a
        // TMEM lane quarter take one half each of the 256 columns; in gate/up mode a half is
        // 64 intermediate units, read from both the gate (columns 0..127) and the up
        // (columns 128..255) block. Each warp stages the biases of its own columns in a
        // warp-private slice of shared memory, so that no epilogue step waits on another warp.
        const int q = warp & 3;
        const int eid = threadIdx.x - 64;
        // TMEM columns per epilogue step: 16 beside the 4-bit kernel's 16 dequantising warps
        // (704 threads leave 80 registers per thread), 32 otherwise
        constexpr int CW = Q4 ? 16 : 32;
        const uint64_t pol_y = policy_evict_last();  // routed-sum reductions
        const int th = S::MH == 2 ? (eid >= 128 ? 1 : 0) : 0;  // token half of this warp
        const int tok = (PAIR ? int(crank) : th) * kBM + q * 32 + lane;  // token row of the tile
        constexpr int NH = S::NH;                               // column halves per warp
        const int h_lo = NH == 1 ? (eid >= 128 ? 1 : 0) : 0;
        float* sb = sbias + (eid >> 5) * 128 * NH;  // this warp's column biases (warp-private)
        uint32_t it = 0;
        for (int tile = tile0; tile < total; tile += tstep, ++it) {
            const TileInfo ti = decode_tile(P, gt, tile, t0);
            const TcProblem& p = P.p[ti.prob];
            const uint32_t ab = it % S::NBUF, aph = (it / S::NBUF) & 1u;
            const bool tv = tok < ti.nvalid;
            const int64_t prow = int64_t(ti.row0) + tok;
            float wslot = 0.f;
            float* yrow = nullptr;
            if (!GATEUP && p.mode == kEpiScatterAdd && tv) {  // this token row's slot, before the wait
                const int slot = p.sorted_slot[prow];
                wslot = p.topk_w[slot];
                yrow = reinterpret_cast<float*>(p.out) + int64_t(slot / p.k) * p.ld_out;
            }
            const bool has_bias = p.bias0 != nullptr;
            if (has_bias) {  // the biases of this warp's columns (128 per half), before the wait
                __syncwarp();  // every lane is done with the previous tile's values
#pragma unroll
                for (int hh = 0; hh < NH; ++hh) {
                    const int half = h_lo + hh;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int j = lane + 32 * i;
                        float b = 0.f;
                        if (GATEUP) {  // j < 64: gate bias of unit u0 + j, else up bias of unit u0 + j - 64
                            const int unit = ti.mb * kBM + half * 64 + (j & 63);
                            const int up = j >= 64 ? 1 : 0;
                            if (unit < p.M)
                                b = p.bias_interleaved ? bf16_at(p.bias0, (int64_t(ti.group) * p.M + unit) * 2 + up)
                                                       : bf16_at(up ? p.bias1 : p.bias0, int64_t(ti.group) * p.M + unit);
                        } else {
                            const int r = ti.mb * 2 * kBM + half * kBM + j;
                            if (r < p.M) b = bf16_at(p.bias0, int64_t(ti.group) * p.M + r);
                        }
                        sb[hh * 128 + j] = b;
                    }
                }
                __syncwarp();
            }
            // the accumulator is ready only after the tile's whole main loop: sleep in the wait
            // rather than take issue slots from the warps that feed the MMA
            if (!mbar_wait_sleep(&acc_full[ab], aph, deadline)) {
                set_status(P.status, MOE_ERR_DEVICE_TIMEOUT);
                break;
            }
            tc_fence_after();
            const uint32_t tb = tmem_base + (uint32_t(q * 32) << 16) + (ab * S::MH + th) * S::ACC_COLS;
            auto release = [&]() {  // the accumulator set is free for the tile after next
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if constexpr (PAIR) mbar_arrive_cluster(mapa_shared(&acc_empty[ab], 0));  // the leader's
                    else mbar_arrive(&acc_empty[ab]);
                }
            };
#pragma unroll 1
            for (int hh = 0; hh < NH; ++hh) {
                const int half = h_lo + hh;
                const bool last_half = hh == NH - 1;
                const float* sbh = sb + hh * 128;
                if constexpr (GATEUP) {
                    // CW units per chunk: gate and up of the same units -> CW values of h
                    const int u0 = ti.mb * kBM + half * 64;
#pragma unroll 1
                    for (int c = 0; c < 64 / CW; ++c) {
                        uint32_t g[CW], u[CW];
                        tmem_ld_issue(tb + half * 64 + CW * c, g);
                        tmem_ld_issue(tb + kBM + half * 64 + CW * c, u);
                        tmem_ld_wait(g);
                        tmem_ld_wait(u);
                        if (c == 64 / CW - 1 && last_half) release();
                        const int ub = u0 + CW * c;
                        if (!tv || ub >= p.M) continue;
                        const float* bg = sbh + CW * c;  // gate biases of these CW units
                        const float* bu = bg + 64;       // their up biases
                        uint32_t hp[CW / 2];
#pragma unroll
                        for (int j = 0; j < CW; j += 2) {
                            float gg0 = __uint_as_float(g[j]), gg1 = __uint_as_float(g[j + 1]);
                            float uu0 = __uint_as_float(u[j]), uu1 = __uint_as_float(u[j + 1]);
                            if (has_bias) {
                                gg0 += bg[j]; gg1 += bg[j + 1];
                                uu0 += bu[j]; uu1 += bu[j + 1];
                            }
                            const float a0 = act_fast(P.act, gg0, uu0, P.limit, P.alpha);
                            const float a1 = act_fast(P.act, gg1, uu1, P.limit, P.alpha);
                            if (p.out_f16) {
                                __half2 v2 = __floats2half2_rn(a0, a1);
                                hp[j / 2] = *reinterpret_cast<uint32_t*>(&v2);
                            } else {
                                __nv_bfloat162 v2 = __floats2bfloat162_rn(a0, a1);
                                hp[j / 2] = *reinterpret_cast<uint32_t*>(&v2);
                            }
                        }
                        uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.out) + prow * p.ld_out + ub);
#pragma unroll
                        for (int v = 0; v < CW / 8; ++v) dst[v] = make_uint4(hp[4 * v], hp[4 * v + 1], hp[4 * v + 2], hp[4 * v + 3]);
                    }
                } else {
                    // CW weight rows (output columns) per chunk; bf16 weights: the next chunk's TMEM
                    // load in flight while this one is stored; 4-bit weights: one at a time
                    const int rb = ti.mb * 2 * kBM + half * kBM;
                    constexpr int NB = Q4 ? 1 : 2;
                    constexpr int NC = kBM / CW;  // chunks per half
                    uint32_t v[NB][CW];
                    tmem_ld_issue(tb + half * kBM, v[0]);
#pragma unroll
                    for (int c = 0; c < NC; ++c) {
                        tmem_ld_wait(v[c % NB]);
                        if (NB == 2 && c < NC - 1) tmem_ld_issue(tb + half * kBM + CW * (c + 1), v[(c + 1) % NB]);
                        if (c == NC - 1 && last_half) release();
                        const int r0 = rb + CW * c;
                        float o[CW];
#pragma unroll
                        for (int j = 0; j < CW; ++j) o[j] = __uint_as_float(v[c % NB][j]);
                        if (NB == 1 && c < NC - 1) tmem_ld_issue(tb + half * kBM + CW * (c + 1), v[0]);
                        if (!tv || r0 >= p.M) continue;
                        if (has_bias) {
#pragma unroll
                            for (int j = 0; j < CW; ++j) o[j] += sbh[CW * c + j];
                        }
                        const bool whole = r0 + CW <= p.M;
                        if (p.mode == kEpiScatterAdd) {
                            // weighted combine into the token's fp32 routed sum, 16 bytes per
                            // reduction (libmir-metal execute: down weighted by routing.weights and
                            // summed per token); M is a multiple of 64 here
#pragma unroll
                            for (int j = 0; j < CW; j += 4)
                                red_add_v4(yrow + r0 + j, wslot * o[j], wslot * o[j + 1], wslot * o[j + 2], wslot * o[j + 3],
                                           pol_y);
                        } else if (p.mode == kEpiStoreF32) {
                            float* dst = reinterpret_cast<float*>(p.out) + prow * p.ld_out + r0;
                            if (whole) {
#pragma unroll
                                for (int j = 0; j < CW; j += 4)
                                    *reinterpret_cast<float4*>(dst + j) = make_float4(o[j], o[j + 1], o[j + 2], o[j + 3]);
                            } else {
#pragma unroll
                                for (int j = 0; j < CW; ++j)
                                    if (r0 + j < p.M) dst[j] = o[j];
                            }
                        } else {  // kEpiStoreAct (+ optional fp32 addend)
                            __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.out) + prow * p.ld_out + r0;
                            const float* ad = p.addend ? p.addend + prow * p.ld_add + r0 : nullptr;
                            if (whole) {
                                if (ad) {
#pragma unroll
                                    for (int j = 0; j < CW; j += 4) {
                                        const float4 a4 = __ldcs(reinterpret_cast<const float4*>(ad + j));
                                        o[j] += a4.x; o[j + 1] += a4.y; o[j + 2] += a4.z; o[j + 3] += a4.w;
                                    }
                                }
#pragma unroll
                                for (int w4 = 0; w4 < CW / 8; ++w4) {
                                    uint32_t hp[4];
#pragma unroll
                                    for (int j = 0; j < 4; ++j) {
                                        __nv_bfloat162 v2 = __floats2bfloat162_rn(o[8 * w4 + 2 * j], o[8 * w4 + 2 * j + 1]);
                                        hp[j] = *reinterpret_cast<uint32_t*>(&v2);
                                    }
                                    reinterpret_cast<uint4*>(dst)[w4] = make_uint4(hp[0], hp[1], hp[2], hp[3]);
                                }
                            } else {
#pragma unroll
                                for (int j = 0; j < CW; ++j)
                                    if (r0 + j < p.M) dst[j] = __float2bfloat16_rn(o[j] + (ad ? ad[j] : 0.f));
                            }
                        }
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    // CTA pairs: neither CTA leaves (nor frees its TMEM) while the other may still arrive on its
    // barriers or the leader's MMAs may read its operands
    if constexpr (PAIR) cluster_sync();
    if (warp == 0) {
        tc_fence_after();
        if constexpr (PAIR)
            asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                         "r"(uint32_t(S::TMEM_COLS)));
        else
            asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                         "r"(uint32_t(S::TMEM_COLS)));
    }
}

// ------------------------------------------------------------------ host side
using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn encode_fn() {
    static EncodeFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeFn>(p);
    });
    return fn;
}

bool encode(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
            const cuuint32_t* box, CUtensorMapDataType type = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
            CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
    EncodeFn fn = encode_fn();
    if (!fn) return false;
    cuuint32_t es[5] = {1, 1, 1, 1, 1};
    return fn(m, type, cuuint32_t(rank), const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() { return device_sm_count(); }

template <bool GATEUP, int BN, int STAGES, bool Q4, bool PAIR = false>
cudaError_t launch_tc_t(TcParams& P, int64_t max_tiles, cudaStream_t s) {
    using S = TcShape<GATEUP, BN, STAGES, Q4, PAIR>;
    auto kern = tc_gemm_kernel<GATEUP, BN, STAGES, Q4, PAIR>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM);
    if (err != cudaSuccess) return err;
    if constexpr (PAIR) {
        // clusters of two CTAs; as many pairs as can be resident at once (a GPC with an odd
        // number of free SMs holds one CTA fewer), each looping over the pair tiles
        cudaLaunchConfig_t cfg = {};
        cfg.blockDim = dim3(S::THREADS);
        cfg.dynamicSmemBytes = S::SMEM;
        cfg.stream = s;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
        cfg.attrs = attr;
        cfg.numAttrs = 2;
        cfg.gridDim = dim3(2 * (sm_count() / 2));
        int resident = 0;
        if ((err = cudaOccupancyMaxActiveClusters(&resident, kern, &cfg)) != cudaSuccess) return err;
        const int pairs = int(std::min<int64_t>(max_tiles, std::min(resident, sm_count() / 2)));
        if (pairs <= 0) return resident <= 0 ? cudaErrorInvalidConfiguration : cudaSuccess;
        cfg.gridDim = dim3(2 * pairs);
        if ((err = cudaLaunchKernelEx(&cfg, kern, P)) != cudaSuccess) return err;
        return cudaGetLastError();
    }
    const int grid = int(std::min<int64_t>(max_tiles, sm_count()));
    if (grid <= 0) return cudaSuccess;
    { const cudaError_t e_ = launch_pdl(kern, dim3(grid), dim3(S::THREADS), S::SMEM, s, P); if (e_ != cudaSuccess) return e_; }
    return cudaGetLastError();
}

}  // namespace

// Weight operand: [E, R, K] bf16 (E = 1 for a dense matrix), or the interleaved
// [E, 2R, K] gate_up plane viewed as [E, R, 2, K].
bool tc_weight_map(CUtensorMap* m, const void* w, int E, int R, int K, bool interleaved) {
    if (interleaved) {
        const cuuint64_t dims[4] = {cuuint64_t(K), 2, cuuint64_t(R), cuuint64_t(E)};
        const cuuint64_t strides[3] = {cuuint64_t(K) * 2, cuuint64_t(K) * 4, cuuint64_t(R) * K * 4};
        const cuuint32_t box[4] = {kBK, 1, kBM, 1};
        return encode(m, w, 4, dims, strides, box);
    }
    const cuuint64_t dims[3] = {cuuint64_t(K), cuuint64_t(R), cuuint64_t(E)};
    const cuuint64_t strides[2] = {cuuint64_t(K) * 2, cuuint64_t(R) * K * 2};
    const cuuint32_t box[3] = {kBK, kBM, 1};
    return encode(m, w, 3, dims, strides, box);
}

// Token operand: [rows, K] bf16, maps m[0..4] with boxes of 16, 32, 64, 128 and 256 rows
// (at most bn).
bool tc_token_map(CUtensorMap* m, const void* u, int64_t rows, int K, int bn) {
    const cuuint64_t dims[2] = {cuuint64_t(K), cuuint64_t(rows)};
    const cuuint64_t strides[1] = {cuuint64_t(K) * 2};
    for (int v = 0; v < 5; ++v) {
        const cuuint32_t box[2] = {kBK, cuuint32_t(std::min(bn, 16 << v))};
        if (!encode(&m[v], u, 2, dims, strides, box)) return false;
    }
    return true;
}

// Packed 4-bit plane [E, R, K / 8] uint32 (K % 64 == 0): box of 8 words x 128 rows. With
// row_step 2 the rows of one unit are every other row of an [E, 2R, K / 8] plane.
bool tc_q4_weight_map(CUtensorMap* m, const void* w, int E, int R, int K, int row_step) {
    const cuuint64_t dims[3] = {cuuint64_t(K / 8), cuuint64_t(R), cuuint64_t(E)};
    const cuuint64_t strides[2] = {cuuint64_t(K / 8) * 4 * row_step, cuuint64_t(R) * (K / 8) * 4 * row_step};
    const cuuint32_t box[3] = {8, kBM, 1};
    return encode(m, w, 3, dims, strides, box, CU_TENSOR_MAP_DATA_TYPE_UINT32, CU_TENSOR_MAP_SWIZZLE_NONE);
}

int device_sm_count() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

cudaError_t launch_tc_gemm(TcParams& P, bool gateup, int64_t max_tiles, cudaStream_t s) {
    bool q4 = false;
    for (int i = 0; i < P.nprob; ++i) q4 = q4 || P.p[i].q4;
    // the tile lists (dense tile counts, the permutation's tile prefix) were built for one
    // tile height, which picks the kernel: 128 rows with 4-bit weights or bf16, 256 with bf16
    const int bn = P.p[0].bn;
    bool grouped = false;
    for (int i = 0; i < P.nprob; ++i) grouped = grouped || P.p[i].grouped;
    // dense problems: as many token tiles per band as fill the resident CTAs (or pairs)
    // together with every weight-row block
    const int conc = (bn == kTcBNWide && !q4 && !grouped) ? sm_count() / 2 : sm_count();
    for (int i = 0; i < P.nprob; ++i)
        if (!P.p[i].grouped && P.p[i].m_blocks > 0)
            P.p[i].band = std::max(1, std::min(P.p[i].n_tiles, conc / P.p[i].m_blocks));
    for (int i = 0; i < P.nprob; ++i)
        if (P.p[i].bn != bn || (q4 && bn != kTcBN) || (bn != kTcBN && bn != kTcBNWide)) return cudaErrorInvalidValue;
    if (q4) {  // six load slots (packed tiles + token tile) feed two dequantised shared-memory operand slots
        if (gateup) return launch_tc_t<true, kTcBN, 6, true>(P, max_tiles, s);
        return launch_tc_t<false, kTcBN, 6, true>(P, max_tiles, s);
    }
    if (bn == kTcBNWide) {
        // Dense launches: CTA pairs (six 32 KB stages per CTA). A pair's M = 256 MMA computes
        // all 256 token rows of a tile, so in grouped launches, where the last tile of most
        // experts is partial, the one-CTA tile (which skips an empty second half) measured
        // faster: latent block at 8192 tokens, expert gate/up 2.64 ms one CTA vs 2.78 ms
        // pairs; with 512 routed rows per expert (every tile full) pairs win, 518 vs 570 us.
        if (!grouped) {
            if (gateup) return launch_tc_t<true, kTcBNWide, 6, false, true>(P, max_tiles, s);
            return launch_tc_t<false, kTcBNWide, 6, false, true>(P, max_tiles, s);
        }
        if (gateup) return launch_tc_t<true, kTcBNWide, 3, false>(P, max_tiles, s);  // three 64 KB stages
        return launch_tc_t<false, kTcBNWide, 3, false>(P, max_tiles, s);
    }
    // 128-token tiles, four 48 KB stages
    if (gateup) return launch_tc_t<true, kTcBN, 4, false>(P, max_tiles, s);
    return launch_tc_t<false, kTcBN, 4, false>(P, max_tiles, s);
}

}  // namespace moe
