// permute_dev.cuh -- stable counting sort of slots by expert (a3), block-level routines.
//
// A stable counting sort of the T*k slots (slot s = t*k + j) by expert id: per-chunk
// histograms, an exclusive prefix over experts (and over earlier chunks of the same
// expert), then every slot's destination = its expert's base + the number of earlier
// slots of the same expert. Within a step of NT slots, ranks come from warp match masks
// plus per-warp counts in shared memory, so equal experts keep ascending slot order. Also
// emits the compact list of experts that received tokens and, when asked, the prefix of
// tensor-core token tiles per expert.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kPermE = 512;  // experts supported by the permutation routines

// Exclusive scan of vals[0..n) (n <= kPermE) in shared memory by an NT-thread block;
// returns the total. warp_tot holds NT/32 + 1 ints.
template <int NT>
__device__ int block_exclusive_scan(int* vals, int n, int* warp_tot) {
    constexpr int NW = NT / 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int per = (n + NT - 1) / NT;  // consecutive elements owned by each thread
    const int b = tid * per;
    int local = 0;
    for (int i = 0; i < per; ++i)
        if (b + i < n) local += vals[b + i];
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int wt = lane < NW ? warp_tot[lane] : 0;
        int wi = wt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += y;
        }
        if (lane < NW) warp_tot[lane] = wi - wt;  // exclusive warp offsets
        if (lane == NW - 1) warp_tot[NW] = wi;
    }
    __syncthreads();
    int run = incl - local + warp_tot[warp];
    for (int i = 0; i < per; ++i) {
        if (b + i < n) {
            const int v = vals[b + i];
            vals[b + i] = run;
            run += v;
        }
    }
    const int total = warp_tot[NW];
    __syncthreads();
    return total;
}

template <int NT>
struct PlaceSmem {
    int base[kPermE];
    int scan_buf[kPermE];
    int flag_buf[kPermE];
    int cnt[NT / 32][kPermE];
    int warp_tot[NT / 32 + 1];
};

// Places the slots of permutation chunk `chunk` (all of them when a.n_chunks == 1, in
// which case the chunk's own histogram is taken here). Chunk 0 also writes offsets, the
// active-expert list and (tile_bn > 0) the tile prefix. Every thread of the block calls it.
template <int NT>
__device__ void place_chunk(const PermuteArgs& a, int chunk, PlaceSmem<NT>& sm) {
    constexpr int NW = NT / 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int E = a.E;
    const int64_t s0 = int64_t(chunk) * a.chunk;
    const int64_t s1 = min(a.S, s0 + a.chunk);

    for (int i = tid; i < NW * kPermE; i += NT) (&sm.cnt[0][0])[i] = 0;
    if (a.n_chunks == 1) {
        for (int e = tid; e < E; e += NT) sm.scan_buf[e] = 0;
        __syncthreads();
        for (int64_t s = s0 + tid; s < s1; s += NT) {
            const int e = a.idx[s];
            if (e >= 0 && e < E) atomicAdd(&sm.scan_buf[e], 1);
            else set_status(a.status, MOE_ERR_DEVICE_CHECK);
        }
        __syncthreads();
        for (int e = tid; e < E; e += NT) sm.base[e] = 0;  // no earlier chunks
    } else {
        for (int e = tid; e < E; e += NT) {
            // this expert's counts of all chunks are contiguous (expert-major histograms)
            const int* hrow = a.chunk_hist + int64_t(e) * a.n_chunks;
            int tot = 0, pre = 0;
#pragma unroll 8
            for (int c = 0; c < a.n_chunks; ++c) {
                const int h = hrow[c];
                tot += h;
                pre += c < chunk ? h : 0;
            }
            sm.scan_buf[e] = tot;
            sm.base[e] = pre;
        }
    }
    __syncthreads();
    for (int e = tid; e < E; e += NT) sm.flag_buf[e] = sm.scan_buf[e] > 0 ? 1 : 0;
    if (chunk == 0 && a.tile_bn > 0) {
        // tensor-core tile prefix: tiles of expert e = ceil(count_e / tile_bn)
        for (int e = tid; e < E; e += NT) sm.cnt[0][e] = (sm.scan_buf[e] + a.tile_bn - 1) / a.tile_bn;
        __syncthreads();
        const int ntiles = block_exclusive_scan<NT>(&sm.cnt[0][0], E, sm.warp_tot);
        for (int e = tid; e < E; e += NT) a.tile_start[e] = sm.cnt[0][e];
        if (tid == 0) a.tile_start[E] = ntiles;
        for (int e = tid; e < E; e += NT) sm.cnt[0][e] = 0;
    }
    __syncthreads();
    const int total = block_exclusive_scan<NT>(sm.scan_buf, E, sm.warp_tot);
    const int n_active = block_exclusive_scan<NT>(sm.flag_buf, E, sm.warp_tot);
    if (chunk == 0) {
        for (int e = tid; e < E; e += NT) {
            a.offsets[e] = sm.scan_buf[e];
            const int next = (e + 1 < E) ? sm.flag_buf[e + 1] : n_active;
            if (next != sm.flag_buf[e]) a.active[1 + sm.flag_buf[e]] = e;
        }
        if (tid == 0) {
            a.offsets[E] = total;
            a.active[0] = n_active;
        }
    }
    for (int e = tid; e < E; e += NT) sm.base[e] += sm.scan_buf[e];
    __syncthreads();

    const unsigned lt_mask = (1u << lane) - 1u;
    for (int64_t step = s0; step < s1; step += NT) {
        const int64_t s = step + tid;
        int e = -1;
        if (s < s1) {
            e = a.idx[s];
            if (e < 0 || e >= E) {
                if (a.n_chunks > 1) set_status(a.status, MOE_ERR_DEVICE_CHECK);
                e = -1;
                a.slot_pos[s] = -1;
            }
        }
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const int rank = __popc(peers & lt_mask);
        const bool leader = (peers & lt_mask) == 0;
        if (e >= 0 && leader) sm.cnt[warp][e] = __popc(peers);
        __syncthreads();
        if (e >= 0) {
            int p = sm.base[e] + rank;
            for (int w = 0; w < warp; ++w) p += sm.cnt[w][e];
            a.sorted_slot[p] = int32_t(s);
            a.slot_pos[s] = p;
        }
        __syncthreads();
        if (e >= 0 && leader) {
            atomicAdd(&sm.base[e], __popc(peers));
            sm.cnt[warp][e] = 0;
        }
        __syncthreads();
    }
}

}  // namespace
}  // namespace moe
