// select.cuh -- CTA-wide exact top-k over keys held in shared memory.
//
// The ranking is "higher score first, equal scores to the lower block id".
// Scores are mapped to order-preserving uint32 keys (score_key), so the k-th
// largest key K* is found with an MSB-first radix select (four 8-bit
// digits), and the selection is
//     { i : key_i > K* }  U  { the first (k - #{key > K*}) positions with key == K* },
// emitted in ascending position order by an ordered stream compaction (warp
// ballots + a CTA prefix).  Because positions are scanned in increasing
// order, the output is sorted ascending, which is the layout the sparse
// attention consumes.
#pragma once

#include "common.cuh"

namespace qsa {

// Shared scratch of one select (lives in static smem of the calling kernel).
struct SelectSmem {
    uint32_t hist[256];
    uint32_t warp_a[32];
    uint32_t warp_b[32];
    uint32_t kstar;
    int32_t take_eq;
    int32_t run_out;
    int32_t run_eq;
};

// Finds K* and the number of keys equal to K* that are taken (k < n).
// Requires every thread of the CTA.  `nt` = blockDim.x (multiple of 32).
__device__ __forceinline__ void radix_kth(const uint32_t *keys, int n, int k, SelectSmem &sm) {
    const int tid = threadIdx.x, nt = blockDim.x;
    uint32_t prefix = 0, mask = 0;
    int k_rem = k;
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int i = tid; i < 256; i += nt) sm.hist[i] = 0;
        __syncthreads();
        for (int i = tid; i < n; i += nt) {
            const uint32_t key = keys[i];
            if ((key & mask) == prefix) atomicAdd(&sm.hist[(key >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (tid < 32) {
            const int lane = tid;
            uint32_t mine = 0;
#pragma unroll
            for (int b = 0; b < 8; ++b) mine += sm.hist[8 * lane + b];
            // exclusive suffix sum over lanes: counts in bins above this lane's range
            uint32_t incl = mine;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                uint32_t v = __shfl_down_sync(0xffffffffu, incl, o);
                if (lane + o < 32) incl += v;
            }
            uint32_t above = incl - mine;
            int found = -1;
            uint32_t cum = above;
            for (int b = 7; b >= 0; --b) {
                const uint32_t h = sm.hist[8 * lane + b];
                if (cum < (uint32_t)k_rem && cum + h >= (uint32_t)k_rem) { found = 8 * lane + b; break; }
                cum += h;
            }
            if (found >= 0) {
                sm.kstar = (uint32_t)found;
                sm.take_eq = k_rem - (int)cum;
            }
        }
        __syncthreads();
        prefix |= sm.kstar << shift;
        mask |= 255u << shift;
        k_rem = sm.take_eq;
        __syncthreads();
    }
    if (tid == 0) {
        sm.kstar = prefix;
        sm.take_eq = k_rem;
    }
    __syncthreads();
}

// Ordered compaction of the selection described by (sm.kstar, sm.take_eq):
// calls emit(out_pos, i) for every selected position i in increasing order of
// i.  With all_valid (n <= k) every position is selected.  Returns the count.
template <typename Emit>
__device__ __forceinline__ int ordered_select(const uint32_t *keys, int n, bool all_valid, SelectSmem &sm,
                                              Emit &&emit) {
    const int tid = threadIdx.x, nt = blockDim.x;
    const int lane = tid & 31, warp = tid >> 5, nwarps = nt >> 5;
    const uint32_t lt = (1u << lane) - 1u;
    const uint32_t kstar = sm.kstar;
    const int take_eq = sm.take_eq;
    if (tid == 0) { sm.run_out = 0; sm.run_eq = 0; }
    __syncthreads();
    for (int base = 0; base < n; base += nt) {
        const int i = base + tid;
        const bool valid = i < n;
        const uint32_t key = valid ? keys[i] : 0u;
        const bool gt = valid && (all_valid || key > kstar);
        const bool eq = valid && !all_valid && key == kstar;
        const uint32_t be = __ballot_sync(0xffffffffu, eq);
        if (lane == 0) sm.warp_a[warp] = __popc(be);
        __syncthreads();
        int eq_before = sm.run_eq;
        for (int w = 0; w < warp; ++w) eq_before += sm.warp_a[w];
        const int eq_rank = eq_before + __popc(be & lt);
        const bool sel = gt || (eq && eq_rank < take_eq);
        const uint32_t bs = __ballot_sync(0xffffffffu, sel);
        if (lane == 0) sm.warp_b[warp] = __popc(bs);
        __syncthreads();
        int out_before = sm.run_out;
        for (int w = 0; w < warp; ++w) out_before += sm.warp_b[w];
        if (sel) emit(out_before + __popc(bs & lt), i);
        __syncthreads();
        if (tid == 0) {
            int te = 0, ts = 0;
            for (int w = 0; w < nwarps; ++w) { te += sm.warp_a[w]; ts += sm.warp_b[w]; }
            sm.run_eq += te;
            sm.run_out += ts;
        }
        __syncthreads();
    }
    return sm.run_out;
}

// Full select: top-k of keys[0..n) -> emit(pos, i) in ascending i; returns the count.
template <typename Emit>
__device__ __forceinline__ int cta_topk(const uint32_t *keys, int n, int k, SelectSmem &sm, Emit &&emit) {
    const bool all = n <= k;
    if (!all) radix_kth(keys, n, k, sm);
    return ordered_select(keys, n, all, sm, emit);
}

}  // namespace qsa
