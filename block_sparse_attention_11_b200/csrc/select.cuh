// select.cuh -- CTA-wide exact top-k over keys held in shared memory.
//
// The ranking is "higher score first, equal scores to the lower block id".
// Scores are mapped to order-preserving uint32 keys (score_key).  The k-th
// largest key K* is found by an MSB-first radix select:
//   1. an 11-bit histogram of the top digit (warp-aggregated atomics: equal
//      digits within a warp are merged with match_any, since scores pile up in
//      a few exponent bins);
//   2. the keys of the bin holding K* are gathered into a small candidate
//      list and the remaining 21 bits are resolved on that list only (two
//      more digits); if the bin is too large for the list, the two digits are
//      resolved on the full key array instead;
// and the selection
//     { i : key_i > K* }  U  { the first (k - #{key > K*}) positions with key == K* }
// is emitted in ascending position order by a two-phase ordered compaction:
// each warp owns a contiguous range, counts its "greater" and "equal" keys,
// and after one exclusive prefix over warps writes its survivors with ballot
// prefix sums.  Ascending output is the layout the sparse attention consumes.
#pragma once

#include "common.cuh"

namespace qsa {

constexpr int kSelCandCap = 1024;

struct SelectSmem {
    uint32_t hist[2048];
    uint32_t cand[kSelCandCap];
    uint32_t warp_gt[32];
    uint32_t warp_eq[32];
    uint32_t kstar;      // K*
    int32_t take_eq;     // how many keys equal to K* are taken (in position order)
    int32_t ncand;
    int32_t digit;
    int32_t k_rem;
    int32_t total;
};

// All threads scan hist[0..nbins) from the top and record the digit whose
// bin holds the k_rem-th largest key and the rank left inside that bin.
// Thread t owns bins [per*t, per*t + per); a suffix scan over threads (warp
// shuffles, then over warps) gives every thread the count above its range.
// Ends with a barrier; sm.digit / sm.k_rem are then valid for all threads.
__device__ __forceinline__ void sel_find_digit(SelectSmem &sm, int nbins, int k_rem) {
    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5, nwarps = nt >> 5;
    const int per = nbins / nt;   // nbins and nt are powers of two, nbins >= nt
    uint32_t mine = 0;
    for (int b = 0; b < per; ++b) mine += sm.hist[per * tid + b];
    uint32_t incl = mine;   // inclusive suffix within the warp (towards higher lanes)
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_down_sync(0xffffffffu, incl, o);
        if (lane + o < 32) incl += v;
    }
    if (lane == 0) sm.warp_eq[warp] = incl;   // warp total
    __syncthreads();
    // count in the warps above this one: lane l holds warp l's total (nwarps <= 32)
    const uint32_t wv = lane < nwarps ? sm.warp_eq[lane] : 0u;
    uint32_t cum = incl - mine + __reduce_add_sync(0xffffffffu, lane > warp ? wv : 0u);
    if (cum < (uint32_t)k_rem && cum + mine >= (uint32_t)k_rem) {
        for (int b = per - 1; b >= 0; --b) {
            const uint32_t h = sm.hist[per * tid + b];
            if (cum + h >= (uint32_t)k_rem) {
                sm.digit = per * tid + b;
                sm.k_rem = k_rem - (int)cum;
                break;
            }
            cum += h;
        }
    }
    __syncthreads();
}

// Histogram of digit (key >> shift) & mask over keys matching (key & pmask) == prefix.
__device__ __forceinline__ void sel_histogram(const uint32_t *keys, int n, int shift, uint32_t mask, uint32_t pmask,
                                              uint32_t prefix, SelectSmem &sm, bool aggregate) {
    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31;
    const int n_round = (n + 31) & ~31;
    for (int i = tid; i < n_round; i += nt) {
        const bool live = i < n;
        const uint32_t key = live ? keys[i] : 0u;
        const bool match = live && (key & pmask) == prefix;
        const uint32_t bin = match ? (key >> shift) & mask : 0xFFFFFFFFu;
        if (aggregate) {
            const uint32_t peers = __match_any_sync(0xffffffffu, bin);
            if (match && lane == __ffs(peers) - 1) atomicAdd(&sm.hist[bin], (uint32_t)__popc(peers));
        } else if (match) {
            atomicAdd(&sm.hist[bin], 1u);
        }
    }
}

// Finds K* and the number of keys equal to K* that are taken (requires k < n).
__device__ __forceinline__ void radix_kth(const uint32_t *keys, int n, int k, SelectSmem &sm) {
    const int tid = threadIdx.x, nt = blockDim.x;
    // ---- top 11 bits
    for (int i = tid; i < 2048; i += nt) sm.hist[i] = 0;
    if (tid == 0) sm.ncand = 0;
    __syncthreads();
    sel_histogram(keys, n, 21, 2047u, 0u, 0u, sm, true);
    __syncthreads();
    sel_find_digit(sm, 2048, k);
    uint32_t prefix = (uint32_t)sm.digit << 21;
    uint32_t pmask = 0xFFE00000u;
    int k_rem = sm.k_rem;
    // ---- gather the keys of that bin
    const int n_round = (n + 31) & ~31;
    for (int i = tid; i < n_round; i += nt) {
        const bool hit = i < n && (keys[i] & pmask) == prefix;
        const uint32_t bal = __ballot_sync(0xffffffffu, hit);
        int base = 0;
        if ((tid & 31) == 0 && bal) base = atomicAdd(&sm.ncand, __popc(bal));
        base = __shfl_sync(0xffffffffu, base, 0);
        if (hit) {
            const int slot = base + __popc(bal & ((1u << (tid & 31)) - 1u));
            if (slot < kSelCandCap) sm.cand[slot] = keys[i];
        }
    }
    __syncthreads();
    const int nc = sm.ncand;
    const bool small = nc <= kSelCandCap;
    const uint32_t *src = small ? sm.cand : keys;
    const int ns = small ? nc : n;
    // ---- bits 20..10, then 9..0
    const int shifts[2] = {10, 0};
    const uint32_t masks[2] = {2047u, 1023u};
    for (int pass = 0; pass < 2; ++pass) {
        const int nb = pass == 0 ? 2048 : 1024;
        for (int i = tid; i < nb; i += nt) sm.hist[i] = 0;
        __syncthreads();
        sel_histogram(src, ns, shifts[pass], masks[pass], pmask, prefix, sm, !small);
        __syncthreads();
        sel_find_digit(sm, nb, k_rem);
        prefix |= (uint32_t)sm.digit << shifts[pass];
        pmask |= masks[pass] << shifts[pass];
        k_rem = sm.k_rem;
        __syncthreads();
    }
    if (tid == 0) {
        sm.kstar = prefix;
        sm.take_eq = k_rem;
    }
    __syncthreads();
}

// Ordered compaction of the selection described by (sm.kstar, sm.take_eq):
// calls emit(out_pos, i) for every selected position i, in increasing i.
// With all_valid (n <= k) every position is selected.  Returns the count.
template <typename Emit>
__device__ __forceinline__ int ordered_select(const uint32_t *keys, int n, bool all_valid, SelectSmem &sm,
                                              Emit &&emit) {
    const int tid = threadIdx.x, nt = blockDim.x;
    const int lane = tid & 31, warp = tid >> 5, nwarps = nt >> 5;
    if (all_valid) {
        for (int i = tid; i < n; i += nt) emit(i, i);
        return n;
    }
    const uint32_t lt = (1u << lane) - 1u;
    const uint32_t kstar = sm.kstar;
    const int take_eq = sm.take_eq;
    const int per = (((n + nwarps - 1) / nwarps) + 31) & ~31;
    const int r0 = min(n, warp * per), r1 = min(n, r0 + per);
    uint32_t cgt = 0, ceq = 0;
    for (int b = r0; b < r1; b += 32) {
        const int i = b + lane;
        const uint32_t key = i < r1 ? keys[i] : 0u;
        cgt += __popc(__ballot_sync(0xffffffffu, i < r1 && key > kstar));
        ceq += __popc(__ballot_sync(0xffffffffu, i < r1 && key == kstar));
    }
    if (lane == 0) { sm.warp_gt[warp] = cgt; sm.warp_eq[warp] = ceq; }
    __syncthreads();
    // exclusive prefix over warps: outputs and equal keys before this warp's range
    int eq_before = 0, out_run = 0, total = 0, eq_run = 0;
    for (int w = 0; w < nwarps; ++w) {
        const int e = (int)sm.warp_eq[w];
        const int s = (int)sm.warp_gt[w] + max(0, min(e, take_eq - eq_before));
        if (w < warp) out_run += s;
        if (w == warp) eq_run = eq_before;
        total += s;
        eq_before += e;
    }
    for (int b = r0; b < r1; b += 32) {
        const int i = b + lane;
        const uint32_t key = i < r1 ? keys[i] : 0u;
        const bool gt = i < r1 && key > kstar;
        const bool eq = i < r1 && key == kstar;
        const uint32_t be = __ballot_sync(0xffffffffu, eq);
        const bool sel = gt || (eq && eq_run + __popc(be & lt) < take_eq);
        const uint32_t bs = __ballot_sync(0xffffffffu, sel);
        if (sel) emit(out_run + __popc(bs & lt), i);
        eq_run += __popc(be);
        out_run += __popc(bs);
    }
    __syncthreads();
    return total;
}

// Full select: top-k of keys[0..n) -> emit(pos, i) in ascending i; returns the count.
template <typename Emit>
__device__ __forceinline__ int cta_topk(const uint32_t *keys, int n, int k, SelectSmem &sm, Emit &&emit) {
    const bool all = n <= k;
    if (!all) radix_kth(keys, n, k, sm);
    return ordered_select(keys, n, all, sm, emit);
}

}  // namespace qsa

namespace qsa {

// ---------------------------------------------------------------------------
// Warp-per-row top-k over scores held in global memory (L2-resident rows).
//
// Same ranking and output as cta_topk, for one row per warp and no CTA
// barriers, so many rows are in flight per SM:
//   pass 1  11-bit histogram of the top digit (shared-memory atomics; two
//           16-bit counters per word for rows below 65536 elements, one
//           32-bit counter per bin for longer rows, kWide);
//   pass 2  the keys of the bin holding K* are gathered into a per-warp list
//           and the remaining 21 bits are resolved on it (if the bin overflows
//           the list, they are resolved on the row instead);
//   pass 3  ordered emission: lane l holds elements 4l..4l+3 of each 128-wide
//           chunk; warp prefix sums give output positions and equal-key ranks.
// ---------------------------------------------------------------------------
constexpr int kWarpSelBuf = 512;

// A bin of the narrow form counts to 65535: rows of fewer than 65536
// elements only; longer rows take kWide (2048 32-bit counters).
template <bool kWide>
struct WarpSelSmemT {
    uint32_t hist[kWide ? 2048 : 1024];
    uint32_t buf[kWarpSelBuf];    // keys of the threshold bin
};
using WarpSelSmem = WarpSelSmemT<false>;
constexpr int kWarpSelNarrowMax = 65535;   // longest row of the narrow form

template <bool kWide>
__device__ __forceinline__ uint32_t wsel_count(const WarpSelSmemT<kWide> &w, int bin) {
    if constexpr (kWide) return w.hist[bin];
    else return (w.hist[bin >> 1] >> (16 * (bin & 1))) & 0xFFFFu;
}

// Find the digit holding the k_rem-th largest among nbins (<= 2048) counters;
// returns digit and updates k_rem.  Lane l owns bins [l*per, l*per + per).
template <bool kWide>
__device__ __forceinline__ int wsel_find(const WarpSelSmemT<kWide> &w, int nbins, int &k_rem) {
    const int lane = threadIdx.x & 31;
    const int per = nbins / 32;
    // the lane's words are visited rotated by its lane index, so the 32 lanes
    // read 32 different banks (in order, all lanes would hit one bank)
    uint32_t mine = 0;
    if constexpr (kWide) {
        for (int j = 0; j < per; ++j) mine += w.hist[per * lane + ((j + lane) & (per - 1))];
    } else {
        const int pw = per / 2;                       // words per lane, two 16-bit counters each
        for (int j = 0; j < pw; ++j) {
            const uint32_t x = w.hist[pw * lane + ((j + lane) & (pw - 1))];
            mine += (x & 0xFFFFu) + (x >> 16);
        }
    }
    uint32_t incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_down_sync(0xffffffffu, incl, o);
        if (lane + o < 32) incl += v;
    }
    uint32_t cum = incl - mine;
    int digit = -1, rem = 0;
    if (cum < (uint32_t)k_rem && cum + mine >= (uint32_t)k_rem) {
        for (int b = per - 1; b >= 0; --b) {
            const uint32_t h = wsel_count(w, per * lane + b);
            if (cum + h >= (uint32_t)k_rem) { digit = per * lane + b; rem = k_rem - (int)cum; break; }
            cum += h;
        }
    }
    const uint32_t who = __ballot_sync(0xffffffffu, digit >= 0);
    const int src = __ffs(who) - 1;
    digit = __shfl_sync(0xffffffffu, digit, src);
    k_rem = __shfl_sync(0xffffffffu, rem, src);
    return digit;
}

template <bool kWide>
__device__ __forceinline__ void wsel_clear(WarpSelSmemT<kWide> &w, int nbins) {
    const int lane = threadIdx.x & 31;
    for (int i = lane; i < (kWide ? nbins : nbins / 2); i += 32) w.hist[i] = 0;
    __syncwarp();
}

// Plain shared-memory atomics: cheaper here than aggregating equal digits
// with match_any (measured on B200: 1.06 vs 1.43 ms for the 32K-token indexer).
template <bool kWide>
__device__ __forceinline__ void wsel_add(WarpSelSmemT<kWide> &w, bool live, uint32_t bin) {
    if constexpr (kWide) {
        if (live) atomicAdd(&w.hist[bin], 1u);
    } else {
        if (live) atomicAdd(&w.hist[bin >> 1], 1u << (16 * (bin & 1)));
    }
}

// Loads element chunk [base + 4*lane, +4) of the row as keys (invalid -> live=false).
__device__ __forceinline__ void wsel_load4(const float *row, int n, int base, uint32_t (&key)[4], bool (&live)[4]) {
    const int lane = threadIdx.x & 31;
    const int i = base + 4 * lane;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (i < n) v = *reinterpret_cast<const float4 *>(row + i);   // row stride keeps 16-byte alignment
    const float f[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        live[c] = i + c < n;
        key[c] = score_key(f[c]);
    }
}

// Four consecutive 128-element chunks [base + 128u, +128), u < 4: the four
// 16-byte loads are issued before any key is used, so each lane keeps four
// loads in flight (one at a time left the row passes latency-bound).
__device__ __forceinline__ void wsel_load4x4(const float *row, int n, int base, uint32_t (&key)[4][4],
                                             bool (&live)[4][4]) {
    const int lane = threadIdx.x & 31;
    float4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int i = base + 128 * u + 4 * lane;
        v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (i < n) v[u] = *reinterpret_cast<const float4 *>(row + i);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int i = base + 128 * u + 4 * lane;
        const float f[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            live[u][c] = i + c < n;
            key[u][c] = score_key(f[c]);
        }
    }
}

// Top-k of one row; emit(pos, i) in ascending i, pos < k.  Returns the count
// (min(n, k)).  Whole warp.  kWide is required for n > kWarpSelNarrowMax.
template <bool kWide, typename Emit>
__device__ __forceinline__ int warp_topk_row(const float *row, int n, int k, WarpSelSmemT<kWide> &w,
                                             Emit &&emit) {
    const int lane = threadIdx.x & 31;
    const uint32_t lt = (1u << lane) - 1u;
    if (n <= k) {
        for (int i = lane; i < n; i += 32) emit(i, i);
        return n;
    }
    // ---- pass 1: top 11 bits (full 512-element steps need no bounds checks)
    wsel_clear(w, 2048);
    const int n_full = n & ~511;
    for (int base = 0; base < n_full; base += 512) {
        float4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = *reinterpret_cast<const float4 *>(row + base + 128 * u + 4 * lane);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            wsel_add(w, true, score_key(v[u].x) >> 21);
            wsel_add(w, true, score_key(v[u].y) >> 21);
            wsel_add(w, true, score_key(v[u].z) >> 21);
            wsel_add(w, true, score_key(v[u].w) >> 21);
        }
    }
    if (n_full < n) {
        uint32_t key[4][4];
        bool live[4][4];
        wsel_load4x4(row, n, n_full, key, live);
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int c = 0; c < 4; ++c) wsel_add(w, live[u][c], key[u][c] >> 21);
    }
    __syncwarp();
    int k_rem = k;
    const uint32_t d1 = (uint32_t)wsel_find(w, 2048, k_rem);
    uint32_t prefix = d1 << 21, pmask = 0xFFE00000u;
    // ---- pass 2: gather the bin's keys (a multiset: order does not matter);
    // each lane's hits of a step as a 16-bit mask, one warp scan for the slots
    int cnt = 0;
    for (int base = 0; base < n; base += 512) {
        uint32_t key[4][4];
        bool live[4][4];
        wsel_load4x4(row, n, base, key, live);
        uint32_t hm = 0;
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int c = 0; c < 4; ++c) hm |= (uint32_t)(live[u][c] && (key[u][c] & pmask) == prefix) << (4 * u + c);
        const int mine = __popc(hm);
        int incl = mine;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        int slot = cnt + incl - mine;
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int c = 0; c < 4; ++c)
                if ((hm >> (4 * u + c)) & 1u) {
                    if (slot < kWarpSelBuf) w.buf[slot] = key[u][c];
                    ++slot;
                }
        cnt += __shfl_sync(0xffffffffu, incl, 31);
    }
    __syncwarp();
    const bool small = cnt <= kWarpSelBuf;
    const int shifts[2] = {10, 0};
    const uint32_t masks[2] = {2047u, 1023u};
    for (int pass = 0; pass < 2; ++pass) {
        const int nb = pass == 0 ? 2048 : 1024;
        wsel_clear(w, nb);
        if (small) {
            for (int i = lane; i < ((cnt + 31) & ~31); i += 32) {
                const bool live = i < cnt && (w.buf[i] & pmask) == prefix;
                const uint32_t key = i < cnt ? w.buf[i] : 0u;
                wsel_add(w, live, (key >> shifts[pass]) & masks[pass]);
            }
        } else {
            for (int base = 0; base < n; base += 128) {
                uint32_t key[4];
                bool live[4];
                wsel_load4(row, n, base, key, live);
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    wsel_add(w, live[c] && (key[c] & pmask) == prefix, (key[c] >> shifts[pass]) & masks[pass]);
            }
        }
        __syncwarp();
        const uint32_t d = (uint32_t)wsel_find(w, nb, k_rem);
        prefix |= d << shifts[pass];
        pmask |= masks[pass] << shifts[pass];
        __syncwarp();
    }
    const uint32_t kstar = prefix;
    const int take_eq = k_rem;
    // ---- pass 3: ordered emission
    int out_run = 0, eq_run = 0;
    for (int base4 = 0; base4 < n; base4 += 512) {
        uint32_t key4[4][4];
        bool live4[4][4];
        wsel_load4x4(row, n, base4, key4, live4);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int base = base4 + 128 * u;
            const uint32_t(&key)[4] = key4[u];
            const bool(&live)[4] = live4[u];
            // element order is (lane, c): ranks come from ballots, lanes below
            // plus this lane's earlier elements
            bool gt[4], eq[4];
            uint32_t be[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                gt[c] = live[c] && key[c] > kstar;
                eq[c] = live[c] && key[c] == kstar;
                be[c] = __ballot_sync(0xffffffffu, eq[c]);
            }
            int eq_before = eq_run;
#pragma unroll
            for (int c = 0; c < 4; ++c) eq_before += __popc(be[c] & lt);
            bool sel[4];
            uint32_t bs[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                sel[c] = gt[c] || (eq[c] && eq_before < take_eq);
                eq_before += eq[c];
                bs[c] = __ballot_sync(0xffffffffu, sel[c]);
            }
            int pos = out_run;
#pragma unroll
            for (int c = 0; c < 4; ++c) pos += __popc(bs[c] & lt);
#pragma unroll
            for (int c = 0; c < 4; ++c)
                if (sel[c]) {
                    if (pos < k) emit(pos, base + 4 * lane + c);   // exact counts give pos < k always
                    ++pos;
                }
            out_run += __popc(bs[0]) + __popc(bs[1]) + __popc(bs[2]) + __popc(bs[3]);
            eq_run += __popc(be[0]) + __popc(be[1]) + __popc(be[2]) + __popc(be[3]);
        }
    }
    return min(out_run, k);
}

}  // namespace qsa
