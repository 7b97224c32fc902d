// k_index.cu -- prefill indexer: block scores on the 5th-generation tensor
// cores (tcgen05, accumulators in TMEM, operands fed by TMA), an fp32 SIMT
// variant for the fp32 mode, and the per-row top-k select.
//
// Score (page "Qwen3.8-Flash-Next: Day-0 Support in SGLang", section "Qwen
// Sparse Attention: Retrieve Coarsely, Attend Precisely", score equation):
//     s_{t,b} = (1/sqrt(128)) * sum_h w_h * phi(<qhat_{t,h}, kbar_b>),  b < nb(t).
// The positive factor 1/sqrt(128) does not change the ranking and is not
// applied; only the ranking leaves this file.
//
// Two operand layouts:
//   * head-sum ("hi/lo"): with phi = identity and w = 1 the score is
//     <sum_h qhat_h, kbar_b>.  The FP32 head sum is split into two BF16 planes
//     hi + lo (16 significant bits, exact for BF16 heads of similar
//     magnitude), so one query row costs two K=128 MMAs instead of four and
//     the ranking keeps FP32 accuracy.  A tile is 128 query rows.
//   * per-head: rows are (query, head) pairs, 32 queries per 128-row tile;
//     the epilogue applies phi and w and sums the 4 heads across 4 lanes.
//
// Tile shape: M = 128 (TMEM lanes), N = 128 key blocks, K = 128 (two
// 64-element 128-byte-swizzled k-atoms).  The query tile is loaded once per
// CTA and stays in shared memory; key tiles stream through a 3-stage TMA
// ring; two TMEM accumulators (128 columns each) let the epilogue of tile j
// overlap the MMAs of tile j+1.  Warp roles: 0 = TMA producer, 1 = MMA issuer
// and TMEM owner, 2..9 = epilogue: two warps per TMEM lane quarter (warp w
// reads lanes 32*(w%4)..+31), one per half of the tile's 128 columns.
#include "internal.h"
#include "select.cuh"

namespace qsa {

namespace {

constexpr int GM = 128;
constexpr int GN = 128;
constexpr int NST = 3;
constexpr int KATOM_BYTES_A = GM * 128;            // 128 rows x 128 bytes
constexpr int KATOM_BYTES_B = GN * 128;
constexpr int A_BYTES = 2 * KATOM_BYTES_A;         // one operand plane, both k-atoms
constexpr int B_STAGE_BYTES = 2 * KATOM_BYTES_B;
constexpr int GEMM_EPI = 8;                        // epilogue warps
constexpr int GEMM_THREADS = (2 + GEMM_EPI) * 32;
constexpr int TMEM_COLS = 2 * GN;

struct GemmSmem {
    alignas(1024) uint8_t a0[A_BYTES];
    alignas(1024) uint8_t a1[A_BYTES];
    alignas(1024) uint8_t b[NST][B_STAGE_BYTES];
    alignas(8) uint64_t a_full;
    uint64_t b_full[NST];
    uint64_t b_empty[NST];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint32_t tmem_base;
    alignas(16) float epi[GEMM_EPI][32][36];   // per epilogue warp: 32 rows x 32 scores, transposed for stores
};

struct GemmParams {
    int64_t n_q, q0, row_begin, row_count, pool_stride, ld;
    int per_head, relu;
    const float *head_w;
    float *scores;
    unsigned *status;
    int nsplit;           // CTAs per row tile, each over `span` key tiles
    int span;
    uint16_t *keys;       // non-null: write the 16-bit order key of each score (ld per row) instead of scores
};

__global__ void __launch_bounds__(GEMM_THREADS, 1)
    score_gemm_kernel(const __grid_constant__ CUtensorMap map_a0, const __grid_constant__ CUtensorMap map_a1,
                      const __grid_constant__ CUtensorMap map_b, GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    GemmSmem &sm = *reinterpret_cast<GemmSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int seq = blockIdx.y;
    const int rows_per_tile = p.per_head ? GM / kIdxHeads : GM;
    // row tile m (heaviest, latest rows first), key tiles [j0, j0 + ntiles) of it
    const int m = (int)(gridDim.x / p.nsplit) - 1 - (int)(blockIdx.x / p.nsplit);
    const int j0 = (int)(blockIdx.x % p.nsplit) * p.span;
    const int64_t r0 = p.row_begin + (int64_t)m * rows_per_tile;
    const int64_t r_end = min(r0 + rows_per_tile, p.row_begin + p.row_count);
    const int64_t t_last = p.q0 + r_end - 1;
    const int64_t nb_tile = (t_last + 1) / kBlock;
    const int ntiles = max(0, min((int)((nb_tile + GN - 1) / GN) - j0, p.span));
    const int kplanes = p.per_head ? 1 : 2;

    if (threadIdx.x == 0) {
        mbar_init(&sm.a_full, 1);
        for (int s = 0; s < NST; ++s) { mbar_init(&sm.b_full[s], 1); mbar_init(&sm.b_empty[s], 1); }
        for (int s = 0; s < 2; ++s) { mbar_init(&sm.acc_full[s], 1); mbar_init(&sm.acc_empty[s], GEMM_EPI); }
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp == 0) {
        // ---------------- TMA producer
        if (lane == 0 && ntiles > 0) {
            prefetch_tmap(&map_a0);
            prefetch_tmap(&map_b);
            const int ay = p.per_head ? (int)((seq * p.n_q + r0) * kIdxHeads) : (int)(seq * p.n_q + r0);
            mbar_arrive_expect_tx(&sm.a_full, kplanes * A_BYTES);
            tma_load_2d(sm.a0, &map_a0, 0, ay, &sm.a_full);
            tma_load_2d(sm.a0 + KATOM_BYTES_A, &map_a0, 64, ay, &sm.a_full);
            if (!p.per_head) {
                tma_load_2d(sm.a1, &map_a1, 0, ay, &sm.a_full);
                tma_load_2d(sm.a1 + KATOM_BYTES_A, &map_a1, 64, ay, &sm.a_full);
            }
            bool ok = true;
            for (int j = 0; j < ntiles && ok; ++j) {
                const int s = j % NST;
                if (j >= NST) ok = mbar_wait(&sm.b_empty[s], ((j / NST) + 1) & 1, p.status);
                if (!ok) break;
                const int by = (int)(seq * p.pool_stride + (int64_t)(j0 + j) * GN);
                mbar_arrive_expect_tx(&sm.b_full[s], B_STAGE_BYTES);
                tma_load_2d(sm.b[s], &map_b, 0, by, &sm.b_full[s]);
                tma_load_2d(sm.b[s] + KATOM_BYTES_B, &map_b, 64, by, &sm.b_full[s]);
            }
            // make sure no copy is still landing in shared memory when the CTA ends
            mbar_wait(&sm.a_full, 0, p.status);
            for (int j = max(0, ntiles - NST); j < ntiles; ++j) mbar_wait(&sm.b_full[j % NST], (j / NST) & 1, p.status);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (one thread)
        if (lane == 0 && ntiles > 0) {
            const uint32_t idesc = idesc_bf16_f32(GM, GN);
            bool ok = mbar_wait(&sm.a_full, 0, p.status);
            tc_fence_after();
            const uint32_t a0 = smem_u32(sm.a0), a1 = smem_u32(sm.a1);
            for (int j = 0; j < ntiles && ok; ++j) {
                const int s = j % NST, ab = j & 1;
                if (j >= 2) ok = mbar_wait(&sm.acc_empty[ab], ((j >> 1) + 1) & 1, p.status);
                if (ok) ok = mbar_wait(&sm.b_full[s], (j / NST) & 1, p.status);
                if (!ok) break;
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(ab * GN);
                const uint32_t bs = smem_u32(sm.b[s]);
                uint32_t acc = 0;
                for (int pl = 0; pl < kplanes; ++pl) {
                    const uint32_t abase = pl ? a1 : a0;
#pragma unroll
                    for (int ka = 0; ka < 2; ++ka)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint64_t adesc = sw128_desc(abase + ka * KATOM_BYTES_A + kk * 32);
                            const uint64_t bdesc = sw128_desc(bs + ka * KATOM_BYTES_B + kk * 32);
                            tc_mma_f16(d, adesc, bdesc, idesc, acc);
                            acc = 1;
                        }
                }
                tc_commit(&sm.b_empty[s]);
                tc_commit(&sm.acc_full[ab]);
            }
        }
        __syncwarp();
    } else {
        // ---------------- epilogue: TMEM -> registers -> global scores
        const int quarter = warp & 3;
        const int ew = warp - 2;                // epilogue warp: staging buffer
        const int chalf = ew >> 2;              // columns [64 chalf, 64 chalf + 64) of each tile
        const int lrow = quarter * 32 + lane;   // TMEM lane = operand row in the tile
        int64_t qrow;                           // query row (within the sequence)
        int head = 0;
        if (p.per_head) { qrow = r0 + lrow / kIdxHeads; head = lrow % kIdxHeads; }
        else qrow = r0 + lrow;
        const bool row_live = qrow < r_end;
        float w = 1.0f;
        if (p.per_head && p.head_w && row_live) w = p.head_w[(seq * p.n_q + qrow) * kIdxHeads + head];
        for (int j = 0; j < ntiles; ++j) {
            const int ab = j & 1;
            if (!mbar_wait(&sm.acc_full[ab], (j >> 1) & 1, p.status)) break;
            tc_fence_after();
            // both 32-column chunks into registers, then the accumulator is released at once:
            // the MMAs of tile j + 2 need not wait for this tile's stores
            uint32_t r2[2][32];
            tmem_ld32(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(ab * GN + 64 * chalf), r2[0]);
            tmem_ld32(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(ab * GN + 64 * chalf + 32), r2[1]);
            tc_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.acc_empty[ab]);
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const int c = 2 * chalf + cc;
                float v[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r2[cc][i]);
                if (p.per_head) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        float x = v[i];
                        if (p.relu) x = fmaxf(x, 0.0f);
                        x *= w;
                        x += __shfl_xor_sync(0xffffffffu, x, 1);
                        x += __shfl_xor_sync(0xffffffffu, x, 2);
                        v[i] = x;
                    }
                }
                if (p.keys) {
                    // the top 16 bits of the order key (sign, exponent, 7 mantissa bits): the
                    // selection ranks by them and re-scores the keys that tie at 16 bits
                    uint16_t(*t16)[40] = reinterpret_cast<uint16_t(*)[40]>(&sm.epi[ew][0][0]);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        uint32_t w4[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            w4[e] = (score_key(v[8 * i + 2 * e]) >> 16) | (score_key(v[8 * i + 2 * e + 1]) & 0xFFFF0000u);
                        *reinterpret_cast<uint4 *>(&t16[lane][8 * i]) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                    }
                    __syncwarp();
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int rr = 8 * i + (lane >> 2);
                        const int lr = quarter * 32 + rr;
                        const int64_t q = p.per_head ? r0 + lr / kIdxHeads : r0 + lr;
                        const bool writer = q < r_end && (!p.per_head || (lr % kIdxHeads) == 0);
                        if (writer) {
                            uint16_t *d = p.keys + ((int64_t)seq * p.row_count + (q - p.row_begin)) * p.ld +
                                          (int64_t)(j0 + j) * GN + c * 32 + 8 * (lane & 3);
                            *reinterpret_cast<uint4 *>(d) = *reinterpret_cast<const uint4 *>(&t16[rr][8 * (lane & 3)]);
                        }
                    }
                    __syncwarp();
                    continue;
                }
                // stage the 32 x 32 block in smem and store it row-contiguously
                float(*tile)[36] = sm.epi[ew];
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    *reinterpret_cast<float4 *>(&tile[lane][4 * i]) = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2],
                                                                                 v[4 * i + 3]);
                __syncwarp();
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int rr = 4 * i + (lane >> 3);
                    const int lr = quarter * 32 + rr;
                    const int64_t q = p.per_head ? r0 + lr / kIdxHeads : r0 + lr;
                    const bool writer = q < r_end && (!p.per_head || (lr % kIdxHeads) == 0);
                    if (writer) {
                        float *d = p.scores + ((int64_t)seq * p.row_count + (q - p.row_begin)) * p.ld +
                                   (int64_t)(j0 + j) * GN + c * 32 + 4 * (lane & 7);
                        *reinterpret_cast<float4 *>(d) = *reinterpret_cast<const float4 *>(&tile[rr][4 * (lane & 7)]);
                    }
                }
                __syncwarp();
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// fp32 mode: plain SIMT scores.  One CTA per (query row, 128-block slab);
// thread b owns one block.  q_hat [B][n_q][4][128] fp32 (rotated, rounded).
__global__ void __launch_bounds__(128) score_simt_kernel(const float *__restrict__ q_hat,
                                                          const float *__restrict__ k_pool, GemmParams p) {
    __shared__ float qs[kIdxHeads][kIdxDim];
    const int seq = blockIdx.z;
    const int64_t row = p.row_begin + blockIdx.y;
    const int64_t t = p.q0 + row;
    const int64_t nb = (t + 1) / kBlock;
    const int64_t b = (int64_t)blockIdx.x * 128 + threadIdx.x;
    for (int i = threadIdx.x; i < kIdxHeads * kIdxDim; i += 128)
        qs[i / kIdxDim][i % kIdxDim] = q_hat[((int64_t)seq * p.n_q + row) * kIdxHeads * kIdxDim + i];
    __syncthreads();
    if (b >= nb) return;
    const float *kb = k_pool + ((int64_t)seq * p.pool_stride + b) * kIdxDim;
    float acc = 0.0f;
#pragma unroll
    for (int h = 0; h < kIdxHeads; ++h) {
        float dsum = 0.0f;
        for (int i = 0; i < kIdxDim; ++i) dsum = fmaf(qs[h][i], kb[i], dsum);
        if (p.relu) dsum = fmaxf(dsum, 0.0f);
        const float w = p.head_w ? p.head_w[((int64_t)seq * p.n_q + row) * kIdxHeads + h] : 1.0f;
        acc += w * dsum;
    }
    p.scores[((int64_t)seq * p.row_count + blockIdx.y) * p.ld + b] = acc;
}

// Per-row top-k over materialised scores: one warp per (row, sequence), 16
// rows per CTA, no CTA barriers (see warp_topk_row).  kWide: rows of more
// than 65535 visible blocks (positions from 262140 on) count in 32 bits.
constexpr int SEL_WARPS = 16;

template <bool kWide>
__global__ void __launch_bounds__(SEL_WARPS * 32, 2)
    select_rows_kernel(const float *__restrict__ scores, int64_t row_begin, int64_t n_q, int64_t q0, int64_t ld,
                       int top_k, int32_t *__restrict__ sel, int32_t *__restrict__ nsel, int64_t row_count) {
    extern __shared__ uint8_t ssm_raw[];
    WarpSelSmemT<kWide> *wsm = reinterpret_cast<WarpSelSmemT<kWide> *>(ssm_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int seq = blockIdx.y;
    const int64_t rloc = (int64_t)blockIdx.x * SEL_WARPS + warp;
    if (rloc >= row_count) return;
    const int64_t row = row_begin + rloc;
    const int64_t t = q0 + row;
    const int n = (int)((t + 1) / kBlock);
    const float *src = scores + ((int64_t)seq * row_count + rloc) * ld;
    int32_t *out = sel + ((int64_t)seq * n_q + row) * top_k;
    const int cnt = warp_topk_row(src, n, top_k, wsm[warp], [&](int pos, int i) { out[pos] = i; });
    for (int i = cnt + lane; i < top_k; i += 32) out[i] = -1;
    if (lane == 0) nsel[(int64_t)seq * n_q + row] = cnt;
}

// ---- long rows: one CTA per row, two passes over the row
//
// The warp kernel reads a row three times (five when the bin of the k-th key
// overflows its list), and one warp keeps too few loads in flight for rows of
// 10^5 scores.  Here a CTA of SR_THREADS takes one row:
//   pass 1  11-bit histogram of the top digit of every key; a CTA scan finds
//           the bin d1 holding the k-th largest key and k_rem, the number of
//           picks that bin supplies;
//   pass 2  every element of a higher bin is picked (exactly k - k_rem of
//           them); the elements of bin d1 are listed as (~key << 32 | id);
//   rank    the list is sorted ascending (key descending, id ascending: the
//           ranking's tie rule) and its first k_rem ids are picked;
//   order   the k picked ids are sorted ascending and written.
// A bin of more than SR_TIE_CAP elements (massive ties) falls back to the
// warp kernel's passes, run by warp 0.
constexpr int SR_THREADS = 256;
constexpr int SR_TIE_CAP = 4096;
constexpr int SR_SPAN = SR_THREADS * 16;   // elements per iteration: four float4 per thread
#ifndef QSA_SELECT_CTA_MIN_BLOCKS
#define QSA_SELECT_CTA_MIN_BLOCKS 32768
#endif
constexpr int SR_MIN_BLOCKS = QSA_SELECT_CTA_MIN_BLOCKS;   // longest row of a launch from which this kernel is used

struct RowSelSmem {
    uint32_t hist[2048];
    union {
        unsigned long long tie[SR_TIE_CAP];
        WarpSelSmemT<true> warp;            // fallback
    };
    uint32_t pick[2048];                    // picked ids (top_k <= 2048)
    uint32_t wsum[SR_THREADS / 32];
    int n_sure, n_tie, d1, k_rem;
};

// Ascending bitonic sort of a[0, P), P a power of two; all threads of the CTA.
template <typename T>
__device__ __forceinline__ void cta_bitonic_sort(T *a, int P) {
    for (int size = 2; size <= P; size <<= 1)
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = threadIdx.x; i < P / 2; i += blockDim.x) {
                const int lo = 2 * i - (i & (stride - 1));
                const int hi = lo + stride;
                const bool up = (lo & size) == 0;
                const T x = a[lo], y = a[hi];
                if ((x > y) == up) {
                    a[lo] = y;
                    a[hi] = x;
                }
            }
            __syncthreads();
        }
}

__device__ __forceinline__ int pow2_ceil(int x) {
    int p = 1;
    while (p < x) p <<= 1;
    return p;
}

// Element i0 + 4 * tid + SR_THREADS * 4 * u + c of the row, u < 4, c < 4.
template <bool kLast>
__device__ __forceinline__ void sr_load(const float *row, int n, int base, float (&f)[4][4]) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int i = base + u * SR_THREADS * 4 + 4 * (int)threadIdx.x;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        // i < n <= ld and ld % 4 == 0: the whole float4 lies inside the row's stride
        if (i < n) v = kLast ? __ldcs(reinterpret_cast<const float4 *>(row + i))
                             : *reinterpret_cast<const float4 *>(row + i);
        f[u][0] = v.x;
        f[u][1] = v.y;
        f[u][2] = v.z;
        f[u][3] = v.w;
    }
}

__global__ void __launch_bounds__(SR_THREADS)
    select_rows_cta_kernel(const float *__restrict__ scores, int64_t row_begin, int64_t n_q, int64_t q0,
                           int64_t ld, int top_k, int32_t *__restrict__ sel, int32_t *__restrict__ nsel,
                           int64_t row_count) {
    extern __shared__ __align__(16) uint8_t rsm_raw[];
    RowSelSmem &sm = *reinterpret_cast<RowSelSmem *>(rsm_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t lt = (1u << lane) - 1u;
    const int seq = blockIdx.y;
    const int64_t rloc = blockIdx.x;
    const int64_t row = row_begin + rloc;
    const int n = (int)((q0 + row + 1) / kBlock);
    const int k = top_k;
    const float *src = scores + ((int64_t)seq * row_count + rloc) * ld;
    int32_t *out = sel + ((int64_t)seq * n_q + row) * top_k;
    int32_t *cnt_out = nsel + (int64_t)seq * n_q + row;
    if (n <= k) {
        for (int i = tid; i < k; i += SR_THREADS) out[i] = i < n ? i : -1;
        if (tid == 0) *cnt_out = n;
        return;
    }
    for (int i = tid; i < 2048; i += SR_THREADS) sm.hist[i] = 0;
    if (tid == 0) sm.n_sure = sm.n_tie = 0;
    __syncthreads();

    // ---- pass 1: histogram of the top 11 bits
    for (int base = 0; base < n; base += SR_SPAN) {
        float f[4][4];
        sr_load<false>(src, n, base, f);
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int c = 0; c < 4; ++c)
                if (base + u * SR_THREADS * 4 + 4 * tid + c < n) atomicAdd(&sm.hist[score_key(f[u][c]) >> 21], 1u);
    }
    __syncthreads();

    // ---- the bin holding the k-th largest key: thread t owns bins 2047-8t .. 2040-8t
    {
        const int top_bin = 2047 - 8 * tid;
        uint32_t mine = 0;
#pragma unroll
        for (int b = 0; b < 8; ++b) mine += sm.hist[top_bin - b];
        uint32_t incl = mine;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        if (lane == 31) sm.wsum[warp] = incl;
        __syncthreads();
        uint32_t cum = incl - mine;
        for (int w = 0; w < warp; ++w) cum += sm.wsum[w];
        if (cum < (uint32_t)k && cum + mine >= (uint32_t)k) {
            for (int b = 0; b < 8; ++b) {
                const uint32_t h = sm.hist[top_bin - b];
                if (cum + h >= (uint32_t)k) {
                    sm.d1 = top_bin - b;
                    sm.k_rem = k - (int)cum;
                    break;
                }
                cum += h;
            }
        }
        __syncthreads();
    }
    const uint32_t d1 = (uint32_t)sm.d1;
    const int k_rem = sm.k_rem;

    // ---- pass 2: pick the higher bins, list bin d1
    for (int base = 0; base < n; base += SR_SPAN) {
        float f[4][4];
        sr_load<true>(src, n, base, f);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i0 = base + u * SR_THREADS * 4 + 4 * tid;
            uint32_t key[4];
            bool above[4], in_bin[4];
            bool any = false;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                key[c] = score_key(f[u][c]);
                const bool live = i0 + c < n;
                above[c] = live && (key[c] >> 21) > d1;
                in_bin[c] = live && (key[c] >> 21) == d1;
                any |= above[c] || in_bin[c];
            }
            if (!__any_sync(0xffffffffu, any)) continue;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const uint32_t ba = __ballot_sync(0xffffffffu, above[c]);
                if (ba) {
                    const int leader = __ffs(ba) - 1;
                    int slot0 = 0;
                    if (lane == leader) slot0 = atomicAdd(&sm.n_sure, __popc(ba));
                    slot0 = __shfl_sync(0xffffffffu, slot0, leader);
                    const int slot = slot0 + __popc(ba & lt);
                    if (above[c] && slot < 2048) sm.pick[slot] = (uint32_t)(i0 + c);
                }
                const uint32_t bt = __ballot_sync(0xffffffffu, in_bin[c]);
                if (bt) {
                    const int leader = __ffs(bt) - 1;
                    int slot0 = 0;
                    if (lane == leader) slot0 = atomicAdd(&sm.n_tie, __popc(bt));
                    slot0 = __shfl_sync(0xffffffffu, slot0, leader);
                    const int slot = slot0 + __popc(bt & lt);
                    if (in_bin[c] && slot < SR_TIE_CAP)
                        sm.tie[slot] = ((unsigned long long)(~key[c]) << 32) | (uint32_t)(i0 + c);
                }
            }
        }
    }
    __syncthreads();
    const int m = sm.n_tie;
    const int n_sure = sm.n_sure;
    if (m > SR_TIE_CAP || n_sure != k - k_rem) {
        // massive ties: the warp kernel's passes (the union's list is no longer needed)
        if (warp == 0) {
            const int cnt = warp_topk_row(src, n, k, sm.warp, [&](int pos, int i) { out[pos] = i; });
            for (int i = cnt + lane; i < k; i += 32) out[i] = -1;
            if (lane == 0) *cnt_out = cnt;
        }
        return;
    }

    // ---- rank bin d1: key descending, id ascending; its first k_rem are picked
    const int P = pow2_ceil(max(m, 2));
    for (int i = m + tid; i < P; i += SR_THREADS) sm.tie[i] = ~0ull;
    __syncthreads();
    cta_bitonic_sort(sm.tie, P);
    for (int j = tid; j < k_rem; j += SR_THREADS) sm.pick[n_sure + j] = (uint32_t)sm.tie[j];
    // ---- ascending ids
    const int P2 = pow2_ceil(max(k, 2));
    for (int i = k + tid; i < P2; i += SR_THREADS) sm.pick[i] = 0xFFFFFFFFu;
    __syncthreads();
    cta_bitonic_sort(sm.pick, P2);
    for (int i = tid; i < k; i += SR_THREADS) out[i] = (int32_t)sm.pick[i];
    if (tid == 0) *cnt_out = k;
}

// ---- rows of 16-bit keys (BF16 modes): one CTA per row
//
// The score GEMM stores the top 16 bits of each score's order key.  Ranking
// by them is exact except among the keys equal to the threshold key; those
// are re-scored in fp32 from the query operand and the compressed keys:
//   pass 1  histogram of the key's top 12 bits (sign, exponent and three
//           significand bits: 8 bins per binade, so the few binades a row's
//           scores crowd into spread over many bins and the shared-memory
//           atomics rarely collide); the bin d1 holding the k-th largest key,
//           and k1, the picks it supplies;
//   pass 2  histogram of the low 4 bits within bin d1: the threshold key
//           T = (d1, d2) and k2, the picks among the keys equal to T;
//   pass 3  ids of keys > T (exactly k - k2) and of keys == T, each list in
//           ascending id order (per 8192-element tile a block scan orders
//           the writes).  Rows of several tiles whose keys above bin d1 and
//           in it number at most SK_LIST skip it: pass 2 lists those keys in
//           id order with their low 4 bits, and the list is split instead;
//   rank    the keys == T are re-scored; the k2 best (score descending, id
//           ascending: the ranking's tie rule) join the picks;
//   merge   both ascending lists merge into the row's ascending selection.
// More than SK_AMB_CAP keys equal to T (massive ties) take an exact radix
// select over the re-scored 32-bit keys of those entries instead.  A row is
// 2 bytes per visible block, so the CTAs resident at once hold a few tens of
// MB of rows: passes 2 and 3 read L2.
constexpr int SK_THREADS = 256;
constexpr int SK_TILE = SK_THREADS * 8;    // elements per tile: one 16-byte load per thread (massive ties)
constexpr int SK_PER = 32;                 // passes 1-3: contiguous keys per thread (four 16-byte loads in flight)
constexpr int SK_STILE = SK_THREADS * SK_PER;
constexpr int SK_LIST = 4096;              // one-read rows: keys above bin d1 and in it, listed in pass 2
constexpr int SK_AMB_CAP = 2048;

struct KeySelSmem {
    uint32_t h2[256];                     // pass 2 (16 bins); the massive-tie radix select (256 bins)
    uint32_t sure[2048];                  // ids with key > T, ascending
    uint32_t amb[SK_AMB_CAP];             // ids with key == T, ascending
    union {
        uint32_t h1[4096];                // pass 1: counts of the keys' top 12 bits
        struct {                          // after pass 3
            float amb_s[SK_AMB_CAP];      // the re-scored values of the keys == T
            uint32_t chosen[2048];        // the picked ids among them, ascending (also rank scratch)
        };
    };
    float q[kIdxHeads * kIdxDim];         // the row's query operand in fp32 (mode 0: the head sum)
    float w[kIdxHeads];
    int wsum[2][SK_THREADS / 32];
    uint32_t d1, k1, n_d1, d2, k2, n_amb, prefix, need;
};

struct KeySelParams {
    const uint16_t *keys;
    int64_t row_begin, row_count, n_q, q0, ld, pool_stride;
    int top_k, mode, relu;
    const __nv_bfloat16 *qa0, *qa1;      // mode 0: hi, lo planes [B][n_q][128]; mode 1: [B][n_q][4][128]
    const __nv_bfloat16 *k_pool;         // [B][pool_stride][128]
    const float *head_w;                 // [B][n_q][4] or null
    int32_t *sel, *nsel;
};

// The k-th largest of 256 bins counted from the top: bin d and the number of
// picks it supplies (k minus the count above it).  Warp 0; lane l owns bins
// 255 - 8 l .. 248 - 8 l.
__device__ __forceinline__ void sk_find_bin(const uint32_t *h, uint32_t k, uint32_t *d_out, uint32_t *k_out) {
    const int lane = threadIdx.x & 31;
    uint32_t mine = 0;
#pragma unroll
    for (int b = 0; b < 8; ++b) mine += h[255 - 8 * lane - b];
    uint32_t incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    uint32_t cum = incl - mine;
    if (cum < k && cum + mine >= k) {
        for (int b = 0; b < 8; ++b) {
            const uint32_t c = h[255 - 8 * lane - b];
            if (cum + c >= k) {
                *d_out = (uint32_t)(255 - 8 * lane - b);
                *k_out = k - cum;
                break;
            }
            cum += c;
        }
    }
}

// Exclusive block scan of two counts; returns this thread's offsets and the totals.
__device__ __forceinline__ void sk_scan2(int a, int b, int (*wsum)[SK_THREADS / 32], int &oa, int &ob, int &ta,
                                         int &tb);

// The k-th largest of 4096 bins counted from the top (the whole CTA): bin d,
// the picks it supplies and its count.  Thread t owns bins 4095 - 16 t .. 4080 - 16 t.
// Ends with a barrier.
__device__ __forceinline__ void sk_find_bin4096(const uint32_t *h, uint32_t k, int (*wsum)[SK_THREADS / 32],
                                                uint32_t *d_out, uint32_t *k_out, uint32_t *n_out) {
    static_assert(SK_THREADS * 16 == 4096, "16 bins per thread");
    const int tid = threadIdx.x;
    const int lo = 16 * (SK_THREADS - 1 - tid);   // this thread's lowest bin
    const uint4 *src = reinterpret_cast<const uint4 *>(h + lo);
    uint32_t mine = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint4 v = src[j];
        mine += (v.x + v.y) + (v.z + v.w);
    }
    int above, unused, ta, tb;   // keys in the bins above this thread's (threads of lower index)
    sk_scan2((int)mine, 0, wsum, above, unused, ta, tb);
    uint32_t cum = (uint32_t)above;
    if (cum < k && cum + mine >= k) {
        for (int j = 15; j >= 0; --j) {
            const uint32_t c = h[lo + j];
            if (cum + c >= k) {
                *d_out = (uint32_t)(lo + j);
                *k_out = k - cum;
                *n_out = c;
                break;
            }
            cum += c;
        }
    }
    __syncthreads();
}

// Exclusive block scan of two counts; returns this thread's offsets and the totals.
__device__ __forceinline__ void sk_scan2(int a, int b, int (*wsum)[SK_THREADS / 32], int &oa, int &ob, int &ta,
                                         int &tb) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int ia = a, ib = b;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, ia, o), y = __shfl_up_sync(0xffffffffu, ib, o);
        if (lane >= o) {
            ia += x;
            ib += y;
        }
    }
    if (lane == 31) {
        wsum[0][warp] = ia;
        wsum[1][warp] = ib;
    }
    __syncthreads();
    int pa = 0, pb = 0;
    ta = tb = 0;
#pragma unroll
    for (int w = 0; w < SK_THREADS / 32; ++w) {
        pa += (w < warp) ? wsum[0][w] : 0;
        pb += (w < warp) ? wsum[1][w] : 0;
        ta += wsum[0][w];
        tb += wsum[1][w];
    }
    __syncthreads();
    oa = pa + ia - a;
    ob = pb + ib - b;
}

// The fp32 score of block b for the row whose operand is in sm.q (one thread).
__device__ __forceinline__ float sk_score(const KeySelSmem &sm, const __nv_bfloat16 *kb, int mode, int relu) {
    const __nv_bfloat162 *k2 = reinterpret_cast<const __nv_bfloat162 *>(kb);
    if (mode == 0) {
        float acc = 0.f;
#pragma unroll 8
        for (int i = 0; i < kIdxDim / 2; ++i) {
            const float2 kv = __bfloat1622float2(k2[i]);
            acc = fmaf(sm.q[2 * i], kv.x, acc);
            acc = fmaf(sm.q[2 * i + 1], kv.y, acc);
        }
        return acc;
    }
    float tot = 0.f;
    for (int h = 0; h < kIdxHeads; ++h) {
        float acc = 0.f;
#pragma unroll 8
        for (int i = 0; i < kIdxDim / 2; ++i) {
            const float2 kv = __bfloat1622float2(k2[i]);
            acc = fmaf(sm.q[h * kIdxDim + 2 * i], kv.x, acc);
            acc = fmaf(sm.q[h * kIdxDim + 2 * i + 1], kv.y, acc);
        }
        if (relu) acc = fmaxf(acc, 0.f);
        tot = fmaf(sm.w[h], acc, tot);
    }
    return tot;
}

// The same score by one warp: lane l multiplies dims 4 l .. 4 l + 3 (one 8-byte
// load of the key), a butterfly sum adds the lanes (every lane ends with the
// same value).
__device__ __forceinline__ float sk_score_warp(const KeySelSmem &sm, const __nv_bfloat16 *kb, int mode, int relu) {
    const int lane = threadIdx.x & 31;
    const uint2 raw = __ldg(reinterpret_cast<const uint2 *>(kb) + lane);
    const float2 k01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.x));
    const float2 k23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.y));
    auto dot = [&](const float *q) {
        const float4 qv = reinterpret_cast<const float4 *>(q)[lane];
        float a = qv.x * k01.x;
        a = fmaf(qv.y, k01.y, a);
        a = fmaf(qv.z, k23.x, a);
        a = fmaf(qv.w, k23.y, a);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
        return a;
    };
    if (mode == 0) return dot(sm.q);
    float tot = 0.f;
#pragma unroll
    for (int h = 0; h < kIdxHeads; ++h) {
        float acc = dot(sm.q + h * kIdxDim);
        if (relu) acc = fmaxf(acc, 0.f);
        tot = fmaf(sm.w[h], acc, tot);
    }
    return tot;
}

__global__ void __launch_bounds__(SK_THREADS, 6) select_keys_kernel(KeySelParams p) {
    extern __shared__ __align__(16) uint8_t ksm_raw[];
    KeySelSmem &sm = *reinterpret_cast<KeySelSmem *>(ksm_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int seq = blockIdx.y;
    const int64_t rloc = blockIdx.x;
    const int64_t row = p.row_begin + rloc;
    const int64_t qrow = (int64_t)seq * p.n_q + row;
    const int n = (int)((p.q0 + row + 1) / kBlock);
    const uint32_t k = (uint32_t)p.top_k;
    int32_t *out = p.sel + qrow * p.top_k;
    pdl_wait();
    pdl_trigger();
    if (n <= (int)k) {
        for (int i = tid; i < (int)k; i += SK_THREADS) out[i] = i < n ? i : -1;
        if (tid == 0) p.nsel[qrow] = n;
        return;
    }
    const uint16_t *src = p.keys + ((int64_t)seq * p.row_count + rloc) * p.ld;
    const __nv_bfloat16 *kp = p.k_pool + (int64_t)seq * p.pool_stride * kIdxDim;
    // the row's query operand (fp32) and head weights: loaded now, stored to shared
    // memory after pass 3 (only the re-score reads them), so no pass waits for them
    static_assert(kIdxDim <= SK_THREADS && kIdxHeads * kIdxDim == 2 * SK_THREADS, "operand staging");
    float qv0 = 0.f, qv1 = 0.f, wv = 1.f;
    if (p.mode == 0) {
        if (tid < kIdxDim)
            qv0 = __bfloat162float(p.qa0[qrow * kIdxDim + tid]) + __bfloat162float(p.qa1[qrow * kIdxDim + tid]);
    } else {
        qv0 = __bfloat162float(p.qa0[qrow * kIdxHeads * kIdxDim + tid]);
        qv1 = __bfloat162float(p.qa0[qrow * kIdxHeads * kIdxDim + SK_THREADS + tid]);
        if (tid < kIdxHeads && p.head_w) wv = p.head_w[qrow * kIdxHeads + tid];
    }
    for (int i = tid; i < 4096 / 4; i += SK_THREADS) reinterpret_cast<uint4 *>(sm.h1)[i] = make_uint4(0, 0, 0, 0);
    for (int i = tid; i < 256; i += SK_THREADS) sm.h2[i] = 0;
    __syncthreads();

    // 8 keys of a tile (thread tid: elements base + 8 tid ..), zero past the row (never counted)
    auto load8 = [&](int base, uint16_t (&kk)[8]) {
        const int i = base + 8 * tid;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (i < n) v = *reinterpret_cast<const uint4 *>(src + i);   // ld is a multiple of 128: in the row
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            kk[2 * e] = (uint16_t)(w4[e] & 0xFFFFu);
            kk[2 * e + 1] = (uint16_t)(w4[e] >> 16);
        }
    };
    // Passes 1-3 walk the row in tiles of SK_STILE keys, thread tid holding keys
    // [base + 32 tid, base + 32 tid + 32): four 16-byte loads in flight per thread,
    // and in pass 3 one ordered block scan per tile.  Returns the live keys held.
    auto load32 = [&](int base, uint32_t (&w)[16]) -> int {
        const int i = base + SK_PER * tid;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint4 v = make_uint4(0, 0, 0, 0);
            if (i + 8 * j < n) v = *reinterpret_cast<const uint4 *>(src + i + 8 * j);   // ld: a multiple of 128
            w[4 * j] = v.x; w[4 * j + 1] = v.y; w[4 * j + 2] = v.z; w[4 * j + 3] = v.w;
        }
        return max(0, min(SK_PER, n - i));
    };
    auto key_of = [](const uint32_t (&w)[16], int e) -> uint32_t { return (w[e >> 1] >> (16 * (e & 1))) & 0xFFFFu; };
    // ---- pass 1: top 12 bits
    for (int base = 0; base < n; base += SK_STILE) {
        uint32_t w[16];
        const int live = load32(base, w);
#pragma unroll
        for (int e = 0; e < SK_PER; ++e)
            if (e < live) atomicAdd(&sm.h1[key_of(w, e) >> 4], 1u);
    }
    // the next pass's first tile is loaded while the bin is searched (likewise before pass 3)
    uint32_t wpre[16];
    int lpre = load32(0, wpre);
    __syncthreads();
    sk_find_bin4096(sm.h1, k, sm.wsum, &sm.d1, &sm.k1, &sm.n_d1);
    const uint32_t d1 = sm.d1, k1 = sm.k1;
    uint32_t T, k2, n_amb;
    if (n > SK_STILE && (k - k1) + sm.n_d1 <= (uint32_t)SK_LIST) {
        // ---- pass 2, rows of several tiles whose keys above bin d1 (k - k1 of
        // them, all picked) and in it fit the list: pass 2 writes them in id
        // order (entry: id | low 4 bits << 16 | above bin d1 << 20) beside the
        // low-4-bit histogram of bin d1, and the row is not read again.  (A
        // one-tile row re-reads its tile from L2 for less than the list costs.)
        uint32_t *list = sm.h1;   // the pass-1 counts are no longer read
        int pos = 0;
        auto tile = [&](const uint32_t (&w)[16], int live, int base) {
            uint32_t am = 0, cm = 0;
            uint32_t nib[4] = {0u, 0u, 0u, 0u};   // low 4 bits of key e at bits 4 (e & 7) of nib[e >> 3]
#pragma unroll
            for (int e = 0; e < SK_PER; ++e) {
                const uint32_t key = key_of(w, e), b = key >> 4;
                const bool in = e < live && b == d1;
                am |= (e < live && b > d1) ? (1u << e) : 0u;
                cm |= in ? (1u << e) : 0u;
                nib[e >> 3] |= (key & 0xFu) << (4 * (e & 7));
                if (in) atomicAdd(&sm.h2[key & 0xFu], 1u);
            }
            uint32_t all = am | cm;
            int o, ob, t, tb;
            sk_scan2(__popc(all), 0, sm.wsum, o, ob, t, tb);
            o += pos;
            const uint32_t id0 = (uint32_t)(base + SK_PER * tid);
            while (all) {   // a few keys per thread and tile
                const int e = __ffs(all) - 1;
                all &= all - 1u;
                const uint32_t nw = e < 16 ? (e < 8 ? nib[0] : nib[1]) : (e < 24 ? nib[2] : nib[3]);
                if (o < SK_LIST) list[o] = (id0 + (uint32_t)e) | (((nw >> (4 * (e & 7))) & 0xFu) << 16) | (((am >> e) & 1u) << 20);
                ++o;
            }
            pos += t;
        };
        tile(wpre, lpre, 0);
        for (int base = SK_STILE; base < n; base += SK_STILE) {
            uint32_t w[16];
            const int live = load32(base, w);
            tile(w, live, base);
        }
        __syncthreads();
        if (warp == 0) {
            sk_find_bin(sm.h2, k1, &sm.d2, &sm.k2);   // bins 16-255 are empty
            __syncwarp();
            if (lane == 0) sm.n_amb = sm.h2[sm.d2];
        }
        __syncthreads();
        const uint32_t d2 = sm.d2;
        T = (d1 << 4) | d2;
        k2 = sm.k2;
        n_amb = sm.n_amb;
        // ---- the list split in id order: keys above T and keys equal to T
        static_assert(SK_LIST == 16 * SK_THREADS, "16 list entries per thread");
        const int nl = min(pos, SK_LIST);
        const int j0 = 16 * tid;
        uint32_t gt = 0, eq = 0;   // bit j: entry j0 + j lies above T / equals T
        for (int j = 0; j < 16 && j0 + j < nl; ++j) {
            const uint32_t ent = list[j0 + j];
            const uint32_t nib = (ent >> 16) & 0xFu;
            const bool above = (ent >> 20) & 1u;
            gt |= (above || nib > d2) ? (1u << j) : 0u;
            eq |= (!above && nib == d2) ? (1u << j) : 0u;
        }
        int os, oa, ts, ta;
        sk_scan2(__popc(gt), __popc(eq), sm.wsum, os, oa, ts, ta);
        // the list is read again below; nothing writes over it before the barrier after this split
        while (gt) {
            const int j = __ffs(gt) - 1;
            gt &= gt - 1u;
            if (os < 2048) sm.sure[os] = list[j0 + j] & 0xFFFFu;
            ++os;
        }
        while (eq) {
            const int j = __ffs(eq) - 1;
            eq &= eq - 1u;
            if (oa < SK_AMB_CAP) sm.amb[oa] = list[j0 + j] & 0xFFFFu;
            ++oa;
        }
    } else {
        // ---- pass 2: low 4 bits within bin d1
        auto pass2_tile = [&](const uint32_t (&w)[16], int live) {
#pragma unroll
            for (int e = 0; e < SK_PER; ++e) {
                const uint32_t key = key_of(w, e);
                if (e < live && (key >> 4) == d1) atomicAdd(&sm.h2[key & 0xFu], 1u);
            }
        };
        pass2_tile(wpre, lpre);
        for (int base = SK_STILE; base < n; base += SK_STILE) {
            uint32_t w[16];
            const int live = load32(base, w);
            pass2_tile(w, live);
        }
        lpre = load32(0, wpre);
        __syncthreads();
        if (warp == 0) {
            sk_find_bin(sm.h2, sm.k1, &sm.d2, &sm.k2);   // bins 16-255 are empty
            __syncwarp();
            if (lane == 0) sm.n_amb = sm.h2[sm.d2];
        }
        __syncthreads();
        T = (d1 << 4) | sm.d2;
        k2 = sm.k2;
        n_amb = sm.n_amb;
        // ---- pass 3: ids above T and equal to T, ascending
        {
            int pos_s = 0, pos_a = 0;
            auto pass3_tile = [&](const uint32_t (&w)[16], int live, int base) {
                uint32_t gt = 0, eq = 0;   // bit e: key e lies above T / equals T
#pragma unroll
                for (int e = 0; e < SK_PER; ++e) {
                    const uint32_t key = key_of(w, e);
                    gt |= (e < live && key > T) ? (1u << e) : 0u;
                    eq |= (e < live && key == T) ? (1u << e) : 0u;
                }
                int os, oa, ts, ta;
                sk_scan2(__popc(gt), __popc(eq), sm.wsum, os, oa, ts, ta);
                os += pos_s;
                oa += pos_a;
                const uint32_t id0 = (uint32_t)(base + SK_PER * tid);
                while (gt) {   // few keys per row pass: walk the set bits
                    const int e = __ffs(gt) - 1;
                    gt &= gt - 1u;
                    if (os < 2048) sm.sure[os] = id0 + (uint32_t)e;
                    ++os;
                }
                while (eq) {
                    const int e = __ffs(eq) - 1;
                    eq &= eq - 1u;
                    if (oa < SK_AMB_CAP) sm.amb[oa] = id0 + (uint32_t)e;
                    ++oa;
                }
                pos_s += ts;
                pos_a += ta;
            };
            pass3_tile(wpre, lpre, 0);
            for (int base = SK_STILE; base < n; base += SK_STILE) {
                uint32_t w[16];
                const int live = load32(base, w);
                pass3_tile(w, live, base);
            }
        }
    }
    const int n_sure = (int)(k - k2);
    if (p.mode == 0) {
        if (tid < kIdxDim) sm.q[tid] = qv0;
    } else {
        sm.q[tid] = qv0;
        sm.q[SK_THREADS + tid] = qv1;
        if (tid < kIdxHeads) sm.w[tid] = wv;
    }
    __syncthreads();
    if (n_amb <= (uint32_t)SK_AMB_CAP) {
        // ---- re-score the keys equal to T (a warp each), rank, pick the k2 best
        for (uint32_t i = warp; i < n_amb; i += SK_THREADS / 32) {
            const float sc = sk_score_warp(sm, kp + (int64_t)sm.amb[i] * kIdxDim, p.mode, p.relu);
            if (lane == 0) sm.amb_s[i] = sc;
        }
        __syncthreads();
        for (uint32_t i = tid; i < n_amb; i += SK_THREADS) {
            const float si = sm.amb_s[i];
            uint32_t r = 0;
            for (uint32_t j = 0; j < n_amb; ++j) {
                const float sj = sm.amb_s[j];
                r += (sj > si || (sj == si && j < i)) ? 1u : 0u;   // the list is in id order
            }
            sm.chosen[i < 2048 ? i : 0] = r;   // n_amb <= SK_AMB_CAP = 2048
        }
        __syncthreads();
        // compact the picked ones in id order
        int pos = 0;
        for (uint32_t base = 0; base < n_amb; base += SK_THREADS) {
            const uint32_t i = base + tid;
            const bool pick = i < n_amb && sm.chosen[i] < k2;
            int o, dummy, t, td;
            sk_scan2(pick ? 1 : 0, 0, sm.wsum, o, dummy, t, td);
            // the ranks of this window are read before any write below (scan barrier)
            if (pick) sm.amb_s[pos + o] = __uint_as_float(sm.amb[i]);
            pos += t;
        }
        __syncthreads();
        for (uint32_t i = tid; i < k2; i += SK_THREADS) sm.chosen[i] = __float_as_uint(sm.amb_s[i]);
        __syncthreads();
    } else {
        // ---- massive ties: exact radix select over the re-scored 32-bit keys of the entries equal to T
        if (tid == 0) {
            sm.prefix = 0;
            sm.need = k2;
        }
        for (int byte = 3; byte >= 0; --byte) {
            for (int i = tid; i < 256; i += SK_THREADS) sm.h2[i] = 0;
            __syncthreads();
            const uint32_t prefix = sm.prefix;
            for (int base = 0; base < n; base += SK_TILE) {
                uint16_t kk[8];
                load8(base, kk);
#pragma unroll 1
                for (int e = 0; e < 8; ++e) {
                    if (base + 8 * tid + e >= n || kk[e] != T) continue;
                    const uint32_t ek = score_key(sk_score(sm, kp + (int64_t)(base + 8 * tid + e) * kIdxDim, p.mode,
                                                           p.relu));
                    const bool match = byte == 3 || (ek >> (8 * (byte + 1))) == prefix;
                    if (match) atomicAdd(&sm.h2[(ek >> (8 * byte)) & 0xFFu], 1u);
                }
            }
            __syncthreads();
            if (warp == 0) {
                sk_find_bin(sm.h2, sm.need, &sm.d2, &sm.k1);   // (d2, k1 reused as scratch: T is kept above)
                __syncwarp();
                if (lane == 0) {
                    sm.prefix = (prefix << 8) | sm.d2;
                    sm.need = sm.k1;
                }
            }
            __syncthreads();
        }
        const uint32_t tx = sm.prefix, need = sm.need;   // exact threshold key; picks among keys == tx
        int pos = 0, peq = 0;
        for (int base = 0; base < n; base += SK_TILE) {
            uint16_t kk[8];
            load8(base, kk);
            uint32_t ek[8];
            int cg = 0, ce = 0;
#pragma unroll 1
            for (int e = 0; e < 8; ++e) {
                ek[e] = 0;
                if (base + 8 * tid + e >= n || kk[e] != T) continue;
                ek[e] = score_key(sk_score(sm, kp + (int64_t)(base + 8 * tid + e) * kIdxDim, p.mode, p.relu));
                cg += ek[e] > tx ? 1 : 0;
                ce += ek[e] == tx ? 1 : 0;
            }
            int og, oe, tg, te;
            sk_scan2(cg, ce, sm.wsum, og, oe, tg, te);
            // picks of this tile: every key > tx, and keys == tx while fewer than `need` were taken
            int taken_eq = peq + oe;
            int mine = 0;
#pragma unroll 1
            for (int e = 0; e < 8; ++e) {
                if (base + 8 * tid + e >= n || kk[e] != T) continue;
                if (ek[e] > tx) ++mine;
                else if (ek[e] == tx && taken_eq < (int)need) {
                    ++mine;
                    ++taken_eq;
                }
            }
            int om, dummy, tm, td;
            sk_scan2(mine, 0, sm.wsum, om, dummy, tm, td);
            om += pos;
            taken_eq = peq + oe;
#pragma unroll 1
            for (int e = 0; e < 8; ++e) {
                if (base + 8 * tid + e >= n || kk[e] != T) continue;
                bool pick = ek[e] > tx;
                if (!pick && ek[e] == tx && taken_eq < (int)need) {
                    pick = true;
                    ++taken_eq;
                }
                if (pick) {
                    if (om < 2048) sm.chosen[om] = (uint32_t)(base + 8 * tid + e);
                    ++om;
                }
            }
            pos += tm;
            peq += te;
        }
        __syncthreads();
    }
    // ---- merge the two ascending lists: sure (n_sure) and chosen (k2)
    for (int i = tid; i < n_sure; i += SK_THREADS) {
        const uint32_t id = sm.sure[i];
        int lo = 0, hi = (int)k2;   // chosen ids below id
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (sm.chosen[mid] < id) lo = mid + 1;
            else hi = mid;
        }
        out[i + lo] = (int32_t)id;
    }
    for (int j = tid; j < (int)k2; j += SK_THREADS) {
        const uint32_t id = sm.chosen[j];
        int lo = 0, hi = n_sure;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (sm.sure[mid] < id) lo = mid + 1;
            else hi = mid;
        }
        out[j + lo] = (int32_t)id;
    }
    if (tid == 0) p.nsel[qrow] = (int)k;
}

// Driver-API tensor-map encoder obtained through the runtime (no -lcuda).
using EncodeTiledFn = decltype(&cuTensorMapEncodeTiled);
EncodeTiledFn get_encode() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// 2-D bf16 map over [rows][128] with a 64 x box_rows box, 128-byte swizzle.
bool make_map(CUtensorMap *map, const void *base, uint64_t rows, uint32_t box_rows) {
    auto enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[2] = {128, rows};
    cuuint64_t strides[1] = {128 * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_score_gemm(const ScoreGemmArgs &a, const void *qa0, const void *qa1, const void *k_pool,
                              unsigned *status, cudaStream_t s) {
    if (a.row_count <= 0) return cudaSuccess;
    const int rows_per_tile = a.per_head ? GM / kIdxHeads : GM;
    const uint64_t a_rows = (uint64_t)a.B * a.n_q * (a.per_head ? kIdxHeads : 1);
    CUtensorMap ma0, ma1, mb;
    if (!make_map(&ma0, qa0, a_rows, GM)) return cudaErrorInvalidValue;
    if (!make_map(&ma1, a.per_head ? qa0 : qa1, a_rows, GM)) return cudaErrorInvalidValue;
    if (!make_map(&mb, k_pool, (uint64_t)a.B * a.pool_stride, GN)) return cudaErrorInvalidValue;
    GemmParams p{a.n_q, a.q0, a.row_begin, a.row_count, a.pool_stride, a.ld, a.per_head, a.relu, a.head_w,
                 a.scores, status, 1, 0, a.keys};
    // Split each row tile's key tiles over several CTAs so that the grid holds
    // about four CTAs per SM whatever the row count (a 2048-row chunk of a
    // 1M-token context has 16 row tiles of 2048 key tiles each).
    const int64_t row_tiles = (a.row_count + rows_per_tile - 1) / rows_per_tile;
    const int64_t max_tiles = ((a.q0 + a.row_begin + a.row_count) / kBlock + GN - 1) / GN;
    const DeviceInfo *di = device_info();
    const int64_t want = 4 * (int64_t)(di ? di->sm_count : 148);
    const int64_t nsplit = std::max<int64_t>(1, std::min<int64_t>(max_tiles, (want + row_tiles * a.B - 1) / (row_tiles * a.B)));
    p.nsplit = (int)nsplit;
    p.span = (int)std::max<int64_t>(1, (max_tiles + nsplit - 1) / nsplit);
    const size_t smem = sizeof(GemmSmem) + 1024;
    static bool attr_done = false;
    if (!attr_done) {
        cudaError_t e = cudaFuncSetAttribute(score_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr_done = true;
    }
    dim3 grid((unsigned)(row_tiles * nsplit), (unsigned)a.B);
    score_gemm_kernel<<<grid, GEMM_THREADS, smem, s>>>(ma0, ma1, mb, p);
    return cudaGetLastError();
}

cudaError_t launch_score_simt_f32(const ScoreGemmArgs &a, const float *q_hat, const float *k_pool, cudaStream_t s) {
    if (a.row_count <= 0) return cudaSuccess;
    const int64_t nb_max = (a.q0 + a.row_begin + a.row_count) / kBlock;
    if (nb_max <= 0) return cudaSuccess;
    GemmParams p{a.n_q, a.q0, a.row_begin, a.row_count, a.pool_stride, a.ld, 0, a.relu, a.head_w, a.scores,
                 nullptr};
    dim3 grid((unsigned)((nb_max + 127) / 128), (unsigned)a.row_count, (unsigned)a.B);
    score_simt_kernel<<<grid, 128, 0, s>>>(q_hat, k_pool, p);
    return cudaGetLastError();
}

cudaError_t launch_select_keys(const uint16_t *keys, int B, int64_t row_begin, int64_t row_count, int64_t n_q,
                               int64_t q0, int64_t ld, int top_k, int mode, int relu, const void *qa0, const void *qa1,
                               const void *k_pool, int64_t pool_stride, const float *head_w, int32_t *sel,
                               int32_t *nsel, cudaStream_t s) {
    if (row_count <= 0) return cudaSuccess;
    KeySelParams p{};
    p.keys = keys;
    p.row_begin = row_begin;
    p.row_count = row_count;
    p.n_q = n_q;
    p.q0 = q0;
    p.ld = ld;
    p.pool_stride = pool_stride;
    p.top_k = top_k;
    p.mode = mode;
    p.relu = relu;
    p.qa0 = static_cast<const __nv_bfloat16 *>(qa0);
    p.qa1 = static_cast<const __nv_bfloat16 *>(qa1);
    p.k_pool = static_cast<const __nv_bfloat16 *>(k_pool);
    p.head_w = head_w;
    p.sel = sel;
    p.nsel = nsel;
    const size_t smem = sizeof(KeySelSmem);
    cudaError_t e = cudaFuncSetAttribute(select_keys_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(select_keys_kernel, dim3((unsigned)row_count, (unsigned)B), dim3(SK_THREADS), smem, s, p);
}

cudaError_t launch_select_rows(const float *scores, int B, int64_t row_begin, int64_t row_count, int64_t n_q,
                               int64_t q0, int64_t ld, int top_k, int32_t *sel, int32_t *nsel, unsigned *status,
                               cudaStream_t s) {
    (void)status;
    if (row_count <= 0) return cudaSuccess;
    const int64_t n_max = (q0 + row_begin + row_count) / kBlock;   // the longest row's blocks
    if (n_max >= SR_MIN_BLOCKS) {
        const size_t smem = sizeof(RowSelSmem);
        cudaError_t e = cudaFuncSetAttribute(select_rows_cta_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        dim3 grid((unsigned)row_count, (unsigned)B);
        select_rows_cta_kernel<<<grid, SR_THREADS, smem, s>>>(scores, row_begin, n_q, q0, ld, top_k, sel, nsel,
                                                              row_count);
        return cudaGetLastError();
    }
    const bool wide = n_max > kWarpSelNarrowMax;
    auto kernel = wide ? select_rows_kernel<true> : select_rows_kernel<false>;
    const size_t smem = SEL_WARPS * (wide ? sizeof(WarpSelSmemT<true>) : sizeof(WarpSelSmemT<false>));
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)((row_count + SEL_WARPS - 1) / SEL_WARPS), (unsigned)B);
    kernel<<<grid, SEL_WARPS * 32, smem, s>>>(scores, row_begin, n_q, q0, ld, top_k, sel, nsel, row_count);
    return cudaGetLastError();
}

}  // namespace qsa
