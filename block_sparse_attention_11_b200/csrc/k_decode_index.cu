// k_decode_index.cu -- decode indexer: scan all compressed keys of each
// sequence for its one new query, keep the top-k blocks.
//
// Page "Qwen3.8-Flash-Next: Day-0 Support in SGLang", section "IndexShare MTP":
// the decode scorer reads all ceil(L/4) compressed blocks and, beyond a few
// thousand tokens, sets the cost of the layer.  So the scan is an HBM-streaming
// kernel: each CTA owns a contiguous chunk of one sequence's compressed keys,
// pulls it through shared memory with TMA (bulk copies in fp32 mode, 128-byte
// swizzled tensor tiles in bf16 mode where the scores come from warp MMAs),
// writes one 4-byte order-preserving score key per block to the workspace and
// adds the chunk's histogram of the keys' top 11 bits into a per-sequence
// histogram.  The selection then runs over the keys (still in L2) in one pass,
// one thread-block cluster per sequence: only the keys of the histogram bin
// holding the k-th largest key need their remaining bits resolved, and one
// CTA of the cluster assembles the ascending output.
#include <algorithm>

#include "internal.h"
#include "select.cuh"

namespace qsa {

namespace {

constexpr int DI_THREADS = 256;
constexpr int DI_NS = 4;
constexpr int DI_STAGE_BYTES = 16384;

struct DecodeParams {
    const int32_t *seq_len;
    const float *head_w;
    int64_t pool_stride, max_blocks, chunk, kstride;
    int chunks, top_k, relu;
    uint32_t *keys;      // [B][kstride] score keys
    uint32_t *hist;      // [B][2048] histogram of the keys' top 11 bits
    unsigned *status;
};

// Adds a CTA's local histogram (smem, 2048 bins) into the sequence's global one.
__device__ __forceinline__ void flush_hist(const uint32_t *lh, uint32_t *gh) {
    for (int b = threadIdx.x; b < 2048; b += blockDim.x)
        if (lh[b]) atomicAdd(&gh[b], lh[b]);
}

template <typename T>
__global__ void __launch_bounds__(DI_THREADS, 2)
    decode_score_kernel(const T *__restrict__ q_idx, const T *__restrict__ k_pool, Rope rope, DecodeParams p) {
    constexpr int VEC = 16 / sizeof(T);          // elements per lane per 16-byte load
    constexpr int LPR = kIdxDim / VEC;           // lanes per key row
    constexpr int RPW = 32 / LPR;                // rows per warp instruction
    constexpr int ROW_BYTES = kIdxDim * sizeof(T);
    constexpr int SROWS = DI_STAGE_BYTES / ROW_BYTES;
    extern __shared__ __align__(128) uint8_t dsm[];
    uint8_t *stage = dsm;                                                   // DI_NS * 16 KB
    __shared__ uint64_t full[DI_NS];
    __shared__ float qh[kIdxHeads][kIdxDim];
    __shared__ float qsum[kIdxDim];
    __shared__ uint32_t lh[2048];

    pdl_trigger();
    const int seq = blockIdx.y, c = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t s_len = p.seq_len[seq];
    int64_t nb = s_len / kBlock;
    if (s_len < 1 || nb > p.pool_stride || nb > p.max_blocks) {
        if (tid == 0 && c == 0) flag(p.status, QSA_DEV_BAD_LENGTH);
        nb = 0;
    }
    const int64_t c0 = (int64_t)c * p.chunk;
    const int64_t c1 = min(c0 + p.chunk, nb);
    const int n = (int)(c1 > c0 ? c1 - c0 : 0);
    if (n == 0) return;
    uint32_t *gkeys = p.keys + (int64_t)seq * p.kstride + c0;
    const int nstages = (n + SROWS - 1) / SROWS;
    const T *kbase = k_pool + ((int64_t)seq * p.pool_stride + c0) * kIdxDim;
    for (int b = tid; b < 2048; b += blockDim.x) lh[b] = 0;
    if (tid == 0) {
        for (int s = 0; s < DI_NS; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
        for (int st = 0; st < min(DI_NS, nstages); ++st) {
            const int rows = min(SROWS, n - st * SROWS);
            mbar_arrive_expect_tx(&full[st], rows * ROW_BYTES);
            bulk_g2s(stage + st * DI_STAGE_BYTES, kbase + (int64_t)st * SROWS * kIdxDim, rows * ROW_BYTES, &full[st]);
        }
    }
    // rotated query heads of the new token (position s_len - 1), rounded to T
    if (tid < kIdxDim) {
        const int e = tid, R = rope.rotary_dim, half = R >> 1;
        const T *src = q_idx + (int64_t)seq * kIdxHeads * kIdxDim;
        double cs = 1.0, sn = 0.0;
        int pr = e;
        if (e < R) {
            pr = e < half ? e + half : e - half;
            const double ang = __dmul_rn(__ddiv_rn((double)(s_len - 1), rope.pos_scale),
                                         rope_inv_freq(rope, e < half ? e : e - half));
            sincos(ang, &sn, &cs);
        }
        float hs = 0.0f;
        for (int h = 0; h < kIdxHeads; ++h) {
            const double xe = to_float(src[h * kIdxDim + e]);
            double o = xe;
            if (e < R) {
                const double xp = to_float(src[h * kIdxDim + pr]);
                o = (e < half) ? __dsub_rn(__dmul_rn(xe, cs), __dmul_rn(xp, sn))
                               : __dadd_rn(__dmul_rn(xe, cs), __dmul_rn(xp, sn));
            }
            const float r = to_float(from_double<T>(o));
            qh[h][e] = r;
            hs = (h == 0) ? r : __fadd_rn(hs, r);
        }
        qsum[e] = hs;
    }
    __syncthreads();
    const bool per_head = p.relu || p.head_w;
    float w[kIdxHeads] = {1.f, 1.f, 1.f, 1.f};
    if (p.head_w)
        for (int h = 0; h < kIdxHeads; ++h) w[h] = p.head_w[(int64_t)seq * kIdxHeads + h];
    const int sub = lane % LPR, rsub = lane / LPR;
    float qv[kIdxHeads][VEC], qs[VEC];
#pragma unroll
    for (int i = 0; i < VEC; ++i) {
        qs[i] = qsum[sub * VEC + i];
#pragma unroll
        for (int h = 0; h < kIdxHeads; ++h) qv[h][i] = qh[h][sub * VEC + i];
    }

    for (int st = 0; st < nstages; ++st) {
        const int slot = st % DI_NS;
        const bool ok = __syncthreads_and(mbar_wait(&full[slot], (st / DI_NS) & 1, p.status));
        if (!ok) return;   // every thread leaves together; the status word says why
        const int rows = min(SROWS, n - st * SROWS);
        const uint8_t *buf = stage + slot * DI_STAGE_BYTES;
        for (int r = warp * RPW + rsub; r < ((rows + RPW - 1) / RPW) * RPW; r += 8 * RPW) {
            const bool live = r < rows;
            float kv[VEC];
            if (live) {
                const uint4 raw = *reinterpret_cast<const uint4 *>(buf + r * ROW_BYTES + sub * 16);
                const T *e = reinterpret_cast<const T *>(&raw);
#pragma unroll
                for (int i = 0; i < VEC; ++i) kv[i] = to_float(e[i]);
            } else {
#pragma unroll
                for (int i = 0; i < VEC; ++i) kv[i] = 0.f;
            }
            float score;
            if (!per_head) {
                float acc = 0.f;
#pragma unroll
                for (int i = 0; i < VEC; ++i) acc = fmaf(qs[i], kv[i], acc);
#pragma unroll
                for (int o = LPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
                score = acc;
            } else {
                float acc[kIdxHeads];
#pragma unroll
                for (int h = 0; h < kIdxHeads; ++h) {
                    float a = 0.f;
#pragma unroll
                    for (int i = 0; i < VEC; ++i) a = fmaf(qv[h][i], kv[i], a);
#pragma unroll
                    for (int o = LPR / 2; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
                    acc[h] = a;
                }
                score = 0.f;
#pragma unroll
                for (int h = 0; h < kIdxHeads; ++h) score += w[h] * (p.relu ? fmaxf(acc[h], 0.f) : acc[h]);
            }
            if (live && sub == 0) {
                const uint32_t key = score_key(score);
                gkeys[st * SROWS + r] = key;
                atomicAdd(&lh[key >> 21], 1u);
            }
        }
        __syncthreads();
        if (tid == 0 && st + DI_NS < nstages) {
            const int st2 = st + DI_NS;
            const int rows2 = min(SROWS, n - st2 * SROWS);
            mbar_arrive_expect_tx(&full[slot], rows2 * ROW_BYTES);
            bulk_g2s(stage + slot * DI_STAGE_BYTES, kbase + (int64_t)st2 * SROWS * kIdxDim, rows2 * ROW_BYTES,
                     &full[slot]);
        }
    }
    __syncthreads();
    flush_hist(lh, p.hist + (int64_t)seq * 2048);
}

// bf16 scorer on the tensor cores.  A 128-key stage arrives by two tensor
// TMA loads (64 dims x 128 keys each, 128-byte swizzle) so ldmatrix reads are
// conflict-free; each warp scores one 16-key tile per stage with 8
// m16n8k16 MMAs: A = keys (16 keys x 16 dims), B = the query as 8 columns
// (hi and lo planes of the FP32 head sum, or the 4 heads), FP32 accumulate.
constexpr int DM_ROWS = 128;                       // keys per stage
constexpr int DM_NS = 3;                           // stages in flight per CTA (2 CTAs per SM)
constexpr int DM_STAGE_BYTES = DM_ROWS * 256;      // two 64-dim k-atoms of 128 rows x 128 B

struct DecodeMmaSmem {
    alignas(1024) uint8_t stage[DM_NS][DM_STAGE_BYTES];
    alignas(16) __nv_bfloat16 qcol[8][kIdxDim];   // B operand source: 8 columns x 128 dims
    float w[kIdxHeads];
    uint64_t full[DM_NS], empty[DM_NS];
    uint32_t lh[2048];                             // local histogram of the keys' top 11 bits
};

__global__ void __launch_bounds__(DI_THREADS, 2)
    decode_score_mma_kernel(const __grid_constant__ CUtensorMap kmap, const __nv_bfloat16 *__restrict__ q_idx,
                            Rope rope, DecodeParams p) {
    extern __shared__ uint8_t dsm_raw[];
    DecodeMmaSmem &sm = *reinterpret_cast<DecodeMmaSmem *>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) &
                                                           ~uintptr_t(1023));
    pdl_trigger();
    const int seq = blockIdx.y, c = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t s_len = p.seq_len[seq];
    int64_t nb = s_len / kBlock;
    if (s_len < 1 || nb > p.pool_stride || nb > p.max_blocks) {
        if (tid == 0 && c == 0) flag(p.status, QSA_DEV_BAD_LENGTH);
        nb = 0;
    }
    const int64_t c0 = (int64_t)c * p.chunk;
    const int64_t c1 = min(c0 + p.chunk, nb);
    const int n = (int)(c1 > c0 ? c1 - c0 : 0);
    if (n == 0) return;
    uint32_t *gkeys = p.keys + (int64_t)seq * p.kstride + c0;
    for (int b = tid; b < 2048; b += blockDim.x) sm.lh[b] = 0;
    const int nstages = (n + DM_ROWS - 1) / DM_ROWS;
    const int y0 = (int)(seq * p.pool_stride + c0);
    if (tid == 0) {
        for (int s = 0; s < DM_NS; ++s) { mbar_init(&sm.full[s], 1); mbar_init(&sm.empty[s], DI_THREADS / 32); }
        fence_mbar_init();
        prefetch_tmap(&kmap);
    }
    __syncthreads();
    if (tid == 0) {
        for (int st = 0; st < min(DM_NS, nstages); ++st) {
            mbar_arrive_expect_tx(&sm.full[st], DM_STAGE_BYTES);
            tma_load_2d(sm.stage[st], &kmap, 0, y0 + st * DM_ROWS, &sm.full[st]);
            tma_load_2d(sm.stage[st] + DM_STAGE_BYTES / 2, &kmap, 64, y0 + st * DM_ROWS, &sm.full[st]);
        }
    }
    const bool per_head = p.relu || p.head_w;
    // rotated query heads of the new token (position s_len - 1), rounded to bf16;
    // columns: hi/lo of the FP32 head sum, or the 4 heads
    if (tid < kIdxDim) {
        const int e = tid, R = rope.rotary_dim, half = R >> 1;
        const __nv_bfloat16 *src = q_idx + (int64_t)seq * kIdxHeads * kIdxDim;
        double cs = 1.0, sn = 0.0;
        int pr = e;
        if (e < R) {
            pr = e < half ? e + half : e - half;
            const double ang = __dmul_rn(__ddiv_rn((double)(s_len - 1), rope.pos_scale),
                                         rope_inv_freq(rope, e < half ? e : e - half));
            sincos(ang, &sn, &cs);
        }
        float hs = 0.0f;
        for (int h = 0; h < kIdxHeads; ++h) {
            const double xe = __bfloat162float(src[h * kIdxDim + e]);
            double o = xe;
            if (e < R) {
                const double xp = __bfloat162float(src[h * kIdxDim + pr]);
                o = (e < half) ? __dsub_rn(__dmul_rn(xe, cs), __dmul_rn(xp, sn))
                               : __dadd_rn(__dmul_rn(xe, cs), __dmul_rn(xp, sn));
            }
            const __nv_bfloat16 r = d2bf(o);
            if (per_head) sm.qcol[h][e] = r;
            hs = (h == 0) ? __bfloat162float(r) : __fadd_rn(hs, __bfloat162float(r));
        }
        const __nv_bfloat16 zero = __float2bfloat16_rn(0.f);
        if (!per_head) {
            const __nv_bfloat16 hi = __float2bfloat16_rn(hs);
            sm.qcol[0][e] = hi;
            sm.qcol[1][e] = __float2bfloat16_rn(__fsub_rn(hs, __bfloat162float(hi)));
            for (int col = 2; col < 8; ++col) sm.qcol[col][e] = zero;
        } else {
            for (int col = 4; col < 8; ++col) sm.qcol[col][e] = zero;
        }
    }
    if (tid < kIdxHeads) sm.w[tid] = p.head_w ? p.head_w[(int64_t)seq * kIdxHeads + tid] : 1.f;
    __syncthreads();
    const int gr = lane >> 2, tq = lane & 3;
    uint32_t qf[8][2];
    {
        const uint32_t *qw = reinterpret_cast<const uint32_t *>(&sm.qcol[gr][0]);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            qf[kk][0] = qw[(16 * kk + 2 * tq) >> 1];
            qf[kk][1] = qw[(16 * kk + 8 + 2 * tq) >> 1];
        }
    }
    const float w0 = sm.w[2 * (tq & 1)], w1 = sm.w[2 * (tq & 1) + 1];
    const int mi = lane >> 3, rr = lane & 7;
    const int trow = 16 * warp + rr + 8 * (mi & 1);      // row of this lane's ldmatrix address in the stage
    const uint32_t row_off = (uint32_t)trow * 128u;
    const uint32_t sw = (uint32_t)(trow & 7);
    bool ok = true;
    for (int st = 0; st < nstages; ++st) {
        const int slot = st % DM_NS;
        ok = mbar_wait(&sm.full[slot], (st / DM_NS) & 1, p.status);
        if (!ok) break;
        const uint32_t base = smem_u32(sm.stage[slot]);
        float acc[4] = {0.f, 0.f, 0.f, 0.f}, acc2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kk = 0; kk < 8; kk += 2) {
            uint32_t a[4], b[4];
            {
                const uint32_t chunk = (uint32_t)(2 * (kk & 3) + (mi >> 1));
                ldsm_x4(base + (kk >> 2) * (DM_STAGE_BYTES / 2) + row_off + ((chunk ^ sw) << 4), a[0], a[1], a[2], a[3]);
            }
            {
                const uint32_t chunk = (uint32_t)(2 * ((kk + 1) & 3) + (mi >> 1));
                ldsm_x4(base + ((kk + 1) >> 2) * (DM_STAGE_BYTES / 2) + row_off + ((chunk ^ sw) << 4), b[0], b[1], b[2],
                        b[3]);
            }
            mma16816(acc, a[0], a[1], a[2], a[3], qf[kk][0], qf[kk][1]);
            mma16816(acc2, b[0], b[1], b[2], b[3], qf[kk + 1][0], qf[kk + 1][1]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[i] += acc2[i];
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.empty[slot]);
        float s0, s1;   // rows gr and gr + 8 of this warp's tile
        if (!per_head) {
            s0 = acc[0] + acc[1];
            s1 = acc[2] + acc[3];
        } else {
            float a0 = acc[0], a1 = acc[1], a2 = acc[2], a3 = acc[3];
            if (p.relu) { a0 = fmaxf(a0, 0.f); a1 = fmaxf(a1, 0.f); a2 = fmaxf(a2, 0.f); a3 = fmaxf(a3, 0.f); }
            s0 = w0 * a0 + w1 * a1;
            s1 = w0 * a2 + w1 * a3;
            s0 += __shfl_xor_sync(0xffffffffu, s0, 1);
            s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
        }
        const int r0 = st * DM_ROWS + 16 * warp + gr;
        if (tq == 0) {
            if (r0 < n) {
                const uint32_t key = score_key(s0);
                gkeys[r0] = key;
                atomicAdd(&sm.lh[key >> 21], 1u);
            }
            if (r0 + 8 < n) {
                const uint32_t key = score_key(s1);
                gkeys[r0 + 8] = key;
                atomicAdd(&sm.lh[key >> 21], 1u);
            }
        }
        if (tid == 0 && st + DM_NS < nstages) {
            ok = mbar_wait(&sm.empty[slot], (st / DM_NS) & 1, p.status);
            if (ok) {
                const int st2 = st + DM_NS;
                mbar_arrive_expect_tx(&sm.full[slot], DM_STAGE_BYTES);
                tma_load_2d(sm.stage[slot], &kmap, 0, y0 + st2 * DM_ROWS, &sm.full[slot]);
                tma_load_2d(sm.stage[slot] + DM_STAGE_BYTES / 2, &kmap, 64, y0 + st2 * DM_ROWS, &sm.full[slot]);
            }
        }
    }
    ok = __syncthreads_and(ok);
    if (!ok) return;
    flush_hist(sm.lh, p.hist + (int64_t)seq * 2048);
}

using EncodeTiledFn = decltype(&cuTensorMapEncodeTiled);

// 2-D bf16 map over the compressed keys [rows][128]: 64 x 128 boxes, 128-byte swizzle.
bool make_kpool_map(CUtensorMap *map, const void *base, uint64_t rows) {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return false;
        fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    cuuint64_t dims[2] = {128, rows};
    cuuint64_t strides[1] = {128 * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)DM_ROWS};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---------------------------------------------------------------------------
// Selection from the score keys: one kernel, one thread-block cluster of up to
// 16 CTAs per sequence.
//
// Every CTA owns a chunk of a sequence's keys (whole tiles of DS_TILE keys,
// 16 contiguous keys per thread, read with four 16-byte loads issued
// together).  With the top-11-bit histogram from the scorer, the bin d1 that
// holds the k-th largest key is known before any key is read.  Each CTA
// writes to its own shared memory, in block order, the ids of its keys above
// bin d1 (all of them are selected; fewer than k in the whole sequence) and
// the (key, id) pairs of its keys in bin d1 (the candidates; past the
// shared-memory capacity they go to a global overflow area).  After a cluster
// barrier, CTA 0 gathers the lists through distributed shared memory, resolves
// the remaining 21 bits of K* on the candidates, keeps the candidates above K*
// and the first ones equal to K* (ties to the lower block id), and merges that
// list with the above-bin ids into the ascending output.
// ---------------------------------------------------------------------------
constexpr int DS_THREADS = 512;
constexpr int DS_PER_THREAD = 16;
constexpr int DS_TILE = DS_THREADS * DS_PER_THREAD;   // keys per CTA tile
constexpr int DS_CLUSTER = 16;                        // CTAs (chunks) per sequence at most (non-portable above 8)
constexpr int DS_LCAND = 2048;                        // candidates a CTA keeps in shared memory
constexpr int DS_CAND_SMEM = 4096;                    // candidates CTA 0 stages in shared memory
constexpr int DS_MAX_K = 2048;                        // largest top_k

struct SelectArgs {
    const int32_t *seq_len;
    int64_t pool_stride, max_blocks, kstride, chunk;   // chunk: keys per CTA, a multiple of DS_TILE
    int gmax, top_k;                                    // gmax: CTAs per cluster (<= DS_CLUSTER)
    const uint32_t *keys;   // [B][kstride] score keys
    const uint32_t *hist;   // [B][2048] histogram of the keys' top 11 bits
    uint2 *cand;            // [B][kstride]: chunk g's candidates past DS_LCAND, at g * chunk + position
    int32_t *sel, *nsel;
};

struct DsSmem {
    SelectSmem s;                       // histogram, warp partials, digit search results
    // this CTA's lists (read by CTA 0 through distributed shared memory)
    int32_t my_above[DS_MAX_K];
    uint32_t my_ck[DS_LCAND];
    uint32_t my_ci[DS_LCAND];
    uint32_t my_na, my_nc;
    // CTA 0
    uint32_t ck[DS_CAND_SMEM];          // candidate keys (block order)
    uint32_t ci[DS_CAND_SMEM];          // candidate block ids
    int32_t alist[DS_MAX_K];            // ids above bin d1 (ascending)
    int32_t slist[DS_MAX_K];            // selected candidate ids (ascending)
    uint32_t aoff[DS_CLUSTER + 1];      // prefix of the above counts per chunk
    uint32_t coff[DS_CLUSTER + 1];      // prefix of the candidate counts per chunk
    uint32_t wsum[DS_THREADS / 32];
};

__device__ __forceinline__ int64_t visible_blocks(const SelectArgs &a, int seq) {
    const int64_t s_len = a.seq_len[seq];
    const int64_t nb = s_len / kBlock;
    return (s_len < 1 || nb > a.pool_stride || nb > a.max_blocks) ? 0 : nb;   // flagged by the scorer
}

// Loads keys [i0, i0 + 16) of a row (i0 a multiple of 16; the row holds
// kstride keys, a multiple of 4); returns how many of them are < n.
__device__ __forceinline__ int load16(const uint32_t *row, int64_t i0, int64_t n, int64_t kstride, uint32_t k[16]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int64_t i = i0 + 4 * j;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (i < n && i < kstride) v = __ldcg(reinterpret_cast<const uint4 *>(row + i));
        k[4 * j] = v.x; k[4 * j + 1] = v.y; k[4 * j + 2] = v.z; k[4 * j + 3] = v.w;
    }
    const int64_t m = n - i0;
    return m <= 0 ? 0 : (m >= 16 ? 16 : (int)m);
}

// Exclusive prefix over the CTA; total in `total`.  Two barriers.
__device__ __forceinline__ uint32_t cta_scan(uint32_t v, uint32_t *wsum, uint32_t &total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    const uint32_t wv = lane < nw ? wsum[lane] : 0u;     // lane l: warp l's total (nw <= 32)
    const uint32_t off = __reduce_add_sync(0xffffffffu, lane < warp ? wv : 0u);
    total = __reduce_add_sync(0xffffffffu, wv);
    __syncthreads();
    return off + x - v;
}

// Largest g < n with off[g] <= j (off ascending): the chunk that holds entry j.
__device__ __forceinline__ int chunk_of(const uint32_t *off, int n, uint32_t j) {
    int g = 0;
    for (int c = 1; c < n; ++c) g = off[c] <= j ? c : g;
    return g;
}

// Entries of the ascending list l[0..n) that are smaller than v.
__device__ __forceinline__ int count_below(const int32_t *l, int n, int32_t v) {
    int lo = 0, hi = n;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (l[mid] < v) lo = mid + 1;
        else hi = mid;
    }
    return lo;
}

__global__ void __launch_bounds__(DS_THREADS)
    decode_select_kernel(SelectArgs a) {
    extern __shared__ __align__(16) uint8_t ds_raw[];
    DsSmem &sm = *reinterpret_cast<DsSmem *>(ds_raw);
    pdl_wait();
    pdl_trigger();
    const int seq = blockIdx.y, tid = threadIdx.x;
    const uint32_t rank = cluster_rank();             // = blockIdx.x: a cluster spans the x extent
    const int64_t nb = visible_blocks(a, seq);
    const int top_k = a.top_k;
    int32_t *out = a.sel + (int64_t)seq * top_k;
    const int64_t c0 = (int64_t)rank * a.chunk, c1 = min(c0 + a.chunk, nb);
    if (nb <= top_k) {                               // every visible block, in order (whole cluster)
        for (int64_t i = c0 + tid; i < c1; i += DS_THREADS) out[i] = (int32_t)i;
        if (rank == 0) {
            for (int i = (int)nb + tid; i < top_k; i += DS_THREADS) out[i] = -1;
            if (tid == 0) a.nsel[seq] = (int)nb;
        }
        return;
    }
    const int gseq = (int)((nb + a.chunk - 1) / a.chunk);   // CTAs with keys (<= cluster size)
    const uint32_t *row = a.keys + (int64_t)seq * a.kstride;
    uint2 *cand_seq = a.cand + (int64_t)seq * a.kstride;
    // first tile's keys in flight before the histogram is read
    uint32_t k[16];
    int m = load16(row, c0 + (int64_t)DS_PER_THREAD * tid, c1, a.kstride, k);
    // bin of the k-th largest key from the scorer's histogram
    static_assert(DS_THREADS * 4 == 2048, "one 16-byte histogram load per thread");
    reinterpret_cast<uint4 *>(sm.s.hist)[tid] = __ldcg(reinterpret_cast<const uint4 *>(a.hist + (int64_t)seq * 2048) + tid);
    if (tid == 0) { sm.s.digit = 0; sm.s.k_rem = 1; }
    __syncthreads();
    sel_find_digit(sm.s, 2048, top_k);
    const uint32_t d1 = (uint32_t)sm.s.digit;
    const int k_rem1 = sm.s.k_rem;

    uint32_t na_run = 0, nc_run = 0;
    for (int64_t t0 = c0; t0 < c1; t0 += DS_TILE) {
        const int64_t i0 = t0 + (int64_t)DS_PER_THREAD * tid;
        if (t0 != c0) m = load16(row, i0, c1, a.kstride, k);
        // bit j: key j lies above bin d1 (amask) or in it (cmask); few keys do
        uint32_t amask = 0, cmask = 0;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const uint32_t dg = k[j] >> 21;
            amask |= (uint32_t)(dg > d1) << j;
            cmask |= (uint32_t)(dg == d1) << j;
        }
        const uint32_t valid = m >= 16 ? 0xFFFFu : ((1u << m) - 1u);
        amask &= valid;
        cmask &= valid;
        uint32_t tot;
        const uint32_t ex = cta_scan(__popc(amask) | (__popc(cmask) << 16), sm.wsum, tot);
        uint32_t pa = na_run + (ex & 0xFFFFu), pc = nc_run + (ex >> 16);
        const uint32_t any = amask | cmask;
        if (any) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                if (((any >> (4 * q)) & 0xFu) == 0) continue;
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const int j = 4 * q + jj;
                    if ((amask >> j) & 1u) {
                        if (pa < (uint32_t)DS_MAX_K) sm.my_above[pa] = (int32_t)(i0 + j);
                        ++pa;
                    } else if ((cmask >> j) & 1u) {
                        if (pc < (uint32_t)DS_LCAND) { sm.my_ck[pc] = k[j]; sm.my_ci[pc] = (uint32_t)(i0 + j); }
                        else cand_seq[c0 + pc] = make_uint2(k[j], (uint32_t)(i0 + j));   // pc < c1 - c0
                        ++pc;
                    }
                }
            }
        }
        na_run += tot & 0xFFFFu;
        nc_run += tot >> 16;
    }
    if (tid == 0) {
        sm.my_na = min(na_run, (uint32_t)min(top_k - 1, DS_MAX_K));
        sm.my_nc = nc_run;
    }
    cluster_sync();                                  // every CTA's lists are complete
    if (rank == 0) {
        // per-chunk offsets of the above ids and of the candidates
        if (tid == 0) {
            uint32_t ea = 0, ec = 0;
            for (int c = 0; c < gseq; ++c) {
                sm.aoff[c] = ea;
                sm.coff[c] = ec;
                ea += ld_dsmem(dsmem_addr(&sm.my_na, c));
                ec += ld_dsmem(dsmem_addr(&sm.my_nc, c));
            }
            sm.aoff[gseq] = ea;
            sm.coff[gseq] = ec;
        }
        __syncthreads();
        const int na_all = (int)min(sm.aoff[gseq], (uint32_t)(top_k - 1));
        const int nc_all = (int)min((int64_t)sm.coff[gseq], nb);
        const bool small = nc_all <= DS_CAND_SMEM;
        for (int j = tid; j < na_all; j += DS_THREADS) {
            const int c = chunk_of(sm.aoff, gseq, (uint32_t)j);
            sm.alist[j] = (int32_t)ld_dsmem(dsmem_addr(&sm.my_above[j - sm.aoff[c]], c));
        }
        auto fetch = [&](int j) -> uint2 {           // candidate j of the sequence, block order
            const int c = chunk_of(sm.coff, gseq, (uint32_t)j);
            const uint32_t jj = (uint32_t)j - sm.coff[c];
            if (jj < (uint32_t)DS_LCAND)
                return make_uint2(ld_dsmem(dsmem_addr(&sm.my_ck[jj], c)), ld_dsmem(dsmem_addr(&sm.my_ci[jj], c)));
            return __ldcg(cand_seq + (int64_t)c * a.chunk + jj);
        };
        if (small)
            for (int j = tid; j < nc_all; j += DS_THREADS) {
                const uint2 v = fetch(j);
                sm.ck[j] = v.x;
                sm.ci[j] = v.y;
            }
        __syncthreads();
        auto cand_at = [&](int j) -> uint2 { return small ? make_uint2(sm.ck[j], sm.ci[j]) : fetch(j); };
        // remaining 21 bits of K*: bits 20..10, then 9..0
        uint32_t prefix = d1 << 21, pmask = 0xFFE00000u;
        int k_rem = k_rem1;
#pragma unroll 1
        for (int pass = 0; pass < 2; ++pass) {
            const int shift = pass == 0 ? 10 : 0, nbins = pass == 0 ? 2048 : 1024;
            const uint32_t mask = (uint32_t)nbins - 1u;
            for (int b = tid; b < nbins; b += DS_THREADS) sm.s.hist[b] = 0;
            __syncthreads();
            for (int j = tid; j < nc_all; j += DS_THREADS) {
                const uint32_t key = cand_at(j).x;
                if ((key & pmask) == prefix) atomicAdd(&sm.s.hist[(key >> shift) & mask], 1u);
            }
            __syncthreads();
            sel_find_digit(sm.s, nbins, k_rem);
            prefix |= (uint32_t)sm.s.digit << shift;
            pmask |= mask << shift;
            k_rem = sm.s.k_rem;
            __syncthreads();
        }
        const uint32_t kstar = prefix;
        const int take_eq = k_rem;
        // selected candidates in block order: keys above K*, and the first take_eq equal to K*.
        // Thread t takes a contiguous run of cpt candidates per round of DS_THREADS * cpt.
        int ns = 0;     // CTA-uniform running count
        uint32_t eq_run = 0;
        const int cpt = min(8, max(1, (nc_all + DS_THREADS - 1) / DS_THREADS));
        for (int base = 0; base < nc_all; base += DS_THREADS * cpt) {
            const int j0 = base + cpt * tid, j1 = min(j0 + cpt, nc_all);
            uint32_t eq = 0;
            for (int j = j0; j < j1; ++j) eq += cand_at(j).x == kstar;
            uint32_t eq_tot;
            const uint32_t r0 = eq_run + cta_scan(eq, sm.wsum, eq_tot);   // rank of my first key == K*
            uint32_t r = r0, nsel_mine = 0;
            for (int j = j0; j < j1; ++j) {
                const uint32_t key = cand_at(j).x;
                nsel_mine += key > kstar || (key == kstar && r++ < (uint32_t)take_eq);
            }
            uint32_t s_tot;
            uint32_t pos = (uint32_t)ns + cta_scan(nsel_mine, sm.wsum, s_tot);
            r = r0;
            for (int j = j0; j < j1; ++j) {
                const uint2 v = cand_at(j);
                if (v.x > kstar || (v.x == kstar && r++ < (uint32_t)take_eq)) {
                    if (pos < (uint32_t)DS_MAX_K) sm.slist[pos] = (int32_t)v.y;
                    ++pos;
                }
            }
            ns += (int)s_tot;
            eq_run += eq_tot;
        }
        ns = min(ns, top_k - na_all);
        __syncthreads();
        // merge the two ascending lists into the output
        for (int j = tid; j < na_all; j += DS_THREADS) {
            const int32_t v = sm.alist[j];
            const int pos = j + count_below(sm.slist, ns, v);
            if (pos < top_k) out[pos] = v;
        }
        for (int j = tid; j < ns; j += DS_THREADS) {
            const int32_t v = sm.slist[j];
            const int pos = j + count_below(sm.alist, na_all, v);
            if (pos < top_k) out[pos] = v;
        }
        const int cnt = na_all + ns;
        for (int i = cnt + tid; i < top_k; i += DS_THREADS) out[i] = -1;
        if (tid == 0) a.nsel[seq] = cnt;
    }
    cluster_sync();                                  // CTA 0 has finished reading the others' lists
}

}  // namespace

DecodePlan decode_index_plan(int B, int64_t max_blocks, bool bf16) {
    (void)bf16;
    const DeviceInfo *di = device_info();
    const int sms = di ? di->sm_count : 148;
    DecodePlan pl;
    // at most two CTAs per SM over all sequences (one wave: a second, partial
    // wave would stream its chunks with a fraction of the SMs), chunks of at
    // least 512 blocks
    int64_t C = std::max<int64_t>(1, (2 * sms) / std::max(B, 1));
    C = std::min<int64_t>(C, std::max<int64_t>(1, (max_blocks + 511) / 512));
    int64_t chunk = (max_blocks + C - 1) / C;
    chunk = std::max<int64_t>(128, (chunk + 127) / 128 * 128);
    C = std::max<int64_t>(1, (max_blocks + chunk - 1) / chunk);
    pl.chunks = (int)C;
    pl.chunk = chunk;
    return pl;
}

namespace {
int64_t key_stride(int64_t max_blocks) { return std::max<int64_t>(4, (max_blocks + 3) / 4 * 4); }
size_t r256(size_t x) { return (x + 255) / 256 * 256; }

struct SelectLayout {
    int64_t chunk;
    int gmax;
};

// Whether clusters of 16 CTAs of the select kernel can be resident (checked once).
bool cluster16_ok();

// Chunks of whole tiles, at most DS_CLUSTER per sequence (8 where 16 cannot run).
SelectLayout select_layout(int64_t max_blocks) {
    const int64_t tiles = std::max<int64_t>(1, (max_blocks + DS_TILE - 1) / DS_TILE);
    const int64_t cmax = (tiles > 8 && cluster16_ok()) ? DS_CLUSTER : 8;
    const int64_t tiles_per_chunk = (tiles + cmax - 1) / cmax;
    SelectLayout l;
    l.chunk = tiles_per_chunk * DS_TILE;
    l.gmax = (int)((tiles + tiles_per_chunk - 1) / tiles_per_chunk);
    return l;
}

bool cluster16_ok() {
    static int ok = -1;
    if (ok < 0) {
        ok = 0;
        if (cudaFuncSetAttribute(decode_select_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
                cudaSuccess &&
            cudaFuncSetAttribute(decode_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)sizeof(DsSmem)) == cudaSuccess) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(DS_CLUSTER, 1, 1);
            cfg.blockDim = dim3(DS_THREADS, 1, 1);
            cfg.dynamicSmemBytes = sizeof(DsSmem);
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = DS_CLUSTER;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, decode_select_kernel, &cfg) == cudaSuccess && n > 0) ok = 1;
        }
        cudaGetLastError();   // a refused query leaves no sticky error
    }
    return ok == 1;
}

// Workspace: keys [B][kstride] u32 | cand overflow [B][kstride] uint2 | hist [B][2048] u32
struct DecodeWs {
    uint32_t *keys;
    uint2 *cand;
    uint32_t *hist;
    size_t zero_bytes;   // hist, cleared before every call
    size_t total;
};

DecodeWs decode_ws(void *base, int B, int64_t max_blocks, int top_k) {
    (void)top_k;
    const int64_t ks = key_stride(max_blocks);
    uint8_t *w = static_cast<uint8_t *>(base);
    DecodeWs d;
    size_t off = 0;
    d.keys = reinterpret_cast<uint32_t *>(w + off);
    off += r256((size_t)B * ks * 4);
    d.cand = reinterpret_cast<uint2 *>(w + off);
    off += r256((size_t)B * ks * 8);
    d.hist = reinterpret_cast<uint32_t *>(w + off);
    d.zero_bytes = (size_t)B * 2048 * 4;
    off += r256(d.zero_bytes);
    d.total = off;
    return d;
}
}  // namespace

size_t decode_index_ws_bytes(int B, int64_t max_blocks, int top_k, bool bf16) {
    (void)bf16;
    return decode_ws(nullptr, B, max_blocks, top_k).total;
}

cudaError_t launch_decode_index(const void *q_idx, const void *k_pool, const float *head_w,
                                const int32_t *seq_len, int B, int64_t pool_stride, int64_t max_blocks,
                                int top_k, int32_t *sel, int32_t *nsel, void *ws, Rope rope, bool relu,
                                bool bf16, unsigned *status, cudaStream_t s) {
    const DecodePlan pl = decode_index_plan(B, max_blocks, bf16);
    const int64_t kstride = key_stride(max_blocks);
    const DecodeWs d = decode_ws(ws, B, max_blocks, top_k);
    cudaError_t e = cudaMemsetAsync(d.hist, 0, d.zero_bytes, s);
    if (e != cudaSuccess) return e;
    DecodeParams p{seq_len, head_w, pool_stride, max_blocks, pl.chunk, kstride, pl.chunks, top_k, relu ? 1 : 0,
                   d.keys, d.hist, status};
    dim3 grid((unsigned)pl.chunks, (unsigned)B);
    if (bf16) {
        CUtensorMap kmap;
        if (!make_kpool_map(&kmap, k_pool, (uint64_t)B * pool_stride)) return cudaErrorInvalidValue;
        const size_t smem = sizeof(DecodeMmaSmem) + 1024;
        e = cudaFuncSetAttribute(decode_score_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        decode_score_mma_kernel<<<grid, DI_THREADS, smem, s>>>(kmap, (const __nv_bfloat16 *)q_idx, rope, p);
    } else {
        const size_t smem = DI_NS * DI_STAGE_BYTES;
        e = cudaFuncSetAttribute(decode_score_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        decode_score_kernel<float><<<grid, DI_THREADS, smem, s>>>((const float *)q_idx, (const float *)k_pool, rope,
                                                                  p);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const SelectLayout l = select_layout(max_blocks);
    SelectArgs sa{seq_len, pool_stride, max_blocks, kstride, l.chunk, l.gmax, top_k, d.keys, d.hist, d.cand, sel,
                  nsel};
    const dim3 sgrid((unsigned)l.gmax, (unsigned)B);
    e = cudaFuncSetAttribute(decode_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(DsSmem));
    if (e != cudaSuccess) return e;
    if (l.gmax > 8) {
        e = cudaFuncSetAttribute(decode_select_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
    }
    return launch_pdl_cluster(decode_select_kernel, sgrid, dim3(DS_THREADS), sizeof(DsSmem), (unsigned)l.gmax, s, sa);
}

}  // namespace qsa
