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
    int64_t pool_stride, max_blocks, chunk, kstride;   // paged: pool_stride = max_pages * page_tokens / 4
    int chunks, top_k, relu;
    uint32_t *keys;      // [B][kstride] score keys
    uint32_t *hist;      // [B][2048] histogram of the keys' top 11 bits
    unsigned *status;
    Paging pg;           // pg.table: the compressed keys are paged (rows slot / 4)
};

// Bulk copy of rows [lr0, lr0 + rows) of sequence seq's compressed keys
// (row_bytes each) into dst, completing on bar: one copy when contiguous, one
// per page run when paged.  Returns the bytes issued (rows of a page outside
// the cache are skipped and flagged), to be posted with expect_tx first: call
// once with issue = false to count, then with issue = true.
__device__ __forceinline__ uint32_t copy_key_rows(const DecodeParams &p, const uint8_t *k_pool, int seq,
                                                  int64_t lr0, int rows, int row_bytes, uint8_t *dst, uint64_t *bar,
                                                  bool issue) {
    if (!p.pg.table) {
        if (issue)
            bulk_g2s(dst, k_pool + ((int64_t)seq * p.pool_stride + lr0) * row_bytes, (uint32_t)(rows * row_bytes),
                     bar);
        return (uint32_t)(rows * row_bytes);
    }
    const int page_rows = p.pg.page_tokens / kBlock;
    uint32_t bytes = 0;
    for (int r = 0; r < rows;) {
        const int64_t lr = lr0 + r;
        const int run = min(rows - r, page_rows - (int)(lr & (page_rows - 1)));
        const int64_t slot = paged_slot(p.pg, seq, lr * kBlock);
        if (slot >= 0) {
            if (issue) bulk_g2s(dst + (int64_t)r * row_bytes, k_pool + (slot / kBlock) * row_bytes,
                                (uint32_t)(run * row_bytes), bar);
            bytes += (uint32_t)(run * row_bytes);
        } else if (!issue) {
            flag(p.status, QSA_DEV_BAD_INDEX);
        }
        r += run;
    }
    return bytes;
}

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

    pdl_wait();      // the compressed keys come from the previous kernel (ring pooling)
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
    const uint8_t *kbytes = reinterpret_cast<const uint8_t *>(k_pool);
    for (int b = tid; b < 2048; b += blockDim.x) lh[b] = 0;
    if (tid == 0) {
        for (int s = 0; s < DI_NS; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
        for (int st = 0; st < min(DI_NS, nstages); ++st) {
            const int rows = min(SROWS, n - st * SROWS);
            const int64_t lr = c0 + (int64_t)st * SROWS;
            uint8_t *dst = stage + st * DI_STAGE_BYTES;
            mbar_arrive_expect_tx(&full[st], copy_key_rows(p, kbytes, seq, lr, rows, ROW_BYTES, dst, &full[st], false));
            copy_key_rows(p, kbytes, seq, lr, rows, ROW_BYTES, dst, &full[st], true);
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
            const int64_t lr = c0 + (int64_t)st2 * SROWS;
            uint8_t *dst = stage + slot * DI_STAGE_BYTES;
            mbar_arrive_expect_tx(&full[slot],
                                  copy_key_rows(p, kbytes, seq, lr, rows2, ROW_BYTES, dst, &full[slot], false));
            copy_key_rows(p, kbytes, seq, lr, rows2, ROW_BYTES, dst, &full[slot], true);
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
constexpr int DM_NS_FP8 = 6;                       // FP8 stages are half the bytes
constexpr int DM_STAGE_BYTES = DM_ROWS * 256;      // two 64-dim k-atoms of 128 rows x 128 B
// FP8 E4M3 compressed keys: a stage is one 128-byte-swizzled box of 128 rows x
// 128 B, the A operand of m16n8k32 E4M3 MMAs as it lands.
constexpr int DM_STAGE_BYTES_FP8 = DM_ROWS * 128;
constexpr int DM_PG_IDS = 1024;                    // paged: page ids a scorer CTA keeps (bounds its chunk)
template <bool FP8> __host__ __device__ constexpr int stage_bytes() { return FP8 ? DM_STAGE_BYTES_FP8 : DM_STAGE_BYTES; }

using EncodeTiledFn = decltype(&cuTensorMapEncodeTiled);

// 2-D map over the compressed keys [rows][128]: bf16 in 64 x 128 boxes, or
// FP8 E4M3 (as bytes) in 128 x 128 boxes; 128-byte swizzle.
bool make_kpool_map(CUtensorMap *map, const void *base, uint64_t rows, bool fp8 = false, int box_rows = DM_ROWS) {
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
    cuuint64_t strides[1] = {fp8 ? 128u : 128u * 2};
    cuuint32_t box[2] = {fp8 ? 128u : 64u, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base),
              dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Streams the n compressed keys of rows y0.. through NS stages, scores them
// against the rotated query and hands each (row, key) to sink; every key's
// top 11 bits are counted in sm.lh.  NT threads form NT / 256 groups of 8
// warps; group g consumes (and refills) the stages st = g mod NT / 256, each
// warp scoring 16 rows of a 128-row stage.  Returns false after a timed-out
// wait, once the copies still in flight have landed (or their waits ran out).
template <int NS, bool FP8, int NT, bool PAGED, typename Smem, typename Sink>
__device__ __forceinline__ bool stream_scores(Smem &sm, const CUtensorMap *kmap,
                                              const __nv_bfloat16 *__restrict__ q_idx, const Rope &rope,
                                              const DecodeParams &p, int seq, int64_t s_len, int n, int y0,
                                              int64_t c0, Sink &&sink) {
    constexpr int G = NT / 256;
    static_assert(NT % 256 == 0 && NS % G == 0, "whole groups; each slot stays with one group");
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int grp = warp >> 3, gw = warp & 7;            // stage group, warp within the group
    const bool leader = (tid & 255) == 0;
    const int nstages = (n + DM_ROWS - 1) / DM_ROWS;
    constexpr int SB = stage_bytes<FP8>();
    const int pr = PAGED ? p.pg.page_tokens / kBlock : 1;   // rows per page (a power of two)
    const int pshift = PAGED ? p.pg.page_shift - 2 : 0;      // log2(pr)
    const int64_t pg_first = PAGED ? c0 >> pshift : 0;       // the chunk's first page index
    auto issue = [&](int slot, int st2) {   // contiguous: rows y0 + 128 st2 .. as one box (per 64-dim atom)
        mbar_arrive_expect_tx(&sm.full[slot], SB);
        tma_load_2d(sm.stage[slot], kmap, 0, y0 + st2 * DM_ROWS, &sm.full[slot]);
        if constexpr (!FP8) tma_load_2d(sm.stage[slot] + SB / 2, kmap, 64, y0 + st2 * DM_ROWS, &sm.full[slot]);
    };
    // Paged stages are issued by a whole warp: lane ch copies box ch of the
    // stage (cr rows: a page, or 128 rows of one) from its page, so the up to
    // 16 boxes of a stage of small pages go out in parallel; boxes past the
    // chunk's keys are skipped.
    auto issue_paged = [&](int slot, int st2) {
        const int cr = min(DM_ROWS, pr);
        const int ch = lane;
        bool live = ch * cr < DM_ROWS && st2 * DM_ROWS + ch * cr < n;
        int y = 0;
        if (live) {
            const int64_t lr = c0 + (int64_t)st2 * DM_ROWS + ch * cr;
            const int32_t id = sm.pg_ids[(lr >> pshift) - pg_first];
            if (id < 0) {
                flag(p.status, QSA_DEV_BAD_INDEX);
                live = false;
            }
            y = (int)(((int64_t)id << pshift) + (lr & (pr - 1)));
        }
        const uint32_t bytes = __reduce_add_sync(0xffffffffu, live ? (uint32_t)cr * (SB / DM_ROWS) : 0u);
        if (lane == 0) mbar_arrive_expect_tx(&sm.full[slot], bytes);
        __syncwarp();
        if (live) {
            tma_load_2d(sm.stage[slot] + ch * cr * 128, kmap, 0, y, &sm.full[slot]);
            if constexpr (!FP8) tma_load_2d(sm.stage[slot] + SB / 2 + ch * cr * 128, kmap, 64, y, &sm.full[slot]);
        }
    };
    if constexpr (PAGED) {
        // the page ids of the chunk's rows, once, into shared memory (-1: outside the cache)
        const int cnt = (int)(((c0 + n + pr - 1) >> pshift) - pg_first);   // <= the window by the launch plan
        for (int i = tid; i < cnt; i += NT) {
            const int64_t pi = pg_first + i;
            int32_t id = -1;
            if (pi < p.pg.max_pages) {
                id = p.pg.table[(int64_t)seq * p.pg.max_pages + pi];
                if (id < 0 || id >= p.pg.num_pages) id = -1;
            }
            sm.pg_ids[i] = id;
        }
        __syncthreads();
    }
    if constexpr (PAGED) {
        if (tid < 32)
            for (int st = 0; st < min(NS, nstages); ++st) issue_paged(st, st);
    } else if (tid == 0) {
        for (int st = 0; st < min(NS, nstages); ++st) issue(st, st);
    }
    const bool per_head = p.relu || p.head_w;
    // Rotated query heads of the new token (position s_len - 1), rounded to
    // bf16, as the B operand's columns.  BF16 keys: hi/lo bf16 planes of the
    // FP32 head sum, or the 4 heads.  FP8 keys (scored as FP16, which holds
    // every E4M3 value): the same values times 2^qexp, which puts the largest
    // magnitude in [2^14, 2^15), as FP16 -- three pieces that add up to the
    // scaled head sum, or one per head (exact for any bf16 value above 2^-31 of
    // the largest); the scores are scaled back by 2^-qexp.
    const int e = tid;
    float rv[kIdxHeads], hs = 0.0f;
    if (tid < kIdxDim) {
        const int R = rope.rotary_dim, half = R >> 1;
        const __nv_bfloat16 *src = q_idx + (int64_t)seq * kIdxHeads * kIdxDim;
        double cs = 1.0, sn = 0.0;
        int pr = e;
        if (e < R) {
            pr = e < half ? e + half : e - half;
            const double ang = __dmul_rn(__ddiv_rn((double)(s_len - 1), rope.pos_scale),
                                         rope_inv_freq(rope, e < half ? e : e - half));
            sincos(ang, &sn, &cs);
        }
#pragma unroll
        for (int h = 0; h < kIdxHeads; ++h) {
            const double xe = __bfloat162float(src[h * kIdxDim + e]);
            double o = xe;
            if (e < R) {
                const double xp = __bfloat162float(src[h * kIdxDim + pr]);
                o = (e < half) ? __dsub_rn(__dmul_rn(xe, cs), __dmul_rn(xp, sn))
                               : __dadd_rn(__dmul_rn(xe, cs), __dmul_rn(xp, sn));
            }
            rv[h] = __bfloat162float(d2bf(o));
            hs = (h == 0) ? rv[0] : __fadd_rn(hs, rv[h]);
        }
        if constexpr (!FP8) {
            const __nv_bfloat16 zero = __float2bfloat16_rn(0.f);
            if (!per_head) {
                const __nv_bfloat16 hi = __float2bfloat16_rn(hs);
                sm.qcol[0][e] = hi;
                sm.qcol[1][e] = __float2bfloat16_rn(__fsub_rn(hs, __bfloat162float(hi)));
                for (int col = 2; col < 8; ++col) sm.qcol[col][e] = zero;
            } else {
                for (int h = 0; h < kIdxHeads; ++h) sm.qcol[h][e] = __float2bfloat16_rn(rv[h]);
                for (int col = 4; col < 8; ++col) sm.qcol[col][e] = zero;
            }
        } else {
            float m = per_head ? fmaxf(fmaxf(fabsf(rv[0]), fabsf(rv[1])), fmaxf(fabsf(rv[2]), fabsf(rv[3])))
                               : fabsf(hs);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            if (lane == 0) sm.qred[warp] = m;
        }
    }
    if (tid < kIdxHeads) sm.w[tid] = p.head_w ? p.head_w[(int64_t)seq * kIdxHeads + tid] : 1.f;
    float qinv = 1.0f;   // FP8: 2^-qexp
    if constexpr (FP8) {
        __syncthreads();
        const float m = fmaxf(fmaxf(sm.qred[0], sm.qred[1]), fmaxf(sm.qred[2], sm.qred[3]));
        int qexp = 0;
        if (m > 0.0f && m <= 3.0e38f) {
            int ex;
            frexpf(m, &ex);                       // m in [2^(ex-1), 2^ex)
            qexp = min(max(15 - ex, -100), 100);
        }
        qinv = ldexpf(1.0f, -qexp);
        if (tid < kIdxDim) {
            const float sc = ldexpf(1.0f, qexp);
            uint16_t(*q16)[kIdxDim] = reinterpret_cast<uint16_t(*)[kIdxDim]>(&sm.qcol[0][0]);
            if (!per_head) {
                float x = __fmul_rn(hs, sc);
#pragma unroll
                for (int j = 0; j < 3; ++j) {
                    const uint16_t b = f2h_bits(x);
                    q16[j][e] = b;
                    x = __fsub_rn(x, h_bits2f(b));
                }
                for (int col = 3; col < 8; ++col) q16[col][e] = 0;
            } else {
#pragma unroll
                for (int h = 0; h < kIdxHeads; ++h) q16[h][e] = f2h_bits(__fmul_rn(rv[h], sc));
                for (int col = 4; col < 8; ++col) q16[col][e] = 0;
            }
        }
    }
    __syncthreads();
    const int gr = lane >> 2, tq = lane & 3;
    // B fragments.  BF16: k-step kk covers dims 16kk .. 16kk + 15.  FP8: the
    // E4M3 A fragment of a 32-dim block j (4 bytes of dims 32j + 4tq + {0..3}
    // per register, as ldmatrix gives them) widens into two FP16 k16 steps
    // whose k order is a permutation of the block's dims: step 2j takes dims
    // 32j + 4tq + {0..3}, step 2j + 1 dims 32j + 16 + 4tq + {0..3}; the query
    // fragments follow the same order.
    uint32_t qf[8][2];
    {
        const uint32_t *qw = reinterpret_cast<const uint32_t *>(&sm.qcol[gr][0]);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const int d0 = FP8 ? 32 * (kk >> 1) + 16 * (kk & 1) + 4 * tq : 16 * kk + 2 * tq;
            const int d1 = FP8 ? d0 + 2 : d0 + 8;
            qf[kk][0] = qw[d0 >> 1];
            qf[kk][1] = qw[d1 >> 1];
        }
    }
    const float w0 = sm.w[2 * (tq & 1)], w1 = sm.w[2 * (tq & 1) + 1];
    const int mi = lane >> 3, rr = lane & 7;
    const int trow = 16 * gw + rr + 8 * (mi & 1);        // row of this lane's ldmatrix address in the stage
    const uint32_t row_off = (uint32_t)trow * 128u;
    const uint32_t sw = (uint32_t)(trow & 7);
    constexpr uint32_t kAtom = DM_STAGE_BYTES / 2;
    bool ok = true;
    int issued = min(NS, nstages);   // the group's stages below this were issued (leader's count)
    int st = grp;
    for (; st < nstages; st += G) {
        const int slot = st % NS;
        ok = mbar_wait(&sm.full[slot], (st / NS) & 1, p.status);
        if (!ok) break;
        const uint32_t base = smem_u32(sm.stage[slot]);
        float acc[4] = {0.f, 0.f, 0.f, 0.f}, acc2[4] = {0.f, 0.f, 0.f, 0.f};
        if constexpr (FP8) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint32_t r[4], lo[4], hi[4];
                const uint32_t chunk = (uint32_t)(2 * j + (mi >> 1));
                ldsm_x4(base + row_off + ((chunk ^ sw) << 4), r[0], r[1], r[2], r[3]);
#pragma unroll
                for (int i = 0; i < 4; ++i) e4m3x4_to_f16x4(r[i], lo[i], hi[i]);
                mma16816_f16(acc, lo[0], lo[1], hi[0], hi[1], qf[2 * j][0], qf[2 * j][1]);
                mma16816_f16(acc2, lo[2], lo[3], hi[2], hi[3], qf[2 * j + 1][0], qf[2 * j + 1][1]);
            }
        } else {
#pragma unroll
            for (int kk = 0; kk < 8; kk += 2) {
                uint32_t a[4], b[4];
                {
                    const uint32_t chunk = (uint32_t)(2 * (kk & 3) + (mi >> 1));
                    ldsm_x4(base + (kk >> 2) * kAtom + row_off + ((chunk ^ sw) << 4), a[0], a[1], a[2], a[3]);
                }
                {
                    const uint32_t chunk = (uint32_t)(2 * ((kk + 1) & 3) + (mi >> 1));
                    ldsm_x4(base + ((kk + 1) >> 2) * kAtom + row_off + ((chunk ^ sw) << 4), b[0], b[1], b[2],
                            b[3]);
                }
                mma16816(acc, a[0], a[1], a[2], a[3], qf[kk][0], qf[kk][1]);
                mma16816(acc2, b[0], b[1], b[2], b[3], qf[kk + 1][0], qf[kk + 1][1]);
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[i] += acc2[i];
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.empty[slot]);
        float s0, s1;   // rows gr and gr + 8 of this warp's tile
        if (!per_head) {
            s0 = acc[0] + acc[1];
            s1 = acc[2] + acc[3];
            if constexpr (FP8) {   // the third piece is column 2, in lane tq = 1
                s0 += __shfl_xor_sync(0xffffffffu, s0, 1);
                s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
            }
        } else {
            float a0 = acc[0], a1 = acc[1], a2 = acc[2], a3 = acc[3];
            if (p.relu) { a0 = fmaxf(a0, 0.f); a1 = fmaxf(a1, 0.f); a2 = fmaxf(a2, 0.f); a3 = fmaxf(a3, 0.f); }
            s0 = w0 * a0 + w1 * a1;
            s1 = w0 * a2 + w1 * a3;
            s0 += __shfl_xor_sync(0xffffffffu, s0, 1);
            s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
        }
        if constexpr (FP8) {
            s0 = __fmul_rn(s0, qinv);
            s1 = __fmul_rn(s1, qinv);
        }
        const int r0 = st * DM_ROWS + 16 * gw + gr;
        if (tq == 0) {
            if (r0 < n) {
                const uint32_t key = score_key(s0);
                sink(r0, key);
                atomicAdd(&sm.lh[key >> 21], 1u);
            }
            if (r0 + 8 < n) {
                const uint32_t key = score_key(s1);
                sink(r0 + 8, key);
                atomicAdd(&sm.lh[key >> 21], 1u);
            }
        }
        if constexpr (PAGED) {
            if (gw == 0 && st + NS < nstages) {   // the group's first warp refills the slot
                bool okw = true;
                if (lane == 0) okw = ok = mbar_wait(&sm.empty[slot], (st / NS) & 1, p.status);
                if (__shfl_sync(0xffffffffu, okw, 0)) {
                    issue_paged(slot, st + NS);
                    issued = st + NS + 1;
                }
            }
        } else if (leader && st + NS < nstages) {
            ok = mbar_wait(&sm.empty[slot], (st / NS) & 1, p.status);
            if (ok) {
                issue(slot, st + NS);
                issued = st + NS + 1;
            }
        }
    }
    ok = __syncthreads_and(ok);
    if (!ok && leader) {
        // let the copies still in flight land before the shared memory is reused
        for (int s2 = st; s2 < issued; s2 += G) mbar_wait(&sm.full[s2 % NS], (s2 / NS) & 1, p.status);
    }
    return ok;
}

template <bool FP8>
struct DecodeMmaSmem {
    static constexpr int NS = FP8 ? DM_NS_FP8 : DM_NS;
    alignas(1024) uint8_t stage[NS][stage_bytes<FP8>()];
    alignas(16) __nv_bfloat16 qcol[8][kIdxDim];   // B operand source: 8 columns x 128 dims (FP8: as FP16)
    float w[kIdxHeads];
    float qred[4];                                 // FP8: per-warp largest query magnitude
    uint64_t full[NS], empty[NS];
    uint32_t lh[2048];                             // local histogram of the keys' top 11 bits
    int32_t pg_ids[DM_PG_IDS];                     // paged: page ids of the chunk's rows
};

// Scorer of the two-kernel path: keys to the workspace, histogram added into
// the sequence's global histogram.  PAGED: paged compressed keys (p.pg).
template <bool FP8, bool PAGED>
__global__ void __launch_bounds__(DI_THREADS, 2)
    decode_score_mma_kernel(const __grid_constant__ CUtensorMap kmap, const __nv_bfloat16 *__restrict__ q_idx,
                            Rope rope, DecodeParams p) {
    extern __shared__ uint8_t dsm_raw[];
    DecodeMmaSmem<FP8> &sm = *reinterpret_cast<DecodeMmaSmem<FP8> *>(
        (reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
    pdl_wait();      // the compressed keys come from the previous kernel (ring pooling)
    pdl_trigger();
    const int seq = blockIdx.y, c = blockIdx.x;
    const int tid = threadIdx.x;
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
    if (tid == 0) {
        for (int s = 0; s < DecodeMmaSmem<FP8>::NS; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 8);   // the warps of the stage's group
        }
        fence_mbar_init();
        prefetch_tmap(&kmap);
    }
    __syncthreads();
    const bool ok = stream_scores<DecodeMmaSmem<FP8>::NS, FP8, DI_THREADS, PAGED>(sm, &kmap, q_idx, rope, p, seq, s_len, n,
                                              (int)(seq * p.pool_stride + c0), c0,
                                         [&](int r, uint32_t key) { gkeys[r] = key; });
    if (!ok) return;
    flush_hist(sm.lh, p.hist + (int64_t)seq * 2048);
}

// ---------------------------------------------------------------------------
// Selection from the score keys, one thread-block cluster per sequence.
//
// Every CTA owns a chunk of a sequence's keys (whole tiles of NT * 16 keys, 16
// contiguous keys per thread).  With the histogram of the keys' top 11 bits,
// the bin d1 that holds the k-th largest key is known before any key is read.
// Each CTA writes to its own shared memory, in block order, the ids of its
// keys above bin d1 (all of them are selected; fewer than k in the whole
// sequence) and the (key, id) pairs of its keys in bin d1 (the candidates;
// past the shared-memory capacity they go to a global overflow area).  After
// a cluster barrier, CTA 0 gathers the lists through distributed shared
// memory, resolves the remaining 21 bits of K* on the candidates, keeps the
// candidates above K* and the first ones equal to K* (ties to the lower block
// id), and merges that list with the above-bin ids into the ascending output.
//
// Two kernels use it: decode_select_kernel reads the keys and the histogram
// that decode_score_*_kernel wrote to the workspace; decode_index_fused_kernel
// scores, keeps its chunk's keys in shared memory and merges the CTAs'
// histograms through distributed shared memory, with no workspace round trip.
// ---------------------------------------------------------------------------
constexpr int DS_THREADS = 512;
constexpr int DS_PER_THREAD = 16;
constexpr int DS_TILE = DS_THREADS * DS_PER_THREAD;   // keys per CTA tile of decode_select_kernel
constexpr int DS_CLUSTER = 16;                        // CTAs (chunks) per sequence at most (non-portable above 8)
constexpr int DS_LCAND = 2048;                        // candidates a CTA keeps in shared memory
constexpr int DS_CAND_SMEM = 4096;                    // candidates CTA 0 stages in shared memory
constexpr int DS_MAX_K = 2048;                        // largest top_k

struct SelectArgs {
    const int32_t *seq_len;
    int64_t pool_stride, max_blocks, kstride, chunk;   // chunk: keys per CTA (whole tiles for the select kernel)
    int gmax, top_k;                                    // gmax: CTAs per cluster (<= DS_CLUSTER)
    const uint32_t *keys;   // [B][kstride] score keys (select kernel)
    uint32_t *hist;         // [B][2048] histogram of the keys' top 11 bits (select kernel; cleared after use)
    uint2 *cand;            // [B][kstride]: chunk g's candidates past DS_LCAND, at g * chunk + position
    int32_t *sel, *nsel;
    unsigned *status;
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
    uint32_t htotal;                    // select kernel: sum of the scorer's histogram
    uint32_t aoff[DS_CLUSTER + 1];      // prefix of the above counts per chunk
    uint32_t coff[DS_CLUSTER + 1];      // prefix of the candidate counts per chunk
    uint32_t wsum[32];
};

__device__ __forceinline__ int64_t visible_blocks(const int32_t *seq_len, int64_t pool_stride, int64_t max_blocks,
                                                  int seq) {
    const int64_t s_len = seq_len[seq];
    const int64_t nb = s_len / kBlock;
    return (s_len < 1 || nb > pool_stride || nb > max_blocks) ? 0 : nb;   // flagged by the scorer
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

// This CTA's lists from its keys [c0, c1): tiles of NT * 16 keys, thread t
// holding keys [16t, 16t + 16) of a tile.  k/m hold the first tile's keys
// (already loaded by the caller); load(i0, k) loads the next ones.
template <int NT, typename Load>
__device__ __forceinline__ void build_lists(DsSmem &sm, Load &&load, int64_t c0, int64_t c1, uint32_t d1, int top_k,
                                            uint2 *cand_seq, uint32_t (&k)[16], int m) {
    const int tid = threadIdx.x;
    uint32_t na_run = 0, nc_run = 0;
    for (int64_t t0 = c0; t0 < c1; t0 += (int64_t)NT * DS_PER_THREAD) {
        const int64_t i0 = t0 + (int64_t)DS_PER_THREAD * tid;
        if (t0 != c0) m = load(i0, k);
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
}

// CTA 0 of the cluster, after the lists of the gseq CTAs with keys are complete.
template <int NT>
__device__ __forceinline__ void select_leader(DsSmem &sm, int gseq, uint32_t d1, int k_rem1, int64_t nb,
                                              int64_t chunk, const uint2 *cand_seq, int top_k, int32_t *out,
                                              int32_t *nsel_out) {
    const int tid = threadIdx.x;
    // per-chunk offsets of the above ids and of the candidates: lane c reads
    // CTA c's counts (all at once), an exclusive warp scan gives the offsets
    if (tid < 32) {
        const int lane = tid;
        uint32_t na = 0, nc = 0;
        if (lane < gseq) {
            na = ld_dsmem(dsmem_addr(&sm.my_na, lane));
            nc = ld_dsmem(dsmem_addr(&sm.my_nc, lane));
        }
        uint32_t ia = na, ic = nc;   // inclusive scans
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t va = __shfl_up_sync(0xffffffffu, ia, o), vc = __shfl_up_sync(0xffffffffu, ic, o);
            if (lane >= o) { ia += va; ic += vc; }
        }
        if (lane < gseq) { sm.aoff[lane] = ia - na; sm.coff[lane] = ic - nc; }
        if (lane == gseq - 1) { sm.aoff[gseq] = ia; sm.coff[gseq] = ic; }
    }
    __syncthreads();
    const int na_all = (int)min(sm.aoff[gseq], (uint32_t)(top_k - 1));
    const int nc_all = (int)min((int64_t)sm.coff[gseq], nb);
    const bool small = nc_all <= DS_CAND_SMEM;
    for (int j = tid; j < na_all; j += NT) {
        const int c = chunk_of(sm.aoff, gseq, (uint32_t)j);
        sm.alist[j] = (int32_t)ld_dsmem(dsmem_addr(&sm.my_above[j - sm.aoff[c]], c));
    }
    auto fetch = [&](int j) -> uint2 {           // candidate j of the sequence, block order
        const int c = chunk_of(sm.coff, gseq, (uint32_t)j);
        const uint32_t jj = (uint32_t)j - sm.coff[c];
        if (jj < (uint32_t)DS_LCAND)
            return make_uint2(ld_dsmem(dsmem_addr(&sm.my_ck[jj], c)), ld_dsmem(dsmem_addr(&sm.my_ci[jj], c)));
        return __ldcg(cand_seq + (int64_t)c * chunk + jj);
    };
    if (small)
        for (int j = tid; j < nc_all; j += NT) {
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
        for (int b = tid; b < nbins; b += NT) sm.s.hist[b] = 0;
        __syncthreads();
        for (int j = tid; j < nc_all; j += NT) {
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
    // Thread t takes a contiguous run of cpt candidates per round of NT * cpt.
    int ns = 0;     // CTA-uniform running count
    uint32_t eq_run = 0;
    const int cpt = min(8, max(1, (nc_all + NT - 1) / NT));
    for (int base = 0; base < nc_all; base += NT * cpt) {
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
    for (int j = tid; j < na_all; j += NT) {
        const int32_t v = sm.alist[j];
        const int pos = j + count_below(sm.slist, ns, v);
        if (pos < top_k) out[pos] = v;
    }
    for (int j = tid; j < ns; j += NT) {
        const int32_t v = sm.slist[j];
        const int pos = j + count_below(sm.alist, na_all, v);
        if (pos < top_k) out[pos] = v;
    }
    const int cnt = na_all + ns;
    for (int i = cnt + tid; i < top_k; i += NT) out[i] = -1;
    if (tid == 0) *nsel_out = cnt;
}

// Every visible block selected (nb <= top_k): ids in order, padded with -1.
template <int NT>
__device__ __forceinline__ void select_all(int64_t c0, int64_t c1, int64_t nb, int top_k, uint32_t rank,
                                           int32_t *out, int32_t *nsel_out) {
    for (int64_t i = c0 + threadIdx.x; i < c1; i += NT) out[i] = (int32_t)i;
    if (rank == 0) {
        for (int i = (int)nb + threadIdx.x; i < top_k; i += NT) out[i] = -1;
        if (threadIdx.x == 0) *nsel_out = (int)nb;
    }
}

__global__ void __launch_bounds__(DS_THREADS)
    decode_select_kernel(SelectArgs a) {
    extern __shared__ __align__(16) uint8_t ds_raw[];
    DsSmem &sm = *reinterpret_cast<DsSmem *>(ds_raw);
    pdl_wait();
    pdl_trigger();
    const int seq = blockIdx.y, tid = threadIdx.x;
    const uint32_t rank = cluster_rank();             // = blockIdx.x: a cluster spans the x extent
    const int64_t nb = visible_blocks(a.seq_len, a.pool_stride, a.max_blocks, seq);
    const int top_k = a.top_k;
    int32_t *out = a.sel + (int64_t)seq * top_k;
    const int64_t c0 = (int64_t)rank * a.chunk, c1 = min(c0 + a.chunk, nb);
    uint32_t *ghist = a.hist + (int64_t)seq * 2048;  // the scorer's counts; zero again when this kernel ends
    if (nb <= top_k) {                               // the whole cluster takes this branch
        select_all<DS_THREADS>(c0, c1, nb, top_k, rank, out, a.nsel + seq);
        if (rank == 0) reinterpret_cast<uint4 *>(ghist)[tid] = make_uint4(0u, 0u, 0u, 0u);
        return;
    }
    const int gseq = (int)((nb + a.chunk - 1) / a.chunk);   // CTAs with keys (<= cluster size)
    const uint32_t *row = a.keys + (int64_t)seq * a.kstride;
    uint2 *cand_seq = a.cand + (int64_t)seq * a.kstride;
    // first tile's keys in flight before the histogram is read
    uint32_t k[16];
    const int m = load16(row, c0 + (int64_t)DS_PER_THREAD * tid, c1, a.kstride, k);
    // bin of the k-th largest key from the scorer's histogram
    static_assert(DS_THREADS * 4 == 2048, "one 16-byte histogram load per thread");
    const uint4 hv = __ldcg(reinterpret_cast<const uint4 *>(ghist) + tid);
    reinterpret_cast<uint4 *>(sm.s.hist)[tid] = hv;
    if (tid == 0) { sm.s.digit = 0; sm.s.k_rem = 1; sm.htotal = 0; }
    __syncthreads();
    if (rank == 0) {   // the counts must add up to the keys scored: else the workspace was not zero
        uint32_t part = hv.x + hv.y + hv.z + hv.w;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        if ((tid & 31) == 0) atomicAdd(&sm.htotal, part);
    }
    sel_find_digit(sm.s, 2048, top_k);
    const uint32_t d1 = (uint32_t)sm.s.digit;
    const int k_rem1 = sm.s.k_rem;
    build_lists<DS_THREADS>(
        sm, [&](int64_t i0, uint32_t (&kk)[16]) { return load16(row, i0, c1, a.kstride, kk); }, c0, c1, d1, top_k,
        cand_seq, k, m);
    cluster_sync();                                  // every CTA's lists are complete (and has read ghist)
    if (rank == 0) {
        reinterpret_cast<uint4 *>(ghist)[tid] = make_uint4(0u, 0u, 0u, 0u);
        if (tid == 0 && sm.htotal != (uint32_t)nb) flag(a.status, QSA_DEV_WORKSPACE);
        select_leader<DS_THREADS>(sm, gseq, d1, k_rem1, nb, a.chunk, cand_seq, top_k, out, a.nsel + seq);
    }
    cluster_sync();                                  // CTA 0 has finished reading the others' lists
}

// ---------------------------------------------------------------------------
// Fused decode indexer (bf16): scorer and selection in one cluster kernel.
// One cluster of up to 16 CTAs per sequence, one CTA per SM; each CTA streams
// its chunk of compressed keys (4 stages in flight, two groups of 8 warps
// taking alternate stages) and keeps the chunk's score
// keys in shared memory.  The CTAs' histograms are summed through distributed
// shared memory (CTA r sums a slice of bins over the cluster and writes the
// sums into every CTA), then the selection above runs on the resident keys.
// ---------------------------------------------------------------------------
constexpr int DF_NS = 4;              // stages in flight per CTA
constexpr int DF_NS_FP8 = 8;          // FP8 stages are half the bytes
template <bool FP8> __host__ __device__ constexpr int fused_stages() { return FP8 ? DF_NS_FP8 : DF_NS; }
constexpr int DF_KEYS = 16384;        // keys a CTA keeps in shared memory
constexpr int DF_THREADS = 512;      // two stage groups of 8 warps

template <bool FP8>
struct FusedSmem {
    union {
        struct {
            uint8_t stage[fused_stages<FP8>()][stage_bytes<FP8>()];     // while streaming
        } st;
        DsSmem ds;                              // selection, once every stage has been consumed
    } u;
    uint32_t skeys[DF_KEYS];
    uint32_t lh[2048];
    alignas(16) __nv_bfloat16 qcol[8][kIdxDim];
    float w[kIdxHeads];
    float qred[4];
    uint64_t full[fused_stages<FP8>()], empty[fused_stages<FP8>()];
    int32_t pg_ids[DF_KEYS / 8];                // paged: page ids of the chunk's rows (pages of >= 8 rows)
};
// The streaming interface of FusedSmem (stage, qcol, w, qred, full, empty, lh).
template <bool FP8>
struct FusedStream {
    uint8_t (&stage)[fused_stages<FP8>()][stage_bytes<FP8>()];
    __nv_bfloat16 (&qcol)[8][kIdxDim];
    float (&w)[kIdxHeads];
    float (&qred)[4];
    uint64_t (&full)[fused_stages<FP8>()];
    uint64_t (&empty)[fused_stages<FP8>()];
    uint32_t (&lh)[2048];
    int32_t (&pg_ids)[DF_KEYS / 8];
};

template <bool FP8, bool PAGED>
__global__ void __launch_bounds__(DF_THREADS, 1)
    decode_index_fused_kernel(const __grid_constant__ CUtensorMap kmap, const __nv_bfloat16 *__restrict__ q_idx,
                              Rope rope, DecodeParams p, SelectArgs a) {
    extern __shared__ uint8_t dsm_raw[];
    FusedSmem<FP8> &sm = *reinterpret_cast<FusedSmem<FP8> *>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) &
                                                             ~uintptr_t(1023));
    pdl_wait();      // the compressed keys come from the previous kernel (ring pooling)
    pdl_trigger();
    const int seq = blockIdx.y, tid = threadIdx.x;
    const uint32_t rank = cluster_rank();             // = blockIdx.x: a cluster spans the x extent
    const int ncta = (int)a.gmax;
    const int64_t s_len = p.seq_len[seq];
    const int64_t nb = visible_blocks(a.seq_len, a.pool_stride, a.max_blocks, seq);
    if ((s_len < 1 || s_len / kBlock > p.pool_stride || s_len / kBlock > p.max_blocks) && tid == 0 && rank == 0)
        flag(p.status, QSA_DEV_BAD_LENGTH);
    const int top_k = a.top_k;
    int32_t *out = a.sel + (int64_t)seq * top_k;
    const int64_t c0 = (int64_t)rank * a.chunk, c1 = min(c0 + a.chunk, nb);
    if (nb <= top_k) {                               // the whole cluster takes this branch; no scores needed
        select_all<DF_THREADS>(c0, c1, nb, top_k, rank, out, a.nsel + seq);
        return;
    }
    const int gseq = (int)((nb + a.chunk - 1) / a.chunk);
    const int n = (int)(c1 > c0 ? c1 - c0 : 0);      // <= DF_KEYS by the launch plan
    uint2 *cand_seq = a.cand + (int64_t)seq * a.kstride;
    for (int b = tid; b < 2048; b += DF_THREADS) sm.lh[b] = 0;
    if (tid == 0) {
        for (int s = 0; s < fused_stages<FP8>(); ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 8);   // the warps of the stage's group
        }
        fence_mbar_init();
        prefetch_tmap(&kmap);
    }
    __syncthreads();
    bool ok = true;
    if (n > 0) {
        FusedStream<FP8> fs{sm.u.st.stage, sm.qcol, sm.w, sm.qred, sm.full, sm.empty, sm.lh, sm.pg_ids};
        ok = stream_scores<fused_stages<FP8>(), FP8, DF_THREADS, PAGED>(fs, &kmap, q_idx, rope, p, seq, s_len, n,
                                                                 (int)(seq * p.pool_stride + c0), c0,
                                  [&](int r, uint32_t key) { sm.skeys[r] = key; });
    }
    (void)ok;   // a timed-out wait is in the status word; the cluster still runs every barrier
    __syncthreads();
    cluster_sync();                                  // every CTA's histogram is complete; stages are free
    // sequence histogram: CTA r sums bins [r * per, (r + 1) * per) over the cluster
    const int per = (2048 + ncta - 1) / ncta;
    for (int b = (int)rank * per + tid; b < min(2048, ((int)rank + 1) * per); b += DF_THREADS) {
        uint32_t sum = 0;
        for (int c = 0; c < ncta; ++c) sum += ld_dsmem(dsmem_addr(&sm.lh[b], (uint32_t)c));
        for (int c = 0; c < ncta; ++c) st_dsmem(dsmem_addr(&sm.u.ds.s.hist[b], (uint32_t)c), sum);
    }
    DsSmem &ds = sm.u.ds;
    if (tid == 0) { ds.s.digit = 0; ds.s.k_rem = 1; }
    cluster_sync();                                  // every CTA holds the sequence histogram
    sel_find_digit(ds.s, 2048, top_k);
    const uint32_t d1 = (uint32_t)ds.s.digit;
    const int k_rem1 = ds.s.k_rem;
    auto load_sm = [&](int64_t i0, uint32_t (&kk)[16]) -> int {
        const int64_t m0 = c1 - i0;
        const int m = m0 <= 0 ? 0 : (m0 >= 16 ? 16 : (int)m0);
        const uint4 *src = reinterpret_cast<const uint4 *>(&sm.skeys[i0 - c0]);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (4 * j < m) v = src[j];
            kk[4 * j] = v.x; kk[4 * j + 1] = v.y; kk[4 * j + 2] = v.z; kk[4 * j + 3] = v.w;
        }
        return m;
    };
    uint32_t k[16];
    const int m = load_sm(c0 + (int64_t)DS_PER_THREAD * tid, k);
    build_lists<DF_THREADS>(ds, load_sm, c0, c1, d1, top_k, cand_seq, k, m);
    cluster_sync();                                  // every CTA's lists are complete
    if (rank == 0) select_leader<DF_THREADS>(ds, gseq, d1, k_rem1, nb, a.chunk, cand_seq, top_k, out, a.nsel + seq);
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

// Fused path: C CTAs per sequence (one cluster), chunks of at most DF_KEYS
// keys, used when B x C CTAs (one per SM) cover at least half the SMs and all
// B clusters can be resident together.
struct FusedPlan {
    bool use;
    int C;
    int64_t chunk;
};

// Clusters of C fused CTAs that can be resident at once (queried once per C).
template <bool FP8>
int fused_active_clusters(int C) {
    static int ok[DS_CLUSTER + 1];
    static bool init = false;
    if (!init) {
        for (int i = 0; i <= DS_CLUSTER; ++i) ok[i] = -1;
        init = true;
    }
    if (C < 1 || C > DS_CLUSTER) return 0;
    if (ok[C] < 0) {
        ok[C] = 0;
        const size_t smem = sizeof(FusedSmem<FP8>) + 1024;
        if (cudaFuncSetAttribute(decode_index_fused_kernel<FP8, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem) == cudaSuccess &&
            (C <= 8 || cudaFuncSetAttribute(decode_index_fused_kernel<FP8, false>,
                                            cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess)) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3((unsigned)C, 1, 1);
            cfg.blockDim = dim3(DF_THREADS, 1, 1);
            cfg.dynamicSmemBytes = smem;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = (unsigned)C;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, decode_index_fused_kernel<FP8, false>, &cfg) == cudaSuccess && n > 0)
                ok[C] = n;
        }
        cudaGetLastError();   // a refused query leaves no sticky error
    }
    return ok[C];
}

FusedPlan fused_plan(int B, int64_t max_blocks, bool bf16, bool fp8) {
    FusedPlan f{false, 1, DF_KEYS};
    const DeviceInfo *di = device_info();
    const int64_t sms = di ? di->sm_count : 148;
    if (!bf16 || B < 1 || max_blocks < 1) return f;
    const int64_t cmin = (max_blocks + DF_KEYS - 1) / DF_KEYS;
    if (cmin > DS_CLUSTER) return f;
    int64_t C = std::max<int64_t>(cmin, std::min<int64_t>(DS_CLUSTER, sms / B));
    int64_t chunk = (max_blocks + C - 1) / C;
    chunk = (chunk + DM_ROWS - 1) / DM_ROWS * DM_ROWS;          // <= DF_KEYS: C >= cmin
    C = (max_blocks + chunk - 1) / chunk;
    f.C = (int)C;
    f.chunk = chunk;
    // one wave of clusters: a sequence whose cluster waited for a free GPC
    // would stream after the others with a fraction of the bandwidth
    f.use = (int64_t)B * C >= sms / 2 &&
            (fp8 ? fused_active_clusters<true>((int)C) : fused_active_clusters<false>((int)C)) >= B;
    return f;
}

// Workspace: keys [B][kstride] u32 | cand overflow [B][kstride] uint2 | hist [B][2048] u32
struct DecodeWs {
    uint32_t *keys;
    uint2 *cand;
    uint32_t *hist;
    size_t hist_bytes;   // zero between calls: the select kernel clears what the scorer added
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
    d.hist_bytes = (size_t)B * 2048 * 4;
    off += r256(d.hist_bytes);
    d.total = off;
    return d;
}
}  // namespace

int decode_index_kernel_count(int B, int64_t max_blocks, bool bf16, bool fp8) {
    return fused_plan(B, std::max<int64_t>(max_blocks, 1), bf16, fp8).use ? 1 : 2;
}

size_t decode_index_ws_bytes(int B, int64_t max_blocks, int top_k, bool bf16) {
    (void)bf16;
    return decode_ws(nullptr, B, max_blocks, top_k).total;
}

cudaError_t launch_decode_index(const void *q_idx, const void *k_pool, const float *head_w,
                                const int32_t *seq_len, int B, int64_t pool_stride, int64_t max_blocks,
                                int top_k, int32_t *sel, int32_t *nsel, void *ws, Rope rope, bool relu,
                                bool bf16, bool fp8, const Paging &pg, unsigned *status, cudaStream_t s) {
    if (fp8 && !bf16) return cudaErrorInvalidValue;
    const int64_t kstride = key_stride(max_blocks);
    const DecodeWs d = decode_ws(ws, B, max_blocks, top_k);
    const FusedPlan fp = fused_plan(B, max_blocks, bf16, fp8);
    // the compressed keys as one 2-D tensor: B * pool_stride rows, or the paged
    // cache's num_pages * page_tokens / 4 rows read in boxes of one page (<= 128 rows)
    const uint64_t map_rows = pg.table ? (uint64_t)pg.num_pages * (pg.page_tokens / kBlock) : (uint64_t)B * pool_stride;
    const int box_rows = pg.table ? std::min(DM_ROWS, pg.page_tokens / kBlock) : DM_ROWS;
    if (fp.use) {
        CUtensorMap kmap;
        if (!make_kpool_map(&kmap, k_pool, map_rows, fp8, box_rows)) return cudaErrorInvalidValue;
        DecodeParams p{seq_len, head_w, pool_stride, max_blocks, fp.chunk, kstride, fp.C, top_k, relu ? 1 : 0,
                       d.keys, d.hist, status, pg};
        SelectArgs sa{seq_len, pool_stride, max_blocks, kstride, fp.chunk, fp.C, top_k, d.keys, d.hist, d.cand,
                      sel, nsel, status};
        auto kern = fp8 ? (pg.table ? decode_index_fused_kernel<true, true> : decode_index_fused_kernel<true, false>)
                        : (pg.table ? decode_index_fused_kernel<false, true> : decode_index_fused_kernel<false, false>);
        const size_t smem = (fp8 ? sizeof(FusedSmem<true>) : sizeof(FusedSmem<false>)) + 1024;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        if (fp.C > 8) {
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
            if (e != cudaSuccess) return e;
        }
        return launch_pdl_cluster(kern, dim3((unsigned)fp.C, (unsigned)B), dim3(DF_THREADS), smem, (unsigned)fp.C, s,
                                  kmap, (const __nv_bfloat16 *)q_idx, rope, p, sa);
    }
    DecodePlan pl = decode_index_plan(B, max_blocks, bf16);
    if (pg.table) {   // a scorer CTA keeps the page ids of its chunk: at most DM_PG_IDS pages
        const int64_t pr = pg.page_tokens / kBlock;
        const int64_t cap = std::max<int64_t>(DM_ROWS, (DM_PG_IDS - 2) * pr / DM_ROWS * DM_ROWS);
        if (pl.chunk > cap) {
            pl.chunk = cap;
            pl.chunks = (int)((max_blocks + cap - 1) / cap);
        }
    }
    cudaError_t e;
    DecodeParams p{seq_len, head_w, pool_stride, max_blocks, pl.chunk, kstride, pl.chunks, top_k, relu ? 1 : 0,
                   d.keys, d.hist, status, pg};
    dim3 grid((unsigned)pl.chunks, (unsigned)B);
    if (bf16) {
        CUtensorMap kmap;
        if (!make_kpool_map(&kmap, k_pool, map_rows, fp8, box_rows)) return cudaErrorInvalidValue;
        auto kern = fp8 ? (pg.table ? decode_score_mma_kernel<true, true> : decode_score_mma_kernel<true, false>)
                        : (pg.table ? decode_score_mma_kernel<false, true> : decode_score_mma_kernel<false, false>);
        const size_t smem = (fp8 ? sizeof(DecodeMmaSmem<true>) : sizeof(DecodeMmaSmem<false>)) + 1024;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        e = launch_pdl(kern, grid, dim3(DI_THREADS), smem, s, kmap, (const __nv_bfloat16 *)q_idx, rope, p);
        if (e != cudaSuccess) return e;
    } else {
        const size_t smem = DI_NS * DI_STAGE_BYTES;
        e = cudaFuncSetAttribute(decode_score_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        e = launch_pdl(decode_score_kernel<float>, grid, dim3(DI_THREADS), smem, s, (const float *)q_idx,
                       (const float *)k_pool, rope, p);
        if (e != cudaSuccess) return e;
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const SelectLayout l = select_layout(max_blocks);
    SelectArgs sa{seq_len, pool_stride, max_blocks, kstride, l.chunk, l.gmax, top_k, d.keys, d.hist, d.cand, sel,
                  nsel, status};
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
