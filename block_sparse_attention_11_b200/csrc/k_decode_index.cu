// k_decode_index.cu -- decode indexer: scan all compressed keys of each
// sequence for its one new query, keep the top-k blocks.
//
// Page "Qwen3.8-Flash-Next: Day-0 Support in SGLang", section "IndexShare MTP":
// the decode scorer reads all ceil(L/4) compressed blocks and, beyond a few
// thousand tokens, sets the cost of the layer.  So this is an HBM-streaming
// kernel: each CTA owns a contiguous chunk of one sequence's compressed keys,
// pulls it through shared memory with 16 KB bulk TMA copies (4 in flight),
// computes the scores with warp-level fp32 dot products, keeps them in shared
// memory, and selects the chunk's local top-k there.  A second kernel merges
// the chunks of each sequence.  Any block of the global top-k is in its
// chunk's local top-k under the same (score desc, id asc) order, so the merge
// is exact; chunks are consecutive id ranges and local lists are ascending,
// so concatenating them keeps ascending id order for the tie rule.
#include <algorithm>

#include "internal.h"
#include "select.cuh"

namespace qsa {

namespace {

constexpr int DI_THREADS = 256;
constexpr int DI_NS = 4;
constexpr int DI_STAGE_BYTES = 16384;
constexpr int64_t DI_MAX_CHUNK = 16384;     // scores of one chunk live in smem (64 KB)
constexpr int DI_MERGE_CAP = 24576;         // candidates one merge CTA holds (key + id = 192 KB)
constexpr int DI_MERGE_THREADS = 1024;

struct DecodeParams {
    const int32_t *seq_len;
    const float *head_w;
    int64_t pool_stride, max_blocks, chunk;
    int chunks, top_k, relu;
    uint32_t *cand_key;
    int32_t *cand_idx;
    int32_t *cand_cnt;
    unsigned *status;
};

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
    uint32_t *keys = reinterpret_cast<uint32_t *>(dsm + DI_NS * DI_STAGE_BYTES);
    __shared__ uint64_t full[DI_NS];
    __shared__ float qh[kIdxHeads][kIdxDim];
    __shared__ float qsum[kIdxDim];
    __shared__ SelectSmem sm;

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
    const int64_t cbase = ((int64_t)seq * p.chunks + c) * p.top_k;
    if (n == 0) {
        if (tid == 0) p.cand_cnt[(int64_t)seq * p.chunks + c] = 0;
        return;
    }
    const int nstages = (n + SROWS - 1) / SROWS;
    const T *kbase = k_pool + ((int64_t)seq * p.pool_stride + c0) * kIdxDim;
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
            if (live && sub == 0) keys[st * SROWS + r] = score_key(score);
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
    uint32_t *ck = p.cand_key + cbase;
    int32_t *ci = p.cand_idx + cbase;
    const int cnt = cta_topk(keys, n, p.top_k, sm, [&](int pos, int i) {
        ck[pos] = keys[i];
        ci[pos] = (int32_t)(c0 + i);
    });
    if (tid == 0) p.cand_cnt[(int64_t)seq * p.chunks + c] = cnt;
}

// bf16 scorer on the tensor cores.  A 128-key stage arrives by two tensor
// TMA loads (64 dims x 128 keys each, 128-byte swizzle) so ldmatrix reads are
// conflict-free; each warp scores one 16-key tile per stage with 8
// m16n8k16 MMAs: A = keys (16 keys x 16 dims), B = the query as 8 columns
// (hi and lo planes of the FP32 head sum, or the 4 heads), FP32 accumulate.
constexpr int DM_ROWS = 128;                       // keys per stage
constexpr int DM_NS = 2;                           // stages in flight per CTA (2 CTAs per SM)
constexpr int DM_STAGE_BYTES = DM_ROWS * 256;      // two 64-dim k-atoms of 128 rows x 128 B

struct DecodeMmaSmem {
    alignas(1024) uint8_t stage[DM_NS][DM_STAGE_BYTES];
    alignas(16) __nv_bfloat16 qcol[8][kIdxDim];   // B operand source: 8 columns x 128 dims
    float w[kIdxHeads];
    uint64_t full[DM_NS], empty[DM_NS];
    SelectSmem sel;
};

__global__ void __launch_bounds__(DI_THREADS, 2)
    decode_score_mma_kernel(const __grid_constant__ CUtensorMap kmap, const __nv_bfloat16 *__restrict__ q_idx,
                            Rope rope, DecodeParams p) {
    extern __shared__ uint8_t dsm_raw[];
    DecodeMmaSmem &sm = *reinterpret_cast<DecodeMmaSmem *>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) &
                                                           ~uintptr_t(1023));
    uint32_t *keys = reinterpret_cast<uint32_t *>(reinterpret_cast<uint8_t *>(&sm) + sizeof(DecodeMmaSmem));
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
    const int64_t cbase = ((int64_t)seq * p.chunks + c) * p.top_k;
    if (n == 0) {
        if (tid == 0) p.cand_cnt[(int64_t)seq * p.chunks + c] = 0;
        return;
    }
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
            if (r0 < n) keys[r0] = score_key(s0);
            if (r0 + 8 < n) keys[r0 + 8] = score_key(s1);
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
    uint32_t *ck = p.cand_key + cbase;
    int32_t *ci = p.cand_idx + cbase;
    const int cnt = cta_topk(keys, n, p.top_k, sm.sel, [&](int pos, int i) {
        ck[pos] = keys[i];
        ci[pos] = (int32_t)(c0 + i);
    });
    if (tid == 0) p.cand_cnt[(int64_t)seq * p.chunks + c] = cnt;
}

__global__ void __launch_bounds__(DI_MERGE_THREADS) decode_merge_kernel(DecodePlan plan, int top_k,
                                                                         const uint32_t *__restrict__ cand_key,
                                                                         const int32_t *__restrict__ cand_idx,
                                                                         const int32_t *__restrict__ cand_cnt,
                                                                         int32_t *__restrict__ sel,
                                                                         int32_t *__restrict__ nsel) {
    extern __shared__ __align__(16) uint32_t msm[];
    __shared__ int off[65];
    __shared__ SelectSmem sm;
    const int seq = blockIdx.x, tid = threadIdx.x;
    const int C = plan.chunks;
    const int cap = C * top_k;
    uint32_t *keys = msm;
    int32_t *ids = reinterpret_cast<int32_t *>(msm + cap);
    if (tid == 0) {
        int a = 0;
        for (int c = 0; c < C; ++c) { off[c] = a; a += cand_cnt[(int64_t)seq * C + c]; }
        off[C] = a;
    }
    __syncthreads();
    const int total = off[C];
    const int64_t base = (int64_t)seq * C * top_k;
    for (int f = tid; f < cap; f += blockDim.x) {
        const int c = f / top_k, i = f % top_k;
        if (off[c] + i < off[c + 1]) {
            keys[off[c] + i] = cand_key[base + f];
            ids[off[c] + i] = cand_idx[base + f];
        }
    }
    __syncthreads();
    int32_t *out = sel + (int64_t)seq * top_k;
    const int cnt = cta_topk(keys, total, top_k, sm, [&](int pos, int i) { out[pos] = ids[i]; });
    for (int i = cnt + tid; i < top_k; i += blockDim.x) out[i] = -1;
    if (tid == 0) nsel[seq] = cnt;
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

}  // namespace

DecodePlan decode_index_plan(int B, int64_t max_blocks, bool bf16) {
    (void)bf16;
    const DeviceInfo *di = device_info();
    const int sms = di ? di->sm_count : 148;
    DecodePlan pl;
    int64_t C = std::max<int64_t>(1, (2 * sms) / std::max(B, 1));
    C = std::min<int64_t>(C, std::max<int64_t>(1, (max_blocks + 255) / 256));
    int64_t chunk = (max_blocks + C - 1) / C;
    chunk = std::max<int64_t>(128, (chunk + 127) / 128 * 128);
    if (chunk > DI_MAX_CHUNK) chunk = DI_MAX_CHUNK;
    C = std::max<int64_t>(1, (max_blocks + chunk - 1) / chunk);
    pl.chunks = (int)C;
    pl.chunk = chunk;
    return pl;
}

size_t decode_index_ws_bytes(int B, int64_t max_blocks, int top_k, bool bf16) {
    const DecodePlan pl = decode_index_plan(B, max_blocks, bf16);
    const size_t n = (size_t)B * pl.chunks * top_k;
    size_t bytes = n * sizeof(uint32_t);
    bytes = (bytes + 255) / 256 * 256;
    bytes += (n * sizeof(int32_t) + 255) / 256 * 256;
    bytes += ((size_t)B * pl.chunks * sizeof(int32_t) + 255) / 256 * 256;
    return bytes;
}

cudaError_t launch_decode_index(const void *q_idx, const void *k_pool, const float *head_w,
                                const int32_t *seq_len, int B, int64_t pool_stride, int64_t max_blocks,
                                int top_k, int32_t *sel, int32_t *nsel, void *ws, Rope rope, bool relu,
                                bool bf16, unsigned *status, cudaStream_t s) {
    const DecodePlan pl = decode_index_plan(B, max_blocks, bf16);
    if ((int64_t)pl.chunks * top_k > DI_MERGE_CAP || pl.chunks > 64) return cudaErrorInvalidConfiguration;
    const size_t n = (size_t)B * pl.chunks * top_k;
    uint8_t *w = static_cast<uint8_t *>(ws);
    uint32_t *ck = reinterpret_cast<uint32_t *>(w);
    w += (n * sizeof(uint32_t) + 255) / 256 * 256;
    int32_t *ci = reinterpret_cast<int32_t *>(w);
    w += (n * sizeof(int32_t) + 255) / 256 * 256;
    int32_t *cc = reinterpret_cast<int32_t *>(w);
    DecodeParams p{seq_len, head_w, pool_stride, max_blocks, pl.chunk, pl.chunks, top_k, relu ? 1 : 0, ck, ci, cc,
                   status};
    dim3 grid((unsigned)pl.chunks, (unsigned)B);
    cudaError_t e;
    if (bf16) {
        CUtensorMap kmap;
        if (!make_kpool_map(&kmap, k_pool, (uint64_t)B * pool_stride)) return cudaErrorInvalidValue;
        const size_t smem = sizeof(DecodeMmaSmem) + 1024 + (size_t)pl.chunk * sizeof(uint32_t);
        e = cudaFuncSetAttribute(decode_score_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        decode_score_mma_kernel<<<grid, DI_THREADS, smem, s>>>(kmap, (const __nv_bfloat16 *)q_idx, rope, p);
    } else {
        const size_t smem = DI_NS * DI_STAGE_BYTES + (size_t)pl.chunk * sizeof(uint32_t);
        e = cudaFuncSetAttribute(decode_score_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        decode_score_kernel<float><<<grid, DI_THREADS, smem, s>>>((const float *)q_idx, (const float *)k_pool, rope,
                                                                  p);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const size_t msmem = (size_t)pl.chunks * top_k * 8;
    e = cudaFuncSetAttribute(decode_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)msmem);
    if (e != cudaSuccess) return e;
    decode_merge_kernel<<<B, DI_MERGE_THREADS, msmem, s>>>(pl, top_k, ck, ci, cc, sel, nsel);
    return cudaGetLastError();
}

}  // namespace qsa
