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

}  // namespace

DecodePlan decode_index_plan(int B, int64_t max_blocks, bool bf16) {
    (void)bf16;
    const DeviceInfo *di = device_info();
    const int sms = di ? di->sm_count : 148;
    DecodePlan pl;
    int64_t C = std::max<int64_t>(1, (2 * sms) / std::max(B, 1));
    C = std::min<int64_t>(C, std::max<int64_t>(1, (max_blocks + 255) / 256));
    int64_t chunk = (max_blocks + C - 1) / C;
    chunk = std::max<int64_t>(64, (chunk + 63) / 64 * 64);
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
    const size_t smem = DI_NS * DI_STAGE_BYTES + (size_t)pl.chunk * sizeof(uint32_t);
    dim3 grid((unsigned)pl.chunks, (unsigned)B);
    cudaError_t e;
    if (bf16) {
        e = cudaFuncSetAttribute(decode_score_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
        if (e != cudaSuccess) return e;
        decode_score_kernel<__nv_bfloat16><<<grid, DI_THREADS, smem, s>>>(
            (const __nv_bfloat16 *)q_idx, (const __nv_bfloat16 *)k_pool, rope, p);
    } else {
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
