// k_dense.cu -- full causal attention for prefill: the dense baseline QSA
// replaces.
//
// Pages "Qwen3.8-Flash-Next, Layer by Layer" (section "Token mixing") and the
// aicontrolled journal (section "Where the measurement ends") compare the QSA
// attention module with full attention during prefill at 1M tokens (16K-token
// chunks).  Not a step of QSA: the kernel exists so that comparison can be made
// on one GPU with kernels of this library.  Query t of a chunk starting at q0
// attends over every cached position 0 .. q0 + t.
//
// Tiled ("flash") form with warp MMAs: a CTA takes the 8 q heads of one kv head
// for 8 consecutive queries (64 rows of Q), streams the kv head's K and V in
// 64-key tiles through two TMA stages (128-byte swizzle), and each of its 4
// warps runs an online softmax over 16 rows (2 queries x 8 heads):
// S = Q K^T and O += P V as m16n8k16 bf16 MMAs with fp32 accumulation, P fed
// from the S accumulators as the A operand.  K/V tiles are loaded once for all
// 64 rows, the reuse a per-query gather (the sparse kernel) does not have.
#include "dense.h"

namespace qsa {

namespace {

constexpr int DP_KEYS = 64;                 // keys per tile
constexpr int DP_Q = 8;                     // queries per CTA
constexpr int DP_WARPS = 4;                 // 2 queries x 8 heads = 16 rows each
constexpr int DP_ATOM = DP_KEYS * 128;      // one 64-dim half of a 64-key tile (bytes)
constexpr int DP_TILE = 2 * DP_ATOM;        // 64 keys x 128 dims, bf16
constexpr float kDpLog2e = 1.4426950408889634f;

struct DpParams {
    const __nv_bfloat16 *q;
    __nv_bfloat16 *out;
    float *lse;
    int64_t n_q, q0, kv_stride;
    int Hkv;
    float scale_log2;
    unsigned *status;
};

struct __align__(1024) DpSmem {
    uint8_t k[2][DP_TILE];
    uint8_t v[2][DP_TILE];
    uint64_t full[2], empty[2];
};

// Byte offset of (key, 16-byte chunk c of 128 dims) in a tile stored as two
// 64-dim halves of 64 rows x 128 B with the TMA 128-byte swizzle.
__device__ __forceinline__ uint32_t dp_off(int key, int c) {
    return (uint32_t)((c >> 3) * DP_ATOM + key * 128 + (((c & 7) ^ (key & 7)) << 4));
}

__global__ void __launch_bounds__(DP_WARPS * 32) dense_prefill_kernel(const __grid_constant__ CUtensorMap kmap,
                                                                     const __grid_constant__ CUtensorMap vmap,
                                                                     DpParams p) {
    extern __shared__ uint8_t dp_raw[];
    DpSmem &sm = *reinterpret_cast<DpSmem *>((reinterpret_cast<uintptr_t>(dp_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gr = lane >> 2, tq = lane & 3;
    // longest rows first: the last query blocks have the most key tiles
    const int64_t nqb = (p.n_q + DP_Q - 1) / DP_Q;
    const int64_t qb = nqb - 1 - blockIdx.x;
    const int g = blockIdx.y, seq = blockIdx.z;
    const int Hq = 8 * p.Hkv;
    const int64_t r0 = qb * DP_Q;                              // first query row of the CTA
    const int64_t last = min(r0 + DP_Q, p.n_q) - 1;            // last row
    const int64_t ntiles = (p.q0 + last) / DP_KEYS + 1;        // key tiles up to the last row's position
    const int64_t y0 = (int64_t)seq * p.kv_stride;
    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], DP_WARPS);
        }
        fence_mbar_init();
        prefetch_tmap(&kmap);
        prefetch_tmap(&vmap);
    }
    __syncthreads();
    pdl_wait();
    pdl_trigger();
    auto issue = [&](int slot, int64_t t) {
        mbar_arrive_expect_tx(&sm.full[slot], 2 * DP_TILE);
        const int y = (int)(y0 + t * DP_KEYS);
        for (int a = 0; a < 2; ++a) {
            tma_load_2d(sm.k[slot] + a * DP_ATOM, &kmap, g * 128 + 64 * a, y, &sm.full[slot]);
            tma_load_2d(sm.v[slot] + a * DP_ATOM, &vmap, g * 128 + 64 * a, y, &sm.full[slot]);
        }
    };
    if (tid == 0)
        for (int64_t t = 0; t < 2 && t < ntiles; ++t) issue((int)t, t);

    // rows gr / gr + 8 of this warp: queries ra / rb (head gr of kv head g)
    const int64_t ra = r0 + 2 * warp, rb = ra + 1;
    const bool va = ra < p.n_q, vb = rb < p.n_q;
    const int64_t pa = p.q0 + ra, pb = p.q0 + rb;              // their positions
    uint32_t qf[8][4];
    {
        const int head = 8 * g + gr;
        const uint32_t *qa = reinterpret_cast<const uint32_t *>(p.q + (((int64_t)seq * p.n_q + ra) * Hq + head) * 128);
        const uint32_t *qb2 = reinterpret_cast<const uint32_t *>(p.q + (((int64_t)seq * p.n_q + rb) * Hq + head) * 128);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            qf[kk][0] = va ? qa[(16 * kk + 2 * tq) >> 1] : 0u;
            qf[kk][1] = vb ? qb2[(16 * kk + 2 * tq) >> 1] : 0u;
            qf[kk][2] = va ? qa[(16 * kk + 8 + 2 * tq) >> 1] : 0u;
            qf[kk][3] = vb ? qb2[(16 * kk + 8 + 2 * tq) >> 1] : 0u;
        }
    }
    float o[16][4];
#pragma unroll
    for (int j = 0; j < 16; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
    const int mi = lane >> 3, rr = lane & 7;
    bool ok = true;
    int64_t t = 0;
    for (; t < ntiles; ++t) {
        const int slot = (int)(t & 1);
        ok = mbar_wait(&sm.full[slot], (uint32_t)((t >> 1) & 1), p.status);
        if (!ok) break;
        const uint32_t kb = smem_u32(sm.k[slot]), vbase = smem_u32(sm.v[slot]);
        // S (16 rows x 64 keys): n-tile j = keys 8j .. 8j + 7
        float s[8][4];
#pragma unroll
        for (int j = 0; j < 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
            for (int pq = 0; pq < 4; ++pq) {   // n-tiles 2pq, 2pq + 1 (keys 16pq .. 16pq + 15)
                uint32_t b0, b1, b2, b3;
                const int key = 16 * pq + 8 * (mi >> 1) + rr;
                ldsm_x4(kb + dp_off(key, 2 * kk + (mi & 1)), b0, b1, b2, b3);
                mma16816(s[2 * pq], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b0, b1);
                mma16816(s[2 * pq + 1], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b2, b3);
            }
        }
        // causal mask on the tiles that reach past a row's position
        const int64_t kbase = t * DP_KEYS;
        if (kbase + DP_KEYS - 1 > pa) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int64_t key = kbase + 8 * j + 2 * tq;
                if (key > pa || !va) s[j][0] = -INFINITY;
                if (key + 1 > pa || !va) s[j][1] = -INFINITY;
                if (key > pb || !vb) s[j][2] = -INFINITY;
                if (key + 1 > pb || !vb) s[j][3] = -INFINITY;
            }
        }
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            mx0 = fmaxf(mx0, fmaxf(s[j][0], s[j][1]));
            mx1 = fmaxf(mx1, fmaxf(s[j][2], s[j][3]));
        }
#pragma unroll
        for (int o2 = 1; o2 < 4; o2 <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o2));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o2));
        }
        const float mn0 = fmaxf(mrow[0], mx0 * p.scale_log2), mn1 = fmaxf(mrow[1], mx1 * p.scale_log2);
        const float al0 = exp2f(mrow[0] - (mn0 == -INFINITY ? 0.f : mn0));
        const float al1 = exp2f(mrow[1] - (mn1 == -INFINITY ? 0.f : mn1));
        mrow[0] = mn0;
        mrow[1] = mn1;
        lrow[0] *= al0;
        lrow[1] *= al1;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            o[j][0] *= al0;
            o[j][1] *= al0;
            o[j][2] *= al1;
            o[j][3] *= al1;
        }
        const float nm0 = mn0 == -INFINITY ? 0.f : -mn0, nm1 = mn1 == -INFINITY ? 0.f : -mn1;
        uint32_t pf[8][2];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float p0 = exp2f(fmaf(s[j][0], p.scale_log2, nm0));
            const float p1 = exp2f(fmaf(s[j][1], p.scale_log2, nm0));
            const float p2 = exp2f(fmaf(s[j][2], p.scale_log2, nm1));
            const float p3 = exp2f(fmaf(s[j][3], p.scale_log2, nm1));
            lrow[0] += p0 + p1;
            lrow[1] += p2 + p3;
            pf[j][0] = pack_bf16(p0, p1);
            pf[j][1] = pack_bf16(p2, p3);
        }
        // O (16 rows x 128 dims) += P (16 x 64) V (64 x 128): k-step ks = keys 16ks ..
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {   // dim n-tiles 2jj, 2jj + 1
                uint32_t b0, b1, b2, b3;
                const int key = 16 * ks + 8 * (mi & 1) + rr;
                ldsm_x4_t(vbase + dp_off(key, 2 * jj + (mi >> 1)), b0, b1, b2, b3);
                mma16816(o[2 * jj], pf[2 * ks][0], pf[2 * ks][1], pf[2 * ks + 1][0], pf[2 * ks + 1][1], b0, b1);
                mma16816(o[2 * jj + 1], pf[2 * ks][0], pf[2 * ks][1], pf[2 * ks + 1][0], pf[2 * ks + 1][1], b2,
                         b3);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.empty[slot]);
        if (tid == 0 && t + 2 < ntiles) {
            ok = mbar_wait(&sm.empty[slot], (uint32_t)((t >> 1) & 1), p.status);
            if (ok) issue(slot, t + 2);
        }
    }
    ok = __syncthreads_and(ok);
    if (!ok) {
        // let the copies still in flight land before the CTA exits
        if (tid == 0)
            for (int64_t c = t; c < t + 2 && c < ntiles; ++c)
                mbar_wait(&sm.full[c & 1], (uint32_t)((c >> 1) & 1), p.status);
        return;
    }
#pragma unroll
    for (int o2 = 1; o2 < 4; o2 <<= 1) {
        lrow[0] += __shfl_xor_sync(0xffffffffu, lrow[0], o2);
        lrow[1] += __shfl_xor_sync(0xffffffffu, lrow[1], o2);
    }
    const float inv0 = lrow[0] > 0.f ? 1.f / lrow[0] : 0.f, inv1 = lrow[1] > 0.f ? 1.f / lrow[1] : 0.f;
    const int head = 8 * g + gr;
    __nv_bfloat16 *oa = p.out + (((int64_t)seq * p.n_q + ra) * Hq + head) * 128;
    __nv_bfloat16 *ob = p.out + (((int64_t)seq * p.n_q + rb) * Hq + head) * 128;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        if (va) *reinterpret_cast<uint32_t *>(oa + 8 * j + 2 * tq) = pack_bf16(o[j][0] * inv0, o[j][1] * inv0);
        if (vb) *reinterpret_cast<uint32_t *>(ob + 8 * j + 2 * tq) = pack_bf16(o[j][2] * inv1, o[j][3] * inv1);
    }
    if (p.lse && tq == 0) {
        if (va) p.lse[((int64_t)seq * p.n_q + ra) * Hq + head] = lrow[0] > 0.f ? (mrow[0] + log2f(lrow[0])) / kDpLog2e
                                                                               : -INFINITY;
        if (vb) p.lse[((int64_t)seq * p.n_q + rb) * Hq + head] = lrow[1] > 0.f ? (mrow[1] + log2f(lrow[1])) / kDpLog2e
                                                                               : -INFINITY;
    }
}

using EncodeTiledFn = decltype(&cuTensorMapEncodeTiled);

// [rows][Hkv * 128] bf16 with 64 x 64 boxes, 128-byte swizzle.
bool make_kv_map(CUtensorMap *map, const void *base, uint64_t rows, int Hkv) {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return false;
        fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    cuuint64_t dims[2] = {(cuuint64_t)Hkv * 128, rows};
    cuuint64_t strides[1] = {(cuuint64_t)Hkv * 128 * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)DP_KEYS};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_dense_prefill(const void *q, const void *k, const void *v, int B, int64_t n_q, int64_t q0,
                                 int64_t kv_stride, int Hkv, float scale, void *out, float *lse, unsigned *status,
                                 cudaStream_t s) {
    if (n_q <= 0) return cudaSuccess;
    CUtensorMap kmap, vmap;
    if (!make_kv_map(&kmap, k, (uint64_t)B * kv_stride, Hkv) || !make_kv_map(&vmap, v, (uint64_t)B * kv_stride, Hkv))
        return cudaErrorInvalidValue;
    DpParams p{(const __nv_bfloat16 *)q, (__nv_bfloat16 *)out, lse, n_q, q0, kv_stride, Hkv, scale * kDpLog2e, status};
    const size_t smem = sizeof(DpSmem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(dense_prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)((n_q + DP_Q - 1) / DP_Q), (unsigned)Hkv, (unsigned)B);
    return launch_pdl(dense_prefill_kernel, grid, dim3(DP_WARPS * 32), smem, s, kmap, vmap, p);
}

}  // namespace qsa
