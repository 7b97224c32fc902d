// k_attn_tc.cu -- prefill sparse attention on the tensor cores, one tile of
// 16 consecutive queries at a time.
//
// Page "Qwen3.8-Flash-Next: Day-0 Support in SGLang", section "Qwen Sparse
// Attention: Retrieve Coarsely, Attend Precisely": each query attends over the
// 4 positions of each of its selected blocks plus its own 0-3 tail tokens,
// with softmax and value aggregation over the original K/V; one selection per
// query serves every head.
//
// Neighbouring queries select overlapping blocks (heavy-tailed keys are chosen
// by many queries; early queries see few blocks), so this kernel gathers each
// block once for a tile of UQ = 16 queries:
//   * a pre-pass (union_build_kernel) merges the 16 selections and tail blocks
//     of a query tile into one ascending list of blocks, each with a 16-bit
//     mask of the queries that attend to it;
//   * for one kv head g, the 16 queries x 8 q heads form the M = 128 rows of
//     two tcgen05 GEMMs per key tile of 32 listed blocks (N = 128 keys):
//       S = Q K^T   (A = Q from tensor memory, B = K tile, 128-byte swizzle)
//       O += P V    (A = P from tensor memory, B = V tile read MN-major)
//     with S, P and O in tensor memory and K/V tiles landing in shared memory
//     by TMA (one 4-token x 64-dim box per block, dim half and tensor);
//   * 4 softmax warps own one TMEM row each ((query, head) = row / 8, row % 8):
//     they mask the keys their query does not attend to (mask bit, and for the
//     blocks at the diagonal key position <= query position), keep the fp32
//     online-softmax state of their row, rescale their O row in tensor memory
//     when the row maximum grows by more than 2^8 (lazy rescaling), and write
//     P back over S as bf16.
// A masked key contributes p = 0 exactly, so each query's result is its own
// softmax over its own positions; the extra products are the price of reading
// each block once.  Warp roles: 0 = TMA producer, 1 = MMA issuer and TMEM
// owner, 2..5 = softmax and epilogue.  A persistent grid walks the work items
// (sequence, query tile, kv head), latest query tiles first.
#include <algorithm>

#include "internal.h"

namespace qsa {

namespace {

constexpr int UQ = 16;                 // queries per tile
constexpr int UG = 8;                  // q heads per kv head
constexpr int UM = UQ * UG;            // MMA rows
constexpr int UB = 32;                 // listed blocks per key tile
constexpr int UN = UB * kBlock;        // keys per tile
constexpr int UD = 128;                // head dim
constexpr int UREG = UN * 128;         // 128 rows x 128 bytes (64 bf16 dims), 128-byte swizzle
constexpr int USTAGE = 4 * UREG;       // K dims 0-63, K dims 64-127, V dims 0-63, V dims 64-127
constexpr int UBOX = kBlock * 128;     // one TMA box: 4 tokens x 64 dims
#ifndef QSA_UT_STAGES
#define QSA_UT_STAGES 3
#endif
constexpr int UNS = QSA_UT_STAGES;     // key tiles in flight
constexpr int UT_THREADS = 192;
constexpr uint32_t TM_S = 0;           // S / P, two buffers of 128 columns
constexpr uint32_t TM_O = 256;         // O, 128 columns
constexpr uint32_t TM_Q = 384;         // Q, 64 columns (bf16 pairs)
constexpr uint32_t TM_COLS = 512;
constexpr int UCHUNK = 16384;          // pre-pass: block ids per pass (one 32-bit mask word each)
constexpr float kLog2e = 1.4426950408889634f;
#ifndef QSA_UT_RESCALE
#define QSA_UT_RESCALE 8.f
#endif
constexpr float kRescale = QSA_UT_RESCALE;   // lazy rescale threshold (log2 units)

struct UtMeta {
    int32_t id[UB];                    // listed block ids of the tile (-1: padding)
    uint32_t mw[UQ];                   // per query: bit j = the query attends to block j of the tile
    int32_t diag;                      // a block of the tile reaches past the tile's first query
    int32_t pad[15];
};

struct UtSmem {
    alignas(1024) uint8_t kv[UNS][USTAGE];
    alignas(1024) uint8_t qs[2 * UREG];            // Q tile staging: 128 rows x 128 dims, two swizzled halves
    UtMeta meta[UNS];
    uint64_t full[UNS], empty[UNS];
    uint64_t q_full, q_empty, q_ready;
    uint64_t s_full[2], p_ready[2], pv_done, o_full, drain;
    uint32_t tmem_base;
};

static_assert(sizeof(UtSmem) + 1024 <= 232448, "shared memory of the attention CTA exceeds 227 KB");

struct UtParams {
    int B;
    int64_t n_q, q0;
    int Hq, Hkv;
    int64_t row0, row_end;   // rows of this launch
    int64_t n_qt;            // query tiles per sequence in this launch
    int cap;                 // list capacity per query tile
    const int32_t *u_count;  // [B][n_qt]
    const uint32_t *u_id;    // [B][n_qt][cap]
    const uint16_t *u_mask;  // [B][n_qt][cap]
    float scale_log2;
    __nv_bfloat16 *out;
    float *lse;
    unsigned *status;
    int64_t items;
};

struct UtItem {
    int seq, g, nrows, n_u;
    int64_t r0, t0;
    const uint32_t *ids;
    const uint16_t *msk;
};

__device__ __forceinline__ UtItem ut_item(const UtParams &p, int64_t i) {
    UtItem it;
    const int64_t per = (int64_t)p.B * p.Hkv;
    const int64_t qt = p.n_qt - 1 - i / per;   // latest (longest) query tiles first
    const int rem = (int)(i % per);
    it.seq = rem / p.Hkv;
    it.g = rem % p.Hkv;
    it.r0 = p.row0 + qt * UQ;
    it.nrows = (int)(p.row_end - it.r0 < UQ ? p.row_end - it.r0 : UQ);
    it.t0 = p.q0 + it.r0;
    const int64_t ti = (int64_t)it.seq * p.n_qt + qt;
    it.n_u = min(max(p.u_count[ti], 0), p.cap);
    it.ids = p.u_id + ti * p.cap;
    it.msk = p.u_mask + ti * p.cap;
    return it;
}

// ---------------------------------------------------------------- pre-pass
// One CTA per (query tile, sequence).  Block ids of the tile's 16 selections
// (validated: 0 <= b < nb(t)) and each query's tail block (when it holds 1-3
// tokens) set bit q in a mask word per id; the non-zero words are compacted
// in id order.  Ids are processed UCHUNK at a time.
__global__ void __launch_bounds__(256) union_build_kernel(const int32_t *__restrict__ sel,
                                                          const int32_t *__restrict__ nsel, int64_t n_q, int64_t q0,
                                                          int top_k, int64_t row0, int64_t row_end, int64_t n_qt,
                                                          int cap, int32_t *__restrict__ u_count,
                                                          uint32_t *__restrict__ u_id, uint16_t *__restrict__ u_mask,
                                                          unsigned *status) {
    extern __shared__ uint32_t ub_bits[];
    __shared__ int s_nsel[UQ];
    __shared__ int s_wsum[8];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int seq = blockIdx.y;
    const int64_t qt = blockIdx.x;
    const int64_t r0 = row0 + qt * UQ;
    const int nrows = (int)(row_end - r0 < UQ ? row_end - r0 : UQ);
    pdl_wait();       // the selection comes from the previous kernel
    pdl_trigger();
    if (tid < UQ) s_nsel[tid] = tid < nrows ? max(0, min(nsel[(int64_t)seq * n_q + r0 + tid], top_k)) : 0;
    __syncthreads();
    const int64_t t_last = q0 + r0 + nrows - 1;
    const int64_t id_end = t_last / kBlock + 1;            // the last query's tail block, exclusive
    const int64_t ti = (int64_t)seq * n_qt + qt;
    uint32_t *oid = u_id + ti * cap;
    uint16_t *om = u_mask + ti * cap;
    int count = 0;
    for (int64_t c0 = 0; c0 < id_end; c0 += UCHUNK) {
        const int span = (int)(id_end - c0 < UCHUNK ? id_end - c0 : UCHUNK);
        for (int i = tid; i < span; i += 256) ub_bits[i] = 0;
        __syncthreads();
        for (int e = tid; e < UQ * top_k; e += 256) {
            const int q = e / top_k, k = e - q * top_k;
            if (k >= s_nsel[q]) continue;
            const int64_t t = q0 + r0 + q;
            const int32_t b = sel[((int64_t)seq * n_q + r0 + q) * top_k + k];
            if (b < 0 || (int64_t)b >= (t + 1) / kBlock) {
                if (c0 == 0) flag(status, QSA_DEV_BAD_INDEX);
                continue;
            }
            if (b >= c0 && b < c0 + span) atomicOr(&ub_bits[b - c0], 1u << q);
        }
        if (tid < nrows) {
            const int64_t t = q0 + r0 + tid;
            const int64_t nb = (t + 1) / kBlock;
            if (t + 1 > kBlock * nb && nb >= c0 && nb < c0 + span) atomicOr(&ub_bits[nb - c0], 1u << tid);
        }
        __syncthreads();
        // compaction in id order: thread tid owns words [tid * W, tid * W + W)
        const int W = (span + 255) / 256;
        int mine = 0;
        for (int i = 0; i < W; ++i) {
            const int w = tid * W + i;
            if (w < span && ub_bits[w]) ++mine;
        }
        int incl = mine;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        if (lane == 31) s_wsum[warp] = incl;
        __syncthreads();
        int before = 0, total = 0;
#pragma unroll
        for (int w = 0; w < 8; ++w) {
            before += (w < warp) ? s_wsum[w] : 0;
            total += s_wsum[w];
        }
        int pos = count + before + incl - mine;
        for (int i = 0; i < W; ++i) {
            const int w = tid * W + i;
            if (w < span) {
                const uint32_t m = ub_bits[w];
                if (m && pos < cap) {
                    oid[pos] = (uint32_t)(c0 + w);
                    om[pos] = (uint16_t)m;
                    ++pos;
                }
            }
        }
        count += total;
        __syncthreads();
    }
    if (tid == 0) u_count[ti] = min(count, cap);
}

// ---------------------------------------------------------------- attention
__global__ void __launch_bounds__(UT_THREADS, 1)
    attn_union_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                      const __grid_constant__ CUtensorMap map_v, UtParams p) {
    extern __shared__ uint8_t ut_raw[];
    UtSmem &sm = *reinterpret_cast<UtSmem *>((reinterpret_cast<uintptr_t>(ut_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // zero the K/V stages once: rows of padding entries are never loaded, and
    // their (masked) products must stay finite
    for (int i = threadIdx.x; i < (int)(sizeof(sm.kv) / 16); i += blockDim.x)
        reinterpret_cast<uint4 *>(&sm.kv[0][0])[i] = make_uint4(0, 0, 0, 0);
    if (threadIdx.x == 0) {
        for (int s = 0; s < UNS; ++s) {
            mbar_init(&sm.full[s], 32);
            mbar_init(&sm.empty[s], 1);
        }
        mbar_init(&sm.q_full, 1);
        mbar_init(&sm.q_empty, 4);
        mbar_init(&sm.q_ready, 4);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.s_full[b], 1);
            mbar_init(&sm.p_ready[b], 4);
        }
        mbar_init(&sm.pv_done, 1);
        mbar_init(&sm.o_full, 1);
        mbar_init(&sm.drain, 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, TM_COLS);
        tmem_relinquish();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    pdl_wait();       // the block lists come from the pre-pass
    pdl_trigger();

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tmap(&map_q);
            prefetch_tmap(&map_k);
            prefetch_tmap(&map_v);
        }
        int64_t c = 0, nq = 0;   // stages issued, Q tiles issued
        bool ok = true;
        for (int64_t i = blockIdx.x; i < p.items && ok; i += gridDim.x) {
            const UtItem it = ut_item(p, i);
            if (nq >= 1) ok = mbar_wait(&sm.q_empty, (int)((nq - 1) & 1), p.status);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            if (lane == 0) {
                mbar_arrive_expect_tx(&sm.q_full, 2 * UREG);
                const int qrow = (int)((int64_t)it.seq * p.n_q + it.r0);
                tma_load_3d(sm.qs, &map_q, 0, UG * it.g, qrow, &sm.q_full);
                tma_load_3d(sm.qs + UREG, &map_q, 64, UG * it.g, qrow, &sm.q_full);
            }
            ++nq;
            const int ntile = (it.n_u + UB - 1) / UB;
            uint32_t e_id = lane < it.n_u ? it.ids[lane] : 0xFFFFFFFFu;
            uint32_t e_m = lane < it.n_u ? it.msk[lane] : 0u;
            for (int u = 0; u < ntile; ++u) {
                const int nx = (u + 1) * UB + lane;            // next tile's entries, loaded ahead
                const uint32_t n_id = nx < it.n_u ? it.ids[nx] : 0xFFFFFFFFu;
                const uint32_t n_m = nx < it.n_u ? it.msk[nx] : 0u;
                const int s = (int)(c % UNS);
                if (c >= UNS) ok = mbar_wait(&sm.empty[s], (int)(((c / UNS) + 1) & 1), p.status);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                const bool live = e_id != 0xFFFFFFFFu;
                UtMeta &mt = sm.meta[s];
                mt.id[lane] = live ? (int32_t)e_id : -1;
                uint32_t mine = 0;
#pragma unroll
                for (int q = 0; q < UQ; ++q) {
                    const uint32_t b = __ballot_sync(0xffffffffu, (e_m >> q) & 1u);
                    if (lane == q) mine = b;
                }
                if (lane < UQ) mt.mw[lane] = mine;
                const int maxid = __reduce_max_sync(0xffffffffu, live ? (int)e_id : -1);
                if (lane == 0) mt.diag = ((int64_t)kBlock * maxid + kBlock - 1 > it.t0) ? 1 : 0;
                const uint32_t nlive = __popc(__ballot_sync(0xffffffffu, live));
                __syncwarp();
                if (lane == 0) mbar_arrive_expect_tx(&sm.full[s], nlive * 4u * UBOX);
                else mbar_arrive(&sm.full[s]);
                if (live) {
                    uint8_t *st = sm.kv[s] + lane * UBOX;
                    const int tok = kBlock * (int)e_id;
                    tma_load_4d(st, &map_k, 0, it.g, tok, it.seq, &sm.full[s]);
                    tma_load_4d(st + UREG, &map_k, 64, it.g, tok, it.seq, &sm.full[s]);
                    tma_load_4d(st + 2 * UREG, &map_v, 0, it.g, tok, it.seq, &sm.full[s]);
                    tma_load_4d(st + 3 * UREG, &map_v, 64, it.g, tok, it.seq, &sm.full[s]);
                }
                ++c;
                e_id = n_id;
                e_m = n_m;
            }
        }
        // no copy may still be landing when the CTA ends (bounded waits)
        if (lane == 0) {
            for (int64_t cc = (c > UNS ? c - UNS : 0); cc < c; ++cc)
                mbar_wait(&sm.full[cc % UNS], (int)((cc / UNS) & 1), p.status);
            if (nq >= 1) mbar_wait(&sm.q_full, (int)((nq - 1) & 1), p.status);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc_qk = idesc_bf16_f32(UM, UN);
            const uint32_t idesc_pv = idesc_bf16_f32(UM, UD) | (1u << 16);   // B = V tile, MN-major
            int64_t c = 0, ic = 0;
            bool ok = true;
            for (int64_t i = blockIdx.x; i < p.items && ok; i += gridDim.x, ++ic) {
                const UtItem it = ut_item(p, i);
                const int ntile = (it.n_u + UB - 1) / UB;
                ok = mbar_wait(&sm.q_ready, (int)(ic & 1), p.status);
                if (!ok) break;
                tc_fence_after();
                for (int u = 0; u <= ntile && ok; ++u) {
                    if (u < ntile) {   // S(u) = Q K(u)^T
                        const int64_t cu = c + u;
                        const int s = (int)(cu % UNS);
                        ok = mbar_wait(&sm.full[s], (int)((cu / UNS) & 1), p.status);
                        if (!ok) break;
                        tc_fence_after();
                        const uint32_t d = tmem + TM_S + (uint32_t)((cu & 1) * 128);
                        const uint32_t kb = smem_u32(sm.kv[s]);
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            tc_mma_ts(d, tmem + TM_Q + 8 * k, sw128_desc(kb + (k >> 2) * UREG + (k & 3) * 32),
                                      idesc_qk, k > 0 ? 1u : 0u);
                        tc_commit(&sm.s_full[cu & 1]);
                    }
                    if (u >= 1) {      // O += P(u-1) V(u-1)
                        const int64_t cp = c + u - 1;
                        ok = mbar_wait(&sm.p_ready[cp & 1], (int)((cp >> 1) & 1), p.status);
                        if (!ok) break;
                        tc_fence_after();
                        const int s = (int)(cp % UNS);
                        const uint32_t vb = smem_u32(sm.kv[s]) + 2 * UREG;
                        const uint32_t pa = tmem + TM_S + (uint32_t)((cp & 1) * 128);
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            tc_mma_ts(tmem + TM_O, pa + 8 * k, sw128_desc_ls(vb + k * 2048, UREG, 1024), idesc_pv,
                                      (u > 1 || k > 0) ? 1u : 0u);
                        tc_commit(&sm.empty[s]);
                        tc_commit(&sm.pv_done);
                    }
                }
                // the item's O is complete: one phase of o_full per item.  (The
                // epilogue cannot wait on pv_done by parity: when it gets there
                // the item's last two products may both still be in flight, two
                // phases behind, which a parity wait cannot tell apart.)
                if (ok) tc_commit(&sm.o_full);
                c += ntile;
            }
            // every MMA issued has completed before the TMEM is released
            tc_commit(&sm.drain);
            mbar_wait(&sm.drain, 0, p.status);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax / epilogue
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;          // TMEM lane: query row / 8, head row % 8
        const int qi = row >> 3, hl = row & 7;
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        const float sl2 = p.scale_log2;
        int64_t c = 0, ic = 0;
        bool ok = true;
        for (int64_t i = blockIdx.x; i < p.items && ok; i += gridDim.x, ++ic) {
            const UtItem it = ut_item(p, i);
            const int ntile = (it.n_u + UB - 1) / UB;
            const int64_t tq = it.t0 + qi;
            // Q tile: staging shared memory -> this row's 64 TMEM columns
            ok = __all_sync(0xffffffffu, mbar_wait(&sm.q_full, (int)(ic & 1), p.status));
            if (!ok) break;
            {
                uint32_t qv[64];
#pragma unroll
                for (int c8 = 0; c8 < 16; ++c8) {
                    const int half = c8 >> 3, ch = c8 & 7;
                    const uint4 v = *reinterpret_cast<const uint4 *>(sm.qs + half * UREG + row * 128 +
                                                                     ((ch ^ (row & 7)) << 4));
                    qv[4 * c8] = v.x;
                    qv[4 * c8 + 1] = v.y;
                    qv[4 * c8 + 2] = v.z;
                    qv[4 * c8 + 3] = v.w;
                }
                tmem_st32(lane_base + TM_Q, *reinterpret_cast<const uint32_t(*)[32]>(&qv[0]));
                tmem_st32(lane_base + TM_Q + 32, *reinterpret_cast<const uint32_t(*)[32]>(&qv[32]));
                tc_wait_st();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&sm.q_ready);
                mbar_arrive(&sm.q_empty);
            }
            float m_run = -INFINITY, l_run = 0.f;
            for (int u = 0; u < ntile; ++u, ++c) {
                const int s = (int)(c % UNS);
                bool w_ok = mbar_wait(&sm.s_full[c & 1], (int)((c >> 1) & 1), p.status);
                if (w_ok) w_ok = mbar_wait(&sm.full[s], (int)((c / UNS) & 1), p.status);   // the tile's meta
                ok = __all_sync(0xffffffffu, w_ok);
                if (!ok) break;
                tc_fence_after();
                const UtMeta &mt = sm.meta[s];
                const uint32_t mw = mt.mw[qi];
                const uint32_t wmask = __reduce_or_sync(0xffffffffu, mw);
                const bool diag = mt.diag != 0;
                const uint32_t sa = lane_base + TM_S + (uint32_t)((c & 1) * 128);
                uint32_t sv[128];
#pragma unroll
                for (int ch = 0; ch < 4; ++ch)
                    tmem_ld32(sa + 32 * ch, *reinterpret_cast<uint32_t(*)[32]>(&sv[32 * ch]));
                tc_wait_ld();
                // logits in log2 units; keys the query does not attend to -> -inf
                float mx = -INFINITY;
#pragma unroll
                for (int j = 0; j < UB; ++j) {
                    const bool on = (mw >> j) & 1u;
                    int64_t kpos = 0;
                    if (diag) kpos = (int64_t)kBlock * mt.id[j];
#pragma unroll
                    for (int tk = 0; tk < kBlock; ++tk) {
                        const bool valid = on && (!diag || kpos + tk <= tq);
                        const float x = valid ? __uint_as_float(sv[kBlock * j + tk]) * sl2 : -INFINITY;
                        sv[kBlock * j + tk] = __float_as_uint(x);
                        mx = fmaxf(mx, x);
                    }
                }
                const bool grow = mx > m_run + kRescale;       // also the first keys of the row
                const bool resc = grow && m_run != -INFINITY;  // O and l already hold earlier keys
                if (__any_sync(0xffffffffu, resc)) {
                    // the previous P V must have landed before O is read.  A parity
                    // wait is exact here: S(c) landing means every MMA issued before
                    // QK(c) is done, P V(c - 2) included, and P V(c) needs this
                    // warp's P(c), so pv_done is at phase c - 1 or c.
                    ok = __all_sync(0xffffffffu, mbar_wait(&sm.pv_done, (int)((c - 1) & 1), p.status));
                    if (!ok) break;
                    tc_fence_after();
                    const float alpha = resc ? exp2f(m_run - mx) : 1.f;
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) {
                        uint32_t ov[32];
                        tmem_ld32(lane_base + TM_O + 32 * ch, ov);
                        tc_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
                        tmem_st32(lane_base + TM_O + 32 * ch, ov);
                    }
                    tc_wait_st();
                    l_run *= alpha;
                }
                if (grow) m_run = mx;
                const float mneg = (m_run == -INFINITY) ? 0.f : -m_run;
                uint32_t pk[64];
                float ls = 0.f;
#pragma unroll
                for (int j = 0; j < UB; ++j) {
                    if ((wmask >> j) & 1u) {   // some query of this warp attends to block j
                        const float p0 = exp2f(__uint_as_float(sv[4 * j]) + mneg);
                        const float p1 = exp2f(__uint_as_float(sv[4 * j + 1]) + mneg);
                        const float p2 = exp2f(__uint_as_float(sv[4 * j + 2]) + mneg);
                        const float p3 = exp2f(__uint_as_float(sv[4 * j + 3]) + mneg);
                        ls += (p0 + p1) + (p2 + p3);
                        pk[2 * j] = pack_bf16(p0, p1);
                        pk[2 * j + 1] = pack_bf16(p2, p3);
                    } else {
                        pk[2 * j] = 0u;
                        pk[2 * j + 1] = 0u;
                    }
                }
                l_run += ls;
                tmem_st32(sa, *reinterpret_cast<const uint32_t(*)[32]>(&pk[0]));
                tmem_st32(sa + 32, *reinterpret_cast<const uint32_t(*)[32]>(&pk[32]));
                tc_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.p_ready[c & 1]);
            }
            if (!ok) break;
            // epilogue: O / l -> bf16 rows of the output; lse
            ok = __all_sync(0xffffffffu, mbar_wait(&sm.o_full, (int)(ic & 1), p.status));
            if (!ok) break;
            tc_fence_after();
            const bool live = qi < it.nrows;
            const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
            __nv_bfloat16 *dst = p.out + (((int64_t)it.seq * p.n_q + it.r0 + qi) * p.Hq + UG * it.g + hl) * UD;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                uint32_t ov[32];
                tmem_ld32(lane_base + TM_O + 32 * ch, ov);
                tc_wait_ld();
                if (ntile == 0)   // no position at all: the output is zero
#pragma unroll
                    for (int e = 0; e < 32; ++e) ov[e] = 0u;
                if (live) {
#pragma unroll
                    for (int v4 = 0; v4 < 4; ++v4) {
                        uint4 w;
                        w.x = pack_bf16(__uint_as_float(ov[8 * v4]) * inv, __uint_as_float(ov[8 * v4 + 1]) * inv);
                        w.y = pack_bf16(__uint_as_float(ov[8 * v4 + 2]) * inv, __uint_as_float(ov[8 * v4 + 3]) * inv);
                        w.z = pack_bf16(__uint_as_float(ov[8 * v4 + 4]) * inv, __uint_as_float(ov[8 * v4 + 5]) * inv);
                        w.w = pack_bf16(__uint_as_float(ov[8 * v4 + 6]) * inv, __uint_as_float(ov[8 * v4 + 7]) * inv);
                        *reinterpret_cast<uint4 *>(dst + 32 * ch + 8 * v4) = w;
                    }
                }
            }
            if (live && p.lse)
                p.lse[((int64_t)it.seq * p.n_q + it.r0 + qi) * p.Hq + UG * it.g + hl] =
                    l_run > 0.f ? (m_run + log2f(l_run)) / kLog2e : -INFINITY;
            tc_fence_before();
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TM_COLS);
    }
}

using EncodeTiledFn = decltype(&cuTensorMapEncodeTiled);
EncodeTiledFn get_encode_fn() {
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

// Rows of one launch and the list capacity of a query tile.
struct UnionPlan {
    int cap;             // list entries per query tile
    int64_t rows;        // query rows per launch (a multiple of UQ)
    size_t count_bytes, id_bytes, mask_bytes;
};

constexpr size_t kUnionBudget = (size_t)512 << 20;   // workspace cap; longer prompts run in several launches

UnionPlan union_plan(int B, int64_t n_q, int top_k) {
    UnionPlan u{};
    u.cap = (UQ * (top_k + 1) + UB - 1) / UB * UB;
    const size_t per_tile = (size_t)u.cap * 6 + 4;
    const int64_t want_tiles = (n_q + UQ - 1) / UQ;
    const int64_t max_tiles = std::max<int64_t>(1, (int64_t)(kUnionBudget / (per_tile * std::max(B, 1))));
    const int64_t tiles = std::max<int64_t>(1, std::min(want_tiles, max_tiles));
    u.rows = tiles * UQ;
    auto r256 = [](size_t x) { return (x + 255) / 256 * 256; };
    u.count_bytes = r256((size_t)B * tiles * 4);
    u.id_bytes = r256((size_t)B * tiles * u.cap * 4);
    u.mask_bytes = r256((size_t)B * tiles * u.cap * 2);
    return u;
}

}  // namespace

bool attn_union_supported(const AttnArgs &a) {
    return !a.decode && !a.kv8 && a.d == UD && a.Hq == UG * a.Hkv && !a.pg.table;
}

size_t attn_union_ws_bytes(int B, int64_t n_q, int top_k) {
    if (B < 1 || n_q < 1) return 0;
    const UnionPlan u = union_plan(B, n_q, top_k);
    return u.count_bytes + u.id_bytes + u.mask_bytes;
}

int attn_union_launches(int B, int64_t n_q, int top_k) {
    if (B < 1 || n_q < 1) return 0;
    const UnionPlan u = union_plan(B, n_q, top_k);
    return (int)((n_q + u.rows - 1) / u.rows);
}

cudaError_t launch_attn_union(const AttnArgs &a, void *ws, unsigned *status, cudaStream_t s) {
    if (a.n_q <= 0) return cudaSuccess;
    const DeviceInfo *di = device_info();
    const int sms = di ? di->sm_count : 148;
    const UnionPlan u = union_plan(a.B, a.n_q, a.top_k);
    uint8_t *w = static_cast<uint8_t *>(ws);
    int32_t *u_count = reinterpret_cast<int32_t *>(w);
    uint32_t *u_id = reinterpret_cast<uint32_t *>(w + u.count_bytes);
    uint16_t *u_mask = reinterpret_cast<uint16_t *>(w + u.count_bytes + u.id_bytes);

    auto enc = get_encode_fn();
    if (!enc) return cudaErrorInvalidValue;
    // q: [B * n_q][Hq][128], box 64 dims x 8 heads x 16 queries
    CUtensorMap mq, mk, mv;
    {
        cuuint64_t dims[3] = {UD, (cuuint64_t)a.Hq, (cuuint64_t)a.B * a.n_q};
        cuuint64_t strides[2] = {UD * 2, (cuuint64_t)a.Hq * UD * 2};
        cuuint32_t box[3] = {64, UG, UQ};
        cuuint32_t estr[3] = {1, 1, 1};
        if (enc(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(a.q), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    // k, v: [B][kv_stride][Hkv][128], box 64 dims x 1 head x 4 tokens x 1 sequence
    for (int t = 0; t < 2; ++t) {
        cuuint64_t dims[4] = {UD, (cuuint64_t)a.Hkv, (cuuint64_t)a.kv_stride, (cuuint64_t)a.B};
        cuuint64_t strides[3] = {UD * 2, (cuuint64_t)a.Hkv * UD * 2, (cuuint64_t)a.kv_stride * a.Hkv * UD * 2};
        cuuint32_t box[4] = {64, 1, kBlock, 1};
        cuuint32_t estr[4] = {1, 1, 1, 1};
        if (enc(t ? &mv : &mk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(t ? a.v : a.k), dims, strides,
                box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    const size_t smem = sizeof(UtSmem) + 1024;
    if (di && smem > di->smem_optin) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(attn_union_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(union_build_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, UCHUNK * 4);
    if (e != cudaSuccess) return e;
    for (int64_t r = 0; r < a.n_q; r += u.rows) {
        const int64_t rows = std::min(u.rows, a.n_q - r);
        const int64_t n_qt = (rows + UQ - 1) / UQ;
        e = launch_pdl(union_build_kernel, dim3((unsigned)n_qt, (unsigned)a.B), dim3(256), (size_t)UCHUNK * 4, s,
                       a.sel, a.nsel, a.n_q, a.q0, a.top_k, r, r + rows, n_qt, u.cap, u_count, u_id, u_mask, status);
        if (e != cudaSuccess) return e;
        UtParams p{};
        p.B = a.B;
        p.n_q = a.n_q;
        p.q0 = a.q0;
        p.Hq = a.Hq;
        p.Hkv = a.Hkv;
        p.row0 = r;
        p.row_end = r + rows;
        p.n_qt = n_qt;
        p.cap = u.cap;
        p.u_count = u_count;
        p.u_id = u_id;
        p.u_mask = u_mask;
        p.scale_log2 = a.scale * kLog2e;
        p.out = static_cast<__nv_bfloat16 *>(a.out);
        p.lse = a.lse;
        p.status = status;
        p.items = (int64_t)a.B * n_qt * a.Hkv;
        const int64_t grid = std::min<int64_t>(p.items, sms);
        e = launch_pdl(attn_union_kernel, dim3((unsigned)grid), dim3(UT_THREADS), smem, s, mq, mk, mv, p);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace qsa
