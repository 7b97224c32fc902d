// k_attn_tc.cu -- prefill sparse attention on the tensor cores, one tile of
// 8 consecutive queries at a time.
//
// Page "Qwen3.8-Flash-Next: Day-0 Support in SGLang", section "Qwen Sparse
// Attention: Retrieve Coarsely, Attend Precisely": each query attends over the
// 4 positions of each of its selected blocks plus its own 0-3 tail tokens,
// with softmax and value aggregation over the original K/V; one selection per
// query serves every head.
//
// Neighbouring queries select overlapping blocks (heavy-tailed keys are chosen
// by many queries; early queries see few blocks), so this kernel gathers each
// block once for a tile of UQ = 8 queries:
//   * a pre-pass (union_build_kernel) merges the 8 selections and tail blocks
//     of a query tile into one ascending list of blocks, each with a mask of
//     the queries that attend to it;
//   * a block of a pair of kv heads (4 tokens x 2 heads x 128 dims = 2 KB per
//     tensor) arrives as ONE 5-D TMA box, already in the 128-byte-swizzled
//     layout the tensor cores read: two 8-row atoms (dims 0-63, dims 64-127),
//     row = head * 4 + token.  Measured on B200, the TMA engine's cost is per
//     request, so whole 2 KB blocks issued by four producer warps gather about
//     7x faster than 4-row boxes of one head from one warp;
//   * the 8 queries x 16 q heads of the kv-head pair form the M = 128 rows of
//     two tcgen05 GEMMs per key tile of 16 listed blocks (N = 128 keys):
//       S = Q K^T          (A = Q, staged once per item in shared memory)
//       O_h += P_h V_h     (A = P from tensor memory, B = V tile read MN-major)
//     A row of S pairs each q head with the keys of both kv heads; the other
//     head's keys are masked (p = 0), the price of one 2 KB request per block.
//     Rows are ordered (kv head, query, q head), so each TMEM lane quarter
//     holds the rows of one kv head;
//   * the key tile is split in two column halves h (blocks 0-7, 8-15), each
//     with its own accumulator O_h in tensor memory and its own running
//     maximum: 8 softmax warps, two per TMEM lane quarter (one per half), run
//     the online softmax of their half with no exchange per key tile, rescale
//     their O_h only when their maximum grows by more than 2^64 (lazy
//     rescaling: P is bf16, with fp32's exponent range, so p <= 2^64 and
//     the fp32 sums of O and l stay far from overflow; the final division
//     cancels the common scale),
//     and write P over their half of S as bf16.  At the end of an item the
//     two halves exchange (maximum, sum) through tensor memory and combine:
//       O = (2^(m_0 - m) O_0 + 2^(m_1 - m) O_1) / (2^(m_0 - m) l_0 + 2^(m_1 - m) l_1),
//     m = max(m_0, m_1), the usual merge of two partial softmaxes.
// A masked key contributes p = 0 exactly (the query's mask bit, the other kv
// head, and at the diagonal key position <= query position), so each query's
// result is its own softmax over its own positions.  Warp roles: 0-2 = TMA
// producers, 3 = MMA issuer and TMEM owner, 4-11 = softmax and epilogue (12
// warps leave 168 registers a thread, so the softmax state never spills).  A
// persistent grid walks the work items (sequence, query tile, kv-head pair),
// latest tiles first.
#include <algorithm>

#include "internal.h"

namespace qsa {

namespace {

constexpr int UQ = 8;                  // queries per tile
constexpr int UG = 8;                  // q heads per kv head
constexpr int UH = 2 * UG;             // q heads of a kv-head pair
constexpr int UM = UQ * UH;            // MMA rows
constexpr int UB = 16;                 // listed blocks per key tile
constexpr int UBLK = 2048;             // one block of a kv-head pair, one tensor: 2 atoms of 8 x 128 B
constexpr int UN = UB * 8;             // S columns per tile: 16 blocks x 4 tokens x 2 heads
constexpr int UD = 128;                // head dim
constexpr int UKV = UB * UBLK;         // one tensor's tile (32 KB)
constexpr int USTAGE = 2 * UKV;        // K tile, V tile
constexpr int UPW = 3;                 // producer warps
constexpr int UBPW = (UB + UPW - 1) / UPW;   // blocks per producer warp per tile (the last takes fewer)
#ifndef QSA_UT_STAGES
#define QSA_UT_STAGES 3
#endif
constexpr int UNS = QSA_UT_STAGES;     // key tiles in flight
constexpr int UPRE = 4;                // key tiles whose block ids the producers hold ahead
#ifndef QSA_UT_SHARE
#define QSA_UT_SHARE 2
#endif
constexpr int kShare = QSA_UT_SHARE;   // queries of a tile that must attend to a block for the tile list
constexpr int UW_MMA = UPW;            // warp index of the MMA issuer
constexpr int USW = 8;                 // softmax warps: two per TMEM lane quarter, one per column half
constexpr int UT_THREADS = (UPW + 1 + USW) * 32;
constexpr int UQH = UM * 128;          // Q in shared memory: one 64-dim half of 128 rows (16 KB)
constexpr uint32_t TM_S = 0;           // S / P, two buffers of 128 columns
constexpr uint32_t TM_O = 256;         // O_0, O_1: 128 columns each
constexpr uint32_t TM_COLS = 512;
constexpr int UCHUNK = 32768;          // pre-pass: block ids per pass (a one-byte query mask each: 32 KB)
constexpr float kLog2e = 1.4426950408889634f;
#ifndef QSA_UT_RESCALE
#define QSA_UT_RESCALE 64.f
#endif
constexpr float kRescale = QSA_UT_RESCALE;   // lazy rescale threshold (log2 units)

struct UtMeta {
    int32_t id[UB];                    // listed block ids of the tile (-1: padding)
    uint32_t mw[UQ];                   // per query: bit j = the query attends to block j of the tile
    int32_t diag;                      // a block of the tile reaches past the tile's first query
    int32_t pad[7];
};

struct UtSmem {
    alignas(1024) uint8_t kv[UNS][USTAGE];
    alignas(1024) uint8_t q[2 * UQH];              // Q: dims 0-63 | dims 64-127, rows of 128 B, 128-B swizzle
    UtMeta meta[UNS];
    uint64_t full[UNS], empty[UNS];
    uint64_t q_ready;
    uint64_t s_full[2], p_ready[2], pv_done, o_full, drain;
    uint32_t tmem_base;
};

static_assert(sizeof(UtSmem) + 1024 <= 232448, "shared memory of the attention CTA exceeds 227 KB");

struct UtParams {
    const __nv_bfloat16 *q;  // [B][n_q][Hq][128]
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
    __nv_bfloat16 *out;      // in: the gather kernel's result over each query's own blocks; out: the total
    const float *lse_q;      // [B][n_q][Hq] its log-sum-exp (natural log)
    float *lse;
    unsigned *status;
    int64_t items;
};

struct UtItem {
    int seq, pair, nrows, n_u;
    int64_t r0, t0;
    const uint32_t *ids;
    const uint16_t *msk;
};

__device__ __forceinline__ UtItem ut_item(const UtParams &p, int64_t i) {
    UtItem it;
    const int npair = p.Hkv / 2;
    const int64_t per = (int64_t)p.B * npair;
    const int64_t qt = p.n_qt - 1 - i / per;   // latest (longest) query tiles first
    const int rem = (int)(i % per);
    it.seq = rem / npair;
    it.pair = rem % npair;
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
// One CTA per query tile of a one-sequence view.  Block ids of the tile's
// selections (validated: 0 <= b < nb(t)) and each query's tail block (when it
// holds 1-3 tokens) set bit q of a one-byte mask per id (four ids to a 32-bit
// word).  Ids are processed UCHUNK at a time, in id order; each non-zero mask
// goes
//   * to the tile's block list (id, mask) when at least kShare queries of the
//     tile attend to it, or it is some query's tail block (the tile kernel
//     masks the tail's later positions): its K/V is gathered once for all;
//   * otherwise to the own list of its one query (sel1 [rows][top_k],
//     ascending ids, counts in nsel1), which the per-query gather kernel
//     attends to (full blocks only).
// Thread tid owns words [tid W, tid W + W) of a chunk; one block-wide
// exclusive scan of its nine counts (list entries, and own-list entries per
// query) gives every destination position.
constexpr int kScanN = UQ + 1;

__device__ __forceinline__ void block_exclusive_scan9(int (&v)[kScanN], int (*s_w)[8], int (&total)[kScanN]) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl[kScanN];
#pragma unroll
    for (int j = 0; j < kScanN; ++j) incl[j] = v[j];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1)
#pragma unroll
        for (int j = 0; j < kScanN; ++j) {
            const int y = __shfl_up_sync(0xffffffffu, incl[j], o);
            if (lane >= o) incl[j] += y;
        }
    if (lane == 31)
#pragma unroll
        for (int j = 0; j < kScanN; ++j) s_w[j][warp] = incl[j];
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kScanN; ++j) {
        int before = 0, tot = 0;
#pragma unroll
        for (int w = 0; w < 8; ++w) {
            const int x = s_w[j][w];
            before += (w < warp) ? x : 0;
            tot += x;
        }
        total[j] = tot;
        v[j] = before + incl[j] - v[j];
    }
    __syncthreads();
}

__global__ void __launch_bounds__(256) union_build_kernel(const int32_t *__restrict__ sel,
                                                          const int32_t *__restrict__ nsel, int64_t n_q, int64_t q0,
                                                          int top_k, int64_t n_qt, int cap,
                                                          int32_t *__restrict__ u_count, uint32_t *__restrict__ u_id,
                                                          uint16_t *__restrict__ u_mask, int32_t *__restrict__ sel1,
                                                          int32_t *__restrict__ nsel1, unsigned *status) {
    extern __shared__ uint32_t ub_words[];   // UCHUNK / 4 words: byte j of word w = mask of id 4 w + j
    __shared__ int s_nsel[UQ];
    __shared__ int64_t s_tail[UQ];           // the query's tail block, or -1
    __shared__ int s_w[kScanN][8];
    const int tid = threadIdx.x;
    const int64_t qt = blockIdx.x;
    const int64_t r0 = qt * UQ;
    const int nrows = (int)(n_q - r0 < UQ ? n_q - r0 : UQ);
    pdl_wait();       // the selection comes from the previous kernel
    pdl_trigger();
    if (tid < UQ) {
        s_nsel[tid] = tid < nrows ? max(0, min(nsel[r0 + tid], top_k)) : 0;
        const int64_t t = q0 + r0 + tid;
        s_tail[tid] = (tid < nrows && (t + 1) % kBlock != 0) ? (t + 1) / kBlock : -1;
    }
    __syncthreads();
    const int64_t t_last = q0 + r0 + nrows - 1;
    const int64_t id_end = t_last / kBlock + 1;            // the last query's tail block, exclusive
    // the tile's tail blocks are consecutive: [tail_lo, tail_hi]
    int64_t tail_lo = INT64_MAX, tail_hi = -1;
#pragma unroll
    for (int q = 0; q < UQ; ++q)
        if (s_tail[q] >= 0) {
            tail_lo = min(tail_lo, s_tail[q]);
            tail_hi = max(tail_hi, s_tail[q]);
        }
    uint32_t *oid = u_id + qt * cap;
    uint16_t *om = u_mask + qt * cap;
    int count = 0;
    int qcount[UQ];
#pragma unroll
    for (int q = 0; q < UQ; ++q) qcount[q] = 0;
    for (int64_t c0 = 0; c0 < id_end; c0 += UCHUNK) {
        const int span = (int)(id_end - c0 < UCHUNK ? id_end - c0 : UCHUNK);
        const int nw = (span + 3) / 4;
        for (int i = tid; i < nw; i += 256) ub_words[i] = 0;
        __syncthreads();
        for (int q = 0; q < nrows; ++q) {
            const int64_t t = q0 + r0 + q;
            const int32_t *row = sel + (r0 + q) * top_k;
            for (int k = tid; k < s_nsel[q]; k += 256) {
                const int32_t b = row[k];
                if (b < 0 || (int64_t)b >= (t + 1) / kBlock) {
                    if (c0 == 0) flag(status, QSA_DEV_BAD_INDEX);
                    continue;
                }
                if (b >= c0 && b < c0 + span) {
                    const int rel = (int)(b - c0);
                    atomicOr(&ub_words[rel >> 2], 1u << (8 * (rel & 3) + q));
                }
            }
        }
        if (tid < UQ && s_tail[tid] >= c0 && s_tail[tid] < c0 + span) {
            const int rel = (int)(s_tail[tid] - c0);
            atomicOr(&ub_words[rel >> 2], 1u << (8 * (rel & 3) + tid));
        }
        __syncthreads();
        const int W = (nw + 255) / 256;
        auto listed = [&](uint32_t m, int64_t id) {
            return __popc(m) >= kShare || (id >= tail_lo && id <= tail_hi);
        };
        int cnt[kScanN];
#pragma unroll
        for (int j = 0; j < kScanN; ++j) cnt[j] = 0;
        for (int i = 0; i < W; ++i) {
            const int w = tid * W + i;
            const uint32_t word = w < nw ? ub_words[w] : 0u;
            if (!word) continue;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t m = (word >> (8 * j)) & 0xFFu;
                if (!m) continue;
                if (listed(m, c0 + 4 * w + j)) ++cnt[UQ];
                else
#pragma unroll
                    for (int q = 0; q < UQ; ++q) cnt[q] += (m >> q) & 1u;
            }
        }
        int total[kScanN];
        block_exclusive_scan9(cnt, s_w, total);   // cnt: this thread's first positions
        int pos = count + cnt[UQ];
        count += total[UQ];
        int qpos[UQ];
#pragma unroll
        for (int q = 0; q < UQ; ++q) {
            qpos[q] = qcount[q] + cnt[q];
            qcount[q] += total[q];
        }
        for (int i = 0; i < W; ++i) {
            const int w = tid * W + i;
            const uint32_t word = w < nw ? ub_words[w] : 0u;
            if (!word) continue;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t m = (word >> (8 * j)) & 0xFFu;
                if (!m) continue;
                const int64_t id = c0 + 4 * w + j;
                if (listed(m, id)) {
                    if (pos < cap) {
                        oid[pos] = (uint32_t)id;
                        om[pos] = (uint16_t)m;
                    }
                    ++pos;
                } else {
#pragma unroll
                    for (int q = 0; q < UQ; ++q)
                        if ((m >> q) & 1u) {
                            if (qpos[q] < top_k) sel1[(r0 + q) * top_k + qpos[q]] = (int32_t)id;
                            ++qpos[q];
                        }
                }
            }
        }
        __syncthreads();
    }
    if (tid == 0) u_count[qt] = min(count, cap);
#pragma unroll
    for (int q = 0; q < UQ; ++q)
        if (tid == q && q < nrows) nsel1[r0 + q] = min(qcount[q], top_k);
}

// ---------------------------------------------------------------- attention
__global__ void __launch_bounds__(UT_THREADS, 1)
    attn_union_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                      UtParams p) {
    extern __shared__ uint8_t ut_raw[];
    UtSmem &sm = *reinterpret_cast<UtSmem *>((reinterpret_cast<uintptr_t>(ut_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // zero the K/V stages once: rows of padding entries are never loaded, and
    // their (masked) products must stay finite
    for (int i = threadIdx.x; i < (int)(sizeof(sm.kv) / 16); i += blockDim.x)
        reinterpret_cast<uint4 *>(&sm.kv[0][0])[i] = make_uint4(0, 0, 0, 0);
    if (threadIdx.x == 0) {
        for (int s = 0; s < UNS; ++s) {
            mbar_init(&sm.full[s], 32 + UPW - 1);   // warp 0's lanes (they write the meta), lane 0 of the others
            mbar_init(&sm.empty[s], 1);
        }
        mbar_init(&sm.q_ready, USW);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.s_full[b], 1);
            mbar_init(&sm.p_ready[b], USW);
        }
        mbar_init(&sm.pv_done, 1);
        mbar_init(&sm.o_full, 1);
        mbar_init(&sm.drain, 1);
        fence_mbar_init();
    }
    if (warp == UW_MMA) {
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

    if (warp < UPW) {
        // ------------------------------------------------------------ TMA producers
        // Every producer warp reads the tile's 16 entries (lanes 0-15); warp 0
        // writes the tile's meta, warp w issues the boxes of blocks
        // [UBPW w, UBPW w + UBPW).
        if (warp == 0 && lane == 0) {
            prefetch_tmap(&map_k);
            prefetch_tmap(&map_v);
        }
        int64_t c = 0;   // stages issued
        int st = 0;      // stage of the next tile
        uint32_t eph = 1;   // parity of the empty phase to wait for (the first round waits for nothing)
        bool ok = true;
        for (int64_t i = blockIdx.x; i < p.items && ok; i += gridDim.x) {
            const UtItem it = ut_item(p, i);
            const int ntile = (it.n_u + UB - 1) / UB;
            const bool rl = lane < UB;
            // the entries of the next UPRE key tiles are in flight (lanes 0-15 of each warp):
            // one tile ahead leaves every stage waiting a full L2 round trip for its ids
            uint32_t rid[UPRE], rmk[UPRE];
#pragma unroll
            for (int k = 0; k < UPRE; ++k) {
                const int x = k * UB + lane;
                rid[k] = (rl && x < it.n_u) ? __ldg(it.ids + x) : 0xFFFFFFFFu;
                rmk[k] = (rl && x < it.n_u) ? (uint32_t)__ldg(it.msk + x) : 0u;
            }
            for (int u0 = 0; u0 < ntile && ok; u0 += UPRE) {
#pragma unroll
                for (int k = 0; k < UPRE; ++k) {
                    const int u = u0 + k;
                    if (u >= ntile) break;
                    const uint32_t e_id = rid[k], e_m = rmk[k];
                    {
                        const int x = (u + UPRE) * UB + lane;
                        rid[k] = (rl && x < it.n_u) ? __ldg(it.ids + x) : 0xFFFFFFFFu;
                        rmk[k] = (rl && x < it.n_u) ? (uint32_t)__ldg(it.msk + x) : 0u;
                    }
                    const int s = st;
                    if (c >= UNS) ok = mbar_wait(&sm.empty[s], eph, p.status);
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                    const bool live = e_id != 0xFFFFFFFFu;
                    if (warp == 0) {
                        UtMeta &mt = sm.meta[s];
                        if (rl) mt.id[lane] = live ? (int32_t)e_id : -1;
                        uint32_t mine = 0;
#pragma unroll
                        for (int q = 0; q < UQ; ++q) {
                            const uint32_t b = __ballot_sync(0xffffffffu, (e_m >> q) & 1u);
                            if (lane == q) mine = b;
                        }
                        if (lane < UQ) mt.mw[lane] = mine;
                        const int maxid = __reduce_max_sync(0xffffffffu, live ? (int)e_id : -1);
                        if (lane == 0) mt.diag = ((int64_t)kBlock * maxid + kBlock - 1 > it.t0) ? 1 : 0;
                    }
                    const bool mine_blk = lane >= UBPW * warp && lane < UBPW * (warp + 1);
                    const uint32_t nlive = __popc(__ballot_sync(0xffffffffu, live && mine_blk));
                    __syncwarp();
                    if (lane == 0) mbar_arrive_expect_tx(&sm.full[s], nlive * 2u * UBLK);
                    else if (warp == 0) mbar_arrive(&sm.full[s]);
                    __syncwarp();
                    if (live && mine_blk) {
                        uint8_t *dst = sm.kv[s] + lane * UBLK;
                        const int tok = kBlock * (int)e_id;
                        tma_load_5d(dst, &map_k, 0, tok, 2 * it.pair, 0, it.seq, &sm.full[s]);
                        tma_load_5d(dst + UKV, &map_v, 0, tok, 2 * it.pair, 0, it.seq, &sm.full[s]);
                    }
                    ++c;
                    if (++st == UNS) {
                        st = 0;
                        eph ^= 1u;
                    }
                }
            }
        }
        // no copy may still be landing when the CTA ends (bounded waits)
        if (lane == 0)
            for (int64_t cc = (c > UNS ? c - UNS : 0); cc < c; ++cc)
                mbar_wait(&sm.full[cc % UNS], (int)((cc / UNS) & 1), p.status);
    } else if (warp == UW_MMA) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc_qk = idesc_bf16_f32(UM, UN);
            const uint32_t idesc_pv = idesc_bf16_f32(UM, UD) | (1u << 16);   // B = V tile, MN-major
            // shared-memory descriptors: the start address (bits 0-13, 16-byte units) of each
            // operand advances by adding to the descriptor of stage 0 / k-step 0
            const uint64_t dq = sw128_desc(smem_u32(sm.q));                     // Q, 8-row groups 1024 B apart
            const uint64_t dk0 = sw128_desc_ls(smem_u32(sm.kv[0]), 16, UBLK);  // K tile, 8-row groups 2048 B apart
            const uint64_t dv0 = sw128_desc_ls(smem_u32(sm.kv[0]) + UKV, 1024, UBLK);   // V tile, MN-major
            constexpr uint64_t kStageD = USTAGE >> 4;
            int64_t c = 0, ic = 0;
            int qs = 0, ps = 0;      // stages of the next QK and the next P V
            uint32_t qph = 0;        // phase of the next QK's stage
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
                        ok = mbar_wait(&sm.full[qs], qph, p.status);
                        if (!ok) break;
                        tc_fence_after();
                        const uint32_t d = tmem + TM_S + (uint32_t)((cu & 1) * 128);
                        const uint64_t dk = dk0 + (uint64_t)qs * kStageD;
                        // k-step k: dims 16 k .. 16 k + 15 = 32-byte column (k & 3) of the 64-dim half k >> 2
                        // (Q: halves 16 KB apart; K tile: block j's dims 0-63 atom at 2048 j, dims 64-127 at + 1024)
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            tc_mma_f16(d, dq + (uint64_t)(((k >> 2) * UQH + (k & 3) * 32) >> 4),
                                       dk + (uint64_t)(((k >> 2) * 1024 + (k & 3) * 32) >> 4), idesc_qk,
                                       k > 0 ? 1u : 0u);
                        tc_commit(&sm.s_full[cu & 1]);
                        if (++qs == UNS) {
                            qs = 0;
                            qph ^= 1u;
                        }
                    }
                    if (u >= 1) {      // O_h += P_h(u-1) V_h(u-1), h = 0, 1
                        const int64_t cp = c + u - 1;
                        ok = mbar_wait(&sm.p_ready[cp & 1], (int)((cp >> 1) & 1), p.status);
                        if (!ok) break;
                        tc_fence_after();
                        const uint64_t dv = dv0 + (uint64_t)ps * kStageD;
                        const uint32_t pa = tmem + TM_S + (uint32_t)((cp & 1) * 128);
                        // P_h: 32 columns at 64 h (keys 64 h .. 64 h + 63); V tile MN-major, 16 rows
                        // (2 blocks) per k-step, dims 64-127 one atom (1024 B) on
#pragma unroll
                        for (int h = 0; h < 2; ++h)
#pragma unroll
                            for (int k = 0; k < 4; ++k)
                                tc_mma_ts(tmem + TM_O + 128 * h, pa + 64 * h + 8 * k,
                                          dv + (uint64_t)(((4 * h + k) * 2 * UBLK) >> 4), idesc_pv,
                                          (u > 1 || k > 0) ? 1u : 0u);
                        tc_commit(&sm.empty[ps]);
                        tc_commit(&sm.pv_done);
                        if (++ps == UNS) ps = 0;
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
        // TMEM lane (row) = 64 hd + 8 query + q head: quarters 0-1 hold kv head 0 of the
        // pair, quarters 2-3 kv head 1.  Warp (quarter, hf) owns S columns [64 hf, 64 hf + 64)
        // (blocks 8 hf .. 8 hf + 7 of the key tile), their running maximum and sum, the
        // accumulator O_hf, and writes Q dims [64 hf, 64 hf + 64) and output dims of the same range.
        const int sw = warp - (UW_MMA + 1);
        const int quarter = warp & 3;
        const int hf = sw >> 2;
        const int row = quarter * 32 + lane;
        const int hd = quarter >> 1;                    // kv head within the pair (warp-uniform)
        const int qi = (row >> 3) & (UQ - 1);           // query of the tile
        const int hq = row & (UG - 1);                  // q head within the kv head's group
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        const uint32_t o_own = lane_base + TM_O + 128 * hf;
        const uint32_t o_oth = lane_base + TM_O + 128 * (hf ^ 1);
        uint8_t *qrow = sm.q + hf * UQH + (row >> 3) * 1024 + (row & 7) * 128;
        const float sl2 = p.scale_log2;
        int64_t c = 0, ic = 0;
        int ms = 0;           // stage of the tile's meta
        uint32_t mph = 0;     // its phase
        bool ok = true;
        for (int64_t i = blockIdx.x; i < p.items && ok; i += gridDim.x, ++ic) {
            const UtItem it = ut_item(p, i);
            const int ntile = (it.n_u + UB - 1) / UB;
            const int64_t tq = it.t0 + qi;
            const int head = UH * it.pair + UG * hd + hq;
            // Q: this row's dims [64 hf, 64 hf + 64) -> shared memory, 128-byte swizzle (rows
            // past the tile's queries hold zeros).  Every QK product of the previous item is
            // complete: its O was read after its last product.
            {
                const bool qlive = qi < it.nrows;
                const uint4 *src = reinterpret_cast<const uint4 *>(
                    p.q + (((int64_t)it.seq * p.n_q + it.r0 + (qlive ? qi : 0)) * p.Hq + head) * UD + 64 * hf);
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    const uint4 v = qlive ? __ldg(src + ch) : make_uint4(0, 0, 0, 0);
                    *reinterpret_cast<uint4 *>(qrow + ((ch ^ (row & 7)) << 4)) = v;
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.q_ready);
            float m_run = -INFINITY, l_run = 0.f;
            for (int u = 0; u < ntile; ++u, ++c) {
                const int s = ms;
                const uint32_t sph = mph;
                if (++ms == UNS) {
                    ms = 0;
                    mph ^= 1u;
                }
                bool w_ok = mbar_wait(&sm.s_full[c & 1], (int)((c >> 1) & 1), p.status);
                if (w_ok) w_ok = mbar_wait(&sm.full[s], sph, p.status);   // the tile's meta
                ok = __all_sync(0xffffffffu, w_ok);
                if (!ok) break;
                tc_fence_after();
                const UtMeta &mt = sm.meta[s];
                const uint32_t mw = (mt.mw[qi] >> (8 * hf)) & 0xFFu;          // this half's 8 blocks
                const bool diag = mt.diag != 0;
                const uint32_t sbuf = lane_base + TM_S + (uint32_t)((c & 1) * 128);
                // S column 64 hf + 8 j + 4 h + tk: block 8 hf + j, kv head h of the pair, token tk;
                // xs[4 j + tk] = this row's kv head hd
                uint32_t sv[64], xs[32];
                tmem_ld32(sbuf + 64 * hf, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
                tmem_ld32(sbuf + 64 * hf + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
                tc_wait_ld();
#pragma unroll
                for (int j = 0; j < 8; ++j)
#pragma unroll
                    for (int tk = 0; tk < kBlock; ++tk) xs[4 * j + tk] = hd ? sv[8 * j + 4 + tk] : sv[8 * j + tk];
                // the keys this row attends to: bit 4 j + tk of vm (the query's mask bit; at the
                // diagonal also key position <= query position)
                uint32_t vm = 0;
#pragma unroll
                for (int j = 0; j < 8; ++j) vm |= ((mw >> j) & 1u) ? (0xFu << (4 * j)) : 0u;
                if (diag) {
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int64_t lim = tq - (int64_t)kBlock * mt.id[8 * hf + j];   // tokens tk <= lim
                        const uint32_t tm = lim >= kBlock - 1 ? 0xFu : (lim < 0 ? 0u : ((2u << lim) - 1u));
                        vm &= ~(0xFu << (4 * j)) | (tm << (4 * j));
                    }
                }
                // pass 1: the row maximum.  The maximum over all of the half's scores bounds the one
                // over the keys this row attends to; only when it could move the running maximum
                // by more than the threshold is the exact (masked) maximum taken.  (sl2 > 0)
                float m4[4] = {__uint_as_float(xs[0]), __uint_as_float(xs[1]), __uint_as_float(xs[2]),
                               __uint_as_float(xs[3])};
#pragma unroll
                for (int e = 4; e < 32; ++e) m4[e & 3] = fmaxf(m4[e & 3], __uint_as_float(xs[e]));
                float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * sl2;
                bool grow = false;
                if (__any_sync(0xffffffffu, mx > m_run + kRescale)) {
#pragma unroll
                    for (int k = 0; k < 4; ++k) m4[k] = -INFINITY;
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        m4[e & 3] = fmaxf(m4[e & 3], ((vm >> e) & 1u) ? __uint_as_float(xs[e]) : -INFINITY);
                    mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * sl2;
                    grow = mx > m_run + kRescale;               // also the first keys of the row
                }
                const bool resc = grow && m_run != -INFINITY;  // O_hf and l already hold earlier keys
                if (__any_sync(0xffffffffu, resc)) {
                    // the previous P V must have landed before O is read.  A parity
                    // wait is exact here: S(c) landing means every MMA issued before
                    // QK(c) is done, P V(c - 2) included, and P V(c) needs this
                    // warp's P(c), so pv_done is at phase c - 1 or c.
                    ok = __all_sync(0xffffffffu, mbar_wait(&sm.pv_done, (int)((c - 1) & 1), p.status));
                    if (!ok) break;
                    tc_fence_after();
                    const float alpha = resc ? ex2_approx(m_run - mx) : 1.f;
#pragma unroll 1
                    for (int ch = 0; ch < 8; ++ch) {   // rare: kept rolled, so its loads do not crowd the registers
                        uint32_t ov[16];
                        tmem_ld16(o_own + 16 * ch, ov);
                        tc_wait_ld();
#pragma unroll
                        for (int e = 0; e < 16; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
                        tmem_st16(o_own + 16 * ch, ov);
                    }
                    tc_wait_st();
                    l_run *= alpha;
                }
                if (grow) m_run = mx;
                const float mneg = (m_run == -INFINITY) ? 0.f : -m_run;
                // pass 2: p for this row's keys (2^-inf = 0 for the others), P (bf16 pairs) over this
                // half's S columns: word 64 hf + 4 j + 2 h + tk / 2 holds tokens tk, tk + 1 of kv head
                // h of block j; the other kv head's words are zero
                float pv[32];
                float l4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    pv[e] = ex2_approx(((vm >> e) & 1u) ? fmaf(__uint_as_float(xs[e]), sl2, mneg) : -INFINITY);
                    l4[e & 3] += pv[e];
                }
                uint32_t pk[32];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint32_t w0 = pack_bf16(pv[4 * j], pv[4 * j + 1]), w1 = pack_bf16(pv[4 * j + 2], pv[4 * j + 3]);
                    pk[4 * j] = hd ? 0u : w0;
                    pk[4 * j + 1] = hd ? 0u : w1;
                    pk[4 * j + 2] = hd ? w0 : 0u;
                    pk[4 * j + 3] = hd ? w1 : 0u;
                }
                const float ls = (l4[0] + l4[1]) + (l4[2] + l4[3]);
                tmem_st32(sbuf + 64 * hf, pk);
                l_run += ls;
                tc_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.p_ready[c & 1]);
            }
            if (!ok) break;
            // epilogue.  o_full: every product of the item is done, so both S buffers
            // are free until the next item's Q is staged; the halves exchange (m, l)
            // through columns [4 hf, 4 hf + 4) of S buffer 0.
            ok = __all_sync(0xffffffffu, mbar_wait(&sm.o_full, (int)(ic & 1), p.status));
            if (!ok) break;
            tc_fence_after();
            {
                const uint32_t xv[4] = {__float_as_uint(m_run), __float_as_uint(l_run), 0u, 0u};
                tmem_st4(lane_base + TM_S + 4 * hf, xv);
                tc_wait_st();
            }
            tc_fence_before();
            named_bar_sync(1, USW * 32);
            tc_fence_after();
            uint32_t yv[4];
            tmem_ld4(lane_base + TM_S + 4 * (hf ^ 1), yv);
            tc_wait_ld();
            const float m_oth = __uint_as_float(yv[0]), l_oth = __uint_as_float(yv[1]);
            // merge three partial softmaxes of the row: the two column halves of the listed
            // blocks, and the gather kernel's (its own blocks and tail; out_q normalised, so its
            // weight is 2^lse_q)
            const bool live = qi < it.nrows;
            const int64_t orow = ((int64_t)it.seq * p.n_q + it.r0 + qi) * p.Hq + head;
            const float lq = live ? p.lse_q[orow] * kLog2e : -INFINITY;
            const bool tile = ntile > 0;
            const float m_all = fmaxf(tile ? fmaxf(m_run, m_oth) : -INFINITY, lq);
            const bool any = m_all != -INFINITY;
            const float a_own = (any && tile) ? ex2_approx(m_run - m_all) : 0.f;
            const float a_oth = (any && tile) ? ex2_approx(m_oth - m_all) : 0.f;
            const float a_q = any ? ex2_approx(lq - m_all) : 0.f;
            const float l_tot = a_own * l_run + a_oth * l_oth + a_q;
            const float inv = l_tot > 0.f ? 1.f / l_tot : 0.f;
            const float c_own = a_own * inv, c_oth = a_oth * inv, c_q = a_q * inv;
            __nv_bfloat16 *dst = p.out + orow * UD + 64 * hf;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                uint32_t o0[16], o1[16];
                tmem_ld16(o_own + 64 * hf + 16 * ch, o0);
                tmem_ld16(o_oth + 64 * hf + 16 * ch, o1);
                uint4 q4[2] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
                if (live) {
                    q4[0] = *reinterpret_cast<const uint4 *>(dst + 16 * ch);
                    q4[1] = *reinterpret_cast<const uint4 *>(dst + 16 * ch + 8);
                }
                tc_wait_ld();
                if (live) {
                    const uint32_t *qw = reinterpret_cast<const uint32_t *>(q4);
                    uint32_t w[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        // nothing was accumulated without a listed block: TMEM holds no values then
                        const float x0 = tile ? __uint_as_float(o0[2 * e]) * c_own + __uint_as_float(o1[2 * e]) * c_oth : 0.f;
                        const float x1 = tile ? __uint_as_float(o0[2 * e + 1]) * c_own +
                                                    __uint_as_float(o1[2 * e + 1]) * c_oth
                                              : 0.f;
                        const float y0 = __uint_as_float(qw[e] << 16), y1 = __uint_as_float(qw[e] & 0xFFFF0000u);
                        w[e] = pack_bf16(fmaf(y0, c_q, x0), fmaf(y1, c_q, x1));
                    }
                    *reinterpret_cast<uint4 *>(dst + 16 * ch) = make_uint4(w[0], w[1], w[2], w[3]);
                    *reinterpret_cast<uint4 *>(dst + 16 * ch + 8) = make_uint4(w[4], w[5], w[6], w[7]);
                }
            }
            if (live && hf == 0 && p.lse) p.lse[orow] = l_tot > 0.f ? (m_all + log2f(l_tot)) / kLog2e : -INFINITY;
            tc_fence_before();
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == UW_MMA) {
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

// Rows of one chunk and the layout of its workspace.
struct UnionPlan {
    int cap;             // list entries per query tile
    int64_t rows;        // query rows per chunk (a multiple of UQ)
    size_t count_bytes, id_bytes, mask_bytes, sel1_bytes, nsel1_bytes, lse_bytes;
    size_t total() const { return count_bytes + id_bytes + mask_bytes + sel1_bytes + nsel1_bytes + lse_bytes; }
};

constexpr size_t kUnionBudget = (size_t)1 << 30;   // workspace cap; longer prompts run in several chunks

UnionPlan union_plan(int64_t n_q, int top_k, int Hq) {
    UnionPlan u{};
    // each listed block holds >= kShare of the 8 x top_k selections, or is one of the <= 3 tail blocks
    u.cap = (UQ * top_k / kShare + 3 + UB) / UB * UB;
    const size_t per_row = (size_t)u.cap * 6 / UQ + 4 + (size_t)top_k * 4 + 4 + (size_t)Hq * 4;
    const int64_t want = (n_q + UQ - 1) / UQ * UQ;
    const int64_t fit = std::max<int64_t>(UQ, (int64_t)(kUnionBudget / per_row) / UQ * UQ);
    u.rows = std::min(want, fit);
    const int64_t tiles = u.rows / UQ;
    auto r256 = [](size_t x) { return (x + 255) / 256 * 256; };
    u.count_bytes = r256((size_t)tiles * 4);
    u.id_bytes = r256((size_t)tiles * u.cap * 4);
    u.mask_bytes = r256((size_t)tiles * u.cap * 2);
    u.sel1_bytes = r256((size_t)u.rows * top_k * 4);
    u.nsel1_bytes = r256((size_t)u.rows * 4);
    u.lse_bytes = r256((size_t)u.rows * Hq * 4);
    return u;
}

}  // namespace

bool attn_union_supported(const AttnArgs &a) {
    // Longer contexts take the gather kernel alone: their block ids no longer fit one
    // pre-pass chunk, and measured at 1M tokens in 16,000-token chunks the split was slower
    // (attention 193 vs 160 ms).
    return !a.decode && !a.kv8 && a.d == UD && a.Hq == UG * a.Hkv && (a.Hkv == 2 || a.Hkv == 4) && !a.pg.table &&
           (a.q0 + a.n_q) / kBlock <= UCHUNK;
}

size_t attn_union_ws_bytes(int B, int64_t n_q, int top_k, int Hq) {
    if (B < 1 || n_q < 1) return 0;
    return union_plan(n_q, top_k, Hq).total();
}

int attn_union_launches(int B, int64_t n_q, int top_k, int Hq) {
    if (B < 1 || n_q < 1) return 0;
    const UnionPlan u = union_plan(n_q, top_k, Hq);
    return B * (int)((n_q + u.rows - 1) / u.rows);
}

cudaError_t launch_attn_union(const AttnArgs &a, void *ws, unsigned *status, cudaStream_t s) {
    if (a.n_q <= 0) return cudaSuccess;
    const DeviceInfo *di = device_info();
    const int sms = di ? di->sm_count : 148;
    const UnionPlan u = union_plan(a.n_q, a.top_k, a.Hq);
    uint8_t *w = static_cast<uint8_t *>(ws);
    int32_t *u_count = reinterpret_cast<int32_t *>(w);
    w += u.count_bytes;
    uint32_t *u_id = reinterpret_cast<uint32_t *>(w);
    w += u.id_bytes;
    uint16_t *u_mask = reinterpret_cast<uint16_t *>(w);
    w += u.mask_bytes;
    int32_t *sel1 = reinterpret_cast<int32_t *>(w);
    w += u.sel1_bytes;
    int32_t *nsel1 = reinterpret_cast<int32_t *>(w);
    w += u.nsel1_bytes;
    float *lse_q = reinterpret_cast<float *>(w);

    auto enc = get_encode_fn();
    if (!enc) return cudaErrorInvalidValue;
    const size_t smem = sizeof(UtSmem) + 1024;
    if (di && smem > di->smem_optin) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(attn_union_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(union_build_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, UCHUNK);
    if (e != cudaSuccess) return e;
    const size_t qrow = (size_t)a.Hq * UD;                 // elements of one query row of q / out
    const size_t kvseq = (size_t)a.kv_stride * a.Hkv * UD;  // elements of one sequence's cache
    for (int b = 0; b < a.B; ++b) {
        CUtensorMap mk, mv;
        // the sequence's k, v: [kv_stride][Hkv][128] seen as (64 dims, token, kv head, dim half); a box of
        // 64 dims x 4 tokens x 2 heads x 2 halves lands as [half][head][token][64 dims]
        for (int t = 0; t < 2; ++t) {
            const cuuint64_t row = (cuuint64_t)a.Hkv * UD * 2;
            cuuint64_t dims[5] = {64, (cuuint64_t)a.kv_stride, (cuuint64_t)a.Hkv, 2, 1};
            cuuint64_t strides[4] = {row, UD * 2, 128, (cuuint64_t)a.kv_stride * row};
            cuuint32_t box[5] = {64, kBlock, 2, 2, 1};
            cuuint32_t estr[5] = {1, 1, 1, 1, 1};
            const __nv_bfloat16 *base = static_cast<const __nv_bfloat16 *>(t ? a.v : a.k) + (size_t)b * kvseq;
            if (enc(t ? &mv : &mk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<__nv_bfloat16 *>(base), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                return cudaErrorInvalidValue;
        }
        for (int64_t r = 0; r < a.n_q; r += u.rows) {
            // rows [r, r + rows) of sequence b as a one-sequence problem
            const int64_t rows = std::min(u.rows, a.n_q - r);
            const int64_t n_qt = (rows + UQ - 1) / UQ;
            const int64_t row_g = (int64_t)b * a.n_q + r;       // first row in the [B][n_q] layouts
            const int32_t *sel_c = a.sel + row_g * a.top_k;
            const int32_t *nsel_c = a.nsel + row_g;
            const __nv_bfloat16 *q_c = static_cast<const __nv_bfloat16 *>(a.q) + row_g * qrow;
            __nv_bfloat16 *out_c = static_cast<__nv_bfloat16 *>(a.out) + row_g * qrow;
            // 1. block lists of the shared blocks, own lists of the others
            e = launch_pdl(union_build_kernel, dim3((unsigned)n_qt), dim3(256), (size_t)UCHUNK, s, sel_c,
                           nsel_c, rows, a.q0 + r, a.top_k, n_qt, u.cap, u_count, u_id, u_mask, sel1, nsel1,
                           status);
            if (e != cudaSuccess) return e;
            // 2. each query over its own blocks and its tail (gather kernel): out, lse_q
            AttnArgs g = a;
            g.q = q_c;
            g.k = static_cast<const __nv_bfloat16 *>(a.k) + (size_t)b * kvseq;
            g.v = static_cast<const __nv_bfloat16 *>(a.v) + (size_t)b * kvseq;
            g.sel = sel1;
            g.nsel = nsel1;
            g.B = 1;
            g.n_q = rows;
            g.q0 = a.q0 + r;
            g.out = out_c;
            g.lse = lse_q;
            g.no_tail = true;
            e = launch_attn_bf16(g, nullptr, status, s);
            if (e != cudaSuccess) return e;
            // 3. the tiles over their shared blocks, merged with step 2
            UtParams p{};
            p.q = q_c;
            p.B = 1;
            p.n_q = rows;
            p.q0 = a.q0 + r;
            p.Hq = a.Hq;
            p.Hkv = a.Hkv;
            p.row0 = 0;
            p.row_end = rows;
            p.n_qt = n_qt;
            p.cap = u.cap;
            p.u_count = u_count;
            p.u_id = u_id;
            p.u_mask = u_mask;
            p.scale_log2 = a.scale * kLog2e;
            p.out = out_c;
            p.lse_q = lse_q;
            p.lse = a.lse ? a.lse + row_g * a.Hq : nullptr;
            p.status = status;
            p.items = n_qt * (a.Hkv / 2);
            const int64_t grid = std::min<int64_t>(p.items, sms);
            e = launch_pdl(attn_union_kernel, dim3((unsigned)grid), dim3(UT_THREADS), smem, s, mk, mv, p);
            if (e != cudaSuccess) return e;
        }
    }
    return cudaSuccess;
}

}  // namespace qsa
