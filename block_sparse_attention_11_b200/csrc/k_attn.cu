// k_attn.cu -- sparse attention over the selected original K/V.
//
// Page "Qwen3.8-Flash-Next: Day-0 Support in SGLang", section "Qwen Sparse
// Attention: Retrieve Coarsely, Attend Precisely": the selected blocks expand
// to 2048 positions, the 0-3 tokens of the query's own incomplete block are
// appended (at most 2051 positions), and softmax and value aggregation use the
// original uncompressed K/V.  One selection per query serves every head.
//
// bf16 kernel.  Each query gathers its own ~2 MB of K/V, so the stage is bound
// by gather bandwidth (about 8 flop per byte), not by the tensor cores.  The
// design keeps the gather engine busy and the math off the critical path:
//   * a producer warp walks the selection and issues one bulk TMA copy per
//     selected block and tensor (a block of all kv heads is one contiguous
//     4 x Hkv x 256-byte span), 8 blocks per stage, 4 stages in flight;
//   * each block lands in its own shared-memory slot, slots padded by 16 bytes
//     so that token j of 8 different blocks fall in 8 different bank groups:
//     every 8x8 ldmatrix tile reads 8 blocks' token j conflict-free;
//   * consumers use swap-AB warp MMAs (m16n8k16): S^T = K Q^T with 16 keys as
//     M and the 8 q heads of one kv head as N (no padding waste for GQA 8),
//     an fp32 online softmax per head column, P^T re-laid out in registers
//     with movmatrix, and O^T += V^T P;
//   * four warps per kv head share the stages: two take alternate stages,
//     and each of those pairs splits a stage's two 16-key tiles, so every
//     warp runs its own short softmax chain per stage; the four softmax
//     states are merged at the end of an item (with 4 kv heads, two warps per
//     head take both tiles of alternate stages);
//   * the producer stages each item's block ids in shared memory once, so
//     no global read sits on the per-stage issue path.
// A persistent grid walks the work items; the pipeline runs across item
// boundaries.  Decode splits each sequence's key list over several items
// (split-KV) and a small kernel combines the partial results.
//
// fp32 kernel.  A plain SIMT warp per (query, head): used for the fp32 mode.
#include <algorithm>

#include "internal.h"

namespace qsa {

namespace {

constexpr int AT_BPS = 8;               // blocks per stage
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescale = 8.f;         // lazy-rescale threshold (log2 units)
constexpr uint32_t kFullStage = 0x924924u;   // 8 slots x 3 bits, each holding 4 tokens

// Tuning knobs (compile time).  Defaults measured best on B200 for the
// 32K-token prefill: 2 resident CTAs per SM, 2 stages in flight per CTA,
// 4 producer warps per CTA.
#ifndef QSA_ATTN_CTAS
#define QSA_ATTN_CTAS 2           // resident CTAs per SM
#endif
#ifndef QSA_ATTN_PW
#define QSA_ATTN_PW 4             // producer warps per CTA (each owns every PW-th slot of a stage)
#endif
#ifndef QSA_ATTN_NS
#define QSA_ATTN_NS 2             // stages in flight per CTA
#endif

#ifndef QSA_ATTN_TILES
#define QSA_ATTN_TILES 2          // 16-key tiles of a stage per consumer warp (1 or 2); 2 with 4 kv heads
#endif

// KV8: K/V caches of FP8 E4M3 values (times per-tensor scales), 1 byte per element.
// D: head dim (128 or 256).  G: q heads per kv head (8, or 12 for the released
// 24q/2kv shape: two 8-head MMA column tiles, the second one half padding).
template <int HKV, bool KV8 = false, int D = 128, int G = 8> struct AttnCfg {
    static constexpr int kD = D;
    static constexpr int kNT = (G + 7) / 8;        // 8-head column tiles per kv head
    static constexpr int kMT = D / 16;             // 16-dim MMA k-steps (QK) and m-tiles (PV)
    // Consumer warp (grp, sub): group grp = kv head g, column tile nt; sub = u * 2
    // + hf takes the stages whose global index is = hf (mod 2), and tiles
    // [u * kTiles, (u + 1) * kTiles) of each.
    static constexpr int kTiles = (HKV == 4 || D > 128) ? 2 : QSA_ATTN_TILES;
    static constexpr int kU = 2 / kTiles;          // warps sharing one stage of one group
    static constexpr int kWph = 2 * kU;            // consumer warps per group
    static constexpr int kGroups = HKV * kNT;
    static constexpr int kConsumers = kWph * kGroups;
    static constexpr int kMinCtas = (HKV == 4 || D > 128) ? 1 : QSA_ATTN_CTAS;   // launch-bounds residency target
    static constexpr int kPw = QSA_ATTN_PW;
    static constexpr int kThreads = (kConsumers + kPw) * 32;
    static constexpr int kEl = KV8 ? 1 : 2;                    // bytes per K/V element
    static constexpr int kTokBytes = HKV * D * kEl;            // one token, all kv heads
    static constexpr int kSpan = kBlock * kTokBytes;           // bytes of one block, all kv heads
    static constexpr int kSlot = kSpan + 16;                   // padded slot
    static constexpr int kStage = 2 * AT_BPS * kSlot;          // K slots then V slots
    static constexpr int kHq = G * HKV;
    static constexpr int kQBytes = kHq * D * 2;
    static constexpr int kNS = QSA_ATTN_NS;
    // Consumer warp hf takes the stages whose global index is = hf (mod 2); with
    // an even number of slots it always uses the same slots, in order, so no
    // mbarrier is ever waited on more than one phase ahead (try_wait.parity
    // only tells the current phase from the previous one).
    static_assert(kNS >= 2 && kNS % 2 == 0, "stages in flight must be even");
    static_assert(AT_BPS % QSA_ATTN_PW == 0, "producer warps must divide the blocks per stage");
    static_assert(kTiles == 1 || kTiles == 2, "a stage holds two 16-key tiles");
};

struct AttnParams {
    const __nv_bfloat16 *q, *k, *v;
    const int32_t *sel, *nsel, *seq_len;
    int B;
    int64_t n_q, q0, kv_stride;
    int top_k;
    float scale_log2;
    int decode;
    int splits;            // decode: items per sequence
    int split_blocks;      // decode: list entries per split (multiple of AT_BPS)
    int64_t items;
    int sel_cap, nst_cap;  // shared-memory block-id list and per-stage table sizes (from top_k)
    __nv_bfloat16 *out;
    float *lse;
    float *part_o;         // decode: [B][splits][Hq][D]
    float *part_lse;       // decode: [B][splits][Hq] (log2 domain)
    const int32_t *cap_len;  // decode, IndexShare: [B] capture rows + 1 (null: plain decode)
    int max_draft;           // IndexShare: largest seq_len - cap_len
    int dense;               // decode: every visible block in order (dense causal attention, no selection)
    unsigned *status;
    float k_scale, v_scale;  // KV8: K = k_scale * stored E4M3 value, V = v_scale * stored value
    Paging pg;               // pg.table: K/V are paged caches [slots][Hkv][D] (kv_stride = table capacity)
    int no_tail;             // prefill: no tail entries (the listed blocks only)
};

// The key list of one work item: positions lbeg..lend of
// [sel[0..nsel), tail blocks].  The tail is positions 4*nb .. t: the query's
// own incomplete block (0-3 tokens), or, for an IndexShare draft step, the
// capture row's incomplete block and every position drafted since (nb is then
// the capture row's visible block count), as ceil(tail / 4) blocks.
struct Item {
    int seq;
    int64_t row;       // prefill: query row; decode: split index
    int64_t t;         // query position
    const int32_t *sel;
    int nsel;
    int64_t nb;
    int tail;
    int lbeg, lend;
    const __nv_bfloat16 *qrow;
};

template <class Cfg>
__device__ __forceinline__ Item get_item(const AttnParams &p, int64_t i) {
    Item it;
    if (!p.decode) {
        it.seq = (int)(i % p.B);
        it.row = p.n_q - 1 - i / p.B;                       // longest rows first
        it.t = p.q0 + it.row;
        const int64_t qi = (int64_t)it.seq * p.n_q + it.row;
        it.sel = p.sel + qi * p.top_k;
        it.nsel = p.nsel[qi];
        it.qrow = p.q + qi * (int64_t)Cfg::kHq * Cfg::kD;
    } else {
        it.seq = (int)(i / p.splits);
        it.row = i % p.splits;
        it.t = (int64_t)p.seq_len[it.seq] - 1;
        it.sel = p.dense ? nullptr : p.sel + (int64_t)it.seq * p.top_k;
        it.nsel = p.dense ? 0 : p.nsel[it.seq];
        it.qrow = p.q + (int64_t)it.seq * Cfg::kHq * Cfg::kD;
    }
    if (it.t < 0 || it.t >= p.kv_stride) {
        if (it.t >= p.kv_stride) flag(p.status, QSA_DEV_BAD_LENGTH);
        it.t = -1;   // nothing visible: the item attends to no position
    }
    int64_t t_sel = it.t;   // the row whose selection the item reads
    if (p.decode && p.cap_len && it.t >= 0) {
        t_sel = (int64_t)p.cap_len[it.seq] - 1;
        if (t_sel < 0 || t_sel > it.t || it.t - t_sel > p.max_draft) {
            flag(p.status, QSA_DEV_BAD_LENGTH);
            t_sel = it.t;   // read as a plain decode step
        }
    }
    it.nb = (t_sel + 1) / kBlock;
    it.tail = p.no_tail ? 0 : (int)(it.t + 1 - kBlock * it.nb);
    it.nsel = p.dense ? (int)it.nb : max(0, min(it.nsel, p.top_k));
    const int len = it.nsel + (it.tail + kBlock - 1) / kBlock;
    if (!p.decode) {
        it.lbeg = 0;
        it.lend = len;
    } else {
        it.lbeg = min(len, (int)it.row * p.split_blocks);
        it.lend = min(len, it.lbeg + p.split_blocks);
    }
    return it;
}

template <class Cfg>
struct __align__(128) AttnSmem {
    uint8_t stage[Cfg::kNS][Cfg::kStage];
    alignas(16) uint8_t qbuf[2][Cfg::kQBytes];
    float xbuf[Cfg::kGroups][Cfg::kWph - 1][32][4 + 4 * Cfg::kMT];
    alignas(16) __nv_bfloat16 obuf[Cfg::kGroups][8][Cfg::kD];
    alignas(16) uint32_t info[Cfg::kNS][Cfg::kPw];
    uint64_t full[Cfg::kNS], empty[Cfg::kNS], qfull[2], qempty[2];
    uint64_t xready[Cfg::kGroups], xdone[Cfg::kGroups];   // merge handshake per group
    // followed in dynamic shared memory by
    //   int32_t  sel_s[sel_cap]             the current item's block ids (each producer fills its own slots)
    //   uint32_t st_info[kPw][nst_cap]      per stage of the item: token counts of the producer's slots
    //   uint32_t st_bytes[kPw][nst_cap]     per stage of the item: bytes the producer copies per tensor
};

template <class Cfg>
size_t attn_smem_bytes(int sel_cap, int nst_cap) {
    return sizeof(AttnSmem<Cfg>) + (size_t)sel_cap * 4 + 2 * (size_t)Cfg::kPw * nst_cap * 4 + 128;
}

// PAGED: K/V are paged caches addressed through p.pg (a separate instantiation,
// so the contiguous kernels carry none of the page-table code).
template <int HKV, int D, int G, bool PAGED, bool KV8>
__global__ void __launch_bounds__(AttnCfg<HKV, KV8, D, G>::kThreads, AttnCfg<HKV, KV8, D, G>::kMinCtas)
    attn_bf16_kernel(AttnParams p) {
    using Cfg = AttnCfg<HKV, KV8, D, G>;
    extern __shared__ uint8_t asm_raw[];
    AttnSmem<Cfg> &sm =
        *reinterpret_cast<AttnSmem<Cfg> *>((reinterpret_cast<uintptr_t>(asm_raw) + 127) & ~uintptr_t(127));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // zero the slots once: masked keys must read finite values (0 * NaN = NaN)
    for (int i = threadIdx.x; i < (int)(sizeof(sm.stage) / 16); i += blockDim.x)
        reinterpret_cast<uint4 *>(&sm.stage[0][0])[i] = make_uint4(0, 0, 0, 0);
    if (threadIdx.x == 0) {
        for (int s = 0; s < Cfg::kNS; ++s) {
            mbar_init(&sm.full[s], Cfg::kPw);
            mbar_init(&sm.empty[s], Cfg::kGroups * Cfg::kU);
        }
        for (int s = 0; s < 2; ++s) { mbar_init(&sm.qfull[s], 1); mbar_init(&sm.qempty[s], Cfg::kConsumers); }
        for (int s = 0; s < Cfg::kGroups; ++s) { mbar_init(&sm.xready[s], Cfg::kWph - 1); mbar_init(&sm.xdone[s], 1); }
        fence_mbar_init();
    }
    fence_proxy_async_smem();
    __syncthreads();
    pdl_wait();      // the selection comes from the previous kernel
    pdl_trigger();

    if (warp >= Cfg::kConsumers) {
        // ------------------------------------------------------------ producers
        // Producer pw owns slots j = pw, pw + PW, ... of every stage.  Per item it
        // copies the block ids to shared memory and precomputes, per stage, the
        // token counts and byte totals of its slots, so the per-stage issue path
        // is: wait for the slot, one expect_tx, one bulk copy per block and tensor.
        constexpr int kSlotsPerPw = AT_BPS / Cfg::kPw;
        const int pw = warp - Cfg::kConsumers;
        int32_t *ids = reinterpret_cast<int32_t *>(&sm + 1);
        uint32_t *st_info = reinterpret_cast<uint32_t *>(ids + p.sel_cap) + pw * p.nst_cap;
        uint32_t *st_bytes = reinterpret_cast<uint32_t *>(ids + p.sel_cap) + (Cfg::kPw + pw) * p.nst_cap;
        int64_t it_count = 0;   // stage counter across items
        int64_t ic = 0;         // item counter
        bool ok = true;
        for (int64_t i = blockIdx.x; i < p.items && ok; i += gridDim.x, ++ic) {
            const Item it = get_item<Cfg>(p, i);
            const int id_end = min(it.lend, it.nsel);
            // list entries of this producer's slots: e - lbeg = 8 * st + PW * jj + pw
            // (dense: the ids are the entries themselves, nothing to stage)
            for (int r = lane; !p.dense && r * Cfg::kPw < id_end - it.lbeg; r += 32) {
                const int rel = (r / kSlotsPerPw) * AT_BPS + (r % kSlotsPerPw) * Cfg::kPw + pw;
                if (rel < id_end - it.lbeg) ids[rel] = it.sel[it.lbeg + rel];
            }
            __syncwarp();
            const int nst = (it.lend - it.lbeg + AT_BPS - 1) / AT_BPS;
            for (int st = lane; !p.dense && st < nst; st += 32) {
                uint32_t info = 0, bytes = 0;
#pragma unroll
                for (int jj = 0; jj < kSlotsPerPw; ++jj) {
                    const int j = Cfg::kPw * jj + pw;
                    const int e = it.lbeg + AT_BPS * st + j;
                    int tokens = 0;
                    if (e < it.lend) {
                        int64_t blk = it.nb + (e - it.nsel);
                        if (e < it.nsel) {
                            const int b = ids[e - it.lbeg];
                            blk = b;
                            if (b >= 0 && b < it.nb) tokens = kBlock;
                            else flag(p.status, QSA_DEV_BAD_INDEX);
                        } else {
                            tokens = min(kBlock, it.tail - kBlock * (e - it.nsel));
                        }
                        if (PAGED && tokens > 0 && paged_slot(p.pg, it.seq, blk * kBlock) < 0) {
                            tokens = 0;   // a page outside the cache: skipped, flagged
                            flag(p.status, QSA_DEV_BAD_INDEX);
                        }
                    }
                    info |= (uint32_t)tokens << (3 * j);
                    bytes += (uint32_t)tokens * Cfg::kTokBytes;
                }
                st_info[st] = info;
                st_bytes[st] = bytes;
            }
            const int qs = (int)(ic & 1);
            if (pw == 0 && ic >= 2) ok = mbar_wait(&sm.qempty[qs], (int)(((ic >> 1) + 1) & 1), p.status);
            __syncwarp();
            if (!ok) break;
            if (pw == 0 && lane == 0) {
                mbar_arrive_expect_tx(&sm.qfull[qs], Cfg::kQBytes);
                bulk_g2s(sm.qbuf[qs], it.qrow, Cfg::kQBytes, &sm.qfull[qs]);
            }
            const int64_t kv0 = (int64_t)it.seq * p.kv_stride;
            for (int st = 0; st < nst && ok; ++st, ++it_count) {
                const int s = (int)(it_count % Cfg::kNS);
                uint32_t sinfo, sbytes;
                if (!p.dense) {
                    sinfo = st_info[st];
                    sbytes = st_bytes[st];
                } else {   // every visible block, then the tail: counts straight from the entry index
                    sinfo = 0;
                    sbytes = 0;
#pragma unroll
                    for (int jj = 0; jj < kSlotsPerPw; ++jj) {
                        const int j = Cfg::kPw * jj + pw;
                        const int e = it.lbeg + AT_BPS * st + j;
                        int tokens = e >= it.lend ? 0
                                     : (e < it.nsel ? kBlock : min(kBlock, it.tail - kBlock * (e - it.nsel)));
                        if (PAGED && tokens > 0 && paged_slot(p.pg, it.seq, (int64_t)e * kBlock) < 0) {
                            tokens = 0;   // a page outside the cache: skipped, flagged
                            flag(p.status, QSA_DEV_BAD_INDEX);
                        }
                        sinfo |= (uint32_t)tokens << (3 * j);
                        sbytes += (uint32_t)tokens * Cfg::kTokBytes;
                    }
                }
                if (it_count >= Cfg::kNS) ok = mbar_wait(&sm.empty[s], (int)(((it_count / Cfg::kNS) + 1) & 1), p.status);
                if (!ok) break;
                if (lane == 0) {
                    sm.info[s][pw] = sinfo;
                    mbar_arrive_expect_tx(&sm.full[s], 2 * sbytes);
                }
                __syncwarp();
                if (lane < kSlotsPerPw) {
                    const int j = Cfg::kPw * lane + pw;
                    const int e = it.lbeg + AT_BPS * st + j;
                    const int tokens = (int)((sinfo >> (3 * j)) & 7u);
                    if (tokens > 0) {
                        const int64_t blk = (e < it.nsel) ? (p.dense ? (int64_t)e : (int64_t)ids[e - it.lbeg])
                                                          : it.nb + (e - it.nsel);
                        const int64_t tok = PAGED ? paged_slot(p.pg, it.seq, blk * kBlock) : kv0 + blk * kBlock;
                        const int64_t off = tok * Cfg::kTokBytes;   // bytes
                        const uint32_t nbytes = (uint32_t)tokens * Cfg::kTokBytes;
                        bulk_g2s(sm.stage[s] + j * Cfg::kSlot, reinterpret_cast<const uint8_t *>(p.k) + off, nbytes,
                                 &sm.full[s]);
                        bulk_g2s(sm.stage[s] + (AT_BPS + j) * Cfg::kSlot, reinterpret_cast<const uint8_t *>(p.v) + off,
                                 nbytes, &sm.full[s]);
                    }
                }
            }
        }
        // drain: wait until the copies of the last stages have landed
        if (lane == 0) {
            for (int64_t c = (it_count > Cfg::kNS ? it_count - Cfg::kNS : 0); c < it_count; ++c)
                mbar_wait(&sm.full[c % Cfg::kNS], (int)((c / Cfg::kNS) & 1), p.status);
            if (pw == 0)
                for (int64_t c = (ic > 2 ? ic - 2 : 0); c < ic; ++c)
                    mbar_wait(&sm.qfull[c & 1], (int)((c >> 1) & 1), p.status);
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    // warp (g, sub), sub = u * 2 + hf: kv head g; takes the stages whose global
    // index is = hf (mod 2) and the 16-key tiles [u * kTiles, (u + 1) * kTiles)
    // of each (tile t = tokens {2t, 2t+1} of the stage's 8 blocks).  Each warp
    // keeps its own online-softmax state; the states of a kv head's warps are
    // merged at the end of an item.
    constexpr int kT = Cfg::kTiles, kMT = Cfg::kMT;
    const int grp = warp / Cfg::kWph;              // group: kv head g, 8-head column tile nt
    const int g = grp / Cfg::kNT, nt = grp % Cfg::kNT;
    const int sub = warp % Cfg::kWph;
    const int hf = sub & 1;
    const int t0 = (sub >> 1) * kT;
    const int gr = lane >> 2, tq = lane & 3;
    const uint32_t stage0 = smem_u32(&sm.stage[0][0]);
    const int mi = lane >> 3, rr = lane & 7;
    // ldmatrix lane addresses: matrix mi = lane / 8 reads row rr (= block) of
    // the stage's 8 slots.  K: token + (mi & 1), 16 bytes + (mi >> 1).  V (bf16,
    // transposed): token + (mi >> 1), 16 bytes + (mi & 1); V (FP8): token +
    // (mi & 1), 16 bytes + (mi >> 1), so registers 0/1 hold the two tokens of
    // one 16-byte column and 2/3 of the next.
    constexpr int kHead = D * Cfg::kEl;              // bytes of one kv head of one token
    const uint32_t k_lane_off =
        (uint32_t)(rr * Cfg::kSlot + (mi & 1) * Cfg::kTokBytes + g * kHead + (mi >> 1) * 16);
    const uint32_t v_lane_off =
        KV8 ? (uint32_t)(AT_BPS * Cfg::kSlot + rr * Cfg::kSlot + (mi & 1) * Cfg::kTokBytes + g * kHead +
                         (mi >> 1) * 16)
            : (uint32_t)(AT_BPS * Cfg::kSlot + rr * Cfg::kSlot + (mi >> 1) * Cfg::kTokBytes + g * kHead +
                         (mi & 1) * 16);
    constexpr uint32_t kTileOff = 2 * Cfg::kTokBytes;   // tokens {2,3} vs {0,1}
    int64_t it_count = 0, ic = 0;
    bool ok = true;
    for (int64_t i = blockIdx.x; i < p.items && ok; i += gridDim.x, ++ic) {
        const Item it = get_item<Cfg>(p, i);
        const int qs = (int)(ic & 1);
        ok = mbar_wait(&sm.qfull[qs], (int)((ic >> 1) & 1), p.status);
        if (!ok) break;
        // this lane's q head (the B column gr of the tile); padding columns of the
        // last tile (G not a multiple of 8) read zeros and are never written out
        const int hloc = 8 * nt + gr;
        const bool hvalid = hloc < G;
        uint32_t qf[kMT][2];
        float sl2 = p.scale_log2;   // logit scale in log2 units
        if constexpr (!KV8) {
            const uint32_t *qw = reinterpret_cast<const uint32_t *>(sm.qbuf[qs]);
            const int head = G * g + hloc;
#pragma unroll
            for (int kk = 0; kk < kMT; ++kk) {
                qf[kk][0] = hvalid ? qw[(head * D + 16 * kk + 2 * tq) >> 1] : 0u;
                qf[kk][1] = hvalid ? qw[(head * D + 16 * kk + 8 + 2 * tq) >> 1] : 0u;
            }
        } else {
            // FP8 keys are scored as FP16 (E4M3 is a subset of FP16); the query
            // goes to FP16 times 2^e (e puts the kv head's largest |q| in
            // [2^14, 2^15)), in the k order of the widened key fragments:
            // k-step 2j takes dims 32j + 4tq + {0..3}, k-step 2j + 1 dims
            // 32j + 16 + 4tq + {0..3}.
            const __nv_bfloat16 *qh = reinterpret_cast<const __nv_bfloat16 *>(sm.qbuf[qs]) + (G * g + hloc) * D;
            float qv[kMT][4];
            float mx = 0.f;
#pragma unroll
            for (int kk = 0; kk < kMT; ++kk)
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    qv[kk][c] = hvalid ? __bfloat162float(qh[32 * (kk >> 1) + 16 * (kk & 1) + 4 * tq + c]) : 0.f;
                    mx = fmaxf(mx, fabsf(qv[kk][c]));
                }
#pragma unroll
            for (int o2 = 16; o2 > 0; o2 >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o2));
            int qexp = 0;
            if (mx > 0.f && mx <= 3.0e38f) {
                int ex;
                frexpf(mx, &ex);
                qexp = min(max(15 - ex, -100), 100);
            }
            const float sc2 = ldexpf(1.0f, qexp);
#pragma unroll
            for (int kk = 0; kk < kMT; ++kk) {
                qf[kk][0] = pack_f16(__fmul_rn(qv[kk][0], sc2), __fmul_rn(qv[kk][1], sc2));
                qf[kk][1] = pack_f16(__fmul_rn(qv[kk][2], sc2), __fmul_rn(qv[kk][3], sc2));
            }
            sl2 = p.scale_log2 * p.k_scale * ldexpf(1.0f, -qexp);
        }
        // The query buffer is refilled by a bulk copy (async proxy) once every
        // consumer has released it.  Its fragments must have arrived in
        // registers first: plain shared loads may still be in flight at the
        // release, and nothing reads them until the first key stage.  Reading
        // every fragment here waits for the loads; the proxy fence orders these
        // reads before the copy's writes.
        {
            uint32_t all = 0;
#pragma unroll
            for (int kk = 0; kk < kMT; ++kk) all ^= qf[kk][0] ^ qf[kk][1];
            asm volatile("" ::"r"(all));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.qempty[qs]);
        float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
        float o[kMT][4];
#pragma unroll
        for (int a = 0; a < kMT; ++a) o[a][0] = o[a][1] = o[a][2] = o[a][3] = 0.f;

        for (int pos = it.lbeg; pos < it.lend; pos += AT_BPS, ++it_count) {
            if ((int)(it_count & 1) != hf) continue;
            const int s = (int)(it_count % Cfg::kNS);
            ok = mbar_wait(&sm.full[s], (int)((it_count / Cfg::kNS) & 1), p.status);
            if (!ok) break;
            uint32_t info = 0;
            if constexpr (Cfg::kPw == 4) {
                const uint4 w4 = *reinterpret_cast<const uint4 *>(&sm.info[s][0]);
                info = (w4.x | w4.y) | (w4.z | w4.w);
            } else {
#pragma unroll
                for (int q2 = 0; q2 < Cfg::kPw; ++q2) info |= sm.info[s][q2];
            }
            const uint32_t sbase = stage0 + (uint32_t)s * Cfg::kStage;
            // S^T for this warp's tiles (16 keys x 8 heads each), unscaled
            float sc[kT][4];
#pragma unroll
            for (int t = 0; t < kT; ++t)
#pragma unroll
                for (int c = 0; c < 4; ++c) sc[t][c] = 0.f;
            if constexpr (!KV8) {
#pragma unroll
                for (int kk = 0; kk < kMT; ++kk) {
#pragma unroll
                    for (int t = 0; t < kT; ++t) {
                        uint32_t a0, a1, a2, a3;
                        ldsm_x4(sbase + k_lane_off + (uint32_t)(t0 + t) * kTileOff + kk * 32, a0, a1, a2, a3);
                        mma16816(sc[t], a0, a1, a2, a3, qf[kk][0], qf[kk][1]);
                    }
                }
            } else {
                // register r: 4 E4M3 keys' dims; r0/r1 tokens 2t/2t+1 at dims
                // 32j + 4tq.., r2/r3 the same at 32j + 16 + 4tq..
#pragma unroll
                for (int j = 0; j < kMT / 2; ++j) {
#pragma unroll
                    for (int t = 0; t < kT; ++t) {
                        uint32_t r[4], lo[4], hi[4];
                        ldsm_x4(sbase + k_lane_off + (uint32_t)(t0 + t) * kTileOff + j * 32, r[0], r[1], r[2], r[3]);
#pragma unroll
                        for (int i = 0; i < 4; ++i) e4m3x4_to_f16x4(r[i], lo[i], hi[i]);
                        mma16816_f16(sc[t], lo[0], lo[1], hi[0], hi[1], qf[2 * j][0], qf[2 * j][1]);
                        mma16816_f16(sc[t], lo[2], lo[3], hi[2], hi[3], qf[2 * j + 1][0], qf[2 * j + 1][1]);
                    }
                }
            }
            // (slot gr, token 2t): heads 2tq, 2tq+1 in sc[t][0..1]; token 2t+1 in sc[t][2..3]
            if (info != kFullStage) {           // a short or missing block: mask its absent tokens
                const int ntok = (int)((info >> (3 * gr)) & 7u);
#pragma unroll
                for (int t = 0; t < kT; ++t) {
                    if (ntok <= 2 * (t0 + t)) sc[t][0] = sc[t][1] = -INFINITY;
                    if (ntok <= 2 * (t0 + t) + 1) sc[t][2] = sc[t][3] = -INFINITY;
                }
            }
            float lm0 = fmaxf(sc[0][0], sc[0][2]), lm1 = fmaxf(sc[0][1], sc[0][3]);
#pragma unroll
            for (int t = 1; t < kT; ++t) {
                lm0 = fmaxf(lm0, fmaxf(sc[t][0], sc[t][2]));
                lm1 = fmaxf(lm1, fmaxf(sc[t][1], sc[t][3]));
            }
            lm0 *= sl2;
            lm1 *= sl2;
            // Lazy rescaling: the reference max of a head column moves only when a
            // score exceeds it by more than kRescale (log2 units), so unscaled
            // probabilities stay below 2^kRescale; otherwise no max reduction and
            // no rescale of the accumulators.
            if (__any_sync(0xffffffffu, lm0 > mrow[0] + kRescale || lm1 > mrow[1] + kRescale)) {
#pragma unroll
                for (int o2 = 4; o2 < 32; o2 <<= 1) {
                    lm0 = fmaxf(lm0, __shfl_xor_sync(0xffffffffu, lm0, o2));
                    lm1 = fmaxf(lm1, __shfl_xor_sync(0xffffffffu, lm1, o2));
                }
                const float mn0 = fmaxf(mrow[0], lm0), mn1 = fmaxf(mrow[1], lm1);
                const float al0 = exp2f(mrow[0] - ((mn0 == -INFINITY) ? 0.f : mn0));
                const float al1 = exp2f(mrow[1] - ((mn1 == -INFINITY) ? 0.f : mn1));
                mrow[0] = mn0;
                mrow[1] = mn1;
                lrow[0] *= al0;
                lrow[1] *= al1;
#pragma unroll
                for (int mt = 0; mt < kMT; ++mt) {
                    o[mt][0] *= al0;
                    o[mt][1] *= al1;
                    o[mt][2] *= al0;
                    o[mt][3] *= al1;
                }
            }
            const float nmu0 = (mrow[0] == -INFINITY) ? 0.f : -mrow[0];
            const float nmu1 = (mrow[1] == -INFINITY) ? 0.f : -mrow[1];
            uint32_t pb[kT][2];
#pragma unroll
            for (int t = 0; t < kT; ++t) {
                const float p0 = exp2f(fmaf(sc[t][0], sl2, nmu0));
                const float p1 = exp2f(fmaf(sc[t][1], sl2, nmu1));
                const float p2 = exp2f(fmaf(sc[t][2], sl2, nmu0));
                const float p3 = exp2f(fmaf(sc[t][3], sl2, nmu1));
                lrow[0] += p0 + p2;
                lrow[1] += p1 + p3;
                pb[t][0] = movm_t(KV8 ? pack_f16(p0, p1) : pack_bf16(p0, p1));
                pb[t][1] = movm_t(KV8 ? pack_f16(p2, p3) : pack_bf16(p2, p3));
            }
            if constexpr (KV8) {
                // transposed E4M3 V: register r holds (block 2tq, dims d, d + 1)
                // and (block 2tq + 1, dims d, d + 1), d = 2gr of its 16-byte
                // column; pairing bytes (0, 2) and (1, 3) gives the A rows of
                // dims d and d + 1 (output rows gr <-> dim 16 mt + 2gr,
                // gr + 8 <-> 16 mt + 2gr + 1)
#pragma unroll
                for (int c2 = 0; c2 < kMT / 2; ++c2) {
#pragma unroll
                    for (int t = 0; t < kT; ++t) {
                        uint32_t r[4], a[8];
                        ldsm_x4_t(sbase + v_lane_off + (uint32_t)(t0 + t) * kTileOff + c2 * 32, r[0], r[1], r[2],
                                  r[3]);
#pragma unroll
                        for (int i = 0; i < 4; ++i) e4m3x4_to_f16x4(__byte_perm(r[i], 0u, 0x3120), a[2 * i], a[2 * i + 1]);
                        mma16816_f16(o[2 * c2], a[0], a[1], a[2], a[3], pb[t][0], pb[t][1]);
                        mma16816_f16(o[2 * c2 + 1], a[4], a[5], a[6], a[7], pb[t][0], pb[t][1]);
                    }
                }
            } else {
#pragma unroll
                for (int mt = 0; mt < kMT; ++mt) {
#pragma unroll
                    for (int t = 0; t < kT; ++t) {
                        uint32_t a0, a1, a2, a3;
                        ldsm_x4_t(sbase + v_lane_off + (uint32_t)(t0 + t) * kTileOff + mt * 32, a0, a1, a2, a3);
                        mma16816(o[mt], a0, a1, a2, a3, pb[t][0], pb[t][1]);
                    }
                }
            }
            fence_proxy_async_smem();   // this stage's shared reads before the next bulk copies into it
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.empty[s]);
        }
        if (!ok) break;
        // row sums across the 8 lane groups
#pragma unroll
        for (int o2 = 4; o2 < 32; o2 <<= 1) {
            lrow[0] += __shfl_xor_sync(0xffffffffu, lrow[0], o2);
            lrow[1] += __shfl_xor_sync(0xffffffffu, lrow[1], o2);
        }
        // merge the warps of this kv head: warps sub >= 1 publish, warp 0 folds
        if (sub != 0) {
            if (ic > 0) ok = mbar_wait(&sm.xdone[grp], (int)((ic - 1) & 1), p.status);
            if (!ok) break;
            float *xb = sm.xbuf[grp][sub - 1][lane];
            xb[0] = mrow[0]; xb[1] = mrow[1]; xb[2] = lrow[0]; xb[3] = lrow[1];
#pragma unroll
            for (int mt = 0; mt < kMT; ++mt)
#pragma unroll
                for (int c = 0; c < 4; ++c) xb[4 + 4 * mt + c] = o[mt][c];
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.xready[grp]);
        } else {
            ok = mbar_wait(&sm.xready[grp], (int)(ic & 1), p.status);
            if (!ok) break;
            // Every fold is symmetric in its two operands (explicitly rounded, no
            // contraction), so the result does not depend on which warp of a
            // tile group took the even or the odd stages:
            //   A = fold(own, sub 1)               tiles of group 0
            //   B = fold(sub 2, sub 3)             tiles of group 1 (two groups only)
            //   result = fold(A, B)
            {
                const float *xb = sm.xbuf[grp][0][lane];
                float f0[2], f1[2];
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const float mo = xb[c], lo = xb[2 + c];
                    const float mn = fmaxf(mrow[c], mo);
                    const float mu = (mn == -INFINITY) ? 0.f : mn;
                    f0[c] = exp2f(mrow[c] - mu);
                    f1[c] = exp2f(mo - mu);
                    lrow[c] = __fadd_rn(__fmul_rn(lrow[c], f0[c]), __fmul_rn(lo, f1[c]));
                    mrow[c] = mn;
                }
#pragma unroll
                for (int mt = 0; mt < kMT; ++mt)
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        o[mt][c] = __fadd_rn(__fmul_rn(o[mt][c], f0[c & 1]), __fmul_rn(xb[4 + 4 * mt + c], f1[c & 1]));
            }
            if constexpr (Cfg::kU == 2) {
                const float *x2 = sm.xbuf[grp][1][lane], *x3 = sm.xbuf[grp][2][lane];
                float f2[2], f3[2], fa[2], fb[2];
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const float mbv = fmaxf(x2[c], x3[c]);
                    const float mub = (mbv == -INFINITY) ? 0.f : mbv;
                    f2[c] = exp2f(x2[c] - mub);
                    f3[c] = exp2f(x3[c] - mub);
                    const float lb = __fadd_rn(__fmul_rn(x2[2 + c], f2[c]), __fmul_rn(x3[2 + c], f3[c]));
                    const float mn = fmaxf(mrow[c], mbv);
                    const float mu = (mn == -INFINITY) ? 0.f : mn;
                    fa[c] = exp2f(mrow[c] - mu);
                    fb[c] = exp2f(mbv - mu);
                    lrow[c] = __fadd_rn(__fmul_rn(lrow[c], fa[c]), __fmul_rn(lb, fb[c]));
                    mrow[c] = mn;
                }
#pragma unroll
                for (int mt = 0; mt < kMT; ++mt)
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const float ob = __fadd_rn(__fmul_rn(x2[4 + 4 * mt + c], f2[c & 1]),
                                                   __fmul_rn(x3[4 + 4 * mt + c], f3[c & 1]));
                        o[mt][c] = __fadd_rn(__fmul_rn(o[mt][c], fa[c & 1]), __fmul_rn(ob, fb[c & 1]));
                    }
            }
            const float l[2] = {lrow[0], lrow[1]}, m[2] = {mrow[0], mrow[1]};
            const float vsc = KV8 ? p.v_scale : 1.f;
            const float inv0 = l[0] > 0.f ? vsc / l[0] : 0.f, inv1 = l[1] > 0.f ? vsc / l[1] : 0.f;
            // output rows gr / gr + 8 of m-tile mt are dims 16 mt + gr / + 8 (FP8 V: 16 mt + 2gr / + 1)
            const int dr0 = KV8 ? 2 * gr : gr, dr1 = KV8 ? 2 * gr + 1 : gr + 8;
            // the tile's heads: columns 2tq, 2tq + 1 are heads h0 + 2tq (+1), valid below G
            const int h0 = G * g + 8 * nt;
            const int nv = min(8, G - 8 * nt);
            const bool cv0 = 2 * tq < nv, cv1 = 2 * tq + 1 < nv;
            if (!p.decode) {
#pragma unroll
                for (int mt = 0; mt < kMT; ++mt) {
                    const float r0 = o[mt][0] * inv0, r1 = o[mt][1] * inv1;
                    const float r2 = o[mt][2] * inv0, r3 = o[mt][3] * inv1;
                    sm.obuf[grp][2 * tq][16 * mt + dr0] = __float2bfloat16_rn(r0);
                    sm.obuf[grp][2 * tq + 1][16 * mt + dr0] = __float2bfloat16_rn(r1);
                    sm.obuf[grp][2 * tq][16 * mt + dr1] = __float2bfloat16_rn(r2);
                    sm.obuf[grp][2 * tq + 1][16 * mt + dr1] = __float2bfloat16_rn(r3);
                }
                __syncwarp();
                const int64_t qi = (int64_t)it.seq * p.n_q + it.row;
                uint4 *dst = reinterpret_cast<uint4 *>(p.out + (qi * Cfg::kHq + h0) * D);
                const uint4 *src = reinterpret_cast<const uint4 *>(&sm.obuf[grp][0][0]);
                for (int c = lane; c < nv * D / 8; c += 32) dst[c] = src[c];
                if (p.lse && gr == 0) {
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        const float v = (l[c] > 0.f) ? (m[c] + log2f(l[c])) / kLog2e : -INFINITY;
                        if (2 * tq + c < nv) p.lse[qi * Cfg::kHq + h0 + 2 * tq + c] = v;
                    }
                }
                __syncwarp();
            } else {
                const int64_t pi = (int64_t)it.seq * p.splits + it.row;
                float *po = p.part_o + (pi * Cfg::kHq + h0) * D;
#pragma unroll
                for (int mt = 0; mt < kMT; ++mt) {
                    if (cv0) po[(2 * tq) * D + 16 * mt + dr0] = o[mt][0] * inv0;
                    if (cv1) po[(2 * tq + 1) * D + 16 * mt + dr0] = o[mt][1] * inv1;
                    if (cv0) po[(2 * tq) * D + 16 * mt + dr1] = o[mt][2] * inv0;
                    if (cv1) po[(2 * tq + 1) * D + 16 * mt + dr1] = o[mt][3] * inv1;
                }
                if (gr == 0) {
#pragma unroll
                    for (int c = 0; c < 2; ++c)
                        if (2 * tq + c < nv)
                            p.part_lse[pi * Cfg::kHq + h0 + 2 * tq + c] = (l[c] > 0.f) ? m[c] + log2f(l[c]) : -INFINITY;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.xdone[grp]);
        }
    }
}

// Decode combine: one CTA of 128 threads per (sequence, q head): out =
// sum_s w_s o_s / sum_s w_s with w_s = 2^(lse_s - max lse).  Warp j sums the
// splits s = j mod 4 (lane l: dims 4l + 128c .. +3), so four independent
// chains of loads are in flight; warps 1-3 hand their sums to warp 0.
template <int D>
__global__ void __launch_bounds__(128) attn_combine_kernel(const float *__restrict__ part_o,
                                                           const float *__restrict__ part_lse, int splits, int Hq,
                                                           __nv_bfloat16 *__restrict__ out, float *__restrict__ lse) {
    constexpr int NC = D / 128;
    __shared__ float4 red_o[3][NC][32];
    __shared__ float red_m[4], red_d[4];
    pdl_wait();
    const int seq = blockIdx.x / Hq, h = blockIdx.x % Hq, tid = threadIdx.x, lane = tid & 31, sg = tid >> 5;
    const float *pl = part_lse + (int64_t)seq * splits * Hq + h;   // split s at pl[s * Hq]
    float mx = -INFINITY;
    for (int s = tid; s < splits; s += 128) mx = fmaxf(mx, pl[(int64_t)s * Hq]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) red_m[sg] = mx;
    __syncthreads();
    mx = fmaxf(fmaxf(red_m[0], red_m[1]), fmaxf(red_m[2], red_m[3]));
    const float *po = part_o + ((int64_t)seq * splits * Hq + h) * D + 4 * lane;
    float den = 0.f;
    float4 acc[NC];
#pragma unroll
    for (int c = 0; c < NC; ++c) acc[c] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int s = sg; s < splits; s += 4) {
        const float v = pl[(int64_t)s * Hq];
        float4 x[NC];
#pragma unroll
        for (int c = 0; c < NC; ++c) x[c] = *reinterpret_cast<const float4 *>(po + (int64_t)s * Hq * D + 128 * c);
        const float w = (mx == -INFINITY || v == -INFINITY) ? 0.f : exp2f(v - mx);
        den += w;
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            acc[c].x += w * x[c].x;
            acc[c].y += w * x[c].y;
            acc[c].z += w * x[c].z;
            acc[c].w += w * x[c].w;
        }
    }
    if (sg > 0) {
#pragma unroll
        for (int c = 0; c < NC; ++c) red_o[sg - 1][c][lane] = acc[c];
        if (lane == 0) red_d[sg] = den;
    }
    __syncthreads();
    if (sg != 0) return;
#pragma unroll
    for (int j = 0; j < 3; ++j) {
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            const float4 o = red_o[j][c][lane];
            acc[c].x += o.x;
            acc[c].y += o.y;
            acc[c].z += o.z;
            acc[c].w += o.w;
        }
        den += red_d[j + 1];
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
#pragma unroll
    for (int c = 0; c < NC; ++c) {
        uint2 v;
        v.x = pack_bf16(acc[c].x * inv, acc[c].y * inv);
        v.y = pack_bf16(acc[c].z * inv, acc[c].w * inv);
        *reinterpret_cast<uint2 *>(out + ((int64_t)seq * Hq + h) * D + 128 * c + 4 * lane) = v;
    }
    if (lse && lane == 0) lse[(int64_t)seq * Hq + h] = den > 0.f ? (mx + log2f(den)) / kLog2e : -INFINITY;
}

// fp32 SIMT attention: one warp per (item, q head); lane owns 4 dims.
__global__ void __launch_bounds__(256) attn_f32_kernel(const float *__restrict__ q, const float *__restrict__ k,
                                                        const float *__restrict__ v, const int32_t *__restrict__ sel,
                                                        const int32_t *__restrict__ nsel_p,
                                                        const int32_t *__restrict__ seq_len, int B, int64_t n_q,
                                                        int64_t q0, int64_t kv_stride, int Hq, int Hkv, int top_k,
                                                        float scale, float *__restrict__ out, float *__restrict__ lse,
                                                        int decode, const int32_t *__restrict__ cap_len, int max_draft,
                                                        int dense, unsigned *status) {
    const int64_t wid = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    const int64_t items = decode ? (int64_t)B : (int64_t)B * n_q;
    if (wid >= items * Hq) return;
    const int h = (int)(wid % Hq);
    const int64_t item = wid / Hq;
    int seq;
    int64_t t, qi;
    if (decode) { seq = (int)item; t = (int64_t)seq_len[seq] - 1; qi = seq; }
    else { seq = (int)(item / n_q); t = q0 + item % n_q; qi = item; }
    const int g = (int)(((int64_t)h * Hkv) / Hq);
    if (t >= kv_stride) {
        if (lane == 0) flag(status, QSA_DEV_BAD_LENGTH);
        t = -1;   // nothing visible
    }
    int64_t t_sel = t;   // the row whose selection is read (IndexShare: the capture row)
    if (decode && cap_len && t >= 0) {
        t_sel = (int64_t)cap_len[seq] - 1;
        if (t_sel < 0 || t_sel > t || t - t_sel > max_draft) {
            if (lane == 0) flag(status, QSA_DEV_BAD_LENGTH);
            t_sel = t;
        }
    }
    const int64_t nb = (t_sel + 1) / kBlock;
    const int tail = (int)(t + 1 - kBlock * nb);     // positions 4*nb .. t
    const int32_t *sl = dense ? nullptr : sel + qi * top_k;
    const int nsel = dense ? (int)nb : max(0, min(nsel_p[qi], top_k));
    const float4 qv = reinterpret_cast<const float4 *>(q + (qi * Hq + h) * 128)[lane];
    float m = -INFINITY, l = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    const int len = nsel + (tail + kBlock - 1) / kBlock;
    for (int e = 0; e < len; ++e) {
        int64_t b;
        int ntok;
        if (e < nsel) {
            b = dense ? e : sl[e];
            ntok = kBlock;
            if (b < 0 || b >= nb) {
                if (lane == 0) flag(status, QSA_DEV_BAD_INDEX);
                continue;
            }
        } else {
            b = nb + (e - nsel);
            ntok = min(kBlock, tail - kBlock * (e - nsel));
        }
        for (int j = 0; j < ntok; ++j) {
            const int64_t row = ((int64_t)seq * kv_stride + b * kBlock + j) * Hkv + g;
            const float4 kv = reinterpret_cast<const float4 *>(k + row * 128)[lane];
            float d = qv.x * kv.x + qv.y * kv.y + qv.z * kv.z + qv.w * kv.w;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
            const float x = d * scale;
            const float mn = fmaxf(m, x);
            const float al = expf(m - mn);
            const float pw = expf(x - mn);
            m = mn;
            l = l * al + pw;
            const float4 vv = reinterpret_cast<const float4 *>(v + row * 128)[lane];
            acc.x = acc.x * al + pw * vv.x;
            acc.y = acc.y * al + pw * vv.y;
            acc.z = acc.z * al + pw * vv.z;
            acc.w = acc.w * al + pw * vv.w;
        }
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
    reinterpret_cast<float4 *>(out + (qi * Hq + h) * 128)[lane] =
        make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    if (lse && lane == 0) lse[qi * Hq + h] = l > 0.f ? m + logf(l) : -INFINITY;
}

// Decode split-KV plan: each sequence's list of at most list_max entries (top_k
// blocks + tail blocks; ceil(list_max/8) stages) is cut into `splits` items of S stages; the persistent grid of `cap`
// CTAs takes ceil(items / cap) rounds.  S minimises rounds x (S + 1) (one stage
// of start-up per item), ties going to fewer splits.
struct SplitPlan {
    int splits, split_blocks;
};

SplitPlan decode_split_plan(int B, int list_max, int64_t cap) {
    const int nst = (list_max + AT_BPS - 1) / AT_BPS;
    SplitPlan best{1, nst * AT_BPS};
    int64_t best_cost = -1;
    for (int S = nst; S >= 1; --S) {
        const int splits = (nst + S - 1) / S;
        if (S > 1 && (nst + S - 2) / (S - 1) == splits) continue;   // same splits with a smaller S
        const int64_t rounds = ((int64_t)B * splits + cap - 1) / cap;
        const int64_t cost = rounds * (S + 1);
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best = SplitPlan{splits, S * AT_BPS};
        }
    }
    return best;
}

}  // namespace

// Tail blocks of one item's list: the query's own incomplete block, or for an
// IndexShare draft step the capture row's (0-3 tokens) plus max_draft positions.
int attn_tail_blocks(bool indexshare, int max_draft) {
    return indexshare ? (3 + max_draft + kBlock - 1) / kBlock : 1;
}

namespace {

template <int HKV, bool KV8, int D, int G>
cudaError_t run_bf16(const AttnArgs &a, void *ws, unsigned *status, cudaStream_t s) {
    using Cfg = AttnCfg<HKV, KV8, D, G>;
    const DeviceInfo *di = device_info();
    const int sms = di ? di->sm_count : 148;
    AttnParams p{};
    p.q = (const __nv_bfloat16 *)a.q;
    p.k = (const __nv_bfloat16 *)a.k;
    p.v = (const __nv_bfloat16 *)a.v;
    p.sel = a.sel;
    p.nsel = a.nsel;
    p.seq_len = a.seq_len;
    p.B = a.B;
    p.n_q = a.n_q;
    p.q0 = a.q0;
    p.kv_stride = a.kv_stride;
    p.top_k = a.top_k;
    p.scale_log2 = a.scale * kLog2e;
    p.decode = a.decode ? 1 : 0;
    p.out = (__nv_bfloat16 *)a.out;
    p.lse = a.lse;
    p.status = status;
    p.cap_len = a.decode ? a.cap_len : nullptr;
    p.max_draft = a.max_draft;
    p.dense = a.decode && a.dense ? 1 : 0;
    p.pg = a.pg;
    p.k_scale = a.k_scale;
    p.v_scale = a.v_scale;
    p.no_tail = (!a.decode && a.no_tail) ? 1 : 0;
    // entries of one item's list: top_k blocks + the tail blocks (dense: every block of the cache)
    const int list_max = p.dense ? (int)(a.kv_stride / kBlock + 1)
                                 : a.top_k + attn_tail_blocks(a.decode && a.cap_len, a.max_draft);
    if (a.decode) {
        const SplitPlan sp = decode_split_plan(a.B, list_max, (int64_t)sms * Cfg::kMinCtas);
        const int splits = sp.splits;
        p.splits = splits;
        p.split_blocks = sp.split_blocks;
        p.items = (int64_t)a.B * splits;
        float *w = static_cast<float *>(ws);
        p.part_o = w;
        p.part_lse = w + (size_t)a.B * splits * Cfg::kHq * D;
    } else {
        p.splits = 1;
        p.split_blocks = 0;
        p.items = (int64_t)a.B * a.n_q;
    }
    if (p.items <= 0) return cudaSuccess;
    // an item's list holds at most top_k ids plus the tail block
    p.sel_cap = p.dense ? 4 : (a.top_k + 3) & ~3;                  // dense: no id list, no stage tables
    p.nst_cap = p.dense ? 1 : (list_max + AT_BPS - 1) / AT_BPS;
    const size_t smem = attn_smem_bytes<Cfg>(p.sel_cap, p.nst_cap);
    if (di && smem > di->smem_optin) return cudaErrorInvalidValue;
    auto kern = p.pg.table ? attn_bf16_kernel<HKV, D, G, true, KV8> : attn_bf16_kernel<HKV, D, G, false, KV8>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, Cfg::kThreads, smem);
    if (e != cudaSuccess) return e;
    const int64_t grid = std::min<int64_t>(p.items, (int64_t)sms * std::max(1, per_sm));
    e = launch_pdl(kern, dim3((unsigned)grid), dim3(Cfg::kThreads), smem, s, p);
    if (e != cudaSuccess || !a.decode) return e;
    return launch_pdl(attn_combine_kernel<D>, dim3((unsigned)(a.B * Cfg::kHq)), dim3(128), 0, s,
                      (const float *)p.part_o, (const float *)p.part_lse, p.splits, (int)Cfg::kHq,
                      (__nv_bfloat16 *)a.out, a.lse);
}

}  // namespace

size_t attn_decode_ws_bytes(int B, int Hq, int d, int top_k, int tail_blocks) {
    // the larger of the split plans run_bf16 can pick (1 or 2 resident CTAs per SM)
    const DeviceInfo *di = device_info();
    const int sms = di ? di->sm_count : 148;
    const int list_max = top_k + tail_blocks;
    const int splits =
        std::max(decode_split_plan(B, list_max, sms).splits, decode_split_plan(B, list_max, 2 * sms).splits);
    size_t n = (size_t)B * splits * Hq;
    return (n * d * sizeof(float) + n * sizeof(float) + 255) / 256 * 256;
}

size_t attn_dense_decode_ws_bytes(int B, int Hq, int d, int64_t kv_stride) {
    const DeviceInfo *di = device_info();
    const int sms = di ? di->sm_count : 148;
    const int list_max = (int)(kv_stride / kBlock + 1);
    const int splits =
        std::max(decode_split_plan(B, list_max, sms).splits, decode_split_plan(B, list_max, 2 * sms).splits);
    size_t n = (size_t)B * splits * Hq;
    return (n * d * sizeof(float) + n * sizeof(float) + 255) / 256 * 256;
}

cudaError_t launch_attn_bf16(const AttnArgs &a, void *ws, unsigned *status, cudaStream_t s) {
    switch (a.Hkv) {
    case 1: return a.kv8 ? run_bf16<1, true, 128, 8>(a, ws, status, s) : run_bf16<1, false, 128, 8>(a, ws, status, s);
    case 2:
        if (a.d == 256)   // the released 24q/2kv, d = 256 shape
            return a.kv8 ? run_bf16<2, true, 256, 12>(a, ws, status, s) : run_bf16<2, false, 256, 12>(a, ws, status, s);
        return a.kv8 ? run_bf16<2, true, 128, 8>(a, ws, status, s) : run_bf16<2, false, 128, 8>(a, ws, status, s);
    case 4: return a.kv8 ? run_bf16<4, true, 128, 8>(a, ws, status, s) : run_bf16<4, false, 128, 8>(a, ws, status, s);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_attn_f32(const AttnArgs &a, unsigned *status, cudaStream_t s) {
    const int64_t items = a.decode ? (int64_t)a.B : (int64_t)a.B * a.n_q;
    const int64_t warps = items * a.Hq;
    if (warps <= 0) return cudaSuccess;
    attn_f32_kernel<<<(unsigned)((warps + 7) / 8), 256, 0, s>>>(
        (const float *)a.q, (const float *)a.k, (const float *)a.v, a.sel, a.nsel, a.seq_len, a.B, a.n_q, a.q0,
        a.kv_stride, a.Hq, a.Hkv, a.top_k, a.scale, (float *)a.out, a.lse, a.decode ? 1 : 0,
        a.decode ? a.cap_len : nullptr, a.max_draft, a.decode && a.dense ? 1 : 0, status);
    return cudaGetLastError();
}

}  // namespace qsa
