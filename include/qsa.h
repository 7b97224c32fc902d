/*
 * qsa.h -- C ABI of libqsa: Qwen Sparse Attention (QSA) on NVIDIA B200 (sm_100a).
 *
 * QSA (page "Qwen3.8-Flash-Next: Day-0 Support in SGLang", section "Qwen Sparse
 * Attention: Retrieve Coarsely, Attend Precisely"; page "Qwen3.8-Flash-Next,
 * Layer by Layer", section "Token mixing") runs in two stages per attention
 * layer:
 *   1. an indexer mean-pools every 4 consecutive raw indexer keys (in FP32),
 *      rotates the mean with the first token's RoPE position, stores it as one
 *      BF16 compressed key, scores every complete visible block for each query
 *      with 4 indexer query heads against the one shared 128-dim key head, and
 *      keeps the best 512 blocks;
 *   2. softmax attention over the original (uncompressed) K/V at exactly the
 *      selected blocks' 4*512 = 2048 positions plus the query's own 0-3 tail
 *      tokens (at most 2051 positions).
 *
 * Conventions shared by every entry point
 *   - Pointers named as device pointers are device memory owned by the
 *     caller; host pointers are named so.  The library allocates nothing and
 *     never synchronises the stream (qsa_check_status excepted).
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL = the legacy default stream).
 *   - All tensors are dense, row-major, with the layouts stated per call.
 *     Element type: `dtype` = QSA_BF16 (bfloat16) or QSA_FP32 (float) for
 *     every floating-point tensor of the call, except head weights (always
 *     float) and the fp32 scratch.
 *   - Indexer geometry is fixed by the pages: 4 query heads, 1 key head,
 *     128 dims, blocks of 4 tokens.  Attention head dim d = 128, or 256 for
 *     the released 24q / 2kv shape.
 *   - Positions: token i of a sequence has RoPE position i.  Block b holds
 *     positions 4b..4b+3 and is visible to the query at position t iff
 *     4b + 3 <= t, so nb(t) = floor((t + 1) / 4) blocks are visible and the
 *     tail is positions 4*nb(t)..t.  A query selects min(top_k, nb(t)) blocks.
 *   - Selections are written as block ids sorted ascending, padded with -1
 *     up to top_k, plus a count.  Ranking: higher score first, equal scores
 *     go to the lower block id.
 *   - Return value: QSA_OK or an error code.  Invalid arguments are rejected
 *     before anything is launched and leave no state behind.  Kernels that
 *     find an out-of-range index or run out of a bounded wait set the
 *     library's device status word instead of trapping; qsa_check_status
 *     reads it.
 */
#ifndef QSA_H
#define QSA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QSA_API __attribute__((visibility("default")))
#else
#define QSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ---- */
#define QSA_OK 0
#define QSA_ERR_INVALID_ARG 1   /* null pointer, bad size, bad stride, bad flag */
#define QSA_ERR_UNSUPPORTED 2   /* shape/dtype/option the library does not implement, or not an sm_100 device */
#define QSA_ERR_CUDA 3          /* a CUDA launch or runtime call failed */
#define QSA_ERR_DEVICE 4        /* a kernel reported a bounds violation or a wait timeout */
#define QSA_ERR_WORKSPACE 5     /* workspace pointer null or smaller than the size query returned */

/* ---- element types ---- */
#define QSA_BF16 0
#define QSA_FP32 1

/* ---- option flags ---- */
/* Score with ReLU of each head's dot product, as in the score equation of
 * "Qwen Sparse Attention: Retrieve Coarsely, Attend Precisely".  Off by
 * default: the default score is the plain sum over heads. */
#define QSA_SCORE_RELU 1u
/* Normalise the FP32 block mean before rotation (unit-weight RMS norm,
 * eps 1e-6); the same section calls the mean normalised without naming
 * the norm.  Off by default. */
#define QSA_POOL_RMSNORM 2u
/* Compressed keys stored as FP8 E4M3 (1 byte per value, round to nearest
 * even from the exact rotated value, saturating at +-448): the FP8
 * indexer-key cache of the page "Qwen3.8-Flash-Next, Layer by Layer"
 * (section "Serving it", the recipe's indexer_kv_dtype fp8).  Accepted by
 * qsa_pool_keys_prefill / qsa_pool_keys_decode (they write FP8 compressed
 * keys) and qsa_index_topk_decode (it reads them); dtype must be QSA_BF16
 * (raw keys, ring and indexer queries stay BF16).  qsa_index_topk_prefill
 * returns QSA_ERR_UNSUPPORTED with it. */
#define QSA_KEYS_FP8 4u

/* RoPE parameters.  Rotate-half convention (style 0): for i < rotary_dim/2
 * the pair (x_i, x_{i + rotary_dim/2}) turns by the angle
 * (pos / pos_scale) * base^(-2i / rotary_dim); dims >= rotary_dim are left
 * alone.  rotary_dim: even, multiple of 16, 16..128.  pos_scale > 0 is a
 * linear position scale (4 stands in for the 1M-token context extension). */
typedef struct {
    double base;
    double pos_scale;
    int32_t rotary_dim;
    int32_t style;      /* 0 = rotate-half; other values -> QSA_ERR_UNSUPPORTED */
} qsa_rope_t;

/* Human-readable text of a status code (static storage). */
QSA_API const char *qsa_strerror(int status);

/* Library version, major*10000 + minor*100 + patch. */
QSA_API int qsa_version(void);

/* Reads and clears the device status word of the current device after
 * synchronising `stream`.  Returns QSA_OK, or QSA_ERR_DEVICE when a kernel
 * flagged an error since the last call.  If detail != NULL it receives the
 * raw status bits (host pointer): 1 a selected block id out of range, 2 a
 * sequence length beyond the caller's capacity, 4 a bounded wait that ran
 * out, 8 an internal inconsistency of a top-k select, 16 a decode-indexer
 * workspace that was not zero-filled before its first use. */
QSA_API int qsa_check_status(void *stream, uint32_t *detail);

/*
 * Self-test of the bounded waits (not a step of the method; the pages have no
 * counterpart).  Every pipeline of the library waits on mbarriers through one
 * bounded wait that gives up after 2 s, records QSA_DEV_TIMEOUT (status bit 4)
 * and lets the kernel release its tensor memory and return, so a broken
 * pipeline ends its kernel instead of hanging the GPU.  This call runs that
 * wait on purpose: one CTA takes TMEM columns, waits on an mbarrier that
 * nothing arrives on with a limit of limit_ns (1 .. 2e9 ns), gives up, frees
 * the TMEM and returns.  It writes 0 to *result (device, 4-byte aligned) when
 * the wait gave up (1 would mean it completed), and qsa_check_status then
 * reports QSA_ERR_DEVICE with detail bit 4.  No fault, no hang.
 */
QSA_API int qsa_selftest_wait_timeout(uint64_t limit_ns, uint32_t *result, void *stream);

/* ========================================================================= */
/* a1. Compressed-key pooling, prefill                                        */
/* ========================================================================= */
/*
 * For each sequence i < B and each complete block j < floor(n_tok / 4) of the
 * raw keys k_raw[i][0..n_tok):
 *     m   = (((k0 + k1) + k2) + k3) * 0.25            (FP32, the pages' "averaged in FP32")
 *     m   = m / sqrt(mean(m^2) + 1e-6)                 (only with QSA_POOL_RMSNORM)
 *     out = RoPE(m, position pos0 + 4j)                (the first token's position)
 *     k_pool[i][pos0/4 + j] = round_to_dtype(out)      (BF16: round to nearest even)
 * Source: "Qwen Sparse Attention: Retrieve Coarsely, Attend Precisely" (four raw
 * index keys averaged in FP32, rotated with the first token's position, one
 * BF16 compressed key per four tokens); flozi.net guide, "How a token moves
 * through the model", item 2 (RoPE after pooling).
 *
 * k_raw   device, [B][raw_stride][128] dtype; tokens pos0 .. pos0+n_tok-1 of
 *         each sequence sit at rows 0 .. n_tok-1.
 * k_pool  device, [B][pool_stride][128] dtype; rows pos0/4 .. pos0/4 +
 *         floor(n_tok/4) - 1 are written, nothing else.
 * pos0    multiple of 4, >= 0.  Trailing n_tok mod 4 tokens are not pooled
 *         (they belong in the decode ring); n_tok < 4 is a no-op (pointers
 *         may then be NULL).
 * Errors: QSA_ERR_INVALID_ARG for null pointers, B < 1, n_tok < 0,
 *         raw_stride < n_tok, pos0 mod 4 != 0, pool_stride < pos0/4 +
 *         floor(n_tok/4), bad flags or rope; QSA_ERR_UNSUPPORTED for a style
 *         other than 0.
 */
QSA_API int qsa_pool_keys_prefill(const void *k_raw, void *k_pool, int32_t B, int64_t n_tok, int64_t pos0,
                          int64_t raw_stride, int64_t pool_stride, qsa_rope_t rope, uint32_t flags,
                          int32_t dtype, void *stream);

/* ========================================================================= */
/* a1d. Compressed-key pooling, decode (four-slot ring)                       */
/* ========================================================================= */
/*
 * One new token per sequence.  seq_len[i] = s counts the tokens including the
 * new one, whose position is p = s - 1.  The new raw key goes to ring slot
 * p mod 4.  When s mod 4 == 0 the block is complete: ring slots 0..3 are
 * pooled exactly as in qsa_pool_keys_prefill (position s - 4) into
 * k_pool[i][s/4 - 1].
 * Source: "Qwen Sparse Attention: Retrieve Coarsely, Attend Precisely" (the raw
 * keys of the unfinished block live in a four-slot per-request ring).
 *
 * k_new    device, [B][128] dtype, raw indexer key of the new token.
 * ring     device, [B][4][128] dtype, updated in place.
 * k_pool   device, [B][pool_stride][128] dtype.
 * seq_len  device, [B] int32, each >= 1.  A sequence whose s/4 > pool_stride
 *          is skipped and flagged in the device status word.
 */
QSA_API int qsa_pool_keys_decode(const void *k_new, void *ring, void *k_pool, const int32_t *seq_len,
                         int32_t B, int64_t pool_stride, qsa_rope_t rope, uint32_t flags,
                         int32_t dtype, void *stream);

/* ========================================================================= */
/* a2-a4. Indexer scores and top-k, prefill                                    */
/* ========================================================================= */
/*
 * For each sequence i and query row r < n_q (position t = q0 + r):
 *     qhat_h = round_to_dtype(RoPE(q_idx[i][r][h], t))           h = 0..3
 *     s_b    = (1/sqrt(128)) * sum_h w_h * phi(<qhat_h, k_pool[i][b]>),  b < nb(t)
 * with phi = ReLU under QSA_SCORE_RELU and the identity otherwise, w_h =
 * head_w[i][r][h] or 1 when head_w is NULL; then the min(top_k, nb(t)) best
 * blocks are written to sel[i][r][0..top_k) ascending (padded with -1) and
 * their count to nsel[i][r].
 * Source: "Qwen Sparse Attention: Retrieve Coarsely, Attend Precisely" (score
 * equation s_{t,b}; keeps the best 512 blocks); "Token mixing" (4 query
 * heads, 1 key head, 128 dims).
 *
 * q_idx    device, [B][n_q][4][128] dtype, RAW (unrotated) indexer queries.
 * k_pool   device, [B][pool_stride][128] dtype, compressed keys of positions
 *          0 .. q0+n_q-1 (rows 0 .. nb(q0+n_q-1)-1 must be valid).
 * head_w   device, [B][n_q][4] float, or NULL.
 * sel      device, [B][n_q][top_k] int32.   nsel  device, [B][n_q] int32.
 * workspace device scratch of at least qsa_index_topk_prefill_workspace()
 *          bytes, 256-byte aligned; contents on entry are ignored.  The
 *          scores of a group of rows are materialised there (groups of at
 *          most 2 GiB), so the size grows with q0 + n_q up to that cap.
 *          QSA_BF16 with rows of at most 32768 blocks ((q0 + n_q) / 4 <=
 *          32768) stores each score as the top 16 bits of its
 *          order-preserving key; the select ranks by them and re-scores in
 *          fp32 the blocks whose 16-bit key equals the k-th largest one, so
 *          the ranking is that of the fp32 scores up to their rounding.
 *          Longer rows (2048 rows a group at a 1M-token context) and
 *          QSA_FP32 store fp32 scores.
 * top_k    1..2048.
 * Chunked prefill: one call per chunk of rows with q0 = the chunk's first
 * position, after that chunk's keys were pooled into k_pool; the selections
 * equal those of one call over all rows (tested to 1,048,576 positions).
 */
/* Kernels one qsa_index_topk_prefill call with these sizes launches: the
 * query rotation, then a score kernel and a row select per group of query rows
 * (groups keep the score block under 2 GiB); 0 for invalid arguments. */
QSA_API int qsa_index_topk_prefill_kernels(int32_t B, int64_t n_q, int64_t q0, uint32_t flags, int32_t dtype);
QSA_API size_t qsa_index_topk_prefill_workspace(int32_t B, int64_t n_q, int64_t q0, int32_t top_k,
                                        uint32_t flags, int32_t dtype);
QSA_API int qsa_index_topk_prefill(const void *q_idx, const void *k_pool, const float *head_w, int32_t B,
                           int64_t n_q, int64_t q0, int64_t pool_stride, int32_t top_k, int32_t *sel,
                           int32_t *nsel, void *workspace, size_t ws_bytes, qsa_rope_t rope,
                           uint32_t flags, int32_t dtype, void *stream);

/* ========================================================================= */
/* a2-a4 (decode). Indexer scores and top-k for one new token per sequence     */
/* ========================================================================= */
/*
 * As qsa_index_topk_prefill for the single query at position t = seq_len[i]-1
 * of each sequence, scanning all nb(t) = floor(seq_len[i]/4) compressed keys
 * (run qsa_pool_keys_decode first so a block completed by the new token is
 * visible).  Source: as above, and "IndexShare MTP" (the decode scorer scans
 * all ceil(L/4) compressed blocks and dominates the layer's cost at long
 * context).
 *
 * q_idx     device, [B][4][128] dtype, RAW indexer query of the new token.
 * k_pool    device, [B][pool_stride][128] dtype.
 * head_w    device, [B][4] float, or NULL.
 * seq_len   device, [B] int32.
 * max_blocks host bound on floor(seq_len[i]/4) for every i (sizes the grid;
 *           a sequence beyond it or beyond pool_stride is flagged and gets
 *           nsel = 0).
 * sel       device, [B][top_k] int32;  nsel device, [B] int32.
 * workspace at least qsa_index_topk_decode_workspace() bytes, zero-filled
 *           once after it is allocated (cudaMemset): it holds per-sequence
 *           score histograms that a call accumulates and clears again, so a
 *           workspace stays zero between calls and serves any number of them
 *           in stream order.  A call that finds a histogram not zero at its
 *           start flags status bit 16 (its selection is then unreliable).
 */
/* Kernels a qsa_index_topk_decode call with these sizes launches on the
 * current device: 1 (scorer and select fused, one thread-block cluster per
 * sequence, when the clusters fit the GPU at once) or 2 (scorer, then
 * select); 0 for invalid arguments or an unsupported device. */
QSA_API int qsa_index_topk_decode_kernels(int32_t B, int64_t max_blocks, uint32_t flags, int32_t dtype);
QSA_API size_t qsa_index_topk_decode_workspace(int32_t B, int64_t max_blocks, int32_t top_k, uint32_t flags,
                                       int32_t dtype);
QSA_API int qsa_index_topk_decode(const void *q_idx, const void *k_pool, const float *head_w,
                          const int32_t *seq_len, int32_t B, int64_t pool_stride, int64_t max_blocks,
                          int32_t top_k, int32_t *sel, int32_t *nsel, void *workspace, size_t ws_bytes,
                          qsa_rope_t rope, uint32_t flags, int32_t dtype, void *stream);

/* ========================================================================= */
/* a5-a6. Sparse attention, prefill                                           */
/* ========================================================================= */
/*
 * For each sequence i, query row r (position t = q0 + r) and q head h
 * (kv head g = floor(h * Hkv / Hq)):
 *     P(t) = {4b .. 4b+3 : b in sel[i][r][0..nsel)}  U  {4*nb(t) .. t}
 *     out[i][r][h] = sum_{j in P(t)} softmax_j(scale * <q[i][r][h], k[i][j][g]>) v[i][j][g]
 *     lse[i][r][h] = log(sum_{j in P(t)} exp(scale * <q, k_j>))     (natural log)
 * Softmax and accumulation in fp32; out rounded to dtype.
 * Source: "Qwen Sparse Attention: Retrieve Coarsely, Attend Precisely" (expand
 * the 512 blocks to 2048 positions, append the 0-3 tail tokens, softmax and
 * value aggregation over the original uncompressed K/V; one selection per
 * query shared by all heads).
 *
 * q        device, [B][n_q][Hq][d] dtype, already rotated (the attention
 *          layer's RoPE is applied by the caller, see qsa_rope_apply).
 * k, v     device, [B][kv_stride][Hkv][d] dtype, rows by position; k rotated.
 * sel/nsel device, as written by qsa_index_topk_prefill.  Ids must satisfy
 *          0 <= b < nb(t); out-of-range ids are skipped and flagged.
 * out      device, [B][n_q][Hq][d] dtype.   lse device, [B][n_q][Hq] float or NULL.
 * Shapes: d == 128 with Hq % Hkv == 0 and, for QSA_BF16, Hq / Hkv == 8 and
 *         Hkv in {1, 2, 4} (any ratio for QSA_FP32); or, QSA_BF16 only, the
 *         released model's shape Hq = 24, Hkv = 2, d = 256 (the architecture
 *         guide page, section "How a token moves through the model", item 2:
 *         24 query heads, two KV heads of dimension 256); kv_stride >= q0 + n_q;
 *         B * n_q and kv_stride below 2^31.
 * workspace: device, 256-byte aligned, at least qsa_sparse_attn_prefill_workspace()
 *          bytes, caller-owned and needing no initialisation; 0 bytes (pass
 *          NULL) for the shapes that run without one.  QSA_BF16 with d = 128,
 *          Hq = 8 Hkv, Hkv = 2 or 4 and contexts of at most 32768 blocks
 *          ((q0 + n_q) / 4 <= 32768) splits the work by sharing over tiles
 *          of 8 consecutive query rows: a pre-pass lists, per tile, the
 *          blocks that 2 or more of its queries select and the tail blocks
 *          (with a mask of the queries attending to each), and per query the
 *          blocks only it selects; the tile's listed blocks run on the tensor
 *          cores, their K/V (a pair of kv heads) gathered once per tile
 *          (masked keys contribute exactly zero), the own blocks in the
 *          per-query gather kernel, and the two partial softmaxes are merged
 *          by their log-sum-exp.  The workspace holds both lists and the
 *          gather part's lse; it is capped near 1 GiB per sequence: longer
 *          prompts run as several chunks of whole query tiles.  Results of a
 *          chunk starting at a row that is a multiple of 8 equal those of the
 *          same rows in one call bit for bit when both calls split (the gather
 *          kernel alone is chunk-independent too).  Too small:
 *          QSA_ERR_WORKSPACE.
 */
/* Kernels one qsa_sparse_attn_prefill call with these sizes launches: 1 (the
 * gather kernels: fp32, d = 256, other GQA ratios) or 3 per sequence and
 * chunk of query tiles (lists, gather kernel, tiles); 0 for invalid
 * arguments. */
QSA_API int qsa_sparse_attn_prefill_kernels(int32_t B, int64_t n_q, int64_t q0, int32_t top_k, int32_t Hq,
                                            int32_t Hkv, int32_t d, int32_t dtype);
QSA_API size_t qsa_sparse_attn_prefill_workspace(int32_t B, int64_t n_q, int64_t q0, int32_t top_k, int32_t Hq, int32_t Hkv,
                                                 int32_t d, int32_t dtype);
QSA_API int qsa_sparse_attn_prefill(const void *q, const void *k, const void *v, const int32_t *sel,
                            const int32_t *nsel, int32_t B, int64_t n_q, int64_t q0, int64_t kv_stride,
                            int32_t Hq, int32_t Hkv, int32_t d, int32_t top_k, float scale, void *out,
                            float *lse, void *workspace, size_t ws_bytes, int32_t dtype, void *stream);

/* ========================================================================= */
/* a5-a6 (decode). Sparse attention for one new token per sequence            */
/* ========================================================================= */
/*
 * As qsa_sparse_attn_prefill for the query at position t = seq_len[i] - 1.
 * The caller has written the new token's rotated k and its v at row t of
 * the caches.  The work of each sequence is split across CTAs and combined
 * (split-KV); the partial results live in the workspace.
 *
 * q        device, [B][Hq][d] dtype (rotated).
 * k, v     device, [B][kv_stride][Hkv][d] dtype.
 * sel/nsel device, [B][top_k] / [B] from qsa_index_topk_decode.
 * out      device, [B][Hq][d] dtype.   lse device, [B][Hq] float or NULL.
 * workspace at least qsa_sparse_attn_decode_workspace() bytes.
 */
QSA_API size_t qsa_sparse_attn_decode_workspace(int32_t B, int32_t Hq, int32_t d, int32_t top_k, int32_t dtype);
QSA_API int qsa_sparse_attn_decode(const void *q, const void *k, const void *v, const int32_t *seq_len,
                           const int32_t *sel, const int32_t *nsel, int32_t B, int64_t kv_stride,
                           int32_t Hq, int32_t Hkv, int32_t d, int32_t top_k, float scale, void *out,
                           float *lse, void *workspace, size_t ws_bytes, int32_t dtype, void *stream);

/* ========================================================================= */
/* IndexShare draft step: decode attention over a frozen selection            */
/* ========================================================================= */
/*
 * Page "Qwen3.8-Flash-Next: Day-0 Support in SGLang", section "IndexShare MTP:
 * Reusing the QSA Selection Across Draft Steps": the selection computed for
 * the last accepted row is held for the whole draft loop; each draft decode
 * step skips the indexer and reads that selection plus the positions drafted
 * since.  The query of sequence i is at t = seq_len[i] - 1; the capture row is
 * t_c = cap_len[i] - 1 (0 <= t_c <= t <= t_c + max_draft).  It attends over
 *   the blocks in sel/nsel (written by qsa_index_topk_decode for the capture
 *   row, i.e. with seq_len = cap_len; ids b < floor(cap_len / 4)), and
 *   every position from 4 * floor(cap_len / 4) through t (the capture row's
 *   incomplete block and the drafted positions, the new token included).
 * Other arguments as qsa_sparse_attn_decode.  A sequence outside the stated
 * range of cap_len is read as a plain decode step and flagged in the status
 * word (QSA_DEV_BAD_LENGTH).  max_draft in [0, 64].
 * workspace at least qsa_sparse_attn_decode_shared_workspace() bytes.
 */
QSA_API size_t qsa_sparse_attn_decode_shared_workspace(int32_t B, int32_t Hq, int32_t d, int32_t top_k,
                                                       int32_t max_draft, int32_t dtype);
QSA_API int qsa_sparse_attn_decode_shared(const void *q, const void *k, const void *v, const int32_t *seq_len,
                                          const int32_t *cap_len, const int32_t *sel, const int32_t *nsel,
                                          int32_t B, int64_t kv_stride, int32_t Hq, int32_t Hkv, int32_t d,
                                          int32_t top_k, int32_t max_draft, float scale, void *out, float *lse,
                                          void *workspace, size_t ws_bytes, int32_t dtype, void *stream);

/* ========================================================================= */
/* Dense causal decode attention (the full-attention baseline)                */
/* ========================================================================= */
/*
 * Not a step of QSA: the full attention QSA replaces.  Pages "Qwen3.8-Flash-
 * Next, Layer by Layer" (section "Token mixing") and the aicontrolled journal
 * (section "Where the measurement ends") compare the QSA attention module with
 * full attention at 1M tokens; this is the full attention, on the same
 * kernels, so that ratio can be measured on one GPU.  The query of sequence i
 * at t = seq_len[i] - 1 attends over every position 0..t.  Arguments as
 * qsa_sparse_attn_decode without a selection; 1 <= seq_len[i] <= kv_stride.
 * workspace at least qsa_dense_attn_decode_workspace() bytes.
 */
QSA_API size_t qsa_dense_attn_decode_workspace(int32_t B, int32_t Hq, int32_t d, int64_t kv_stride, int32_t dtype);
QSA_API int qsa_dense_attn_decode(const void *q, const void *k, const void *v, const int32_t *seq_len, int32_t B,
                                  int64_t kv_stride, int32_t Hq, int32_t Hkv, int32_t d, float scale, void *out,
                                  float *lse, void *workspace, size_t ws_bytes, int32_t dtype, void *stream);

/* ========================================================================= */
/* Decode sparse attention without a workspace (allocation-free callers)      */
/* ========================================================================= */
/*
 * Not a step of the method: the source pages have no counterpart.  This is a
 * convenience for callers that cannot allocate device memory where they call
 * QSA (an engine that gives all free memory to its KV pool and forbids
 * allocation in the decode loop, a host thread that must not block on
 * cudaMalloc/cudaFree, a fixed pre-planned memory budget).
 *
 * Same arguments, results and errors as qsa_sparse_attn_decode, minus the
 * workspace: the split-KV partial results live in a scratch area compiled
 * into the library, QSA_NOALLOC_SCRATCH_BYTES of device memory on every GPU
 * that loads the library, held until the process exits.  Calls needing more
 * (roughly B * splits * Hq * 516 bytes, splits ~ 2 * SMs / B) return
 * QSA_ERR_WORKSPACE (for example B = 64 with Hq = 32: 4,227,072 bytes).
 * Allocates nothing.  The scratch's device address is looked up
 * (cudaGetSymbolAddress) by the first call of any entry point of this library
 * on a device, with that device current, and cached; make that first call (for
 * example qsa_check_status) before any stream capture, since a lookup inside
 * a capture can fail with QSA_ERR_CUDA depending on the capture mode.  The
 * fp32 path keeps no partial results and uses no scratch.  Every call on a
 * device shares the one scratch area: calls whose work can overlap on the GPU
 * (different streams without ordering) race and must be serialised by the
 * caller.  Nothing needs clearing between calls.
 */
#define QSA_NOALLOC_SCRATCH_BYTES (4u << 20)
QSA_API int qsa_sparse_attn_decode_noalloc(const void *q, const void *k, const void *v, const int32_t *seq_len,
                                           const int32_t *sel, const int32_t *nsel, int32_t B, int64_t kv_stride,
                                           int32_t Hq, int32_t Hkv, int32_t d, int32_t top_k, float scale, void *out,
                                           float *lse, int32_t dtype, void *stream);

/*
 * The prefill counterpart: full causal attention of query rows q0 .. q0 +
 * n_q - 1 over every cached position up to each row's own (the baseline the
 * pages' 7.6x prefill ratio is quoted against).  Tiled over queries and keys
 * (each K/V tile is loaded once for 8 queries of a kv head).  QSA_BF16 with
 * Hq = 8 Hkv, Hkv in {1, 2, 4}, d = 128.  q, out [B][n_q][Hq][d]; k, v
 * [B][kv_stride][Hkv][d]; lse [B][n_q][Hq] float or NULL; kv_stride >= q0 +
 * n_q and B * kv_stride <= 2^31.  No workspace.
 */
QSA_API int qsa_dense_attn_prefill(const void *q, const void *k, const void *v, int32_t B, int64_t n_q, int64_t q0,
                                   int64_t kv_stride, int32_t Hq, int32_t Hkv, int32_t d, float scale, void *out,
                                   float *lse, int32_t dtype, void *stream);

/* ========================================================================= */
/* FP8 K/V caches                                                             */
/* ========================================================================= */
/*
 * Page "Qwen3.8-Flash-Next, Layer by Layer", section "Serving it": with an
 * FP8 cache the QSA keys and values take 12 KiB per token, and the serving
 * recipe there runs with an FP8 KV cache.  The pages give no scaling
 * scheme; here the caches hold FP8 E4M3 bytes with one scale per tensor
 * (K = k_scale * stored value, V = v_scale * stored value, the engines'
 * per-tensor form), q and out stay BF16.  Scores use the exact products of
 * the BF16 query and the dequantized keys (FP16 tensor-core MMAs, the query
 * scaled by a power of two), probabilities are rounded to FP16 for the value
 * MMAs.  As qsa_sparse_attn_prefill / qsa_sparse_attn_decode otherwise
 * (Hq = 8 Hkv with Hkv in {1, 2, 4} and d = 128, or 24q / 2kv with d = 256);
 * k, v are [B][kv_stride][Hkv][d]
 * bytes; k_scale, v_scale finite and > 0.  Decode workspace as
 * qsa_sparse_attn_decode_workspace(..., QSA_BF16).
 */
QSA_API int qsa_sparse_attn_prefill_kv8(const void *q, const void *k, const void *v, float k_scale, float v_scale,
                                        const int32_t *sel, const int32_t *nsel, int32_t B, int64_t n_q, int64_t q0,
                                        int64_t kv_stride, int32_t Hq, int32_t Hkv, int32_t d, int32_t top_k,
                                        float scale, void *out, float *lse, void *stream);
QSA_API int qsa_sparse_attn_decode_kv8(const void *q, const void *k, const void *v, float k_scale, float v_scale,
                                       const int32_t *seq_len, const int32_t *sel, const int32_t *nsel, int32_t B,
                                       int64_t kv_stride, int32_t Hq, int32_t Hkv, int32_t d, int32_t top_k,
                                       float scale, void *out, float *lse, void *workspace, size_t ws_bytes,
                                       void *stream);

/* ========================================================================= */
/* Paged caches (decode)                                                      */
/* ========================================================================= */
/*
 * Page "Qwen3.8-Flash-Next: Day-0 Support in SGLang", section "Qwen Sparse
 * Attention: Retrieve Coarsely, Attend Precisely": serving keeps the
 * original K/V in the engine's paged pool, and a paged scorer reads the
 * compressed keys there.  The K/V cache is a pool of fixed-size pages
 * and addresses the compressed-key cache at full_slot / 4, so the 4 tokens of
 * a block share one page and their compressed key is one row of a paged
 * compressed-key cache.  A page table maps each sequence's positions to
 * slots:
 *   slot(b, i) = page_table[b][i / page_tokens] * page_tokens + i % page_tokens
 * The K/V caches are [num_pages * page_tokens][Hkv][d]; the compressed-key
 * cache is [num_pages * page_tokens / 4][128] and block j of sequence b is
 * its row slot(b, 4j) / 4.  page_tokens is a power of two >= 32; positions
 * 0 .. max_pages * page_tokens - 1 of a sequence are addressable.  A page id
 * outside [0, num_pages) met by a kernel is flagged (status bit 1) and its
 * rows are skipped.  BF16 only (QSA_ERR_UNSUPPORTED otherwise); results are
 * those of the contiguous entry points on the same logical caches.
 */
typedef struct {
    const int32_t *page_table;   /* device, [B][max_pages] int32 page ids */
    int64_t max_pages;           /* entries per table row */
    int64_t num_pages;           /* pages in the caches */
    int32_t page_tokens;         /* token slots per page */
} qsa_paging_t;

/* qsa_pool_keys_prefill into a paged compressed-key cache (k_pool as above). */
QSA_API int qsa_pool_keys_prefill_paged(const void *k_raw, void *k_pool, qsa_paging_t paging, int32_t B,
                                        int64_t n_tok, int64_t pos0, int64_t raw_stride, qsa_rope_t rope,
                                        uint32_t flags, int32_t dtype, void *stream);
/* qsa_pool_keys_decode into a paged compressed-key cache (the ring stays
 * [B][4][128] per sequence). */
QSA_API int qsa_pool_keys_decode_paged(const void *k_new, void *ring, void *k_pool, qsa_paging_t paging,
                                       const int32_t *seq_len, int32_t B, qsa_rope_t rope, uint32_t flags,
                                       int32_t dtype, void *stream);
/* qsa_index_topk_decode over a paged compressed-key cache; max_blocks as
 * there (<= max_pages * page_tokens / 4); workspace sized and kept as for
 * qsa_index_topk_decode (qsa_index_topk_decode_workspace). */
QSA_API int qsa_index_topk_decode_paged(const void *q_idx, const void *k_pool, qsa_paging_t paging,
                                        const float *head_w, const int32_t *seq_len, int32_t B, int64_t max_blocks,
                                        int32_t top_k, int32_t *sel, int32_t *nsel, void *workspace,
                                        size_t ws_bytes, qsa_rope_t rope, uint32_t flags, int32_t dtype,
                                        void *stream);
/* qsa_sparse_attn_decode over paged K/V caches; workspace as
 * qsa_sparse_attn_decode_workspace(). */
QSA_API int qsa_sparse_attn_decode_paged(const void *q, const void *k, const void *v, qsa_paging_t paging,
                                         const int32_t *seq_len, const int32_t *sel, const int32_t *nsel, int32_t B,
                                         int32_t Hq, int32_t Hkv, int32_t d, int32_t top_k, float scale, void *out,
                                         float *lse, void *workspace, size_t ws_bytes, int32_t dtype, void *stream);

/* ========================================================================= */
/* Helper: the attention layer's RoPE                                         */
/* ========================================================================= */
/*
 * Rotates x[i][r][h][0..d) in place at position pos0 + r (fp64 angles,
 * result rounded to dtype), for i < B, r < n, h < H.  This is the rotation
 * the pages keep in the full-attention layers ("Token mixing": the
 * full-attention layers keep rotary position embeddings); callers use it to
 * produce the rotated q/k the sparse attention consumes.
 * x: device, [B][n][H][d] dtype, d even, rotary_dim <= d.
 */
QSA_API int qsa_rope_apply(void *x, int32_t B, int64_t n, int32_t H, int32_t d, int64_t pos0, qsa_rope_t rope,
                   int32_t dtype, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* QSA_H */
