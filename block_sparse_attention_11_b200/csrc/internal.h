// internal.h -- host-side launchers shared between the kernel files and the
// C-ABI layer (qsa_api.cu).  Nothing here is exported from libqsa.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"

namespace qsa {

// Launch with programmatic stream serialization (see pdl_wait in common.cuh).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// As launch_pdl, with the grid split into clusters of cluster_x CTAs along x.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, unsigned cluster_x,
                               cudaStream_t s, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster_x;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

struct DeviceInfo {
    int sm_count = 0;
    int major = 0, minor = 0;
    size_t smem_optin = 0;
    unsigned *status = nullptr;   // device address of the library status word
    void *noalloc_scratch = nullptr;   // device address of the allocation-free decode scratch
};

// Per-device info of the current device (cached).  Returns nullptr on error.
const DeviceInfo *device_info();

// Device address of the allocation-free decode scratch on the current device
// (qsa_noalloc.cu); device_info() looks it up once per device.
cudaError_t noalloc_scratch_address(void **out);

// Argument checks shared by the sparse attention entry points (qsa_api.cu):
// null pointers, top_k, head shapes, scale, dtype and 16-byte alignment.
int attn_common_checks(const void *q, const void *k, const void *v, const int32_t *sel, const int32_t *nsel,
                       int32_t B, int32_t Hq, int32_t Hkv, int32_t d, int32_t top_k, float scale, const void *out,
                       int32_t dtype);

// ---- self-test of the bounded waits (k_selftest.cu): one CTA waits on an
// mbarrier nothing arrives on, with the given limit; writes 0 to *result when
// the wait gave up (and QSA_DEV_TIMEOUT to the status word), 1 otherwise.
cudaError_t launch_wait_timeout_selftest(uint64_t limit_ns, unsigned *status, unsigned *result, cudaStream_t s);

// ---- pooling / rotation (k_rope.cu)
// fp8: the compressed keys are stored as FP8 E4M3 (bf16 raw keys only).
// pg.table != nullptr: the compressed-key cache is paged (pool_stride unused).
cudaError_t launch_pool_prefill(const void *k_raw, void *k_pool, int B, int64_t nblk, int64_t pos0,
                                int64_t raw_stride, int64_t pool_stride, Rope rope, bool rmsnorm, bool bf16,
                                bool fp8, const Paging &pg, unsigned *status, cudaStream_t s);
cudaError_t launch_pool_decode(const void *k_new, void *ring, void *k_pool, const int32_t *seq_len, int B,
                               int64_t pool_stride, Rope rope, bool rmsnorm, bool bf16, bool fp8, const Paging &pg,
                               unsigned *status, cudaStream_t s);
cudaError_t launch_rope_apply(void *x, int B, int64_t n, int H, int d, int64_t pos0, Rope rope, bool bf16,
                              cudaStream_t s);
// Indexer queries for prefill: mode 0 -> hi/lo bf16 planes of the head sum
// ([rows][128] each); mode 1 -> per-head bf16 [rows][4][128]; mode 2 -> per-head fp32.
cudaError_t launch_rotate_index_q(const void *q_idx, int B, int64_t n_q, int64_t q0, Rope rope, int mode,
                                  void *out0, void *out1, cudaStream_t s);

// ---- indexer scores (k_index.cu)
struct ScoreGemmArgs {
    int B;
    int64_t n_q;          // query rows per sequence in this call
    int64_t q0;           // position of query row 0
    int64_t row_begin;    // first query row of this chunk (within each sequence)
    int64_t row_count;    // rows of this chunk
    int64_t pool_stride;
    int64_t ld;           // score row stride (floats)
    int per_head;         // 0: hi/lo head-sum operands, 1: per-head operands
    int relu;
    const float *head_w;  // [B][n_q][4] or null
    float *scores;        // [B][row_count][ld]
    uint16_t *keys = nullptr;   // BF16 modes: [B][row_count][ld] 16-bit order keys, written instead of scores
};
cudaError_t launch_score_gemm(const ScoreGemmArgs &a, const void *qa0, const void *qa1, const void *k_pool,
                              unsigned *status, cudaStream_t s);
cudaError_t launch_score_simt_f32(const ScoreGemmArgs &a, const float *q_hat, const float *k_pool,
                                  cudaStream_t s);
cudaError_t launch_select_rows(const float *scores, int B, int64_t row_begin, int64_t row_count, int64_t n_q,
                               int64_t q0, int64_t ld, int top_k, int32_t *sel, int32_t *nsel,
                               unsigned *status, cudaStream_t s);
// Row top-k over 16-bit keys (BF16 modes): keys that tie with the threshold at
// 16 bits are re-scored in fp32 from the query operand (qa0/qa1 as the
// rotation wrote them: mode 0 hi/lo planes, mode 1 per-head) and k_pool.
cudaError_t launch_select_keys(const uint16_t *keys, int B, int64_t row_begin, int64_t row_count, int64_t n_q,
                               int64_t q0, int64_t ld, int top_k, int mode, int relu, const void *qa0, const void *qa1,
                               const void *k_pool, int64_t pool_stride, const float *head_w, int32_t *sel,
                               int32_t *nsel, cudaStream_t s);

// ---- decode indexer (k_decode_index.cu)
struct DecodePlan {
    int chunks;          // chunks per sequence
    int64_t chunk;       // blocks per chunk
};
DecodePlan decode_index_plan(int B, int64_t max_blocks, bool bf16);
size_t decode_index_ws_bytes(int B, int64_t max_blocks, int top_k, bool bf16);
// Kernels one decode-index call launches: 1 (fused scorer-select) or 2 (scorer, select).
int decode_index_kernel_count(int B, int64_t max_blocks, bool bf16, bool fp8);
cudaError_t launch_decode_index(const void *q_idx, const void *k_pool, const float *head_w,
                                const int32_t *seq_len, int B, int64_t pool_stride, int64_t max_blocks,
                                int top_k, int32_t *sel, int32_t *nsel, void *ws, Rope rope, bool relu,
                                bool bf16, bool fp8, const Paging &pg, unsigned *status, cudaStream_t s);

// ---- sparse attention (k_attn.cu)
struct AttnArgs {
    const void *q, *k, *v;
    const int32_t *sel, *nsel;
    const int32_t *seq_len;   // decode: [B]; prefill: null
    int B;
    int64_t n_q, q0, kv_stride;
    int Hq, Hkv, d, top_k;
    float scale;
    void *out;
    float *lse;
    bool decode;
    const int32_t *cap_len = nullptr;   // decode, IndexShare draft step: [B] capture rows + 1
    int max_draft = 0;                  // IndexShare: largest seq_len - cap_len
    bool dense = false;                 // decode: dense causal attention over every position (no selection)
    Paging pg;                          // pg.table: paged K/V caches (bf16 kernels), kv_stride = its capacity
    bool kv8 = false;                   // K/V caches of FP8 E4M3 (bf16 q/out): K = k_scale * k8, V = v_scale * v8
    float k_scale = 1.f, v_scale = 1.f;
    bool no_tail = false;               // prefill: the rows attend to their listed blocks only (the split prefill
                                        // gives each query's tail to the tile kernel)
};
int attn_tail_blocks(bool indexshare, int max_draft);
size_t attn_decode_ws_bytes(int B, int Hq, int d, int top_k, int tail_blocks = 1);
size_t attn_dense_decode_ws_bytes(int B, int Hq, int d, int64_t kv_stride);
cudaError_t launch_attn_bf16(const AttnArgs &a, void *ws, unsigned *status, cudaStream_t s);
// Prefill split by sharing (k_attn_tc.cu): BF16, d = 128, 8 q heads per kv
// head, contiguous BF16 K/V.  Blocks that several queries of a tile of 8
// attend to run on the tensor cores once per tile; the rest run in the gather
// kernel (launch_attn_bf16) per query; the tile kernel merges the two.  Its
// workspace holds the block lists, the per-query lists and their lse.  Used
// for contexts of at most 32768 blocks (q0 + n_q <= 131075 positions).
bool attn_union_supported(const AttnArgs &a);
size_t attn_union_ws_bytes(int B, int64_t n_q, int top_k, int Hq);
int attn_union_launches(int B, int64_t n_q, int top_k, int Hq);   // chunks per call (3 kernels each)
cudaError_t launch_attn_union(const AttnArgs &a, void *ws, unsigned *status, cudaStream_t s);
cudaError_t launch_attn_f32(const AttnArgs &a, unsigned *status, cudaStream_t s);

}  // namespace qsa
