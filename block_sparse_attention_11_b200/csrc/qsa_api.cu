// qsa_api.cu -- the C ABI of libqsa (declared in include/qsa.h).
//
// Argument checking, workspace carving and kernel launches.  Every entry
// point validates its arguments before launching anything, never allocates
// device memory and never synchronises (qsa_check_status excepted).
#include <algorithm>
#include <cmath>
#include <mutex>

#include "../../include/qsa.h"
#include "dense.h"
#include "internal.h"

namespace qsa {

// One status word per device; kernels OR QSA_DEV_* bits into it.
__device__ unsigned g_status;

namespace {
constexpr int kMaxDevices = 64;
DeviceInfo g_info[kMaxDevices];
bool g_info_ok[kMaxDevices];
std::mutex g_info_mu;
}  // namespace

const DeviceInfo *device_info() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_info_mu);
    if (!g_info_ok[dev]) {
        DeviceInfo d;
        if (cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return nullptr;
        if (cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return nullptr;
        if (cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return nullptr;
        int optin = 0;
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        d.smem_optin = (size_t)optin;
        void *addr = nullptr;
        if (cudaGetSymbolAddress(&addr, g_status) != cudaSuccess) return nullptr;
        d.status = static_cast<unsigned *>(addr);
        if (noalloc_scratch_address(&d.noalloc_scratch) != cudaSuccess || !d.noalloc_scratch) return nullptr;
        g_info[dev] = d;
        g_info_ok[dev] = true;
    }
    return &g_info[dev];
}

}  // namespace qsa

using namespace qsa;

namespace {

int check_device(const DeviceInfo **out) {
    const DeviceInfo *di = device_info();
    if (!di) return QSA_ERR_CUDA;
    if (di->major != 10) return QSA_ERR_UNSUPPORTED;   // sm_100 family only
    *out = di;
    return QSA_OK;
}

int check_rope(const qsa_rope_t &r) {
    if (r.style != 0) return QSA_ERR_UNSUPPORTED;
    if (!(r.base > 1.0) || !std::isfinite(r.base) || !(r.pos_scale > 0.0) || !std::isfinite(r.pos_scale))
        return QSA_ERR_INVALID_ARG;
    if (r.rotary_dim < 16 || r.rotary_dim > 128 || (r.rotary_dim % 16) != 0) return QSA_ERR_INVALID_ARG;
    return QSA_OK;
}

Rope to_rope(const qsa_rope_t &r) {
    Rope k{};
    for (int i = 0; i < r.rotary_dim / 2; ++i) k.inv_freq[i] = std::pow(r.base, -(2.0 * i) / (double)r.rotary_dim);
    k.pos_scale = r.pos_scale;
    k.rotary_dim = r.rotary_dim;
    return k;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int cuda_status(cudaError_t e) { return e == cudaSuccess ? QSA_OK : QSA_ERR_CUDA; }

constexpr uint32_t kAllFlags = QSA_SCORE_RELU | QSA_POOL_RMSNORM | QSA_KEYS_FP8;

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

// Prefill indexer workspace layout: [rotated queries][scores of one query chunk].
struct PrefillPlan {
    int mode;            // 0 hi/lo, 1 per-head bf16, 2 per-head fp32
    size_t q_bytes;      // rotated query buffer(s)
    int64_t ld;          // score row stride
    int64_t chunk;       // query rows per chunk
    size_t score_bytes;
    bool key16;          // 16-bit order keys (BF16, rows of at most 32768 blocks), else fp32 scores
};

PrefillPlan prefill_plan(int B, int64_t n_q, int64_t q0, uint32_t flags, int dtype, bool has_w) {
    PrefillPlan p{};
    const bool per_head = (flags & QSA_SCORE_RELU) || has_w;
    p.mode = dtype == QSA_FP32 ? 2 : (per_head ? 1 : 0);
    const int64_t nb_max0 = (q0 + n_q) / kBlock;
    // BF16 rows of at most 32768 blocks store 16-bit keys (the key select); longer rows keep
    // fp32 scores and the fp32 selects, measured faster there (1M context in 16,000-token
    // chunks: indexer 395 vs 479 ms)
    p.key16 = p.mode != 2 && nb_max0 <= 32768;
    const size_t rows = (size_t)B * (size_t)n_q;
    if (p.mode == 0) p.q_bytes = 2 * round256(rows * kIdxDim * 2);
    else if (p.mode == 1) p.q_bytes = round256(rows * kIdxHeads * kIdxDim * 2);
    else p.q_bytes = round256(rows * kIdxHeads * kIdxDim * 4);
    const int64_t nb_max = (q0 + n_q) / kBlock;
    p.ld = std::max<int64_t>(128, (nb_max + 127) / 128 * 128);
    // BF16 modes store 16-bit order keys, fp32 mode the scores; keep one chunk under 2 GiB;
    // chunks are multiples of 128 rows
    const int64_t el = p.key16 ? 2 : 4;
    const int64_t budget_rows = std::max<int64_t>(128, ((int64_t)1 << 31) / (p.ld * el * std::max(B, 1)) / 128 * 128);
    p.chunk = std::min<int64_t>(std::max<int64_t>(n_q, 1), budget_rows);
    p.score_bytes = round256((size_t)B * p.chunk * p.ld * el);
    return p;
}

}  // namespace

namespace qsa {
int attn_common_checks(const void *q, const void *k, const void *v, const int32_t *sel, const int32_t *nsel,
                       int32_t B, int32_t Hq, int32_t Hkv, int32_t d, int32_t top_k, float scale, const void *out,
                       int32_t dtype) {
    if (!q || !k || !v || !sel || !nsel || !out || B < 1) return QSA_ERR_INVALID_ARG;
    if (top_k < 1 || top_k > 2048) return QSA_ERR_INVALID_ARG;
    if (Hq < 1 || Hkv < 1 || (Hq % Hkv) != 0) return QSA_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !std::isfinite(scale)) return QSA_ERR_INVALID_ARG;
    if (dtype != QSA_BF16 && dtype != QSA_FP32) return QSA_ERR_UNSUPPORTED;
    // shapes: d = 128 with 8 q heads per kv head (1, 2 or 4 kv heads; fp32: any GQA),
    // and the released 24q / 2kv, d = 256 shape (bf16)
    const bool released = dtype == QSA_BF16 && d == 256 && Hkv == 2 && Hq == 24;
    if (d != 128 && !released) return QSA_ERR_UNSUPPORTED;
    if (dtype == QSA_BF16 && !released && (Hq != 8 * Hkv || (Hkv != 1 && Hkv != 2 && Hkv != 4)))
        return QSA_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return QSA_ERR_INVALID_ARG;
    return QSA_OK;
}
}  // namespace qsa

extern "C" {

const char *qsa_strerror(int status) {
    switch (status) {
    case QSA_OK: return "ok";
    case QSA_ERR_INVALID_ARG: return "invalid argument";
    case QSA_ERR_UNSUPPORTED: return "unsupported shape, dtype, option or device";
    case QSA_ERR_CUDA: return "CUDA error";
    case QSA_ERR_DEVICE: return "kernel reported an out-of-range index or a wait timeout";
    case QSA_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
    }
}

int qsa_version(void) { return 100; }

int qsa_check_status(void *stream, uint32_t *detail) {
    const DeviceInfo *di = nullptr;
    int st = check_device(&di);
    if (st != QSA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned v = 0;
    if (cudaStreamSynchronize(s) != cudaSuccess) return QSA_ERR_CUDA;
    if (cudaMemcpy(&v, di->status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return QSA_ERR_CUDA;
    const unsigned zero = 0;
    if (cudaMemcpy(di->status, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return QSA_ERR_CUDA;
    if (detail) *detail = v;
    return v ? QSA_ERR_DEVICE : QSA_OK;
}

int qsa_selftest_wait_timeout(uint64_t limit_ns, uint32_t *result, void *stream) {
    if (!result || limit_ns < 1 || limit_ns > kWaitNs) return QSA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(result) & 3u) != 0) return QSA_ERR_INVALID_ARG;
    const DeviceInfo *di = nullptr;
    int st = check_device(&di);
    if (st != QSA_OK) return st;
    return cuda_status(launch_wait_timeout_selftest(limit_ns, di->status, result, static_cast<cudaStream_t>(stream)));
}

int qsa_pool_keys_prefill(const void *k_raw, void *k_pool, int32_t B, int64_t n_tok, int64_t pos0,
                          int64_t raw_stride, int64_t pool_stride, qsa_rope_t rope, uint32_t flags, int32_t dtype,
                          void *stream) {
    if (B < 1 || n_tok < 0 || pos0 < 0 || (pos0 % kBlock) != 0 || raw_stride < n_tok) return QSA_ERR_INVALID_ARG;
    if (n_tok < kBlock) return QSA_OK;   // no complete block: nothing to pool
    if (!k_raw || !k_pool) return QSA_ERR_INVALID_ARG;
    if (flags & ~kAllFlags) return QSA_ERR_INVALID_ARG;
    if (dtype != QSA_BF16 && dtype != QSA_FP32) return QSA_ERR_UNSUPPORTED;
    if ((flags & QSA_KEYS_FP8) && dtype != QSA_BF16) return QSA_ERR_UNSUPPORTED;
    const int64_t nblk = n_tok / kBlock;
    if (pool_stride < pos0 / kBlock + nblk) return QSA_ERR_INVALID_ARG;
    if (!aligned16(k_raw) || !aligned16(k_pool)) return QSA_ERR_INVALID_ARG;
    int st = check_rope(rope);
    if (st != QSA_OK) return st;
    const DeviceInfo *di = nullptr;
    if ((st = check_device(&di)) != QSA_OK) return st;
    return cuda_status(launch_pool_prefill(k_raw, k_pool, B, nblk, pos0, raw_stride, pool_stride, to_rope(rope),
                                           (flags & QSA_POOL_RMSNORM) != 0, dtype == QSA_BF16,
                                           (flags & QSA_KEYS_FP8) != 0, Paging{}, di->status,
                                           static_cast<cudaStream_t>(stream)));
}

int qsa_pool_keys_decode(const void *k_new, void *ring, void *k_pool, const int32_t *seq_len, int32_t B,
                         int64_t pool_stride, qsa_rope_t rope, uint32_t flags, int32_t dtype, void *stream) {
    if (!k_new || !ring || !k_pool || !seq_len || B < 1 || pool_stride < 1) return QSA_ERR_INVALID_ARG;
    if (flags & ~kAllFlags) return QSA_ERR_INVALID_ARG;
    if (dtype != QSA_BF16 && dtype != QSA_FP32) return QSA_ERR_UNSUPPORTED;
    if ((flags & QSA_KEYS_FP8) && dtype != QSA_BF16) return QSA_ERR_UNSUPPORTED;
    int st = check_rope(rope);
    if (st != QSA_OK) return st;
    const DeviceInfo *di = nullptr;
    if ((st = check_device(&di)) != QSA_OK) return st;
    return cuda_status(launch_pool_decode(k_new, ring, k_pool, seq_len, B, pool_stride, to_rope(rope),
                                          (flags & QSA_POOL_RMSNORM) != 0, dtype == QSA_BF16,
                                          (flags & QSA_KEYS_FP8) != 0, Paging{}, di->status,
                                          static_cast<cudaStream_t>(stream)));
}

size_t qsa_index_topk_prefill_workspace(int32_t B, int64_t n_q, int64_t q0, int32_t top_k, uint32_t flags,
                                        int32_t dtype) {
    (void)top_k;
    if (B < 1 || n_q < 0 || q0 < 0) return 0;
    // head weights force the per-head layout; size for the larger of the two
    const PrefillPlan a = prefill_plan(B, n_q, q0, flags, dtype, false);
    const PrefillPlan b = prefill_plan(B, n_q, q0, flags, dtype, true);
    return std::max(a.q_bytes, b.q_bytes) + a.score_bytes;
}

int qsa_index_topk_prefill(const void *q_idx, const void *k_pool, const float *head_w, int32_t B, int64_t n_q,
                           int64_t q0, int64_t pool_stride, int32_t top_k, int32_t *sel, int32_t *nsel,
                           void *workspace, size_t ws_bytes, qsa_rope_t rope, uint32_t flags, int32_t dtype,
                           void *stream) {
    if (!q_idx || !k_pool || !sel || !nsel || B < 1 || n_q < 0 || q0 < 0) return QSA_ERR_INVALID_ARG;
    if (top_k < 1 || top_k > 2048) return QSA_ERR_INVALID_ARG;
    if (flags & ~kAllFlags) return QSA_ERR_INVALID_ARG;
    if (dtype != QSA_BF16 && dtype != QSA_FP32) return QSA_ERR_UNSUPPORTED;
    if (flags & QSA_KEYS_FP8) return QSA_ERR_UNSUPPORTED;   // the prefill GEMM reads BF16 compressed keys
    if (n_q == 0) return QSA_OK;
    const int64_t nb_max = (q0 + n_q) / kBlock;
    if (pool_stride < std::max<int64_t>(nb_max, 1)) return QSA_ERR_INVALID_ARG;
    if (!aligned16(q_idx) || !aligned16(k_pool)) return QSA_ERR_INVALID_ARG;
    if ((B * n_q * kIdxHeads > INT32_MAX) || (B * pool_stride > INT32_MAX)) return QSA_ERR_UNSUPPORTED;
    int st = check_rope(rope);
    if (st != QSA_OK) return st;
    const DeviceInfo *di = nullptr;
    if ((st = check_device(&di)) != QSA_OK) return st;
    const PrefillPlan pl = prefill_plan(B, n_q, q0, flags, dtype, head_w != nullptr);
    if (!workspace || ws_bytes < pl.q_bytes + pl.score_bytes) return QSA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return QSA_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    void *q0buf = ws;
    void *q1buf = ws + pl.q_bytes / 2;
    float *scores = reinterpret_cast<float *>(ws + pl.q_bytes);
    cudaError_t e = launch_rotate_index_q(q_idx, B, n_q, q0, to_rope(rope), pl.mode, q0buf, q1buf, s);
    if (e != cudaSuccess) return QSA_ERR_CUDA;
    for (int64_t r = 0; r < n_q; r += pl.chunk) {
        ScoreGemmArgs a{};
        a.B = B;
        a.n_q = n_q;
        a.q0 = q0;
        a.row_begin = r;
        a.row_count = std::min(pl.chunk, n_q - r);
        a.pool_stride = pool_stride;
        a.ld = pl.ld;
        a.per_head = pl.mode != 0;
        a.relu = (flags & QSA_SCORE_RELU) ? 1 : 0;
        a.head_w = head_w;
        a.scores = scores;
        if (!pl.key16) {
            if (pl.mode == 2)
                e = launch_score_simt_f32(a, static_cast<const float *>(q0buf), static_cast<const float *>(k_pool), s);
            else
                e = launch_score_gemm(a, q0buf, q1buf, k_pool, di->status, s);
            if (e != cudaSuccess) return QSA_ERR_CUDA;
            e = launch_select_rows(scores, B, r, a.row_count, n_q, q0, pl.ld, top_k, sel, nsel, di->status, s);
        } else {
            a.keys = reinterpret_cast<uint16_t *>(scores);
            e = launch_score_gemm(a, q0buf, q1buf, k_pool, di->status, s);
            if (e != cudaSuccess) return QSA_ERR_CUDA;
            e = launch_select_keys(a.keys, B, r, a.row_count, n_q, q0, pl.ld, top_k, pl.mode, a.relu, q0buf, q1buf,
                                   k_pool, pool_stride, head_w, sel, nsel, s);
        }
        if (e != cudaSuccess) return QSA_ERR_CUDA;
    }
    return QSA_OK;
}

int qsa_index_topk_prefill_kernels(int32_t B, int64_t n_q, int64_t q0, uint32_t flags, int32_t dtype) {
    if (B < 1 || n_q < 0 || q0 < 0 || (flags & ~kAllFlags) || (dtype != QSA_BF16 && dtype != QSA_FP32)) return 0;
    if (n_q == 0) return 0;
    const PrefillPlan pl = prefill_plan(B, n_q, q0, flags, dtype, false);
    // query rotation, then per chunk of rows: scores and the row select
    return 1 + 2 * (int)((n_q + pl.chunk - 1) / pl.chunk);
}

size_t qsa_index_topk_decode_workspace(int32_t B, int64_t max_blocks, int32_t top_k, uint32_t flags, int32_t dtype) {
    (void)flags;
    if (B < 1 || max_blocks < 0 || top_k < 1) return 0;
    return decode_index_ws_bytes(B, std::max<int64_t>(max_blocks, 1), top_k, dtype == QSA_BF16);
}

int qsa_index_topk_decode_kernels(int32_t B, int64_t max_blocks, uint32_t flags, int32_t dtype) {
    if (B < 1 || max_blocks < 0 || (flags & ~kAllFlags) || (dtype != QSA_BF16 && dtype != QSA_FP32)) return 0;
    const DeviceInfo *di = nullptr;
    if (check_device(&di) != QSA_OK) return 0;
    return decode_index_kernel_count(B, max_blocks, dtype == QSA_BF16, (flags & QSA_KEYS_FP8) != 0);
}

int qsa_index_topk_decode(const void *q_idx, const void *k_pool, const float *head_w, const int32_t *seq_len,
                          int32_t B, int64_t pool_stride, int64_t max_blocks, int32_t top_k, int32_t *sel,
                          int32_t *nsel, void *workspace, size_t ws_bytes, qsa_rope_t rope, uint32_t flags,
                          int32_t dtype, void *stream) {
    if (!q_idx || !k_pool || !seq_len || !sel || !nsel || B < 1 || pool_stride < 1 || max_blocks < 0)
        return QSA_ERR_INVALID_ARG;
    if (top_k < 1 || top_k > 2048) return QSA_ERR_INVALID_ARG;
    if (flags & ~kAllFlags) return QSA_ERR_INVALID_ARG;
    if (dtype != QSA_BF16 && dtype != QSA_FP32) return QSA_ERR_UNSUPPORTED;
    if ((flags & QSA_KEYS_FP8) && dtype != QSA_BF16) return QSA_ERR_UNSUPPORTED;
    if (!aligned16(q_idx) || !aligned16(k_pool)) return QSA_ERR_INVALID_ARG;
    int st = check_rope(rope);
    if (st != QSA_OK) return st;
    const DeviceInfo *di = nullptr;
    if ((st = check_device(&di)) != QSA_OK) return st;
    const int64_t mb = std::max<int64_t>(max_blocks, 1);
    const size_t need = decode_index_ws_bytes(B, mb, top_k, dtype == QSA_BF16);
    if (!workspace || ws_bytes < need) return QSA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return QSA_ERR_INVALID_ARG;
    cudaError_t e = launch_decode_index(q_idx, k_pool, head_w, seq_len, B, pool_stride, mb, top_k, sel, nsel,
                                        workspace, to_rope(rope), (flags & QSA_SCORE_RELU) != 0, dtype == QSA_BF16,
                                        (flags & QSA_KEYS_FP8) != 0, Paging{}, di->status,
                                        static_cast<cudaStream_t>(stream));
    if (e == cudaErrorInvalidConfiguration) return QSA_ERR_UNSUPPORTED;
    return cuda_status(e);
}


size_t qsa_sparse_attn_prefill_workspace(int32_t B, int64_t n_q, int64_t q0, int32_t top_k, int32_t Hq, int32_t Hkv,
                                         int32_t d, int32_t dtype) {
    if (B < 1 || n_q < 1 || q0 < 0 || top_k < 1 || top_k > 2048 || Hq < 1 || Hkv < 1) return 0;
    AttnArgs a{};
    a.n_q = n_q;
    a.q0 = q0;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.d = d;
    if (dtype != QSA_BF16 || !attn_union_supported(a)) return 0;
    return attn_union_ws_bytes(B, n_q, top_k, Hq);
}

int qsa_sparse_attn_prefill_kernels(int32_t B, int64_t n_q, int64_t q0, int32_t top_k, int32_t Hq, int32_t Hkv,
                                    int32_t d, int32_t dtype) {
    if (B < 1 || n_q < 1 || q0 < 0 || top_k < 1 || top_k > 2048 || Hq < 1 || Hkv < 1) return 0;
    AttnArgs a{};
    a.n_q = n_q;
    a.q0 = q0;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.d = d;
    if (dtype != QSA_BF16 || !attn_union_supported(a)) return 1;
    return 3 * attn_union_launches(B, n_q, top_k, Hq);   // per chunk: block lists, gather kernel, tiles
}

int qsa_sparse_attn_prefill(const void *q, const void *k, const void *v, const int32_t *sel, const int32_t *nsel,
                            int32_t B, int64_t n_q, int64_t q0, int64_t kv_stride, int32_t Hq, int32_t Hkv, int32_t d,
                            int32_t top_k, float scale, void *out, float *lse, void *workspace, size_t ws_bytes,
                            int32_t dtype, void *stream) {
    int st = attn_common_checks(q, k, v, sel, nsel, B, Hq, Hkv, d, top_k, scale, out, dtype);
    if (st != QSA_OK) return st;
    if (n_q < 0 || q0 < 0 || kv_stride < q0 + n_q) return QSA_ERR_INVALID_ARG;
    if (n_q == 0) return QSA_OK;
    if ((int64_t)B * n_q > INT32_MAX || (int64_t)kv_stride > INT32_MAX) return QSA_ERR_UNSUPPORTED;   // TMA coordinates
    const DeviceInfo *di = nullptr;
    if ((st = check_device(&di)) != QSA_OK) return st;
    AttnArgs a{q, k, v, sel, nsel, nullptr, B, n_q, q0, kv_stride, Hq, Hkv, d, top_k, scale, out, lse, false};
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dtype == QSA_BF16 && attn_union_supported(a)) {
        const size_t need = attn_union_ws_bytes(B, n_q, top_k, Hq);
        if (!workspace || ws_bytes < need) return QSA_ERR_WORKSPACE;
        if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return QSA_ERR_INVALID_ARG;
        return cuda_status(launch_attn_union(a, workspace, di->status, s));
    }
    cudaError_t e = dtype == QSA_BF16 ? launch_attn_bf16(a, nullptr, di->status, s) : launch_attn_f32(a, di->status, s);
    return cuda_status(e);
}

size_t qsa_sparse_attn_decode_workspace(int32_t B, int32_t Hq, int32_t d, int32_t top_k, int32_t dtype) {
    if (B < 1 || Hq < 1 || d < 1 || top_k < 1) return 0;
    if (dtype == QSA_FP32) return 0;
    return attn_decode_ws_bytes(B, Hq, d, top_k);
}

int qsa_sparse_attn_decode(const void *q, const void *k, const void *v, const int32_t *seq_len, const int32_t *sel,
                           const int32_t *nsel, int32_t B, int64_t kv_stride, int32_t Hq, int32_t Hkv, int32_t d,
                           int32_t top_k, float scale, void *out, float *lse, void *workspace, size_t ws_bytes,
                           int32_t dtype, void *stream) {
    int st = attn_common_checks(q, k, v, sel, nsel, B, Hq, Hkv, d, top_k, scale, out, dtype);
    if (st != QSA_OK) return st;
    if (!seq_len || kv_stride < 1) return QSA_ERR_INVALID_ARG;
    const DeviceInfo *di = nullptr;
    if ((st = check_device(&di)) != QSA_OK) return st;
    AttnArgs a{q, k, v, sel, nsel, seq_len, B, 1, 0, kv_stride, Hq, Hkv, d, top_k, scale, out, lse, true};
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dtype == QSA_BF16) {
        const size_t need = attn_decode_ws_bytes(B, Hq, d, top_k);
        if (!workspace || ws_bytes < need) return QSA_ERR_WORKSPACE;
        return cuda_status(launch_attn_bf16(a, workspace, di->status, s));
    }
    return cuda_status(launch_attn_f32(a, di->status, s));
}

size_t qsa_sparse_attn_decode_shared_workspace(int32_t B, int32_t Hq, int32_t d, int32_t top_k, int32_t max_draft,
                                               int32_t dtype) {
    if (B < 1 || Hq < 1 || d < 1 || top_k < 1 || max_draft < 0 || max_draft > 64) return 0;
    if (dtype != QSA_BF16) return 0;
    return attn_decode_ws_bytes(B, Hq, d, top_k, attn_tail_blocks(true, max_draft));
}

int qsa_sparse_attn_decode_shared(const void *q, const void *k, const void *v, const int32_t *seq_len,
                                  const int32_t *cap_len, const int32_t *sel, const int32_t *nsel, int32_t B,
                                  int64_t kv_stride, int32_t Hq, int32_t Hkv, int32_t d, int32_t top_k,
                                  int32_t max_draft, float scale, void *out, float *lse, void *workspace,
                                  size_t ws_bytes, int32_t dtype, void *stream) {
    int st = attn_common_checks(q, k, v, sel, nsel, B, Hq, Hkv, d, top_k, scale, out, dtype);
    if (st != QSA_OK) return st;
    if (!seq_len || !cap_len || kv_stride < 1 || max_draft < 0 || max_draft > 64) return QSA_ERR_INVALID_ARG;
    const DeviceInfo *di = nullptr;
    if ((st = check_device(&di)) != QSA_OK) return st;
    AttnArgs a{q, k, v, sel, nsel, seq_len, B, 1, 0, kv_stride, Hq, Hkv, d, top_k, scale, out, lse, true};
    a.cap_len = cap_len;
    a.max_draft = max_draft;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dtype == QSA_BF16) {
        const size_t need = attn_decode_ws_bytes(B, Hq, d, top_k, attn_tail_blocks(true, max_draft));
        if (!workspace || ws_bytes < need) return QSA_ERR_WORKSPACE;
        return cuda_status(launch_attn_bf16(a, workspace, di->status, s));
    }
    return cuda_status(launch_attn_f32(a, di->status, s));
}

size_t qsa_dense_attn_decode_workspace(int32_t B, int32_t Hq, int32_t d, int64_t kv_stride, int32_t dtype) {
    if (B < 1 || Hq < 1 || d < 1 || kv_stride < 1 || kv_stride > ((int64_t)1 << 30)) return 0;
    if (dtype != QSA_BF16) return 0;
    return attn_dense_decode_ws_bytes(B, Hq, d, kv_stride);
}

int qsa_dense_attn_decode(const void *q, const void *k, const void *v, const int32_t *seq_len, int32_t B,
                          int64_t kv_stride, int32_t Hq, int32_t Hkv, int32_t d, float scale, void *out, float *lse,
                          void *workspace, size_t ws_bytes, int32_t dtype, void *stream) {
    // the shape rules of the sparse kernels, with a dummy (unused) selection
    const int32_t dummy = 0;
    int st = attn_common_checks(q, k, v, &dummy, &dummy, B, Hq, Hkv, d, 1, scale, out, dtype);
    if (st != QSA_OK) return st;
    if (!seq_len || kv_stride < 1 || kv_stride > ((int64_t)1 << 30)) return QSA_ERR_INVALID_ARG;
    const DeviceInfo *di = nullptr;
    if ((st = check_device(&di)) != QSA_OK) return st;
    AttnArgs a{q, k, v, nullptr, nullptr, seq_len, B, 1, 0, kv_stride, Hq, Hkv, d, 1, scale, out, lse, true};
    a.dense = true;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dtype == QSA_BF16) {
        const size_t need = attn_dense_decode_ws_bytes(B, Hq, d, kv_stride);
        if (!workspace || ws_bytes < need) return QSA_ERR_WORKSPACE;
        return cuda_status(launch_attn_bf16(a, workspace, di->status, s));
    }
    return cuda_status(launch_attn_f32(a, di->status, s));
}

int qsa_rope_apply(void *x, int32_t B, int64_t n, int32_t H, int32_t d, int64_t pos0, qsa_rope_t rope, int32_t dtype,
                   void *stream) {
    if (!x || B < 1 || n < 0 || H < 1 || d < 2 || (d % 2) != 0 || pos0 < 0) return QSA_ERR_INVALID_ARG;
    if (dtype != QSA_BF16 && dtype != QSA_FP32) return QSA_ERR_UNSUPPORTED;
    int st = check_rope(rope);
    if (st != QSA_OK) return st;
    if (rope.rotary_dim > d) return QSA_ERR_INVALID_ARG;
    const DeviceInfo *di = nullptr;
    if ((st = check_device(&di)) != QSA_OK) return st;
    return cuda_status(launch_rope_apply(x, B, n, H, d, pos0, to_rope(rope), dtype == QSA_BF16,
                                         static_cast<cudaStream_t>(stream)));
}

// ---------------------------------------------------------------- dense causal prefill (baseline)

int qsa_dense_attn_prefill(const void *q, const void *k, const void *v, int32_t B, int64_t n_q, int64_t q0,
                           int64_t kv_stride, int32_t Hq, int32_t Hkv, int32_t d, float scale, void *out, float *lse,
                           int32_t dtype, void *stream) {
    if (!q || !k || !v || !out || B < 1 || n_q < 0 || q0 < 0 || kv_stride < q0 + n_q) return QSA_ERR_INVALID_ARG;
    if (Hq < 1 || Hkv < 1 || (Hq % Hkv) != 0) return QSA_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !std::isfinite(scale)) return QSA_ERR_INVALID_ARG;
    if (dtype != QSA_BF16 || d != 128 || Hq != 8 * Hkv || (Hkv != 1 && Hkv != 2 && Hkv != 4))
        return QSA_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return QSA_ERR_INVALID_ARG;
    if ((int64_t)B * kv_stride > ((int64_t)1 << 31)) return QSA_ERR_UNSUPPORTED;   // TMA row coordinates
    if (n_q == 0) return QSA_OK;
    const DeviceInfo *di = nullptr;
    int st = check_device(&di);
    if (st != QSA_OK) return st;
    return cuda_status(launch_dense_prefill(q, k, v, B, n_q, q0, kv_stride, Hkv, scale, out, lse, di->status,
                                            static_cast<cudaStream_t>(stream)));
}

// ---------------------------------------------------------------- FP8 K/V caches

namespace {
int kv8_checks(const void *q, const void *k, const void *v, const int32_t *sel, const int32_t *nsel, int32_t B,
               int32_t Hq, int32_t Hkv, int32_t d, int32_t top_k, float scale, float k_scale, float v_scale,
               const void *out) {
    int st = attn_common_checks(q, k, v, sel, nsel, B, Hq, Hkv, d, top_k, scale, out, QSA_BF16);
    if (st != QSA_OK) return st;
    if (!(k_scale > 0.f) || !std::isfinite(k_scale) || !(v_scale > 0.f) || !std::isfinite(v_scale))
        return QSA_ERR_INVALID_ARG;
    return QSA_OK;
}
}  // namespace

int qsa_sparse_attn_prefill_kv8(const void *q, const void *k, const void *v, float k_scale, float v_scale,
                                const int32_t *sel, const int32_t *nsel, int32_t B, int64_t n_q, int64_t q0,
                                int64_t kv_stride, int32_t Hq, int32_t Hkv, int32_t d, int32_t top_k, float scale,
                                void *out, float *lse, void *stream) {
    int st = kv8_checks(q, k, v, sel, nsel, B, Hq, Hkv, d, top_k, scale, k_scale, v_scale, out);
    if (st != QSA_OK) return st;
    if (n_q < 0 || q0 < 0 || kv_stride < q0 + n_q) return QSA_ERR_INVALID_ARG;
    if (n_q == 0) return QSA_OK;
    const DeviceInfo *di = nullptr;
    if ((st = check_device(&di)) != QSA_OK) return st;
    AttnArgs a{q, k, v, sel, nsel, nullptr, B, n_q, q0, kv_stride, Hq, Hkv, d, top_k, scale, out, lse, false};
    a.kv8 = true;
    a.k_scale = k_scale;
    a.v_scale = v_scale;
    return cuda_status(launch_attn_bf16(a, nullptr, di->status, static_cast<cudaStream_t>(stream)));
}

int qsa_sparse_attn_decode_kv8(const void *q, const void *k, const void *v, float k_scale, float v_scale,
                               const int32_t *seq_len, const int32_t *sel, const int32_t *nsel, int32_t B,
                               int64_t kv_stride, int32_t Hq, int32_t Hkv, int32_t d, int32_t top_k, float scale,
                               void *out, float *lse, void *workspace, size_t ws_bytes, void *stream) {
    int st = kv8_checks(q, k, v, sel, nsel, B, Hq, Hkv, d, top_k, scale, k_scale, v_scale, out);
    if (st != QSA_OK) return st;
    if (!seq_len || kv_stride < 1) return QSA_ERR_INVALID_ARG;
    const DeviceInfo *di = nullptr;
    if ((st = check_device(&di)) != QSA_OK) return st;
    const size_t need = attn_decode_ws_bytes(B, Hq, d, top_k);
    if (!workspace || ws_bytes < need) return QSA_ERR_WORKSPACE;
    AttnArgs a{q, k, v, sel, nsel, seq_len, B, 1, 0, kv_stride, Hq, Hkv, d, top_k, scale, out, lse, true};
    a.kv8 = true;
    a.k_scale = k_scale;
    a.v_scale = v_scale;
    return cuda_status(launch_attn_bf16(a, workspace, di->status, static_cast<cudaStream_t>(stream)));
}

// ---------------------------------------------------------------- paged caches

namespace {
// Validates a paging descriptor for capacity `need_tokens` (positions 0 ..
// need_tokens - 1 of a sequence must fit the table row).
int check_paging(const qsa_paging_t &pg, int64_t need_tokens, Paging *out) {
    if (!pg.page_table || pg.max_pages < 1 || pg.num_pages < 1) return QSA_ERR_INVALID_ARG;
    const int pt = pg.page_tokens;
    if (pt < 32 || (pt & (pt - 1)) != 0) return QSA_ERR_INVALID_ARG;   // a power of two >= 32
    if (pg.num_pages > ((int64_t)1 << 31) / pt) return QSA_ERR_INVALID_ARG;
    if (need_tokens > pg.max_pages * (int64_t)pt) return QSA_ERR_INVALID_ARG;
    out->table = pg.page_table;
    out->max_pages = pg.max_pages;
    out->num_pages = pg.num_pages;
    out->page_tokens = pt;
    out->page_shift = 0;
    while ((1 << out->page_shift) < pt) ++out->page_shift;
    return QSA_OK;
}
}  // namespace

int qsa_pool_keys_prefill_paged(const void *k_raw, void *k_pool, qsa_paging_t paging, int32_t B, int64_t n_tok,
                                int64_t pos0, int64_t raw_stride, qsa_rope_t rope, uint32_t flags, int32_t dtype,
                                void *stream) {
    if (B < 1 || n_tok < 0 || pos0 < 0 || (pos0 % kBlock) != 0 || raw_stride < n_tok) return QSA_ERR_INVALID_ARG;
    Paging pg;
    int st = check_paging(paging, pos0 + n_tok, &pg);
    if (st != QSA_OK) return st;
    if (n_tok < kBlock) return QSA_OK;
    if (!k_raw || !k_pool) return QSA_ERR_INVALID_ARG;
    if (flags & ~kAllFlags) return QSA_ERR_INVALID_ARG;
    if (dtype != QSA_BF16) return QSA_ERR_UNSUPPORTED;
    if (!aligned16(k_raw) || !aligned16(k_pool)) return QSA_ERR_INVALID_ARG;
    if ((st = check_rope(rope)) != QSA_OK) return st;
    const DeviceInfo *di = nullptr;
    if ((st = check_device(&di)) != QSA_OK) return st;
    return cuda_status(launch_pool_prefill(k_raw, k_pool, B, n_tok / kBlock, pos0, raw_stride, 0, to_rope(rope),
                                           (flags & QSA_POOL_RMSNORM) != 0, true, (flags & QSA_KEYS_FP8) != 0, pg,
                                           di->status, static_cast<cudaStream_t>(stream)));
}

int qsa_pool_keys_decode_paged(const void *k_new, void *ring, void *k_pool, qsa_paging_t paging,
                               const int32_t *seq_len, int32_t B, qsa_rope_t rope, uint32_t flags, int32_t dtype,
                               void *stream) {
    if (!k_new || !ring || !k_pool || !seq_len || B < 1) return QSA_ERR_INVALID_ARG;
    Paging pg;
    int st = check_paging(paging, 0, &pg);
    if (st != QSA_OK) return st;
    if (flags & ~kAllFlags) return QSA_ERR_INVALID_ARG;
    if (dtype != QSA_BF16) return QSA_ERR_UNSUPPORTED;
    if ((st = check_rope(rope)) != QSA_OK) return st;
    const DeviceInfo *di = nullptr;
    if ((st = check_device(&di)) != QSA_OK) return st;
    return cuda_status(launch_pool_decode(k_new, ring, k_pool, seq_len, B, 0, to_rope(rope),
                                          (flags & QSA_POOL_RMSNORM) != 0, true, (flags & QSA_KEYS_FP8) != 0, pg,
                                          di->status, static_cast<cudaStream_t>(stream)));
}

int qsa_index_topk_decode_paged(const void *q_idx, const void *k_pool, qsa_paging_t paging, const float *head_w,
                                const int32_t *seq_len, int32_t B, int64_t max_blocks, int32_t top_k, int32_t *sel,
                                int32_t *nsel, void *workspace, size_t ws_bytes, qsa_rope_t rope, uint32_t flags,
                                int32_t dtype, void *stream) {
    if (!q_idx || !k_pool || !seq_len || !sel || !nsel || B < 1 || max_blocks < 0) return QSA_ERR_INVALID_ARG;
    Paging pg;
    int st = check_paging(paging, max_blocks * kBlock, &pg);
    if (st != QSA_OK) return st;
    if (top_k < 1 || top_k > 2048) return QSA_ERR_INVALID_ARG;
    if (flags & ~kAllFlags) return QSA_ERR_INVALID_ARG;
    if (dtype != QSA_BF16) return QSA_ERR_UNSUPPORTED;
    if (!aligned16(q_idx) || !aligned16(k_pool)) return QSA_ERR_INVALID_ARG;
    if ((st = check_rope(rope)) != QSA_OK) return st;
    const DeviceInfo *di = nullptr;
    if ((st = check_device(&di)) != QSA_OK) return st;
    const int64_t mb = std::max<int64_t>(max_blocks, 1);
    const size_t need = decode_index_ws_bytes(B, mb, top_k, true);
    if (!workspace || ws_bytes < need) return QSA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return QSA_ERR_INVALID_ARG;
    const int64_t capacity_rows = pg.max_pages * (pg.page_tokens / kBlock);
    cudaError_t e = launch_decode_index(q_idx, k_pool, head_w, seq_len, B, capacity_rows, mb, top_k, sel, nsel,
                                        workspace, to_rope(rope), (flags & QSA_SCORE_RELU) != 0, true,
                                        (flags & QSA_KEYS_FP8) != 0, pg, di->status,
                                        static_cast<cudaStream_t>(stream));
    if (e == cudaErrorInvalidConfiguration) return QSA_ERR_UNSUPPORTED;
    return cuda_status(e);
}

int qsa_sparse_attn_decode_paged(const void *q, const void *k, const void *v, qsa_paging_t paging,
                                 const int32_t *seq_len, const int32_t *sel, const int32_t *nsel, int32_t B,
                                 int32_t Hq, int32_t Hkv, int32_t d, int32_t top_k, float scale, void *out,
                                 float *lse, void *workspace, size_t ws_bytes, int32_t dtype, void *stream) {
    int st = attn_common_checks(q, k, v, sel, nsel, B, Hq, Hkv, d, top_k, scale, out, dtype);
    if (st != QSA_OK) return st;
    if (!seq_len) return QSA_ERR_INVALID_ARG;
    Paging pg;
    if ((st = check_paging(paging, 0, &pg)) != QSA_OK) return st;
    if (dtype != QSA_BF16) return QSA_ERR_UNSUPPORTED;
    const DeviceInfo *di = nullptr;
    if ((st = check_device(&di)) != QSA_OK) return st;
    const int64_t capacity = pg.max_pages * (int64_t)pg.page_tokens;
    AttnArgs a{q, k, v, sel, nsel, seq_len, B, 1, 0, capacity, Hq, Hkv, d, top_k, scale, out, lse, true};
    a.pg = pg;
    const size_t need = attn_decode_ws_bytes(B, Hq, d, top_k);
    if (!workspace || ws_bytes < need) return QSA_ERR_WORKSPACE;
    return cuda_status(launch_attn_bf16(a, workspace, di->status, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
