// qsa_noalloc.cu -- decode sparse attention without a caller-provided workspace.
//
// Some callers cannot allocate device memory where they call into QSA: a
// serving engine that hands all free device memory to its KV pool at start-up
// and forbids allocation inside its decode loop, a host thread that must not
// block (cudaMalloc and cudaFree can synchronise the device), or a host with
// a fixed, pre-planned memory budget.  For them, qsa_sparse_attn_decode_noalloc
// runs the same split-KV decode attention as qsa_sparse_attn_decode, but keeps
// its split partial results in a fixed scratch area compiled into the library
// (QSA_NOALLOC_SCRATCH_BYTES of device memory on every GPU that loads it,
// held until the process exits).
//
// The scratch is shared by every call on a device: calls whose work overlaps on
// the GPU (different streams, no ordering between them) race on it.  Every
// partial result is written before it is read within one call, so nothing has
// to be cleared between calls.
#include <cmath>
#include <mutex>

#include "../../include/qsa.h"
#include "internal.h"

// File-scope device scratch: the split-KV partial outputs and log-sum-exps.
static __device__ __align__(256) unsigned char g_noalloc_scratch[QSA_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDev = 64;
std::mutex g_scratch_mu;
void *g_scratch_ptr[kMaxDev];
bool g_scratch_ok[kMaxDev];

// Device address of the scratch on the current device.  The host-side symbol
// is only a stand-in, so the address is looked up once per device (with that
// device current) and cached.
int scratch_address(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return QSA_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_ok[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return QSA_ERR_CUDA;
        g_scratch_ptr[dev] = p;
        g_scratch_ok[dev] = true;
    }
    *out = g_scratch_ptr[dev];
    return QSA_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int qsa_sparse_attn_decode_noalloc(const void *q, const void *k, const void *v, const int32_t *seq_len,
                                              const int32_t *sel, const int32_t *nsel, int32_t B, int64_t kv_stride,
                                              int32_t Hq, int32_t Hkv, int32_t d, int32_t top_k, float scale,
                                              void *out, float *lse, int32_t dtype, void *stream) {
    if (!q || !k || !v || !sel || !nsel || !out || !seq_len || B < 1 || kv_stride < 1) return QSA_ERR_INVALID_ARG;
    if (top_k < 1 || top_k > 2048) return QSA_ERR_INVALID_ARG;
    if (Hq < 1 || Hkv < 1 || (Hq % Hkv) != 0) return QSA_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !std::isfinite(scale)) return QSA_ERR_INVALID_ARG;
    if (dtype != QSA_BF16 && dtype != QSA_FP32) return QSA_ERR_UNSUPPORTED;
    if (d != 128) return QSA_ERR_UNSUPPORTED;
    if (dtype == QSA_BF16 && (Hq != 8 * Hkv || (Hkv != 1 && Hkv != 2 && Hkv != 4))) return QSA_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return QSA_ERR_INVALID_ARG;
    const qsa::DeviceInfo *di = qsa::device_info();
    if (!di) return QSA_ERR_CUDA;
    if (di->major != 10) return QSA_ERR_UNSUPPORTED;
    qsa::AttnArgs a{q, k, v, sel, nsel, seq_len, B, 1, 0, kv_stride, Hq, Hkv, d, top_k, scale, out, lse, true};
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dtype == QSA_FP32)   // the fp32 kernel keeps no partial results
        return qsa::launch_attn_f32(a, di->status, s) == cudaSuccess ? QSA_OK : QSA_ERR_CUDA;
    if (qsa::attn_decode_ws_bytes(B, Hq, d, top_k) > (size_t)QSA_NOALLOC_SCRATCH_BYTES) return QSA_ERR_WORKSPACE;
    void *scratch = nullptr;
    const int st = scratch_address(&scratch);
    if (st != QSA_OK) return st;
    return qsa::launch_attn_bf16(a, scratch, di->status, s) == cudaSuccess ? QSA_OK : QSA_ERR_CUDA;
}
