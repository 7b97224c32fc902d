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
#include "../../include/qsa.h"
#include "internal.h"

// File-scope device scratch: the split-KV partial outputs and log-sum-exps.
static __device__ __align__(256) unsigned char g_noalloc_scratch[QSA_NOALLOC_SCRATCH_BYTES];

namespace qsa {

// The host-side symbol is only a stand-in for the scratch: its device address
// is looked up here, with the device in question current.  device_info()
// calls this once per device and caches the address, so any earlier library
// call on that device (qsa_check_status included) has done the lookup.
cudaError_t noalloc_scratch_address(void **out) {
    *out = nullptr;
    return cudaGetSymbolAddress(out, g_noalloc_scratch);
}

}  // namespace qsa

extern "C" int qsa_sparse_attn_decode_noalloc(const void *q, const void *k, const void *v, const int32_t *seq_len,
                                              const int32_t *sel, const int32_t *nsel, int32_t B, int64_t kv_stride,
                                              int32_t Hq, int32_t Hkv, int32_t d, int32_t top_k, float scale,
                                              void *out, float *lse, int32_t dtype, void *stream) {
    // the same argument rules as qsa_sparse_attn_decode
    int st = qsa::attn_common_checks(q, k, v, sel, nsel, B, Hq, Hkv, d, top_k, scale, out, dtype);
    if (st != QSA_OK) return st;
    if (!seq_len || kv_stride < 1) return QSA_ERR_INVALID_ARG;
    const qsa::DeviceInfo *di = qsa::device_info();
    if (!di) return QSA_ERR_CUDA;
    if (di->major != 10) return QSA_ERR_UNSUPPORTED;
    qsa::AttnArgs a{q, k, v, sel, nsel, seq_len, B, 1, 0, kv_stride, Hq, Hkv, d, top_k, scale, out, lse, true};
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dtype == QSA_FP32)   // the fp32 kernel keeps no partial results
        return qsa::launch_attn_f32(a, di->status, s) == cudaSuccess ? QSA_OK : QSA_ERR_CUDA;
    if (qsa::attn_decode_ws_bytes(B, Hq, d, top_k) > (size_t)QSA_NOALLOC_SCRATCH_BYTES) return QSA_ERR_WORKSPACE;
    return qsa::launch_attn_bf16(a, di->noalloc_scratch, di->status, s) == cudaSuccess ? QSA_OK : QSA_ERR_CUDA;
}
