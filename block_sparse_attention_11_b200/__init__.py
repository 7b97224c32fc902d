"""Python binding of libqsa, the C-ABI CUDA library for Qwen Sparse Attention
(QSA) on NVIDIA B200 (sm_100a).

Argument marshalling only: every function takes torch tensors (device
memory and the current CUDA stream come from PyTorch), checks dtype and
contiguity, and calls the C entry point of the same name through ctypes.
All arithmetic happens in the CUDA kernels of ``libqsa.so``.  There is no CPU
fallback: if the library is missing the import fails loudly.

Layouts and semantics are those of ``include/qsa.h``.  QSA itself is described
on the page "Qwen3.8-Flash-Next: Day-0 Support in SGLang", section "Qwen
Sparse Attention: Retrieve Coarsely, Attend Precisely".
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

__all__ = [
    "QSAError", "Rope", "lib", "LIB_PATH",
    "qsa_pool_keys_prefill", "qsa_pool_keys_decode",
    "qsa_index_topk_prefill", "qsa_index_topk_prefill_workspace",
    "qsa_index_topk_decode", "qsa_index_topk_decode_workspace", "qsa_index_topk_decode_kernels",
    "qsa_sparse_attn_prefill", "qsa_sparse_attn_prefill_workspace", "qsa_sparse_attn_prefill_kernels",
    "qsa_index_topk_prefill_kernels", "qsa_sparse_attn_decode", "qsa_sparse_attn_decode_workspace",
    "qsa_sparse_attn_decode_noalloc", "qsa_sparse_attn_decode_shared", "qsa_sparse_attn_decode_shared_workspace",
    "qsa_dense_attn_decode", "qsa_dense_attn_decode_workspace", "qsa_dense_attn_prefill",
    "qsa_pool_keys_prefill_paged", "qsa_pool_keys_decode_paged", "qsa_index_topk_decode_paged",
    "qsa_sparse_attn_decode_paged", "qsa_sparse_attn_prefill_kv8", "qsa_sparse_attn_decode_kv8",
    "qsa_rope_apply", "qsa_check_status", "qsa_selftest_wait_timeout", "qsa_strerror", "qsa_version",
    "QSA_SCORE_RELU", "QSA_POOL_RMSNORM", "QSA_KEYS_FP8", "QSA_BF16", "QSA_FP32",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libqsa.so")

QSA_OK, QSA_ERR_INVALID_ARG, QSA_ERR_UNSUPPORTED, QSA_ERR_CUDA, QSA_ERR_DEVICE, QSA_ERR_WORKSPACE = range(6)
QSA_BF16, QSA_FP32 = 0, 1
QSA_SCORE_RELU, QSA_POOL_RMSNORM, QSA_KEYS_FP8 = 1, 2, 4
QSA_NOALLOC_SCRATCH_BYTES = 4 << 20   # as in include/qsa.h


class QSAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {qsa_strerror(status)} (status {status})")


class _Paging(ctypes.Structure):
    _fields_ = [("page_table", ctypes.c_void_p), ("max_pages", ctypes.c_int64), ("num_pages", ctypes.c_int64),
                ("page_tokens", ctypes.c_int32)]


class _Rope(ctypes.Structure):
    _fields_ = [("base", ctypes.c_double), ("pos_scale", ctypes.c_double),
                ("rotary_dim", ctypes.c_int32), ("style", ctypes.c_int32)]


@dataclass(frozen=True)
class Rope:
    """RoPE parameters (rotate-half): angle_i = (pos / pos_scale) * base^(-2i/rotary_dim)."""
    base: float = 10000.0
    pos_scale: float = 1.0
    rotary_dim: int = 128
    style: int = 0

    def c(self) -> _Rope:
        return _Rope(self.base, self.pos_scale, self.rotary_dim, self.style)


if not os.path.exists(LIB_PATH):
    raise ImportError(f"libqsa.so not found at {LIB_PATH}: build it with "
                      "`python block_sparse_attention_11_b200/build.py` (nvcc, sm_100a)")

lib = ctypes.CDLL(LIB_PATH)

_i32, _i64, _u32, _sz, _vp, _f32, _d = (ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32, ctypes.c_size_t,
                                         ctypes.c_void_p, ctypes.c_float, ctypes.c_double)


def _sig(name, res, *args):
    f = getattr(lib, name)
    f.restype = res
    f.argtypes = list(args)
    return f


_sig("qsa_strerror", ctypes.c_char_p, ctypes.c_int)
_sig("qsa_version", ctypes.c_int)
_sig("qsa_check_status", ctypes.c_int, _vp, ctypes.POINTER(_u32))
_sig("qsa_selftest_wait_timeout", ctypes.c_int, ctypes.c_uint64, _vp, _vp)
_sig("qsa_pool_keys_prefill", ctypes.c_int, _vp, _vp, _i32, _i64, _i64, _i64, _i64, _Rope, _u32, _i32, _vp)
_sig("qsa_pool_keys_decode", ctypes.c_int, _vp, _vp, _vp, _vp, _i32, _i64, _Rope, _u32, _i32, _vp)
_sig("qsa_index_topk_prefill_workspace", _sz, _i32, _i64, _i64, _i32, _u32, _i32)
_sig("qsa_index_topk_prefill", ctypes.c_int, _vp, _vp, _vp, _i32, _i64, _i64, _i64, _i32, _vp, _vp, _vp, _sz,
     _Rope, _u32, _i32, _vp)
_sig("qsa_index_topk_decode_workspace", _sz, _i32, _i64, _i32, _u32, _i32)
_sig("qsa_index_topk_decode_kernels", ctypes.c_int, _i32, _i64, _u32, _i32)
_sig("qsa_index_topk_decode", ctypes.c_int, _vp, _vp, _vp, _vp, _i32, _i64, _i64, _i32, _vp, _vp, _vp, _sz,
     _Rope, _u32, _i32, _vp)
_sig("qsa_sparse_attn_prefill", ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _i32, _i64, _i64, _i64, _i32, _i32, _i32,
     _i32, _f32, _vp, _vp, _vp, _sz, _i32, _vp)
_sig("qsa_sparse_attn_decode_workspace", _sz, _i32, _i32, _i32, _i32, _i32)
_sig("qsa_sparse_attn_prefill_workspace", _sz, _i32, _i64, _i64, _i32, _i32, _i32, _i32, _i32)
_sig("qsa_sparse_attn_prefill_kernels", ctypes.c_int, _i32, _i64, _i64, _i32, _i32, _i32, _i32, _i32)
_sig("qsa_index_topk_prefill_kernels", ctypes.c_int, _i32, _i64, _i64, _u32, _i32)
_sig("qsa_sparse_attn_decode", ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i64, _i32, _i32, _i32, _i32,
     _f32, _vp, _vp, _vp, _sz, _i32, _vp)
_sig("qsa_sparse_attn_decode_shared_workspace", _sz, _i32, _i32, _i32, _i32, _i32, _i32)
_sig("qsa_sparse_attn_decode_shared", ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i64, _i32, _i32, _i32,
     _i32, _i32, _f32, _vp, _vp, _vp, _sz, _i32, _vp)
_sig("qsa_dense_attn_decode_workspace", _sz, _i32, _i32, _i32, _i64, _i32)
_sig("qsa_dense_attn_decode", ctypes.c_int, _vp, _vp, _vp, _vp, _i32, _i64, _i32, _i32, _i32, _f32, _vp, _vp, _vp, _sz,
     _i32, _vp)
_sig("qsa_rope_apply", ctypes.c_int, _vp, _i32, _i64, _i32, _i32, _i64, _Rope, _i32, _vp)
_sig("qsa_pool_keys_prefill_paged", ctypes.c_int, _vp, _vp, _Paging, _i32, _i64, _i64, _i64, _Rope, _u32, _i32, _vp)
_sig("qsa_pool_keys_decode_paged", ctypes.c_int, _vp, _vp, _vp, _Paging, _vp, _i32, _Rope, _u32, _i32, _vp)
_sig("qsa_index_topk_decode_paged", ctypes.c_int, _vp, _vp, _Paging, _vp, _vp, _i32, _i64, _i32, _vp, _vp, _vp, _sz,
     _Rope, _u32, _i32, _vp)
_sig("qsa_sparse_attn_decode_paged", ctypes.c_int, _vp, _vp, _vp, _Paging, _vp, _vp, _vp, _i32, _i32, _i32, _i32,
     _i32, _f32, _vp, _vp, _vp, _sz, _i32, _vp)
_sig("qsa_dense_attn_prefill", ctypes.c_int, _vp, _vp, _vp, _i32, _i64, _i64, _i64, _i32, _i32, _i32, _f32, _vp, _vp,
     _i32, _vp)
_sig("qsa_sparse_attn_prefill_kv8", ctypes.c_int, _vp, _vp, _vp, _f32, _f32, _vp, _vp, _i32, _i64, _i64, _i64, _i32,
     _i32, _i32, _i32, _f32, _vp, _vp, _vp)
_sig("qsa_sparse_attn_decode_kv8", ctypes.c_int, _vp, _vp, _vp, _f32, _f32, _vp, _vp, _vp, _i32, _i64, _i32, _i32,
     _i32, _i32, _f32, _vp, _vp, _vp, _sz, _vp)
_sig("qsa_sparse_attn_decode_noalloc", ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i64, _i32, _i32, _i32,
     _i32, _f32, _vp, _vp, _i32, _vp)


def qsa_strerror(status: int) -> str:
    return lib.qsa_strerror(int(status)).decode()


def qsa_version() -> int:
    return lib.qsa_version()


# ----------------------------------------------------------------------------- helpers

def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return QSA_BF16
    if t.dtype == torch.float32:
        return QSA_FP32
    raise TypeError(f"unsupported dtype {t.dtype}: QSA takes bfloat16 or float32")


def _ptr(t, dtype=None, name="tensor"):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def _kpool_ptr(k_pool, dtype, flags):
    """Compressed-key cache pointer: `dtype` (the computation type), or one
    byte per value (float8_e4m3fn or uint8) under QSA_KEYS_FP8."""
    if flags & QSA_KEYS_FP8:
        if not isinstance(k_pool, torch.Tensor) or k_pool.dtype not in (torch.float8_e4m3fn, torch.uint8):
            raise TypeError("k_pool must be float8_e4m3fn (or uint8) with QSA_KEYS_FP8")
        return _ptr(k_pool, None, "k_pool")
    return _ptr(k_pool, dtype, "k_pool")


def _stream(t: torch.Tensor, stream=None):
    if stream is None:
        stream = torch.cuda.current_stream(t.device)
    return stream.cuda_stream


def _check(status: int, where: str):
    if status != QSA_OK:
        raise QSAError(status, where)


def _ws(nbytes: int, device, workspace, zero=False):
    """Workspace pointer and size; allocated here when none is given (zero-filled
    for an entry point whose workspace must start zero)."""
    if nbytes == 0:
        return None, 0
    if workspace is None:
        workspace = (torch.zeros if zero else torch.empty)(nbytes, dtype=torch.uint8, device=device)
    if workspace.numel() * workspace.element_size() < nbytes:
        raise ValueError(f"workspace too small: need {nbytes} bytes")
    return workspace.data_ptr(), workspace.numel() * workspace.element_size()


# ----------------------------------------------------------------------------- entry points

def qsa_pool_keys_prefill(k_raw, k_pool, pos0=0, rope=Rope(), flags=0, n_tok=None, stream=None):
    """k_raw [B][S][128] -> k_pool[:, pos0/4 : pos0/4 + n_tok//4] (n_tok defaults to S)."""
    dt = _dtype_code(k_raw)
    B, S, D = k_raw.shape
    assert D == 128 and k_pool.dim() == 3 and k_pool.shape[0] == B and k_pool.shape[2] == 128
    n_tok = S if n_tok is None else n_tok
    st = lib.qsa_pool_keys_prefill(_ptr(k_raw, None, "k_raw"), _kpool_ptr(k_pool, k_raw.dtype, flags), B, n_tok, pos0, S,
                                   k_pool.shape[1], rope.c(), flags, dt, _stream(k_raw, stream))
    _check(st, "qsa_pool_keys_prefill")


def qsa_pool_keys_decode(k_new, ring, k_pool, seq_len, rope=Rope(), flags=0, stream=None):
    dt = _dtype_code(k_new)
    B = k_new.shape[0]
    st = lib.qsa_pool_keys_decode(_ptr(k_new, None, "k_new"), _ptr(ring, k_new.dtype, "ring"),
                                  _kpool_ptr(k_pool, k_new.dtype, flags), _ptr(seq_len, torch.int32, "seq_len"), B,
                                  k_pool.shape[1], rope.c(), flags, dt, _stream(k_new, stream))
    _check(st, "qsa_pool_keys_decode")


def qsa_index_topk_prefill_workspace(B, n_q, q0, top_k, flags=0, dtype=QSA_BF16) -> int:
    return lib.qsa_index_topk_prefill_workspace(B, n_q, q0, top_k, flags, dtype)


def qsa_index_topk_prefill(q_idx, k_pool, sel, nsel, q0=0, top_k=512, head_w=None, rope=Rope(), flags=0,
                           workspace=None, stream=None):
    """q_idx [B][n_q][4][128] raw; k_pool [B][P][128]; sel [B][n_q][top_k] int32; nsel [B][n_q] int32."""
    dt = _dtype_code(q_idx)
    B, n_q = q_idx.shape[0], q_idx.shape[1]
    need = qsa_index_topk_prefill_workspace(B, n_q, q0, top_k, flags, dt)
    wp, wb = _ws(need, q_idx.device, workspace)
    st = lib.qsa_index_topk_prefill(_ptr(q_idx, None, "q_idx"), _ptr(k_pool, q_idx.dtype, "k_pool"),
                                    _ptr(head_w, torch.float32, "head_w"), B, n_q, q0, k_pool.shape[1], top_k,
                                    _ptr(sel, torch.int32, "sel"), _ptr(nsel, torch.int32, "nsel"), wp, wb,
                                    rope.c(), flags, dt, _stream(q_idx, stream))
    _check(st, "qsa_index_topk_prefill")


def qsa_index_topk_decode_kernels(B, max_blocks, flags=0, dtype=QSA_BF16) -> int:
    """Kernels one qsa_index_topk_decode call launches (1 fused, 2 scorer + select)."""
    return lib.qsa_index_topk_decode_kernels(B, max_blocks, flags, dtype)


def qsa_index_topk_decode_workspace(B, max_blocks, top_k, flags=0, dtype=QSA_BF16) -> int:
    return lib.qsa_index_topk_decode_workspace(B, max_blocks, top_k, flags, dtype)


def qsa_index_topk_decode(q_idx, k_pool, seq_len, sel, nsel, max_blocks=None, top_k=512, head_w=None, rope=Rope(),
                          flags=0, workspace=None, stream=None):
    """q_idx [B][4][128] raw; k_pool [B][P][128]; seq_len [B] int32 (incl. the new token)."""
    dt = _dtype_code(q_idx)
    B = q_idx.shape[0]
    max_blocks = k_pool.shape[1] if max_blocks is None else max_blocks
    need = qsa_index_topk_decode_workspace(B, max_blocks, top_k, flags, dt)
    wp, wb = _ws(need, q_idx.device, workspace, zero=True)   # zero-filled once; calls leave it zero
    st = lib.qsa_index_topk_decode(_ptr(q_idx, None, "q_idx"), _kpool_ptr(k_pool, q_idx.dtype, flags),
                                   _ptr(head_w, torch.float32, "head_w"), _ptr(seq_len, torch.int32, "seq_len"), B,
                                   k_pool.shape[1], max_blocks, top_k, _ptr(sel, torch.int32, "sel"),
                                   _ptr(nsel, torch.int32, "nsel"), wp, wb, rope.c(), flags, dt,
                                   _stream(q_idx, stream))
    _check(st, "qsa_index_topk_decode")


def qsa_sparse_attn_prefill_kernels(B, n_q, top_k, Hq, Hkv, d, dtype=QSA_BF16, q0=0) -> int:
    return lib.qsa_sparse_attn_prefill_kernels(B, n_q, q0, top_k, Hq, Hkv, d, dtype)


def qsa_index_topk_prefill_kernels(B, n_q, q0=0, flags=0, dtype=QSA_BF16) -> int:
    return lib.qsa_index_topk_prefill_kernels(B, n_q, q0, flags, dtype)


def qsa_sparse_attn_prefill_workspace(B, n_q, top_k, Hq, Hkv, d, dtype=QSA_BF16, q0=0) -> int:
    return lib.qsa_sparse_attn_prefill_workspace(B, n_q, q0, top_k, Hq, Hkv, d, dtype)


def qsa_sparse_attn_prefill(q, k, v, sel, nsel, out, q0=0, top_k=None, scale=None, lse=None, workspace=None,
                            stream=None):
    """q [B][n_q][Hq][d]; k, v [B][L][Hkv][d]; sel [B][n_q][top_k]; out like q.  workspace: a uint8
    device tensor of at least qsa_sparse_attn_prefill_workspace() bytes (allocated here when None)."""
    dt = _dtype_code(q)
    B, n_q, Hq, d = q.shape
    Hkv = k.shape[2]
    top_k = sel.shape[-1] if top_k is None else top_k
    scale = (1.0 / d ** 0.5) if scale is None else scale
    need = qsa_sparse_attn_prefill_workspace(B, max(n_q, 1), top_k, Hq, Hkv, d, dt, q0=q0)
    wp, wb = _ws(need, q.device, workspace) if need else (None, 0)
    st = lib.qsa_sparse_attn_prefill(_ptr(q, None, "q"), _ptr(k, q.dtype, "k"), _ptr(v, q.dtype, "v"),
                                     _ptr(sel, torch.int32, "sel"), _ptr(nsel, torch.int32, "nsel"), B, n_q, q0,
                                     k.shape[1], Hq, Hkv, d, top_k, scale, _ptr(out, q.dtype, "out"),
                                     _ptr(lse, torch.float32, "lse"), wp, wb, dt, _stream(q, stream))
    _check(st, "qsa_sparse_attn_prefill")


def qsa_sparse_attn_decode_workspace(B, Hq, d, top_k, dtype=QSA_BF16) -> int:
    return lib.qsa_sparse_attn_decode_workspace(B, Hq, d, top_k, dtype)


def qsa_sparse_attn_decode(q, k, v, seq_len, sel, nsel, out, top_k=None, scale=None, lse=None, workspace=None,
                           stream=None):
    """q [B][Hq][d]; k, v [B][L][Hkv][d] (new token already written); out [B][Hq][d]."""
    dt = _dtype_code(q)
    B, Hq, d = q.shape
    Hkv = k.shape[2]
    top_k = sel.shape[-1] if top_k is None else top_k
    scale = (1.0 / d ** 0.5) if scale is None else scale
    need = qsa_sparse_attn_decode_workspace(B, Hq, d, top_k, dt)
    wp, wb = _ws(need, q.device, workspace)
    st = lib.qsa_sparse_attn_decode(_ptr(q, None, "q"), _ptr(k, q.dtype, "k"), _ptr(v, q.dtype, "v"),
                                    _ptr(seq_len, torch.int32, "seq_len"), _ptr(sel, torch.int32, "sel"),
                                    _ptr(nsel, torch.int32, "nsel"), B, k.shape[1], Hq, Hkv, d, top_k, scale,
                                    _ptr(out, q.dtype, "out"), _ptr(lse, torch.float32, "lse"), wp, wb, dt,
                                    _stream(q, stream))
    _check(st, "qsa_sparse_attn_decode")


def qsa_sparse_attn_decode_shared_workspace(B, Hq, d, top_k, max_draft, dtype=QSA_BF16) -> int:
    return lib.qsa_sparse_attn_decode_shared_workspace(B, Hq, d, top_k, max_draft, dtype)


def qsa_sparse_attn_decode_shared(q, k, v, seq_len, cap_len, sel, nsel, out, max_draft, top_k=None, scale=None,
                                  lse=None, workspace=None, stream=None):
    """IndexShare draft step: attention of the token at seq_len - 1 over the
    selection made for the capture row cap_len - 1 (sel/nsel) plus positions
    4 * (cap_len // 4) .. seq_len - 1.  q [B][Hq][d]; k, v [B][L][Hkv][d]."""
    dt = _dtype_code(q)
    B, Hq, d = q.shape
    Hkv = k.shape[2]
    top_k = sel.shape[-1] if top_k is None else top_k
    scale = (1.0 / d ** 0.5) if scale is None else scale
    need = qsa_sparse_attn_decode_shared_workspace(B, Hq, d, top_k, max_draft, dt)
    wp, wb = _ws(need, q.device, workspace)
    st = lib.qsa_sparse_attn_decode_shared(_ptr(q, None, "q"), _ptr(k, q.dtype, "k"), _ptr(v, q.dtype, "v"),
                                           _ptr(seq_len, torch.int32, "seq_len"),
                                           _ptr(cap_len, torch.int32, "cap_len"), _ptr(sel, torch.int32, "sel"),
                                           _ptr(nsel, torch.int32, "nsel"), B, k.shape[1], Hq, Hkv, d, top_k,
                                           max_draft, scale, _ptr(out, q.dtype, "out"),
                                           _ptr(lse, torch.float32, "lse"), wp, wb, dt, _stream(q, stream))
    _check(st, "qsa_sparse_attn_decode_shared")


def qsa_dense_attn_decode_workspace(B, Hq, d, kv_stride, dtype=QSA_BF16) -> int:
    return lib.qsa_dense_attn_decode_workspace(B, Hq, d, kv_stride, dtype)


def qsa_dense_attn_decode(q, k, v, seq_len, out, scale=None, lse=None, workspace=None, stream=None):
    """Full causal attention of the token at seq_len - 1 over positions 0..seq_len - 1
    (the baseline QSA replaces).  q [B][Hq][d]; k, v [B][L][Hkv][d]."""
    dt = _dtype_code(q)
    B, Hq, d = q.shape
    Hkv = k.shape[2]
    scale = (1.0 / d ** 0.5) if scale is None else scale
    need = qsa_dense_attn_decode_workspace(B, Hq, d, k.shape[1], dt)
    wp, wb = _ws(need, q.device, workspace)
    st = lib.qsa_dense_attn_decode(_ptr(q, None, "q"), _ptr(k, q.dtype, "k"), _ptr(v, q.dtype, "v"),
                                   _ptr(seq_len, torch.int32, "seq_len"), B, k.shape[1], Hq, Hkv, d, scale,
                                   _ptr(out, q.dtype, "out"), _ptr(lse, torch.float32, "lse"), wp, wb, dt,
                                   _stream(q, stream))
    _check(st, "qsa_dense_attn_decode")


def qsa_sparse_attn_decode_noalloc(q, k, v, seq_len, sel, nsel, out, top_k=None, scale=None, lse=None, stream=None):
    """As qsa_sparse_attn_decode, for callers that cannot allocate device memory
    at the call: the library keeps the split partials in its own fixed scratch
    (QSA_NOALLOC_SCRATCH_BYTES per GPU).  Calls that overlap on the GPU share
    that scratch and race; the first call on a device should precede any
    stream capture."""
    dt = _dtype_code(q)
    B, Hq, d = q.shape
    Hkv = k.shape[2]
    top_k = sel.shape[-1] if top_k is None else top_k
    scale = (1.0 / d ** 0.5) if scale is None else scale
    st = lib.qsa_sparse_attn_decode_noalloc(_ptr(q, None, "q"), _ptr(k, q.dtype, "k"), _ptr(v, q.dtype, "v"),
                                            _ptr(seq_len, torch.int32, "seq_len"), _ptr(sel, torch.int32, "sel"),
                                            _ptr(nsel, torch.int32, "nsel"), B, k.shape[1], Hq, Hkv, d, top_k, scale,
                                            _ptr(out, q.dtype, "out"), _ptr(lse, torch.float32, "lse"), dt,
                                            _stream(q, stream))
    _check(st, "qsa_sparse_attn_decode_noalloc")


def _paging(page_table, num_pages, page_tokens):
    """Paging descriptor: page_table [B][max_pages] int32 on the device."""
    return _Paging(_ptr(page_table, torch.int32, "page_table"), page_table.shape[1], int(num_pages), int(page_tokens))


def qsa_pool_keys_prefill_paged(k_raw, k_pool, page_table, page_tokens, pos0=0, rope=Rope(), flags=0, n_tok=None,
                                stream=None):
    """k_raw [B][S][128] -> rows slot(b, 4j) / 4 of the paged compressed-key cache
    k_pool [num_pages * page_tokens / 4][128] for blocks j of positions pos0 .. pos0 + n_tok."""
    dt = _dtype_code(k_raw)
    B, S, D = k_raw.shape
    assert D == 128 and k_pool.dim() == 2 and k_pool.shape[1] == 128
    n_tok = S if n_tok is None else n_tok
    pg = _paging(page_table, k_pool.shape[0] * 4 // page_tokens, page_tokens)
    st = lib.qsa_pool_keys_prefill_paged(_ptr(k_raw, None, "k_raw"), _kpool_ptr(k_pool, k_raw.dtype, flags), pg, B,
                                         n_tok, pos0, S, rope.c(), flags, dt, _stream(k_raw, stream))
    _check(st, "qsa_pool_keys_prefill_paged")


def qsa_pool_keys_decode_paged(k_new, ring, k_pool, page_table, page_tokens, seq_len, rope=Rope(), flags=0,
                               stream=None):
    dt = _dtype_code(k_new)
    B = k_new.shape[0]
    pg = _paging(page_table, k_pool.shape[0] * 4 // page_tokens, page_tokens)
    st = lib.qsa_pool_keys_decode_paged(_ptr(k_new, None, "k_new"), _ptr(ring, k_new.dtype, "ring"),
                                        _kpool_ptr(k_pool, k_new.dtype, flags), pg,
                                        _ptr(seq_len, torch.int32, "seq_len"), B, rope.c(), flags, dt,
                                        _stream(k_new, stream))
    _check(st, "qsa_pool_keys_decode_paged")


def qsa_index_topk_decode_paged(q_idx, k_pool, page_table, page_tokens, seq_len, sel, nsel, max_blocks=None,
                                top_k=512, head_w=None, rope=Rope(), flags=0, workspace=None, stream=None):
    """As qsa_index_topk_decode over the paged compressed-key cache k_pool
    [num_pages * page_tokens / 4][128]."""
    dt = _dtype_code(q_idx)
    B = q_idx.shape[0]
    max_blocks = page_table.shape[1] * page_tokens // 4 if max_blocks is None else max_blocks
    need = qsa_index_topk_decode_workspace(B, max_blocks, top_k, flags, dt)
    wp, wb = _ws(need, q_idx.device, workspace, zero=True)
    pg = _paging(page_table, k_pool.shape[0] * 4 // page_tokens, page_tokens)
    st = lib.qsa_index_topk_decode_paged(_ptr(q_idx, None, "q_idx"), _kpool_ptr(k_pool, q_idx.dtype, flags), pg,
                                         _ptr(head_w, torch.float32, "head_w"), _ptr(seq_len, torch.int32, "seq_len"),
                                         B, max_blocks, top_k, _ptr(sel, torch.int32, "sel"),
                                         _ptr(nsel, torch.int32, "nsel"), wp, wb, rope.c(), flags, dt,
                                         _stream(q_idx, stream))
    _check(st, "qsa_index_topk_decode_paged")


def qsa_sparse_attn_decode_paged(q, k, v, page_table, page_tokens, seq_len, sel, nsel, out, top_k=None, scale=None,
                                 lse=None, workspace=None, stream=None):
    """As qsa_sparse_attn_decode over paged K/V caches k, v [num_pages * page_tokens][Hkv][d]."""
    dt = _dtype_code(q)
    B, Hq, d = q.shape
    Hkv = k.shape[1]
    top_k = sel.shape[-1] if top_k is None else top_k
    scale = (1.0 / d ** 0.5) if scale is None else scale
    need = qsa_sparse_attn_decode_workspace(B, Hq, d, top_k, dt)
    wp, wb = _ws(need, q.device, workspace)
    pg = _paging(page_table, k.shape[0] // page_tokens, page_tokens)
    st = lib.qsa_sparse_attn_decode_paged(_ptr(q, None, "q"), _ptr(k, q.dtype, "k"), _ptr(v, q.dtype, "v"), pg,
                                          _ptr(seq_len, torch.int32, "seq_len"), _ptr(sel, torch.int32, "sel"),
                                          _ptr(nsel, torch.int32, "nsel"), B, Hq, Hkv, d, top_k, scale,
                                          _ptr(out, q.dtype, "out"), _ptr(lse, torch.float32, "lse"), wp, wb, dt,
                                          _stream(q, stream))
    _check(st, "qsa_sparse_attn_decode_paged")


def qsa_dense_attn_prefill(q, k, v, out, q0=0, scale=None, lse=None, stream=None):
    """Full causal attention of query rows q0 .. q0 + n_q - 1 over every cached position up
    to each row's own (the dense baseline).  q, out [B][n_q][Hq][d]; k, v [B][L][Hkv][d]."""
    dt = _dtype_code(q)
    B, n_q, Hq, d = q.shape
    Hkv = k.shape[2]
    scale = (1.0 / d ** 0.5) if scale is None else scale
    st = lib.qsa_dense_attn_prefill(_ptr(q, None, "q"), _ptr(k, q.dtype, "k"), _ptr(v, q.dtype, "v"), B, n_q, q0,
                                    k.shape[1], Hq, Hkv, d, scale, _ptr(out, q.dtype, "out"),
                                    _ptr(lse, torch.float32, "lse"), dt, _stream(q, stream))
    _check(st, "qsa_dense_attn_prefill")


def _kv8_ptr(t, name):
    if not isinstance(t, torch.Tensor) or t.dtype not in (torch.float8_e4m3fn, torch.uint8):
        raise TypeError(f"{name} must be float8_e4m3fn (or uint8)")
    return _ptr(t, None, name)


def qsa_sparse_attn_prefill_kv8(q, k, v, k_scale, v_scale, sel, nsel, out, q0=0, top_k=None, scale=None, lse=None,
                                stream=None):
    """As qsa_sparse_attn_prefill with FP8 E4M3 K/V caches (K = k_scale * k, V = v_scale * v);
    q, out bfloat16 [B][n_q][Hq][d]; k, v [B][L][Hkv][d] float8_e4m3fn."""
    B, n_q, Hq, d = q.shape
    Hkv = k.shape[2]
    top_k = sel.shape[-1] if top_k is None else top_k
    scale = (1.0 / d ** 0.5) if scale is None else scale
    st = lib.qsa_sparse_attn_prefill_kv8(_ptr(q, torch.bfloat16, "q"), _kv8_ptr(k, "k"), _kv8_ptr(v, "v"),
                                         float(k_scale), float(v_scale), _ptr(sel, torch.int32, "sel"),
                                         _ptr(nsel, torch.int32, "nsel"), B, n_q, q0, k.shape[1], Hq, Hkv, d, top_k,
                                         scale, _ptr(out, torch.bfloat16, "out"), _ptr(lse, torch.float32, "lse"),
                                         _stream(q, stream))
    _check(st, "qsa_sparse_attn_prefill_kv8")


def qsa_sparse_attn_decode_kv8(q, k, v, k_scale, v_scale, seq_len, sel, nsel, out, top_k=None, scale=None, lse=None,
                               workspace=None, stream=None):
    """As qsa_sparse_attn_decode with FP8 E4M3 K/V caches (K = k_scale * k, V = v_scale * v)."""
    B, Hq, d = q.shape
    Hkv = k.shape[2]
    top_k = sel.shape[-1] if top_k is None else top_k
    scale = (1.0 / d ** 0.5) if scale is None else scale
    need = qsa_sparse_attn_decode_workspace(B, Hq, d, top_k, QSA_BF16)
    wp, wb = _ws(need, q.device, workspace)
    st = lib.qsa_sparse_attn_decode_kv8(_ptr(q, torch.bfloat16, "q"), _kv8_ptr(k, "k"), _kv8_ptr(v, "v"),
                                        float(k_scale), float(v_scale), _ptr(seq_len, torch.int32, "seq_len"),
                                        _ptr(sel, torch.int32, "sel"), _ptr(nsel, torch.int32, "nsel"), B,
                                        k.shape[1], Hq, Hkv, d, top_k, scale, _ptr(out, torch.bfloat16, "out"),
                                        _ptr(lse, torch.float32, "lse"), wp, wb, _stream(q, stream))
    _check(st, "qsa_sparse_attn_decode_kv8")


def qsa_rope_apply(x, pos0=0, rope=Rope(), stream=None):
    """Rotate x [B][n][H][d] in place at positions pos0 + r."""
    dt = _dtype_code(x)
    B, n, H, d = x.shape
    st = lib.qsa_rope_apply(_ptr(x, None, "x"), B, n, H, d, pos0, rope.c(), dt, _stream(x, stream))
    _check(st, "qsa_rope_apply")


def qsa_selftest_wait_timeout(limit_ns, result, stream=None):
    """Run the bounded-wait self-test: one CTA waits on an mbarrier nothing
    arrives on, gives up after limit_ns, frees its TMEM and returns; result
    (a 1-element int32 device tensor) receives 0 when the wait gave up."""
    _check(lib.qsa_selftest_wait_timeout(int(limit_ns), _ptr(result, torch.int32, "result"), _stream(result, stream)),
           "qsa_selftest_wait_timeout")


def qsa_check_status(stream=None, device=None):
    """Synchronise and read/clear the library's device status word; raises on a flagged error."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    s = (stream or torch.cuda.current_stream(dev)).cuda_stream
    detail = _u32()
    st = lib.qsa_check_status(s, ctypes.byref(detail))
    if st != QSA_OK:
        raise QSAError(st, f"qsa_check_status (bits 0x{detail.value:x})")
    return detail.value
