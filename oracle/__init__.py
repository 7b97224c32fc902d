"""CPU oracle for Qwen Sparse Attention (QSA) -- test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports it, and this package never imports the
product.

The arithmetic lives in ``qsa_oracle.c`` (plain loops, fp64 accumulation,
POSIX threads only across independent query rows).  This module compiles it
with gcc and wraps it with ctypes; every array crosses the boundary as a
contiguous numpy array.  Inputs are float32 arrays holding the exact values
of the (bf16 or fp32) tensors the GPU path reads.

Sources: "Qwen3.8-Flash-Next: Day-0 Support in SGLang", section "Qwen Sparse
Attention: Retrieve Coarsely, Attend Precisely" (pooling, score equation,
selection, expansion, attention over the original K/V); "Qwen3.8-Flash-Next,
Layer by Layer", section "Token mixing" (indexer shape, 512 blocks).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qsa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

IDX_HEADS = 4
IDX_DIM = 128
BLOCK = 4


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
               "-shared", "-pthread", "-o", _LIB, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


_lib = None


def _L():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _lib.oracle_round_bf16.restype = ctypes.c_double
        _lib.oracle_round_bf16.argtypes = [ctypes.c_double]
        _lib.oracle_round_e4m3.restype = ctypes.c_double
        _lib.oracle_round_e4m3.argtypes = [ctypes.c_double]
        _lib.oracle_topk.restype = ctypes.c_int
    return _lib


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _p(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.c_void_p)


def nthreads_default() -> int:
    return max(1, os.cpu_count() or 1)


def round_bf16(x: float) -> float:
    """Nearest bfloat16 value of a double, ties to even."""
    return _L().oracle_round_bf16(float(x))


def rope_rows(x, pos, base=10000.0, pos_scale=1.0, rotary_dim=128):
    """Rotate rows x[n][dim] at positions pos[n]; fp64 result."""
    x = _f32(x)
    n, dim = x.shape
    pos = np.ascontiguousarray(pos, dtype=np.int64)
    out = np.empty((n, dim), np.float64)
    _L().oracle_rope_rows(_p(x), ctypes.c_int64(n), ctypes.c_int(dim), _p(pos),
                          ctypes.c_double(base), ctypes.c_double(pos_scale),
                          ctypes.c_int(rotary_dim), _p(out))
    return out


def _store_code(store_bf16, store_fp8):
    return 2 if store_fp8 else int(bool(store_bf16))


def round_e4m3(x):
    """Elementwise round-to-nearest-even to FP8 E4M3 (saturating at +-448), from float64."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    f = _L().oracle_round_e4m3
    return np.vectorize(lambda v: f(ctypes.c_double(v)))(x)


def pool_keys(k_raw, pos0=0, base=10000.0, pos_scale=1.0, rotary_dim=128,
              rmsnorm=False, store_bf16=True, store_fp8=False):
    """Compressed keys [n/4][128] from raw indexer keys [n][128] (first token
    at position pos0, a multiple of 4); stored as BF16, FP32 or FP8 E4M3 values."""
    k_raw = _f32(k_raw)
    n = k_raw.shape[0]
    out = np.empty((n // BLOCK, IDX_DIM), np.float32)
    _L().oracle_pool_keys(_p(k_raw), ctypes.c_int64(n), ctypes.c_int64(pos0),
                          ctypes.c_double(base), ctypes.c_double(pos_scale),
                          ctypes.c_int(rotary_dim), ctypes.c_int(int(rmsnorm)),
                          ctypes.c_int(_store_code(store_bf16, store_fp8)), _p(out))
    return out


def pool_decode(k_new, ring, k_pool, seq_len, base=10000.0, pos_scale=1.0,
                rotary_dim=128, rmsnorm=False, store_bf16=True, store_fp8=False):
    """One decode pooling step for one sequence; updates ring [4][128] and
    k_pool [cap][128] (float32 arrays) in place."""
    assert ring.dtype == np.float32 and ring.flags.c_contiguous
    assert k_pool.dtype == np.float32 and k_pool.flags.c_contiguous
    k_new = _f32(k_new)
    _L().oracle_pool_decode(_p(k_new), _p(ring), _p(k_pool), ctypes.c_int64(int(seq_len)),
                            ctypes.c_double(base), ctypes.c_double(pos_scale),
                            ctypes.c_int(rotary_dim), ctypes.c_int(int(rmsnorm)),
                            ctypes.c_int(_store_code(store_bf16, store_fp8)))


def topk(scores, k):
    """Top-k of a score vector: (sel[k] ascending padded with -1, nsel, kth, next)."""
    s = np.ascontiguousarray(scores, dtype=np.float64)
    sel = np.empty(k, np.int32)
    kth = ctypes.c_double()
    nxt = ctypes.c_double()
    nsel = _L().oracle_topk(_p(s), ctypes.c_int64(s.shape[0]), ctypes.c_int(k), _p(sel),
                            ctypes.byref(kth), ctypes.byref(nxt))
    return sel, nsel, kth.value, nxt.value


def prefill_rows(rows, *, q_idx=None, k_pool=None, head_w=None, relu=False, store_bf16=True,
                 top_k=512, base=10000.0, pos_scale=1.0, rotary_dim=128,
                 q=None, k=None, v=None, Hq=16, Hkv=2, d=128, scale=None, q0=0,
                 sel_in=None, nsel_in=None, want_scores=False, nthreads=None):
    """Prefill QSA for the given query rows.

    Returns a dict with sel [n][top_k], nsel [n], kth [n], next [n],
    scores [n][cap] (when want_scores), out [n][Hq][d] and lse [n][Hq]
    (when q/k/v are given).  Row i is the query at position q0 + i.
    """
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    n = rows.shape[0]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    nthreads = nthreads or nthreads_default()
    res = {}
    q_idx_a = _f32(q_idx) if q_idx is not None else None
    k_pool_a = _f32(k_pool) if k_pool is not None else None
    head_w_a = _f32(head_w) if head_w is not None else None
    q_a = _f32(q) if q is not None else None
    k_a = _f32(k) if k is not None else None
    v_a = _f32(v) if v is not None else None
    sel_in_a = np.ascontiguousarray(sel_in, dtype=np.int32) if sel_in is not None else None
    nsel_in_a = np.ascontiguousarray(nsel_in, dtype=np.int32) if nsel_in is not None else None
    sel = np.full((n, top_k), -1, np.int32)
    nsel = np.zeros(n, np.int32)
    kth = np.full(n, np.nan)
    nxt = np.full(n, np.nan)
    cap = 0
    scores = None
    if want_scores:
        cap = int(((q0 + rows.max() + 1) // BLOCK)) if n else 0
        scores = np.full((n, max(cap, 1)), np.nan)
    out = np.zeros((n, Hq, d)) if q is not None else None
    lse = np.zeros((n, Hq)) if q is not None else None
    _L().oracle_prefill_rows(
        _p(q_idx_a), _p(k_pool_a), _p(head_w_a), ctypes.c_int(int(relu)), ctypes.c_int(int(store_bf16)),
        ctypes.c_int(top_k), ctypes.c_double(base), ctypes.c_double(pos_scale), ctypes.c_int(rotary_dim),
        _p(q_a), _p(k_a), _p(v_a), ctypes.c_int(Hq), ctypes.c_int(Hkv), ctypes.c_int(d),
        ctypes.c_double(scale), ctypes.c_int64(q0), _p(rows), ctypes.c_int64(n),
        _p(sel_in_a), _p(nsel_in_a), _p(sel), _p(nsel), _p(kth), _p(nxt),
        _p(scores), ctypes.c_int64(cap), _p(out), _p(lse), ctypes.c_int(nthreads))
    res.update(sel=sel, nsel=nsel, kth=kth, next=nxt)
    if want_scores:
        res["scores"] = scores
    if q is not None:
        res.update(out=out, lse=lse)
    return res


def dense_rows(rows, q, k, v, Hq, Hkv, d, scale=None, q0=0, nthreads=None):
    """Textbook causal attention over positions 0..t for the given rows."""
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    n = rows.shape[0]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    q_a, k_a, v_a = _f32(q), _f32(k), _f32(v)
    out = np.zeros((n, Hq, d))
    _L().oracle_dense_rows(_p(q_a), _p(k_a), _p(v_a), ctypes.c_int(Hq), ctypes.c_int(Hkv),
                           ctypes.c_int(d), ctypes.c_double(scale), ctypes.c_int64(q0), _p(rows),
                           ctypes.c_int64(n), _p(out), ctypes.c_int(nthreads or nthreads_default()))
    return out


def decode(q_idx, k_pool, seq_len, *, head_w=None, q=None, k=None, v=None, relu=False,
           store_bf16=True, top_k=512, Hq=16, Hkv=2, d=128, scale=None, base=10000.0,
           pos_scale=1.0, rotary_dim=128, nthreads=None, cap_len=None, want_scores=False):
    """One decode step for B sequences (after pooling).

    q_idx [B][4][128]; k_pool [B][stride][128]; seq_len [B]; q [B][Hq][d];
    k, v [B][kv_stride][Hkv][d].  Returns sel, nsel, kth, next, out, lse.
    cap_len [B] (IndexShare draft step): the selection is that of row
    cap_len - 1 (q_idx is that row's indexer query); the attention at row
    seq_len - 1 reads those blocks plus positions 4*floor(cap_len/4) .. seq_len - 1.
    want_scores: also return scores [B][cap], the block scores the selection
    ranked (NaN past each sequence's visible blocks).
    """
    q_idx_a = _f32(q_idx)
    k_pool_a = _f32(k_pool)
    B = q_idx_a.shape[0]
    pool_stride = k_pool_a.shape[1]
    seq = np.ascontiguousarray(seq_len, dtype=np.int32)
    cap = np.ascontiguousarray(cap_len, dtype=np.int32) if cap_len is not None else None
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    head_w_a = _f32(head_w) if head_w is not None else None
    q_a = _f32(q) if q is not None else None
    k_a = _f32(k) if k is not None else None
    v_a = _f32(v) if v is not None else None
    kv_stride = k_a.shape[1] if k_a is not None else 0
    sel = np.full((B, top_k), -1, np.int32)
    nsel = np.zeros(B, np.int32)
    kth = np.full(B, np.nan)
    nxt = np.full(B, np.nan)
    out = np.zeros((B, Hq, d)) if q is not None else None
    lse = np.zeros((B, Hq)) if q is not None else None
    scores, score_cap = None, 0
    if want_scores:
        rows_sel = cap if cap is not None else seq
        score_cap = max(1, int(max(int(x) for x in rows_sel)) // BLOCK) if B else 1
        scores = np.full((B, score_cap), np.nan)
    _L().oracle_decode(_p(q_idx_a), _p(k_pool_a), ctypes.c_int64(pool_stride), _p(head_w_a),
                       _p(q_a), _p(k_a), _p(v_a), ctypes.c_int64(kv_stride), _p(seq), _p(cap),
                       ctypes.c_int64(B), ctypes.c_int(int(relu)), ctypes.c_int(int(store_bf16)),
                       ctypes.c_int(top_k), ctypes.c_int(Hq), ctypes.c_int(Hkv), ctypes.c_int(d),
                       ctypes.c_double(scale), ctypes.c_double(base), ctypes.c_double(pos_scale),
                       ctypes.c_int(rotary_dim), _p(sel), _p(nsel), _p(kth), _p(nxt), _p(out),
                       _p(lse), _p(scores), ctypes.c_int64(score_cap), ctypes.c_int(nthreads or nthreads_default()))
    res = dict(sel=sel, nsel=nsel, kth=kth, next=nxt)
    if want_scores:
        res["scores"] = scores
    if q is not None:
        res.update(out=out, lse=lse)
    return res
