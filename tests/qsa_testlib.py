"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
(Python binding) and compare it with the CPU oracle.

Acceptance rules (fixed by the method's target):
  * pooled keys and block ids are compared bit-exactly;
  * a query row whose oracle k-th and (k+1)-th scores are closer than 1e-4
    (relative) may legitimately select differently: there the test checks
    that every block in the symmetric difference scores within 1e-4 of the
    oracle's k-th score, i.e. that the GPU selection is one of the valid ones;
  * attention output: max abs error <= 2e-2 in bf16, <= 1e-4 in fp32.
"""
from __future__ import annotations

import numpy as np
import torch

import block_sparse_attention_11_b200 as qsa
import oracle

GAP_REL = 1e-4
TOL = {"bf16": 2e-2, "fp32": 1e-4}


def np32(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy()


def rope_of(w) -> qsa.Rope:
    return qsa.Rope(base=w.rope_base, pos_scale=w.pos_scale, rotary_dim=128)


def gpu_prefill(x, w, T=None, top_k=None, flags=0, head_w=None, attn=True):
    """Pool, index and attend on the GPU; returns dict of device tensors."""
    q_idx, k_idx, q, k, v = x["q_idx"], x["k_idx"], x["q"], x["k"], x["v"]
    B, T0 = k_idx.shape[0], k_idx.shape[1]
    T = T or T0
    top_k = top_k or w.top_k
    dev = k_idx.device
    rope = rope_of(w)
    k_pool = torch.zeros(B, max(T // 4, 1), 128, dtype=k_idx.dtype, device=dev)
    qsa.qsa_pool_keys_prefill(k_idx, k_pool, rope=rope, flags=flags)
    sel = torch.full((B, T, top_k), -7, dtype=torch.int32, device=dev)
    nsel = torch.full((B, T), -7, dtype=torch.int32, device=dev)
    qsa.qsa_index_topk_prefill(q_idx, k_pool, sel, nsel, top_k=top_k, head_w=head_w, rope=rope, flags=flags)
    res = dict(k_pool=k_pool, sel=sel, nsel=nsel)
    if attn:
        out = torch.empty_like(q)
        lse = torch.empty(B, T, q.shape[2], dtype=torch.float32, device=dev)
        qsa.qsa_sparse_attn_prefill(q, k, v, sel, nsel, out, lse=lse)
        res.update(out=out, lse=lse)
    qsa.qsa_check_status()
    return res


def oracle_prefill(x, w, rows, b=0, top_k=None, flags=0, head_w=None, attn=True, k_pool=None, sel_in=None,
                   nsel_in=None):
    store_bf16 = w.dtype == "bf16"
    k_raw = np32(x["k_idx"][b])
    if k_pool is None:
        k_pool = oracle.pool_keys(k_raw, base=w.rope_base, pos_scale=w.pos_scale, rotary_dim=128,
                                  rmsnorm=bool(flags & qsa.QSA_POOL_RMSNORM), store_bf16=store_bf16)
    kw = dict(top_k=top_k or w.top_k, base=w.rope_base, pos_scale=w.pos_scale, rotary_dim=128,
              relu=bool(flags & qsa.QSA_SCORE_RELU), store_bf16=store_bf16, Hq=w.Hq, Hkv=w.Hkv, d=w.d)
    if sel_in is None:
        kw.update(q_idx=np32(x["q_idx"][b]), k_pool=k_pool,
                  head_w=None if head_w is None else head_w[b].cpu().numpy())
    else:
        kw.update(sel_in=sel_in, nsel_in=nsel_in)
    if attn:
        kw.update(q=np32(x["q"][b]), k=np32(x["k"][b]), v=np32(x["v"][b]))
    res = oracle.prefill_rows(rows, **kw)
    res["k_pool"] = k_pool
    return res


def selection_report(g_sel, g_nsel, ref, score_fn, rows):
    """Compare GPU and oracle selections row by row.

    Returns (exact_mask, overlap) and asserts the acceptance rule."""
    n = len(rows)
    assert np.array_equal(g_nsel, ref["nsel"]), "selection counts differ"
    exact = np.all(g_sel == ref["sel"], axis=1)
    overlap = []
    bad = np.nonzero(~exact)[0]
    if len(bad):
        scores = score_fn([rows[i] for i in bad])
        for j, i in enumerate(bad):
            ns = ref["nsel"][i]
            a = set(g_sel[i, :ns].tolist())
            o = set(ref["sel"][i, :ns].tolist())
            kth = ref["kth"][i]
            tol = GAP_REL * max(abs(kth), 1e-30)
            for blk in a ^ o:
                assert 0 <= blk < scores.shape[1], f"row {rows[i]}: block {blk} out of range"
                assert abs(scores[j, blk] - kth) <= tol, (
                    f"row {rows[i]}: block {blk} (score {scores[j, blk]}) differs from the oracle selection "
                    f"but is not within {GAP_REL} of the k-th score {kth}")
            assert np.all(np.diff(g_sel[i, :ns]) > 0), "selection not strictly ascending"
            assert np.all(g_sel[i, ns:] == -1), "padding is not -1"
            overlap.append(len(a & o) / max(ns, 1))
    return exact, (float(np.mean(overlap)) if overlap else 1.0), len(bad)


def check_prefill_workload(x, w, rows, top_k=None, flags=0, head_w=None, b=0, check_attn=True, gpu=None):
    """Full-pipeline parity on the listed rows of sequence b."""
    g = gpu or gpu_prefill(x, w, top_k=top_k, flags=flags, head_w=head_w)
    ref = oracle_prefill(x, w, rows, b=b, top_k=top_k, flags=flags, head_w=head_w, attn=check_attn)
    # pooled keys: bit-exact
    assert np.array_equal(np32(g["k_pool"][b])[: ref["k_pool"].shape[0]], ref["k_pool"]), "pooled keys differ"
    g_sel = g["sel"][b].cpu().numpy()[rows]
    g_nsel = g["nsel"][b].cpu().numpy()[rows]

    def score_fn(rr):
        kw = dict(q_idx=np32(x["q_idx"][b]), k_pool=ref["k_pool"], top_k=top_k or w.top_k,
                  base=w.rope_base, pos_scale=w.pos_scale, relu=bool(flags & qsa.QSA_SCORE_RELU),
                  store_bf16=w.dtype == "bf16",
                  head_w=None if head_w is None else head_w[b].cpu().numpy(), want_scores=True)
        return oracle.prefill_rows(rr, **kw)["scores"]

    exact, overlap, nbad = selection_report(g_sel, g_nsel, ref, score_fn, rows)
    err = 0.0
    if check_attn:
        go = np32(g["out"][b])[rows]
        diff = np.abs(go - ref["out"])[exact]
        err = float(diff.max()) if diff.size else 0.0
        assert err <= TOL[w.dtype], f"attention max abs error {err} > {TOL[w.dtype]}"
        gl = g["lse"][b].cpu().numpy()[rows][exact]
        lerr = float(np.abs(gl - ref["lse"][exact]).max()) if gl.size else 0.0
        assert lerr <= (1e-3 if w.dtype == "bf16" else 1e-4), f"lse error {lerr}"
    return dict(exact=exact, overlap=overlap, nbad=nbad, err=err, g=g, ref=ref)


def decode_selection_matches(g_sel, g_nsel, ref, i=0):
    """Compare one decode sequence's GPU selection with the oracle's (ref from
    oracle.decode(..., want_scores=True), sequence i of it).

    Returns True when the selections are equal.  Otherwise asserts the
    acceptance rule -- every block in the symmetric difference scores within
    GAP_REL of the oracle's k-th score, ids ascending, padding -1 -- and
    returns False (the caller then checks the attention on the oracle's
    selection instead)."""
    ns = int(ref["nsel"][i])
    assert int(g_nsel) == ns, f"selection count {int(g_nsel)} != oracle {ns}"
    o_sel = ref["sel"][i]
    if np.array_equal(g_sel, o_sel):
        return True
    scores = ref["scores"][i]
    kth = ref["kth"][i]
    tol = GAP_REL * max(abs(kth), 1e-30)
    a, o = set(g_sel[:ns].tolist()), set(o_sel[:ns].tolist())
    for blk in a ^ o:
        assert 0 <= blk < scores.shape[0] and np.isfinite(scores[blk]), f"block {blk} out of range"
        assert abs(scores[blk] - kth) <= tol, (
            f"block {blk} (score {scores[blk]}) differs from the oracle selection but is not within "
            f"{GAP_REL} of the k-th score {kth}")
    assert np.all(np.diff(g_sel[:ns]) > 0), "selection not strictly ascending"
    assert np.all(g_sel[ns:] == -1), "padding is not -1"
    return False


def stage_isolated_decode(refs, attn_fn, B, top_k, tol, lse_tol=None):
    """For the decode sequences whose selection differed (refs: {b: oracle
    result of that sequence}), run the GPU attention of the whole batch on
    the oracle's selections (attn_fn(sel, nsel) -> (out, lse or None), device
    tensors) and compare those sequences with the oracle's attention."""
    if not refs:
        return
    dev = "cuda"
    sel = torch.full((B, top_k), -1, dtype=torch.int32)
    nsel = torch.zeros(B, dtype=torch.int32)
    for b, r in refs.items():
        sel[b] = torch.from_numpy(r["sel"][0])
        nsel[b] = int(r["nsel"][0])
    out, lse = attn_fn(sel.to(dev), nsel.to(dev))
    qsa.qsa_check_status()
    for b, r in refs.items():
        err = float(np.abs(np32(out[b]) - r["out"][0]).max())
        assert err <= tol, f"seq {b}: attention on the oracle's selection, error {err}"
        if lse is not None and lse_tol is not None:
            assert float(np.abs(lse[b].cpu().numpy() - r["lse"][0]).max()) <= lse_tol
