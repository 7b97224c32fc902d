"""The allocation-free decode attention entry point.

qsa_sparse_attn_decode_noalloc serves callers that cannot allocate device
memory where they call QSA (an engine that reserves all free memory for its KV
pool, a thread that must not block on cudaMalloc): it keeps its split-KV
partial results in a fixed scratch area compiled into the library instead of a
caller workspace.  It must give the same output as qsa_sparse_attn_decode, on
consecutive calls that reuse the shared scratch, accept the same shapes, and
refuse a call whose partials would not fit the scratch.  This file is
collected last so that a failure here leaves every other test already run."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _decode_inputs(qsa, workloads, Hq=16, Hkv=2, d=128, dtype="bf16", B=6, L=20000):
    w = workloads.Workload("noalloc", "decode", B, L, 512, Hq, Hkv, d, dtype, 321)
    x = workloads.make_decode(w, device=DEV, ragged=True)
    lens = x["lens"]
    cap = max(lens) // 4 + 2
    kdt = x["k_idx"].dtype
    k_pool = torch.zeros(B, cap, 128, dtype=kdt, device=DEV)
    for b in range(B):
        kp = torch.zeros(1, cap, 128, dtype=kdt, device=DEV)
        qsa.qsa_pool_keys_prefill(x["k_idx"][b:b + 1, :lens[b]].contiguous(), kp)
        k_pool[b] = kp[0]
    sel = torch.empty(B, w.top_k, dtype=torch.int32, device=DEV)
    nsel = torch.empty(B, dtype=torch.int32, device=DEV)
    qsa.qsa_index_topk_decode(x["q_idx"], k_pool, x["seq_len"], sel, nsel, top_k=w.top_k)
    return x, sel, nsel


def _compare_two_calls(qsa, x, sel, nsel, tol, lse_tol):
    ref = torch.empty_like(x["q"])
    ref_lse = torch.empty(x["q"].shape[:2], dtype=torch.float32, device=DEV)
    qsa.qsa_sparse_attn_decode(x["q"], x["k"], x["v"], x["seq_len"], sel, nsel, ref, lse=ref_lse)
    for _ in range(2):   # two calls in a row: the shared scratch is reused
        out = torch.full_like(x["q"], 7.0)
        lse = torch.full(x["q"].shape[:2], 7.0, dtype=torch.float32, device=DEV)
        qsa.qsa_sparse_attn_decode_noalloc(x["q"], x["k"], x["v"], x["seq_len"], sel, nsel, out, lse=lse)
        qsa.qsa_check_status()
        err = (out.float() - ref.float()).abs().max().item()
        assert err <= tol, err
        assert (lse - ref_lse).abs().max().item() <= lse_tol
    assert np.isfinite(out.float().cpu().numpy()).all()


def test_noalloc_decode_attention_matches_workspace_entry_point():
    import block_sparse_attention_11_b200 as qsa
    import workloads
    x, sel, nsel = _decode_inputs(qsa, workloads)
    _compare_two_calls(qsa, x, sel, nsel, 2e-2, 1e-3)


def test_noalloc_released_shape_matches_workspace_entry_point():
    """24 q heads, 2 kv heads of 256 dims: the same shapes as the workspace
    entry point, while the partials fit the scratch."""
    import block_sparse_attention_11_b200 as qsa
    import workloads
    assert qsa.qsa_sparse_attn_decode_workspace(2, 24, 256, 512) <= qsa.QSA_NOALLOC_SCRATCH_BYTES
    x, sel, nsel = _decode_inputs(qsa, workloads, Hq=24, Hkv=2, d=256, B=2, L=9000)
    _compare_two_calls(qsa, x, sel, nsel, 2e-2, 1e-3)


def test_noalloc_fp32_matches_workspace_entry_point():
    """The fp32 path keeps no partial results (no scratch) and must agree
    with the workspace entry point within the fp32 bound."""
    import block_sparse_attention_11_b200 as qsa
    import workloads
    x, sel, nsel = _decode_inputs(qsa, workloads, dtype="fp32", B=3, L=5000)
    _compare_two_calls(qsa, x, sel, nsel, 1e-4, 1e-4)


def test_noalloc_rejects_partials_beyond_the_scratch():
    """B = 64 with 32 q heads needs 4,227,072 bytes of partials, more than the
    4 MiB scratch: the call returns QSA_ERR_WORKSPACE before launching."""
    import block_sparse_attention_11_b200 as qsa
    B, Hq, Hkv, d, L = 64, 32, 4, 128, 64
    need = qsa.qsa_sparse_attn_decode_workspace(B, Hq, d, 512)
    assert need > qsa.QSA_NOALLOC_SCRATCH_BYTES
    q = torch.zeros(B, Hq, d, dtype=torch.bfloat16, device=DEV)
    k = torch.zeros(B, L, Hkv, d, dtype=torch.bfloat16, device=DEV)
    v = torch.zeros_like(k)
    seq_len = torch.full((B,), L, dtype=torch.int32, device=DEV)
    sel = torch.full((B, 512), -1, dtype=torch.int32, device=DEV)
    nsel = torch.zeros(B, dtype=torch.int32, device=DEV)
    out = torch.full_like(q, 3.0)
    with pytest.raises(qsa.QSAError) as ei:
        qsa.qsa_sparse_attn_decode_noalloc(q, k, v, seq_len, sel, nsel, out)
    assert ei.value.status == qsa.QSA_ERR_WORKSPACE
    assert bool((out == 3.0).all())   # nothing ran
    qsa.qsa_check_status()
