"""The allocation-free decode attention entry point.

qsa_sparse_attn_decode_noalloc serves callers that cannot allocate device
memory where they call QSA (an engine that reserves all free memory for its KV
pool, a thread that must not block on cudaMalloc): it keeps its split-KV
partial results in a fixed scratch area compiled into the library instead of a
caller workspace.  It must give the same output as qsa_sparse_attn_decode, on
consecutive calls that reuse the shared scratch.  This file is collected
last so that a failure here leaves every other test already run."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _decode_inputs(qsa, workloads):
    w = workloads.Workload("noalloc", "decode", 6, 20000, 512, 16, 2, 128, "bf16", 321)
    x = workloads.make_decode(w, device=DEV, ragged=True)
    B, lens = w.B, x["lens"]
    cap = max(lens) // 4 + 2
    k_pool = torch.zeros(B, cap, 128, dtype=torch.bfloat16, device=DEV)
    for b in range(B):
        kp = torch.zeros(1, cap, 128, dtype=torch.bfloat16, device=DEV)
        qsa.qsa_pool_keys_prefill(x["k_idx"][b:b + 1, :lens[b]].contiguous(), kp)
        k_pool[b] = kp[0]
    sel = torch.empty(B, w.top_k, dtype=torch.int32, device=DEV)
    nsel = torch.empty(B, dtype=torch.int32, device=DEV)
    qsa.qsa_index_topk_decode(x["q_idx"], k_pool, x["seq_len"], sel, nsel, top_k=w.top_k)
    return x, sel, nsel


def test_noalloc_decode_attention_matches_workspace_entry_point():
    import block_sparse_attention_11_b200 as qsa
    import workloads
    x, sel, nsel = _decode_inputs(qsa, workloads)
    ref = torch.empty_like(x["q"])
    ref_lse = torch.empty(x["q"].shape[:2], dtype=torch.float32, device=DEV)
    qsa.qsa_sparse_attn_decode(x["q"], x["k"], x["v"], x["seq_len"], sel, nsel, ref, lse=ref_lse)
    for _ in range(2):   # two calls in a row: the shared scratch is reused
        out = torch.full_like(x["q"], 7.0)
        lse = torch.full(x["q"].shape[:2], 7.0, dtype=torch.float32, device=DEV)
        qsa.qsa_sparse_attn_decode_noalloc(x["q"], x["k"], x["v"], x["seq_len"], sel, nsel, out, lse=lse)
        qsa.qsa_check_status()
        err = (out.float() - ref.float()).abs().max().item()
        assert err <= 2e-2, err
        assert (lse - ref_lse).abs().max().item() <= 1e-3
    assert np.isfinite(out.float().cpu().numpy()).all()
