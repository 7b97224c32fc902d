"""Stage-by-stage GPU parity against the CPU oracle on sizes the oracle
finishes in seconds (several tiles plus a ragged tail), plus edge cases.

Each stage is fed the same inputs as the oracle's stage: the GPU attention
runs on the oracle's selection, so a tie decided differently upstream can
neither hide nor fake an attention error."""
import numpy as np
import pytest
import torch

import workloads
from qsa_testlib import (TOL, check_prefill_workload, decode_selection_matches, np32, rope_of,
                         selection_report, stage_isolated_decode)

pytestmark = pytest.mark.gpu

import oracle  # noqa: E402


@pytest.fixture(scope="module")
def qsa():
    import block_sparse_attention_11_b200 as m
    assert torch.cuda.is_available()
    return m


DEV = "cuda"


def W(T, top_k=64, Hq=16, Hkv=2, dtype="bf16", seed=11, **kw):
    return workloads.Workload(f"t{T}", "prefill", kw.pop("B", 1), T, top_k, Hq, Hkv, 128, dtype, seed, **kw)


# ----------------------------------------------------------------------------- pooling

@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("n_tok,pos0,R,ps,flags", [(4099, 0, 128, 1.0, 0), (1000, 4 * 12345, 128, 1.0, 0),
                                                  (4096, 1 << 20, 128, 4.0, 0), (515, 0, 64, 1.0, 0),
                                                  (512, 8, 128, 1.0, 2)])
def test_pool_prefill_bit_exact(qsa, dtype, n_tok, pos0, R, ps, flags):
    g = torch.Generator(device=DEV).manual_seed(n_tok + pos0)
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    k_raw = torch.randn(2, n_tok, 128, generator=g, device=DEV).to(dt)
    cap = pos0 // 4 + n_tok // 4 + 3
    k_pool = torch.full((2, cap, 128), 7.0, dtype=dt, device=DEV)
    rope = qsa.Rope(pos_scale=ps, rotary_dim=R)
    qsa.qsa_pool_keys_prefill(k_raw, k_pool, pos0=pos0, rope=rope, flags=flags)
    qsa.qsa_check_status()
    for b in range(2):
        ref = oracle.pool_keys(np32(k_raw[b]), pos0=pos0, pos_scale=ps, rotary_dim=R, rmsnorm=bool(flags & 2),
                               store_bf16=dtype == "bf16")
        got = np32(k_pool[b])
        assert np.array_equal(got[pos0 // 4: pos0 // 4 + n_tok // 4], ref)
        assert np.all(got[: pos0 // 4] == 7.0) and np.all(got[pos0 // 4 + n_tok // 4:] == 7.0)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_pool_decode_ring_matches_oracle(qsa, dtype):
    B, steps = 5, 23
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    g = torch.Generator(device=DEV).manual_seed(3)
    start = torch.tensor([0, 1, 2, 3, 101], dtype=torch.int32)
    keys = torch.randn(B, steps, 128, generator=g, device=DEV).to(dt)
    ring = torch.zeros(B, 4, 128, dtype=dt, device=DEV)
    cap = (int(start.max()) + steps) // 4 + 1
    k_pool = torch.zeros(B, cap, 128, dtype=dt, device=DEV)
    o_ring = np.zeros((B, 4, 128), np.float32)
    o_pool = np.zeros((B, cap, 128), np.float32)
    rope = qsa.Rope(pos_scale=4.0)
    for s in range(steps):
        seq_len = (start + s + 1).to(DEV)
        qsa.qsa_pool_keys_decode(keys[:, s].contiguous(), ring, k_pool, seq_len, rope=rope)
        kn = np32(keys[:, s])
        for b in range(B):
            oracle.pool_decode(kn[b], o_ring[b], o_pool[b], int(start[b]) + s + 1, pos_scale=4.0,
                               store_bf16=dtype == "bf16")
    qsa.qsa_check_status()
    assert np.array_equal(np32(ring), o_ring)
    assert np.array_equal(np32(k_pool), o_pool)


@pytest.mark.parametrize("n_tok,pos0,amp,flags", [(4099, 0, 1.0, 0), (1000, 4 * 12345, 300.0, 0),
                                                  (515, 8, 1.0, 2), (2048, 1 << 20, 0.01, 0)])
def test_pool_prefill_fp8_bit_exact(qsa, n_tok, pos0, amp, flags):
    """FP8 E4M3 compressed keys: bit-exact against the oracle's rounding of
    the exact rotated mean, including saturation (amp 300: rotated values
    beyond 448) and subnormals (amp 0.01)."""
    g = torch.Generator(device=DEV).manual_seed(n_tok + pos0 + 1)
    k_raw = (torch.randn(2, n_tok, 128, generator=g, device=DEV) * amp).to(torch.bfloat16)
    cap = pos0 // 4 + n_tok // 4 + 3
    k_pool = torch.full((2, cap, 128), 7.0, device=DEV).to(torch.float8_e4m3fn)
    rope = qsa.Rope(pos_scale=2.0)
    qsa.qsa_pool_keys_prefill(k_raw, k_pool, pos0=pos0, rope=rope, flags=flags | qsa.QSA_KEYS_FP8)
    qsa.qsa_check_status()
    for b in range(2):
        ref = oracle.pool_keys(np32(k_raw[b]), pos0=pos0, pos_scale=2.0, rmsnorm=bool(flags & 2), store_fp8=True)
        got = np32(k_pool[b])
        assert np.array_equal(got[pos0 // 4: pos0 // 4 + n_tok // 4], ref)
        assert np.all(got[: pos0 // 4] == 7.0) and np.all(got[pos0 // 4 + n_tok // 4:] == 7.0)
    if amp > 100:
        assert np.abs(np32(k_pool)).max() == 448.0


def test_pool_decode_ring_fp8_matches_oracle(qsa):
    B, steps = 5, 23
    g = torch.Generator(device=DEV).manual_seed(4)
    start = torch.tensor([0, 1, 2, 3, 101], dtype=torch.int32)
    keys = (torch.randn(B, steps, 128, generator=g, device=DEV) * 60).to(torch.bfloat16)
    ring = torch.zeros(B, 4, 128, dtype=torch.bfloat16, device=DEV)
    cap = (int(start.max()) + steps) // 4 + 1
    k_pool = torch.zeros(B, cap, 128, device=DEV).to(torch.float8_e4m3fn)
    o_ring = np.zeros((B, 4, 128), np.float32)
    o_pool = np.zeros((B, cap, 128), np.float32)
    for s in range(steps):
        seq_len = (start + s + 1).to(DEV)
        qsa.qsa_pool_keys_decode(keys[:, s].contiguous(), ring, k_pool, seq_len, flags=qsa.QSA_KEYS_FP8)
        kn = np32(keys[:, s])
        for b in range(B):
            oracle.pool_decode(kn[b], o_ring[b], o_pool[b], int(start[b]) + s + 1, store_fp8=True)
    qsa.qsa_check_status()
    assert np.array_equal(np32(ring), o_ring)
    assert np.array_equal(np32(k_pool), o_pool)


def test_rope_apply_matches_oracle(qsa):
    g = torch.Generator(device=DEV).manual_seed(5)
    x = torch.randn(2, 300, 3, 128, generator=g, device=DEV).to(torch.bfloat16)
    ref_in = np32(x)
    qsa.qsa_rope_apply(x, pos0=77, rope=qsa.Rope(rotary_dim=64))
    got = np32(x)
    for b in range(2):
        for h in range(3):
            rot = oracle.rope_rows(ref_in[b, :, h], np.arange(77, 377), rotary_dim=64)
            exp = np.vectorize(oracle.round_bf16)(rot)
            assert np.array_equal(got[b, :, h], exp.astype(np.float32))


# ----------------------------------------------------------------------------- prefill indexer + attention

@pytest.mark.parametrize("T,top_k,flags,weights,dtype", [
    (4099, 64, 0, False, "bf16"),      # hi/lo tensor-core path, ragged tail, many tiles
    (4099, 512, 0, False, "bf16"),     # top-512: nb < k for the first 2048 rows
    (2315, 64, 1, False, "bf16"),      # ReLU: per-head tensor-core path
    (2315, 64, 0, True, "bf16"),       # head weights: per-head path
    (1024, 64, 0, False, "fp32"),      # fp32 SIMT path (tiny workload shape)
    (1031, 64, 1, True, "fp32"),
    (7, 4, 0, False, "bf16"),          # fewer than one tile, rows with 0 and 1 blocks
    (1, 4, 0, False, "bf16"),          # single token: attends to itself
])
def test_prefill_pipeline(qsa, T, top_k, flags, weights, dtype):
    w = W(T, top_k=top_k, dtype=dtype, Hq=8 if dtype == "fp32" else 16, Hkv=1 if dtype == "fp32" else 2)
    x = workloads.make_prefill(w, device=DEV)
    head_w = None
    if weights:
        head_w = torch.rand(1, T, 4, generator=torch.Generator(device=DEV).manual_seed(9), device=DEV) * 2
    rows = list(range(T))
    r = check_prefill_workload(x, w, rows, top_k=top_k, flags=flags, head_w=head_w)
    assert r["nbad"] <= max(2, T // 200), f"too many near-tie rows: {r['nbad']}"


def test_prefill_batched_and_chunked(qsa):
    """B = 2 sequences; and chunked prefill (pooling and queries in chunks
    against the growing cache) gives the same selections as one shot."""
    w = W(3000, top_k=128, B=2, seed=21)
    x = workloads.make_prefill(w, device=DEV)
    g = check_prefill_workload(x, w, list(range(0, 3000, 7)), b=1)["g"]
    rope = rope_of(w)
    k_pool = torch.zeros(2, 750, 128, dtype=torch.bfloat16, device=DEV)
    sel = torch.empty(2, 3000, 128, dtype=torch.int32, device=DEV)
    nsel = torch.empty(2, 3000, dtype=torch.int32, device=DEV)
    out = torch.empty_like(x["q"])
    for c0, c1 in [(0, 1024), (1024, 2048), (2048, 3000)]:
        qsa.qsa_pool_keys_prefill(x["k_idx"][:, c0:c1].contiguous(), k_pool, pos0=c0, rope=rope)
        s = torch.empty(2, c1 - c0, 128, dtype=torch.int32, device=DEV)
        n = torch.empty(2, c1 - c0, dtype=torch.int32, device=DEV)
        qsa.qsa_index_topk_prefill(x["q_idx"][:, c0:c1].contiguous(), k_pool, s, n, q0=c0, top_k=128, rope=rope)
        o = torch.empty(2, c1 - c0, 16, 128, dtype=torch.bfloat16, device=DEV)
        qsa.qsa_sparse_attn_prefill(x["q"][:, c0:c1].contiguous(), x["k"], x["v"], s, n, o, q0=c0)
        sel[:, c0:c1] = s
        nsel[:, c0:c1] = n
        out[:, c0:c1] = o
    qsa.qsa_check_status()
    assert torch.equal(k_pool, g["k_pool"])
    assert torch.equal(sel, g["sel"]) and torch.equal(nsel, g["nsel"])
    assert torch.equal(out, g["out"])


def test_attention_stage_isolated_on_oracle_selection(qsa):
    """GPU attention fed the oracle's selection, compared with the oracle's attention."""
    for dtype, Hq, Hkv in [("bf16", 16, 2), ("bf16", 8, 1), ("bf16", 32, 4), ("fp32", 8, 1), ("fp32", 12, 4)]:
        w = W(2500, top_k=96, Hq=Hq, Hkv=Hkv, dtype=dtype, seed=33)
        x = workloads.make_prefill(w, device=DEV)
        rows = list(range(2500))
        kp = oracle.pool_keys(np32(x["k_idx"][0]), store_bf16=dtype == "bf16")
        ref = oracle.prefill_rows(rows, q_idx=np32(x["q_idx"][0]), k_pool=kp, top_k=96,
                                  store_bf16=dtype == "bf16", q=np32(x["q"][0]), k=np32(x["k"][0]),
                                  v=np32(x["v"][0]), Hq=Hq, Hkv=Hkv, d=128)
        sel = torch.from_numpy(ref["sel"][None]).to(DEV)
        nsel = torch.from_numpy(ref["nsel"][None]).to(DEV)
        out = torch.empty_like(x["q"])
        lse = torch.empty(1, 2500, Hq, dtype=torch.float32, device=DEV)
        qsa.qsa_sparse_attn_prefill(x["q"], x["k"], x["v"], sel, nsel, out, lse=lse)
        qsa.qsa_check_status()
        err = np.abs(np32(out[0]) - ref["out"]).max()
        assert err <= TOL[dtype], (dtype, Hq, Hkv, err)
        assert np.abs(lse[0].cpu().numpy() - ref["lse"]).max() <= (1e-3 if dtype == "bf16" else 1e-4)


def _to_e4m3(t):
    """Per-tensor FP8 E4M3 cache of t (scale = amax / 448) and its scale."""
    scale = float(t.float().abs().max()) / 448.0
    return (t.float() / scale).to(torch.float8_e4m3fn), scale


@pytest.mark.parametrize("Hq,Hkv,T,top_k", [(16, 2, 2500, 96), (8, 1, 1031, 64), (32, 4, 777, 32), (16, 2, 7, 4)])
def test_attention_fp8_kv_prefill_on_oracle_selection(qsa, Hq, Hkv, T, top_k):
    """FP8 E4M3 K/V caches (per-tensor scales): the GPU attention on the
    oracle's selection equals the oracle's attention over the dequantized
    K/V within the BF16 tolerance."""
    w = W(T, top_k=top_k, Hq=Hq, Hkv=Hkv, seed=34 + Hq)
    x = workloads.make_prefill(w, device=DEV)
    k8, ks = _to_e4m3(x["k"])
    v8, vs = _to_e4m3(x["v"])
    kd = k8.float() * ks
    vd = v8.float() * vs
    rows = list(range(T))
    kp = oracle.pool_keys(np32(x["k_idx"][0]))
    ref = oracle.prefill_rows(rows, q_idx=np32(x["q_idx"][0]), k_pool=kp, top_k=top_k, q=np32(x["q"][0]),
                              k=kd[0].cpu().numpy(), v=vd[0].cpu().numpy(), Hq=Hq, Hkv=Hkv, d=128)
    sel = torch.from_numpy(ref["sel"][None]).to(DEV)
    nsel = torch.from_numpy(ref["nsel"][None]).to(DEV)
    out = torch.empty_like(x["q"])
    lse = torch.empty(1, T, Hq, dtype=torch.float32, device=DEV)
    qsa.qsa_sparse_attn_prefill_kv8(x["q"], k8, v8, ks, vs, sel, nsel, out, lse=lse)
    qsa.qsa_check_status()
    err = np.abs(np32(out[0]) - ref["out"]).max()
    assert err <= TOL["bf16"], err
    assert np.abs(lse[0].cpu().numpy() - ref["lse"]).max() <= 1e-3


@pytest.mark.parametrize("B,L", [(6, 20000), (3, 70001), (5, 2)])
def test_attention_fp8_kv_decode(qsa, B, L):
    """Decode attention over FP8 K/V caches against the oracle's decode step
    on the dequantized caches (same compressed keys, so the same selection)."""
    w = workloads.Workload("dec_kv8", "decode", B, L, 256, 16, 2, 128, "bf16", 80)
    x = workloads.make_decode(w, device=DEV, ragged=True)
    rope = rope_of(w)
    lens = x["lens"]
    k8, ks = _to_e4m3(x["k"])
    v8, vs = _to_e4m3(x["v"])
    cap = max(lens) // 4 + 2
    k_pool = torch.zeros(B, cap, 128, dtype=torch.bfloat16, device=DEV)
    sel = torch.empty(B, w.top_k, dtype=torch.int32, device=DEV)
    nsel = torch.empty(B, dtype=torch.int32, device=DEV)
    # compressed keys of all L + 1 keys (the new token's block included) by prefill pooling
    for b in range(B):
        kp = torch.zeros(1, cap, 128, dtype=torch.bfloat16, device=DEV)
        full = torch.cat([x["k_idx"][b, :lens[b]], x["k_idx_new"][b:b + 1]], 0)[None].contiguous()
        qsa.qsa_pool_keys_prefill(full, kp, rope=rope)
        k_pool[b] = kp[0]
    qsa.qsa_index_topk_decode(x["q_idx"], k_pool, x["seq_len"], sel, nsel, top_k=w.top_k, rope=rope)
    out = torch.empty_like(x["q"])
    lse = torch.empty(B, 16, dtype=torch.float32, device=DEV)
    qsa.qsa_sparse_attn_decode_kv8(x["q"], k8, v8, ks, vs, x["seq_len"], sel, nsel, out, lse=lse)
    qsa.qsa_check_status()
    kd, vd = k8.float() * ks, v8.float() * vs
    differ = {}
    for b in range(B):
        s = lens[b] + 1
        ref = oracle.decode(np32(x["q_idx"][b:b + 1]), np32(k_pool[b])[None], [s], q=np32(x["q"][b:b + 1]),
                            k=kd[b:b + 1].cpu().numpy(), v=vd[b:b + 1].cpu().numpy(), top_k=w.top_k,
                            want_scores=True)
        if not decode_selection_matches(sel[b].cpu().numpy(), nsel[b], ref):
            differ[b] = ref
            continue
        assert np.abs(np32(out[b]) - ref["out"][0]).max() <= TOL["bf16"], b
        assert np.abs(lse[b].cpu().numpy() - ref["lse"][0]).max() <= 1e-3

    def attn_on(s_, n_):
        o_ = torch.empty_like(x["q"])
        l_ = torch.empty(B, 16, dtype=torch.float32, device=DEV)
        qsa.qsa_sparse_attn_decode_kv8(x["q"], k8, v8, ks, vs, x["seq_len"], s_, n_, o_, lse=l_)
        return o_, l_

    stage_isolated_decode(differ, attn_on, B, w.top_k, TOL["bf16"], 1e-3)


@pytest.mark.parametrize("T,top_k,kv8", [(2500, 96, False), (2500, 96, True), (7, 4, False), (1031, 512, False)])
def test_attention_released_shape_prefill(qsa, T, top_k, kv8):
    """The released 24q / 2kv, d = 256 shape (two 8-head column tiles per kv
    head, the second half padding) on the oracle's selection, BF16 or FP8 K/V."""
    w = workloads.Workload(f"t{T}", "prefill", 1, T, top_k, 24, 2, 256, "bf16", 35)
    x = workloads.make_prefill(w, device=DEV)
    k, v = x["k"], x["v"]
    ks = vs = 1.0
    if kv8:
        k, ks = _to_e4m3(x["k"])
        v, vs = _to_e4m3(x["v"])
    kd = k.float() * ks
    vd = v.float() * vs
    rows = list(range(T))
    kp = oracle.pool_keys(np32(x["k_idx"][0]))
    ref = oracle.prefill_rows(rows, q_idx=np32(x["q_idx"][0]), k_pool=kp, top_k=top_k, q=np32(x["q"][0]),
                              k=kd[0].cpu().numpy(), v=vd[0].cpu().numpy(), Hq=24, Hkv=2, d=256)
    sel = torch.from_numpy(ref["sel"][None]).to(DEV)
    nsel = torch.from_numpy(ref["nsel"][None]).to(DEV)
    out = torch.full_like(x["q"], 7.0)
    lse = torch.empty(1, T, 24, dtype=torch.float32, device=DEV)
    if kv8:
        qsa.qsa_sparse_attn_prefill_kv8(x["q"], k, v, ks, vs, sel, nsel, out, lse=lse)
    else:
        qsa.qsa_sparse_attn_prefill(x["q"], k, v, sel, nsel, out, lse=lse)
    qsa.qsa_check_status()
    err = np.abs(np32(out[0]) - ref["out"]).max()
    assert err <= TOL["bf16"], err
    assert np.abs(lse[0].cpu().numpy() - ref["lse"]).max() <= 1e-3


@pytest.mark.parametrize("B,L,kv8", [(6, 20000, False), (3, 70001, True), (5, 2, False)])
def test_attention_released_shape_decode(qsa, B, L, kv8):
    """Decode attention with the released 24q / 2kv, d = 256 shape against the
    oracle's decode step (selection and attention), and the dense decode
    baseline against textbook attention."""
    w = workloads.Workload("dec_rel", "decode", B, L, 256, 24, 2, 256, "bf16", 81)
    x = workloads.make_decode(w, device=DEV, ragged=True)
    rope = rope_of(w)
    lens = x["lens"]
    k, v = x["k"], x["v"]
    ks = vs = 1.0
    if kv8:
        k, ks = _to_e4m3(x["k"])
        v, vs = _to_e4m3(x["v"])
    cap = max(lens) // 4 + 2
    k_pool = torch.zeros(B, cap, 128, dtype=torch.bfloat16, device=DEV)
    for b in range(B):
        kp = torch.zeros(1, cap, 128, dtype=torch.bfloat16, device=DEV)
        full = torch.cat([x["k_idx"][b, :lens[b]], x["k_idx_new"][b:b + 1]], 0)[None].contiguous()
        qsa.qsa_pool_keys_prefill(full, kp, rope=rope)
        k_pool[b] = kp[0]
    sel = torch.empty(B, w.top_k, dtype=torch.int32, device=DEV)
    nsel = torch.empty(B, dtype=torch.int32, device=DEV)
    qsa.qsa_index_topk_decode(x["q_idx"], k_pool, x["seq_len"], sel, nsel, top_k=w.top_k, rope=rope)
    out = torch.empty_like(x["q"])
    lse = torch.empty(B, 24, dtype=torch.float32, device=DEV)
    if kv8:
        qsa.qsa_sparse_attn_decode_kv8(x["q"], k, v, ks, vs, x["seq_len"], sel, nsel, out, lse=lse)
    else:
        qsa.qsa_sparse_attn_decode(x["q"], k, v, x["seq_len"], sel, nsel, out, lse=lse)
    qsa.qsa_check_status()
    kd, vd = k.float() * ks, v.float() * vs
    differ = {}
    for b in range(B):
        s = lens[b] + 1
        ref = oracle.decode(np32(x["q_idx"][b:b + 1]), np32(k_pool[b])[None], [s], q=np32(x["q"][b:b + 1]),
                            k=kd[b:b + 1].cpu().numpy(), v=vd[b:b + 1].cpu().numpy(), top_k=w.top_k,
                            Hq=24, Hkv=2, d=256, want_scores=True)
        if not decode_selection_matches(sel[b].cpu().numpy(), nsel[b], ref):
            differ[b] = ref
            continue
        assert np.abs(np32(out[b]) - ref["out"][0]).max() <= TOL["bf16"], b
        assert np.abs(lse[b].cpu().numpy() - ref["lse"][0]).max() <= 1e-3

    def attn_on(s_, n_):
        o_ = torch.empty_like(x["q"])
        l_ = torch.empty(B, 24, dtype=torch.float32, device=DEV)
        if kv8:
            qsa.qsa_sparse_attn_decode_kv8(x["q"], k, v, ks, vs, x["seq_len"], s_, n_, o_, lse=l_)
        else:
            qsa.qsa_sparse_attn_decode(x["q"], k, v, x["seq_len"], s_, n_, o_, lse=l_)
        return o_, l_

    stage_isolated_decode(differ, attn_on, B, w.top_k, TOL["bf16"], 1e-3)
    if not kv8:
        outd = torch.empty_like(x["q"])
        qsa.qsa_dense_attn_decode(x["q"], x["k"], x["v"], x["seq_len"], outd)
        qsa.qsa_check_status()
        for b in range(min(B, 2)):
            t = lens[b]
            refd = oracle.dense_rows([0], q=np32(x["q"][b])[None], k=np32(x["k"][b]), v=np32(x["v"][b]), Hq=24,
                                     Hkv=2, d=256, q0=t)
            assert np.abs(np32(outd[b]) - refd[0]).max() <= TOL["bf16"], b


@pytest.mark.parametrize("Hq,Hkv,T,q0,B", [(16, 2, 1000, 0, 1), (8, 1, 333, 0, 2), (32, 4, 200, 0, 1),
                                          (16, 2, 700, 600, 1), (16, 2, 5, 0, 1)])
def test_dense_prefill_matches_textbook_attention(qsa, Hq, Hkv, T, q0, B):
    """Full causal prefill attention (the dense baseline) against textbook
    attention over positions 0..t on every row; q0 > 0: a chunk of rows after
    a cached prefix."""
    g = torch.Generator(device=DEV).manual_seed(T + q0 + Hq)
    L = q0 + T + 3
    q = torch.randn(B, T, Hq, 128, generator=g, device=DEV).to(torch.bfloat16)
    k = torch.randn(B, L, Hkv, 128, generator=g, device=DEV).to(torch.bfloat16)
    v = torch.randn(B, L, Hkv, 128, generator=g, device=DEV).to(torch.bfloat16)
    out = torch.full_like(q, 9.0)
    lse = torch.empty(B, T, Hq, dtype=torch.float32, device=DEV)
    qsa.qsa_dense_attn_prefill(q, k, v, out, q0=q0, lse=lse)
    qsa.qsa_check_status()
    rows = list(range(T))
    for b in range(B):
        ref = oracle.dense_rows(rows, q=np32(q[b]), k=np32(k[b]), v=np32(v[b]), Hq=Hq, Hkv=Hkv, d=128, q0=q0)
        assert np.abs(np32(out[b]) - ref).max() <= TOL["bf16"], b


@pytest.mark.parametrize("q0", [262100, 262130, 1048000])
def test_prefill_chunk_beyond_65535_blocks_all_ties(qsa, q0):
    """Chunked prefill rows near and beyond position 262143, from which a row
    scores more than 65535 blocks: the cache's indexer keys are zero except
    300 planted blocks, so nearly every block scores exactly 0 and falls in
    one histogram bin of the row select (ties go to the lower block id).
    Selections (bit-exact) and attention against the oracle.  Chunk 262100
    ends at 65533 blocks per row, chunk 262130 crosses the line, chunk
    1048000 sits at a 1M-token context."""
    n_q = 32
    L = q0 + n_q
    g = torch.Generator(device=DEV).manual_seed(q0)
    k_idx = torch.zeros(1, L, 128, device=DEV)
    planted = torch.randperm(L // 4, generator=g, device=DEV)[:300]
    tok = (4 * planted[:, None] + torch.arange(4, device=DEV)).reshape(-1)
    k_idx[0, tok] = 3 * torch.randn(tok.numel(), 128, generator=g, device=DEV)
    k_idx = k_idx.to(torch.bfloat16)
    q_idx = torch.randn(1, n_q, 4, 128, generator=g, device=DEV).to(torch.bfloat16)
    q = torch.randn(1, n_q, 16, 128, generator=g, device=DEV).to(torch.bfloat16)
    k = torch.randn(1, L, 2, 128, generator=g, device=DEV).to(torch.bfloat16)
    v = torch.randn(1, L, 2, 128, generator=g, device=DEV).to(torch.bfloat16)
    rope = qsa.Rope()
    k_pool = torch.zeros(1, L // 4, 128, dtype=torch.bfloat16, device=DEV)
    qsa.qsa_pool_keys_prefill(k_idx, k_pool, rope=rope)
    sel = torch.full((1, n_q, 512), -7, dtype=torch.int32, device=DEV)
    nsel = torch.full((1, n_q), -7, dtype=torch.int32, device=DEV)
    qsa.qsa_index_topk_prefill(q_idx, k_pool, sel, nsel, q0=q0, top_k=512, rope=rope)
    out = torch.empty_like(q)
    qsa.qsa_sparse_attn_prefill(q, k, v, sel, nsel, out, q0=q0)
    qsa.qsa_check_status()
    kp = oracle.pool_keys(np32(k_idx[0]), store_bf16=True)
    assert np.array_equal(np32(k_pool[0]), kp)
    rows = [0, 5, 11, 18, 31]
    ref = oracle.prefill_rows(rows, q_idx=np32(q_idx[0]), k_pool=kp, top_k=512, store_bf16=True, q=np32(q[0]),
                              k=np32(k[0]), v=np32(v[0]), Hq=16, Hkv=2, d=128, q0=q0)
    assert np.array_equal(nsel[0].cpu().numpy()[rows], ref["nsel"])
    assert np.array_equal(sel[0].cpu().numpy()[rows], ref["sel"])
    assert np.abs(np32(out[0])[rows] - ref["out"]).max() <= TOL["bf16"]


@pytest.mark.parametrize("keys", ["groups", "random"])
def test_prefill_long_rows_select(qsa, keys):
    """Rows of about 33000 blocks (the CTA-per-row select).  "groups": every
    block's key is one of 64 vectors and the rotation is the identity
    (pos_scale 1e15), so each row's scores take 64 values, each shared
    exactly by ~515 blocks: the top-512 end inside a group of exact ties
    ranked by block id (bit-exact against the oracle).  "random": the usual
    case under the near-tie acceptance rule."""
    n_q, q0 = 32, 131968
    L = q0 + n_q
    g = torch.Generator(device=DEV).manual_seed(L)
    if keys == "groups":
        rope = qsa.Rope(pos_scale=1e15)
        vecs = torch.randn(64, 128, generator=g, device=DEV).to(torch.bfloat16)
        grp = torch.randint(0, 64, (L // 4,), generator=g, device=DEV)
        k_idx = vecs[grp].repeat_interleave(4, dim=0)[None].contiguous()
    else:
        rope = qsa.Rope()
        k_idx = torch.randn(1, L, 128, generator=g, device=DEV).to(torch.bfloat16)
    q_idx = torch.randn(1, n_q, 4, 128, generator=g, device=DEV).to(torch.bfloat16)
    k_pool = torch.zeros(1, L // 4, 128, dtype=torch.bfloat16, device=DEV)
    qsa.qsa_pool_keys_prefill(k_idx, k_pool, rope=rope)
    sel = torch.full((1, n_q, 512), -7, dtype=torch.int32, device=DEV)
    nsel = torch.full((1, n_q), -7, dtype=torch.int32, device=DEV)
    qsa.qsa_index_topk_prefill(q_idx, k_pool, sel, nsel, q0=q0, top_k=512, rope=rope)
    qsa.qsa_check_status()
    kp = oracle.pool_keys(np32(k_idx[0]), pos_scale=rope.pos_scale, store_bf16=True)
    assert np.array_equal(np32(k_pool[0]), kp)
    rows = list(range(n_q))
    kw = dict(q_idx=np32(q_idx[0]), k_pool=kp, top_k=512, store_bf16=True, pos_scale=rope.pos_scale, q0=q0)
    ref = oracle.prefill_rows(rows, **kw)
    g_sel, g_nsel = sel[0].cpu().numpy(), nsel[0].cpu().numpy()
    if keys == "groups":
        assert np.array_equal(g_nsel, ref["nsel"])
        assert np.array_equal(g_sel, ref["sel"])
    else:
        from qsa_testlib import selection_report
        _, _, nbad = selection_report(g_sel, g_nsel, ref,
                                      lambda rr: oracle.prefill_rows(rr, want_scores=True, **kw)["scores"], rows)
        assert nbad <= 2


def test_attention_flags_out_of_range_ids(qsa):
    """A selection id outside [0, nb(t)) is skipped and reported through the
    status word (no trap)."""
    w = W(64, top_k=4, seed=5)
    x = workloads.make_prefill(w, device=DEV)
    sel = torch.full((1, 64, 4), -1, dtype=torch.int32, device=DEV)
    nsel = torch.zeros(1, 64, dtype=torch.int32, device=DEV)
    sel[0, 40, 0] = 10            # nb(40) = 10: id 10 is not visible
    nsel[0, 40] = 1
    out = torch.empty_like(x["q"])
    qsa.qsa_sparse_attn_prefill(x["q"], x["k"], x["v"], sel, nsel, out)
    with pytest.raises(qsa.QSAError):
        qsa.qsa_check_status()
    qsa.qsa_check_status()        # cleared


# ----------------------------------------------------------------------------- decode

@pytest.mark.parametrize("dtype,flags,weights,L,B", [("bf16", 0, False, 20000, 6), ("bf16", 1, True, 9001, 3),
                                                     ("fp32", 0, False, 5000, 4), ("bf16", 0, False, 2, 5),
                                                     ("bf16", 0, False, 70001, 3), ("fp32", 1, True, 40000, 2),
                                                     # FP8 E4M3 compressed keys: fused indexer (B 6) and
                                                     # two-kernel path (B 3), tiny sequences
                                                     ("bf16", 4, False, 20000, 6), ("bf16", 5, True, 70001, 3),
                                                     ("bf16", 4, False, 2, 5), ("bf16", 6, False, 9001, 12)])
def test_decode_pipeline(qsa, dtype, flags, weights, L, B):
    w = workloads.Workload("dec", "decode", B, L, 256, 16, 2, 128, dtype, 77, pos_scale=2.0)
    x = workloads.make_decode(w, device=DEV, ragged=True)
    fp8 = bool(flags & qsa.QSA_KEYS_FP8)
    dt = torch.float8_e4m3fn if fp8 else x["k"].dtype
    rope = rope_of(w)
    lens = x["lens"]
    cap = max(lens) // 4 + 2
    # pooled cache of the prefix (prefill pooling), ring holding the unfinished block
    k_pool = torch.zeros(B, cap, 128, dtype=dt, device=DEV)
    ring = torch.zeros(B, 4, 128, dtype=x["k"].dtype, device=DEV)
    for b in range(B):
        kp = torch.zeros(1, cap, 128, dtype=dt, device=DEV)
        qsa.qsa_pool_keys_prefill(x["k_idx"][b:b + 1, :lens[b]].contiguous(), kp, rope=rope, flags=flags & 6)
        k_pool[b] = kp[0]
        nb0 = lens[b] // 4
        r = lens[b] - 4 * nb0
        if r:
            ring[b, :r] = x["k_idx"][b, 4 * nb0: lens[b]]
    head_w = torch.rand(B, 4, device=DEV) * 2 if weights else None
    qsa.qsa_pool_keys_decode(x["k_idx_new"], ring, k_pool, x["seq_len"], rope=rope, flags=flags & 6)
    sel = torch.full((B, w.top_k), -7, dtype=torch.int32, device=DEV)
    nsel = torch.full((B,), -7, dtype=torch.int32, device=DEV)
    qsa.qsa_index_topk_decode(x["q_idx"], k_pool, x["seq_len"], sel, nsel, top_k=w.top_k, head_w=head_w,
                              rope=rope, flags=flags)
    out = torch.empty_like(x["q"])
    lse = torch.empty(B, 16, dtype=torch.float32, device=DEV)
    qsa.qsa_sparse_attn_decode(x["q"], x["k"], x["v"], x["seq_len"], sel, nsel, out, lse=lse)
    qsa.qsa_check_status()
    # oracle, sequence by sequence
    differ = {}
    for b in range(B):
        s = lens[b] + 1
        kr = np32(x["k_idx"][b, :lens[b]])
        kp = np.zeros((cap, 128), np.float32)
        kp[: lens[b] // 4] = oracle.pool_keys(kr, pos_scale=2.0, rmsnorm=bool(flags & 2),
                                              store_bf16=dtype == "bf16", store_fp8=fp8)
        rg = np.zeros((4, 128), np.float32)
        nb0 = lens[b] // 4
        rg[: lens[b] - 4 * nb0] = kr[4 * nb0:]
        oracle.pool_decode(np32(x["k_idx_new"][b]), rg, kp, s, pos_scale=2.0, rmsnorm=bool(flags & 2),
                           store_bf16=dtype == "bf16", store_fp8=fp8)
        assert np.array_equal(np32(k_pool[b]), kp), f"pooled cache differs (seq {b})"
        ref = oracle.decode(np32(x["q_idx"][b:b + 1]), kp[None], [s],
                            head_w=None if head_w is None else head_w[b:b + 1].cpu().numpy(),
                            q=np32(x["q"][b:b + 1]), k=np32(x["k"][b:b + 1]), v=np32(x["v"][b:b + 1]),
                            relu=bool(flags & 1), store_bf16=dtype == "bf16", top_k=w.top_k, pos_scale=2.0,
                            want_scores=True)
        if not decode_selection_matches(sel[b].cpu().numpy(), nsel[b], ref):
            differ[b] = ref
            continue
        err = np.abs(np32(out[b]) - ref["out"][0]).max()
        assert err <= TOL[dtype], (b, err)
        assert np.abs(lse[b].cpu().numpy() - ref["lse"][0]).max() <= (1e-3 if dtype == "bf16" else 1e-4)

    def attn_on(s_, n_):
        o_ = torch.empty_like(x["q"])
        l_ = torch.empty(B, 16, dtype=torch.float32, device=DEV)
        qsa.qsa_sparse_attn_decode(x["q"], x["k"], x["v"], x["seq_len"], s_, n_, o_, lse=l_)
        return o_, l_

    stage_isolated_decode(differ, attn_on, B, w.top_k, TOL[dtype], 1e-3 if dtype == "bf16" else 1e-4)


@pytest.mark.parametrize("B", [1, 40])
def test_decode_fp8_keys_every_code_scored_exactly(qsa, B):
    """Every finite FP8 E4M3 code but -0 (subnormals included) is one block's
    key, in dim 127, which the rotation (rotary_dim 64) leaves alone; the
    query is the unit vector there, so each score is exactly the key's value.
    The top-k for k around the subnormals must then match the oracle's: a
    widening that lost a subnormal would tie it with zero and pick lower
    block ids.  B = 40 runs the fused indexer, B = 1 the two-kernel path."""
    codes = np.array([c for c in range(256) if c not in (0x7F, 0x80, 0xFF)], np.uint8)
    nb = len(codes)
    cap = nb + 1
    rng = np.random.default_rng(17)
    k_pool = torch.zeros(B, cap, 128, dtype=torch.uint8)
    for b in range(B):
        k_pool[b, :nb, 127] = torch.from_numpy(codes[rng.permutation(nb)])
    k_pool = k_pool.view(torch.float8_e4m3fn).to(DEV)
    q_idx = torch.zeros(B, 4, 128, dtype=torch.bfloat16, device=DEV)
    q_idx[:, 0, 127] = 1.0
    seq_len = torch.full((B,), 4 * nb + 1, dtype=torch.int32, device=DEV)
    rope = qsa.Rope(rotary_dim=64)
    kp = np32(k_pool)
    for top_k in [1, 100, 119, 120, 123, 126, 127, 128, 130, 252]:
        sel = torch.full((B, top_k), -7, dtype=torch.int32, device=DEV)
        nsel = torch.full((B,), -7, dtype=torch.int32, device=DEV)
        qsa.qsa_index_topk_decode(q_idx, k_pool, seq_len, sel, nsel, top_k=top_k, rope=rope,
                                  flags=qsa.QSA_KEYS_FP8)
        qsa.qsa_check_status()
        ref = oracle.decode(np32(q_idx), kp, seq_len.cpu().numpy(), top_k=top_k, rotary_dim=64)
        assert np.array_equal(nsel.cpu().numpy(), ref["nsel"])
        assert np.array_equal(sel.cpu().numpy(), ref["sel"]), top_k


@pytest.mark.parametrize("dtype,flags,lens", [("bf16", 0, [40000, 65537, 2049]), ("bf16", 1, [40000, 65537, 2049]),
                                              ("fp32", 0, [40000, 65537, 2049]),
                                              ("bf16", 0, [65537, 40000, 2049, 17, 65000, 60001, 1, 64000, 65536,
                                                          30000])])
def test_decode_select_all_ties(qsa, dtype, flags, lens):
    """All compressed keys zero: every score is 0, so the top-k is the k lowest
    block ids; with 10000+ blocks the tie bin spans several select chunks (and,
    with 10 sequences, the single-kernel cluster path with candidate overflow)."""
    B, top_k = len(lens), 512
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    cap = max(lens) // 4 + 1
    k_pool = torch.zeros(B, cap, 128, dtype=dt, device=DEV)
    g = torch.Generator().manual_seed(5)
    q_idx = torch.randn(B, 4, 128, generator=g).to(dt).to(DEV)
    seq_len = torch.tensor(lens, dtype=torch.int32, device=DEV)
    sel = torch.full((B, top_k), -7, dtype=torch.int32, device=DEV)
    nsel = torch.full((B,), -7, dtype=torch.int32, device=DEV)
    qsa.qsa_index_topk_decode(q_idx, k_pool, seq_len, sel, nsel, top_k=top_k, flags=flags)
    qsa.qsa_check_status()
    for b, L in enumerate(lens):
        nb = L // 4
        n = min(nb, top_k)
        assert int(nsel[b]) == n
        exp = np.full(top_k, -1, np.int32)
        exp[:n] = np.arange(n)
        assert np.array_equal(sel[b].cpu().numpy(), exp), b


def _paged_layout(lens, page_tokens, extra_pages, seed):
    """A page table that scatters each sequence's pages over a shuffled pool;
    table entries past a sequence's pages are -1 (never read)."""
    rng = np.random.default_rng(seed)
    need = [(L + page_tokens) // page_tokens for L in lens]          # positions 0 .. L (the new token)
    max_pages = max(need) + 1
    num_pages = sum(need) + extra_pages
    perm = rng.permutation(num_pages)
    table = np.full((len(lens), max_pages), -1, np.int32)
    k = 0
    for b, n in enumerate(need):
        table[b, :n] = perm[k:k + n]
        k += n
    return table, num_pages


@pytest.mark.parametrize("B,L,page_tokens,keys", [(6, 20000, 64, "bf16"), (3, 70001, 256, "bf16"),
                                                  (12, 9001, 32, "fp8"), (5, 2, 64, "bf16"),
                                                  (4, 5000, 1024, "bf16")])
def test_decode_paged_matches_contiguous(qsa, B, L, page_tokens, keys):
    """Paged caches (a shuffled page pool, one table row per sequence) give the
    contiguous results bit for bit: pooled rows, selections, attention output."""
    w = workloads.Workload("dec_paged", "decode", B, L, 256, 16, 2, 128, "bf16", 78, pos_scale=2.0)
    x = workloads.make_decode(w, device=DEV, ragged=True)
    rope = rope_of(w)
    lens = x["lens"]
    fp8 = keys == "fp8"
    kf = qsa.QSA_KEYS_FP8 if fp8 else 0
    kdt = torch.float8_e4m3fn if fp8 else torch.bfloat16
    table_np, num_pages = _paged_layout(lens, page_tokens, 3, B + L)
    table = torch.from_numpy(table_np).to(DEV)
    pt = page_tokens
    # contiguous reference pipeline
    cap = max(lens) // 4 + 2
    k_pool = torch.zeros(B, cap, 128, dtype=kdt, device=DEV)
    ring = torch.zeros(B, 4, 128, dtype=torch.bfloat16, device=DEV)
    for b in range(B):
        kp = torch.zeros(1, cap, 128, dtype=kdt, device=DEV)
        qsa.qsa_pool_keys_prefill(x["k_idx"][b:b + 1, :lens[b]].contiguous(), kp, rope=rope, flags=kf)
        k_pool[b] = kp[0]
        nb0 = lens[b] // 4
        if lens[b] > 4 * nb0:
            ring[b, :lens[b] - 4 * nb0] = x["k_idx"][b, 4 * nb0: lens[b]]
    ring_p = ring.clone()
    qsa.qsa_pool_keys_decode(x["k_idx_new"], ring, k_pool, x["seq_len"], rope=rope, flags=kf)
    sel = torch.empty(B, w.top_k, dtype=torch.int32, device=DEV)
    nsel = torch.empty(B, dtype=torch.int32, device=DEV)
    qsa.qsa_index_topk_decode(x["q_idx"], k_pool, x["seq_len"], sel, nsel, top_k=w.top_k, rope=rope, flags=kf)
    out = torch.empty_like(x["q"])
    qsa.qsa_sparse_attn_decode(x["q"], x["k"], x["v"], x["seq_len"], sel, nsel, out)
    # paged caches: K/V scattered to their slots, compressed keys pooled straight into pages
    slots = [torch.from_numpy((table_np[b, np.arange(lens[b] + 1) // pt].astype(np.int64) * pt
                               + np.arange(lens[b] + 1) % pt)).to(DEV) for b in range(B)]
    k_pg = torch.zeros(num_pages * pt, 2, 128, dtype=torch.bfloat16, device=DEV)
    v_pg = torch.zeros_like(k_pg)
    for b in range(B):
        k_pg[slots[b]] = x["k"][b, :lens[b] + 1]
        v_pg[slots[b]] = x["v"][b, :lens[b] + 1]
    kpool_pg = torch.zeros(num_pages * pt // 4, 128, dtype=kdt, device=DEV)
    for b in range(B):
        qsa.qsa_pool_keys_prefill_paged(x["k_idx"][b:b + 1, :lens[b]].contiguous(), kpool_pg, table[b:b + 1], pt,
                                        rope=rope, flags=kf)
    qsa.qsa_pool_keys_decode_paged(x["k_idx_new"], ring_p, kpool_pg, table, pt, x["seq_len"], rope=rope, flags=kf)
    sel_p = torch.full((B, w.top_k), -7, dtype=torch.int32, device=DEV)
    nsel_p = torch.full((B,), -7, dtype=torch.int32, device=DEV)
    qsa.qsa_index_topk_decode_paged(x["q_idx"], kpool_pg, table, pt, x["seq_len"], sel_p, nsel_p, top_k=w.top_k,
                                    rope=rope, flags=kf)
    out_p = torch.empty_like(x["q"])
    qsa.qsa_sparse_attn_decode_paged(x["q"], k_pg, v_pg, table, pt, x["seq_len"], sel_p, nsel_p, out_p)
    qsa.qsa_check_status()                       # no page outside the table was touched
    assert torch.equal(ring_p, ring)
    for b in range(B):
        nbk = (lens[b] + 1) // 4
        rows = slots[b][0:4 * nbk:4] // 4
        assert torch.equal(kpool_pg[rows].view(torch.uint8), k_pool[b, :nbk].view(torch.uint8)), b
    assert torch.equal(nsel_p, nsel) and torch.equal(sel_p, sel)
    assert torch.equal(out_p, out)


def test_decode_paged_flags_a_page_outside_the_cache(qsa):
    B, L, pt = 2, 3000, 64
    w = workloads.Workload("dec_paged_bad", "decode", B, L, 64, 16, 2, 128, "bf16", 79)
    x = workloads.make_decode(w, device=DEV)
    table_np, num_pages = _paged_layout([L] * B, pt, 0, 5)
    table_np[1, 3] = num_pages + 7               # one page id past the pool
    table = torch.from_numpy(table_np).to(DEV)
    kpool = torch.zeros(num_pages * pt // 4, 128, dtype=torch.bfloat16, device=DEV)
    kv = torch.zeros(num_pages * pt, 2, 128, dtype=torch.bfloat16, device=DEV)
    sel = torch.empty(B, w.top_k, dtype=torch.int32, device=DEV)
    nsel = torch.empty(B, dtype=torch.int32, device=DEV)
    qsa.qsa_index_topk_decode_paged(x["q_idx"], kpool, table, pt, x["seq_len"], sel, nsel, top_k=w.top_k,
                                    rope=rope_of(w))
    with pytest.raises(qsa.QSAError):
        qsa.qsa_check_status()
    out = torch.empty_like(x["q"])
    sel_all = torch.arange(w.top_k, dtype=torch.int32, device=DEV).repeat(B, 1) + 40   # blocks 40.. cross page 3
    nsel_all = torch.full((B,), w.top_k, dtype=torch.int32, device=DEV)
    qsa.qsa_sparse_attn_decode_paged(x["q"], kv, kv, table, pt, x["seq_len"], sel_all, nsel_all, out)
    with pytest.raises(qsa.QSAError):
        qsa.qsa_check_status()


def test_decode_index_workspace_stays_zero_and_dirty_one_is_flagged(qsa):
    """The two-kernel decode indexer leaves its workspace zero after a call,
    so one zero-filled workspace serves any number of calls; a workspace whose
    histogram was not zero is flagged (status bit 16)."""
    w = workloads.Workload("dec_ws", "decode", 2, 20001, 256, 16, 2, 128, "bf16", 93)
    x = workloads.make_decode(w, device=DEV)
    rope = rope_of(w)
    cap = w.T // 4 + 1
    k_pool = torch.zeros(2, cap, 128, dtype=torch.bfloat16, device=DEV)
    qsa.qsa_pool_keys_prefill(x["k_idx"], k_pool, rope=rope)
    need = qsa.qsa_index_topk_decode_workspace(2, cap, w.top_k)
    ws = torch.zeros(need, dtype=torch.uint8, device=DEV)
    sel = torch.empty(2, w.top_k, dtype=torch.int32, device=DEV)
    nsel = torch.empty(2, dtype=torch.int32, device=DEV)
    run = lambda: qsa.qsa_index_topk_decode(x["q_idx"], k_pool, x["seq_len"], sel, nsel, max_blocks=cap,
                                            top_k=w.top_k, rope=rope, workspace=ws)
    run()
    qsa.qsa_check_status()
    first = sel.clone()
    hist_bytes = (2 * 2048 * 4 + 255) // 256 * 256        # the workspace ends with [B][2048] u32 counts
    assert int(ws[need - hist_bytes:].count_nonzero()) == 0
    run()
    qsa.qsa_check_status()
    assert torch.equal(sel, first)
    ws[need - hist_bytes] = 1                              # one stray count in sequence 0's lowest bin
    run()
    with pytest.raises(qsa.QSAError):
        qsa.qsa_check_status()
    assert torch.equal(sel, first)                         # a count in the lowest bin moves nothing
    assert int(ws[need - hist_bytes:].count_nonzero()) == 0
    run()
    qsa.qsa_check_status()


def test_decode_step_graph_replay_matches_eager(qsa):
    """A decode step (ring pooling, indexer, attention with caller workspaces)
    captured in a CUDA graph and replayed gives the eager results bit for bit."""
    w = workloads.Workload("dec_graph", "decode", 6, 30001, 512, 16, 2, 128, "bf16", 91)
    x = workloads.make_decode(w, device=DEV, ragged=True)
    rope = rope_of(w)
    B = w.B
    cap = max(x["lens"]) // 4 + 2
    k_pool = torch.zeros(B, cap, 128, dtype=torch.bfloat16, device=DEV)
    for b in range(B):
        kp = torch.zeros(1, cap, 128, dtype=torch.bfloat16, device=DEV)
        qsa.qsa_pool_keys_prefill(x["k_idx"][b:b + 1, :x["lens"][b]].contiguous(), kp, rope=rope)
        k_pool[b] = kp[0]
    ring0 = torch.zeros(B, 4, 128, dtype=torch.bfloat16, device=DEV)
    max_blocks = cap
    ws_i = torch.zeros(qsa.qsa_index_topk_decode_workspace(B, max_blocks, w.top_k), dtype=torch.uint8, device=DEV)
    ws_a = torch.empty(qsa.qsa_sparse_attn_decode_workspace(B, w.Hq, w.d, w.top_k), dtype=torch.uint8, device=DEV)

    def step(ring, pool, sel, nsel, out):
        qsa.qsa_pool_keys_decode(x["k_idx_new"], ring, pool, x["seq_len"], rope=rope)
        qsa.qsa_index_topk_decode(x["q_idx"], pool, x["seq_len"], sel, nsel, max_blocks=max_blocks, top_k=w.top_k,
                                  rope=rope, workspace=ws_i)
        qsa.qsa_sparse_attn_decode(x["q"], x["k"], x["v"], x["seq_len"], sel, nsel, out, workspace=ws_a)

    def buffers():
        return (ring0.clone(), k_pool.clone(), torch.empty(B, w.top_k, dtype=torch.int32, device=DEV),
                torch.empty(B, dtype=torch.int32, device=DEV), torch.empty_like(x["q"]))

    eager = buffers()
    step(*eager)
    graphed = buffers()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step(*buffers())                        # warm-up outside the capture
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step(*graphed)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    qsa.qsa_check_status()
    for a, b in zip(eager, graphed):
        assert torch.equal(a, b)


# ----------------------------------------------------------------------------- IndexShare draft steps

@pytest.mark.parametrize("dtype,Hq,Hkv,B,L,top_k,max_draft", [("bf16", 16, 2, 6, 9000, 256, 8),
                                                               ("bf16", 8, 1, 3, 2500, 64, 13),
                                                               ("fp32", 8, 1, 3, 3000, 64, 5),
                                                               ("bf16", 32, 4, 2, 1800, 512, 3)])
def test_indexshare_draft_step_on_oracle_selection(qsa, dtype, Hq, Hkv, B, L, top_k, max_draft):
    """Draft steps after a capture row: the GPU attention, fed the selection the
    oracle made for the capture row, matches the oracle's draft step for every
    number of drafted positions 0..max_draft (ragged over sequences)."""
    d = 128
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    g = torch.Generator().manual_seed(L + B)
    kv_len = L + max_draft + 8
    k = torch.randn(B, kv_len, Hkv, d, generator=g).to(dt)
    v = torch.randn(B, kv_len, Hkv, d, generator=g).to(dt)
    q = torch.randn(B, Hq, d, generator=g).to(dt)
    k_raw = torch.randn(B, kv_len, 128, generator=g).to(dt)
    q_idx = torch.randn(B, 4, 128, generator=g).to(dt)
    # capture rows t_c = cap_len - 1 with every residue mod 4 (and a short one)
    cap = [L - (i % 4) for i in range(B)]
    cap[-1] = 3 if B > 2 else cap[-1]
    pool_cap = kv_len // 4 + 1
    kp = np.zeros((B, pool_cap, 128), np.float32)
    for b in range(B):
        nb = cap[b] // 4
        if nb:
            kp[b, :nb] = oracle.pool_keys(np32(k_raw[b, :4 * nb]), store_bf16=dtype == "bf16")
    ref_sel = oracle.decode(np32(q_idx), kp, cap, top_k=top_k, store_bf16=dtype == "bf16")
    sel = torch.from_numpy(ref_sel["sel"]).to(DEV)
    nsel = torch.from_numpy(ref_sel["nsel"]).to(DEV)
    kd, vd, qd = k.to(DEV), v.to(DEV), q.to(DEV)
    for step in range(max_draft + 1):
        drafted = [(step + b) % (max_draft + 1) for b in range(B)]
        seq = [cap[b] + drafted[b] for b in range(B)]
        out = torch.empty_like(qd)
        lse = torch.empty(B, Hq, dtype=torch.float32, device=DEV)
        qsa.qsa_sparse_attn_decode_shared(qd, kd, vd, torch.tensor(seq, dtype=torch.int32, device=DEV),
                                          torch.tensor(cap, dtype=torch.int32, device=DEV), sel, nsel, out,
                                          max_draft, top_k=top_k, lse=lse)
        qsa.qsa_check_status()
        ref = oracle.decode(np32(q_idx), kp, seq, cap_len=cap, q=np32(q), k=np32(k), v=np32(v), top_k=top_k,
                            Hq=Hq, Hkv=Hkv, d=d, store_bf16=dtype == "bf16")
        np.testing.assert_array_equal(ref["sel"], ref_sel["sel"])
        err = np.abs(np32(out) - ref["out"]).max()
        assert err <= TOL[dtype], (step, err)
        assert np.abs(lse.cpu().numpy() - ref["lse"]).max() <= (1e-3 if dtype == "bf16" else 1e-4)


def test_indexshare_flags_out_of_range_capture(qsa):
    """seq_len < cap_len, or more drafted positions than max_draft, is read as
    a plain decode step and reported through the status word (no trap)."""
    B, Hq, Hkv, d, L = 2, 16, 2, 128, 600
    g = torch.Generator().manual_seed(3)
    k = torch.randn(B, L + 40, Hkv, d, generator=g).to(torch.bfloat16).to(DEV)
    v = torch.randn(B, L + 40, Hkv, d, generator=g).to(torch.bfloat16).to(DEV)
    q = torch.randn(B, Hq, d, generator=g).to(torch.bfloat16).to(DEV)
    sel = torch.full((B, 64), -1, dtype=torch.int32, device=DEV)
    nsel = torch.zeros(B, dtype=torch.int32, device=DEV)
    out = torch.empty_like(q)
    for seq, cap in [([L, L], [L + 1, L]), ([L + 9, L], [L, L])]:   # behind the capture; 9 > max_draft 4
        qsa.qsa_sparse_attn_decode_shared(q, k, v, torch.tensor(seq, dtype=torch.int32, device=DEV),
                                          torch.tensor(cap, dtype=torch.int32, device=DEV), sel, nsel, out, 4)
        with pytest.raises(qsa.QSAError):
            qsa.qsa_check_status()
        qsa.qsa_check_status()        # cleared


# ----------------------------------------------------------------------------- dense decode baseline

@pytest.mark.parametrize("dtype,Hq,Hkv,B,L", [("bf16", 16, 2, 4, 20001), ("bf16", 8, 1, 3, 3), ("fp32", 8, 1, 3, 7000),
                                             ("bf16", 32, 4, 2, 9000)])
def test_dense_decode_matches_textbook_attention(qsa, dtype, Hq, Hkv, B, L):
    """Full causal decode attention (the baseline QSA replaces) against the
    oracle's textbook causal attention, ragged lengths."""
    d = 128
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    g = torch.Generator().manual_seed(L)
    k = torch.randn(B, L + 4, Hkv, d, generator=g).to(dt)
    v = torch.randn(B, L + 4, Hkv, d, generator=g).to(dt)
    q = torch.randn(B, Hq, d, generator=g).to(dt)
    lens = [max(1, L - i) for i in range(B)]
    out = torch.empty(B, Hq, d, dtype=dt, device=DEV)
    qsa.qsa_dense_attn_decode(q.to(DEV), k.to(DEV), v.to(DEV), torch.tensor(lens, dtype=torch.int32, device=DEV), out)
    qsa.qsa_check_status()
    for b in range(B):
        t = lens[b] - 1
        ref = oracle.dense_rows([0], q=np32(q[b])[None], k=np32(k[b]), v=np32(v[b]), Hq=Hq, Hkv=Hkv, d=d, q0=t)
        err = np.abs(np32(out[b]) - ref[0]).max()
        assert err <= TOL[dtype], (b, err)


# ----------------------------------------------------------------------------- tensor-core prefill over query tiles

def _overlapping_selection(T, top_k, seed, hot=64, short_every=5):
    """Seeded selections whose neighbouring rows overlap (a shared hot set of
    blocks plus row-specific ones), some rows shorter than min(top_k, nb)."""
    rng = np.random.default_rng(seed)
    sel = np.full((T, top_k), -1, np.int32)
    nsel = np.zeros(T, np.int32)
    hot_ids = rng.permutation(max(T // 4, 1))[:hot]
    for t in range(T):
        nb = (t + 1) // 4
        if nb == 0:
            continue
        want = min(top_k, nb)
        if t % short_every == 0:
            want = max(1, want // 3)
        cand = [b for b in hot_ids if b < nb][: want // 2]
        rest = rng.permutation(nb)
        chosen = list(dict.fromkeys(list(cand) + list(rest)))[:want]
        chosen = np.sort(np.array(chosen, np.int32))
        sel[t, :len(chosen)] = chosen
        nsel[t] = len(chosen)
    return sel, nsel


@pytest.mark.parametrize("Hq,Hkv,T,top_k", [(16, 2, 1500, 96), (8, 1, 777, 64), (32, 4, 2049, 128),
                                           (16, 2, 9000, 2048), (16, 2, 5, 4)])
def test_tile_attention_on_overlapping_selections(qsa, Hq, Hkv, T, top_k):
    """Hand-built overlapping selections (hot blocks shared by many rows, rows
    with fewer than min(top_k, nb) blocks, a last partial 8-row tile): the
    split prefill (shared blocks on the tensor cores, the rest in the gather
    kernel) equals the oracle's attention over the same selections, B = 2
    sequences with different selections."""
    w = W(T, top_k=top_k, Hq=Hq, Hkv=Hkv, B=2, seed=90 + Hq)
    x = workloads.make_prefill(w, device=DEV)
    sels, nsels = zip(*[_overlapping_selection(T, top_k, seed=7 + b) for b in range(2)])
    sel = torch.from_numpy(np.stack(sels)).to(DEV)
    nsel = torch.from_numpy(np.stack(nsels)).to(DEV)
    out = torch.full_like(x["q"], 9.0)
    lse = torch.empty(2, T, Hq, dtype=torch.float32, device=DEV)
    qsa.qsa_sparse_attn_prefill(x["q"], x["k"], x["v"], sel, nsel, out, lse=lse)
    qsa.qsa_check_status()
    rows = list(range(T)) if T <= 2100 else sorted(set(range(0, T, 3)) | set(range(T - 40, T)))
    for b in range(2):
        ref = oracle.prefill_rows(rows, sel_in=sels[b][rows], nsel_in=nsels[b][rows], top_k=top_k,
                                  q=np32(x["q"][b]), k=np32(x["k"][b]), v=np32(x["v"][b]), Hq=Hq, Hkv=Hkv, d=128)
        err = np.abs(np32(out[b])[rows] - ref["out"]).max()
        assert err <= TOL["bf16"], (b, err)
        assert np.abs(lse[b].cpu().numpy()[rows] - ref["lse"]).max() <= 1e-3


def test_tile_attention_chunks_off_the_tile_grid(qsa):
    """Chunks that start off the 8-row tile grid (q0 = 1000, 1001 are not both
    multiples of 8) form other tiles than one call does; every row still
    matches the oracle."""
    T, top_k = 1700, 64
    w = W(T, top_k=top_k, seed=95)
    x = workloads.make_prefill(w, device=DEV)
    sel_np, nsel_np = _overlapping_selection(T, top_k, seed=3)
    sel = torch.from_numpy(sel_np[None]).to(DEV)
    nsel = torch.from_numpy(nsel_np[None]).to(DEV)
    out = torch.empty_like(x["q"])
    for c0, c1 in [(0, 1000), (1000, 1001), (1001, 1700)]:
        o = torch.empty(1, c1 - c0, 16, 128, dtype=torch.bfloat16, device=DEV)
        qsa.qsa_sparse_attn_prefill(x["q"][:, c0:c1].contiguous(), x["k"], x["v"], sel[:, c0:c1].contiguous(),
                                    nsel[:, c0:c1].contiguous(), o, q0=c0)
        out[:, c0:c1] = o
    qsa.qsa_check_status()
    rows = list(range(T))
    ref = oracle.prefill_rows(rows, sel_in=sel_np, nsel_in=nsel_np, top_k=top_k, q=np32(x["q"][0]),
                              k=np32(x["k"][0]), v=np32(x["v"][0]), Hq=16, Hkv=2, d=128)
    assert np.abs(np32(out[0]) - ref["out"]).max() <= TOL["bf16"]


def test_tile_attention_aligned_chunks_are_bit_exact(qsa):
    """Chunks starting on the 8-row tile grid reproduce one call bit for bit
    (same tiles, same lists, same order of accumulation)."""
    T, top_k = 2000, 96
    w = W(T, top_k=top_k, seed=96)
    x = workloads.make_prefill(w, device=DEV)
    sel_np, nsel_np = _overlapping_selection(T, top_k, seed=4)
    sel = torch.from_numpy(sel_np[None]).to(DEV)
    nsel = torch.from_numpy(nsel_np[None]).to(DEV)
    one = torch.empty_like(x["q"])
    qsa.qsa_sparse_attn_prefill(x["q"], x["k"], x["v"], sel, nsel, one)
    out = torch.empty_like(x["q"])
    for c0, c1 in [(0, 512), (512, 1536), (1536, 2000)]:
        o = torch.empty(1, c1 - c0, 16, 128, dtype=torch.bfloat16, device=DEV)
        qsa.qsa_sparse_attn_prefill(x["q"][:, c0:c1].contiguous(), x["k"], x["v"], sel[:, c0:c1].contiguous(),
                                    nsel[:, c0:c1].contiguous(), o, q0=c0)
        out[:, c0:c1] = o
    qsa.qsa_check_status()
    assert torch.equal(out, one)


@pytest.mark.parametrize("Hq,Hkv", [(16, 2), (32, 4)])
def test_split_attention_repeats_bit_identically(qsa, Hq, Hkv):
    """The split prefill on the oracle's selection: four calls give the same
    bits (output and lse), and match the oracle.  (A race in the gather
    kernel's query buffer once made rare rows differ from run to run when
    its lists were short, as the split's own lists are.)"""
    T = 2500
    w = W(T, top_k=96, Hq=Hq, Hkv=Hkv, seed=33)
    x = workloads.make_prefill(w, device=DEV)
    rows = list(range(T))
    kp = oracle.pool_keys(np32(x["k_idx"][0]), store_bf16=True)
    ref = oracle.prefill_rows(rows, q_idx=np32(x["q_idx"][0]), k_pool=kp, top_k=96, store_bf16=True,
                              q=np32(x["q"][0]), k=np32(x["k"][0]), v=np32(x["v"][0]), Hq=Hq, Hkv=Hkv, d=128)
    sel = torch.from_numpy(ref["sel"][None]).to(DEV)
    nsel = torch.from_numpy(ref["nsel"][None]).to(DEV)
    outs = []
    for _ in range(4):
        out = torch.empty_like(x["q"])
        lse = torch.empty(1, T, Hq, dtype=torch.float32, device=DEV)
        qsa.qsa_sparse_attn_prefill(x["q"], x["k"], x["v"], sel, nsel, out, lse=lse)
        outs.append((out, lse))
    qsa.qsa_check_status()
    for out, lse in outs[1:]:
        assert torch.equal(out, outs[0][0]) and torch.equal(lse, outs[0][1])
    assert np.abs(np32(outs[0][0][0]) - ref["out"]).max() <= TOL["bf16"]
    assert np.abs(outs[0][1][0].cpu().numpy() - ref["lse"]).max() <= 1e-3


@pytest.mark.parametrize("Hq,Hkv", [(16, 2), (32, 4), (8, 1)])
def test_attention_tail_only_rows(qsa, Hq, Hkv):
    """Selections of no block at all (nsel = 0): each row attends to its own
    0-3 tail tokens only, rows whose position ends a block attend to nothing
    (zero output, lse = -inf); three calls give the same bits."""
    T = 2500
    w = W(T, top_k=96, Hq=Hq, Hkv=Hkv, seed=34)
    x = workloads.make_prefill(w, device=DEV)
    sel = torch.full((1, T, 96), -1, dtype=torch.int32, device=DEV)
    nsel = torch.zeros(1, T, dtype=torch.int32, device=DEV)
    outs = []
    for _ in range(3):
        out = torch.full_like(x["q"], 5.0)
        lse = torch.empty(1, T, Hq, dtype=torch.float32, device=DEV)
        qsa.qsa_sparse_attn_prefill(x["q"], x["k"], x["v"], sel, nsel, out, lse=lse)
        outs.append((out, lse))
    qsa.qsa_check_status()
    for out, lse in outs[1:]:
        assert torch.equal(out, outs[0][0]) and torch.equal(lse, outs[0][1])
    rows = list(range(T))
    ref = oracle.prefill_rows(rows, sel_in=sel[0].cpu().numpy(), nsel_in=nsel[0].cpu().numpy(), top_k=96,
                              q=np32(x["q"][0]), k=np32(x["k"][0]), v=np32(x["v"][0]), Hq=Hq, Hkv=Hkv, d=128)
    assert np.abs(np32(outs[0][0][0]) - ref["out"]).max() <= TOL["bf16"]
    g, r = outs[0][1][0].cpu().numpy(), ref["lse"]
    assert np.array_equal(np.isinf(g), np.isinf(r))
    fin = np.isfinite(r)
    assert np.abs(g[fin] - r[fin]).max() <= 1e-3


@pytest.mark.parametrize("flags", [0, 1])
def test_prefill_select_massive_16bit_ties(qsa, flags):
    """Zero compressed keys: every score is exactly 0, so all keys of a row
    tie at 16 bits (more than 2048 of them from position 8192 on) and the
    select takes its exact radix over re-scored keys; the ties go to the
    lowest ids, as in the oracle (bit-exact), for the linear and the ReLU
    per-head scores."""
    T, top_k = 40000, 512
    g = torch.Generator(device=DEV).manual_seed(41)
    q_idx = torch.randn(1, T, 4, 128, generator=g, device=DEV).to(torch.bfloat16)
    k_pool = torch.zeros(1, T // 4, 128, dtype=torch.bfloat16, device=DEV)
    sel = torch.full((1, T, top_k), -7, dtype=torch.int32, device=DEV)
    nsel = torch.full((1, T), -7, dtype=torch.int32, device=DEV)
    qsa.qsa_index_topk_prefill(q_idx, k_pool, sel, nsel, top_k=top_k, rope=qsa.Rope(), flags=flags)
    qsa.qsa_check_status()
    rows = [0, 3, 2047, 2048, 2051, 8191, 8200, 20000, 39999]
    ref = oracle.prefill_rows(rows, q_idx=np32(q_idx[0]), k_pool=np32(k_pool[0]), top_k=top_k, store_bf16=True,
                              relu=bool(flags & qsa.QSA_SCORE_RELU))
    assert np.array_equal(nsel[0].cpu().numpy()[rows], ref["nsel"])
    assert np.array_equal(sel[0].cpu().numpy()[rows], ref["sel"])


@pytest.mark.parametrize("eps", [0.02, 0.03])
def test_prefill_select_crowded_bins_multi_tile(qsa, eps):
    """Compressed keys 1 + U(-eps, eps): every score of a row is close to the
    same value, so a row's keys crowd into one or two 12-bit bins and tie in
    the hundreds at 16 bits.  Rows of more than 8192 blocks whose keys above
    and in the threshold's 12-bit bin exceed the select's 4096-entry list
    (eps 0.02: about 6900 and 10000 at rows 36000 and 39999) read the row a
    third time; the others (eps 0.03, row 39999: about 1070) are listed in
    pass 2.  Both agree with the oracle under the 1e-4 gap rule."""
    T, top_k = 40000, 512
    g = torch.Generator().manual_seed(43)
    q_idx = torch.randn(1, T, 4, 128, generator=g).to(torch.bfloat16)
    k_pool = (1.0 + eps * (2 * torch.rand(1, T // 4, 128, generator=g) - 1)).to(torch.bfloat16)
    q_idx, k_pool = q_idx.to(DEV), k_pool.to(DEV)
    sel = torch.full((1, T, top_k), -7, dtype=torch.int32, device=DEV)
    nsel = torch.full((1, T), -7, dtype=torch.int32, device=DEV)
    qsa.qsa_index_topk_prefill(q_idx, k_pool, sel, nsel, top_k=top_k, rope=qsa.Rope())
    qsa.qsa_check_status()
    rows = [32775, 36000, 38000, 39999]
    qi, kp = np32(q_idx[0]), np32(k_pool[0])
    ref = oracle.prefill_rows(rows, q_idx=qi, k_pool=kp, top_k=top_k, store_bf16=True)

    def score_fn(rr):
        return oracle.prefill_rows(rr, q_idx=qi, k_pool=kp, top_k=top_k, store_bf16=True, want_scores=True)["scores"]

    selection_report(sel[0].cpu().numpy()[rows], nsel[0].cpu().numpy()[rows], ref, score_fn, rows)
