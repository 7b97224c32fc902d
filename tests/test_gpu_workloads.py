"""Full-size parity of the five workloads the method is measured on, in the
launch configuration the benchmark times, against the CPU oracle on sampled
rows (prefill) or every sequence (decode)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from qsa_testlib import (TOL, check_prefill_workload, decode_selection_matches, np32, rope_of,
                         stage_isolated_decode)

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def qsa():
    import block_sparse_attention_11_b200 as m
    return m


def _free():
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def test_tiny_prefill_fp32_all_rows(qsa):
    w = workloads.WORKLOADS["tiny_prefill_t1k_fp32"]
    x = workloads.make_prefill(w, device=DEV)
    r = check_prefill_workload(x, w, list(range(w.T)))
    assert r["nbad"] <= 2
    assert r["err"] <= TOL["fp32"]


def test_prefill_32k_needles(qsa):
    w = workloads.WORKLOADS["prefill_t32k_needles"]
    x = workloads.make_prefill(w, device=DEV)
    rows = workloads.sample_rows(w.T, x["needles"], n_uniform=1024)
    r = check_prefill_workload(x, w, rows)
    # every needle block is selected by each of its aligned queries
    g_sel = r["g"]["sel"][0].cpu().numpy()
    g_nsel = r["g"]["nsel"][0].cpu().numpy()
    assert len(x["needles"]) == w.needles
    for b, ts in x["needles"]:
        for t in ts:
            assert b in set(g_sel[t, :g_nsel[t]].tolist()), f"needle block {b} missed by query {t}"
    assert r["nbad"] <= len(rows) // 50
    del x, r
    _free()


def test_prefill_dense_reduction_t2048(qsa):
    """T = 2048 with top-512: every visible block is selected, so the sparse
    path must equal textbook causal attention."""
    w = workloads.Workload("dense2048", "prefill", 1, 2048, 512, 16, 2, 128, "bf16", 99)
    x = workloads.make_prefill(w, device=DEV)
    from qsa_testlib import gpu_prefill
    g = gpu_prefill(x, w)
    rows = np.arange(0, 2048, 3)
    ref = oracle.dense_rows(rows, np32(x["q"][0]), np32(x["k"][0]), np32(x["v"][0]), 16, 2, 128)
    err = np.abs(np32(g["out"][0])[rows] - ref).max()
    assert err <= TOL["bf16"], err
    nb = (np.arange(2048) + 1) // 4
    assert np.array_equal(g["nsel"][0].cpu().numpy(), np.minimum(nb, 512))


def test_prefill_128k_heavy_tail(qsa):
    w = workloads.WORKLOADS["prefill_t128k_heavytail"]
    x = workloads.make_prefill(w, device=DEV)
    rows = workloads.sample_rows(w.T, n_uniform=1024)
    r = check_prefill_workload(x, w, rows)
    assert r["nbad"] <= len(rows) // 50
    del x, r
    _free()


def _attn_decode(qsa, x, sel, nsel):
    out = torch.empty_like(x["q"])
    qsa.qsa_sparse_attn_decode(x["q"], x["k"], x["v"], x["seq_len"], sel, nsel, out)
    return out, None


def _decode_check(qsa, w, B=None, L=None, ragged=False):
    x = workloads.make_decode(w, device=DEV, B=B, L=L, ragged=ragged)
    B = x["q"].shape[0]
    lens = x["lens"]
    rope = rope_of(w)
    dt = x["k"].dtype
    fp8 = w.extra.get("keys") == "fp8"          # compressed keys stored as FP8 E4M3
    kflags = qsa.QSA_KEYS_FP8 if fp8 else 0
    kdt = torch.float8_e4m3fn if fp8 else dt
    cap = max(lens) // 4 + 1
    k_pool = torch.zeros(B, cap, 128, dtype=kdt, device=DEV)
    ring = torch.zeros(B, 4, 128, dtype=dt, device=DEV)
    for b in range(B):
        kp = torch.zeros(1, cap, 128, dtype=kdt, device=DEV)
        qsa.qsa_pool_keys_prefill(x["k_idx"][b:b + 1, :lens[b]].contiguous(), kp, rope=rope, flags=kflags)
        k_pool[b] = kp[0]
        nb0 = lens[b] // 4
        if lens[b] > 4 * nb0:
            ring[b, :lens[b] - 4 * nb0] = x["k_idx"][b, 4 * nb0: lens[b]]
    qsa.qsa_pool_keys_decode(x["k_idx_new"], ring, k_pool, x["seq_len"], rope=rope, flags=kflags)
    sel = torch.empty(B, w.top_k, dtype=torch.int32, device=DEV)
    nsel = torch.empty(B, dtype=torch.int32, device=DEV)
    qsa.qsa_index_topk_decode(x["q_idx"], k_pool, x["seq_len"], sel, nsel, top_k=w.top_k, rope=rope, flags=kflags)
    out = torch.empty_like(x["q"])
    qsa.qsa_sparse_attn_decode(x["q"], x["k"], x["v"], x["seq_len"], sel, nsel, out)
    qsa.qsa_check_status()
    differ = {}
    for b in range(B):
        s = lens[b] + 1
        kr = np32(x["k_idx"][b, :lens[b]])
        kp = np.zeros((cap, 128), np.float32)
        kp[: lens[b] // 4] = oracle.pool_keys(kr, base=w.rope_base, pos_scale=w.pos_scale, store_fp8=fp8)
        rg = np.zeros((4, 128), np.float32)
        nb0 = lens[b] // 4
        rg[: lens[b] - 4 * nb0] = kr[4 * nb0:]
        oracle.pool_decode(np32(x["k_idx_new"][b]), rg, kp, s, base=w.rope_base, pos_scale=w.pos_scale,
                           store_fp8=fp8)
        assert np.array_equal(np32(k_pool[b]), kp), f"pooled keys differ (seq {b})"
        ref = oracle.decode(np32(x["q_idx"][b:b + 1]), kp[None], [s], q=np32(x["q"][b:b + 1]),
                            k=np32(x["k"][b:b + 1]), v=np32(x["v"][b:b + 1]), top_k=w.top_k,
                            base=w.rope_base, pos_scale=w.pos_scale, want_scores=True)
        if not decode_selection_matches(sel[b].cpu().numpy(), nsel[b], ref):
            differ[b] = ref
            continue
        err = np.abs(np32(out[b]) - ref["out"][0]).max()
        assert err <= TOL["bf16"], (b, err)
    assert len(differ) <= max(1, B // 16)
    stage_isolated_decode(differ, lambda s_, n_: _attn_decode(qsa, x, s_, n_), B, w.top_k, TOL["bf16"])
    del x
    _free()


def test_decode_128k_b64(qsa):
    _decode_check(qsa, workloads.WORKLOADS["decode_b64_l128k"])


def test_decode_128k_ragged_tails(qsa):
    _decode_check(qsa, workloads.WORKLOADS["decode_b64_l128k"], B=8, ragged=True)


def test_decode_1m_b8_scaled_positions(qsa):
    _decode_check(qsa, workloads.WORKLOADS["decode_b8_l1m_scale4"])


def test_decode_128k_b64_fp8_keys(qsa):
    _decode_check(qsa, workloads.WORKLOADS["decode_b64_l128k_fp8keys"])


def test_decode_1m_b8_fp8_keys(qsa):
    _decode_check(qsa, workloads.WORKLOADS["decode_b8_l1m_scale4_fp8keys"])


def _bench_decode_check(qsa, name):
    """One decode step of the benchmark's own runner (its caches, layout and
    calls: paged, FP8 keys, FP8 K/V, head shape as the workload says) against
    the oracle, sequence by sequence, on the same seeded inputs."""
    import bench
    w = workloads.WORKLOADS[name]
    r = bench.DecodeRunner(w, torch.device(DEV))
    out = r.step().float().cpu().numpy()
    sel, nsel = r.sel.cpu().numpy(), r.nsel.cpu().numpy()
    qsa.qsa_check_status()
    del r
    _free()
    x = workloads.make_decode(w, device=DEV)
    fp8 = w.extra.get("keys") == "fp8"
    k, v = x["k"], x["v"]
    if w.extra.get("kv") == "fp8":
        k8, ks = workloads.to_e4m3(x["k"])
        v8, vs = workloads.to_e4m3(x["v"])
        k, v = k8.float() * ks, v8.float() * vs
        del k8, v8
    differ = {}
    for b in range(w.B):
        L = x["lens"][b]
        kr = np32(x["k_idx"][b, :L])
        kp = np.zeros((L // 4 + 1, 128), np.float32)
        kp[: L // 4] = oracle.pool_keys(kr, base=w.rope_base, pos_scale=w.pos_scale, store_fp8=fp8)
        rg = np.zeros((4, 128), np.float32)
        rg[: L - 4 * (L // 4)] = kr[4 * (L // 4):]
        oracle.pool_decode(np32(x["k_idx_new"][b]), rg, kp, L + 1, base=w.rope_base, pos_scale=w.pos_scale,
                           store_fp8=fp8)
        ref = oracle.decode(np32(x["q_idx"][b:b + 1]), kp[None], [L + 1], q=np32(x["q"][b:b + 1]),
                            k=np32(k[b:b + 1]), v=np32(v[b:b + 1]), top_k=w.top_k, base=w.rope_base,
                            pos_scale=w.pos_scale, Hq=w.Hq, Hkv=w.Hkv, d=w.d, want_scores=True)
        if not decode_selection_matches(sel[b], nsel[b], ref):
            differ[b] = ref
            continue
        err = np.abs(out[b] - ref["out"][0]).max()
        assert err <= TOL["bf16"], (b, err)
    assert len(differ) <= max(1, w.B // 16)
    if differ:
        # the attention of the same runner layout (paged / FP8 / d = 256) on the oracle's selections
        r = bench.DecodeRunner(w, torch.device(DEV))

        def attn_on(s_, n_):
            r.sel.copy_(s_)
            r.nsel.copy_(n_)
            return r.attend(), None

        stage_isolated_decode(differ, attn_on, w.B, w.top_k, TOL["bf16"])
        del r
    del x, k, v
    _free()


@pytest.mark.parametrize("name", ["decode_b64_l128k_paged", "decode_b64_l128k_fp8", "decode_b64_l128k_d256",
                                  "decode_b64_l128k_d256_fp8"])
def test_bench_decode_runner_full_size(qsa, name):
    _bench_decode_check(qsa, name)


def test_bench_prefill_1m_chunked_runner(qsa):
    """The benchmark's 1M-token prompt prefilled in 16,000-token chunks by its
    own runner (chunk offsets, growing compressed cache, score chunks and the
    CTA-per-row select of long rows) against the oracle on sampled rows: the
    first and last rows, both sides of chunk boundaries, of 131072 (32768
    blocks: the select changes kernel) and of 262144 (65536 blocks), and
    uniform rows."""
    import bench
    from qsa_testlib import selection_report
    w = workloads.WORKLOADS["prefill_l1m_chunk16k"]
    r = bench.PrefillRunner(w, torch.device(DEV))
    assert len(r.chunks) == 66
    r.step()
    qsa.qsa_check_status()
    # the runner keeps one chunk's selection: rerun the chunk of each sampled row for it
    T = w.T
    g = torch.Generator().manual_seed(5)
    rows = {0, 1, 15999, 16000, 16001, 65535, 65536, 131071, 131072, 262139, 262143, 262144, 523999, 524000,
            T - 2, T - 1}
    rows |= set(torch.randint(0, T, (10,), generator=g).tolist())
    rows = sorted(rows)
    ri = torch.tensor(rows, device=DEV)
    out = r.out[0, ri].float().cpu().numpy()
    sel = np.zeros((len(rows), w.top_k), np.int32)
    nsel = np.zeros(len(rows), np.int32)
    for c0, c1 in r.chunks:
        mine = [i for i, t in enumerate(rows) if c0 <= t < c1]
        if not mine:
            continue
        n = c1 - c0
        s, ns = r.sel[:, :n], r.nsel[:, :n]
        qsa.qsa_index_topk_prefill(r.x["q_idx"][:, c0:c1], r.k_pool, s, ns, q0=c0, top_k=w.top_k, rope=r.rope,
                                   workspace=r.ws)
        for i in mine:
            sel[i] = s[0, rows[i] - c0].cpu().numpy()
            nsel[i] = int(ns[0, rows[i] - c0])
    qsa.qsa_check_status()
    kp = oracle.pool_keys(np32(r.x["k_idx"][0]), base=w.rope_base, pos_scale=w.pos_scale)
    assert np.array_equal(np32(r.k_pool[0]), kp)
    q_idx = np32(r.x["q_idx"][0, ri])
    q = np32(r.x["q"][0, ri])
    k, v = np32(r.x["k"][0]), np32(r.x["v"][0])
    del r
    _free()
    ref = {"sel": [], "nsel": [], "kth": [], "out": []}
    for i, t in enumerate(rows):          # the oracle takes rows relative to q0: one row per call
        o = oracle.prefill_rows([0], q_idx=q_idx[i:i + 1], k_pool=kp, top_k=w.top_k, base=w.rope_base,
                                pos_scale=w.pos_scale, q=q[i:i + 1], k=k, v=v, Hq=w.Hq, Hkv=w.Hkv, d=w.d, q0=t)
        for key in ref:
            ref[key].append(o[key][0])
    ref = {key: np.stack(val) for key, val in ref.items()}

    def score_fn(idx_rows):
        res = []
        for rr in idx_rows:
            i = rows.index(rr)
            sc = oracle.prefill_rows([0], q_idx=q_idx[i:i + 1], k_pool=kp, top_k=w.top_k, base=w.rope_base,
                                     pos_scale=w.pos_scale, q0=rr, want_scores=True)["scores"][0]
            res.append(np.pad(sc, (0, kp.shape[0] - sc.shape[0]), constant_values=np.nan))
        return np.stack(res)

    exact, _, nbad = selection_report(sel, nsel, ref, score_fn, rows)
    assert nbad <= 2
    err = np.abs(out - ref["out"])[exact].max()
    assert err <= TOL["bf16"], err
