"""Pins of the CPU oracle against facts fixed by the pages and by mathematics.

Each test checks the oracle against something other than itself: a library
routine (torch's bfloat16 conversion, torch's scaled-dot-product attention),
a complex-number restatement of the rotation, a full sort, closed forms,
invariants, or the structural numbers the pages print
(tests/golden/structure.json).  No test retypes the oracle's formula.

Sources: "Qwen3.8-Flash-Next: Day-0 Support in SGLang", section "Qwen Sparse
Attention: Retrieve Coarsely, Attend Precisely"; "Qwen3.8-Flash-Next, Layer
by Layer", section "Token mixing"; flozi.net architecture guide, "How a token
moves through the model", item 2.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


def bf16(x):
    """Values of a float array after torch's float32 -> bfloat16 (RNE)."""
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).float().numpy()


def complex_rotate(x, pos, base=10000.0, pos_scale=1.0, rotary_dim=128):
    """Rotate-half RoPE restated as complex multiplication: z_i = x_i + j x_{i+R/2}
    times exp(j * angle_i)."""
    x = np.asarray(x, np.float64)
    half = rotary_dim // 2
    i = np.arange(half)
    ang = (pos / pos_scale) * base ** (-(2.0 * i) / rotary_dim)
    z = (x[..., :half] + 1j * x[..., half:rotary_dim]) * np.exp(1j * ang)
    out = x.copy()
    out[..., :half] = z.real
    out[..., half:rotary_dim] = z.imag
    return out


# ----------------------------------------------------------------------------- rounding

def test_round_bf16_ties_and_library():
    r = oracle.round_bf16
    assert r(1.0) == 1.0
    assert r(1.0 + 2.0 ** -8) == 1.0                    # tie -> even (1.0000000)
    assert r(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6    # tie -> even (1.0000010)
    assert r(1.0 + 2.0 ** -8 + 2.0 ** -40) == 1.0 + 2.0 ** -7   # above the tie
    assert r(-(1.0 + 2.0 ** -8 + 2.0 ** -40)) == -(1.0 + 2.0 ** -7)
    assert r(1.5 * 2.0 ** -133) == 2.0 ** -132         # subnormal tie -> even
    assert math.isinf(r(3.4e38))
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(20000), rng.standard_normal(2000) * 1e-39,
                        rng.standard_normal(2000) * 1e30]).astype(np.float32)
    got = np.array([r(float(v)) for v in x])
    np.testing.assert_array_equal(got, bf16(x))


# ----------------------------------------------------------------------------- RoPE

def test_rope_matches_complex_restatement_and_preserves_norm():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((64, 128)).astype(np.float32)
    pos = rng.integers(0, 1 << 20, 64)
    for base, ps, R in [(10000.0, 1.0, 128), (10000.0, 4.0, 128), (1e6, 1.0, 64)]:
        y = oracle.rope_rows(x, pos, base, ps, R)
        ref = np.stack([complex_rotate(x[i], pos[i], base, ps, R) for i in range(64)])
        np.testing.assert_allclose(y, ref, rtol=0, atol=1e-9)
        np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x.astype(np.float64), axis=1),
                                   rtol=1e-12)
        if R < 128:
            np.testing.assert_array_equal(y[:, R:], x[:, R:].astype(np.float64))


def test_rope_relative_position_invariance_and_scale():
    rng = np.random.default_rng(2)
    q = rng.standard_normal((1, 128)).astype(np.float32)
    k = rng.standard_normal((1, 128)).astype(np.float32)
    ref = None
    for delta in [0, 1, 17, 4096, 300000]:
        a = oracle.rope_rows(q, [1000 + delta])
        b = oracle.rope_rows(k, [37 + delta])
        dot = float((a * b).sum())
        ref = dot if ref is None else ref
        assert abs(dot - ref) < 1e-9 * max(1.0, abs(ref))
    # linear position scaling: pos_scale 4 at position 4p == scale 1 at p
    np.testing.assert_allclose(oracle.rope_rows(q, [4 * 12345], pos_scale=4.0),
                               oracle.rope_rows(q, [12345]), rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------- pooling

def test_pool_block0_is_the_block_mean():
    # position 0 -> no rotation; small integers keep every sum exact
    rng = np.random.default_rng(3)
    k = rng.integers(-8, 9, (4, 128)).astype(np.float32)
    out = oracle.pool_keys(k, store_bf16=True)
    np.testing.assert_array_equal(out[0], bf16(k.mean(axis=0)))


def test_pool_fp32_matches_mean_then_complex_rotation():
    rng = np.random.default_rng(4)
    n = 64 * 4
    k = rng.standard_normal((n, 128)).astype(np.float32)
    for pos0, ps in [(0, 1.0), (4 * 9999, 1.0), (1 << 20, 4.0)]:
        out = oracle.pool_keys(k, pos0=pos0, pos_scale=ps, store_bf16=False)
        kb = k.reshape(-1, 4, 128)
        m = (((kb[:, 0] + kb[:, 1]) + kb[:, 2]) + kb[:, 3]) * np.float32(0.25)   # float32 mean
        ref = np.stack([complex_rotate(m[j], pos0 + 4 * j, pos_scale=ps) for j in range(m.shape[0])])
        np.testing.assert_allclose(out, ref.astype(np.float32), rtol=2e-7, atol=1e-7)


def test_pool_bf16_is_correctly_rounded():
    rng = np.random.default_rng(5)
    k = bf16(rng.standard_normal((400, 128)))
    out = oracle.pool_keys(k, pos0=4 * 777, store_bf16=True)
    kb = k.reshape(-1, 4, 128)
    m = (((kb[:, 0] + kb[:, 1]) + kb[:, 2]) + kb[:, 3]) * np.float32(0.25)
    exact = np.stack([complex_rotate(m[j], 4 * 777 + 4 * j) for j in range(m.shape[0])])
    # representable in bf16 ...
    np.testing.assert_array_equal(bf16(out), out)
    # ... and within half an ulp of the exact value
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(exact), 1e-30))) - 7)
    assert np.all(np.abs(out - exact) <= 0.5 * ulp * (1 + 1e-9))


def test_rope_after_pooling_differs_from_rope_before_pooling():
    rng = np.random.default_rng(6)
    k = rng.standard_normal((8, 128)).astype(np.float32)
    out = oracle.pool_keys(k, store_bf16=False)
    # RoPE each token at its own position, then average
    rot = np.stack([complex_rotate(k[i], i) for i in range(8)])
    before = rot.reshape(2, 4, 128).mean(axis=1)
    assert np.max(np.abs(out[1] - before[1])) > 0.1          # block 1 differs
    # block 0: rotation at the first token's position (0) is the identity
    kb = k[:4]
    m0 = (((kb[0] + kb[1]) + kb[2]) + kb[3]) * np.float32(0.25)
    np.testing.assert_array_equal(out[0], m0)


def test_pool_rmsnorm_flag_unit_rms():
    rng = np.random.default_rng(7)
    k = rng.standard_normal((16, 128)).astype(np.float32) * 3
    out = oracle.pool_keys(k, rmsnorm=True, store_bf16=False)
    rms = np.sqrt((out.astype(np.float64) ** 2).mean(axis=1))
    np.testing.assert_allclose(rms, 1.0, rtol=1e-5)


def test_pool_offset_consistency_and_decode_ring():
    rng = np.random.default_rng(8)
    k = bf16(rng.standard_normal((64, 128)))
    full = oracle.pool_keys(k)
    part = oracle.pool_keys(k[16:], pos0=16)
    np.testing.assert_array_equal(full[4:], part)
    # incremental ring pooling equals prefill pooling
    ring = np.zeros((4, 128), np.float32)
    kp = np.zeros((16, 128), np.float32)
    for t in range(64):
        oracle.pool_decode(k[t], ring, kp, t + 1)
    np.testing.assert_array_equal(kp, full)


# ----------------------------------------------------------------------------- top-k

def _sorted_ref(s, k):
    order = sorted(range(len(s)), key=lambda b: (-s[b], b))
    sel = sorted(order[:k])
    return sel


@pytest.mark.parametrize("n,k,kind", [(0, 8, "rand"), (5, 8, "rand"), (8, 8, "rand"), (1000, 64, "rand"),
                                      (4096, 512, "rand"), (3000, 512, "ties"), (777, 100, "ties"),
                                      (2000, 512, "allequal")])
def test_topk_equals_full_sort(n, k, kind):
    rng = np.random.default_rng(n + k)
    if kind == "rand":
        s = rng.standard_normal(n)
    elif kind == "ties":
        s = rng.integers(0, 7, n).astype(np.float64)
    else:
        s = np.zeros(n)
    sel, nsel, kth, nxt = oracle.topk(s, k)
    ref = _sorted_ref(list(s), k)
    assert nsel == min(n, k)
    assert list(sel[:nsel]) == ref
    assert np.all(sel[nsel:] == -1)
    if n >= k and k > 0:
        srt = sorted(s, reverse=True)
        assert kth == srt[k - 1]
        if n > k:
            assert nxt == srt[k]


# ----------------------------------------------------------------------------- scores

def _query_raw_for(values_per_head, t, j):
    """Raw indexer query whose rotation at t is values_per_head[h] * e_j."""
    q = np.zeros((4, 128))
    for h, a in enumerate(values_per_head):
        e = np.zeros(128)
        e[j] = a
        q[h] = complex_rotate(e, -t)           # inverse rotation
    return q.astype(np.float32)


@pytest.mark.parametrize("relu,w", [(False, None), (True, None), (False, (0.5, 1.0, 2.0, 0.0)),
                                    (True, (0.5, 1.0, 2.0, 0.0))])
def test_score_closed_form(relu, w):
    # Block 0 is rotated at position 0 (identity).  The query at t = 3 sees
    # exactly block 0.  With rotated query heads a_h * e_j the score is
    # (1/sqrt(128)) * sum_h w_h phi(a_h * kbar_0[j]).
    rng = np.random.default_rng(11)
    k_raw = np.abs(rng.integers(1, 9, (4, 128))).astype(np.float32)   # positive mean
    kbar = oracle.pool_keys(k_raw, store_bf16=False)
    a = np.array([1.0, -2.0, 3.0, 0.5])
    j = 5
    q_idx = _query_raw_for(a, 3, j)[None]             # position 3 -> row 3
    q_idx = np.concatenate([np.zeros((3, 4, 128), np.float32), q_idx])
    head_w = None if w is None else np.tile(np.array(w, np.float32), (4, 1))
    res = oracle.prefill_rows([3], q_idx=q_idx, k_pool=kbar, head_w=head_w, relu=relu,
                              store_bf16=False, top_k=8, want_scores=True)
    dots = a * kbar[0, j]
    if relu:
        dots = np.maximum(dots, 0)
    ww = np.ones(4) if w is None else np.array(w)
    expect = (ww * dots).sum() / math.sqrt(128)
    assert abs(res["scores"][0, 0] - expect) <= 1e-6 * abs(expect)
    assert res["nsel"][0] == 1 and res["sel"][0, 0] == 0


def test_relu_all_negative_scores_tie_to_lowest_blocks():
    # With ReLU and every dot product negative all scores are exactly 0: the
    # tie rule must then select blocks 0..k-1.
    T, k = 4 * 300, 64
    rng = np.random.default_rng(12)
    k_raw = np.abs(rng.standard_normal((T, 128))).astype(np.float32)   # pooled keys ~ positive
    kbar = oracle.pool_keys(k_raw, store_bf16=False)
    t = T - 1
    q = np.zeros((T, 4, 128), np.float32)
    # make every rotated query head the negated mean direction -> negative dots
    direction = -np.abs(kbar).mean(axis=0)
    q[t] = _query_raw_for([1, 1, 1, 1], t, 0)[0] * 0      # zero, then fill below
    for h in range(4):
        q[t, h] = complex_rotate(direction, -t).astype(np.float32)
    res = oracle.prefill_rows([t], q_idx=q, k_pool=kbar, relu=True, store_bf16=False, top_k=k,
                              want_scores=True)
    nb = (t + 1) // 4
    assert np.all(res["scores"][0, :nb] == 0.0)
    assert list(res["sel"][0]) == list(range(k))


# ----------------------------------------------------------------------------- counts / structure

def test_selection_structure_matches_pages():
    gold = json.load(open(os.path.join(HERE, "golden", "structure.json")))
    B4 = gold["block_tokens"]["value"]
    K = gold["top_k_blocks"]["value"]
    assert K * B4 == gold["selected_tokens"]["value"]
    T = 4 * 600
    rng = np.random.default_rng(13)
    k_raw = bf16(rng.standard_normal((T, 128)))
    q_idx = bf16(rng.standard_normal((T, 4, 128)))
    kbar = oracle.pool_keys(k_raw)
    rows = [0, 1, 2, 3, 4, 7, 2046, 2047, 2048, 2049, 2050, 2051, 2052, T - 4, T - 3, T - 2, T - 1]
    res = oracle.prefill_rows(rows, q_idx=q_idx, k_pool=kbar, top_k=K)
    max_pos = 0
    for r, t in enumerate(rows):
        nb = (t + 1) // B4
        tail = t + 1 - B4 * nb
        nsel = res["nsel"][r]
        sel = res["sel"][r, :nsel]
        assert nsel == min(K, nb)
        assert len(set(sel.tolist())) == nsel and np.all(np.diff(sel) > 0)
        assert np.all((sel >= 0) & (sel < nb))
        assert 0 <= tail <= gold["tail_tokens_max"]["value"]
        npos = B4 * nsel + tail
        max_pos = max(max_pos, npos)
        assert npos <= gold["max_positions"]["value"]
    # t = T-2 = 2398: 599 complete blocks (>= 512) and a 3-token tail -> 2051 positions
    assert max_pos == gold["max_positions"]["value"]
    assert gold["index_query_heads"]["value"] == oracle.IDX_HEADS
    assert gold["index_dim"]["value"] == oracle.IDX_DIM


# ----------------------------------------------------------------------------- attention

def _sdpa_causal(q, k, v, Hq, Hkv):
    """torch's scaled-dot-product attention (fp64, CPU) with a causal mask."""
    qt = torch.from_numpy(q.astype(np.float64)).permute(1, 0, 2)[None]      # [1][Hq][T][d]
    kt = torch.from_numpy(k.astype(np.float64)).permute(1, 0, 2)[None]
    vt = torch.from_numpy(v.astype(np.float64)).permute(1, 0, 2)[None]
    rep = Hq // Hkv
    kt = kt.repeat_interleave(rep, dim=1)
    vt = vt.repeat_interleave(rep, dim=1)
    o = F.scaled_dot_product_attention(qt, kt, vt, is_causal=True)
    return o[0].permute(1, 0, 2).numpy()                                     # [T][Hq][d]


@pytest.mark.parametrize("T,k,Hq,Hkv", [(1024, 256, 8, 1), (2048, 512, 16, 2), (259, 64, 4, 2)])
def test_qsa_equals_dense_causal_when_every_block_fits(T, k, Hq, Hkv):
    # When k >= nb(t) for every row the selection is every visible block plus
    # the tail, i.e. positions 0..t: QSA reduces to full causal attention.
    assert k >= T // 4
    rng = np.random.default_rng(T + k)
    d = 128
    q_idx = bf16(rng.standard_normal((T, 4, 128)))
    kbar = oracle.pool_keys(bf16(rng.standard_normal((T, 128))))
    q = bf16(rng.standard_normal((T, Hq, d)))
    kk = bf16(rng.standard_normal((T, Hkv, d)))
    v = bf16(rng.standard_normal((T, Hkv, d)))
    ref = _sdpa_causal(q, kk, v, Hq, Hkv)
    rows = np.unique(np.concatenate([np.arange(0, 8), np.arange(T - 8, T),
                                     rng.integers(0, T, 48)]))
    res = oracle.prefill_rows(rows, q_idx=q_idx, k_pool=kbar, top_k=k, q=q, k=kk, v=v,
                              Hq=Hq, Hkv=Hkv, d=d)
    np.testing.assert_allclose(res["out"], ref[rows], rtol=0, atol=1e-10)
    dense = oracle.dense_rows(rows, q, kk, v, Hq, Hkv, d)
    np.testing.assert_allclose(dense, ref[rows], rtol=0, atol=1e-10)


def test_dense_rows_with_a_chunk_offset_match_the_full_sequence():
    # rows of a chunk starting at q0 attend over positions 0 .. q0 + i: they are
    # rows q0 + i of textbook causal attention over the whole sequence
    T, q0, Hq, Hkv, d = 300, 203, 8, 2, 128
    rng = np.random.default_rng(77)
    q = bf16(rng.standard_normal((T, Hq, d)))
    kk = bf16(rng.standard_normal((T, Hkv, d)))
    v = bf16(rng.standard_normal((T, Hkv, d)))
    ref = _sdpa_causal(q, kk, v, Hq, Hkv)
    rows = np.arange(T - q0)
    dense = oracle.dense_rows(rows, q[q0:], kk, v, Hq, Hkv, d, q0=q0)
    np.testing.assert_allclose(dense, ref[q0:], rtol=0, atol=1e-10)


def test_attention_special_cases():
    T, Hq, Hkv, d = 64, 4, 2, 128
    rng = np.random.default_rng(21)
    q = rng.standard_normal((T, Hq, d)).astype(np.float32)
    k = rng.standard_normal((T, Hkv, d)).astype(np.float32)
    v = rng.standard_normal((T, Hkv, d)).astype(np.float32)
    # t = 0 attends to itself only: o = v_0 of the head's kv group
    res = oracle.prefill_rows([0], q=q, k=k, v=v, Hq=Hq, Hkv=Hkv, d=d, top_k=4,
                              sel_in=np.full((1, 4), -1, np.int32), nsel_in=np.zeros(1, np.int32))
    for h in range(Hq):
        np.testing.assert_allclose(res["out"][0, h], v[0, h * Hkv // Hq], rtol=0, atol=1e-12)
    # constant keys: uniform softmax -> mean of V over P(t)
    kc = np.ones_like(k)
    t = 41                                      # nb = 10, tail = 2 (positions 40, 41)
    sel = np.array([[1, 4, 7, -1]], np.int32)
    res = oracle.prefill_rows([t], q=q, k=kc, v=v, Hq=Hq, Hkv=Hkv, d=d, top_k=4, sel_in=sel,
                              nsel_in=np.array([3], np.int32))
    pos = [4, 5, 6, 7, 16, 17, 18, 19, 28, 29, 30, 31, 40, 41]
    for h in range(Hq):
        g = h * Hkv // Hq
        np.testing.assert_allclose(res["out"][0, h], v[pos, g].astype(np.float64).mean(axis=0),
                                   rtol=0, atol=1e-12)
        # lse of equal logits = logit + log(|P|)
        logit = float(np.dot(q[t, h].astype(np.float64), kc[0, g].astype(np.float64))) / math.sqrt(d)
        assert abs(res["lse"][0, h] - (logit + math.log(len(pos)))) < 1e-9


# ----------------------------------------------------------------------------- decode vs prefill

def test_decode_step_equals_prefill_row():
    T, k, Hq, Hkv, d = 4 * 150 + 2, 64, 4, 2, 128
    rng = np.random.default_rng(31)
    q_idx = bf16(rng.standard_normal((T, 4, 128)))
    k_raw = bf16(rng.standard_normal((T, 128)))
    q = bf16(rng.standard_normal((T, Hq, d)))
    kk = bf16(rng.standard_normal((T, Hkv, d)))
    v = bf16(rng.standard_normal((T, Hkv, d)))
    kbar = oracle.pool_keys(k_raw)
    for t in [T - 1, T - 2, T - 3, T - 4, 100, 3, 0]:
        # decode: cache of t tokens + the new one at position t
        ring = np.zeros((4, 128), np.float32)
        kp = np.zeros((T // 4 + 1, 128), np.float32)
        for s in range(t + 1):
            oracle.pool_decode(k_raw[s], ring, kp, s + 1)
        dec = oracle.decode(q_idx[t][None], kp[None], [t + 1], q=q[t][None], k=kk[None], v=v[None],
                            top_k=k, Hq=Hq, Hkv=Hkv, d=d, want_scores=True)
        pre = oracle.prefill_rows([t], q_idx=q_idx, k_pool=kbar, top_k=k, q=q, k=kk, v=v,
                                  Hq=Hq, Hkv=Hkv, d=d, want_scores=True)
        nb = (t + 1) // 4
        if nb:   # the scores the decode selection ranked are the prefill row's
            np.testing.assert_array_equal(dec["scores"][0][:nb], pre["scores"][0][:nb])
        assert dec["nsel"][0] == pre["nsel"][0]
        np.testing.assert_array_equal(dec["sel"][0], pre["sel"][0])
        np.testing.assert_array_equal(dec["out"][0], pre["out"][0])


# ----------------------------------------------------------------------------- needles

def test_needle_recall_small():
    import workloads
    w = workloads.Workload("needles_small", "prefill", 1, 8192, 512, 4, 1, 128, "bf16", 77, needles=16)
    x = workloads.make_prefill(w, device="cpu")
    q_idx = x["q_idx"][0].float().numpy()
    k_raw = x["k_idx"][0].float().numpy()
    kbar = oracle.pool_keys(k_raw)
    rows, blocks = [], []
    for b, ts in x["needles"]:
        for t in ts:
            rows.append(t)
            blocks.append(b)
    res = oracle.prefill_rows(rows, q_idx=q_idx, k_pool=kbar, top_k=w.top_k)
    for r, b in enumerate(blocks):
        assert b in set(res["sel"][r, :res["nsel"][r]].tolist())


# ----------------------------------------------------------------------------- IndexShare draft steps

def _pooled_cache(k_raw, n_tok, cap):
    """Compressed keys of the first n_tok raw keys (complete blocks only)."""
    kp = np.zeros((cap, 128), np.float32)
    nb = n_tok // 4
    if nb:
        kp[:nb] = oracle.pool_keys(k_raw[:4 * nb])
    return kp


@pytest.mark.parametrize("t_c,drafts", [(4 * 300 + 2, [0, 1, 2, 5, 9]), (4 * 300 + 3, [0, 1, 4, 8]),
                                         (4 * 300, [0, 3, 6])])
def test_indexshare_draft_equals_dense_when_every_block_fits(t_c, drafts):
    # With k >= nb(t_c) the frozen selection is every block visible to the
    # capture row, and the draft step adds t_c's incomplete block and every
    # drafted position: positions 0..t, i.e. full causal attention at t.
    T = t_c + max(drafts) + 1
    Hq, Hkv, d, k = 8, 2, 128, 512
    assert k >= (t_c + 1) // 4
    rng = np.random.default_rng(t_c)
    k_raw = bf16(rng.standard_normal((T, 128)))
    q_idx = bf16(rng.standard_normal((T, 4, 128)))
    q = bf16(rng.standard_normal((T, Hq, d)))
    kk = bf16(rng.standard_normal((T, Hkv, d)))
    v = bf16(rng.standard_normal((T, Hkv, d)))
    ref = _sdpa_causal(q, kk, v, Hq, Hkv)
    kp = _pooled_cache(k_raw, t_c + 1, T // 4 + 1)
    for j in drafts:
        t = t_c + j
        res = oracle.decode(q_idx[t_c][None], kp[None], [t + 1], cap_len=[t_c + 1], q=q[t][None], k=kk[None],
                            v=v[None], top_k=k, Hq=Hq, Hkv=Hkv, d=d)
        assert res["nsel"][0] == (t_c + 1) // 4
        np.testing.assert_allclose(res["out"][0], ref[t], rtol=0, atol=1e-12)


def test_indexshare_capture_row_is_a_plain_decode_step():
    # At t == t_c the draft step reads the capture row's own selection and tail.
    T, k, Hq, Hkv, d = 4 * 200 + 1, 32, 4, 1, 128
    rng = np.random.default_rng(5)
    k_raw = bf16(rng.standard_normal((T, 128)))
    q_idx = bf16(rng.standard_normal((T, 4, 128)))
    q = bf16(rng.standard_normal((T, Hq, d)))
    kk = bf16(rng.standard_normal((T, Hkv, d)))
    v = bf16(rng.standard_normal((T, Hkv, d)))
    t = T - 1
    kp = _pooled_cache(k_raw, T, T // 4 + 1)
    plain = oracle.decode(q_idx[t][None], kp[None], [T], q=q[t][None], k=kk[None], v=v[None], top_k=k, Hq=Hq,
                          Hkv=Hkv, d=d)
    shared = oracle.decode(q_idx[t][None], kp[None], [T], cap_len=[T], q=q[t][None], k=kk[None], v=v[None],
                           top_k=k, Hq=Hq, Hkv=Hkv, d=d)
    np.testing.assert_array_equal(plain["sel"], shared["sel"])
    np.testing.assert_array_equal(plain["out"], shared["out"])


def test_indexshare_keeps_the_frozen_selection_and_sees_drafted_positions():
    # The draft step at t = t_c + 3 must (1) attend over the blocks selected for
    # t_c, not re-select, and (2) see the drafted positions t_c + 1 .. t: a key
    # planted only at a drafted position, aligned with the query, carries its
    # value to the output.
    T, k, Hq, Hkv, d = 4 * 400 + 2, 16, 1, 1, 128
    rng = np.random.default_rng(9)
    k_raw = bf16(rng.standard_normal((T + 8, 128)))
    q_idx = bf16(rng.standard_normal((T + 8, 4, 128)))
    q = bf16(rng.standard_normal((T + 8, Hq, d)) * 0.1)
    kk = bf16(rng.standard_normal((T + 8, Hkv, d)) * 0.1)
    v = np.zeros((T + 8, Hkv, d), np.float32)
    t_c, t = T - 1, T + 2
    u = np.zeros(d, np.float32)
    u[7] = 1.0
    q[t, 0] = 30.0 * u
    kk[t_c + 2, 0] = 30.0 * u          # drafted position
    v[t_c + 2, 0, 3] = 1.0
    kp = _pooled_cache(k_raw, T, (T + 8) // 4 + 1)
    res = oracle.decode(q_idx[t_c][None], kp[None], [t + 1], cap_len=[t_c + 1], q=q[t][None], k=kk[None],
                        v=v[None], top_k=k, Hq=Hq, Hkv=Hkv, d=d)
    cap = oracle.decode(q_idx[t_c][None], kp[None], [t_c + 1], top_k=k)
    np.testing.assert_array_equal(res["sel"], cap["sel"])          # frozen, not re-selected
    assert res["out"][0, 0, 3] > 0.99                                # the drafted key wins


# ----------------------------------------------------------------------------- FP8 E4M3 storage

def _e4m3_codes():
    """Every finite E4M3 value, from the bit layout (1 sign, 4 exponent bits with
    bias 7, 3 mantissa bits; exponent 15 with mantissa 7 is NaN)."""
    vals = []
    for e in range(16):
        for m in range(8):
            if e == 15 and m == 7:
                continue
            v = (m / 8.0) * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7)
            vals.append(v)
    pos = sorted(set(vals))
    return np.array(sorted(set([-v for v in pos] + pos)))


def test_e4m3_code_points_round_trip_and_max():
    codes = _e4m3_codes()
    assert codes.max() == 448.0 and len(codes) == 253      # 126 positive, 126 negative, zero
    np.testing.assert_array_equal(oracle.round_e4m3(codes), codes)


def test_e4m3_ties_to_even_and_nearest():
    pos = _e4m3_codes()
    pos = pos[pos >= 0]
    lo, hi = pos[:-1], pos[1:]
    mid = (lo + hi) / 2
    # the code of a value is even iff its mantissa's last bit is 0; consecutive
    # codes alternate, starting with 0 (even)
    even_lo = (np.arange(len(lo)) % 2) == 0
    exp_tie = np.where(even_lo, lo, hi)
    np.testing.assert_array_equal(oracle.round_e4m3(mid), exp_tie)
    np.testing.assert_array_equal(oracle.round_e4m3(-mid), -exp_tie)
    eps = (hi - lo) * 1e-3
    np.testing.assert_array_equal(oracle.round_e4m3(mid - eps), lo)
    np.testing.assert_array_equal(oracle.round_e4m3(mid + eps), hi)


def test_e4m3_saturates_and_matches_torch_in_range():
    np.testing.assert_array_equal(oracle.round_e4m3([448.0, 460.0, 464.0, 500.0, 1e9, np.inf, -np.inf]),
                                  [448.0, 448.0, 448.0, 448.0, 448.0, 448.0, -448.0])
    rng = np.random.default_rng(2)
    x = (rng.standard_normal(20000) * np.exp(rng.uniform(-8, 5, 20000))).astype(np.float32)
    x = x[np.abs(x) < 440]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).float().numpy()
    np.testing.assert_array_equal(oracle.round_e4m3(x.astype(np.float64)), ref)


def test_pooled_keys_in_fp8_are_the_rounded_bf16_free_values():
    # FP8 storage rounds the same fp64 rotated mean that BF16 storage rounds:
    # pooled FP32 keys (no storage rounding) rounded to E4M3 equal the FP8 path.
    rng = np.random.default_rng(4)
    k_raw = bf16(rng.standard_normal((4 * 300, 128)))
    exact = oracle.pool_keys(k_raw, store_bf16=False)       # fp32 store of the fp64 value
    fp8 = oracle.pool_keys(k_raw, store_fp8=True)
    codes = set(_e4m3_codes().tolist())
    assert set(np.unique(fp8).tolist()) <= codes
    # fp32 storage is within half an fp32 ulp of the fp64 value, so re-rounding
    # it to E4M3 differs only where it straddles an E4M3 midpoint: never here
    np.testing.assert_array_equal(oracle.round_e4m3(exact.astype(np.float64)), fp8)
