"""Seeded synthetic workloads for QSA (shared by the tests and the benchmark).

This module only draws inputs.  It computes no output of the method: no
pooling, scoring, selection or attention.  The one piece of arithmetic it
carries is the inverse position rotation used to plant "needles" whose
direction must survive the rotation the method applies; it builds inputs and
is written here on its own, independent of the oracle and of the CUDA path.

Workload shapes follow the pages ("Qwen3.8-Flash-Next: Day-0 Support in
SGLang", "Qwen Sparse Attention: Retrieve Coarsely, Attend Precisely";
"Qwen3.8-Flash-Next, Layer by Layer", "Token mixing"): an indexer of 4 query
heads and one shared 128-dim key head, blocks of 4 tokens, top-512 blocks.

Conventions
  * indexer inputs are RAW (before RoPE): the method rotates them itself;
  * attention q and k are given AFTER the attention layer's RoPE (the sparse
    attention consumes rotated q/k, as a paged KV cache stores them);
  * all tensors are contiguous: q_idx [B][T][4][128], k_idx [B][T][128],
    q [B][T][Hq][d], k/v [B][T][Hkv][d].
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

IDX_HEADS = 4
IDX_DIM = 128
BLOCK = 4


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str                 # "prefill", "decode", "draft" (IndexShare draft step after a decode capture)
                              # or "dense" (full causal decode attention, the baseline QSA replaces)
    B: int
    T: int                    # prefill tokens, or decode cache length before the new token
    top_k: int
    Hq: int
    Hkv: int
    d: int
    dtype: str                # "bf16" or "fp32"
    seed: int
    rope_base: float = 10000.0
    pos_scale: float = 1.0
    needles: int = 0
    heavy_tail: bool = False
    extra: dict = field(default_factory=dict)


WORKLOADS = {
    "tiny_prefill_t1k_fp32": Workload("tiny_prefill_t1k_fp32", "prefill", 1, 1024, 64, 8, 1, 128,
                                      "fp32", 1001),
    "prefill_t32k_needles": Workload("prefill_t32k_needles", "prefill", 1, 32768, 512, 16, 2, 128,
                                     "bf16", 1002, needles=64),
    "decode_b64_l128k": Workload("decode_b64_l128k", "decode", 64, 131072, 512, 16, 2, 128,
                                 "bf16", 1003),
    "prefill_t128k_heavytail": Workload("prefill_t128k_heavytail", "prefill", 1, 131072, 512, 16, 2,
                                        128, "bf16", 1004, heavy_tail=True),
    "decode_b8_l1m_scale4": Workload("decode_b8_l1m_scale4", "decode", 8, 1048576, 512, 16, 2, 128,
                                     "bf16", 1005, pos_scale=4.0),
    # the decode workloads with the compressed keys stored as FP8 E4M3 (same data and seeds)
    "decode_b64_l128k_fp8keys": Workload("decode_b64_l128k_fp8keys", "decode", 64, 131072, 512, 16, 2, 128,
                                         "bf16", 1003, extra={"keys": "fp8"}),
    "decode_b8_l1m_scale4_fp8keys": Workload("decode_b8_l1m_scale4_fp8keys", "decode", 8, 1048576, 512, 16, 2,
                                             128, "bf16", 1005, pos_scale=4.0, extra={"keys": "fp8"}),
    # FP8 serving configuration: FP8 E4M3 compressed keys and FP8 E4M3 K/V caches (per-tensor scales)
    "decode_b64_l128k_fp8": Workload("decode_b64_l128k_fp8", "decode", 64, 131072, 512, 16, 2, 128, "bf16", 1003,
                                     extra={"keys": "fp8", "kv": "fp8"}),
    "decode_b8_l1m_scale4_fp8": Workload("decode_b8_l1m_scale4_fp8", "decode", 8, 1048576, 512, 16, 2, 128, "bf16",
                                         1005, pos_scale=4.0, extra={"keys": "fp8", "kv": "fp8"}),
    # the 32K prefill workload with FP8 E4M3 K/V caches
    "prefill_t32k_needles_kv8": Workload("prefill_t32k_needles_kv8", "prefill", 1, 32768, 512, 16, 2, 128, "bf16",
                                         1002, needles=64, extra={"kv": "fp8"}),
    # full causal prefill attention on the QSA prefill workloads' q/k/v (the dense baseline)
    "dense_prefill_t32k": Workload("dense_prefill_t32k", "dense_prefill", 1, 32768, 512, 16, 2, 128, "bf16", 1002,
                                   needles=64),
    "dense_prefill_t128k": Workload("dense_prefill_t128k", "dense_prefill", 1, 131072, 512, 16, 2, 128, "bf16",
                                    1004, heavy_tail=True),
    # a 1M-token prompt prefilled in chunks of 16,000 tokens (the pages' speed comparison), QSA and full
    # attention on the same inputs (heavy-tailed like the 128K workload)
    "prefill_l1m_chunk16k": Workload("prefill_l1m_chunk16k", "prefill", 1, 1048576, 512, 16, 2, 128, "bf16", 1007,
                                     heavy_tail=True, extra={"chunk": 16000}),
    "dense_prefill_l1m_chunk16k": Workload("dense_prefill_l1m_chunk16k", "dense_prefill", 1, 1048576, 512, 16, 2,
                                           128, "bf16", 1007, heavy_tail=True, extra={"chunk": 16000}),
    # the released model's attention shape: 24 q heads, 2 kv heads of 256 dims (BF16, and the FP8 serving form)
    "prefill_t32k_d256": Workload("prefill_t32k_d256", "prefill", 1, 32768, 512, 24, 2, 256, "bf16", 1002,
                                  needles=64),
    "decode_b64_l128k_d256": Workload("decode_b64_l128k_d256", "decode", 64, 131072, 512, 24, 2, 256, "bf16", 1003),
    "decode_b64_l128k_d256_fp8": Workload("decode_b64_l128k_d256_fp8", "decode", 64, 131072, 512, 24, 2, 256, "bf16",
                                          1003, extra={"keys": "fp8", "kv": "fp8"}),
    # the 128K decode workload over paged caches (64-token pages, shuffled page pool)
    "decode_b64_l128k_paged": Workload("decode_b64_l128k_paged", "decode", 64, 131072, 512, 16, 2, 128, "bf16",
                                       1003, extra={"page_tokens": 64}),
    # full causal decode attention on the same caches as the QSA decode workloads
    "dense_b64_l128k": Workload("dense_b64_l128k", "dense", 64, 131072, 512, 16, 2, 128, "bf16", 1003),
    "dense_b8_l1m_scale4": Workload("dense_b8_l1m_scale4", "dense", 8, 1048576, 512, 16, 2, 128, "bf16", 1005,
                                    pos_scale=4.0),
    # IndexShare draft step: 3 positions drafted since the capture row (at most 4)
    "draft_b64_l128k": Workload("draft_b64_l128k", "draft", 64, 131072, 512, 16, 2, 128, "bf16", 1006,
                                extra={"drafted": 3, "max_draft": 4}),
}


def to_e4m3(t: torch.Tensor):
    """A per-tensor FP8 E4M3 cache of t: (values / scale) rounded to E4M3, and
    scale = amax / 448, so that scale * cache approximates t."""
    scale = float(t.float().abs().max()) / 448.0
    return (t.float() / scale).to(torch.float8_e4m3fn), scale


def torch_dtype(w: Workload):
    return torch.bfloat16 if w.dtype == "bf16" else torch.float32


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randn(shape, g, device, dtype=torch.float32):
    return torch.randn(shape, generator=g, device=device, dtype=dtype)


def _heavy_scale(n, g, device):
    """Per-vector norm multiplier s = u^(-1/1.5), u ~ U(0,1], clipped at 64
    (a Pareto tail with alpha = 1.5)."""
    u = torch.rand(n, generator=g, device=device, dtype=torch.float32)
    u = 1.0 - u                      # (0, 1]
    return torch.clamp(u.pow(-1.0 / 1.5), max=64.0)


def _inverse_rotation(u: torch.Tensor, pos: torch.Tensor, base: float, pos_scale: float) -> torch.Tensor:
    """Return x with rotate-half rotation R(pos) x == u (fp64), batched:
    u [..., 128], pos broadcastable to u[..., 0].  Pairs (i, i + 64) turn by
    (pos / pos_scale) * base^(-2i/128); the inverse turns by the negative
    angle."""
    half = IDX_DIM // 2
    i = torch.arange(half, dtype=torch.float64, device=u.device)
    inv_freq = torch.pow(torch.tensor(base, dtype=torch.float64, device=u.device), -(2.0 * i) / IDX_DIM)
    ang = (pos.to(torch.float64) / pos_scale).unsqueeze(-1) * inv_freq
    c, s = torch.cos(-ang), torch.sin(-ang)
    a, b = u[..., :half], u[..., half:]
    return torch.cat([a * c - b * s, b * c + a * s], dim=-1)


def make_prefill(w: Workload, device="cuda", T: int | None = None):
    """Inputs of a prefill workload (optionally truncated to T tokens).

    Returns dict(q_idx, k_idx, q, k, v, needles) with needles a list of
    (block, [query positions]) when the workload plants them.
    """
    assert w.kind in ("prefill", "dense_prefill")
    T = T or w.T
    g = _gen(device, w.seed)
    B = w.B
    dt = torch_dtype(w)
    q_idx = _randn((B, T, IDX_HEADS, IDX_DIM), g, device)
    k_idx = _randn((B, T, IDX_DIM), g, device)
    q = _randn((B, T, w.Hq, w.d), g, device)
    k = _randn((B, T, w.Hkv, w.d), g, device)
    v = _randn((B, T, w.Hkv, w.d), g, device)
    needles = []
    if w.heavy_tail:
        k_idx *= _heavy_scale(B * T, g, device).view(B, T, 1)
        k *= _heavy_scale(B * T * w.Hkv, g, device).view(B, T, w.Hkv, 1)
    if w.needles:
        needles = _plant_needles(w, T, g, device, q_idx, k_idx, q, k)
    return dict(q_idx=q_idx.to(dt).contiguous(), k_idx=k_idx.to(dt).contiguous(),
                q=q.to(dt).contiguous(), k=k.to(dt).contiguous(), v=v.to(dt).contiguous(),
                needles=needles)


def _plant_needles(w, T, g, device, q_idx, k_idx, q, k, alpha=8.0, beta=8.0, per_needle=16,
                   min_query=2048):
    """Plant `w.needles` blocks whose indexer keys (after the method's pooling
    and rotation) point along a unit direction u_j, and add beta * u_j (in
    the rotated frame) to the indexer queries of up to 16 later positions per
    needle, drawn from [max(min_query, 4b+4), T).  The attention keys of the
    block and the queries at those positions get a shared direction too, so
    the attention mass follows the needle.  Needles need T > min_query + 4.
    Vectorised: a handful of kernel launches whatever the needle count."""
    n = w.needles
    hi = (T - 4) // BLOCK
    blocks = torch.randperm(hi, generator=g, device=device)[:n]
    lo = torch.clamp(BLOCK * blocks + BLOCK, min=min_query)
    keep = lo < T
    blocks, lo = blocks[keep], lo[keep]
    n = int(blocks.numel())
    u = _randn((n, IDX_DIM), g, device).double()
    u = u / u.norm(dim=-1, keepdim=True)
    ua = _randn((n, w.d), g, device).double()
    ua = ua / ua.norm(dim=-1, keepdim=True)
    span = (T - lo).to(torch.float64)
    ts = lo.unsqueeze(1) + torch.floor(torch.rand((n, per_needle), generator=g, device=device,
                                                  dtype=torch.float64) * span.unsqueeze(1)).long()
    noise_k = 0.1 * _randn((n, BLOCK, IDX_DIM), g, device).double()
    noise_a = 0.1 * _randn((n, BLOCK, w.Hkv, w.d), g, device).double()
    tok = (BLOCK * blocks).unsqueeze(1) + torch.arange(BLOCK, device=device)          # [n][4]
    kvec = alpha * _inverse_rotation(u, (BLOCK * blocks).to(torch.float64), w.rope_base, w.pos_scale)
    kvec = kvec.unsqueeze(1) + noise_k                                                  # [n][4][128]
    avec = alpha * ua[:, None, None, :] + noise_a                                        # [n][4][Hkv][d]
    # unique (needle, query position) pairs
    pair = torch.unique(torch.stack([torch.arange(n, device=device).unsqueeze(1).expand(n, per_needle), ts],
                                    dim=-1).view(-1, 2), dim=0)
    j, t = pair[:, 0], pair[:, 1]
    qadd = beta * _inverse_rotation(u[j], t.to(torch.float64), w.rope_base, w.pos_scale)   # [m][128]
    for bi in range(w.B):
        k_idx[bi].index_copy_(0, tok.reshape(-1), kvec.reshape(-1, IDX_DIM).float())
        k[bi].index_copy_(0, tok.reshape(-1), avec.reshape(-1, w.Hkv, w.d).float())
        q_idx[bi].index_add_(0, t, qadd.float().unsqueeze(1).expand(-1, IDX_HEADS, IDX_DIM).contiguous())
        q[bi].index_add_(0, t, (beta * ua[j]).float().unsqueeze(1).expand(-1, w.Hq, w.d).contiguous())
    bl = blocks.tolist()
    tl = [[] for _ in range(n)]
    for jj, tt in zip(j.tolist(), t.tolist()):
        tl[jj].append(tt)
    return [(bl[i], sorted(tl[i])) for i in range(n)]


def make_decode(w: Workload, device="cuda", L: int | None = None, B: int | None = None,
                ragged: bool = False):
    """Inputs of a decode workload.

    Each sequence i has a cache of L_i tokens before the new one (L, or with
    ragged=True L - (i mod 4), which covers tails 0..3 and in-step pooling).
    Returns dict(k_idx [B][Lmax][128] raw indexer keys of the cache,
                 q_idx [B][4][128], k_idx_new [B][128] raw indexer key of the
                 new token, q [B][Hq][d], k, v [B][Lmax+1][Hkv][d] caches that
                 already hold the new token at position L_i, seq_len [B]
                 int32 = L_i + 1).  Draft workloads ("drafted" in extra) get
    extra[drafted] more cache rows: the positions drafted after the new token.
    """
    assert w.kind in ("decode", "draft", "dense")
    L = L or w.T
    B = B or w.B
    g = _gen(device, w.seed)
    dt = torch_dtype(w)
    lens = [max(0, L - (i % 4 if ragged else 0)) for i in range(B)]
    Lmax = max(lens)
    extra = int(w.extra.get("drafted", 0))   # draft workloads: cache rows for the drafted positions
    k_idx = _randn((B, Lmax, IDX_DIM), g, device, dt)
    q_idx = _randn((B, IDX_HEADS, IDX_DIM), g, device, dt)
    k_idx_new = _randn((B, IDX_DIM), g, device, dt)
    q = _randn((B, w.Hq, w.d), g, device, dt)
    k = _randn((B, Lmax + 1 + extra, w.Hkv, w.d), g, device, dt)
    v = _randn((B, Lmax + 1 + extra, w.Hkv, w.d), g, device, dt)
    seq_len = torch.tensor([x + 1 for x in lens], dtype=torch.int32, device=device)
    return dict(k_idx=k_idx, q_idx=q_idx, k_idx_new=k_idx_new, q=q, k=k, v=v, seq_len=seq_len,
                lens=lens)


def sample_rows(T: int, needles=(), n_uniform: int = 2048, seed: int = 7) -> list[int]:
    """Query rows checked at full size: the first and last 16, four around
    every multiple of 2048, all needle queries, and n_uniform uniform rows."""
    rows = set(range(min(16, T))) | set(range(max(0, T - 16), T))
    for m in range(2048, T, 2048):
        rows |= {m - 2, m - 1, m, m + 1}
    for _, ts in needles:
        rows |= set(ts)
    g = torch.Generator().manual_seed(seed)
    rows |= set(torch.randint(0, T, (n_uniform,), generator=g).tolist())
    return sorted(r for r in rows if 0 <= r < T)


def scale_default(d: int) -> float:
    return 1.0 / math.sqrt(d)
