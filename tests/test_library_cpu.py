"""Host-side checks of the C-ABI library that need no GPU: it builds, loads,
exports every entry point include/qsa.h declares, and rejects invalid
arguments before launching anything."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qsa.h")


def declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^QSA_API\s+[\w\s\*]+?\b(qsa_\w+)\s*\(", src, flags=re.M)))


@pytest.fixture(scope="module")
def qsa():
    import __graft_entry__
    __graft_entry__._load_build_module().build()
    import block_sparse_attention_11_b200 as m
    return m


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ["qsa_pool_keys_prefill", "qsa_pool_keys_decode", "qsa_index_topk_prefill", "qsa_index_topk_decode",
              "qsa_sparse_attn_prefill", "qsa_sparse_attn_decode", "qsa_check_status", "qsa_rope_apply"]:
        assert n in names


def test_library_exports_every_declared_symbol(qsa):
    lib = ctypes.CDLL(qsa.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, f"not exported: {missing}"


def test_strerror_and_version(qsa):
    assert qsa.qsa_strerror(0) == "ok"
    assert "invalid" in qsa.qsa_strerror(1)
    assert qsa.qsa_strerror(99) == "unknown status"
    assert qsa.qsa_version() >= 100


def test_invalid_arguments_are_rejected_before_launch(qsa):
    lib = qsa.lib
    rope = qsa.Rope().c()
    # null pointers
    assert lib.qsa_pool_keys_prefill(None, None, 1, 16, 0, 16, 4, rope, 0, 0, None) == qsa.QSA_ERR_INVALID_ARG
    assert lib.qsa_pool_keys_prefill(None, None, 1, 3, 0, 3, 0, rope, 0, 0, None) == qsa.QSA_OK   # nothing to pool
    # pos0 not a multiple of 4 (checked before any pointer is touched)
    fake = ctypes.c_void_p(4096)
    assert lib.qsa_pool_keys_prefill(fake, fake, 1, 16, 2, 16, 8, rope, 0, 0, None) == qsa.QSA_ERR_INVALID_ARG
    # pooled cache too small
    assert lib.qsa_pool_keys_prefill(fake, fake, 1, 16, 0, 16, 3, rope, 0, 0, None) == qsa.QSA_ERR_INVALID_ARG
    # unknown flag bits
    assert lib.qsa_pool_keys_prefill(fake, fake, 1, 16, 0, 16, 4, rope, 8, 0, None) == qsa.QSA_ERR_INVALID_ARG
    # unsupported dtype
    assert lib.qsa_pool_keys_prefill(fake, fake, 1, 16, 0, 16, 4, rope, 0, 7, None) == qsa.QSA_ERR_UNSUPPORTED
    # rope: unsupported style, bad rotary_dim
    bad_style = qsa.Rope(style=1).c()
    assert lib.qsa_pool_keys_prefill(fake, fake, 1, 16, 0, 16, 4, bad_style, 0, 0, None) == qsa.QSA_ERR_UNSUPPORTED
    bad_dim = qsa.Rope(rotary_dim=20).c()
    assert lib.qsa_pool_keys_prefill(fake, fake, 1, 16, 0, 16, 4, bad_dim, 0, 0, None) == qsa.QSA_ERR_INVALID_ARG
    # top_k out of range
    assert lib.qsa_index_topk_prefill(fake, fake, None, 1, 16, 0, 4, 0, fake, fake, fake, 1 << 20, rope, 0, 0,
                                      None) == qsa.QSA_ERR_INVALID_ARG
    # attention: bf16 needs GQA ratio 8, d = 128
    assert lib.qsa_sparse_attn_prefill(fake, fake, fake, fake, fake, 1, 4, 0, 4, 16, 4, 128, 8, 0.1, fake, None,
                                       None, 0, 0, None) == qsa.QSA_ERR_UNSUPPORTED
    assert lib.qsa_sparse_attn_prefill(fake, fake, fake, fake, fake, 1, 4, 0, 4, 16, 2, 64, 8, 0.1, fake, None,
                                       None, 0, 0, None) == qsa.QSA_ERR_UNSUPPORTED
    # kv cache shorter than the queries
    assert lib.qsa_sparse_attn_prefill(fake, fake, fake, fake, fake, 1, 8, 0, 4, 16, 2, 128, 8, 0.1, fake, None,
                                       None, 0, 0, None) == qsa.QSA_ERR_INVALID_ARG
    # IndexShare draft step: capture lengths required, max_draft in [0, 64]
    assert lib.qsa_sparse_attn_decode_shared(fake, fake, fake, fake, None, fake, fake, 1, 64, 16, 2, 128, 8, 4, 0.1,
                                             fake, None, fake, 1 << 20, 0, None) == qsa.QSA_ERR_INVALID_ARG
    assert lib.qsa_sparse_attn_decode_shared(fake, fake, fake, fake, fake, fake, fake, 1, 64, 16, 2, 128, 8, 65,
                                             0.1, fake, None, fake, 1 << 20, 0, None) == qsa.QSA_ERR_INVALID_ARG
    assert lib.qsa_sparse_attn_decode_shared_workspace(4, 16, 128, 512, -1, 0) == 0
    assert lib.qsa_sparse_attn_decode_shared_workspace(4, 16, 128, 512, 8, 1) == 0     # fp32 needs none
    # dense decode baseline: a cache length is required
    assert lib.qsa_dense_attn_decode(fake, fake, fake, fake, 1, 0, 16, 2, 128, 0.1, fake, None, fake, 1 << 20, 0,
                                     None) == qsa.QSA_ERR_INVALID_ARG
    assert lib.qsa_dense_attn_decode(fake, fake, fake, None, 1, 64, 16, 2, 128, 0.1, fake, None, fake, 1 << 20, 0,
                                     None) == qsa.QSA_ERR_INVALID_ARG
    # FP8 compressed keys: BF16 only; the prefill indexer reads BF16 keys
    fp8 = qsa.QSA_KEYS_FP8
    assert lib.qsa_pool_keys_prefill(fake, fake, 1, 16, 0, 16, 4, rope, fp8, 1, None) == qsa.QSA_ERR_UNSUPPORTED
    assert lib.qsa_pool_keys_decode(fake, fake, fake, fake, 1, 4, rope, fp8, 1, None) == qsa.QSA_ERR_UNSUPPORTED
    assert lib.qsa_index_topk_prefill(fake, fake, None, 1, 16, 0, 4, 4, fake, fake, fake, 1 << 20, rope, fp8, 0,
                                      None) == qsa.QSA_ERR_UNSUPPORTED
    assert lib.qsa_index_topk_decode(fake, fake, None, fake, 1, 4, 4, 4, fake, fake, fake, 1 << 20, rope, fp8, 1,
                                     None) == qsa.QSA_ERR_UNSUPPORTED
    # paged caches: a table is required, page_tokens a power of two >= 32, BF16 only
    pg = qsa._Paging(4096, 8, 16, 64)
    assert lib.qsa_pool_keys_decode_paged(fake, fake, fake, qsa._Paging(None, 8, 16, 64), fake, 1, rope, 0, 0,
                                          None) == qsa.QSA_ERR_INVALID_ARG
    assert lib.qsa_pool_keys_decode_paged(fake, fake, fake, qsa._Paging(4096, 8, 16, 48), fake, 1, rope, 0, 0,
                                          None) == qsa.QSA_ERR_INVALID_ARG
    assert lib.qsa_pool_keys_decode_paged(fake, fake, fake, qsa._Paging(4096, 8, 16, 16), fake, 1, rope, 0, 0,
                                          None) == qsa.QSA_ERR_INVALID_ARG
    assert lib.qsa_pool_keys_decode_paged(fake, fake, fake, pg, fake, 1, rope, 0, 1, None) == qsa.QSA_ERR_UNSUPPORTED
    # max_blocks beyond the table's capacity (8 pages x 64 tokens = 128 blocks)
    assert lib.qsa_index_topk_decode_paged(fake, fake, pg, None, fake, 1, 129, 64, fake, fake, fake, 1 << 20, rope,
                                           0, 0, None) == qsa.QSA_ERR_INVALID_ARG
    assert lib.qsa_pool_keys_prefill_paged(fake, fake, pg, 1, 16, 512, 16, rope, 0, 0, None) == qsa.QSA_ERR_INVALID_ARG
    assert lib.qsa_sparse_attn_decode_paged(fake, fake, fake, pg, fake, fake, fake, 1, 16, 2, 128, 64, 0.1, fake,
                                            None, fake, 1 << 20, 1, None) == qsa.QSA_ERR_UNSUPPORTED
    assert lib.qsa_index_topk_decode_kernels(0, 100, 0, 0) == 0
    # FP8 K/V attention: scales must be finite and positive; bf16 shapes only (GQA 8)
    assert lib.qsa_sparse_attn_prefill_kv8(fake, fake, fake, 0.0, 1.0, fake, fake, 1, 4, 0, 4, 16, 2, 128, 8, 0.1,
                                           fake, None, None) == qsa.QSA_ERR_INVALID_ARG
    assert lib.qsa_sparse_attn_decode_kv8(fake, fake, fake, 1.0, float("inf"), fake, fake, fake, 1, 64, 16, 2, 128,
                                          8, 0.1, fake, None, fake, 1 << 20, None) == qsa.QSA_ERR_INVALID_ARG
    assert lib.qsa_sparse_attn_prefill_kv8(fake, fake, fake, 1.0, 1.0, fake, fake, 1, 4, 0, 4, 12, 4, 128, 8, 0.1,
                                           fake, None, None) == qsa.QSA_ERR_UNSUPPORTED
    # misaligned pointer
    odd = ctypes.c_void_p(4098)
    assert lib.qsa_pool_keys_prefill(odd, fake, 1, 16, 0, 16, 4, rope, 0, 0, None) == qsa.QSA_ERR_INVALID_ARG


def test_binding_rejects_host_tensors(qsa):
    import torch
    x = torch.zeros(1, 8, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        qsa.qsa_pool_keys_prefill(x, torch.zeros(1, 2, 128, dtype=torch.bfloat16))


def test_prefill_index_workspace_grows_with_context_up_to_its_cap(qsa):
    """The prefill indexer materialises scores of row groups of at most 2 GiB:
    its workspace grows with the context, stays below the cap plus the rotated
    queries, and a 16,000-row chunk at a 1M-token context is supported."""
    ws = qsa.qsa_index_topk_prefill_workspace
    sizes = [ws(1, 16000, q0, 512) for q0 in (0, 48000, 112000, 496000, 1032576)]
    assert all(a <= b for a, b in zip(sizes, sizes[1:]))
    q_bytes = 2 * 16000 * 128 * 2
    assert sizes[-1] <= (1 << 31) + 4 * q_bytes + (1 << 20)
    assert sizes[-1] >= 2048 * 262144 * 4                      # at least one 2048-row group of 1M-context scores
    assert ws(0, 16000, 0, 512) == 0 and ws(1, 16000, -1, 512) == 0     # invalid shapes: 0


def test_binding_constants_match_the_header(qsa):
    src = open(HEADER).read()
    m = re.search(r"#define QSA_NOALLOC_SCRATCH_BYTES \((\d+)u << (\d+)\)", src)
    assert m and qsa.QSA_NOALLOC_SCRATCH_BYTES == int(m.group(1)) << int(m.group(2))


def test_prefill_attention_workspace_sizes(qsa):
    """The split prefill (BF16, d = 128, 8 q heads per kv head, 2 or 4 kv
    heads) keeps in the workspace, per chunk of rows: the lists of blocks
    shared within each 8-query tile (8 * top_k / 2 entries of 6 bytes, rounded
    up to a key tile of 16; each listed block holds at least 2 of the tile's
    selections), every query's own list (top_k ids and a count) and the lse of
    the gather kernel's part (Hq floats a row); chunks are capped near 1 GiB;
    the other shapes need none."""
    ws = qsa.qsa_sparse_attn_prefill_workspace
    cap = (8 * 512 // 2 + 3 + 16) // 16 * 16
    rows = 131072
    tiles = rows // 8
    r256 = lambda x: (x + 255) // 256 * 256
    assert ws(1, rows, 512, 16, 2, 128, qsa.QSA_BF16) == (
        r256(tiles * 4) + r256(tiles * cap * 4) + r256(tiles * cap * 2) + r256(rows * 512 * 4) + r256(rows * 4)
        + r256(rows * 16 * 4))
    assert ws(1, 1, 512, 16, 2, 128, qsa.QSA_BF16) > 0
    assert 0 < ws(1, 131072, 2048, 16, 2, 128, qsa.QSA_BF16) <= (1 << 30) + 8192
    assert ws(1, 16000, 512, 16, 2, 128, qsa.QSA_BF16, q0=1032576) == 0   # contexts past 32768 blocks: gather kernel
    assert ws(4, 4096, 512, 16, 2, 128, qsa.QSA_BF16) == ws(1, 4096, 512, 16, 2, 128, qsa.QSA_BF16)  # per sequence
    assert ws(1, 4096, 512, 24, 2, 256, qsa.QSA_BF16) == 0      # released shape: the gather kernel
    assert ws(1, 4096, 512, 8, 1, 128, qsa.QSA_BF16) == 0       # one kv head: the gather kernel
    assert ws(1, 4096, 512, 8, 1, 128, qsa.QSA_FP32) == 0       # fp32: the SIMT kernel
    assert ws(0, 4096, 512, 16, 2, 128, qsa.QSA_BF16) == 0      # invalid


def test_prefill_kernel_counts(qsa):
    """Launch counts the benchmark reports: the indexer at 128K runs its score
    kernel and row select in 4 chunks of 32768 rows (16-bit keys under 2 GiB); the
    split attention runs three kernels per sequence and chunk of rows (lists,
    gather kernel, tiles)."""
    assert qsa.qsa_index_topk_prefill_kernels(1, 131072, 0, 0, qsa.QSA_BF16) == 1 + 2 * 4
    assert qsa.qsa_index_topk_prefill_kernels(1, 131072, 0, 0, qsa.QSA_FP32) == 1 + 2 * 8   # fp32 scores
    assert qsa.qsa_index_topk_prefill_kernels(1, 32768, 0, 0, qsa.QSA_BF16) == 1 + 2 * 1
    assert qsa.qsa_sparse_attn_prefill_kernels(1, 131072, 512, 16, 2, 128, qsa.QSA_BF16) == 3
    assert qsa.qsa_sparse_attn_prefill_kernels(2, 4096, 512, 16, 2, 128, qsa.QSA_BF16) == 6
    assert qsa.qsa_sparse_attn_prefill_kernels(1, 131072, 512, 24, 2, 256, qsa.QSA_BF16) == 1
    assert qsa.qsa_sparse_attn_prefill_kernels(1, 131072, 512, 8, 1, 128, qsa.QSA_BF16) == 1
    assert qsa.qsa_sparse_attn_prefill_kernels(1, 131072, 2048, 16, 2, 128, qsa.QSA_BF16) >= 3
    assert qsa.qsa_sparse_attn_prefill_kernels(1, 16000, 512, 16, 2, 128, qsa.QSA_BF16, q0=1032576) == 1
    assert qsa.qsa_index_topk_prefill_kernels(1, 16000, 1032576, 0, qsa.QSA_BF16) == 1 + 2 * 8   # fp32 scores
