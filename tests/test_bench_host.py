"""Host-side pieces of the benchmark that need no GPU: chunking of a prompt
for chunked prefill, the workloads' chunk settings, and the one-thread oracle
figure reported beside the all-core one."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import workloads  # noqa: E402


def test_chunk_bounds_cover_the_prompt_in_order():
    for T, chunk in [(1048576, 16000), (32768, None), (100, 30), (7, 16000), (16000, 16000)]:
        cb = bench.chunk_bounds(T, chunk)
        assert cb[0][0] == 0 and cb[-1][1] == T
        assert all(a1 == b0 for (_, a1), (b0, _) in zip(cb, cb[1:]))      # contiguous
        assert all(0 < c1 - c0 <= (chunk or T) for c0, c1 in cb)
        if chunk is None or chunk % 4 == 0:                             # block-aligned chunk, aligned offsets
            assert all(c0 % 4 == 0 for c0, _ in cb)
    cb = bench.chunk_bounds(1048576, 16000)
    assert len(cb) == 66 and cb[-1] == (1040000, 1048576)


def test_1m_workloads_chunk_in_16000_tokens():
    for name in ("prefill_l1m_chunk16k", "dense_prefill_l1m_chunk16k"):
        w = workloads.WORKLOADS[name]
        assert w.T == 1 << 20 and w.extra["chunk"] == 16000 and w.B == 1


def test_oracle_sample_reports_one_thread_rate():
    w = workloads.WORKLOADS["tiny_prefill_t1k_fp32"]
    bench.ORACLE_EXTRA.clear()
    value, sample, threads, unit = bench.run_oracle_sample(w, budget_s=0.5)
    assert unit == "tokens/s" and value > 0 and threads >= 1
    assert bench.ORACLE_EXTRA["value_1thread"] > 0
    # all cores are not slower than one (within timing noise on a loaded host)
    assert value >= 0.5 * bench.ORACLE_EXTRA["value_1thread"]


def test_default_run_is_the_metrics_configurations():
    """The metric is quoted at 128K-1M context: the default line is the 128K
    prefill, and the same run measures the 1M and 128K decode steps."""
    w = workloads.WORKLOADS[bench.DEFAULT_WORKLOAD]
    assert w.kind == "prefill" and w.T == 131072 and w.heavy_tail
    dec = [workloads.WORKLOADS[n] for n in bench.DEFAULT_DECODE]
    assert [(d.kind, d.B, d.T) for d in dec] == [("decode", 8, 1 << 20), ("decode", 64, 131072)]
